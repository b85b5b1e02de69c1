"""Thin Python binding of libkda.so (the C ABI declared in include/kda.h).

Argument marshalling only: tensors are checked for device/dtype/layout, their device pointers and
the current CUDA stream are handed to the C entry points, and status codes become exceptions.
Every step of the operator runs in the library's CUDA kernels; there is no fallback of any kind,
and importing a missing or unbuilt library raises.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Tuple

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libkda.so")

KDA_BF16, KDA_F32 = 0, 1
STATUS = {0: "KDA_OK", 1: "KDA_ERR_INVALID_ARG", 2: "KDA_ERR_UNSUPPORTED", 3: "KDA_ERR_CUDA",
          4: "KDA_ERR_TIMEOUT", 5: "KDA_ERR_WORKSPACE", 6: "KDA_ERR_BAD_SEQLENS"}

# The C ABI, as declared in include/kda.h (name -> (restype, argtypes)).
_P, _I, _SZ = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t


class KdaOptions(ctypes.Structure):
    """``kda_options`` of include/kda.h (zero = the plain entry points' behaviour)."""
    _fields_ = [("num_qk_heads", ctypes.c_int), ("prologue", ctypes.c_uint), ("reserved", ctypes.c_int * 6)]


class KdaOutputGate(ctypes.Structure):
    """``kda_output_gate`` of include/kda.h (the output gate of ``kda_chunk_fwd_gated``)."""
    _fields_ = [("z", ctypes.c_void_p), ("weight", ctypes.c_void_p), ("group", ctypes.c_int),
                ("eps", ctypes.c_float), ("act", ctypes.c_int), ("reserved", ctypes.c_int * 3)]


GATE_ACT = {"none": 0, "sigmoid": 1}  # kda_gate_act

# kda_options.prologue bits (KDA_PROLOGUE_* in include/kda.h)
PROLOGUE_L2NORM_QK = 1     # q and k normalised per (token, q/k head) over d_k inside the kernels
PROLOGUE_GATE_LOGITS = 2   # log_alpha holds raw gate logits a: log_alpha = log sigmoid(a)
PROLOGUE_BETA_LOGITS = 4   # beta holds raw logits b: beta = sigmoid(b)
PROLOGUE_GATE_BF16 = 8     # log_alpha (or its logits) is bf16; set by the binding from log_alpha's dtype


ABI = {
    "kda_status_string": (ctypes.c_char_p, [_I]),
    "kda_version": (ctypes.c_char_p, []),
    "kda_chunk_fwd_workspace_size": (_I, [_I, _I, _I, _I, _I, _I, _I, _I, ctypes.POINTER(_SZ)]),
    "kda_chunk_fwd": (_I, [_P, _P, _P, _P, _P, _P, _P, _I, _P, _P, _I, _I, _I, _I, _I, _I, _P, _SZ, _P]),
    "kda_decode_step": (_I, [_P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _P]),
    "kda_chunk_fwd_ex": (_I, [_P, _P, _P, _P, _P, _P, _P, _I, _P, _P, _I, _I, _I, _I, _I, _I,
                              ctypes.POINTER(KdaOptions), _P, _SZ, _P]),
    "kda_decode_step_ex": (_I, [_P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, ctypes.POINTER(KdaOptions), _P]),
    "kda_gated_rmsnorm": (_I, [_P, _P, _P, _P, ctypes.c_longlong, _I, _I, ctypes.c_float, _I, _I, _P]),
    "kda_chunk_fwd_gated": (_I, [_P, _P, _P, _P, _P, _P, _P, _I, _P, _P, _I, _I, _I, _I, _I, _I,
                                 ctypes.POINTER(KdaOptions), ctypes.POINTER(KdaOutputGate), _P, _SZ, _P]),
    "kda_chunk_fwd_noalloc": (_I, [_P, _P, _P, _P, _P, _P, _P, _I, _P, _P, _I, _I, _I, _I, _I, _I, _P]),
    "kda_chunk_bwd_workspace_size": (_I, [_I, _I, _I, _I, _I, _I, _I, _I, ctypes.POINTER(KdaOptions),
                                         ctypes.POINTER(_SZ)]),
    "kda_chunk_bwd": (_I, [_P, _P, _P, _P, _P, _P, _P, _I, _P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I,
                           ctypes.POINTER(KdaOptions), _P, _SZ, _P]),
    "kda_chunk_fwd_host_workspace_size": (_I, [_I, _I, _I, _I, _I, _I, ctypes.POINTER(KdaOptions), _I,
                                              ctypes.POINTER(_SZ)]),
    "kda_chunk_fwd_host": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, ctypes.POINTER(KdaOptions),
                                _I, _P, _SZ, _P]),
    "kda_host_release": (_I, []),
    "kda_check": (_I, [_P]),
    "kda_selftest_timeout": (_I, [_P]),
    "kda_profile_begin": (_I, []),
    "kda_profile_end": (_I, []),
    "kda_profile_kernels": (_I, [_I, ctypes.POINTER(ctypes.c_char_p), ctypes.POINTER(_I),
                                 ctypes.POINTER(ctypes.c_double)]),
}

_lib = None


class KdaError(RuntimeError):
    def __init__(self, fn: str, code: int):
        super().__init__(f"{fn} returned {STATUS.get(code, code)}")
        self.code = code


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load libkda.so (build it first with ``python -m gated_delta_rule_83_b200.build``)."""
    global _lib
    if _lib is None or path != LIB_PATH:
        if not os.path.exists(path):
            raise ImportError(f"{path} is missing: build it with `python -m gated_delta_rule_83_b200.build`")
        lib = ctypes.CDLL(path)
        for name, (res, args) in ABI.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        if path != LIB_PATH:
            return lib
        _lib = lib
    return _lib


def _check(fn: str, code: int):
    if code != 0:
        raise KdaError(fn, code)


def _dt(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return KDA_BF16
    if t.dtype == torch.float32:
        return KDA_F32
    raise TypeError(f"q/k/v must be bfloat16 or float32, got {t.dtype}")


def _gate_bits(log_alpha: torch.Tensor, prologue: int) -> int:
    """log_alpha may be fp32 or bf16; bf16 selects PROLOGUE_GATE_BF16 (exact widening in the kernels)."""
    if log_alpha.dtype == torch.bfloat16:
        return prologue | PROLOGUE_GATE_BF16
    if log_alpha.dtype != torch.float32:
        raise TypeError(f"log_alpha must be float32 or bfloat16, got {log_alpha.dtype}")
    if prologue & PROLOGUE_GATE_BF16:
        raise TypeError("PROLOGUE_GATE_BF16 set for a float32 log_alpha")
    return prologue


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else t.data_ptr()


def _req(t: torch.Tensor, name: str, dtype=None, device=None):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if device is not None and t.device != device:
        raise ValueError(f"{name} is on {t.device}, expected {device}")


def _stream_handle(stream: Optional[torch.cuda.Stream], device) -> int:
    s = stream if stream is not None else torch.cuda.current_stream(device)
    return s.cuda_stream


_workspaces = {}  # (device, stream handle) -> the largest workspace a call on that stream has needed


def release_workspaces() -> None:
    """Drop the cached per-stream workspaces (the backward's can be several GB).  Calls made after
    this allocate again on first use; pass ``workspace=`` to manage the memory yourself."""
    _workspaces.clear()


def release_host_resources() -> None:
    """Destroy the copy streams and events that ``chunk_fwd_host`` keeps per (device, stream)
    (``kda_host_release``); later calls create them again."""
    _check("kda_host_release", load_library().kda_host_release())


def workspace_size(B: int, T: int, H: int, dk: int, dv: int, varlen: bool = False, num_seqs: int = 0,
                   dtype: torch.dtype = torch.bfloat16) -> int:
    lib = load_library()
    n = ctypes.c_size_t(0)
    dt = KDA_BF16 if dtype == torch.bfloat16 else KDA_F32
    _check("kda_chunk_fwd_workspace_size",
           lib.kda_chunk_fwd_workspace_size(B, T, H, dk, dv, int(bool(varlen)), num_seqs, dt, ctypes.byref(n)))
    return n.value


def _get_workspace(nbytes: int, device, stream_handle: int) -> torch.Tensor:
    key = (device, stream_handle)
    ws = _workspaces.get(key)
    if ws is None or ws.numel() < nbytes:
        ws = torch.empty(max(nbytes, 256), dtype=torch.uint8, device=device)
        _workspaces[key] = ws
    return ws


def chunk_fwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, log_alpha: torch.Tensor, beta: torch.Tensor,
              S0: Optional[torch.Tensor] = None, cu_seqlens: Optional[torch.Tensor] = None,
              out: Optional[torch.Tensor] = None, S_final: Optional[torch.Tensor] = None,
              output_final_state: bool = True, workspace: Optional[torch.Tensor] = None,
              stream: Optional[torch.cuda.Stream] = None, prologue: int = 0,
              z: Optional[torch.Tensor] = None, gate_weight: Optional[torch.Tensor] = None, gate_group: int = 0,
              gate_eps: float = 1e-6, gate_act: str = "none") -> Tuple[torch.Tensor, Optional[torch.Tensor]]:
    """Chunked KDA prefill (``kda_chunk_fwd``).

    q, k: [B, T, Hk, dk]; log_alpha: [B, T, H, dk]; v: [B, T, H, dv]; beta: [B, T, H]; q/k/v bf16 or
    fp32, beta fp32, log_alpha fp32 or bf16 (``kda_chunk_fwd_ex`` with PROLOGUE_GATE_BF16).  Hk = H, or
    a divisor of H (grouped heads, ``kda_chunk_fwd_ex``: value head h reads q/k head h // (H // Hk)).
    S0 / S_final: [N, H, dk, dv] fp32 (N = B, or len(cu_seqlens) - 1 for packed varlen input with B = 1).
    ``prologue``: PROLOGUE_* bits (raw q/k and gate logits transformed inside the kernels).
    Returns (out [B, T, H, dv] in q's dtype, S_final or None).  S_final may be S0 (in place).

    With ``z`` ([B, T, H, dv], q's dtype) the output gate is applied inside the prefill
    (``kda_chunk_fwd_gated``): out = o / sqrt(mean_group(o^2) + gate_eps) * gate_weight * act(z),
    gate_weight [dv] fp32 or None, gate_group 0 (= dv) or a power of two >= 8, gate_act "none" or
    "sigmoid"; o itself is not returned."""
    lib = load_library()
    _req(q, "q")
    dev = q.device
    dtq = q.dtype
    if q.dim() != 4 or v.dim() != 4:
        raise ValueError("q must be [B, T, Hk, dk] and v [B, T, H, dv]")
    B, T, Hk, dk = q.shape
    H, dv = v.shape[2], v.shape[-1]
    _req(k, "k", dtq, dev)
    _req(v, "v", dtq, dev)
    _req(log_alpha, "log_alpha", None, dev)
    prologue = _gate_bits(log_alpha, prologue)
    _req(beta, "beta", torch.float32, dev)
    if k.shape != q.shape or tuple(log_alpha.shape) != (B, T, H, dk) or tuple(v.shape) != (B, T, H, dv) or \
            tuple(beta.shape) != (B, T, H) or H % Hk != 0:
        raise ValueError("inconsistent shapes")
    N = B
    if cu_seqlens is not None:
        _req(cu_seqlens, "cu_seqlens", torch.int32, dev)
        N = cu_seqlens.numel() - 1
        if B != 1:
            raise ValueError("packed varlen input needs B == 1")
    if S0 is not None:
        _req(S0, "S0", torch.float32, dev)
        if tuple(S0.shape) != (N, H, dk, dv):
            raise ValueError(f"S0 must be [{N}, {H}, {dk}, {dv}]")
    if out is None:
        out = torch.empty((B, T, H, dv), dtype=dtq, device=dev)
    else:
        _req(out, "out", dtq, dev)
    if S_final is None and output_final_state:
        S_final = torch.empty((N, H, dk, dv), dtype=torch.float32, device=dev)
    elif S_final is not None:
        _req(S_final, "S_final", torch.float32, dev)
    sh = _stream_handle(stream, dev)
    ws_bytes = workspace_size(B, T, H, dk, dv, cu_seqlens is not None, N, dtq)
    if workspace is None:
        workspace = _get_workspace(ws_bytes, dev, sh)
    else:
        _req(workspace, "workspace", torch.uint8, dev)
    if z is not None:
        _req(z, "z", dtq, dev)
        if tuple(z.shape) != (B, T, H, dv):
            raise ValueError(f"z must be [{B}, {T}, {H}, {dv}]")
        if z.data_ptr() == out.data_ptr() and z.numel():
            raise ValueError("z must not alias out")
        if gate_weight is not None:
            _req(gate_weight, "gate_weight", torch.float32, dev)
            if tuple(gate_weight.shape) != (dv,):
                raise ValueError(f"gate_weight must be [{dv}]")
        if gate_act not in GATE_ACT:
            raise ValueError(f"gate_act must be one of {sorted(GATE_ACT)}")
        g = KdaOutputGate(z=_ptr(z), weight=_ptr(gate_weight), group=gate_group, eps=gate_eps,
                          act=GATE_ACT[gate_act])
        opt = KdaOptions(num_qk_heads=Hk, prologue=prologue)
        rc = lib.kda_chunk_fwd_gated(_ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(beta), _ptr(S0),
                                     _ptr(cu_seqlens), N, _ptr(out), _ptr(S_final), B, T, H, dk, dv, _dt(q),
                                     ctypes.byref(opt), ctypes.byref(g), _ptr(workspace), workspace.numel(), sh)
        _check("kda_chunk_fwd_gated", rc)
    elif Hk == H and not prologue:
        rc = lib.kda_chunk_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(beta), _ptr(S0), _ptr(cu_seqlens),
                               N, _ptr(out), _ptr(S_final), B, T, H, dk, dv, _dt(q), _ptr(workspace),
                               workspace.numel(), sh)
        _check("kda_chunk_fwd", rc)
    else:
        opt = KdaOptions(num_qk_heads=Hk, prologue=prologue)
        rc = lib.kda_chunk_fwd_ex(_ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(beta), _ptr(S0),
                                  _ptr(cu_seqlens), N, _ptr(out), _ptr(S_final), B, T, H, dk, dv, _dt(q),
                                  ctypes.byref(opt), _ptr(workspace), workspace.numel(), sh)
        _check("kda_chunk_fwd_ex", rc)
    return out, S_final


def _host(t: torch.Tensor, name: str, dtype=None):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.is_cuda:
        raise ValueError(f"{name} must be a host tensor (pinned for overlap)")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")


def chunk_fwd_host(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, log_alpha: torch.Tensor, beta: torch.Tensor,
                   S0: Optional[torch.Tensor] = None, out: Optional[torch.Tensor] = None,
                   S_final: Optional[torch.Tensor] = None, output_final_state: bool = True, prologue: int = 0,
                   segment_tokens: int = 4096, device=None, workspace: Optional[torch.Tensor] = None,
                   stream: Optional[torch.cuda.Stream] = None, synchronize: bool = True):
    """``kda_chunk_fwd_host``: the prefill on HOST tensors (pinned for overlap), pipelined in
    segments of ``segment_tokens`` tokens: copies in, kernels and copies out overlap.  Same shapes
    and options as ``chunk_fwd`` (regular batches).  Outputs are host tensors (pinned when
    allocated here).  With ``synchronize`` the call waits for the stream before returning."""
    lib = load_library()
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    _host(q, "q")
    dtq = q.dtype
    B, T, Hk, dk = q.shape
    H, dv = v.shape[2], v.shape[-1]
    _host(k, "k", dtq)
    _host(v, "v", dtq)
    _host(log_alpha, "log_alpha")
    prologue = _gate_bits(log_alpha, prologue)
    _host(beta, "beta", torch.float32)
    if k.shape != q.shape or tuple(log_alpha.shape) != (B, T, H, dk) or tuple(v.shape) != (B, T, H, dv) or \
            tuple(beta.shape) != (B, T, H) or H % Hk != 0:
        raise ValueError("inconsistent shapes")
    if S0 is not None:
        _host(S0, "S0", torch.float32)
    if out is None:
        out = torch.empty((B, T, H, dv), dtype=dtq).pin_memory()
    else:
        _host(out, "out", dtq)
    if S_final is None and output_final_state:
        S_final = torch.empty((B, H, dk, dv), dtype=torch.float32).pin_memory()
    elif S_final is not None:
        _host(S_final, "S_final", torch.float32)
    opt = KdaOptions(num_qk_heads=Hk, prologue=prologue)
    n = ctypes.c_size_t(0)
    _check("kda_chunk_fwd_host_workspace_size",
           lib.kda_chunk_fwd_host_workspace_size(B, T, H, dk, dv, _dt(q), ctypes.byref(opt), segment_tokens,
                                                 ctypes.byref(n)))
    sh = _stream_handle(stream, dev)
    if workspace is None:
        workspace = _get_workspace(n.value, dev, sh)
    else:
        _req(workspace, "workspace", torch.uint8, dev)
    rc = lib.kda_chunk_fwd_host(_ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(beta), _ptr(S0), _ptr(out),
                                _ptr(S_final), B, T, H, dk, dv, _dt(q), ctypes.byref(opt), segment_tokens,
                                _ptr(workspace), workspace.numel(), sh)
    _check("kda_chunk_fwd_host", rc)
    if synchronize:
        (stream or torch.cuda.current_stream(dev)).synchronize()
    return out, S_final


def bwd_workspace_size(B: int, T: int, H: int, dk: int, dv: int, varlen: bool = False, num_seqs: int = 0,
                       dtype: torch.dtype = torch.bfloat16, qk_heads: Optional[int] = None, prologue: int = 0) -> int:
    lib = load_library()
    n = ctypes.c_size_t(0)
    dt = KDA_BF16 if dtype == torch.bfloat16 else KDA_F32
    opt = KdaOptions(num_qk_heads=qk_heads or 0, prologue=prologue)
    _check("kda_chunk_bwd_workspace_size",
           lib.kda_chunk_bwd_workspace_size(B, T, H, dk, dv, int(bool(varlen)), num_seqs, dt, ctypes.byref(opt),
                                            ctypes.byref(n)))
    return n.value


def chunk_bwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, log_alpha: torch.Tensor, beta: torch.Tensor,
              dout: torch.Tensor, S0: Optional[torch.Tensor] = None, dS_final: Optional[torch.Tensor] = None,
              cu_seqlens: Optional[torch.Tensor] = None, want_dS0: bool = True, grads: Optional[dict] = None,
              workspace: Optional[torch.Tensor] = None, stream: Optional[torch.cuda.Stream] = None,
              prologue: int = 0) -> dict:
    """Backward pass of ``chunk_fwd`` (``kda_chunk_bwd``): the derivatives of
    ``L = sum(dout * out) + sum(dS_final * S_final)`` with respect to every input.

    Inputs as ``chunk_fwd`` (q, k with H or Hk heads; log_alpha fp32 or bf16) plus ``dout``
    (layout and dtype of ``out``) and ``dS_final`` ([N, H, dk, dv] fp32 or None).  Returns a dict
    ``dq, dk, dv`` (dtype of q), ``dlog_alpha`` (fp32), ``dbeta`` (fp32) and ``dS0`` (fp32, or None
    when ``want_dS0`` is False).  ``grads`` may hold preallocated output tensors under those keys.
    ``prologue``: the PROLOGUE_* bits the forward call used; the gradients are then those of the raw
    inputs."""
    lib = load_library()
    _req(q, "q")
    dev, dtq = q.device, q.dtype
    B, T, Hk, dk = q.shape
    H, dv = v.shape[2], v.shape[-1]
    for t, name in ((k, "k"), (v, "v"), (dout, "dout")):
        _req(t, name, dtq, dev)
    _req(log_alpha, "log_alpha", None, dev)
    pro = _gate_bits(log_alpha, prologue)
    _req(beta, "beta", torch.float32, dev)
    if k.shape != q.shape or tuple(log_alpha.shape) != (B, T, H, dk) or tuple(v.shape) != (B, T, H, dv) or \
            tuple(beta.shape) != (B, T, H) or dout.shape != v.shape or H % Hk != 0:
        raise ValueError("inconsistent shapes")
    N = B
    if cu_seqlens is not None:
        _req(cu_seqlens, "cu_seqlens", torch.int32, dev)
        N = cu_seqlens.numel() - 1
        if B != 1:
            raise ValueError("packed varlen input needs B == 1")
    for t, name in ((S0, "S0"), (dS_final, "dS_final")):
        if t is not None:
            _req(t, name, torch.float32, dev)
            if tuple(t.shape) != (N, H, dk, dv):
                raise ValueError(f"{name} must be [{N}, {H}, {dk}, {dv}]")
    g = dict(grads or {})
    want = {"dq": (q.shape, dtq), "dk": (q.shape, dtq), "dv": (v.shape, dtq),
            "dlog_alpha": (log_alpha.shape, torch.float32), "dbeta": (beta.shape, torch.float32)}
    if want_dS0:
        want["dS0"] = ((N, H, dk, dv), torch.float32)
    for key, (shape, dt) in want.items():
        if g.get(key) is None:
            g[key] = torch.empty(shape, dtype=dt, device=dev)
        else:
            _req(g[key], key, dt, dev)
            if tuple(g[key].shape) != tuple(shape):
                raise ValueError(f"{key} must be {tuple(shape)}")
    if not want_dS0:
        g["dS0"] = None
    sh = _stream_handle(stream, dev)
    ws_bytes = bwd_workspace_size(B, T, H, dk, dv, cu_seqlens is not None, N, dtq, qk_heads=Hk, prologue=pro)
    if workspace is None:
        workspace = _get_workspace(ws_bytes, dev, sh)
    else:
        _req(workspace, "workspace", torch.uint8, dev)
    opt = KdaOptions(num_qk_heads=Hk, prologue=pro)
    rc = lib.kda_chunk_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(beta), _ptr(S0), _ptr(cu_seqlens), N,
                           _ptr(dout), _ptr(dS_final), _ptr(g["dq"]), _ptr(g["dk"]), _ptr(g["dv"]),
                           _ptr(g["dlog_alpha"]), _ptr(g["dbeta"]), _ptr(g["dS0"]), B, T, H, dk, dv, _dt(q),
                           ctypes.byref(opt), _ptr(workspace), workspace.numel(), sh)
    _check("kda_chunk_bwd", rc)
    return g


NOALLOC_SCRATCH_BYTES = 64 * 1024 * 1024  # KDA_NOALLOC_SCRATCH_BYTES in include/kda.h


def _check_noalloc_args(q, k, v, log_alpha, beta, S0, out, S_final, cu_seqlens):
    """Argument checks of ``chunk_fwd_noalloc``, types and shapes first, placement last, so that a
    malformed call raises before any pointer reaches the library.  Returns (B, T, H, dk, dv, N)."""
    named = (("q", q), ("k", k), ("v", v), ("log_alpha", log_alpha), ("beta", beta), ("out", out))
    for name, t in named + (("S0", S0), ("S_final", S_final), ("cu_seqlens", cu_seqlens)):
        if t is not None and not isinstance(t, torch.Tensor):
            raise TypeError(f"{name} must be a torch.Tensor")
    for name, t in named:
        if t is None:
            raise TypeError(f"{name} is required")
    if q.dtype not in (torch.bfloat16, torch.float32):
        raise TypeError(f"q must be bfloat16 or float32, got {q.dtype}")
    for name, t in (("k", k), ("v", v), ("out", out)):
        if t.dtype != q.dtype:
            raise TypeError(f"{name} must be {q.dtype}, got {t.dtype}")
    # the entry point takes float* gates: a bf16 log_alpha would be read past its end
    for name, t in (("log_alpha", log_alpha), ("beta", beta), ("S0", S0), ("S_final", S_final)):
        if t is not None and t.dtype != torch.float32:
            raise TypeError(f"{name} must be torch.float32, got {t.dtype}")
    if q.dim() != 4 or v.dim() != 4:
        raise ValueError("q must be [B, T, H, dk] and v [B, T, H, dv]")
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    if tuple(k.shape) != (B, T, H, dk) or tuple(v.shape) != (B, T, H, dv) or \
            tuple(log_alpha.shape) != (B, T, H, dk) or tuple(beta.shape) != (B, T, H):
        raise ValueError("inconsistent shapes (the allocation-free entry point has no grouped q/k heads)")
    if tuple(out.shape) != (B, T, H, dv):
        raise ValueError(f"out must be [{B}, {T}, {H}, {dv}]")
    N = B
    if cu_seqlens is not None:
        if cu_seqlens.dtype != torch.int32 or cu_seqlens.dim() != 1 or cu_seqlens.numel() < 2:
            raise TypeError("cu_seqlens must be a 1-D torch.int32 tensor of N + 1 offsets")
        if B != 1:
            raise ValueError("packed varlen input needs B == 1")
        N = cu_seqlens.numel() - 1
    for name, t in (("S0", S0), ("S_final", S_final)):
        if t is not None and tuple(t.shape) != (N, H, dk, dv):
            raise ValueError(f"{name} must be [{N}, {H}, {dk}, {dv}]")
    dev = q.device
    for name, t in named + (("S0", S0), ("S_final", S_final), ("cu_seqlens", cu_seqlens)):
        if t is not None:
            _req(t, name, None, dev)
    return B, T, H, dk, dv, N


def chunk_fwd_noalloc(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, log_alpha: torch.Tensor,
                      beta: torch.Tensor, S0: Optional[torch.Tensor], out: torch.Tensor,
                      S_final: Optional[torch.Tensor], cu_seqlens: Optional[torch.Tensor] = None,
                      stream: Optional[torch.cuda.Stream] = None) -> None:
    """``kda_chunk_fwd_noalloc``: the chunked prefill for callers that cannot allocate device memory
    (the library's built-in scratch replaces the workspace).  Every buffer, ``out`` and ``S_final``
    included, is the caller's; nothing is allocated here either.  Shapes as ``chunk_fwd`` with
    Hk = H; log_alpha, beta, S0 and S_final fp32 (S0 None = zero state, S_final None = not
    written).  Problems whose workspace would exceed ``NOALLOC_SCRATCH_BYTES`` raise ``KdaError``
    (KDA_ERR_WORKSPACE)."""
    B, T, H, dk, dv, N = _check_noalloc_args(q, k, v, log_alpha, beta, S0, out, S_final, cu_seqlens)
    lib = load_library()
    with torch.cuda.device(q.device):  # the scratch address is looked up on the current device
        rc = lib.kda_chunk_fwd_noalloc(_ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(beta), _ptr(S0),
                                       _ptr(cu_seqlens), N, _ptr(out), _ptr(S_final), B, T, H, dk, dv, _dt(q),
                                       _stream_handle(stream, q.device))
    _check("kda_chunk_fwd_noalloc", rc)


def decode_step(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, log_alpha: torch.Tensor, beta: torch.Tensor,
                S: torch.Tensor, out: Optional[torch.Tensor] = None,
                stream: Optional[torch.cuda.Stream] = None, prologue: int = 0) -> torch.Tensor:
    """One KDA decode step (``kda_decode_step``); ``S`` [N, H, dk, dv] fp32 is updated in place.
    q, k: [N, Hk, dk]; log_alpha: [N, H, dk]; v: [N, H, dv]; beta: [N, H], with Hk = H or a divisor of
    H (grouped heads, ``kda_decode_step_ex``); log_alpha fp32 or bf16.  ``prologue``: PROLOGUE_* bits.
    Returns out [N, H, dv]."""
    lib = load_library()
    _req(q, "q")
    dev, dtq = q.device, q.dtype
    N, Hk, dk = q.shape
    H, dv = v.shape[1], v.shape[-1]
    _req(k, "k", dtq, dev)
    _req(v, "v", dtq, dev)
    _req(log_alpha, "log_alpha", None, dev)
    prologue = _gate_bits(log_alpha, prologue)
    _req(beta, "beta", torch.float32, dev)
    _req(S, "S", torch.float32, dev)
    if k.shape != q.shape or tuple(log_alpha.shape) != (N, H, dk) or tuple(v.shape) != (N, H, dv) or \
            tuple(beta.shape) != (N, H) or tuple(S.shape) != (N, H, dk, dv) or H % Hk != 0:
        raise ValueError("inconsistent shapes")
    if out is None:
        out = torch.empty((N, H, dv), dtype=dtq, device=dev)
    else:
        _req(out, "out", dtq, dev)
    if Hk == H and not prologue:
        rc = lib.kda_decode_step(_ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(beta), _ptr(S), _ptr(out), N, H,
                                 dk, dv, _dt(q), _stream_handle(stream, dev))
        _check("kda_decode_step", rc)
    else:
        opt = KdaOptions(num_qk_heads=Hk, prologue=prologue)
        rc = lib.kda_decode_step_ex(_ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(beta), _ptr(S), _ptr(out), N,
                                    H, dk, dv, _dt(q), ctypes.byref(opt), _stream_handle(stream, dev))
        _check("kda_decode_step_ex", rc)
    return out


def gated_rmsnorm(o: torch.Tensor, z: torch.Tensor, weight: Optional[torch.Tensor] = None, group: int = 0,
                  eps: float = 1e-6, gate: str = "none", out: Optional[torch.Tensor] = None,
                  stream: Optional[torch.cuda.Stream] = None) -> torch.Tensor:
    """Output gate ``y = o / sqrt(mean_group(o^2) + eps) * weight * act(z)`` (``kda_gated_rmsnorm``).
    o, z: [..., d] (bf16 or fp32, same shape), d in {64, 128}; weight [d] fp32 or None; group 0 (= d)
    or a power of two >= 8 dividing d; gate "none" or "sigmoid".  ``out`` may be ``o`` (in place)."""
    lib = load_library()
    _req(o, "o")
    dev, dt = o.device, o.dtype
    _req(z, "z", dt, dev)
    if z.shape != o.shape:
        raise ValueError("o and z must have the same shape")
    if weight is not None:
        _req(weight, "weight", torch.float32, dev)
    if out is None:
        out = torch.empty_like(o)
    else:
        _req(out, "out", dt, dev)
    d = o.shape[-1]
    rows = o.numel() // d if d else 0
    act = {"none": 0, "sigmoid": 1}[gate]
    rc = lib.kda_gated_rmsnorm(_ptr(o), _ptr(z), _ptr(weight), _ptr(out), rows, d, group, eps, act, _dt(o),
                               _stream_handle(stream, dev))
    _check("kda_gated_rmsnorm", rc)
    return out


def check(stream: Optional[torch.cuda.Stream] = None):
    """Synchronise and raise if a kernel recorded a device-side error (``kda_check``)."""
    lib = load_library()
    dev = torch.device("cuda", torch.cuda.current_device())
    _check("kda_check", lib.kda_check(_stream_handle(stream, dev)))


def profile_begin():
    """Start recording per-launch device times of the library's kernels (``kda_profile_begin``)."""
    _check("kda_profile_begin", load_library().kda_profile_begin())


def profile_end() -> dict:
    """Stop recording and return ``{kernel name: (launches, total device ms)}``."""
    lib = load_library()
    _check("kda_profile_end", lib.kda_profile_end())
    cap = 64
    names = (ctypes.c_char_p * cap)()
    launches = (ctypes.c_int * cap)()
    ms = (ctypes.c_double * cap)()
    n = lib.kda_profile_kernels(cap, names, launches, ms)
    if n < 0:
        raise KdaError("kda_profile_kernels", 3)
    return {names[i].decode(): (launches[i], ms[i]) for i in range(n)}


def version() -> str:
    return load_library().kda_version().decode()
