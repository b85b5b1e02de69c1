"""fp64 CPU oracle for the Kimi Delta Attention (KDA) operator -- TEST INFRASTRUCTURE.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py`` may import
this package.  The CUDA library never imports, links or executes anything here, and this package
imports nothing from the CUDA library.

The arithmetic lives in ``kda_oracle.c`` (plain C, fp64); this module only marshals numpy
arrays into it.  Every function follows a passage of the pages:

* ``seq``         -- the recurrence ``S_t = (I - b_t k_t k_t^T) Diag(a_t) S_{t-1} + b_t k_t v_t^T``
                     with readout ``o_t = S_t^T q_t``; "Kimi Linear" explainer (xugj520.cn),
                     section "Kimi Delta Attention的技术内核"; attention review (lanjinlin.com.cn),
                     entry "KLA 25.10 kimi".
* ``bruteforce``  -- the same recurrence with the dense transition matrix
                     ``M_t = (I - b k k^T) Diag(a)`` materialised (textbook matrix products).
* ``chunked``     -- the chunk-parallel / WY / UT form listed in the explainer's section
                     "硬件效率的深度优化" (chunk size C, any C >= 1).
* ``decode_step`` -- one token per sequence, in the loop order (decay, delta, update, output) of
                     the review's GDN pseudo-code.

``bwd`` is the reverse-mode derivative of ``seq`` (the training backward pass): the recurrence's
step differentiated as written, walking the tokens backwards.

``gated_rmsnorm`` is the output gate (grouped RMS norm times the gate z).

``prologue`` is the input transform of the kernels' optional prologue (q/k L2 normalisation,
log-sigmoid gate logits, sigmoid beta logits), applied in front of the other functions;
``prologue_bwd`` carries gradients back through it (the chain rule of each transform).

``seq``, ``chunked`` and ``decode_step`` also take q and k with fewer heads than v (grouped heads:
value head h reads q/k head h // (H // Hk)), as in the head-count comments of the review's GDN
pseudo-code.

Pins (checked in ``tests/test_oracle_pins.py``): the beta=0 closed form, exact write/retrieve
with orthonormal keys at alpha=1 and beta=1, an exact rational worked example, the per-step
delta invariant, brute force vs sequential, chunked vs sequential for several C, linearity in
(V, S0), state passing, varlen vs separate runs, decode vs prefill, and a norm bound.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import sys

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "kda_oracle.c")
_LIB = os.path.join(_HERE, "libkda_oracle.so")
_lib = None
_lib_path = None


def build(force: bool = False) -> str:
    """Compile ``kda_oracle.c`` into ``libkda_oracle.so`` next to it (gcc, -O2, no fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-fPIC", "-shared", "-std=c11", "-Wall", "-Wextra", "-fno-fast-math",
               "-ffp-contract=off", "-o", _LIB, _SRC, "-lm", "-lpthread"]
        subprocess.run(cmd, check=True)
    return _LIB


def use_library(path: str) -> None:
    """Point this wrapper at another build of the oracle (used by the mutant tests, which compile
    deliberately broken copies of ``kda_oracle.c`` and check that the pins reject them)."""
    global _lib, _lib_path
    _lib, _lib_path = None, path


def _load():
    global _lib
    if _lib is None:
        if _lib_path is None:
            build()
        lib = ctypes.CDLL(_lib_path or _LIB)
        P = ctypes.c_void_p
        I = ctypes.c_int
        for name in ("kda_oracle_seq", "kda_oracle_bruteforce"):
            f = getattr(lib, name)
            f.argtypes = [P, P, P, P, P, P, P, I, I, I, I, P, P, P, I]
            f.restype = I
        lib.kda_oracle_chunked.argtypes = [P, P, P, P, P, P, P, I, I, I, I, P, P, P, I, I]
        lib.kda_oracle_chunked.restype = I
        lib.kda_oracle_decode_step.argtypes = [P, P, P, P, P, P, I, I, I, I, P]
        lib.kda_oracle_decode_step.restype = I
        lib.kda_oracle_seq_grouped.argtypes = [P, P, P, P, P, P, P, I, I, I, I, I, P, P, P, I]
        lib.kda_oracle_seq_grouped.restype = I
        lib.kda_oracle_chunked_grouped.argtypes = [P, P, P, P, P, P, P, I, I, I, I, I, P, P, P, I, I]
        lib.kda_oracle_chunked_grouped.restype = I
        lib.kda_oracle_decode_step_grouped.argtypes = [P, P, P, P, P, P, I, I, I, I, I, P]
        lib.kda_oracle_decode_step_grouped.restype = I
        lib.kda_oracle_bwd.argtypes = [P, P, P, P, P, P, P, P, P, I, I, I, I, P, P, P, P, P, P, P, I]
        lib.kda_oracle_bwd.restype = I
        _lib = lib
    return _lib


def _f32(x):
    return np.ascontiguousarray(np.asarray(x, dtype=np.float32))


def _ptr(a):
    return None if a is None else a.ctypes.data


def default_threads() -> int:
    return max(1, len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else os.cpu_count() or 1)


def _prep(q, k, v, log_alpha, beta, S0, cu_seqlens):
    """q, k may have fewer heads (Hk) than v, log_alpha and beta (H), with H a multiple of Hk:
    value head h then reads q/k head h // (H // Hk) (grouped heads)."""
    q, k, v, la, b = _f32(q), _f32(k), _f32(v), _f32(log_alpha), _f32(beta)
    if q.ndim == 4:  # [B, T, H, d] regular batch -> packed with cu_seqlens
        B, T, Hk, dk = q.shape
        H, dv = v.shape[2], v.shape[-1]
        if cu_seqlens is not None:
            raise ValueError("cu_seqlens is only meaningful for packed [Ttot, H, d] inputs")
        cu = np.arange(B + 1, dtype=np.int64) * T
        q, k = (x.reshape(B * T, Hk, dk) for x in (q, k))
        la = la.reshape(B * T, H, dk)
        v = v.reshape(B * T, H, dv)
        b = b.reshape(B * T, H)
    else:
        Ttot, Hk, dk = q.shape
        H, dv = v.shape[1], v.shape[-1]
        cu = (np.array([0, Ttot], dtype=np.int64) if cu_seqlens is None
              else np.ascontiguousarray(np.asarray(cu_seqlens, dtype=np.int64)))
    N = len(cu) - 1
    Ttot = q.shape[0]
    if k.shape != q.shape or la.shape != (Ttot, H, dk) or v.shape[:2] != (Ttot, H) or b.shape != (Ttot, H) \
            or H % Hk != 0:
        raise ValueError("inconsistent shapes")
    s0 = None if S0 is None else np.ascontiguousarray(np.asarray(S0, dtype=np.float64).reshape(N, H, dk, dv))
    return q, k, v, la, b, s0, cu, N, H, Hk, dk, dv


def _call(fname, q, k, v, log_alpha, beta, S0, cu_seqlens, pairs, threads, extra=()):
    shape4 = np.asarray(q).ndim == 4
    q, k, v, la, b, s0, cu, N, H, Hk, dk, dv = _prep(q, k, v, log_alpha, beta, S0, cu_seqlens)
    Ttot = q.shape[0]
    out = np.zeros((Ttot, H, dv), dtype=np.float64)
    sf = np.zeros((N, H, dk, dv), dtype=np.float64)
    mask = None
    if pairs is not None:
        mask = np.zeros(N * H, dtype=np.int32)
        for n, h in pairs:
            mask[n * H + h] = 1
    lib = _load()
    if Hk != H:
        if fname != "kda_oracle_seq":
            raise ValueError(f"{fname} takes one q/k head per value head")
        rc = lib.kda_oracle_seq_grouped(_ptr(q), _ptr(k), _ptr(v), _ptr(la), _ptr(b), _ptr(s0), _ptr(cu), N, H,
                                        Hk, dk, dv, _ptr(out), _ptr(sf), _ptr(mask), threads or default_threads())
    else:
        rc = getattr(lib, fname)(_ptr(q), _ptr(k), _ptr(v), _ptr(la), _ptr(b), _ptr(s0), _ptr(cu), N, H, dk, dv,
                                 _ptr(out), _ptr(sf), _ptr(mask), *extra, threads or default_threads())
    if rc != 0:
        raise RuntimeError(f"{fname} failed with status {rc}")
    if shape4:
        B = N
        out = out.reshape(B, Ttot // B, H, dv)
    return out, sf


def seq(q, k, v, log_alpha, beta, S0=None, cu_seqlens=None, pairs=None, threads=None):
    """The definition.  Inputs ``[B,T,H,d]`` or packed ``[Ttot,H,d]`` (+ ``cu_seqlens``).

    Returns ``(out, S_final)`` in float64: out has the layout of ``v``, S_final is
    ``[N, H, dk, dv]``.  ``pairs`` restricts the work to a list of ``(seq, head)`` pairs
    (the other outputs stay zero)."""
    return _call("kda_oracle_seq", q, k, v, log_alpha, beta, S0, cu_seqlens, pairs, threads)


def bruteforce(q, k, v, log_alpha, beta, S0=None, cu_seqlens=None, pairs=None, threads=None):
    """Dense transition-matrix form (short sequences)."""
    return _call("kda_oracle_bruteforce", q, k, v, log_alpha, beta, S0, cu_seqlens, pairs, threads)


def chunked(q, k, v, log_alpha, beta, S0=None, cu_seqlens=None, C=64, pairs=None, threads=None):
    """Chunked WY/UT form with chunk size ``C``."""
    # the C entry point takes C before the thread count
    shape4 = np.asarray(q).ndim == 4
    q_, k_, v_, la, b, s0, cu, N, H, Hk, dk, dv = _prep(q, k, v, log_alpha, beta, S0, cu_seqlens)
    Ttot = q_.shape[0]
    out = np.zeros((Ttot, H, dv), dtype=np.float64)
    sf = np.zeros((N, H, dk, dv), dtype=np.float64)
    mask = None
    if pairs is not None:
        mask = np.zeros(N * H, dtype=np.int32)
        for n, h in pairs:
            mask[n * H + h] = 1
    rc = _load().kda_oracle_chunked_grouped(_ptr(q_), _ptr(k_), _ptr(v_), _ptr(la), _ptr(b), _ptr(s0), _ptr(cu),
                                            N, H, Hk, dk, dv, _ptr(out), _ptr(sf), _ptr(mask), int(C),
                                            threads or default_threads())
    if rc != 0:
        raise RuntimeError(f"kda_oracle_chunked failed with status {rc}")
    if shape4:
        out = out.reshape(N, Ttot // N, H, dv)
    return out, sf


def decode_step(q, k, v, log_alpha, beta, S):
    """One token for each of N sequences.  ``q,k [N,Hk,dk]``, ``log_alpha [N,H,dk]``, ``v [N,H,dv]``,
    ``beta [N,H]``, ``S [N,H,dk,dv]`` (float64, returned updated as a new array); Hk = H, or a
    divisor of H (value head h reads q/k head h // (H // Hk)).
    Returns ``(out [N,H,dv] float64, S_new)``."""
    q, k, v, la, b = _f32(q), _f32(k), _f32(v), _f32(log_alpha), _f32(beta)
    N, Hk, dk = q.shape
    H, dv = v.shape[1], v.shape[-1]
    if k.shape != q.shape or la.shape != (N, H, dk) or b.shape != (N, H) or H % Hk != 0:
        raise ValueError("inconsistent shapes")
    S = np.array(S, dtype=np.float64, copy=True, order="C").reshape(N, H, dk, dv)
    out = np.zeros((N, H, dv), dtype=np.float64)
    rc = _load().kda_oracle_decode_step_grouped(_ptr(q), _ptr(k), _ptr(v), _ptr(la), _ptr(b), _ptr(S), N, H, Hk,
                                                dk, dv, _ptr(out))
    if rc != 0:
        raise RuntimeError(f"kda_oracle_decode_step failed with status {rc}")
    return out, S


def bwd(q, k, v, log_alpha, beta, dout, S0=None, dS_final=None, cu_seqlens=None, pairs=None, threads=None):
    """Reverse-mode derivative of ``seq`` for the loss ``sum(dout * out) + sum(dS_final * S_final)``.

    Same inputs as ``seq`` plus the cotangents ``dout`` (layout of ``v``) and ``dS_final``
    ``[N, H, dk, dv]`` (None = 0).  Grouped q/k heads: the per-value-head derivatives of q and k
    are summed over each group (value head h reads q/k head h // (H // Hk)).
    Returns a dict of float64 arrays ``dq, dk`` (layout of q), ``dv`` (of v), ``dlog_alpha``,
    ``dbeta`` and ``dS0`` ``[N, H, dk, dv]``."""
    shape4 = np.asarray(q).ndim == 4
    q_, k_, v_, la, b, s0, cu, N, H, Hk, dk, dv = _prep(q, k, v, log_alpha, beta, S0, cu_seqlens)
    Ttot = q_.shape[0]
    G = H // Hk
    if G != 1:  # one q/k copy per value head
        q_, k_ = (np.ascontiguousarray(np.repeat(x, G, axis=1)) for x in (q_, k_))
    do = np.ascontiguousarray(np.asarray(dout, dtype=np.float64).reshape(Ttot, H, dv))
    dsf = None if dS_final is None else np.ascontiguousarray(
        np.asarray(dS_final, dtype=np.float64).reshape(N, H, dk, dv))
    dq = np.zeros((Ttot, H, dk)); dk_ = np.zeros((Ttot, H, dk)); dv_ = np.zeros((Ttot, H, dv))
    dla = np.zeros((Ttot, H, dk)); db = np.zeros((Ttot, H)); ds0 = np.zeros((N, H, dk, dv))
    mask = None
    if pairs is not None:
        mask = np.zeros(N * H, dtype=np.int32)
        for n, h in pairs:
            mask[n * H + h] = 1
    rc = _load().kda_oracle_bwd(_ptr(q_), _ptr(k_), _ptr(v_), _ptr(la), _ptr(b), _ptr(s0), _ptr(do), _ptr(dsf),
                                _ptr(cu), N, H, dk, dv, _ptr(dq), _ptr(dk_), _ptr(dv_), _ptr(dla), _ptr(db),
                                _ptr(ds0), _ptr(mask), threads or default_threads())
    if rc != 0:
        raise RuntimeError(f"kda_oracle_bwd failed with status {rc}")
    if G != 1:
        dq, dk_ = (x.reshape(Ttot, Hk, G, dk).sum(axis=2) for x in (dq, dk_))
    res = dict(dq=dq, dk=dk_, dv=dv_, dlog_alpha=dla, dbeta=db, dS0=ds0)
    if shape4:
        T = Ttot // N
        for key in ("dq", "dk", "dv", "dlog_alpha", "dbeta"):
            res[key] = res[key].reshape((N, T) + res[key].shape[1:])
    return res


QK_NORM_EPS = 1e-6  # x / sqrt(sum x^2 + eps): the epsilon of the in-kernel q/k normalisation


def prologue(q, k, log_alpha, beta, l2norm_qk=False, gate_logits=False, beta_logits=False):
    """The input prologue in fp64, as a preprocessing step in front of ``seq`` / ``chunked`` /
    ``decode_step``: q and k normalised over their last (d_k) axis, ``x / sqrt(sum x^2 + eps)``;
    gate logits a turned into ``log_alpha = log sigmoid(a)`` (the log-space forget gate of the
    coreui.cn article, section 4.2); beta logits b into ``beta = sigmoid(b)``.  Library routines
    (numpy, scipy.special.log_expit / expit) carry every step.  Returns float64 arrays."""
    import scipy.special as sp
    q, k, la, b = (np.asarray(x, dtype=np.float64) for x in (q, k, log_alpha, beta))
    if l2norm_qk:
        q = q / np.sqrt(np.sum(q * q, axis=-1, keepdims=True) + QK_NORM_EPS)
        k = k / np.sqrt(np.sum(k * k, axis=-1, keepdims=True) + QK_NORM_EPS)
    if gate_logits:
        la = sp.log_expit(la)
    if beta_logits:
        b = sp.expit(b)
    return q, k, la, b


def prologue_bwd(q, k, log_alpha, beta, grads, l2norm_qk=False, gate_logits=False, beta_logits=False):
    """The chain rule through ``prologue``: given the raw inputs and the gradients with respect to
    the transformed ones (a dict from ``bwd`` on ``prologue``'s outputs), return the gradients with
    respect to the raw inputs (a new dict; dv and dS0 pass through).  fp64 numpy:

    * x_hat = x / n, n = sqrt(sum x^2 + eps):  dx = dx_hat / n - x (x . dx_hat) / n^3
    * log_alpha = log sigmoid(a):              da = dlog_alpha * sigmoid(-a)
    * beta = sigmoid(b):                       db = dbeta * sigmoid(b) (1 - sigmoid(b))"""
    import scipy.special as sp
    q, k, la, b = (np.asarray(x, dtype=np.float64) for x in (q, k, log_alpha, beta))
    g = dict(grads)
    if l2norm_qk:
        for name, x in (("dq", q), ("dk", k)):
            n = np.sqrt(np.sum(x * x, axis=-1, keepdims=True) + QK_NORM_EPS)
            dxh = np.asarray(g[name], dtype=np.float64)
            g[name] = dxh / n - x * np.sum(x * dxh, axis=-1, keepdims=True) / n ** 3
    if gate_logits:
        g["dlog_alpha"] = np.asarray(g["dlog_alpha"], dtype=np.float64) * sp.expit(-la)
    if beta_logits:
        s = sp.expit(b)
        g["dbeta"] = np.asarray(g["dbeta"], dtype=np.float64) * s * (1.0 - s)
    return g


def gated_rmsnorm(o, z, weight=None, group=None, eps=1e-6, gate="none"):
    """The output gate of the review's GDN pseudo-code (section "门控归一化": the normalised attention
    output times the output gate z), with the grouped RMS norm of the Ring-linear notes (the norm
    taken over groups of ``group`` channels of the last axis, each group on its own):

        y = o / sqrt(mean_group(o^2) + eps) * weight * act(z),   act = identity or sigmoid.

    fp64 numpy; ``weight`` [d] or None (ones); ``group`` None = the whole last axis."""
    import scipy.special as sp
    o = np.asarray(o, dtype=np.float64)
    d = o.shape[-1]
    g = d if group is None else int(group)
    if d % g:
        raise ValueError("group must divide the last axis")
    og = o.reshape(o.shape[:-1] + (d // g, g))
    y = (og / np.sqrt(np.mean(og * og, axis=-1, keepdims=True) + eps)).reshape(o.shape)
    if weight is not None:
        y = y * np.asarray(weight, dtype=np.float64)
    zz = np.asarray(z, dtype=np.float64)
    return y * (sp.expit(zz) if gate == "sigmoid" else zz)


if __name__ == "__main__":  # pragma: no cover
    print(build(force="--force" in sys.argv))
