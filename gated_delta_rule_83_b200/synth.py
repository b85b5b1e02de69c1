"""Seeded synthetic inputs for the KDA operator (shared by the CUDA path's tests/bench and the oracle).

This module draws random inputs only; it holds none of the operator's arithmetic.  The value
distributions follow the operator's documented workloads:

* q, k ~ N(0, 1), then L2-normalised per (token, head) over the key axis in fp32, then cast to
  the q/k/v dtype (bf16 rounding is round-to-nearest-even, done by torch).
* v ~ N(0, 1).
* log_alpha = log sigmoid(x), x ~ N(3, 1), drawn independently per (token, head, key channel);
  evaluated in fp64 and stored as fp32.
* beta = sigmoid(x), x ~ N(0, 1), per (token, head), fp32.
* S0 ~ N(0, 0.02^2) (standard deviation 0.02) where a workload starts from a random state.
* varlen lengths: 8 integers uniform in [1024, 16384] summing to 65536, by seeded rejection
  sampling (7 draws, the 8th is the remainder, redraw until it is in range).

Everything is generated with a ``torch.Generator`` on the requested device.  A test or the bench
hands the same tensors to the CUDA library and (as float32/float64 copies) to the oracle, so both
sides always see identical bits.
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import Optional

import numpy as np
import torch


@dataclass(frozen=True)
class Workload:
    """One named synthetic workload of the operator."""
    name: str
    kind: str                 # "prefill" or "decode"
    B: int                    # batch (prefill, regular) or number of sequences (decode)
    T: int                    # tokens per sequence (prefill); decode steps (decode)
    H: int
    dk: int
    dv: int
    dtype: str                # "bf16" or "f32" (q/k/v/out); gates and state are always fp32
    seed: int
    s0_std: float = 0.0       # 0 -> S0 = 0 (passed as NULL)
    varlen: Optional[tuple] = None   # (num_seqs, total, lo, hi) for packed varlen prefill
    desc: str = field(default="", compare=False)


WORKLOADS = {
    "tiny_fp32": Workload("tiny_fp32", "prefill", 1, 256, 2, 64, 64, "f32", 0,
                          desc="B=1 H=2 T=256 dk=dv=64, fp32 everything, S0=0"),
    "prefill_32k": Workload("prefill_32k", "prefill", 1, 32768, 32, 128, 128, "bf16", 1, s0_std=0.02,
                            desc="B=1 H=32 T=32768 dk=dv=128, bf16 q/k/v, fp32 gates/state, S0~N(0,0.02^2)"),
    "varlen_64k": Workload("varlen_64k", "prefill", 1, 65536, 32, 128, 128, "bf16", 2,
                           varlen=(8, 65536, 1024, 16384),
                           desc="8 packed sequences, lengths U[1024,16384] summing to 65536, H=32, dk=dv=128, bf16, S0=0"),
    "long_1m": Workload("long_1m", "prefill", 1, 1048576, 32, 128, 128, "bf16", 3,
                        desc="B=1 H=32 T=1048576 dk=dv=128, bf16 q/k/v, fp32 gates/state, S0=0"),
    "decode_256x512": Workload("decode_256x512", "decode", 256, 512, 32, 128, 128, "bf16", 4, s0_std=0.02,
                               desc="256 sequences x H=32, dk=dv=128, fp32 state ~N(0,0.02^2), 512 steps"),
}


def torch_dtype(name: str) -> torch.dtype:
    return {"bf16": torch.bfloat16, "f32": torch.float32}[name]


def varlen_lengths(seed: int, num: int = 8, total: int = 65536, lo: int = 1024, hi: int = 16384) -> list:
    """Seeded rejection sampling of ``num`` lengths in [lo, hi] that sum to ``total``."""
    rng = np.random.default_rng(seed)
    while True:
        head = rng.integers(lo, hi + 1, size=num - 1)
        last = total - int(head.sum())
        if lo <= last <= hi:
            return [int(x) for x in head] + [last]


def cu_from_lengths(lengths) -> np.ndarray:
    cu = np.zeros(len(lengths) + 1, dtype=np.int64)
    cu[1:] = np.cumsum(np.asarray(lengths, dtype=np.int64))
    return cu


def _gen(device, seed):
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def _normal(shape, g, device, mean=0.0, std=1.0, dtype=torch.float32):
    return torch.randn(shape, generator=g, device=device, dtype=dtype) * std + mean


def qk_normalised(shape, g, device, dtype):
    """N(0,1) draws, L2-normalised over the last axis in fp32, then cast to ``dtype``."""
    x = _normal(shape, g, device)
    x = x / torch.linalg.vector_norm(x, dim=-1, keepdim=True).clamp_min(1e-30)
    return x.to(dtype)


def log_sigmoid_gate(shape, g, device, mean=3.0, std=1.0):
    """log sigmoid(x), x ~ N(mean, std^2), evaluated in fp64, stored fp32."""
    x = _normal(shape, g, device, mean, std, dtype=torch.float64)
    return torch.nn.functional.logsigmoid(x).to(torch.float32)


def sigmoid_beta(shape, g, device):
    return torch.sigmoid(_normal(shape, g, device)).to(torch.float32)


def prefill_inputs(w: Workload, device="cpu", T: Optional[int] = None, H: Optional[int] = None,
                   seed: Optional[int] = None, lengths=None) -> dict:
    """Inputs for a prefill workload.  ``T``/``H``/``seed``/``lengths`` override the preset (for
    smaller parity cases of the same distributions).  Returns a dict with
    q, k, v ([B,T,H,d] or packed [1,Ttot,H,d]), log_alpha, beta, S0 (or None), cu_seqlens (int32
    tensor on ``device`` or None), lengths (list or None)."""
    T = w.T if T is None else T
    H = w.H if H is None else H
    seed = w.seed if seed is None else seed
    dt = torch_dtype(w.dtype)
    g = _gen(device, seed)
    if lengths is None and w.varlen is not None:
        n, total, lo, hi = w.varlen
        lengths = varlen_lengths(seed, n, total, lo, hi)
    if lengths is not None:
        B, Ttot, N = 1, int(sum(lengths)), len(lengths)
    else:
        B, Ttot, N = w.B, T, w.B
    q = qk_normalised((B, Ttot, H, w.dk), g, device, dt)
    k = qk_normalised((B, Ttot, H, w.dk), g, device, dt)
    v = _normal((B, Ttot, H, w.dv), g, device).to(dt)
    la = log_sigmoid_gate((B, Ttot, H, w.dk), g, device)
    beta = sigmoid_beta((B, Ttot, H), g, device)
    S0 = _normal((N, H, w.dk, w.dv), g, device, 0.0, w.s0_std) if w.s0_std > 0 else None
    cu = None
    if lengths is not None:
        cu = torch.from_numpy(cu_from_lengths(lengths).astype(np.int32)).to(device)
    return dict(q=q, k=k, v=v, log_alpha=la, beta=beta, S0=S0, cu_seqlens=cu, lengths=lengths)


def decode_state(w: Workload, device="cpu", N: Optional[int] = None, seed: Optional[int] = None):
    N = w.B if N is None else N
    g = _gen(device, (w.seed if seed is None else seed) * 1000003 + 17)
    return _normal((N, w.H, w.dk, w.dv), g, device, 0.0, w.s0_std)


def decode_inputs(w: Workload, step: int, device="cpu", N: Optional[int] = None, seed: Optional[int] = None,
                  steps: int = 1) -> dict:
    """Per-step decode inputs (fresh draws per step).  With ``steps > 1`` the tensors get a
    leading step axis: q,k [steps,N,H,dk], v [steps,N,H,dv], log_alpha [steps,N,H,dk],
    beta [steps,N,H]."""
    N = w.B if N is None else N
    dt = torch_dtype(w.dtype)
    g = _gen(device, (w.seed if seed is None else seed) * 7919 + step)
    lead = (steps,) if steps > 1 else ()
    q = qk_normalised(lead + (N, w.H, w.dk), g, device, dt)
    k = qk_normalised(lead + (N, w.H, w.dk), g, device, dt)
    v = _normal(lead + (N, w.H, w.dv), g, device).to(dt)
    la = log_sigmoid_gate(lead + (N, w.H, w.dk), g, device)
    beta = sigmoid_beta(lead + (N, w.H), g, device)
    return dict(q=q, k=k, v=v, log_alpha=la, beta=beta)


def to_oracle(x):
    """float32 numpy copy of a tensor (exact for bf16/fp32 values)."""
    if x is None:
        return None
    return x.detach().to("cpu", torch.float32).numpy()
