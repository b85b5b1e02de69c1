"""Shared helpers for the GPU parity tests: tolerances, comparisons, oracle calls on test inputs."""
import numpy as np
import torch

import oracle
from gated_delta_rule_83_b200 import synth

# Tolerances fixed for the operator: bf16 q/k/v with fp32 gates/state -> max-abs error on outputs
# <= 2e-2 * max|o| and relative Frobenius error on final states <= 1e-2; all-fp32 -> 1e-4 for both.
TOL = {"bf16": (2e-2, 1e-2), "f32": (1e-4, 1e-4)}


def out_err(o_gpu, o_ref):
    o_gpu = np.asarray(o_gpu, np.float64)
    o_ref = np.asarray(o_ref, np.float64)
    return float(np.max(np.abs(o_gpu - o_ref)) / max(np.max(np.abs(o_ref)), 1e-30))


def state_err(s_gpu, s_ref):
    s_gpu = np.asarray(s_gpu, np.float64)
    s_ref = np.asarray(s_ref, np.float64)
    return float(np.linalg.norm(s_gpu - s_ref) / max(np.linalg.norm(s_ref), 1e-30))


def np64(t):
    return t.detach().to("cpu", torch.float64).numpy()


def oracle_prefill(inp, pairs=None, threads=None):
    """Oracle on the exact values in ``inp`` (a synth.prefill_inputs dict)."""
    q, k, v, la, b = (synth.to_oracle(inp[x]) for x in ("q", "k", "v", "log_alpha", "beta"))
    S0 = None if inp["S0"] is None else inp["S0"].detach().cpu().double().numpy()
    if inp["cu_seqlens"] is not None:
        cu = inp["cu_seqlens"].cpu().numpy().astype(np.int64)
        out, sf = oracle.seq(q[0], k[0], v[0], la[0], b[0], S0=S0, cu_seqlens=cu, pairs=pairs, threads=threads)
        return out[None], sf
    return oracle.seq(q, k, v, la, b, S0=S0, pairs=pairs, threads=threads)


def to_device(inp, device):
    return {k: (v.to(device) if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
