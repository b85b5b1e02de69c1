"""GPU parity of kda_decode_step (through the C ABI) against the fp64 oracle."""
import numpy as np
import pytest
import torch

import oracle
from gated_delta_rule_83_b200 import synth
from tests.kda_testutil import TOL, np64, oracle_prefill, out_err, state_err

pytestmark = pytest.mark.gpu
DEV = "cuda"


def kda():
    import gated_delta_rule_83_b200 as m
    return m


@pytest.mark.parametrize("dtype,dk,dv", [("bf16", 128, 128), ("f32", 128, 128), ("bf16", 64, 64),
                                         ("f32", 64, 128), ("f32", 128, 64)])
def test_decode_small(dtype, dk, dv):
    m = kda()
    w = synth.Workload("t", "decode", 5, 6, 3, dk, dv, dtype, 31, s0_std=0.3)
    S = synth.decode_state(w, device=DEV)
    S_ref = np64(S)
    for step in range(6):
        inp = synth.decode_inputs(w, step, device=DEV)
        out = m.decode_step(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"], S)
        m.check()
        o_ref, S_ref = oracle.decode_step(*(synth.to_oracle(inp[x]) for x in ("q", "k", "v", "log_alpha", "beta")),
                                          S_ref)
        assert out_err(np64(out), o_ref) <= TOL[dtype][0]
    assert state_err(np64(S), S_ref) <= TOL[dtype][1]


def test_decode_256x512_sampled():
    """The 256-sequence x 32-head workload, 512 steps, three (sequence, head) pairs followed by the oracle."""
    m = kda()
    w = synth.WORKLOADS["decode_256x512"]
    S = synth.decode_state(w, device=DEV)
    pairs = [(0, 0), (100, 7), (255, 31)]
    S_ref = np.stack([np64(S[n, h]) for n, h in pairs])[:, None]        # [P,1,dk,dv]
    worst = 0.0
    for step in range(w.T):
        inp = synth.decode_inputs(w, step, device=DEV)
        out = m.decode_step(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"], S)
        sel = {x: torch.stack([inp[x][n, h] for n, h in pairs])[:, None] for x in ("q", "k", "v", "log_alpha", "beta")}
        o_ref, S_ref = oracle.decode_step(*(synth.to_oracle(sel[x]) for x in ("q", "k", "v", "log_alpha", "beta")),
                                          S_ref)
        og = np.stack([np64(out[n, h]) for n, h in pairs])[:, None]
        worst = max(worst, out_err(og, o_ref))
    m.check()
    sg = np.stack([np64(S[n, h]) for n, h in pairs])[:, None]
    es = state_err(sg, S_ref)
    print(f"\nPARITY decode_256x512 pairs {pairs}: worst max-abs out error / max|o| over 512 steps = {worst:.3e} "
          f"(tol {TOL['bf16'][0]:g}); relative Frobenius state error after 512 steps = {es:.3e} "
          f"(tol {TOL['bf16'][1]:g})")
    assert worst <= TOL["bf16"][0]
    assert es <= TOL["bf16"][1]


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_decode_equals_prefill(dtype):
    """512 decode steps and one 512-token prefill on the same tokens agree with the oracle (and so
    with each other)."""
    m = kda()
    N, H, T = 3, 2, 512
    w = synth.Workload("t", "prefill", N, T, H, 128, 128, dtype, 77, s0_std=0.1)
    inp = synth.prefill_inputs(w, T=T)
    d = {k: (v.to(DEV) if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
    out_p, s_p = m.chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], S0=d["S0"])
    S = d["S0"].clone()
    outs = []
    for t in range(T):
        outs.append(m.decode_step(d["q"][:, t].contiguous(), d["k"][:, t].contiguous(), d["v"][:, t].contiguous(),
                                  d["log_alpha"][:, t].contiguous(), d["beta"][:, t].contiguous(), S))
    m.check()
    o_ref, s_ref = oracle_prefill(inp)
    out_d = torch.stack(outs, 1)
    assert out_err(np64(out_d), o_ref) <= TOL[dtype][0]
    assert out_err(np64(out_p), o_ref) <= TOL[dtype][0]
    assert state_err(np64(S), s_ref) <= TOL[dtype][1]
    assert state_err(np64(s_p), s_ref) <= TOL[dtype][1]


def test_decode_zero_batch():
    m = kda()
    e = torch.empty(0, 2, 64, device=DEV)
    out = m.decode_step(e.bfloat16(), e.bfloat16(), e.bfloat16(), e, torch.empty(0, 2, device=DEV),
                        torch.empty(0, 2, 64, 64, device=DEV))
    assert out.numel() == 0
