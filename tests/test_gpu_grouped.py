"""GPU parity of grouped q/k heads (kda_chunk_fwd_ex / kda_decode_step_ex with
kda_options.num_qk_heads = Hk < H): value head h reads q/k head h // (H // Hk), every other tensor
keeps H heads.  Checked against the fp64 oracle's grouped form on the same input bits, and against
the plain entry points run on q and k repeated over each group (which must give identical bits)."""
import numpy as np
import pytest
import torch

import oracle
from gated_delta_rule_83_b200 import synth
from tests.kda_testutil import TOL, np64, out_err, state_err

pytestmark = pytest.mark.gpu
DEV = "cuda"


def kda():
    import gated_delta_rule_83_b200 as m
    return m


def grouped_inputs(dtype, d, H, Hk, T=None, lengths=None, B=2, seed=5):
    w = synth.Workload("grouped", "prefill", B if lengths is None else 1, 0, H, d, d, dtype, seed, s0_std=0.5)
    inp = synth.prefill_inputs(w, T=T, lengths=lengths)
    inp["q"] = inp["q"][:, :, :Hk].contiguous()   # the first Hk heads: L2-normalised like all of them
    inp["k"] = inp["k"][:, :, :Hk].contiguous()
    return inp


def oracle_grouped(inp):
    q, k, v, la, b = (synth.to_oracle(inp[x]) for x in ("q", "k", "v", "log_alpha", "beta"))
    S0 = None if inp["S0"] is None else inp["S0"].double().numpy()
    if inp["cu_seqlens"] is not None:
        cu = inp["cu_seqlens"].numpy().astype(np.int64)
        o, s = oracle.seq(q[0], k[0], v[0], la[0], b[0], S0=S0, cu_seqlens=cu)
        return o[None], s
    return oracle.seq(q, k, v, la, b, S0=S0)


@pytest.mark.parametrize("dtype,d,H,Hk,T", [("bf16", 128, 4, 2, 200), ("bf16", 128, 4, 1, 130),
                                              ("f32", 64, 4, 2, 150), ("bf16", 64, 6, 3, 97),
                                              ("f32", 128, 2, 1, 70)])
def test_grouped_prefill_matches_oracle(dtype, d, H, Hk, T):
    m = kda()
    inp = grouped_inputs(dtype, d, H, Hk, T=T)
    g = {k_: (v_.to(DEV) if isinstance(v_, torch.Tensor) else v_) for k_, v_ in inp.items()}
    out, sf = m.chunk_fwd(g["q"], g["k"], g["v"], g["log_alpha"], g["beta"], S0=g["S0"])
    m.check()
    o_ref, s_ref = oracle_grouped(inp)
    tol_o, tol_s = TOL[dtype]
    assert out_err(np64(out), o_ref) <= tol_o
    assert state_err(np64(sf), s_ref) <= tol_s
    # identical bits to the one-head-per-value-head call on repeated q and k
    G = H // Hk
    out2, sf2 = m.chunk_fwd(g["q"].repeat_interleave(G, dim=2).contiguous(),
                            g["k"].repeat_interleave(G, dim=2).contiguous(), g["v"], g["log_alpha"], g["beta"],
                            S0=g["S0"])
    m.check()
    assert torch.equal(out, out2) and torch.equal(sf, sf2)


def test_grouped_varlen_prefill():
    m = kda()
    inp = grouped_inputs("bf16", 128, 6, 3, lengths=[70, 130, 64, 1])
    g = {k_: (v_.to(DEV) if isinstance(v_, torch.Tensor) else v_) for k_, v_ in inp.items()}
    out, sf = m.chunk_fwd(g["q"], g["k"], g["v"], g["log_alpha"], g["beta"], S0=g["S0"], cu_seqlens=g["cu_seqlens"])
    m.check()
    o_ref, s_ref = oracle_grouped(inp)
    tol_o, tol_s = TOL["bf16"]
    assert out_err(np64(out), o_ref) <= tol_o
    assert state_err(np64(sf), s_ref) <= tol_s


@pytest.mark.parametrize("dtype,d,H,Hk", [("bf16", 128, 6, 2), ("f32", 128, 4, 1), ("bf16", 64, 4, 2)])
def test_grouped_decode_matches_oracle(dtype, d, H, Hk):
    m = kda()
    N, steps = 5, 4
    w = synth.Workload("gd", "decode", N, steps, H, d, d, dtype, 41, s0_std=0.3)
    S = (torch.randn(N, H, d, d, generator=torch.Generator().manual_seed(42)) * 0.3).to(DEV)
    S_ref = np64(S)
    for t in range(steps):
        st = synth.decode_inputs(w, t, device=DEV)
        q, k = st["q"][:, :Hk].contiguous(), st["k"][:, :Hk].contiguous()
        o = m.decode_step(q, k, st["v"], st["log_alpha"], st["beta"], S)
        m.check()
        o_ref, S_ref = oracle.decode_step(*(synth.to_oracle(x.cpu()) for x in (q, k, st["v"], st["log_alpha"],
                                                                                  st["beta"])), S_ref)
        assert out_err(np64(o), o_ref) <= TOL[dtype][0]
    assert state_err(np64(S), S_ref) <= TOL[dtype][1]
