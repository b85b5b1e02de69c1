"""GPU parity of bf16 gate input (kda_options.prologue bit KDA_PROLOGUE_GATE_BF16, chosen by the
binding when log_alpha is a bf16 tensor).  The kernels widen each bf16 value to fp32 exactly, so the
prefill must give the same bits as the fp32 call on the widened values; both are also checked
against the fp64 oracle on those values (bf16 -> fp64 is exact)."""
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


def inputs(dtype, d, H, T=None, lengths=None, B=2, seed=21):
    w = synth.Workload("gate16", "prefill", B if lengths is None else 1, 0, H, d, d, dtype, seed, s0_std=0.5)
    inp = synth.prefill_inputs(w, T=T, lengths=lengths)
    inp["log_alpha"] = inp["log_alpha"].to(torch.bfloat16)
    return inp


def oracle_ref(inp, flags=0):
    q, k, v, la, b = (synth.to_oracle(inp[x]) for x in ("q", "k", "v", "log_alpha", "beta"))
    if flags:
        q, k, la, b = oracle.prologue(q, k, la, b, l2norm_qk=bool(flags & 1), gate_logits=bool(flags & 2),
                                      beta_logits=bool(flags & 4))
    S0 = None if inp["S0"] is None else inp["S0"].double().numpy()
    if inp["cu_seqlens"] is not None:
        cu = inp["cu_seqlens"].numpy().astype(np.int64)
        o, s = oracle.seq(q[0], k[0], v[0], la[0], b[0], S0=S0, cu_seqlens=cu)
        return o[None], s
    return oracle.seq(q, k, v, la, b, S0=S0)


def run_both(inp, flags=0):
    m = kda()
    g = {k_: (v_.to(DEV) if isinstance(v_, torch.Tensor) else v_) for k_, v_ in inp.items()}
    o16, s16 = m.chunk_fwd(g["q"], g["k"], g["v"], g["log_alpha"], g["beta"], S0=g["S0"],
                           cu_seqlens=g["cu_seqlens"], prologue=flags)
    o32, s32 = m.chunk_fwd(g["q"], g["k"], g["v"], g["log_alpha"].float(), g["beta"], S0=g["S0"],
                           cu_seqlens=g["cu_seqlens"], prologue=flags)
    m.check()
    return o16, s16, o32, s32


@pytest.mark.parametrize("dtype,d,H,T", [("bf16", 128, 4, 200), ("bf16", 128, 3, 64), ("f32", 64, 3, 150),
                                          ("bf16", 64, 2, 97), ("f32", 128, 2, 70)])
def test_bf16_gates_match_fp32_gates_bitwise(dtype, d, H, T):
    inp = inputs(dtype, d, H, T=T)
    o16, s16, o32, s32 = run_both(inp)
    assert torch.equal(o16, o32) and torch.equal(s16, s32)
    o_ref, s_ref = oracle_ref(inp)
    tol_o, tol_s = TOL[dtype]
    assert out_err(np64(o16), o_ref) <= tol_o
    assert state_err(np64(s16), s_ref) <= tol_s


def test_bf16_gates_varlen_ragged():
    """Sequences ending inside a chunk: the rows past the end of the bf16 box (another sequence's
    gates, or the zeros past the tensor) must stay identity steps."""
    inp = inputs("bf16", 128, 3, lengths=[1, 63, 65, 130, 7])
    o16, s16, o32, s32 = run_both(inp)
    assert torch.equal(o16, o32) and torch.equal(s16, s32)
    o_ref, s_ref = oracle_ref(inp)
    assert out_err(np64(o16), o_ref) <= TOL["bf16"][0]
    assert state_err(np64(s16), s_ref) <= TOL["bf16"][1]


def test_bf16_gate_logits_with_full_prologue():
    """Raw bf16 gate logits (log sigmoid inside the scan) together with the q/k and beta transforms."""
    g = torch.Generator().manual_seed(3)
    B, T, H, d = 2, 140, 4, 128
    q = (torch.randn(B, T, H, d, generator=g) * 3.0).to(torch.bfloat16)
    k = (torch.randn(B, T, H, d, generator=g) * 0.2).to(torch.bfloat16)
    v = torch.randn(B, T, H, d, generator=g).to(torch.bfloat16)
    a = (torch.randn(B, T, H, d, generator=g) + 3.0).to(torch.bfloat16)
    b = torch.randn(B, T, H, generator=g)
    S0 = torch.randn(B, H, d, d, generator=g) * 0.3
    inp = dict(q=q, k=k, v=v, log_alpha=a, beta=b, S0=S0, cu_seqlens=None)
    o16, s16, o32, s32 = run_both(inp, flags=7)
    assert torch.equal(o16, o32) and torch.equal(s16, s32)
    o_ref, s_ref = oracle_ref(inp, flags=7)
    assert out_err(np64(o16), o_ref) <= TOL["bf16"][0]
    assert state_err(np64(s16), s_ref) <= TOL["bf16"][1]


@pytest.mark.parametrize("dtype,d", [("bf16", 128), ("f32", 64)])
def test_bf16_gates_decode(dtype, d):
    m = kda()
    N, H, steps = 6, 4, 3
    w = synth.Workload("gate16d", "decode", N, steps, H, d, d, dtype, 23, s0_std=0.3)
    S0 = (torch.randn(N, H, d, d, generator=torch.Generator().manual_seed(24)) * 0.3).to(DEV)
    S16, S32, S_ref = S0.clone(), S0.clone(), np64(S0)
    for t in range(steps):
        st = synth.decode_inputs(w, t, device=DEV)
        la16 = st["log_alpha"].to(torch.bfloat16)
        o16 = m.decode_step(st["q"], st["k"], st["v"], la16, st["beta"], S16)
        o32 = m.decode_step(st["q"], st["k"], st["v"], la16.float(), st["beta"], S32)
        m.check()
        o_ref, S_ref = oracle.decode_step(*(synth.to_oracle(x.cpu()) for x in (st["q"], st["k"], st["v"], la16,
                                                                                  st["beta"])), S_ref)
        # same inputs, another kernel instance: equal up to the order the compiler gives the fp32 ops
        assert (o16.float() - o32.float()).abs().max() <= 1e-6 * (1.0 + o32.float().abs().max())
        assert out_err(np64(o16), o_ref) <= TOL[dtype][0]
    assert state_err(np64(S16), S_ref) <= TOL[dtype][1]
    assert (S16 - S32).abs().max() <= 1e-6 * (1.0 + S32.abs().max())
