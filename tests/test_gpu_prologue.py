"""GPU parity of the input prologue (kda_options.prologue): raw q/k normalised inside the kernels,
raw gate logits turned into log sigmoid, raw beta logits into sigmoid.  Reference: the fp64
``oracle.prologue`` transform followed by the oracle recurrence, on the same raw input bits."""
import numpy as np
import pytest
import torch

import oracle
from gated_delta_rule_83_b200 import synth
from tests.kda_testutil import TOL, np64, out_err, state_err

pytestmark = pytest.mark.gpu
DEV = "cuda"
ALL = 7  # L2NORM_QK | GATE_LOGITS | BETA_LOGITS


def kda():
    import gated_delta_rule_83_b200 as m
    return m


def raw_inputs(dtype, d, H, Hk=None, B=2, T=None, lengths=None, seed=9):
    """Un-normalised q/k (scaled so the norm matters), gate logits ~ N(3, 1), beta logits ~ N(0, 1)."""
    g = torch.Generator().manual_seed(seed)
    dt = torch.bfloat16 if dtype == "bf16" else torch.float32
    Hk = H if Hk is None else Hk
    if lengths is not None:
        B, Ttot = 1, int(sum(lengths))
        cu = torch.tensor(np.concatenate([[0], np.cumsum(lengths)]), dtype=torch.int32)
    else:
        Ttot, cu = T, None
    N = B if cu is None else len(lengths)
    q = (torch.randn(B, Ttot, Hk, d, generator=g) * 3.0).to(dt)
    k = (torch.randn(B, Ttot, Hk, d, generator=g) * 0.2).to(dt)
    v = torch.randn(B, Ttot, H, d, generator=g).to(dt)
    a = torch.randn(B, Ttot, H, d, generator=g) + 3.0
    b = torch.randn(B, Ttot, H, generator=g)
    S0 = torch.randn(N, H, d, d, generator=g) * 0.3
    return dict(q=q, k=k, v=v, log_alpha=a, beta=b, S0=S0, cu_seqlens=cu)


def oracle_ref(inp, flags):
    q, k, v, la, b = (synth.to_oracle(inp[x]) for x in ("q", "k", "v", "log_alpha", "beta"))
    q, k, la, b = oracle.prologue(q, k, la, b, l2norm_qk=bool(flags & 1), gate_logits=bool(flags & 2),
                                  beta_logits=bool(flags & 4))
    S0 = inp["S0"].double().numpy()
    if inp["cu_seqlens"] is not None:
        cu = inp["cu_seqlens"].numpy().astype(np.int64)
        o, s = oracle.seq(q[0], k[0], v[0], la[0], b[0], S0=S0, cu_seqlens=cu)
        return o[None], s
    return oracle.seq(q, k, v, la, b, S0=S0)


def run(inp, flags, dtype):
    m = kda()
    g = {k_: (v_.to(DEV) if isinstance(v_, torch.Tensor) else v_) for k_, v_ in inp.items()}
    out, sf = m.chunk_fwd(g["q"], g["k"], g["v"], g["log_alpha"], g["beta"], S0=g["S0"],
                          cu_seqlens=g["cu_seqlens"], prologue=flags)
    m.check()
    o_ref, s_ref = oracle_ref(inp, flags)
    tol_o, tol_s = TOL[dtype]
    eo, es = out_err(np64(out), o_ref), state_err(np64(sf), s_ref)
    assert eo <= tol_o, f"output error {eo:.3e}"
    assert es <= tol_s, f"state error {es:.3e}"


@pytest.mark.parametrize("flags", [1, 2, 4, ALL])
def test_prologue_tensor_core_path(flags):
    """bf16, d = 128 (tensor-core path), two sequences with a ragged last chunk."""
    inp = raw_inputs("bf16", 128, 4, T=200)
    if not flags & 1:  # without in-kernel normalisation the keys must already be unit vectors
        inp["q"] = torch.nn.functional.normalize(inp["q"].float(), dim=-1).to(torch.bfloat16)
        inp["k"] = torch.nn.functional.normalize(inp["k"].float(), dim=-1).to(torch.bfloat16)
    if not flags & 2:
        inp["log_alpha"] = torch.nn.functional.logsigmoid(inp["log_alpha"])
    if not flags & 4:
        inp["beta"] = torch.sigmoid(inp["beta"])
    run(inp, flags, "bf16")


@pytest.mark.parametrize("dtype,d", [("f32", 64), ("bf16", 64), ("f32", 128)])
def test_prologue_cuda_core_path(dtype, d):
    run(raw_inputs(dtype, d, 3, T=150), ALL, dtype)


def test_prologue_varlen_tails_are_identity_steps():
    """Sequences whose last chunk is partial: the padded rows must stay identity steps after the
    activations (a zero logit would otherwise mean alpha = beta = 1/2)."""
    run(raw_inputs("bf16", 128, 2, lengths=[1, 63, 65, 130]), ALL, "bf16")


def test_prologue_with_grouped_heads():
    run(raw_inputs("bf16", 128, 4, Hk=2, T=140), ALL, "bf16")


@pytest.mark.parametrize("dtype,d,Hk", [("bf16", 128, 4), ("f32", 64, 4), ("bf16", 128, 2)])
def test_prologue_decode(dtype, d, Hk):
    m = kda()
    N, H, steps = 5, 4, 3
    g = torch.Generator().manual_seed(77)
    dt = torch.bfloat16 if dtype == "bf16" else torch.float32
    S = (torch.randn(N, H, d, d, generator=g) * 0.3).to(DEV)
    S_ref = np64(S)
    for _ in range(steps):
        q = (torch.randn(N, Hk, d, generator=g) * 2.0).to(dt)
        k = (torch.randn(N, Hk, d, generator=g) * 0.5).to(dt)
        v = torch.randn(N, H, d, generator=g).to(dt)
        a = torch.randn(N, H, d, generator=g) + 3.0
        b = torch.randn(N, H, generator=g)
        o = m.decode_step(q.to(DEV), k.to(DEV), v.to(DEV), a.to(DEV), b.to(DEV), S, prologue=ALL)
        m.check()
        qn, kn, la, bb = oracle.prologue(*(synth.to_oracle(x) for x in (q, k, a, b)), l2norm_qk=True,
                                         gate_logits=True, beta_logits=True)
        o_ref, S_ref = oracle.decode_step(qn, kn, synth.to_oracle(v), la, bb, S_ref)
        assert out_err(np64(o), o_ref) <= TOL[dtype][0]
    assert state_err(np64(S), S_ref) <= TOL[dtype][1]
