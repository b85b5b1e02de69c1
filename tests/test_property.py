"""Property-based parity: random small shapes, length mixes and gate ranges, drawn by hypothesis
with a fixed derandomised seed (the same examples every run).

* CPU (oracle): the chunked WY/UT form equals the step-by-step recurrence for any chunk size, and
  a packed varlen call equals separate calls, on every drawn case.
* GPU: the library's prefill (tensor-core or CUDA-core path, by dtype and d) and its backward match
  the oracle on every drawn case, within the operator's tolerances."""
import numpy as np
import pytest
import torch
from hypothesis import HealthCheck, given, settings
from hypothesis import strategies as st

import oracle
from gated_delta_rule_83_b200 import synth
from tests.kda_testutil import TOL, np64, out_err, state_err

SETTINGS = dict(derandomize=True, deadline=None, suppress_health_check=list(HealthCheck), database=None)


def case_inputs(seed, lengths, H, dk, dv, gate_lo, dtype="f32", s0=True):
    """Seeded inputs with the workload's distributions, except the gate: log alpha uniform in
    [gate_lo, 0] per channel (from almost no decay to strong decay)."""
    g = torch.Generator().manual_seed(seed)
    Ttot = int(sum(lengths))
    dt = torch.bfloat16 if dtype == "bf16" else torch.float32
    q = torch.nn.functional.normalize(torch.randn(1, Ttot, H, dk, generator=g), dim=-1).to(dt)
    k = torch.nn.functional.normalize(torch.randn(1, Ttot, H, dk, generator=g), dim=-1).to(dt)
    v = torch.randn(1, Ttot, H, dv, generator=g).to(dt)
    la = gate_lo * torch.rand(1, Ttot, H, dk, generator=g)
    b = torch.rand(1, Ttot, H, generator=g)
    N = len(lengths)
    S0 = torch.randn(N, H, dk, dv, generator=g) * 0.3 if s0 else None
    cu = torch.tensor(np.concatenate([[0], np.cumsum(lengths)]), dtype=torch.int32)
    return dict(q=q, k=k, v=v, log_alpha=la, beta=b, S0=S0, cu_seqlens=cu)


lengths_st = st.lists(st.integers(min_value=0, max_value=150), min_size=1, max_size=4).filter(lambda x: sum(x) > 0)


@settings(max_examples=25, **SETTINGS)
@given(seed=st.integers(0, 10_000), lengths=lengths_st, H=st.integers(1, 3), dk=st.sampled_from([2, 3, 8]),
       dv=st.sampled_from([1, 4, 5]), C=st.sampled_from([1, 3, 16, 64]), gate_lo=st.sampled_from([-0.05, -2.0, -30.0]))
def test_oracle_chunked_equals_sequential(seed, lengths, H, dk, dv, C, gate_lo):
    inp = case_inputs(seed, lengths, H, dk, dv, gate_lo)
    args = [synth.to_oracle(inp[x])[0] for x in ("q", "k", "v", "log_alpha", "beta")]
    cu = inp["cu_seqlens"].numpy().astype(np.int64)
    S0 = inp["S0"].double().numpy()
    o1, s1 = oracle.seq(*args, S0=S0, cu_seqlens=cu)
    o2, s2 = oracle.chunked(*args, S0=S0, cu_seqlens=cu, C=C)
    scale = max(np.max(np.abs(o1)), 1e-300)
    assert np.max(np.abs(o1 - o2)) <= 1e-9 * scale
    assert np.max(np.abs(s1 - s2)) <= 1e-9 * max(np.max(np.abs(s1)), 1e-300)


@settings(max_examples=15, **SETTINGS)
@given(seed=st.integers(0, 10_000), lengths=lengths_st, H=st.integers(1, 2), dk=st.sampled_from([2, 4]),
       dv=st.sampled_from([1, 3]))
def test_oracle_varlen_equals_separate(seed, lengths, H, dk, dv):
    inp = case_inputs(seed, lengths, H, dk, dv, -1.0)
    args = [synth.to_oracle(inp[x])[0] for x in ("q", "k", "v", "log_alpha", "beta")]
    cu = inp["cu_seqlens"].numpy().astype(np.int64)
    S0 = inp["S0"].double().numpy()
    o, s = oracle.seq(*args, S0=S0, cu_seqlens=cu)
    for n in range(len(lengths)):
        sl = slice(cu[n], cu[n + 1])
        on, sn = oracle.seq(*(a[sl] for a in args), S0=S0[n:n + 1])
        np.testing.assert_array_equal(o[sl], on)
        np.testing.assert_array_equal(s[n], sn[0])


def _kda():
    import gated_delta_rule_83_b200 as m
    return m


@pytest.mark.gpu
@settings(max_examples=20, **SETTINGS)
@given(seed=st.integers(0, 10_000), lengths=lengths_st, H=st.integers(1, 3),
       cfg=st.sampled_from([("bf16", 128, 128), ("f32", 64, 64), ("bf16", 64, 128), ("f32", 128, 64)]),
       gate_lo=st.sampled_from([-0.05, -1.0, -12.0]))
def test_gpu_prefill_matches_oracle(seed, lengths, H, cfg, gate_lo):
    dtype, dk, dv = cfg
    m = _kda()
    inp = case_inputs(seed, lengths, H, dk, dv, gate_lo, dtype)
    d = {k_: (v_.to("cuda") if isinstance(v_, torch.Tensor) else v_) for k_, v_ in inp.items()}
    out, sf = m.chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], S0=d["S0"], cu_seqlens=d["cu_seqlens"])
    m.check()
    args = [synth.to_oracle(inp[x])[0] for x in ("q", "k", "v", "log_alpha", "beta")]
    o_ref, s_ref = oracle.seq(*args, S0=inp["S0"].double().numpy(), cu_seqlens=inp["cu_seqlens"].numpy().astype(np.int64))
    tol_o, tol_s = TOL[dtype]
    assert out_err(np64(out)[0], o_ref) <= tol_o
    assert state_err(np64(sf), s_ref) <= tol_s


@pytest.mark.gpu
@settings(max_examples=10, **SETTINGS)
@given(seed=st.integers(0, 10_000), lengths=lengths_st, H=st.integers(1, 2),
       cfg=st.sampled_from([("bf16", 128, 128), ("f32", 64, 64)]), gate_lo=st.sampled_from([-0.05, -1.0, -12.0]))
def test_gpu_backward_matches_oracle(seed, lengths, H, cfg, gate_lo):
    dtype, dk, dv = cfg
    m = _kda()
    inp = case_inputs(seed, lengths, H, dk, dv, gate_lo, dtype)
    g = torch.Generator().manual_seed(seed + 1)
    do = torch.randn(inp["v"].shape, generator=g).to(inp["v"].dtype)
    d = {k_: (v_.to("cuda") if isinstance(v_, torch.Tensor) else v_) for k_, v_ in inp.items()}
    gr = m.chunk_bwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], do.to("cuda"), S0=d["S0"],
                     cu_seqlens=d["cu_seqlens"])
    m.check()
    args = [synth.to_oracle(inp[x])[0] for x in ("q", "k", "v", "log_alpha", "beta")]
    ref = oracle.bwd(*args, do.double().numpy()[0], S0=inp["S0"].double().numpy(),
                     cu_seqlens=inp["cu_seqlens"].numpy().astype(np.int64))
    tol = {"f32": 1e-3, "bf16": 1e-2}[dtype]
    for key in ("dq", "dk", "dv", "dlog_alpha", "dbeta", "dS0"):
        got = np64(gr[key])
        got = got if key == "dS0" else got[0]
        err = np.max(np.abs(got - ref[key])) / max(np.max(np.abs(ref[key])), 1e-30)
        assert err <= tol, f"{key}: {err:.3e}"
