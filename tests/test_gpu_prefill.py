"""GPU parity of kda_chunk_fwd (through the C ABI) against the fp64 oracle, element by element.

Small cases span several chunks and ragged tails; full-size workloads are compared on sampled
(sequence, head) pairs that the oracle recomputes from the very same input bits.
"""
import math

import numpy as np
import pytest
import torch

from gated_delta_rule_83_b200 import synth
from tests.kda_testutil import TOL, np64, oracle_prefill, out_err, state_err

pytestmark = pytest.mark.gpu

DEV = "cuda"


def kda():
    import gated_delta_rule_83_b200 as m
    return m


def small_workload(dtype="bf16", dk=128, dv=128, s0_std=0.5, seed=123):
    return synth.Workload("test", "prefill", 2, 0, 2, dk, dv, dtype, seed, s0_std=s0_std)


def run_and_compare(inp, dtype, pairs=None, check_all=True, tol=None):
    m = kda()
    d = {k: (v.to(DEV) if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
    out, sf = m.chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], S0=d["S0"], cu_seqlens=d["cu_seqlens"])
    m.check()
    o_ref, s_ref = oracle_prefill(inp, pairs=pairs)
    o_gpu, s_gpu = np64(out), np64(sf)
    tol_o, tol_s = tol or TOL[dtype]
    if pairs is None:
        eo, es = out_err(o_gpu, o_ref), state_err(s_gpu, s_ref)
        assert np.all(np.isfinite(o_gpu)) and np.all(np.isfinite(s_gpu))
        assert eo <= tol_o, f"output error {eo:.3e} > {tol_o}"
        assert es <= tol_s, f"state error {es:.3e} > {tol_s}"
        return eo, es
    worst = (0.0, 0.0)
    cu = None if inp["cu_seqlens"] is None else inp["cu_seqlens"].cpu().numpy()
    for n, h in pairs:
        if cu is None:
            og, orf = o_gpu[n, :, h], o_ref[n, :, h]
        else:
            og, orf = o_gpu[0, cu[n]:cu[n + 1], h], o_ref[0, cu[n]:cu[n + 1], h]
        eo, es = out_err(og, orf), state_err(s_gpu[n, h], s_ref[n, h])
        assert eo <= tol_o, f"pair {(n, h)}: output error {eo:.3e} > {tol_o}"
        assert es <= tol_s, f"pair {(n, h)}: state error {es:.3e} > {tol_s}"
        worst = (max(worst[0], eo), max(worst[1], es))
    return worst


def test_tiny_fp32_workload():
    """The all-fp32 tiny workload (B=1, H=2, T=256, d=64, S0=0), every output element."""
    w = synth.WORKLOADS["tiny_fp32"]
    run_and_compare(synth.prefill_inputs(w), "f32")


@pytest.mark.parametrize("T", [1, 63, 64, 65, 127, 300])
def test_bf16_d128_ragged(T):
    w = small_workload()
    run_and_compare(synth.prefill_inputs(w, T=T), "bf16")


@pytest.mark.parametrize("dtype,dk,dv,T", [("bf16", 64, 64, 200), ("f32", 128, 128, 130), ("f32", 128, 64, 97),
                                           ("f32", 64, 128, 129), ("bf16", 128, 64, 150), ("bf16", 64, 128, 70)])
def test_dtypes_and_dims(dtype, dk, dv, T):
    w = small_workload(dtype, dk, dv)
    run_and_compare(synth.prefill_inputs(w, T=T), dtype)


@pytest.mark.parametrize("B,H,T", [(1, 72, 130), (3, 21, 257), (2, 1, 1000), (4, 16, 64), (1, 2, 1), (1, 4, 65)])
def test_tc_launch_shapes(B, H, T):
    """Tensor-core prefill over many heads, several sequences of a regular batch, one long chain,
    one chunk per sequence and ragged tails."""
    w = synth.Workload("test", "prefill", B, 0, H, 128, 128, "bf16", 322, s0_std=0.5)
    run_and_compare(synth.prefill_inputs(w, T=T), "bf16")


def test_tc_many_sequences():
    """17 packed sequences of 4 heads, empty and one-token sequences among them."""
    w = synth.Workload("test", "prefill", 1, 0, 4, 128, 128, "bf16", 321, s0_std=0.5)
    lengths = [3, 64, 65, 1, 200, 0, 129, 64, 70, 17, 5, 90, 128, 33, 64, 100, 2]
    run_and_compare(synth.prefill_inputs(w, lengths=lengths), "bf16")


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_varlen_small(dtype):
    w = small_workload(dtype)
    inp = synth.prefill_inputs(w, lengths=[1, 63, 64, 65, 200, 17, 128])
    run_and_compare(inp, dtype)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("case", ["beta0", "alpha1", "strong_decay", "mixed_decay"])
def test_gate_edge_cases(dtype, case):
    w = small_workload(dtype)
    inp = synth.prefill_inputs(w, T=200)
    if case == "beta0":
        inp["beta"].zero_()
    elif case == "alpha1":
        inp["log_alpha"].zero_()
    elif case == "strong_decay":
        inp["log_alpha"].fill_(-30.0)
    else:  # a few channels decay extremely fast, the rest normally
        inp["log_alpha"][..., ::7] = -30.0
    run_and_compare(inp, dtype)


def test_zero_length_and_s0_none():
    m = kda()
    w = small_workload("bf16")
    inp = synth.prefill_inputs(w, T=0)
    d = {k: (v.to(DEV) if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
    out, sf = m.chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], S0=d["S0"])
    m.check()
    assert out.numel() == 0
    assert torch.equal(sf, d["S0"])
    # S0 = None -> zero initial state
    inp = synth.prefill_inputs(small_workload("f32", s0_std=0.0), T=70)
    run_and_compare(inp, "f32")


def test_inplace_state_passing_and_split():
    """S_final may alias S0; running T1 then T2 with the carried state equals one run of T1+T2."""
    m = kda()
    w = small_workload("f32")
    inp = synth.prefill_inputs(w, T=250)
    d = {k: (v.to(DEV) if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
    out_full, s_full = m.chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], S0=d["S0"])
    S = d["S0"].clone()
    outs = []
    for a, b in [(0, 100), (100, 101), (101, 250)]:
        sl = lambda x: x[:, a:b].contiguous()
        o, _ = m.chunk_fwd(sl(d["q"]), sl(d["k"]), sl(d["v"]), sl(d["log_alpha"]), sl(d["beta"]), S0=S, S_final=S)
        outs.append(o)
    m.check()
    o_ref, s_ref = oracle_prefill(inp)
    assert out_err(np64(torch.cat(outs, 1)), o_ref) < 1e-4
    assert state_err(np64(S), s_ref) < 1e-4
    assert state_err(np64(s_full), s_ref) < 1e-4


def test_canaries_untouched():
    """Guard bands around out and S_final stay bit-identical."""
    m = kda()
    w = small_workload("bf16")
    inp = synth.prefill_inputs(w, T=131)
    d = {k: (v.to(DEV) if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
    B, T, H, dv = d["v"].shape
    G = 4096
    ob = torch.full((2 * G + B * T * H * dv,), 7.25, dtype=torch.bfloat16, device=DEV)
    sb = torch.full((2 * G + B * H * 128 * dv,), -3.5, dtype=torch.float32, device=DEV)
    out = ob[G:G + B * T * H * dv].view(B, T, H, dv)
    sf = sb[G:G + B * H * 128 * dv].view(B, H, 128, dv)
    m.chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], S0=d["S0"], out=out, S_final=sf)
    m.check()
    assert torch.all(ob[:G] == 7.25) and torch.all(ob[-G:] == 7.25)
    assert torch.all(sb[:G] == -3.5) and torch.all(sb[-G:] == -3.5)


def test_bad_cu_seqlens_reported():
    m = kda()
    w = small_workload("bf16")
    inp = synth.prefill_inputs(w, lengths=[10, 20, 30])
    d = {k: (v.to(DEV) if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
    bad = torch.tensor([0, 20, 10, 60], dtype=torch.int32, device=DEV)   # decreasing
    out = torch.full_like(d["v"], 5.0)
    sf = torch.full((3, 2, 128, 128), 9.0, device=DEV)
    m.chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], cu_seqlens=bad, out=out, S_final=sf)
    with pytest.raises(m.KdaError) as ei:
        m.check()
    assert ei.value.code == 6
    assert torch.all(out == 5.0) and torch.all(sf == 9.0)
    m.check()  # the error word was cleared
    bad_total = torch.tensor([0, 10, 30, 59], dtype=torch.int32, device=DEV)   # cN != T
    m.chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], cu_seqlens=bad_total, out=out, S_final=sf)
    with pytest.raises(m.KdaError):
        m.check()


# ------------------------------------------------------------------------------------------------
# full-size workloads, sampled (sequence, head) pairs
# ------------------------------------------------------------------------------------------------
def report(name, eo, es):
    """Achieved errors of a full-size case against the tolerances (shown with ``pytest -s``)."""
    tol_o, tol_s = TOL["bf16"]
    print(f"\nPARITY {name}: max-abs out error / max|o| = {eo:.3e} (tol {tol_o:g}, margin {tol_o / max(eo, 1e-30):.1f}x); "
          f"relative Frobenius state error = {es:.3e} (tol {tol_s:g}, margin {tol_s / max(es, 1e-30):.1f}x)")


def test_prefill_32k_sampled():
    w = synth.WORKLOADS["prefill_32k"]
    inp = synth.prefill_inputs(w, device=DEV)
    report("prefill_32k heads 0/17/31", *run_and_compare(inp, "bf16", pairs=[(0, 0), (0, 17), (0, 31)]))


def test_varlen_64k_sampled():
    w = synth.WORKLOADS["varlen_64k"]
    inp = synth.prefill_inputs(w, device=DEV)
    report("varlen_64k pairs (0,5)/(3,12)/(7,31)", *run_and_compare(inp, "bf16", pairs=[(0, 5), (3, 12), (7, 31)]))


def test_long_1m_sampled():
    """T = 1,048,576: head 0 compared over the whole sequence (outputs and final state)."""
    m = kda()
    w = synth.WORKLOADS["long_1m"]
    inp = synth.prefill_inputs(w, device=DEV)
    out, sf = m.chunk_fwd(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"], S0=None)
    m.check()
    h = 0
    sub = {k: (inp[k][:, :, h:h + 1].contiguous() if k != "beta" else inp[k][:, :, h:h + 1].contiguous())
           for k in ("q", "k", "v", "log_alpha", "beta")}
    sub.update(S0=None, cu_seqlens=None)
    o_ref, s_ref = oracle_prefill(sub)
    og = np64(out[:, :, h:h + 1])
    eo, es = out_err(og, o_ref), state_err(np64(sf[:, h:h + 1]), s_ref)
    report("long_1m head 0", eo, es)
    assert eo <= TOL["bf16"][0]
    assert es <= TOL["bf16"][1]
