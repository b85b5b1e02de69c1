"""GPU parity of kda_chunk_fwd_gated (the prefill with the output gate applied in its epilogue) against
the fp64 oracle: the oracle's recurrence output, then the oracle's grouped gated RMS norm, on the same
input bits.

Groups of 8, 16 and 32 channels are normalised inside one phase-B CTA; groups of 64 and 128 are summed
across the CTAs of a 4-CTA cluster, which the row-norm property test checks over every row of the
full-size workload.
"""
import numpy as np
import pytest
import torch

import oracle
from gated_delta_rule_83_b200 import synth
from tests.kda_testutil import TOL, np64, oracle_prefill, out_err

pytestmark = pytest.mark.gpu
DEV = "cuda"
EPS = 1e-6


def kda():
    import gated_delta_rule_83_b200 as m
    return m


def gate_inputs(shape, dv, dtype, seed):
    g = torch.Generator().manual_seed(seed)
    z = torch.randn(*shape, generator=g).to(dtype)
    w = torch.rand(dv, generator=g) + 0.5
    return z, w


def run_gated(inp, z, w, group, act, tol=None, pairs=None, prologue=0, Hk=None):
    m = kda()
    d = {k: (v.to(DEV) if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
    q, k = d["q"], d["k"]
    if Hk is not None:  # grouped q/k heads: every (H / Hk)-th head's q/k
        r = q.shape[2] // Hk
        q, k = q[:, :, ::r].contiguous(), k[:, :, ::r].contiguous()
    y, sf = m.chunk_fwd(q, k, d["v"], d["log_alpha"], d["beta"], S0=d["S0"], cu_seqlens=d["cu_seqlens"],
                        z=z.to(DEV), gate_weight=None if w is None else w.to(DEV), gate_group=group,
                        gate_eps=EPS, gate_act=act, prologue=prologue)
    m.check()
    ref_in = dict(inp)
    if Hk is not None:
        r = inp["q"].shape[2] // Hk
        ref_in["q"] = inp["q"][:, :, ::r].repeat_interleave(r, dim=2)
        ref_in["k"] = inp["k"][:, :, ::r].repeat_interleave(r, dim=2)
    o_ref, _ = oracle_prefill(ref_in, pairs=pairs)
    y_ref = oracle.gated_rmsnorm(o_ref, np64(z), weight=None if w is None else w.numpy(),
                                 group=None if group == 0 else group, eps=EPS, gate=act)
    y_gpu = np64(y)
    assert np.all(np.isfinite(y_gpu))
    tol = tol or TOL["bf16" if inp["q"].dtype == torch.bfloat16 else "f32"][0]
    if pairs is None:
        e = out_err(y_gpu, y_ref)
        assert e <= tol, f"gated output error {e:.3e} > {tol}"
        return e
    worst = 0.0
    for n, h in pairs:
        e = out_err(y_gpu[n, :, h], y_ref[n, :, h])
        assert e <= tol, f"pair {(n, h)}: gated output error {e:.3e} > {tol}"
        worst = max(worst, e)
    return worst


@pytest.mark.parametrize("group", [0, 64, 32, 16, 8])
@pytest.mark.parametrize("act", ["none", "sigmoid"])
def test_gated_prefill_groups(group, act):
    """Every group size of the tensor-core path, both activations, with and without a weight."""
    w = synth.Workload("test", "prefill", 2, 0, 3, 128, 128, "bf16", 400 + group, s0_std=0.5)
    inp = synth.prefill_inputs(w, T=200)
    z, wt = gate_inputs((2, 200, 3, 128), 128, torch.bfloat16, seed=group)
    run_gated(inp, z, wt if group in (0, 16) else None, group, act)


@pytest.mark.parametrize("B,H,T", [(1, 72, 130), (3, 21, 257), (1, 2, 1), (4, 16, 64), (2, 1, 1000)])
def test_gated_prefill_launch_shapes(B, H, T):
    """Cluster-reduced groups (128) over many heads, several sequences, single tokens and one long chain."""
    w = synth.Workload("test", "prefill", B, 0, H, 128, 128, "bf16", 410 + T, s0_std=0.5)
    inp = synth.prefill_inputs(w, T=T)
    z, wt = gate_inputs((B, T, H, 128), 128, torch.bfloat16, seed=T)
    run_gated(inp, z, wt, 0, "sigmoid")


@pytest.mark.parametrize("group", [128, 32])
def test_gated_prefill_varlen(group):
    """Packed sequences, empty and one-token ones among them."""
    w = synth.Workload("test", "prefill", 1, 0, 4, 128, 128, "bf16", 421, s0_std=0.5)
    lengths = [3, 64, 65, 1, 200, 0, 129, 17, 90]
    inp = synth.prefill_inputs(w, lengths=lengths)
    z, wt = gate_inputs((1, sum(lengths), 4, 128), 128, torch.bfloat16, seed=group)
    run_gated(inp, z, wt, group, "sigmoid")


def test_gated_prefill_grouped_heads_and_prologue():
    """The gate combined with grouped q/k heads (Hk = H / 2) and the in-kernel input prologue."""
    m = kda()
    w = synth.Workload("test", "prefill", 1, 0, 4, 128, 128, "bf16", 431, s0_std=0.5)
    inp = synth.prefill_inputs(w, T=150)
    z, wt = gate_inputs((1, 150, 4, 128), 128, torch.bfloat16, seed=3)
    run_gated(inp, z, wt, 64, "sigmoid", Hk=2)
    # beta passed as logits: the oracle sees sigmoid(logit) of the same values
    inp2 = dict(inp)
    b = inp["beta"].double().clamp(1e-6, 1 - 1e-6)
    inp2["beta"] = torch.log(b / (1 - b)).float()
    ref = dict(inp2)
    ref["beta"] = torch.sigmoid(inp2["beta"].double()).float()
    y2, _ = m.chunk_fwd(*(inp2[x].to(DEV) for x in ("q", "k", "v", "log_alpha", "beta")), S0=inp2["S0"].to(DEV),
                        z=z.to(DEV), gate_weight=wt.to(DEV), gate_act="sigmoid", prologue=m.PROLOGUE_BETA_LOGITS)
    m.check()
    o_ref, _ = oracle_prefill(ref)
    y_ref = oracle.gated_rmsnorm(o_ref, np64(z), weight=wt.numpy(), eps=EPS, gate="sigmoid")
    assert out_err(np64(y2), y_ref) <= TOL["bf16"][0]


@pytest.mark.parametrize("dtype,dk,dv,group", [("f32", 128, 128, 0), ("f32", 64, 64, 16), ("bf16", 64, 64, 0),
                                               ("bf16", 128, 64, 32)])
def test_gated_prefill_cuda_core_paths(dtype, dk, dv, group):
    """Shapes and dtypes outside the tensor-core path: the prefill, then the gate in place."""
    w = synth.Workload("test", "prefill", 2, 0, 2, dk, dv, dtype, 441, s0_std=0.5)
    inp = synth.prefill_inputs(w, T=130)
    z, wt = gate_inputs((2, 130, 2, dv), dv, synth.torch_dtype(dtype), seed=dv)
    run_gated(inp, z, wt, group, "sigmoid")


def test_gated_prefill_leaves_z_and_neighbours_untouched():
    m = kda()
    w = synth.Workload("test", "prefill", 1, 0, 4, 128, 128, "bf16", 451, s0_std=0.5)
    inp = synth.prefill_inputs(w, T=100, device=DEV)
    z, _ = gate_inputs((1, 100, 4, 128), 128, torch.bfloat16, seed=9)
    z = z.to(DEV)
    z_before = z.clone()
    n = 100 * 4 * 128
    buf = torch.full((n + 256,), 5, dtype=torch.bfloat16, device=DEV)
    out = buf[:n].view(1, 100, 4, 128)
    m.chunk_fwd(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"], S0=inp["S0"], out=out, z=z,
                gate_act="sigmoid")
    m.check()
    assert torch.equal(z, z_before)
    assert torch.all(buf[n:] == 5)


def test_gated_prefill_rejects_bad_gates():
    m = kda()
    w = synth.Workload("test", "prefill", 1, 0, 2, 128, 128, "bf16", 461, s0_std=0.5)
    inp = synth.prefill_inputs(w, T=64, device=DEV)
    z = torch.zeros(1, 64, 2, 128, dtype=torch.bfloat16, device=DEV)
    args = (inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"])
    for kw in ({"gate_group": 24}, {"gate_group": 256}, {"gate_group": 4}, {"gate_eps": 0.0}):
        with pytest.raises(m.KdaError):
            m.chunk_fwd(*args, z=z, **kw)
    with pytest.raises(ValueError):
        m.chunk_fwd(*args, z=z, gate_act="relu")
    with pytest.raises(TypeError):
        m.chunk_fwd(*args, z=z.float())


# ------------------------------------------------------------------------------------------------
# full-size workload
# ------------------------------------------------------------------------------------------------
def test_gated_prefill_32k_sampled_and_row_norms():
    """T = 32,768, H = 32, the 128-channel group reduced across each head's cluster: heads 0, 17 and
    31 against the oracle over all tokens; and with z = 1, w = 1, act = identity every row of every
    head has mean(y^2) = |o|^2 / (|o|^2 + 128 eps) (= 1 up to eps) -- a missing or doubled share of
    the cross-CTA sum would move it by 25 % or more."""
    m = kda()
    w = synth.WORKLOADS["prefill_32k"]
    inp = synth.prefill_inputs(w, device=DEV)
    z, wt = gate_inputs((1, 32768, 32, 128), 128, torch.bfloat16, seed=32)
    pairs = [(0, 0), (0, 17), (0, 31)]
    e = run_gated(inp, z, wt, 0, "sigmoid", pairs=pairs)
    print(f"\nPARITY prefill_32k gated (group 128, sigmoid) heads 0/17/31: max-abs y error / max|y| = {e:.3e} "
          f"(tol {TOL['bf16'][0]:g})")
    ones = torch.ones(1, 32768, 32, 128, dtype=torch.bfloat16, device=DEV)
    y, _ = m.chunk_fwd(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"], S0=inp["S0"], z=ones)
    m.check()
    ms = y.float().pow(2).mean(-1)
    dev = (ms - 1).abs().max().item()
    print(f"PARITY prefill_32k gated row norms: max |mean(y^2) - 1| = {dev:.3e} over {ms.numel()} rows")
    assert dev <= 2e-2
