"""GPU parity of the chunked backward pass (``kda_chunk_bwd``) against the fp64 oracle's reverse-mode
derivative of the recurrence (``oracle.bwd``), on the same input bits and cotangents.

Tolerances (max-abs error over max |reference|, per gradient): the kernels work in fp32, so the
fp32 outputs (dlog_alpha, dbeta, dS0, and every gradient of an fp32 call) are held to 1e-3; bf16
calls return dq, dk, dv rounded to bf16 (relative step 2^-8), held to 1e-2."""
import numpy as np
import pytest
import torch

import oracle
from gated_delta_rule_83_b200 import synth
from tests.kda_testutil import np64

pytestmark = pytest.mark.gpu
DEV = "cuda"
BWD_TOL = {"f32": {"dq": 1e-3, "dk": 1e-3, "dv": 1e-3, "dlog_alpha": 1e-3, "dbeta": 1e-3, "dS0": 1e-3},
           "bf16": {"dq": 1e-2, "dk": 1e-2, "dv": 1e-2, "dlog_alpha": 1e-3, "dbeta": 1e-3, "dS0": 1e-3}}
KEYS = ("dq", "dk", "dv", "dlog_alpha", "dbeta", "dS0")


def kda():
    import gated_delta_rule_83_b200 as m
    return m


def max_rel(a, b):
    a, b = np.asarray(a, np.float64), np.asarray(b, np.float64)
    return float(np.max(np.abs(a - b)) / max(np.max(np.abs(b)), 1e-30))


def cotangents(inp, seed, with_dsf=True):
    g = torch.Generator().manual_seed(seed)
    v = inp["v"]
    N = v.shape[0] if inp["cu_seqlens"] is None else inp["cu_seqlens"].numel() - 1
    H, dk, dv = v.shape[2], inp["q"].shape[-1], v.shape[-1]
    do = torch.randn(v.shape, generator=g).to(v.dtype)
    dsf = torch.randn((N, H, dk, dv), generator=g) * 0.5 if with_dsf else None
    return do, dsf


def oracle_bwd(inp, do, dsf, pairs=None):
    q, k, v, la, b = (synth.to_oracle(inp[x].cpu()) for x in ("q", "k", "v", "log_alpha", "beta"))
    S0 = None if inp["S0"] is None else inp["S0"].detach().cpu().double().numpy()
    d_o = do.detach().cpu().double().numpy()
    d_sf = None if dsf is None else dsf.detach().cpu().double().numpy()
    if inp["cu_seqlens"] is not None:
        cu = inp["cu_seqlens"].cpu().numpy().astype(np.int64)
        g = oracle.bwd(q[0], k[0], v[0], la[0], b[0], d_o[0], S0=S0, dS_final=d_sf, cu_seqlens=cu, pairs=pairs)
        for key in ("dq", "dk", "dv", "dlog_alpha", "dbeta"):
            g[key] = g[key][None]
        return g
    return oracle.bwd(q, k, v, la, b, d_o, S0=S0, dS_final=d_sf, pairs=pairs)


def run_and_compare(inp, dtype, seed=1, with_dsf=True):
    m = kda()
    do, dsf = cotangents(inp, seed, with_dsf)
    d = {k_: (v_.to(DEV) if isinstance(v_, torch.Tensor) else v_) for k_, v_ in inp.items()}
    g = m.chunk_bwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], do.to(DEV), S0=d["S0"],
                    dS_final=None if dsf is None else dsf.to(DEV), cu_seqlens=d["cu_seqlens"])
    m.check()
    ref = oracle_bwd(inp, do, dsf)
    errs = {key: max_rel(np64(g[key]), ref[key]) for key in KEYS}
    bad = {key: e for key, e in errs.items() if not e <= BWD_TOL[dtype][key]}
    assert not bad, f"gradient errors above tolerance: {bad} (all: {errs})"
    return errs


@pytest.mark.parametrize("dtype,d,H,T", [("bf16", 128, 2, 200), ("f32", 64, 3, 150), ("f32", 128, 2, 130),
                                          ("bf16", 64, 2, 97), ("f32", 128, 1, 64)])
def test_backward_matches_oracle(dtype, d, H, T):
    w = synth.Workload("bwd", "prefill", 2, T, H, d, d, dtype, 31, s0_std=0.5)
    run_and_compare(synth.prefill_inputs(w), dtype)


@pytest.mark.parametrize("dk,dv", [(64, 128), (128, 64)])
def test_backward_rectangular_state(dk, dv):
    w = synth.Workload("bwd", "prefill", 1, 150, 2, dk, dv, "f32", 32, s0_std=0.5)
    run_and_compare(synth.prefill_inputs(w), "f32")


def test_backward_varlen_ragged():
    w = synth.Workload("bwdv", "prefill", 1, 0, 3, 128, 128, "bf16", 33, s0_std=0.5)
    run_and_compare(synth.prefill_inputs(w, lengths=[1, 63, 65, 130, 7]), "bf16")


def test_backward_without_state_inputs():
    """S0 = None and dS_final = None: zero initial state, no cotangent on the final state."""
    w = synth.Workload("bwd0", "prefill", 2, 100, 2, 128, 128, "bf16", 34)
    run_and_compare(synth.prefill_inputs(w), "bf16", with_dsf=False)


def test_backward_strong_decay_exact_factors():
    """Gates down to log alpha = -8: the in-chunk gate spread exceeds the factorised range, so the
    kernels take the exact per-element factors; the chunk-end decay underflows to 0."""
    w = synth.Workload("bwdw", "prefill", 1, 140, 2, 64, 64, "f32", 35, s0_std=0.5)
    inp = synth.prefill_inputs(w)
    g = torch.Generator().manual_seed(36)
    inp["log_alpha"] = -8.0 * torch.rand(inp["log_alpha"].shape, generator=g)
    run_and_compare(inp, "f32")


@pytest.mark.parametrize("channels", ["all", "first_tile"])
def test_backward_strong_decay_exact_factors_bf16(channels):
    """The same on the bf16 d = 128 path, whose input-side kernel runs on the tensor cores: a
    32-channel tile with a wide gate spread takes the exact per-element factors; with only the first
    tile's channels decaying fast, the other tiles keep the factorised form in the same unit."""
    w = synth.Workload("bwdw16", "prefill", 1, 140, 2, 128, 128, "bf16", 38, s0_std=0.5)
    inp = synth.prefill_inputs(w)
    g = torch.Generator().manual_seed(39)
    strong = -8.0 * torch.rand(inp["log_alpha"].shape, generator=g)
    if channels == "all":
        inp["log_alpha"] = strong
    else:
        inp["log_alpha"][..., :32] = strong[..., :32]
    run_and_compare(inp, "bf16")


def test_backward_bf16_gates():
    """log_alpha passed as bf16 (KDA_PROLOGUE_GATE_BF16): same result as the fp32 call on the
    widened values."""
    m = kda()
    w = synth.Workload("bwdg", "prefill", 2, 130, 2, 128, 128, "bf16", 37, s0_std=0.5)
    inp = synth.prefill_inputs(w)
    inp["log_alpha"] = inp["log_alpha"].to(torch.bfloat16)
    run_and_compare(inp, "bf16")
    do, dsf = cotangents(inp, 2)
    d = {k_: (v_.to(DEV) if isinstance(v_, torch.Tensor) else v_) for k_, v_ in inp.items()}
    g16 = m.chunk_bwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], do.to(DEV), S0=d["S0"],
                      dS_final=dsf.to(DEV))
    g32 = m.chunk_bwd(d["q"], d["k"], d["v"], d["log_alpha"].float(), d["beta"], do.to(DEV), S0=d["S0"],
                      dS_final=dsf.to(DEV))
    m.check()
    for key in KEYS:
        assert torch.equal(g16[key], g32[key]), key


def test_backward_directional_derivative_of_forward():
    """Property that holds at any size: <grad, delta> matches the change of the forward loss along
    delta (the CUDA forward itself, fp32 inputs, central difference)."""
    m = kda()
    w = synth.Workload("bwdfd", "prefill", 1, 256, 2, 64, 64, "f32", 38, s0_std=0.5)
    inp = {k_: (v_.to(DEV) if isinstance(v_, torch.Tensor) else v_) for k_, v_ in synth.prefill_inputs(w).items()}
    do, dsf = cotangents(inp, 3)
    do, dsf = do.to(DEV), dsf.to(DEV)
    g = m.chunk_bwd(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"], do, S0=inp["S0"], dS_final=dsf)
    gen = torch.Generator(device=DEV).manual_seed(39)
    eps = 1e-3
    names = {"q": "dq", "k": "dk", "v": "dv", "log_alpha": "dlog_alpha", "beta": "dbeta"}
    for name, key in names.items():
        delta = torch.randn(inp[name].shape, generator=gen, device=DEV)

        def loss(x):
            a = dict(inp)
            a[name] = x
            out, sf = m.chunk_fwd(a["q"], a["k"], a["v"], a["log_alpha"], a["beta"], S0=a["S0"])
            return float((out.double() * do.double()).sum() + (sf.double() * dsf.double()).sum())

        fd = (loss(inp[name] + eps * delta) - loss(inp[name] - eps * delta)) / (2 * eps)
        an = float((g[key].double() * delta.double()).sum())
        assert abs(fd - an) <= 2e-3 * abs(an) + 1e-3, f"{name}: fd {fd} vs grad {an}"
    m.check()


def test_backward_prefill_32k_sampled():
    """The full 32K x 32-head workload through the backward; heads 0 and 17 compared over the whole
    sequence (heads are independent, so the oracle runs on those two heads alone)."""
    m = kda()
    w = synth.WORKLOADS["prefill_32k"]
    inp = synth.prefill_inputs(w, device=DEV)
    g = torch.Generator(device=DEV).manual_seed(40)
    do = torch.randn(inp["v"].shape, generator=g, device=DEV).to(inp["v"].dtype)
    gr = m.chunk_bwd(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"], do, S0=inp["S0"])
    m.check()
    heads = [0, 17]
    sub = {k_: inp[k_][:, :, heads].contiguous() for k_ in ("q", "k", "v", "log_alpha", "beta")}
    sub.update(S0=None if inp["S0"] is None else inp["S0"][:, heads].contiguous(), cu_seqlens=None)
    ref = oracle_bwd(sub, do[:, :, heads].contiguous(), None)
    for key in KEYS:
        got = gr[key][:, heads] if key == "dS0" else gr[key][:, :, heads]
        e = max_rel(np64(got), ref[key])
        assert e <= BWD_TOL["bf16"][key], f"{key}: {e:.3e}"


@pytest.mark.parametrize("dtype,d,H,Hk,T", [("bf16", 128, 4, 2, 200), ("f32", 64, 6, 3, 150), ("bf16", 128, 4, 1, 97)])
def test_backward_grouped_heads(dtype, d, H, Hk, T):
    """Grouped q/k heads (num_qk_heads = Hk): dq and dk come back with Hk heads, each the sum over the
    value heads that read it (the oracle repeats q/k per value head and sums)."""
    w = synth.Workload("bwdg", "prefill", 2, T, H, d, d, dtype, 61, s0_std=0.5)
    inp = synth.prefill_inputs(w)
    inp["q"] = inp["q"][:, :, :Hk].contiguous()
    inp["k"] = inp["k"][:, :, :Hk].contiguous()
    run_and_compare(inp, dtype)


def test_backward_grouped_varlen():
    w = synth.Workload("bwdgv", "prefill", 1, 0, 6, 128, 128, "bf16", 62, s0_std=0.5)
    inp = synth.prefill_inputs(w, lengths=[70, 1, 130, 64])
    inp["q"] = inp["q"][:, :, :2].contiguous()
    inp["k"] = inp["k"][:, :, :2].contiguous()
    run_and_compare(inp, "bf16")


@pytest.mark.parametrize("dtype,d,flags,Hk", [("bf16", 128, 7, 4), ("f32", 64, 7, 4), ("bf16", 128, 1, 2),
                                               ("bf16", 128, 2, 4), ("f32", 128, 4, 4)])
def test_backward_through_prologue(dtype, d, flags, Hk):
    """The prologue bits of the forward (q/k L2 norm, gate logits, beta logits): gradients of the raw
    inputs.  Reference: oracle.prologue (the kernels' rounding of the normalised q/k to the input
    precision applied too), oracle.bwd on the transformed inputs, then oracle.prologue_bwd."""
    m = kda()
    g = torch.Generator().manual_seed(71)
    B, T, H = 2, 150, 4
    dt = torch.bfloat16 if dtype == "bf16" else torch.float32
    q = (torch.randn(B, T, Hk, d, generator=g) * 3.0).to(dt)
    k = (torch.randn(B, T, Hk, d, generator=g) * 0.2).to(dt)
    v = torch.randn(B, T, H, d, generator=g).to(dt)
    a = torch.randn(B, T, H, d, generator=g) + 3.0
    b = torch.randn(B, T, H, generator=g)
    if not flags & 1:
        q = torch.nn.functional.normalize(q.float(), dim=-1).to(dt)
        k = torch.nn.functional.normalize(k.float(), dim=-1).to(dt)
    if not flags & 2:
        a = torch.nn.functional.logsigmoid(a)
    if not flags & 4:
        b = torch.sigmoid(b)
    S0 = torch.randn(B, H, d, d, generator=g) * 0.3
    do = torch.randn(B, T, H, d, generator=g).to(dt)
    dsf = torch.randn(B, H, d, d, generator=g) * 0.5
    gr = m.chunk_bwd(q.to(DEV), k.to(DEV), v.to(DEV), a.to(DEV), b.to(DEV), do.to(DEV), S0=S0.to(DEV),
                     dS_final=dsf.to(DEV), prologue=flags)
    m.check()
    raw = [synth.to_oracle(x) for x in (q, k, a, b)]
    fl = dict(l2norm_qk=bool(flags & 1), gate_logits=bool(flags & 2), beta_logits=bool(flags & 4))
    qh, kh, la, bb = oracle.prologue(*raw, **fl)
    if flags & 1:  # the kernels round the normalised q, k to the input precision
        qh = torch.from_numpy(qh).to(dt).double().numpy()
        kh = torch.from_numpy(kh).to(dt).double().numpy()
    ref = oracle.bwd(qh, kh, synth.to_oracle(v), la, bb, do.double().numpy(), S0=S0.double().numpy(),
                     dS_final=dsf.double().numpy())
    ref = oracle.prologue_bwd(*raw, ref, **fl)
    errs = {key: max_rel(np64(gr[key]), ref[key]) for key in KEYS}
    tol = {key: max(t, 2e-3) for key, t in BWD_TOL[dtype].items()}  # fp32 prologue arithmetic on both ends
    bad = {key: e for key, e in errs.items() if not e <= tol[key]}
    assert not bad, f"gradient errors above tolerance: {bad} (all: {errs})"


def test_backward_empty_and_zero_length_sequences():
    """Packed sequences of length 0 among others, and a call with no tokens at all: the empty
    sequences get dS0 = dS_final and the others match the oracle."""
    m = kda()
    w = synth.Workload("bwde", "prefill", 1, 0, 2, 64, 64, "f32", 81, s0_std=0.5)
    inp = synth.prefill_inputs(w, lengths=[0, 5, 0, 64, 3])
    run_and_compare(inp, "f32")
    # no tokens: every gradient is empty and dS0 equals dS_final
    z = lambda *s: torch.zeros(*s, device=DEV)  # noqa: E731
    cu = torch.tensor([0, 0, 0], dtype=torch.int32, device=DEV)
    dsf = torch.randn(2, 2, 64, 64, device=DEV)
    g = m.chunk_bwd(z(1, 0, 2, 64), z(1, 0, 2, 64), z(1, 0, 2, 64), z(1, 0, 2, 64), z(1, 0, 2), z(1, 0, 2, 64),
                    S0=z(2, 2, 64, 64), dS_final=dsf, cu_seqlens=cu)
    m.check()
    assert torch.equal(g["dS0"], dsf)
