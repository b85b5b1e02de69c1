"""Pins for the oracle's backward pass (``oracle.bwd``), against facts that do not come from its code.

The loss is f = sum(dout * out) + sum(dS_final * S_final) over the recurrence
S_t = (I - b_t k_t k_t^T) Diag(a_t) S_{t-1} + b_t k_t v_t^T, o_t = S_t^T q_t ('Kimi Linear'
explainer, section 'Kimi Delta Attention的技术内核').  Its derivative is pinned by:

* central finite differences of the (separately pinned) forward oracle, with perturbations that are
  exact in float32 so the difference quotient carries only its O(eps^2) truncation error;
* the closed form of a single step from a zero state;
* structure: packed variable-length sequences give the gradients of separate runs; grouped q/k
  heads sum the per-value-head gradients.
"""
import numpy as np
import pytest

import oracle

EPS = 2.0 ** -12  # perturbation step; inputs and directions sit on a 2^-8 grid -> x +- EPS d exact


def grid(rng, shape, scale=1.0, lo=None, hi=None):
    x = rng.standard_normal(shape) * scale
    if lo is not None:
        x = rng.uniform(lo, hi, shape)
    return (np.round(x * 256) / 256).astype(np.float32)


def case(seed, lengths, H=2, dk=4, dv=3, Hk=None):
    rng = np.random.default_rng(seed)
    Ttot = int(sum(lengths))
    Hk = H if Hk is None else Hk
    q = grid(rng, (Ttot, Hk, dk))
    k = grid(rng, (Ttot, Hk, dk), 0.5)
    v = grid(rng, (Ttot, H, dv))
    la = grid(rng, (Ttot, H, dk), lo=-0.6, hi=-0.01)
    b = grid(rng, (Ttot, H), lo=0.05, hi=1.0)
    N = len(lengths)
    S0 = rng.standard_normal((N, H, dk, dv)) * 0.5
    do = rng.standard_normal((Ttot, H, dv))
    dsf = rng.standard_normal((N, H, dk, dv))
    cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int64)
    return dict(q=q, k=k, v=v, log_alpha=la, beta=b, S0=S0, cu_seqlens=cu), do, dsf


def loss(inp, do, dsf, o=oracle):
    out, sf = o.seq(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"], S0=inp["S0"],
                    cu_seqlens=inp["cu_seqlens"])
    return float(np.sum(out * do) + np.sum(sf * dsf))


GRAD = {"q": "dq", "k": "dk", "v": "dv", "log_alpha": "dlog_alpha", "beta": "dbeta"}


def test_bwd_matches_finite_differences(o=oracle):
    """Every derivative at once, on sequences that cross the backward's 64-step checkpoints (1, 70
    and 130 tokens).  Catches: a dropped term, a wrong sign, a missing beta or alpha factor, the
    readout taken from the wrong state, a cotangent not carried (or not decayed) across steps."""
    inp, do, dsf = case(3, [1, 70, 130])
    g = o.bwd(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"], do, S0=inp["S0"], dS_final=dsf,
              cu_seqlens=inp["cu_seqlens"])
    rng = np.random.default_rng(4)
    for name, key in GRAD.items():
        d = (rng.integers(-8, 9, inp[name].shape) / 8.0).astype(np.float32)
        plus, minus = dict(inp), dict(inp)
        plus[name] = (inp[name] + EPS * d).astype(np.float32)
        minus[name] = (inp[name] - EPS * d).astype(np.float32)
        assert np.array_equal(plus[name].astype(np.float64) - minus[name], 2 * EPS * d.astype(np.float64))
        fd = loss(plus, do, dsf, o) - loss(minus, do, dsf, o)
        an = float(np.sum(g[key] * (2 * EPS * d)))
        assert abs(fd - an) <= 1e-5 * abs(an) + 1e-12, f"{name}: fd {fd!r} vs analytic {an!r}"
    dS = np.random.default_rng(5).standard_normal(inp["S0"].shape) * EPS
    plus, minus = dict(inp), dict(inp)
    plus["S0"], minus["S0"] = inp["S0"] + dS, inp["S0"] - dS
    fd = loss(plus, do, dsf, o) - loss(minus, do, dsf, o)
    an = float(np.sum(g["dS0"] * 2 * dS))
    assert abs(fd - an) <= 1e-5 * abs(an), f"S0: fd {fd!r} vs analytic {an!r}"


def test_bwd_single_step_closed_form(o=oracle):
    """One token from S0 = 0: o = b (q.k) v, so df/dq = b (v.do) k, df/dk = b (v.do) q,
    df/dv = b (q.k) do, df/db = (q.k)(v.do), df/dlog_alpha = 0 and
    df/dS0 = Diag(a) (I - b k k^T) q do^T."""
    rng = np.random.default_rng(11)
    dk, dv = 5, 3
    q = rng.standard_normal((1, 1, dk)).astype(np.float32)
    k = rng.standard_normal((1, 1, dk)).astype(np.float32)
    v = rng.standard_normal((1, 1, dv)).astype(np.float32)
    la = -rng.uniform(0.1, 1.0, (1, 1, dk)).astype(np.float32)
    b = np.array([[0.625]], np.float32)
    do = rng.standard_normal((1, 1, dv))
    g = o.bwd(q, k, v, la, b, do)
    q64, k64, v64, do64 = (x.astype(np.float64).ravel() for x in (q, k, v, do))
    bb, qk, vd = 0.625, q64 @ k64, v64 @ do64
    np.testing.assert_allclose(g["dq"].ravel(), bb * vd * k64, rtol=1e-13, atol=1e-15)
    np.testing.assert_allclose(g["dk"].ravel(), bb * vd * q64, rtol=1e-13, atol=1e-15)
    np.testing.assert_allclose(g["dv"].ravel(), bb * qk * do64, rtol=1e-13, atol=1e-15)
    np.testing.assert_allclose(g["dbeta"].ravel(), [qk * vd], rtol=1e-13)
    np.testing.assert_array_equal(g["dlog_alpha"], 0.0)
    a = np.exp(la.astype(np.float64).ravel())
    ds0 = a[:, None] * np.outer((np.eye(dk) - bb * np.outer(k64, k64)) @ q64, do64)
    np.testing.assert_allclose(g["dS0"][0, 0], ds0, rtol=1e-13, atol=1e-15)


def test_bwd_varlen_equals_separate_runs(o=oracle):
    """Packed sequences are independent: their gradients are those of separate calls (catches a
    cotangent leaking across a sequence boundary)."""
    lengths = [5, 67, 2]
    inp, do, dsf = case(7, lengths, H=2, dk=3, dv=4)
    g = o.bwd(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"], do, S0=inp["S0"], dS_final=dsf,
              cu_seqlens=inp["cu_seqlens"])
    cu = inp["cu_seqlens"]
    for n in range(len(lengths)):
        s = slice(cu[n], cu[n + 1])
        gn = o.bwd(inp["q"][s], inp["k"][s], inp["v"][s], inp["log_alpha"][s], inp["beta"][s], do[s],
                   S0=inp["S0"][n:n + 1], dS_final=dsf[n:n + 1])
        for key in GRAD.values():
            np.testing.assert_array_equal(g[key][s], gn[key])
        np.testing.assert_array_equal(g["dS0"][n], gn["dS0"][0])


def test_bwd_zero_cotangent_gives_zero(o=oracle):
    inp, do, dsf = case(8, [9], H=1)
    g = o.bwd(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"], 0 * do, S0=inp["S0"],
              cu_seqlens=inp["cu_seqlens"])
    for key in list(GRAD.values()) + ["dS0"]:
        assert not np.any(g[key])


def test_bwd_grouped_heads(o=oracle):
    """Grouped q/k heads: df/dq of a shared head is the sum over the value heads that read it,
    checked by finite differences on the shared q."""
    inp, do, dsf = case(9, [6, 3], H=4, dk=3, dv=2, Hk=2)
    g = o.bwd(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"], do, S0=inp["S0"], dS_final=dsf,
              cu_seqlens=inp["cu_seqlens"])
    assert g["dq"].shape == inp["q"].shape and g["dk"].shape == inp["k"].shape
    rng = np.random.default_rng(10)
    for name in ("q", "k"):
        d = (rng.integers(-8, 9, inp[name].shape) / 8.0).astype(np.float32)
        plus, minus = dict(inp), dict(inp)
        plus[name] = (inp[name] + EPS * d).astype(np.float32)
        minus[name] = (inp[name] - EPS * d).astype(np.float32)
        fd = loss(plus, do, dsf, o) - loss(minus, do, dsf, o)
        an = float(np.sum(g[GRAD[name]] * (2 * EPS * d)))
        assert abs(fd - an) <= 1e-5 * abs(an)


@pytest.mark.parametrize("T", [64, 65, 128])
def test_bwd_checkpoint_boundaries(T, o=oracle):
    """Sequence lengths at and next to the checkpoint spacing: the gradients of the first tokens
    must not depend on how the sequence is cut (catches an off-by-one in the recomputed states)."""
    inp, do, dsf = case(12, [T], H=1, dk=3, dv=2)
    g = o.bwd(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"], do, S0=inp["S0"], dS_final=dsf,
              cu_seqlens=inp["cu_seqlens"])
    rng = np.random.default_rng(13)
    d = (rng.integers(-8, 9, inp["log_alpha"].shape) / 8.0).astype(np.float32)
    plus, minus = dict(inp), dict(inp)
    plus["log_alpha"] = (inp["log_alpha"] + EPS * d).astype(np.float32)
    minus["log_alpha"] = (inp["log_alpha"] - EPS * d).astype(np.float32)
    fd = loss(plus, do, dsf, o) - loss(minus, do, dsf, o)
    an = float(np.sum(g["dlog_alpha"] * (2 * EPS * d)))
    assert abs(fd - an) <= 1e-5 * abs(an)


def test_prologue_bwd_matches_finite_differences(o=oracle):
    """The chain rule through the input prologue (L2-normalised q/k, log-sigmoid gate logits, sigmoid
    beta logits), pinned by finite differences of the composition prologue -> recurrence.  The
    transformed inputs are kept in fp64 on both sides of the difference (the oracle recurrence takes
    float32, so the perturbation goes through the exact fp64 prologue and a float32 rounding that is
    the same for the base point and the analytic side).  Catches: a missing 1/n or projection term in
    the norm, sigma(a) in place of sigma(-a), a missing (1 - sigma) factor."""
    rng = np.random.default_rng(21)
    T, H, dk, dv = 9, 2, 4, 3
    q = rng.standard_normal((T, H, dk)) * 2.0
    k = rng.standard_normal((T, H, dk)) * 0.7
    v = rng.standard_normal((T, H, dv))
    a = rng.normal(2.0, 1.0, (T, H, dk))
    b = rng.standard_normal((T, H))
    do = rng.standard_normal((T, H, dv))
    flags = dict(l2norm_qk=True, gate_logits=True, beta_logits=True)

    def f(q_, k_, a_, b_):
        qq, kk, la, bb = o.prologue(q_, k_, a_, b_, **flags)
        out, _ = o.seq(qq, kk, v, la, bb)
        return float(np.sum(out * do))

    qq, kk, la, bb = o.prologue(q, k, a, b, **flags)
    g = o.bwd(qq, kk, v, la, bb, do)
    g = o.prologue_bwd(q, k, a, b, g, **flags)
    eps = 1e-4
    for name, key, x in (("q", "dq", q), ("k", "dk", k), ("a", "dlog_alpha", a), ("b", "dbeta", b)):
        d = rng.standard_normal(x.shape)
        args = dict(q_=q, k_=k, a_=a, b_=b)
        plus, minus = dict(args), dict(args)
        plus[name + "_"] = x + eps * d
        minus[name + "_"] = x - eps * d
        fd = (f(**plus) - f(**minus)) / (2 * eps)
        an = float(np.sum(g[key] * d))
        # float32 rounding of the transformed inputs inside the oracle recurrence bounds the agreement
        assert abs(fd - an) <= 2e-3 * abs(an) + 1e-6, f"{name}: fd {fd!r} vs analytic {an!r}"
