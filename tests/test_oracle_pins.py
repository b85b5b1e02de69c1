"""Pins for the fp64 oracle: facts the pages and the mathematics fix, independent of the oracle's code.

Each test states which mistake it is there to catch.  The recurrence being pinned is
S_t = (I - b_t k_t k_t^T) Diag(a_t) S_{t-1} + b_t k_t v_t^T, o_t = S_t^T q_t ('Kimi Linear'
explainer, section 'Kimi Delta Attention的技术内核'; attention review, entry 'KLA 25.10 kimi').
"""
import json
import os

import numpy as np
import pytest

HERE = os.path.dirname(os.path.abspath(__file__))


def rel(a, b):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


def rand_case(seed, Ttot, H, dk, dv, unit_k=True, s0=True, beta_lo=0.0):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((Ttot, H, dk)).astype(np.float32)
    k = rng.standard_normal((Ttot, H, dk))
    if unit_k:
        k /= np.linalg.norm(k, axis=-1, keepdims=True)
    k = k.astype(np.float32)
    v = rng.standard_normal((Ttot, H, dv)).astype(np.float32)
    la = np.log(1.0 / (1.0 + np.exp(-rng.normal(3.0, 1.0, (Ttot, H, dk))))).astype(np.float32)
    beta = rng.uniform(beta_lo, 1.0, (Ttot, H)).astype(np.float32)
    S0 = rng.standard_normal((1, H, dk, dv)) * 0.5 if s0 else None
    return q, k, v, la, beta, S0


# ---------------------------------------------------------------------------------------------
# 1. hand-worked example (orientation, order of decay/delta/update/readout, beta placement)
# ---------------------------------------------------------------------------------------------
def test_hand_worked_example(oracle):
    """Catches: S q instead of S^T q, correction on the undecayed state, readout from S_{t-1},
    beta on the wrong term.  Values worked by hand in tests/golden/kda_hand_example.json."""
    g = json.load(open(os.path.join(HERE, "golden", "kda_hand_example.json")))
    T = len(g["beta"])
    q = np.array(g["q"], np.float32).reshape(T, 1, 2)
    k = np.array(g["k"], np.float32).reshape(T, 1, 2)
    v = np.array(g["v"], np.float32).reshape(T, 1, 2)
    la = np.log(np.array(g["alpha"], np.float64)).astype(np.float32).reshape(T, 1, 2)
    b = np.array(g["beta"], np.float32).reshape(T, 1)
    S0 = np.array(g["S0"], np.float64).reshape(1, 1, 2, 2)
    tol = g["tolerance"]
    for fn in (oracle.seq, oracle.bruteforce):
        out, sf = fn(q, k, v, la, b, S0=S0)
        np.testing.assert_allclose(out[:, 0], np.array(g["out"]), atol=tol, rtol=0)
        np.testing.assert_allclose(sf[0, 0], np.array(g["S_final"]), atol=tol, rtol=0)
    for C in (1, 2, 64):
        out, sf = oracle.chunked(q, k, v, la, b, S0=S0, C=C)
        np.testing.assert_allclose(out[:, 0], np.array(g["out"]), atol=tol, rtol=0)
        np.testing.assert_allclose(sf[0, 0], np.array(g["S_final"]), atol=tol, rtol=0)
    # decode form, one token at a time
    S = S0.copy()
    for t in range(T):
        o, S = oracle.decode_step(q[t:t + 1], k[t:t + 1], v[t:t + 1], la[t:t + 1], b[t:t + 1], S)
        np.testing.assert_allclose(o[0, 0], np.array(g["out"][t]), atol=tol, rtol=0)
    np.testing.assert_allclose(S[0, 0], np.array(g["S_final"]), atol=tol, rtol=0)


# ---------------------------------------------------------------------------------------------
# 2. beta = 0: the delta term vanishes and the state is the closed-form decayed S0
# ---------------------------------------------------------------------------------------------
@pytest.mark.parametrize("form", ["seq", "chunked16", "chunked64", "bruteforce"])
def test_beta_zero_closed_form(oracle, form):
    """Catches: a wrong decay (missing exp, gate on the value axis, cumulative gate off by one,
    gate not restarted correctly across chunks).  S_t = Diag(exp(sum_{i<=t} log a_i)) S0."""
    Ttot, H, dk, dv = 70 if form != "bruteforce" else 12, 2, 8, 6
    q, k, v, la, beta, S0 = rand_case(1, Ttot, H, dk, dv)
    beta[:] = 0.0
    G = np.cumsum(la.astype(np.float64), axis=0)                      # [T,H,dk]
    S_t = np.exp(G)[:, :, :, None] * S0[0][None]                      # [T,H,dk,dv]
    o_ref = np.einsum("thc,thcj->thj", q.astype(np.float64), S_t)
    fn = {"seq": oracle.seq, "bruteforce": oracle.bruteforce,
          "chunked16": lambda *a, **kw: oracle.chunked(*a, C=16, **kw),
          "chunked64": lambda *a, **kw: oracle.chunked(*a, C=64, **kw)}[form]
    out, sf = fn(q, k, v, la, beta, S0=S0)
    assert rel(out, o_ref) < 1e-12
    assert rel(sf[0], S_t[-1]) < 1e-12


# ---------------------------------------------------------------------------------------------
# 3. alpha = 1, beta = 1, orthonormal keys: the delta rule writes, q = k_i retrieves v_i exactly
# ---------------------------------------------------------------------------------------------
@pytest.mark.parametrize("form", ["seq", "chunked", "bruteforce"])
def test_orthonormal_write_retrieve(oracle, form):
    """Catches: a missing/mis-signed rank-1 correction, beta applied to the wrong term, a
    transposed update k v^T vs v k^T.  With (I - k k^T) a projector the write is exact
    (the 'precise memory update' of the delta rule), whatever S0 is."""
    dk = dv = 8
    Tw = 6
    rng = np.random.default_rng(7)
    Qm, _ = np.linalg.qr(rng.standard_normal((dk, dk)))
    keys = Qm[:, :Tw].T.astype(np.float32)                 # Tw orthonormal keys (float32-rounded)
    vals = rng.standard_normal((Tw, dv)).astype(np.float32)
    T = 2 * Tw
    q = np.zeros((T, 1, dk), np.float32)
    k = np.zeros((T, 1, dk), np.float32)
    v = np.zeros((T, 1, dv), np.float32)
    la = np.zeros((T, 1, dk), np.float32)
    b = np.zeros((T, 1), np.float32)
    k[:Tw, 0] = keys
    v[:Tw, 0] = vals
    b[:Tw] = 1.0
    q[Tw:, 0] = keys                                      # query phase: beta=0, k=0 -> state frozen
    S0 = rng.standard_normal((1, 1, dk, dv))
    fn = {"seq": oracle.seq, "bruteforce": oracle.bruteforce,
          "chunked": lambda *a, **kw: oracle.chunked(*a, C=4, **kw)}[form]
    out, _ = fn(q, k, v, la, b, S0=S0)
    # float32 keys are orthonormal to ~1e-7; the retrieval error is of that order
    np.testing.assert_allclose(out[Tw:, 0], vals, atol=2e-6, rtol=0)
    # right after each write, o_t = S_t^T q_t with q_t = 0 is 0 (readout uses q, not k)
    np.testing.assert_allclose(out[:Tw, 0], 0.0, atol=0)


# ---------------------------------------------------------------------------------------------
# 4. per-step delta invariant, |k| = 1:  S_t^T k_t = (1 - b_t) S'_t^T k_t + b_t v_t
# ---------------------------------------------------------------------------------------------
def test_per_step_invariant(oracle):
    """Catches: decay applied after the correction, correction on the undecayed state."""
    N, H, dk, dv = 3, 2, 16, 8
    rng = np.random.default_rng(11)
    S = rng.standard_normal((N, H, dk, dv))
    for t in range(20):
        q = rng.standard_normal((N, H, dk)).astype(np.float32)
        k = rng.standard_normal((N, H, dk))
        k = (k / np.linalg.norm(k, axis=-1, keepdims=True)).astype(np.float32)
        kk = k.astype(np.float64)
        kk /= np.linalg.norm(kk, axis=-1, keepdims=True)      # the float32 key, renormalised in fp64
        k = kk.astype(np.float32)
        v = rng.standard_normal((N, H, dv)).astype(np.float32)
        la = (-rng.uniform(0, 0.5, (N, H, dk))).astype(np.float32)
        b = rng.uniform(0, 1, (N, H)).astype(np.float32)
        Sd = np.exp(la.astype(np.float64))[..., None] * S
        _, S = oracle.decode_step(q, k, v, la, b, S)
        k64 = k.astype(np.float64)
        lhs = np.einsum("nhcj,nhc->nhj", S, k64)
        rhs = (1 - b[..., None].astype(np.float64)) * np.einsum("nhcj,nhc->nhj", Sd, k64) + \
            b[..., None].astype(np.float64) * v.astype(np.float64)
        # |k|^2 = 1 only to float32 precision
        assert np.max(np.abs(lhs - rhs)) < 1e-6 * (1 + np.max(np.abs(rhs)))


# ---------------------------------------------------------------------------------------------
# 5. brute force (dense transition matrices) vs sequential
# ---------------------------------------------------------------------------------------------
@pytest.mark.parametrize("T", [1, 5, 16])
def test_bruteforce_vs_seq(oracle, T):
    q, k, v, la, b, S0 = rand_case(3, T, 3, 8, 5, unit_k=False)
    o1, s1 = oracle.seq(q, k, v, la, b, S0=S0)
    o2, s2 = oracle.bruteforce(q, k, v, la, b, S0=S0)
    assert rel(o1, o2) < 1e-12 and rel(s1, s2) < 1e-12


# ---------------------------------------------------------------------------------------------
# 6. chunked WY/UT form vs sequential, several C, T not a multiple of C
# ---------------------------------------------------------------------------------------------
@pytest.mark.parametrize("C", [1, 4, 16, 64])
def test_chunked_vs_seq(oracle, C):
    q, k, v, la, b, S0 = rand_case(5, 150, 2, 16, 12)
    o1, s1 = oracle.seq(q, k, v, la, b, S0=S0)
    o2, s2 = oracle.chunked(q, k, v, la, b, S0=S0, C=C)
    assert rel(o1, o2) < 1e-10 and rel(s1, s2) < 1e-10


def test_chunked_strong_decay(oracle):
    """log alpha = -30 per step: products of gates underflow; the chunked form must not overflow."""
    q, k, v, la, b, S0 = rand_case(6, 100, 1, 8, 8)
    la[:] = -30.0
    o1, s1 = oracle.seq(q, k, v, la, b, S0=S0)
    o2, s2 = oracle.chunked(q, k, v, la, b, S0=S0, C=64)
    assert np.all(np.isfinite(o2)) and np.all(np.isfinite(s2))
    assert rel(o1, o2) < 1e-10 and rel(s1, s2) < 1e-10


# ---------------------------------------------------------------------------------------------
# 7. linearity in (V, S0) for fixed (q, k, alpha, beta)
# ---------------------------------------------------------------------------------------------
def test_linearity(oracle):
    """Catches: any term that is not linear in (v, S) -- e.g. a stray constant or a squared v."""
    q, k, v1, la, b, S01 = rand_case(8, 40, 2, 8, 8)
    rng = np.random.default_rng(9)
    v2 = rng.standard_normal(v1.shape).astype(np.float32)
    S02 = rng.standard_normal(S01.shape)
    c = np.float32(2.0)
    o1, s1 = oracle.seq(q, k, v1, la, b, S0=S01)
    o2, s2 = oracle.seq(q, k, v2, la, b, S0=S02)
    o3, s3 = oracle.seq(q, k, (v1 + c * v2).astype(np.float32), la, b, S0=S01 + 2.0 * S02)
    assert rel(o3, o1 + 2 * o2) < 1e-6 and rel(s3, s1 + 2 * s2) < 1e-6   # v1 + 2 v2 rounded to f32


# ---------------------------------------------------------------------------------------------
# 8. state passing: run(T) = run(T2; S0 = S_final(run(T1)))
# ---------------------------------------------------------------------------------------------
@pytest.mark.parametrize("split", [1, 37, 64, 100])
def test_state_passing(oracle, split):
    q, k, v, la, b, S0 = rand_case(10, 130, 2, 8, 8)
    o, s = oracle.chunked(q, k, v, la, b, S0=S0, C=16)
    oa, sa = oracle.chunked(q[:split], k[:split], v[:split], la[:split], b[:split], S0=S0, C=16)
    ob, sb = oracle.chunked(q[split:], k[split:], v[split:], la[split:], b[split:], S0=sa, C=16)
    assert rel(np.concatenate([oa, ob]), o) < 1e-10 and rel(sb, s) < 1e-10


# ---------------------------------------------------------------------------------------------
# 9. varlen (packed with cu_seqlens) = separate runs
# ---------------------------------------------------------------------------------------------
@pytest.mark.parametrize("form", ["seq", "chunked"])
def test_varlen_equals_separate(oracle, form):
    lens = [1, 63, 64, 65, 130]
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    q, k, v, la, b, _ = rand_case(12, int(cu[-1]), 2, 8, 8)
    rng = np.random.default_rng(13)
    S0 = rng.standard_normal((len(lens), 2, 8, 8))
    fn = oracle.seq if form == "seq" else (lambda *a, **kw: oracle.chunked(*a, C=64, **kw))
    o, s = fn(q, k, v, la, b, S0=S0, cu_seqlens=cu)
    for n in range(len(lens)):
        a, e = cu[n], cu[n + 1]
        on, sn = oracle.seq(q[a:e], k[a:e], v[a:e], la[a:e], b[a:e], S0=S0[n:n + 1])
        assert rel(o[a:e], on) < 1e-10 and rel(s[n], sn[0]) < 1e-10


# ---------------------------------------------------------------------------------------------
# 10. decode (per-token loop order) = prefill (recurrence) on the same tokens
# ---------------------------------------------------------------------------------------------
def test_decode_equals_prefill(oracle):
    N, H, dk, dv, T = 3, 2, 8, 8, 32
    rng = np.random.default_rng(14)
    q, k, v, la, b, _ = rand_case(15, N * T, H, dk, dv)
    S0 = rng.standard_normal((N, H, dk, dv))
    cu = np.arange(N + 1, dtype=np.int64) * T
    o_ref, s_ref = oracle.seq(q, k, v, la, b, S0=S0, cu_seqlens=cu)
    S = S0.copy()
    for t in range(T):
        idx = cu[:-1] + t
        o, S = oracle.decode_step(q[idx], k[idx], v[idx], la[idx], b[idx], S)
        assert rel(o, o_ref[idx]) < 1e-12
    assert rel(S, s_ref) < 1e-12


# ---------------------------------------------------------------------------------------------
# 11. norm bound: |k| = 1, beta in [0,1], alpha <= 1  =>  |S_t|_F <= |S_{t-1}|_F + beta |v|
# ---------------------------------------------------------------------------------------------
def test_norm_bound(oracle):
    rng = np.random.default_rng(16)
    N, H, dk, dv = 2, 2, 16, 16
    S = rng.standard_normal((N, H, dk, dv))
    for t in range(30):
        q = rng.standard_normal((N, H, dk)).astype(np.float32)
        k = rng.standard_normal((N, H, dk))
        k = (k / np.linalg.norm(k, axis=-1, keepdims=True)).astype(np.float32)
        v = rng.standard_normal((N, H, dv)).astype(np.float32)
        la = (-rng.uniform(0, 0.3, (N, H, dk))).astype(np.float32)
        b = rng.uniform(0, 1, (N, H)).astype(np.float32)
        n0 = np.linalg.norm(S, axis=(-2, -1))
        _, S = oracle.decode_step(q, k, v, la, b, S)
        n1 = np.linalg.norm(S, axis=(-2, -1))
        bound = n0 + b.astype(np.float64) * np.linalg.norm(v.astype(np.float64), axis=-1)
        assert np.all(n1 <= bound * (1 + 1e-6))


# ---------------------------------------------------------------------------------------------
# 12. special cases: zero-length sequences, beta=0 & alpha=1 (identity step), S0 = None
# ---------------------------------------------------------------------------------------------
def test_identity_and_empty(oracle):
    q, k, v, la, b, S0 = rand_case(17, 10, 1, 4, 4)
    la[:] = 0.0
    b[:] = 0.0
    out, sf = oracle.seq(q, k, v, la, b, S0=S0)
    np.testing.assert_allclose(sf[0], S0[0], rtol=0, atol=0)
    np.testing.assert_allclose(out, np.einsum("thc,hcj->thj", q.astype(np.float64), S0[0]), rtol=1e-13)
    # empty sequences in a varlen pack keep their S0 and produce no rows
    cu = np.array([0, 0, 10, 10], np.int64)
    S0s = np.random.default_rng(1).standard_normal((3, 1, 4, 4))
    out, sf = oracle.chunked(q, k, v, la, b, S0=S0s, cu_seqlens=cu, C=4)
    np.testing.assert_allclose(sf[0], S0s[0], atol=0)
    np.testing.assert_allclose(sf[2], S0s[2], atol=0)
    # S0 = None means zero state
    q, k, v, la, b, _ = rand_case(18, 9, 1, 4, 4)
    o1, s1 = oracle.seq(q, k, v, la, b, S0=None)
    o2, s2 = oracle.seq(q, k, v, la, b, S0=np.zeros((1, 1, 4, 4)))
    np.testing.assert_array_equal(o1, o2)
    np.testing.assert_array_equal(s1, s2)


# ---------------------------------------------------------------------------------------------
# 13. grouped q/k heads (the head-count comments of the review's GDN pseudo-code: fewer q/k heads
#     than value heads, each q/k head shared by a group of value heads)
# ---------------------------------------------------------------------------------------------
@pytest.mark.parametrize("form", ["seq", "chunked", "decode"])
def test_grouped_heads_equal_repeated_qk(oracle, form):
    """A grouped call must equal the one-head-per-value-head call on q and k repeated by numpy
    (np.repeat along the head axis).  Catches: value head h reading q/k head h % Hk instead of
    h // (H // Hk), or reading the value-head index into the smaller q/k array."""
    H, Hk, dk, dv = 6, 2, 8, 8
    G = H // Hk
    if form == "decode":
        rng = np.random.default_rng(21)
        N = 3
        q = rng.standard_normal((N, Hk, dk)).astype(np.float32)
        k = rng.standard_normal((N, Hk, dk)).astype(np.float32)
        v = rng.standard_normal((N, H, dv)).astype(np.float32)
        la = np.log(1.0 / (1.0 + np.exp(-rng.normal(3.0, 1.0, (N, H, dk))))).astype(np.float32)
        b = rng.uniform(0.0, 1.0, (N, H)).astype(np.float32)
        S = rng.standard_normal((N, H, dk, dv))
        o_g, s_g = oracle.decode_step(q, k, v, la, b, S)
        o_r, s_r = oracle.decode_step(np.repeat(q, G, axis=1), np.repeat(k, G, axis=1), v, la, b, S)
    else:
        Ttot = 150
        q, k, v, la, b, S0 = rand_case(22, Ttot, H, dk, dv)
        q, k = q[:, :Hk], k[:, :Hk]
        cu = np.array([0, 70, 150], dtype=np.int64)
        S0 = np.random.default_rng(23).standard_normal((2, H, dk, dv))
        fn = oracle.seq if form == "seq" else (lambda *a, **kw: oracle.chunked(*a, C=16, **kw))
        o_g, s_g = fn(q, k, v, la, b, S0=S0, cu_seqlens=cu)
        o_r, s_r = fn(np.repeat(q, G, axis=1), np.repeat(k, G, axis=1), v, la, b, S0=S0, cu_seqlens=cu)
    assert np.array_equal(o_g, o_r) and np.array_equal(s_g, s_r)
    # and the groups really share: value heads of one group differ only through v, gates and state
    assert rel(o_g[..., 0, :], o_g[..., 1, :]) > 1e-3


# ---------------------------------------------------------------------------------------------
# 14. input prologue: q/k L2 normalisation, log-sigmoid gate logits, sigmoid beta logits
# ---------------------------------------------------------------------------------------------
def test_prologue_transforms(oracle):
    """Pinned by facts of the functions themselves, not by their code.  Catches: a normalisation over
    the wrong axis or without the square root, log sigmoid with a wrong sign or branch, sigmoid of
    -b, and transforms applied when their flag is off."""
    rng = np.random.default_rng(31)
    q = rng.standard_normal((5, 3, 16)) * 3.0
    k = rng.standard_normal((5, 3, 16)) * 0.1
    a = np.array([-60.0, -5.0, -1.0, 0.0, 1.0, 3.0, 40.0])
    b = np.array([-3.0, 0.0, 2.0])
    qn, kn, la, bb = oracle.prologue(q, k, a, b, l2norm_qk=True, gate_logits=True, beta_logits=True)
    # unit rows (up to the 1e-6 epsilon under the square root), same directions
    nq, nk = np.linalg.norm(qn, axis=-1), np.linalg.norm(kn, axis=-1)
    assert np.allclose(nq, np.sqrt(np.sum(q * q, -1) / (np.sum(q * q, -1) + 1e-6)), rtol=1e-14)
    assert np.all(np.abs(nq - 1) < 1e-6) and np.all(np.abs(nk - 1) < 1e-3)
    assert np.allclose(qn * np.linalg.norm(q, axis=-1, keepdims=True), q * nq[..., None], rtol=1e-12)
    z, _, _, _ = oracle.prologue(np.zeros((1, 4)), np.zeros((1, 4)), 0.0, 0.0, l2norm_qk=True)
    assert np.all(z == 0)                                        # a zero row stays zero
    # log sigmoid: log(1/2) at 0; ~x for x << 0; ~-e^{-x} for x >> 0; log of sigma(x) elsewhere
    assert la[3] == np.log(0.5)
    assert abs(la[0] - (-60.0)) < 1e-20 and abs(la[6] + np.exp(-40.0)) < 1e-30
    mid = a[1:6]
    assert np.allclose(la[1:6], np.log(1.0 / (1.0 + np.exp(-mid))), rtol=1e-13)
    assert np.all(la <= 0)
    # sigmoid: 1/2 at 0, symmetric s(-x) = 1 - s(x)
    assert bb[1] == 0.5 and abs(bb[0] - (1 - oracle.prologue(q, k, a, -b, beta_logits=True)[3][0])) < 1e-15
    # flags off: inputs returned unchanged
    q2, k2, la2, b2 = oracle.prologue(q, k, a, b)
    assert np.array_equal(q2, q) and np.array_equal(k2, k) and np.array_equal(la2, a) and np.array_equal(b2, b)


# ---------------------------------------------------------------------------------------------
# 15. output gate: grouped RMS norm times the gate z
# ---------------------------------------------------------------------------------------------
def test_gated_rmsnorm(oracle):
    """Pinned by torch's own rms_norm (float64, a library routine) and by facts of the norm.  Catches:
    the norm over the wrong axis or group, a missing square root or mean, the gate not applied or
    applied before the norm, the weight dropped."""
    import torch
    rng = np.random.default_rng(41)
    o = rng.standard_normal((3, 5, 64)) * 4.0
    z = rng.standard_normal((3, 5, 64))
    w = rng.uniform(0.5, 1.5, 64)
    y = oracle.gated_rmsnorm(o, z, weight=w, eps=1e-6)
    ref = torch.nn.functional.rms_norm(torch.from_numpy(o), (64,), torch.from_numpy(w), eps=1e-6).numpy() * z
    assert np.allclose(y, ref, rtol=1e-12, atol=1e-14)
    # grouped: each group of 16 normalised on its own = rms_norm over a reshaped last axis
    yg = oracle.gated_rmsnorm(o, np.ones_like(o), group=16, eps=1e-6)
    refg = torch.nn.functional.rms_norm(torch.from_numpy(o.reshape(3, 5, 4, 16)), (16,), eps=1e-6).numpy()
    assert np.allclose(yg, refg.reshape(o.shape), rtol=1e-12)
    # unit RMS per group (up to eps), invariant to a positive scale of o
    ms = np.mean(yg.reshape(3, 5, 4, 16) ** 2, axis=-1)
    assert np.all(np.abs(ms - 1) < 1e-6)
    assert np.allclose(oracle.gated_rmsnorm(7.5 * o, z), oracle.gated_rmsnorm(o, z), rtol=1e-6)
    # sigmoid gate: z = 0 halves the normalised output
    y0 = oracle.gated_rmsnorm(o, np.zeros_like(o), gate="sigmoid")
    assert np.allclose(y0, 0.5 * oracle.gated_rmsnorm(o, np.ones_like(o)), rtol=1e-14)
