"""Pins of the CPU oracle to things other than itself.

Each test checks an oracle function against a closed form, a hand-computed
golden case (tests/golden/), a library routine that computes the same
quantity by another route, a brute-force enumeration on tiny inputs, or an
invariant of the mathematics -- chosen so that a dropped term, a wrong sign or
index, or a transposed operand fails at least one of them.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest
import torch

from oracle import ssa_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def small_problem(**kw):
    base = dict(batch=1, n_q=32, n_kv=32, h_q=1, h_kv=1, d=4, block=4, topk=2, window=4,
                dtype=O.F32, sigma=O.FULL, beta=2.0)
    base.update(kw)
    return O.Problem(**base)


# ------------------------------------------------------------------ rounding

def test_round_bf16_matches_torch_and_ties_to_even():
    rng = np.random.default_rng(1)
    x = np.concatenate([rng.standard_normal(20000).astype(np.float32) * 10.0 ** rng.integers(-6, 6, 20000),
                        np.float32([1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -1.0 - 2 ** -8, 0.0, -0.0, 3.0e38])])
    ours = O.round_bf16(x)
    ref = torch.from_numpy(x.astype(np.float32)).to(torch.bfloat16).to(torch.float64).numpy()
    assert np.array_equal(ours, ref)
    # exact halfway cases round to the even neighbour
    assert O.round_bf16(np.float32(1.0 + 2 ** -8)) == 1.0
    assert O.round_bf16(np.float32(1.0 + 3 * 2 ** -8)) == 1.0 + 2 ** -6


def test_round_f32_matches_numpy_cast():
    x = np.random.default_rng(2).standard_normal(1000) * 1e3
    assert np.array_equal(O.round_f32(x), x.astype(np.float32).astype(np.float64))


# ------------------------------------------------------------------ summaries

def test_summaries_golden_two_blocks():
    g = golden("cumulant_routing_outlier.json")
    K = np.array(g["keys"], dtype=np.float64).reshape(1, 4, 1, 2)
    pd = small_problem(n_q=4, n_kv=4, d=2, block=2, sigma=O.DIAG)
    mu, var = O.block_summaries(K, pd)
    assert np.array_equal(mu[0, 0], np.array(g["mu"], dtype=float))
    assert np.array_equal(var[0, 0], np.array(g["var"], dtype=float))
    pf = small_problem(n_q=4, n_kv=4, d=2, block=2, sigma=O.FULL)
    _, cov = O.block_summaries(K, pf)
    assert np.array_equal(cov[0, 0], np.array(g["cov"], dtype=float))


def test_summaries_match_numpy_mean_and_population_cov():
    rng = np.random.default_rng(3)
    K = rng.standard_normal((2, 24, 3, 5))
    p = small_problem(batch=2, n_q=24, n_kv=24, h_q=3, h_kv=3, d=5, block=8, sigma=O.FULL)
    mu, cov = O.block_summaries(K, p)
    _, var = O.block_summaries(K, O.Problem(**{**p.__dict__, "sigma": O.DIAG}))
    for bi in range(2):
        for h in range(3):
            for c in range(3):
                keys = K[bi, c * 8:(c + 1) * 8, h]
                np.testing.assert_allclose(mu[bi, h, c], keys.mean(axis=0), rtol=0, atol=1e-14)
                np.testing.assert_allclose(cov[bi, h, c], np.cov(keys.T, bias=True), rtol=0, atol=1e-13)
                np.testing.assert_allclose(var[bi, h, c], keys.var(axis=0), rtol=0, atol=1e-14)


def test_summary_invariants_shift_scale_psd():
    rng = np.random.default_rng(4)
    K = rng.standard_normal((1, 16, 1, 6))
    p = small_problem(n_q=16, n_kv=16, d=6, block=8, sigma=O.FULL)
    mu, cov = O.block_summaries(K, p)
    shift = rng.standard_normal(6)
    K2 = K.copy()
    K2[0, :8, 0] += shift                      # shift block 0 only
    mu2, cov2 = O.block_summaries(K2, p)
    np.testing.assert_allclose(mu2[0, 0, 0], mu[0, 0, 0] + shift, atol=1e-13)
    np.testing.assert_allclose(mu2[0, 0, 1], mu[0, 0, 1], atol=0)
    np.testing.assert_allclose(cov2, cov, atol=1e-13)
    mu3, cov3 = O.block_summaries(3.0 * K, p)
    np.testing.assert_allclose(cov3, 9.0 * cov, rtol=1e-13)
    for c in range(2):
        S = cov[0, 0, c]
        assert np.allclose(S, S.T)
        assert np.linalg.eigvalsh(S).min() > -1e-12
    # a block of identical keys has zero spread
    K4 = np.repeat(O.round_bf16(rng.standard_normal((1, 1, 1, 6))), 16, axis=1)
    _, cov4 = O.block_summaries(K4, p)
    assert np.abs(cov4).max() == 0


def test_stored_table_is_bf16_of_f32():
    rng = np.random.default_rng(5)
    K = torch.randn(1, 64, 2, 8, generator=torch.Generator().manual_seed(5)).to(torch.bfloat16).float().numpy()
    p = small_problem(n_q=64, n_kv=64, h_q=2, h_kv=2, d=8, block=16, dtype=O.BF16, sigma=O.DIAG)
    mu, var = O.block_summaries(K, p)
    mu32, var32, tab = O.stored_summaries(mu, var, p)
    t = torch.from_numpy(np.concatenate([mu, var], axis=-1)).to(torch.float32).to(torch.bfloat16).double().numpy()
    assert np.array_equal(tab, t)
    assert tab.shape == (1, 2, 4, 16)
    del rng


# ------------------------------------------------------------------ routing score

def test_routing_golden_outlier_block():
    g = golden("cumulant_routing_outlier.json")
    K = np.array(g["keys"], dtype=np.float64).reshape(1, 4, 1, 2)
    Q = np.array(g["q"], dtype=np.float64).reshape(1, 1, 1, 2)
    for beta, key_r, key_top in ((2.0, "r_beta2", "top1_beta2"), (0.0, "r_beta0", "top1_beta0")):
        for sigma in (O.DIAG, O.FULL):
            p = small_problem(n_q=1, n_kv=4, d=2, block=2, topk=1, window=1, q_offset=3,
                              beta=beta, sigma=sigma)
            stored = O.stored_summaries(*O.block_summaries(K, p), p)
            s = O.route_scores_row(Q, stored, p, 0, 0, 0)
            assert np.array_equal(s, np.array(g[key_r], dtype=float))
            sel, _ = O.select_topk(s, 1)
            assert sel[0] == g[key_top]


def _dyadic_keys(rng, shape):
    return rng.integers(-4, 5, size=shape).astype(np.float64)   # exact in fp32 and after /4, /16


def test_full_sigma_score_equals_logit_mean_plus_half_beta_logit_variance():
    """r_c(q) computed from mu_c / Sigma_c must equal the mean of the block's
    logits q.k_j plus (beta/2) times their population variance."""
    rng = np.random.default_rng(6)
    for beta in (0.0, 0.5, 2.0, -1.0):
        K = _dyadic_keys(rng, (1, 32, 1, 4))
        Q = _dyadic_keys(rng, (1, 32, 1, 4))
        p = small_problem(beta=beta)
        stored = O.stored_summaries(*O.block_summaries(K, p), p)
        for i in (3, 17, 31):
            s = O.route_scores_row(Q, stored, p, 0, i, 0)
            nv = O.visible_blocks(i, p)
            for c in range(nv):
                logits = [float(np.dot(Q[0, i, 0], K[0, c * 4 + j, 0])) for j in range(4)]
                m = sum(logits) / 4
                v = sum((x - m) ** 2 for x in logits) / 4
                assert s[c] == pytest.approx(m + beta / 2 * v, rel=1e-12, abs=1e-12)


def test_diag_score_matches_per_dimension_variance_and_full_when_uncorrelated():
    rng = np.random.default_rng(7)
    K = _dyadic_keys(rng, (1, 32, 1, 4))
    Q = _dyadic_keys(rng, (1, 32, 1, 4))
    p = small_problem(sigma=O.DIAG)
    stored = O.stored_summaries(*O.block_summaries(K, p), p)
    s = O.route_scores_row(Q, stored, p, 0, 31, 0)
    q = Q[0, 31, 0]
    for c in range(8):
        keys = K[0, c * 4:(c + 1) * 4, 0]
        direct = q @ keys.mean(axis=0) + 1.0 * np.sum(q * q * keys.var(axis=0))
        assert s[c] == pytest.approx(direct, rel=1e-12, abs=1e-12)
    # keys with exactly diagonal covariance: rows of a Hadamard pattern
    H = np.array([[1, 1, 1], [1, -1, -1], [-1, 1, -1], [-1, -1, 1]], dtype=np.float64)
    K2 = np.zeros((1, 8, 1, 3))
    K2[0, :4, 0] = H * np.array([1.0, 2.0, 0.5]) + 1.0
    K2[0, 4:, 0] = H * np.array([3.0, 0.25, 1.0]) - 2.0
    Q2 = np.tile(np.array([0.5, -1.0, 2.0]), (1, 8, 1, 1))
    pd = small_problem(n_q=8, n_kv=8, d=3, block=4, sigma=O.DIAG)
    pf = small_problem(n_q=8, n_kv=8, d=3, block=4, sigma=O.FULL)
    sd = O.route_scores_row(Q2, O.stored_summaries(*O.block_summaries(K2, pd), pd), pd, 0, 7, 0)
    sf = O.route_scores_row(Q2, O.stored_summaries(*O.block_summaries(K2, pf), pf), pf, 0, 7, 0)
    np.testing.assert_allclose(sd, sf, rtol=1e-14)


def test_beta_zero_is_centroid_routing():
    rng = np.random.default_rng(8)
    K = rng.standard_normal((1, 64, 1, 8)).astype(np.float32).astype(np.float64)
    Q = rng.standard_normal((1, 64, 1, 8)).astype(np.float32).astype(np.float64)
    p = small_problem(n_q=64, n_kv=64, d=8, block=8, beta=0.0, sigma=O.FULL)
    stored = O.stored_summaries(*O.block_summaries(K, p), p)
    s = O.route_scores_row(Q, stored, p, 0, 63, 0)
    mean_logit = np.array([np.mean(K[0, c * 8:(c + 1) * 8, 0] @ Q[0, 63, 0]) for c in range(8)])
    np.testing.assert_allclose(s, mean_logit, rtol=1e-6, atol=1e-6)   # fp32-rounded mu


def test_group_score_is_sum_of_head_scores():
    rng = np.random.default_rng(9)
    K = _dyadic_keys(rng, (1, 32, 2, 4))
    Q = _dyadic_keys(rng, (1, 32, 8, 4))
    for sigma in (O.DIAG, O.FULL):
        p = small_problem(h_q=8, h_kv=2, sigma=sigma)
        stored = O.stored_summaries(*O.block_summaries(K, p), p)
        s = O.route_scores_row(Q, stored, p, 0, 30, 1)
        per_head = np.zeros_like(s)
        for h in range(4, 8):
            ph = small_problem(h_q=1, h_kv=1, sigma=sigma)
            st = O.stored_summaries(*O.block_summaries(K[:, :, 1:2], ph), ph)
            per_head += O.route_scores_row(Q[:, :, h:h + 1], st, ph, 0, 30, 0)
        np.testing.assert_allclose(s, per_head, rtol=1e-13)


def test_bf16_features_exact_case_equals_group_score():
    """With small-integer queries every feature rounding is exact, so the bf16
    route equals the exact group score on the bf16 table."""
    rng = np.random.default_rng(10)
    K = torch.randn(1, 64, 2, 8, generator=torch.Generator().manual_seed(10)).to(torch.bfloat16).float().numpy()
    Q = rng.integers(-3, 4, size=(1, 64, 4, 8)).astype(np.float64)
    p = O.Problem(batch=1, n_q=64, n_kv=64, h_q=4, h_kv=2, d=8, block=16, topk=2, window=16,
                  dtype=O.BF16, sigma=O.DIAG, beta=2.0)
    stored = O.stored_summaries(*O.block_summaries(K, p), p)
    tab = stored[2]
    F = O.route_features(Q, p)
    for g in range(2):
        qs = Q[0, 40, 2 * g:2 * g + 2].sum(axis=0)
        qq = (Q[0, 40, 2 * g:2 * g + 2] ** 2).sum(axis=0)
        np.testing.assert_array_equal(F[0, g, 40], np.concatenate([qs, qq]))
        s = O.route_scores_row(Q, stored, p, 0, 40, g)
        direct = sum(Q[0, 40, h] @ tab[0, g, :, :8].T + (Q[0, 40, h] ** 2) @ tab[0, g, :, 8:].T
                     for h in (2 * g, 2 * g + 1))[:2]
        np.testing.assert_allclose(s, direct, rtol=1e-14)
    # the full-row and the per-row route agree
    S = O.route_scores(Q, stored, p, 0, 1)
    np.testing.assert_allclose(S[40, :2], O.route_scores_row(Q, stored, p, 0, 40, 1), rtol=1e-14)


def _golden_feature_query(g):
    """The golden query as a [1, 1, G, d] array (heads by dimension in the file)."""
    return np.asarray(g["q_heads_by_dim"], dtype=np.float64).T[None, None]


def _bf16_torch(x):
    return torch.from_numpy(np.asarray(x, dtype=np.float32)).to(torch.bfloat16).double().numpy()


def _feature_variant(Q, beta, order="forward", acc=np.float32, round_first=False):
    """Routing features of a wrong-on-purpose variant: heads summed in another
    order, in another precision, or the squared sum rounded to bf16 before the
    (beta/2) multiply.  Rounding by torch, so nothing here is the oracle's."""
    q = np.asarray(Q[0, 0], dtype=acc)                      # [G, d]
    heads = range(q.shape[0]) if order == "forward" else reversed(range(q.shape[0]))
    qs = np.zeros(q.shape[1], dtype=acc)
    qq = np.zeros(q.shape[1], dtype=acc)
    for h in heads:
        qs = (qs + q[h]).astype(acc)
        qq = (qq + q[h] * q[h]).astype(acc)
    hb = np.float32(beta / 2)
    if round_first:
        fq = _bf16_torch((hb * _bf16_torch(qq).astype(np.float32)).astype(np.float32))
    else:
        fq = _bf16_torch((hb * qq).astype(np.float32) if acc == np.float32 else hb * qq)
    return np.concatenate([_bf16_torch(qs), fq])


def test_bf16_features_golden_rounding_order():
    """Hand-derived case (tests/golden/feature_rounding.json) in which the
    float32 head-order sums, the float32 (beta/2) multiply and the final
    round-to-nearest-even each decide a feature: the oracle must give the
    derived values, and summing in float64, summing the heads in reverse
    order, or rounding the squared sum before the (beta/2) multiply must each
    give a different (also hand-derived) row."""
    g = golden("feature_rounding.json")
    Q = _golden_feature_query(g)
    d, G = g["d"], g["G"]
    p = O.Problem(batch=1, n_q=1, n_kv=64, h_q=G, h_kv=1, d=d, block=16, topk=2, window=16,
                  dtype=O.BF16, sigma=O.DIAG, beta=g["beta"])
    f = O.route_features(Q, p)[0, 0, 0]
    assert np.array_equal(f, np.asarray(g["features"]))
    variants = {
        "features_reversed_head_order": _feature_variant(Q, g["beta"], order="reversed"),
        "features_float64_sums": _feature_variant(Q, g["beta"], acc=np.float64),
        "features_rounded_before_half_beta": _feature_variant(Q, g["beta"], round_first=True),
    }
    for key, v in variants.items():
        assert np.array_equal(v, np.asarray(g[key])), key
        assert not np.array_equal(v, f), key
    # the correct variant written the same way reproduces the oracle
    assert np.array_equal(_feature_variant(Q, g["beta"]), f)
    # and the routing score against a unit table row reads one feature back
    table = np.eye(2 * d)
    assert np.array_equal(table @ f, f)


def test_visible_blocks_brute_force():
    p = small_problem(n_kv=64, block=8)
    for pos in range(64):
        brute = sum(1 for c in range(8) if (c + 1) * 8 - 1 <= pos)
        assert O.visible_blocks(pos, p) == brute


# ------------------------------------------------------------------ top-k

def test_topk_brute_force_with_ties():
    rng = np.random.default_rng(11)
    for trial in range(300):
        nv = int(rng.integers(1, 8))
        k = int(rng.integers(1, 6))
        s = rng.integers(-3, 3, size=nv).astype(np.float64)      # many exact ties
        sel, gap = O.select_topk(s, k)
        take = min(k, nv)
        # brute force: the unique subset whose every member beats every non-member
        # under (higher score, then lower index)
        beats = lambda a, b: s[a] > s[b] or (s[a] == s[b] and a < b)
        found = None
        for sub in itertools.combinations(range(nv), take):
            rest = [c for c in range(nv) if c not in sub]
            if all(beats(a, b) for a in sub for b in rest):
                assert found is None
                found = sub
        assert list(sel[:take]) == sorted(found)
        assert all(x == -1 for x in sel[take:])
        if nv > k:
            srt = sorted(s, reverse=True)
            expect = (srt[k - 1] - srt[k]) / abs(srt[k - 1]) if srt[k - 1] != 0 else (
                np.inf if srt[k - 1] > srt[k] else 0.0)
            assert gap == expect


# ------------------------------------------------------------------ key set

def test_key_set_brute_force():
    p = small_problem(n_kv=64, block=8, window=11)
    rng = np.random.default_rng(12)
    for _ in range(100):
        pos = int(rng.integers(0, 64))
        nv = O.visible_blocks(pos, p)
        cand = list(range(nv))
        rng.shuffle(cand)
        sel = np.array(sorted(cand[:3]) + [-1] * (3 - min(3, nv)))
        S = O.key_set(pos, sel, p)
        brute = [j for j in range(64) if (j // 8 in set(sel[sel >= 0])) or (pos - 11 < j <= pos)]
        assert list(S) == brute
        assert all(j <= pos for j in S)


# ------------------------------------------------------------------ attention

def test_softmax_golden_three_keys():
    g = golden("softmax_three_keys.json")
    q = np.array([g["q"]])
    Ks = np.array(g["keys"])[:, None]
    Vs = np.array(g["values"])[:, None]
    o, lse = O.softmax_attend(q, Ks, Vs, 1.0)
    assert o[0, 0] == pytest.approx(g["o"], rel=1e-15)
    assert lse[0] == pytest.approx(g["lse"], rel=1e-15)


def test_full_budget_equals_dense_causal_attention():
    """With k >= number of blocks and W >= B every earlier key is attended,
    so the layer must reduce to dense causal softmax attention."""
    rng = np.random.default_rng(13)
    for G, sigma in ((1, O.FULL), (4, O.DIAG)):
        p = O.Problem(batch=2, n_q=48, n_kv=48, h_q=2 * G, h_kv=2, d=8, block=8, topk=6, window=8,
                      dtype=O.F32, sigma=sigma)
        Q = rng.standard_normal((2, 48, 2 * G, 8))
        K = rng.standard_normal((2, 48, 2, 8))
        V = rng.standard_normal((2, 48, 2, 8))
        out = O.forward(Q, K, V, p)
        Od, Ld = O.dense_causal_attention(Q, K, V, p)
        np.testing.assert_allclose(out["O"], Od, rtol=0, atol=1e-12)
        np.testing.assert_allclose(out["lse"], Ld, rtol=0, atol=1e-12)
    # decode: the single query at the last position equals the dense last row
    p = O.Problem(batch=1, n_q=1, n_kv=48, h_q=4, h_kv=2, d=8, block=8, topk=6, window=8,
                  q_offset=47, dtype=O.F32, sigma=O.DIAG)
    Qd = rng.standard_normal((1, 1, 4, 8))
    out = O.forward(Qd, K[:1], V[:1], p)
    Od, _ = O.dense_causal_attention(Qd, K[:1], V[:1], p)
    np.testing.assert_allclose(out["O"], Od, atol=1e-12)


def test_recovery_law_golden_and_exact_construction():
    for c in golden("recovery_law.json")["cases"]:
        assert O.recovery_weight(c["beta"], c["delta"], c["mu"]) == pytest.approx(c["w"], rel=1e-12)
    # exact construction: q = a e1, mu distractors orthogonal to e1, one target
    # at first coordinate Delta/a; V = e1 on the target only.  The attention
    # output's first coordinate is the target weight w* at beta = scale.
    d, a = 8, 2.0
    rng = np.random.default_rng(14)
    for mu, delta in ((7, 1.5), (63, 4.0), (255, 6.0)):
        Ks = np.zeros((mu + 1, d))
        Ks[:mu, 1:] = rng.standard_normal((mu, d - 1))
        Ks[mu, 0] = delta / a
        Vs = np.zeros((mu + 1, d))
        Vs[mu, 0] = 1.0
        q = np.zeros((1, d))
        q[0, 0] = a
        scale = 1 / math.sqrt(d)
        o, _ = O.softmax_attend(q, Ks, Vs, scale)
        assert o[0, 0] == pytest.approx(O.recovery_weight(scale, delta, mu), rel=1e-12)


def test_selection_cuts_distractors_recovery_improves():
    """Selection cuts mu from the causal prefix to the budget: the recovered
    target weight under SSA equals w* with mu = |S|-1, which is larger than
    dense attention's w* with mu = pos."""
    d, B = 8, 8
    n = 256
    K = np.zeros((1, n, 1, d))
    rng = np.random.default_rng(15)
    K[0, :, 0, 1:] = rng.standard_normal((n, d - 1)) * 0.0     # all distractor logits 0
    tgt = 40
    delta = 12.0
    K[0, tgt, 0, 0] = delta / 2.0
    V = np.zeros((1, n, 1, d))
    V[0, tgt, 0, 0] = 1.0
    Q = np.zeros((1, n, 1, d))
    Q[0, :, 0, 0] = 2.0
    p = O.Problem(batch=1, n_q=n, n_kv=n, h_q=1, h_kv=1, d=d, block=B, topk=2, window=8,
                  dtype=O.F32, sigma=O.DIAG)
    out = O.forward(Q, K, V, p, rows=[(0, 255)])
    Od, _ = O.dense_causal_attention(Q, K, V, p)
    S = O.key_set(255, out["block_idx"][0, 255, 0], p)
    assert tgt in S
    w_sparse = out["O"][0, 255, 0, 0]
    assert w_sparse == pytest.approx(O.recovery_weight(p.scale, delta, len(S) - 1), rel=1e-12)
    assert Od[0, 255, 0, 0] == pytest.approx(O.recovery_weight(p.scale, delta, 255), rel=1e-12)
    assert w_sparse > Od[0, 255, 0, 0]


def test_dropped_mass_identity_and_bound():
    """o_S - o_dense = eps (o_S - o_D), eps = dense softmax mass outside S and
    o_D the dense-normalised average of the dropped values; hence
    |o_S - o_dense|_inf <= eps * max_t (max_j v_jt - min_j v_jt)."""
    rng = np.random.default_rng(16)
    p = O.Problem(batch=1, n_q=128, n_kv=128, h_q=2, h_kv=1, d=8, block=8, topk=3, window=8,
                  dtype=O.F32, sigma=O.DIAG)
    Q = rng.standard_normal((1, 128, 2, 8)) * 1.5
    K = rng.standard_normal((1, 128, 1, 8))
    V = rng.standard_normal((1, 128, 1, 8))
    rows = [(0, i) for i in (40, 77, 127)]
    out = O.forward(Q, K, V, p, rows=rows)
    Od, _ = O.dense_causal_attention(Q, K, V, p)
    for _, i in rows:
        S = O.key_set(i, out["block_idx"][0, i, 0], p)
        D = np.setdiff1d(np.arange(i + 1), S)
        for h in range(2):
            logits = (K[0, :i + 1, 0] @ Q[0, i, h]) * p.scale
            w = np.exp(logits - logits.max())
            w /= w.sum()
            eps = w[D].sum()
            oD = (w[D, None] * V[0, D, 0]).sum(axis=0) / eps
            oS = out["O"][0, i, h]
            np.testing.assert_allclose(oS - Od[0, i, h], eps * (oS - oD), atol=1e-10)
            spread = V[0, :i + 1, 0].max(axis=0) - V[0, :i + 1, 0].min(axis=0)
            assert np.abs(oS - Od[0, i, h]).max() <= eps * spread.max() + 1e-12


def test_cumulant_routing_recovers_needles_centroid_misses():
    """On clustered keys with planted needles, second-cumulant routing (beta=2)
    puts the needle's block in the budget far more often than centroid
    routing (beta=0)."""
    from content_routed_block_ssa_b200.workload import WORKLOADS, make_inputs
    w = WORKLOADS["gqa_bf16_128k"].scaled(n=4096, needles=48, topk=4)
    Q, K, V, plan = make_inputs(w)
    Q, K = Q.float().numpy(), K.float().numpy()
    hits = {}
    for beta in (2.0, 0.0):
        p = O.Problem(batch=1, n_q=w.n, n_kv=w.n, h_q=w.h_q, h_kv=w.h_kv, d=w.d, block=w.block,
                      topk=w.topk, window=w.window, beta=beta, dtype=O.BF16, sigma=O.DIAG)
        stored = O.stored_summaries(*O.block_summaries(K, p), p)
        h = 0
        for (bi, i, head, j) in plan:
            s = O.route_scores_row(Q, stored, p, bi, i, head // p.group)
            sel, _ = O.select_topk(s, p.topk)
            h += int(j // p.block in set(sel))
        hits[beta] = h / len(plan)
    assert hits[2.0] >= 0.95
    assert hits[2.0] > hits[0.0] + 0.3


# ---------------------------------------------------------------- sub-block routing, tempered family

def test_subblock_summaries_are_summaries_of_the_smaller_blocks():
    rng = np.random.default_rng(21)
    K = O.round_bf16(rng.standard_normal((2, 256, 2, 16)))
    for S in (2, 4):
        p = O.Problem(2, 256, 256, 4, 2, 16, 64, 4, 64, subblocks=S, dtype="f32", sigma="full")
        q = O.Problem(2, 256, 256, 4, 2, 16, 64 // S, 4, 64, dtype="f32", sigma="full")
        mu_a, sig_a = O.block_summaries(K, p)
        mu_b, sig_b = O.block_summaries(K, q)
        assert mu_a.shape == (2, 2, 4 * S, 16)
        np.testing.assert_array_equal(mu_a, mu_b)
        np.testing.assert_array_equal(sig_a, sig_b)


def _direct_block_score(Qh, Kc, beta):
    """Sum over query heads of mean + (beta/2) population variance of the
    logits q_h . k_j over the keys Kc, from the keys themselves."""
    tot = 0.0
    for q in Qh:
        s = Kc @ q
        tot += s.mean() + 0.5 * beta * s.var()
    return tot


@pytest.mark.parametrize("sigma", ["full", "diag"])
def test_pooled_score_is_the_best_subblock_score_from_the_keys(sigma):
    rng = np.random.default_rng(22)
    B, S, d, G = 64, 4, 8, 2
    K = O.round_f32(rng.standard_normal((1, 4 * B, 1, d)))
    Q = O.round_f32(rng.standard_normal((1, 4 * B, G, d)))
    p = O.Problem(1, 4 * B, 4 * B, G, 1, d, B, 2, 16, subblocks=S, dtype="f32", sigma=sigma, beta=1.5)
    st = O.stored_summaries(*O.block_summaries(K, p), p)
    i = 4 * B - 1
    got = O.route_scores_row(Q, st, p, 0, i, 0)
    assert got.shape == (4,)
    Kn = K[0, :, 0]
    for c in range(4):
        want = max(_direct_block_score(Q[0, i], Kn[c * B + s * (B // S): c * B + (s + 1) * (B // S)], 1.5)
                   for s in range(S))
        if sigma == "diag":   # the diagonal form drops the cross-covariances: compare per-dimension
            want = max(sum(Q[0, i, h] @ Kn[c * B + s * 16: c * B + (s + 1) * 16].mean(0)
                           + 0.75 * (Q[0, i, h] ** 2) @ Kn[c * B + s * 16: c * B + (s + 1) * 16].var(0)
                           for h in range(G)) for s in range(S))
        assert abs(got[c] - want) <= 1e-5 * max(1.0, abs(want))


def test_subblock_pooling_rescues_a_spike_that_the_block_variance_dilutes():
    """A block whose only signal is one spike key loses to a block of
    uniformly spread keys under whole-block summaries, and wins once each
    block is summarised in four sub-blocks (the spike is then 1 key of 16,
    not 1 of 64)."""
    B, d = 64, 16
    K = np.zeros((1, 8 * B, 1, d))
    K[0, 3 * B:4 * B, 0, 0] = np.where(np.arange(B) % 2 == 0, 1.0, -1.0) * math.sqrt(2.0) / 4.0   # block 3
    K[0, 5 * B + 37, 0, 0] = 2.0                                                                   # block 5
    Q = np.zeros((1, 8 * B, 1, d))
    Q[0, :, 0, 0] = 4.0
    res = {}
    for S in (1, 4):
        p = O.Problem(1, 8 * B, 8 * B, 1, 1, d, B, 1, 1, subblocks=S, dtype="f32", sigma="diag", beta=2.0)
        st = O.stored_summaries(*O.block_summaries(K, p), p)
        s = O.route_scores_row(Q, st, p, 0, 8 * B - 1, 0)
        res[S] = O.select_topk(s, 1)[0][0]
    assert res[1] == 3 and res[4] == 5


def test_tempered_score_limits_and_cumulant_expansion():
    rng = np.random.default_rng(23)
    Kc = rng.standard_normal((64, 8))
    q = rng.standard_normal(8)
    s = Kc @ q
    mean, var = s.mean(), s.var()
    k3 = np.mean((s - mean) ** 3)
    assert O.tempered_block_score(q, Kc, 0.0) == pytest.approx(mean, rel=1e-12)
    assert O.tempered_block_score(q, Kc, 1e-6) == pytest.approx(mean, abs=1e-5)
    # T_beta = mean + (beta/2) var + (beta^2/6) k3 + O(beta^3): the cumulant score is the second-order term
    for beta in (1e-2, 3e-3):
        t = O.tempered_block_score(q, Kc, beta)
        assert (t - (mean + 0.5 * beta * var)) / beta ** 2 == pytest.approx(k3 / 6.0, rel=2e-2)
    # beta -> infinity: the exact maximum, approached as max - log(B)/beta for a unique max
    beta = 400.0
    assert O.tempered_block_score(q, Kc, beta) == pytest.approx(s.max() - math.log(64) / beta, abs=1e-9)
    # non-decreasing in beta (power-mean inequality)
    vals = [O.tempered_block_score(q, Kc, b) for b in (0.0, 0.1, 0.5, 1.0, 2.0, 8.0, 50.0)]
    assert all(a <= b + 1e-12 for a, b in zip(vals, vals[1:]))


# ------------------------------------------------------------------ hierarchical router

def _hier_problem(rng, n=512, d=16, block=4, G=2, h_kv=2, topk=4, node_keys=None, spread=4.0):
    """A bf16 problem and its stored summaries.  node_keys = M * block gives
    keys drawn around one centre per node (benign geometry: blocks of a node
    alike, nodes far apart); None gives iid keys."""
    p = O.Problem(1, n, n, G * h_kv, h_kv, d, block, topk, block, dtype=O.BF16, sigma=O.DIAG)
    if node_keys is None:
        K = rng.standard_normal((1, n, h_kv, d))
    else:
        cen = spread * rng.standard_normal((1, n // node_keys, h_kv, d))
        K = np.repeat(cen, node_keys, axis=1) + 0.1 * rng.standard_normal((1, n, h_kv, d))
    K = O.round_bf16(K)
    Q = O.round_bf16(rng.standard_normal((1, n, G * h_kv, d)))
    stored = O.stored_summaries(*O.block_summaries(K, p), p)
    return p, Q, stored


def test_hier_node_bound_is_admissible_and_tight_at_fanout_one():
    """Every block's score is at most its node's bound f.[m;v] + ||f_s|| R for
    features with a non-negative variance half, including features aimed at
    the farthest block; with one block per node the bound is the score."""
    rng = np.random.default_rng(31)
    d, nb = 8, 64
    mu = O.round_bf16(rng.standard_normal((1, 1, nb, d)) * rng.uniform(0.1, 3.0, (1, 1, nb, 1)))
    sg = O.round_bf16(rng.chisquare(2, (1, 1, nb, d)))
    table = np.concatenate([mu, sg], axis=-1)
    for M in (2, 4, 8):
        nt, rad, r_star, _t = O.hier_nodes(table, M)
        assert nt.shape == (1, 1, nb // M, 2 * d)
        assert r_star[0, 0] == rad[0, 0].max()
        for trial in range(200):
            fs = O.round_bf16(rng.standard_normal(d) * 2)
            fq = O.round_bf16(np.abs(rng.standard_normal(d)))
            if trial % 4 == 0:   # aim the mean half at the block farthest from its centre
                N = trial % (nb // M)
                far = np.argmax(np.linalg.norm(mu[0, 0, N * M:(N + 1) * M] - nt[0, 0, N, :d], axis=1))
                fs = O.round_bf16(mu[0, 0, N * M + far] - nt[0, 0, N, :d])
                fq = np.zeros(d)
            f = np.concatenate([fs, fq])
            bound = nt[0, 0] @ f + np.linalg.norm(fs) * rad[0, 0]
            score = (table[0, 0] @ f).reshape(nb // M, M)
            assert np.all(score.max(axis=1) <= bound + 1e-9)
            if trial % 4 == 0:   # Cauchy-Schwarz is attained in the aimed direction
                N = trial % (nb // M)
                assert score[N].max() >= bound[N] - 1e-2 * np.linalg.norm(fs) * rad[0, 0, N]
    nt1, rad1, r1, _t = O.hier_nodes(table, 1)
    np.testing.assert_array_equal(nt1, table)
    np.testing.assert_array_equal(rad1, 0.0)
    assert r1[0, 0] == 0.0


def test_hier_nodes_shift_and_radius_invariants():
    """Shifting every block mean by a vector shifts the node centres by it and
    keeps radii and variance caps; the radius is the largest centre distance
    (rounded up to float32), the cap the per-dimension maximum."""
    rng = np.random.default_rng(32)
    d, nb, M = 8, 32, 4
    mu = rng.integers(-16, 16, (1, 2, nb, d)) / 4.0      # exact in bf16, and so are node means
    sg = rng.integers(0, 64, (1, 2, nb, d)) / 8.0
    v = rng.integers(-8, 8, d) / 2.0
    a = O.hier_nodes(np.concatenate([mu, sg], -1), M)
    b = O.hier_nodes(np.concatenate([mu + v, sg], -1), M)
    np.testing.assert_array_equal(b[0][..., :d], a[0][..., :d] + v)
    np.testing.assert_array_equal(b[0][..., d:], a[0][..., d:])
    np.testing.assert_array_equal(b[1], a[1])
    for g in range(2):
        for N in range(nb // M):
            blk = mu[0, g, N * M:(N + 1) * M]
            np.testing.assert_array_equal(a[0][0, g, N, :d], blk.mean(axis=0))
            np.testing.assert_array_equal(a[0][0, g, N, d:], sg[0, g, N * M:(N + 1) * M].max(axis=0))
            dist = max(math.sqrt(sum((x - c) ** 2 for x, c in zip(row, blk.mean(axis=0)))) for row in blk)
            r = a[1][0, g, N]
            assert dist <= r <= dist * (1 + 2.0 ** -23)
            assert np.float32(r) == r


def _flat(Q, stored, p, bi, i, g):
    f = O.route_features(Q[bi:bi + 1, i:i + 1], p)[0, g, 0]
    nv = O.visible_blocks(p.q_offset + i, p)
    return O.select_topk(stored[2][bi, g, :nv] @ f, p.topk)[0]


@pytest.mark.parametrize("benign", [False, True])
def test_hier_certified_rows_hold_the_exact_topk(benign):
    """A certified row's kept blocks are the flat top-k of all its visible
    blocks; on benign geometry the certificate fires on most rows, on iid keys
    it rarely does (the bound is loose), and uncertified rows occur."""
    rng = np.random.default_rng(33 + benign)
    fired = total = 0
    for M, probe, topk in ((2, 2, 4), (4, 1, 4), (4, 3, 8), (8, 2, 4)):
        p, Q, stored = _hier_problem(rng, topk=topk, node_keys=(M * 4 if benign else None))
        rows = [(0, i) for i in range(0, p.n_q, 3)]
        bidx, cert, info = O.hier_route(Q, stored, p, M, probe, rows=rows)
        for (bi, i) in rows:
            for g in range(p.h_kv):
                total += 1
                if cert[bi, i, g]:
                    fired += 1
                    np.testing.assert_array_equal(bidx[bi, i, g], _flat(Q, stored, p, bi, i, g))
    if benign:
        assert fired > 0.6 * total
    else:
        assert fired < 0.6 * total
    assert fired < total


def test_hier_ranking_and_kept_set_brute_force():
    """The expanded nodes are the probe best by w_N (ties to the lower node),
    and the kept set is the top-k of the expanded nodes' blocks plus the
    visible blocks outside complete nodes, by explicit enumeration."""
    rng = np.random.default_rng(35)
    p, Q, stored = _hier_problem(rng, n=256, topk=3)
    M, probe = 4, 2
    nt, rad, r_star, t_star = O.hier_nodes(stored[2], M)
    f_all = O.route_features(Q, p)[0]
    for i in range(0, 256, 7):
        for g in range(p.h_kv):
            f = f_all[g, i]
            pos = i
            nvn = min(nt.shape[2], (pos + 1) // (M * p.block))
            nv = O.visible_blocks(pos, p)
            w = [(-(nt[0, g, N] @ f), N) for N in range(nvn)]
            exp = sorted(N for _, N in sorted(w)[:probe])
            kept, ok, info = O.hier_route_row(f, stored[2][0, g], (nt[0, g], rad[0, g], r_star[0, g], t_star[0, g]),
                                              pos, p, M, probe)
            assert list(info["expanded"]) == exp
            cand = [c for N in exp for c in range(N * M, N * M + M)] + list(range(nvn * M, nv))
            ranked = sorted(cand, key=lambda c: (-(stored[2][0, g, c] @ f), c))
            want = sorted(ranked[:p.topk]) + [-1] * max(0, p.topk - len(cand))
            assert list(kept) == want
            if nvn <= probe:
                assert ok


def test_hier_full_probe_and_escalation_equal_flat_and_twins_never_certify():
    rng = np.random.default_rng(36)
    p, Q, stored = _hier_problem(rng, n=256, topk=4)
    flat, _ = O.route_topk(Q, stored, p)
    M = 4
    nn = p.nb // M
    b1, c1, _ = O.hier_route(Q, stored, p, M, nn)            # every node expanded
    np.testing.assert_array_equal(b1, flat)
    assert c1.all()
    b2, c2, _ = O.hier_route(Q, stored, p, M, 1, escalate=True)
    np.testing.assert_array_equal(b2, flat)
    assert not c2.all()
    # two identical nodes: expanding one can never rule out the other
    tw = stored[2].copy()
    tw[:, :, 4:8] = tw[:, :, 0:4]
    st2 = (stored[0], stored[1], tw)
    _b, c3, info = O.hier_route(Q, st2, p, M, 1, rows=[(0, i) for i in range(64, 256)])
    for i in range(64, 256):
        for g in range(p.h_kv):
            if list(info[(0, i, g)]["expanded"]) in ([0], [1]) and ((i + 1) // (M * p.block)) > 1:
                assert not c3[0, i, g]


def test_hier_certificate_hand_cases_radius_and_margin():
    """Hand-computed rows (d = 2, one key per block, the whole sequence visible).

    Radius: nodes {b0, b1} with means (1,0), (1,0) and {b2, b3} with (-0.5,0),
    (1.5,0); f = [1, 0 ; 0, 0].  Node 0: centre (1,0), R = 0, w = 1; node 1:
    centre (0.5,0), R = 1, w = 0.5.  Probe 1 expands node 0, k = 1 keeps b0 with
    tau = 1, but the bound of node 1 is 0.5 + 1 * 1 = 1.5 > 1: not certified --
    rightly, b3 scores 1.5.
    Margin: one block per node, means (1,1) and (1,0), f = [1, e ; 0, 0]:
    tau = 1 + e against w_next = 1, R* = 0, margin = 2^-12 ||f|| sqrt(2);
    e = 2^-12 is inside the margin (not certified), e = 2^-10 outside it."""
    def row(table, f, M, probe, k):
        nb = table.shape[0]
        p = O.Problem(1, nb, nb, 1, 1, 2, 1, k, 1, dtype=O.BF16, sigma=O.DIAG)
        nt, rad, rs, ts = O.hier_nodes(table[None, None], M)
        return O.hier_route_row(np.asarray(f, float), table, (nt[0, 0], rad[0, 0], rs[0, 0], ts[0, 0]),
                                nb - 1, p, M, probe)
    t = np.array([[1, 0, 0, 0], [1, 0, 0, 0], [-0.5, 0, 0, 0], [1.5, 0, 0, 0]], float)
    kept, ok, info = row(t, [1, 0, 0, 0], 2, 1, 1)
    assert list(info["expanded"]) == [0] and list(kept) == [0] and info["tau"] == 1.0
    assert info["bound"] == pytest.approx(1.5 + 2.0 ** -12 * 1.5)
    assert not ok
    t2 = np.array([[1, 1, 0, 0], [1, 0, 0, 0]], float)
    for e, want in ((2.0 ** -12, False), (2.0 ** -10, True)):
        kept, ok, info = row(t2, [1, e, 0, 0], 1, 1, 1)
        assert list(kept) == [0] and ok is want


def test_hier_two_levels_hand_cases_recursive_radius_and_row_norm():
    """Hand-computed two-level rows (d = 2, one key per block, M = 2, probe 1,
    k = 1, f = [1, 0 ; 0, 0], the whole sequence visible).

    Nodes are tight (two equal blocks each, R_N = 0, so R* = 0) and the
    super-nodes' spread is all in the recursive radius.  Super-node 0 = nodes
    {2, 2}, {0, 0}: centre 1, R_S = max(|2 - 1| + 0, |0 - 1| + 0) = 1.
    (A) super-node 1 = nodes {-1, -1}, {2.5, 2.5}: centre 0.75,
    R_S = 1.75.  The row expands super-node 0 (w 1 > 0.75), then node 0, and
    keeps b0 with tau = 2; the node level holds (tau > 0 + 0 + margin) but the
    super level's bound 0.75 + 1.75 = 2.5 does not -- rightly, b6 scores 2.5.
    (B) super-node 1 = nodes {0.25, 0.25}, {1.25, 1.25}: centre 0.75,
    R_S = 0.5, R2* = 1; bound 0.75 + 1 = 1.75 < 2: certified, and b0 is the
    flat top-1.
    Row norm: a super-node's cap takes each dimension's largest node cap, so
    its row can be the longest one, and T* covers it."""
    def run(means):
        nb = len(means)
        table = np.zeros((nb, 4))
        table[:, 0] = means
        p = O.Problem(1, nb, nb, 1, 1, 2, 1, 1, 1, dtype=O.BF16, sigma=O.DIAG)
        nt, rad, rs, t1 = O.hier_nodes(table[None, None], 2)
        st, srad, r2, t2 = O.hier_super_nodes(nt, rad, t1, 2)
        kept, ok, info = O.hier_route_row2(np.array([1.0, 0, 0, 0]), table, (nt[0, 0], rad[0, 0], rs[0, 0], t1[0, 0]),
                                           (st[0, 0], srad[0, 0], r2[0, 0], t2[0, 0]), nb - 1, p, 2, 1)
        return kept, ok, info, rs[0, 0], srad[0, 0], r2[0, 0], t2[0, 0]
    kept, ok, info, r1, srad, r2, t2 = run([2, 2, 0, 0, -1, -1, 2.5, 2.5])
    assert r1 == 0.0 and list(srad) == [1.0, 1.75] and r2 == 1.75 and t2 == 2.5
    assert list(info["super_expanded"]) == [0] and list(info["expanded"]) == [0]
    assert list(kept) == [0] and info["tau"] == 2.0
    m = 2.0 ** -12 * 1.0 * 2.5
    assert info["bounds"][0] == pytest.approx(0.0 + m) and info["bounds"][1] == pytest.approx(2.5 + m)
    assert not ok
    kept, ok, info, r1, srad, r2, t2 = run([2, 2, 0, 0, 0.25, 0.25, 1.25, 1.25])
    assert list(srad) == [1.0, 0.5] and r2 == 1.0
    assert list(kept) == [0] and info["bounds"][1] == pytest.approx(1.75 + 2.0 ** -12 * 2.0)
    assert ok
    # the longest row is a super-node's: caps 1 in dimension 0 (node 0) and
    # in dimension 1 (node 1) give the super row (0, 0 ; 1, 1), norm sqrt(2),
    # against 1 for every block and node row
    table = np.zeros((1, 1, 8, 4))
    table[0, 0, 0:2, 2] = 1.0
    table[0, 0, 2:4, 3] = 1.0
    nt, rad, rs, t1 = O.hier_nodes(table, 2)
    st, srad, r2, t2 = O.hier_super_nodes(nt, rad, t1, 2)
    assert t1[0, 0] == 1.0
    assert math.sqrt(2) <= t2[0, 0] <= math.sqrt(2) * (1 + 2.0 ** -23)


def test_hier_listed_blocks_and_the_summaries_of_the_rest():
    """Listed blocks by explicit enumeration (the variance half's 2-norm above
    lambda times the node's (M/2)-th smallest); the node's centre, cap and
    radius over its unlisted blocks written out; the node bound is
    admissible for those blocks (features aimed at the farthest included);
    a very large lambda lists nothing and gives the plain node summaries."""
    rng = np.random.default_rng(47)
    d, nb = 8, 64
    mu = O.round_bf16(rng.standard_normal((1, 1, nb, d)))
    sg = O.round_bf16(rng.chisquare(2, (1, 1, nb, d)) * rng.choice([1.0, 1.0, 1.0, 9.0], (1, 1, nb, 1)))
    table = np.concatenate([mu, sg], axis=-1)
    for M, lam in ((4, 1.5), (8, 2.0), (8, 1.0), (16, 3.0)):
        listed = O.hier_listed_blocks(table, M, lam)
        nt, rad, r_star, _t = O.hier_nodes(table, M, listed)
        for N in range(nb // M):
            ids = list(range(N * M, (N + 1) * M))
            norms = [math.sqrt(float(sum(x * x for x in table[0, 0, c, d:]))) for c in ids]
            lm = sorted(norms)[M // 2 - 1]
            want = [norms[j] > lam * lm for j in range(M)]
            assert [bool(listed[0, 0, c]) for c in ids] == want
            keep = [c for c, lst in zip(ids, want) if not lst]
            assert len(keep) >= M // 2
            centre = O.round_bf16(O.round_f32(sum(table[0, 0, c, :d] for c in keep) / len(keep)))
            np.testing.assert_array_equal(nt[0, 0, N, :d], centre)
            np.testing.assert_array_equal(nt[0, 0, N, d:], np.max([table[0, 0, c, d:] for c in keep], axis=0))
            far = max(float(np.linalg.norm(table[0, 0, c, :d] - centre)) for c in keep)
            assert far <= rad[0, 0, N] <= far * (1 + 2.0 ** -23)
            for trial in range(40):
                fs = O.round_bf16(rng.standard_normal(d))
                fq = O.round_bf16(np.abs(rng.standard_normal(d)))
                if trial % 4 == 0:
                    c = max(keep, key=lambda c: np.linalg.norm(table[0, 0, c, :d] - centre))
                    fs, fq = O.round_bf16(table[0, 0, c, :d] - centre), np.zeros(d)
                f = np.concatenate([fs, fq])
                bound = nt[0, 0, N] @ f + np.linalg.norm(fs) * rad[0, 0, N]
                assert max(table[0, 0, c] @ f for c in keep) <= bound + 1e-9
    assert not O.hier_listed_blocks(table, 4, 1e30).any()
    plain = O.hier_nodes(table, 4)
    none = O.hier_nodes(table, 4, O.hier_listed_blocks(table, 4, 1e30))
    for a, b in zip(plain, none):
        np.testing.assert_array_equal(a, b)


def test_hier_listed_blocks_certify_nodes_with_one_extreme_key():
    """Nodes of alike blocks, a third of them holding one extreme key (its
    block's variance is large in every dimension).  Without listing those
    blocks lift their nodes' caps and the certificate rarely fires; listed
    (lambda = 2), they are scored exactly and it fires on most rows.  Either
    way a certified row holds the flat top-k, and escalation gives the flat
    router on every row."""
    rng = np.random.default_rng(48)
    M, probe, topk = 4, 2, 4
    p, Q, _ = _hier_problem(rng, n=512, topk=topk)      # the problem and its queries
    # keys around one centre per node, then the extreme keys planted
    n, h_kv, d, block = 512, 2, 16, 4
    cen = 4.0 * rng.standard_normal((1, n // (M * block), h_kv, d))
    K = np.repeat(cen, M * block, axis=1) + 0.1 * rng.standard_normal((1, n, h_kv, d))
    for node in range(0, n // (M * block), 3):
        j = node * M * block + int(rng.integers(0, M * block))
        K[0, j] = 12.0 * rng.choice([-1.0, 1.0], (h_kv, d))
    K = O.round_bf16(K)
    stored = O.stored_summaries(*O.block_summaries(K, p), p)
    rows = [(0, i) for i in range(64, p.n_q, 3)]
    rates = {}
    for lam in (None, 2.0):
        bidx, cert, _ = O.hier_route(Q, stored, p, M, probe, rows=rows, list_factor=lam)
        fired = 0
        for (bi, i) in rows:
            for g in range(p.h_kv):
                if cert[bi, i, g]:
                    fired += 1
                    np.testing.assert_array_equal(bidx[bi, i, g], _flat(Q, stored, p, bi, i, g))
        rates[lam] = fired / (len(rows) * p.h_kv)
    assert rates[2.0] > 0.6 and rates[None] < 0.5 * rates[2.0]
    flat, _ = O.route_topk(Q, stored, p)
    b2, _c, _ = O.hier_route(Q, stored, p, M, 1, escalate=True, list_factor=2.0)
    np.testing.assert_array_equal(b2, flat)


def test_unquantised_selection_is_the_float32_route_of_the_same_summaries():
    """The informational unquantised selection of a bf16 problem is the float32
    problem's selection from the float32 summaries, and its scores are the
    sum over the group's heads of <q_h, mu> + (beta/2) q_h^2 . sigma^2 from
    the float64 query heads (checked row by row against a direct sum)."""
    rng = np.random.default_rng(41)
    p = O.Problem(1, 96, 96, 4, 2, 8, 4, 3, 4, dtype=O.BF16, sigma=O.DIAG)
    K = O.round_bf16(rng.standard_normal((1, 96, 2, 8)))
    Q = O.round_bf16(rng.standard_normal((1, 96, 4, 8)))
    stored = O.stored_summaries(*O.block_summaries(K, p), p)
    bidx, gaps = O.route_topk_unquantised(Q, stored, p)
    mu32, sig32, _ = stored
    for i in range(0, 96, 5):
        for g in range(2):
            nv = O.visible_blocks(i, p)
            qh = Q[0, i, 2 * g:2 * g + 2]
            sc = np.array([sum(qh[h] @ mu32[0, g, c] + 1.0 * (qh[h] ** 2) @ sig32[0, g, c] for h in range(2))
                           for c in range(nv)])
            want, _ = O.select_topk(sc, p.topk)
            np.testing.assert_array_equal(bidx[0, i, g], want)


def test_hier_bound_constants_are_the_largest_radius_and_row_norm():
    """R* is the largest node radius and T* the largest 2-norm over the block
    rows and the node rows of each (batch, kv-head), rounded up to float32; a
    node row can be longer than every block row (its cap takes each
    dimension's largest variance)."""
    rng = np.random.default_rng(43)
    d, nb, M = 4, 16, 4
    mu = np.zeros((1, 2, nb, d))
    sg = np.zeros((1, 2, nb, d))
    for c in range(nb):                       # block c's variance sits in one dimension only
        sg[0, :, c, c % d] = 4.0
    mu[0, 1] = O.round_bf16(rng.standard_normal((nb, d)))
    table = np.concatenate([mu, sg], -1)
    nt, rad, r_star, t_star = O.hier_nodes(table, M)
    for g in range(2):
        assert r_star[0, g] == rad[0, g].max()
        norms = [np.linalg.norm(table[0, g, c]) for c in range(nb)] + \
                [np.linalg.norm(nt[0, g, N]) for N in range(nb // M)]
        assert max(norms) <= t_star[0, g] <= max(norms) * (1 + 2.0 ** -23)
    # kv-head 0: every block row has norm 4, every node row (cap 4 in all four
    # dimensions) norm 8
    assert t_star[0, 0] == 8.0


# ------------------------------------------------------------------ outlier channel

def test_outlier_channel_golden_block():
    """Hand case (tests/golden/outlier_channel.json): cumulant routing ranks
    the block of four moderate keys first; the outlier row (the largest-norm
    key, zero covariance) recovers the block holding the largest logit.
    Checked through both the float32 and the bf16 routing rows."""
    g = golden("outlier_channel.json")
    K = np.asarray(g["keys"], dtype=np.float64)[None, :, None, :]      # [1, 8, 1, 2]
    q = np.asarray(g["q"], dtype=np.float64)
    for dtype in (O.F32, O.BF16):
        kw = dict(batch=1, n_q=8, n_kv=8, h_q=1, h_kv=1, d=2, block=4, topk=1, window=1,
                  dtype=dtype, sigma=O.DIAG, beta=g["beta"])
        base = O.Problem(**kw)
        out = O.Problem(**kw, outlier=True)
        mu, sig = O.block_summaries(K, base)
        np.testing.assert_array_equal(mu[0, 0], g["mu"])
        np.testing.assert_array_equal(sig[0, 0], g["var"])
        mu2, sig2 = O.block_summaries(K, out)
        np.testing.assert_array_equal(mu2[0, 0, 1::2], g["outlier_key"])
        np.testing.assert_array_equal(sig2[0, 0, 1::2], np.zeros((2, 2)))
        Q = np.zeros((1, 8, 1, 2))
        Q[0, 7, 0] = q
        s0 = O.route_scores_row(Q, O.stored_summaries(mu, sig, base), base, 0, 7, 0)
        s1 = O.route_scores_row(Q, O.stored_summaries(mu2, sig2, out), out, 0, 7, 0)
        np.testing.assert_array_equal(s0, g["r_cumulant"])
        np.testing.assert_array_equal(s1, g["r_pooled"])
        assert O.select_topk(s0, 1)[0][0] == g["top1_cumulant"]
        assert O.select_topk(s1, 1)[0][0] == g["top1_with_outlier"]


def test_outlier_keys_brute_force_with_ties():
    """The outlier key is the first key of largest squared norm, by a direct
    scan; small integer keys make equal norms common."""
    rng = np.random.default_rng(21)
    p = O.Problem(batch=2, n_q=32, n_kv=32, h_q=2, h_kv=2, d=3, block=8, topk=2, window=8,
                  dtype=O.F32, sigma=O.FULL, outlier=True)
    for _ in range(20):
        K = rng.integers(-2, 3, size=(2, 32, 2, 3)).astype(np.float64)
        ko = O.outlier_keys(K, p)
        for b in range(2):
            for h in range(2):
                for c in range(4):
                    best, arg = -1.0, None
                    for j in range(8):
                        k = K[b, c * 8 + j, h]
                        n2 = float(k @ k)
                        if n2 > best:
                            best, arg = n2, k
                    np.testing.assert_array_equal(ko[b, h, c], arg)
        # the full-Sigma rows of the outlier channel are zero matrices, and the
        # block rows are the plain block summaries
        mu2, sig2 = O.block_summaries(K, p)
        mu1, sig1 = O.block_summaries(K, O.Problem(**{**p.__dict__, "outlier": False}))
        np.testing.assert_array_equal(mu2[:, :, 0::2], mu1)
        np.testing.assert_array_equal(sig2[:, :, 0::2], sig1)
        assert not sig2[:, :, 1::2].any()


def test_outlier_score_is_the_exact_group_logit_of_the_max_norm_key():
    """A block's outlier-row score equals sum_h q_h . k*_c computed directly
    from the keys, and the pooled score is the larger of it and the
    cumulant score."""
    rng = np.random.default_rng(22)
    p = O.Problem(batch=1, n_q=64, n_kv=64, h_q=4, h_kv=2, d=8, block=16, topk=2, window=16,
                  dtype=O.F32, sigma=O.DIAG, beta=2.0, outlier=True)
    K = rng.standard_normal((1, 64, 2, 8))
    Q = rng.standard_normal((1, 64, 4, 8))
    stored = O.stored_summaries(*O.block_summaries(K, p), p)
    base = O.Problem(**{**p.__dict__, "outlier": False})
    stored0 = O.stored_summaries(*O.block_summaries(K, base), base)
    for g in range(2):
        s = O.route_scores_row(Q, stored, p, 0, 63, g)
        s0 = O.route_scores_row(Q, stored0, base, 0, 63, g)
        for c in range(4):
            Kc = K[0, c * 16:(c + 1) * 16, g]
            ks = O.round_f32(Kc[np.argmax((Kc * Kc).sum(axis=1))])
            logit = sum(O.round_f32(Q[0, 63, h]) @ ks for h in (2 * g, 2 * g + 1))
            assert abs(s[c] - max(s0[c], logit)) <= 1e-12 * max(1.0, abs(s[c]))
    with pytest.raises(ValueError):
        O.block_summaries(K, O.Problem(**{**p.__dict__, "subblocks": 2}))


# ------------------------------------------------------------------ two-level tree

def test_hier_super_node_bound_is_admissible_and_radius_recursive():
    """Every block's score is at most its super-node's bound f.[m_S;v_S] +
    ||f_s|| R_S (features aimed at the farthest block included); R_S is the
    largest ||m_N - m_S|| + R_N over its nodes, rounded up to float32, so it
    covers the true largest distance of a block mean from m_S."""
    rng = np.random.default_rng(41)
    d, nb = 8, 128
    mu = O.round_bf16(rng.standard_normal((1, 1, nb, d)) * rng.uniform(0.1, 3.0, (1, 1, nb, 1)))
    sg = O.round_bf16(rng.chisquare(2, (1, 1, nb, d)))
    table = np.concatenate([mu, sg], axis=-1)
    for M in (2, 4):
        nt, rad, _r1, t1 = O.hier_nodes(table, M)
        st, srad, r2, t2 = O.hier_super_nodes(nt, rad, t1, M)
        ns = nb // (M * M)
        assert st.shape == (1, 1, ns, 2 * d) and r2[0, 0] == srad[0, 0].max() and t2[0, 0] >= t1[0, 0]
        for S in range(ns):
            kids = nt[0, 0, S * M:(S + 1) * M]
            rec = max(float(np.linalg.norm(kids[j, :d] - st[0, 0, S, :d])) + float(rad[0, 0, S * M + j])
                      for j in range(M))
            assert rec <= srad[0, 0, S] <= rec * (1 + 2.0 ** -22)
            true = np.linalg.norm(mu[0, 0, S * M * M:(S + 1) * M * M] - st[0, 0, S, :d], axis=1).max()
            assert true <= srad[0, 0, S]
            np.testing.assert_array_equal(st[0, 0, S, d:], kids[:, d:].max(axis=0))
        for trial in range(200):
            fs = O.round_bf16(rng.standard_normal(d) * 2)
            fq = O.round_bf16(np.abs(rng.standard_normal(d)))
            if trial % 4 == 0:
                S = trial % ns
                blk = mu[0, 0, S * M * M:(S + 1) * M * M]
                far = np.argmax(np.linalg.norm(blk - st[0, 0, S, :d], axis=1))
                fs = O.round_bf16(blk[far] - st[0, 0, S, :d])
                fq = np.zeros(d)
            f = np.concatenate([fs, fq])
            bound = st[0, 0] @ f + np.linalg.norm(fs) * srad[0, 0]
            score = (table[0, 0, :ns * M * M] @ f).reshape(ns, M * M)
            assert np.all(score.max(axis=1) <= bound + 1e-9)


def test_hier_two_levels_brute_force_ranking():
    """Both levels by explicit enumeration: the probe best super-nodes by w_S
    (ties to the lower index), then the probe best of their nodes and the
    nodes outside complete super-nodes by w_N, then the top-k of the expanded
    nodes' blocks and the blocks outside complete nodes."""
    rng = np.random.default_rng(42)
    p, Q, stored = _hier_problem(rng, n=512, topk=3)
    M, probe = 2, 2
    nt, rad, r1, t1 = O.hier_nodes(stored[2], M)
    st, srad, r2, t2 = O.hier_super_nodes(nt, rad, t1, M)
    f_all = O.route_features(Q, p)[0]
    T = stored[2]
    for i in range(0, 512, 11):
        for g in range(p.h_kv):
            f = f_all[g, i]
            nv = O.visible_blocks(i, p)
            nvn = min(nt.shape[2], (i + 1) // (M * p.block))
            nvs = min(st.shape[2], (i + 1) // (M * M * p.block))
            sexp = sorted(sorted(range(nvs), key=lambda S: (-(st[0, g, S] @ f), S))[:probe])
            ncand = [N for S in sexp for N in range(S * M, S * M + M)] + list(range(nvs * M, nvn))
            nexp = sorted(sorted(ncand, key=lambda N: (-(nt[0, g, N] @ f), N))[:probe])
            cand = [c for N in nexp for c in range(N * M, N * M + M)] + list(range(nvn * M, nv))
            ranked = sorted(cand, key=lambda c: (-(T[0, g, c] @ f), c))
            want = sorted(ranked[:p.topk]) + [-1] * max(0, p.topk - len(cand))
            kept, ok, info = O.hier_route_row2(f, T[0, g], (nt[0, g], rad[0, g], r1[0, g], t1[0, g]),
                                               (st[0, g], srad[0, g], r2[0, g], t2[0, g]), i, p, M, probe)
            assert list(info["super_expanded"]) == sexp and list(info["expanded"]) == nexp
            assert list(kept) == want
            if nvs <= probe and len(ncand) <= probe:
                assert ok


@pytest.mark.parametrize("benign", [False, True])
def test_hier_two_levels_certified_rows_hold_the_exact_topk(benign):
    """A certified row of the two-level tree keeps the flat top-k of all its
    visible blocks; probing every super-node and node gives the flat router;
    escalation gives the flat router on every row."""
    rng = np.random.default_rng(43 + benign)
    fired = total = 0
    for M, probe, topk in ((2, 2, 4), (4, 2, 4), (2, 3, 8)):
        p, Q, stored = _hier_problem(rng, n=512, topk=topk, node_keys=(M * 4 if benign else None))
        rows = [(0, i) for i in range(0, p.n_q, 5)]
        bidx, cert, _ = O.hier_route(Q, stored, p, M, probe, rows=rows, levels=2)
        for (bi, i) in rows:
            for g in range(p.h_kv):
                total += 1
                if cert[bi, i, g]:
                    fired += 1
                    np.testing.assert_array_equal(bidx[bi, i, g], _flat(Q, stored, p, bi, i, g))
    assert 0 < fired < total
    p, Q, stored = _hier_problem(rng, n=256, topk=4)
    flat, _ = O.route_topk(Q, stored, p)
    M = 2
    b1, c1, _ = O.hier_route(Q, stored, p, M, p.nb // M, levels=2)   # everything expanded
    np.testing.assert_array_equal(b1, flat)
    assert c1.all()
    b2, _c2, _ = O.hier_route(Q, stored, p, M, 1, escalate=True, levels=2)
    np.testing.assert_array_equal(b2, flat)
