"""Pins for the oracle's row warping, sampling and lossless block verify.

What the pages fix, and how each is checked here:
  * losslessness (LoopUno "How it works" / "Training is self-distillation"; the model
    card's "lossless verification"): at every reached block position the emitted token
    is distributed exactly as the verifier's warped distribution p_i. Checked by exact
    enumeration of the uniforms' joint law on tiny vocabularies, and by Monte Carlo;
  * acceptance probability is exactly 1 - TV (LoopUno "Training is self-distillation");
  * position 0 is always the exact AR token, so a step never moves backward;
  * tokens per step vs per-position acceptance ("Scaling with training": TPF 2.1-2.2 at
    acceptance 0.54 with block 8) fixes the counting convention;
  * sampler settings (model card "Evaluation protocol"): hand-worked warping fixtures.
"""
import itertools
import json
import os

import numpy as np
import pytest
from scipy.special import softmax

import oracle
from tests.conftest import GOLDEN


# ---------------------------------------------------------------------------------------
# warping and sampling
# ---------------------------------------------------------------------------------------
def test_warp_golden():
    d = json.load(open(os.path.join(GOLDEN, "warp_rows_hand.json")))
    for c in d["cases"]:
        dist, _, nk = oracle.warp_row(c["logits"], c["temperature"], c["top_k"], c["top_p"])
        np.testing.assert_allclose(dist, c["dist"], rtol=0, atol=1e-15, err_msg=c["name"])
        assert nk == int(np.count_nonzero(np.array(c["dist"]))), c["name"]


def test_warp_unfiltered_is_softmax():
    rng = np.random.default_rng(5)
    for V, T in ((7, 1.0), (1000, 0.7), (33, 2.5)):
        z = rng.standard_normal(V) * 3
        dist, margin, nk = oracle.warp_row(z, T, 0, 1.0)
        np.testing.assert_allclose(dist, softmax(z / T), rtol=1e-13, atol=1e-300)  # library routine
        assert margin == np.inf and nk == V


def test_topk_equals_sort_selection():
    rng = np.random.default_rng(6)
    for trial in range(20):
        V = int(rng.integers(5, 200))
        k = int(rng.integers(1, V))
        z = np.round(rng.standard_normal(V) * 2, 1)  # coarse values: many ties
        order = np.lexsort((np.arange(V), -z))       # library sort: z desc, id asc
        keep = np.zeros(V, bool)
        keep[order[:k]] = True
        expect = np.where(keep, np.exp(z - z[keep].max()), 0.0)
        expect /= expect.sum()
        dist, _, nk = oracle.warp_row(z, 1.0, k, 1.0)
        assert nk == k
        np.testing.assert_allclose(dist, expect, rtol=1e-13, atol=1e-300)


def test_topp_keeps_shortest_prefix():
    rng = np.random.default_rng(7)
    for trial in range(20):
        V = int(rng.integers(3, 60))
        z = rng.standard_normal(V) * 2
        top_p = float(rng.uniform(0.05, 0.99))
        dist, margin, nk = oracle.warp_row(z, 1.0, 0, top_p)
        p = softmax(z)
        kept = dist > 0
        # every kept token is at least as probable as every dropped one
        if (~kept).any():
            assert p[kept].min() >= p[~kept].max()
        # the kept mass reaches top_p and dropping the smallest kept token falls below it
        assert p[kept].sum() >= top_p - 1e-12
        assert p[kept].sum() - p[kept].min() < top_p + 1e-12
        np.testing.assert_allclose(dist[kept], p[kept] / p[kept].sum(), rtol=1e-12)
        assert margin >= 0


def test_temperature_scale_invariance():
    rng = np.random.default_rng(8)
    z = rng.standard_normal(50)
    a, _, _ = oracle.warp_row(z, 1.0, 10, 0.9)
    b, _, _ = oracle.warp_row(z * 2.5, 2.5, 10, 0.9)
    np.testing.assert_allclose(a, b, rtol=1e-12, atol=1e-300)


def test_inv_cdf_golden():
    d = json.load(open(os.path.join(GOLDEN, "inv_cdf_hand.json")))
    for c in d["cases"]:
        t, m = oracle.inv_cdf(c["weights"], c["u"])
        assert t == c["token"], c


def test_inv_cdf_law_matches_weights():
    """The length of the u-interval mapped to each token equals its probability."""
    w = np.array([0.1, 0.0, 0.35, 0.05, 0.5])
    grid = (np.arange(100000) + 0.5) / 100000
    toks = np.array([oracle.inv_cdf(w, u)[0] for u in grid[::10]])
    freq = np.bincount(toks, minlength=5) / toks.size
    np.testing.assert_allclose(freq, w, atol=2e-4)


# ---------------------------------------------------------------------------------------
# exact enumeration of the verify step on tiny vocabularies
# ---------------------------------------------------------------------------------------
def _cells_from_dist(dist):
    """(midpoint u, weight, token) for each token's u-interval under inverse-CDF."""
    c = np.concatenate([[0.0], np.cumsum(dist)])
    c[-1] = 1.0
    return [((c[t] + c[t + 1]) / 2, dist[t], t) for t in range(len(dist)) if dist[t] > 0]


def _position_cells(P, Q, first):
    """Cells (u0, u1, u2, weight) of one block position's uniforms."""
    if first:
        return [(u0, 0.5, 0.5, w) for (u0, w, _) in _cells_from_dist(P)]
    res = np.maximum(P - Q, 0.0)
    res = res / res.sum() if res.sum() > 0 else P
    out = []
    for (u0, wq, d) in _cells_from_dist(Q):
        ratio = P[d] / Q[d]
        if ratio >= 1.0:
            out.append((u0, 0.5, 0.5, wq))
            continue
        if ratio > 0:
            out.append((u0, ratio / 2, 0.5, wq * ratio))
        for (u2, wr, _) in _cells_from_dist(res):
            out.append((u0, (1 + ratio) / 2, u2, wq * (1 - ratio) * wr))
    return out


def _enumerate(Pl, Ql, T=1.0, top_k=0, top_p=1.0):
    K, V = Pl.shape
    P = np.stack([oracle.warp_row(Pl[i], T, top_k, top_p)[0] for i in range(K)])
    Q = np.stack([oracle.warp_row(Ql[i], T, top_k, top_p)[0] for i in range(K)])
    cells = [_position_cells(P[i], Q[i], i == 0) for i in range(K)]
    combos = list(itertools.product(*cells))
    n = len(combos)
    u = np.array([[c[:3] for c in combo] for combo in combos])          # [n, K, 3]
    w = np.array([np.prod([c[3] for c in combo]) for combo in combos])  # [n]
    out = oracle.block_verify(np.broadcast_to(Pl, (n, K, V)), np.broadcast_to(Ql, (n, K, V)), u,
                              T, top_k, top_p)
    return P, Q, w, out


@pytest.mark.parametrize("case", range(6))
def test_exact_losslessness(case):
    rng = np.random.default_rng(100 + case)
    K, V = 3, 4
    Pl = rng.standard_normal((K, V)) * 1.5
    Ql = rng.standard_normal((K, V)) * 1.5
    T, top_k, top_p = [(1.0, 0, 1.0), (1.0, 2, 1.0), (1.0, 0, 0.8), (0.7, 3, 0.9), (1.3, 0, 1.0),
                       (1.0, 1, 1.0)][case]
    P, Q, w, out = _enumerate(Pl, Ql, T, top_k, top_p)
    assert abs(w.sum() - 1.0) < 1e-12
    count, toks, nxt = out["count"], out["tokens"], out["next"]
    tv = 0.5 * np.abs(P - Q).sum(axis=1)
    # position 0 is always emitted and is distributed as P_0
    assert (count >= 1).all()
    marg0 = np.bincount(toks[:, 0], weights=w, minlength=V)
    np.testing.assert_allclose(marg0, P[0], atol=1e-12)
    for i in range(1, K):
        reached = count >= i
        pr = w[reached].sum()
        assert abs(pr - np.prod(1.0 - tv[1:i])) < 1e-12
        if pr == 0.0:  # an earlier position has TV = 1: position i is never reached
            continue
        emitted = np.where(count > i, toks[:, i], nxt)
        marg = np.bincount(emitted[reached], weights=w[reached], minlength=V) / pr
        np.testing.assert_allclose(marg, P[i], atol=1e-12, err_msg=f"position {i}")
        acc = w[count > i].sum() / pr
        assert abs(acc - (1.0 - tv[i])) < 1e-12, (i, acc, 1 - tv[i])
    expect_n = 1.0 + sum(np.prod(1.0 - tv[1:k + 1]) for k in range(1, K))
    assert abs((w * count).sum() - expect_n) < 1e-12
    # emitted tokens after the count are -1; next is -1 exactly when all were accepted
    for i in range(K):
        assert (toks[count <= i, i] == -1).all()
    assert ((nxt == -1) == (count == K)).all()


def test_exact_disjoint_support_always_rejects():
    """TV = 1 (top-1 on different argmaxes): every draft rejected, correction ~ P."""
    Pl = np.array([[0.0, 5.0, 1.0, 2.0], [3.0, 0.0, 1.0, 0.5]])
    Ql = np.array([[0.0, 0.0, 0.0, 0.0], [0.0, 4.0, 1.0, 0.5]])
    P, Q, w, out = _enumerate(Pl, Ql, 1.0, 1, 1.0)
    assert (out["count"] == 1).all()
    assert (out["next"] == 0).all()  # argmax of P_1
    assert (out["tokens"][:, 0] == 1).all()


# ---------------------------------------------------------------------------------------
# Monte Carlo and closed forms
# ---------------------------------------------------------------------------------------
def test_monte_carlo_acceptance_and_marginal():
    rng = np.random.default_rng(9)
    K, V, n = 4, 16, 200000
    Pl = rng.standard_normal((K, V)) * 2
    Ql = 0.6 * Pl + 0.8 * rng.standard_normal((K, V)) * 2
    u = rng.random((n, K, 3))
    out = oracle.block_verify(np.broadcast_to(Pl, (n, K, V)), np.broadcast_to(Ql, (n, K, V)), u)
    P = softmax(Pl, axis=1)
    Q = softmax(Ql, axis=1)
    tv = 0.5 * np.abs(P - Q).sum(axis=1)
    acc1 = (out["count"] > 1).mean()
    assert abs(acc1 - (1 - tv[1])) < 5 * np.sqrt(tv[1] * (1 - tv[1]) / n)
    emitted = np.where(out["count"] > 1, out["tokens"][:, 1], out["next"])
    freq = np.bincount(emitted, minlength=V) / n
    assert (np.abs(freq - P[1]) < 5 * np.sqrt(P[1] * (1 - P[1]) / n) + 1e-9).all()
    expect_n = 1.0 + sum(np.prod(1.0 - tv[1:k + 1]) for k in range(1, K))
    sd = out["count"].std()
    assert abs(out["count"].mean() - expect_n) < 5 * sd / np.sqrt(n)


def test_tpf_vs_acceptance_counting_convention():
    d = json.load(open(os.path.join(GOLDEN, "tpf_acceptance.json")))
    a, K = d["acceptance"], d["block"]
    closed = (1 - a ** K) / (1 - a)
    assert abs(closed - d["expected_count"]) < 1e-6
    assert d["tpf_low"] <= closed <= d["tpf_high"]
    assert not (d["tpf_low"] <= closed + 1 <= d["tpf_high"])  # counting the correction too would not fit
    # two-token rows with TV = 1 - a at every draft position
    p = np.array([0.5 + (1 - a) / 2 + 0.04, 0.0])
    p[1] = 1 - p[0]
    q = np.array([p[0] - (1 - a), 0.0])
    q[1] = 1 - q[0]
    assert abs(0.5 * np.abs(p - q).sum() - (1 - a)) < 1e-12
    n = 200000
    Pl = np.broadcast_to(np.log(p), (n, K, 2))
    Ql = np.broadcast_to(np.log(q), (n, K, 2))
    u = np.random.default_rng(10).random((n, K, 3))
    out = oracle.block_verify(Pl, Ql, u)
    c = out["count"]
    assert abs(c.mean() - closed) < 5 * c.std() / np.sqrt(n)
    assert d["tpf_low"] <= c.mean() <= d["tpf_high"]


def test_identical_rows_accept_everything():
    rng = np.random.default_rng(11)
    B, K, V = 50, 6, 30
    L = rng.standard_normal((B, K, V)) * 3
    out = oracle.block_verify(L, L, rng.random((B, K, 3)), 1.0, 5, 0.9)
    assert (out["count"] == K).all() and (out["next"] == -1).all()
    np.testing.assert_allclose(out["tv"], 0.0, atol=1e-15)


def test_greedy_top1_is_argmax_verify():
    rng = np.random.default_rng(12)
    B, K, V = 40, 5, 12
    P = np.round(rng.standard_normal((B, K, V)), 1)
    Q = np.where(rng.random((B, K, V)) < 0.5, P, np.round(rng.standard_normal((B, K, V)), 1))
    out = oracle.block_verify(P, Q, rng.random((B, K, 3)), 1.0, 1, 1.0)
    ap = P.argmax(axis=2)  # library argmax: first (lowest) index among ties
    aq = Q.argmax(axis=2)
    for b in range(B):
        assert out["tokens"][b, 0] == ap[b, 0]
        n = 1
        while n < K and aq[b, n] == ap[b, n]:
            n += 1
        assert out["count"][b] == n
        np.testing.assert_array_equal(out["tokens"][b, 1:n], aq[b, 1:n])
        assert out["next"][b] == (ap[b, n] if n < K else -1)


def test_position0_is_the_ar_token():
    rng = np.random.default_rng(13)
    B, K, V = 20, 4, 50
    P, Q = rng.standard_normal((B, K, V)) * 2, rng.standard_normal((B, K, V)) * 2
    u = rng.random((B, K, 3))
    out = oracle.block_verify(P, Q, u, 0.8, 7, 0.93)
    for b in range(B):
        dist, _, _ = oracle.warp_row(P[b, 0], 0.8, 7, 0.93)
        assert out["tokens"][b, 0] == oracle.inv_cdf(dist, u[b, 0, 0])[0]
        assert abs(out["p_tok"][b, 0] - dist[out["tokens"][b, 0]]) < 1e-15
    pos0 = rng.integers(0, V, B).astype(np.int32)
    out2 = oracle.block_verify(P, Q, u, 0.8, 7, 0.93, pos0=pos0)
    np.testing.assert_array_equal(out2["tokens"][:, 0], pos0)
    assert (out2["count"] >= 1).all()
    # an entry < 0 (a previous step's next token when all its drafts were accepted) means
    # "draw from p_0": those sequences equal the run without pos0
    pos0[::3] = -1
    out3 = oracle.block_verify(P, Q, u, 0.8, 7, 0.93, pos0=pos0)
    for b in range(B):
        ref = out if pos0[b] < 0 else out2
        np.testing.assert_array_equal(out3["tokens"][b], ref["tokens"][b])
        assert out3["count"][b] == ref["count"][b] and out3["next"][b] == ref["next"][b]


def test_supplied_drafts_zero_probabilities():
    """q(d) = 0 < p(d): ratio is infinite, accept. p(d) = 0: reject; p == q: residual empty -> p."""
    K, V = 2, 4
    Pl = np.array([[0.0, 1.0, 2.0, 3.0], [0.0, 1.0, 2.0, 3.0]])
    Ql = np.array([[0.0, 1.0, 2.0, 3.0], [3.0, 2.0, 1.0, 0.0]])
    u = np.full((1, K, 3), 0.5)
    # top-2: P_1 keeps {2,3}, Q_1 keeps {0,1}; draft 3 has q = 0 -> accepted
    out = oracle.block_verify(Pl[None], Ql[None], u, 1.0, 2, 1.0, drafts=np.array([[0, 3]], np.int32))
    assert out["count"][0] == 2 and out["tokens"][0, 1] == 3
    # draft 0 has p = 0 -> rejected; correction from max(0, P - Q) = P_1 on {2, 3}
    out = oracle.block_verify(Pl[None], Ql[None], u, 1.0, 2, 1.0, drafts=np.array([[0, 0]], np.int32))
    assert out["count"][0] == 1 and out["next"][0] in (2, 3)
    # P_1 == Q_1 and a draft outside the support: rejected with an empty residual -> sample P_1
    out = oracle.block_verify(Pl[None], Pl[None], u, 1.0, 2, 1.0, drafts=np.array([[0, 1]], np.int32))
    dist, _, _ = oracle.warp_row(Pl[1], 1.0, 2, 1.0)
    assert out["count"][0] == 1 and out["next"][0] == oracle.inv_cdf(dist, 0.5)[0]


def test_block_of_one():
    rng = np.random.default_rng(14)
    P = rng.standard_normal((3, 1, 9))
    out = oracle.block_verify(P, P, rng.random((3, 1, 3)))
    assert (out["count"] == 1).all() and (out["next"] == -1).all()


def test_tv_output_is_one_minus_acceptance_probability():
    rng = np.random.default_rng(15)
    B, K, V = 4, 3, 20
    P, Q = rng.standard_normal((B, K, V)), rng.standard_normal((B, K, V))
    out = oracle.block_verify(P, Q, rng.random((B, K, 3)), 1.0, 8, 0.95)
    for b in range(B):
        for i in range(1, K):
            p, _, _ = oracle.warp_row(P[b, i], 1.0, 8, 0.95)
            q, _, _ = oracle.warp_row(Q[b, i], 1.0, 8, 0.95)
            assert abs(out["tv"][b, i] - (1 - np.minimum(p, q).sum())) < 1e-14
