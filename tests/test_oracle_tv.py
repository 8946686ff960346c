"""Pins for the oracle's TV self-distillation loss and its gradient.

LoopUno project page, "Training is self-distillation": the loss is the total-variation
distance between the frozen teacher's and the student's next-token distributions on the
response tokens. Pinned by: TV(p, p) = 0, symmetry and range, the two-token closed form
|sigmoid(a) - sigmoid(b)| (library expit), acceptance = 1 - TV = sum min(p, q), the
gradient's zero row sum, and fp64 central finite differences of the mean.
"""
import numpy as np
from scipy.special import expit, softmax

import oracle


def test_identical_is_zero():
    rng = np.random.default_rng(20)
    t = rng.standard_normal((5, 40)) * 3
    out = oracle.tv_loss(t, t)
    assert (out["tv"] == 0).all() and out["mean"] == 0
    assert (out["grad"] == 0).all()


def test_range_symmetry_and_overlap_identity():
    rng = np.random.default_rng(21)
    t, s = rng.standard_normal((8, 100)) * 3, rng.standard_normal((8, 100)) * 3
    a, b = oracle.tv_loss(t, s), oracle.tv_loss(s, t)
    np.testing.assert_allclose(a["tv"], b["tv"], rtol=1e-14)
    assert ((a["tv"] >= 0) & (a["tv"] <= 1)).all()
    p, q = softmax(t, axis=1), softmax(s, axis=1)
    np.testing.assert_allclose(a["tv"], 1 - np.minimum(p, q).sum(axis=1), atol=1e-14)


def test_two_token_closed_form():
    rng = np.random.default_rng(22)
    t, s = rng.standard_normal((50, 2)) * 4, rng.standard_normal((50, 2)) * 4
    out = oracle.tv_loss(t, s)
    expect = np.abs(expit(t[:, 1] - t[:, 0]) - expit(s[:, 1] - s[:, 0]))
    np.testing.assert_allclose(out["tv"], expect, rtol=1e-12, atol=1e-15)


def test_disjoint_mass_is_one():
    out = oracle.tv_loss(np.array([[60.0, 0.0, 0.0]]), np.array([[0.0, 0.0, 60.0]]))
    assert abs(out["tv"][0] - 1.0) < 1e-20 + 2e-26 * 1e6


def test_mean_over_mask_and_masked_gradient():
    rng = np.random.default_rng(23)
    t, s = rng.standard_normal((6, 30)), rng.standard_normal((6, 30))
    mask = np.array([1, 0, 1, 1, 0, 0], np.uint8)
    out = oracle.tv_loss(t, s, mask=mask, grad_scale=2.0)
    assert abs(out["mean"] - out["tv"][mask == 1].mean()) < 1e-15
    assert (out["grad"][mask == 0] == 0).all()
    full = oracle.tv_loss(t, s, grad_scale=2.0)
    np.testing.assert_allclose(out["grad"][mask == 1], full["grad"][mask == 1] * 6 / 3, rtol=1e-13)
    empty = oracle.tv_loss(t, s, mask=np.zeros(6, np.uint8))
    assert empty["mean"] == 0 and (empty["grad"] == 0).all()


def test_gradient_rows_sum_to_zero():
    rng = np.random.default_rng(24)
    t, s = rng.standard_normal((10, 500)) * 3, rng.standard_normal((10, 500)) * 3
    g = oracle.tv_loss(t, s)["grad"]
    assert np.abs(g.sum(axis=1)).max() < 1e-17 + 1e-14 * np.abs(g).sum(axis=1).max()


def test_gradient_finite_differences():
    """Central differences of the masked mean w.r.t. each student logit (fp64)."""
    rng = np.random.default_rng(25)
    N, V = 3, 7
    t, s = rng.standard_normal((N, V)) * 2, rng.standard_normal((N, V)) * 2
    mask = np.array([1, 1, 0], np.uint8)
    out = oracle.tv_loss(t, s, mask=mask, grad_scale=1.7)
    h = 1e-6
    for n in range(N):
        for v in range(V):
            sp, sm = s.copy(), s.copy()
            sp[n, v] += h
            sm[n, v] -= h
            fd = 1.7 * (oracle.tv_loss(t, sp, mask=mask)["mean"] - oracle.tv_loss(t, sm, mask=mask)["mean"]) / (2 * h)
            assert abs(fd - out["grad"][n, v]) < 1e-8, (n, v, fd, out["grad"][n, v])


def test_absdiff_output():
    rng = np.random.default_rng(26)
    t, s = rng.standard_normal((2, 9)), rng.standard_normal((2, 9))
    out = oracle.tv_loss(t, s, want_absdiff=True)
    np.testing.assert_allclose(out["absdiff"], np.abs(softmax(t, axis=1) - softmax(s, axis=1)), atol=1e-15)
