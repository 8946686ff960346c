"""Pins for the oracle's gated-LoRA linear (fp64).

The oracle states y = x W0^T + scale * g * (x A^T) B^T with explicit loops. It is pinned by
a hand-worked example, by the special cases the pages fix (gate 0 / B = 0 / scale 0 is the
frozen base layer, LoopUno "How it works"; model card introduction), which reduce to a
library matmul, by linearity in the gate, and by a brute-force per-element check.
"""
import json
import os

import numpy as np

import oracle
from tests.conftest import GOLDEN


def _rand(shape, rng, s=1.0):
    return rng.standard_normal(shape) * s


def test_hand_example():
    d = json.load(open(os.path.join(GOLDEN, "gated_lora_hand.json")))
    y = oracle.gated_lora(np.array(d["x"], float), np.array(d["w0"], float), np.array(d["a"], float),
                          np.array(d["b"], float), np.array(d["gate"], float), d["scale"])
    np.testing.assert_array_equal(y, np.array(d["y"], float))


def test_ungated_rows_are_the_base_layer():
    rng = np.random.default_rng(0)
    M, din, dout, r = 9, 40, 24, 5
    x, w0 = _rand((M, din), rng), _rand((dout, din), rng, 0.1)
    a, b = _rand((r, din), rng, 0.1), _rand((dout, r), rng, 0.1)
    base = np.matmul(x, w0.T)  # library routine
    for y in (oracle.gated_lora(x, w0, a, b, np.zeros(M), 2.0),
              oracle.gated_lora(x, w0, a, b, None, 2.0),
              oracle.gated_lora(x, w0, a, np.zeros_like(b), np.ones(M), 2.0),
              oracle.gated_lora(x, w0, a, b, np.ones(M), 0.0)):
        np.testing.assert_allclose(y, base, rtol=1e-13, atol=1e-13)


def test_linear_in_gate_and_scale():
    rng = np.random.default_rng(1)
    M, din, dout, r = 7, 32, 16, 4
    x, w0 = _rand((M, din), rng), _rand((dout, din), rng, 0.1)
    a, b = _rand((r, din), rng, 0.1), _rand((dout, r), rng, 0.1)
    y0 = oracle.gated_lora(x, w0, a, b, np.zeros(M), 1.0)
    y1 = oracle.gated_lora(x, w0, a, b, np.ones(M), 1.0)
    g = rng.standard_normal(M)
    yg = oracle.gated_lora(x, w0, a, b, g, 3.0)
    np.testing.assert_allclose(yg, y0 + 3.0 * g[:, None] * (y1 - y0), rtol=1e-11, atol=1e-12)


def test_adapter_term_is_rank_r_in_row_space():
    """(y(g=1) - y(g=0)) = (x A^T) B^T has rank <= r and lies in the span of B's columns."""
    rng = np.random.default_rng(2)
    M, din, dout, r = 12, 20, 18, 3
    x, w0 = _rand((M, din), rng), _rand((dout, din), rng)
    a, b = _rand((r, din), rng), _rand((dout, r), rng)
    delta = oracle.gated_lora(x, w0, a, b, np.ones(M), 1.0) - oracle.gated_lora(x, w0, a, b, np.zeros(M), 1.0)
    sv = np.linalg.svd(delta, compute_uv=False)
    assert sv[r] < 1e-10 * sv[0]
    coef, res, *_ = np.linalg.lstsq(b, delta.T, rcond=None)  # library least squares
    np.testing.assert_allclose(b @ coef, delta.T, atol=1e-10)


def test_brute_force_elements():
    rng = np.random.default_rng(3)
    M, din, dout, r = 4, 6, 5, 2
    x, w0 = _rand((M, din), rng), _rand((dout, din), rng)
    a, b = _rand((r, din), rng), _rand((dout, r), rng)
    g = np.array([0.0, 1.0, 1.0, 0.5])
    y = oracle.gated_lora(x, w0, a, b, g, 1.5)
    for m in range(M):
        for o in range(dout):
            acc = 0.0
            for k in range(din):
                acc += x[m, k] * w0[o, k]
            for j in range(r):
                t = 0.0
                for k in range(din):
                    t += x[m, k] * a[j, k]
                acc += 1.5 * g[m] * t * b[o, j]
            assert abs(acc - y[m, o]) < 1e-12


def test_single_row_selection_matches_full():
    """Oracle rows are independent: evaluating a subset of rows gives the same values."""
    rng = np.random.default_rng(4)
    M, din, dout, r = 10, 16, 8, 2
    x, w0 = _rand((M, din), rng), _rand((dout, din), rng)
    a, b = _rand((r, din), rng), _rand((dout, r), rng)
    g = rng.random(M)
    full = oracle.gated_lora(x, w0, a, b, g, 2.0)
    rows = np.array([7, 2, 9])
    part = oracle.gated_lora(x[rows], w0, a, b, g[rows], 2.0)
    np.testing.assert_array_equal(part, full[rows])
