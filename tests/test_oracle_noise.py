"""Pins of the block-noising oracle (noise mode random_uniform): values worked by hand
from the definition, the special cases of the uniform, the gate pattern, and a chi-square
test that the noised tokens are uniform over the vocabulary.

LoopUno project page, "Training is self-distillation" (the student reads a block-noised
copy); uno-qwen3-8B model card, "Evaluation protocol" (noise mode random_uniform)."""
import numpy as np
from scipy import stats

import oracle


def test_hand_example():
    # out[b,0] = clean[b,0]; out[b,i] = floor(u * V) for i >= 1, V = 10, u the float32
    # value: float32(0.7) = 0.699999988..., so 10 u = 6.99999988 gives 6
    clean = np.array([[7, 1, 2, 3], [9, 9, 9, 9]], np.int32)
    u = np.array([[0.99, 0.0, 0.05, 0.5], [0.0, 0.123, 0.9999, 0.7]], np.float32)
    r = oracle.block_noise(clean, u, 10)
    assert r["tokens"].tolist() == [[7, 0, 0, 5], [9, 1, 9, 6]]
    assert r["gate"].tolist() == [0, 1, 1, 1, 0, 1, 1, 1]


def test_extremes_of_the_uniform():
    V = 151936
    below_one = np.nextafter(np.float32(1), np.float32(0))
    clean = np.zeros((1, 4), np.int32)
    # u = 1 (outside [0, 1), which some generators produce) is clamped to the last token
    r = oracle.block_noise(clean, np.array([[0.5, 0.0, below_one, 1.0]], np.float32), V)
    assert r["tokens"][0, 1] == 0 and r["tokens"][0, 2] == V - 1 and r["tokens"][0, 3] == V - 1


def test_block_of_one_keeps_the_block():
    clean = np.array([[5], [6]], np.int32)
    r = oracle.block_noise(clean, np.array([[0.3], [0.9]], np.float32), 100)
    assert r["tokens"].tolist() == [[5], [6]] and r["gate"].tolist() == [0, 0]


def test_noised_tokens_are_uniform():
    V, B, K = 16, 4000, 16
    rng = np.random.default_rng(5)
    u = rng.random((B, K), dtype=np.float32)
    r = oracle.block_noise(np.zeros((B, K), np.int32), u, V)
    counts = np.bincount(r["tokens"][:, 1:].ravel(), minlength=V)
    assert counts.sum() == B * (K - 1)
    assert stats.chisquare(counts).pvalue > 1e-4
    # and each noised token is the one its uniform selects
    assert (r["tokens"][:, 1:] == np.floor(u[:, 1:].astype(np.float64) * V).astype(np.int32)).all()
