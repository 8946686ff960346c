"""The seeded input generator: dtype rounding, determinism, and per-row regeneration."""
import numpy as np

from diffusion_drafted_lossless_b200 import workloads as W


def test_bf16_round_to_nearest_even():
    f = np.array([1.0, -2.0, 1.00390625, 1.01171875, 1.0 + 2 ** -8 + 2 ** -20, 3.140625, 0.0, -0.0],
                 dtype=np.float32)
    # 1 + 2^-8 is a tie between 1.0 and 1.0078125 -> even (1.0); 1 + 3*2^-8 ties up to 1.015625
    expect = np.array([0x3F80, 0xC000, 0x3F80, 0x3F82, 0x3F81, 0x4049, 0x0000, 0x8000], dtype=np.uint16)
    np.testing.assert_array_equal(W.bf16_bits(f), expect)
    np.testing.assert_array_equal(W.bf16_to_f32(expect)[:2], f[:2])


def test_bf16_matches_torch_rounding():
    import torch
    x = np.random.default_rng(0).standard_normal(100000).astype(np.float32) * 7
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(W.bf16_bits(x), ref)


def test_rows_regenerate_independently():
    full = W.normal_rows(5, 7, 200, 33, 3.0)
    rows = np.array([199, 0, 64, 65, 127, 3])
    np.testing.assert_array_equal(W.normal_rows(5, 7, 200, 33, 3.0, rows), full[rows])
    assert abs(full.std() - 3.0) < 0.1


def test_verify_rows_and_correlation():
    w = W.VerifyWorkload("t", 9, B=4, K=8, V=4096, sigma=3.0, rho=0.8, temperature=1.0, top_k=50, top_p=0.95)
    p, q = W.verify_logits(w)
    assert p.shape == (32, 4096) and p.dtype == np.uint16
    pf, qf = W.bf16_to_f32(p), W.bf16_to_f32(q)
    assert abs(np.corrcoef(pf.ravel(), qf.ravel())[0, 1] - 0.8) < 0.01
    assert abs(qf.std() - 3.0) < 0.05
    rows = np.array([31, 5])
    p2, q2 = W.verify_logits(w, rows)
    np.testing.assert_array_equal(p2, p[rows])
    np.testing.assert_array_equal(q2, q[rows])
    u = W.verify_uniforms(w)
    assert u.shape == (4, 8, 3) and (u >= 0).all() and (u < 1).all()


def test_gate_pattern():
    g = W.row_gate(32, 16)
    assert g[0] == 0 and g[16] == 0 and g[1:16].all() and g.sum() == 30


def test_linear_inputs_shapes():
    x = W.linear_inputs(W.TINY_LINEAR, W.TINY_LINEAR.shapes[0])
    assert x["x"].shape == (16, 256) and x["x"].dtype == np.float32
    assert x["a"].shape == (8, 256) and x["b"].shape == (256, 8)
    assert abs(x["w0"].std() - 0.02) < 0.002
