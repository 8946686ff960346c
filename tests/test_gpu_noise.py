"""GPU parity of uno_block_noise (noise mode random_uniform) against the oracle: bit-exact
tokens and gates, with the uniform's extremes, in place, and the degenerate shapes."""
import numpy as np
import pytest
import torch

import oracle
from diffusion_drafted_lossless_b200 import _lib
from diffusion_drafted_lossless_b200 import workloads as W

pytestmark = pytest.mark.gpu


def _inputs(B, K, V, seed):
    rng = np.random.default_rng(seed)
    clean = rng.integers(0, V, size=(B, K), dtype=np.int32)
    u = W.uniforms(seed, (B, K))
    below_one = np.nextafter(np.float32(1), np.float32(0))
    flat = u.reshape(-1)
    flat[: min(8, flat.size)] = np.array([0.0, below_one, 1.0, 0.5, 0.25, 1.0 / 3, 0.7, 1e-30],
                                         np.float32)[: min(8, flat.size)]
    return clean, u


@pytest.mark.parametrize("B,K,V", [(64, 16, 151936), (256, 8, 166144), (3, 1, 10), (5, 7, 1), (1, 33, 16777215)])
def test_noise_parity(B, K, V):
    clean, u = _inputs(B, K, V, 17 + B + K)
    ref = oracle.block_noise(clean, u, V)
    c, ud = torch.from_numpy(clean).cuda(), torch.from_numpy(np.ascontiguousarray(u)).cuda()
    out = torch.full((B, K), -7, dtype=torch.int32, device="cuda")
    gate = torch.full((B * K,), -1.0, device="cuda")
    _lib.uno_block_noise(c, ud, V, out, gate)
    torch.cuda.synchronize()
    assert (out.cpu().numpy() == ref["tokens"]).all()
    assert (gate.cpu().numpy() == ref["gate"]).all()


def test_noise_in_place_and_without_gate():
    B, K, V = 64, 16, 151936
    clean, u = _inputs(B, K, V, 3)
    ref = oracle.block_noise(clean, u, V)
    c = torch.from_numpy(clean).cuda()
    _lib.uno_block_noise(c, torch.from_numpy(np.ascontiguousarray(u)).cuda(), V, c)
    torch.cuda.synchronize()
    assert (c.cpu().numpy() == ref["tokens"]).all()


def test_noise_empty_batch():
    e = torch.empty((0, 16), dtype=torch.int32, device="cuda")
    _lib.uno_block_noise(e, torch.empty((0, 16), device="cuda"), 100, e)
    torch.cuda.synchronize()
