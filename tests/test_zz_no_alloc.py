"""uno_block_verify_noalloc: the block verify for callers that cannot allocate device
memory (for instance a plugin that only receives device pointers and a stream from its host
application, or a serving loop that may not call cudaMalloc). It runs on a fixed scratch
array inside the library and must give exactly what uno_block_verify gives with a
caller-supplied workspace. This file is collected last; its tests pass alone in a fresh
process and after the rest of the suite."""
import ctypes

import numpy as np
import pytest
import torch

from diffusion_drafted_lossless_b200 import _lib
from diffusion_drafted_lossless_b200 import workloads as W
from tests.gpu_util import PROB_TOL, dev

pytestmark = pytest.mark.gpu


def _outs(B, K):
    return [torch.full((B, K), -9, dtype=torch.int32, device="cuda"),
            torch.full((B,), -9, dtype=torch.int32, device="cuda"),
            torch.full((B,), -9, dtype=torch.int32, device="cuda"),
            torch.full((B, K), -1.0, device="cuda"), torch.full((B, K), -1.0, device="cuda"),
            torch.full((B, K), -1.0, device="cuda")]


def _host(outs):
    torch.cuda.synchronize()
    return [o.cpu().numpy() for o in outs]


def _batch(top_k, top_p, seed):
    w = W.VerifyWorkload("noalloc", seed, B=64, K=16, V=151936, sigma=3.0, rho=0.8, temperature=1.0,
                         top_k=top_k, top_p=top_p)
    P, Q = W.verify_logits(w)
    u = W.verify_uniforms(w)
    return (dev(P, "bf16").view(64, 16, -1), dev(Q, "bf16").view(64, 16, -1), 1.0, top_k, top_p,
            torch.from_numpy(u).cuda())


def test_noalloc_matches_workspace_entry_point():
    # two batches that use the shared array differently: the top-k path (top-k 50) and the
    # full-vocabulary path (top-k off), with different logits and uniforms
    batches = [_batch(50, 0.95, 4292), _batch(0, 0.95, 4242)]
    refs = []
    for args in batches:
        ref = _outs(64, 16)
        _lib.uno_block_verify(*args, *ref)
        refs.append(_host(ref))
    # the no-alloc calls alternate between the batches, so each call finds the array as the
    # other batch left it; every call must still give the workspace entry point's results
    for call, which in enumerate((0, 0, 1, 0, 1, 1)):
        got = _outs(64, 16)
        _lib.uno_block_verify_noalloc(*batches[which], *got)
        got = _host(got)
        for a, b in zip(got[:3], refs[which][:3]):
            np.testing.assert_array_equal(a, b, err_msg=f"call {call}")
        for a, b in zip(got[3:], refs[which][3:]):
            np.testing.assert_allclose(a, b, atol=PROB_TOL, rtol=0, err_msg=f"call {call}")
    assert _lib.uno_read_device_status() == 0


def test_noalloc_rejects_batches_beyond_the_array():
    lib = _lib.load()
    need = lib.uno_block_verify_workspace_size(1024, 16, 151936, 50, 0.95, 0)
    assert need > (16 << 20)
    fake = ctypes.c_void_p(0x7F0000000000)  # never dereferenced: the size check comes first
    st = lib.uno_block_verify_noalloc(fake, fake, 0, 1024, 16, 151936, 1.0, 50, 0.95, None, None, fake, fake, fake,
                                      None, None, None, None, None)
    assert st == _lib.UNO_ERR_UNSUPPORTED
    assert b"scratch" in lib.uno_last_error_string()
