"""GPU parity of uno_tv_loss against the fp64 oracle (through the C ABI): per-token TV,
the masked mean and the bf16 gradient, at small ragged sizes, with masks, fp32 inputs,
and at the full 16384 x 151936 workload on sampled rows."""
import numpy as np
import pytest
import torch

import oracle
from diffusion_drafted_lossless_b200 import _lib
from diffusion_drafted_lossless_b200 import workloads as W
from tests.gpu_util import PROB_TOL, bf16_ulp, dev

pytestmark = pytest.mark.gpu


def _psum(Tf, Sf):
    """p + q per element (scale for the sign-decision band)."""
    from scipy.special import softmax
    return softmax(Tf, axis=1) + softmax(Sf, axis=1)


def _run(T, S, dtype, mask=None, grad_scale=1.0, want_grad=True):
    N, V = T.shape
    td, sd = dev(T, dtype), dev(S, dtype)
    tv = torch.full((N,), -1.0, device="cuda")
    mean = torch.full((1,), -1.0, device="cuda")
    g = torch.empty((N, V), dtype=td.dtype, device="cuda") if want_grad else None
    md = None if mask is None else torch.from_numpy(mask.astype(np.uint8)).cuda()
    _lib.uno_tv_loss(td, sd, tv, mean, g, md, grad_scale)
    torch.cuda.synchronize()
    gg = None if g is None else g.float().cpu().numpy()
    return tv.cpu().numpy(), float(mean.cpu()[0]), gg


def _compare_grad(g_gpu, ref_grad, absdiff, psum):
    """Within one bf16 ulp of the fp64 gradient. Mismatches are excused only where
    sign(q - p) is not decided at fp32 resolution (|p - q| <= 1e-6 (p + q)); those are
    counted and must stay below 0.1% of the elements."""
    undecided = absdiff <= 1e-6 * psum
    err = np.abs(g_gpu.astype(np.float64) - ref_grad)
    ok = err <= bf16_ulp(ref_grad) + 1e-38
    bad = ~ok & ~undecided
    assert not bad.any(), (np.argwhere(bad)[:5], err[bad][:5], ref_grad[bad][:5])
    assert (~ok & undecided).mean() < 1e-3


# bf16 rows whose length is a multiple of 8 run on the cluster kernel (on B200: cluster size 1
# for V = 1000 and 12000, 2 for 20000, 4 for 40000, 8 for 151936 and 16 for 166144); the
# others on the per-row kernel
@pytest.mark.parametrize("N,V,dtype", [(7, 1000, "bf16"), (5, 4099, "bf16"), (3, 20000, "f32"), (4, 777, "f32"),
                                       (2, 1, "bf16"), (9, 151936, "bf16"), (5, 20000, "bf16"),
                                       (5, 12000, "bf16"), (3, 40000, "bf16"), (4, 166144, "bf16"), (600, 2048, "bf16"),
                                       (1, 8, "bf16")])
def test_tv_parity(N, V, dtype):
    w = W.TVWorkload("t", 40 + N + V, N=N, V=V)
    T, S = W.tv_logits(w)
    if dtype == "f32":
        T, S = W.bf16_to_f32(T), W.bf16_to_f32(S)
    mask = np.ones(N, bool)
    mask[1::3] = False
    tv, mean, g = _run(T, S, dtype, mask=mask, grad_scale=1.5)
    Tf, Sf = W.to_f64(T, dtype), W.to_f64(S, dtype)
    ref = oracle.tv_loss(Tf, Sf, mask=mask, grad_scale=np.float32(1.5), want_absdiff=True)
    np.testing.assert_allclose(tv, ref["tv"], atol=PROB_TOL, rtol=0)
    assert abs(mean - ref["mean"]) <= PROB_TOL
    _compare_grad(g, ref["grad"], ref["absdiff"], _psum(Tf, Sf))


@pytest.mark.parametrize("env,N,V", [
    ({"UNO_TV_CLUSTER": "16"}, 5, 151936),   # a larger cluster than needed
    ({"UNO_TV_CLUSTER": "16"}, 3, 64),       # half of the CTAs hold an empty slice
    ({"UNO_TV_CLUSTER": "16"}, 4, 1000),     # ragged last slice
    ({"UNO_TV_CLUSTER": "2"}, 300, 151936),  # does not fit: falls back to the chosen size
    ({"UNO_TV_CLUSTER": "6", "UNO_TV_KEEP": "0"}, 50, 151936),  # exp(student) recomputed
    ({"UNO_TV_CLUSTER": "8", "UNO_TV_KEEP": "1"}, 40, 151936),  # exp(student) kept
    ({"UNO_TV_KEEP": "1"}, 7, 5000),
    ({"UNO_TV_CLUSTER": "3", "UNO_TV_KEEP": "0"}, 9, 4000),      # ragged slices at a size of 3
    ({"UNO_TV_KERNEL": "rows"}, 6, 151936),  # the per-row kernel on bf16 rows
    ({"UNO_TV_KERNEL": "teams"}, 37, 151936),  # the two-team kernel: many rows per team
    ({"UNO_TV_KERNEL": "teams"}, 5, 1000),
    ({"UNO_TV_KERNEL": "teams", "UNO_TV_CLUSTER": "16"}, 9, 4000),  # CTAs with empty slices
    ({"UNO_TV_KERNEL": "teams"}, 3, 166144),
    ({"UNO_TV_KERNEL": "teams", "UNO_TV_KEEP": "0"}, 37, 151936),  # exp(student) recomputed
    ({"UNO_TV_KERNEL": "teams", "UNO_TV_KEEP": "0"}, 5, 1000),
    ({"UNO_TV_KERNEL": "teams", "UNO_TV_CLUSTER": "8"}, 11, 151936),  # keep does not fit at 8
])
def test_tv_kernel_variants(monkeypatch, env, N, V):
    """Every kernel variant and cluster size gives the oracle's result."""
    for k, v in env.items():
        monkeypatch.setenv(k, v)
    w = W.TVWorkload("t", 7 + N + V, N=N, V=V)
    T, S = W.tv_logits(w)
    mask = np.ones(N, bool)
    mask[::4] = False
    tv, mean, g = _run(T, S, "bf16", mask=mask, grad_scale=0.75)
    Tf, Sf = W.to_f64(T, "bf16"), W.to_f64(S, "bf16")
    ref = oracle.tv_loss(Tf, Sf, mask=mask, grad_scale=np.float32(0.75), want_absdiff=True)
    np.testing.assert_allclose(tv, ref["tv"], atol=PROB_TOL, rtol=0)
    assert abs(mean - ref["mean"]) <= PROB_TOL
    _compare_grad(g, ref["grad"], ref["absdiff"], _psum(Tf, Sf))


def test_tv_identical_rows_zero_gradient():
    """p == q: TV 0 and a gradient of exactly 0 (sign(q - p) = 0 everywhere), on both kernels."""
    T, _ = W.tv_logits(W.TVWorkload("t", 43, N=5, V=151936))
    tv, mean, g = _run(T, T, "bf16")
    assert np.abs(tv).max() == 0.0 and mean == 0.0 and (g == 0).all()
    T, _ = W.tv_logits(W.TVWorkload("t", 44, N=3, V=4099))
    tv, mean, g = _run(T, T, "bf16")
    assert np.abs(tv).max() == 0.0 and mean == 0.0 and (g == 0).all()


def test_tv_identical_and_no_grad():
    T, _ = W.tv_logits(W.TVWorkload("t", 41, N=3, V=5000))
    tv, mean, g = _run(T, T, "bf16", want_grad=False)
    assert np.abs(tv).max() < 1e-6 and abs(mean) < 1e-6 and g is None


def test_tv_empty_mask_and_empty_batch():
    T, S = W.tv_logits(W.TVWorkload("t", 42, N=4, V=3000))
    tv, mean, g = _run(T, S, "bf16", mask=np.zeros(4, bool))
    assert mean == 0.0 and (g == 0).all() and (tv > 0).all()
    e = torch.empty((0, 10), dtype=torch.bfloat16, device="cuda")
    out_tv = torch.empty((0,), device="cuda")
    mean_t = torch.full((1,), 5.0, device="cuda")
    _lib.uno_tv_loss(e, e, out_tv, mean_t)
    torch.cuda.synchronize()
    assert float(mean_t.cpu()[0]) == 0.0


def test_tv_full_size_rows_and_mean():
    """N = 16384 tokens, V = 151936, bf16: the whole batch runs on the GPU. The oracle
    recomputes the TV of every row (in blocks of rows, without the gradient) and so the mean,
    and the gradient of 284 rows spread over the batch (every 59th row and a few edges: every
    residue of the row index modulo any count of co-resident clusters below 59 is among them,
    so every cluster's share is checked)."""
    w = W.TV_LOSS
    T, S = W.tv_logits(w)
    tv, mean, g = _run(T, S, "bf16")
    ref_tv = np.empty(w.N)
    for r0 in range(0, w.N, 1024):
        Tf, Sf = W.to_f64(T[r0:r0 + 1024], "bf16"), W.to_f64(S[r0:r0 + 1024], "bf16")
        ref_tv[r0:r0 + 1024] = oracle.tv_loss(Tf, Sf, want_grad=False)["tv"]
    np.testing.assert_allclose(tv, ref_tv, atol=PROB_TOL, rtol=0)
    assert abs(mean - ref_tv.mean()) <= PROB_TOL
    rows = np.unique(np.concatenate([np.arange(0, w.N, 59), [1, 4095, 4096, 8191, 16382, 16383]]))
    assert len(rows) >= 256
    Tf, Sf = W.to_f64(T[rows], "bf16"), W.to_f64(S[rows], "bf16")
    ref = oracle.tv_loss(Tf, Sf, want_absdiff=True)
    # the oracle's per-row gradient carries 1/N_mask = 1/len(rows); the batch's is 1/N
    _compare_grad(g[rows], ref["grad"] * len(rows) / w.N, ref["absdiff"], _psum(Tf, Sf))
