"""GPU parity of uno_block_verify against the fp64 oracle (called through the C ABI).

Sizes span several 256-element tiles with ragged tails (V not a multiple of the tile, and
V not a multiple of the 16-byte vector so that rows are misaligned), every top-k capacity
class, both dtypes, heavy ties, adversarial orderings, supplied drafts / position-0
tokens, K = 1 and K = 32, and the serving-scale workload (B=64, K=16, V=151936) checked on
sampled sequences.
"""
import zlib

import numpy as np
import pytest
import torch

import oracle
from diffusion_drafted_lossless_b200 import workloads as W
from tests.gpu_util import NEAR_FP64, compare_verify, f32, verify_gpu

pytestmark = pytest.mark.gpu


def _inputs(B, K, V, dtype, seed, sigma=3.0, rho=0.8):
    w = W.VerifyWorkload("t", seed, B=B, K=K, V=V, sigma=sigma, rho=rho, temperature=1.0, top_k=0, top_p=1.0,
                         dtype=dtype)
    P, Q = W.verify_logits(w)
    return P.reshape(B, K, V), Q.reshape(B, K, V), W.verify_uniforms(w)


def _oracle(P, Q, u, T, top_k, top_p, dtype, drafts=None, pos0=None):
    return oracle.block_verify(W.to_f64(P, dtype), W.to_f64(Q, dtype), u.astype(np.float64), f32(T), top_k,
                               f32(top_p) if top_p < 1 else 1.0, drafts=drafts, pos0=pos0)


def _check(P, Q, u, T, top_k, top_p, dtype, drafts=None, pos0=None):
    """Both paths take the top-p cut, the draws and the acceptance test in fp64, as the oracle
    does: a difference is excused only where a decision before it lies within NEAR_FP64 of its
    threshold, and such decisions must stay below 0.1% of all."""
    gpu = verify_gpu(P, Q, u, T, top_k, top_p, dtype, drafts=drafts, pos0=pos0)
    ref = _oracle(P, Q, u, T, top_k, top_p, dtype, drafts, pos0)
    cmp = compare_verify(gpu, ref, band=NEAR_FP64).check()
    assert (gpu["count"] >= 1).all()
    return gpu, ref, cmp


CASES = [
    ("bf16", 3, 5, 3000, 1.0, 50, 0.95),
    ("bf16", 4, 8, 20000, 0.7, 1, 1.0),
    ("bf16", 2, 16, 4099, 1.3, 64, 0.5),
    ("bf16", 3, 4, 5000, 1.0, 100, 0.9),
    ("bf16", 2, 3, 9000, 1.0, 700, 0.99),
    ("f32", 3, 6, 2500, 1.0, 50, 0.95),
    ("f32", 2, 5, 777, 2.0, 20, 1.0),
    ("bf16", 5, 32, 1200, 1.0, 5, 0.8),
    ("bf16", 3, 1, 500, 1.0, 10, 0.9),
    ("bf16", 6, 16, 151936, 1.0, 50, 0.95),
]


@pytest.mark.parametrize("case", CASES, ids=[f"{c[0]}-B{c[1]}K{c[2]}V{c[3]}k{c[5]}" for c in CASES])
def test_topk_parity(case):
    dtype, B, K, V, T, k, p = case
    P, Q, u = _inputs(B, K, V, dtype, seed=zlib.crc32(str(case).encode()) % 10007)
    gpu, ref, cmp = _check(P, Q, u, T, k, p, dtype)
    assert cmp.excused == 0


def test_heavy_ties():
    B, K, V = 4, 6, 6000
    rng = np.random.default_rng(31)
    Pf = np.round(rng.standard_normal((B, K, V)) * 2) / 2  # values on a 0.5 grid: many ties
    Qf = np.round((0.7 * Pf + 0.7 * rng.standard_normal((B, K, V))) * 2) / 2
    P, Q = W.bf16_bits(Pf.astype(np.float32)), W.bf16_bits(Qf.astype(np.float32))
    u = rng.random((B, K, 3), dtype=np.float32)
    for k in (1, 7, 50, 200):
        _check(P, Q, u, 1.0, k, 0.9, "bf16")


@pytest.mark.parametrize("order", ["ascending", "descending", "constant", "one_hot"])
def test_adversarial_orders(order):
    B, K, V = 2, 4, 5000
    base = np.linspace(-5, 5, V, dtype=np.float32)
    if order == "descending":
        base = base[::-1].copy()
    elif order == "constant":
        base = np.zeros(V, np.float32)
    elif order == "one_hot":
        base = np.full(V, -3.0, np.float32)
        base[V // 2] = 4.0
    P = np.broadcast_to(W.bf16_bits(base), (B, K, V)).copy()
    Q = np.broadcast_to(W.bf16_bits(base[::-1].copy()), (B, K, V)).copy()
    u = np.random.default_rng(32).random((B, K, 3), dtype=np.float32)
    for k in (1, 50, 64, 300):
        _check(P, Q, u, 1.0, k, 0.95, "bf16")


def test_identical_rows_accept_all():
    P, _, u = _inputs(4, 8, 10000, "bf16", seed=33)
    gpu, ref, _ = _check(P, P, u, 1.0, 50, 0.95, "bf16")
    assert (gpu["count"] == 8).all() and (gpu["next"] == -1).all()
    np.testing.assert_allclose(gpu["tv"], 0.0, atol=1e-6)


def test_supplied_drafts_and_pos0():
    B, K, V = 5, 6, 3000
    P, Q, u = _inputs(B, K, V, "bf16", seed=34)
    rng = np.random.default_rng(34)
    drafts = rng.integers(0, V, (B, K)).astype(np.int32)
    # make some drafts the verifier's argmax so that acceptances happen
    drafts[:, 1:3] = W.bf16_to_f32(P).reshape(B, K, V)[:, 1:3].argmax(axis=2)
    pos0 = rng.integers(0, V, B).astype(np.int32)
    gpu, ref, _ = _check(P, Q, u, 1.0, 50, 0.95, "bf16", drafts=drafts, pos0=pos0)
    assert (gpu["tokens"][:, 0] == pos0).all()


def test_empty_batch():
    from diffusion_drafted_lossless_b200 import _lib
    z = torch.empty((0, 4, 100), dtype=torch.bfloat16, device="cuda")
    u = torch.empty((0, 4, 3), device="cuda")
    t = torch.empty((0, 4), dtype=torch.int32, device="cuda")
    c = torch.empty((0,), dtype=torch.int32, device="cuda")
    _lib.uno_block_verify(z, z, 1.0, 50, 0.95, u, t, c)
    torch.cuda.synchronize()


def test_repeated_calls_reuse_workspace():
    """Counters in the workspace are reset by each call: two calls give the same result."""
    from diffusion_drafted_lossless_b200 import _lib
    B, K, V = 3, 5, 7000
    P, Q, u = _inputs(B, K, V, "bf16", seed=35)
    ws = torch.empty(_lib.uno_block_verify_workspace_size(B, K, V, 50, 0.95), dtype=torch.uint8, device="cuda")
    outs = []
    for _ in range(3):
        from tests.gpu_util import dev
        t = torch.empty((B, K), dtype=torch.int32, device="cuda")
        c = torch.empty((B,), dtype=torch.int32, device="cuda")
        nx = torch.empty((B,), dtype=torch.int32, device="cuda")
        _lib.uno_block_verify(dev(P, "bf16"), dev(Q, "bf16"), 1.0, 50, 0.95, torch.from_numpy(u).cuda(), t, c,
                              nx, workspace=ws)
        torch.cuda.synchronize()
        outs.append((t.cpu().numpy(), c.cpu().numpy(), nx.cpu().numpy()))
    for o in outs[1:]:
        for a, b in zip(o, outs[0]):
            np.testing.assert_array_equal(a, b)


def test_serving_scale_all_sequences():
    """B=64, K=16, V=151936 bf16, T=1, top-k 50, top-p 0.95 (the serving workload): the full
    batch on the GPU, every sequence recomputed by the oracle and compared."""
    w = W.SERVING_VERIFY
    P, Q = W.verify_logits(w)
    u = W.verify_uniforms(w)
    B, K, V = w.B, w.K, w.V
    gpu = verify_gpu(P.reshape(B, K, V), Q.reshape(B, K, V), u, w.temperature, w.top_k, w.top_p)
    ref = oracle.block_verify(W.to_f64(P, "bf16").reshape(B, K, V), W.to_f64(Q, "bf16").reshape(B, K, V),
                              u.astype(np.float64), f32(w.temperature), w.top_k, f32(w.top_p))
    cmp = compare_verify(gpu, ref, band=NEAR_FP64).check()
    assert cmp.n == B and cmp.excused == 0
    assert (gpu["count"] >= 1).all() and (gpu["count"] <= K).all()
    # every sequence: tokens after the count are -1, next is -1 exactly when all accepted
    for b in range(B):
        c = gpu["count"][b]
        assert (gpu["tokens"][b, c:] == -1).all() and (gpu["tokens"][b, :c] >= 0).all()
        assert (gpu["next"][b] == -1) == (c == K)


def test_threshold_guess_fallback():
    """Rows whose first loads hold a few large spikes: the streaming kernel's sampled
    threshold guess then leaves fewer than k candidates, and the row is redone exactly."""
    B, K, V = 2, 3, 200000
    rng = np.random.default_rng(36)
    base = (rng.standard_normal((B, K, V)) * 0.5).astype(np.float32)
    base[:, :, 0:96:8] = 6.0 + rng.random((B, K, 12), dtype=np.float32)  # 12 spikes, one per lane-chunk
    P = W.bf16_bits(base)
    Q = W.bf16_bits(base[:, :, ::-1].copy())
    u = rng.random((B, K, 3), dtype=np.float32)
    for k in (20, 50):
        _check(P, Q, u, 1.0, k, 0.95, "bf16")


@pytest.mark.parametrize("env", [{"UNO_VERIFY_STREAM": "warps"}, {"UNO_VERIFY_STREAM": "tma"},
                                 {"UNO_VERIFY_STREAM": "warps", "UNO_VERIFY_SEGMENTS": "3"},
                                 {"UNO_VERIFY_TOPK": "local"}],
                         ids=["stream_warps", "stream_tma", "stream_warps_s3", "cluster_local"])
def test_alternate_topk_paths_parity(env):
    """The top-k tests on the other top-k paths: the streaming kernel with one CTA per row
    segment (UNO_VERIFY_STREAM=warps, the path of fp32 and unaligned rows), its TMA-fed
    variant (UNO_VERIFY_STREAM=tma) and the cluster kernel with per-CTA lists
    (UNO_VERIFY_TOPK=local, with the streaming path for the batches it does not take); run
    in a subprocess so that the selection is clean."""
    import os
    import subprocess
    import sys
    code = ("import sys; sys.argv=['x']; import pytest; "
            "sys.exit(pytest.main(['-q', '-p', 'no:cacheprovider', '-m', 'gpu', "
            "'tests/test_gpu_verify.py::test_topk_parity', 'tests/test_gpu_verify.py::test_heavy_ties', "
            "'tests/test_gpu_verify.py::test_threshold_guess_fallback', "
            "'tests/test_gpu_verify.py::test_adversarial_orders']))")
    r = subprocess.run([sys.executable, "-c", code], env=dict(os.environ, **env), capture_output=True, text=True,
                       cwd=os.path.dirname(os.path.dirname(__file__)))
    assert r.returncode == 0, r.stdout[-3000:] + r.stderr[-2000:]


TOPK_CLUSTER_CASES = [
    (16, 16, 5000, 1.0, 50, 0.95),
    (8, 8, 12000, 0.7, 1, 1.0),       # greedy
    (4, 6, 20000, 1.3, 256, 0.5),     # the largest k of the cluster kernel
    (3, 5, 2048, 1.0, 100, 0.9),
    (6, 16, 151936, 1.0, 50, 0.95),   # the serving row length
]


@pytest.mark.parametrize("mode", ["local", "window"])
@pytest.mark.parametrize("cl", [1, 2, 4, 8, 16])
@pytest.mark.parametrize("case", TOPK_CLUSTER_CASES, ids=[f"B{c[0]}K{c[1]}V{c[2]}k{c[4]}p{c[5]}" for c in TOPK_CLUSTER_CASES])
def test_topk_cluster_kernel(case, cl, mode, monkeypatch):
    """The cluster kernels' top-k modes against the oracle, for every cluster size that fits:
    "local" (k <= 128: every CTA takes its slice's exact top-k, a head CTA merges the lists,
    selected by UNO_VERIFY_TOPK=local) and "window" (the row's k-th value from per-value counts over its 256 largest values,
    selected by UNO_VERIFY_TOPK=window; it also serves 128 < k <= 256). UNO_VERIFY_FULL=cluster
    makes any other path an error."""
    B, K, V, T, k, p = case
    from diffusion_drafted_lossless_b200._lib import UnoError
    monkeypatch.setenv("UNO_VERIFY_FULL", "cluster")
    monkeypatch.setenv("UNO_VERIFY_FULL_CLUSTER", str(cl))
    monkeypatch.setenv("UNO_VERIFY_TOPK", mode)
    P, Q, u = _inputs(B, K, V, "bf16", seed=zlib.crc32(str((case, cl)).encode()) % 10007)
    try:
        _check(P, Q, u, T, k, p, "bf16")
    except UnoError as e:  # the rows do not fit in the shared memory of this cluster size
        assert "UNSUPPORTED" in str(e) and V > 50000, e
        pytest.skip(f"V = {V} does not fit clusters of {cl}")


# ---------------------------------------------------------------------------------------
# full-vocabulary path (no top-k): the cut, the draws and the tests are decided in fp64 from
# per-value counts, so the same band as the top-k path
# ---------------------------------------------------------------------------------------
FULL_BAND = NEAR_FP64


def _check_full(P, Q, u, T, top_p, dtype, drafts=None, pos0=None):
    gpu = verify_gpu(P, Q, u, T, 0, top_p, dtype, drafts=drafts, pos0=pos0)
    ref = _oracle(P, Q, u, T, 0, top_p, dtype, drafts, pos0)
    cmp = compare_verify(gpu, ref, band=FULL_BAND).check()
    assert (gpu["count"] >= 1).all()
    return gpu, ref, cmp


def test_tiny_config_unfiltered():
    """2 sequences x block 8, V = 1000, fp32 logits ~ N(0, 2^2), T = 1, no filter."""
    w = W.TINY_VERIFY
    P, Q = W.verify_logits(w)
    u = W.verify_uniforms(w)
    _, _, cmp = _check_full(P.reshape(2, 8, 1000), Q.reshape(2, 8, 1000), u, 1.0, 1.0, "f32")
    assert cmp.excused == 0


FULL_CASES = [
    ("bf16", 3, 5, 5000, 1.0, 1.0),
    ("bf16", 3, 6, 20000, 1.0, 0.95),
    ("f32", 2, 4, 3001, 0.8, 0.9),
    ("bf16", 2, 16, 4099, 1.2, 0.5),
    ("bf16", 3, 1, 700, 1.0, 0.95),
    ("f32", 4, 3, 2048, 1.0, 1.0),
]


@pytest.mark.parametrize("case", FULL_CASES, ids=[f"{c[0]}-B{c[1]}K{c[2]}V{c[3]}p{c[5]}" for c in FULL_CASES])
def test_full_vocab_parity(case):
    dtype, B, K, V, T, p = case
    P, Q, u = _inputs(B, K, V, dtype, seed=zlib.crc32(str(case).encode()) % 10007)
    _check_full(P, Q, u, T, p, dtype)


@pytest.mark.parametrize("case", [c for c in FULL_CASES if c[0] == "bf16"],
                         ids=[f"B{c[1]}K{c[2]}V{c[3]}p{c[5]}" for c in FULL_CASES if c[0] == "bf16"])
def test_full_vocab_parity_without_lists(case, monkeypatch):
    """UNO_VERIFY_LISTS=off: the row pass records no candidate lists, so every item is weighed
    from the logits by the row-streaming item kernel instead of from its rows' lists; both
    give the oracle's results."""
    monkeypatch.setenv("UNO_VERIFY_LISTS", "off")
    dtype, B, K, V, T, p = case
    P, Q, u = _inputs(B, K, V, dtype, seed=zlib.crc32(str(case).encode()) % 10007)
    _check_full(P, Q, u, T, p, dtype)


def test_full_vocab_smallest_workspace():
    """A workspace of uno_block_verify_min_workspace_size bytes (no room for the candidate
    lists) is accepted and gives the same outputs as the full workspace; one byte less is
    rejected."""
    from diffusion_drafted_lossless_b200 import _lib
    from tests.gpu_util import dev
    B, K, V = 3, 6, 20000
    P, Q, u = _inputs(B, K, V, "bf16", seed=46)
    outs = []
    for size in (_lib.uno_block_verify_workspace_size(B, K, V, 0, 0.95),
                 _lib.uno_block_verify_min_workspace_size(B, K, V, 0, 0.95)):
        ws = torch.empty(size, dtype=torch.uint8, device="cuda")
        t = torch.empty((B, K), dtype=torch.int32, device="cuda")
        c = torch.empty((B,), dtype=torch.int32, device="cuda")
        nx = torch.empty((B,), dtype=torch.int32, device="cuda")
        pt = torch.empty((B, K), dtype=torch.float32, device="cuda")
        _lib.uno_block_verify(dev(P, "bf16"), dev(Q, "bf16"), 1.0, 0, 0.95, torch.from_numpy(u).cuda(), t, c, nx,
                              out_p_tok=pt, workspace=ws)
        torch.cuda.synchronize()
        outs.append((t.cpu().numpy(), c.cpu().numpy(), nx.cpu().numpy(), pt.cpu().numpy()))
    for a, b in zip(outs[0][:3], outs[1][:3]):
        np.testing.assert_array_equal(a, b)
    np.testing.assert_allclose(outs[0][3], outs[1][3], rtol=1e-6, atol=0)
    ws = torch.empty(_lib.uno_block_verify_min_workspace_size(B, K, V, 0, 0.95) - 256, dtype=torch.uint8,
                     device="cuda")
    t = torch.empty((B, K), dtype=torch.int32, device="cuda")
    c = torch.empty((B,), dtype=torch.int32, device="cuda")
    with pytest.raises(Exception):
        _lib.uno_block_verify(dev(P, "bf16"), dev(Q, "bf16"), 1.0, 0, 0.95, torch.from_numpy(u).cuda(), t, c,
                              workspace=ws)


def test_full_vocab_ties_and_supplied_tokens():
    B, K, V = 3, 5, 4000
    rng = np.random.default_rng(41)
    Pf = np.round(rng.standard_normal((B, K, V)) * 2) / 2
    Qf = np.round((0.7 * Pf + 0.7 * rng.standard_normal((B, K, V))) * 2) / 2
    P, Q = W.bf16_bits(Pf.astype(np.float32)), W.bf16_bits(Qf.astype(np.float32))
    u = rng.random((B, K, 3), dtype=np.float32)
    for top_p in (1.0, 0.9, 0.3):
        _check_full(P, Q, u, 1.0, top_p, "bf16")
    # every token tied: the cut keeps the lowest ids (top_p * V is kept away from an integer,
    # where the cut itself would sit on its threshold)
    const = np.zeros((B, K, V), np.float32)
    _check_full(W.bf16_bits(const), W.bf16_bits(const), u, 1.0, 0.3001, "bf16")
    drafts = rng.integers(0, V, (B, K)).astype(np.int32)
    pos0 = rng.integers(0, V, B).astype(np.int32)
    gpu, _, _ = _check_full(P, Q, u, 1.0, 0.9, "bf16", drafts=drafts, pos0=pos0)
    assert (gpu["tokens"][:, 0] == pos0).all()


CLUSTER_CASES = [
    (16, 16, 5000, 1.0, 0.95),   # clusters of 8 and 16 hold CTAs with short slices
    (16, 16, 5000, 0.8, 1.0),    # no cut: every token survives
    (4, 8, 12000, 1.2, 0.5),     # a ragged last slice at every cluster size
    (3, 5, 2048, 1.0, 0.9),
    (2, 3, 104, 1.0, 0.9),       # 13 vectors: at 16 CTAs per cluster some hold nothing
]


@pytest.mark.parametrize("cl", [1, 2, 4, 8, 16])
@pytest.mark.parametrize("case", CLUSTER_CASES, ids=[f"B{c[0]}K{c[1]}V{c[2]}T{c[3]}p{c[4]}" for c in CLUSTER_CASES])
def test_full_vocab_cluster_kernel(case, cl, monkeypatch):
    """The cluster kernel of the full-vocabulary path (an item's two rows resident in the
    shared memory of a CL-CTA cluster, two teams per CTA on alternate items, the next item's
    rows copied in while the other team computes) against the oracle, for every cluster size.
    With UNO_VERIFY_FULL=cluster a case that could not take the cluster kernel is an error,
    so these runs cannot pass on the generic kernel. B * K = 256 items for the first cases:
    many items per team, so every barrier's phase wraps many times."""
    monkeypatch.setenv("UNO_VERIFY_FULL", "cluster")
    monkeypatch.setenv("UNO_VERIFY_FULL_CLUSTER", str(cl))
    B, K, V, T, p = case
    P, Q, u = _inputs(B, K, V, "bf16", seed=zlib.crc32(str((case, cl)).encode()) % 10007)
    _check_full(P, Q, u, T, p, "bf16")


def test_full_vocab_cluster_ties_and_repeatability(monkeypatch):
    """Heavy ties at the top-p cut (logits on a 1/2 grid: thousands of tokens share the cut
    value, so the kept ties end inside one CTA's slice) through the cluster kernel, and the
    same call twice gives identical outputs (every CTA of a cluster combines the same
    partials in the same order)."""
    monkeypatch.setenv("UNO_VERIFY_FULL", "cluster")
    monkeypatch.setenv("UNO_VERIFY_FULL_CLUSTER", "4")
    B, K, V = 6, 7, 12000
    rng = np.random.default_rng(43)
    Pf = np.round(rng.standard_normal((B, K, V)) * 2) / 2
    Qf = np.round((0.7 * Pf + 0.7 * rng.standard_normal((B, K, V))) * 2) / 2
    P, Q = W.bf16_bits(Pf.astype(np.float32)), W.bf16_bits(Qf.astype(np.float32))
    u = rng.random((B, K, 3), dtype=np.float32)
    for top_p in (0.9, 0.3):
        a, _, _ = _check_full(P, Q, u, 1.0, top_p, "bf16")
        b = verify_gpu(P, Q, u, 1.0, 0, top_p, "bf16")
        for k in ("tokens", "count", "next", "p_tok", "q_tok", "tv"):
            assert (a[k] == b[k]).all(), k


def test_full_vocab_generic_kernel_matches(monkeypatch):
    """UNO_VERIFY_FULL=generic sends every item to the generic kernel (the path of fp32 and
    unaligned rows, and of items the cluster kernel leaves to it); on bf16 rows it gives the
    oracle's results as well."""
    monkeypatch.setenv("UNO_VERIFY_FULL", "generic")
    P, Q, u = _inputs(3, 6, 20000, "bf16", seed=44)
    _check_full(P, Q, u, 1.0, 0.95, "bf16")


def test_full_vocab_tiny_magnitudes_go_to_the_generic_kernel():
    """Rows whose largest magnitude is far above the values near the cut: the counted band
    (2048 bf16 steps below the largest magnitude) then misses the tokens where the cut falls,
    so the cluster kernel hands the items to the generic kernel, whose result must still be
    the oracle's."""
    B, K, V = 2, 4, 8000
    rng = np.random.default_rng(45)
    base = (rng.standard_normal((B, K, V)) * 1e-3).astype(np.float32)
    base[:, :, 7] = -3.0e5  # one huge negative magnitude widens nothing above the cut
    P = W.bf16_bits(base)
    Q = W.bf16_bits((base * 0.9 + rng.standard_normal((B, K, V)).astype(np.float32) * 1e-3).astype(np.float32))
    u = rng.random((B, K, 3), dtype=np.float32)
    _check_full(P, Q, u, 1.0, 0.9, "bf16")


def test_full_vocab_cluster_required_rejects_unaligned(monkeypatch):
    """V not a multiple of 8 cannot take the cluster kernel: with UNO_VERIFY_FULL=cluster the
    call fails with UNO_ERR_UNSUPPORTED (no kernel runs); by default it takes the generic
    kernel."""
    from diffusion_drafted_lossless_b200._lib import UnoError
    B, K, V = 2, 3, 4099
    P, Q, u = _inputs(B, K, V, "bf16", seed=5)
    monkeypatch.setenv("UNO_VERIFY_FULL", "cluster")
    with pytest.raises(UnoError, match="UNSUPPORTED"):
        verify_gpu(P, Q, u, 1.0, 0, 0.9, "bf16")
    monkeypatch.delenv("UNO_VERIFY_FULL")
    _check_full(P, Q, u, 1.0, 0.9, "bf16")


def test_looped_verify_sampled_sequences():
    """B=256, K=8, V=166144 bf16, T=1, top-p 0.95, no top-k (the looped-3B step's verify):
    the whole batch on the GPU; 64 sequences spread over the batch recomputed by the oracle
    and compared output by output. The top-p cut over 166144 tokens sits next to tokens of
    probability ~4e-6, so nearly every cut is within 1e-5 of top_p: it is decided exactly
    here, and only decisions within 1e-9 of their threshold may be excused (below 0.1%)."""
    w = W.LOOPED_VERIFY
    P, Q = W.verify_logits(w)
    u = W.verify_uniforms(w)
    B, K, V = w.B, w.K, w.V
    gpu = verify_gpu(P.reshape(B, K, V), Q.reshape(B, K, V), u, w.temperature, 0, w.top_p)
    seqs = list(range(0, B, 4))
    rows = np.concatenate([np.arange(s * K, (s + 1) * K) for s in seqs])
    ref = oracle.block_verify(W.to_f64(P[rows], "bf16").reshape(len(seqs), K, V),
                              W.to_f64(Q[rows], "bf16").reshape(len(seqs), K, V),
                              u[seqs].astype(np.float64), 1.0, 0, f32(w.top_p))
    sub = {k: (v[seqs] if v is not None else None) for k, v in gpu.items()}
    cmp = compare_verify(sub, ref, band=FULL_BAND).check()
    assert cmp.n == 64
    # the stated 1e-4 band would excuse nearly everything at this vocabulary size
    assert cmp.literal_near > 0.3 * cmp.n
    assert (gpu["count"] >= 1).all() and (gpu["count"] <= K).all()


@pytest.mark.parametrize("top_k", [50, 0])
def test_pos0_entries_below_zero_draw_from_p0(top_k):
    """pos0_tokens[b] < 0 (a previous step's next token when all its drafts were accepted)
    draws x_0 from p_0, on both paths; the other entries are taken as given."""
    B, K, V = 6, 5, 4000
    P, Q, u = _inputs(B, K, V, "bf16", seed=91 + top_k)
    pos0 = np.random.default_rng(91).integers(0, V, B).astype(np.int32)
    pos0[::2] = -1
    if top_k:
        gpu, ref, _ = _check(P, Q, u, 1.0, top_k, 0.95, "bf16", pos0=pos0)
    else:
        gpu, ref, _ = _check_full(P, Q, u, 1.0, 0.95, "bf16", pos0=pos0)
    assert (gpu["tokens"][1::2, 0] == pos0[1::2]).all()
    assert (gpu["tokens"][::2, 0] >= 0).all()


@pytest.mark.parametrize("k", [1, 50, 128])
def test_topk_outlier_slices_go_to_the_generic_kernel(k, monkeypatch):
    """A few huge logits put the largest values of their slice far above the rest, so that
    slice holds fewer than k tokens among its 256 largest values: the cluster kernel hands
    those items to the generic kernel, and every result must still be the oracle's. The
    streaming path (the default) gets the same rows."""
    B, K, V = 3, 4, 40000
    rng = np.random.default_rng(46 + k)
    base = rng.standard_normal((B, K, V)).astype(np.float32)
    base[:, :, 5] = 4000.0
    base[:, ::2, 20011] = -3000.0
    P = W.bf16_bits(base)
    Q = W.bf16_bits((0.8 * base + 0.6 * rng.standard_normal((B, K, V))).astype(np.float32))
    u = rng.random((B, K, 3), dtype=np.float32)
    _check(P, Q, u, 1.0, k, 0.9, "bf16")
    monkeypatch.setenv("UNO_VERIFY_TOPK", "local")
    _check(P, Q, u, 1.0, k, 0.9, "bf16")
