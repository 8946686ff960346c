"""GPU parity of uno_gated_lora_linear against the fp64 oracle (through the C ABI).

Tolerance: max|err| / max|ref| <= 5e-3 against the exact fp64 value computed from the
same (bf16-representable) inputs. Cases span several 128 x BN tiles with ragged M and
ragged N, every rank class (the LoRA K tail is shorter than a 64-wide K tile for r < 64),
fp32 storage (rounded to bf16 on the device), the special cases that reduce to the base
layer (gate 0, B = 0), and every Qwen3-8B and looped-3B projection at full size (q and
down of the Qwen3-8B layer on every row, the others on one row of every 128-row tile).
"""
import zlib

import numpy as np
import pytest
import torch

import oracle
from diffusion_drafted_lossless_b200 import _lib
from diffusion_drafted_lossless_b200 import workloads as W
from tests.gpu_util import dev

pytestmark = pytest.mark.gpu
TOL = 5e-3


def _run(inp, M, d_in, d_out, r):
    dt = inp["dtype"]
    x, w0, a, b = (dev(inp[k], dt) for k in ("x", "w0", "a", "b"))
    g = torch.from_numpy(np.ascontiguousarray(inp["gate"], np.float32)).cuda()
    y = torch.empty((M, d_out), dtype=x.dtype, device="cuda")
    _lib.uno_gated_lora_linear(x, w0, a, b, g, inp["scale"], y)
    torch.cuda.synchronize()
    return y.float().cpu().numpy()


def _ref(inp, rows=None):
    dt = inp["dtype"]
    x = W.to_f64(inp["x"], dt)
    g = inp["gate"].astype(np.float64)
    if rows is not None:
        x, g = x[rows], g[rows]
    return oracle.gated_lora(x, W.to_f64(inp["w0"], dt), W.to_f64(inp["a"], dt), W.to_f64(inp["b"], dt), g,
                             float(np.float32(inp["scale"])))


def _rel(y, ref):
    return np.abs(y - ref).max() / np.abs(ref).max()


def test_tiny_fp32_config():
    w = W.TINY_LINEAR
    sh = w.shapes[0]
    inp = W.linear_inputs(w, sh)
    y = _run(inp, w.M, sh.d_in, sh.d_out, w.rank)
    # the device rounds fp32 inputs to bf16 before the tensor cores: compare with the
    # exact product of the rounded inputs, and with the unrounded fp32 inputs
    inp16 = dict(inp, dtype="bf16", **{k: W.bf16_bits(inp[k]) for k in ("x", "w0", "a", "b")})
    assert _rel(y, _ref(inp16)) <= TOL
    assert _rel(y, _ref(inp)) <= TOL


@pytest.mark.parametrize("M,d_in,d_out,r", [(200, 512, 384, 16), (129, 256, 640, 128), (300, 1024, 256, 64),
                                            (64, 320, 192, 8), (1000, 768, 1024, 256), (5, 128, 64, 24)])
def test_bf16_ragged_tiles(M, d_in, d_out, r):
    w = W.GatedLoraWorkload("t", 77 + M, M=M, block=8, rank=r, scale=2.0, shapes=(W.LinearShape("t", d_in, d_out),))
    inp = W.linear_inputs(w, w.shapes[0])
    y = _run(inp, M, d_in, d_out, r)
    assert _rel(y, _ref(inp)) <= TOL


def test_gate_zero_and_b_zero_are_the_base_layer():
    M, d_in, d_out, r = 256, 512, 512, 32
    w = W.GatedLoraWorkload("t", 91, M=M, block=8, rank=r, scale=2.0, shapes=(W.LinearShape("t", d_in, d_out),))
    inp = W.linear_inputs(w, w.shapes[0])
    base = W.to_f64(inp["x"], "bf16") @ W.to_f64(inp["w0"], "bf16").T
    y0 = _run(dict(inp, gate=np.zeros(M, np.float32)), M, d_in, d_out, r)
    assert _rel(y0, base) <= TOL
    yb = _run(dict(inp, b=np.zeros_like(inp["b"])), M, d_in, d_out, r)
    assert _rel(yb, base) <= TOL
    # and the gated rows do differ from the base layer
    y = _run(inp, M, d_in, d_out, r)
    assert np.abs(y - base)[inp["gate"] > 0].max() > 10 * TOL * np.abs(base).max()


def _tile_rows(M, seed):
    """One row from every 128-row tile (at a different offset in each), plus the first and
    last rows: a fault confined to one tile of rows cannot pass."""
    rng = np.random.default_rng(seed)
    rows = [t + int(rng.integers(0, min(128, M - t))) for t in range(0, M, 128)]
    return np.unique(np.array(rows + [0, M - 1]))


@pytest.mark.parametrize("wl,name", [(W.QWEN3_8B, s.name) for s in W.QWEN3_8B_LINEARS] +
                         [(W.LOOPED_3B, s.name) for s in W.LOOPED_3B_LINEARS])
def test_full_shapes(wl, name):
    """Every projection of the Qwen3-8B layer (M = 1024, rank 128) and of the looped 3B-class
    layer (M = 2048, rank 64) at full size. q and down of the Qwen3-8B layer are compared on
    every row and column; the others on every column of one row per 128-row tile."""
    sh = [s for s in wl.shapes if s.name == name][0]
    inp = W.linear_inputs(wl, sh)
    y = _run(inp, wl.M, sh.d_in, sh.d_out, wl.rank)
    assert np.isfinite(y).all()
    if wl is W.QWEN3_8B and name in ("q", "down"):
        assert _rel(y, _ref(inp)) <= TOL
    else:
        rows = _tile_rows(wl.M, zlib.crc32(name.encode()))
        assert _rel(y[rows], _ref(inp, rows)) <= TOL


@pytest.mark.parametrize("name", ["k", "down"])
def test_one_loop_drafting_verify_prefix(name):
    """One-loop drafting's second loop: the looped-3B projections over the 256 verify rows
    only (gate 0), passed as the first rows of the 2048-row activations (a prefix view),
    against the oracle's base layer on every row."""
    wl = W.LOOPED_3B
    sh = [s for s in wl.shapes if s.name == name][0]
    inp = W.linear_inputs(wl, sh)
    n_verify = wl.M // wl.block
    x = dev(inp["x"], "bf16")[:n_verify]
    w0, a, b = (dev(inp[k], "bf16") for k in ("w0", "a", "b"))
    g = torch.zeros(n_verify, device="cuda")
    y = torch.empty((n_verify, sh.d_out), dtype=torch.bfloat16, device="cuda")
    _lib.uno_gated_lora_linear(x, w0, a, b, g, wl.scale, y)
    torch.cuda.synchronize()
    ref = oracle.gated_lora(W.to_f64(inp["x"], "bf16")[:n_verify], W.to_f64(inp["w0"], "bf16"),
                            W.to_f64(inp["a"], "bf16"), W.to_f64(inp["b"], "bf16"), np.zeros(n_verify), 2.0)
    assert _rel(y.float().cpu().numpy(), ref) <= TOL


@pytest.mark.parametrize("ks", [2, 3, 7])
def test_output_split_k(monkeypatch, ks):
    """Output tiles split over K (selected with UNO_LORA_KSPLIT): the fp32 partials are
    summed by the split that finishes a tile last. Ragged M and N, every rank class, fp32 storage, and
    two calls in a row (the tickets of the second call must not count the first's)."""
    monkeypatch.setenv("UNO_LORA_KSPLIT", str(ks))
    for M, d_in, d_out, r in [(200, 512, 384, 16), (300, 1024, 256, 64), (129, 256, 640, 128)]:
        w = W.GatedLoraWorkload("t", 177 + M + ks, M=M, block=8, rank=r, scale=2.0,
                                shapes=(W.LinearShape("t", d_in, d_out),))
        inp = W.linear_inputs(w, w.shapes[0])
        ref = _ref(inp)
        for _ in range(2):
            assert _rel(_run(inp, M, d_in, d_out, r), ref) <= TOL
    w = W.TINY_LINEAR
    sh = w.shapes[0]
    inp = W.linear_inputs(w, sh)
    inp16 = dict(inp, dtype="bf16", **{k: W.bf16_bits(inp[k]) for k in ("x", "w0", "a", "b")})
    assert _rel(_run(inp, w.M, sh.d_in, sh.d_out, w.rank), _ref(inp16)) <= TOL


def test_calls_back_to_back_on_one_workspace():
    """Two calls with different gates on the same workspace: the second call's output
    tiles must use its own adapter rows, not the ones the first call left behind."""
    M, d_in, d_out, r = 512, 1024, 1024, 64
    w = W.GatedLoraWorkload("t", 93, M=M, block=8, rank=r, scale=2.0, shapes=(W.LinearShape("t", d_in, d_out),))
    inp = W.linear_inputs(w, w.shapes[0])
    import torch
    from diffusion_drafted_lossless_b200 import _lib
    dv = {k: torch.from_numpy(inp[k].view(np.int16)).view(torch.bfloat16).cuda() for k in ("x", "w0", "a", "b")}
    ws = torch.empty(_lib.uno_gated_lora_linear_workspace_size(M, d_in, d_out, r), dtype=torch.uint8, device="cuda")
    outs = []
    gates = [inp["gate"], (1.0 - inp["gate"]).astype(np.float32)]
    for gt in gates:
        y = torch.empty((M, d_out), dtype=torch.bfloat16, device="cuda")
        _lib.uno_gated_lora_linear(dv["x"], dv["w0"], dv["a"], dv["b"], torch.from_numpy(gt).cuda(), 2.0, y,
                                   workspace=ws)
        outs.append(y)
    torch.cuda.synchronize()
    for y, gt in zip(outs, gates):
        ref = _ref(dict(inp, gate=gt))
        assert _rel(y.float().cpu().numpy(), ref) <= TOL


@pytest.mark.parametrize("splits", ["3", "64"])
def test_split_adapter_path(monkeypatch, splits):
    """The adapter product split over K into bf16 partials of T, each run through the output
    tiles' (T, B) K tiles in turn, gives the oracle's result; 64 splits exceed the K tiles
    and are clamped."""
    monkeypatch.setenv("UNO_LORA_SPLITS", splits)
    for M, d_in, d_out, r in [(300, 1024, 256, 64), (1000, 768, 1024, 256), (129, 256, 640, 128)]:
        w = W.GatedLoraWorkload("t", 5 + M, M=M, block=8, rank=r, scale=2.0,
                                shapes=(W.LinearShape("t", d_in, d_out),))
        inp = W.linear_inputs(w, w.shapes[0])
        y = _run(inp, M, d_in, d_out, r)
        assert _rel(y, _ref(inp)) <= TOL


@pytest.mark.parametrize("env", [{"UNO_LORA_CG": "2"}, {"UNO_LORA_CG": "2", "UNO_LORA_SPLITS": "3"},
                                 {"UNO_LORA_CG": "2", "UNO_LORA_BN": "128"}, {"UNO_LORA_CG": "2", "UNO_LORA_BN": "64"},
                                 {"UNO_LORA_CG": "1"}])
def test_cta_pair_and_single_forms(monkeypatch, env):
    """The CTA-pair form (256-row tiles of 256, 128 or 64 columns, one MMA stream over two
    SMs) and the single-CTA form give the oracle's result on ragged shapes (M not a multiple
    of 256, rank 8/24/256)."""
    for k, v in env.items():
        monkeypatch.setenv(k, v)
    for M, d_in, d_out, r in [(300, 1024, 512, 64), (1000, 768, 1024, 256), (257, 256, 768, 8),
                              (512, 512, 256, 24), (1024, 4096, 4096, 128)]:
        w = W.GatedLoraWorkload("t", 11 + M + r, M=M, block=8, rank=r, scale=2.0,
                                shapes=(W.LinearShape("t", d_in, d_out),))
        inp = W.linear_inputs(w, w.shapes[0])
        y = _run(inp, M, d_in, d_out, r)
        assert _rel(y, _ref(inp)) <= TOL, (M, d_in, d_out, r)


def test_withheld_adapter_flags_time_out(monkeypatch):
    """The failure path of a bounded device wait. With UNO_LORA_TEST_WITHHOLD_FLAGS=1 the
    adapter items never publish their rows of T, so every output tile's wait for them runs
    out. The call must end by itself (no hang, no fault), the device status word must then
    read UNO_ERR_TIMEOUT, and the next normal call must give the oracle's result: the
    context stays usable."""
    M, d_in, d_out, r = 512, 1024, 1024, 64
    w = W.GatedLoraWorkload("t", 97, M=M, block=8, rank=r, scale=2.0, shapes=(W.LinearShape("t", d_in, d_out),))
    inp = W.linear_inputs(w, w.shapes[0])
    assert _lib.uno_read_device_status() == _lib.UNO_OK
    monkeypatch.setenv("UNO_LORA_TEST_WITHHOLD_FLAGS", "1")
    _run(inp, M, d_in, d_out, r)
    assert _lib.uno_read_device_status() == _lib.UNO_ERR_TIMEOUT
    monkeypatch.delenv("UNO_LORA_TEST_WITHHOLD_FLAGS")
    assert _rel(_run(inp, M, d_in, d_out, r), _ref(inp)) <= TOL
    assert _lib.uno_read_device_status() == _lib.UNO_OK


@pytest.mark.parametrize("epi", ["tma", "rows"])
def test_output_epilogues(epi, monkeypatch):
    """Both bf16 epilogues: output tiles staged in shared memory (64-byte swizzle) and written
    by TMA stores (the default), and per-lane row stores (UNO_LORA_EPI=rows). Ragged M (the
    stores leave rows past M out), every tile width, several tiles per CTA, and two calls in
    a row."""
    if epi == "rows":
        monkeypatch.setenv("UNO_LORA_EPI", "rows")
    for M, d_in, d_out, r in [(300, 1024, 512, 64), (1000, 768, 1024, 256), (129, 256, 640, 128),
                              (1024, 4096, 4096, 128), (2048, 2560, 640, 64), (5, 128, 64, 24)]:
        w = W.GatedLoraWorkload("t", 23 + M + r, M=M, block=8, rank=r, scale=2.0,
                                shapes=(W.LinearShape("t", d_in, d_out),))
        inp = W.linear_inputs(w, w.shapes[0])
        ref = _ref(inp)
        for _ in range(2):
            assert _rel(_run(inp, M, d_in, d_out, r), ref) <= TOL, (M, d_in, d_out, r)

def test_k_and_v_as_one_call():
    """k and v of the Qwen3-8B layer as one call over [W0_k; W0_v], [A_k; A_v] and
    diag(B_k, B_v) (rank 2r): the output's column halves equal the two separate calls bit
    for bit (the zero blocks of B add exact zeros) and the oracle on sampled rows."""
    wl = W.QWEN3_8B
    sh = {s.name: s for s in wl.shapes}
    ik, iv = W.linear_inputs(wl, sh["k"]), W.linear_inputs(wl, sh["v"])
    M, d_in, dk, r = wl.M, sh["k"].d_in, sh["k"].d_out, wl.rank
    iv = dict(iv, x=ik["x"], gate=ik["gate"])  # the same input rows and gate
    yk = _run(ik, M, d_in, dk, r)
    yv = _run(iv, M, d_in, dk, r)
    bf = np.zeros((2 * dk, 2 * r), dtype=ik["b"].dtype)
    bf[:dk, :r] = ik["b"]
    bf[dk:, r:] = iv["b"]
    fused = dict(ik, w0=np.concatenate([ik["w0"], iv["w0"]]), a=np.concatenate([ik["a"], iv["a"]]), b=bf)
    y = _run(fused, M, d_in, 2 * dk, 2 * r)
    assert np.array_equal(y[:, :dk], yk) and np.array_equal(y[:, dk:], yv)
    rows = _tile_rows(M, 7)
    assert _rel(y[rows], _ref(fused, rows)) <= TOL
