"""GPU parity of uno_gated_lora_linear against the fp64 oracle (through the C ABI).

Tolerance: max|err| / max|ref| <= 5e-3 against the exact fp64 value computed from the
same (bf16-representable) inputs. Cases span several 128 x BN tiles with ragged M and
ragged N, every rank class (the LoRA K tail is shorter than a 64-wide K tile for r < 64),
fp32 storage (rounded to bf16 on the device), the special cases that reduce to the base
layer (gate 0, B = 0), and the Qwen3-8B and looped-3B projection shapes at full size,
checked on sampled rows.
"""
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


@pytest.mark.parametrize("wl,name", [(W.QWEN3_8B, s.name) for s in W.QWEN3_8B_LINEARS] +
                         [(W.LOOPED_3B, s.name) for s in W.LOOPED_3B_LINEARS if s.name in ("q", "k", "down")])
def test_full_shapes_sampled_rows(wl, name):
    sh = [s for s in wl.shapes if s.name == name][0]
    inp = W.linear_inputs(wl, sh)
    y = _run(inp, wl.M, sh.d_in, sh.d_out, wl.rank)
    rows = np.array([0, 1, 15, 16, 127, 128, wl.M // 2 + 3, wl.M - 1])
    ref = _ref(inp, rows)
    assert _rel(y[rows], ref) <= TOL
    assert np.isfinite(y).all()
