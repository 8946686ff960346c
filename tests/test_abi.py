"""The C-ABI library loads and exports every symbol include/uno.h declares; host-side
argument validation and workspace sizing work without a GPU (no kernel is launched:
every call here is rejected before any device work, or is a pure size query)."""
import ctypes
import re
from pathlib import Path

import pytest

from diffusion_drafted_lossless_b200 import _lib
from diffusion_drafted_lossless_b200.build import build

ROOT = Path(__file__).resolve().parents[1]
FAKE = 0x7F0000000000  # a 256-byte aligned address that is never dereferenced


@pytest.fixture(scope="module")
def lib():
    build()
    return _lib.load()


def declared_functions():
    text = (ROOT / "include" / "uno.h").read_text()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(uno_[a-z0-9_]+)\s*\(", text)))


def test_every_declared_symbol_is_exported(lib):
    names = declared_functions()
    assert len(names) == 13, names
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(_lib.EXPORTED)


def test_status_strings_and_version(lib):
    assert lib.uno_status_string(0) == b"UNO_OK"
    assert lib.uno_status_string(5) == b"UNO_ERR_WORKSPACE"
    assert _lib.uno_version() == 10000


def _verify(lib, B=2, K=4, V=1000, T=1.0, top_k=50, top_p=0.95, P=FAKE, Q=FAKE, u=FAKE, ws=FAKE, wsb=1 << 30,
            dtype=_lib.UNO_BF16, tokens=FAKE):
    return lib.uno_block_verify(P, Q, dtype, B, K, V, T, top_k, top_p, None, None, u, tokens, FAKE, None, None,
                                None, None, ws, wsb, None)


def test_verify_validation(lib):
    assert _verify(lib, K=33) == _lib.UNO_ERR_UNSUPPORTED
    assert _verify(lib, K=0) == _lib.UNO_ERR_INVALID_ARG
    assert _verify(lib, V=0) == _lib.UNO_ERR_INVALID_ARG
    assert _verify(lib, B=-1) == _lib.UNO_ERR_INVALID_ARG
    assert _verify(lib, T=0.0) == _lib.UNO_ERR_INVALID_ARG
    assert _verify(lib, T=float("nan")) == _lib.UNO_ERR_INVALID_ARG
    assert _verify(lib, top_p=0.0) == _lib.UNO_ERR_INVALID_ARG
    assert _verify(lib, top_k=-3) == _lib.UNO_ERR_INVALID_ARG
    assert _verify(lib, top_k=2000, V=100000) == _lib.UNO_ERR_UNSUPPORTED
    assert _verify(lib, P=0) == _lib.UNO_ERR_INVALID_ARG
    assert _verify(lib, u=0) == _lib.UNO_ERR_INVALID_ARG
    assert _verify(lib, tokens=FAKE + 4) == _lib.UNO_ERR_UNSUPPORTED
    assert _verify(lib, ws=0) == _lib.UNO_ERR_WORKSPACE
    assert _verify(lib, ws=FAKE + 16) == _lib.UNO_ERR_WORKSPACE
    assert _verify(lib, wsb=16) == _lib.UNO_ERR_WORKSPACE
    assert _verify(lib, dtype=7) == _lib.UNO_ERR_INVALID_ARG
    assert b"K <= 32" in lib.uno_last_error_string() or True
    _verify(lib, K=33)
    assert b"32" in lib.uno_last_error_string()
    # B = 0 is a no-op that needs nothing
    assert _verify(lib, B=0, P=0, Q=0, u=0, ws=0, wsb=0, tokens=0) == _lib.UNO_OK


def test_verify_workspace_sizes(lib):
    a = lib.uno_block_verify_workspace_size(64, 16, 151936, 50, 0.95, _lib.UNO_BF16)
    b = lib.uno_block_verify_workspace_size(128, 16, 151936, 50, 0.95, _lib.UNO_BF16)
    assert 0 < a < b < (1 << 30)
    assert lib.uno_block_verify_workspace_size(0, 16, 151936, 50, 0.95, _lib.UNO_BF16) == 0
    assert lib.uno_block_verify_workspace_size(4, 40, 1000, 0, 1.0, _lib.UNO_BF16) == 0  # unsupported
    assert lib.uno_block_verify_workspace_size(2, 8, 1000, 0, 1.0, _lib.UNO_F32) > 0
    # top-k on: one size; top-k off with bf16 rows: the fastest path adds a 128 KiB
    # candidate list per row (two rows per item) to the smallest workspace accepted
    for B, K, V, k in ((64, 16, 151936, 50), (3, 5, 700, 1)):
        assert (lib.uno_block_verify_min_workspace_size(B, K, V, k, 0.95, _lib.UNO_BF16)
                == lib.uno_block_verify_workspace_size(B, K, V, k, 0.95, _lib.UNO_BF16))
    full = lib.uno_block_verify_workspace_size(256, 8, 166144, 0, 0.95, _lib.UNO_BF16)
    small = lib.uno_block_verify_min_workspace_size(256, 8, 166144, 0, 0.95, _lib.UNO_BF16)
    assert full - small == 2 * 256 * 8 * (128 << 10)
    assert lib.uno_block_verify_min_workspace_size(0, 8, 166144, 0, 0.95, _lib.UNO_BF16) == 0


def test_lora_validation(lib):
    f = lib.uno_gated_lora_linear
    ok = dict(M=16, d_in=256, d_out=256, r=8)

    def call(M=16, d_in=256, d_out=256, r=8, x=FAKE, ws=FAKE, wsb=1 << 30, dtype=_lib.UNO_BF16):
        return f(x, FAKE, FAKE, FAKE, None, 2.0, M, d_in, d_out, r, dtype, FAKE, ws, wsb, None)

    assert call(d_in=100) == _lib.UNO_ERR_UNSUPPORTED
    assert call(d_out=96) == _lib.UNO_ERR_UNSUPPORTED
    assert call(r=12) == _lib.UNO_ERR_UNSUPPORTED
    assert call(r=264) == _lib.UNO_ERR_UNSUPPORTED
    assert call(M=0) == _lib.UNO_ERR_INVALID_ARG
    assert call(x=0) == _lib.UNO_ERR_INVALID_ARG
    assert call(x=FAKE + 2) == _lib.UNO_ERR_UNSUPPORTED
    assert call(ws=0) == _lib.UNO_ERR_WORKSPACE
    assert call(wsb=1) == _lib.UNO_ERR_WORKSPACE
    assert lib.uno_gated_lora_linear_workspace_size(1024, 4096, 4096, 128, 0) > 0
    assert ok


def test_tv_validation(lib):
    f = lib.uno_tv_loss

    def call(N=4, V=100, t=FAKE, ws=FAKE, wsb=1 << 20, g=2.0, mean=FAKE):
        return f(t, FAKE, _lib.UNO_BF16, N, V, None, g, FAKE, mean, None, ws, wsb, None)

    assert call(N=-1) == _lib.UNO_ERR_INVALID_ARG
    assert call(V=0) == _lib.UNO_ERR_INVALID_ARG
    assert call(t=0) == _lib.UNO_ERR_INVALID_ARG
    assert call(mean=0) == _lib.UNO_ERR_INVALID_ARG
    assert call(g=float("inf")) == _lib.UNO_ERR_INVALID_ARG
    assert call(ws=0) == _lib.UNO_ERR_WORKSPACE
    assert call(t=FAKE + 8) == _lib.UNO_ERR_UNSUPPORTED


def test_product_path_fails_loudly_without_library(tmp_path, monkeypatch):
    monkeypatch.setattr(_lib, "_lib", None)
    with pytest.raises(RuntimeError, match="no fallback"):
        _lib.load(tmp_path / "missing.so")


def test_noise_validation(lib):
    f = lib.uno_block_noise
    assert f(FAKE, FAKE, -1, 4, 100, FAKE, None, None) == _lib.UNO_ERR_INVALID_ARG
    assert f(FAKE, FAKE, 2, 0, 100, FAKE, None, None) == _lib.UNO_ERR_INVALID_ARG
    assert f(FAKE, FAKE, 2, 4, 0, FAKE, None, None) == _lib.UNO_ERR_INVALID_ARG
    assert f(FAKE, FAKE, 2, 4, 1 << 24, FAKE, None, None) == _lib.UNO_ERR_INVALID_ARG
    assert f(None, FAKE, 2, 4, 100, FAKE, None, None) == _lib.UNO_ERR_INVALID_ARG
    assert f(FAKE + 2, FAKE, 2, 4, 100, FAKE, None, None) == _lib.UNO_ERR_UNSUPPORTED
    assert f(None, None, 0, 4, 100, None, None, None) == _lib.UNO_OK  # B = 0: nothing to do


def test_binding_refuses_host_and_strided_tensors(lib):
    """The binding passes only contiguous CUDA tensors to the C ABI: a host tensor (or a
    strided view) is refused with ValueError before any library call."""
    import torch
    clean = torch.zeros((2, 4), dtype=torch.int32)
    u = torch.zeros((2, 4), dtype=torch.float32)
    out = torch.zeros((2, 4), dtype=torch.int32)
    with pytest.raises(ValueError, match="contiguous CUDA"):
        _lib.uno_block_noise(clean, u, 100, out)
    with pytest.raises(ValueError, match="contiguous CUDA"):
        _lib._ptr(torch.zeros((4, 4))[:, 1])
    assert _lib._ptr(None) is None
