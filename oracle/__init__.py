"""fp64 CPU oracle for the Uno draft-and-verify hot path (ctypes wrapper around uno_oracle.c).

TEST INFRASTRUCTURE ONLY: the test suite, the smoke check and the benchmark's CPU-baseline
leg use this package; the product path never does. It shares no code with the CUDA
library. Inputs are widened exactly to float64 before the C code sees them.

Every function here is pinned by tests/test_oracle_*.py against values that the pages and
the mathematics fix (closed forms, invariants, library routines on special cases, brute
force on tiny inputs, hand-worked fixtures under tests/golden/).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from pathlib import Path

import numpy as np

_HERE = Path(__file__).resolve().parent
_SRC = _HERE / "uno_oracle.c"
_LIB_PATH = _HERE / "liboracle.so"
_lib = None

_f64p = ctypes.POINTER(ctypes.c_double)
_i32p = ctypes.POINTER(ctypes.c_int32)
_i64p = ctypes.POINTER(ctypes.c_int64)
_u8p = ctypes.POINTER(ctypes.c_uint8)
_i64 = ctypes.c_int64
_f64 = ctypes.c_double


def compile_source(src: Path, out: Path) -> Path:
    """gcc -O2 -fopenmp, IEEE fp64 (no fast-math)."""
    tmp = Path(str(out) + f".{os.getpid()}.tmp")
    subprocess.run(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11", "-Wall",
                    "-o", str(tmp), str(src), "-lm"], check=True)
    os.replace(tmp, out)
    return out


def build(force: bool = False) -> Path:
    """Compile uno_oracle.c into liboracle.so (rebuilt when the source is newer)."""
    if force or not _LIB_PATH.exists() or _LIB_PATH.stat().st_mtime < _SRC.stat().st_mtime:
        compile_source(_SRC, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is None:
        build()
        _lib = _bind(ctypes.CDLL(str(_LIB_PATH)))
    return _lib


class use_library:
    """Context manager: route the wrappers to another build of uno_oracle.c (used by the
    test that plants mistakes in a copy of the oracle to show that the pins catch them)."""

    def __init__(self, path):
        self.path = str(path)

    def __enter__(self):
        global _lib
        _load()
        self.saved = _lib
        _lib = _bind(ctypes.CDLL(self.path))
        return self

    def __exit__(self, *exc):
        global _lib
        _lib = self.saved
        return False


def _bind(lib):
    lib.oracle_gated_lora.argtypes = [_f64p, _f64p, _f64p, _f64p, _f64p, _f64, _i64, _i64, _i64, _i64, _f64p]
    lib.oracle_warp_row.argtypes = [_f64p, _i64, _f64, _i64, _f64, _f64p, _f64p, _i64p]
    lib.oracle_warp_row.restype = _f64
    lib.oracle_inv_cdf.argtypes = [_f64p, _i64, _f64, _f64, _f64p]
    lib.oracle_inv_cdf.restype = _i64
    lib.oracle_block_verify.argtypes = [_f64p, _f64p, _i64, _i64, _i64, _f64, _i64, _f64,
                                        _i32p, _i32p, _f64p, _i32p, _i32p, _i32p,
                                        _f64p, _f64p, _f64p, _f64p]
    lib.oracle_tv_loss.argtypes = [_f64p, _f64p, _i64, _i64, _u8p, _f64, _f64p, _f64p, _f64p, _f64p]
    lib.oracle_block_noise.argtypes = [_i32p, ctypes.POINTER(ctypes.c_float), _i64, _i64, _i64, _i32p, _f64p]
    lib.oracle_block_noise.restype = ctypes.c_int
    lib.oracle_num_threads.restype = ctypes.c_int
    lib.oracle_set_num_threads.argtypes = [ctypes.c_int]
    return lib


def _p(a, t):
    return None if a is None else a.ctypes.data_as(t)


def _f64c(a):
    return np.ascontiguousarray(a, dtype=np.float64)


def num_threads() -> int:
    return int(_load().oracle_num_threads())


def set_num_threads(n: int) -> None:
    _load().oracle_set_num_threads(int(n))


def gated_lora(x, w0, a, b, gate, scale):
    """y = x W0^T + scale * diag(gate) (x A^T) B^T in fp64. x [M,d_in], w0 [d_out,d_in],
    a [r,d_in], b [d_out,r], gate [M] or None (all zeros)."""
    x, w0, a, b = _f64c(x), _f64c(w0), _f64c(a), _f64c(b)
    M, d_in = x.shape
    d_out = w0.shape[0]
    r = a.shape[0]
    g = None if gate is None else _f64c(gate)
    y = np.empty((M, d_out), dtype=np.float64)
    rc = _load().oracle_gated_lora(_p(x, _f64p), _p(w0, _f64p), _p(a, _f64p), _p(b, _f64p), _p(g, _f64p),
                                   float(scale), M, d_in, d_out, r, _p(y, _f64p))
    assert rc == 0
    return y


def warp_row(logits, temperature=1.0, top_k=0, top_p=1.0):
    """Warped row: returns (dist [V] normalised, topp_margin, n_keep)."""
    z = _f64c(logits)
    w = np.empty_like(z)
    m = ctypes.c_double()
    nk = ctypes.c_int64()
    Z = _load().oracle_warp_row(_p(z, _f64p), z.size, float(temperature), int(top_k), float(top_p),
                                _p(w, _f64p), ctypes.byref(m), ctypes.byref(nk))
    return w / Z, m.value, nk.value


def inv_cdf(weights, u):
    """(token, margin): smallest id whose cumulative weight exceeds u * sum(weights)."""
    w = _f64c(weights)
    m = ctypes.c_double()
    t = _load().oracle_inv_cdf(_p(w, _f64p), w.size, float(w.sum()), float(u), ctypes.byref(m))
    return int(t), m.value


def block_verify(P, Q, uniforms, temperature=1.0, top_k=0, top_p=1.0, drafts=None, pos0=None):
    """Lossless block verify over logits P, Q [B,K,V] (any real dtype, widened to fp64).

    Returns a dict: tokens [B,K] int32, count [B], next [B], p_tok [B,K], q_tok [B,K],
    tv [B,K], margins [B,K,5] (see uno_oracle.c for the margin layout).
    """
    P, Q = _f64c(P), _f64c(Q)
    B, K, V = P.shape
    u = _f64c(uniforms).reshape(B, K, 3)
    d = None if drafts is None else np.ascontiguousarray(drafts, dtype=np.int32)
    p0 = None if pos0 is None else np.ascontiguousarray(pos0, dtype=np.int32)
    out = {
        "tokens": np.empty((B, K), np.int32), "count": np.empty(B, np.int32), "next": np.empty(B, np.int32),
        "p_tok": np.empty((B, K)), "q_tok": np.empty((B, K)), "tv": np.empty((B, K)),
        "margins": np.empty((B, K, 5)),
    }
    rc = _load().oracle_block_verify(
        _p(P, _f64p), _p(Q, _f64p), B, K, V, float(temperature), int(top_k), float(top_p),
        _p(d, _i32p), _p(p0, _i32p), _p(u, _f64p),
        _p(out["tokens"], _i32p), _p(out["count"], _i32p), _p(out["next"], _i32p),
        _p(out["p_tok"], _f64p), _p(out["q_tok"], _f64p), _p(out["tv"], _f64p), _p(out["margins"], _f64p))
    assert rc == 0
    return out


def tv_loss(teacher, student, mask=None, grad_scale=1.0, want_grad=True, want_absdiff=False):
    """TV self-distillation loss: returns dict tv [N], mean, grad [N,V] or None, absdiff or None."""
    t, s = _f64c(teacher), _f64c(student)
    N, V = t.shape
    m = None if mask is None else np.ascontiguousarray(mask, dtype=np.uint8)
    tv = np.empty(N)
    mean = ctypes.c_double()
    g = np.empty((N, V)) if want_grad else None
    ad = np.empty((N, V)) if want_absdiff else None
    rc = _load().oracle_tv_loss(_p(t, _f64p), _p(s, _f64p), N, V, _p(m, _u8p), float(grad_scale),
                                _p(tv, _f64p), ctypes.byref(mean), _p(g, _f64p), _p(ad, _f64p))
    assert rc == 0
    return {"tv": tv, "mean": mean.value, "grad": g, "absdiff": ad}


def block_noise(clean, uniforms, V):
    """Block-noised copy, random_uniform mode: dict tokens [B, K] int32, gate [B*K] (see
    oracle_block_noise)."""
    c = np.ascontiguousarray(clean, dtype=np.int32)
    B, K = c.shape
    u = np.ascontiguousarray(uniforms, dtype=np.float32).reshape(B, K)
    out = np.empty((B, K), np.int32)
    gate = np.empty(B * K)
    rc = _load().oracle_block_noise(_p(c, _i32p), u.ctypes.data_as(ctypes.POINTER(ctypes.c_float)), B, K, int(V),
                                    _p(out, _i32p), _p(gate, _f64p))
    assert rc == 0
    return {"tokens": out, "gate": gate}
