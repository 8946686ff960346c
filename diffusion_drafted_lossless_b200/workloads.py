"""Seeded synthetic inputs for the Uno draft-and-verify hot path.

This module draws random numbers and rounds them to their storage dtype. It holds none of
the method's arithmetic: the CUDA path's tests and benchmark and the CPU oracle both read
what it produces, so it is the one piece of code the two sides share.

Shapes and value distributions follow the workloads the Uno pages describe (the LoopUno
project page, "Setup / Recipe" and "Experiment data"; the uno-qwen3-8B model card,
"Evaluation protocol"). No model weights or datasets are involved: every tensor is a
normal draw of the stated scale, rounded to bf16 with round-to-nearest-even.

Rows are generated in blocks of ``ROW_BLOCK`` from a PCG64 stream keyed by
``(seed, tag, block)``, so any row of a large tensor can be regenerated on its own (the
full-size parity tests check sampled rows against the oracle that way).
"""
from __future__ import annotations

import os
import zlib
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass, field

import numpy as np

ROW_BLOCK = 64

# Stream tags: one independent PCG64 stream family per tensor role.
TAG_X, TAG_W0, TAG_A, TAG_B = 1, 2, 3, 4
TAG_VERIFIER, TAG_DRAFT_NOISE, TAG_UNIFORM = 11, 12, 13
TAG_TEACHER, TAG_STUDENT_NOISE = 21, 22


# --------------------------------------------------------------------------------------
# storage dtype conversion (bf16 held as raw uint16 bits; numpy has no bfloat16)
# --------------------------------------------------------------------------------------
def bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round float32 values to bf16 with round-to-nearest-even; return the raw bits."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)
    rounding = ((u >> np.uint32(16)) & np.uint32(1)) + np.uint32(0x7FFF)
    return ((u + rounding) >> np.uint32(16)).astype(np.uint16)


def bf16_to_f32(bits: np.ndarray) -> np.ndarray:
    """Widen raw bf16 bits to float32 (exact)."""
    return (np.ascontiguousarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def _rng(seed: int, tag: int, block: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64([int(seed), int(tag), int(block)]))


def _threads() -> int:
    return max(1, min(16, os.cpu_count() or 1))


def _blocks_for(rows: np.ndarray) -> dict[int, np.ndarray]:
    out: dict[int, list[int]] = {}
    for i, r in enumerate(rows.tolist()):
        out.setdefault(r // ROW_BLOCK, []).append(i)
    return {b: np.asarray(v) for b, v in out.items()}


def normal_rows(seed: int, tag: int, n_rows: int, n_cols: int, sigma: float,
                rows: np.ndarray | None = None) -> np.ndarray:
    """float32 draws ~ N(0, sigma^2) for the given rows of an [n_rows, n_cols] tensor.

    ``sigma`` is the standard deviation. With ``rows=None`` every row is produced.
    Row ``r`` is the ``r % ROW_BLOCK``-th row of block ``r // ROW_BLOCK``'s stream.
    """
    rows = np.arange(n_rows) if rows is None else np.asarray(rows, dtype=np.int64)
    out = np.empty((len(rows), n_cols), dtype=np.float32)

    def work(item):
        blk, idx = item
        need = int(rows[idx].max() % ROW_BLOCK) + 1
        block_rows = min(need, n_rows - blk * ROW_BLOCK)
        z = _rng(seed, tag, blk).standard_normal((block_rows, n_cols), dtype=np.float32)
        out[idx] = z[rows[idx] % ROW_BLOCK] * np.float32(sigma)

    items = list(_blocks_for(rows).items())
    if len(items) == 1:
        work(items[0])
    else:
        with ThreadPoolExecutor(_threads()) as ex:
            list(ex.map(work, items))
    return out


def uniforms(seed: int, shape: tuple[int, ...]) -> np.ndarray:
    """float32 U[0,1) draws (the verify step's supplied random numbers)."""
    u = _rng(seed, TAG_UNIFORM, 0).random(shape, dtype=np.float32)
    return np.minimum(u, np.float32(np.nextafter(np.float32(1), np.float32(0))))


# --------------------------------------------------------------------------------------
# the five workloads
# --------------------------------------------------------------------------------------
@dataclass(frozen=True)
class LinearShape:
    name: str
    d_in: int
    d_out: int


@dataclass(frozen=True)
class GatedLoraWorkload:
    """Row-gated LoRA linears: M rows of B sequences x block K; row 0 of each block ungated."""
    name: str
    seed: int
    M: int
    block: int
    rank: int
    scale: float
    shapes: tuple[LinearShape, ...]
    dtype: str = "bf16"          # "bf16" or "f32" storage for X / weights
    x_sigma: float = 1.0
    w_sigma: float = 0.02


@dataclass(frozen=True)
class VerifyWorkload:
    name: str
    seed: int
    B: int
    K: int
    V: int
    sigma: float
    rho: float | None            # None: drafter independent of the verifier
    temperature: float
    top_k: int                   # 0 = off
    top_p: float                 # >= 1 = off
    dtype: str = "bf16"


@dataclass(frozen=True)
class TVWorkload:
    name: str
    seed: int
    N: int
    V: int
    teacher_sigma: float = 3.0
    noise_sigma: float = 1.0


QWEN3_8B_LINEARS = (
    LinearShape("q", 4096, 4096), LinearShape("k", 4096, 1024), LinearShape("v", 4096, 1024),
    LinearShape("o", 4096, 4096), LinearShape("gate", 4096, 12288), LinearShape("up", 4096, 12288),
    LinearShape("down", 12288, 4096),
)
LOOPED_3B_LINEARS = (
    LinearShape("q", 2560, 2560), LinearShape("k", 2560, 640), LinearShape("v", 2560, 640),
    LinearShape("o", 2560, 2560), LinearShape("gate", 2560, 9728), LinearShape("up", 2560, 9728),
    LinearShape("down", 9728, 2560),
)

# 1: tiny CPU-checkable step (fp32 storage)
TINY_LINEAR = GatedLoraWorkload("tiny_linear_256x256_r8_m16", 1001, M=16, block=8, rank=8, scale=2.0,
                                shapes=(LinearShape("tiny", 256, 256),), dtype="f32")
TINY_VERIFY = VerifyWorkload("tiny_verify_b2_k8_v1000", 1001, B=2, K=8, V=1000, sigma=2.0, rho=None,
                             temperature=1.0, top_k=0, top_p=1.0, dtype="f32")
# 2: Qwen3-8B-shaped projections, M = 64 sequences x block 16
QWEN3_8B = GatedLoraWorkload("qwen3_8b_linears_m1024_r128", 1002, M=1024, block=16, rank=128, scale=2.0,
                             shapes=QWEN3_8B_LINEARS)
# 3: verify at serving scale (the headline workload)
SERVING_VERIFY = VerifyWorkload("verify_b64_k16_v151936", 1003, B=64, K=16, V=151936, sigma=3.0, rho=0.8,
                                temperature=1.0, top_k=50, top_p=0.95)
# 4: looped 3B-class step: 22 layers applied twice, M = 256 x block 8
LOOPED_3B = GatedLoraWorkload("looped_3b_linears_m2048_r64", 1004, M=2048, block=8, rank=64, scale=2.0,
                              shapes=LOOPED_3B_LINEARS)
LOOPED_3B_LAYERS, LOOPED_3B_LOOPS = 22, 2
LOOPED_VERIFY = VerifyWorkload("verify_b256_k8_v166144", 1004, B=256, K=8, V=166144, sigma=3.0, rho=0.8,
                               temperature=1.0, top_k=0, top_p=0.95)
# 5: TV self-distillation loss over 8 x 2048 response tokens
TV_LOSS = TVWorkload("tv_n16384_v151936", 1005, N=16384, V=151936)


def row_gate(M: int, block: int) -> np.ndarray:
    """Per-row adapter gate: 0 on position 0 of every block, 1 on the draft-noise rows."""
    g = np.ones(M, dtype=np.float32)
    g[::block] = 0.0
    return g


# --------------------------------------------------------------------------------------
# generators
# --------------------------------------------------------------------------------------
def _store(a: np.ndarray, dtype: str) -> np.ndarray:
    return bf16_bits(a) if dtype == "bf16" else np.ascontiguousarray(a, dtype=np.float32)


def linear_inputs(w: GatedLoraWorkload, shape: LinearShape, rows: np.ndarray | None = None,
                  layer: int = 0) -> dict:
    """X [M,d_in], W0 [d_out,d_in], A [r,d_in], B [d_out,r], gate [M] in storage dtype.

    ``layer`` offsets the weight streams so different layers get different weights.
    ``rows`` restricts X and the gate to those rows (weights are always whole).
    """
    s = w.seed
    lk = 1000 * (layer + 1) + zlib.crc32(shape.name.encode()) % 997
    x = normal_rows(s, TAG_X * 7919 + shape.d_in, w.M, shape.d_in, w.x_sigma, rows)
    w0 = normal_rows(s, TAG_W0 * 7919 + lk, shape.d_out, shape.d_in, w.w_sigma)
    a = normal_rows(s, TAG_A * 7919 + lk, w.rank, shape.d_in, w.w_sigma)
    b = normal_rows(s, TAG_B * 7919 + lk, shape.d_out, w.rank, w.w_sigma)
    g = row_gate(w.M, w.block)
    if rows is not None:
        g = g[np.asarray(rows)]
    return {"x": _store(x, w.dtype), "w0": _store(w0, w.dtype), "a": _store(a, w.dtype),
            "b": _store(b, w.dtype), "gate": g, "scale": w.scale, "dtype": w.dtype}


def verify_logits(w: VerifyWorkload, rows: np.ndarray | None = None) -> tuple[np.ndarray, np.ndarray]:
    """Verifier and drafter logits for the flattened [B*K] rows, storage dtype, [n, V].

    The verifier is N(0, sigma^2). With ``rho`` set, the drafter is
    rho * v + sqrt(1 - rho^2) * sigma * eps with v the verifier draw before rounding and
    eps ~ N(0, 1); without it the drafter is an independent N(0, sigma^2) draw.
    """
    n = w.B * w.K
    v = normal_rows(w.seed, TAG_VERIFIER, n, w.V, w.sigma, rows)
    e = normal_rows(w.seed, TAG_DRAFT_NOISE, n, w.V, 1.0 if w.rho is not None else w.sigma, rows)
    if w.rho is not None:
        q = np.float32(w.rho) * v + np.float32(np.sqrt(1.0 - w.rho * w.rho) * w.sigma) * e
    else:
        q = e
    return _store(v, w.dtype), _store(q, w.dtype)


def verify_uniforms(w: VerifyWorkload) -> np.ndarray:
    """[B, K, 3] float32 U[0,1): (sample, accept, resample) per block position."""
    return uniforms(w.seed + 1000, (w.B, w.K, 3))


def _block_rows(seed: int, tag: int, blk: int, n_rows: int, n_cols: int, need: int) -> np.ndarray:
    """The first `need` standard-normal rows of block `blk` of an [n_rows, n_cols] tensor."""
    return _rng(seed, tag, blk).standard_normal((min(need, n_rows - blk * ROW_BLOCK), n_cols), dtype=np.float32)


def tv_logits(w: TVWorkload, rows: np.ndarray | None = None) -> tuple[np.ndarray, np.ndarray]:
    """Teacher ~ N(0, 3^2) and student = teacher + N(0, 1), both bf16 bits [n, V].

    The noise is added to the teacher draw before rounding; each is rounded once. Each
    block of rows is generated and rounded by one worker thread, so only the bf16 outputs
    are ever held in full. Row r equals normal_rows(...)[r] of the same streams.
    """
    rows = np.arange(w.N) if rows is None else np.asarray(rows, dtype=np.int64)
    T = np.empty((len(rows), w.V), dtype=np.uint16)
    S = np.empty((len(rows), w.V), dtype=np.uint16)

    def work(item):
        blk, idx = item
        need = int(rows[idx].max() % ROW_BLOCK) + 1
        sel = rows[idx] % ROW_BLOCK
        t = _block_rows(w.seed, TAG_TEACHER, blk, w.N, w.V, need)[sel]
        t *= np.float32(w.teacher_sigma)
        e = _block_rows(w.seed, TAG_STUDENT_NOISE, blk, w.N, w.V, need)[sel]
        e *= np.float32(w.noise_sigma)
        T[idx] = bf16_bits(t)
        e += t
        S[idx] = bf16_bits(e)

    items = list(_blocks_for(rows).items())
    with ThreadPoolExecutor(_threads()) as ex:
        list(ex.map(work, items))
    return T, S


def to_f64(a: np.ndarray, dtype: str) -> np.ndarray:
    """Storage array (bf16 bits or float32) widened exactly to float64."""
    if dtype == "bf16":
        return bf16_to_f32(a).astype(np.float64)
    return np.asarray(a, dtype=np.float32).astype(np.float64)
