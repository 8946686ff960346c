"""Helpers for the GPU parity tests: device transfer of the seeded inputs, calls through the
C-ABI binding, and comparison with the oracle under the stated tolerances.

Tolerances (from the problem statement's parity bar):
  * tokens and counts bit-exact, except decisions within 1e-4 of a threshold (oracle
    margin), which are counted and must stay below 0.1% of all decisions;
  * probabilities and TV: absolute error <= 1e-5 (fp32 outputs);
  * gated LoRA: max|err| / max|ref| <= 5e-3;
  * TV gradient (bf16 output): within one bf16 ulp of the fp64 value, excluding elements
    whose |p - q| < 1e-7 (their sign(q - p) is not decided at fp32), counted, < 0.1%.
"""
from __future__ import annotations

import numpy as np
import torch

from diffusion_drafted_lossless_b200 import _lib

NEAR = 1e-4          # the stated threshold band
NEAR_FP64 = 1e-9     # band for decisions both sides take in fp64 (they differ only in summation order)
PROB_TOL = 1e-5


def dev(a: np.ndarray, dtype: str) -> torch.Tensor:
    if dtype == "bf16":
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).cuda()
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).cuda()


def f32(x) -> float:
    """The float32 value the kernels see for a Python float parameter."""
    return float(np.float32(x))


def verify_gpu(P, Q, u, temperature, top_k, top_p, dtype="bf16", drafts=None, pos0=None, want_tv=True):
    """P, Q: [B,K,V] storage arrays (bf16 bits or f32); u: [B,K,3] f32. Returns numpy dict."""
    B, K, V = P.shape
    Pd, Qd = dev(P, dtype), dev(Q, dtype)
    ud = torch.from_numpy(np.ascontiguousarray(u, dtype=np.float32)).cuda()
    out = {
        "tokens": torch.full((B, K), -7, dtype=torch.int32, device="cuda"),
        "count": torch.full((B,), -7, dtype=torch.int32, device="cuda"),
        "next": torch.full((B,), -7, dtype=torch.int32, device="cuda"),
        "p_tok": torch.full((B, K), -1.0, device="cuda"),
        "q_tok": torch.full((B, K), -1.0, device="cuda"),
        "tv": torch.full((B, K), -1.0, device="cuda") if want_tv else None,
    }
    dd = None if drafts is None else torch.from_numpy(np.ascontiguousarray(drafts, np.int32)).cuda()
    pd = None if pos0 is None else torch.from_numpy(np.ascontiguousarray(pos0, np.int32)).cuda()
    _lib.uno_block_verify(Pd, Qd, temperature, top_k, top_p, ud, out["tokens"], out["count"], out["next"],
                          out["p_tok"], out["q_tok"], out["tv"], draft_tokens=dd, pos0_tokens=pd)
    torch.cuda.synchronize()
    return {k: (None if v is None else v.cpu().numpy()) for k, v in out.items()}


def decision_path_margin(ref, b):
    """Smallest oracle margin among the decisions sequence b's output depends on."""
    K = ref["tokens"].shape[1]
    n = int(ref["count"][b])
    last = min(n, K - 1)  # positions 0..n (n = first rejection) are decided
    m = ref["margins"][b, : last + 1]
    return float(np.min(m)) if m.size else np.inf


def compare_verify(gpu, ref, check_tv=True, near_eps=NEAR):
    """Compare GPU and oracle verify outputs sequence by sequence.

    A sequence whose decision path has an oracle margin below `near_eps` is excused (not
    compared) and counted. Returns (n_sequences, n_excused, mismatch descriptions,
    n_literal_near) where the last counts sequences with a margin below the stated 1e-4.
    """
    B, K = ref["tokens"].shape
    bad, near, literal = [], 0, 0
    for b in range(B):
        m = decision_path_margin(ref, b)
        literal += m < NEAR
        if m < near_eps:
            near += 1
            continue
        if gpu["count"][b] != ref["count"][b]:
            bad.append(f"seq {b}: count {gpu['count'][b]} vs {ref['count'][b]}")
            continue
        if not np.array_equal(gpu["tokens"][b], ref["tokens"][b]):
            bad.append(f"seq {b}: tokens {gpu['tokens'][b]} vs {ref['tokens'][b]}")
        if gpu["next"][b] != ref["next"][b]:
            bad.append(f"seq {b}: next {gpu['next'][b]} vs {ref['next'][b]}")
        n = int(ref["count"][b])
        upto = min(n + 1, K)
        ep = np.abs(gpu["p_tok"][b, :upto] - ref["p_tok"][b, :upto]).max()
        eq = np.abs(gpu["q_tok"][b, :upto] - ref["q_tok"][b, :upto]).max()
        if ep > PROB_TOL or eq > PROB_TOL:
            bad.append(f"seq {b}: p/q error {ep:.3g} {eq:.3g}")
        if check_tv and gpu.get("tv") is not None:
            rows_ok = np.min(ref["margins"][b, :, 3:5], axis=1) >= near_eps  # top-p cuts decided
            et = np.abs(gpu["tv"][b] - ref["tv"][b])[rows_ok]
            if et.size and et.max() > PROB_TOL:
                bad.append(f"seq {b}: tv error {et.max():.3g}")
    return B, near, bad, literal


def bf16_ulp(x: np.ndarray) -> np.ndarray:
    """Spacing of bf16 numbers at |x| (8 significant bits); tiny floor for zeros."""
    ax = np.abs(x)
    e = np.floor(np.log2(np.maximum(ax, 1e-38)))
    return np.exp2(e - 7)
