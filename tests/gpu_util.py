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


def _path(ref, b):
    """The oracle's decisions for sequence b in the order they are taken, as
    (position, margin) pairs: per reached position the top-p cuts of P_i and Q_i, the draw
    and the acceptance test; at the first rejection the residual draw. A margin of inf is a
    decision that was not taken (a supplied token, top-p off, i = 0 for the drafter)."""
    K = ref["tokens"].shape[1]
    n = int(ref["count"][b])
    out = []
    for i in range(min(n, K - 1) + 1):
        m = ref["margins"][b, i]
        for c in (3, 4, 0, 1):
            if np.isfinite(m[c]):
                out.append((i, float(m[c])))
        if i == n and n < K and np.isfinite(m[2]):
            out.append((i, float(m[2])))
    return out


class Comparison:
    """Result of comparing GPU and oracle verify outputs (see compare_verify)."""

    def __init__(self):
        self.n = 0               # sequences
        self.matched = 0         # sequences whose outputs all agree
        self.excused = 0         # sequences with a difference explained by a decision in the band
        self.decisions = 0       # decisions taken on the oracle's paths
        self.near = 0            # of them within the band
        self.literal_near = 0    # of them within the stated 1e-4
        self.bad = []

    def check(self, min_matched=0.9, max_excused_frac=1e-3):
        """No unexplained difference; at least `min_matched` of the sequences compared in
        full; excused decisions below `max_excused_frac` of all decisions."""
        assert not self.bad, self.bad[:5]
        assert self.matched >= min_matched * self.n, f"only {self.matched} of {self.n} sequences compared"
        assert self.excused <= max_excused_frac * self.decisions, \
            f"{self.excused} excused of {self.decisions} decisions"
        return self


def compare_verify(gpu, ref, check_tv=True, band=NEAR_FP64):
    """Compare GPU and oracle verify outputs sequence by sequence, every output.

    A difference is excused only if a decision taken before it on the oracle's path (or the
    differing decision itself) has an oracle margin below `band`: that decision may go the
    other way when both sides evaluate it in fp64 with different summation orders. Every
    other difference is a failure. Outputs after the first difference depend on it and are
    not compared further.
    """
    B, K = ref["tokens"].shape
    c = Comparison()
    c.n = B
    for b in range(B):
        path = _path(ref, b)
        c.decisions += len(path)
        c.near += sum(m < band for _, m in path)
        c.literal_near += sum(m < NEAR for _, m in path)
        n_ref, n_gpu = int(ref["count"][b]), int(gpu["count"][b])
        first = None   # first differing position (K for a difference in the correction token only)
        why = None
        for i in range(K):
            if gpu["tokens"][b, i] != ref["tokens"][b, i]:
                first, why = i, f"token {i}: {gpu['tokens'][b, i]} vs {ref['tokens'][b, i]}"
                break
        if first is None and n_gpu != n_ref:
            first, why = min(n_gpu, n_ref), f"count {n_gpu} vs {n_ref}"
        if first is None and gpu["next"][b] != ref["next"][b]:
            first, why = K, f"next {gpu['next'][b]} vs {ref['next'][b]}"
        if first is None:
            upto = min(n_ref + 1, K)
            ep = np.abs(gpu["p_tok"][b, :upto] - ref["p_tok"][b, :upto]).max()
            eq = np.abs(gpu["q_tok"][b, :upto] - ref["q_tok"][b, :upto]).max()
            if ep > PROB_TOL or eq > PROB_TOL:
                c.bad.append(f"seq {b}: p/q error {ep:.3g} {eq:.3g}")
                continue
            if check_tv and gpu.get("tv") is not None:
                rows_ok = np.min(ref["margins"][b, :, 3:5], axis=1) >= band  # top-p cuts decided
                et = np.abs(gpu["tv"][b] - ref["tv"][b])[rows_ok]
                if et.size and et.max() > PROB_TOL:
                    c.bad.append(f"seq {b}: tv error {et.max():.3g}")
                    continue
            c.matched += 1
            continue
        before = [m for i, m in path if i <= first]
        if before and min(before) < band:
            c.excused += 1
        else:
            c.bad.append(f"seq {b}: {why} (smallest margin on the path {min(before) if before else np.inf:.3g})")
    return c


def bf16_ulp(x: np.ndarray) -> np.ndarray:
    """Spacing of bf16 numbers at |x| (8 significant bits); tiny floor for zeros."""
    ax = np.abs(x)
    e = np.floor(np.log2(np.maximum(ax, 1e-38)))
    return np.exp2(e - 7)
