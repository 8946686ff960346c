"""Benchmark of the Uno draft-and-verify hot path on B200.

One step = one pass of the whole hot path over one batch of 64 sequences x block 16
(V = 151936, Qwen3-8B shapes):
  1. the seven row-gated LoRA projections of one decoder layer (q, k, v, o, gate, up,
     down) at M = 64 x 16 = 1024 rows, rank 128, position 0 of each block ungated; k and v
     share their input, so they run as one call over the concatenated weights (W0 and A
     stacked, B block-diagonal: each adapter still acts only on its own outputs, and the
     outputs are bit-identical to two calls); the FLOPs counted are the seven projections'
     own;
  2. the lossless block verify over the [64, 16, 151936] verifier / drafter logits
     (bf16, T = 1, top-k 50, top-p 0.95; drafter correlated with the verifier, rho 0.8);
  3. the TV self-distillation loss and its gradient over the same 1024 logit rows
     (teacher = verifier logits, student = drafter logits).
Metric: verified draft rows per second = B * K / t_verify, with t_verify the mean time of
the verify inside the timed steps (CUDA events on the library's stream), summed over GPUs;
the whole step's rate is reported beside it ("step"), and "e2e" is the whole step through
the C ABI with every input copied in from pinned host memory and every result copied back.

Inputs are seeded synthetic tensors of those shapes (no weights or datasets); every
tensor is larger than L2 or read once per step, so no L2 flush is needed.

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--impl uno|reference]
For N > 1 run under torch.distributed.run (one process per GPU); each rank runs its own
replica (data parallel, weak scaling) and the time is the maximum over ranks.
"""
from __future__ import annotations

import argparse
import json
import os
import subprocess
import sys
import tempfile
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from diffusion_drafted_lossless_b200 import workloads as W  # noqa: E402

METRIC = "verified draft rows/s (B=64, block 16, V=151936); TFLOP/s & GB/s vs B200 peak"
UNIT = "rows/s"
WORKLOAD = "uno_step_b64_k16_v151936_qwen3_8b"
LINEARS = W.QWEN3_8B
VERIFY = W.SERVING_VERIFY
LAUNCHES_PER_STEP = 6 + 2 + 2  # 6 projection calls (k and v as one) + verify (row streaming, finish) + TV (mask, rows)


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        d = json.load(open(path))
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained"), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


def profiled_traffic(kernel):
    """DRAM bytes (read + write) per launch of `kernel` from the committed ncu summary
    profiles/<kernel>_traffic.txt ("key: value" lines), or None when there is none or when
    the kernel's source has changed since the capture (the summary records its SHA-256)."""
    import hashlib
    path = os.path.join(ROOT, "profiles", f"{kernel}_traffic.txt")
    if not os.path.exists(path):
        return None
    d = {}
    for line in open(path):
        if ":" in line:
            k, v = line.split(":", 1)
            d[k.strip()] = v.strip()
    src = os.path.join(ROOT, d.get("source", ""))
    if not os.path.isfile(src) or hashlib.sha256(open(src, "rb").read()).hexdigest() != d.get("source_sha256"):
        return None
    return float(d["dram_bytes_per_launch"])


# ---------------------------------------------------------------------------------------
# workload
# ---------------------------------------------------------------------------------------
def gemm_flops(shape, M, rank, n_gated):
    return 2 * M * shape.d_in * shape.d_out + 2 * M * shape.d_in * rank + 2 * n_gated * rank * shape.d_out


def verify_bytes(w):
    """Bytes the verify must read: verifier rows 0..K-1 and drafter rows 1..K-1."""
    return w.B * (2 * w.K - 1) * w.V * 2


def tv_bytes(n, v):
    return n * v * (2 + 2 + 2)  # read teacher and student, write the bf16 gradient


class Step:
    """Device-resident inputs and outputs of one step, and the calls that make it."""

    def __init__(self, torch, dev):
        from diffusion_drafted_lossless_b200 import _lib
        self.torch, self.lib, self.dev = torch, _lib, dev
        bf = torch.bfloat16

        def t(a):
            return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(bf).to(dev)

        w = LINEARS
        self.lin = []
        xs = {}
        for sh in w.shapes:
            inp = W.linear_inputs(w, sh)
            if sh.d_in not in xs:
                xs[sh.d_in] = t(inp["x"])
            y = torch.empty((w.M, sh.d_out), dtype=bf, device=dev)
            ws = torch.empty(_lib.uno_gated_lora_linear_workspace_size(w.M, sh.d_in, sh.d_out, w.rank),
                             dtype=torch.uint8, device=dev)
            self.lin.append(dict(shape=sh, x=xs[sh.d_in], w0=t(inp["w0"]), a=t(inp["a"]), b=t(inp["b"]),
                                 g=torch.from_numpy(inp["gate"]).to(dev), y=y, ws=ws))
        # the calls a step makes: k and v as one call over [W0_k; W0_v], [A_k; A_v] and
        # diag(B_k, B_v) (rank 2r), whose output holds k's columns, then v's
        by = {L["shape"].name: L for L in self.lin}
        self.calls = []
        for L in self.lin:
            name = L["shape"].name
            if name == "v" and "k" in by:
                continue
            if name == "k" and "v" in by:
                K_, V_ = by["k"], by["v"]
                dk, dv, r = K_["shape"].d_out, V_["shape"].d_out, w.rank
                bf_ = torch.zeros((dk + dv, 2 * r), dtype=bf, device=dev)
                bf_[:dk, :r] = K_["b"]
                bf_[dk:, r:] = V_["b"]
                self.calls.append(dict(x=K_["x"], w0=torch.cat([K_["w0"], V_["w0"]], 0).contiguous(),
                                       a=torch.cat([K_["a"], V_["a"]], 0).contiguous(), b=bf_, g=K_["g"],
                                       y=torch.empty((w.M, dk + dv), dtype=bf, device=dev),
                                       ws=torch.empty(_lib.uno_gated_lora_linear_workspace_size(
                                           w.M, K_["shape"].d_in, dk + dv, 2 * r), dtype=torch.uint8, device=dev)))
                continue
            self.calls.append(L)
        self.n_gated = int((W.row_gate(w.M, w.block) > 0).sum())
        self.x_host = {k: v.cpu() for k, v in xs.items()}
        v = VERIFY
        P, Q = W.verify_logits(v)
        self.P, self.Q = t(P).view(v.B, v.K, v.V), t(Q).view(v.B, v.K, v.V)
        self.P_host, self.Q_host = self.P.cpu(), self.Q.cpu()
        self.u = torch.from_numpy(W.verify_uniforms(v)).to(dev)
        self.tokens = torch.empty((v.B, v.K), dtype=torch.int32, device=dev)
        self.count = torch.empty((v.B,), dtype=torch.int32, device=dev)
        self.next = torch.empty((v.B,), dtype=torch.int32, device=dev)
        self.vws = torch.empty(_lib.uno_block_verify_workspace_size(v.B, v.K, v.V, v.top_k, v.top_p),
                               dtype=torch.uint8, device=dev)
        n = v.B * v.K
        self.tv = torch.empty((n,), device=dev)
        self.mean = torch.empty((1,), device=dev)
        self.grad = torch.empty((n, v.V), dtype=bf, device=dev)
        self.tws = torch.empty(_lib.uno_tv_loss_workspace_size(n, v.V), dtype=torch.uint8, device=dev)

    def linears(self):
        for L in self.calls:
            self.lib.uno_gated_lora_linear(L["x"], L["w0"], L["a"], L["b"], L["g"], LINEARS.scale, L["y"],
                                           workspace=L["ws"])

    def verify(self):
        v = VERIFY
        self.lib.uno_block_verify(self.P, self.Q, v.temperature, v.top_k, v.top_p, self.u, self.tokens,
                                  self.count, self.next, workspace=self.vws)

    def tv_loss(self):
        v = VERIFY
        n = v.B * v.K
        self.lib.uno_tv_loss(self.P.view(n, v.V), self.Q.view(n, v.V), self.tv, self.mean, self.grad,
                             workspace=self.tws)

    def run(self):
        self.linears()
        self.verify()
        self.tv_loss()

    # end to end: host inputs in pinned memory, copied in every step; results copied back
    def setup_host(self):
        torch = self.torch

        def pinned_like(t):
            return torch.empty(t.shape, dtype=t.dtype, device="cpu").pin_memory()

        self.hx = {k: v.pin_memory() for k, v in self.x_host.items()}
        self.hP, self.hQ = self.P_host.pin_memory(), self.Q_host.pin_memory()
        self.hu = self.u.cpu().pin_memory()
        # every result of the step: the seven projection outputs, the verify's tokens, counts
        # and correction tokens, the per-token TV, the mean TV and the TV gradient
        self.d_out = [L["y"] for L in self.calls] + [self.tokens, self.count, self.next, self.tv, self.mean, self.grad]
        self.h_out = [pinned_like(t) for t in self.d_out]
        self.h2d = sum(t.numel() * t.element_size() for t in list(self.hx.values()) + [self.hP, self.hQ, self.hu])
        self.d2h = sum(t.numel() * t.element_size() for t in self.h_out)
        # copies in and out run on their own streams, so that one step's results travel back
        # while the next step's inputs travel in (the link is full duplex)
        self.s_in, self.s_out = torch.cuda.Stream(), torch.cuda.Stream()

    def run_e2e(self, steps):
        """`steps` steps through the C ABI from pinned host memory: every step copies all of
        its inputs in and all of its results back. Step i + 1's inputs are copied in once
        step i's kernels are done with the device inputs, step i + 1's kernels start once
        those copies and step i's copy-back are done, and the calling stream ends waiting for
        the last copy-back (so events on it bracket every copy)."""
        torch = self.torch
        cur = torch.cuda.current_stream()
        after = torch.cuda.Event()
        after.record(cur)  # no copy starts before work already queued on the calling stream
        comp_done = out_done = None
        for _ in range(steps):
            self.s_in.wait_event(comp_done if comp_done is not None else after)
            with torch.cuda.stream(self.s_in):
                for k, h in self.hx.items():
                    next(L["x"] for L in self.lin if L["shape"].d_in == k).copy_(h, non_blocking=True)
                self.P.copy_(self.hP, non_blocking=True)
                self.Q.copy_(self.hQ, non_blocking=True)
                self.u.copy_(self.hu, non_blocking=True)
            in_done = torch.cuda.Event()
            in_done.record(self.s_in)
            cur.wait_event(in_done)
            if out_done is not None:
                cur.wait_event(out_done)  # the previous step's results have left
            self.run()
            comp_done = torch.cuda.Event()
            comp_done.record(cur)
            self.s_out.wait_event(comp_done)
            with torch.cuda.stream(self.s_out):
                for h, d in zip(self.h_out, self.d_out):
                    h.copy_(d, non_blocking=True)
            out_done = torch.cuda.Event()
            out_done.record(self.s_out)
        cur.wait_event(out_done)


# ---------------------------------------------------------------------------------------
# clocks during the timed region
# ---------------------------------------------------------------------------------------
class ClockSampler:
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.idx = gpu_index
        self.proc = None
        self.f = None

    def __enter__(self):
        try:
            self.f = tempfile.NamedTemporaryFile("w+", delete=False, suffix=".csv")
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.idx}", f"--query-gpu={self.QUERY}",
                                          "--format=csv,noheader,nounits", "-lms", "50"],
                                         stdout=self.f, stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
        return False

    def summary(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.f.flush()
        rows = [r.split(",") for r in open(self.f.name).read().strip().splitlines() if r.strip()]
        os.unlink(self.f.name)
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            r = [c.strip() for c in r]
            if len(r) < 9:
                continue
            try:
                sm.append(float(r[1]))
                mx = float(r[2])
            except ValueError:
                continue
            for n, v in zip(names, r[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": float(np.median(sm)) if sm else None, "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# ---------------------------------------------------------------------------------------
# CPU oracle baseline (bounded sample)
# ---------------------------------------------------------------------------------------
def oracle_sample(n_seq=2, threads=None):
    """Time the fp64 oracle on a bounded sample of the step: n_seq sequences through the
    verify, the same n_seq * 16 rows through the seven linears and through the TV loss.
    Returns the headline metric (verify rows per second of the oracle's verify) and the
    whole-step rate. `threads` sets the oracle's OpenMP thread count for the call."""
    import oracle
    v = VERIFY
    rows = np.arange(n_seq * v.K)
    P, Q = W.verify_logits(v, rows)
    u = W.verify_uniforms(v)[:n_seq]
    lin = [W.linear_inputs(LINEARS, sh, rows=rows) for sh in LINEARS.shapes]
    Pf, Qf = W.to_f64(P, "bf16"), W.to_f64(Q, "bf16")
    before = oracle.num_threads()
    if threads:
        oracle.set_num_threads(threads)
    try:
        t0 = time.perf_counter()
        oracle.block_verify(Pf.reshape(n_seq, v.K, v.V), Qf.reshape(n_seq, v.K, v.V), u.astype(np.float64),
                            v.temperature, v.top_k, float(np.float32(v.top_p)))
        t1 = time.perf_counter()
        for inp in lin:
            oracle.gated_lora(W.to_f64(inp["x"], "bf16"), W.to_f64(inp["w0"], "bf16"), W.to_f64(inp["a"], "bf16"),
                              W.to_f64(inp["b"], "bf16"), inp["gate"].astype(np.float64), inp["scale"])
        oracle.tv_loss(Pf, Qf, want_grad=True)
        t2 = time.perf_counter()
        cores = oracle.num_threads()
    finally:
        oracle.set_num_threads(before)
    n_rows = n_seq * v.K
    return {"value": n_rows / (t1 - t0), "unit": UNIT, "cores": cores, "kind": "oracle",
            "sample": f"{n_seq} of 64 sequences ({n_rows} rows): the verify alone gives the value "
                      f"({t1 - t0:.2f} s); the same rows through the seven linears and the TV loss too "
                      f"({t2 - t0:.1f} s of fp64 CPU work in all)",
            "step_rows_per_s": n_rows / (t2 - t0)}


# ---------------------------------------------------------------------------------------
def fuse_kv(lw, rank):
    """A layer's projection calls with k and v as one: (shape, W0, A, B) for k and for v
    become one call over [W0_k; W0_v], [A_k; A_v] and diag(B_k, B_v) at rank 2 rank (they
    share their input rows and gate; each adapter acts only on its own outputs)."""
    import torch
    by = {c[0].name: c for c in lw}
    if "k" not in by or "v" not in by or by["k"][0].d_in != by["v"][0].d_in:
        return lw
    (sk, wk, ak, bk), (sv, wv, av, bv) = by["k"], by["v"]
    b = torch.zeros((sk.d_out + sv.d_out, 2 * rank), dtype=bk.dtype, device=bk.device)
    b[:sk.d_out, :rank] = bk
    b[sk.d_out:, rank:] = bv
    kv = (W.LinearShape("kv", sk.d_in, sk.d_out + sv.d_out), torch.cat([wk, wv], 0).contiguous(),
          torch.cat([ak, av], 0).contiguous(), b)
    out = []
    for c in lw:
        if c[0].name == "k":
            out.append(kv)
        elif c[0].name != "v":
            out.append(c)
    return out


def measure_configs(torch, dev, lib, pk, reduce):
    """The other single-GPU configurations of the path, each timed with CUDA events after
    warm-up (inputs resident in HBM, larger than L2): the looped 3B-class step (7 gated
    projections x 22 layers x 2 loops at M = 2048, then the verify at B = 256, K = 8,
    V = 166144, top-p 0.95), its one-loop drafting variant (second loop over the 256 verify
    rows only) and the TV loss at 16384 x 151936. Inputs are drawn on the
    device from a seeded generator with the configurations' distributions."""
    gen = torch.Generator(device=dev)
    bf = torch.bfloat16

    def normal(shape, sigma, seed):
        gen.manual_seed(seed)
        t = torch.randn(shape, generator=gen, device=dev, dtype=torch.float32)
        return (t * sigma).to(bf)

    def timed(fn, reps):
        fn()
        torch.cuda.synchronize()
        s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s.record()
        for _ in range(reps):
            fn()
        e.record()
        torch.cuda.synchronize()
        return reduce(s.elapsed_time(e) / reps)

    out = {}
    # ---- looped 3B-class step: 7 projections x 22 layers x 2 loops, shared across loops ----
    w = W.LOOPED_3B
    M = w.M
    gate = torch.from_numpy(W.row_gate(M, w.block)).to(dev)
    n_gated = int((gate > 0).sum().item())
    xs = {d: normal((M, d), w.x_sigma, 7000 + d) for d in sorted({sh.d_in for sh in w.shapes})}
    layers = []
    for l in range(W.LOOPED_3B_LAYERS):
        lw = []
        for i, sh in enumerate(w.shapes):
            seed = 8000 + 10 * l + i
            lw.append((sh, normal((sh.d_out, sh.d_in), w.w_sigma, seed), normal((w.rank, sh.d_in), w.w_sigma, seed + 3000),
                       normal((sh.d_out, w.rank), w.w_sigma, seed + 6000)))
        layers.append(fuse_kv(lw, w.rank))
    calls = [c[0] for c in layers[0]]  # the call shapes (k and v as one), the same in every layer
    ranks = {c[0].name: c[2].shape[0] for c in layers[0]}
    ys = {sh.name: torch.empty((M, sh.d_out), dtype=bf, device=dev) for sh in calls}
    wss = {sh.name: torch.empty(lib.uno_gated_lora_linear_workspace_size(M, sh.d_in, sh.d_out, ranks[sh.name]),
                                dtype=torch.uint8, device=dev) for sh in calls}

    def looped():
        for _ in range(W.LOOPED_3B_LOOPS):
            for lw in layers:
                for sh, w0, a, b in lw:
                    lib.uno_gated_lora_linear(xs[sh.d_in], w0, a, b, gate, w.scale, ys[sh.name], workspace=wss[sh.name])

    ms = timed(looped, 3)
    fl = W.LOOPED_3B_LAYERS * W.LOOPED_3B_LOOPS * sum(gemm_flops(sh, M, w.rank, n_gated) for sh in w.shapes)
    out["looped_3b_linears_m2048_x44"] = {"ms": ms, "tflops": fl / (ms * 1e-3) / 1e12,
                                          "frac": fl / (ms * 1e-3) / 1e12 / pk["bf16_tflops_sustained"],
                                          "peak": "bf16_tflops_sustained (a seconds-long loop)",
                                          "launches": len(calls) * W.LOOPED_3B_LAYERS * W.LOOPED_3B_LOOPS}
    # ---- one-loop drafting: the draft rows leave after the first loop; the verify rows (the
    # gate-0 rows, laid out first) go through the second loop alone, a prefix of the batch ----
    n_verify = M - n_gated
    gate_vf = torch.cat([torch.zeros(n_verify), torch.ones(n_gated)]).to(dev)
    gate_v = torch.zeros(n_verify, device=dev)
    ys_v = {sh.name: torch.empty((n_verify, sh.d_out), dtype=bf, device=dev) for sh in calls}
    wss_v = {sh.name: torch.empty(lib.uno_gated_lora_linear_workspace_size(n_verify, sh.d_in, sh.d_out,
                                                                           ranks[sh.name]),
                                  dtype=torch.uint8, device=dev) for sh in calls}

    def one_loop():
        for lw in layers:
            for sh, w0, a, b in lw:
                lib.uno_gated_lora_linear(xs[sh.d_in], w0, a, b, gate_vf, w.scale, ys[sh.name], workspace=wss[sh.name])
        for lw in layers:
            for sh, w0, a, b in lw:
                lib.uno_gated_lora_linear(xs[sh.d_in][:n_verify], w0, a, b, gate_v, w.scale, ys_v[sh.name],
                                          workspace=wss_v[sh.name])

    ms1 = timed(one_loop, 3)
    fl1 = W.LOOPED_3B_LAYERS * sum(gemm_flops(sh, M, w.rank, n_gated) + gemm_flops(sh, n_verify, w.rank, 0)
                                   for sh in w.shapes)
    out["looped_3b_linears_one_loop_drafting"] = {
        "ms": ms1, "tflops": fl1 / (ms1 * 1e-3) / 1e12,
        "frac": fl1 / (ms1 * 1e-3) / 1e12 / pk["bf16_tflops_sustained"],
        "saving_vs_two_loops": 1.0 - ms1 / ms, "verify_rows": n_verify,
        "launches": len(calls) * W.LOOPED_3B_LAYERS * 2}
    del layers, xs, ys, wss, ys_v, wss_v
    v = W.LOOPED_VERIFY
    P = normal((v.B, v.K, v.V), v.sigma, 9001)
    Q = (v.rho * P.float() + (1 - v.rho ** 2) ** 0.5 * normal((v.B, v.K, v.V), v.sigma, 9002).float()).to(bf)
    gen.manual_seed(9003)
    u = torch.rand((v.B, v.K, 3), generator=gen, device=dev, dtype=torch.float32)
    tok = torch.empty((v.B, v.K), dtype=torch.int32, device=dev)
    cnt = torch.empty((v.B,), dtype=torch.int32, device=dev)
    nxt = torch.empty((v.B,), dtype=torch.int32, device=dev)
    vws = torch.empty(lib.uno_block_verify_workspace_size(v.B, v.K, v.V, v.top_k, v.top_p), dtype=torch.uint8,
                      device=dev)
    ms = timed(lambda: lib.uno_block_verify(P, Q, v.temperature, v.top_k, v.top_p, u, tok, cnt, nxt, workspace=vws), 5)
    vb = verify_bytes(v)
    out["looped_3b_verify_b256_k8_v166144"] = {"ms": ms, "gbs": vb / (ms * 1e-3) / 1e9,
                                               "frac": vb / (ms * 1e-3) / 1e9 / pk["hbm_gbs"],
                                               "rows_per_s": v.B * v.K / (ms * 1e-3),
                                               "mean_tokens_per_step": float(cnt.float().mean().item())}
    del P, Q, u, vws
    # ---- TV loss at 8 x 2048 response tokens ----
    t = W.TV_LOSS
    T_ = normal((t.N, t.V), t.teacher_sigma, 9101)
    S_ = torch.empty_like(T_)
    for i in range(0, t.N, 2048):  # student = teacher + N(0, 1), in slices to bound the fp32 temporaries
        S_[i:i + 2048] = (T_[i:i + 2048].float() + normal((min(2048, t.N - i), t.V), t.noise_sigma, 9102 + i).float()).to(bf)
    tv = torch.empty((t.N,), device=dev)
    mean = torch.empty((1,), device=dev)
    grad = torch.empty((t.N, t.V), dtype=bf, device=dev)
    tws = torch.empty(lib.uno_tv_loss_workspace_size(t.N, t.V), dtype=torch.uint8, device=dev)
    ms = timed(lambda: lib.uno_tv_loss(T_, S_, tv, mean, grad, workspace=tws), 3)
    tb = tv_bytes(t.N, t.V)
    out["tv_loss_n16384_v151936"] = {"ms": ms, "gbs": tb / (ms * 1e-3) / 1e9, "frac": tb / (ms * 1e-3) / 1e9 / pk["hbm_gbs"]}
    del T_, S_, grad
    torch.cuda.empty_cache()
    # ---- the draft/verify step driver at the serving shapes: noising, the seven gated
    #      projections, the verify, the carried token; eager and replayed from a CUDA graph ----
    try:
        from diffusion_drafted_lossless_b200.driver import DraftVerifyDriver
        d = DraftVerifyDriver(LINEARS, VERIFY)
        counts = []
        for _ in range(3):
            counts.append(d.step()[1].cpu().numpy())
        ms_eager = timed(lambda: d.step(), 10)
        d.capture()
        ms_graph = timed(lambda: d.step(), 20)
        for _ in range(5):
            counts.append(d.step()[1].cpu().numpy())
        out["draft_verify_driver_b64_k16"] = {"ms_eager": ms_eager, "ms_graph": ms_graph,
                                              "tokens_per_forward": DraftVerifyDriver.tokens_per_forward(counts),
                                              "library_launches_per_step": 1 + 7 + 3,
                                              "torch_copies_per_step": 2}
        del d
    except Exception as e:  # reported, never fatal to the bench line
        out["draft_verify_driver_b64_k16"] = {"error": f"{type(e).__name__}: {e}"[:300]}
    torch.cuda.empty_cache()
    return out


def reduce_max(x, dist, device):
    """The maximum of x over all ranks (x itself without a process group): every rank's
    time is the slowest rank's, as the job finishes when the last replica does."""
    if dist is None:
        return float(x)
    import torch
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(rows_per_rank, world, ms_per_step):
    """Rows per second of the whole job: every rank runs its own replica of the step (weak
    scaling), and the step time is the maximum over ranks."""
    return world * rows_per_rank / (ms_per_step * 1e-3)


def run_uno(args):
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300), device_id=dev)

    st = Step(torch, dev)

    def barrier():
        if dist is not None:
            dist.barrier()
        torch.cuda.synchronize()

    def max_over_ranks(x):
        return reduce_max(x, dist, dev)

    for _ in range(args.warmup):
        st.run()
    barrier()
    # CUDA events around each phase of every timed step, on the stream the library launches
    # on (the current stream): the per-phase (and so per-kernel) times come from the timed
    # region itself
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clk:
        time.sleep(0.3)  # let the sampler start before the timed region
        barrier()
        s.record()
        for i in range(args.steps):
            ev[i][0].record()
            st.linears()
            ev[i][1].record()
            st.verify()
            ev[i][2].record()
            st.tv_loss()
            ev[i][3].record()
        e.record()
        barrier()
    ms = max_over_ranks(s.elapsed_time(e) / args.steps)
    clocks = clk.summary()
    ph = {name: max_over_ranks(float(np.mean([ev[i][k].elapsed_time(ev[i][k + 1]) for i in range(args.steps)])))
          for k, name in enumerate(("gated_lora_linears", "block_verify", "tv_loss"))}

    # end to end through the C ABI with host buffers
    st.setup_host()
    st.run_e2e(2)
    barrier()
    with_e2e = max(1, min(args.steps, 5))
    s.record()
    st.run_e2e(with_e2e)
    e.record()
    barrier()
    e2e_ms = max_over_ranks(s.elapsed_time(e) / with_e2e)

    v, pk = VERIFY, peaks()
    configs = None if args.no_configs else measure_configs(torch, dev, st.lib, pk, max_over_ranks)
    rows = v.B * v.K
    # the headline: B * K / t_verify (the verify's mean time inside the timed steps)
    value = whole_job_rate(rows, world, ph["block_verify"])
    gemm_fl = sum(gemm_flops(L["shape"], LINEARS.M, LINEARS.rank, st.n_gated) for L in st.lin)
    # The roofline of the metric's kernel: the value is B * K over the verify's time, and the
    # verify is the streaming kernel (about 80% of it) and the per-sequence finish kernel, both
    # inside one library call; its algorithmic bytes are the logit rows it must read once.
    # The other phases' fractions (the projections against the tensor peak, the TV loss
    # against HBM) are in "phases".
    ach = verify_bytes(v) / (ph["block_verify"] * 1e-3) / 1e9
    roof = {"kernel": "block_verify (row-streaming top-k kernel + per-sequence finish kernel, one call)",
            "bound": "hbm", "achieved": ach, "peak": pk["hbm_gbs"], "unit": "GB/s", "frac": ach / pk["hbm_gbs"],
            "traffic": profiled_traffic("block_verify"), "algorithmic_per_launch": verify_bytes(v)}
    roof["peak_source"] = pk["source"]
    gl_tf = gemm_fl / (ph["gated_lora_linears"] * 1e-3) / 1e12
    vb_gbs = verify_bytes(v) / (ph["block_verify"] * 1e-3) / 1e9
    tv_gbs = tv_bytes(rows, v.V) / (ph["tv_loss"] * 1e-3) / 1e9
    phases = {
        "gated_lora_linears": {"ms": ph["gated_lora_linears"], "tflops": gl_tf,
                               "frac": gl_tf / (pk["bf16_tflops_sustained"] or pk["bf16_tflops"]),
                               "peak": "bf16 sustained (the projections run back to back inside the step)"},
        "block_verify": {"ms": ph["block_verify"], "gbs": vb_gbs, "frac": vb_gbs / pk["hbm_gbs"],
                         "rows_per_s": rows / (ph["block_verify"] * 1e-3)},
        "tv_loss": {"ms": ph["tv_loss"], "gbs": tv_gbs, "frac": tv_gbs / pk["hbm_gbs"],
                    "traffic": profiled_traffic("tv_loss")},
    }
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu:
        cpu = oracle_sample()
        one = oracle_sample(n_seq=1, threads=1)
        cpu["single_thread"] = {"value": one["value"], "cores": one["cores"], "sample": one["sample"],
                                "step_rows_per_s": one["step_rows_per_s"]}
    mean_count = float(st.count.float().mean().item())
    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": WORKLOAD, "B": v.B, "K": v.K, "V": v.V, "global_batch": world * rows,
                       "seq_len": v.K, "parallelism": f"dp{world}",
                       "value": "B*K / mean verify time inside the timed steps (each step: 7 projections, "
                                "verify, TV loss)",
                       "linears": "Qwen3-8B layer: q,k,v,o,gate,up,down at M=1024, rank 128, scale 2; k and v as "
                                  "one call over their concatenated weights",
                       "verify": "T=1, top-k 50, top-p 0.95, drafts sampled in-kernel",
                       "tv": "1024 rows x 151936, teacher=verifier, student=drafter logits",
                       "l2": "no flush: every input (logits 622 MB, weights 380 MB) exceeds L2 or is read once"},
            "roofline": roof, "phases": phases, "configs": configs, "cpu_baseline": cpu,
            "step": {"ms": ms, "rows_per_s": whole_job_rate(rows, world, ms),
                     "what": "the whole step (7 projections + verify + TV loss), device time"},
            "e2e": {"value": world * rows / (e2e_ms * 1e-3), "unit": UNIT, "h2d_bytes_per_step": st.h2d,
                    "d2h_bytes_per_step": st.d2h, "ms_per_step": e2e_ms,
                    "what": "the whole step through the C ABI: activations, logits and uniforms copied in "
                            "from pinned host memory, every result (projection outputs, tokens, counts, "
                            "correction tokens, per-token TV, mean TV, TV gradient) copied back, every "
                            "step; copies in and out on their own streams, one step's copy-back "
                            "overlapping the next step's copy-in"},
            "gpu_launches": LAUNCHES_PER_STEP * args.steps, "clocks": clocks,
            "diagnostics": {"mean_tokens_per_step": mean_count},
        }
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()


def run_reference(args):
    """The reference arm: the fp64 CPU oracle on the host cores, on bounded samples (one
    sequence per step), measured on this arm's metric: verify rows per second."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    for _ in range(args.warmup):
        oracle_sample(n_seq=1)
    runs = [oracle_sample(n_seq=1) for _ in range(args.steps)]
    value = float(np.median([r["value"] for r in runs]))
    base = runs[-1]
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": VERIFY.K / value * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": WORKLOAD, "B": 64, "K": 16, "V": 151936,
                       "sample": "1 of the 64 sequences per step (16 rows)"},
            "cpu_baseline": dict(base, value=value),
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def run_kernel_case(args):
    """One workload alone, for profiling its kernels (a profiling aid, not a bench line):
      looped_verify   the looped 3B-class verify (block 8, V = 166144, top-p 0.95, no top-k)
                      at --case-batch sequences;
      serving_verify  the serving verify (block 16, V = 151936, top-k 50, top-p 0.95) at
                      --case-batch sequences;
      qwen3_linears   the seven Qwen3-8B gated projections at M = 1024 (one call = 7 launches);
      tv_rows         the TV loss and gradient over --case-batch x 16 rows of V = 151936.
    Runs W warm-up calls and then K calls and prints the mean time per call as JSON."""
    import torch
    from diffusion_drafted_lossless_b200 import _lib as lib
    dev = torch.device("cuda", 0)
    gen = torch.Generator(device=dev)
    bf = torch.bfloat16

    def normal(shape, sigma, seed):
        gen.manual_seed(seed)
        return (torch.randn(shape, generator=gen, device=dev) * sigma).to(bf)

    B = args.case_batch
    if args.kernel_case in ("looped_verify", "serving_verify"):
        v = W.LOOPED_VERIFY if args.kernel_case == "looped_verify" else W.SERVING_VERIFY
        P = normal((B, v.K, v.V), v.sigma, 9001)
        Q = (v.rho * P.float() + (1 - v.rho ** 2) ** 0.5 * normal((B, v.K, v.V), v.sigma, 9002).float()).to(bf)
        gen.manual_seed(9003)
        u = torch.rand((B, v.K, 3), generator=gen, device=dev)
        tok = torch.empty((B, v.K), dtype=torch.int32, device=dev)
        cnt = torch.empty((B,), dtype=torch.int32, device=dev)
        nxt = torch.empty((B,), dtype=torch.int32, device=dev)
        ws = torch.empty(lib.uno_block_verify_workspace_size(B, v.K, v.V, v.top_k, v.top_p), dtype=torch.uint8,
                         device=dev)

        def call():
            lib.uno_block_verify(P, Q, v.temperature, v.top_k, v.top_p, u, tok, cnt, nxt, workspace=ws)
    elif args.kernel_case == "qwen3_linears":
        w = LINEARS
        gate = torch.from_numpy(W.row_gate(w.M, w.block)).to(dev)
        lin = []
        for i, sh in enumerate(w.shapes):
            lin.append((normal((w.M, sh.d_in), w.x_sigma, 100 + i), normal((sh.d_out, sh.d_in), w.w_sigma, 200 + i),
                        normal((w.rank, sh.d_in), w.w_sigma, 300 + i), normal((sh.d_out, w.rank), w.w_sigma, 400 + i),
                        torch.empty((w.M, sh.d_out), dtype=bf, device=dev),
                        torch.empty(lib.uno_gated_lora_linear_workspace_size(w.M, sh.d_in, sh.d_out, w.rank),
                                    dtype=torch.uint8, device=dev)))

        def call():
            for x, w0, a, b, y, ws in lin:
                lib.uno_gated_lora_linear(x, w0, a, b, gate, w.scale, y, workspace=ws)
    else:
        n, V = B * 16, W.TV_LOSS.V
        T_ = normal((n, V), 3.0, 9101)
        S_ = (T_.float() + normal((n, V), 1.0, 9102).float()).to(bf)
        tv = torch.empty((n,), device=dev)
        mean = torch.empty((1,), device=dev)
        grad = torch.empty((n, V), dtype=bf, device=dev)
        ws = torch.empty(lib.uno_tv_loss_workspace_size(n, V), dtype=torch.uint8, device=dev)

        def call():
            lib.uno_tv_loss(T_, S_, tv, mean, grad, workspace=ws)

    for _ in range(args.warmup):
        call()
    torch.cuda.synchronize()
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record()
    for _ in range(args.steps):
        call()
    e.record()
    torch.cuda.synchronize()
    print(json.dumps({"kernel_case": args.kernel_case, "batch": B, "calls": args.steps,
                      "ms_per_call": s.elapsed_time(e) / args.steps,
                      "device_status": lib.uno_read_device_status()}), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=300)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["uno", "reference"], default="uno")
    ap.add_argument("--no-cpu", action="store_true", help="skip the CPU oracle baseline")
    ap.add_argument("--no-configs", action="store_true", help="skip the other configurations' measurements")
    ap.add_argument("--kernel-case", choices=["looped_verify", "serving_verify", "qwen3_linears", "tv_rows"],
                    default=None,
                    help="run one workload alone (for kernel profiling) instead of the bench")
    ap.add_argument("--case-batch", type=int, default=32, help="sequences of the --kernel-case workload")
    args = ap.parse_args()
    if args.kernel_case:
        run_kernel_case(args)
        return
    if args.warmup < 3 and args.impl == "uno":
        args.warmup = 3
    if args.gpus > 1 and "WORLD_SIZE" not in os.environ:
        cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={args.gpus}",
               "--master-addr=127.0.0.1", "--master-port=29511", __file__] + sys.argv[1:]
        sys.exit(subprocess.call(cmd))
    if args.impl == "reference":
        run_reference(args)
    else:
        run_uno(args)


if __name__ == "__main__":
    main()
