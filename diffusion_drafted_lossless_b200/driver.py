"""Linear draft/verify step driver: the decode step's operations chained on one stream.

Per step (LoopUno project page, "How it works": a block is drafted in one forward with the
LoRA on the noise positions only, the unmodified model verifies it, the longest correct
prefix is kept and the first position is the exact AR token):
  1. uno_block_noise: the block's input tokens — position 0 is the token carried from the
     previous step (its correction token; -1 when every draft was accepted, or at the
     first step), positions 1..K-1 random_uniform noise — and the row gate (0 at
     position 0, 1 on the noise rows);
  2. uno_gated_lora_linear over the seven projections of one decoder layer on the block's
     B x K rows, gated by that row gate;
  3. uno_block_verify with pos0_tokens = the carried tokens (an entry < 0 draws x_0 from
     p_0), drafts sampled in the kernel;
  4. the correction token becomes the next step's carried token.
There is no model: the projections' activations and the verifier / drafter logits are
seeded synthetic inputs of the right shapes (a model's forward would compute them from the
noised tokens). Each step's activations and uniforms come from a small pool and are copied
into the step's input buffers before its launches, so consecutive steps compute on
different data. Every step is the same sequence of launches, so it can be captured once in
a CUDA graph and replayed.
tokens_per_forward() is the mean accepted count per sequence and step.
"""
from __future__ import annotations

import dataclasses

import numpy as np
import torch

from . import _lib
from . import workloads as W


class DraftVerifyDriver:
    def __init__(self, linears: W.GatedLoraWorkload, verify: W.VerifyWorkload, pool: int = 3, device: str = "cuda"):
        v = verify
        assert linears.M == v.B * v.K, "the projections run on the block's B x K rows"
        self.lw, self.v, self.dev = linears, v, torch.device(device)
        bf = torch.bfloat16

        def t(a):
            return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(bf).to(self.dev)

        self.lin = []
        self.x = {}  # the step's activations, one buffer per input width (read by the captured launches)
        for sh in linears.shapes:
            inp = W.linear_inputs(linears, sh)
            ws = torch.empty(_lib.uno_gated_lora_linear_workspace_size(linears.M, sh.d_in, sh.d_out, linears.rank),
                             dtype=torch.uint8, device=self.dev)
            if sh.d_in not in self.x:
                self.x[sh.d_in] = torch.empty((linears.M, sh.d_in), dtype=bf, device=self.dev)
            self.lin.append(dict(shape=sh, x=self.x[sh.d_in], w0=t(inp["w0"]), a=t(inp["a"]), b=t(inp["b"]), ws=ws,
                                 y=torch.empty((linears.M, sh.d_out), dtype=bf, device=self.dev)))
        # pool entry s draws its activations from the workload's seed + s (entry 0 is the
        # workload's own X); they stay on the device and are copied in per step
        self.pool_x = []
        for s in range(pool):
            lw = dataclasses.replace(linears, seed=linears.seed + s)
            self.pool_x.append({d: t(W.linear_inputs(lw, next(sh for sh in linears.shapes if sh.d_in == d))["x"])
                                for d in self.x})
        P, Q = W.verify_logits(v)
        self.P_host, self.Q_host = P, Q
        self.P = t(P).view(v.B, v.K, v.V)
        self.Q = t(Q).view(v.B, v.K, v.V)
        self.pool_u = [W.uniforms(v.seed + 2000 + s, (v.B, v.K, 3)) for s in range(pool)]
        self.pool_noise = [W.uniforms(v.seed + 3000 + s, (v.B, v.K)) for s in range(pool)]
        self.u = torch.empty((v.B, v.K, 3), device=self.dev)
        self.u_noise = torch.empty((v.B, v.K), device=self.dev)
        self.carry = torch.full((v.B, v.K), -1, dtype=torch.int32, device=self.dev)  # column 0 is read
        self.noised = torch.empty((v.B, v.K), dtype=torch.int32, device=self.dev)
        self.gate = torch.empty((v.B * v.K,), device=self.dev)
        self.pos0 = torch.empty((v.B,), dtype=torch.int32, device=self.dev)
        self.tokens = torch.empty((v.B, v.K), dtype=torch.int32, device=self.dev)
        self.count = torch.empty((v.B,), dtype=torch.int32, device=self.dev)
        self.next = torch.empty((v.B,), dtype=torch.int32, device=self.dev)
        self.vws = torch.empty(_lib.uno_block_verify_workspace_size(v.B, v.K, v.V, v.top_k, v.top_p),
                               dtype=torch.uint8, device=self.dev)
        self.steps = 0
        self.graph = None

    def pool_inputs(self, s: int):
        """The uniforms of step s (verify [B, K, 3], noise [B, K])."""
        return self.pool_u[s % len(self.pool_u)], self.pool_noise[s % len(self.pool_noise)]

    def pool_linear_workload(self, s: int) -> W.GatedLoraWorkload:
        """The workload whose X (W.linear_inputs) step s's projections read."""
        return dataclasses.replace(self.lw, seed=self.lw.seed + s % len(self.pool_x))

    def _ops(self):
        v, lw = self.v, self.lw
        _lib.uno_block_noise(self.carry, self.u_noise, v.V, self.noised, self.gate)
        for L in self.lin:
            _lib.uno_gated_lora_linear(L["x"], L["w0"], L["a"], L["b"], self.gate, lw.scale, L["y"],
                                       workspace=L["ws"])
        self.pos0.copy_(self.noised[:, 0])
        _lib.uno_block_verify(self.P, self.Q, v.temperature, v.top_k, v.top_p, self.u, self.tokens, self.count,
                              self.next, pos0_tokens=self.pos0, workspace=self.vws)
        self.carry[:, 0].copy_(self.next)

    def capture(self):
        """Capture one step in a CUDA graph; later steps replay it."""
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            self._ops()
        self.graph = g

    def step(self):
        """One decode step; returns (tokens [B, K], count [B], next [B]) on the device."""
        u, un = self.pool_inputs(self.steps)
        self.u.copy_(torch.from_numpy(u))
        self.u_noise.copy_(torch.from_numpy(un))
        for d, x in self.pool_x[self.steps % len(self.pool_x)].items():
            self.x[d].copy_(x)
        if self.graph is not None:
            self.graph.replay()
        else:
            self._ops()
        self.steps += 1
        return self.tokens, self.count, self.next

    @staticmethod
    def tokens_per_forward(counts) -> float:
        return float(np.mean([np.asarray(c).mean() for c in counts]))
