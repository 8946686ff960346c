"""The linear draft/verify step driver on the GPU: each step's block noising, gated
projection and verify agree with the oracle chained the same way (the carried token feeds
the next step's position 0), and the CUDA-graph replay gives the eager results for every
output of every step while the activations change from step to step (also with the
adapter product and the output tiles split over K, whose partial sums are combined by
tickets that carry the execution's epoch)."""
import numpy as np
import pytest
import torch

import oracle
from diffusion_drafted_lossless_b200 import workloads as W
from diffusion_drafted_lossless_b200.driver import DraftVerifyDriver
from tests.gpu_util import NEAR_FP64, decision_path_margin

pytestmark = pytest.mark.gpu

V = W.VerifyWorkload("drv", 4242, B=8, K=16, V=32000, sigma=3.0, rho=0.8, temperature=1.0, top_k=50, top_p=0.95)
L = W.GatedLoraWorkload("drv", 4243, M=8 * 16, block=16, rank=16, scale=2.0,
                        shapes=(W.LinearShape("q", 512, 512), W.LinearShape("k", 512, 128), W.LinearShape("v", 512, 128),
                                W.LinearShape("o", 512, 512), W.LinearShape("gate", 512, 1024),
                                W.LinearShape("up", 512, 1024), W.LinearShape("down", 1024, 512)))


def _run(steps, graph):
    d = DraftVerifyDriver(L, V)
    out = []
    for s in range(steps):
        if graph and s == 1:
            d.capture()
        tok, cnt, nxt = d.step()
        torch.cuda.synchronize()
        out.append((tok.cpu().numpy().copy(), cnt.cpu().numpy().copy(), nxt.cpu().numpy().copy(),
                    d.noised.cpu().numpy().copy(), d.gate.cpu().numpy().copy(),
                    [Lr["y"].float().cpu().numpy() for Lr in d.lin]))
    return d, out


def _oracle_y(d, s, i, gate):
    """The oracle's projection i at step s: that step's activations, the layer's weights."""
    sh = L.shapes[i]
    x = W.linear_inputs(d.pool_linear_workload(s), sh)["x"]
    inp = W.linear_inputs(L, sh)
    return oracle.gated_lora(W.to_f64(x, "bf16"), W.to_f64(inp["w0"], "bf16"), W.to_f64(inp["a"], "bf16"),
                             W.to_f64(inp["b"], "bf16"), gate, float(np.float32(L.scale)))


def test_steps_match_the_chained_oracle():
    d, out = _run(4, graph=False)
    Pf = W.to_f64(d.P_host, "bf16").reshape(V.B, V.K, V.V)
    Qf = W.to_f64(d.Q_host, "bf16").reshape(V.B, V.K, V.V)
    carry = np.full(V.B, -1, np.int32)
    counts = []
    for s, (tok, cnt, nxt, noised, gate, ys) in enumerate(out):
        u, un = d.pool_inputs(s)
        clean = np.zeros((V.B, V.K), np.int32)
        clean[:, 0] = carry
        nz = oracle.block_noise(clean, un, V.V)
        assert (noised == nz["tokens"]).all() and (gate == nz["gate"]).all()
        ref = oracle.block_verify(Pf, Qf, u.astype(np.float64), V.temperature, V.top_k,
                                  float(np.float32(V.top_p)), pos0=nz["tokens"][:, 0])
        for b in range(V.B):
            if decision_path_margin(ref, b) < NEAR_FP64:
                continue  # a decision within rounding of its threshold
            assert cnt[b] == ref["count"][b] and nxt[b] == ref["next"][b], (s, b)
            assert (tok[b] == ref["tokens"][b]).all(), (s, b)
        # the gated projection reads this step's activations and the noise kernel's gate
        yref = _oracle_y(d, s, 0, nz["gate"])
        assert np.abs(ys[0] - yref).max() / np.abs(yref).max() <= 5e-3
        carry = nxt.copy()
        counts.append(cnt)
    tpf = DraftVerifyDriver.tokens_per_forward(counts)
    assert 1.0 <= tpf <= V.K


@pytest.mark.parametrize("env", [{}, {"UNO_LORA_SPLITS": "2"}, {"UNO_LORA_KSPLIT": "2"}],
                         ids=["default", "adapter_split2", "output_ksplit2"])
def test_graph_replay_equals_eager(env, monkeypatch):
    for k, v in env.items():
        monkeypatch.setenv(k, v)
    _, eager = _run(5, graph=False)
    d, graph = _run(5, graph=True)
    for s, (a, b) in enumerate(zip(eager, graph)):
        for x, y in zip(a[:5], b[:5]):
            assert (x == y).all(), s
        for i, (ya, yb) in enumerate(zip(a[5], b[5])):
            assert (ya == yb).all(), (s, i)  # every projection, every step
        # replayed steps (1..4) against the oracle for the step's own activations
        for i in (0, 1, 6):
            yref = _oracle_y(d, s, i, b[4])
            assert np.abs(b[5][i] - yref).max() / np.abs(yref).max() <= 5e-3, (s, i)
