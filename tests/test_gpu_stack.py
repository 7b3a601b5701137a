"""GPU parity of the 30-layer stack (x <- x + MoE_l(RMSNorm(x)), full-size
layers with independent seeded routers and Zipf(1.1) biases per layer,
154.8 GB of int4 experts resident) against the fp64 oracle, through
coli_moe_stack_forward.

The batch of 64 tokens runs the separate-kernel path, a single token the
persistent decode kernel; one sampled token (whose top-8 selection has a
clear margin at every layer, so the fp32 residual stream cannot flip a
near-tie) is followed through all 30 layers by the oracle, generating only
the experts it selects. fp32-path tolerance: max|x - x_ref| <= 1e-3 max|x_ref|.
"""
import numpy as np
import pytest

import oracle
import synth
from tests import cases

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")

LAYERS = 30
FP32_TOL = 1e-3
MARGIN = 1e-3  # smallest accepted gap between the 8th and 9th logit of the sampled token


@pytest.fixture(scope="module")
def coli():
    import int4_expert_ffn_router_b200 as m
    return m


def _oracle_stack(c, x, n_layers):
    """Oracle residual stack for the rows of x (fp32, modified copy returned)
    and the smallest top-k margin met on the way."""
    x = np.ascontiguousarray(x, np.float32).copy()
    cfg = cases.oracle_cfg(c)
    margin = np.inf
    for l in range(n_layers):
        wr = synth.router(0, l, c["E"], c["H"])
        bias = synth.zipf_bias(0, l, c["E"])[0]
        logits = oracle.router_logits(wr, bias, oracle.rmsnorm(x).astype(np.float32))
        srt = np.sort(logits, axis=1)[:, ::-1]
        margin = min(margin, float((srt[:, c["K"] - 1] - srt[:, c["K"]]).min()))
        ids, _ = oracle.topk(logits, c["K"])
        experts = [None] * (c["E"] + c["S"])
        for e in set(ids.ravel().tolist()) | {c["E"] + j for j in range(c["S"])}:
            experts[e] = synth.expert(0, l, e, c["H"], c["I"])
        oracle.stack_step(cfg, wr, bias, experts, x)
    return x, margin


def test_full_stack_30_layers(gpu, coli):
    from tests import gpu_cases
    c = cases.FULL
    T = 64
    layers = []
    try:
        for l in range(LAYERS):
            bias = synth.zipf_bias(0, l, c["E"])[0]
            layers.append(gpu_cases.device_layer(c, seed=0, layer=l, bias=bias, max_tokens=T))
        x = synth.x_f32(7, 0, T, c["H"])
        xd = torch.from_numpy(x).to(gpu)
        coli.stack_forward(layers, xd)                      # batch 64: separate kernels
        # a token with a clear routing margin at every layer
        for t in (17, 5, 40, 63):
            x_ref, margin = _oracle_stack(c, x[t:t + 1], LAYERS)
            if margin > MARGIN:
                break
        assert margin > MARGIN
        x1 = torch.from_numpy(np.ascontiguousarray(x[t:t + 1])).to(gpu)
        coli.stack_forward(layers, x1)                      # batch 1: persistent decode kernel
        torch.cuda.synchronize()
        ref = x_ref.astype(np.float64)
        scale = np.abs(ref).max()
        got64 = xd.cpu().numpy()[t:t + 1].astype(np.float64)
        got1 = x1.cpu().numpy().astype(np.float64)
        assert np.isfinite(got64).all() and np.isfinite(got1).all()
        assert np.abs(got64 - ref).max() <= FP32_TOL * scale
        assert np.abs(got1 - ref).max() <= FP32_TOL * scale
        # every token of the batch went through all layers (residual stream moved, stayed finite)
        xs = xd.cpu().numpy()
        assert np.isfinite(xs).all() and np.abs(xs - x).max() > 0
    finally:
        for L in layers:
            L.close()
        torch.cuda.empty_cache()
