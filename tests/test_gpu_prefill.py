"""GPU parity of the tensor-core path (the tcgen05 grouped GEMMs of bf16
batches) against the fp64 oracle, through the C ABI. The tiny layer here has
the persistent small-batch kernel switched off, so every batch size, down to
5 tokens, runs the batch kernels.

Routing and the batch-union plan bit for bit; outputs within the bf16-path
tolerance ||y - y_ref||_2 <= 5e-3 ||y_ref||_2. Cases span ragged token tiles
(an expert with more tokens than one tile holds, tiles of 1..15 tokens), the
shared expert over every token, K = E, no shared expert and two shared
experts, and the switch back to the CUDA-core kernels.
"""
import numpy as np
import pytest

import oracle
import synth
from tests import cases
from tests.test_gpu_parity import (BF16_TOL, _bf16_to_f32, _check_plan, _host_layer_to_device, _l2_rel,
                                   _oracle_for_tokens)

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")

TILE = 128  # tokens per tensor-core tile


@pytest.fixture(scope="module")
def coli():
    import int4_expert_ffn_router_b200 as m
    return m


def _bf16_x(seed, step, T, H, gpu):
    xb = synth.x_bf16(seed, step, T, H)
    return xb, torch.from_numpy(xb.view(np.int16)).to(gpu).view(torch.bfloat16)


def _y_f64(yd):
    return _bf16_to_f32(yd.view(torch.int16).cpu().numpy().view(np.uint16)).astype(np.float64)


@pytest.fixture(scope="module")
def tiny_big(coli):
    """The tiny layer (H 512, I 256, 16 experts top-2, 1 shared) with room for 1024 tokens."""
    c = cases.TINY
    L = cases.host_layer(c, seed=c["seed"])
    layer = _host_layer_to_device(coli, c, L, max_tokens=1024)
    layer.set_tensor_cores(True)  # the shapes qualify: raises otherwise
    layer.set_fused(False)        # small batches too take the batch kernels
    yield c, L, layer
    layer.close()


@pytest.mark.parametrize("T", [5, 13, 64, 300, 1024])
def test_tiny_bf16_tensor_cores(gpu, tiny_big, T):
    c, L, layer = tiny_big
    xb, xd = _bf16_x(c["seed"], 400 + T, T, c["H"], gpu)
    yd = torch.full_like(xd, float("nan"))
    layer.forward(xd, yd)
    layer.sync()
    y_ref, ids_ref, w_ref = oracle.moe_forward(cases.oracle_cfg(c), L["wr"], None, L["experts"], xb)
    plan = layer.plan(T)
    _check_plan(plan, ids_ref, c["E"])
    np.testing.assert_allclose(plan["weights"], w_ref, rtol=0, atol=1e-6)
    y = _y_f64(yd)
    assert np.isfinite(y).all()
    assert _l2_rel(y, y_ref) <= BF16_TOL
    # per token as well: no token may carry a large share of the error
    for t in range(0, T, max(1, T // 16)):
        assert _l2_rel(y[t], y_ref[t]) <= 2 * BF16_TOL
    if T == 1024:
        assert plan["cnt"].max() > TILE  # an expert spans several token tiles


def test_tiny_bf16_cuda_core_switch(gpu, tiny_big):
    """set_tensor_cores(False) sends bf16 batches to the CUDA-core kernels;
    both paths match the oracle and each other."""
    c, L, layer = tiny_big
    T = 40
    xb, xd = _bf16_x(c["seed"], 77, T, c["H"], gpu)
    y_tc = torch.empty_like(xd)
    y_cc = torch.empty_like(xd)
    layer.forward(xd, y_tc)
    layer.set_tensor_cores(False)
    try:
        layer.forward(xd, y_cc)
    finally:
        layer.set_tensor_cores(True)
    layer.sync()
    y_ref, _, _ = oracle.moe_forward(cases.oracle_cfg(c), L["wr"], None, L["experts"], xb)
    a, b = _y_f64(y_tc), _y_f64(y_cc)
    assert _l2_rel(a, y_ref) <= BF16_TOL
    assert _l2_rel(b, y_ref) <= BF16_TOL
    assert _l2_rel(a, b) <= BF16_TOL


def test_tiny_bf16_repeatable(gpu, tiny_big):
    """Back-to-back launches reuse the tile list and workspace: the same input
    gives the same routing and outputs equal up to the order of fp32 additions."""
    c, L, layer = tiny_big
    T = 200
    xb, xd = _bf16_x(c["seed"], 5, T, c["H"], gpu)
    ys = []
    for _ in range(3):
        yd = torch.empty_like(xd)
        layer.forward(xd, yd)
        ys.append(_y_f64(yd))
    layer.sync()
    for y in ys[1:]:
        assert _l2_rel(y, ys[0]) <= 1e-3


@pytest.mark.parametrize("K,S", [(16, 1), (1, 0), (3, 2)])
def test_tiny_bf16_variants(gpu, coli, K, S):
    """All experts selected (K = E), no shared expert, two shared experts,
    with Zipf-skewed routing."""
    c = dict(cases.TINY, K=K, S=S)
    L = cases.host_layer(c, seed=3)
    bias = synth.zipf_bias(3, 0, c["E"], kappa=2.0)[0]
    layer = _host_layer_to_device(coli, c, L, max_tokens=160, bias=bias)
    layer.set_tensor_cores(True)
    T = 150
    xb, xd = _bf16_x(3, 0, T, c["H"], gpu)
    yd = torch.empty_like(xd)
    layer.forward(xd, yd)
    layer.sync()
    y_ref, ids_ref, _ = oracle.moe_forward(cases.oracle_cfg(c), L["wr"], bias, L["experts"], xb)
    _check_plan(layer.plan(T), ids_ref, c["E"])
    assert _l2_rel(_y_f64(yd), y_ref) <= BF16_TOL
    layer.close()


def test_tiny_bf16_large_activations(gpu, tiny_big):
    """Inputs far from unit scale (rows scaled by 2^-20 .. 2^20) take the
    power-of-two token scales: no overflow, same relative accuracy."""
    c, L, layer = tiny_big
    T = 24
    xb = synth.x_bf16(c["seed"], 900, T, c["H"])
    xf = _bf16_to_f32(xb.view(np.uint16)).reshape(T, c["H"])
    scale = np.float32(2.0) ** np.linspace(-20, 20, T).astype(np.int32)[:, None].astype(np.float32)
    xs = (xf * scale).astype(np.float32)
    xsb = (xs.view(np.uint32) >> 16).astype(np.uint16)  # exact: power-of-two scaling of bf16 values
    xd = torch.from_numpy(xsb.view(np.int16)).to(gpu).view(torch.bfloat16)
    yd = torch.empty_like(xd)
    layer.forward(xd, yd)
    layer.sync()
    y_ref, ids_ref, _ = oracle.moe_forward(cases.oracle_cfg(c), L["wr"], None, L["experts"], xsb)
    _check_plan(layer.plan(T), ids_ref, c["E"])
    y = _y_f64(yd)
    assert np.isfinite(y).all()
    for t in range(T):
        assert _l2_rel(y[t], y_ref[t]) <= 2 * BF16_TOL


def test_full_prefill_2048_hot_expert_tokens(gpu, coli):
    """Full-size prefill (2048 bf16 tokens, Zipf(1.1) routing): the tokens of
    the most popular expert (several token tiles) and of a one-token expert
    match the oracle."""
    from tests import gpu_cases
    c = cases.FULL
    bias, _ = synth.zipf_bias(0, 0, c["E"])
    layer = gpu_cases.device_layer(c, seed=0, layer=0, bias=bias, max_tokens=2048)
    layer.set_tensor_cores(True)
    T = 2048
    xb, xd = _bf16_x(3001, 0, T, c["H"], gpu)
    yd = torch.empty_like(xd)
    layer.forward(xd, yd)
    layer.sync()
    wr = synth.router(0, 0, c["E"], c["H"])
    ids_ref, _ = oracle.topk(oracle.router_logits(wr, bias, xb), c["K"])
    plan = layer.plan(T)
    _check_plan(plan, ids_ref, c["E"])
    cnt = plan["cnt"]
    hot = int(np.argmax(cnt))
    assert cnt[hot] > TILE
    hot_tokens = np.nonzero((ids_ref == hot).any(axis=1))[0]
    pick = list(hot_tokens[[0, len(hot_tokens) // 2, -1]])
    rare = [e for e in range(c["E"]) if cnt[e] == cnt[cnt > 0].min()]
    pick.append(int(np.nonzero((ids_ref == rare[0]).any(axis=1))[0][0]))
    y = _y_f64(yd)
    for t in pick:
        y_ref, _, _ = _oracle_for_tokens(c, wr, bias, xb[t:t + 1])
        assert _l2_rel(y[t:t + 1], y_ref) <= BF16_TOL
    layer.close()


@pytest.mark.parametrize("T", [5, 40, 200])
def test_tiny_fp32_tensor_cores_and_cuda_cores(gpu, tiny_big, T):
    """fp32 batches on the batch kernels run on the CUDA cores by default; mode
    2 runs them on the tensor cores with hi + lo operand rows (tiles of up to
    64 tokens). Both meet the fp32-path tolerance on one layer."""
    c, L, layer = tiny_big
    x = synth.x_f32(c["seed"], 600 + T, T, c["H"])
    xd = torch.from_numpy(x).to(gpu)
    y_tc = torch.full_like(xd, float("nan"))
    y_cc = torch.full_like(xd, float("nan"))
    layer.forward(xd, y_cc)
    layer.set_tensor_cores(2)
    try:
        layer.forward(xd, y_tc)
    finally:
        layer.set_tensor_cores(1)
    layer.sync()
    y_ref, ids_ref, _ = oracle.moe_forward(cases.oracle_cfg(c), L["wr"], None, L["experts"], x)
    _check_plan(layer.plan(T), ids_ref, c["E"])
    scale = np.abs(y_ref).max()
    for y in (y_tc, y_cc):
        yv = y.cpu().numpy().astype(np.float64)
        assert np.isfinite(yv).all()
        assert np.abs(yv - y_ref).max() <= 1e-3 * scale
