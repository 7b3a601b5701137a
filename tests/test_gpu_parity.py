"""GPU parity: the CUDA path through the C ABI against the fp64 oracle.

Routing (ids, order, weights' selection), the batch-union plan (counts,
offsets, unique set, permutation) are compared bit for bit; outputs within
these tolerances:
  fp32 path: max|y - y_ref| <= 1e-3 * max|y_ref|
  bf16 path: ||y - y_ref||_2 <= 5e-3 * ||y_ref||_2
"""
import numpy as np
import pytest

import oracle
import synth
from tests import cases

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")

FP32_TOL = 1e-3
BF16_TOL = 5e-3


@pytest.fixture(scope="module")
def coli():
    import int4_expert_ffn_router_b200 as m
    return m


def _bf16_to_f32(a):
    return (a.astype(np.uint32) << 16).view(np.float32)


def _check_plan(plan, ids_ref, E):
    u = oracle.union(ids_ref, E)
    np.testing.assert_array_equal(plan["ids"], ids_ref)
    np.testing.assert_array_equal(plan["cnt"], u["cnt"])
    np.testing.assert_array_equal(plan["off"], u["off"])
    np.testing.assert_array_equal(plan["unique"], u["unique"])
    np.testing.assert_array_equal(plan["pos"], u["pos"])
    np.testing.assert_array_equal(plan["tok"], u["tok"])


def _max_rel(y, y_ref):
    return float(np.abs(y - y_ref).max() / np.abs(y_ref).max())


def _l2_rel(y, y_ref):
    return float(np.linalg.norm(y - y_ref) / np.linalg.norm(y_ref))


def _host_layer_to_device(coli, c, L, max_tokens, bias=None):
    E, S = c["E"], c["S"]
    q = np.concatenate([e[0] for e in L["experts"]])
    s = np.concatenate([e[1] for e in L["experts"]])
    nq, ns = synth.expert_sizes(c["H"], c["I"])
    cfg = coli.make_config(c["H"], c["I"], E, c["K"], S, max_tokens)
    return coli.Layer(cfg, L["wr"], bias, q[:E * nq], s[:E * ns], q[E * nq:] if S else None,
                      s[E * ns:] if S else None, device=0)


# ------------------------------------------------------------------ generator


def test_device_generator_matches_host(gpu):
    H, I = 512, 256
    nq, ns = synth.expert_sizes(H, I)
    q = torch.empty(3 * nq, dtype=torch.uint8, device=gpu)
    s = torch.empty(3 * ns, dtype=torch.int16, device=gpu)
    synth.expert_dev(11, 2, 5, 3, H, I, q.data_ptr(), s.data_ptr())
    torch.cuda.synchronize()
    for i in range(3):
        qh, sh = synth.expert(11, 2, 5 + i, H, I)
        assert np.array_equal(q[i * nq:(i + 1) * nq].cpu().numpy(), qh)
        assert np.array_equal(s[i * ns:(i + 1) * ns].cpu().numpy().view(np.uint16), sh)
    wr = torch.empty(16 * H, dtype=torch.float32, device=gpu)
    synth.router_dev(11, 2, 16, H, wr.data_ptr())
    x = torch.empty(3 * H, dtype=torch.float32, device=gpu)
    synth.x_dev(11, 7, 3, H, 0, x.data_ptr())
    xb = torch.empty(3 * H, dtype=torch.int16, device=gpu)
    synth.x_dev(11, 7, 3, H, 1, xb.data_ptr())
    torch.cuda.synchronize()
    assert np.array_equal(wr.cpu().numpy().reshape(16, H), synth.router(11, 2, 16, H))
    assert np.array_equal(x.cpu().numpy().reshape(3, H), synth.x_f32(11, 7, 3, H))
    assert np.array_equal(xb.cpu().numpy().view(np.uint16).reshape(3, H), synth.x_bf16(11, 7, 3, H))


def test_device_generator_matches_host_full_size_expert(gpu):
    H, I = 6144, 2048
    nq, ns = synth.expert_sizes(H, I)
    q = torch.empty(nq, dtype=torch.uint8, device=gpu)
    s = torch.empty(ns, dtype=torch.int16, device=gpu)
    synth.expert_dev(0, 0, 256, 1, H, I, q.data_ptr(), s.data_ptr())
    torch.cuda.synchronize()
    qh, sh = synth.expert(0, 0, 256, H, I)
    assert np.array_equal(q.cpu().numpy(), qh)
    assert np.array_equal(s.cpu().numpy().view(np.uint16), sh)


# ----------------------------------------------------------------- tiny layer


@pytest.fixture(scope="module")
def tiny(coli):
    c = cases.TINY
    L = cases.host_layer(c, seed=c["seed"])
    layer = _host_layer_to_device(coli, c, L, max_tokens=64)
    yield c, L, layer
    layer.close()


@pytest.mark.parametrize("T", [4, 1, 5, 13, 64])
def test_tiny_fp32_parity(gpu, tiny, T):
    c, L, layer = tiny
    x = synth.x_f32(c["seed"], T, T, c["H"])
    xd = torch.from_numpy(x).to(gpu)
    yd = torch.full_like(xd, float("nan"))
    layer.forward(xd, yd)
    torch.cuda.synchronize()
    y_ref, ids_ref, w_ref = oracle.moe_forward(cases.oracle_cfg(c), L["wr"], None, L["experts"], x)
    plan = layer.plan(T)
    _check_plan(plan, ids_ref, c["E"])
    np.testing.assert_allclose(plan["weights"], w_ref, rtol=0, atol=1e-6)
    assert _max_rel(yd.cpu().numpy().astype(np.float64), y_ref) <= FP32_TOL


@pytest.mark.parametrize("fused", [True, False])
@pytest.mark.parametrize("T", [1, 2, 3, 4])
def test_tiny_small_batch_both_paths(gpu, tiny, T, fused):
    """n_tokens <= 4 runs the persistent kernel by default; both paths must
    route identically and match the oracle."""
    c, L, layer = tiny
    layer.set_fused(fused)
    try:
        x = synth.x_f32(c["seed"], 50 + T, T, c["H"])
        xd = torch.from_numpy(x).to(gpu)
        yd = torch.full_like(xd, float("nan"))
        for _ in range(3):  # repeated launches reuse the control block
            layer.forward(xd, yd)
        layer.sync()
        y_ref, ids_ref, w_ref = oracle.moe_forward(cases.oracle_cfg(c), L["wr"], None, L["experts"], x)
        plan = layer.plan(T)
        _check_plan(plan, ids_ref, c["E"])
        np.testing.assert_allclose(plan["weights"], w_ref, rtol=0, atol=1e-6)
        assert _max_rel(yd.cpu().numpy().astype(np.float64), y_ref) <= FP32_TOL
    finally:
        layer.set_fused(True)


def test_tiny_bf16_parity(gpu, tiny):
    c, L, layer = tiny
    T = 6
    xb = synth.x_bf16(c["seed"], 100, T, c["H"])
    xd = torch.from_numpy(xb.view(np.int16)).to(gpu).view(torch.bfloat16)
    yd = torch.empty_like(xd)
    layer.forward(xd, yd)
    torch.cuda.synchronize()
    y_ref, ids_ref, _ = oracle.moe_forward(cases.oracle_cfg(c), L["wr"], None, L["experts"], xb)
    _check_plan(layer.plan(T), ids_ref, c["E"])
    y = _bf16_to_f32(yd.view(torch.int16).cpu().numpy().view(np.uint16)).astype(np.float64)
    assert _l2_rel(y, y_ref) <= BF16_TOL


def test_tiny_route_entry_point(gpu, tiny):
    c, L, layer = tiny
    T = 9
    x = synth.x_f32(c["seed"], 200, T, c["H"])
    xd = torch.from_numpy(x).to(gpu)
    ids = torch.empty((T, c["K"]), dtype=torch.int32, device=gpu)
    w = torch.empty((T, c["K"]), dtype=torch.float32, device=gpu)
    layer.route(xd, ids, w)
    torch.cuda.synchronize()
    logits = oracle.router_logits(L["wr"], None, x)
    ids_ref, w_ref = oracle.topk(logits, c["K"])
    np.testing.assert_array_equal(ids.cpu().numpy(), ids_ref)
    np.testing.assert_allclose(w.cpu().numpy(), w_ref, rtol=0, atol=1e-6)


def test_zero_tokens_is_a_no_op(gpu, tiny):
    c, L, layer = tiny
    x = torch.zeros((1, c["H"]), device=gpu)
    y = torch.full_like(x, 7.0)
    layer.forward(x, y, n_tokens=0)
    torch.cuda.synchronize()
    assert torch.all(y == 7.0)


def test_too_many_tokens_is_rejected(gpu, tiny, coli):
    c, L, layer = tiny
    x = torch.zeros((65, c["H"]), device=gpu)
    y = torch.empty_like(x)
    with pytest.raises(coli.ColiError) as e:
        layer.forward(x, y)
    assert e.value.status == coli.COLI_EINVAL


@pytest.mark.parametrize("K,S", [(16, 1), (1, 0), (3, 2)])
def test_tiny_variants(gpu, coli, K, S):
    """All experts selected (K = E), no shared expert, two shared experts."""
    c = dict(cases.TINY, K=K, S=S)
    L = cases.host_layer(c, seed=3)
    bias = synth.zipf_bias(3, 0, c["E"], kappa=2.0)[0]
    layer = _host_layer_to_device(coli, c, L, max_tokens=8, bias=bias)
    T = 7
    x = synth.x_f32(3, 0, T, c["H"])
    xd = torch.from_numpy(x).to(gpu)
    yd = torch.empty_like(xd)
    layer.forward(xd, yd)
    torch.cuda.synchronize()
    L["bias"] = bias
    y_ref, ids_ref, _ = oracle.moe_forward(cases.oracle_cfg(c), L["wr"], bias, L["experts"], x)
    _check_plan(layer.plan(T), ids_ref, c["E"])
    assert _max_rel(yd.cpu().numpy().astype(np.float64), y_ref) <= FP32_TOL
    layer.close()


def test_tiny_stack_matches_oracle_steps(gpu, coli):
    c = cases.TINY
    layers_h = [cases.host_layer(c, seed=5, layer=l) for l in range(3)]
    layers = [_host_layer_to_device(coli, c, Lh, max_tokens=8) for Lh in layers_h]
    T = 3
    x = (synth.x_f32(5, 0, T, c["H"]) * 4.0).astype(np.float32)
    xd = torch.from_numpy(x.copy()).to(gpu)
    coli.stack_forward(layers, xd)
    torch.cuda.synchronize()
    xr = x.copy()
    for Lh in layers_h:
        oracle.stack_step(cases.oracle_cfg(c), Lh["wr"], None, Lh["experts"], xr)
    assert _max_rel(xd.cpu().numpy().astype(np.float64), xr.astype(np.float64)) <= FP32_TOL
    for l in layers:
        l.close()


# ------------------------------------------------------------- full-size layer


@pytest.fixture(scope="module")
def full(coli):
    from tests import gpu_cases
    c = cases.FULL
    layer = gpu_cases.device_layer(c, seed=0, layer=0, max_tokens=64)
    wr = synth.router(0, 0, c["E"], c["H"])
    yield c, layer, wr
    layer.close()


def _oracle_for_tokens(c, wr, bias, x, seed=0, layer=0):
    """Oracle forward for the rows of x, generating only the experts they select."""
    logits = oracle.router_logits(wr, bias, x)
    ids, _ = oracle.topk(logits, c["K"])
    need = set(ids.ravel().tolist()) | {c["E"] + j for j in range(c["S"])}
    experts = [None] * (c["E"] + c["S"])
    for e in need:
        experts[e] = synth.expert(seed, layer, e, c["H"], c["I"])
    return oracle.moe_forward(cases.oracle_cfg(c), wr, bias, experts, x)


@pytest.mark.parametrize("step,fused", [(0, True), (1, True), (0, False)])
def test_full_decode_batch1(gpu, full, step, fused):
    """One full-size layer (H 6144, I 2048, 256 experts top-8 + shared), one token."""
    c, layer, wr = full
    layer.set_fused(fused)
    x = synth.x_f32(1000 + step, 0, 1, c["H"])
    xd = torch.from_numpy(x).to(gpu)
    yd = torch.empty_like(xd)
    layer.forward(xd, yd)
    layer.sync()
    layer.set_fused(True)
    y_ref, ids_ref, _ = _oracle_for_tokens(c, wr, None, x)
    _check_plan(layer.plan(1), ids_ref, c["E"])
    nu, nbytes = layer.stats()
    assert nu == 8 and nbytes == 9 * 20_054_016 + 6_291_456
    assert _max_rel(yd.cpu().numpy().astype(np.float64), y_ref) <= FP32_TOL


@pytest.mark.parametrize("T", [2, 4])
def test_full_decode_small_batch_fused_matches_oracle(gpu, full, T):
    """T tokens through the persistent kernel (no router bias): routing and
    union bit-exact, every output against the oracle. At 2 tokens the
    kernel's producer stages each item's token operands into a buffer per
    item-queue slot; at 4 the consumers stage them into one buffer."""
    c, layer, wr = full
    x = synth.x_f32(4000, 0, T, c["H"])
    xd = torch.from_numpy(x).to(gpu)
    yd = torch.empty_like(xd)
    layer.forward(xd, yd)
    layer.sync()
    y_ref, ids_ref, _ = _oracle_for_tokens(c, wr, None, x)
    _check_plan(layer.plan(T), ids_ref, c["E"])
    assert _max_rel(yd.cpu().numpy().astype(np.float64), y_ref) <= FP32_TOL


def test_full_decode_batch32_zipf(gpu, coli):
    """Batch 32 with Zipf(1.1)-skewed routing: routing and union bit-exact for
    every token; outputs of two sampled tokens against the oracle."""
    from tests import gpu_cases
    c = cases.FULL
    bias, _ = synth.zipf_bias(0, 0, c["E"])
    layer = gpu_cases.device_layer(c, seed=0, layer=0, bias=bias, max_tokens=32)
    T = 32
    x = synth.x_f32(2000, 0, T, c["H"])
    xd = torch.from_numpy(x).to(gpu)
    yd = torch.empty_like(xd)
    layer.forward(xd, yd)
    torch.cuda.synchronize()
    wr = synth.router(0, 0, c["E"], c["H"])
    logits = oracle.router_logits(wr, bias, x)
    ids_ref, _ = oracle.topk(logits, c["K"])
    _check_plan(layer.plan(T), ids_ref, c["E"])
    nu, nbytes = layer.stats()
    assert nu == len(set(ids_ref.ravel().tolist()))
    y = yd.cpu().numpy().astype(np.float64)
    for t in (0, 17):
        y_ref, _, _ = _oracle_for_tokens(c, wr, bias, x[t:t + 1])
        assert _max_rel(y[t:t + 1], y_ref) <= FP32_TOL
    layer.close()


def test_full_prefill_2048_bf16_zipf(gpu, coli):
    """Prefill of 2048 bf16 tokens with Zipf(1.1)-skewed routing: routing and
    union bit-exact for all tokens; outputs of sampled tokens within the bf16
    tolerance."""
    from tests import gpu_cases
    c = cases.FULL
    bias, _ = synth.zipf_bias(0, 0, c["E"])
    layer = gpu_cases.device_layer(c, seed=0, layer=0, bias=bias, max_tokens=2048)
    T = 2048
    xb = synth.x_bf16(3000, 0, T, c["H"])
    xd = torch.from_numpy(xb.view(np.int16)).to(gpu).view(torch.bfloat16)
    yd = torch.empty_like(xd)
    layer.forward(xd, yd)
    torch.cuda.synchronize()
    wr = synth.router(0, 0, c["E"], c["H"])
    ids_ref, _ = oracle.topk(oracle.router_logits(wr, bias, xb), c["K"])
    _check_plan(layer.plan(T), ids_ref, c["E"])
    assert layer.stats()[0] == len(set(ids_ref.ravel().tolist()))
    y = _bf16_to_f32(yd.view(torch.int16).cpu().numpy().view(np.uint16)).astype(np.float64)
    for t in (0, 1234, 2047):
        y_ref, _, _ = _oracle_for_tokens(c, wr, bias, xb[t:t + 1])
        assert _l2_rel(y[t:t + 1], y_ref) <= BF16_TOL
    layer.close()
