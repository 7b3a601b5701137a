"""GPU parity of the router of token batches (64 tokens and more): router rows
and tokens as four signed 8-bit digit planes under power-of-two row scales,
every logit from one exact int8 tensor-core GEMM with a rigorous bound of its
representation error, the top-K set, its order and its weights taken from
those logits where the bounds prove them, and every logit of the other tokens
(near ties) recomputed in fp64.

The ids and their order must equal the fp64 oracle's bit for bit, also for
tokens whose selection the bounds cannot settle: router rows that are exact
copies of each other put exact ties at the boundary (fallback), and rows that
differ by a relative 2^-20 put near ties there that the bounds must resolve.
"""
import numpy as np
import pytest

import oracle
import synth
from tests import cases

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def coli():
    import int4_expert_ffn_router_b200 as m
    return m


def _layer(coli, c, wr, L, max_tokens):
    E = c["E"]
    q = np.concatenate([e[0] for e in L["experts"]])
    s = np.concatenate([e[1] for e in L["experts"]])
    nq, ns = synth.expert_sizes(c["H"], c["I"])
    cfg = coli.make_config(c["H"], c["I"], E, c["K"], c["S"], max_tokens)
    return coli.Layer(cfg, wr, L["bias"], q[:E * nq], s[:E * ns], q[E * nq:], s[E * ns:], device=0)


def _route(coli, layer, x, gpu, K):
    T = x.shape[0]
    if x.dtype == np.uint16:
        xd = torch.from_numpy(x.view(np.int16)).to(gpu).view(torch.bfloat16)
    else:
        xd = torch.from_numpy(x).to(gpu)
    ids = torch.empty((T, K), dtype=torch.int32, device=gpu)
    w = torch.empty((T, K), dtype=torch.float32, device=gpu)
    layer.route(xd, ids, w)
    torch.cuda.synchronize()
    return ids.cpu().numpy(), w.cpu().numpy().astype(np.float64)


@pytest.mark.parametrize("T,bf16", [(64, False), (200, False), (64, True), (1000, True)])
def test_certified_router_matches_the_oracle(gpu, coli, T, bf16):
    c = dict(cases.TINY, E=64, K=8)
    bias, _ = synth.zipf_bias(31, 0, c["E"])
    L = cases.host_layer(c, seed=31, bias=bias)
    layer = _layer(coli, c, L["wr"], L, T)
    x = synth.x_bf16(31, T, T, c["H"]) if bf16 else synth.x_f32(31, T, T, c["H"])
    ids, w = _route(coli, layer, x, gpu, c["K"])
    ids_ref, w_ref = oracle.topk(oracle.router_logits(L["wr"], bias, x), c["K"])
    np.testing.assert_array_equal(ids, ids_ref)
    np.testing.assert_allclose(w, w_ref, rtol=0, atol=1e-6)
    # random logits: the bounds (about 1e-9 of ||Wr_e|| ||x_t||) settle every token
    assert layer.router_fallbacks() == (True, 0)
    layer.close()


@pytest.mark.parametrize("T", [64, 300])
def test_near_ties_at_the_boundary_fall_back_to_fp64(gpu, coli, T):
    """Rows 1 and 2 are exact copies of row 0, rows 4 and 5 near copies of row
    3 (relative 2^-20): an exact pair within or at the edge of the top-K has
    equal logits, which no bound separates, so the fp64 fallback decides
    (equal logits to the lower id); the near copies differ by far more than
    the bounds and are settled by them."""
    c = dict(cases.TINY, E=32, K=4)
    L = cases.host_layer(c, seed=32)
    wr = L["wr"].copy()
    wr[0] *= np.float32(8.0)
    wr[1] = wr[0]
    wr[2] = wr[0]
    wr[3] *= np.float32(8.0)
    wr[4] = (wr[3].astype(np.float64) * (1 + 2.0 ** -20)).astype(np.float32)
    wr[5] = (wr[3].astype(np.float64) * (1 - 2.0 ** -20)).astype(np.float32)
    L["bias"] = None
    layer = _layer(coli, c, wr, L, T)
    x = synth.x_f32(32, T, T, c["H"])
    ids, w = _route(coli, layer, x, gpu, c["K"])
    ids_ref, w_ref = oracle.topk(oracle.router_logits(wr, None, x), c["K"])
    np.testing.assert_array_equal(ids, ids_ref)
    np.testing.assert_allclose(w, w_ref, rtol=0, atol=1e-6)
    # the ties really were at the boundary for some tokens: one of a pair selected without the other
    rows = [set(r) for r in ids_ref.tolist()]
    assert any((0 in r) != (1 in r) or (1 in r) != (2 in r) for r in rows)
    assert any((3 in r) != (4 in r) or (3 in r) != (5 in r) for r in rows)
    # some tokens went to the fp64 fallback, and only tokens with a copied row among their
    # K + 1 largest logits (random rows leave no other near tie)
    certified, n_fb = layer.router_fallbacks()
    lg = oracle.router_logits(wr, None, x)
    order = np.argsort(-lg, axis=1, kind="stable")
    near = sum(1 for t in range(T) if {0, 1, 2, 3, 4, 5} & set(order[t, :c["K"] + 1].tolist()))
    assert certified and 0 < n_fb <= near
    # and the forward takes the same routing
    yd = torch.empty((T, c["H"]), device=gpu)
    layer.set_fused(False)
    layer.forward(torch.from_numpy(x).to(gpu), yd)
    layer.sync()
    np.testing.assert_array_equal(layer.plan(T)["ids"], ids_ref)
    layer.close()


@pytest.mark.parametrize("with_bias", [True, False])
def test_extreme_and_zero_rows(gpu, coli, with_bias):
    """Row scales at the ends of the fp32 range (1e30, 1e-30, all-subnormal
    rows) exercise the per-token power-of-two scale; an all-zero row has
    logits equal to the bias, or, without bias, all equal, which no bound
    separates (fp64 fallback: the K lowest ids, equal weights)."""
    c = dict(cases.TINY, E=64, K=8)
    bias = synth.zipf_bias(33, 0, c["E"])[0] if with_bias else None
    L = cases.host_layer(c, seed=33, bias=bias)
    T = 96
    layer = _layer(coli, c, L["wr"], L, T)
    x = synth.x_f32(33, T, T, c["H"]).copy()
    x[3] = 0.0
    x[10] *= np.float32(1e30)
    x[20] *= np.float32(1e-30)
    x[30] = (x[30].astype(np.float64) * 2.0 ** -140).astype(np.float32)  # subnormal fp32 row
    ids, w = _route(coli, layer, x, gpu, c["K"])
    ids_ref, w_ref = oracle.topk(oracle.router_logits(L["wr"], bias, x), c["K"])
    np.testing.assert_array_equal(ids, ids_ref)
    np.testing.assert_allclose(w, w_ref, rtol=0, atol=1e-6)
    if not with_bias:
        np.testing.assert_array_equal(ids[3], np.arange(c["K"]))
        assert layer.router_fallbacks()[1] >= 1
    layer.close()


@pytest.mark.parametrize("bf16", [True, False])
def test_full_size_router_every_token(gpu, coli, bf16):
    """The full-size router (256 experts, hidden 6144) on 2048 tokens with
    Zipf bias: ids and order of every token bit-exact against the fp64
    oracle, weights within 1e-6, and no token left to the fp64 fallback. The
    layer is rank 0 of a 32-way expert-parallel split (8 routed experts in
    HBM, no expert weights loaded): routing through `coli_moe_route` always
    covers all experts."""
    c = cases.FULL
    T, E, K = 2048, c["E"], c["K"]
    wr = synth.router(40, 0, E, c["H"])
    bias, _ = synth.zipf_bias(40, 0, E)
    cfg = coli.make_config(c["H"], c["I"], E, K, c["S"], T)
    layer = coli.Layer(cfg, wr, bias, device=0, ep=(0, 32))
    x = synth.x_bf16(40, 0, T, c["H"]) if bf16 else synth.x_f32(40, 0, T, c["H"])
    ids, w = _route(coli, layer, x, gpu, K)
    ids_ref, w_ref = oracle.topk(oracle.router_logits(wr, bias, x), K)
    np.testing.assert_array_equal(ids, ids_ref)
    np.testing.assert_allclose(w, w_ref, rtol=0, atol=1e-6)
    assert layer.router_fallbacks() == (True, 0)
    print(f"full-size router, {T} {'bf16' if bf16 else 'fp32'} tokens: ids bit-exact, max |w - w_ref| "
          f"{np.abs(w - w_ref).max():.2e}")
    layer.close()
