"""GPU parity of the router of token batches (64 tokens and more): logits in
fp32 with a rigorous error bound per logit, the top-K set taken from them when
the bound separates it from the other experts, the K selected logits then
recomputed in fp64 for their order and weights, and every logit of the other
tokens (near ties at the K-th place) recomputed in fp64.

The ids and their order must equal the fp64 oracle's bit for bit, also for
tokens whose selection the bound cannot settle: router rows that are exact or
near copies of each other (relative difference 2^-20, far below the fp32
bound) put such ties at the boundary.
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
    layer.close()


@pytest.mark.parametrize("T", [64, 300])
def test_near_ties_at_the_boundary_fall_back_to_fp64(gpu, coli, T):
    """Rows 1 and 2 are exact copies of row 0, rows 4 and 5 near copies of row
    3 (relative 2^-20): whenever such a pair straddles the K-th place the
    fp32 bound cannot separate it, and the fp64 fallback decides (equal
    logits to the lower id)."""
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
    # and the forward takes the same routing
    yd = torch.empty((T, c["H"]), device=gpu)
    layer.set_fused(False)
    layer.forward(torch.from_numpy(x).to(gpu), yd)
    layer.sync()
    np.testing.assert_array_equal(layer.plan(T)["ids"], ids_ref)
    layer.close()
