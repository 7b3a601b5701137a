"""GPU parity of the adaptive expert top-p routing variant (opt-in;
"colibri: 1300 lines of C ...", usage section: topp=0.7 expert top-p).

Against the oracle on the same seeded inputs: the kept prefix of every
token's slots is bit-exact (ids and order), each dropped slot reports slot 0's
id with weight 0, the kept weights are within 1e-6, the batch-union's unique
experts are exactly the distinct kept experts, and the outputs are within the
path's tolerance. The seeded inputs are checked to keep every token's running
weight sum away from p (the decision is fp64 on both sides; only a sum within
rounding of p could go either way).
"""
import numpy as np
import pytest

import oracle
import synth
from tests import cases

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")

C4 = dict(cases.TINY, K=4)
P = 0.7


@pytest.fixture(scope="module")
def coli():
    import int4_expert_ffn_router_b200 as m
    return m


@pytest.fixture(scope="module")
def host():
    bias, _ = synth.zipf_bias(7, 0, C4["E"])
    return cases.host_layer(C4, seed=7, bias=bias)


def _layer(coli, L, max_tokens=64, resident=None):
    c = C4
    E = c["E"]
    q = np.concatenate([e[0] for e in L["experts"]])
    s = np.concatenate([e[1] for e in L["experts"]])
    nq, ns = synth.expert_sizes(c["H"], c["I"])
    cfg = coli.make_config(c["H"], c["I"], E, c["K"], c["S"], max_tokens)
    return coli.Layer(cfg, L["wr"], L["bias"], q[:E * nq], s[:E * ns], q[E * nq:], s[E * ns:], device=0,
                      resident=resident)


def _margin_ok(logits, K, p):
    _, w = oracle.topk(logits, K)
    cum = np.cumsum(w, axis=1)
    return np.abs(cum - p).min() > 1e-9


def _check_plan(plan, ids_ref, w_ref):
    keep = (ids_ref >= 0).sum(axis=1)
    for t in range(ids_ref.shape[0]):
        n = keep[t]
        assert plan["ids"][t, :n].tolist() == ids_ref[t, :n].tolist(), f"token {t}"
        assert (plan["ids"][t, n:] == ids_ref[t, 0]).all()
        assert (plan["weights"][t, n:] == 0).all()
        np.testing.assert_allclose(plan["weights"][t, :n], w_ref[t, :n], rtol=0, atol=1e-6)
    kept = set(ids_ref[ids_ref >= 0].ravel().tolist())
    assert sorted(plan["unique"].tolist()) == sorted(kept)
    return keep


@pytest.mark.parametrize("path,T", [("i8", 1), ("i8", 3), ("i8", 8), ("i8", 64), ("core", 5), ("core", 64),
                                    ("tc", 64), ("tc", 200)])
def test_expert_top_p_matches_the_oracle(gpu, coli, host, path, T):
    L = host
    layer = _layer(coli, L, max_tokens=256)
    layer.set_expert_top_p(P)
    if path != "i8":
        layer.set_fused(False)
    if path == "tc":
        x = synth.x_bf16(70, T, T, C4["H"])
        xd = torch.from_numpy(x.view(np.int16)).to(gpu).view(torch.bfloat16)
    else:
        x = synth.x_f32(70, T, T, C4["H"])
        xd = torch.from_numpy(x).to(gpu)
    logits = oracle.router_logits(L["wr"], L["bias"], x)
    assert _margin_ok(logits, C4["K"], P)
    yd = torch.full_like(xd, float("nan"))
    layer.forward(xd, yd)
    layer.sync()
    plan = layer.plan(T)
    y_ref, ids_ref, w_ref = oracle.moe_forward(cases.oracle_cfg(C4, top_p=P), L["wr"], L["bias"], L["experts"], x)
    keep = _check_plan(plan, ids_ref, w_ref)
    y = yd.float().cpu().numpy().astype(np.float64)
    if path == "tc":
        err = np.linalg.norm(y - y_ref) / np.linalg.norm(y_ref)
        assert err <= 5e-3
    else:
        err = np.abs(y - y_ref).max() / np.abs(y_ref).max()
        assert err <= 1e-3
    print(f"top-p {P} {path} T={T}: kept {keep.mean():.2f} of {C4['K']} per token, err {err:.2e}")
    # route() gives the same routing
    ids = torch.empty((T, C4["K"]), dtype=torch.int32, device=gpu)
    w = torch.empty((T, C4["K"]), dtype=torch.float32, device=gpu)
    layer.route(xd, ids, w)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(ids.cpu().numpy(), plan["ids"])
    np.testing.assert_array_equal(w.cpu().numpy(), plan["weights"])
    layer.close()


def test_expert_top_p_one_is_plain_top_k_and_bad_values_are_refused(gpu, coli, host):
    L = host
    a, b = _layer(coli, L), _layer(coli, L)
    b.set_expert_top_p(1.0)
    x = synth.x_f32(71, 0, 8, C4["H"])
    xd = torch.from_numpy(x).to(gpu)
    ya, yb = torch.empty_like(xd), torch.empty_like(xd)
    a.forward(xd, ya)
    b.forward(xd, yb)
    torch.cuda.synchronize()
    assert torch.equal(ya, yb)
    for bad in (0.0, -0.5, 1.5, float("nan")):
        with pytest.raises(coli.ColiError):
            a.set_expert_top_p(bad)
    a.close()
    b.close()


def test_expert_top_p_on_a_cached_layer(gpu, coli, host):
    """The cache sees only the kept experts: a cached layer with top-p equals
    an all-slot cached layer with top-p, and misses no more than without it."""
    L = host
    cached, full = _layer(coli, L, max_tokens=2, resident=8), _layer(coli, L, max_tokens=2, resident=C4["E"])
    plain = _layer(coli, L, max_tokens=2, resident=8)
    for l in (cached, full):
        l.set_expert_top_p(P)
    for step in range(30):
        x = synth.x_f32(72, step, 2, C4["H"])
        xd = torch.from_numpy(x).to(gpu)
        outs = []
        for l in (cached, full, plain):
            yd = torch.empty_like(xd)
            l.forward(xd, yd)
            l.sync()
            outs.append(yd.cpu().numpy())
        assert np.array_equal(outs[0], outs[1]), f"step {step}"
    sc, sp = cached.cache_stats(), plain.cache_stats()
    print(f"cached top-p: {sc['hits'] + sc['misses']} needed, {sc['misses']} misses; plain: "
          f"{sp['hits'] + sp['misses']} needed, {sp['misses']} misses")
    assert sc["hits"] + sc["misses"] < sp["hits"] + sp["misses"]
    for l in (cached, full, plain):
        l.close()


def test_full_size_decode_batch32_expert_top_p(gpu, coli):
    """Full-size layer, Zipf routing, batch 32, p = 0.7: routing of every token
    against the oracle, two tokens' outputs, and the distinct experts per step
    against the plain top-8."""
    from tests import gpu_cases
    c = cases.FULL
    bias, _ = synth.zipf_bias(0, 0, c["E"])
    layer = gpu_cases.device_layer(c, seed=0, layer=0, bias=bias, max_tokens=32)
    x = synth.x_f32(2100, 0, 32, c["H"])
    wr = synth.router(0, 0, c["E"], c["H"])
    logits = oracle.router_logits(wr, bias, x)
    assert _margin_ok(logits, c["K"], P)
    xd = torch.from_numpy(x).to(gpu)
    yd = torch.empty_like(xd)
    layer.forward(xd, yd)
    n_plain = layer.stats()[0]
    layer.set_expert_top_p(P)
    layer.forward(xd, yd)
    layer.sync()
    plan = layer.plan(32)
    n_topp = layer.stats()[0]
    y = yd.cpu().numpy().astype(np.float64)
    layer.close()
    ids_ref, w_ref = oracle.topk(logits, c["K"], top_p=P)
    _check_plan(plan, ids_ref, w_ref)
    toks = [0, 17]
    experts = [None] * (c["E"] + c["S"])
    for e in set(ids_ref[toks][ids_ref[toks] >= 0].ravel().tolist()) | {c["E"]}:
        experts[e] = synth.expert(0, 0, e, c["H"], c["I"])
    y_ref, _, _ = oracle.moe_forward(cases.oracle_cfg(c, top_p=P), wr, bias, experts, x[toks])
    err = np.abs(y[toks] - y_ref).max() / np.abs(y_ref).max()
    kept = (ids_ref >= 0).sum() / 32
    print(f"full b32 top-p {P}: {kept:.2f} experts kept per token, distinct {n_topp} vs {n_plain} plain; err {err:.2e}")
    assert n_topp < n_plain
    assert err <= 1e-3
