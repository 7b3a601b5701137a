"""GPU tests of the expert cache: a layer with only R of its E routed experts
in HBM, the rest fetched from page-locked host memory on demand, per-layer
least-recently-used eviction, pinned (learned hot) experts and the router run
one layer ahead to prefetch ("Colibri: 2400 lines of pure C ...", section 二;
project page, placement tiers).

Over a Zipf-routed token stream the cached layer must give the outputs of a
layer that holds every expert, bit for bit when both take the same routing
(a cache of R = E slots runs the same host-routed sequence), and the same ids
and outputs within 1e-6 of the largest magnitude against the resident layer
(whose persistent kernel routes inside itself).
"""
import numpy as np
import pytest

import oracle
import synth
from tests import cases

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")

# 64 routed experts top-4, batches of up to 4 tokens: a batch needs at most 16 slots
MID = dict(H=512, I=256, E=64, K=4, S=1)
R = 20
MAXT = 4


@pytest.fixture(scope="module")
def coli():
    import int4_expert_ffn_router_b200 as m
    return m


@pytest.fixture(scope="module")
def host():
    bias, _ = synth.zipf_bias(5, 0, MID["E"])
    return [cases.host_layer(MID, seed=5, layer=l, bias=bias) for l in range(3)]


def _make(coli, L, resident, max_tokens=MAXT):
    c = MID
    E, S = c["E"], c["S"]
    q = np.concatenate([e[0] for e in L["experts"]])
    s = np.concatenate([e[1] for e in L["experts"]])
    nq, ns = synth.expert_sizes(c["H"], c["I"])
    cfg = coli.make_config(c["H"], c["I"], E, c["K"], S, max_tokens)
    return coli.Layer(cfg, L["wr"], L["bias"], q[:E * nq], s[:E * ns], q[E * nq:], s[E * ns:], device=0,
                      resident=resident)


def _stream(n, seed=50):
    rng = np.random.default_rng(seed)
    return [int(t) for t in rng.integers(1, MAXT + 1, n)]


def _fwd(layer, x, gpu):
    xd = torch.from_numpy(x).to(gpu)
    yd = torch.full_like(xd, float("nan"))
    layer.forward(xd, yd)
    layer.sync()
    return yd.cpu().numpy()


@pytest.mark.parametrize("path", ["i8", "core", "tc"])
def test_cached_layer_equals_resident_layer_over_a_zipf_stream(gpu, coli, host, path):
    """40 batches of 1-4 tokens through a cache of 20 slots (all full from the
    start, so every miss evicts). i8: the persistent kernel; core: the
    CUDA-core kernels (fp32); tc: the tensor-core kernels (bf16), whose fp32
    atomic combine may change the last bits between runs, so there the
    comparison is a relative L2 of 1e-4 instead of equality."""
    L = host[0]
    cached, full, resident = _make(coli, L, R), _make(coli, L, MID["E"]), _make(coli, L, None)
    if path != "i8":
        for l in (cached, full, resident):
            l.set_fused(False)
    bf16 = path == "tc"
    distinct = 0
    for step, T in enumerate(_stream(40)):
        if bf16:
            xb = synth.x_bf16(60, step, T, MID["H"])
            xd = torch.from_numpy(xb.view(np.int16)).to(gpu).view(torch.bfloat16)
        else:
            x = synth.x_f32(60, step, T, MID["H"])
            xd = torch.from_numpy(x).to(gpu)
        outs, plans = [], []
        for l in (cached, full, resident):
            yd = torch.full_like(xd, float("nan"))
            l.forward(xd, yd)
            l.sync()
            outs.append(yd.float().cpu().numpy().astype(np.float64))
            plans.append(l.plan(T))
        distinct += len(set(plans[0]["ids"].ravel().tolist()))
        for other in plans[1:]:
            np.testing.assert_array_equal(plans[0]["ids"], other["ids"])
        if bf16:
            for other in outs[1:]:
                assert np.linalg.norm(outs[0] - other) <= 1e-4 * np.linalg.norm(other), f"step {step}"
        else:
            assert np.array_equal(outs[0], outs[1]), f"step {step}: cached and all-slot layers differ"
            if path == "core":  # the resident layer routes with the same kernels here
                assert np.array_equal(outs[0], outs[2]), f"step {step}: cached and resident layers differ"
            else:  # the persistent kernel of the resident layer sums the logits in another order
                assert np.abs(outs[0] - outs[2]).max() <= 1e-6 * np.abs(outs[2]).max(), f"step {step}"
        if step % 13 == 0 and not bf16:  # and against the oracle
            y_ref, ids_ref, _ = oracle.moe_forward(cases.oracle_cfg(MID), L["wr"], L["bias"], L["experts"], x)
            np.testing.assert_array_equal(plans[0]["ids"], ids_ref)
            assert np.abs(outs[0] - y_ref).max() <= 1e-3 * np.abs(y_ref).max()
    st = cached.cache_stats(usage=True)
    print(f"cache {path}: {st['hits']} hits, {st['misses']} misses, {st['bytes_h2d']} B copied")
    assert st["hits"] + st["misses"] == distinct
    assert st["misses"] > 0 and st["hits"] > 0
    per_copy = st["bytes_h2d"] // st["misses"]
    assert st["bytes_h2d"] == st["misses"] * per_copy and per_copy >= coli.expert_bytes(MID["H"], MID["I"])
    assert st["usage"].sum() == distinct
    assert full.cache_stats()["misses"] == 0
    for l in (cached, full, resident):
        l.close()


def test_pinned_experts_stay_resident_and_prefetch_hits(gpu, coli, host):
    L = host[0]
    cached, full = _make(coli, L, R), _make(coli, L, MID["E"])
    steps = _stream(30, seed=51)
    for step, T in enumerate(steps[:15]):
        x = synth.x_f32(61, step, T, MID["H"])
        cached.forward(torch.from_numpy(x).to(gpu), torch.empty((T, MID["H"]), device=gpu))
    cached.sync()
    hot = cached.pin_hot(4)
    st = cached.cache_stats(usage=True, reset=True)
    assert st["n_pinned"] == 4
    assert list(hot) == list(np.argsort(-st["usage"], kind="stable")[:4])
    with pytest.raises(coli.ColiError):  # 20 slots - 16 for a batch: at most 4 pinned
        cached.pin(list(range(5)))
    for step, T in enumerate(steps[15:]):
        x = synth.x_f32(61, 100 + step, T, MID["H"])
        assert np.array_equal(_fwd(cached, x, gpu), _fwd(full, x, gpu))
    # the pinned experts were never evicted: a prefetch of them copies nothing
    before = cached.cache_stats()["prefetched"]
    cached.prefetch(hot)
    assert cached.cache_stats()["prefetched"] == before
    slots = cached.cache_slots()
    assert all(slots[e] >= 0 for e in hot)
    assert sorted(slots[slots >= 0].tolist()) == list(range(R))
    # prefetch a batch's experts (one with some not in HBM), then that batch misses nothing
    for seed in range(62, 200):
        x = synth.x_f32(seed, 0, MAXT, MID["H"])
        ids, _ = oracle.topk(oracle.router_logits(L["wr"], L["bias"], x), MID["K"])
        need = np.unique(ids)
        if (slots[need] < 0).any():
            break
    n_new = int((slots[need] < 0).sum())
    p0 = cached.cache_stats()
    cached.prefetch(need)
    assert (cached.cache_slots()[need] >= 0).all()
    assert all(cached.cache_slots()[e] >= 0 for e in hot)
    ya, yb = _fwd(cached, x, gpu), _fwd(full, x, gpu)
    assert np.array_equal(ya, yb)
    st = cached.cache_stats()
    assert st["misses"] == p0["misses"]
    assert st["prefetched"] - p0["prefetched"] == n_new
    assert st["prefetch_used"] - p0["prefetch_used"] >= n_new  # (pinned copies also count as prefetched)
    cached.pin([])
    assert cached.cache_stats()["n_pinned"] == 0
    cached.close()
    full.close()


def test_cached_stack_with_lookahead_equals_resident_stack(gpu, coli, host):
    """Three cached layers (the second and third accept the previous layer's
    prediction) against three all-slot layers: the residual stream must be
    identical after every step; the predictions are counted."""
    cached = [_make(coli, L, R) for L in host]
    full = [_make(coli, L, MID["E"]) for L in host]
    for l in full:
        l.set_lookahead(False)
    for step, T in enumerate(_stream(20, seed=52)):
        x = synth.x_f32(63, step, T, MID["H"])
        xa = torch.from_numpy(x).to(gpu)
        xb = xa.clone()
        coli.stack_forward(cached, xa)
        coli.stack_forward(full, xb)
        torch.cuda.synchronize()
        assert torch.equal(xa, xb), f"step {step}"
    st = [l.cache_stats() for l in cached]
    print("lookahead:", [(s["predicted"], s["predicted_of"], s["prefetched"], s["prefetch_used"]) for s in st])
    assert st[0]["predicted_of"] == 0
    for s in st[1:]:
        assert s["predicted_of"] > 0 and s["prefetched"] > 0
    assert all(s["predicted_of"] == 0 for s in (l.cache_stats() for l in full))
    for l in cached + full:
        l.close()


def test_cached_layer_argument_errors(gpu, coli, host):
    L = host[0]
    with pytest.raises(coli.ColiError):
        _make(coli, L, 15)          # fewer than max_tokens * top_k = 16 slots
    with pytest.raises(coli.ColiError):
        _make(coli, L, MID["E"] + 1)
    resident = _make(coli, L, None)
    with pytest.raises(coli.ColiError):
        resident.cache_stats()
    with pytest.raises(coli.ColiError):
        resident.prefetch([1])
    resident.close()
    cached = _make(coli, L, R)
    with pytest.raises(coli.ColiError):
        cached.prefetch([MID["E"]])
    with pytest.raises(coli.ColiError):
        cached.pin([-1])
    cached.close()
