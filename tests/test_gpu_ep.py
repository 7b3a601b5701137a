"""GPU tests of the expert-parallel layer (experts sharded over ranks, router
replicated, partial outputs summed by the caller). The ranks of one layer are
emulated on one GPU as separate layers run one after the other: nothing waits
on another rank, and the exchange is a host-side sum here (on several GPUs it
is an all-reduce).

Checks, on the persistent kernel, the CUDA-core kernels and the tcgen05
kernels: each rank's plan lists only its own experts and marks the other
slots empty (id -1, position -1) while keeping the routing weights; the
ranks' distinct experts partition the whole layer's; the partial outputs sum
to the whole layer's output (within the fp32 reassociation of the sum) and to
the oracle's.
"""
import numpy as np
import pytest

import oracle
import synth
from tests import cases

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")

C = dict(cases.TINY, E=32, K=4)


@pytest.fixture(scope="module")
def coli():
    import int4_expert_ffn_router_b200 as m
    return m


@pytest.fixture(scope="module")
def host():
    bias, _ = synth.zipf_bias(9, 0, C["E"])
    return cases.host_layer(C, seed=9, bias=bias)


def _layer(coli, L, ep=None, max_tokens=512):
    E = C["E"]
    q = np.concatenate([e[0] for e in L["experts"]])
    s = np.concatenate([e[1] for e in L["experts"]])
    nq, ns = synth.expert_sizes(C["H"], C["I"])
    cfg = coli.make_config(C["H"], C["I"], E, C["K"], C["S"], max_tokens)
    return coli.Layer(cfg, L["wr"], L["bias"], q[:E * nq], s[:E * ns], q[E * nq:], s[E * ns:], device=0, ep=ep)


def _run(layer, xd, T):
    yd = torch.full_like(xd, float("nan"))
    layer.forward(xd, yd)
    layer.sync()
    return yd.float().cpu().numpy().astype(np.float64), layer.plan(T)


@pytest.mark.parametrize("path,T,world", [("i8", 1, 2), ("i8", 8, 4), ("i8", 64, 3), ("core", 100, 2),
                                          ("tc", 300, 4), ("i8", 8, 32)])
def test_partial_outputs_sum_to_the_layer(gpu, coli, host, path, T, world):
    L = host
    full = _layer(coli, L)
    ranks = [_layer(coli, L, ep=(r, world)) for r in range(world)]
    if path != "i8":
        for l in [full] + ranks:
            l.set_fused(False)
    if path == "tc":
        x = synth.x_bf16(80, T, T, C["H"])
        xd = torch.from_numpy(x.view(np.int16)).to(gpu).view(torch.bfloat16)
    else:
        x = synth.x_f32(80, T, T, C["H"])
        xd = torch.from_numpy(x).to(gpu)
    y_full, plan_full = _run(full, xd, T)
    y_sum = np.zeros_like(y_full)
    uniques = []
    for r, l in enumerate(ranks):
        y_r, plan = _run(l, xd, T)
        lo, hi = coli.ep_range(C["E"], r, world)
        ids_full = plan_full["ids"]
        local = (ids_full >= lo) & (ids_full < hi)
        np.testing.assert_array_equal(plan["ids"], np.where(local, ids_full, -1))
        np.testing.assert_array_equal(plan["pos"][~local], -1)
        np.testing.assert_array_equal(plan["weights"], plan_full["weights"])
        assert all(lo <= e < hi for e in plan["unique"])
        uniques.append(set(plan["unique"].tolist()))
        y_sum += y_r
    assert set().union(*uniques) == set(plan_full["unique"].tolist())
    assert sum(len(u) for u in uniques) == len(plan_full["unique"])
    scale = np.abs(y_full).max()
    if path == "tc":
        err = np.linalg.norm(y_sum - y_full) / np.linalg.norm(y_full)
        assert err <= 5e-3
    else:
        err = np.abs(y_sum - y_full).max() / scale
        assert err <= 1e-5
    if path != "tc":
        y_ref, _, _ = oracle.moe_forward(cases.oracle_cfg(C), L["wr"], L["bias"], L["experts"], x)
        assert np.abs(y_sum - y_ref).max() <= 1e-3 * np.abs(y_ref).max()
    print(f"expert parallel {path} T={T} world={world}: partial sum vs whole layer {err:.2e}")
    for l in [full] + ranks:
        l.close()


def test_expert_parallel_with_expert_top_p(gpu, coli, host):
    L = host
    world, T = 2, 8
    full = _layer(coli, L)
    full.set_expert_top_p(0.7)
    ranks = [_layer(coli, L, ep=(r, world)) for r in range(world)]
    for l in ranks:
        l.set_expert_top_p(0.7)
    x = synth.x_f32(81, 0, T, C["H"])
    xd = torch.from_numpy(x).to(gpu)
    y_full, _ = _run(full, xd, T)
    y_sum = sum(_run(l, xd, T)[0] for l in ranks)
    assert np.abs(y_sum - y_full).max() <= 1e-5 * np.abs(y_full).max()
    y_ref, _, _ = oracle.moe_forward(cases.oracle_cfg(C, top_p=0.7), L["wr"], L["bias"], L["experts"], x)
    assert np.abs(y_sum - y_ref).max() <= 1e-3 * np.abs(y_ref).max()
    for l in [full] + ranks:
        l.close()


def test_expert_parallel_argument_errors(gpu, coli, host):
    with pytest.raises(coli.ColiError):
        _layer(coli, host, ep=(2, 2))
    with pytest.raises(coli.ColiError):
        _layer(coli, host, ep=(0, C["E"] + 1))
