"""Failure handling on the GPU, without making the GPU fault or hang.

Out of memory is made on the host: coli_moe_debug_fail_alloc makes the nth
device (or page-locked host) allocation of layer creation fail as if the
memory were full. Each
failing create must return COLI_ENOMEM, leave nothing allocated (the
device's free memory is the same before and after) and leave the library
usable.
"""
import numpy as np
import pytest

import oracle
import synth
from tests import cases

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


def _host_args(coli, c, max_tokens=8):
    L = cases.host_layer(c, seed=c["seed"])
    q = np.concatenate([e[0] for e in L["experts"]])
    s = np.concatenate([e[1] for e in L["experts"]])
    nq, ns = synth.expert_sizes(c["H"], c["I"])
    E = c["E"]
    cfg = coli.make_config(c["H"], c["I"], E, c["K"], c["S"], max_tokens)
    return L, (cfg, L["wr"], None, q[:E * nq], s[:E * ns], q[E * nq:], s[E * ns:])


@pytest.mark.parametrize("resident", [None, 6])
def test_create_out_of_memory_at_each_allocation(gpu, resident):
    """resident=6: an expert cache of 6 slots, whose create also allocates
    page-locked host memory (those allocations fail the same way)."""
    import int4_expert_ffn_router_b200 as coli

    c = cases.TINY
    L, args = _host_args(coli, c, max_tokens=2)
    coli.Layer(*args, device=0, resident=resident).close()  # module loading and the context are not counted below
    torch.cuda.synchronize()
    free0 = torch.cuda.mem_get_info()[0]
    failed = 0
    try:
        for nth in range(1, 16):
            coli.debug_fail_alloc(nth)
            try:
                layer = coli.Layer(*args, device=0, resident=resident)
            except coli.ColiError as e:
                assert e.status == coli.COLI_ENOMEM, str(e)
                failed += 1
                assert torch.cuda.mem_get_info()[0] == free0, f"allocation {nth}: device memory leaked"
                continue
            layer.close()  # fewer than nth allocations: the create succeeded
            break
    finally:
        coli.debug_fail_alloc(0)
    # weights, router, bias, workspace and the staging buffer of host sources;
    # a cache adds the repack buffer, the slot table, and four page-locked
    # buffers: expert pool, table staging, routed ids, predicted ids
    assert failed == (5 if resident is None else 11)
    assert torch.cuda.mem_get_info()[0] == free0
    # the library still works: a forward through a fresh layer matches the oracle
    layer = coli.Layer(*args, device=0, resident=resident)
    x = synth.x_f32(c["seed"], 3, 2, c["H"])
    xd = torch.from_numpy(x).to(gpu)
    yd = torch.empty_like(xd)
    layer.forward(xd, yd)
    layer.sync()
    y_ref, _, _ = oracle.moe_forward(cases.oracle_cfg(c), L["wr"], None, L["experts"], x)
    y = yd.cpu().numpy().astype(np.float64)
    assert np.abs(y - y_ref).max() <= 1e-3 * np.abs(y_ref).max()
    layer.close()


@pytest.mark.parametrize("T", [3, 1])
def test_bounded_wait_expiry_returns_an_error_and_the_layer_recovers(gpu, T):
    """A testing aid makes one gate/up item of the persistent kernel wait on a
    flag that nothing sets, with every wait bounded to 2 ms. The launch gives
    up by itself (its CTAs drain their copies and exit): coli_moe_sync reports
    COLI_ECUDA promptly, and the next forward on the same layer matches the
    oracle. Nothing faults or hangs. At 1 token the kernel's producer stages
    the other items' operands into per-slot buffers, which the drain covers."""
    import time

    import int4_expert_ffn_router_b200 as coli

    c = cases.TINY
    L, args = _host_args(coli, c)
    layer = coli.Layer(*args, device=0)
    x = synth.x_f32(c["seed"], 4, T, c["H"])
    xd = torch.from_numpy(x).to(gpu)
    yd = torch.empty_like(xd)
    layer.forward(xd, yd)  # warm: module loaded, control block in use once
    layer.sync()
    layer.debug_wait_test(True, 2_000_000)
    t0 = time.time()
    layer.forward(xd, yd)
    with pytest.raises(coli.ColiError) as e:
        layer.sync()
    elapsed = time.time() - t0
    assert e.value.status == coli.COLI_ECUDA and "timed out" in str(e.value)
    assert elapsed < 2.0, f"the launch took {elapsed:.2f} s to give up"
    layer.debug_wait_test(False, 0)
    for _ in range(2):
        yd.fill_(float("nan"))
        layer.forward(xd, yd)
        layer.sync()
        y_ref, _, _ = oracle.moe_forward(cases.oracle_cfg(c), L["wr"], None, L["experts"], x)
        y = yd.cpu().numpy().astype(np.float64)
        assert np.abs(y - y_ref).max() <= 1e-3 * np.abs(y_ref).max()
    layer.close()


@pytest.mark.parametrize("E,sites", [(16, r"4[1-4]"), (300, r"2[1-9]")])
def test_bounded_wait_expiry_in_the_batch_kernels(gpu, E, sites):
    """The same testing aid on a 96-token bf16 batch: the certified router's
    int8 GEMM and both tensor-core grouped GEMMs each make one MMA warp wait
    on a barrier that nothing completes, every wait bounded to 2 ms. Each
    launch gives up by itself (its copies drain, no MMA is left running when
    tensor memory is released): coli_moe_sync reports COLI_ECUDA promptly,
    naming a site of the first launch that gave up, and the next forwards on
    the same layer match the oracle. With 16 experts that is the router GEMM
    (sites 41-44); with 300 experts (more than the certified router takes) the
    router is the fp64 one, and the grouped GEMMs report (sites 21-29)."""
    import time

    import int4_expert_ffn_router_b200 as coli

    c = dict(cases.TINY, E=E)
    T = 96
    L, args = _host_args(coli, c, max_tokens=T)
    layer = coli.Layer(*args, device=0)
    assert layer.router_fallbacks()[0] == (E <= 256)  # the certified router serves this batch
    xb = synth.x_bf16(c["seed"], 5, T, c["H"])
    xd = torch.from_numpy(xb.view(np.int16)).to(gpu).view(torch.bfloat16)
    yd = torch.empty_like(xd)
    layer.forward(xd, yd)
    layer.sync()
    layer.debug_wait_test(True, 2_000_000)
    t0 = time.time()
    layer.forward(xd, yd)
    with pytest.raises(coli.ColiError) as e:
        layer.sync()
    elapsed = time.time() - t0
    # the first wait to give up belongs to the first launch with the aid: its MMA warp's, or
    # the wait of another warp for the same barrier
    import re
    assert e.value.status == coli.COLI_ECUDA and re.search(r"timed out \(site " + sites + r"\)", str(e.value))
    assert elapsed < 2.0, f"the launches took {elapsed:.2f} s to give up"
    layer.debug_wait_test(False, 0)
    y_ref, _, _ = oracle.moe_forward(cases.oracle_cfg(c), L["wr"], None, L["experts"], xb)
    for _ in range(2):
        yd.fill_(float("nan"))
        layer.forward(xd, yd)
        layer.sync()
        y = yd.float().cpu().numpy().astype(np.float64)
        assert np.linalg.norm(y - y_ref) <= 5e-3 * np.linalg.norm(y_ref)
        ids_ref, _ = oracle.topk(oracle.router_logits(L["wr"], None, xb), c["K"])
        np.testing.assert_array_equal(layer.plan(T)["ids"], ids_ref)
    layer.close()
