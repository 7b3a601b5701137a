"""Host logic of the expert-parallel layer on CPU (no GPU): the partition of
the routed experts over the ranks, and the exchange step on two and three
`gloo` ranks. Each rank forms its partial output the way an expert-parallel
layer defines it (its own routed experts, the shared experts on rank 0 only;
computed here by the fp64 oracle with the other ranks' experts zeroed), the
partial outputs are summed by `bench.ep_combine` (an all-reduce), and the sum
must be the whole layer's output.
"""
import os
import socket

import numpy as np
import pytest

torch = pytest.importorskip("torch")
import torch.distributed as dist  # noqa: E402
import torch.multiprocessing as mp  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.mark.parametrize("E", [1, 7, 16, 256])
def test_expert_ranges_partition_the_experts(E):
    import int4_expert_ffn_router_b200 as coli
    for world in range(1, min(E, 8) + 1):
        ranges = [coli.ep_range(E, r, world) for r in range(world)]
        assert ranges[0][0] == 0 and ranges[-1][1] == E
        for (a0, a1), (b0, b1) in zip(ranges, ranges[1:]):
            assert a1 == b0                      # contiguous, disjoint
        sizes = [b - a for a, b in ranges]
        assert max(sizes) - min(sizes) <= 1 and min(sizes) >= 1
    with pytest.raises(coli.ColiError):
        coli.ep_range(E, 0, 0)
    with pytest.raises(coli.ColiError):
        coli.ep_range(E, 1, 1)


def _partial(c, L, x, rank, world):
    """This rank's partial output by the oracle: other ranks' routed experts
    and (off rank 0) the shared experts replaced by all-zero experts, whose
    output is exactly 0."""
    import oracle
    import int4_expert_ffn_router_b200 as coli
    from tests import cases
    lo, hi = coli.ep_range(c["E"], rank, world)
    zero = (np.zeros_like(L["experts"][0][0]), np.zeros_like(L["experts"][0][1]))
    experts = [L["experts"][e] if lo <= e < hi else zero for e in range(c["E"])]
    experts += L["experts"][c["E"]:] if rank == 0 else [zero] * c["S"]
    y, ids, _ = oracle.moe_forward(cases.oracle_cfg(c), L["wr"], L["bias"], experts, x)
    return y, ids


def _rank_main(rank, world, port, out):
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    import bench
    import oracle
    import synth
    from tests import cases
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        c = cases.TINY
        bias, _ = synth.zipf_bias(3, 0, c["E"])
        L = cases.host_layer(c, seed=3, bias=bias)
        x = synth.x_f32(3, 0, 6, c["H"])
        y_r, _ = _partial(c, L, x, rank, world)
        y = torch.from_numpy(y_r.copy())
        bench.ep_combine(y, dist)
        y_full, _, _ = oracle.moe_forward(cases.oracle_cfg(c), L["wr"], L["bias"], L["experts"], x)
        out[rank] = (float(np.abs(y.numpy() - y_full).max() / np.abs(y_full).max()),
                     float(np.abs(y_r).max()))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_partial_outputs_sum_to_the_layer_over_gloo_ranks(world):
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_rank_main, args=(world, _free_port(), out), nprocs=world, start_method="spawn", join=True)
    assert sorted(out.keys()) == list(range(world))
    for r in range(world):
        assert out[r][0] <= 1e-13      # every rank holds the whole layer's output after the exchange
    assert sum(out[r][1] > 0 for r in range(world)) >= 2   # the work was really split


def test_single_process_combine_is_the_identity():
    import bench
    y = torch.arange(6, dtype=torch.float32)
    bench.ep_combine(y, None)
    assert y.tolist() == list(range(6))
