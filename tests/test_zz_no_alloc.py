"""The allocation-free routing entry point.

Some callers cannot allocate device memory where they route (inside a CUDA
graph capture, on a fixed memory budget from another framework's pool).
coli_moe_route_noalloc serves them from a fixed scratch array inside the
library. Here it must give what the layer's coli_moe_route gives for the same
inputs, on two calls in a row (the shared scratch keeps the previous call's
values, which must not leak into the next result). This file is collected
last so that a failure here leaves the rest of the suite already run.
"""
import numpy as np
import pytest

import synth

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.mark.parametrize("H,E,K,T,bf16", [(512, 16, 2, 5, False), (6144, 256, 8, 63, False), (6144, 256, 8, 3, True)])
def test_route_noalloc_matches_layer_route(gpu, H, E, K, T, bf16):
    import int4_expert_ffn_router_b200 as coli

    I, S = 256, 1
    wr = synth.router(7, 0, E, H)
    bias = synth.zipf_bias(7, 0, E)[0]
    # a layer only to call the existing entry point (routing needs no experts)
    layer = coli.Layer(coli.make_config(H, I, E, K, S, T), wr, bias)
    wr_d = torch.from_numpy(wr).to(gpu)
    bias_d = torch.from_numpy(bias).to(gpu)
    for call in range(2):  # two calls in a row through the shared scratch
        if bf16:
            xh = synth.x_bf16(100 + call, 0, T, H)
            x = torch.from_numpy(xh.view(np.int16)).to(gpu).view(torch.bfloat16)
        else:
            x = torch.from_numpy(synth.x_f32(100 + call, 0, T, H)).to(gpu)
        ids_a = torch.full((T, K), -1, dtype=torch.int32, device=gpu)
        w_a = torch.zeros((T, K), dtype=torch.float32, device=gpu)
        ids_b = torch.full((T, K), -2, dtype=torch.int32, device=gpu)
        w_b = torch.ones((T, K), dtype=torch.float32, device=gpu)
        layer.route(x, ids_a, w_a)
        coli.route_noalloc(wr_d, bias_d, E, H, K, x, ids_b, w_b)
        torch.cuda.synchronize()
        np.testing.assert_array_equal(ids_b.cpu().numpy(), ids_a.cpu().numpy())
        np.testing.assert_allclose(w_b.cpu().numpy(), w_a.cpu().numpy(), rtol=0, atol=1e-6)
    layer.close()


def test_route_noalloc_rejects_sizes_beyond_its_scratch(gpu):
    import int4_expert_ffn_router_b200 as coli

    H, E, K = 512, 16, 2
    T = coli.NOALLOC_MAX_TOKENS + 1
    wr = torch.zeros((E, H), device=gpu)
    x = torch.zeros((T, H), device=gpu)
    ids = torch.empty((T, K), dtype=torch.int32, device=gpu)
    w = torch.empty((T, K), dtype=torch.float32, device=gpu)
    with pytest.raises(coli.ColiError) as e:
        coli.route_noalloc(wr, None, E, H, K, x, ids, w)
    assert e.value.status == coli.COLI_EINVAL and "n_tokens" in str(e.value)
    with pytest.raises(coli.ColiError):
        coli.route_noalloc(wr, None, coli.NOALLOC_MAX_EXPERTS + 1, H, K, x[:1], ids[:1], w[:1])
