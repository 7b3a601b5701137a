"""Device-side builders for the GPU tests and the benchmark: a layer generated
straight into HBM by the generator's device twin, then handed to the C ABI."""
from __future__ import annotations

import numpy as np
import torch

import synth
import int4_expert_ffn_router_b200 as coli


def device_layer(c, seed=0, layer=0, bias=None, max_tokens=64, device=0, resident=None):
    """Create a layer whose canonical weights are generated on the device
    (``resident``: routed-expert slots of an expert cache, None: all in HBM).

    Peak device memory: the canonical buffers (E+S experts) plus the layer."""
    H, I, E, S = c["H"], c["I"], c["E"], c["S"]
    nq, ns = synth.expert_sizes(H, I)
    dev = torch.device("cuda", device)
    stream = torch.cuda.current_stream(dev).cuda_stream
    wr = torch.empty(E * H, dtype=torch.float32, device=dev)
    synth.router_dev(seed, layer, E, H, wr.data_ptr(), stream)
    q = torch.empty((E + S) * nq, dtype=torch.uint8, device=dev)
    s = torch.empty((E + S) * ns, dtype=torch.int16, device=dev)
    synth.expert_dev(seed, layer, 0, E + S, H, I, q.data_ptr(), s.data_ptr(), stream)
    b = None if bias is None else torch.from_numpy(np.ascontiguousarray(bias, np.float32)).to(dev)
    torch.cuda.synchronize(dev)
    cfg = coli.make_config(H, I, E, c["K"], S, max_tokens)
    L = coli.Layer(cfg, wr, b, q[:E * nq], s[:E * ns], q[E * nq:] if S else None, s[E * ns:] if S else None,
                   device=device, resident=resident)
    del q, s
    torch.cuda.empty_cache()
    return L


def x_device(seed, step, T, H, bf16=False, device=0):
    dev = torch.device("cuda", device)
    x = torch.empty((T, H), dtype=torch.bfloat16 if bf16 else torch.float32, device=dev)
    if T:
        synth.x_dev(seed, step, T, H, 1 if bf16 else 0, x.data_ptr(), torch.cuda.current_stream(dev).cuda_stream)
    return x
