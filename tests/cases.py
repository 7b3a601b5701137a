"""Workload shapes and host-side input builders shared by the tests.

Shapes follow the MoE layer of the Colibri pages (256 routed experts, 8 per
token, ~19 MB per int4 expert, groups of 64) at full size, plus a tiny layer
the CPU oracle finishes in well under a second.
"""
from __future__ import annotations

import numpy as np

import synth

# Tiny layer: hidden 512, expert intermediate 256, 16 routed experts top-2,
# one shared expert, 4 tokens, seed 0.
TINY = dict(H=512, I=256, E=16, K=2, S=1, T=4, seed=0)
# Full-size layer: hidden 6144, intermediate 2048 (20,054,016 B per int4
# expert with its fp16 scales), 256 routed experts top-8, one shared expert.
FULL = dict(H=6144, I=2048, E=256, K=8, S=1)


def oracle_cfg(c, top_p=0.0):
    import oracle
    return oracle.Cfg(hidden=c["H"], inter=c["I"], n_experts=c["E"], top_k=c["K"], n_shared=c["S"],
                      expert_top_p=top_p)


def host_layer(c, seed=0, layer=0, which=None, bias=None):
    """Router weights and canonical experts on the host.

    ``which``: iterable of expert ids to generate (routed 0..E-1, shared E..);
    None = all. Others are None (the oracle rejects selecting a missing one).
    """
    H, I, E, S = c["H"], c["I"], c["E"], c["S"]
    wr = synth.router(seed, layer, E, H)
    ids = range(E + S) if which is None else sorted(set(which))
    experts = [None] * (E + S)
    for e in ids:
        experts[e] = synth.expert(seed, layer, e, H, I)
    return dict(wr=wr, bias=bias, experts=experts)


def pack_codes(codes: np.ndarray) -> np.ndarray:
    """Signed codes [rows][cols] in [-8, 7] -> canonical bytes [rows][cols/2]."""
    c = (codes.astype(np.int16) & 0xF).astype(np.uint8)
    return (c[:, 0::2] | (c[:, 1::2] << 4)).astype(np.uint8)


def f16_bits(v) -> np.ndarray:
    return np.asarray(v, np.float32).astype(np.float16).view(np.uint16)


def expert_from_codes(G, U, D, sG, sU, sD):
    """Canonical expert from integer codes and fp32 per-group scales
    (G, U: [I][H]; D: [H][I]; scales [rows][cols/64], exactly representable in fp16)."""
    q = np.concatenate([pack_codes(G).ravel(), pack_codes(U).ravel(), pack_codes(D).ravel()])
    s = np.concatenate([f16_bits(sG).ravel(), f16_bits(sU).ravel(), f16_bits(sD).ravel()])
    return q, s
