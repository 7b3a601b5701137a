"""Roofline arithmetic of bench.py on CPU: the algorithmic work per launch of
the dominant kernel and its fraction of the measured peak, and the guard that
drops recorded ncu traffic once a kernel's sources change."""
import pytest

import bench

PEAKS = {"hbm_gbs": 6000.0, "bf16_tflops": 1500.0, "bf16_tflops_sustained": 1200.0}


def test_decode_roofline_bytes_and_fraction():
    # persistent kernel: 9 active experts + router + x and y (fp32, one token), 80 us per launch
    stages = {"fused": 80e-3 * 10, "router": 0.0}
    dom, roof = bench.dominant_roofline(stages, 10, 1, 8.0, 256, 4, False, PEAKS)
    assert dom == "fused" and roof["bound"] == "hbm" and roof["unit"] == "GB/s"
    want = 9 * bench.EXPERT_BYTES + 256 * bench.H * 4 + 2 * bench.H * 4
    assert roof["bytes_per_launch"] == want
    assert roof["achieved"] == pytest.approx(want / 80e-6 / 1e9, rel=1e-3)
    assert roof["frac"] == pytest.approx(roof["achieved"] / 6000.0, rel=1e-3)


def test_tensor_roofline_counts_algorithmic_flops():
    # 2048 tokens, K = 8 routed + 1 shared: gate/up is 2 * T(K+S) * H * 2I flops
    stages = {"gateup": 1.5 * 4, "down": 0.8 * 4}
    dom, roof = bench.dominant_roofline(stages, 4, 2048, 256.0, 256, 2, True, PEAKS)
    assert dom == "gateup" and roof["bound"] == "tensor" and roof["unit"] == "TFLOP/s"
    flops = 2.0 * 2048 * 9 * bench.H * 2 * bench.I
    assert roof["flops_per_launch"] == flops
    assert roof["achieved"] == pytest.approx(flops / 1.5e-3 / 1e12, rel=1e-3)
    assert roof["frac"] == pytest.approx(roof["achieved"] / 1500.0, rel=1e-3)
    assert roof["frac_of_sustained"] == pytest.approx(roof["achieved"] / 1200.0, rel=1e-3)


def _digest(files):
    import hashlib
    import os
    h = hashlib.sha256()
    for f in files:
        with open(os.path.join(bench.ROOT, "int4_expert_ffn_router_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def test_recorded_traffic_needs_unchanged_sources(monkeypatch):
    key = ("moe_decode_i8_kernel", "decode_b1")
    assert bench.ncu_traffic("moe_decode_i8_kernel", "decode_b32") == (None, None)
    rec = dict(bytes=190_000_000, sources=("decode_i8.cu", "common.cuh"), note="test record")
    monkeypatch.setitem(bench.NCU_TRAFFIC, key, dict(rec, sha256_16=_digest(rec["sources"])))
    assert bench.ncu_traffic(*key) == (190_000_000, "test record")  # sources as captured
    monkeypatch.setitem(bench.NCU_TRAFFIC, key, dict(rec, sha256_16="0" * 16))
    b, note = bench.ncu_traffic(*key)
    assert b is None and "changed" in note
