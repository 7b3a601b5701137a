"""The C-ABI library loads, exports every declared symbol, and rejects bad
arguments before touching a GPU (no compute calls: these run on the CPU)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "coli_moe.h")


def _declared():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(coli_\w+)\s*\(", text)))


@pytest.fixture(scope="module")
def lib():
    import __graft_entry__  # noqa: F401  (build helper)
    from int4_expert_ffn_router_b200 import build as b
    if not os.path.exists(b.SO):
        b.build()
    import int4_expert_ffn_router_b200 as m
    return m


def test_every_declared_symbol_is_exported(lib):
    names = _declared()
    assert "coli_moe_layer_create" in names and "coli_moe_forward" in names and "coli_moe_route" in names
    raw = ctypes.CDLL(lib.LIB_PATH)
    for n in names:
        assert hasattr(raw, n), f"{n} declared in coli_moe.h but not exported"
    assert sorted(lib.EXPORTS) == names


def test_status_strings_and_expert_bytes(lib):
    assert lib.lib.coli_status_string(0) == b"ok"
    assert lib.lib.coli_status_string(1) == b"invalid argument"
    # 6144 x 2048 expert: 18,874,368 nibble bytes + 1,179,648 B of fp16 scales (~19 MB)
    assert lib.expert_bytes(6144, 2048) == 20_054_016


def _create(lib, **over):
    cfg = lib.make_config(512, 256, 16, 2, 1, 4)
    for k, v in over.items():
        setattr(cfg, k, v)
    h = ctypes.c_void_p()
    dummy = (ctypes.c_float * 16)()
    st = lib.lib.coli_moe_layer_create(ctypes.byref(cfg), ctypes.cast(dummy, ctypes.c_void_p), None, None, None,
                                       None, None, 0, ctypes.byref(h))
    return st, h, lib.lib.coli_last_error().decode()


@pytest.mark.parametrize("field,value,msg", [
    ("hidden", 500, "hidden"), ("hidden", 0, "hidden"), ("inter", 100, "inter"), ("group_size", 128, "group_size"),
    ("n_experts", 0, "n_experts"), ("n_experts", 2048, "n_experts"), ("top_k", 17, "top_k"), ("top_k", 0, "top_k"),
    ("n_shared", -1, "n_shared"), ("max_tokens", 0, "max_tokens"),
])
def test_create_rejects_bad_config_before_any_cuda_call(lib, field, value, msg):
    st, h, err = _create(lib, **{field: value})
    assert st == lib.COLI_EINVAL and h.value is None and msg in err


def test_null_arguments_are_rejected(lib):
    L = lib.lib
    assert L.coli_moe_layer_create(None, None, None, None, None, None, None, 0, None) == lib.COLI_EINVAL
    assert L.coli_moe_forward(None, None, None, 0, 1, None) == lib.COLI_EINVAL
    assert L.coli_moe_route(None, None, 0, 1, None, None, None) == lib.COLI_EINVAL
    assert L.coli_moe_get_stats(None, None, None, None) == lib.COLI_EINVAL
    assert L.coli_moe_stack_forward(None, 1, None, 1, 1e-6, None) == lib.COLI_EINVAL
    n = ctypes.c_int64(-1)
    assert L.coli_moe_get_launch_count(None, ctypes.byref(n)) == lib.COLI_EINVAL and n.value == -1
    assert L.coli_moe_set_tensor_cores(None, 1) == lib.COLI_EINVAL
    L.coli_moe_layer_destroy(None)  # no-op


def test_debug_fail_alloc_validates_its_argument(lib):
    assert lib.lib.coli_moe_debug_fail_alloc(-1) == lib.COLI_EINVAL
    assert lib.lib.coli_moe_debug_fail_alloc(0) == lib.COLI_OK
