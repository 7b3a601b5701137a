"""Python binding of the int4 expert-FFN MoE layer (``libcoli_moe.so``).

Argument marshalling only: every step of the layer runs in the CUDA library
behind the C ABI declared in ``include/coli_moe.h``. Tensors are passed as raw
pointers (``torch.Tensor.data_ptr()`` or numpy arrays for host inputs of
``Layer``); streams as ``torch.cuda.Stream.cuda_stream`` handles. If the
library is missing this module raises at import: there is no fallback.
"""
from __future__ import annotations

import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libcoli_moe.so")

COLI_OK, COLI_EINVAL, COLI_ENOMEM, COLI_ECUDA, COLI_EUNSUPPORTED = range(5)
F32, BF16 = 0, 1

# Every symbol the header declares.
EXPORTS = (
    "coli_moe_layer_create", "coli_moe_layer_set_experts", "coli_moe_layer_destroy", "coli_moe_layer_config",
    "coli_moe_route", "coli_moe_forward", "coli_moe_stack_forward", "coli_moe_get_stats", "coli_moe_get_plan",
    "coli_moe_expert_bytes", "coli_status_string", "coli_last_error", "coli_moe_set_profiling",
    "coli_moe_get_profile", "coli_moe_stage_name", "coli_moe_sync", "coli_moe_set_fused", "coli_moe_set_tensor_cores",
    "coli_moe_set_trace", "coli_moe_set_ring", "coli_moe_route_noalloc", "coli_moe_get_launch_count",
    "coli_moe_debug_fail_alloc", "coli_clock_stamp", "coli_moe_debug_wait_test", "coli_moe_layer_create_cached",
    "coli_moe_cache_stats", "coli_moe_cache_pin", "coli_moe_cache_prefetch", "coli_moe_cache_set_lookahead",
    "coli_moe_cache_slots", "coli_moe_set_expert_top_p", "coli_moe_layer_create_ep", "coli_moe_ep_range",
    "coli_moe_router_fallbacks",
)
NOALLOC_MAX_TOKENS, NOALLOC_MAX_EXPERTS = 63, 1024
N_STAGES = 8


class Config(ctypes.Structure):
    _fields_ = [("hidden", ctypes.c_int), ("inter", ctypes.c_int), ("n_experts", ctypes.c_int),
                ("top_k", ctypes.c_int), ("n_shared", ctypes.c_int), ("group_size", ctypes.c_int),
                ("max_tokens", ctypes.c_int)]


class CacheStats(ctypes.Structure):
    _fields_ = [("hits", ctypes.c_int64), ("misses", ctypes.c_int64), ("bytes_h2d", ctypes.c_int64),
                ("prefetched", ctypes.c_int64), ("prefetch_used", ctypes.c_int64), ("predicted", ctypes.c_int64),
                ("predicted_of", ctypes.c_int64), ("resident_slots", ctypes.c_int32), ("n_pinned", ctypes.c_int32)]


class ColiError(RuntimeError):
    def __init__(self, status: int, where: str, detail: str):
        super().__init__(f"{where}: status {status} ({detail})")
        self.status = status


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with __graft_entry__.build() "
                          "(the CUDA library is required; there is no CPU path)")
    L = ctypes.CDLL(LIB_PATH)
    vp, i32, f32 = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
    pcfg = ctypes.POINTER(Config)
    L.coli_moe_layer_create.argtypes = [pcfg, vp, vp, vp, vp, vp, vp, i32, ctypes.POINTER(vp)]
    L.coli_moe_layer_set_experts.argtypes = [vp, i32, i32, vp, vp]
    L.coli_moe_layer_destroy.argtypes = [vp]
    L.coli_moe_layer_destroy.restype = None
    L.coli_moe_layer_config.argtypes = [vp, pcfg]
    L.coli_moe_route.argtypes = [vp, vp, i32, i32, vp, vp, vp]
    L.coli_moe_forward.argtypes = [vp, vp, vp, i32, i32, vp]
    L.coli_moe_stack_forward.argtypes = [vp, i32, vp, i32, f32, vp]
    L.coli_moe_get_stats.argtypes = [vp, ctypes.POINTER(i32), ctypes.POINTER(ctypes.c_int64), vp]
    L.coli_moe_get_launch_count.argtypes = [vp, ctypes.POINTER(ctypes.c_int64)]
    L.coli_moe_get_plan.argtypes = [vp, vp, vp, vp, vp, vp, ctypes.POINTER(i32), vp, vp]
    L.coli_moe_expert_bytes.argtypes = [i32, i32]
    L.coli_moe_expert_bytes.restype = ctypes.c_int64
    L.coli_moe_set_profiling.argtypes = [vp, i32]
    L.coli_moe_get_profile.argtypes = [vp, vp, ctypes.POINTER(ctypes.c_int64)]
    L.coli_moe_stage_name.argtypes = [i32]
    L.coli_moe_stage_name.restype = ctypes.c_char_p
    L.coli_moe_sync.argtypes = [vp]
    L.coli_moe_set_trace.argtypes = [vp, vp, i32]
    L.coli_moe_set_ring.argtypes = [vp, i32, i32]
    L.coli_moe_route_noalloc.argtypes = [vp, vp, i32, i32, i32, vp, i32, i32, vp, vp, vp]
    L.coli_moe_set_fused.argtypes = [vp, i32]
    L.coli_moe_set_tensor_cores.argtypes = [vp, i32]
    L.coli_moe_debug_fail_alloc.argtypes = [i32]
    L.coli_clock_stamp.argtypes = [vp, i32, vp]
    L.coli_moe_debug_wait_test.argtypes = [vp, i32, ctypes.c_int64]
    L.coli_moe_layer_create_cached.argtypes = [pcfg, vp, vp, vp, vp, vp, vp, i32, i32, ctypes.POINTER(vp)]
    L.coli_moe_cache_stats.argtypes = [vp, ctypes.POINTER(CacheStats), vp, i32]
    L.coli_moe_cache_pin.argtypes = [vp, vp, i32]
    L.coli_moe_cache_prefetch.argtypes = [vp, vp, i32]
    L.coli_moe_cache_set_lookahead.argtypes = [vp, i32]
    L.coli_moe_cache_slots.argtypes = [vp, vp]
    L.coli_moe_set_expert_top_p.argtypes = [vp, ctypes.c_double]
    L.coli_moe_layer_create_ep.argtypes = [pcfg, vp, vp, vp, vp, vp, vp, i32, i32, i32, ctypes.POINTER(vp)]
    L.coli_moe_ep_range.argtypes = [i32, i32, i32, ctypes.POINTER(i32), ctypes.POINTER(i32)]
    L.coli_moe_router_fallbacks.argtypes = [vp, ctypes.POINTER(i32), ctypes.POINTER(i32)]
    L.coli_status_string.argtypes = [i32]
    L.coli_status_string.restype = ctypes.c_char_p
    L.coli_last_error.argtypes = []
    L.coli_last_error.restype = ctypes.c_char_p
    return L


lib = _load()


def _check(status: int, where: str) -> None:
    if status != COLI_OK:
        raise ColiError(status, where, (lib.coli_last_error() or b"").decode())


def _ptr(a) -> int | None:
    """Address of a torch tensor or numpy array (None stays None)."""
    if a is None:
        return None
    if hasattr(a, "data_ptr"):
        return a.data_ptr() if a.numel() else None
    if hasattr(a, "ctypes"):
        if not a.flags["C_CONTIGUOUS"]:
            raise ValueError("array must be C-contiguous")
        return a.ctypes.data
    return int(a)


def _stream(stream) -> int | None:
    if stream is None:
        try:
            import torch
            return torch.cuda.current_stream().cuda_stream
        except Exception:
            return None
    return getattr(stream, "cuda_stream", stream)


def _dtype_of(t) -> int:
    name = str(getattr(t, "dtype", ""))
    if name.endswith("float32"):
        return F32
    if name.endswith("bfloat16") or name.endswith("uint16") or name.endswith("int16"):
        return BF16
    raise TypeError(f"unsupported activation dtype {name}")


def expert_bytes(hidden: int, inter: int) -> int:
    return lib.coli_moe_expert_bytes(hidden, inter)


class Layer:
    """One MoE layer on a CUDA device: every expert resident in HBM; with
    ``resident`` = R, an expert cache of R routed experts in HBM over a
    page-locked host copy of all of them; with ``ep`` = (rank, world), rank's
    share of an expert-parallel layer (forward writes its partial output)."""

    def __init__(self, cfg: Config, router_w, router_bias=None, expert_q=None, expert_scales=None,
                 shared_q=None, shared_scales=None, device: int = 0, resident: int | None = None, ep=None):
        h = ctypes.c_void_p()
        args = (ctypes.byref(cfg), _ptr(router_w), _ptr(router_bias), _ptr(expert_q), _ptr(expert_scales),
                _ptr(shared_q), _ptr(shared_scales))
        if ep is not None:
            if resident is not None:
                raise ValueError("an expert-parallel layer has no expert cache")
            _check(lib.coli_moe_layer_create_ep(*args, int(ep[0]), int(ep[1]), device, ctypes.byref(h)),
                   "coli_moe_layer_create_ep")
        elif resident is None:
            _check(lib.coli_moe_layer_create(*args, device, ctypes.byref(h)), "coli_moe_layer_create")
        else:
            _check(lib.coli_moe_layer_create_cached(*args, resident, device, ctypes.byref(h)),
                   "coli_moe_layer_create_cached")
        self._h = h
        self.cfg = cfg
        self.device = device
        self.resident = resident

    @property
    def handle(self) -> ctypes.c_void_p:
        if self._h is None:
            raise ValueError("layer is destroyed")
        return self._h

    def set_experts(self, first: int, count: int, q, scales) -> None:
        _check(lib.coli_moe_layer_set_experts(self.handle, first, count, _ptr(q), _ptr(scales)),
               "coli_moe_layer_set_experts")

    def close(self) -> None:
        if getattr(self, "_h", None) is not None:
            lib.coli_moe_layer_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def route(self, x, ids, weights, n_tokens: int | None = None, stream=None) -> None:
        T = x.shape[0] if n_tokens is None else n_tokens
        _check(lib.coli_moe_route(self.handle, _ptr(x), _dtype_of(x), T, _ptr(ids), _ptr(weights), _stream(stream)),
               "coli_moe_route")

    def router_fallbacks(self) -> tuple[bool, int]:
        """(the certified router routes this layer's batches of 64 tokens and more,
        tokens of its last batch that took the fp64 fallback); synchronises."""
        c, n = ctypes.c_int32(), ctypes.c_int32()
        _check(lib.coli_moe_router_fallbacks(self.handle, ctypes.byref(c), ctypes.byref(n)),
               "coli_moe_router_fallbacks")
        return bool(c.value), int(n.value)

    def forward(self, x, y, n_tokens: int | None = None, stream=None) -> None:
        T = x.shape[0] if n_tokens is None else n_tokens
        _check(lib.coli_moe_forward(self.handle, _ptr(x), _ptr(y), _dtype_of(x), T, _stream(stream)),
               "coli_moe_forward")

    def stats(self, counts=None):
        nu = ctypes.c_int()
        b = ctypes.c_int64()
        _check(lib.coli_moe_get_stats(self.handle, ctypes.byref(nu), ctypes.byref(b), _ptr(counts)),
               "coli_moe_get_stats")
        return nu.value, b.value

    def launch_count(self) -> int:
        """Kernels of the library this layer's route/forward/stack calls enqueued so far."""
        n = ctypes.c_int64()
        _check(lib.coli_moe_get_launch_count(self.handle, ctypes.byref(n)), "coli_moe_get_launch_count")
        return n.value

    def sync(self) -> None:
        """Wait for the last forward; raises if the device reported a timeout."""
        _check(lib.coli_moe_sync(self.handle), "coli_moe_sync")

    def set_fused(self, on) -> None:
        """True: the persistent kernel for batches of up to 64 tokens (default); False: separate kernels."""
        _check(lib.coli_moe_set_fused(self.handle, 1 if on else 0), "coli_moe_set_fused")

    def set_expert_top_p(self, p: float) -> None:
        """Adaptive expert top-p (opt-in; changes routing): keep the shortest
        prefix of each token's top-K whose weights reach p. 1.0: plain top-K."""
        _check(lib.coli_moe_set_expert_top_p(self.handle, float(p)), "coli_moe_set_expert_top_p")

    def debug_wait_test(self, enable: bool, wait_ns: int = 0) -> None:
        """Testing aid: bound the persistent kernel's waits to wait_ns and, when
        enabled, make each launch give up on a flag that nothing sets."""
        _check(lib.coli_moe_debug_wait_test(self.handle, 1 if enable else 0, wait_ns), "coli_moe_debug_wait_test")

    def set_tensor_cores(self, mode) -> None:
        """0 / False: CUDA-core kernels; 1 / True: tensor cores for bf16 (default);
        2: tensor cores for fp32 too (fp16 hi + lo tokens)."""
        _check(lib.coli_moe_set_tensor_cores(self.handle, int(mode)), "coli_moe_set_tensor_cores")

    def set_trace(self, buffer, capacity: int) -> None:
        """Record the persistent kernel's item timeline into a zeroed device
        int64 buffer of 16 + 8 * capacity entries (None disables)."""
        _check(lib.coli_moe_set_trace(self.handle, _ptr(buffer), capacity), "coli_moe_set_trace")

    def set_ring(self, stages: int, blocks_per_stage: int = 8) -> None:
        _check(lib.coli_moe_set_ring(self.handle, stages, blocks_per_stage), "coli_moe_set_ring")

    def set_profiling(self, on: bool) -> None:
        _check(lib.coli_moe_set_profiling(self.handle, 1 if on else 0), "coli_moe_set_profiling")

    def profile(self):
        """(stage name -> total device ms, number of forwards) since profiling was enabled."""
        buf = (ctypes.c_double * N_STAGES)()
        n = ctypes.c_int64()
        _check(lib.coli_moe_get_profile(self.handle, ctypes.cast(buf, ctypes.c_void_p), ctypes.byref(n)),
               "coli_moe_get_profile")
        return {lib.coli_moe_stage_name(i).decode(): float(buf[i]) for i in range(N_STAGES)}, n.value

    def cache_stats(self, reset: bool = False, usage: bool = False):
        """Counters of a cached layer (dict); with usage=True also the per-expert
        routing counts (numpy int64 [E]) under "usage"."""
        import numpy as np
        st = CacheStats()
        use = np.zeros(self.cfg.n_experts, np.int64) if usage else None
        _check(lib.coli_moe_cache_stats(self.handle, ctypes.byref(st), _ptr(use), 1 if reset else 0),
               "coli_moe_cache_stats")
        out = {name: getattr(st, name) for name, _ in CacheStats._fields_}
        if usage:
            out["usage"] = use
        return out

    def pin(self, ids) -> None:
        """Pin these experts (resident, never evicted); an empty list unpins all."""
        import numpy as np
        a = np.ascontiguousarray(ids, dtype=np.int32)
        _check(lib.coli_moe_cache_pin(self.handle, _ptr(a) if a.size else None, int(a.size)), "coli_moe_cache_pin")

    def pin_hot(self, n: int, usage=None):
        """Pin the n experts routed to most often (from `usage`, e.g. counts saved
        by an earlier session, else this layer's own); returns their ids."""
        import numpy as np
        u = self.cache_stats(usage=True)["usage"] if usage is None else np.asarray(usage)
        ids = np.argsort(-u, kind="stable")[:n].astype(np.int32)
        self.pin(ids)
        return ids

    def prefetch(self, ids) -> None:
        """Copy these experts into HBM ahead of need (asynchronous, copy stream)."""
        import numpy as np
        a = np.ascontiguousarray(ids, dtype=np.int32)
        _check(lib.coli_moe_cache_prefetch(self.handle, _ptr(a) if a.size else None, int(a.size)),
               "coli_moe_cache_prefetch")

    def cache_slots(self):
        """Slot of each routed expert in HBM (numpy int32 [E]; -1: not resident)."""
        import numpy as np
        out = np.zeros(self.cfg.n_experts, np.int32)
        _check(lib.coli_moe_cache_slots(self.handle, _ptr(out)), "coli_moe_cache_slots")
        return out

    def set_lookahead(self, on: bool) -> None:
        _check(lib.coli_moe_cache_set_lookahead(self.handle, 1 if on else 0), "coli_moe_cache_set_lookahead")

    def plan(self, T: int):
        """Host copies of the last forward's routing and batch-union plan."""
        import numpy as np
        E, K = self.cfg.n_experts, self.cfg.top_k
        out = dict(ids=np.zeros((T, K), np.int32), weights=np.zeros((T, K), np.float32),
                   cnt=np.zeros(E, np.int32), off=np.zeros(E + 1, np.int32), unique=np.zeros(E, np.int32),
                   pos=np.zeros((T, K), np.int32), tok=np.zeros(max(T * K, 1), np.int32))
        nu = ctypes.c_int()
        _check(lib.coli_moe_get_plan(self.handle, _ptr(out["ids"]), _ptr(out["weights"]), _ptr(out["cnt"]),
                                     _ptr(out["off"]), _ptr(out["unique"]), ctypes.byref(nu), _ptr(out["pos"]),
                                     _ptr(out["tok"])), "coli_moe_get_plan")
        out["unique"] = out["unique"][:nu.value]
        out["tok"] = out["tok"][:T * K]
        return out


def ep_range(n_experts: int, rank: int, world: int) -> tuple[int, int]:
    """The routed experts [first, end) rank `rank` of `world` holds."""
    a, b = ctypes.c_int(), ctypes.c_int()
    _check(lib.coli_moe_ep_range(n_experts, rank, world, ctypes.byref(a), ctypes.byref(b)), "coli_moe_ep_range")
    return a.value, b.value


def route_noalloc(router_w, router_bias, n_experts: int, hidden: int, top_k: int, x, ids, weights,
                  n_tokens: int | None = None, stream=None) -> None:
    """Routing without a layer and without any device allocation (fixed
    504 KiB scratch in the library; at most 63 tokens and 1024 experts)."""
    T = x.shape[0] if n_tokens is None else n_tokens
    _check(lib.coli_moe_route_noalloc(_ptr(router_w), _ptr(router_bias), n_experts, hidden, top_k, _ptr(x),
                                      _dtype_of(x), T, _ptr(ids), _ptr(weights), _stream(stream)),
           "coli_moe_route_noalloc")


def stack_forward(layers, x, n_tokens: int | None = None, eps: float = 1e-6, stream=None) -> None:
    """x <- x + MoE_l(RMSNorm(x)) over the layers, in place on fp32 x."""
    T = x.shape[0] if n_tokens is None else n_tokens
    arr = (ctypes.c_void_p * len(layers))(*[l.handle.value for l in layers])
    _check(lib.coli_moe_stack_forward(ctypes.cast(arr, ctypes.c_void_p), len(layers), _ptr(x), T, eps,
                                      _stream(stream)), "coli_moe_stack_forward")


def debug_fail_alloc(nth: int) -> None:
    """Make the nth device allocation of the library from now on fail (0: off)."""
    _check(lib.coli_moe_debug_fail_alloc(nth), "coli_moe_debug_fail_alloc")


def clock_stamp(buffer, n_blocks: int, stream=None) -> None:
    """Per-SM {SM id, clock counter, global timer ns} into a device int64 buffer [n_blocks][3]."""
    _check(lib.coli_clock_stamp(_ptr(buffer), n_blocks, _stream(stream)), "coli_clock_stamp")


def sm_clock_mhz(stamp0, stamp1):
    """Mean clock rate (MHz) of each SM between two stamps (host int64 arrays [n][3]),
    over the SMs present in both; a list of floats."""
    first = {int(r[0]): (int(r[1]), int(r[2])) for r in stamp0}
    out = {}
    for r in stamp1:
        sm = int(r[0])
        if sm in first and sm not in out:
            dc, dt = int(r[1]) - first[sm][0], int(r[2]) - first[sm][1]
            if dt > 0 and dc > 0:
                out[sm] = dc / dt * 1e3
    return list(out.values())


def make_config(hidden, inter, n_experts, top_k, n_shared, max_tokens) -> Config:
    return Config(hidden=hidden, inter=inter, n_experts=n_experts, top_k=top_k, n_shared=n_shared,
                  group_size=64, max_tokens=max_tokens)
