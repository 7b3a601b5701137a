#!/usr/bin/env python
"""Benchmark of the int4 expert-FFN MoE layer on B200.

Default workload: one full-size MoE layer (hidden 6144, expert intermediate
2048, 256 routed experts top-8 with softmax-renormalised weights, one shared
expert; int4 gs64 weights with fp16 scales, N(0, 0.02) before encoding; router
fp32, bias 0), decode batch 1, a fresh seeded N(0,1) fp32 token every step.

One step = one forward of the layer (router, top-k, batch-union plan, fused
int4 gate/up + SwiGLU, down, weighted combine with the shared expert) for one
batch. Inputs are resident in HBM before the timed region; L2 is flushed
between steps by a 256 MiB memset recorded outside the per-step events.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload decode_b1|decode_b32|prefill_2048|stack30_b1|stack30_b8|stack30_b64|
                                decode_b1_cached|stack4_b1_cached]

Prints one JSON line (rank 0). N > 1 runs N independent replicas (one per
rank, launched by torch.distributed.run), weak scaling, max time over ranks.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "MoE int4 layer tokens/s; streamed-expert HBM GB/s vs ~8 TB/s (batch 1–2048)"
H, I, E_FULL, K, S = 6144, 2048, 256, 8, 1
E = E_FULL
EXPERT_BYTES = 20_054_016          # int4 nibbles + fp16 scales of one expert
GU_BYTES = 13_369_344              # gate + up of one expert
DOWN_BYTES = 6_684_672             # down of one expert
ROUTER_BYTES = E * H * 4           # fp32 router matrix

WORKLOADS = {
    "decode_b1": dict(T=1, zipf=False, bf16=False,
                      desc="one full-size layer, decode batch 1, bias 0, fresh fp32 token per step"),
    "decode_b32": dict(T=32, zipf=True, bf16=False,
                       desc="one full-size layer, decode batch 32, Zipf(1.1) router bias, fp32"),
    "prefill_2048": dict(T=2048, zipf=True, bf16=True,
                         desc="one full-size layer, prefill 2048 tokens, Zipf(1.1) router bias, bf16"),
    # profiling case: the decode step with 16 routed experts (same 9 active
    # experts per token, 0.34 GB resident instead of 5.16 GB)
    "decode_b1_e16": dict(T=1, zipf=False, bf16=False, E=16,
                          desc="full-size experts, 16 routed experts top-8 + shared, decode batch 1 (profiling case)"),
    # profiling case for the tensor-core kernels: 64 routed experts, 512 bf16
    # tokens (about 64 tokens per expert, as in the full prefill; 1.3 GB resident)
    "prefill_e64": dict(T=512, zipf=True, bf16=True, E=64,
                        desc="full-size experts, 64 routed experts top-8 + shared, 512 bf16 tokens, Zipf(1.1) (profiling case)"),
    # 30 full-size layers (154.8 GB of int4 experts resident), x <- x + MoE_l(RMSNorm(x)),
    # independent seeded routers and Zipf(1.1) biases per layer, fp32 residual stream
    "stack30_b1": dict(T=1, zipf=True, bf16=False, layers=30,
                       desc="30-layer stack of the full-size layer, decode batch 1, Zipf(1.1) per layer"),
    "stack30_b8": dict(T=8, zipf=True, bf16=False, layers=30,
                       desc="30-layer stack of the full-size layer, decode batch 8, Zipf(1.1) per layer"),
    "stack30_b64": dict(T=64, zipf=True, bf16=False, layers=30,
                        desc="30-layer stack of the full-size layer, decode batch 64, Zipf(1.1) per layer"),
    # expert cache over page-locked host memory: 64 of the 256 routed experts of a layer in HBM,
    # all 256 in host memory; Zipf(1.1) routing; after an untimed learning pass the 48 experts
    # routed to most often are pinned (the learned hot set), least-recently-used eviction in the
    # other 16 slots; every miss is one host-to-HBM copy of the expert's 20 MB
    "decode_b1_cached": dict(T=1, zipf=True, bf16=False, resident=64, pin=48,
                             desc="one full-size layer as an expert cache (64 of 256 routed experts in HBM, 48 "
                                  "pinned by learned usage, LRU), decode batch 1, Zipf(1.1) router bias, fp32"),
    # speculative verify: one sequence's current token and 3 draft positions as one batch, so
    # the batch-union reads each distinct expert once for all four; positions of one sequence
    # share part of their hidden state (x_j = 0.6 x_0 + 0.8 z_j); accepted tokens per forward
    # taken as 2.5 (the pages report 2.2-2.8 with an int8 draft head)
    "verify_b4": dict(T=4, zipf=True, bf16=False, verify=dict(rho=0.6, tau=2.5),
                      desc="one full-size layer, speculative verify batch of 1 + 3 draft positions of one "
                           "sequence (correlated tokens), Zipf(1.1) router bias, fp32"),
    "verify_b4_cached": dict(T=4, zipf=True, bf16=False, resident=64, pin=32, verify=dict(rho=0.6, tau=2.5),
                             desc="speculative verify batch (1 + 3 draft positions) on an expert-cache layer "
                                  "(64 of 256 in HBM, 32 pinned, LRU), Zipf(1.1), fp32"),
    "stack4_b1_cached": dict(T=1, zipf=True, bf16=False, layers=4, resident=64, pin=48,
                             desc="4-layer stack of expert-cache layers (64 of 256 in HBM each, 48 pinned, LRU), "
                                  "each next layer's router run one layer ahead to prefetch, decode batch 1, "
                                  "Zipf(1.1) per layer"),
}
X_SEED0 = 1000  # step s draws its activations with seed X_SEED0 + s
TOPP = 1.0      # --expert-top-p: adaptive expert top-p of every layer (1: plain top-K)


def topp_arg():
    """The oracle's top_p argument for TOPP (None: plain top-K)."""
    return TOPP if TOPP < 1.0 else None
LEARN_SEED0 = 500_000  # the cache workloads' learning pass draws its own tokens
FUSED_MODE = {"i8": 1, "separate": 0}


DEFAULT_STEPS = {"decode_b1": 10000, "decode_b32": 2000, "prefill_2048": 100, "decode_b1_e16": 1000, "prefill_e64": 100,
                 "stack30_b1": 300, "stack30_b8": 200, "stack30_b64": 100, "decode_b1_cached": 2000,
                 "stack4_b1_cached": 500, "verify_b4": 5000, "verify_b4_cached": 1000}


def step_seed(step, rank):
    """Seed of the activations of `step` on `rank`: every replica draws its own token stream."""
    return X_SEED0 + step + 100000 * rank


def max_over_ranks(value, dist, device):
    """The largest of the ranks' values (every rank gets it); `dist` None: single process."""
    if dist is None:
        return value
    import torch
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def fill_tokens(torch, synth, wl, xs, seed_of, stream):
    """Step i's tokens into xs[i] (device): N(0,1) rows drawn with seed
    seed_of(i); for a verify workload rows 1.. become positions of the same
    sequence as row 0, x_j = rho x_0 + sqrt(1 - rho^2) z_j."""
    T = xs.shape[1]
    for i in range(xs.shape[0]):
        synth.x_dev(seed_of(i), 0, T, H, 1 if wl["bf16"] else 0, xs[i].data_ptr(), stream.cuda_stream)
    v = wl.get("verify")
    if v:
        rho = v["rho"]
        xs[:, 1:] = rho * xs[:, :1] + (1.0 - rho * rho) ** 0.5 * xs[:, 1:]


def verify_report(wl, mean_loads, forwards_per_s):
    """Expert loads and accepted tokens of a verify workload (loads = distinct
    routed experts of the batch + the shared experts)."""
    v = wl["verify"]
    return {"positions": wl["T"], "rho": v["rho"], "tokens_per_forward_assumed": v["tau"],
            "expert_loads_per_forward": round(mean_loads, 2),
            "expert_loads_per_token": round(mean_loads / v["tau"], 2),
            "expert_loads_per_token_plain_decode": K + S,
            "accepted_tokens_per_s": round(forwards_per_s * v["tau"], 1),
            "note": ("accepted tokens per forward is a property of the draft head, not of this layer; "
                     "the value assumed is the middle of the pages' 2.2-2.8")}


def ep_combine(y, dist):
    """Exchange step of the expert-parallel layer: every rank's partial output
    is replaced by the sum over the ranks (all-reduce; NCCL on GPUs)."""
    if dist is not None and dist.is_initialized() and dist.get_world_size() > 1:
        dist.all_reduce(y, op=dist.ReduceOp.SUM)
    return y


def job_tokens_per_s(world_size, steps, tokens_per_step, total_ms):
    """Whole-job throughput: the tokens every replica processed over the slowest rank's time."""
    return world_size * steps * tokens_per_step / (total_ms * 1e-3)


# DRAM bytes per launch (dram__bytes_read.sum + dram__bytes_write.sum) from
# one ncu capture, keyed by (kernel, workload). A value stands only while the
# kernel's sources hash to the recorded digest; otherwise `traffic` is null.
NCU_TRAFFIC = {
    ("moe_decode_i8_kernel", "decode_b1"): dict(
        bytes=190_110_000,
        sources=('decode_i8.cu', 'common.cuh', 'topk.cuh', 'kernels.cuh'),
        sha256_16="f065e23c972e8b9a",
        note="ncu capture of the 16-expert decode case (184.21 MB read + written per launch) + 5.90 MB for "
             "the 256-expert router"),
    ("moe_prefill_tc_kernel (gateup)", "prefill_2048"): dict(
        bytes=4_531_153_152,
        sources=('prefill_tc.cu', 'tcgen05.cuh', 'common.cuh', 'kernels.cuh'),
        sha256_16="4bbb8b0b50917590",
        note="ncu capture (dram__bytes_read.sum + dram__bytes_write.sum, one pass) of the first gate/up launch of "
             "this workload: 4,464 MB read + 67 MB written, against 3,738 MB algorithmic (1.21x: a hot expert's "
             "weights are read again per token tile, the token rows again per pair of row tiles)"),
}


def ncu_traffic(kernel, workload):
    rec = NCU_TRAFFIC.get((kernel, workload))
    if rec is None:
        return None, None
    import hashlib
    h = hashlib.sha256()
    for f in rec["sources"]:
        with open(os.path.join(ROOT, "int4_expert_ffn_router_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    if h.hexdigest()[:16] != rec["sha256_16"]:
        return None, "kernel sources changed since the ncu capture"
    return rec["bytes"], rec["note"]


def step_percentiles(step_ms):
    """p10 / median / p90 of this rank's per-step device times (ms)."""
    v = sorted(step_ms)
    if not v:
        return None
    pick = lambda q: v[min(len(v) - 1, int(round(q * (len(v) - 1))))]
    return {"p10": round(pick(0.1), 5), "p50": round(pick(0.5), 5), "p90": round(pick(0.9), 5)}


def load_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return json.load(f)
    except OSError:
        return {}


def dominant_roofline(stages, n_launches, T, mean_unique, E, elt, tc, peaks):
    """Roofline of the kernel with the largest device time.

    stages: total device ms per stage over `n_launches` launches of each stage
    kernel. Algorithmic work per launch:
      persistent decode kernel: active experts + router bytes + x and y;
      CUDA-core gate/up: active gate/up bytes + x + h (fp32);
      CUDA-core down: active down bytes + h + o (fp32);
      tensor-core gate/up: 2 * T (K + S) * H * 2I flops; down: 2 * T (K + S) * I * H.
    """
    dom = max(stages, key=lambda k: stages[k])
    avg_s = stages[dom] / max(n_launches, 1) * 1e-3
    pairs = T * (K + S)
    router_bytes = E * H * 4
    act = 2 * T * H * elt
    if tc and dom in ("gateup", "down"):
        flops = 2.0 * pairs * H * 2 * I if dom == "gateup" else 2.0 * pairs * I * H
        ach = flops / avg_s / 1e12
        peak = peaks.get("bf16_tflops", 1590.0)
        roof = {"bound": "tensor", "kernel": f"moe_prefill_tc_kernel ({dom})", "achieved": round(ach, 1),
                "peak": peak, "unit": "TFLOP/s", "frac": round(ach / peak, 4), "traffic": None,
                "peak_source": "measured burst (MEASURED_PEAKS.json bf16_tflops; the f16 MMA rate equals bf16)"
                if "bf16_tflops" in peaks else "fallback 1.59 PFLOP/s",
                "flops_per_launch": flops, "avg_launch_us": round(avg_s * 1e6, 2)}
        if "bf16_tflops_sustained" in peaks:
            roof["frac_of_sustained"] = round(ach / peaks["bf16_tflops_sustained"], 4)
        return dom, roof
    alg = {"gateup": (mean_unique + S) * GU_BYTES + T * H * elt + pairs * I * 4,
           "down": (mean_unique + S) * DOWN_BYTES + pairs * (I + H) * 4,
           "router": router_bytes + T * H * elt,
           "fused": (mean_unique + S) * EXPERT_BYTES + router_bytes + act}
    if dom not in alg:
        return dom, None
    ach = alg[dom] / avg_s / 1e9
    peak = peaks.get("hbm_gbs", 6650.0)
    names = {"fused": "moe_decode_i8_kernel", "gateup": "gateup_core_kernel", "down": "down_core_kernel",
             "router": "router kernels"}
    return dom, {"bound": "hbm", "kernel": names[dom], "achieved": round(ach, 1), "peak": peak, "unit": "GB/s",
                 "frac": round(ach / peak, 4), "traffic": None,
                 "peak_source": "measured (MEASURED_PEAKS.json hbm_gbs)" if "hbm_gbs" in peaks else "fallback 6.65 TB/s",
                 "bytes_per_launch": int(alg[dom]), "avg_launch_us": round(avg_s * 1e6, 2)}


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None, help="default: 10000 (decode_b1), 2000 (decode_b32), 100 (prefill)")
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=sorted(WORKLOADS), default="decode_b1")
    ap.add_argument("--cpu-seconds", type=float, default=20.0, help="budget of the CPU-oracle sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--parallel", choices=["replicas", "ep"], default="replicas",
                    help="N > 1: independent replicas (default, weak scaling) or one layer with its experts "
                         "sharded over the ranks (expert parallelism, strong scaling)")
    ap.add_argument("--expert-top-p", type=float, default=1.0,
                    help="adaptive expert top-p of every layer, in (0, 1] (opt-in routing variant; 1: plain top-8)")
    ap.add_argument("--decode-kernel", choices=["i8", "separate"], default="i8",
                    help="batches of up to 64 tokens: the persistent integer-MMA kernel (default) or the separate "
                         "kernels")
    a = ap.parse_args()
    if a.steps is None:
        a.steps = DEFAULT_STEPS[a.workload]
    return a


def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


# --------------------------------------------------------------- CPU oracle leg
class OracleLeg:
    """The fp64 oracle on the host cores, one bounded sample per step (input
    generation, including the selected experts, is untimed and cached)."""

    def __init__(self, wl):
        import oracle
        import synth
        self.oracle, self.synth, self.wl = oracle, synth, wl
        self.E = E = wl.get("E", E_FULL)
        self.bias = synth.zipf_bias(0, 0, E)[0] if wl["zipf"] else None
        self.wr = synth.router(0, 0, E, H)
        self.cfg = oracle.Cfg(hidden=H, inter=I, n_experts=E, top_k=K, n_shared=S, expert_top_p=topp_arg() or 0.0)
        self.cache = {}
        self.Ts = wl["T"] if wl["T"] <= 2 else 2   # tokens of a step the sample covers
        self.layers = wl.get("layers", 0)
        if self.layers:
            # stack: one token through the first Ls layers, time scaled to all layers
            self.Ts, self.Ls = 1, 2
            self.wrs = [synth.router(0, l, E, H) for l in range(self.Ls)]
            self.biases = [synth.zipf_bias(0, l, E)[0] for l in range(self.Ls)]

    def step(self, i):
        """Returns (tokens, oracle seconds) of the sample of step i."""
        import numpy as np
        wl, syn = self.wl, self.synth
        if self.layers:
            return self._stack_step(i)
        x = syn.x_bf16(X_SEED0 + i, 0, wl["T"], H) if wl["bf16"] else syn.x_f32(X_SEED0 + i, 0, wl["T"], H)
        if wl.get("verify"):  # positions of one sequence, as fill_tokens forms them
            rho = wl["verify"]["rho"]
            x[1:] = (np.float32(rho) * x[:1] + np.float32((1.0 - rho * rho) ** 0.5) * x[1:]).astype(np.float32)
        x = np.ascontiguousarray(x[:self.Ts])
        ids, _ = self.oracle.topk(self.oracle.router_logits(self.wr, self.bias, x), K, top_p=topp_arg())
        E = self.E
        experts = [None] * (E + S)
        for e in {e for e in ids.ravel().tolist() if e >= 0} | set(range(E, E + S)):
            if e not in self.cache:
                self.cache[e] = syn.expert(0, 0, e, H, I)
            experts[e] = self.cache[e]
        t0 = time.perf_counter()
        self.oracle.moe_forward(self.cfg, self.wr, self.bias, experts, x)
        return self.Ts, time.perf_counter() - t0

    def _stack_step(self, i):
        import numpy as np
        syn, orc, E = self.synth, self.oracle, self.E
        x = np.ascontiguousarray(syn.x_f32(X_SEED0 + i, 0, self.wl["T"], H)[:1])
        spent = 0.0
        for l in range(self.Ls):
            xn = orc.rmsnorm(x).astype(np.float32)  # the layer input the oracle step forms
            ids, _ = orc.topk(orc.router_logits(self.wrs[l], self.biases[l], xn), K, top_p=topp_arg())
            experts = [None] * (E + S)
            for e in {e for e in ids.ravel().tolist() if e >= 0} | set(range(E, E + S)):
                if (l, e) not in self.cache:
                    self.cache[(l, e)] = syn.expert(0, l, e, H, I)
                experts[e] = self.cache[(l, e)]
            t0 = time.perf_counter()
            orc.stack_step(self.cfg, self.wrs[l], self.biases[l], experts, x)
            spent += time.perf_counter() - t0
        return 1, spent * self.layers / self.Ls

    def cores(self):
        return int(os.environ.get("OMP_NUM_THREADS", os.cpu_count() or 1))


def oracle_sample(wl, budget_s):
    leg = OracleLeg(wl)
    tokens, spent, steps = 0, 0.0, 0
    wall = time.time()
    while spent < budget_s and time.time() - wall < 4 * budget_s:
        n, dt = leg.step(steps)
        tokens += n
        spent += dt
        steps += 1
    what = (f"{steps} steps x 1 token through the first {leg.Ls} of {leg.layers} layers (time scaled to "
            f"{leg.layers} layers)") if leg.layers else f"{steps} steps x {leg.Ts} token(s) of the workload"
    return dict(value=round(tokens / spent, 4), unit="tokens/s", cores=leg.cores(), kind="oracle",
                sample=f"{what} through the fp64 oracle, {spent:.1f} s of oracle time (input and expert "
                       f"generation untimed)")


# -------------------------------------------------------------------- GPU side
class Clocks:
    """SM clocks over the timed region, two ways: nvidia-smi sampled every
    20 ms (clock and throttle reasons), and per-SM clock-counter / global-timer
    stamps taken by a one-block-per-SM kernel just before and just after the
    timed loop, which give each SM's mean clock rate over the region however
    short it is."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    REASONS = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]

    def __init__(self, index, coli=None, torch=None, stream=None):
        self.index = index
        self.coli, self.torch, self.stream = coli, torch, stream
        self.file = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(index), f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "20"],
                                         stdout=self.file, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
        self.stamps = None
        if coli is not None:
            n = torch.cuda.get_device_properties(index).multi_processor_count
            self.n_sm = n
            self.stamps = torch.zeros((2, n, 3), dtype=torch.int64, device=torch.device("cuda", index))
            coli.clock_stamp(self.stamps[0], n, stream=stream)

    def end_region(self):
        """Second stamp, enqueued right after the timed loop."""
        if self.stamps is not None:
            self.coli.clock_stamp(self.stamps[1], self.n_sm, stream=self.stream)

    @staticmethod
    def query_once(index):
        """One nvidia-smi reading (max clock and throttle reasons right now)."""
        try:
            out = subprocess.run(["nvidia-smi", "-i", str(index), f"--query-gpu={Clocks.FIELDS}",
                                  "--format=csv,noheader,nounits"], capture_output=True, text=True, timeout=20)
            return [out.stdout.strip().split(",")]
        except Exception:
            return []

    def stop(self):
        rows = []
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(5)
            except Exception:
                self.proc.kill()
            self.file.flush()
            self.file.seek(0)
            rows = [r.split(",") for r in self.file.read().strip().splitlines() if r.strip()]
        os.unlink(self.file.name)
        sampled = len(rows)
        if not rows:
            rows = self.query_once(self.index)
        sm, mx, reasons = [], 0.0, set()
        for r in rows:
            try:
                if sampled:
                    sm.append(float(r[1]))
                mx = max(mx, float(r[2]))
                for n, v in zip(self.REASONS, r[5:9]):
                    if v.strip().lower() == "active":
                        reasons.add(n)
            except (ValueError, IndexError):
                continue
        out = {"sm_max_mhz": mx or None, "reasons": sorted(reasons), "samples": sampled}
        if sm:
            out["sm_mhz"] = statistics.median(sm)
            out["sm_mhz_source"] = "nvidia-smi, sampled every 20 ms during the timed region"
        if self.stamps is not None:
            st = self.stamps.cpu().numpy()
            mhz = self.coli.sm_clock_mhz(st[0], st[1])
            if mhz:
                out["sm_mhz_stamps"] = round(statistics.median(mhz), 1)
                out["sm_mhz_stamps_min"] = round(min(mhz), 1)
                out["stamped_sms"] = len(mhz)
                if "sm_mhz" not in out:
                    out["sm_mhz"] = out["sm_mhz_stamps"]
                    out["sm_mhz_source"] = ("median over SMs of clock cycles / global-timer ns between "
                                            "stamps taken right before and after the timed loop")
        if not sampled:
            out["reasons_note"] = "region shorter than one sample: reasons read once right after it"
        return out


def build_layer(torch, coli, synth, wl, device, max_tokens, layer_idx=0, resident=None, ep=None):
    """Layer `layer_idx` of the workload: router, Zipf bias and experts drawn
    with the generator's layer index (resident: slots of an expert cache;
    ep: (rank, world) of an expert-parallel layer)."""
    E = wl.get("E", E_FULL)
    nq, ns = synth.expert_sizes(H, I)
    dev = torch.device("cuda", device)
    stream = torch.cuda.current_stream(dev).cuda_stream
    wr = torch.empty(E * H, dtype=torch.float32, device=dev)
    synth.router_dev(0, layer_idx, E, H, wr.data_ptr(), stream)
    q = torch.empty((E + S) * nq, dtype=torch.uint8, device=dev)
    s = torch.empty((E + S) * ns, dtype=torch.int16, device=dev)
    synth.expert_dev(0, layer_idx, 0, E + S, H, I, q.data_ptr(), s.data_ptr(), stream)
    bias = None
    if wl["zipf"]:
        bias = torch.from_numpy(synth.zipf_bias(0, layer_idx, E)[0]).to(dev)
    torch.cuda.synchronize(dev)
    cfg = coli.make_config(H, I, E, K, S, max_tokens)
    layer = coli.Layer(cfg, wr, bias, q[:E * nq], s[:E * ns], q[E * nq:], s[E * ns:], device=device,
                       resident=resident, ep=ep)
    del q, s, wr
    torch.cuda.empty_cache()
    return layer


E2E_METHOD = ("pipelined through the public API: pinned host x of step j copied to a device buffer on an upload "
              "stream, the forward on the compute stream, y copied back to pinned host memory on a download "
              "stream; two buffers per side, so step j+1's upload and step j-1's download overlap step j's "
              "forward; one event pair around all steps; L2 not flushed (each step reads its weights from HBM)")


def small_batch_limit(kernel):
    return {"i8": 64, "separate": 0}[kernel]


def path_dtype(kernel, T, bf16, tc):
    """Arithmetic of the path a batch of T tokens takes."""
    if T <= small_batch_limit(kernel):
        return "s8xu8->s32 + f32"
    if tc:
        return "f16->f32"
    return "f32"


def compute_desc(kernel, T, tc):
    if T <= small_batch_limit(kernel):
        return ("one persistent kernel; int4 codes x 8-bit token parts (15-bit block floating point per 64 "
                "inputs) on mma.sync s32, exact per group, f32 scales and accumulation; fp64 router")
    if tc:
        return ("int4 weights dequantised to f16 in tensor memory, tcgen05 f16 MMA, f32 accumulate; "
                "bf16 tokens scaled by powers of two to f16 (exact)")
    return "int4 weights dequantised to f32 on CUDA cores, fp64 router"


def e2e_pipelined(torch, dev, stream, xdev_steps, forward, shape, dtype, steps, dist, inplace=False):
    """Device ms for `steps` end-to-end steps: H2D of the step's input from
    pinned host memory, forward(x, y), D2H of y into pinned host memory
    (inplace: forward(x, None) updates x, which is downloaded)."""
    xh = xdev_steps[:steps].cpu().pin_memory()
    yh = [torch.empty(shape, dtype=dtype).pin_memory() for _ in range(2)]
    xin = [torch.empty(shape, dtype=dtype, device=dev) for _ in range(2)]
    yout = [torch.empty(shape, dtype=dtype, device=dev) for _ in range(2)]
    up, down = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev = lambda: torch.cuda.Event()
    h2d = [ev() for _ in range(steps)]
    fwd = [ev() for _ in range(steps)]
    d2h = [ev() for _ in range(steps)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if dist:
        dist.barrier()
    torch.cuda.synchronize(dev)
    t0.record(stream)
    up.wait_event(t0)
    for j in range(steps):
        b = j % 2
        if j >= 2:
            # xin[b] is free once forward j-2 has read it (and, in place, once it is downloaded)
            up.wait_event(d2h[j - 2] if inplace else fwd[j - 2])
        with torch.cuda.stream(up):
            xin[b].copy_(xh[j], non_blocking=True)
        h2d[j].record(up)
        stream.wait_event(h2d[j])
        if j >= 2:
            stream.wait_event(d2h[j - 2])  # yout[b] is free once its download is done
        forward(xin[b], None if inplace else yout[b])
        fwd[j].record(stream)
        down.wait_event(fwd[j])
        with torch.cuda.stream(down):
            yh[b].copy_(xin[b] if inplace else yout[b], non_blocking=True)
        d2h[j].record(down)
    stream.wait_event(d2h[steps - 1])
    t1.record(stream)
    torch.cuda.synchronize(dev)
    ms = t0.elapsed_time(t1)
    return max_over_ranks(ms, dist, dev)


def output_error(torch, coli, synth, wl, layer, x_step, y, stream, n_tok=2):
    """Error of one step's outputs against the fp64 oracle, on its first
    n_tok tokens (only the experts they select are generated): max relative
    error for fp32, relative L2 for bf16."""
    import numpy as np
    import oracle
    if layer is not None:  # (None: y already holds the step's output)
        layer.forward(x_step, y, stream=stream)
    torch.cuda.synchronize()
    T = x_step.shape[0]
    n = min(n_tok, T)
    E = wl.get("E", E_FULL)
    if wl["bf16"]:
        xh = x_step[:n].view(torch.int16).cpu().numpy().view(np.uint16)
        yg = (y[:n].view(torch.int16).cpu().numpy().view(np.uint16).astype(np.uint32) << 16).view(np.float32)
    else:
        xh = x_step[:n].cpu().numpy()
        yg = y[:n].cpu().numpy()
    bias = synth.zipf_bias(0, 0, E)[0] if wl["zipf"] else None
    wr = synth.router(0, 0, E, H)
    ids, _ = oracle.topk(oracle.router_logits(wr, bias, xh), K, top_p=topp_arg())
    experts = [None] * (E + S)
    for e in {e for e in ids.ravel().tolist() if e >= 0} | set(range(E, E + S)):
        experts[e] = synth.expert(0, 0, e, H, I)
    cfg = oracle.Cfg(hidden=H, inter=I, n_experts=E, top_k=K, n_shared=S, expert_top_p=topp_arg() or 0.0)
    y_ref, _, _ = oracle.moe_forward(cfg, wr, bias, experts, xh)
    yg = yg.astype(np.float64)
    if wl["bf16"]:
        val = float(np.linalg.norm(yg - y_ref) / np.linalg.norm(y_ref))
        kind = "relative L2 error (bf16 path)"
    else:
        val = float(np.abs(yg - y_ref).max() / np.abs(y_ref).max())
        kind = "max |y - y_oracle| / max |y_oracle| (fp32 path)"
    return {"value": val, "kind": kind, "sample": f"tokens 0..{n - 1} of the first timed step vs the fp64 oracle"}


def run_ours(args, wl, ws, rank, local):
    import torch
    import synth
    import int4_expert_ffn_router_b200 as coli

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dist = None
    if ws > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300), device_id=dev)

    T = wl["T"]
    # expert parallelism: every rank holds 1/ws of the experts and sees the same tokens;
    # replicas: every rank holds the whole layer and draws its own tokens
    ep = args.parallel == "ep" and ws > 1
    layer = build_layer(torch, coli, synth, wl, local, max_tokens=T, ep=(rank, ws) if ep else None)
    layer.set_fused(FUSED_MODE[args.decode_kernel])
    layer.set_expert_top_p(TOPP)
    nsteps = args.warmup + args.steps
    xdt = torch.bfloat16 if wl["bf16"] else torch.float32
    xs = torch.empty((nsteps, T, H), dtype=xdt, device=dev)
    stream = torch.cuda.current_stream(dev)
    fill_tokens(torch, synth, wl, xs, lambda i: step_seed(i, 0 if ep else rank), stream)
    y = torch.empty((T, H), dtype=xdt, device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)

    def fwd(x, yout):
        layer.forward(x, yout, stream=stream)
        if ep:
            ep_combine(yout, dist)  # the exchange step: all-reduce of the partial outputs (NCCL)

    # routing statistics of every step (untimed pre-pass): unique experts -> bytes
    uniq = []
    for i in range(nsteps):
        layer.forward(xs[i], y, stream=stream)
        uniq.append(layer.stats()[0])
    torch.cuda.synchronize(dev)
    uniq_local = list(uniq)
    if ep:  # distinct experts of the whole layer = the sum of the ranks' (disjoint) sets
        u = torch.tensor(uniq, dtype=torch.float64, device=dev)
        dist.all_reduce(u)
        uniq = u.cpu().tolist()

    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(nsteps)]
    # warm-up
    for i in range(args.warmup):
        fwd(xs[i], y)
        flush.zero_()
    torch.cuda.synchronize(dev)
    if dist:
        dist.barrier()
    torch.cuda.synchronize(dev)
    clocks = Clocks(local, coli, torch, stream)
    n0 = layer.launch_count()
    for i in range(args.warmup, nsteps):
        ev[i][0].record(stream)
        fwd(xs[i], y)
        ev[i][1].record(stream)
        flush.zero_()
    clocks.end_region()
    torch.cuda.synchronize(dev)
    clk = clocks.stop()
    launches = layer.launch_count() - n0
    if dist:
        dist.barrier()
    torch.cuda.synchronize(dev)
    step_ms = [ev[i][0].elapsed_time(ev[i][1]) for i in range(args.warmup, nsteps)]
    # per-stage device times from a separate pass (the stage events are not in the timed region)
    layer.set_profiling(True)
    for i in range(args.warmup, min(nsteps, args.warmup + 200)):
        fwd(xs[i], y)
        flush.zero_()
    torch.cuda.synchronize(dev)
    stages, nprof = layer.profile()
    layer.set_profiling(False)
    total_ms = sum(step_ms)
    total_ms = max_over_ranks(total_ms, dist, dev)

    # end to end through the C ABI with host buffers (pinned x in, y out)
    e2e_ms = e2e_pipelined(torch, dev, stream, xs[args.warmup:], fwd, (T, H), xdt, args.steps, dist)
    if ep:
        fwd(xs[args.warmup], y)  # every rank takes part in the exchange; rank 0 checks the sum
        torch.cuda.synchronize(dev)
    err = output_error(torch, coli, synth, wl, None if ep else layer, xs[args.warmup], y, stream) if rank == 0 else None

    if rank != 0:
        layer.close()
        if dist:
            dist.destroy_process_group()
        return None

    u = uniq[args.warmup:]
    mean_unique = sum(u) / len(u)
    router_bytes = wl.get("E", E_FULL) * H * 4
    bytes_step = [(n + S) * EXPERT_BYTES + router_bytes for n in u]
    gbs = sum(bytes_step) / (sum(step_ms) * 1e-3) / 1e9
    peaks = load_peaks()
    peak_gbs = peaks.get("hbm_gbs", 6650.0)
    tc = wl["bf16"] and T > small_batch_limit(args.decode_kernel)  # larger bf16 batches: tcgen05 grouped GEMMs
    # the roofline of this rank's kernel: its own distinct experts (expert parallelism) or all of them
    mean_local = sum(uniq_local[args.warmup:]) / len(uniq_local[args.warmup:])
    dom, roof = dominant_roofline(stages, nprof, T, mean_local, wl.get("E", E_FULL), xs.element_size(), tc, peaks)
    if roof is not None:
        roof["traffic"], roof["traffic_note"] = ncu_traffic(roof["kernel"], args.workload)
    out = {
        "metric": METRIC, "value": round(job_tokens_per_s(1 if ep else ws, args.steps, T, total_ms), 2), "unit": "tokens/s",
        "n_gpus": ws,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(total_ms / args.steps, 5),
        "step_ms_rank0": step_percentiles(step_ms),
        "higher_is_better": True, "scaling": "strong" if ep else "weak", "vs_baseline": None,
        "dtype": path_dtype(args.decode_kernel, T, wl["bf16"], tc),
        "stage_note": "stage_us from a separate profiled pass (stage events add host gaps)",
        "data": "synthetic (seeded generator; random-init int4 weights of the full-size layer shape)",
        "config": {"workload": args.workload, "desc": wl["desc"], "hidden": H, "inter": I, "experts": wl.get("E", E_FULL),
                   "top_k": K, "shared": S, "tokens_per_step": T, "weights": "int4 gs64 + fp16 scales",
                   "l2": "flushed between steps (256 MiB memset outside the step events)",
                   "parallelism": (f"expert parallel x{ws} (NCCL all-reduce of partial outputs)" if ep else
                                   f"replicas x{ws}" if ws > 1 else "single GPU"),
                   "expert_top_p": TOPP},
        "hbm_gbs": round(gbs, 1), "hbm_frac_of_8tbs": round(gbs / 8000.0, 4),
        "hbm_frac_of_measured": round(gbs / peak_gbs, 4),
        "unique_experts_per_step": round(mean_unique, 2),
        "bytes_per_step": int(sum(bytes_step) / len(bytes_step)),
        "stage_us": {k: round(v / max(nprof, 1) * 1e3, 2) for k, v in stages.items() if v > 0},
        "roofline": roof,
        "gpu_launches": launches,
        "gpu_launches_note": "forward kernels in the timed loop; two clock-stamp kernels bracket the loop",
        "max_rel_err": err,
        "verify": verify_report(wl, mean_unique + S, args.steps / (sum(step_ms) * 1e-3)) if wl.get("verify") else None,
        "compute": compute_desc(args.decode_kernel, T, tc),
        "e2e": {"value": round(job_tokens_per_s(1 if ep else ws, args.steps, T, e2e_ms), 2), "unit": "tokens/s",
                "h2d_bytes_per_step": T * H * xs.element_size(), "d2h_bytes_per_step": T * H * xs.element_size(),
                "method": E2E_METHOD},
        "clocks": clk,
    }
    if T >= 64:  # batches of 64 tokens and more: the certified integer-MMA router, if the layer uses it
        cert, n_fb = layer.router_fallbacks()
        out["router"] = {"certified": cert, "fallback_tokens_last_batch": n_fb, "tokens_per_batch": T,
                         "note": "tokens whose logits and top-K the certified router left to the fp64 fallback"}
    layer.close()
    if dist:
        dist.destroy_process_group()
    return out


def stack_output_error(torch, coli, synth, wl, layers, x_step, stream, n_layers=2):
    """Error of token 0 of a step through the first n_layers layers of the
    stack against the fp64 oracle (max relative error)."""
    import numpy as np
    import oracle
    E = wl.get("E", E_FULL)
    xw = x_step[:1].clone()
    coli.stack_forward(layers[:n_layers], xw, stream=stream)
    torch.cuda.synchronize()
    xr = x_step[:1].cpu().numpy().copy()
    cfg = oracle.Cfg(hidden=H, inter=I, n_experts=E, top_k=K, n_shared=S, expert_top_p=topp_arg() or 0.0)
    for l in range(n_layers):
        wr = synth.router(0, l, E, H)
        bias = synth.zipf_bias(0, l, E)[0]
        xn = oracle.rmsnorm(xr).astype(np.float32)
        ids, _ = oracle.topk(oracle.router_logits(wr, bias, xn), K, top_p=topp_arg())
        experts = [None] * (E + S)
        for e in {e for e in ids.ravel().tolist() if e >= 0} | set(range(E, E + S)):
            experts[e] = synth.expert(0, l, e, H, I)
        oracle.stack_step(cfg, wr, bias, experts, xr)
    yg = xw.cpu().numpy().astype(np.float64)
    ref = xr.astype(np.float64)
    val = float(np.abs(yg - ref).max() / np.abs(ref).max())
    return {"value": val, "kind": "max |x - x_oracle| / max |x_oracle| (fp32 residual stream)",
            "sample": f"token 0 of the first timed step through the first {n_layers} layers vs the fp64 oracle"}


def run_stack(args, wl, ws, rank, local):
    """The 30-layer stack workloads: x <- x + MoE_l(RMSNorm(x)) for l = 0..L-1
    (coli_moe_stack_forward), one step = one batch through all layers."""
    import torch
    import synth
    import int4_expert_ffn_router_b200 as coli

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dist = None
    if ws > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=600), device_id=dev)
    T, NL = wl["T"], wl["layers"]
    layers = [build_layer(torch, coli, synth, wl, local, max_tokens=T, layer_idx=l) for l in range(NL)]
    for L in layers:
        L.set_fused(FUSED_MODE[args.decode_kernel])
        L.set_expert_top_p(TOPP)
    nsteps = args.warmup + args.steps
    xs = torch.empty((nsteps, T, H), dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)
    for i in range(nsteps):
        synth.x_dev(step_seed(i, rank), 0, T, H, 0, xs[i].data_ptr(), stream.cuda_stream)
    xw = torch.empty((T, H), dtype=torch.float32, device=dev)

    # routing statistics from a few untimed steps: distinct experts per layer -> bytes
    per_step, uniq = [], []
    for i in range(min(4, nsteps)):
        xw.copy_(xs[i])
        coli.stack_forward(layers, xw, stream=stream)
        u = [L.stats()[0] for L in layers]
        uniq.append(sum(u) / NL)
        per_step.append(sum((n + S) * EXPERT_BYTES + E_FULL * H * 4 for n in u))
    mean_unique = sum(uniq) / len(uniq)
    bytes_step = sum(per_step) / len(per_step)
    torch.cuda.synchronize(dev)

    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(nsteps)]
    for i in range(args.warmup):
        xw.copy_(xs[i])
        coli.stack_forward(layers, xw, stream=stream)
    torch.cuda.synchronize(dev)
    if dist:
        dist.barrier()
    torch.cuda.synchronize(dev)
    clocks = Clocks(local, coli, torch, stream)
    n0 = sum(L.launch_count() for L in layers)
    for i in range(args.warmup, nsteps):
        xw.copy_(xs[i])
        ev[i][0].record(stream)
        coli.stack_forward(layers, xw, stream=stream)
        ev[i][1].record(stream)
    clocks.end_region()
    torch.cuda.synchronize(dev)
    clk = clocks.stop()
    launches = sum(L.launch_count() for L in layers) - n0
    if dist:
        dist.barrier()
    torch.cuda.synchronize(dev)
    step_ms = [ev[i][0].elapsed_time(ev[i][1]) for i in range(args.warmup, nsteps)]
    total_ms = sum(step_ms)
    # per-stage device times from a separate pass (not in the timed region)
    for L in layers:
        L.set_profiling(True)
    for i in range(args.warmup, min(nsteps, args.warmup + 20)):
        xw.copy_(xs[i])
        coli.stack_forward(layers, xw, stream=stream)
    torch.cuda.synchronize(dev)
    stages = {}
    nprof = 0
    for L in layers:
        st, n = L.profile()
        nprof = n
        for k, v in st.items():
            stages[k] = stages.get(k, 0.0) + v
        L.set_profiling(False)
    total_ms = max_over_ranks(total_ms, dist, dev)

    # end to end through the C ABI with host buffers (pinned x in, result out)
    e2e_ms = e2e_pipelined(torch, dev, stream, xs[args.warmup:],
                           lambda xin, _: coli.stack_forward(layers, xin, stream=stream), (T, H), torch.float32,
                           args.steps, dist, inplace=True)
    err = stack_output_error(torch, coli, synth, wl, layers, xs[args.warmup], stream) if rank == 0 else None
    for L in layers:
        L.close()
    if rank != 0:
        if dist:
            dist.destroy_process_group()
        return None

    gbs = bytes_step / (total_ms / args.steps * 1e-3) / 1e9
    peaks = load_peaks()
    peak_gbs = peaks.get("hbm_gbs", 6650.0)
    # stage totals are summed over the layers: nprof forwards of each of NL layers
    dom, roof = dominant_roofline(stages, nprof * NL, T, mean_unique, E_FULL, 4, False, peaks)
    out = {
        "metric": METRIC, "value": round(job_tokens_per_s(ws, args.steps, T, total_ms), 2), "unit": "tokens/s", "n_gpus": ws,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(total_ms / args.steps, 5),
        "step_ms_rank0": step_percentiles(step_ms),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": path_dtype(args.decode_kernel, T, False, False),
        "data": "synthetic (seeded generator; random-init int4 weights of the full-size layer shape, per layer)",
        "config": {"workload": args.workload, "desc": wl["desc"], "layers": NL, "hidden": H, "inter": I,
                   "experts": E_FULL, "top_k": K, "shared": S, "tokens_per_step": T,
                   "weights": "int4 gs64 + fp16 scales, 154.8 GB resident",
                   "l2": f"not flushed: each step streams {bytes_step / 1e9:.2f} GB of weights (L2 is 126 MB)",
                   "parallelism": f"replicas x{ws}" if ws > 1 else "single GPU",
                   "expert_top_p": TOPP},
        "hbm_gbs": round(gbs, 1), "hbm_frac_of_8tbs": round(gbs / 8000.0, 4),
        "hbm_frac_of_measured": round(gbs / peak_gbs, 4),
        "bytes_per_step": int(bytes_step), "unique_experts_per_layer": round(mean_unique, 2),
        "stage_us": {k: round(v / max(nprof, 1) * 1e3, 2) for k, v in stages.items() if v > 0},
        "roofline": roof,
        "gpu_launches": launches,
        "gpu_launches_note": "forward kernels in the timed loop; two clock-stamp kernels bracket the loop",
        "max_rel_err": err,
        "e2e": {"value": round(job_tokens_per_s(ws, args.steps, T, e2e_ms), 2), "unit": "tokens/s",
                "h2d_bytes_per_step": T * H * 4, "d2h_bytes_per_step": T * H * 4, "method": E2E_METHOD},
        "clocks": clk,
    }
    if dist:
        dist.destroy_process_group()
    return out


def host_link_gbs(torch, dev, nbytes=1 << 30, reps=3):
    """Best of `reps` plain copies of `nbytes` from page-locked host memory to
    HBM (CUDA events): the host link's measured rate for the cache workloads."""
    src = torch.empty(nbytes, dtype=torch.uint8, pin_memory=True)
    dst = torch.empty(nbytes, dtype=torch.uint8, device=dev)
    best = 0.0
    for _ in range(reps):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        dst.copy_(src, non_blocking=True)
        b.record()
        b.synchronize()
        best = max(best, nbytes / (a.elapsed_time(b) * 1e-3) / 1e9)
    del src, dst
    torch.cuda.empty_cache()
    return best


def run_cached(args, wl, ws, rank, local):
    """Expert-cache workloads: layers with `resident` of their 256 routed
    experts in HBM over a page-locked host copy of all of them. An untimed
    learning pass (its own tokens) counts routing per expert; the `pin` most
    used are pinned; the counters are then reset, and the timed steps measure
    hits, misses and host-to-HBM bytes. One layer: coli_moe_forward; several:
    coli_moe_stack_forward, whose next-layer lookahead prefetches."""
    import numpy as np
    import torch
    import synth
    import int4_expert_ffn_router_b200 as coli

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dist = None
    if ws > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=600), device_id=dev)
    T, NL, R = wl["T"], wl.get("layers", 1), wl["resident"]
    stack = NL > 1
    link = host_link_gbs(torch, dev)
    layers = [build_layer(torch, coli, synth, wl, local, max_tokens=T, layer_idx=l, resident=R) for l in range(NL)]
    for L in layers:
        L.set_fused(FUSED_MODE[args.decode_kernel])
        L.set_expert_top_p(TOPP)
    nsteps = args.warmup + args.steps
    stream = torch.cuda.current_stream(dev)
    xs = torch.empty((nsteps, T, H), dtype=torch.float32, device=dev)
    fill_tokens(torch, synth, wl, xs, lambda i: step_seed(i, rank), stream)
    xw = torch.empty((T, H), dtype=torch.float32, device=dev)
    y = torch.empty((T, H), dtype=torch.float32, device=dev)

    def step(x):
        if stack:
            xw.copy_(x)
            coli.stack_forward(layers, xw, stream=stream)
        else:
            layers[0].forward(x, y, stream=stream)

    # learning pass: routing counts per expert, then the hot set is pinned
    n_learn, n_cold = 400, 100
    xl = torch.empty((n_learn, T, H), dtype=torch.float32, device=dev)
    fill_tokens(torch, synth, wl, xl, lambda i: LEARN_SEED0 + i + 10_000 * rank, stream)
    for i in range(n_learn):
        step(xl[i])
        if i == n_cold - 1:  # the first forwards from the initial placement: a cold cache
            torch.cuda.synchronize(dev)
            cold = [L.cache_stats() for L in layers]
    torch.cuda.synchronize(dev)
    for L in layers:
        L.pin_hot(wl["pin"])
    for i in range(args.warmup):
        step(xs[i])
    torch.cuda.synchronize(dev)
    for L in layers:
        L.cache_stats(reset=True)
    if dist:
        dist.barrier()
    torch.cuda.synchronize(dev)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(nsteps)]
    clocks = Clocks(local, coli, torch, stream)
    n0 = sum(L.launch_count() for L in layers)
    for i in range(args.warmup, nsteps):
        ev[i][0].record(stream)
        step(xs[i])
        ev[i][1].record(stream)
    clocks.end_region()
    torch.cuda.synchronize(dev)
    clk = clocks.stop()
    launches = sum(L.launch_count() for L in layers) - n0
    st = [L.cache_stats(reset=True) for L in layers]
    if dist:
        dist.barrier()
    torch.cuda.synchronize(dev)
    step_ms = [ev[i][0].elapsed_time(ev[i][1]) for i in range(args.warmup, nsteps)]
    total_ms = max_over_ranks(sum(step_ms), dist, dev)
    # per-stage device times from a separate pass (not in the timed region)
    for L in layers:
        L.set_profiling(True)
    for i in range(args.warmup, min(nsteps, args.warmup + 100)):
        step(xs[i])
    torch.cuda.synchronize(dev)
    stages, nprof = {}, 0
    for L in layers:
        sp, nprof = L.profile()
        for k, v in sp.items():
            stages[k] = stages.get(k, 0.0) + v
        L.set_profiling(False)
    for L in layers:
        L.cache_stats(reset=True)
    # end to end through the C ABI with host buffers
    if stack:
        e2e_ms = e2e_pipelined(torch, dev, stream, xs[args.warmup:],
                               lambda xin, _: coli.stack_forward(layers, xin, stream=stream), (T, H), torch.float32,
                               args.steps, dist, inplace=True)
    else:
        e2e_ms = e2e_pipelined(torch, dev, stream, xs[args.warmup:],
                               lambda xin, yout: layers[0].forward(xin, yout, stream=stream), (T, H), torch.float32,
                               args.steps, dist)
    if stack:
        err = stack_output_error(torch, coli, synth, wl, layers, xs[args.warmup], stream) if rank == 0 else None
    else:
        err = output_error(torch, coli, synth, wl, layers[0], xs[args.warmup], y, stream) if rank == 0 else None
    for L in layers:
        L.close()
    if rank != 0:
        if dist:
            dist.destroy_process_group()
        return None

    cold_hits = sum(x["hits"] for x in cold)
    cold_misses = sum(x["misses"] for x in cold)
    hits = sum(x["hits"] for x in st)
    misses = sum(x["misses"] for x in st)
    h2d = sum(x["bytes_h2d"] for x in st)
    secs = sum(step_ms) * 1e-3
    pred = sum(x["predicted"] for x in st)
    pred_of = sum(x["predicted_of"] for x in st)
    pref = sum(x["prefetched"] for x in st)
    pref_used = sum(x["prefetch_used"] for x in st)
    needed_per_step = (hits + misses) / args.steps
    hbm_bytes = needed_per_step * EXPERT_BYTES + NL * (S * EXPERT_BYTES + E_FULL * H * 4)
    peaks = load_peaks()
    kernel_stages = {k: v for k, v in stages.items() if k != "cache"}
    dom, roof = dominant_roofline(kernel_stages, nprof * NL, T, needed_per_step / NL, E_FULL, 4, False, peaks)
    cache_ms = stages.get("cache", 0.0) / max(nprof, 1)
    out = {
        "metric": METRIC, "value": round(job_tokens_per_s(ws, args.steps, T, total_ms), 2), "unit": "tokens/s",
        "n_gpus": ws, "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(total_ms / args.steps, 5),
        "step_ms_rank0": step_percentiles(step_ms),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": path_dtype(args.decode_kernel, T, False, False),
        "data": "synthetic (seeded generator; random-init int4 weights of the full-size layer shape)",
        "config": {"workload": args.workload, "desc": wl["desc"], "layers": NL, "hidden": H, "inter": I,
                   "experts": E_FULL, "top_k": K, "shared": S, "tokens_per_step": T, "resident_slots": R,
                   "pinned": wl["pin"], "learning_steps": n_learn,
                   "l2": "not flushed: every step copies experts from host memory or streams them from HBM",
                   "parallelism": f"replicas x{ws}" if ws > 1 else "single GPU",
                   "expert_top_p": TOPP},
        "cache": {
            "cold_hit_rate": round(cold_hits / max(cold_hits + cold_misses, 1), 4),
            "cold_misses_per_step": round(cold_misses / n_cold, 3),
            "cold_note": f"the first {n_cold} forwards of the learning pass, from experts 0..R-1 resident, no pins",
            "hit_rate": round(hits / max(hits + misses, 1), 4),
            "misses_per_step": round(misses / args.steps, 3),
            "needed_per_step": round(needed_per_step, 3),
            "h2d_bytes_per_step": int(h2d / args.steps),
            "h2d_gbs": round(h2d / secs / 1e9, 2),
            "host_link_gbs_measured": round(link, 2),
            "host_link_frac": round(h2d / secs / 1e9 / link, 4),
            "host_pool_bytes_per_layer": E_FULL * EXPERT_BYTES,
            "hbm_expert_bytes_per_layer": (R + S) * EXPERT_BYTES,
            "cache_stage_us": round(cache_ms * 1e3 / NL, 2),
            "lookahead_accuracy": round(pred / pred_of, 4) if pred_of else None,
            "prefetched_per_step": round(pref / args.steps, 3),
            "prefetch_used_frac": round(pref_used / pref, 4) if pref else None,
            "note": ("hit = a needed expert already in HBM; h2d = page-locked host to HBM copies (misses and "
                     "prefetches); lookahead accuracy = needed experts of layers 1.. that the previous layer's "
                     "lookahead routing named"),
        },
        "hbm_bytes_per_step": int(hbm_bytes),
        "verify": verify_report(wl, needed_per_step + NL * S, args.steps / secs) if wl.get("verify") else None,
        "stage_us": {k: round(v / max(nprof, 1) * 1e3, 2) for k, v in stages.items() if v > 0},
        "roofline": roof,
        "gpu_launches": launches,
        "gpu_launches_note": "forward kernels in the timed loop; two clock-stamp kernels bracket the loop",
        "max_rel_err": err,
        "e2e": {"value": round(job_tokens_per_s(ws, args.steps, T, e2e_ms), 2), "unit": "tokens/s",
                "h2d_bytes_per_step": T * H * 4, "d2h_bytes_per_step": T * H * 4, "method": E2E_METHOD},
        "clocks": clk,
    }
    if dist:
        dist.destroy_process_group()
    return out


def main():
    global TOPP
    args = parse()
    if not 0.0 < args.expert_top_p <= 1.0:
        raise SystemExit("--expert-top-p must be in (0, 1]")
    TOPP = args.expert_top_p
    wl = WORKLOADS[args.workload]
    ws, rank, local = dist_env()
    if args.impl == "reference":
        if rank != 0:
            return 0
        leg = OracleLeg(wl)
        for i in range(args.warmup):
            leg.step(i)
        tok, total = 0, 0.0
        for i in range(args.warmup, args.warmup + args.steps):
            n, dt = leg.step(i)
            tok += n
            total += dt
        val = tok / total
        cb = {"value": round(val, 4), "unit": "tokens/s", "cores": leg.cores(), "kind": "oracle",
              "sample": (f"{args.steps} steps, each the fp64 oracle on 1 token through the first {leg.Ls} of "
                         f"{leg.layers} layers, time scaled to {leg.layers} layers" if leg.layers else
                         f"{args.steps} steps, each the fp64 oracle on {leg.Ts} token(s) of the step's batch") +
                        " (input and expert generation untimed)"}
        print(json.dumps({"impl": "reference", "metric": METRIC, "value": round(val, 4), "unit": "tokens/s",
                          "n_gpus": ws, "steps": args.steps, "warmup": args.warmup,
                          "ms_per_step": round(total / args.steps * 1e3, 3), "higher_is_better": True,
                          "scaling": "weak", "vs_baseline": None, "dtype": "f64",
                          "data": "synthetic", "config": {"workload": args.workload, "desc": wl["desc"],
                                                                "expert_top_p": TOPP},
                          "cpu_baseline": cb,
                          "e2e": {"value": round(val, 4), "unit": "tokens/s", "h2d_bytes_per_step": 0,
                                  "d2h_bytes_per_step": 0}}))
        return 0

    # the CPU oracle sample runs first (before any CUDA call in this process)
    cpu = None
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        cpu = oracle_sample(wl, args.cpu_seconds)
    if wl.get("resident"):
        out = run_cached(args, wl, ws, rank, local)
    elif wl.get("layers"):
        out = run_stack(args, wl, ws, rank, local)
    else:
        out = run_ours(args, wl, ws, rank, local)
    if out is not None:
        out["cpu_baseline"] = cpu
        print(json.dumps(out))
    return 0


if __name__ == "__main__":
    sys.exit(main())
