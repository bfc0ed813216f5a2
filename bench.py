#!/usr/bin/env python
"""Benchmark of the MoE layer's forward + backward on B200s.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl reference]

One step = moe_layer_fwd + moe_layer_bwd over one batch of the workload (default: the largest
layer, the Mixtral-style dropless top-2 layer, T=16384, d=4096, E=8, SwiGLU F=14336, softmax over
the two chosen logits, bf16), inputs resident in HBM.  K steps are timed with CUDA events on the launching stream, one pair per step,
with an L2 flush between steps (outside the timed pairs: a 256 MiB write, then a 256 MiB read of a
second buffer, which evicts the written lines so that their write-back to HBM is not charged to
the first kernel of the next step); the run is bracketed by
a barrier and a device synchronise, and the max over ranks is taken.  value = tokens processed
by all ranks / that time.  Several GPUs run independent replicas (the layer has no exchange step
on one device), so scaling is weak.

Also reported: e2e (the same steps through the C ABI with every step's inputs copied from pinned
host memory and its outputs read back inside the timed region, the copies on two streams
overlapped with the compute), per-phase device times from the library's profiling events (a
separate pass before the timed one: events between phases would break the overlap of
consecutive launches), the roofline of the dominant kernel (timed live in a third pass with
events around that phase only), SM clocks sampled during the timed region, the number of library
kernel launches in the timed region, and the CPU oracle timed on a bounded sample (rank 0, one
GPU).

--impl reference times the CPU oracle itself on this host's cores as the reference arm.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "MoE-layer tokens/s fwd+bwd on 1 B200; % bf16 TC peak (GEMM), % HBM BW (rest)"
FLUSH_BYTES = 256 << 20


class L2Flush:
    """Between timed steps: write FLUSH_BYTES (twice the 126 MB L2), then read as many bytes of a
    second buffer, so that L2 ends up holding clean lines of neither the step's inputs nor its
    outputs (a write alone leaves L2 full of dirty lines, written back during the next step)."""

    def __init__(self, dev):
        import torch
        self._amax = torch.amax
        self.w = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
        self.r = torch.zeros(FLUSH_BYTES // 4, dtype=torch.int32, device=dev)

    def __call__(self):
        self.w.zero_()
        self._amax(self.r)
GEMM_PHASES = {"expert_up", "expert_down", "dgrad_h", "dgrad_x", "wgrad_w1", "wgrad_w2"}


# DRAM traffic of a phase from one ncu capture (dram__bytes_read.sum + dram__bytes_write.sum of the
# phase's launches in one step, averaged over the run's steps), keyed by workload and phase.  It
# stands only for the kernel sources it was taken on: the SHA-256 of those files is stored with it
# and the bench reports null once they have changed.  The large layers' figures come from the
# one-pass launch lists (gpu__time_duration.sum and the two DRAM byte counters) of
# `python bench.py [--workload W] --steps 1 --warmup 1 --no-cpu-baseline`; "profile" names the
# summary of the capture under profiles/.
GEMM_SOURCES = ["gemm_tc.cu", "tc_ptx.cuh", "act_fast.cuh", "common.cuh"]
WGRAD_SOURCES = GEMM_SOURCES + ["transpose.cu"]
NCU_TRAFFIC = {
    # weight-gradient phase: transpose64_kernel + the dW1 and dW3 launches
    ("mixtral_dropless", "wgrad_w1"): {
        "bytes": 15686405478,
        "sources": WGRAD_SOURCES,
        "sha256": "bdf5917b14f1a7688c880b17a52e5d21bea257f7a01a57c65a5477a036629f53",
        "profile": "profiles/launches_mixtral_dropless.md",
    },
    ("mixtral_dropless", "expert_up"): {
        "bytes": 11330623053,
        "sources": GEMM_SOURCES,
        "sha256": "9935fc610e25e1760dc0152fe0942080d209f33a55c7ce35a6db03ea2ef1e2e3",
        "profile": "profiles/launches_mixtral_dropless.md",
    },
    ("deepseek_v2", "wgrad_w1"): {   # the dW1 and dW3 launches (no transposes on this layer)
        "bytes": 2882665472,
        "sources": WGRAD_SOURCES,
        "sha256": "bdf5917b14f1a7688c880b17a52e5d21bea257f7a01a57c65a5477a036629f53",
        "profile": "profiles/launches_deepseek_v2.md",
    },
    ("deepseek_v2", "expert_up"): {
        "bytes": 2031581773,
        "sources": GEMM_SOURCES,
        "sha256": "9935fc610e25e1760dc0152fe0942080d209f33a55c7ce35a6db03ea2ef1e2e3",
        "profile": "profiles/launches_deepseek_v2.md",
    },
    ("gpt2_gshard", "expert_up"): {
        "bytes": 146722355,
        "sources": GEMM_SOURCES,
        "sha256": "9935fc610e25e1760dc0152fe0942080d209f33a55c7ce35a6db03ea2ef1e2e3",
        "profile": "profiles/launches_gpt2_gshard.md",
    },
}


def sources_sha256(files):
    h = hashlib.sha256()
    for f in files:
        with open(os.path.join(ROOT, "mixture_experts_layer_23_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()


def measured_traffic(workload, phase):
    e = NCU_TRAFFIC.get((workload, phase))
    if e is None or sources_sha256(e["sources"]) != e["sha256"]:
        return None, None
    return e["bytes"], e["profile"]


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="mixtral_dropless")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--aux-loss-coef", type=float, default=0.0,
                    help="also compute the load-balancing loss (and its gradient) with this weight")
    ap.add_argument("--choice-major", action="store_true",
                    help="drop priority: all first choices, then second choices, ... (else token order)")
    ap.add_argument("--cpu-seconds", type=float, default=12.0,
                    help="target CPU time of the oracle baseline sample")
    ap.add_argument("--ep", action="store_true",
                    help="expert parallelism instead of replicas: each of the N ranks owns E/N "
                         "experts and its own batch (layers without shared experts)")
    ap.add_argument("--ep-chunks", type=int, default=1,
                    help="expert groups per rank whose exchange overlaps the previous group's GEMMs")
    return ap.parse_args()


def rank_barrier(world):
    """Barrier over the replicas (no-op on one rank)."""
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def reduce_max(v: float, world: int, device) -> float:
    """The maximum of v over all ranks (each rank's own device time: the job is as slow as its
    slowest replica)."""
    if world == 1:
        return v
    import torch
    import torch.distributed as dist
    t = torch.tensor([v], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_tokens_per_s(world: int, T: int, steps: int, total_ms: float) -> float:
    """Whole-job throughput: every replica processes T tokens per step; total_ms is the
    max-over-ranks time of the steps."""
    return world * T * steps / (total_ms * 1e-3)


def dist_env():
    return (int(os.environ.get("RANK", 0)), int(os.environ.get("LOCAL_RANK", 0)),
            int(os.environ.get("WORLD_SIZE", 1)))


def peaks():
    """(HBM GB/s, bf16 TFLOP/s burst, bf16 TFLOP/s sustained, source).  The measured copy
    bandwidth and cuBLAS bf16 rates of this machine's B200s when the file is there, else an
    earlier measurement of the same parts (sustained: under the 1 kW power cap)."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            j = json.load(f)
        return (j["hbm_gbs"], j["bf16_tflops"], j.get("bf16_tflops_sustained", j["bf16_tflops"]),
                "measured")
    return 6650.0, 1590.0, 1400.0, "fallback"


# A kernel timed inside back-to-back steps that last longer than this (or during which the power
# cap held the clock down) runs at the power cap's sustained clock, so its tensor-core fraction is
# taken against the sustained peak.
SUSTAINED_AFTER_S = 1.0


def workload_config(shape, world: int) -> dict:
    """The `config` object of the JSON line: the workload only (both arms print the same one)."""
    from mixture_experts_layer_23_b200.configs import WORKLOAD_TEXT
    return {"workload": WORKLOAD_TEXT[shape.name], "name": shape.name, "T": shape.T,
            "d": shape.d, "E": shape.E, "k": shape.k, "d_ff": shape.d_ff,
            "n_shared": shape.n_shared, "act": ["gelu", "swiglu"][shape.act],
            "gate_norm": ["softmax_all", "softmax_topk"][shape.gate_norm],
            "capacity_factor": shape.capacity_factor, "bias": shape.bias,
            "aux_loss_coef": shape.aux_loss_coef,
            "drop_order": "choice-major" if shape.choice_major else "token",
            "l2": "GPU arm: 256 MiB write + 256 MiB read of another buffer between timed "
                  "steps, outside the timed events",
            "parallelism": f"replicas x{world}"}


def bench_shape(args):
    from dataclasses import replace
    from mixture_experts_layer_23_b200.configs import BY_NAME
    shape = BY_NAME[args.workload]
    if args.aux_loss_coef or args.choice_major:
        shape = replace(shape, aux_loss_coef=args.aux_loss_coef, choice_major=args.choice_major)
    return shape


# ----------------------------------------------------------------------------- CPU oracle leg

def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return os.cpu_count() or 1


def oracle_step(shape, inp, n_tok):
    """One oracle forward + backward on the first n_tok tokens of the workload (capacity
    recomputed for n_tok tokens).  Returns seconds."""
    from mixture_experts_layer_23_b200.synth import to_f64
    from oracle import moe_oracle as mo
    dt = shape.dtype
    x = to_f64(inp["x"][:n_tok], dt)
    dy = to_f64(inp["dy"][:n_tok], dt) if inp["dy"] is not None else None
    Wg = to_f64(inp["Wg"], dt)
    W1, W2 = inp["_W1_64"], inp["_W2_64"]
    W3 = inp.get("_W3_64")
    t0 = time.perf_counter()
    f = mo.layer_forward(x, Wg, inp["bias"], W1, W3, W2, k=shape.k, act=shape.act,
                         gate_norm=shape.gate_norm, capacity_factor=shape.capacity_factor,
                         n_shared=shape.n_shared, aux_loss_coef=shape.aux_loss_coef,
                         choice_major=shape.choice_major)
    if dy is not None:
        mo.layer_backward(f, x, Wg, W1, W3, W2, dy)
    return time.perf_counter() - t0


def prepare_oracle_weights(shape, inp):
    from mixture_experts_layer_23_b200.synth import to_f64
    inp["_W1_64"] = to_f64(inp["W1"], shape.dtype)
    inp["_W2_64"] = to_f64(inp["W2"], shape.dtype)
    if inp["W3"] is not None:
        inp["_W3_64"] = to_f64(inp["W3"], shape.dtype)


def calibrate_sample(shape, inp, target_s):
    """Token count whose oracle step takes about target_s seconds (>= 64, <= T).  One probe step
    on 64 tokens; a layer whose weight gradients alone take longer than target_s (the Mixtral-style
    layer: 2.8 G weights) stays at 64 tokens."""
    n = min(shape.T, 64)
    t = oracle_step(shape, inp, n)
    want = int(n * target_s / max(t, 1e-3))
    return max(n, min(shape.T, want)), t


def cpu_baseline(shape, inp, target_s):
    prepare_oracle_weights(shape, inp)
    n, _ = calibrate_sample(shape, inp, target_s)
    # a layer whose step cost is mostly the weight gradients (fixed in n) reaches the target with
    # repeated steps on the sample rather than a larger one (at most four)
    t, reps = oracle_step(shape, inp, n), 1
    while t < 0.8 * target_s and reps < 4:
        t += oracle_step(shape, inp, n)
        reps += 1
    steps = f"{reps} float64 forward+backward steps" if reps > 1 else "one float64 forward+backward"
    return {"value": n * reps / t, "unit": "tokens/s", "cores": blas_threads(), "kind": "oracle",
            "sample": f"first {n} of {shape.T} tokens, {steps} of the same layer (capacity "
                      f"recomputed for {n} tokens), {t:.1f} s"}


def run_reference(args):
    rank, _, world = dist_env()
    if rank != 0:
        return 0
    from mixture_experts_layer_23_b200.synth import make_inputs
    shape = bench_shape(args)
    inp = make_inputs(shape, 0)
    prepare_oracle_weights(shape, inp)
    budget = 150.0 / max(1, args.steps + args.warmup)
    n, _ = calibrate_sample(shape, inp, min(2.0, budget))
    for _ in range(args.warmup):
        oracle_step(shape, inp, n)
    times = [oracle_step(shape, inp, n) for _ in range(args.steps)]
    total = sum(times)
    value = n * args.steps / total
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * total / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(shape, world),
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": blas_threads(),
                         "kind": "oracle",
                         "sample": f"first {n} of {shape.T} tokens per step, float64 oracle "
                                   "forward+backward (capacity recomputed for the sample)"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------------------------- GPU leg

class ClockSampler:
    """Samples the SM clock and the active clock-event reasons through NVML on a thread while
    the timed region runs (every ~2 ms; reads only, changes no setting)."""

    REASONS = (("hw_slowdown", "nvmlClocksEventReasonHwSlowdown"),
               ("hw_thermal_slowdown", "nvmlClocksEventReasonHwThermalSlowdown"),
               ("sw_thermal_slowdown", "nvmlClocksEventReasonSwThermalSlowdown"),
               ("hw_power_brake", "nvmlClocksEventReasonHwPowerBrakeSlowdown"),
               ("sw_power_cap", "nvmlClocksEventReasonSwPowerCap"))

    def __init__(self, gpu_uuid: str):
        import threading
        self.sm, self.reasons, self.max_mhz, self.err = [], set(), None, None
        self._stop = threading.Event()
        try:
            import pynvml as nv
            nv.nvmlInit()
            self.nv = nv
            self.h = nv.nvmlDeviceGetHandleByUUID(gpu_uuid)
            self.max_mhz = nv.nvmlDeviceGetMaxClockInfo(self.h, nv.NVML_CLOCK_SM)
        except Exception as e:  # NVML missing: report it, never guess
            self.err = f"nvml unavailable: {e}"
            self.t = None
            return
        self.t = threading.Thread(target=self._run, daemon=True)
        self.t.start()

    def _run(self):
        nv = self.nv
        get_r = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons",
                        getattr(nv, "nvmlDeviceGetCurrentClocksThrottleReasons", None))
        while not self._stop.is_set():
            try:
                self.sm.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
                r = get_r(self.h)
                for name, const in self.REASONS:
                    if r & getattr(nv, const, 0):
                        self.reasons.add(name)
            except Exception as e:
                self.err = str(e)
                break
            time.sleep(0.002)

    def stop(self):
        if self.t is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "samples": 0, "reasons": [self.err]}
        self._stop.set()
        self.t.join(timeout=5)
        return {"sm_mhz": statistics.median(self.sm) if self.sm else None,
                "sm_max_mhz": self.max_mhz, "samples": len(self.sm),
                "reasons": sorted(self.reasons)}


# fp32 layers run their GEMMs on the CUDA cores: peak = 148 SMs x 128 FP32 lanes x 2 FLOP (FMA)
# x 1965 MHz (the B200's maximum SM clock)
FP32_FMA_TFLOPS = 148 * 128 * 2 * 1965e6 / 1e12


def phase_work(shape, n_kept):
    """Algorithmic work per phase: FLOPs for the GEMMs (kept rows only), bytes for the rest.  The
    GEMMs of bf16 layers are tensor-core bound, those of fp32 layers ALU (FMA) bound."""
    b = 2 if shape.dtype == 1 else 4
    mm = "tensor" if shape.dtype == 1 else "alu"
    T, d, F, S, E, k = shape.T, shape.d, shape.d_ff, shape.n_shared, shape.E, shape.k
    rows = n_kept + S * T
    g = 2 if shape.act == 1 else 1
    Td, Nd = T * d * b, n_kept * d * b
    # dlogits travel as fp32 on the CUDA-core path and as a bf16 copy (rows padded to 8) on the
    # tensor-core path
    dl = T * ((E + 7) // 8 * 8) * 2 if shape.dtype == 1 and d % 64 == 0 else T * E * 4
    return {
        "router": ("hbm", Td + E * d * b + T * E * 4 + T * k * 8),
        "dispatch": ("hbm", Td + Nd + T * k * 8 + (T * E * 4 if shape.aux_loss_coef else 0)),
        "expert_up": (mm, 2.0 * rows * d * F * g),
        "expert_down": (mm, 2.0 * rows * F * d),
        "combine": ("hbm", Nd + S * Td + Td + T * k * 8),
        # read dy, the kept O rows and the logits; write dO rows, dg and the logit gradient
        "combine_bwd": ("hbm", Td + 2 * Nd + T * E * 4 + T * k * 12 + dl),
        # read x and the logit gradient, write dWg
        "router_bwd": ("hbm", Td + dl + E * d * 4),
        "dgrad_h": (mm, 2.0 * rows * d * F),
        "dgrad_x": (mm, 2.0 * rows * F * d * g),
        "wgrad_w1": (mm, 2.0 * rows * F * d * g),
        "wgrad_w2": (mm, 2.0 * rows * d * F),
        # read the kept and shared dXd rows, the logit gradient and Wg; write dx
        "undispatch": ("hbm", Nd + S * Td + Td + dl + E * d * b + T * k * 4),
    }


def gemm_min_bytes(shape, n_kept):
    """HBM bytes each GEMM phase cannot do without: every operand read once and every output
    written once (kept and shared rows only, no padding).  With the FLOPs of phase_work this gives
    each GEMM's own roofline, max(FLOPs / tensor peak, bytes / HBM bandwidth): the small layers'
    weight gradients, for one, are bound by writing their fp32 output."""
    b = 2 if shape.dtype == 1 else 4
    T, d, F, S, Et = shape.T, shape.d, shape.d_ff, shape.n_shared, shape.E_tot
    rows = n_kept + S * T
    g = 2 if shape.act == 1 else 1
    Xr, Fr, W = rows * d * b, rows * F * b, Et * F * d * b
    return {
        "expert_up": Xr + g * W + (g + 1) * Fr,          # Xd, W1 (W3) -> Gu (Gv), H
        "expert_down": Fr + W + Xr,                      # H, W2 -> O
        "dgrad_h": Xr + W + 2 * g * Fr,                  # dO, W2, Gu (Gv) -> dU (dV)
        "dgrad_x": g * Fr + g * W + Xr,                  # dU (dV), W1 (W3) -> dXd
        "wgrad_w1": g * (Fr + Xr + Et * F * d * 4),      # dU (dV), Xd -> fp32 dW1 (dW3)
        "wgrad_w2": Xr + Fr + Et * F * d * 4,            # dO, H -> fp32 dW2
    }


def run_ours(args):
    import numpy as np
    import torch
    import torch.distributed as dist

    rank, local_rank, world = dist_env()
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=dev)

    from mixture_experts_layer_23_b200 import build as moe_build
    moe_build.build()
    from mixture_experts_layer_23_b200 import moe
    from mixture_experts_layer_23_b200.layer import MoELayer, to_device
    from mixture_experts_layer_23_b200.synth import make_inputs

    shape = bench_shape(args)
    inp = make_inputs(shape, 0)
    w = {n: to_device(inp[n], shape, dev) for n in ("Wg", "W1", "W3", "W2")}
    bias = None if inp["bias"] is None else torch.from_numpy(inp["bias"]).to(dev)
    x = to_device(inp["x"], shape, dev)
    dy = None if shape.fwd_only else to_device(inp["dy"], shape, dev)
    layer = MoELayer(shape, device=dev)
    flush = L2Flush(dev)
    stream = torch.cuda.current_stream(dev)

    def step():
        layer.forward(x, w["Wg"], bias, w["W1"], w["W3"], w["W2"])
        if dy is not None:
            layer.backward(dy, x, w["Wg"], w["W1"], w["W3"], w["W2"])

    def barrier():
        rank_barrier(world)

    def max_over_ranks(v: float) -> float:
        return reduce_max(v, world, dev)

    for _ in range(args.warmup):
        step()
        flush()
    torch.cuda.synchronize(dev)
    st = layer.status()
    if st != moe.MOE_OK:
        raise RuntimeError(f"device status after warm-up: {moe.STATUS_NAMES.get(st, st)}")

    K = args.steps
    mk = lambda: torch.cuda.Event(enable_timing=True)
    nf, nb = len(moe.FWD_PHASES), len(moe.BWD_PHASES)
    uuid = "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)

    # 1. per-phase breakdown: K steps with the library's phase events recorded on the launching
    #    stream (events between kernels keep consecutive launches from overlapping, so this pass is
    #    separate from the timed one)
    fev = [[mk() for _ in range(nf + 1)] for _ in range(K)]
    bev = [[mk() for _ in range(nb + 1)] for _ in range(K)]
    ps, pe = [mk() for _ in range(K)], [mk() for _ in range(K)]
    for i in range(K):
        moe.set_profile_events(fev[i], None if dy is None else bev[i])
        ps[i].record(stream)
        step()
        pe[i].record(stream)
        moe.set_profile_events(None, None)
        flush()
    torch.cuda.synchronize(dev)
    phased_ms = sum(s.elapsed_time(e) for s, e in zip(ps, pe)) / K
    phase_ms = {}
    for j, name in enumerate(moe.FWD_PHASES):
        phase_ms[name] = sum(fev[i][j].elapsed_time(fev[i][j + 1]) for i in range(K)) / K
    if dy is not None:
        for j, name in enumerate(moe.BWD_PHASES):
            phase_ms[name] = sum(bev[i][j].elapsed_time(bev[i][j + 1]) for i in range(K)) / K
    top = max(phase_ms, key=phase_ms.get)
    in_fwd = top in moe.FWD_PHASES
    tj = (moe.FWD_PHASES if in_fwd else moe.BWD_PHASES).index(top)

    # 2. timed region: K whole steps, one event pair per step and nothing inside the steps
    starts, ends = [mk() for _ in range(K)], [mk() for _ in range(K)]
    barrier()
    torch.cuda.synchronize(dev)
    clocks = ClockSampler(uuid)
    n0 = moe.kernel_launches()
    t_wall = time.perf_counter()
    for i in range(K):
        starts[i].record(stream)
        step()
        ends[i].record(stream)
        flush()
    launches = moe.kernel_launches() - n0
    torch.cuda.synchronize(dev)
    timed_wall_s = time.perf_counter() - t_wall
    clk = clocks.stop()
    barrier()
    total_ms = sum(s.elapsed_time(e) for s, e in zip(starts, ends))
    total_ms = max_over_ranks(total_ms)
    st = layer.status()
    if st != moe.MOE_OK:
        raise RuntimeError(f"device status after timing: {moe.STATUS_NAMES.get(st, st)}")

    # 3. the dominant phase, live: K more steps with the library's events around that phase only
    #    (on the launching stream), for the roofline of its kernel
    t0s, t1s = [mk() for _ in range(K)], [mk() for _ in range(K)]

    def top_events(i):
        arr = [None] * ((nf if in_fwd else nb) + 1)
        arr[tj], arr[tj + 1] = t0s[i], t1s[i]
        return arr

    barrier()
    torch.cuda.synchronize(dev)
    top_clocks = ClockSampler(uuid)
    for i in range(K):
        if in_fwd:
            moe.set_profile_events(top_events(i), None)
        else:
            moe.set_profile_events(None, top_events(i))
        step()
        moe.set_profile_events(None, None)
        flush()
    torch.cuda.synchronize(dev)
    top_clk = top_clocks.stop()
    barrier()
    top_ms_live = max_over_ranks(sum(a.elapsed_time(b) for a, b in zip(t0s, t1s)) / K)

    n_kept = int(layer.view("kept").sum().item())
    work = phase_work(shape, n_kept)
    hbm_gbs, bf16_tf, bf16_sus, peak_src = peaks()
    # the dominant kernel is timed inside back-to-back steps: once the power cap holds the clock
    # down during them (or they last more than about a second) the GPU runs at its power-capped
    # clock, and the sustained bf16 rate is the matching peak
    capped = "sw_power_cap" in (clk.get("reasons") or []) or \
        "sw_power_cap" in (top_clk.get("reasons") or [])
    sustained = capped or timed_wall_s > SUSTAINED_AFTER_S
    mm_peak = bf16_sus if sustained else bf16_tf
    mm_peak_name = "sustained" if sustained else "burst"
    phases = {}
    min_bytes = gemm_min_bytes(shape, n_kept)
    for name, ms in phase_ms.items():
        bound, amount = work[name]
        if bound in ("tensor", "alu"):
            ach = amount / (ms * 1e-3) / 1e12
            peak = mm_peak if bound == "tensor" else FP32_FMA_TFLOPS
            phases[name] = {"ms": ms, "bound": bound, "achieved_tflops": ach, "frac": ach / peak}
            if bound == "tensor":
                phases[name]["frac_burst"] = ach / bf16_tf
                # the GEMM's own roofline: the slower of its tensor time and its HBM time
                mb = min_bytes[name]
                t_roof = max(amount / (peak * 1e12), mb / (hbm_gbs * 1e9))
                phases[name].update(min_hbm_bytes=mb, roofline_ms=t_roof * 1e3,
                                    roofline_bound="tensor" if amount / (peak * 1e12) >=
                                    mb / (hbm_gbs * 1e9) else "hbm",
                                    frac_roofline=t_roof * 1e3 / ms)
        else:
            ach = amount / (ms * 1e-3) / 1e9
            phases[name] = {"ms": ms, "bound": bound, "achieved_gbs": ach, "frac": ach / hbm_gbs}
    tb, tw = work[top]
    traffic, traffic_src = measured_traffic(shape.name, top)
    if tb == "tensor":
        ach = tw / (top_ms_live * 1e-3) / 1e12
        roof = {"kernel": top, "bound": "tensor", "achieved": ach, "peak": mm_peak,
                "unit": "TFLOP/s", "frac": ach / mm_peak, "traffic": traffic,
                "peak_source": f"{peak_src} bf16 dense ({mm_peak_name}: the kernel is timed "
                               f"inside {timed_wall_s:.2f} s of back-to-back steps"
                               f"{', power cap active' if capped else ''})",
                "frac_burst": ach / bf16_tf, "frac_sustained": ach / bf16_sus}
    elif tb == "alu":
        ach = tw / (top_ms_live * 1e-3) / 1e12
        roof = {"kernel": top, "bound": "alu", "achieved": ach, "peak": FP32_FMA_TFLOPS,
                "unit": "TFLOP/s", "frac": ach / FP32_FMA_TFLOPS, "traffic": traffic,
                "peak_source": "derived: 148 SMs x 128 FP32 FMA lanes x 2 x 1965 MHz"}
    else:
        ach = tw / (top_ms_live * 1e-3) / 1e9
        roof = {"kernel": top, "bound": "hbm", "achieved": ach, "peak": hbm_gbs, "unit": "GB/s",
                "frac": ach / hbm_gbs, "traffic": traffic, "peak_source": f"{peak_src} HBM copy"}
    roof["ms_per_launch"] = top_ms_live
    roof["work_per_launch"] = tw
    roof["clocks_sm_mhz"] = top_clk.get("sm_mhz")
    if traffic is not None:
        roof["traffic_unit"] = "bytes per launch"
        roof["traffic_source"] = traffic_src

    # the same step captured once into a CUDA graph and replayed (MoEStepGraph): one host call per
    # step instead of one per launch; reported beside the eager value, which stays the headline
    graph, sg = None, None
    try:
        from mixture_experts_layer_23_b200.layer import MoEStepGraph
        n0 = moe.kernel_launches()
        sg = MoEStepGraph(layer, x, w["Wg"], bias, w["W1"], w["W3"], w["W2"], dy)
        per_step = (moe.kernel_launches() - n0) // 2   # the eager warm-up pass, then the capture
    except Exception as err:   # capture not possible here: report why, keep the eager numbers
        graph = {"error": str(err)[:300]}
    # every rank takes the same collective steps: time the replays only if all ranks captured
    if reduce_max(0.0 if sg is not None else 1.0, world, dev) > 0.0:
        if graph is None:
            graph = {"error": "graph capture failed on another rank"}
        sg = None
    else:
        for _ in range(args.warmup):
            sg.replay()
            flush()
        gs, ge = [mk() for _ in range(K)], [mk() for _ in range(K)]
        barrier()
        torch.cuda.synchronize(dev)
        for i in range(K):
            gs[i].record(stream)
            sg.replay()
            ge[i].record(stream)
            flush()
        torch.cuda.synchronize(dev)
        barrier()
        g_ms = max_over_ranks(sum(a.elapsed_time(b) for a, b in zip(gs, ge)))
        graph = {"value": job_tokens_per_s(world, shape.T, K, g_ms), "unit": "tokens/s",
                 "ms_per_step": g_ms / K, "launches_per_step": per_step}
        del sg

    # end to end through the C ABI with host buffers: every step is one moe_layer_step_host call,
    # which copies that step's x and dy up from pinned host memory, runs the forward and backward
    # and copies y and dx back down.  Two layer instances alternate on two streams, so one step's
    # copies overlap the other's compute (as a training loop prefetching its next batch would).
    # Forward-only layers (no dy) run moe_layer_fwd between torch copies instead.
    e2e_ms, h2d, d2h = None, 0, 0
    layers = [layer, MoELayer(shape, device=dev)]
    x_pin = x.cpu().pin_memory()
    dy_pin = None if dy is None else dy.cpu().pin_memory()
    y_host = [torch.empty(layer.y.shape, dtype=layer.y.dtype).pin_memory() for _ in range(2)]
    dx_host = [torch.empty(layer.dx.shape, dtype=layer.dx.dtype).pin_memory() for _ in range(2)]
    xs = [torch.empty_like(x) for _ in range(2)]
    dys = [None if dy is None else torch.empty_like(dy) for _ in range(2)]
    h2d = x_pin.numel() * x_pin.element_size() + (0 if dy_pin is None else
                                                  dy_pin.numel() * dy_pin.element_size())
    d2h = y_host[0].numel() * y_host[0].element_size() + (0 if dy is None else
                                                          dx_host[0].numel() * dx_host[0].element_size())
    streams = [torch.cuda.Stream(dev), torch.cuda.Stream(dev)]

    def e2e_step(i):
        b = i % 2
        L = layers[b]
        st = streams[b]
        if dy is not None:
            moe.layer_step_host(L.cfg, x_pin, dy_pin, y_host[b], dx_host[b], xs[b], dys[b], w["Wg"],
                                bias, w["W1"], w["W3"], w["W2"], L.y, L.dx, L.dWg, L.dW1, L.dW3,
                                L.dW2, L.ctx, L.scratch, st)
        else:
            with torch.cuda.stream(st):
                xs[b].copy_(x_pin, non_blocking=True)
                L.forward(xs[b], w["Wg"], bias, w["W1"], w["W3"], w["W2"], st)
                y_host[b].copy_(L.y, non_blocking=True)

    for i in range(2):                    # untimed: first-call set-up of both instances
        e2e_step(i)
    torch.cuda.synchronize(dev)
    e_start, e_end = mk(), mk()
    barrier()
    torch.cuda.synchronize(dev)
    e_start.record(stream)
    for st in streams:
        st.wait_stream(stream)
    for i in range(K):
        e2e_step(i)
    for st in streams:
        stream.wait_stream(st)
    e_end.record(stream)
    torch.cuda.synchronize(dev)
    barrier()
    e2e_ms = max_over_ranks(e_start.elapsed_time(e_end))
    for L in layers:
        st = L.status()
        if st != moe.MOE_OK:
            raise RuntimeError(f"device status after the end-to-end pass: {moe.STATUS_NAMES.get(st, st)}")
    del layers[1]
    # no L2 flush between these steps: each step's inputs arrive fresh from the host, and the
    # per-step working set (weights + saved forward state) is compared with L2 below
    work_set = sum(t.numel() * t.element_size() for t in w.values() if t is not None) + \
        layer.L.ctx_bytes
    e2e_l2 = ("no flush; per-step working set %.0f MB > 126 MB L2" % (work_set / 1e6)
              if work_set > 126e6 else
              "no flush; per-step working set %.1f MB fits in L2 (warm)" % (work_set / 1e6))

    # forward-only layers: the one-launch fused forward (moe_layer_fwd_fused), where it applies
    fused = None
    if dy is None:
        yf = torch.empty_like(layer.y)

        def fused_step():
            moe.layer_fwd_fused(layer.cfg, x, w["Wg"], bias, w["W1"], w["W3"], w["W2"], yf)
        try:
            fused_step()
        except moe.MoEError as err:
            if err.status != 2:    # MOE_ERR_UNSUPPORTED: the layer is too large for it
                raise
        else:
            for _ in range(args.warmup):
                fused_step()
                flush()
            fs, fe = [mk() for _ in range(K)], [mk() for _ in range(K)]
            barrier()
            torch.cuda.synchronize(dev)
            for i in range(K):
                fs[i].record(stream)
                fused_step()
                fe[i].record(stream)
                flush()
            torch.cuda.synchronize(dev)
            barrier()
            f_ms = max_over_ranks(sum(a.elapsed_time(b) for a, b in zip(fs, fe)))
            fused = {"entry": "moe_layer_fwd_fused", "value": job_tokens_per_s(world, shape.T, K, f_ms),
                     "unit": "tokens/s", "ms_per_step": f_ms / K, "launches_per_step": 1}

    value = job_tokens_per_s(world, shape.T, K, total_ms)
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": total_ms / K, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16" if shape.dtype == 1 else "f32", "data": "synthetic",
        "config": workload_config(shape, world),
        "run": {"kept_assignments": n_kept,
                "gemm_engine": ["cuda_core", "tcgen05"][moe.gemm_engine(layer.cfg)],
                "timed_wall_s": timed_wall_s},
        "roofline": roof,
        "phases": phases,
        "fused_fwd": fused,
        "graph_replay": graph,
        "phased_ms_per_step": phased_ms,
        "e2e": {"value": job_tokens_per_s(world, shape.T, K, e2e_ms), "unit": "tokens/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "ms_per_step": e2e_ms / K,
                "copies": "every step is one moe_layer_step_host call (C ABI, host buffers): x "
                          "and dy copied up from pinned host memory, y and dx copied back, two "
                          "layer instances alternating on two streams so one step's copies "
                          "overlap the other's compute; the weights and the weight gradients stay "
                          "on the device, as in a training loop whose optimizer runs on the GPU",
                "l2": e2e_l2},
        "gpu_launches": launches,
        "clocks": clk,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(shape, inp, args.cpu_seconds)
    else:
        line["cpu_baseline"] = None
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()
    return 0


def run_ep(args):
    """Expert-parallel layer over the N ranks (mixture_experts_layer_23_b200.ep): every rank routes
    its own batch of T tokens, owns E/N experts, and exchanges rows with the others through NCCL.
    K steps timed with CUDA events after W warm-up steps, max over ranks; prints one JSON line."""
    import torch
    import torch.distributed as dist
    from datetime import timedelta
    rank, local_rank, world = dist_env()
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
    os.environ.setdefault("MASTER_PORT", "29541")
    dist.init_process_group("nccl", rank=rank, world_size=world, timeout=timedelta(seconds=120),
                            device_id=dev)
    from mixture_experts_layer_23_b200 import build as moe_build
    moe_build.build()
    from mixture_experts_layer_23_b200 import moe
    from mixture_experts_layer_23_b200.ep import DistExchange, EPRank, step
    from mixture_experts_layer_23_b200.layer import to_device
    from mixture_experts_layer_23_b200.synth import make_inputs
    shape = bench_shape(args)
    El = shape.E // world
    base = make_inputs(shape, 0, with_dy=False)
    mine = make_inputs(shape, 100 + rank)
    W = {n: to_device(base[n], shape, dev) for n in ("Wg", "W1", "W3", "W2")}
    bias = None if base["bias"] is None else torch.from_numpy(base["bias"]).to(dev)
    sl = slice(rank * El, (rank + 1) * El)
    W1l, W2l = W["W1"][sl].contiguous(), W["W2"][sl].contiguous()
    W3l = None if W["W3"] is None else W["W3"][sl].contiguous()
    x, dy = to_device(mine["x"], shape, dev), to_device(mine["dy"], shape, dev)
    F, d = shape.d_ff, shape.d
    grads = (torch.empty(El, F, d, device=dev),
             None if W3l is None else torch.empty(El, F, d, device=dev),
             torch.empty(El, d, F, device=dev))
    r = EPRank(shape, rank, world, device=dev, chunks=args.ep_chunks)
    ex = DistExchange()
    flush = L2Flush(dev)
    stream = torch.cuda.current_stream(dev)
    for _ in range(args.warmup):
        step(r, ex, x, W["Wg"], bias, W1l, W3l, W2l, dy, grads)
        flush()
    torch.cuda.synchronize(dev)
    K = args.steps
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    dist.barrier()
    torch.cuda.synchronize(dev)
    for i in range(K):
        starts[i].record(stream)
        step(r, ex, x, W["Wg"], bias, W1l, W3l, W2l, dy, grads)
        ends[i].record(stream)
        flush()
    torch.cuda.synchronize(dev)
    dist.barrier()
    total_ms = reduce_max(sum(a.elapsed_time(b) for a, b in zip(starts, ends)), world, dev)
    st = r.status()
    if st != moe.MOE_OK:
        raise RuntimeError(f"device status: {moe.STATUS_NAMES.get(st, st)}")
    if rank == 0:
        print(json.dumps({
            "metric": METRIC, "value": job_tokens_per_s(world, shape.T, K, total_ms),
            "unit": "tokens/s", "n_gpus": world, "steps": K, "warmup": args.warmup,
            "ms_per_step": total_ms / K, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16" if shape.dtype == 1 else "f32",
            "data": "synthetic",
            "config": dict(workload_config(shape, world),
                           parallelism=f"expert parallel x{world}, {El} experts per rank, "
                                       f"{args.ep_chunks} exchange chunk(s)"),
            "note": "expert-parallel mode: each step includes the host sync of the kept counts, "
                    "the exchanges and the router-gradient all-reduce"}), flush=True)
    dist.destroy_process_group()
    return 0


def main():
    args = parse()
    if args.impl == "reference":
        return run_reference(args)
    if args.ep:
        return run_ep(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
