#!/usr/bin/env python3
"""Benchmark of the Q4_0 decode hot path on B200.

One step = one decode pass of the whole path at M draft rows:
  * the 64-layer Q4_0 weight stream (per layer: gate 5120->17408, up
    5120->17408, down 17408->5120, in 5120->6144, out 6144->5120) plus the
    5120->151936 output head: 321 q4_gemv calls, 12.33 GB of weights;
  * Q4-KV decode attention for 16 layers (24 query heads, 4 KV heads,
    head_dim 256) at ctx_len 262144: 16 q4kv_attn_decode calls, 4.83 GB.
Every matrix and cache is distinct (17.2 GB per step, far above the 126 MB
L2), so no L2 flush is needed between steps.  The metric is achieved HBM
TB/s = algorithmic bytes / device time.

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--M m] [--impl reference]
Under torchrun each rank runs an independent replica on its own GPU (the
path has no exchange step); the time is the max over ranks.
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

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "Q4 decode GEMV/attn: achieved HBM TB/s (% of B200 peak), µs per call at M=1..5"
HIDDEN, FFN, QKV, HEAD_N, LAYERS = 5120, 17408, 6144, 151936, 64
ATTN_LAYERS, N_Q, N_KV, HEAD_DIM, CTX = 16, 24, 4, 256, 262144
LAYER_SHAPES = [(FFN, HIDDEN), (FFN, HIDDEN), (HIDDEN, FFN), (QKV, HIDDEN), (HIDDEN, QKV)]  # (N, K)
L2_BYTES = 126 * 1024 * 1024


def q4_bytes(N, K):
    return N * (K // 256) * 144


def gemv_alg_bytes(M, N, K):
    return q4_bytes(N, K) + 2 * M * K + 4 * M * N


def attn_alg_bytes(M, ctx, row_bytes=144):
    """K and V rows (144 B per token and KV head for Q4_0, 272 B for Q8_0)
    plus the bf16 queries and fp32 outputs."""
    return 2 * N_KV * ctx * row_bytes + M * N_Q * HEAD_DIM * (2 + 4)


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


def kernel_source_hash():
    """Hash of the sources the measured kernels are built from (every file of
    csrc/ but the wait self-test, which no measured launch runs)."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "bit_weight_streaming_dequant_b200", "csrc")
    for name in sorted(os.listdir(csrc)):
        if name.startswith("q4d_selftest"):
            continue
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(name.encode() + f.read())
    return h.hexdigest()[:16]


def recorded_traffic(kernel, M):
    """DRAM bytes (read + write) per launch of the step's kernel at M rows, from
    the committed ncu record profiles/dram_traffic.json, if it was taken on the
    current kernel sources (else None)."""
    path = os.path.join(ROOT, "profiles", "dram_traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f)
    except Exception:
        return None
    if rec.get("source_hash") != kernel_source_hash():
        return None
    e = rec.get("step", {}).get(kernel, {}).get(f"M{M}")
    return None if not e else e.get("bytes_per_launch")


# ------------------------------------------------------------------ clocks --
class ClockSampler:
    """SM clock, power and clock-event reasons sampled every few milliseconds
    from a background thread through NVML (read-only queries) while the timed
    region runs; nvidia-smi polling is the fallback when NVML is missing."""

    REASONS = [("hw_slowdown", "nvmlClocksEventReasonHwSlowdown"),
               ("hw_thermal_slowdown", "nvmlClocksEventReasonHwThermalSlowdown"),
               ("sw_thermal_slowdown", "nvmlClocksEventReasonSwThermalSlowdown"),
               ("sw_power_cap", "nvmlClocksEventReasonSwPowerCap"),
               ("hw_power_brake", "nvmlClocksEventReasonHwPowerBrakeSlowdown")]

    def __init__(self, torch_dev_index, period_s=0.002):
        import threading

        self.samples = []
        self.err = None
        self._stop = threading.Event()
        self._nvml = None
        try:
            import pynvml

            pynvml.nvmlInit()
            visible = os.environ.get("CUDA_VISIBLE_DEVICES")
            idx = torch_dev_index
            if visible:
                ids = [v.strip() for v in visible.split(",") if v.strip()]
                if torch_dev_index < len(ids) and ids[torch_dev_index].isdigit():
                    idx = int(ids[torch_dev_index])
            self._h = pynvml.nvmlDeviceGetHandleByIndex(idx)
            self._nvml = pynvml
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
        except Exception as e:  # noqa: BLE001
            self.err = f"nvml: {e}"
            self.max_mhz = None
        self._period = period_s
        self._thread = threading.Thread(target=self._run, daemon=True)

    def _run(self):
        nv = self._nvml
        masks = [(name, getattr(nv, attr, 0)) for name, attr in self.REASONS]
        while not self._stop.is_set():
            try:
                mhz = nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM)
                rs = nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                pw = nv.nvmlDeviceGetPowerUsage(self._h) / 1000.0
                self.samples.append((mhz, pw, [n for n, m in masks if m and rs & m]))
            except Exception as e:  # noqa: BLE001
                self.err = f"nvml sample: {e}"
                break
            self._stop.wait(self._period)

    def start(self):
        if self._nvml is not None:
            self._thread.start()

    def stop(self):
        if self._nvml is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0,
                    "error": self.err}
        self._stop.set()
        self._thread.join(timeout=5)
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0,
                    "error": self.err or "no sample inside the timed region"}
        mhz = [m for m, _, _ in self.samples]
        reasons = sorted({r for _, _, rs in self.samples for r in rs})
        return {"sm_mhz": statistics.median(mhz), "sm_max_mhz": self.max_mhz,
                "sm_min_mhz": min(mhz), "power_w_median": statistics.median(
                    [p for _, p, _ in self.samples]),
                "reasons": reasons, "samples": len(self.samples), "source": "nvml"}


# --------------------------------------------------------------- CPU arms --
def cpu_cores():
    try:
        from threadpoolctl import threadpool_info

        n = max((i.get("num_threads", 1) for i in threadpool_info()), default=1)
    except Exception:
        n = 1
    return int(n)


def reduce_over_ranks(values, device, world, op="max"):
    """Element-wise max (or min) of per-rank floats over all ranks of the
    process group (the timed regions' durations: the job takes as long as its
    slowest rank).  With one rank, the values themselves."""
    import torch

    t = torch.tensor(list(values), dtype=torch.float64, device=device)
    if world > 1:
        import torch.distributed as dist

        dist.all_reduce(t, op=dist.ReduceOp.MAX if op == "max" else dist.ReduceOp.MIN)
    return t.tolist()


def job_tbps(bytes_per_rank_step, steps, world, max_ms):
    """Whole-job throughput: every rank moves bytes_per_rank_step per step
    (weak scaling), the job lasts max_ms (the slowest rank)."""
    return bytes_per_rank_step * steps * world / (max_ms * 1e-3) / 1e12


def oracle_sample_step(seed=0):
    """One bounded sample of the workload on the CPU oracle: a 5120->6144
    GEMV at M rows and one attention layer at ctx 4096.  Returns
    (algorithmic bytes, seconds)."""
    import oracle
    import synth

    N, K = QKV, HIDDEN
    W = synth.q4_0_weights(1000 + seed, N, K)
    x = synth.activations(2000 + seed, ARGS.M, K)
    ctx = 4096
    Kc, Vc = synth.q4_0_kv_cache(3000 + seed, N_KV, ctx), synth.q4_0_kv_cache(4000 + seed, N_KV, ctx)
    Q = synth.queries(5000 + seed, ARGS.M, N_Q)
    t0 = time.perf_counter()
    oracle.gemv(W, x, ARGS.M, N, K)
    oracle.attn_decode(Q, Kc, Vc, ctx, N_Q, N_KV, HEAD_DIM, ARGS.M)
    dt = time.perf_counter() - t0
    return gemv_alg_bytes(ARGS.M, N, K) + attn_alg_bytes(ARGS.M, ctx), dt


SAMPLE_DESC = ("fp64 numpy oracle: one 5120->6144 Q4_0 GEMV plus one attention layer at "
               "ctx 4096 (24/4 heads) per sample, M as the GPU arm; inputs generated "
               "outside the timed part")


def cpu_baseline(min_seconds=10.0, max_samples=40):
    """The oracle on the host cores: samples until ~10 s of oracle time (at
    most 40 samples), so the default bench run stays within minutes."""
    total_b, total_t, n = 0, 0.0, 0
    while n < max_samples and total_t < min_seconds:
        b, t = oracle_sample_step(n)
        total_b += b
        total_t += t
        n += 1
    out = {"value": total_b / total_t / 1e12, "unit": "TB/s", "cores": cpu_cores(),
           "kind": "oracle", "seconds": total_t, "sample": f"{n} samples; " + SAMPLE_DESC}
    try:  # the same oracle on one thread
        from threadpoolctl import threadpool_limits

        with threadpool_limits(limits=1):
            b, t = oracle_sample_step(n)
        out["single_thread"] = {"value": b / t / 1e12, "cores": 1, "sample": "1 sample"}
    except Exception as e:  # noqa: BLE001
        out["single_thread"] = {"error": str(e)[:200]}
    return out


def run_reference(args, rank, world):
    if rank != 0:
        return
    for s in range(args.warmup):
        oracle_sample_step(100 + s)
    bs, ts = [], []
    for s in range(args.steps):
        b, t = oracle_sample_step(s)
        bs.append(b)
        ts.append(t)
    value = sum(bs) / sum(ts) / 1e12
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "TB/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * sum(ts) / len(ts), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": workload_config(args),
            "cpu_baseline": {"kind": "oracle", "cores": cpu_cores(), "value": value,
                             "unit": "TB/s", "sample": "each step: " + SAMPLE_DESC},
            "e2e": {"value": value, "unit": "TB/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def workload_config(args):
    return {"workload": (f"decode step at M={args.M}: 64-layer Q4_0 weight stream "
                         "(5120->17408 x2, 17408->5120, 5120->6144, 6144->5120) + "
                         "5120->151936 head = 321 GEMVs, then 16-layer Q4-KV attention "
                         f"(24 q / 4 kv heads, head_dim 256) at ctx_len {CTX}"),
            "M": args.M, "ctx_len": CTX, "layers": LAYERS, "attn_layers": ATTN_LAYERS,
            "bytes_per_step": step_bytes(args.M),
            "l2": "inputs larger than L2 (17.2 GB of distinct weights/caches per step)",
            "gemv_launch": ("one q4_gemv_batch_ex launch of the 321 matrices per step, each "
                            "waiting for its predecessor in the layer chain"),
            "parallelism": f"replicas x{args.gpus}"}


def step_bytes(M):
    g = sum(gemv_alg_bytes(M, N, K) for N, K in LAYER_SHAPES) * LAYERS
    g += gemv_alg_bytes(M, HEAD_N, HIDDEN)
    return g + ATTN_LAYERS * attn_alg_bytes(M, CTX)


# ------------------------------------------------------------- GPU arm --
def main():
    global ARGS
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--M", type=int, default=1, choices=[1, 2, 3, 4, 5])
    ap.add_argument("--impl", default="libq4dec", choices=["libq4dec", "reference"])
    ap.add_argument("--no-per-call", action="store_true")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--case", default="step", choices=["step", "gemv", "gemv_batch", "attn"],
                    help="gemv/gemv_batch/attn: a few launches of one kernel (small case for "
                         "profilers)")
    ap.add_argument("--layers", type=int, default=2, help="--case gemv_batch: layers per launch")
    ap.add_argument("--shape", default="17408x5120", help="--case gemv: NxK")
    ap.add_argument("--ctx", type=int, default=65536, help="--case attn: ctx_len")
    ap.add_argument("--launches", type=int, default=8, help="--case gemv/attn: launches")
    ap.add_argument("--q8", action="store_true", help="--case attn: the Q8_0 K/V cache")
    ap.add_argument("--nvtx", action="store_true",
                    help="mark the step's weight stream and attention layers as NVTX ranges "
                         "(for a profiler's range filters; off for the reported numbers)")
    args = ap.parse_args()
    DecodeStep.nvtx = args.nvtx
    ARGS = args
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        run_reference(args, rank, world)
        return

    import torch
    import torch.distributed as dist

    import synth
    from bit_weight_streaming_dequant_b200 import q4dec

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if args.case != "step":
        run_case(args, torch, dev)
        return
    if world > 1:
        from datetime import timedelta

        dist.init_process_group("nccl", timeout=timedelta(seconds=120),
                                device_id=dev)
    q4dec.lib()
    M = args.M

    # -------- resident state: weights and caches (generated on the device)
    gen_t0 = time.time()
    layers = []
    for l in range(LAYERS):
        layers.append([synth.device_q4_0_weights(1000 + 5 * l + i, N, K, device=dev)
                       for i, (N, K) in enumerate(LAYER_SHAPES)])
    head = synth.device_q4_0_weights(999, HEAD_N, HIDDEN, device=dev)
    kv = [(synth.device_q4_0_kv_cache(2000 + l, N_KV, CTX, device=dev),
           synth.device_q4_0_kv_cache(2100 + l, N_KV, CTX, device=dev))
          for l in range(ATTN_LAYERS)]
    L = q4dec.lib()
    step = DecodeStep(torch, q4dec, synth, dev, layers, head, kv, M)
    m5 = DecodeStep(torch, q4dec, synth, dev, layers, head, kv, 5) if M != 5 else None
    torch.cuda.synchronize()
    gen_s = time.time() - gen_t0

    stream = torch.cuda.current_stream()

    def barrier():
        if world > 1:
            dist.barrier()

    clocks = ClockSampler(local)
    for _ in range(args.warmup):
        step.gemv_stream()
        step.attn_stream()
    torch.cuda.synchronize()

    # -------- timed region
    K_ = args.steps
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True),
           torch.cuda.Event(enable_timing=True)) for _ in range(K_)]
    step.launches = 0
    barrier()
    torch.cuda.synchronize()
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    clocks.start()
    t_start.record(stream)
    for k in range(K_):
        ev[k][0].record(stream)
        step.gemv_stream()
        ev[k][1].record(stream)
        step.attn_stream()
        ev[k][2].record(stream)
    t_end.record(stream)
    torch.cuda.synchronize()
    barrier()
    timed_launches = step.launches
    total_ms = t_start.elapsed_time(t_end)
    gemv_ms = sum(e[0].elapsed_time(e[1]) for e in ev)
    attn_ms = sum(e[1].elapsed_time(e[2]) for e in ev)
    clock = clocks.stop()

    total_ms, gemv_ms, attn_ms = reduce_over_ranks([total_ms, gemv_ms, attn_ms], dev, world)

    bytes_step = step_bytes(M)
    value = job_tbps(bytes_step, K_, world, total_ms)
    peak_gbs, peak_kind = peaks()
    gemv_bytes = gemv_step_bytes(M)
    gemv_launch_s = gemv_ms * 1e-3 / K_            # one batch launch per step
    achieved_gbs = gemv_bytes / gemv_launch_s / 1e9
    attn_gbs = ATTN_LAYERS * attn_alg_bytes(M, CTX) * K_ / (attn_ms * 1e-3) / 1e9

    # -------- the same weight stream as 321 separate launches (one per matrix,
    # weight prefetch under programmatic dependent launch), for comparison
    sep = time_region(torch, stream, lambda: step.gemv_stream_per_matrix(), max(3, K_ // 5))
    sep_ms = reduce_over_ranks([sep], dev, world)[0]
    per_matrix = {"ms_per_step": sep_ms, "value": gemv_bytes / (sep_ms * 1e-3) / 1e12,
                  "unit": "TB/s", "launches_per_step": step.n_gemv}

    # -------- the step at M = 5 (target verification of a 4-token draft)
    m5_rec = None
    if m5 is not None:
        for _ in range(args.warmup):
            m5.gemv_stream()
            m5.attn_stream()
        k5 = max(5, K_ // 5)
        g5 = time_region(torch, stream, m5.gemv_stream, k5)
        a5 = time_region(torch, stream, m5.attn_stream, k5)
        t5 = time_region(torch, stream, lambda: (m5.gemv_stream(), m5.attn_stream()), k5)
        s5 = time_region(torch, stream, m5.gemv_stream_per_matrix, k5)
        g5, a5, t5, s5 = reduce_over_ranks([g5, a5, t5, s5], dev, world)
        gb5 = gemv_step_bytes(5) / (g5 * 1e-3) / 1e9
        ab5 = ATTN_LAYERS * attn_alg_bytes(5, CTX) / (a5 * 1e-3) / 1e9
        m5_rec = {"M": 5, "steps": k5, "ms_per_step": t5,
                  "value": job_tbps(step_bytes(5), 1, world, t5), "unit": "TB/s",
                  "bytes_per_step": step_bytes(5),
                  "roofline": {"bound": "hbm", "kernel": "q4_gemv_kernel<5> (one launch)",
                               "achieved": gb5, "peak": peak_gbs, "unit": "GB/s",
                               "frac": gb5 / peak_gbs, "launch_us": g5 * 1e3,
                               "traffic": recorded_traffic("q4_gemv_kernel", 5)},
                  "attention": {"achieved_gbs": ab5, "frac": ab5 / peak_gbs,
                                "us_per_layer": a5 * 1e3 / ATTN_LAYERS,
                                "traffic": recorded_traffic("q4kv_attn", 5)},
                  "gemv_one_launch_per_matrix": {
                      "ms_per_step": s5, "value": gemv_step_bytes(5) / (s5 * 1e-3) / 1e12,
                      "unit": "TB/s", "launches_per_step": m5.n_gemv}}
        del m5

    # -------- the same step replayed as one CUDA graph
    graph = None
    g = None
    try:
        g = torch.cuda.CUDAGraph()
        s_cap = torch.cuda.Stream()
        s_cap.wait_stream(stream)
        with torch.cuda.stream(s_cap):
            step.gemv_stream()
            step.attn_stream()
        torch.cuda.synchronize()
        with torch.cuda.graph(g, stream=s_cap):
            step.gemv_stream()
            step.attn_stream()
        torch.cuda.synchronize()
        for _ in range(args.warmup):
            g.replay()
        torch.cuda.synchronize()
        graph_err = None
    except Exception as e:  # noqa: BLE001 - report, keep the eager numbers
        graph_err = f"{type(e).__name__}: {e}"[:300]
        torch.cuda.synchronize()
    ok = reduce_over_ranks([0.0 if graph_err else 1.0], dev, world, op="min")[0]
    if ok == 1.0:
        barrier()
        gms = time_region(torch, stream, g.replay, K_)
        barrier()
        gms = reduce_over_ranks([gms], dev, world)[0]
        graph = {"ms_per_step": gms, "value": job_tbps(bytes_step, 1, world, gms),
                 "unit": "TB/s", "replays": K_}
    else:
        graph = {"error": graph_err or "capture failed on another rank"}
    del g
    torch.cuda.synchronize()

    # -------- end to end through the public API with host buffers
    e2e_steps = max(3, min(K_, 10))
    step.e2e_step()
    torch.cuda.synchronize()
    barrier()
    e2e_ms = time_region(torch, stream, step.e2e_step, e2e_steps)
    barrier()
    e2e_ms = reduce_over_ranks([e2e_ms], dev, world)[0]
    e2e_value = job_tbps(bytes_step, 1, world, e2e_ms)

    # -------- per-call latencies (cold L2), rank 0
    per_call = None
    if rank == 0 and not args.no_per_call:
        per_call = per_call_table(torch, L, dev, layers, kv, peak_gbs)

    base = None
    if rank == 0 and world == 1 and not args.no_cpu:
        base = cpu_baseline()

    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return
    line = {
        "metric": METRIC, "value": value, "unit": "TB/s", "n_gpus": world, "steps": K_,
        "warmup": args.warmup, "ms_per_step": total_ms / K_, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": workload_config(args),
        "frac_of_peak": value / world / (peak_gbs / 1e3),
        "roofline": {"bound": "hbm", "kernel": f"q4_gemv_kernel<{M}> (one launch per step)",
                     "achieved": achieved_gbs,
                     "peak": peak_gbs, "peak_source": f"{peak_kind} hbm_gbs", "unit": "GB/s",
                     "frac": achieved_gbs / peak_gbs,
                     "traffic": recorded_traffic("q4_gemv_kernel", M),
                     "algorithmic_bytes_per_launch": gemv_bytes,
                     "launch_us": gemv_launch_s * 1e6,
                     "matrices_per_launch": step.n_gemv},
        "attention": {"achieved_gbs": attn_gbs, "frac": attn_gbs / peak_gbs,
                      "us_per_layer": attn_ms * 1e3 / (K_ * ATTN_LAYERS),
                      "traffic": recorded_traffic("q4kv_attn", M)},
        "m5": m5_rec,
        "gemv_one_launch_per_matrix": per_matrix,
        "cpu_baseline": base,
        "e2e": {"value": e2e_value, "unit": "TB/s", "h2d_bytes_per_step": step.h2d,
                "d2h_bytes_per_step": step.d2h, "steps": e2e_steps},
        "gpu_launches": timed_launches,
        "clocks": clock,
        "graph": graph,
        "per_call": per_call,
        "setup_s": gen_s,
    }
    print(json.dumps(line), flush=True)


def time_region(torch, stream, fn, reps):
    """Device time of `reps` calls of fn on `stream` (CUDA events, synchronised
    on both sides); ms per call."""
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(reps):
        fn()
    b.record(stream)
    torch.cuda.synchronize()
    return a.elapsed_time(b) / reps


def gemv_step_bytes(M):
    return sum(gemv_alg_bytes(M, N, K) for N, K in LAYER_SHAPES) * LAYERS + \
        gemv_alg_bytes(M, HEAD_N, HIDDEN)


class DecodeStep:
    """One decode step at M rows on resident weights and caches.

    The 321 GEMVs run as one batch launch (q4_gemv_batch_ex) in the order of a
    layer -- in-projection, out-projection, gate, up, down -- then the head,
    with the dependencies of a real layer: out waits for in, gate and up for
    out (not for each other), down for up (and so gate), the next layer's in
    for down, the head for the last down.  Each matrix type writes its own
    output buffer; the activations are fixed synthetic inputs (a real chain
    would feed each output on, through the attention and norm steps that are
    not part of this path)."""

    def __init__(self, torch, q4dec, synth, dev, layers, head, kv, M):
        self.torch, self.q4dec, self.L, self.dev, self.M = torch, q4dec, q4dec.lib(), dev, M
        self.layers, self.head, self.kv = layers, head, kv
        self.xs = {K: synth.device_bf16_normal(7 + K + 100 * M, (M, K), device=dev)
                   for K in (HIDDEN, FFN, QKV)}
        names = ("gate", "up", "down", "in", "out")
        self.ys = {n: torch.empty((M, N), dtype=torch.float32, device=dev)
                   for n, (N, K) in zip(names, LAYER_SHAPES)}
        self.ys["head"] = torch.empty((M, HEAD_N), dtype=torch.float32, device=dev)
        self.Qs = [synth.device_bf16_normal(2200 + l + 100 * M, (M, N_Q, HEAD_DIM), scale=1 / 16,
                                            device=dev) for l in range(ATTN_LAYERS)]
        self.outs = [torch.empty((M, N_Q, HEAD_DIM), dtype=torch.float32, device=dev)
                     for _ in range(ATTN_LAYERS)]
        order = (3, 4, 0, 1, 2)                      # in, out, gate, up, down
        jobs, prev_down = [], -1
        for l in range(LAYERS):
            base = len(jobs)
            waits = {3: prev_down, 4: base, 0: base + 1, 1: base + 1, 2: base + 3}
            for i in order:
                N, K = LAYER_SHAPES[i]
                jobs.append(dict(W=layers[l][i], x=self.xs[K], y=self.ys[names[i]], N=N, K=K,
                                 wait_for=waits[i]))
            prev_down = base + 4
        jobs.append(dict(W=head, x=self.xs[HIDDEN], y=self.ys["head"], N=HEAD_N, K=HIDDEN,
                         wait_for=prev_down))
        self.jobs = jobs
        self.n_gemv = len(jobs)
        self.batch = q4dec.GemvBatch(jobs)
        self.aws = self.L.q4d_attn_workspace_bytes(CTX, N_Q, N_KV, HEAD_DIM, M)
        self.attn_ws = torch.empty(max(self.aws, 16), dtype=torch.uint8, device=dev)
        # GEMV workspace: zero-filled once, every launch leaves it so
        self.gemv_ws = torch.zeros(max(16, max(self.L.q4d_gemv_workspace_bytes(M, N, K)
                                               for N, K in LAYER_SHAPES + [(HEAD_N, HIDDEN)])),
                                   dtype=torch.uint8, device=dev)
        self.launches = 0
        self.h2d = self.d2h = 0
        self.h_x = {K: torch.empty((M, K), dtype=torch.bfloat16, pin_memory=True)
                    for K in self.xs}
        for K in self.xs:
            self.h_x[K].copy_(self.xs[K])
        self.h_q = [torch.empty((M, N_Q, HEAD_DIM), dtype=torch.bfloat16, pin_memory=True)
                    for _ in self.Qs]
        for q, h in zip(self.Qs, self.h_q):
            h.copy_(q)
        self.h_y = {n: torch.empty_like(y, device="cpu").pin_memory() for n, y in self.ys.items()}
        self.h_o = [torch.empty((M, N_Q, HEAD_DIM), dtype=torch.float32, pin_memory=True)
                    for _ in self.outs]

    nvtx = False   # NVTX ranges around the step's phases (bench.py --nvtx)

    def _range(self, name):
        if self.nvtx:
            self.torch.cuda.nvtx.range_push(name)

    def _end(self):
        if self.nvtx:
            self.torch.cuda.nvtx.range_pop()

    def gemv_stream(self):
        # one launch; the weights of later matrices stream while earlier ones
        # finish (programmatic dependent launch against the previous kernel)
        self._range(f"weight stream M={self.M}")
        self.batch.run(weight_prefetch=True)
        self._end()
        self.launches += 1

    def gemv_stream_per_matrix(self):
        torch, L, M = self.torch, self.L, self.M
        sptr = torch.cuda.current_stream().cuda_stream
        for j in self.jobs:
            st = L.q4_gemv_ex2(j["W"].data_ptr(), j["x"].data_ptr(), j["y"].data_ptr(), M,
                               j["N"], j["K"], sptr, self.gemv_ws.data_ptr(),
                               self.gemv_ws.numel(), self.q4dec.GEMV_WEIGHT_PREFETCH)
            if st:
                raise RuntimeError(f"q4_gemv_ex2 failed: {st}")

    def attn(self, l):
        torch, L, M = self.torch, self.L, self.M
        Kc, Vc = self.kv[l]
        st = L.q4kv_attn_decode_ex(self.Qs[l].data_ptr(), Kc.data_ptr(), Vc.data_ptr(),
                                   self.outs[l].data_ptr(), CTX, N_Q, N_KV, HEAD_DIM, M, CTX,
                                   1.0, torch.cuda.current_stream().cuda_stream,
                                   self.attn_ws.data_ptr(), self.attn_ws.numel())
        if st:
            raise RuntimeError(f"q4kv_attn_decode_ex failed: {st}")
        self.launches += 2 if self.aws else 1

    def attn_stream(self):
        for l in range(ATTN_LAYERS):
            self._range(f"attention layer {l}")
            self.attn(l)
            self._end()

    def e2e_step(self):
        # the step's inputs (the activation rows of each width, every attention
        # layer's queries) come from pinned host memory; its results (the last
        # output of each matrix type, the logits, every attention output) go
        # back to it; the kernels are the timed step's.  As a decode loop would,
        # the copies that nothing waits for run on a second stream beside the
        # kernels: the queries go up while the weight stream runs, the GEMV
        # results and each attention layer's output come down while the next
        # layers run; the step ends when both streams have finished (every
        # copy is inside the timed region).
        torch = self.torch
        main = torch.cuda.current_stream()
        if not hasattr(self, "side"):
            self.side = torch.cuda.Stream(device=main.device)
        side = self.side
        self.h2d = self.d2h = 0
        for K in self.xs:
            self.xs[K].copy_(self.h_x[K], non_blocking=True)
            self.h2d += self.xs[K].numel() * 2
        side.wait_stream(main)      # after the previous step, inside this one
        with torch.cuda.stream(side):
            for q, h in zip(self.Qs, self.h_q):
                q.copy_(h, non_blocking=True)
                self.h2d += q.numel() * 2
        q_ready = side.record_event()
        self.gemv_stream()
        gemv_done = main.record_event()
        side.wait_event(gemv_done)
        with torch.cuda.stream(side):
            for n, y in self.ys.items():
                self.h_y[n].copy_(y, non_blocking=True)
                self.d2h += y.numel() * y.element_size()
        main.wait_event(q_ready)
        for l, (o, h) in enumerate(zip(self.outs, self.h_o)):
            self.attn(l)
            side.wait_event(main.record_event())   # layer l's output is written
            with torch.cuda.stream(side):
                h.copy_(o, non_blocking=True)
            self.d2h += o.numel() * 4
        main.wait_stream(side)      # the step ends with both streams


def per_call_table(torch, L, dev, layers, kv, peak_gbs, reps=15):
    """Median device time of single calls, L2 flushed before each call by
    reading a buffer twice its size (which also writes back any dirty lines
    before the timed call starts)."""
    flush_buf = torch.ones(2 * L2_BYTES // 4, dtype=torch.int32, device=dev)

    class _Flush:
        def fill_(self, _):
            flush_buf.sum()

    flush = _Flush()
    gemv_need = max([L.q4d_gemv_workspace_bytes(M, N, K) for M in range(1, 6)
                     for N, K in LAYER_SHAPES] + [16])
    gemv_ws = torch.zeros(gemv_need, dtype=torch.uint8, device=dev)  # kept zero by the GEMV
    need = max([L.q4d_attn_workspace_bytes(c, N_Q, N_KV, HEAD_DIM, M) for M in (1, 5)
                for c in (4096, 65536, CTX)] +
               [L.q8kv_attn_workspace_bytes(c, N_Q, N_KV, HEAD_DIM, M) for M in (1, 5)
                for c in (65536, CTX)] + [16])
    ws = torch.empty(need, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()
    sptr = stream.cuda_stream
    table = {"gemv": [], "attn": [], "l2": "flushed before every call (252 MB read)"}
    names = {(FFN, HIDDEN): "5120->17408", (HIDDEN, FFN): "17408->5120",
             (QKV, HIDDEN): "5120->6144", (HIDDEN, QKV): "6144->5120"}
    shape_idx = {(FFN, HIDDEN): 0, (HIDDEN, FFN): 2, (QKV, HIDDEN): 3, (HIDDEN, QKV): 4}
    for (N, K), name in names.items():
        for M in (1, 2, 3, 4, 5):
            x = torch.randn((M, K), device=dev).to(torch.bfloat16)
            y = torch.empty((M, N), dtype=torch.float32, device=dev)
            times = []
            for r in range(reps + 2):
                W = layers[r % len(layers)][shape_idx[(N, K)]]
                flush.fill_(r & 0xFF)
                a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record(stream)
                st = L.q4_gemv_ex(W.data_ptr(), x.data_ptr(), y.data_ptr(), M, N, K, sptr,
                                  gemv_ws.data_ptr(), gemv_ws.numel())
                b.record(stream)
                if st:
                    raise RuntimeError(f"q4_gemv_ex failed: {st}")
                torch.cuda.synchronize()
                if r >= 2:
                    times.append(a.elapsed_time(b) * 1e3)
            us = statistics.median(times)
            gbs = gemv_alg_bytes(M, N, K) / (us * 1e-6) / 1e9
            table["gemv"].append({"shape": name, "M": M, "us": us, "GBps": gbs,
                                  "frac": gbs / peak_gbs})
    for ctx in (4096, 65536, 262144):
        for M in (1, 5):
            Q = torch.randn((M, N_Q, HEAD_DIM), device=dev).div_(16).to(torch.bfloat16)
            out = torch.empty((M, N_Q, HEAD_DIM), dtype=torch.float32, device=dev)
            times = []
            for r in range(reps + 2):
                Kc, Vc = kv[r % len(kv)]
                flush.fill_(r & 0xFF)
                a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record(stream)
                st = L.q4kv_attn_decode_ex(Q.data_ptr(), Kc.data_ptr(), Vc.data_ptr(),
                                           out.data_ptr(), ctx, N_Q, N_KV, HEAD_DIM, M, CTX,
                                           1.0, sptr, ws.data_ptr(), ws.numel())
                b.record(stream)
                if st:
                    raise RuntimeError(f"q4kv_attn_decode_ex failed: {st}")
                torch.cuda.synchronize()
                if r >= 2:
                    times.append(a.elapsed_time(b) * 1e3)
            us = statistics.median(times)
            gbs = attn_alg_bytes(M, ctx) / (us * 1e-6) / 1e9
            table["attn"].append({"ctx": ctx, "M": M, "us": us, "GBps": gbs,
                                  "frac": gbs / peak_gbs})
    # the same attention over the Q8_0 cache (272-byte rows), own caches
    import synth
    kv8 = [(synth.device_q8_0_kv_cache(9000 + 2 * i, N_KV, CTX, device=dev),
            synth.device_q8_0_kv_cache(9001 + 2 * i, N_KV, CTX, device=dev)) for i in range(2)]
    table["attn_q8"] = []
    for ctx in (65536, 262144):
        for M in (1, 5):
            Q = torch.randn((M, N_Q, HEAD_DIM), device=dev).div_(16).to(torch.bfloat16)
            out = torch.empty((M, N_Q, HEAD_DIM), dtype=torch.float32, device=dev)
            times = []
            for r in range(reps + 2):
                Kc, Vc = kv8[r % len(kv8)]
                flush.fill_(r & 0xFF)
                a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record(stream)
                st = L.q8kv_attn_decode_ex(Q.data_ptr(), Kc.data_ptr(), Vc.data_ptr(),
                                           out.data_ptr(), ctx, N_Q, N_KV, HEAD_DIM, M, CTX,
                                           1.0, sptr, ws.data_ptr(), ws.numel())
                b.record(stream)
                if st:
                    raise RuntimeError(f"q8kv_attn_decode_ex failed: {st}")
                torch.cuda.synchronize()
                if r >= 2:
                    times.append(a.elapsed_time(b) * 1e3)
            us = statistics.median(times)
            gbs = attn_alg_bytes(M, ctx, 272) / (us * 1e-6) / 1e9
            table["attn_q8"].append({"ctx": ctx, "M": M, "us": us, "GBps": gbs,
                                     "frac": gbs / peak_gbs})
    del kv8
    # t(M=5) / t(M=1) per GEMV shape: about 1 is what makes verification cheap
    by = {(r["shape"], r["M"]): r["us"] for r in table["gemv"]}
    table["gemv_m5_over_m1"] = {name: by[(name, 5)] / by[(name, 1)] for name in names.values()}
    # fused gate / up + SwiGLU (one 2 x 17408 x 5120 interleaved matrix) vs the
    # two separate 5120 -> 17408 GEMVs of the table above
    import synth
    from bit_weight_streaming_dequant_b200 import q4dec
    Wgu = [synth.device_q4_0_weights(7000 + i, 2 * FFN, HIDDEN, device=dev) for i in range(2)]
    table["gate_up_swiglu"] = []
    for M in (1, 5):
        x = torch.randn((M, HIDDEN), device=dev).to(torch.bfloat16)
        row = {"M": M}
        # fp32 h, and bf16 h (Q4D_GEMV_OUT_BF16: the down projection's input format)
        for key, dt, flags in (("us", torch.float32, 0),
                               ("us_bf16_out", torch.bfloat16, q4dec.GEMV_OUT_BF16)):
            h = torch.empty((M, FFN), dtype=dt, device=dev)
            times = []
            for r in range(reps + 2):
                flush.fill_(r & 0xFF)
                a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record(stream)
                st = L.q4_gemv_swiglu_ex(Wgu[r % 2].data_ptr(), x.data_ptr(), h.data_ptr(), M,
                                         FFN, HIDDEN, sptr, ws.data_ptr(), ws.numel(), flags)
                b.record(stream)
                if st:
                    raise RuntimeError(f"q4_gemv_swiglu_ex failed: {st}")
                torch.cuda.synchronize()
                if r >= 2:
                    times.append(a.elapsed_time(b) * 1e3)
            row[key] = statistics.median(times)
        us = row["us"]
        gbs = (2 * q4_bytes(FFN, HIDDEN) + 2 * M * HIDDEN + 4 * M * FFN) / (us * 1e-6) / 1e9
        row.update({"GBps": gbs, "frac": gbs / peak_gbs,
                    "separate_gate_plus_up_us": 2 * by[("5120->17408", M)]})
        table["gate_up_swiglu"].append(row)
    del Wgu
    # K/V append of M verified tokens (4 KV heads), a small cache of its own
    stride = 4096
    Kc = torch.zeros(N_KV * stride * 144, dtype=torch.uint8, device=dev)
    Vc = torch.zeros_like(Kc)
    table["kv_append"] = []
    for M in (1, 5):
        kn = torch.randn((M, N_KV, HEAD_DIM), device=dev)
        vn = torch.randn((M, N_KV, HEAD_DIM), device=dev)
        times = []
        for r in range(reps + 2):
            flush.fill_(r & 0xFF)
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            st = L.q4kv_append(Kc.data_ptr(), Vc.data_ptr(), kn.data_ptr(), vn.data_ptr(), N_KV,
                               stride, stride - M, M, sptr)
            b.record(stream)
            if st:
                raise RuntimeError(f"q4kv_append failed: {st}")
            torch.cuda.synchronize()
            if r >= 2:
                times.append(a.elapsed_time(b) * 1e3)
        table["kv_append"].append({"M": M, "n_kv_heads": N_KV, "us": statistics.median(times),
                                   "bytes_written": 2 * M * N_KV * 144})
    del flush
    return table


def run_case(args, torch, dev):
    """A few launches of one kernel over distinct buffers whose total exceeds
    L2 (for profilers).  Prints the median device time per launch."""
    import synth
    from bit_weight_streaming_dequant_b200 import q4dec

    L = q4dec.lib()
    M = args.M
    stream = torch.cuda.current_stream()
    sptr = stream.cuda_stream
    times = []
    if args.case == "gemv_batch":
        # the step's batch launch over `layers` layers (5 matrices each, in the
        # step's order and dependencies), on distinct weights per launch
        copies = 2
        sets = [[[synth.device_q4_0_weights(300 + 50 * c + 5 * l + i, N, K, device=dev)
                  for i, (N, K) in enumerate(LAYER_SHAPES)] for l in range(args.layers)]
                for c in range(copies)]
        steps = [DecodeStepGemvOnly(torch, q4dec, synth, dev, sets[c], M) for c in range(copies)]
        for i in range(args.launches):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            steps[i % copies].batch.run()
            b.record(stream)
            torch.cuda.synchronize()
            times.append(a.elapsed_time(b) * 1e3)
        nbytes = sum(gemv_alg_bytes(M, N, K) for N, K in LAYER_SHAPES) * args.layers
        what = f"q4_gemv batch of {args.layers} layers ({5 * args.layers} matrices) M={M}"
    elif args.case == "gemv":
        N, K = (int(v) for v in args.shape.lower().split("x"))
        copies = max(2, -(-3 * L2_BYTES // q4_bytes(N, K)))
        Ws = [synth.device_q4_0_weights(50 + i, N, K, device=dev) for i in range(copies)]
        x = synth.device_bf16_normal(1, (M, K), device=dev)
        y = torch.empty((M, N), dtype=torch.float32, device=dev)
        ws = torch.zeros(max(16, L.q4d_gemv_workspace_bytes(M, N, K)), dtype=torch.uint8,
                         device=dev)
        for i in range(args.launches):
            W = Ws[i % copies]
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            st = L.q4_gemv_ex(W.data_ptr(), x.data_ptr(), y.data_ptr(), M, N, K, sptr,
                              ws.data_ptr(), ws.numel())
            b.record(stream)
            if st:
                raise RuntimeError(f"q4_gemv_ex failed: {st}")
            torch.cuda.synchronize()
            times.append(a.elapsed_time(b) * 1e3)
        nbytes = gemv_alg_bytes(M, N, K)
        what = f"q4_gemv {N}x{K} M={M}"
    else:
        ctx = args.ctx
        row = 272 if args.q8 else 144
        gen = synth.device_q8_0_kv_cache if args.q8 else synth.device_q4_0_kv_cache
        fn = L.q8kv_attn_decode_ex if args.q8 else L.q4kv_attn_decode_ex
        wsfn = L.q8kv_attn_workspace_bytes if args.q8 else L.q4d_attn_workspace_bytes
        copies = max(2, -(-3 * L2_BYTES // (2 * N_KV * ctx * row)))
        caches = [(gen(60 + i, N_KV, ctx, device=dev), gen(80 + i, N_KV, ctx, device=dev))
                  for i in range(copies)]
        Q = synth.device_bf16_normal(2, (M, N_Q, HEAD_DIM), scale=1 / 16, device=dev)
        out = torch.empty((M, N_Q, HEAD_DIM), dtype=torch.float32, device=dev)
        ws = torch.empty(max(16, wsfn(ctx, N_Q, N_KV, HEAD_DIM, M)), dtype=torch.uint8,
                         device=dev)
        for i in range(args.launches):
            Kc, Vc = caches[i % copies]
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            st = fn(Q.data_ptr(), Kc.data_ptr(), Vc.data_ptr(), out.data_ptr(), ctx, N_Q, N_KV,
                    HEAD_DIM, M, ctx, 1.0, sptr, ws.data_ptr(), ws.numel())
            b.record(stream)
            if st:
                raise RuntimeError(f"attention call failed: {st}")
            torch.cuda.synchronize()
            times.append(a.elapsed_time(b) * 1e3)
        nbytes = attn_alg_bytes(M, ctx, row)
        what = f"{'q8' if args.q8 else 'q4'}kv_attn ctx={ctx} M={M}"
    us = statistics.median(times[1:] if len(times) > 1 else times)
    print(json.dumps({"case": what, "us_median": us, "GBps": nbytes / (us * 1e-6) / 1e9,
                      "copies": copies, "launches": args.launches}), flush=True)


class DecodeStepGemvOnly:
    """The step's GEMV batch over the given layers only (no head, no caches):
    a small case of the same launch for profilers."""

    def __init__(self, torch, q4dec, synth, dev, layers, M):
        xs = {K: synth.device_bf16_normal(7 + K, (M, K), device=dev) for K in (HIDDEN, FFN, QKV)}
        names = ("gate", "up", "down", "in", "out")
        ys = {n: torch.empty((M, N), dtype=torch.float32, device=dev)
              for n, (N, K) in zip(names, LAYER_SHAPES)}
        jobs, prev_down = [], -1
        for layer in layers:
            base = len(jobs)
            waits = {3: prev_down, 4: base, 0: base + 1, 1: base + 1, 2: base + 3}
            for i in (3, 4, 0, 1, 2):
                N, K = LAYER_SHAPES[i]
                jobs.append(dict(W=layer[i], x=xs[K], y=ys[names[i]], N=N, K=K, wait_for=waits[i]))
            prev_down = base + 4
        self.keep = (xs, ys)
        self.batch = q4dec.GemvBatch(jobs)


ARGS = None

if __name__ == "__main__":
    main()
