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


def recorded_traffic(kernel):
    """DRAM bytes per launch from a committed ncu capture (the json block of
    profiles/dram_traffic.md), if it was taken on the current kernel sources
    (else None)."""
    path = os.path.join(ROOT, "profiles", "dram_traffic.md")
    try:
        with open(path) as f:
            text = f.read()
        rec = json.loads(text.split("```json", 1)[1].split("```", 1)[0])
    except Exception:
        return None
    e = rec.get(kernel)
    if not e or e.get("source_hash") != kernel_source_hash():
        return None
    return e.get("bytes_per_launch")


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
            "gemv_launch": "q4_gemv_ex2 with Q4D_GEMV_WEIGHT_PREFETCH",
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
    ap.add_argument("--case", default="step", choices=["step", "gemv", "attn"],
                    help="gemv/attn: a few launches of one kernel (small case for profilers)")
    ap.add_argument("--shape", default="17408x5120", help="--case gemv: NxK")
    ap.add_argument("--ctx", type=int, default=65536, help="--case attn: ctx_len")
    ap.add_argument("--launches", type=int, default=8, help="--case gemv/attn: launches")
    ap.add_argument("--q8", action="store_true", help="--case attn: the Q8_0 K/V cache")
    args = ap.parse_args()
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
    # per-step inputs and outputs
    xs = {K: synth.device_bf16_normal(7 + K, (M, K), device=dev) for K in (HIDDEN, FFN, QKV)}
    ys = {N: torch.empty((M, N), dtype=torch.float32, device=dev)
          for N in (FFN, HIDDEN, QKV, HEAD_N)}
    Qs = [synth.device_bf16_normal(2200 + l, (M, N_Q, HEAD_DIM), scale=1 / 16, device=dev)
          for l in range(ATTN_LAYERS)]
    outs = [torch.empty((M, N_Q, HEAD_DIM), dtype=torch.float32, device=dev)
            for _ in range(ATTN_LAYERS)]
    L = q4dec.lib()
    gws = max([L.q4d_gemv_workspace_bytes(M, N, K) for N, K in LAYER_SHAPES + [(HEAD_N, HIDDEN)]])
    aws = L.q4d_attn_workspace_bytes(CTX, N_Q, N_KV, HEAD_DIM, M)
    ws = torch.empty(max(gws, aws, 16), dtype=torch.uint8, device=dev)
    torch.cuda.synchronize()
    gen_s = time.time() - gen_t0

    stream = torch.cuda.current_stream()
    sptr = stream.cuda_stream
    launches = {"n": 0}

    def gemv(W, x, y, N, K):
        # weights are immutable: each call may stream its first stages while
        # the kernel before it finishes (programmatic dependent launch)
        st = L.q4_gemv_ex2(W.data_ptr(), x.data_ptr(), y.data_ptr(), M, N, K,
                           torch.cuda.current_stream().cuda_stream, ws.data_ptr(), ws.numel(),
                           q4dec.GEMV_WEIGHT_PREFETCH)
        if st:
            raise RuntimeError(f"q4_gemv_ex2 failed: {st}")
        launches["n"] += 1 + (1 if L.q4d_gemv_workspace_bytes(M, N, K) else 0)

    def attn(l):
        Kc, Vc = kv[l]
        st = L.q4kv_attn_decode_ex(Qs[l].data_ptr(), Kc.data_ptr(), Vc.data_ptr(),
                                   outs[l].data_ptr(), CTX, N_Q, N_KV, HEAD_DIM, M, CTX,
                                   1.0, torch.cuda.current_stream().cuda_stream,
                                   ws.data_ptr(), ws.numel())
        if st:
            raise RuntimeError(f"q4kv_attn_decode_ex failed: {st}")
        launches["n"] += 2 if aws else 1

    def gemv_stream():
        for l in range(LAYERS):
            for i, (N, K) in enumerate(LAYER_SHAPES):
                gemv(layers[l][i], xs[K], ys[N], N, K)
        gemv(head, xs[HIDDEN], ys[HEAD_N], HEAD_N, HIDDEN)

    def attn_stream():
        for l in range(ATTN_LAYERS):
            attn(l)

    def barrier():
        if world > 1:
            dist.barrier()

    clocks = ClockSampler(local)

    for _ in range(args.warmup):
        gemv_stream()
        attn_stream()
    torch.cuda.synchronize()

    # -------- timed region
    K_ = args.steps
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True),
           torch.cuda.Event(enable_timing=True)) for _ in range(K_)]
    launches["n"] = 0
    barrier()
    torch.cuda.synchronize()
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    clocks.start()
    t_start.record(stream)
    for k in range(K_):
        ev[k][0].record(stream)
        gemv_stream()
        ev[k][1].record(stream)
        attn_stream()
        ev[k][2].record(stream)
    t_end.record(stream)
    torch.cuda.synchronize()
    barrier()
    timed_launches = launches["n"]
    total_ms = t_start.elapsed_time(t_end)
    gemv_ms = sum(e[0].elapsed_time(e[1]) for e in ev)
    attn_ms = sum(e[1].elapsed_time(e[2]) for e in ev)
    clock = clocks.stop()

    total_ms, gemv_ms, attn_ms = reduce_over_ranks([total_ms, gemv_ms, attn_ms], dev, world)

    bytes_step = step_bytes(M)
    value = job_tbps(bytes_step, K_, world, total_ms)
    peak_gbs, peak_kind = peaks()
    n_gemv = LAYERS * len(LAYER_SHAPES) + 1
    gemv_bytes = sum(gemv_alg_bytes(M, N, K) for N, K in LAYER_SHAPES) * LAYERS + \
        gemv_alg_bytes(M, HEAD_N, HIDDEN)
    per_launch_bytes = gemv_bytes / n_gemv
    per_launch_s = gemv_ms * 1e-3 / (K_ * n_gemv)
    achieved_gbs = per_launch_bytes / per_launch_s / 1e9
    attn_gbs = ATTN_LAYERS * attn_alg_bytes(M, CTX) * K_ / (attn_ms * 1e-3) / 1e9

    # -------- the same step replayed as one CUDA graph (353 kernel nodes; the
    # weight-prefetching GEMVs keep their programmatic dependencies)
    graph = None
    g = None
    try:
        g = torch.cuda.CUDAGraph()
        s_cap = torch.cuda.Stream()
        s_cap.wait_stream(stream)
        with torch.cuda.stream(s_cap):
            gemv_stream()
            attn_stream()
        torch.cuda.synchronize()
        with torch.cuda.graph(g, stream=s_cap):
            gemv_stream()
            attn_stream()
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
        torch.cuda.synchronize()
        g0, g1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        g0.record(stream)
        for _ in range(K_):
            g.replay()
        g1.record(stream)
        torch.cuda.synchronize()
        barrier()
        gms = reduce_over_ranks([g0.elapsed_time(g1) / K_], dev, world)[0]
        graph = {"ms_per_step": gms, "value": job_tbps(bytes_step, 1, world, gms),
                 "unit": "TB/s", "replays": K_}
    else:
        graph = {"error": graph_err or "capture failed on another rank"}
    del g
    torch.cuda.synchronize()

    # -------- end to end through the public API with host buffers
    import torch as _t

    e2e_steps = max(3, min(K_, 10))
    h_x = {K: _t.empty((M, K), dtype=_t.bfloat16, pin_memory=True) for K in xs}
    for K in xs:
        h_x[K].copy_(xs[K])
    h_q = [_t.empty((M, N_Q, HEAD_DIM), dtype=_t.bfloat16, pin_memory=True) for _ in Qs]
    for l in range(ATTN_LAYERS):
        h_q[l].copy_(Qs[l])
    h_y = {N: _t.empty((M, N), dtype=_t.float32, pin_memory=True) for N in ys}
    h_o = [_t.empty((M, N_Q, HEAD_DIM), dtype=_t.float32, pin_memory=True) for _ in outs]
    h2d = d2h = 0

    def e2e_step():
        # the step's inputs (the activation rows of each width, the queries of
        # every attention layer) come from pinned host memory; the step's
        # results (the last output of each GEMV width, the logits, every
        # attention output) go back to it; the kernels are the timed step's
        nonlocal h2d, d2h
        h2d = d2h = 0
        for K in xs:
            xs[K].copy_(h_x[K], non_blocking=True)
            h2d += xs[K].numel() * 2
        for l in range(ATTN_LAYERS):
            Qs[l].copy_(h_q[l], non_blocking=True)
            h2d += Qs[l].numel() * 2
        for l in range(LAYERS):
            for i, (N, K) in enumerate(LAYER_SHAPES):
                gemv(layers[l][i], xs[K], ys[N], N, K)
        gemv(head, xs[HIDDEN], ys[HEAD_N], HEAD_N, HIDDEN)
        for l in range(ATTN_LAYERS):
            attn(l)
        for N in ys:
            h_y[N].copy_(ys[N], non_blocking=True)
            d2h += ys[N].numel() * 4
        for l in range(ATTN_LAYERS):
            h_o[l].copy_(outs[l], non_blocking=True)
            d2h += outs[l].numel() * 4

    e2e_step()
    torch.cuda.synchronize()
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(e2e_steps):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize()
    barrier()
    e2e_ms = reduce_over_ranks([e0.elapsed_time(e1)], dev, world)[0]
    e2e_value = job_tbps(bytes_step, e2e_steps, world, e2e_ms)

    # -------- per-call latencies (cold L2), rank 0
    per_call = None
    if rank == 0 and not args.no_per_call:
        per_call = per_call_table(torch, L, dev, layers, kv, ws, peak_gbs)

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
        "roofline": {"bound": "hbm", "kernel": "q4_gemv_kernel", "achieved": achieved_gbs,
                     "peak": peak_gbs, "peak_source": f"{peak_kind} hbm_gbs", "unit": "GB/s",
                     "frac": achieved_gbs / peak_gbs,
                     "traffic": recorded_traffic("q4_gemv_kernel"),
                     "algorithmic_bytes_per_launch": per_launch_bytes,
                     "launch_us": per_launch_s * 1e6},
        "attention": {"achieved_gbs": attn_gbs, "frac": attn_gbs / peak_gbs,
                      "us_per_layer": attn_ms * 1e3 / (K_ * ATTN_LAYERS)},
        "cpu_baseline": base,
        "e2e": {"value": e2e_value, "unit": "TB/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "steps": e2e_steps},
        "gpu_launches": timed_launches,
        "clocks": clock,
        "graph": graph,
        "per_call": per_call,
        "setup_s": gen_s,
    }
    print(json.dumps(line), flush=True)


def per_call_table(torch, L, dev, layers, kv, ws, peak_gbs, reps=15):
    """Median device time of single calls with L2 flushed before each call."""
    flush = torch.empty(2 * L2_BYTES, dtype=torch.uint8, device=dev)
    need = max([L.q4d_gemv_workspace_bytes(M, N, K) for M in range(1, 6)
                for N, K in LAYER_SHAPES] +
               [L.q4d_attn_workspace_bytes(c, N_Q, N_KV, HEAD_DIM, M) for M in (1, 5)
                for c in (4096, 65536, CTX)] +
               [L.q8kv_attn_workspace_bytes(c, N_Q, N_KV, HEAD_DIM, M) for M in (1, 5)
                for c in (65536, CTX)] + [16])
    ws = torch.empty(need, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()
    sptr = stream.cuda_stream
    table = {"gemv": [], "attn": [], "l2": "flushed before every call (256 MB write)"}
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
                                  ws.data_ptr(), ws.numel())
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
    if args.case == "gemv":
        N, K = (int(v) for v in args.shape.lower().split("x"))
        copies = max(2, -(-3 * L2_BYTES // q4_bytes(N, K)))
        Ws = [synth.device_q4_0_weights(50 + i, N, K, device=dev) for i in range(copies)]
        x = synth.device_bf16_normal(1, (M, K), device=dev)
        y = torch.empty((M, N), dtype=torch.float32, device=dev)
        ws = torch.empty(max(16, L.q4d_gemv_workspace_bytes(M, N, K)), dtype=torch.uint8,
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


ARGS = None

if __name__ == "__main__":
    main()
