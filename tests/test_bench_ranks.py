"""The multi-rank side of bench.py on the CPU: two gloo ranks agree on the
slowest rank's durations (max) and on a shared success flag (min), the
whole-job throughput counts every rank's bytes over the slowest rank's time,
and the reference arm prints one line from rank 0 only."""
import json
import os
import socket
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, queue):
    import torch.distributed as dist

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        mx = bench.reduce_over_ranks([1.0 + rank, 10.0 - rank, 3.0], "cpu", world)
        mn = bench.reduce_over_ranks([1.0 if rank == 0 else 0.0], "cpu", world, op="min")
        queue.put((rank, mx, mn))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_reduce_timings():
    import torch.multiprocessing as mp

    ctx = mp.get_context("spawn")
    queue = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, queue)) for r in range(2)]
    for p in procs:
        p.start()
    got = {}
    for _ in procs:
        rank, mx, mn = queue.get(timeout=120)
        got[rank] = (mx, mn)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank in (0, 1):
        assert got[rank][0] == [2.0, 10.0, 3.0]   # element-wise max over the ranks
        assert got[rank][1] == [0.0]              # one rank failed: all see it


def test_single_rank_reduction_is_identity_and_job_throughput():
    assert bench.reduce_over_ranks([4.0, 5.0], "cpu", 1) == [4.0, 5.0]
    # 2 ranks x 3 steps x 1 GB in 1.5 s (the slowest rank) = 4 TB/s
    assert bench.job_tbps(1e9, 3, 2, 1500.0) == pytest.approx(4e-3)


def _reference(rank, world):
    env = dict(os.environ, RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                           "--gpus", str(world), "--steps", "1", "--warmup", "3"],
                          capture_output=True, text=True, timeout=300, env=env, cwd=ROOT)


def test_reference_arm_prints_from_rank_zero_only():
    other = _reference(1, 2)
    assert other.returncode == 0 and other.stdout.strip() == ""
    first = _reference(0, 2)
    assert first.returncode == 0, first.stderr[-2000:]
    lines = [ln for ln in first.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1
    line = json.loads(lines[0])
    assert line["impl"] == "reference" and line["n_gpus"] == 2 and line["steps"] == 1
    for key in ("metric", "value", "unit", "higher_is_better", "cpu_baseline", "e2e", "config"):
        assert key in line
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["value"] > 0


def test_algorithmic_bytes_of_the_step():
    # Q4_0: 18 bytes per 32 weights; x bf16 in, y fp32 out per matrix; K and V
    # super-blocks (144 B) per token and KV head, bf16 queries, fp32 outputs
    hidden, ffn, qkv, head_n = 5120, 17408, 6144, 151936
    layer = [(ffn, hidden), (ffn, hidden), (hidden, ffn), (qkv, hidden), (hidden, qkv)]
    for M in (1, 5):
        mats = layer * 64 + [(head_n, hidden)]
        gemv = sum(N * K // 32 * 18 + 2 * M * K + 4 * M * N for N, K in mats)
        attn = 16 * (2 * 4 * 262144 * 144 + M * 24 * 256 * 6)
        assert bench.gemv_step_bytes(M) == gemv
        assert bench.step_bytes(M) == gemv + attn
    assert bench.gemv_step_bytes(1) == 12347133440      # the 12.35 GB quoted for M = 1
    assert bench.gemv_step_bytes(5) == 12421957120
    assert bench.attn_alg_bytes(1, 262144) == 302026752
    assert bench.step_bytes(1) == 17179561472


def test_recorded_traffic_follows_the_source_hash(monkeypatch):
    rec = json.load(open(os.path.join(ROOT, "profiles", "dram_traffic.json")))
    monkeypatch.setattr(bench, "kernel_source_hash", lambda: rec["source_hash"])
    got = bench.recorded_traffic("q4_gemv_kernel", 1)
    assert got == rec["step"]["q4_gemv_kernel"]["M1"]["bytes_per_launch"]
    monkeypatch.setattr(bench, "kernel_source_hash", lambda: "0" * 16)
    assert bench.recorded_traffic("q4_gemv_kernel", 1) is None


def test_kernel_source_hash_covers_the_kernels_but_not_the_self_tests():
    import hashlib
    csrc = os.path.join(ROOT, "bit_weight_streaming_dequant_b200", "csrc")
    names = sorted(os.listdir(csrc))
    assert "q4_gemv.cuh" in names and "q4d_selftest.cu" in names

    def digest(skip):
        h = hashlib.sha256()
        for n in names:
            if n not in skip:
                h.update(n.encode() + open(os.path.join(csrc, n), "rb").read())
        return h.hexdigest()[:16]

    assert bench.kernel_source_hash() == digest({"q4d_selftest.cu"})
    assert bench.kernel_source_hash() != digest(set())
