"""GPU tests of the multi-matrix GEMV launch (q4d_gemv_batch_prepare +
q4_gemv_batch_ex, through the C ABI via the binding's GemvBatch).

Every job of a batch must give, bit for bit, what the single-GEMV entry point
gives (same partition, same summation order); dependent jobs must read their
input only after the job they wait for has written it; the completion and
completion counters and partial-slot entries must leave the descriptor and
the workspace ready for the next launch (repeated launches, CUDA-graph
replays): the counters back at zero, the workspace zero-filled again."""
import numpy as np
import pytest
import torch

import oracle
import synth
from bit_weight_streaming_dequant_b200 import q4dec
from gpu_util import assert_gemv_close, dev_bf16, dev_bytes

pytestmark = pytest.mark.gpu


def _weights(seed, N, K, device_gen=False):
    if device_gen:
        return synth.device_q4_0_weights(seed, N, K)
    return dev_bytes(synth.q4_0_weights(seed, N, K))


def test_independent_jobs_equal_single_calls(cuda_ok):
    M = 3
    shapes = [(512, 1024), (6144, 5120), (5120, 6144), (37, 4352), (17408, 5120), (5120, 17408)]
    jobs, refs = [], []
    for i, (N, K) in enumerate(shapes):
        W = _weights(700 + i, N, K, device_gen=N * K > 1 << 24)
        x = dev_bf16(synth.activations(710 + i, M, K))
        y = torch.full((M, N), float("nan"), device="cuda")
        jobs.append(dict(W=W, x=x, y=y, N=N, K=K))
        refs.append(q4dec.q4_gemv(W, x, N=N, K=K))
    b = q4dec.GemvBatch(jobs)
    for launch in range(3):
        for j in jobs:
            j["y"].fill_(float("nan"))
        b.run()
        torch.cuda.synchronize()
        for i, (j, r) in enumerate(zip(jobs, refs)):
            assert torch.equal(j["y"], r), f"launch {launch} job {i} {shapes[i]}"
    assert q4dec.device_error() == 0


def test_small_jobs_against_the_oracle(cuda_ok):
    M = 2
    shapes = [(1, 256), (3, 512), (300, 1280), (64, 65536), (129, 2048)]
    jobs, ref = [], []
    for i, (N, K) in enumerate(shapes):
        Wnp, xnp = synth.q4_0_weights(720 + i, N, K), synth.activations(730 + i, M, K)
        jobs.append(dict(W=dev_bytes(Wnp), x=dev_bf16(xnp),
                         y=torch.empty((M, N), device="cuda"), N=N, K=K,
                         wait_for=-1 if i == 0 else i - 1))
        ref.append(oracle.gemv(Wnp, xnp, M, N, K))
    q4dec.GemvBatch(jobs).run()
    torch.cuda.synchronize()
    for i, (j, (y_ref, S)) in enumerate(zip(jobs, ref)):
        assert_gemv_close(j["y"], y_ref, S, f"job {i} {shapes[i]}")


def test_dependent_chain_reads_the_previous_output(cuda_ok):
    # job k reads job k-1's bf16 output as its x: a chain 5120 -> 6144 ->
    # 5120 -> 17408 -> 5120 with every link waiting for the one before
    M = 2
    dims = [5120, 6144, 5120, 17408, 5120]
    Ws = [_weights(740 + k, dims[k + 1], dims[k], device_gen=True) for k in range(len(dims) - 1)]
    x0 = dev_bf16(synth.activations(750, M, dims[0]))
    outs = [torch.empty((M, dims[k + 1]), dtype=torch.bfloat16, device="cuda")
            for k in range(len(Ws))]
    jobs = [dict(W=Ws[k], x=x0 if k == 0 else outs[k - 1], y=outs[k], N=dims[k + 1],
                 K=dims[k], wait_for=k - 1) for k in range(len(Ws))]
    b = q4dec.GemvBatch(jobs)
    # reference: the same chain as single calls, one after another
    ref, x = [], x0
    for k in range(len(Ws)):
        ref.append(q4dec.q4_gemv(Ws[k], x, N=dims[k + 1], K=dims[k], out_dtype=torch.bfloat16))
        x = ref[-1]
    torch.cuda.synchronize()
    for launch in range(3):
        for o in outs:
            o.fill_(float("nan"))
        b.run()
        torch.cuda.synchronize()
        for k in range(len(Ws)):
            assert torch.equal(outs[k], ref[k]), f"launch {launch} link {k}"
    assert q4dec.device_error() == 0


def test_swiglu_job_and_workspace_left_zero(cuda_ok):
    M = 5
    N, K = 1024, 5120
    Wgu = _weights(760, 2 * N, K)
    W2 = _weights(761, 6144, 5120)
    x = dev_bf16(synth.activations(762, M, K))
    h = torch.empty((M, N), device="cuda")
    y2 = torch.empty((M, 6144), dtype=torch.bfloat16, device="cuda")
    b = q4dec.GemvBatch([dict(W=Wgu, x=x, y=h, N=N, K=K, swiglu=True),
                         dict(W=W2, x=x, y=y2, N=6144, K=5120, wait_for=0)])
    h_ref = q4dec.q4_gemv_swiglu(Wgu, x, N=N, K=K)
    y2_ref = q4dec.q4_gemv(W2, x, N=6144, K=5120, out_dtype=torch.bfloat16)
    assert b.workspace_bytes > 0            # both jobs share row blocks across CTAs
    for launch in range(3):
        h.fill_(float("nan"))
        b.run()
        torch.cuda.synchronize()
        assert torch.equal(h, h_ref) and torch.equal(y2, y2_ref), f"launch {launch}"
        # every partial-slot entry written was read and cleared
        assert int(torch.count_nonzero(b.workspace)) == 0, f"launch {launch}"
    assert q4dec.device_error() == 0


def test_batch_replays_as_a_cuda_graph(cuda_ok):
    M = 1
    shapes = [(6144, 5120), (5120, 6144), (17408, 5120)]
    jobs = []
    for i, (N, K) in enumerate(shapes):
        jobs.append(dict(W=_weights(770 + i, N, K, device_gen=True),
                         x=dev_bf16(synth.activations(780 + i, M, K)),
                         y=torch.empty((M, N), device="cuda"), N=N, K=K,
                         wait_for=i - 1))
    b = q4dec.GemvBatch(jobs)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        b.run(weight_prefetch=True)
    torch.cuda.synchronize()
    eager = [j["y"].clone() for j in jobs]
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        b.run(weight_prefetch=True)
    for _ in range(3):
        for j in jobs:
            j["y"].fill_(float("nan"))
        g.replay()
        torch.cuda.synchronize()
        for i, j in enumerate(jobs):
            assert torch.equal(j["y"], eager[i]), f"replay job {i}"
    del g
    assert q4dec.device_error() == 0


def test_wait_for_orders_a_write_after_an_earlier_jobs_read(cuda_ok):
    # job 0 reads x0; job 2 (no data dependence on job 0) writes its output
    # into x0's memory and waits for job 0, so job 0 must still see the old x0;
    # job 1 is independent and runs in between; job 3 waits for job 1, two jobs
    # back
    M, K = 2, 5120
    x0 = dev_bf16(synth.activations(800, M, K))
    x0_copy = x0.clone()
    x1 = dev_bf16(synth.activations(801, M, K))
    W = [_weights(810 + i, 5120, K, device_gen=True) for i in range(4)]
    y = [torch.empty((M, 5120), dtype=torch.bfloat16, device="cuda") for _ in range(4)]
    jobs = [dict(W=W[0], x=x0, y=y[0], N=5120, K=K),
            dict(W=W[1], x=x1, y=y[1], N=5120, K=K),
            dict(W=W[2], x=x1, y=x0, N=5120, K=K, wait_for=0),   # overwrites job 0's input
            dict(W=W[3], x=y[1], y=y[3], N=5120, K=K, wait_for=1)]
    ref0 = q4dec.q4_gemv(W[0], x0_copy, N=5120, K=K, out_dtype=torch.bfloat16)
    ref1 = q4dec.q4_gemv(W[1], x1, N=5120, K=K, out_dtype=torch.bfloat16)
    ref2 = q4dec.q4_gemv(W[2], x1, N=5120, K=K, out_dtype=torch.bfloat16)
    ref3 = q4dec.q4_gemv(W[3], ref1, N=5120, K=K, out_dtype=torch.bfloat16)
    b = q4dec.GemvBatch(jobs)
    for launch in range(3):
        x0.copy_(x0_copy)
        for t in y:
            t.fill_(float("nan"))
        torch.cuda.synchronize()
        b.run()
        torch.cuda.synchronize()
        assert torch.equal(y[0], ref0), f"launch {launch}: job 0 saw the later x0"
        assert torch.equal(y[1], ref1) and torch.equal(x0, ref2) and torch.equal(y[3], ref3), launch
        assert int(torch.count_nonzero(b.workspace)) == 0
    assert q4dec.device_error() == 0


def test_ffn_chain_in_one_launch(cuda_ok):
    # the feed-forward block as a batch: fused gate / up + SwiGLU writing bf16 h,
    # then the down projection reading h (waits for it); beside them a fused
    # job whose 2N = 2000 rows end in a ragged row block of gate / up pairs
    for M in (1, 4):
        hid, ffn = 1024, 2048
        Wgu = _weights(830, 2 * ffn, hid)
        Wdn = _weights(831, hid, ffn)
        Wr = _weights(832, 2 * 1000, hid)
        x = dev_bf16(synth.activations(833 + M, M, hid))
        h = torch.empty((M, ffn), dtype=torch.bfloat16, device="cuda")
        y = torch.empty((M, hid), device="cuda")
        hr = torch.empty((M, 1000), device="cuda")
        b = q4dec.GemvBatch([dict(W=Wgu, x=x, y=h, N=ffn, K=hid, swiglu=True),
                             dict(W=Wr, x=x, y=hr, N=1000, K=hid, swiglu=True),
                             dict(W=Wdn, x=h, y=y, N=hid, K=ffn, wait_for=0)])
        h_ref = q4dec.q4_gemv_swiglu(Wgu, x, N=ffn, K=hid, out_dtype=torch.bfloat16)
        hr_ref = q4dec.q4_gemv_swiglu(Wr, x, N=1000, K=hid)
        y_ref = q4dec.q4_gemv(Wdn, h_ref, N=hid, K=ffn)
        for launch in range(2):
            for t in (h, y, hr):
                t.fill_(float("nan"))
            b.run(weight_prefetch=bool(launch))
            torch.cuda.synchronize()
            assert torch.equal(h, h_ref) and torch.equal(hr, hr_ref), (M, launch)
            assert torch.equal(y, y_ref), (M, launch)
            assert int(torch.count_nonzero(b.workspace)) == 0
    # the ragged job against the oracle's SwiGLU bound
    Wr_np = synth.q4_0_weights(840, 2 * 1000, 1024)
    xr_np = synth.activations(841, 2, 1024)
    hr2 = torch.empty((2, 1000), device="cuda")
    q4dec.GemvBatch([dict(W=dev_bytes(Wr_np), x=dev_bf16(xr_np), y=hr2, N=1000, K=1024,
                          swiglu=True)]).run()
    torch.cuda.synchronize()
    h_o, tol = oracle.gemv_swiglu(Wr_np, xr_np, 2, 1000, 1024)
    err = np.abs(hr2.cpu().numpy().astype(np.float64) - h_o)
    assert (err <= tol).all(), float((err / tol).max())
    assert q4dec.device_error() == 0
