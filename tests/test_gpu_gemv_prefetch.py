"""GPU tests of q4_gemv_ex2 with Q4D_GEMV_WEIGHT_PREFETCH (programmatic
dependent launch): results equal the plain launch bit for bit, and stream
order still holds for everything except the weight stream -- a call reads its
activations only after the previous kernel finished writing them, and writes
its output only after the previous kernel finished reading that memory."""
import numpy as np
import pytest
import torch

import oracle
import synth
from bit_weight_streaming_dequant_b200 import q4dec
from gpu_util import assert_gemv_close, dev_bf16, dev_bytes

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("M,N,K", [(1, 17408, 5120), (5, 5120, 17408), (3, 6144, 5120),
                                   (2, 64, 65536), (1, 300, 1280)])
def test_prefetch_equals_plain_launch(cuda_ok, M, N, K):
    W = synth.device_q4_0_weights(31, N, K)
    x = synth.device_bf16_normal(32, (M, K))
    a = q4dec.q4_gemv(W, x, N=N, K=K)
    b = q4dec.q4_gemv(W, x, N=N, K=K, weight_prefetch=True)
    torch.cuda.synchronize()
    assert torch.equal(a, b)
    assert q4dec.device_error() == 0


def test_prefetch_chain_reads_before_the_next_call_overwrites(cuda_ok):
    # call 1 reads x from a buffer that call 2 (prefetching) overwrites with
    # its output: call 1 must still see the old x
    M, K, N1, N2 = 1, 5120, 17408, 5120
    W1 = synth.device_q4_0_weights(41, N1, K)
    W2 = synth.device_q4_0_weights(42, N2, 6144)
    x2 = synth.device_bf16_normal(43, (M, 6144))
    shared = torch.empty(M * N2 * 4, dtype=torch.uint8, device="cuda")
    x1_view = shared[: M * K * 2].view(torch.bfloat16).view(M, K)
    y2_view = shared.view(torch.float32).view(M, N2)
    x1_vals = [synth.device_bf16_normal(50 + i, (M, K)) for i in range(3)]
    refs1 = [q4dec.q4_gemv(W1, xv, N=N1, K=K) for xv in x1_vals]
    ref2 = q4dec.q4_gemv(W2, x2, N=N2, K=6144)
    torch.cuda.synchronize()
    y1 = torch.empty((M, N1), dtype=torch.float32, device="cuda")
    for it in range(12):
        x1_view.copy_(x1_vals[it % 3])
        q4dec.q4_gemv(W1, x1_view, y1, N=N1, K=K, weight_prefetch=True)
        q4dec.q4_gemv(W2, x2, y2_view, N=N2, K=6144, weight_prefetch=True)
        torch.cuda.synchronize()
        assert torch.equal(y1, refs1[it % 3]), f"iteration {it}: call 1 saw a later x"
        assert torch.equal(y2_view, ref2)
    assert q4dec.device_error() == 0


def test_prefetch_chain_sees_the_previous_kernels_output(cuda_ok):
    # a decode-like chain: y = gemv(W_i, x); x <- bf16(y[:, :K]) by a torch
    # kernel; every call (prefetching) must read the x the kernel before it wrote
    M, K = 2, 5120
    Ws = [synth.q4_0_weights(60 + i, K, K) for i in range(4)]
    x0 = synth.activations(70, M, K)
    Wd = [dev_bytes(w) for w in Ws]
    x = dev_bf16(x0)
    y = torch.empty((M, K), dtype=torch.float32, device="cuda")
    outs = []
    for i in range(4):
        q4dec.q4_gemv(Wd[i], x, y, N=K, K=K, weight_prefetch=True)
        outs.append(y.clone())
        x.copy_((y / 64).to(torch.bfloat16))
    torch.cuda.synchronize()
    # replay on the oracle with the same bf16 roundings between the steps
    xb = x0
    for i in range(4):
        ref, S = oracle.gemv(Ws[i], xb, M, K, K)
        assert_gemv_close(outs[i], ref, S, f"chain step {i}")
        xb = (outs[i].cpu() / 64).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
