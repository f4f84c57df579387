"""GPU parity of q4_gemv (through the C ABI) against the fp64 oracle.

Tolerance: |y_gpu - y_ref| <= 2e-3 * sum_k |w x| + 1e-5 per element; exact
cases (all q = 8, dyadic inputs) must match bit for bit."""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import synth
from bit_weight_streaming_dequant_b200 import q4dec
from gpu_util import assert_gemv_close, dev_bf16, dev_bytes, host_bytes

pytestmark = pytest.mark.gpu

LAYER_SHAPES = [(17408, 5120), (5120, 17408), (6144, 5120), (5120, 6144)]  # (N, K)


def _run(Wnp, xnp, N, K):
    W, x = dev_bytes(Wnp), dev_bf16(xnp)
    y = q4dec.q4_gemv(W, x, N=N, K=K)
    torch.cuda.synchronize()
    return y


def test_config0_single_gemv(cuda_ok):
    N, K, M = 512, 1024, 1
    Wnp = synth.q4_0_weights(0, N, K)
    xnp = synth.activations(0, M, K)
    y_ref, S = oracle.gemv(Wnp, xnp, M, N, K)
    assert_gemv_close(_run(Wnp, xnp, N, K), y_ref, S, "config 0")


SMALL = [(1, 256), (3, 512), (37, 4352), (300, 1280), (64, 65536), (7, 32768),
         (149, 512), (1000, 2048), (2, 17408)]


@pytest.mark.parametrize("N,K", SMALL)
@pytest.mark.parametrize("M", [1, 2, 3, 4, 5])
def test_ragged_shapes(cuda_ok, N, K, M):
    Wnp = synth.q4_0_weights(N * 31 + K, N, K)
    xnp = synth.activations(M * 7 + K, M, K)
    y_ref, S = oracle.gemv(Wnp, xnp, M, N, K)
    assert_gemv_close(_run(Wnp, xnp, N, K), y_ref, S, f"N={N} K={K} M={M}")


@pytest.mark.parametrize("shape", range(4))
def test_layer_shapes_m1(cuda_ok, shape):
    N, K = LAYER_SHAPES[shape]
    Wnp = synth.q4_0_weights(1 + shape, N, K)
    xnp = synth.activations(1 + shape, 1, K)
    y_ref, S = oracle.gemv(Wnp, xnp, 1, N, K)
    assert_gemv_close(_run(Wnp, xnp, N, K), y_ref, S, f"layer shape {N}x{K}")


@pytest.mark.parametrize("shape", range(4))
def test_layer_shapes_verify_m2_to_m5(cuda_ok, shape):
    N, K = LAYER_SHAPES[shape]
    Wnp = synth.q4_0_weights(10 + shape, N, K)
    w = oracle.dequant_weights(Wnp, N, K)
    W = dev_bytes(Wnp)
    for M in (2, 3, 4, 5):
        xnp = synth.activations(100 + M, M, K)
        xf = oracle.bf16_bits_to_f64(xnp)
        y_ref, S = xf @ w.T, np.abs(xf) @ np.abs(w).T
        y = q4dec.q4_gemv(W, dev_bf16(xnp), N=N, K=K)
        torch.cuda.synchronize()
        assert_gemv_close(y, y_ref, S, f"{N}x{K} M={M}")


@pytest.mark.parametrize("N,K", [(300, 1280), (64, 65536), (17408, 5120)])
@pytest.mark.parametrize("M", [1, 3, 5])
def test_all_q8_gives_exact_zero(cuda_ok, N, K, M):
    q = np.full((N, K), 8, dtype=np.uint8)
    d = np.abs(np.random.default_rng(N).standard_normal((N, K // 32))).astype(np.float32)
    y = _run(synth.weights_from_parts(q, d), synth.activations(3, M, K), N, K)
    assert torch.count_nonzero(y).item() == 0


@pytest.mark.parametrize("M", [1, 2, 5])
def test_dyadic_inputs_are_bit_exact(cuda_ok, M):
    N, K = 257, 5120
    rng = np.random.default_rng(77 + M)
    q = rng.integers(0, 16, size=(N, K), dtype=np.uint8)
    d = (2.0 ** -rng.integers(0, 6, size=(N, K // 32))).astype(np.float32)
    xi = rng.integers(-3, 4, size=(M, K)).astype(np.float32)
    Wnp, xnp = synth.weights_from_parts(q, d), synth.f32_to_bf16_bits(xi)
    y_ref, _ = oracle.gemv(Wnp, xnp, M, N, K)
    y = _run(Wnp, xnp, N, K).cpu().numpy().astype(np.float64)
    assert np.array_equal(y, y_ref)


def test_repeat_calls_are_bitwise_identical(cuda_ok):
    N, K = 5120, 17408
    W = dev_bytes(synth.q4_0_weights(5, N, K))
    for M in (1, 5):
        x = dev_bf16(synth.activations(6, M, K))
        a = q4dec.q4_gemv(W, x, N=N, K=K)
        b = q4dec.q4_gemv(W, x, N=N, K=K)
        torch.cuda.synchronize()
        assert torch.equal(a, b)


def test_plain_entry_point_and_side_stream(cuda_ok):
    N, K, M = 64, 65536, 2                     # uses split-K (library workspace)
    Wnp, xnp = synth.q4_0_weights(8, N, K), synth.activations(9, M, K)
    y_ref, S = oracle.gemv(Wnp, xnp, M, N, K)
    W, x = dev_bytes(Wnp), dev_bf16(xnp)
    y = torch.full((M, N), float("nan"), device="cuda")
    torch.cuda.synchronize()
    st = q4dec.lib().q4_gemv(W.data_ptr(), x.data_ptr(), y.data_ptr(), M, N, K)
    torch.cuda.synchronize()
    assert st == 0
    assert_gemv_close(y, y_ref, S, "plain entry")
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        y2 = q4dec.q4_gemv(W, x, N=N, K=K)
    s.synchronize()
    assert torch.equal(y, y2)


def test_one_zeroed_workspace_serves_every_shape(cuda_ok):
    # a caller-owned workspace, zero-filled once, is used by calls of several
    # shapes and M (each sharing row blocks across CTAs); after every call all
    # of it is zero again and the results equal calls with fresh workspaces
    L = q4dec.lib()
    shapes = [(64, 65536, 2), (17408, 5120, 1), (5120, 17408, 5), (6144, 5120, 3), (300, 1280, 4)]
    need = max(L.q4d_gemv_workspace_bytes(M, N, K) for N, K, M in shapes)
    ws = torch.zeros(need, dtype=torch.uint8, device="cuda")
    for i, (N, K, M) in enumerate(shapes * 2):
        assert L.q4d_gemv_workspace_bytes(M, N, K) > 0, (N, K, M)
        W = synth.device_q4_0_weights(1100 + i % len(shapes), N, K)
        x = synth.device_bf16_normal(1110 + i % len(shapes), (M, K))
        ref = q4dec.q4_gemv(W, x, N=N, K=K)
        y = q4dec.q4_gemv(W, x, N=N, K=K, workspace=ws, weight_prefetch=bool(i & 1))
        torch.cuda.synchronize()
        assert torch.equal(y, ref), (N, K, M)
        assert int(torch.count_nonzero(ws)) == 0, (N, K, M)
    assert q4dec.device_error() == 0


def test_bad_calls_launch_nothing(cuda_ok):
    N, K = 64, 512
    W = dev_bytes(synth.q4_0_weights(1, N, K))
    x = dev_bf16(synth.activations(1, 1, K))
    y = torch.full((1, N), 7.0, device="cuda")
    L = q4dec.lib()
    assert L.q4_gemv_ex(W.data_ptr(), x.data_ptr(), y.data_ptr(), 6, N, K, None, None, 0) == 2
    assert L.q4_gemv_ex(W.data_ptr() + 1, x.data_ptr(), y.data_ptr(), 1, N, K, None, None, 0) == 3
    # a shape that needs split-K partials but gets no workspace
    need = L.q4d_gemv_workspace_bytes(2, 64, 65536)
    assert need > 0
    assert L.q4_gemv_ex(W.data_ptr(), x.data_ptr(), y.data_ptr(), 2, 64, 65536, None, None, 0) == 4
    torch.cuda.synchronize()
    assert torch.all(y == 7.0)
    assert q4dec.device_error() == 0


def test_output_head_sampled_rows(cuda_ok):
    # 5120 -> 151936 output head generated on the device; rows sampled for
    # the oracle from the same device bytes
    N, K = 151936, 5120
    W = synth.device_q4_0_weights(1063, N, K)
    for M in (1, 5):
        x = synth.device_bf16_normal(1064 + M, (M, K))
        y = q4dec.q4_gemv(W, x, N=N, K=K)
        torch.cuda.synchronize()
        rows = np.sort(np.random.default_rng(M).choice(N, 1024, replace=False))
        rows = np.concatenate([[0, 1, N - 2, N - 1], rows])
        # the sampled rows keep the column-major super-block layout
        idx = torch.from_numpy(rows).cuda()
        Wr = host_bytes(W.view(K // 256, N, 144)[:, idx, :].contiguous().reshape(-1))
        xb = x.cpu().view(torch.int16).numpy().view(np.uint16)
        y_ref, S = oracle.gemv(Wr, xb, M, len(rows), K)
        assert_gemv_close(y[:, torch.from_numpy(rows).cuda()], y_ref, S, f"head M={M}")


@pytest.mark.parametrize("N,K", [(2048, 5120), (300, 1280), (64, 65536), (17408, 5120)])
@pytest.mark.parametrize("M", [3, 4, 5])
def test_verify_rows_equal_single_row_calls_bitwise(cuda_ok, N, K, M):
    # row m of an M-row verification call is the M = 1 call on x[m], bit for
    # bit: the rows are independent columns of the MMAs and every row sees the
    # same blocking, K ranges and summation order -- also across the change of
    # reduction slots (one per consumer warp up to M = 3, one per block index
    # from M = 4: column 0 + column 1 first in both)
    W = dev_bytes(synth.q4_0_weights(600 + N, N, K))
    x = synth.activations(601 + N, M, K)
    yM = q4dec.q4_gemv(W, dev_bf16(x), N=N, K=K)
    for m in range(M):
        y1 = q4dec.q4_gemv(W, dev_bf16(x[m:m + 1]), N=N, K=K)
        torch.cuda.synchronize()
        assert torch.equal(yM[m:m + 1], y1), f"row {m} of M={M}"
