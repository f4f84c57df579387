"""GPU parity of q4kv_attn_decode (through the C ABI) against the fp64
oracle; tolerance 3e-3 absolute on outputs (V has unit variance)."""
import numpy as np
import pytest
import torch

import oracle
import synth
from bit_weight_streaming_dequant_b200 import q4dec
from gpu_util import assert_attn_close, dev_bf16, dev_bytes, host_bf16_bits, host_bytes

pytestmark = pytest.mark.gpu


def _case(seed, ctx, n_q, n_kv, M):
    return (synth.queries(seed + 2, M, n_q), synth.q4_0_kv_cache(seed, n_kv, ctx),
            synth.q4_0_kv_cache(seed + 1, n_kv, ctx))


def _gpu(Q, K, V, ctx, n_q, n_kv, M, **kw):
    out = q4dec.q4kv_attn_decode(dev_bf16(Q.reshape(M, n_q, 256)), dev_bytes(K), dev_bytes(V),
                                 ctx_len=ctx, n_kv_heads=n_kv, **kw)
    torch.cuda.synchronize()
    return out


CASES = [(1, 4, 1, 1), (2, 24, 4, 2), (5, 24, 4, 5), (63, 6, 2, 3), (64, 24, 4, 1),
         (65, 24, 4, 5), (200, 8, 1, 4), (1000, 24, 4, 5), (4097, 24, 4, 1), (300, 64, 4, 5),
         (129, 4, 4, 2), (777, 48, 1, 5)]


@pytest.mark.parametrize("ctx,n_q,n_kv,M", CASES)
def test_shapes_against_oracle(cuda_ok, ctx, n_q, n_kv, M):
    Q, K, V = _case(ctx + n_q, ctx, n_q, n_kv, M)
    ref = oracle.attn_decode(Q, K, V, ctx, n_q, n_kv, 256, M)
    assert_attn_close(_gpu(Q, K, V, ctx, n_q, n_kv, M), ref, f"ctx={ctx} {n_q}/{n_kv} M={M}")


@pytest.mark.parametrize("M", [1, 5])
def test_config4_ctx4096_all_layers(cuda_ok, M):
    ctx, n_q, n_kv = 4096, 24, 4
    for layer in range(16):
        seed = 2000 + layer
        K = synth.q4_0_kv_cache(seed, n_kv, ctx)
        V = synth.q4_0_kv_cache(seed + 100, n_kv, ctx)
        Q = synth.queries(seed + 200 + M, M, n_q)
        ref = oracle.attn_decode(Q, K, V, ctx, n_q, n_kv, 256, M)
        assert_attn_close(_gpu(Q, K, V, ctx, n_q, n_kv, M), ref, f"layer {layer} M={M}")


@pytest.mark.parametrize("ctx", [65536, 262144])
@pytest.mark.parametrize("M", [1, 5])
def test_config4_long_context_sampled_layers(cuda_ok, ctx, M):
    n_q, n_kv = 24, 4
    for layer in (0, 15):
        seed = 2000 + layer
        K = synth.device_q4_0_kv_cache(seed, n_kv, ctx)
        V = synth.device_q4_0_kv_cache(seed + 100, n_kv, ctx)
        Q = synth.device_bf16_normal(seed + 200 + M, (M, n_q, 256), scale=1.0 / 16)
        out = q4dec.q4kv_attn_decode(Q, K, V, ctx_len=ctx, n_kv_heads=n_kv)
        torch.cuda.synchronize()
        ref = oracle.attn_decode(host_bf16_bits(Q), host_bytes(K), host_bytes(V), ctx, n_q,
                                 n_kv, 256, M)
        assert_attn_close(out, ref, f"ctx={ctx} layer {layer} M={M}")
        del K, V


def test_kv_stride_and_softmax_scale(cuda_ok):
    ctx, cap, n_q, n_kv, M = 700, 1024, 24, 4, 3
    K = synth.q4_0_kv_cache(41, n_kv, cap)
    V = synth.q4_0_kv_cache(42, n_kv, cap)
    Q = synth.queries(43, M, n_q)
    ref = oracle.attn_decode(Q, K, V, ctx, n_q, n_kv, 256, M, kv_stride=cap, scale=1.7)
    out = _gpu(Q, K, V, ctx, n_q, n_kv, M, kv_stride_tokens=cap, softmax_scale=1.7)
    assert_attn_close(out, ref, "stride/scale")


def test_uniform_keys_give_mean_of_visible_values(cuda_ok):
    ctx, n_q, n_kv, M = 333, 24, 4, 5
    kq = np.full((n_kv * ctx, 256), 8, dtype=np.uint8)
    K = synth.from_parts(kq, np.ones((n_kv * ctx, 8), dtype=np.float32))
    V = synth.q4_0_kv_cache(51, n_kv, ctx)
    Q = synth.queries(52, M, n_q)
    out = _gpu(Q, K, V, ctx, n_q, n_kv, M).cpu().numpy()
    Vh = oracle.dequant(V, n_kv * ctx, 256).reshape(n_kv, ctx, 256)
    for m in range(M):
        vis = Vh[:, : ctx - M + m + 1]
        mean = vis.mean(axis=1)                                 # [n_kv][256]
        # the kernels may round each product d*(q - 8) once to fp16 before the
        # P.V contraction: at most 2^-11 of |v| per term, so of the mean |v|
        bound = 2.0 ** -11 * np.abs(vis).mean(axis=1) + 1e-6
        err = np.abs(out[m] - np.repeat(mean, n_q // n_kv, axis=0))
        assert (err <= np.repeat(bound, n_q // n_kv, axis=0)).all(), err.max()


def test_constant_values_and_single_token(cuda_ok):
    ctx, n_q, n_kv, M = 1000, 24, 4, 5
    vq = np.full((n_kv * ctx, 256), 11, dtype=np.uint8)
    V = synth.from_parts(vq, np.full((n_kv * ctx, 8), 0.25, dtype=np.float32))
    Q, K, _ = _case(61, ctx, n_q, n_kv, M)
    out = _gpu(Q, K, V, ctx, n_q, n_kv, M)
    assert torch.allclose(out, torch.full_like(out, 0.75), rtol=0, atol=1e-6)
    Q1, K1, V1 = _case(62, 1, 4, 1, 1)
    out1 = _gpu(Q1, K1, V1, 1, 4, 1, 1).cpu().numpy()
    assert np.array_equal(out1[0], np.repeat(oracle.dequant(V1, 1, 256), 4, axis=0).astype(np.float32))


def test_causal_rows_ignore_later_tokens(cuda_ok):
    ctx, n_q, n_kv, M = 517, 24, 4, 5
    Q, K, V = _case(71, ctx, n_q, n_kv, M)
    base = _gpu(Q, K, V, ctx, n_q, n_kv, M)
    K2 = K.copy().reshape(n_kv, ctx, 144)
    V2 = V.copy().reshape(n_kv, ctx, 144)
    K2[:, ctx - 1, :128] ^= 0x5A
    V2[:, ctx - 1, :128] ^= 0xA5
    pert = _gpu(Q, K2.reshape(-1), V2.reshape(-1), ctx, n_q, n_kv, M)
    assert torch.equal(pert[: M - 1], base[: M - 1])
    assert not torch.allclose(pert[M - 1], base[M - 1])


def test_repeat_calls_bitwise_identical(cuda_ok):
    ctx, n_q, n_kv, M = 65536, 24, 4, 5
    K = synth.device_q4_0_kv_cache(81, n_kv, ctx)
    V = synth.device_q4_0_kv_cache(82, n_kv, ctx)
    Q = synth.device_bf16_normal(83, (M, n_q, 256), scale=1.0 / 16)
    a = q4dec.q4kv_attn_decode(Q, K, V, ctx_len=ctx, n_kv_heads=n_kv)
    b = q4dec.q4kv_attn_decode(Q, K, V, ctx_len=ctx, n_kv_heads=n_kv)
    torch.cuda.synchronize()
    assert torch.equal(a, b)
    assert q4dec.device_error() == 0


def test_plain_entry_point(cuda_ok):
    ctx, n_q, n_kv, M = 20000, 24, 4, 2
    Q, K, V = _case(91, ctx, n_q, n_kv, M)
    ref = oracle.attn_decode(Q, K, V, ctx, n_q, n_kv, 256, M)
    Qd, Kd, Vd = dev_bf16(Q.reshape(M, n_q, 256)), dev_bytes(K), dev_bytes(V)
    out = torch.empty((M, n_q, 256), device="cuda")
    torch.cuda.synchronize()
    st = q4dec.lib().q4kv_attn_decode(Qd.data_ptr(), Kd.data_ptr(), Vd.data_ptr(),
                                      out.data_ptr(), ctx, n_q, n_kv, 256, M)
    torch.cuda.synchronize()
    assert st == 0
    assert_attn_close(out, ref, "plain entry")
