"""GPU parity of q8kv_attn_decode_ex (the Q8_0 K/V cache, through the C ABI)
against the fp64 oracle; tolerance 3e-3 absolute on outputs, as for the Q4
cache."""
import numpy as np
import pytest
import torch

import oracle
import synth
from bit_weight_streaming_dequant_b200 import q4dec
from gpu_util import assert_attn_close, dev_bf16, dev_bytes, host_bf16_bits, host_bytes

pytestmark = pytest.mark.gpu


def _case(seed, ctx, n_q, n_kv, M, cap=None):
    cap = ctx if cap is None else cap
    return (synth.queries(seed + 2, M, n_q), synth.q8_0_kv_cache(seed, n_kv, cap),
            synth.q8_0_kv_cache(seed + 1, n_kv, cap))


def _gpu(Q, K, V, ctx, n_q, n_kv, M, **kw):
    out = q4dec.q8kv_attn_decode(dev_bf16(Q.reshape(M, n_q, 256)), dev_bytes(K), dev_bytes(V),
                                 ctx_len=ctx, n_kv_heads=n_kv, **kw)
    torch.cuda.synchronize()
    return out


# ragged tails, single-tile and multi-split contexts, 1..5 draft rows, GQA
# groups of 1..48 heads (up to 8 row groups)
CASES = [(1, 4, 1, 1), (2, 24, 4, 2), (5, 24, 4, 5), (63, 6, 2, 3), (128, 24, 4, 1),
         (129, 24, 4, 5), (200, 8, 1, 4), (1000, 24, 4, 5), (4097, 24, 4, 1), (300, 64, 4, 5),
         (777, 48, 1, 5), (2500, 24, 4, 3)]


@pytest.mark.parametrize("ctx,n_q,n_kv,M", CASES)
def test_q8_shapes_against_oracle(cuda_ok, ctx, n_q, n_kv, M):
    Q, K, V = _case(ctx + n_q, ctx, n_q, n_kv, M)
    ref = oracle.attn_decode(Q, K, V, ctx, n_q, n_kv, 256, M, fmt="q8_0")
    assert_attn_close(_gpu(Q, K, V, ctx, n_q, n_kv, M), ref, f"q8 ctx={ctx} {n_q}/{n_kv} M={M}")
    assert q4dec.device_error() == 0


@pytest.mark.parametrize("ctx", [65536, 262144])
@pytest.mark.parametrize("M", [1, 5])
def test_q8_long_context(cuda_ok, ctx, M):
    n_q, n_kv = 24, 4
    K = synth.device_q8_0_kv_cache(3000 + ctx, n_kv, ctx)
    V = synth.device_q8_0_kv_cache(3100 + ctx, n_kv, ctx)
    Q = synth.device_bf16_normal(3200 + M, (M, n_q, 256), scale=1.0 / 16)
    out = q4dec.q8kv_attn_decode(Q, K, V, ctx_len=ctx, n_kv_heads=n_kv)
    torch.cuda.synchronize()
    ref = oracle.attn_decode(host_bf16_bits(Q), host_bytes(K), host_bytes(V), ctx, n_q, n_kv,
                             256, M, fmt="q8_0")
    assert_attn_close(out, ref, f"q8 ctx={ctx} M={M}")
    del K, V


def test_q8_stride_and_softmax_scale(cuda_ok):
    ctx, cap, n_q, n_kv, M = 700, 1024, 24, 4, 3
    Q, K, V = _case(41, ctx, n_q, n_kv, M, cap=cap)
    ref = oracle.attn_decode(Q, K, V, ctx, n_q, n_kv, 256, M, kv_stride=cap, scale=1.7,
                             fmt="q8_0")
    out = _gpu(Q, K, V, ctx, n_q, n_kv, M, kv_stride_tokens=cap, softmax_scale=1.7)
    assert_attn_close(out, ref, "q8 stride/scale")


def test_q8_extreme_codes_and_scales(cuda_ok):
    # codes -128 and 127 in every block of K, K scales up to 4 (values up to
    # 512 in magnitude: still finite in fp16); V at the unit scale of the
    # tolerance (|v| <= 2)
    ctx, n_q, n_kv, M = 300, 24, 4, 5
    rng = np.random.default_rng(7)
    rows = n_kv * ctx
    q = rng.integers(-128, 128, size=(rows, 256), dtype=np.int64)
    q[:, ::32], q[:, 1::32] = -128, 127
    d = rng.uniform(0.5, 4.0, size=(rows, 8)).astype(np.float16)
    K = synth.pack_q8_superblocks(q.astype(np.int8), d.view(np.uint16))
    Vq = rng.integers(-128, 128, size=(rows, 256), dtype=np.int64).astype(np.int8)
    dv = rng.uniform(1 / 256, 1 / 64, size=(rows, 8)).astype(np.float16)
    V = synth.pack_q8_superblocks(Vq, dv.view(np.uint16))
    Q = synth.bf16_normal(8, (M, n_q, 256), scale=1.0 / 4096)
    ref = oracle.attn_decode(Q, K, V, ctx, n_q, n_kv, 256, M, fmt="q8_0")
    assert_attn_close(_gpu(Q, K, V, ctx, n_q, n_kv, M), ref, "q8 extremes")


def test_q8_causal_rows_ignore_later_tokens(cuda_ok):
    ctx, n_q, n_kv, M = 517, 24, 4, 5
    Q, K, V = _case(71, ctx, n_q, n_kv, M)
    base = _gpu(Q, K, V, ctx, n_q, n_kv, M)
    K2 = K.copy().reshape(n_kv, ctx, 272)
    V2 = V.copy().reshape(n_kv, ctx, 272)
    K2[:, ctx - 1, :256] ^= 0x5A
    V2[:, ctx - 1, :256] ^= 0xA5
    pert = _gpu(Q, K2.reshape(-1), V2.reshape(-1), ctx, n_q, n_kv, M)
    assert torch.equal(pert[: M - 1], base[: M - 1])
    assert not torch.allclose(pert[M - 1], base[M - 1])


def test_q8_single_token_is_the_value_row(cuda_ok):
    # one visible token: softmax weight 1, out = fp16(d * q) of the V row
    # (exactly representable here: d a power of two, |q| <= 127)
    n_q, n_kv = 4, 1
    rng = np.random.default_rng(9)
    q = rng.integers(-127, 128, size=(1, 256)).astype(np.int8)
    V = synth.pack_q8_superblocks(q, np.full((1, 8), 0x3400, dtype=np.uint16))  # d = 0.25
    K = synth.q8_0_kv_cache(10, n_kv, 1)
    Q = synth.queries(11, 1, n_q)
    out = _gpu(Q, K, V, 1, n_q, n_kv, 1).cpu().numpy()
    for h in range(n_q):
        assert np.array_equal(out[0, h], 0.25 * q[0].astype(np.float32))


def test_q8_matches_q4_on_the_same_values(cuda_ok):
    # a Q4 cache rewritten exactly in the 8-bit layout: both kernels within
    # the bound of the same oracle output
    ctx, n_q, n_kv, M = 900, 24, 4, 2
    K4, V4 = synth.q4_0_kv_cache(81, n_kv, ctx), synth.q4_0_kv_cache(82, n_kv, ctx)
    Q = synth.queries(83, M, n_q)

    def as_q8(buf):
        raw = buf.reshape(-1, 144)
        out = np.zeros((raw.shape[0], 272), dtype=np.uint8)
        for b in range(8):
            nib = raw[:, 16 * b: 16 * b + 16]
            out[:, 32 * b: 32 * b + 16] = ((nib & 15).astype(np.int16) - 8).astype(np.int8).view(np.uint8)
            out[:, 32 * b + 16: 32 * b + 32] = ((nib >> 4).astype(np.int16) - 8).astype(np.int8).view(np.uint8)
        out[:, 256:] = raw[:, 128:]
        return out.reshape(-1)

    ref = oracle.attn_decode(Q, K4, V4, ctx, n_q, n_kv, 256, M)
    o4 = q4dec.q4kv_attn_decode(dev_bf16(Q.reshape(M, n_q, 256)), dev_bytes(K4), dev_bytes(V4),
                                ctx_len=ctx, n_kv_heads=n_kv)
    o8 = _gpu(Q, as_q8(K4), as_q8(V4), ctx, n_q, n_kv, M)
    assert_attn_close(o4, ref, "q4")
    assert_attn_close(o8, ref, "q8 of the q4 values")


def test_q8_repeat_calls_bitwise_identical(cuda_ok):
    ctx, n_q, n_kv, M = 65536, 24, 4, 5
    K = synth.device_q8_0_kv_cache(91, n_kv, ctx)
    V = synth.device_q8_0_kv_cache(92, n_kv, ctx)
    Q = synth.device_bf16_normal(93, (M, n_q, 256), scale=1.0 / 16)
    a = q4dec.q8kv_attn_decode(Q, K, V, ctx_len=ctx, n_kv_heads=n_kv)
    b = q4dec.q8kv_attn_decode(Q, K, V, ctx_len=ctx, n_kv_heads=n_kv)
    torch.cuda.synchronize()
    assert torch.equal(a, b)
    assert q4dec.device_error() == 0
