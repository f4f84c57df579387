"""GPU parity of both attention kernels at the edge of the supported value
range: K/V block scales as large as the library accepts (Q4: |d| <= 8188, so
that every d * (q - 8) lies within +-65504; Q8: |d| <= 511.75, every d * q
within +-65504), with the largest magnitude reached exactly on one block.

The cache is the usual N(0,1) synthetic cache with every scale multiplied by
the same power of two 2^k (exact in fp16) and the softmax scale 2^-k, so the
scores are unchanged and the exact output is 2^k times that of the unscaled
cache: every rounding in the kernels is relative, and the 3e-3 bound for
unit-variance values becomes 3e-3 * 2^k.  M = 1 runs the warp-local kernel
for the Q4 cache, M = 5 the tensor-memory kernel; both must stay within that
bound of the fp64 oracle (and so agree with each other)."""
import numpy as np
import pytest
import torch

import oracle
import synth
from bit_weight_streaming_dequant_b200 import q4dec
from gpu_util import ATTN_TOL, dev_bf16, dev_bytes

pytestmark = pytest.mark.gpu

Q4_D_MAX, Q8_D_MAX = 8188.0, 511.75


def _scale_cache(buf, row_bytes, scale_at, ctx, n_kv, d_max, extreme_code):
    """Every fp16 scale times 2^k (k as large as keeps |d| <= d_max), then
    token 0 of head 0, block 0: scale = d_max and its first code the one of
    largest magnitude (so that value is exactly -65504)."""
    rows = np.array(buf, dtype=np.uint8).reshape(n_kv * ctx, row_bytes)
    d = rows[:, scale_at:scale_at + 16].copy().view(np.float16).astype(np.float64)
    k = int(np.floor(np.log2(d_max / np.abs(d).max())))
    scaled = (d * 2.0 ** k).astype(np.float16)
    assert np.array_equal(scaled.astype(np.float64), d * 2.0 ** k)      # exact in fp16
    rows[:, scale_at:scale_at + 16] = scaled.view(np.uint8).reshape(-1, 16)
    rows[0, scale_at:scale_at + 2] = np.array([d_max], dtype=np.float16).view(np.uint8)
    rows[0, 0] = extreme_code(rows[0, 0])
    return rows.reshape(-1), k


@pytest.mark.parametrize("fmt", ["q4_0", "q8_0"])
@pytest.mark.parametrize("ctx", [300, 4097])
def test_largest_supported_scales(cuda_ok, fmt, ctx):
    n_q, n_kv = 24, 4
    if fmt == "q4_0":
        K0, V0 = synth.q4_0_kv_cache(900 + ctx, n_kv, ctx), synth.q4_0_kv_cache(901 + ctx, n_kv, ctx)
        args = (144, 128, ctx, n_kv, Q4_D_MAX, lambda b: b & 0xF0)      # low nibble q = 0
        call = q4dec.q4kv_attn_decode
    else:
        K0, V0 = synth.q8_0_kv_cache(900 + ctx, n_kv, ctx), synth.q8_0_kv_cache(901 + ctx, n_kv, ctx)
        args = (272, 256, ctx, n_kv, Q8_D_MAX, lambda b: 0x80)           # q = -128
        call = q4dec.q8kv_attn_decode
    K, kk = _scale_cache(K0, *args)
    V, kv = _scale_cache(V0, *args)
    assert kk == kv and kk >= 8
    scale = 2.0 ** -kk
    Kd, Vd = dev_bytes(K), dev_bytes(V)
    outs = {}
    for M in (1, 5):
        Q = synth.queries(902 + ctx + M, M, n_q)
        ref = oracle.attn_decode(Q, K, V, ctx, n_q, n_kv, 256, M, scale=scale, fmt=fmt)
        out = call(dev_bf16(Q.reshape(M, n_q, 256)), Kd, Vd, ctx_len=ctx, n_kv_heads=n_kv,
                   softmax_scale=scale)
        torch.cuda.synchronize()
        o = out.cpu().numpy().astype(np.float64)
        assert np.isfinite(o).all(), f"{fmt} ctx={ctx} M={M}: non-finite output"
        err = np.abs(o - ref).max()
        assert err <= ATTN_TOL * 2.0 ** kv, (fmt, ctx, M, err, ATTN_TOL * 2.0 ** kv)
        outs[M] = o
    assert q4dec.device_error() == 0
