"""GPU parity of q4kv_append (through the C ABI) against the oracle: the
quantised cache bytes must match bit for bit; then attention over the grown
cache matches the oracle (the verify step of speculative decoding)."""
import numpy as np
import pytest
import torch

import oracle
import synth
from bit_weight_streaming_dequant_b200 import q4dec
from gpu_util import assert_attn_close, dev_bf16, dev_bytes, host_bf16_bits, host_bytes

pytestmark = pytest.mark.gpu


def _append(Kc, Vc, kn, vn, n_kv, stride, pos):
    K, V = dev_bytes(Kc), dev_bytes(Vc)
    k, v = torch.from_numpy(kn).cuda(), torch.from_numpy(vn).cuda()
    q4dec.q4kv_append(K, V, k, v, pos=pos, kv_stride_tokens=stride)
    torch.cuda.synchronize()
    return host_bytes(K), host_bytes(V)


@pytest.mark.parametrize("n_kv,stride,pos,M", [(4, 64, 0, 1), (4, 64, 59, 5), (1, 8, 3, 5),
                                               (8, 300, 123, 3), (4, 4096, 4091, 5)])
def test_append_matches_oracle_bytes(cuda_ok, n_kv, stride, pos, M):
    rng = np.random.default_rng(n_kv * 1000 + pos)
    Kc = synth.q4_0_kv_cache(11 + pos, n_kv, stride)
    Vc = synth.q4_0_kv_cache(12 + pos, n_kv, stride)
    kn = (rng.standard_normal((M, n_kv, 256)) * 2.5).astype(np.float32)
    vn = rng.standard_normal((M, n_kv, 256)).astype(np.float32)
    K1, V1 = _append(Kc, Vc, kn, vn, n_kv, stride, pos)
    K2, V2 = oracle.kv_append(Kc, Vc, kn, vn, n_kv, stride, pos, M)
    np.testing.assert_array_equal(K1, K2)
    np.testing.assert_array_equal(V1, V2)


def test_append_edge_values(cuda_ok):
    n_kv, stride, pos, M = 2, 16, 4, 4
    kn = np.zeros((M, n_kv, 256), dtype=np.float32)
    kn[0, 0, :32] = -0.0                                   # all -0: d = +0, q = 8
    kn[1, 0, :4] = [-3.0, 3.0, 1.0, -1.0]                  # tie on |v|: first wins
    kn[1, 1, :32] = np.float32(1e-6)                       # subnormal fp16 scale
    kn[2, 0, :32] = np.linspace(-7.0, 9.5, 32, dtype=np.float32)   # positive amax
    kn[2, 1, :32] = np.float32(3e-9)                       # scale rounds to zero
    kn[3] = np.random.default_rng(3).standard_normal((n_kv, 256)).astype(np.float32) * 1e3
    vn = kn[::-1].copy()
    Kc = np.zeros(n_kv * stride * 144, dtype=np.uint8)
    Vc = np.full(n_kv * stride * 144, 0xA5, dtype=np.uint8)
    K1, V1 = _append(Kc, Vc, kn, vn, n_kv, stride, pos)
    K2, V2 = oracle.kv_append(Kc, Vc, kn, vn, n_kv, stride, pos, M)
    np.testing.assert_array_equal(K1, K2)
    np.testing.assert_array_equal(V1, V2)


def test_append_then_attend_matches_oracle(cuda_ok):
    # a verify round: the M draft tokens' K/V are appended at ctx_len - M, then
    # the M query rows attend causally over the grown cache
    n_q, n_kv, M, ctx = 24, 4, 5, 777
    stride = 1024
    Kc = synth.q4_0_kv_cache(21, n_kv, stride)
    Vc = synth.q4_0_kv_cache(22, n_kv, stride)
    rng = np.random.default_rng(23)
    kn = rng.standard_normal((M, n_kv, 256)).astype(np.float32)
    vn = rng.standard_normal((M, n_kv, 256)).astype(np.float32)
    Q = synth.queries(24, M, n_q)
    K, V = dev_bytes(Kc), dev_bytes(Vc)
    q4dec.q4kv_append(K, V, torch.from_numpy(kn).cuda(), torch.from_numpy(vn).cuda(),
                      pos=ctx - M, kv_stride_tokens=stride)
    Qd = dev_bf16(Q.reshape(M, n_q, 256))
    out = q4dec.q4kv_attn_decode(Qd, K, V, ctx_len=ctx, n_kv_heads=n_kv, kv_stride_tokens=stride)
    torch.cuda.synchronize()
    K2, V2 = oracle.kv_append(Kc, Vc, kn, vn, n_kv, stride, ctx - M, M)
    ref = oracle.attn_decode(Q, K2, V2, ctx, n_q, n_kv, 256, M, kv_stride=stride)
    assert_attn_close(out, ref, "append + attend")
    assert q4dec.device_error() == 0
