"""The debug build on the GPU (libq4dec_debug.so: the same sources with
Q4D_DEBUG, every global access of every kernel index-checked into the device
error record).  On valid inputs no check fails and every result is bit for
bit the release build's (the checks change no arithmetic); a check made to
fail -- a declared weight extent smaller than the real buffer, so that the
redirected copies still read memory that exists -- is reported with its site
and offset (by the failing call itself: a debug-build call waits for its
work and returns the record's status), and the launch ends normally."""
import numpy as np
import pytest
import torch

import oracle
import synth
from bit_weight_streaming_dequant_b200 import q4dec
from gpu_util import assert_attn_close, assert_gemv_close, dev_bf16, dev_bytes, host_bytes

pytestmark = pytest.mark.gpu


@pytest.fixture
def debug_lib(cuda_ok):
    q4dec.use_debug_library(True)
    try:
        assert q4dec.debug_build()
        q4dec.device_error_record(reset=True)
        yield
        # no check failed and no wait ran out in the test's launches
        assert q4dec.device_error_record(reset=True) == (0, 0, 0, 0)
    finally:
        q4dec.debug_limit_weights(0)
        q4dec.use_debug_library(False)


def _release(fn):
    """fn() through the release library (the debug one stays selected)."""
    q4dec.use_debug_library(False)
    try:
        out = fn()
        torch.cuda.synchronize()
        assert not q4dec.debug_build()
        return out
    finally:
        q4dec.use_debug_library(True)


def _debug(fn):
    out = fn()
    torch.cuda.synchronize()
    return out


GEMV_CASES = [(1, 256, 1), (37, 4352, 3), (300, 1280, 5), (1000, 2048, 2), (149, 512, 4),
              (64, 65536, 1), (6144, 5120, 5), (17408, 5120, 1)]


@pytest.mark.parametrize("N,K,M", GEMV_CASES)
def test_gemv_no_check_fails_and_results_equal_the_release_build(debug_lib, N, K, M):
    Wnp = synth.q4_0_weights(N + 3 * K, N, K)
    xnp = synth.activations(M + K, M, K)
    W, x = dev_bytes(Wnp), dev_bf16(xnp)
    y_dbg = _debug(lambda: q4dec.q4_gemv(W, x, N=N, K=K))
    y_rel = _release(lambda: q4dec.q4_gemv(W, x, N=N, K=K))
    assert torch.equal(y_dbg, y_rel)
    if N * K <= 2_000_000:
        y_ref, S = oracle.gemv(Wnp, xnp, M, N, K)
        assert_gemv_close(y_dbg, y_ref, S, f"debug build N={N} K={K} M={M}")


def test_batch_chain_swiglu_and_bf16_no_check_fails(debug_lib):
    hid, ffn, M = 1024, 2048, 3
    Wgu = dev_bytes(synth.q4_0_weights(850, 2 * ffn, hid))
    Wdn = dev_bytes(synth.q4_0_weights(851, hid, ffn))
    Wr = dev_bytes(synth.q4_0_weights(852, 2 * 1000, hid))
    x = dev_bf16(synth.activations(853, M, hid))

    def run():
        h = torch.empty((M, ffn), dtype=torch.bfloat16, device="cuda")
        y = torch.empty((M, hid), device="cuda")
        hr = torch.empty((M, 1000), device="cuda")
        b = q4dec.GemvBatch([dict(W=Wgu, x=x, y=h, N=ffn, K=hid, swiglu=True),
                             dict(W=Wr, x=x, y=hr, N=1000, K=hid, swiglu=True),
                             dict(W=Wdn, x=h, y=y, N=hid, K=ffn, wait_for=0)])
        b.run(weight_prefetch=True)
        torch.cuda.synchronize()
        assert int(torch.count_nonzero(b.workspace)) == 0
        return h, hr, y

    dbg = _debug(run)
    rel = _release(run)
    for a, b in zip(dbg, rel):
        assert torch.equal(a, b)


ATTN_CASES = [(1, 4, 1, 1), (5, 24, 4, 5), (1000, 24, 4, 5), (4097, 24, 4, 1), (300, 64, 4, 5),
              (777, 48, 1, 5)]


@pytest.mark.parametrize("ctx,n_q,n_kv,M", ATTN_CASES)
def test_attention_no_check_fails_and_results_equal_the_release_build(debug_lib, ctx, n_q,
                                                                       n_kv, M):
    Q = synth.queries(ctx + 2, M, n_q)
    Kc, Vc = synth.q4_0_kv_cache(ctx, n_kv, ctx), synth.q4_0_kv_cache(ctx + 1, n_kv, ctx)
    Qd, K, V = dev_bf16(Q.reshape(M, n_q, 256)), dev_bytes(Kc), dev_bytes(Vc)
    call = lambda: q4dec.q4kv_attn_decode(Qd, K, V, ctx_len=ctx, n_kv_heads=n_kv)
    out_dbg = _debug(call)
    assert torch.equal(out_dbg, _release(call))
    ref = oracle.attn_decode(Q, Kc, Vc, ctx, n_q, n_kv, 256, M)
    assert_attn_close(out_dbg, ref, f"debug build ctx={ctx} {n_q}/{n_kv} M={M}")


@pytest.mark.parametrize("ctx,M", [(129, 1), (2500, 5)])
def test_q8_attention_no_check_fails(debug_lib, ctx, M):
    n_q, n_kv = 24, 4
    Q = synth.queries(ctx + 5, M, n_q)
    Kc, Vc = synth.q8_0_kv_cache(ctx, n_kv, ctx), synth.q8_0_kv_cache(ctx + 1, n_kv, ctx)
    Qd, K, V = dev_bf16(Q.reshape(M, n_q, 256)), dev_bytes(Kc), dev_bytes(Vc)
    call = lambda: q4dec.q8kv_attn_decode(Qd, K, V, ctx_len=ctx, n_kv_heads=n_kv)
    out_dbg = _debug(call)
    assert torch.equal(out_dbg, _release(call))


def test_append_no_check_fails_and_bytes_equal_the_oracle(debug_lib):
    n_kv, stride, pos, M = 4, 300, 295, 5
    rng = np.random.default_rng(7)
    Kc, Vc = synth.q4_0_kv_cache(21, n_kv, stride), synth.q4_0_kv_cache(22, n_kv, stride)
    kn = (rng.standard_normal((M, n_kv, 256)) * 2.5).astype(np.float32)
    vn = rng.standard_normal((M, n_kv, 256)).astype(np.float32)
    K, V = dev_bytes(Kc), dev_bytes(Vc)
    q4dec.q4kv_append(K, V, torch.from_numpy(kn).cuda(), torch.from_numpy(vn).cuda(), pos=pos,
                      kv_stride_tokens=stride)
    torch.cuda.synchronize()
    K2, V2 = oracle.kv_append(Kc, Vc, kn, vn, n_kv, stride, pos, M)
    np.testing.assert_array_equal(host_bytes(K), K2)
    np.testing.assert_array_equal(host_bytes(V), V2)


def test_weight_copy_check_reports_site_and_offset(debug_lib):
    N, K, M = 512, 1024, 2                      # 294912 bytes of weights, 4 row blocks
    Wnp = synth.q4_0_weights(860, N, K)
    xnp = synth.activations(861, M, K)
    W, x = dev_bytes(Wnp), dev_bf16(xnp)
    limit = 100_000                             # the copies past it read the first rows instead
    q4dec.debug_limit_weights(limit)
    try:
        # a debug-build call waits for its work and reports the record itself
        with pytest.raises(q4dec.Q4DecError) as failed:
            q4dec.q4_gemv(W, x, N=N, K=K)
        assert failed.value.status == 7
    finally:
        q4dec.debug_limit_weights(0)
    st, bits, site, index = q4dec.device_error_record(reset=True)
    assert st == 7 and bits == 2, (st, bits)                 # Q4D_ERR_DEVICE_INDEX, no time-out
    assert q4dec.CHECK_SITES[site] == "gemv weights"
    piece = 128 * 144                                        # one column of a row block
    assert limit - piece < index < N * (K // 256) * 144 and index % 144 == 0, index
    # the launch ended normally: the context is usable and the next call is right
    y = q4dec.q4_gemv(W, x, N=N, K=K)
    torch.cuda.synchronize()
    y_ref, S = oracle.gemv(Wnp, xnp, M, N, K)
    assert_gemv_close(y, y_ref, S, "after a failed check")


@pytest.mark.parametrize("debug", [True, False])
def test_index_check_selftest_records_the_first_failure(cuda_ok, debug):
    q4dec.use_debug_library(debug)
    try:
        L = q4dec.lib()
        base = (1 << 40) + 7
        for n_fail in (0, 1, 5, 64):
            rec = torch.zeros(4, dtype=torch.int32, device="cuda")
            assert L.q4d_index_check_selftest(rec.data_ptr(), base, n_fail, None) == 0
            torch.cuda.synchronize()
            r = [int(v) & 0xFFFFFFFF for v in rec.cpu()]
            if n_fail == 0:
                assert r == [0, 0, 0, 0]
                continue
            assert r[0] == 2 and r[1] == 255, r           # the bit, the site; no wrong verdict
            assert base <= r[2] + (r[3] << 32) < base + n_fail, r
    finally:
        q4dec.use_debug_library(False)
