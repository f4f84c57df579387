"""The allocation-free attention entry point, q4kv_attn_decode_noalloc.

It serves callers that may not allocate device memory while running (runtimes
that reserve all memory in their own arena at start-up; decode loops where a
cudaMalloc would synchronise the device).  Its scratch is a static 16 MiB
device array inside the library, so its results must equal those of the
workspace entry point, q4kv_attn_decode_ex, on every call -- including a second
call that finds the previous call's states still in the array.

This file is collected last so that a run stopping at the first failure has
already run every other test; it also passes alone in a fresh process.
"""
import ctypes

import pytest
import torch

import synth
from bit_weight_streaming_dequant_b200 import q4dec

ATTN_TOL = 3e-3

# (ctx_len, n_q_heads, n_kv_heads, M): long contexts use many splits (scratch
# of several MiB), short ones a single pass (no scratch at all)
CASES = [(262144, 24, 4, 5), (65536, 24, 4, 1), (4096, 24, 4, 5), (300, 24, 4, 2),
         (20000, 8, 1, 3)]


def _inputs(ctx, n_q, n_kv, M, seed):
    K = synth.device_q4_0_kv_cache(seed, n_kv, ctx)
    V = synth.device_q4_0_kv_cache(seed + 1, n_kv, ctx)
    Q = synth.device_bf16_normal(seed + 2, (M, n_q, 256), scale=1.0 / 16)
    return Q, K, V


def _with_workspace(Q, K, V, ctx, n_q, n_kv, M):
    L = q4dec.lib()
    need = L.q4d_attn_workspace_bytes(ctx, n_q, n_kv, 256, M)
    ws = torch.empty(max(need, 16), dtype=torch.uint8, device="cuda")
    out = torch.empty((M, n_q, 256), dtype=torch.float32, device="cuda")
    st = L.q4kv_attn_decode_ex(Q.data_ptr(), K.data_ptr(), V.data_ptr(), out.data_ptr(), ctx,
                               n_q, n_kv, 256, M, ctx, ctypes.c_float(1.0), None,
                               ws.data_ptr(), ws.numel())
    assert st == 0
    return out


def _no_alloc(Q, K, V, ctx, n_q, n_kv, M):
    out = torch.full((M, n_q, 256), float("nan"), dtype=torch.float32, device="cuda")
    torch.cuda.synchronize()
    st = q4dec.lib().q4kv_attn_decode_noalloc(Q.data_ptr(), K.data_ptr(), V.data_ptr(),
                                              out.data_ptr(), ctx, n_q, n_kv, 256, M, ctx,
                                              ctypes.c_float(1.0), None)
    assert st == 0, q4dec.STATUS.get(st, st)
    return out


@pytest.mark.gpu
def test_no_alloc_matches_workspace_entry_point_twice(cuda_ok):
    for i, (ctx, n_q, n_kv, M) in enumerate(CASES):
        Q, K, V = _inputs(ctx, n_q, n_kv, M, 700 + 10 * i)
        ref = _with_workspace(Q, K, V, ctx, n_q, n_kv, M)
        for call in range(2):
            out = _no_alloc(Q, K, V, ctx, n_q, n_kv, M)
            torch.cuda.synchronize()
            err = (out - ref).abs().max().item()
            assert err <= ATTN_TOL, f"ctx={ctx} M={M} call {call}: max |err| {err}"
        del Q, K, V
    assert q4dec.device_error() == 0


def test_no_alloc_rejects_bad_arguments_before_cuda():
    L = q4dec.lib()
    fake = 0x10000
    one = ctypes.c_float(1.0)
    assert L.q4kv_attn_decode_noalloc(fake, fake, fake, fake, 100, 24, 4, 128, 1, 100, one,
                                      None) == 2
    assert L.q4kv_attn_decode_noalloc(None, fake, fake, fake, 100, 24, 4, 256, 1, 100, one,
                                      None) == 1
    assert L.q4kv_attn_decode_noalloc(fake + 8, fake, fake, fake, 100, 24, 4, 256, 1, 100, one,
                                      None) == 3
    assert L.q4kv_attn_decode_noalloc(fake, fake, fake, fake, 100, 24, 4, 256, 1, 100,
                                      ctypes.c_float(float("nan")), None) == 1
