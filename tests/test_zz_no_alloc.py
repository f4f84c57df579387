"""The allocation-free attention entry point, q4kv_attn_decode_noalloc.

It serves callers that may not allocate device memory while running (runtimes
that reserve all memory in their own arena at start-up; decode loops where a
cudaMalloc would synchronise the device).  Its scratch is a static 16 MiB
device array inside the library, so its results must equal those of the
workspace entry point, q4kv_attn_decode_ex, on every call -- including a second
call that finds the previous call's states still in the array.

Both entry points run the same launch plan and the same kernels; only the
address of the split states differs, so the outputs must be equal bit for bit.

This file is collected last so that a run stopping at the first failure has
already run every other test; it also passes alone in a fresh process.
"""
import ctypes

import pytest
import torch

import synth
from bit_weight_streaming_dequant_b200 import q4dec

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
            assert torch.equal(out, ref), (
                f"ctx={ctx} M={M} call {call}: max |diff| {(out - ref).abs().max().item()}")
        del Q, K, V
    assert q4dec.device_error() == 0


@pytest.mark.gpu
def test_no_alloc_python_wrapper(cuda_ok):
    # the binding's checks and stream handling, then the same bitwise equality
    ctx, n_q, n_kv, M = 65536, 24, 4, 5
    Q, K, V = _inputs(ctx, n_q, n_kv, M, 790)
    ref = _with_workspace(Q, K, V, ctx, n_q, n_kv, M)
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    for call in range(2):
        out = torch.full((M, n_q, 256), float("nan"), dtype=torch.float32, device="cuda")
        with torch.cuda.stream(side):
            got = q4dec.q4kv_attn_decode_noalloc(Q, K, V, out, ctx_len=ctx, n_kv_heads=n_kv)
        torch.cuda.synchronize()
        assert got is out and torch.equal(out, ref), f"wrapper call {call}"
    bad = torch.empty((M, n_q, 128), dtype=torch.float32, device="cuda")
    with pytest.raises(ValueError):
        q4dec.q4kv_attn_decode_noalloc(Q, K, V, bad, ctx_len=ctx, n_kv_heads=n_kv)
    with pytest.raises(ValueError):  # caches shorter than the stated stride
        q4dec.q4kv_attn_decode_noalloc(Q, K, V, out, ctx_len=ctx, n_kv_heads=n_kv,
                                       kv_stride_tokens=2 * ctx)
    assert q4dec.device_error() == 0


def test_no_alloc_wrapper_refuses_host_tensors():
    # no CPU fallback: host tensors are refused before anything runs
    import torch as t
    Q = t.zeros((1, 24, 256), dtype=t.bfloat16)
    K = t.zeros(4 * 16 * 144, dtype=t.uint8)
    out = t.zeros((1, 24, 256), dtype=t.float32)
    with pytest.raises(TypeError):
        q4dec.q4kv_attn_decode_noalloc(Q, K, K, out, ctx_len=16, n_kv_heads=4)


def test_no_alloc_scratch_holds_every_plan():
    # The split states of a plan take n_splits * M * n_q * (256 + 2) * 4 bytes.
    # With one CTA per (split, KV head, row group) and splits sized to fill
    # the SMs once, n_splits * n_kv * row_groups < 2 * num_sms and at most 32
    # query rows share a CTA, so a plan needs < 2 * num_sms * 32 * 1032 bytes:
    # 9.8 MB on 148 SMs, inside the 16 MiB array for any shape.
    L = q4dec.lib()
    plan = q4dec.AttnPlan()
    worst = 0
    for sms in (148, 132, 160, 240):
        for n_q, n_kv in ((24, 4), (1, 1), (8, 1), (32, 1), (48, 1), (64, 64), (64, 8),
                          (128, 1), (96, 3), (40, 8), (512, 1), (28, 4), (150, 150)):
            for M in range(1, 6):
                for ctx in (M, 1000, 4096, 65536, 262144, 1 << 20):
                    st = L.q4d_plan_attn(ctx, n_q, n_kv, 256, M, sms, ctypes.byref(plan))
                    assert st == 0
                    assert plan.workspace_bytes < 2 * sms * 32 * 1032
                    assert plan.workspace_bytes <= q4dec.NOALLOC_SCRATCH_BYTES
                    worst = max(worst, plan.workspace_bytes)
    assert worst > 0


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
