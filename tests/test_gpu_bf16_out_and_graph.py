"""GPU tests of the bf16-output option of q4_gemv_ex2 / q4_gemv_swiglu_ex
(Q4D_GEMV_OUT_BF16) and of one decode layer's calls captured into a CUDA
graph.

bf16 outputs are specified as the fp32 result rounded to nearest even, so the
first check is bit equality with the fp32 call's output converted by torch
(also round-to-nearest-even); the second is parity with the oracle, within the
GEMV bound plus half a bf16 unit in the last place (2^-8 relative)."""
import numpy as np
import pytest
import torch

import oracle
import synth
from bit_weight_streaming_dequant_b200 import q4dec
from gpu_util import assert_attn_close, dev_bf16, dev_bytes

pytestmark = pytest.mark.gpu

# (N, K): one pass, several passes with a ragged tail, a K split (few rows,
# long K), the layer shapes' widths
GEMV_CASES = [(37, 4352), (300, 1280), (64, 65536), (2048, 5120), (5120, 6144)]


@pytest.mark.parametrize("N,K", GEMV_CASES)
@pytest.mark.parametrize("M", [1, 3, 5])
def test_gemv_bf16_output_is_the_rounded_fp32_output(cuda_ok, N, K, M):
    W = synth.q4_0_weights(700 + N + M, N, K)
    x = synth.activations(800 + K + M, M, K)
    Wd, xd = dev_bytes(W), dev_bf16(x)
    y32 = q4dec.q4_gemv(Wd, xd, N=N, K=K)
    y16 = q4dec.q4_gemv(Wd, xd, N=N, K=K, out_dtype=torch.bfloat16)
    y16p = q4dec.q4_gemv(Wd, xd, N=N, K=K, out_dtype=torch.bfloat16, weight_prefetch=True)
    torch.cuda.synchronize()
    assert y16.dtype == torch.bfloat16
    assert torch.equal(y16, y32.to(torch.bfloat16))
    assert torch.equal(y16p, y16)
    y_ref, S = oracle.gemv(W, x, M, N, K)
    err = np.abs(y16.float().cpu().numpy().astype(np.float64) - y_ref)
    assert (err <= oracle.gemv_tolerance(S) + 2.0 ** -8 * np.abs(y_ref)).all()
    assert q4dec.device_error() == 0


@pytest.mark.parametrize("N,K", [(3, 512), (300, 1280), (8, 65536)])
@pytest.mark.parametrize("M", [1, 5])
def test_swiglu_bf16_output_is_the_rounded_fp32_output(cuda_ok, N, K, M):
    W = synth.q4_0_weights(900 + N + M, 2 * N, K)
    x = synth.activations(950 + K + M, M, K)
    Wd, xd = dev_bytes(W), dev_bf16(x)
    h32 = q4dec.q4_gemv_swiglu(Wd, xd, N=N, K=K)
    h16 = q4dec.q4_gemv_swiglu(Wd, xd, N=N, K=K, out_dtype=torch.bfloat16)
    torch.cuda.synchronize()
    assert torch.equal(h16, h32.to(torch.bfloat16))
    h_ref, tol = oracle.gemv_swiglu(W, x, M, N, K)
    err = np.abs(h16.float().cpu().numpy().astype(np.float64) - h_ref)
    assert (err <= tol + 2.0 ** -8 * np.abs(h_ref)).all()


def test_bf16_output_feeds_the_next_gemv(cuda_ok):
    # h (bf16) from the fused gate / up call is the down projection's x
    N_ffn, K_hid, M = 1024, 2048, 2
    Wgu = dev_bytes(synth.q4_0_weights(31, 2 * N_ffn, K_hid))
    Wdn = dev_bytes(synth.q4_0_weights(32, K_hid, N_ffn))
    x = dev_bf16(synth.activations(33, M, K_hid))
    h16 = q4dec.q4_gemv_swiglu(Wgu, x, N=N_ffn, K=K_hid, out_dtype=torch.bfloat16)
    y = q4dec.q4_gemv(Wdn, h16, N=K_hid, K=N_ffn)
    h32 = q4dec.q4_gemv_swiglu(Wgu, x, N=N_ffn, K=K_hid)
    y_ref = q4dec.q4_gemv(Wdn, h32.to(torch.bfloat16), N=K_hid, K=N_ffn)
    torch.cuda.synchronize()
    assert torch.equal(y, y_ref)


def test_output_dtype_checks(cuda_ok):
    W = dev_bytes(synth.q4_0_weights(5, 16, 256))
    x = dev_bf16(synth.activations(6, 1, 256))
    with pytest.raises(ValueError):
        q4dec.q4_gemv(W, x, N=16, K=256, out_dtype=torch.float16)
    with pytest.raises(TypeError):
        q4dec.q4_gemv(W, x, torch.empty((1, 16), device="cuda"), N=16, K=256,
                      out_dtype=torch.bfloat16)


def test_decode_layer_calls_replay_as_one_cuda_graph(cuda_ok):
    """One decode layer's library calls -- K/V append of the verified rows,
    attention, output projection, fused gate / up + SwiGLU with bf16 output,
    down projection -- captured on a side stream into one CUDA graph; two
    replays reproduce the eager results bit for bit, and the attention part
    matches the oracle on the appended cache."""
    n_q, n_kv, M, ctx, cap = 24, 4, 3, 1000, 1024
    hid, ffn = 1024, 2048
    dev = torch.device("cuda")
    K0, V0 = synth.q4_0_kv_cache(41, n_kv, cap), synth.q4_0_kv_cache(42, n_kv, cap)
    Q = dev_bf16(synth.queries(43, M, n_q).reshape(M, n_q, 256))
    k_new = torch.from_numpy(np.random.default_rng(44).standard_normal((M, n_kv, 256))
                             .astype(np.float32)).to(dev)
    v_new = torch.from_numpy(np.random.default_rng(45).standard_normal((M, n_kv, 256))
                             .astype(np.float32)).to(dev)
    Wo = dev_bytes(synth.q4_0_weights(46, hid, n_q * 256))
    Wgu = dev_bytes(synth.q4_0_weights(47, 2 * ffn, hid))
    Wdn = dev_bytes(synth.q4_0_weights(48, hid, ffn))
    x_ffn = dev_bf16(synth.activations(49, M, hid))

    def layer(Kc, Vc, out, attn_bf16, y_o, h, y_dn, stream, ws):
        q4dec.q4kv_append(Kc, Vc, k_new, v_new, pos=ctx - M, kv_stride_tokens=cap, stream=stream)
        q4dec.q4kv_attn_decode(Q, Kc, Vc, out, ctx_len=ctx, n_kv_heads=n_kv, kv_stride_tokens=cap,
                               stream=stream, workspace=ws["attn"])
        attn_bf16.copy_(out.reshape(M, n_q * 256))
        q4dec.q4_gemv(Wo, attn_bf16, y_o, N=hid, K=n_q * 256, stream=stream,
                      workspace=ws["o"], weight_prefetch=True)
        q4dec.q4_gemv_swiglu(Wgu, x_ffn, h, N=ffn, K=hid, stream=stream, workspace=ws["gu"],
                             weight_prefetch=True)
        q4dec.q4_gemv(Wdn, h, y_dn, N=hid, K=ffn, stream=stream, workspace=ws["dn"],
                      weight_prefetch=True)

    def buffers():
        L = q4dec.lib()
        ws = {"attn": torch.empty(max(16, L.q4d_attn_workspace_bytes(ctx, n_q, n_kv, 256, M)),
                                  dtype=torch.uint8, device=dev),
              # GEMV workspaces: zero-filled before first use
              "o": torch.zeros(max(16, L.q4d_gemv_workspace_bytes(M, hid, n_q * 256)),
                               dtype=torch.uint8, device=dev),
              "gu": torch.zeros(max(16, L.q4d_gemv_swiglu_workspace_bytes(M, ffn, hid)),
                                dtype=torch.uint8, device=dev),
              "dn": torch.zeros(max(16, L.q4d_gemv_workspace_bytes(M, hid, ffn)),
                                dtype=torch.uint8, device=dev)}
        return (dev_bytes(K0), dev_bytes(V0), torch.empty((M, n_q, 256), device=dev),
                torch.empty((M, n_q * 256), dtype=torch.bfloat16, device=dev),
                torch.empty((M, hid), device=dev),
                torch.empty((M, ffn), dtype=torch.bfloat16, device=dev),
                torch.empty((M, hid), device=dev), ws)

    eager = buffers()
    layer(*eager[:7], None, eager[7])
    torch.cuda.synchronize()

    cap_bufs = buffers()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            layer(*cap_bufs[:7], s, cap_bufs[7])
    torch.cuda.synchronize()
    for _ in range(2):
        g.replay()
        torch.cuda.synchronize()
        for a, b in zip(eager[:7], cap_bufs[:7]):
            assert torch.equal(a, b)
    assert q4dec.device_error() == 0

    # attention after the append: the oracle on the cache the oracle appends to
    Kr, Vr = oracle.kv_append(K0, V0, k_new.cpu().numpy(), v_new.cpu().numpy(), n_kv, cap,
                              ctx - M, M)
    ref = oracle.attn_decode(synth.queries(43, M, n_q), Kr, Vr, ctx, n_q, n_kv, 256, M,
                             kv_stride=cap)
    assert_attn_close(cap_bufs[2], ref, "graph-captured attention")
    del g
