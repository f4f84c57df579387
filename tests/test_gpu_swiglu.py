"""GPU parity of q4_gemv_swiglu_ex (through the C ABI) against the oracle's
fused gate / up GEMV + SwiGLU, within the bound propagated from the GEMV
tolerance; and agreement with two plain GEMVs on the de-interleaved rows."""
import numpy as np
import pytest
import torch

import oracle
import synth
from bit_weight_streaming_dequant_b200 import q4dec
from gpu_util import dev_bf16, dev_bytes

pytestmark = pytest.mark.gpu


def _interleave(Wg, Wu, N, K):
    rg = oracle.weight_rows(Wg, N, K).reshape(N, -1)
    ru = oracle.weight_rows(Wu, N, K).reshape(N, -1)
    inter = np.empty((2 * N, rg.shape[1]), dtype=np.uint8)
    inter[0::2], inter[1::2] = rg, ru
    return synth.column_major(inter.reshape(-1), 2 * N, K)


def _check(h_gpu, h_ref, tol, what):
    h = h_gpu.detach().cpu().numpy().astype(np.float64)
    err = np.abs(h - h_ref)
    bad = err > tol
    assert not bad.any(), f"{what}: {bad.sum()} elements out of bound, worst {(err - tol).max():.3e}"


@pytest.mark.parametrize("N,K", [(1, 256), (3, 512), (37, 4352), (300, 1280), (2048, 5120),
                                 (8, 65536)])
@pytest.mark.parametrize("M", [1, 3, 5])
def test_swiglu_matches_oracle(cuda_ok, N, K, M):
    W = synth.q4_0_weights(400 + N + M, 2 * N, K)
    x = synth.activations(500 + K + M, M, K)
    h_ref, tol = oracle.gemv_swiglu(W, x, M, N, K)
    h = q4dec.q4_gemv_swiglu(dev_bytes(W), dev_bf16(x), N=N, K=K)
    torch.cuda.synchronize()
    _check(h, h_ref, tol, f"N={N} K={K} M={M}")


def test_swiglu_equals_two_plain_gemvs_then_silu(cuda_ok):
    N, K, M = 1024, 5120, 2
    Wg, Wu = synth.q4_0_weights(61, N, K), synth.q4_0_weights(62, N, K)
    xnp = synth.activations(63, M, K)
    x = dev_bf16(xnp)
    h = q4dec.q4_gemv_swiglu(dev_bytes(_interleave(Wg, Wu, N, K)), x, N=N, K=K,
                             weight_prefetch=True)
    g = q4dec.q4_gemv(dev_bytes(Wg), x, N=N, K=K)
    u = q4dec.q4_gemv(dev_bytes(Wu), x, N=N, K=K)
    torch.cuda.synchronize()
    ref = (g / (1 + torch.exp(-g)) * u).double().cpu().numpy()
    # The fused matrix has 2N rows, so its K ranges split at other places than
    # the plain N-row GEMVs': g and u agree up to fp32 reassociation of their
    # sums (far below 1e-5 of sum |w x|), carried through silu(g) * u, plus
    # the two epilogues' fp32 roundings.
    _, Sg = oracle.gemv(Wg, xnp, M, N, K)
    _, Su = oracle.gemv(Wu, xnp, M, N, K)
    gd, ud = g.double().cpu().numpy(), u.double().cpu().numpy()
    bound = oracle.swiglu_tolerance(gd, ud, 1e-5 * Sg, 1e-5 * Su) + 1e-6 * np.abs(ref)
    err = np.abs(h.double().cpu().numpy() - ref)
    assert (err <= bound).all(), f"worst {(err / bound).max():.3f} of the bound"
    assert q4dec.device_error() == 0
