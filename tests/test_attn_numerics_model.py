"""Error budget of the tensor-memory attention kernel's arithmetic, on the CPU.

A host restatement of the roundings that kernel performs -- K and V entering
the MMAs as fp16 d*(q-8) (Q4) or d*q (Q8), Q as fp16, scores summed in fp32,
softmax in base 2 over 128-token tiles with the running maximum of the tiles
seen so far, P rounded to fp16 and summed in fp32 for the row sums, P.V in
fp32 -- compared with the fp64 oracle.  It shows, independently of a GPU, that
these readings keep the output well inside the 3e-3 parity bound, including
for extreme codes and scales."""
import numpy as np
import pytest

import oracle
import synth

TILE = 128


def _model(Q_bits, Khat, Vhat, ctx, n_q, n_kv, M, scale=1.0):
    """Khat / Vhat: exact fp64 dequantised caches [n_kv][ctx][256]."""
    g = n_q // n_kv
    Q = oracle.bf16_bits_to_f64(np.asarray(Q_bits).reshape(M, n_q, 256))
    Qh = Q.astype(np.float16).astype(np.float32)
    K16 = Khat.astype(np.float16).astype(np.float32)       # one rounding of d*(q-8) or d*q
    V16 = Vhat.astype(np.float16).astype(np.float32)
    out = np.empty((M, n_q, 256))
    c = np.float32(scale * np.log2(np.e))
    for m in range(M):
        pos = ctx - M + m
        for h in range(n_q):
            kv = h // g
            m_run, l, o = -np.inf, np.float32(0), np.zeros(256, np.float32)
            for t0 in range(0, pos + 1, TILE):
                t1 = min(pos + 1, t0 + TILE)
                s = (K16[kv, t0:t1] @ Qh[m, h]).astype(np.float32) * c
                m_new = max(m_run, float(s.max()))
                alpha = np.float32(2.0 ** (m_run - m_new)) if m_run != -np.inf else np.float32(0)
                p = np.exp2(s - np.float32(m_new)).astype(np.float16).astype(np.float32)
                l = l * alpha + p.sum(dtype=np.float32)
                o = o * alpha + p @ V16[kv, t0:t1]
                m_run = m_new
            out[m, h] = o / l
    return out


def _check(Q, K, V, ctx, n_q, n_kv, M, fmt):
    deq = oracle.dequant if fmt == "q4_0" else oracle.dequant_q8
    Kh = deq(K, n_kv * ctx, 256).reshape(n_kv, ctx, 256)
    Vh = deq(V, n_kv * ctx, 256).reshape(n_kv, ctx, 256)
    ref = oracle.attn_decode(Q, K, V, ctx, n_q, n_kv, 256, M, fmt=fmt)
    err = np.abs(_model(Q, Kh, Vh, ctx, n_q, n_kv, M) - ref).max()
    return err


@pytest.mark.parametrize("fmt", ["q4_0", "q8_0"])
@pytest.mark.parametrize("seed", [1, 2])
def test_tc_arithmetic_is_inside_the_bound(fmt, seed):
    ctx, n_q, n_kv, M = 700, 12, 2, 5
    cache = synth.q4_0_kv_cache if fmt == "q4_0" else synth.q8_0_kv_cache
    K, V = cache(100 + seed, n_kv, ctx), cache(200 + seed, n_kv, ctx)
    Q = synth.queries(300 + seed, M, n_q)
    assert _check(Q, K, V, ctx, n_q, n_kv, M, fmt) < 3e-4      # a tenth of the 3e-3 bound


def test_tc_arithmetic_extreme_q8_codes_and_scales():
    # the GPU test's extreme case: K codes -128 / 127 in every block with
    # scales up to 4 (|k| up to 512), V at unit scale
    ctx, n_q, n_kv, M = 300, 12, 2, 5
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
    assert _check(Q, K, V, ctx, n_q, n_kv, M, "q8_0") < 1e-3
