"""Plain, slow fp64 CPU oracle of the Q4_0 decode path.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and
``bench.py``'s CPU-baseline / reference legs may import or run this file.  It
shares no code, tables or constants with the CUDA path and imports nothing
from it; both sides read the same input bytes produced by ``synth``.

What it computes, and where the pages stand on it
-------------------------------------------------
The pages ("Qwen3.8-27B at 256K on a 24GB RTX PRO 4000 SFF (432 GB/s): 50
tok/s with MTP", the paragraph beginning "NVIDIA quotes 432 GB/s") attribute
decode speed to two costs: repeatedly streaming quantised weights, and reading
a Q4 K/V cache that grows with context.  The same page (paragraph on public
GGUFs at 40K context) names the Q4_0 weight format; the paragraph on the 16
full-attention layers says only those layers keep a K/V cache, stored as Q4.
"Qwen3.8-27B on RTX 4090: 5,000 tok/s Prefill Reproduced" (section "MTP helps
ordinary prose, but acceptance controls the gain") explains that the target
model verifies a drafted block of tokens, which is where the M = 1..5 rows of
one decode step come from.  The pages define none of the formulas; this file
writes out the definitions the library implements:

* Q4_0 block: 32 weights, one fp16 scale ``d``, 16 bytes of nibbles; byte
  ``j`` holds element ``j`` (low nibble) and ``j + 16`` (high nibble);
  ``w = d * (q - 8)``.
* super-block storage: 8 blocks in 144 bytes, nibbles first (``16*b + j``),
  then the 8 fp16 scales at ``128 + 2*b`` (little endian).
* weight matrix W[N][K]: K/256 super-block columns one after another; column
  s holds super-block s of rows 0..N-1 in order, i.e. super-block (n, s) sits
  at byte (s*N + n)*144.
* K/V cache: one super-block per (KV head, token) at byte
  (h*kv_stride + t)*144 (head_dim 256).
* GEMV: ``y[m, n] = sum_k w[n, k] * x[m, k]`` for M bf16 rows x.
* decode attention: query head ``h`` reads KV head ``h // (n_q / n_kv)``; draft
  row ``m`` sits at position ``p_m = ctx_len - M + m`` and sees tokens
  ``t <= p_m``; ``s = scale * Q . K_hat``, ``P = softmax(s)``, ``out = P V_hat``.

* fused gate/up GEMV with a SwiGLU epilogue (the feed-forward block the page
  on the 64-layer model describes as gate, up and down projections): the
  weight matrix holds 2N rows, gate row n at 2n and up row n at 2n + 1;
  ``h[m, n] = silu(g) * u`` with ``silu(g) = g / (1 + exp(-g))``.
* K/V append: new K/V values (fp32) are quantised per 32-element block: amax =
  the signed element of largest magnitude (first on ties), d = fp16(amax/-8),
  q = clamp(floor(v/d + 8.5), 0, 15) with the division and the addition
  rounded in fp32 (the precision the device decides the codes in); a block
  whose d is zero stores d = +0 and q = 8.  The pages say only that the
  cache is Q4 (the paragraph on the 16 full-attention layers).

* Q8_0 K/V cache (the 8-bit cache type the page "Running Qwen3.8-27B on an
  RTX 4090" launches its server with, ``--cache-type-k/v q8_0``): 32 int8
  values and one fp16 scale per block, value ``d * q``; stored, like the Q4
  cache, as one super-block per token: the 256 int8 values first (element
  ``j`` of block ``b`` at byte ``32*b + j``), then the 8 fp16 scales at
  ``256 + 2*b`` -- 272 bytes.  Attention over it is the same computation with
  this dequantisation.

Readings taken where nothing fixes a detail: output is fp32 on the device
(fp64 here); the softmax scale defaults to 1 (queries arrive pre-scaled);
GQA groups are contiguous; non-finite inputs are out of scope.

Everything is fp64 numpy; the matrix products are numpy's (a library
primitive), with no blocking, reordering or fusion beyond the definitions.
"""
from __future__ import annotations

import numpy as np

SB_ELEMS = 256          # elements per super-block
SB_BYTES = 144          # bytes per super-block
NIBBLE_BYTES = 128      # bytes of nibbles per super-block (8 blocks x 16)
Q8_SB_BYTES = 272       # bytes per Q8_0 super-block (256 int8 values + 8 fp16 scales)


def bf16_bits_to_f64(bits) -> np.ndarray:
    """Exact value of bf16 bit patterns: the 16 bits are the top half of an
    IEEE binary32 number."""
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    return b.view(np.float32).astype(np.float64)


def f16_bits_to_f64(bits) -> np.ndarray:
    """Exact value of IEEE binary16 bit patterns."""
    return np.asarray(bits, dtype=np.uint16).view(np.float16).astype(np.float64)


def unpack_superblocks(buf, rows: int, K: int):
    """Read ``rows`` rows of ``K`` Q4_0 elements from super-block bytes.

    Returns ``q`` (uint8 [rows][K], values 0..15) and ``d`` (float64
    [rows][K/32], the per-block scale of each group of 32 elements).
    """
    if K % SB_ELEMS:
        raise ValueError("K must be a multiple of 256")
    nsb = K // SB_ELEMS
    raw = np.asarray(buf, dtype=np.uint8).reshape(-1)
    need = rows * nsb * SB_BYTES
    if raw.size < need:
        raise ValueError(f"buffer holds {raw.size} bytes, need {need}")
    sb = raw[:need].reshape(rows, nsb, SB_BYTES)
    q = np.empty((rows, nsb, 8, 32), dtype=np.uint8)
    d_bits = np.empty((rows, nsb, 8), dtype=np.uint16)
    for b in range(8):
        qs = sb[:, :, 16 * b: 16 * b + 16]           # 16 bytes of block b
        q[:, :, b, 0:16] = qs & 0x0F                  # element j
        q[:, :, b, 16:32] = qs >> 4                   # element j + 16
        lo = sb[:, :, 128 + 2 * b].astype(np.uint16)
        hi = sb[:, :, 128 + 2 * b + 1].astype(np.uint16)
        d_bits[:, :, b] = lo | (hi << 8)              # little endian fp16
    return q.reshape(rows, K), f16_bits_to_f64(d_bits).reshape(rows, K // 32)


def dequant(buf, rows: int, K: int) -> np.ndarray:
    """fp64 weights ``w = d * (q - 8)`` of ``rows x K`` Q4_0 elements."""
    q, d = unpack_superblocks(buf, rows, K)
    return np.repeat(d, 32, axis=1) * (q.astype(np.float64) - 8.0)


def weight_rows(W_buf, N: int, K: int) -> np.ndarray:
    """Reorder a weight matrix stored super-block-column-major ([K/256][N]
    super-blocks) into row order ([N][K/256] super-blocks), flat bytes."""
    nsb = K // SB_ELEMS
    raw = np.asarray(W_buf, dtype=np.uint8).reshape(-1)[: nsb * N * SB_BYTES]
    return raw.reshape(nsb, N, SB_BYTES).transpose(1, 0, 2).reshape(-1)


def dequant_weights(W_buf, N: int, K: int) -> np.ndarray:
    """fp64 weights [N][K] of a matrix in the column-major super-block layout."""
    return dequant(weight_rows(W_buf, N, K), N, K)


def gemv(W_buf, x_bits, M: int, N: int, K: int):
    """Dequant-GEMV: ``y[m, n] = sum_k w[n, k] x[m, k]`` in fp64.

    ``W_buf``: the N x K weight matrix in the column-major super-block layout;
    ``x_bits``: bf16 bit patterns [M][K].  Returns ``(y, S)``, both float64
    [M][N], where ``S[m, n] = sum_k |w[n, k] x[m, k]|`` scales the parity
    tolerance.
    """
    w = dequant_weights(W_buf, N, K)
    x = bf16_bits_to_f64(np.asarray(x_bits).reshape(M, K))
    y = x @ w.T
    S = np.abs(x) @ np.abs(w).T
    return y, S


def gemv_tolerance(S: np.ndarray) -> np.ndarray:
    """Per-element bound ``2e-3 * S + 1e-5`` that the device result must meet."""
    return 2e-3 * S + 1e-5


def unpack_q8_superblocks(buf, rows: int, K: int):
    """Read ``rows`` rows of ``K`` Q8_0 elements from 272-byte super-blocks.

    Returns ``q`` (int64 [rows][K], values -128..127) and ``d`` (float64
    [rows][K/32])."""
    if K % SB_ELEMS:
        raise ValueError("K must be a multiple of 256")
    nsb = K // SB_ELEMS
    raw = np.asarray(buf, dtype=np.uint8).reshape(-1)
    need = rows * nsb * Q8_SB_BYTES
    if raw.size < need:
        raise ValueError(f"buffer holds {raw.size} bytes, need {need}")
    sb = raw[:need].reshape(rows, nsb, Q8_SB_BYTES)
    u = sb[:, :, :256].astype(np.int64)
    q = np.where(u >= 128, u - 256, u)                # two's complement bytes
    lo = sb[:, :, 256::2].astype(np.uint16)
    hi = sb[:, :, 257::2].astype(np.uint16)
    d_bits = lo | (hi << 8)                           # little endian fp16, block b at 256 + 2b
    return q.reshape(rows, K), f16_bits_to_f64(d_bits).reshape(rows, K // 32)


def dequant_q8(buf, rows: int, K: int) -> np.ndarray:
    """fp64 values ``d * q`` of ``rows x K`` Q8_0 elements."""
    q, d = unpack_q8_superblocks(buf, rows, K)
    return np.repeat(d, 32, axis=1) * q.astype(np.float64)


def _kv_hat(buf, n_kv: int, ctx_len: int, head_dim: int, kv_stride: int,
            fmt: str = "q4_0") -> np.ndarray:
    """Dequantised cache [n_kv][ctx_len][head_dim] (rows of one super-block
    per token when head_dim == 256; ``kv_stride`` tokens between heads)."""
    if fmt not in ("q4_0", "q8_0"):
        raise ValueError(f"unknown cache format {fmt!r}")
    sb_bytes, deq = (SB_BYTES, dequant) if fmt == "q4_0" else (Q8_SB_BYTES, dequant_q8)
    out = np.empty((n_kv, ctx_len, head_dim), dtype=np.float64)
    row_bytes = (head_dim // SB_ELEMS) * sb_bytes
    raw = np.asarray(buf, dtype=np.uint8).reshape(-1)
    for h in range(n_kv):
        start = h * kv_stride * row_bytes
        out[h] = deq(raw[start: start + ctx_len * row_bytes], ctx_len, head_dim)
    return out


def attn_probs(Q_bits, K_buf, ctx_len: int, n_q_heads: int, n_kv_heads: int,
               head_dim: int, M: int, kv_stride: int | None = None,
               scale: float = 1.0, fmt: str = "q4_0") -> np.ndarray:
    """Softmax weights ``P[m, h, t]`` (zero for masked tokens), fp64."""
    kv_stride = ctx_len if kv_stride is None else kv_stride
    g = n_q_heads // n_kv_heads
    Q = bf16_bits_to_f64(np.asarray(Q_bits).reshape(M, n_q_heads, head_dim))
    Kh = _kv_hat(K_buf, n_kv_heads, ctx_len, head_dim, kv_stride, fmt)
    P = np.zeros((M, n_q_heads, ctx_len), dtype=np.float64)
    for m in range(M):
        p_m = ctx_len - M + m                 # absolute position of draft row m
        for h in range(n_q_heads):
            kv = h // g
            s = scale * (Kh[kv, : p_m + 1] @ Q[m, h])
            e = np.exp(s - s.max())
            P[m, h, : p_m + 1] = e / e.sum()
    return P


def attn_decode(Q_bits, K_buf, V_buf, ctx_len: int, n_q_heads: int, n_kv_heads: int,
                head_dim: int, M: int, kv_stride: int | None = None,
                scale: float = 1.0, fmt: str = "q4_0") -> np.ndarray:
    """Causal GQA decode attention over a Q4_0 (or, ``fmt="q8_0"``, Q8_0) K/V
    cache, fp64.

    Returns ``out[m, h, :] = sum_t P[m, h, t] * V_hat[h // g, t, :]``.
    """
    kv_stride = ctx_len if kv_stride is None else kv_stride
    g = n_q_heads // n_kv_heads
    P = attn_probs(Q_bits, K_buf, ctx_len, n_q_heads, n_kv_heads, head_dim, M,
                   kv_stride, scale, fmt)
    Vh = _kv_hat(V_buf, n_kv_heads, ctx_len, head_dim, kv_stride, fmt)
    out = np.empty((M, n_q_heads, head_dim), dtype=np.float64)
    for m in range(M):
        for h in range(n_q_heads):
            out[m, h] = P[m, h] @ Vh[h // g]
    return out


def quantize_q4_0_rows(v) -> np.ndarray:
    """Quantise fp32 rows ``v[rows][K]`` (K % 256 == 0) into super-blocks in
    row order (the K/V layout), following the K/V append reading above: the
    codes are decided in fp32 (numpy float32 division and addition, each
    rounded to nearest), the scale is rounded to fp16."""
    v = np.asarray(v, dtype=np.float32)
    rows, K = v.shape
    if K % SB_ELEMS:
        raise ValueError("K must be a multiple of 256")
    out = np.zeros((rows, K // SB_ELEMS, SB_BYTES), dtype=np.uint8)
    for r in range(rows):
        for blk in range(K // 32):
            vals = v[r, 32 * blk: 32 * blk + 32]
            i = int(np.argmax(np.abs(vals)))            # first index of the largest |v|
            d16 = np.float16(vals[i] / np.float32(-8.0))
            if d16 == 0:
                d16 = np.float16(0.0)                   # +0, and every code 8
                q = np.full(32, 8, dtype=np.int64)
            else:
                d32 = np.float32(d16)
                q = np.floor(vals / d32 + np.float32(8.5)).astype(np.int64)
                q = np.clip(q, 0, 15)
            s_, b = divmod(blk, 8)
            sb = out[r, s_]
            sb[16 * b: 16 * b + 16] = (q[:16] | (q[16:] << 4)).astype(np.uint8)
            sb[128 + 2 * b: 130 + 2 * b] = np.array([d16], dtype=np.float16).view(np.uint8)
    return out.reshape(-1)


def kv_append(K_buf, V_buf, k_new, v_new, n_kv_heads: int, kv_stride: int, pos: int, M: int):
    """Caches after appending M tokens at positions pos .. pos+M-1 of every KV
    head: token m of head h gets quantize_q4_0_rows(new[m][h]).  ``k_new`` /
    ``v_new``: fp32 [M][n_kv_heads][256].  Returns new (K, V) byte arrays."""
    outs = []
    for buf, new in ((K_buf, k_new), (V_buf, v_new)):
        b = np.array(buf, dtype=np.uint8).reshape(-1).copy()
        new = np.asarray(new, dtype=np.float32).reshape(M, n_kv_heads, SB_ELEMS)
        for m in range(M):
            for h in range(n_kv_heads):
                at = (h * kv_stride + pos + m) * SB_BYTES
                b[at: at + SB_BYTES] = quantize_q4_0_rows(new[m, h][None, :])
        outs.append(b)
    return outs[0], outs[1]


def silu(g):
    """``g / (1 + exp(-g))`` in fp64 (written so that it does not overflow)."""
    g = np.asarray(g, dtype=np.float64)
    out = np.empty_like(g)
    pos = g >= 0
    out[pos] = g[pos] / (1.0 + np.exp(-g[pos]))
    e = np.exp(g[~pos])
    out[~pos] = g[~pos] * e / (1.0 + e)
    return out


def silu_prime(g):
    """d/dg silu(g) = s + g s (1 - s), s = 1 / (1 + e^-g), in fp64."""
    g = np.asarray(g, dtype=np.float64)
    s = 1.0 / (1.0 + np.exp(-np.clip(g, -700.0, 700.0)))
    return s * (1.0 + g * (1.0 - s))


def _silu_prime_critical_point() -> float:
    """The positive root of silu''(g) = s(1 - s)(2 - g tanh(g / 2)), i.e. of
    g tanh(g / 2) = 2 (increasing in g > 0), by bisection in fp64.  silu' has
    its only extrema at +-this point (a maximum at +, a minimum at -)."""
    lo, hi = 1.0, 4.0
    for _ in range(200):
        mid = 0.5 * (lo + hi)
        if mid * np.tanh(mid / 2.0) < 2.0:
            lo = mid
        else:
            hi = mid
    return 0.5 * (lo + hi)


SILU_PRIME_CRIT = _silu_prime_critical_point()

# Relative error of the device's fp32 SwiGLU epilogue h = g / (1 + expf(-g)) * u
# for given fp32 g and u: expf is documented to 2 ulp (2 * 2^-23 relative),
# and the add, the IEEE division and the multiply each round once to nearest
# (2^-24 relative each); the errors compound to at most
# (1 + 2^-22)(1 + 2^-24)^3 - 1 < 7 * 2^-24 * (1 + 1e-6).
SWIGLU_EPILOGUE_REL = 7.0 * 2.0 ** -24 * (1.0 + 1e-6)


def silu_prime_max(g, t):
    """max |silu'(xi)| over xi in [g - t, g + t]: silu' is monotonic between
    its extrema at -SILU_PRIME_CRIT and +SILU_PRIME_CRIT, so the maximum of
    its magnitude is at an end of the interval or at an extremum inside it."""
    g, t = np.broadcast_arrays(np.asarray(g, dtype=np.float64), np.asarray(t, dtype=np.float64))
    lo, hi = g - t, g + t
    best = np.maximum(np.abs(silu_prime(lo)), np.abs(silu_prime(hi)))
    for c in (-SILU_PRIME_CRIT, SILU_PRIME_CRIT):
        inside = (lo <= c) & (c <= hi)
        best = np.where(inside, np.maximum(best, abs(float(silu_prime(c)))), best)
    return best


def swiglu_tolerance(g, u, tg, tu):
    """Bound on |h_dev - silu(g) u| when the device computed g and u to within
    tg and tu (the GEMV bound) and then evaluated the SwiGLU epilogue in fp32.

    With g~ = g + dg, u~ = u + du (|dg| <= tg, |du| <= tu):
      silu(g~) u~ - silu(g) u = (silu(g~) - silu(g)) u~ + silu(g) du,
    and by the mean value theorem |silu(g~) - silu(g)| <= D tg with
    D = max |silu'| over [g - tg, g + tg] (D <= |silu'(g)| + tg / 2, since
    |silu''| <= 1/2); |u~| <= |u| + tu.  So
      |dh| <= D tg (|u| + tu) + |silu(g)| tu:
    the first-order terms |silu'(g) u| tg + |silu(g)| tu, the cross term
    D tg tu, and the curvature of silu over the interval through D.  The fp32
    epilogue adds SWIGLU_EPILOGUE_REL times a bound on |silu(g~) u~|, and 1e-30
    absolute covers fp32 underflow of silu(g~) for g~ < -87."""
    g, u = np.asarray(g, dtype=np.float64), np.asarray(u, dtype=np.float64)
    dsilu_span = silu_prime_max(g, tg) * tg
    u_span = np.abs(u) + tu
    prop = dsilu_span * u_span + np.abs(silu(g)) * tu
    h_max = (np.abs(silu(g)) + dsilu_span) * u_span
    return prop + SWIGLU_EPILOGUE_REL * h_max + 1e-30 * u_span


def gemv_swiglu(W_buf, x_bits, M: int, N: int, K: int):
    """Fused gate/up GEMV + SwiGLU: ``W_buf`` holds 2N rows in the weight
    layout (gate row n at 2n, up row n at 2n + 1).  Returns ``(h, tol)``:
    ``h[m, n] = silu(g) * u`` in fp64 and the per-element bound the device
    result must meet: the GEMV bound ``t = 2e-3 S + 1e-5`` of g and of u,
    carried through the SwiGLU by ``swiglu_tolerance``."""
    y, S = gemv(W_buf, x_bits, M, 2 * N, K)
    g, u = y[:, 0::2], y[:, 1::2]
    tg, tu = gemv_tolerance(S[:, 0::2]), gemv_tolerance(S[:, 1::2])
    h = silu(g) * u
    return h, swiglu_tolerance(g, u, tg, tu)
