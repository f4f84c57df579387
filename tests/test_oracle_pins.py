"""Pins for the CPU oracle: each test ties it to something other than itself --
a hand-worked fixture, literal bit patterns, closed forms, invariants, or a
brute-force pure-Python evaluation with exact rational arithmetic."""
import math
import os
from fractions import Fraction

import numpy as np
import pytest

import oracle
import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ----------------------------------------------------------------- helpers ---
def _fraction_bf16(bits: int) -> Fraction:
    """Exact value of a bf16 bit pattern by the IEEE binary32 field definition
    (sign, 8-bit exponent, 7 stored fraction bits), in rationals."""
    sign = -1 if bits & 0x8000 else 1
    exp = (bits >> 7) & 0xFF
    frac = bits & 0x7F
    if exp == 0:
        return sign * Fraction(frac, 128) * Fraction(2) ** (-126)
    return sign * (1 + Fraction(frac, 128)) * Fraction(2) ** (exp - 127)


def _fraction_f16(bits: int) -> Fraction:
    """Exact value of an IEEE binary16 bit pattern (5-bit exponent, 10 bits)."""
    sign = -1 if bits & 0x8000 else 1
    exp = (bits >> 10) & 0x1F
    frac = bits & 0x3FF
    if exp == 0:
        return sign * Fraction(frac, 1024) * Fraction(2) ** (-14)
    return sign * (1 + Fraction(frac, 1024)) * Fraction(2) ** (exp - 15)


def _brute_weights(buf, rows, K, column_major=False):
    """Pure-Python reading of the super-block layout, in rationals: rows of
    consecutive super-blocks (K/V caches), or the weight layout where
    super-block (r, s) sits at (s * rows + r) * 144."""
    raw = bytes(np.asarray(buf, dtype=np.uint8).tobytes())
    nsb = K // 256
    w = [[Fraction(0)] * K for _ in range(rows)]
    for r in range(rows):
        for s in range(nsb):
            base = ((s * rows + r) if column_major else (r * nsb + s)) * 144
            for b in range(8):
                d = _fraction_f16(raw[base + 128 + 2 * b] | (raw[base + 129 + 2 * b] << 8))
                for j in range(16):
                    byte = raw[base + 16 * b + j]
                    k0 = s * 256 + b * 32
                    w[r][k0 + j] = d * ((byte & 15) - 8)
                    w[r][k0 + j + 16] = d * ((byte >> 4) - 8)
    return w


# ------------------------------------------------------- number formats ----
def test_bf16_literal_values():
    cases = {0x3F80: 1.0, 0xBF80: -1.0, 0x4049: 3.140625, 0x3E20: 0.15625,
             0x0000: 0.0, 0x0001: 2.0 ** -133, 0x0080: 2.0 ** -126,
             0x7F7F: 3.3895313892515355e38, 0xC2F7: -123.5}
    got = oracle.bf16_bits_to_f64(np.array(list(cases), dtype=np.uint16))
    assert list(got) == list(cases.values())


def test_f16_literal_values():
    cases = {0x3800: 0.5, 0x3C00: 1.0, 0xB400: -0.25, 0x0001: 2.0 ** -24,
             0x0400: 2.0 ** -14, 0x7BFF: 65504.0, 0xC500: -5.0, 0x2E66: 0.0999755859375}
    got = oracle.f16_bits_to_f64(np.array(list(cases), dtype=np.uint16))
    assert list(got) == list(cases.values())


def test_bf16_decode_matches_field_definition_exhaustively():
    bits = np.arange(0, 1 << 16, dtype=np.uint32).astype(np.uint16)
    finite = ((bits.astype(np.uint32) >> 7) & 0xFF) != 0xFF
    got = oracle.bf16_bits_to_f64(bits[finite])
    sample = np.random.default_rng(5).choice(np.flatnonzero(finite), 2000, replace=False)
    for i in sample:
        b = int(bits[i])
        assert Fraction(got[np.searchsorted(np.flatnonzero(finite), i)]) == _fraction_bf16(b)


def test_rounding_helpers_are_nearest_even():
    # 1 + 2^-8 is halfway between bf16 1.0 and 1.0078125 -> ties to even (1.0)
    v = np.array([1 + 2 ** -8, 1 + 3 * 2 ** -8, -2.5, 1e-3], dtype=np.float32)
    bits = synth.f32_to_bf16_bits(v)
    assert list(bits[:3]) == [0x3F80, 0x3F82, 0xC020]
    assert abs(oracle.bf16_bits_to_f64(bits[3:])[0] - 1e-3) <= 2 ** -9 * 1e-3


# ---------------------------------------------------------- Q4_0 layout ----
def _read_golden():
    blocks, expect = [], []
    with open(os.path.join(GOLDEN, "q4_0_superblock_worked.txt")) as f:
        lines = [ln.strip() for ln in f if ln.strip() and not ln.startswith("#")]
    for head, vals in zip(lines[0::2], lines[1::2]):
        parts = dict(p.split("=") for p in head.split()[2:])
        blocks.append((int(parts["d"], 16), bytes.fromhex(parts["bytes"])))
        expect.extend(float(v) for v in vals.split())
    return blocks, expect


def test_worked_superblock_fixture():
    blocks, expect = _read_golden()
    assert len(blocks) == 8 and len(expect) == 256
    sb = bytearray(144)
    for b, (dbits, qs) in enumerate(blocks):
        sb[16 * b: 16 * b + 16] = qs
        sb[128 + 2 * b] = dbits & 0xFF
        sb[129 + 2 * b] = dbits >> 8
    w = oracle.dequant(np.frombuffer(bytes(sb), dtype=np.uint8), 1, 256)
    assert list(w[0]) == expect


def test_pack_unpack_roundtrip():
    rng = np.random.default_rng(11)
    q = rng.integers(0, 16, size=(7, 768), dtype=np.uint8)
    dbits = rng.integers(0, 0x7C00, size=(7, 24)).astype(np.uint16)
    buf = synth.pack_superblocks(q, dbits)
    assert buf.size == 7 * 3 * 144
    q2, d2 = oracle.unpack_superblocks(buf, 7, 768)
    assert np.array_equal(q2, q)
    assert np.array_equal(d2, oracle.f16_bits_to_f64(dbits))


def test_superblock_offsets_single_nibble():
    # one nonzero nibble (q = 9, all others q = 8) at row 2, super-block 1,
    # block 5, byte 3, high nibble -> element 256 + 5*32 + 3 + 16 only
    N, K = 4, 512
    q = np.full((N, K), 8, dtype=np.uint8)
    d = np.full((N, K // 32), 0.5, dtype=np.float32)
    q[2, 256 + 5 * 32 + 3 + 16] = 9
    buf = synth.from_parts(q, d)
    raw = buf.reshape(N, 2, 144)
    assert raw[2, 1, 16 * 5 + 3] == (8 | (9 << 4))
    w = oracle.dequant(buf, N, K)
    nz = np.argwhere(w != 0)
    assert nz.tolist() == [[2, 256 + 5 * 32 + 3 + 16]] and w[2, 435] == 0.5


def test_oracle_reading_matches_bruteforce_reader():
    rows = synth.pack_superblocks(np.random.default_rng(21).integers(0, 16, size=(3, 512)),
                                  np.random.default_rng(22).integers(0, 0x7C00, size=(3, 16)))
    w = oracle.dequant(rows, 3, 512)
    wb = _brute_weights(rows, 3, 512)
    for r in range(3):
        assert [Fraction(v) for v in w[r]] == wb[r]
    buf = synth.q4_0_weights(21, 5, 768)
    w = oracle.dequant_weights(buf, 5, 768)
    wb = _brute_weights(buf, 5, 768, column_major=True)
    for r in range(5):
        assert [Fraction(v) for v in w[r]] == wb[r]


def test_weight_layout_single_nibble():
    # weights are super-block-column-major: super-block (n, s) at (s*N + n)*144
    N, K = 4, 768
    q = np.full((N, K), 8, dtype=np.uint8)
    d = np.full((N, K // 32), 0.25, dtype=np.float32)
    q[2, 256 + 3 * 32 + 5] = 12                     # row 2, super-block 1, block 3, byte 5 lo
    buf = synth.weights_from_parts(q, d)
    assert buf.size == N * 3 * 144
    off = (1 * N + 2) * 144 + 16 * 3 + 5
    assert buf[off] == (12 | (8 << 4))
    assert np.count_nonzero(buf.reshape(-1, 144)[:, :128] != 0x88) == 1
    w = oracle.dequant_weights(buf, N, K)
    assert np.argwhere(w != 0).tolist() == [[2, 256 + 3 * 32 + 5]] and w[2, 357] == 1.0
    assert np.array_equal(oracle.weight_rows(buf, N, K).reshape(N, 3, 144)[2, 1],
                          buf.reshape(3, N, 144)[1, 2])


# ----------------------------------------------------------------- GEMV ----
def test_one_hot_x_picks_one_weight_column():
    N, K = 5, 512
    buf = synth.q4_0_weights(3, N, K)
    w = oracle.dequant_weights(buf, N, K)
    for k in (0, 17, 31, 32, 255, 256, 511):
        x = np.zeros((1, K), dtype=np.uint16)
        x[0, k] = 0x3F80  # 1.0
        y, S = oracle.gemv(buf, x, 1, N, K)
        assert np.array_equal(y[0], w[:, k]) and np.array_equal(S[0], np.abs(w[:, k]))


def test_all_q8_gives_exact_zero():
    N, K, M = 6, 1024, 3
    q = np.full((N, K), 8, dtype=np.uint8)
    d = np.abs(np.random.default_rng(1).standard_normal((N, K // 32))).astype(np.float32)
    buf = synth.weights_from_parts(q, d)
    x = synth.activations(2, M, K)
    y, S = oracle.gemv(buf, x, M, N, K)
    assert np.all(y == 0.0) and np.all(S == 0.0)


def test_linear_in_one_block_scale():
    # dyadic values keep every fp64 operation exact, so the change must equal
    # the one block's contribution exactly
    N, K = 3, 512
    rng = np.random.default_rng(4)
    q = rng.integers(0, 16, size=(N, K), dtype=np.uint8)
    d = (2.0 ** -rng.integers(1, 6, size=(N, K // 32))).astype(np.float32)
    x = synth.f32_to_bf16_bits(rng.integers(-4, 5, size=(1, K)).astype(np.float32))
    y0, _ = oracle.gemv(synth.weights_from_parts(q, d), x, 1, N, K)
    b = 9
    d2 = d.copy()
    d2[:, b] *= 2
    y1, _ = oracle.gemv(synth.weights_from_parts(q, d2), x, 1, N, K)
    xs = oracle.bf16_bits_to_f64(x)[0, 32 * b: 32 * b + 32]
    contrib = (d[:, b:b + 1].astype(np.float64) * (q[:, 32 * b:32 * b + 32] - 8.0)) @ xs
    assert np.array_equal(y1[0] - y0[0], contrib)


def test_linear_in_x():
    N, K = 4, 768
    rng = np.random.default_rng(8)
    buf = synth.weights_from_parts(rng.integers(0, 16, size=(N, K), dtype=np.uint8),
                                   (2.0 ** -rng.integers(2, 8, size=(N, K // 32))).astype(np.float32))
    a = rng.integers(-3, 4, size=(1, K)).astype(np.float32)
    b = rng.integers(-3, 4, size=(1, K)).astype(np.float32)
    ya, _ = oracle.gemv(buf, synth.f32_to_bf16_bits(a), 1, N, K)
    yb, _ = oracle.gemv(buf, synth.f32_to_bf16_bits(b), 1, N, K)
    yab, _ = oracle.gemv(buf, synth.f32_to_bf16_bits(3 * a + b), 1, N, K)
    assert np.array_equal(yab, 3 * ya + yb)


def test_rows_are_independent():
    N, K, M = 8, 512, 5
    buf = synth.q4_0_weights(12, N, K)
    x = synth.activations(13, M, K)
    y5, _ = oracle.gemv(buf, x, M, N, K)
    for m in range(M):
        y1, _ = oracle.gemv(buf, x[m:m + 1], 1, N, K)
        assert np.array_equal(y1[0], y5[m])


def test_exact_integer_case_against_python_ints():
    # d = 2^-k and small-integer x make y an exact dyadic rational
    N, K, M = 4, 512, 2
    rng = np.random.default_rng(31)
    q = rng.integers(0, 16, size=(N, K), dtype=np.uint8)
    kexp = rng.integers(0, 6, size=(N, K // 32))
    xi = rng.integers(-7, 8, size=(M, K))
    buf = synth.weights_from_parts(q, (2.0 ** -kexp).astype(np.float32))
    y, _ = oracle.gemv(buf, synth.f32_to_bf16_bits(xi.astype(np.float32)), M, N, K)
    for m in range(M):
        for n in range(N):
            ref = sum(Fraction(int(q[n, k]) - 8, 2 ** int(kexp[n, k // 32])) * int(xi[m, k])
                      for k in range(K))
            assert Fraction(y[m, n]) == ref


def test_gemv_against_rational_bruteforce():
    N, K, M = 3, 256, 2
    buf = synth.q4_0_weights(41, N, K)
    x = synth.activations(42, M, K)
    y, S = oracle.gemv(buf, x, M, N, K)
    w = _brute_weights(buf, N, K, column_major=True)
    for m in range(M):
        xs = [_fraction_bf16(int(b)) for b in x[m]]
        for n in range(N):
            exact = sum(wk * xk for wk, xk in zip(w[n], xs))
            sabs = sum(abs(wk * xk) for wk, xk in zip(w[n], xs))
            assert abs(Fraction(y[m, n]) - exact) <= Fraction(1, 10 ** 12) * (sabs + 1)
            assert abs(Fraction(S[m, n]) - sabs) <= Fraction(1, 10 ** 12) * (sabs + 1)


def test_tolerance_formula():
    S = np.array([[0.0, 1.0, 250.0]])
    assert np.allclose(oracle.gemv_tolerance(S), [[1e-5, 2e-3 + 1e-5, 0.5 + 1e-5]])


# ------------------------------------------------------------- attention ----
def _kv_from_parts(q, d):
    return synth.from_parts(q, d)


def _attn_case(seed, ctx, n_q, n_kv, M):
    K = synth.q4_0_kv_cache(seed, n_kv, ctx)
    V = synth.q4_0_kv_cache(seed + 1, n_kv, ctx)
    Q = synth.queries(seed + 2, M, n_q)
    return Q, K, V


def test_softmax_rows_sum_to_one_and_mask():
    ctx, n_q, n_kv, M = 40, 6, 2, 5
    Q, K, _ = _attn_case(3, ctx, n_q, n_kv, M)
    P = oracle.attn_probs(Q, K, ctx, n_q, n_kv, 256, M)
    assert np.allclose(P.sum(-1), 1.0, rtol=0, atol=1e-14)
    for m in range(M):
        assert np.all(P[m, :, ctx - M + m + 1:] == 0) and np.all(P[m, :, : ctx - M + m + 1] > 0)


def test_all_keys_q8_gives_mean_of_visible_values():
    ctx, n_q, n_kv, M = 23, 4, 2, 3
    kq = np.full((n_kv * ctx, 256), 8, dtype=np.uint8)
    K = _kv_from_parts(kq, np.ones((n_kv * ctx, 8), dtype=np.float32))
    V = synth.q4_0_kv_cache(7, n_kv, ctx)
    Q = synth.queries(8, M, n_q)
    out = oracle.attn_decode(Q, K, V, ctx, n_q, n_kv, 256, M)
    Vh = oracle.dequant(V, n_kv * ctx, 256).reshape(n_kv, ctx, 256)
    for m in range(M):
        vis = ctx - M + m + 1
        for h in range(n_q):
            mean = [math.fsum(Vh[h // 2, t, c] for t in range(vis)) / vis for c in range(256)]
            assert np.allclose(out[m, h], mean, rtol=0, atol=1e-13)


def test_constant_values_give_that_constant():
    ctx, n_q, n_kv, M = 31, 6, 3, 2
    vq = np.full((n_kv * ctx, 256), 11, dtype=np.uint8)          # q - 8 = 3
    V = _kv_from_parts(vq, np.full((n_kv * ctx, 8), 0.25, dtype=np.float32))
    Q, K, _ = _attn_case(9, ctx, n_q, n_kv, M)
    out = oracle.attn_decode(Q, K, V, ctx, n_q, n_kv, 256, M)
    assert np.allclose(out, 0.75, rtol=0, atol=1e-14)


def test_single_token_returns_its_value_row():
    Q, K, V = _attn_case(15, 1, 4, 1, 1)
    out = oracle.attn_decode(Q, K, V, 1, 4, 1, 256, 1)
    Vh = oracle.dequant(V, 1, 256)
    assert np.array_equal(out[0], np.repeat(Vh, 4, axis=0))


def test_dominant_key_selects_its_value():
    ctx, M = 16, 1
    kq = np.full((ctx, 256), 8, dtype=np.uint8)
    kq[5, :] = 15                                    # q - 8 = 7 on every dim
    K = _kv_from_parts(kq, np.full((ctx, 8), 1.0, dtype=np.float32))
    V = synth.q4_0_kv_cache(17, 1, ctx)
    Q = synth.f32_to_bf16_bits(np.full((1, 1, 256), 1.0, dtype=np.float32))
    out = oracle.attn_decode(Q, K, V, ctx, 1, 1, 256, M)     # logit gap 7*256
    Vh = oracle.dequant(V, ctx, 256)
    assert np.array_equal(out[0, 0], Vh[5])


def test_causal_rows_ignore_later_tokens():
    ctx, n_q, n_kv, M = 20, 6, 2, 5
    Q, K, V = _attn_case(19, ctx, n_q, n_kv, M)
    base = oracle.attn_decode(Q, K, V, ctx, n_q, n_kv, 256, M)
    # perturb the last token (position ctx-1) of every head: only row M-1 sees it
    K2 = K.copy().reshape(n_kv, ctx, 144)
    V2 = V.copy().reshape(n_kv, ctx, 144)
    K2[:, ctx - 1, :128] ^= 0x5A
    V2[:, ctx - 1, :128] ^= 0xA5
    pert = oracle.attn_decode(Q, K2.reshape(-1), V2.reshape(-1), ctx, n_q, n_kv, 256, M)
    assert np.array_equal(pert[: M - 1], base[: M - 1])
    assert not np.allclose(pert[M - 1], base[M - 1])


def test_gqa_head_mapping_is_contiguous_groups():
    ctx, n_q, n_kv, M = 9, 6, 3, 1
    vq = np.concatenate([np.full((ctx, 256), 8 + h, dtype=np.uint8) for h in range(n_kv)])
    V = _kv_from_parts(vq, np.ones((n_kv * ctx, 8), dtype=np.float32))
    Q, K, _ = _attn_case(23, ctx, n_q, n_kv, M)
    out = oracle.attn_decode(Q, K, V, ctx, n_q, n_kv, 256, M)
    for h in range(n_q):
        assert np.allclose(out[0, h], h // 2, rtol=0, atol=1e-14)


def test_mha_equals_independent_single_heads():
    ctx, n, M = 12, 3, 2
    Q, K, V = _attn_case(29, ctx, n, n, M)
    out = oracle.attn_decode(Q, K, V, ctx, n, n, 256, M)
    Kr, Vr = K.reshape(n, ctx * 144), V.reshape(n, ctx * 144)
    Qr = Q.reshape(M, n, 256)
    for h in range(n):
        one = oracle.attn_decode(Qr[:, h:h + 1].copy(), Kr[h], Vr[h], ctx, 1, 1, 256, M)
        assert np.array_equal(one[:, 0], out[:, h])


def test_softmax_scale_equals_scaled_queries():
    ctx, n_q, n_kv, M = 14, 4, 2, 2
    Q, K, V = _attn_case(33, ctx, n_q, n_kv, M)
    Q2 = synth.f32_to_bf16_bits(2 * oracle.bf16_bits_to_f64(Q).astype(np.float32))
    a = oracle.attn_decode(Q, K, V, ctx, n_q, n_kv, 256, M, scale=2.0)
    b = oracle.attn_decode(Q2, K, V, ctx, n_q, n_kv, 256, M)
    assert np.allclose(a, b, rtol=0, atol=1e-13)


def test_kv_stride_reads_the_right_rows():
    ctx, cap, n_q, n_kv, M = 10, 16, 4, 2, 2
    Kf = synth.q4_0_kv_cache(35, n_kv, cap)
    Vf = synth.q4_0_kv_cache(36, n_kv, cap)
    Q = synth.queries(37, M, n_q)
    out = oracle.attn_decode(Q, Kf, Vf, ctx, n_q, n_kv, 256, M, kv_stride=cap)
    Kc = Kf.reshape(n_kv, cap, 144)[:, :ctx].reshape(-1)
    Vc = Vf.reshape(n_kv, cap, 144)[:, :ctx].reshape(-1)
    ref = oracle.attn_decode(Q, Kc, Vc, ctx, n_q, n_kv, 256, M)
    assert np.array_equal(out, ref)


def test_attention_against_python_bruteforce():
    ctx, n_q, n_kv, M = 7, 4, 2, 3
    Q, K, V = _attn_case(39, ctx, n_q, n_kv, M)
    out = oracle.attn_decode(Q, K, V, ctx, n_q, n_kv, 256, M)
    Kw = _brute_weights(K, n_kv * ctx, 256)
    Vw = _brute_weights(V, n_kv * ctx, 256)
    Qf = np.asarray(Q).reshape(M, n_q, 256)
    for m in range(M):
        vis = ctx - M + m + 1
        for h in range(n_q):
            kv = h // (n_q // n_kv)
            q = [_fraction_bf16(int(b)) for b in Qf[m, h]]
            s = [float(sum(a * b for a, b in zip(q, Kw[kv * ctx + t]))) for t in range(vis)]
            mx = max(s)
            e = [math.exp(v - mx) for v in s]
            z = math.fsum(e)
            for c in range(0, 256, 37):
                ref = math.fsum(e[t] * float(Vw[kv * ctx + t][c]) for t in range(vis)) / z
                assert out[m, h, c] == pytest.approx(ref, abs=1e-12)


def test_quantizer_recipe_on_literal_block():
    v = np.zeros((1, 256), dtype=np.float32)
    v[0, :32] = np.linspace(-1.0, 2.0, 32, dtype=np.float32)   # amax = +2.0
    q, d = synth.quantize_blocks(v)
    assert d[0, 0] == 0xB400                                    # fp16(-0.25)
    assert q[0, 31] == 0 and q[0, 0] == 12                      # 2/-0.25+8.5 -> 0; -1/-0.25+8.5 -> 12
    assert np.all(q[0, 32:] == 8) and np.all(d[0, 1:] == 0)


# ---------------------------------------------------------------- K/V append
def _one_block_row(vals):
    """A 256-element row whose first block is ``vals`` and the rest zero."""
    row = np.zeros((1, 256), dtype=np.float32)
    row[0, :len(vals)] = vals
    return row


def test_quantizer_hand_worked_block():
    # amax = -4 (largest |v|, negative) -> d = -4 / -8 = 0.5 (exact in fp16);
    # q = floor(v / 0.5 + 8.5): -4 -> 0, -3.9 -> 0 (floor(0.7)), 0 -> 8,
    # 0.25 -> 9, 3.5 -> 15, 3.74 -> 15 (floor(15.98)), 3.76 -> 16 -> clamp 15,
    # -0.26 -> floor(7.98) = 7, 1.0 -> 10, -1.25 -> floor(6.0) = 6
    vals = [-4.0, -3.9, 0.0, 0.25, 3.5, 3.74, 3.76, -0.26, 1.0, -1.25]
    sb = oracle.quantize_q4_0_rows(_one_block_row(vals))
    q = np.concatenate([sb[0:16] & 0x0F, sb[0:16] >> 4])
    assert list(q[:10]) == [0, 0, 8, 9, 15, 15, 15, 7, 10, 6]
    assert all(q[10:] == 8)                                 # zeros -> code 8
    assert sb[128:130].view(np.float16)[0] == np.float16(0.5)
    # blocks 1..7 are all-zero: d = +0 (bits 0x0000), every code 8
    assert all(sb[16:128] == 0x88) and all(sb[130:144] == 0)


def test_quantizer_positive_amax_flips_sign_and_maps_exactly():
    # amax = +2 -> d = -0.25; the amax element itself maps to q = 0, i.e.
    # -0.25 * (0 - 8) = 2 exactly; -2 maps to q = 16 -> 15 (one step short)
    vals = [2.0, -2.0, 0.5, -0.5]
    sb = oracle.quantize_q4_0_rows(_one_block_row(vals))
    q = np.concatenate([sb[0:16] & 0x0F, sb[0:16] >> 4])
    assert list(q[:4]) == [0, 15, 6, 10]
    assert sb[128:130].view(np.float16)[0] == np.float16(-0.25)
    w = oracle.dequant(sb, 1, 256)[0]
    assert w[0] == 2.0 and w[1] == -1.75 and w[2] == 0.5 and w[3] == -0.5


def test_quantizer_ties_take_the_first_index_and_zero_block_stores_plus_zero():
    sb = oracle.quantize_q4_0_rows(_one_block_row([-3.0, 3.0]))
    assert sb[128:130].view(np.float16)[0] == np.float16(0.375)   # from -3 (first)
    z = oracle.quantize_q4_0_rows(np.zeros((1, 256), dtype=np.float32))
    assert all(z[:128] == 0x88) and all(z[128:] == 0)
    # -0.0 everywhere is an all-zero block too: d = +0, not -0
    nz = oracle.quantize_q4_0_rows(np.full((1, 256), -0.0, dtype=np.float32))
    assert all(nz[128:] == 0)


def test_quantizer_error_bound_on_random_rows():
    # |dequant(quant(v)) - v| <= |d| / 2, except the clamped top code (<= |d|)
    rng = np.random.default_rng(9)
    v = rng.standard_normal((6, 512)).astype(np.float32) * np.float32(3.0)
    sb = oracle.quantize_q4_0_rows(v)
    w = oracle.dequant(sb, 6, 512)
    _, d = oracle.unpack_superblocks(sb, 6, 512)
    dd = np.repeat(np.abs(d), 32, axis=1)
    err = np.abs(w - v.astype(np.float64))
    assert np.all(err <= dd * 1.0 + 1e-12)
    assert np.mean(err <= dd * 0.5 + 1e-12) > 0.95


def test_kv_append_writes_only_the_target_tokens():
    n_kv, stride, pos, M = 2, 10, 3, 2
    K0 = np.arange(n_kv * stride * 144, dtype=np.int64).astype(np.uint8)
    V0 = K0[::-1].copy()
    rng = np.random.default_rng(4)
    kn = rng.standard_normal((M, n_kv, 256)).astype(np.float32)
    vn = rng.standard_normal((M, n_kv, 256)).astype(np.float32)
    K1, V1 = oracle.kv_append(K0, V0, kn, vn, n_kv, stride, pos, M)
    for h in range(n_kv):
        for t in range(stride):
            at = slice((h * stride + t) * 144, (h * stride + t + 1) * 144)
            if pos <= t < pos + M:
                assert np.array_equal(K1[at], oracle.quantize_q4_0_rows(kn[t - pos, h][None]))
                assert np.array_equal(V1[at], oracle.quantize_q4_0_rows(vn[t - pos, h][None]))
            else:
                assert np.array_equal(K1[at], K0[at]) and np.array_equal(V1[at], V0[at])


# ------------------------------------------------------- gate/up + SwiGLU
def test_silu_closed_forms():
    g = np.array([0.0, 1.0, -1.0, 40.0, -40.0, 800.0, -800.0])
    s = oracle.silu(g)
    assert s[0] == 0.0
    assert abs(s[1] - 1.0 / (1.0 + math.exp(-1.0))) < 1e-15
    assert abs(s[2] - (-1.0) / (1.0 + math.exp(1.0))) < 1e-15
    assert abs(s[3] - 40.0) < 1e-12 and abs(s[4]) < 1e-15
    assert s[5] == 800.0
    assert abs(s[6]) < 1e-300


def test_gemv_swiglu_composes_two_plain_gemvs():
    # interleaving gate and up rows and fusing must equal silu(gate GEMV) * up GEMV
    N, K, M = 6, 512, 2
    Wg = synth.q4_0_weights(31, N, K)
    Wu = synth.q4_0_weights(32, N, K)
    x = synth.activations(33, M, K)
    rows_g = oracle.weight_rows(Wg, N, K).reshape(N, -1)
    rows_u = oracle.weight_rows(Wu, N, K).reshape(N, -1)
    inter = np.empty((2 * N, rows_g.shape[1]), dtype=np.uint8)
    inter[0::2], inter[1::2] = rows_g, rows_u
    Wgu = synth.column_major(inter.reshape(-1), 2 * N, K)
    h, tol = oracle.gemv_swiglu(Wgu, x, M, N, K)
    g, _ = oracle.gemv(Wg, x, M, N, K)
    u, _ = oracle.gemv(Wu, x, M, N, K)
    np.testing.assert_allclose(h, oracle.silu(g) * u, rtol=0, atol=1e-12)
    assert np.all(tol > 0)


def test_gemv_swiglu_hand_worked():
    # K = 256, one row pair: gate weights all d * (q - 8) = 0.5 * 1 on element 0
    # only (others q = 8), up weights 0.25 * (-2) on element 1 only; x[0] = 2,
    # x[1] = 3: g = 1.0, u = -1.5, h = silu(1) * -1.5
    q = np.full((2, 256), 8, dtype=np.uint8)
    q[0, 0] = 9
    q[1, 1] = 6
    d = np.zeros((2, 8), dtype=np.float32)
    d[0, 0] = 0.5
    d[1, 0] = 0.25
    W = synth.weights_from_parts(q, d)
    x = np.zeros((1, 256), dtype=np.float32)
    x[0, 0], x[0, 1] = 2.0, 3.0
    xb = synth.f32_to_bf16_bits(x)
    h, _ = oracle.gemv_swiglu(W, xb, 1, 1, 256)
    assert abs(h[0, 0] - (1.0 / (1.0 + math.exp(-1.0))) * -1.5) < 1e-15


# ---------------------------------------------------- Q8_0 K/V variant ----
def _read_q8_golden():
    blocks, expect = [], []
    with open(os.path.join(GOLDEN, "q8_0_superblock_worked.txt")) as f:
        lines = [ln.strip() for ln in f if ln.strip() and not ln.startswith("#")]
    for head, vals in zip(lines[0::2], lines[1::2]):
        parts = dict(p.split("=") for p in head.split()[2:])
        blocks.append((int(parts["d"], 16), bytes.fromhex(parts["bytes"])))
        expect.extend(float(v) for v in vals.split())
    return blocks, expect


def test_q8_worked_superblock_fixture():
    blocks, expect = _read_q8_golden()
    assert len(blocks) == 8 and len(expect) == 256
    sb = bytearray(272)
    for b, (dbits, qs) in enumerate(blocks):
        assert len(qs) == 32
        sb[32 * b: 32 * b + 32] = qs
        sb[256 + 2 * b] = dbits & 0xFF
        sb[257 + 2 * b] = dbits >> 8
    v = oracle.dequant_q8(np.frombuffer(bytes(sb), dtype=np.uint8), 1, 256)
    assert list(v[0]) == expect


def test_q8_superblock_offsets_single_value():
    # one nonzero value (q = -3) at row 1, super-block 2, block 6, element 17:
    # byte 32*6 + 17 of that super-block; its block scale is the only 1.0
    rows, K = 3, 768
    buf = np.zeros(rows * 3 * 272, dtype=np.uint8)
    at = (1 * 3 + 2) * 272
    buf[at + 32 * 6 + 17] = 0xFD
    buf[at + 256 + 2 * 6: at + 258 + 2 * 6] = [0x00, 0x3C]
    v = oracle.dequant_q8(buf, rows, K)
    nz = np.argwhere(v != 0)
    assert nz.tolist() == [[1, 512 + 6 * 32 + 17]]
    assert v[1, 512 + 6 * 32 + 17] == -3.0


def test_q8_generator_recipe():
    # every block: d = fp16(amax / 127), |q| <= 127, and the largest |q| is 127
    # (the element that set amax) unless the block is all zero
    c = synth.q8_0_kv_cache(5, 2, 9)
    q, d = oracle.unpack_q8_superblocks(c, 18, 256)
    assert np.abs(q).max() <= 127
    qb = np.abs(q.reshape(18, 8, 32)).max(axis=-1)
    assert ((qb == 127) | (d == 0)).all()
    assert (d > 0).all()


def _q4_cache_as_q8(buf4, rows):
    """The same values in the 8-bit layout: q8 = q4 - 8 with the same scale,
    written byte by byte from the nibble definition (no oracle code)."""
    raw = np.asarray(buf4, dtype=np.uint8).reshape(rows, 144)
    out = np.zeros((rows, 272), dtype=np.uint8)
    for b in range(8):
        nib = raw[:, 16 * b: 16 * b + 16]
        lo = (nib & 0x0F).astype(np.int16) - 8           # elements j
        hi = (nib >> 4).astype(np.int16) - 8              # elements j + 16
        out[:, 32 * b: 32 * b + 16] = lo.astype(np.int8).view(np.uint8)
        out[:, 32 * b + 16: 32 * b + 32] = hi.astype(np.int8).view(np.uint8)
    out[:, 256:272] = raw[:, 128:144]
    return out.reshape(-1)


@pytest.mark.parametrize("ctx,n_q,n_kv,M", [(5, 4, 1, 1), (33, 24, 4, 5), (70, 8, 2, 3)])
def test_q8_attention_equals_q4_attention_on_the_same_values(ctx, n_q, n_kv, M):
    # a Q4 cache re-expressed exactly in the 8-bit layout must give the same
    # attention output: pins the Q8 path to the Q4 path's pins
    K4 = synth.q4_0_kv_cache(90 + ctx, n_kv, ctx)
    V4 = synth.q4_0_kv_cache(91 + ctx, n_kv, ctx)
    Q = synth.queries(92 + ctx, M, n_q)
    K8, V8 = _q4_cache_as_q8(K4, n_kv * ctx), _q4_cache_as_q8(V4, n_kv * ctx)
    assert np.array_equal(oracle.dequant_q8(K8, n_kv * ctx, 256), oracle.dequant(K4, n_kv * ctx, 256))
    o4 = oracle.attn_decode(Q, K4, V4, ctx, n_q, n_kv, 256, M)
    o8 = oracle.attn_decode(Q, K8, V8, ctx, n_q, n_kv, 256, M, fmt="q8_0")
    assert np.allclose(o8, o4, rtol=0, atol=1e-13)


def test_q8_attention_single_token_and_stride():
    # one visible token: the output is that token's V row for every query
    # head of the group; a stride leaves the tokens beyond ctx unread
    n_kv, cap = 2, 7
    V = synth.q8_0_kv_cache(3, n_kv, cap)
    K = synth.q8_0_kv_cache(4, n_kv, cap)
    Q = synth.queries(5, 1, 6)
    out = oracle.attn_decode(Q, K, V, 1, 6, n_kv, 256, 1, kv_stride=cap, fmt="q8_0")
    Vh = oracle.dequant_q8(V, n_kv * cap, 256).reshape(n_kv, cap, 256)
    for h in range(6):
        assert np.array_equal(out[0, h], Vh[h // 3, 0])
    with pytest.raises(ValueError):
        oracle.attn_decode(Q, K, V, 1, 6, n_kv, 256, 1, fmt="q5_0")


# ------------------------------------------- SwiGLU propagated tolerance ----
def _f32_ulps(v, k):
    """fp32 value v moved by k ulps (k may be negative)."""
    v = np.float32(v)
    for _ in range(abs(k)):
        v = np.nextafter(v, np.float32(np.inf if k > 0 else -np.inf), dtype=np.float32)
    return v


def _device_epilogue(g32, u32, exp_ulps):
    """h = g / (1 + expf(-g)) * u with every fp32 operation rounded to nearest
    and expf off by exp_ulps ulps (the documented bound is 2)."""
    e = _f32_ulps(np.float32(math.exp(-float(g32))), exp_ulps)
    den = np.float32(np.float32(1.0) + e)
    return float(np.float32(np.float32(g32 / den) * u32))


def _within(v, center, t):
    """Closest fp32 value to v that lies within [center - t, center + t]."""
    v = np.float32(v)
    while abs(float(v) - center) > t:
        v = np.nextafter(v, np.float32(center), dtype=np.float32)
    return v


def _worst_ratio(g, u, tg, tu, scale=1.0):
    """max over a grid of device results (g~, u~ within tg, tu of g, u; expf
    off by -2, 0, +2 ulps) of |h_dev - silu(g) u| / (scale * tolerance)."""
    tol = float(oracle.swiglu_tolerance(np.array(g), np.array(u), tg, tu)) * scale
    exact = float(oracle.silu(np.array([g]))[0]) * u
    worst = 0.0
    for dg in np.linspace(-tg, tg, 21):
        g32 = _within(g + dg, g, tg)
        for du in np.linspace(-tu, tu, 11):
            u32 = _within(u + du, u, tu)
            for k in (-2, 0, 2):
                worst = max(worst, abs(_device_epilogue(g32, u32, k) - exact) / tol)
    return worst


SWIGLU_CASES = [(g, u, tg, tu) for g in (-30.0, -8.0, -1.278, 0.0, 0.7, 2.4, 8.0, 30.0)
                for u in (-3.0, 1e-3, 5.0)
                for tg, tu in ((0.02, 0.03), (0.5, 0.8), (2.0, 1.5))]


def test_silu_prime_extrema_and_interval_maximum():
    # silu'' = s(1 - s)(2 - g tanh(g / 2)) vanishes at +-SILU_PRIME_CRIT only,
    # and max |silu'| over an interval (the bound's D) equals a dense-grid
    # maximum of |silu'| over that interval
    c = oracle.SILU_PRIME_CRIT
    assert abs(c * math.tanh(c / 2) - 2.0) < 1e-12 and 2.39 < c < 2.41
    g = np.linspace(-30.0, 30.0, 240001)  # 1 - s stays > 0 in fp64 here
    s = 1.0 / (1.0 + np.exp(-g))
    d2 = s * (1.0 - s) * (2.0 - g * np.tanh(g / 2.0))
    sign_changes = g[1:][np.sign(d2[1:]) != np.sign(d2[:-1])]
    assert len(sign_changes) == 2 and np.allclose(sign_changes, [-c, c], atol=1e-3)
    h = 1e-5
    fd = (oracle.silu_prime(g[::997] + h) - oracle.silu_prime(g[::997] - h)) / (2 * h)
    np.testing.assert_allclose(fd, d2[::997], atol=1e-8)
    for center in (-30.0, -8.0, -2.4, -1.0, 0.0, 1.5, 2.4, 3.0, 30.0):
        for t in (0.01, 0.3, 2.0, 6.0):
            grid = np.linspace(center - t, center + t, 200001)
            dense = np.abs(oracle.silu_prime(grid)).max()
            got = float(oracle.silu_prime_max(center, t))
            assert dense * (1 - 1e-12) <= got <= dense * (1 + 1e-9) + 1e-15


def test_silu_prime_is_the_derivative():
    g = np.linspace(-40.0, 40.0, 4001)
    h = 1e-6
    fd = (oracle.silu(g + h) - oracle.silu(g - h)) / (2 * h)
    np.testing.assert_allclose(oracle.silu_prime(g), fd, atol=1e-8)


@pytest.mark.parametrize("g,u,tg,tu", SWIGLU_CASES)
def test_swiglu_tolerance_covers_every_perturbation(g, u, tg, tu):
    # every (g~, u~) within the GEMV bound of (g, u), evaluated as the device
    # does in fp32 with expf at its documented 2-ulp limit, stays within the bound
    assert _worst_ratio(g, u, tg, tu) <= 1.0


@pytest.mark.parametrize("g", [-30.0, -8.0, 0.0, 8.0, 30.0])
def test_swiglu_tolerance_halved_fails(g):
    # the bound is tight to within a factor 2 at these gates: half of it is
    # exceeded by some perturbation inside (tg, tu)
    worst = max(_worst_ratio(g, u, tg, tu, scale=0.5)
                for (gg, u, tg, tu) in SWIGLU_CASES if gg == g)
    assert worst > 1.0


def test_swiglu_tolerance_is_the_propagated_gemv_bound():
    # the fused oracle carries the GEMV bound of each output through the SwiGLU
    N, K, M = 5, 512, 2
    W = synth.q4_0_weights(71, 2 * N, K)
    x = synth.activations(72, M, K)
    h, tol = oracle.gemv_swiglu(W, x, M, N, K)
    y, S = oracle.gemv(W, x, M, 2 * N, K)
    t = oracle.gemv_tolerance(S)
    np.testing.assert_array_equal(
        tol, oracle.swiglu_tolerance(y[:, 0::2], y[:, 1::2], t[:, 0::2], t[:, 1::2]))
    # first-order part alone is a lower bound of it
    g, u = y[:, 0::2], y[:, 1::2]
    first = np.abs(oracle.silu_prime(g) * u) * t[:, 0::2] + np.abs(oracle.silu(g)) * t[:, 1::2]
    assert np.all(tol >= first)
