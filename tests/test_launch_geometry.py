"""CPU model of the kernels' launch geometry, driven by the library's own
planner: every row, K range and token is covered exactly once, every bulk
copy stays inside its source buffer and its shared-memory slot, and every
load, store and workspace index stays in bounds.  These run before anything
touches a GPU."""
import pytest

from bit_weight_streaming_dequant_b200 import q4dec

TX_LIMIT = (1 << 20) - 1           # mbarrier transaction-count range
SMEM_OPTIN = 227 * 1024            # B200 opt-in shared memory per block


def _next_pow2(v):
    p = 1
    while p < v:
        p *= 2
    return p


def _gemv_rsr(M):
    return 4 if M <= 2 else 2


GEMV_SHAPES = [(1, 512, 1024), (1, 17408, 5120), (1, 5120, 17408), (1, 6144, 5120),
               (1, 5120, 6144), (1, 151936, 5120), (2, 5120, 17408), (3, 17408, 5120),
               (4, 6144, 5120), (5, 5120, 17408), (5, 151936, 5120), (1, 1, 256),
               (5, 3, 256), (1, 37, 4352), (3, 300, 1280), (2, 64, 65536), (5, 7, 32768),
               (4, 100, 256), (1, 147, 512), (1, 149, 512)]


@pytest.mark.parametrize("M,N,K", GEMV_SHAPES)
@pytest.mark.parametrize("sms", [148, 132, 7])
def test_gemv_geometry(M, N, K, sms):
    p = q4dec.plan_gemv(M, N, K, sms)
    W, rsr = p.words_per_thread, p.rows_per_stream
    assert rsr == _gemv_rsr(M) and W == {1: 4, 2: 2}.get(M, 1)
    tps = 32 // W
    nsb = K // 256
    ks = p.k_splits
    assert p.threads % 32 == 0 and p.threads <= 640 and p.threads % p.row_streams == 0
    tpr = p.threads // p.row_streams
    assert tpr % 32 == 0 and tpr >= p.sb_per_split * tps
    vpad = _next_pow2(rsr * M)
    assert vpad <= 32 and p.row_streams * rsr * M <= p.threads
    slot = p.row_streams * rsr * p.sb_per_split * 144
    nwarps = p.threads // 32
    assert p.smem_bytes == p.stages * slot + 2 * nwarps * vpad * 4 + p.stages * 8
    assert p.smem_bytes <= SMEM_OPTIN and (p.stages * slot + 2 * nwarps * vpad * 4) % 8 == 0
    assert p.workspace_bytes == (ks * M * N * 4 if ks > 1 else 0)
    w_bytes = N * nsb * 144
    out_len = ks * M * N if ks > 1 else M * N

    # K ranges partition the super-blocks
    sb_base, sb_rem = nsb // ks, nsb % ks
    covered = []
    for k in range(ks):
        cnt = sb_base + (1 if k < sb_rem else 0)
        sb0 = k * sb_base + min(k, sb_rem)
        assert 1 <= cnt <= p.sb_per_split
        covered.extend(range(sb0, sb0 + cnt))
    assert covered == list(range(nsb))

    # threads of one row stream: words and scales inside the row segment,
    # activations inside x
    for k in range(ks):
        cnt = sb_base + (1 if k < sb_rem else 0)
        sb0 = k * sb_base + min(k, sb_rem)
        seg = cnt * 144
        seen = set()
        for tid in range(p.threads):
            stream, idx = divmod(tid, tpr)
            assert stream < p.row_streams
            sb_local, word0 = idx // tps, (idx % tps) * W
            if sb_local >= cnt:
                continue
            blk = word0 >> 2
            word_off = sb_local * 144 + word0 * 4
            scale_off = sb_local * 144 + 128 + blk * 2
            assert word_off % (4 * W) == 0 and word_off + 4 * W <= sb_local * 144 + 128
            assert scale_off + 2 <= seg
            for w in range(W):
                klo = (sb0 + sb_local) * 256 + blk * 32 + 4 * ((word0 + w) & 3)
                assert klo % 4 == 0 and klo + 16 + 4 <= K and (sb0 + sb_local) * 256 <= klo
                if stream == 0:
                    for c in range(4):
                        seen.add(klo + c)
                        seen.add(klo + 16 + c)
        assert seen == set(range(sb0 * 256, (sb0 + cnt) * 256))

    # rows: CTAs partition [0, N); copies stay inside W and the slot
    rows = []
    per_stage = p.row_streams * rsr
    for k in range(ks):
        cnt = sb_base + (1 if k < sb_rem else 0)
        sb0 = k * sb_base + min(k, sb_rem)
        seg = cnt * 144
        for cta in range(p.grid_rows):
            rb, re_ = N * cta // p.grid_rows, N * (cta + 1) // p.grid_rows
            assert re_ > rb
            if k == 0:
                rows.extend(range(rb, re_))
            n_st = (re_ - rb + per_stage - 1) // per_stage
            for st in range(n_st):
                r0 = rb + st * per_stage
                nr = min(per_stage, re_ - r0)
                assert nr >= 1 and nr * seg <= slot and nr * seg <= TX_LIMIT
                if ks == 1:
                    lo, hi = r0 * nsb * 144, r0 * nsb * 144 + nr * seg
                    assert lo % 16 == 0 and hi <= w_bytes
                else:
                    for r in range(nr):
                        lo = ((r0 + r) * nsb + sb0) * 144
                        assert lo % 16 == 0 and lo + seg <= w_bytes
                # final stores
                for tid in range(per_stage * M):
                    lr, m = divmod(tid, M)
                    if lr < nr:
                        assert (k * M + m) * N + r0 + lr < out_len
    assert rows == list(range(N))


ATTN_CASES = [(4096, 24, 4, 1), (4096, 24, 4, 5), (65536, 24, 4, 5), (262144, 24, 4, 1),
              (262144, 24, 4, 5), (1, 4, 1, 1), (5, 24, 4, 5), (63, 6, 2, 3), (65, 6, 2, 3),
              (1000, 8, 1, 5), (300, 64, 4, 5), (129, 4, 4, 2), (70000, 48, 1, 5)]


@pytest.mark.parametrize("ctx,nq,nkv,M", ATTN_CASES)
@pytest.mark.parametrize("stride_extra", [0, 37])
def test_attn_geometry(ctx, nq, nkv, M, stride_extra):
    sms = 148
    p = q4dec.plan_attn(ctx, nq, nkv, 256, M, sms)
    TT, RM = p.tile_tokens, 32
    stride = ctx + stride_extra
    g = nq // nkv
    assert TT == 64 and p.split_tokens % TT == 0 and p.threads == 256
    assert p.rows_per_cta <= RM and p.row_groups * p.rows_per_cta >= g * M
    cache_bytes = nkv * stride * 144
    tokens = []
    for c in range(p.n_splits):
        tb, te = c * p.split_tokens, min(ctx, (c + 1) * p.split_tokens)
        assert te > tb
        tokens.extend(range(tb, te))
        n_tiles = (te - tb + TT - 1) // TT
        for tile in range(n_tiles):
            t0 = tb + tile * TT
            nbytes = min(TT, te - t0) * 144
            assert 2 * nbytes <= TX_LIMIT
            for kh in range(nkv):
                lo = (kh * stride + t0) * 144
                assert lo % 16 == 0 and lo + nbytes <= cache_bytes
    assert tokens == list(range(ctx))
    rows = []
    for z in range(p.row_groups):
        r0 = z * p.rows_per_cta
        R = min(p.rows_per_cta, g * M - r0)
        assert 1 <= R <= RM
        rows.extend(range(r0, r0 + R))
    assert rows == list(range(g * M))
    # workspace indices of the split states and the output rows
    nrows = M * nq
    if p.n_splits > 1:
        assert p.workspace_bytes == p.n_splits * nrows * 258 * 4
        assert (p.n_splits - 1) * nrows * 256 + (nrows - 1) * 256 + 255 < p.n_splits * nrows * 256
    else:
        assert p.workspace_bytes == 0
    for kh in range(nkv):
        for rr in range(g * M):
            m, j = divmod(rr, g)
            row = m * nq + kh * g + j
            assert 0 <= row < nrows
    ring = p.stages * 2 * TT * 144
    assert p.smem_bytes == RM * 256 * 4 + ring + TT * RM * 4 + 3 * RM * 4 + p.stages * 8
    assert (RM * 256 * 4 + ring + TT * RM * 4 + 3 * RM * 4) % 8 == 0
    assert 2 * p.smem_bytes <= 228 * 1024  # two CTAs per SM
