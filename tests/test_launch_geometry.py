"""CPU model of the kernels' launch geometry, driven by the library's own
planner: every row, K range and token is covered exactly once, every bulk
copy stays inside its source buffer and its shared-memory slot, and every
load, store and workspace index stays in bounds.  These run before anything
touches a GPU."""
import numpy as np
import pytest

from bit_weight_streaming_dequant_b200 import q4dec

TX_LIMIT = (1 << 20) - 1           # mbarrier transaction-count range
SMEM_OPTIN = 227 * 1024            # B200 opt-in shared memory per block


GEMV_ROWS, GEMV_COLS, GEMV_WARPS, GEMV_THREADS = 128, 2, 16, 608
GEMV_WBOX = GEMV_ROWS * 144


GEMV_XPITCH = GEMV_COLS * 512 + 32   # activation rows of a stage: 1 KB at a 1056-byte pitch


def _gemv_pair_slots(M):
    # one reduction slot per block index (column 1 adds to column 0) at M >= 4
    return M >= 4


def _gemv_stage_bytes(M):
    align = 16 if _gemv_pair_slots(M) else 128
    return -(-(GEMV_COLS * GEMV_WBOX + M * GEMV_XPITCH) // align) * align


def _gemv_red_layout(M):
    # (buffers, slots per buffer): two buffers for M <= 2; a slot per consumer
    # warp, or per block index with pair slots
    return (2 if M <= 2 else 1), (8 if _gemv_pair_slots(M) else 16)


def _unit_begin(c, U, G):
    return c * U // G


def _unit_owner(u, U, G):
    return ((u + 1) * G - 1) // U


GEMV_SHAPES = [(1, 512, 1024), (1, 17408, 5120), (1, 5120, 17408), (1, 6144, 5120),
               (1, 5120, 6144), (1, 151936, 5120), (2, 5120, 17408), (3, 17408, 5120),
               (4, 6144, 5120), (5, 5120, 17408), (5, 151936, 5120), (1, 1, 256),
               (5, 3, 256), (1, 37, 4352), (3, 300, 1280), (2, 64, 65536), (5, 7, 32768),
               (4, 100, 256), (1, 147, 512), (1, 149, 512), (5, 1000, 2048), (2, 2, 17408),
               (1, 1300, 512), (3, 40000, 768), (5, 34816, 5120)]


@pytest.mark.parametrize("M,N,K", GEMV_SHAPES)
@pytest.mark.parametrize("sms", [148, 132, 7])
def test_gemv_geometry(M, N, K, sms):
    p = q4dec.plan_gemv(M, N, K, sms)
    nsb = K // 256
    rbs, upr = -(-N // GEMV_ROWS), -(-nsb // GEMV_COLS)
    U, G = rbs * upr, p.grid
    assert p.threads == GEMV_THREADS and p.row_blocks == rbs and p.units_per_row_block == upr
    assert p.units == U and 1 <= G <= min(sms, U)
    stage = _gemv_stage_bytes(M)
    assert stage % 16 == 0                    # every stage starts where a bulk copy may land
    # reduction buffers (consumers -> epilogue), slots of [M][132] fp32 (128
    # rows + 4 floats of padding: the 8 rows x 4 columns a warp stores at once
    # hit distinct banks), with pair slots one barrier per slot (the column-0
    # warp's sums are in) besides the two per buffer
    bufs, slots_per_buf = _gemv_red_layout(M)
    red = bufs * slots_per_buf * M * 132 * 4
    assert p.smem_bytes == (p.stages * stage + red + 16 + p.stages * 16 + bufs * 16 +
                            (bufs * 8 * 8 if _gemv_pair_slots(M) else 0))
    if sms == 148:
        assert p.stages == 5                  # five stages at every M on B200
    banks = {((2 * t + e) * 132 + g) % 32 for t in range(4) for g in range(8) for e in (0,)
             if 2 * t + e < M}
    assert len(banks) == 8 * len([t for t in range(4) if 2 * t < M])
    assert p.smem_bytes + stage + 16 > SMEM_OPTIN or p.stages == 8   # as many stages as fit
    assert 2 <= p.stages <= 8 and p.smem_bytes <= SMEM_OPTIN
    # the units are shared out exactly once, every CTA getting at least one
    ranges = [(_unit_begin(c, U, G), _unit_begin(c + 1, U, G)) for c in range(G)]
    assert ranges[0][0] == 0 and ranges[-1][1] == U
    assert all(b > a for a, b in ranges) and all(ranges[i][1] == ranges[i + 1][0]
                                                   for i in range(G - 1))
    assert max(b - a for a, b in ranges) - min(b - a for a, b in ranges) <= 1
    for c, (a, b) in enumerate(ranges):
        assert _unit_owner(a, U, G) == c and _unit_owner(b - 1, U, G) == c
    # contributors per row block, their slots, the workspace carve-up
    slots = 0
    for rb in range(rbs):
        first, last = _unit_owner(rb * upr, U, G), _unit_owner(rb * upr + upr - 1, U, G)
        if last > first:
            slots = max(slots, last - first + 1)
            for c in range(first, last + 1):        # every one of them holds a unit of rb
                a, b = ranges[c]
                assert a < (rb + 1) * upr and b > rb * upr
    assert p.slots == slots
    # one 8-byte entry (fp32 value + tag) per row, column and slot of each row block
    assert p.workspace_bytes == rbs * slots * M * 128 * 8
    # every copy stays inside its source buffer and its stage slot
    w_bytes, x_bytes = N * nsb * 144, M * K * 2
    for c in {0, G // 2, G - 1}:
        a, b = ranges[c]
        for u in range(a, b):
            rb, cp = divmod(u, upr)
            col0 = 2 * cp
            kc = min(2, nsb - col0)
            rows = min(GEMV_ROWS, N - rb * GEMV_ROWS)
            assert kc >= 1 and rows >= 1
            assert kc * (rows * 144 + M * 512) <= TX_LIMIT
            for j in range(kc):
                src = ((col0 + j) * N + rb * GEMV_ROWS) * 144
                assert src % 16 == 0 and src + rows * 144 <= w_bytes
                assert j * GEMV_WBOX + rows * 144 <= GEMV_COLS * GEMV_WBOX
            for m in range(M):
                xsrc = (m * nsb + col0) * 256 * 2
                assert xsrc % 16 == 0 and xsrc + kc * 512 <= x_bytes
                dst = GEMV_COLS * GEMV_WBOX + m * GEMV_XPITCH
                assert dst % 16 == 0 and dst + kc * 512 <= stage
    # per-warp shared-memory reads stay inside the stage: weights (rows g and
    # g + 8 of 8 tiles), scales, activations (column g < M)
    for warp in range(GEMV_WARPS):
        col, blk = warp >> 3, warp & 7
        for g in range(8):
            for t in range(4):
                pa = col * GEMV_WBOX + g * 144 + blk * 16 + t * 4
                assert pa + (16 * 7 + 8) * 144 + 4 <= (col + 1) * GEMV_WBOX
                pd = col * GEMV_WBOX + g * 144 + 128 + blk * 2
                assert pd + (16 * 7 + 8) * 144 + 2 <= (col + 1) * GEMV_WBOX
                if g < M:
                    xo = GEMV_COLS * GEMV_WBOX + g * GEMV_XPITCH + col * 512 + (blk * 32 + 4 * t) * 2
                    assert xo % 8 == 0 and xo + 32 + 8 <= stage
    # bank pattern of the A-word loads: 32 lanes (g, t) read row g, word t at a
    # 144-byte pitch
    banks = {((g * 144 + 4 * t) // 4) % 32 for g in range(8) for t in range(4)}
    assert len(banks) == 32
    # activation fragment loads (8 bytes per lane, a half-warp per pass): the
    # rows g < M of either half-warp hit distinct banks
    for half in (range(0, 4), range(4, 8)):
        for col in range(2):
            for blk in range(8):
                words = [(GEMV_COLS * GEMV_WBOX + g * GEMV_XPITCH + col * 512 +
                          (blk * 32 + 4 * t) * 2) // 4 + i
                         for g in half if g < M for t in range(4) for i in range(2)]
                assert len({w % 32 for w in words}) == len(words)


@pytest.mark.parametrize("M,N,K", [(1, 17408, 5120), (3, 5120, 17408), (2, 6144, 5120),
                                   (5, 37, 4352), (1, 300, 1280), (4, 1000, 2048)])
def test_gemv_stream_k_sums_every_product_once(M, N, K):
    # a model of the partition and of the finisher's reduction: partial sums
    # of each CTA's segments, slot by slot, rebuild the full product exactly
    p = q4dec.plan_gemv(M, N, K, 148)
    nsb = K // 256
    rbs, upr, U, G = p.row_blocks, p.units_per_row_block, p.units, p.grid
    rng = np.random.default_rng(N + K)
    w = rng.integers(-8, 8, size=(N, K)).astype(np.float64)
    x = rng.integers(-4, 5, size=(M, K)).astype(np.float64)
    y = np.zeros((M, N))
    parts = {}
    for c in range(G):
        a, b = _unit_begin(c, U, G), _unit_begin(c + 1, U, G)
        u = a
        while u < b:
            rb = u // upr
            seg_end = min(b, (rb + 1) * upr)
            cols = slice(2 * (u - rb * upr) * 256, min(2 * (seg_end - rb * upr), nsb) * 256)
            rows = slice(rb * 128, min(N, rb * 128 + 128))
            s = x[:, cols] @ w[rows, cols].T
            first = _unit_owner(rb * upr, U, G)
            last = _unit_owner(rb * upr + upr - 1, U, G)
            if first == last:
                y[:, rows] = s
            else:
                assert 0 <= c - first < p.slots
                parts.setdefault(rb, {})[c - first] = s
            u = seg_end
    for rb, d in parts.items():
        assert sorted(d) == list(range(len(d)))
        y[:, rb * 128: min(N, rb * 128 + 128)] = sum(d[k] for k in range(len(d)))
    assert np.array_equal(y, x @ w.T)


ATTN_CASES = [(4096, 24, 4, 1), (4096, 24, 4, 5), (65536, 24, 4, 5), (262144, 24, 4, 1),
              (262144, 24, 4, 5), (1, 4, 1, 1), (5, 24, 4, 5), (63, 6, 2, 3), (65, 6, 2, 3),
              (1000, 8, 1, 5), (300, 64, 4, 5), (129, 4, 4, 2), (70000, 48, 1, 5)]


TT_ATTN, Q_PITCH, ROW = 128, 576, 144
TT_R8, WARPS_R8 = 192, 12          # warp-local variant (at most 8 rows per CTA)


TC_THREADS, TC_V_BYTES = 448, 256 * 128 * 2   # tensor-memory variant: 14 warps, fp16 V tile


def _tc_nr(rows_per_cta):
    return 16 if rows_per_cta <= 16 else 32


ROW_Q8 = 272                        # bytes per token row of the Q8_0 cache
SMEM_Q8_BUDGET = 227 * 1024


def _tc_pbufs(nr, q8):
    return 1 if (q8 and nr == 32) else 2


def _tc_offsets(stages, nr, row=ROW, pb=2):
    """Carve-up of the tensor-memory variant's shared memory: ring, Q (fp16,
    K-major), V tile (fp16, M-major), `pb` P^T buffers (fp16, N-major), row
    statistics ([4][32] warp partials, running max, max used, alpha, sums,
    causal limits), flags, barriers (2 per ring stage + 12) and the
    tensor-memory address."""
    ring = stages * 2 * TT_ATTN * row
    q = ring
    v = q + 512 * nr
    pt = v + TC_V_BYTES
    stats = pt + pb * (nr // 8) * 2048
    flags = stats + 4 * 32 * 4 + 5 * 32 * 4
    bars = flags + 16
    end = bars + (2 * stages + 12) * 8 + 8
    return dict(ring=ring, q=q, v=v, pt=pt, stats=stats, flags=flags, bars=bars, end=end)


def _attn_smem(stages, rows_per_cta):
    if rows_per_cta <= 8:      # ring + Q fragments + per-warp / per-row stats + barriers + abort
        return stages * 2 * TT_R8 * ROW + 8 * Q_PITCH + WARPS_R8 * 8 * 2 * 4 + 8 * 2 * 4 \
            + stages * 16 + 16
    return _tc_offsets(stages, _tc_nr(rows_per_cta))["end"]


def _chunks(addrs):
    """16-byte bank groups hit by eight ldmatrix row addresses (one phase)."""
    return {(a % 128) // 16 for a in addrs}


def test_attn_shared_memory_banks():
    # K ldmatrix (warp-local kernel) and 16-byte row loads (tensor-memory
    # kernel): eight token rows at a 144-byte pitch, same column
    for col in range(0, 144, 16):
        assert len(_chunks([r * ROW + col for r in range(8)])) == 8
    # Q fragment loads (16 bytes per lane): each group of eight lanes covers
    # eight distinct 16-byte bank groups
    for blk in range(8):
        for q in range(4):
            lanes = range(8 * q, 8 * q + 8)
            assert len(_chunks([(ln >> 2) * Q_PITCH + (blk * 4 + (ln & 3)) * 16
                                for ln in lanes])) == 8
    # block scales in the score step: tokens g at a 144-byte pitch, distinct banks
    assert len({((g * ROW + 128) // 4) % 32 for g in range(8)}) == 8
    # tensor-memory kernel: V-tile and P^T stores, lane = token k of a 32-token
    # quadrant, 16 bytes at (k >> 3) * 128 + (k & 7) * 16 from the chunk base
    for quad in range(4):
        for phase in range(4):
            ks = [32 * quad + 8 * phase + i for i in range(8)]
            assert len(_chunks([(k >> 3) * 128 + (k & 7) * 16 for k in ks])) == 8


@pytest.mark.parametrize("ctx,nq,nkv,M", ATTN_CASES)
@pytest.mark.parametrize("stride_extra", [0, 37])
def test_attn_geometry(ctx, nq, nkv, M, stride_extra):
    sms = 148
    p = q4dec.plan_attn(ctx, nq, nkv, 256, M, sms)
    TT = p.tile_tokens
    stride = ctx + stride_extra
    g = nq // nkv
    rows8 = p.rows_per_cta <= 8
    assert TT == (TT_R8 if rows8 else TT_ATTN) and p.split_tokens % TT == 0
    assert p.threads == (WARPS_R8 * 32 if rows8 else TC_THREADS)
    assert 1 <= p.n_splits <= 256
    assert p.rows_per_cta <= 32 and p.row_groups * p.rows_per_cta >= g * M
    assert 2 <= p.stages <= 8
    assert p.smem_bytes == _attn_smem(p.stages, p.rows_per_cta) <= SMEM_OPTIN
    ring = p.stages * 2 * TT * ROW
    if rows8:
        # the final combine parks [12 warps][8 rows][256] fp32 in the ring;
        # Q fragments follow the ring (16-byte aligned), barriers 8-aligned
        assert ring >= WARPS_R8 * 8 * 256 * 4
        assert ring % 16 == 0 and (ring + 8 * Q_PITCH + WARPS_R8 * 64 + 64) % 8 == 0
    else:
        o = _tc_offsets(p.stages, _tc_nr(p.rows_per_cta))
        # operands of the tensor-core descriptors 16-byte aligned, barriers 8
        assert all(o[k] % 16 == 0 for k in ("q", "v", "pt", "stats", "flags", "bars"))
    assert (TT * ROW) % 16 == 0
    cache_bytes = nkv * stride * 144
    tokens = []
    for c in range(p.n_splits):
        tb, te = c * p.split_tokens, min(ctx, (c + 1) * p.split_tokens)
        assert te > tb
        tokens.extend(range(tb, te))
        n_tiles = (te - tb + TT - 1) // TT
        for tile in range(n_tiles):
            t0 = tb + tile * TT
            nbytes = min(TT, te - t0) * ROW
            assert 2 * nbytes <= TX_LIMIT and nbytes % 16 == 0 and nbytes <= TT * ROW
            for kh in range(nkv):
                lo = (kh * stride + t0) * ROW
                assert lo % 16 == 0 and lo + nbytes <= cache_bytes
    assert tokens == list(range(ctx))
    rows = []
    for z in range(p.row_groups):
        r0 = z * p.rows_per_cta
        R = min(p.rows_per_cta, g * M - r0)
        assert 1 <= R <= 32
        rows.extend(range(r0, r0 + R))
    assert rows == list(range(g * M))
    nrt = -(-p.rows_per_cta // 8)
    if rows8:
        for warp in range(WARPS_R8):
            for lane in range(32):
                # ldmatrix rows (K and V) and the 16-byte scale vectors of
                # tokens 2t, 2t + 1, 2t + 8, 2t + 9
                tok = 16 * warp + (lane & 15)
                for b in range(0, 8, 2):
                    assert tok < TT and (lane >> 4) * 16 + b * 16 + 16 <= 128
                for i in range(4):
                    tk = 16 * warp + 2 * (lane & 3) + (i & 1) + (i >> 1) * 8
                    assert tk < TT and (tk * ROW + 128) % 16 == 0
                # park index of the final combine
                g_, t_ = lane >> 2, lane & 3
                hi = (warp * 8 + 2 * t_ + 1) * 256 + 32 * 7 + 2 * g_ + 1 + 16
                assert hi < WARPS_R8 * 8 * 256
        _attn_q_and_workspace(p, M, nq, nkv, g)
        return
    _tc_layout_checks(_tc_nr(p.rows_per_cta))
    _attn_q_and_workspace(p, M, nq, nkv, g)


def _pair_elements(word, low):
    """Elements of a Q4_0 block held by the fp16 pair unpacked from bits 0-3
    (low) or 4-7 of bytes 0 and 2 of `word` (a 4-byte group, word 0 = bytes
    0..3): byte j holds element j in its low nibble, j + 16 in its high."""
    b0, b2 = 4 * (word // 4) + (word % 4), 4 * (word // 4) + (word % 4) + 2
    return (b0, b2) if low else (b0 + 16, b2 + 16)


def _tc_unpacked_element(kk):
    # restatement of the kernel's element order: column c = kk // 2 holds
    # pair i = c % 4 of word t = c // 4
    c, h = kk >> 1, kk & 1
    t, i = c >> 2, c & 3
    return (16 if i & 1 else 0) + 4 * t + (i >> 1) + 2 * h


def test_tc_element_order_matches_nibble_unpacking():
    # word t of a block unpacks as q8_pair<low>(w), q8_pair<high>(w),
    # q8_pair<low>(w >> 8), q8_pair<high>(w >> 8): bytes (4t, 4t+2) then
    # (4t+1, 4t+3)
    order = []
    for t in range(4):
        order += _pair_elements(4 * t, True) + _pair_elements(4 * t, False)
        order += _pair_elements(4 * t + 1, True) + _pair_elements(4 * t + 1, False)
    assert order == [_tc_unpacked_element(kk) for kk in range(32)]
    assert sorted(order) == list(range(32))


def _tc_layout_checks(nr):
    # Q, K-major canonical layout: (kp, n) -> (kp>>3)*nr*16 + (n>>3)*128 + (n&7)*16 + (kp&7)*2
    q_off = {(kp >> 3) * nr * 16 + (n >> 3) * 128 + (n & 7) * 16 + (kp & 7) * 2
             for kp in range(256) for n in range(nr)}
    assert q_off == set(range(0, 512 * nr, 2))
    # QK B operand, step s: core matrices at base + s*nr*32 + kg*LBO + ng*SBO (LBO nr*16, SBO 128)
    reads = set()
    for s_ in range(16):
        for kg in range(2):
            for ng in range(nr // 8):
                reads.add(s_ * nr * 32 + kg * nr * 16 + ng * 128)
    assert reads == set(range(0, 512 * nr, 128))
    # V tile, M-major: V warp (8..11) lane -> token k, chunk (4b + t) of 8 dimensions
    v_off = []
    for warp in range(8, 12):
        for lane in range(32):
            k = 32 * (warp & 3) + lane
            for b in range(8):
                for t in range(4):
                    v_off.append((4 * b + t) * 2048 + (k >> 3) * 128 + (k & 7) * 16)
    assert sorted(v_off) == list(range(0, TC_V_BYTES, 16))
    # PV A operand (half h, step j): core matrices base + h*32768 + j*256 + kg*128 + mg*2048
    a_reads = {h * 32768 + j * 256 + kg * 128 + mg * 2048
               for h in range(2) for j in range(8) for kg in range(2) for mg in range(16)}
    assert a_reads == set(range(0, TC_V_BYTES, 128))
    # P^T, N-major: softmax warp (0..3) lane -> token k, rows 8c .. 8c + 7
    p_off = []
    for warp in range(4):
        for lane in range(32):
            k = 32 * warp + lane
            for c in range(nr // 8):
                p_off.append(c * 2048 + (k >> 3) * 128 + (k & 7) * 16)
    assert sorted(p_off) == list(range(0, (nr // 8) * 2048, 16))
    b_reads = {j * 256 + kg * 128 + ng * 2048 for j in range(8) for kg in range(2)
               for ng in range(nr // 8)}
    assert b_reads == set(range(0, (nr // 8) * 2048, 128))
    # tensor memory: K tiles [2][128], S^T [2][nr], O^T [2][nr] in 512 columns
    assert 256 + 4 * nr <= 512
    # the epilogue's lane -> dimension map is a bijection of 0..255 that
    # inverts the Q element order
    dims = [(mm & ~31) + _tc_unpacked_element(mm & 31) for mm in range(256)]
    assert sorted(dims) == list(range(256))


def _attn_q_and_workspace(p, M, nq, nkv, g):
    # Q reads (global, 8-byte vectors) stay inside [M][n_q][256]
    q_elems = M * nq * 256
    for kh in range(nkv):
        for rr in range(g * M):
            m, j = divmod(rr, g)
            row = m * nq + kh * g + j
            assert 0 <= row < M * nq
            for b in range(8):
                for t in range(4):
                    e = row * 256 + b * 32 + 4 * t
                    assert e % 4 == 0 and e + 16 + 4 <= q_elems
    # workspace: split outputs then (max, sum) pairs
    nrows = M * nq
    if p.n_splits > 1:
        assert p.workspace_bytes == p.n_splits * nrows * 258 * 4
    else:
        assert p.workspace_bytes == 0


def _simulate_in_warp_producer(n_tiles, S, warps, seed):
    """Random schedules of the warp-local variant's copy protocol: lane 0 of
    warp 0 issues tile k into slot k % S only once every warp has released
    tile k - S; at the start of its tile i it issues what it can without
    waiting, and waits only when tile i itself is not issued yet.  Every
    schedule must finish (no state where all warps wait forever)."""
    import random

    rnd = random.Random(seed)
    done = [0] * warps              # tiles finished per warp
    issued = min(S, n_tiles)        # prologue
    pending = [True] * warps        # warp 0's refill step still to run at its current tile
    released = lambda k: all(d > k for d in done)
    steps = 0
    while min(done) < n_tiles:
        steps += 1
        assert steps < 100000
        movable = []
        for w in range(warps):
            i = done[w]
            if i >= n_tiles:
                continue
            if w == 0 and pending[0]:
                # can the refill step finish now?
                blocked = False
                k = issued
                while k < n_tiles and k < i + S:
                    if not released(k - S):
                        blocked = k <= i
                        break
                    k += 1
                if not blocked:
                    movable.append(w)
                continue
            if issued > i:          # tile i's copies were issued: its full barrier completes
                movable.append(w)
        assert movable, f"deadlock: done={done} issued={issued}"
        w = rnd.choice(movable)
        if w == 0 and pending[0]:
            i = done[0]
            while issued < n_tiles and issued < i + S and released(issued - S):
                # slot issued % S held tile issued - S, which every warp has left
                assert all(d >= issued - S + 1 for d in done)
                issued += 1
            pending[0] = False
            continue
        done[w] += 1
        if w == 0:
            pending[0] = True


@pytest.mark.parametrize("n_tiles,S", [(1, 2), (2, 2), (3, 2), (7, 3), (37, 4), (40, 4), (5, 8)])
def test_in_warp_producer_never_deadlocks(n_tiles, S):
    for seed in range(40):
        _simulate_in_warp_producer(n_tiles, S, WARPS_R8, seed)


@pytest.mark.parametrize("N,K", [(1, 256), (3, 512), (37, 4352), (17408, 5120), (2048, 5120),
                                 (8, 65536), (75968, 5120)])
@pytest.mark.parametrize("sms", [148, 7])
def test_swiglu_partition_keeps_row_pairs_together(N, K, sms):
    # the fused variant plans 2N rows; row blocks (128 rows) start on even rows,
    # so a gate / up pair (rows 2n, 2n + 1) never straddles two row blocks and
    # the final write of a block sees both rows of each of its pairs
    p = q4dec.plan_gemv(1, 2 * N, K, sms)
    assert p.row_blocks == -(-2 * N // 128)
    owned = []
    for rb in range(p.row_blocks):
        r0, r1 = rb * 128, min(2 * N, rb * 128 + 128)
        assert r0 % 2 == 0 and (r1 - r0) % 2 == 0
        owned.extend(range(r0 // 2, r1 // 2))
    assert owned == list(range(N))


@pytest.mark.parametrize("ctx,nq,nkv,M", ATTN_CASES + [(1, 4, 1, 1), (200, 48, 1, 5)])
@pytest.mark.parametrize("stride_extra", [0, 37])
def test_attn_q8_geometry(ctx, nq, nkv, M, stride_extra):
    # the Q8_0 cache: every row count on the tensor-memory kernel, 272-byte rows
    sms = 148
    p = q4dec.plan_attn(ctx, nq, nkv, 256, M, sms, q8=True)
    g = nq // nkv
    nr = _tc_nr(p.rows_per_cta)
    pb = _tc_pbufs(nr, True)
    assert p.tile_tokens == TT_ATTN and p.threads == TC_THREADS and p.split_tokens % TT_ATTN == 0
    assert 2 <= p.stages <= 8 and 1 <= p.n_splits <= 256
    o = _tc_offsets(p.stages, nr, ROW_Q8, pb)
    assert p.smem_bytes == o["end"] <= SMEM_Q8_BUDGET
    assert all(o[k] % 16 == 0 for k in ("q", "v", "pt", "stats", "flags", "bars"))
    # a third stage would not fit: the planner takes as many as fit
    assert _tc_offsets(p.stages + 1, nr, ROW_Q8, pb)["end"] > SMEM_Q8_BUDGET or p.stages == 8
    stride = ctx + stride_extra
    cache_bytes = nkv * stride * ROW_Q8
    tokens = []
    for c in range(p.n_splits):
        tb, te = c * p.split_tokens, min(ctx, (c + 1) * p.split_tokens)
        assert te > tb
        tokens.extend(range(tb, te))
        for tile in range((te - tb + TT_ATTN - 1) // TT_ATTN):
            t0 = tb + tile * TT_ATTN
            nbytes = min(TT_ATTN, te - t0) * ROW_Q8
            assert 2 * nbytes <= TX_LIMIT and nbytes % 16 == 0
            for kh in range(nkv):
                lo = (kh * stride + t0) * ROW_Q8
                assert lo % 16 == 0 and lo + nbytes <= cache_bytes
    assert tokens == list(range(ctx))
    # per token row: block b's 32 values at 32b .. 32b+31 (two 16-byte loads),
    # the 16 scale bytes at 256; rows at a 272-byte pitch hit distinct 16-byte
    # bank groups for eight consecutive tokens
    for b in range(8):
        assert 32 * b + 32 <= 256
    for col in range(0, ROW_Q8, 16):
        assert len(_chunks([r * ROW_Q8 + col for r in range(8)])) == 8
    _tc_layout_checks(nr)
    _attn_q_and_workspace(p, M, nq, nkv, g)
    assert p.workspace_bytes == q4dec.lib().q8kv_attn_workspace_bytes(ctx, nq, nkv, 256, M) or \
        sms != 148


def _prmt(a, b, sel):
    """PTX prmt.b32 (default mode): result byte i = byte (sel >> 4i) & 7 of
    the eight bytes {a, b} (a's bytes 0..3, b's bytes 4..7)."""
    src = [(a >> (8 * i)) & 0xFF for i in range(4)] + [(b >> (8 * i)) & 0xFF for i in range(4)]
    return sum(src[(sel >> (4 * i)) & 7] << (8 * i) for i in range(4))


def test_q8_unpack_constants_give_exact_codes():
    # the tensor-memory kernel's Q8 unpack: x = w ^ 0x80808080, pairs
    # prmt(x, 0x64646464, 0x4140 / 0x4342) read as fp16 are 1024 + q + 128;
    # fma(., 1.0 (0x3C00), -1152 (0xE480)) is exactly q, in element order
    one, m1152 = np.uint16(0x3C00).view(np.float16), np.uint16(0xE480).view(np.float16)
    assert float(one) == 1.0 and float(m1152) == -1152.0
    for q0 in range(-128, 128, 7):
        qs = [q0, (q0 + 37) % 256 - 128, (q0 + 101) % 256 - 128, -q0 - 1]
        w = sum((q & 0xFF) << (8 * i) for i, q in enumerate(qs))
        x = w ^ 0x80808080
        got = []
        for sel in (0x4140, 0x4342):
            r = _prmt(x, 0x64646464, sel)
            for half in (r & 0xFFFF, r >> 16):
                v = np.uint16(half).view(np.float16)
                got.append(float(np.float16(np.float32(v) * np.float32(one) + np.float32(m1152))))
        assert got == [float(q) for q in qs]


def _bf16(bits):
    return float(np.array([bits << 16], dtype=np.uint32).view(np.float32)[0])


def _f16(bits):
    return float(np.uint16(bits).view(np.float16))


def test_q4_unpack_constants_give_exact_codes():
    # GEMV (bf16): (w & 0x000F000F) | 0x43004300 is 128 + q in each half;
    # subtracting bf16 136 (0x4308) leaves q - 8 exactly
    assert _bf16(0x4300) == 128.0 and _bf16(0x4308) == 136.0
    for q in range(16):
        v = _bf16(0x4300 | q)
        assert v == 128.0 + q and float(np.float32(v) - np.float32(136.0)) == q - 8
    # attention (fp16): low nibble 0x6400 | q = 1024 + q, fma(., 1, -1032);
    # high nibble 0x6400 | (q << 4) = 1024 + 16 q, fma(., 1/16, -72); both q - 8
    assert _f16(0x3C00) == 1.0 and _f16(0xE408) == -1032.0
    assert _f16(0x2C00) == 1.0 / 16 and _f16(0xD480) == -72.0
    for q in range(16):
        lo, hi = _f16(0x6400 | q), _f16(0x6400 | (q << 4))
        assert lo == 1024.0 + q and hi == 1024.0 + 16 * q
        # each fma is exact (the result is a small integer), so fp16 rounding is moot
        assert float(np.float16(lo * 1.0 - 1032.0)) == q - 8
        assert float(np.float16(hi * (1.0 / 16) - 72.0)) == q - 8


@pytest.mark.parametrize("M", [1, 2, 3, 4, 5])
def test_gemv_shared_memory_carve_up(M):
    """Every shared-memory access of the GEMV in bounds, for the planned ring:
    consumer slot stores (and, with pair slots, column-1 adds), the
    epilogue's sums, for every reduction buffer; then the abort flag and the
    barriers (2 per stage, 2 per buffer, with pair slots one per slot of each
    buffer), ending at the planned size."""
    p = q4dec.plan_gemv(M, 17408, 5120, 148)
    S, stage = p.stages, _gemv_stage_bytes(M)
    bufs, nslot = _gemv_red_layout(M)
    red_floats = bufs * nslot * M * 132
    buf_base = lambda b: b * nslot * M * 132               # the kernel's gemv_red_buffer
    for b in range(bufs):
        top = buf_base(b) + nslot * M * 132
        assert top <= red_floats
        for blk in range(nslot):                            # consumer: its slot
            for t in range(4):
                for e in range(2):
                    m = 2 * t + e
                    if m >= M:
                        continue
                    for p_ in range(8):
                        for g in range(8):
                            for r in (g, g + 8):
                                i = buf_base(b) + blk * M * 132 + m * 132 + 16 * p_ + r
                                assert buf_base(b) <= i < top
        for e in range(2):                                  # epilogue warp e: rows 64e..64e+63
            for lane in range(32):
                for k in range(2 * M):
                    row = 64 * e + 32 * (k & 1) + lane
                    for w in range(nslot):
                        i = buf_base(b) + (k >> 1) * 132 + row + w * M * 132
                        assert buf_base(b) <= i < top
    red_off = S * stage
    bars = red_off + red_floats * 4 + 16                    # abort flag (padded to 16) first
    n_bars = 2 * S + 2 * bufs + (8 * bufs if _gemv_pair_slots(M) else 0)
    assert bars % 8 == 0 and bars + 8 * n_bars == p.smem_bytes <= SMEM_OPTIN
