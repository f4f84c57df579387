// Causal GQA flash-decode attention over a Q4_0 K/V cache, on tensor cores.
//
// What it computes: for draft row m at position p_m = ctx_len - M + m and
// query head h, softmax over tokens t <= p_m of s = scale * Q . Khat, applied
// to Vhat -- the K/V read that grows with context ("Qwen3.8-27B at 256K on a
// 24GB RTX PRO 4000 SFF (432 GB/s): 50 tok/s with MTP", paragraphs on the 16
// full-attention layers and on the 432 GB/s ceiling).
//
// Work split: grid = (context split, KV head, query-row group).  One CTA holds
// every query row that reads its KV head (g grouped heads x M draft rows, at
// most 32) so each K/V byte of its split leaves HBM once; the splits' softmax
// states are merged by a second kernel (log-sum-exp, base 2).  K and V tiles
// (contiguous: one super-block per token) stream into a ring of shared-memory
// stages by bulk copies on full/empty mbarriers with bounded waits.
//
// The kernel below (at most 8 query rows per CTA) computes, per tile:
//  1. Scores, exact up to fp32 rounding: ldmatrix hands lane (g, t) word t
//     of the 16-byte nibble piece of tokens g and g+8 (the A-fragment layout);
//     the nibbles become exact fp16 (q - 8); Q, converted to fp16 once, is
//     the B operand in the same element order; one fresh MMA accumulator per
//     32-element block is scaled by the token's block scale in fp32.
//     S^T = Khat Q^T arrives as (token, row) fragments.
//  2. Online softmax in base 2 (scale * log2 e folded in); P = 2^(s - m) is
//     rounded to fp16 and the row sums add the same rounded values, so
//     numerator and denominator see identical weights.
//  3. P.V as O^T = (q - 8)^T (P^T d): ldmatrix.trans pairs two tokens' bytes
//     of a V piece in one register, so the A operand (q - 8)^T [dims][tokens]
//     unpacks in registers, exact in fp16; the V block scale d goes into the
//     B operand, P^T times d of the same tokens in one fp16 multiply
//     (|P d| <= |d|: no overflow).  O^T accumulates in fp32.
// Each warp owns its own tokens, softmax state and full O^T.  More query rows
// per CTA (9..32) go to the tensor-memory kernel in q4kv_attn_tc.cuh; both
// write the same split states for the merge kernel at the end of this file.
// Built with Q4D_DEBUG, the K / V copies, the query loads and the output and
// state stores are index-checked (the *_in_range helpers below).
#pragma once

#include "q4dec_device.cuh"

namespace q4d {

constexpr int kAttnMaxRows = 32;                              // query rows per CTA, at most
constexpr int kHeadDim = 256;
constexpr int kRowBytes = 144;                                // one super-block per token

struct AttnArgs {
  const uint16_t* Q;   // bf16 bits [M][n_q][256]
  const uint8_t* K;    // [n_kv][kv_stride] super-blocks
  const uint8_t* V;
  float* out;          // [M][n_q][256]
  float* ws_o;         // [n_splits][M*n_q][256]
  float* ws_ml;        // [n_splits][M*n_q][2] (running max in log2 units, sum)
  unsigned* err;
  int ctx_len, n_q, n_kv, M, g, kv_stride;
  float scale_log2;    // softmax scale * log2(e)
  int n_splits, split_tokens, rows_per_cta, stages;
  long long ws_floats; // floats of the workspace (split states) that index checks allow
};

// Index checks shared by the attention kernels (always true without
// Q4D_DEBUG).  Token rows [t0, t0 + n) of KV head kh lie in the cache.
__device__ __forceinline__ bool kv_rows_in_range(const AttnArgs& a, int kh, int t0, int n) {
  return Q4D_CHECK(kh < a.n_kv && t0 >= 0 && n >= 1 && t0 + n <= a.kv_stride, a.err, kSiteAttnKV,
                   (long long)kh * a.kv_stride + t0);
}
// Query row m, head h exists.
__device__ __forceinline__ bool query_in_range(const AttnArgs& a, int m, int h) {
  return Q4D_CHECK(m < a.M && h < a.n_q, a.err, kSiteAttnQuery, (long long)m * a.n_q + h);
}
// Output row `row` (m * n_q + h) exists, and so does split `split`'s state
// for it, with every split's states inside the workspace.
__device__ __forceinline__ bool out_row_in_range(const AttnArgs& a, size_t row) {
  return Q4D_CHECK(row < size_t(a.M) * a.n_q, a.err, kSiteAttnOutput, row);
}
__device__ __forceinline__ bool state_in_range(const AttnArgs& a, int split, size_t row) {
  return Q4D_CHECK(split < a.n_splits && row < size_t(a.M) * a.n_q &&
                       size_t(a.n_splits) * a.M * a.n_q * (kHeadDim + 2) <= size_t(a.ws_floats),
                   a.err, kSiteAttnStates, (long long)split * a.M * a.n_q + row);
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                        uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_trans(uint32_t addr, uint32_t& r0, uint32_t& r1,
                                              uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x2_trans(uint32_t addr, uint32_t& r0, uint32_t& r1) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x2.trans.shared.b16 {%0,%1}, [%2];"
               : "=r"(r0), "=r"(r1)
               : "r"(addr));
}
__device__ __forceinline__ uint32_t movmatrix_trans(uint32_t x) {
  uint32_t r;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(r) : "r"(x));
  return r;
}
__device__ __forceinline__ uint32_t f16x2_fma(uint32_t a, uint32_t b, uint32_t c) {
  uint32_t r;
  asm("fma.rn.f16x2 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(c));
  return r;
}
__device__ __forceinline__ uint32_t f16x2_mul(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}
__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}
__device__ __forceinline__ void mma_f16(float (&c)[4], uint32_t a0, uint32_t a1,
                                              uint32_t a2, uint32_t a3, uint32_t b0,
                                              uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Fp16 pair q - 8 (exact) for the two tokens held in the halves of `r`:
// the nibble at bits 0-3 (LOW) or 4-7 (!LOW) of each half.  0x6400 | q is the
// fp16 value 1024 + q and 0x6400 | (q << 4) is 1024 + 16 q; one fma whose
// exact result is q - 8 finishes it.
template <bool LOW>
__device__ __forceinline__ uint32_t q8_pair(uint32_t r) {
  if (LOW)
    return f16x2_fma(lop3_and_or(r, 0x000F000Fu, 0x64006400u), 0x3C003C00u,
                     0xE408E408u /* -1032 */);
  return f16x2_fma(lop3_and_or(r, 0x00F000F0u, 0x64006400u), 0x2C002C00u /* 1/16 */,
                   0xD480D480u /* -72 */);
}

// Q fragments of one row, block b, lane t (16 bytes, fp16): the pairs
// (q[4t], q[4t+2]), (q[16+4t], q[16+4t+2]), (q[4t+1], q[4t+3]),
// (q[16+4t+1], q[16+4t+3]) of the block -- the element order in which word t
// of a K row's nibbles unpacks (k_pairs).  bf16 -> fp16 is exact for
// |q| in [2^-14, 65504]; smaller magnitudes round to fp16 subnormals.
__device__ __forceinline__ uint4 q_frag_f16(const uint16_t* q /* row + 32 b + 4 t */) {
  const uint2 lo = *reinterpret_cast<const uint2*>(q);
  const uint2 hi = *reinterpret_cast<const uint2*>(q + 16);
  auto f = [](uint32_t bits16) { return __uint_as_float(bits16 << 16); };
  uint4 v;
  v.x = pack_f16x2(f(lo.x & 0xFFFFu), f(lo.y & 0xFFFFu));
  v.y = pack_f16x2(f(hi.x & 0xFFFFu), f(hi.y & 0xFFFFu));
  v.z = pack_f16x2(f(lo.x >> 16), f(lo.y >> 16));
  v.w = pack_f16x2(f(hi.x >> 16), f(hi.y >> 16));
  return v;
}

// The eight nibbles of K word w as exact fp16 pairs q - 8, in the order
// (byte0.lo, byte2.lo), (byte0.hi, byte2.hi), (byte1.lo, byte3.lo),
// (byte1.hi, byte3.hi): one shift per word.
__device__ __forceinline__ void k_pairs(uint32_t w, uint32_t (&r)[4]) {
  r[0] = q8_pair<true>(w);
  r[1] = q8_pair<false>(w);
  r[2] = q8_pair<true>(w >> 8);
  r[3] = q8_pair<false>(w >> 8);
}

constexpr int kR8Warps = 12;                                   // consumer warps
constexpr int kR8QPitch = 8 * 4 * 16 + 64;                     // bytes per row of Q fragments
constexpr int kR8Threads = kR8Warps * 32;
constexpr int kR8Tile = 16 * kR8Warps;                         // 192 tokens per tile
constexpr uint32_t kR8StageBytes = 2u * kR8Tile * kRowBytes;   // K tile + V tile

// Shared memory of the warp-local variant: the ring (which also holds the
// final cross-warp combine, 96 KB), Q fragments of 8 rows, per-warp and
// per-row statistics, barriers, the abort flag (padded to 16).
__host__ __device__ constexpr size_t attn_rows8_smem_bytes(int stages) {
  return size_t(stages) * kR8StageBytes + 8 * kR8QPitch + size_t(kR8Warps) * 8 * 2 * 4 +
         8 * 2 * 4 + size_t(stages) * 16 + 16;
}

// Warp-local variant for at most 8 query rows per CTA (one row tile: plain
// decode, M = 1).  Twelve warps, each owning tokens 16w .. 16w + 15 of every
// 192-token tile, carry their own online softmax and their own O^T for all
// 256 dimensions (64 fp32 registers): a tile needs no CTA-wide barrier.  The
// score fragments (token, row) are rounded to fp16 and transposed in
// registers with movmatrix into the P^T operand of P.V.  Lane 0 of warp 0
// also issues the bulk copies (a separate producer warp would cut every
// thread's register budget); it blocks only for the tile it needs next.  The
// warps' states are combined once, at the end of the split.
__global__ void __launch_bounds__(kR8Threads, 1) q4kv_attn_split_rows8_kernel(const AttnArgs a) {
  constexpr int TT = kR8Tile;
  extern __shared__ __align__(128) uint8_t smem[];
  const int S = a.stages;
  uint8_t* ring = smem;
  uint8_t* Qf = ring + size_t(S) * kR8StageBytes;                 // [row] x kR8QPitch
  float* wml = reinterpret_cast<float*>(Qf + 8 * kR8QPitch);       // [warp][row][m, l]
  float* rml = wml + kR8Warps * 8 * 2;                              // [row][M, L]
  uint64_t* full = reinterpret_cast<uint64_t*>(rml + 8 * 2);
  uint64_t* empty = full + S;
  // set by the first wait that times out: from then on no wait blocks and no
  // further copy is issued (the results are void; the error word says so)
  volatile int* abort_flag = reinterpret_cast<volatile int*>(empty + S);

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int split = blockIdx.x, kh = blockIdx.y, rgrp = blockIdx.z;
  const int row0 = rgrp * a.rows_per_cta;
  const int R = min(a.rows_per_cta, a.g * a.M - row0);
  const int t_begin = split * a.split_tokens;
  const int t_end = min(a.ctx_len, t_begin + a.split_tokens);
  const int n_tiles = (t_end - t_begin + TT - 1) / TT;
  const bool producer = tid == 0;
  const uint8_t* Kh = a.K + size_t(kh) * a.kv_stride * kRowBytes;
  const uint8_t* Vh = a.V + size_t(kh) * a.kv_stride * kRowBytes;
  const uint64_t pol = l2_evict_first_policy();
  auto issue = [&](int tile) {
    int t0 = t_begin + tile * TT, n = min(TT, t_end - t0);
    const uint8_t *kp = Kh, *vp = Vh;
    if (!kv_rows_in_range(a, kh, t0, n)) {  // copy rows of the first head instead
      kp = a.K;
      vp = a.V;
      t0 = 0;
      n = max(1, min(n, a.ctx_len));
    }
    const uint32_t bytes = uint32_t(n) * kRowBytes;
    const int slot = tile % S;
    const uint32_t bar = smem_addr(&full[slot]);
    const uint32_t dk = smem_addr(ring + size_t(slot) * kR8StageBytes);
    mbar_arrive_expect_tx(bar, 2 * bytes);
    bulk_g2s(dk, kp + size_t(t0) * kRowBytes, bytes, bar, pol);
    bulk_g2s(dk + TT * kRowBytes, vp + size_t(t0) * kRowBytes, bytes, bar, pol);
  };

  int issued = 0;
  if (producer) {
    griddep_launch_dependents();  // a following weight-prefetching GEMV may start
    for (int s = 0; s < S; ++s) {
      mbar_init(smem_addr(&full[s]), 1);
      mbar_init(smem_addr(&empty[s]), kR8Warps);
    }
    *abort_flag = 0;
    mbar_init_fence();
    // start streaming before anything else
    for (; issued < min(S, n_tiles); ++issued) issue(issued);
  }
  // Q fragments (zero for padding rows)
  for (int i = tid; i < 8 * 32; i += kR8Threads) {
    const int r = i >> 5, b = (i >> 2) & 7, tt = i & 3;
    uint4 v = make_uint4(0u, 0u, 0u, 0u);
    if (r < R) {
      const int rr = row0 + r, m = rr / a.g, j = rr - m * a.g;
      if (query_in_range(a, m, kh * a.g + j))
        v = q_frag_f16(a.Q + (size_t(m) * a.n_q + kh * a.g + j) * kHeadDim + b * 32 + 4 * tt);
    }
    *reinterpret_cast<uint4*>(Qf + r * kR8QPitch + (i & 31) * 16) = v;
  }
  __syncthreads();

  const int g = lane >> 2, t = lane & 3;
  int row_pos[2];
  float m_run[2], l_run[2];
  #pragma unroll
  for (int e = 0; e < 2; ++e) {
    const int r = 2 * t + e;
    row_pos[e] = r < R ? a.ctx_len - a.M + (row0 + r) / a.g : -1;
    m_run[e] = -INFINITY;
    l_run[e] = 0.f;
  }
  float o[8][2][4];  // O^T: [block][dim tile][fragment]
  #pragma unroll
  for (int b = 0; b < 8; ++b)
    #pragma unroll
    for (int d = 0; d < 2; ++d) o[b][d][0] = o[b][d][1] = o[b][d][2] = o[b][d][3] = 0.f;

  const int tok0 = 16 * warp;
  // ldmatrix rows of this warp's 16 tokens: lanes 0-15 tokens tok0 + lane at
  // block b, lanes 16-31 tokens tok0 + lane - 16 at block b + 1
  const uint32_t lrow = uint32_t(tok0 + (lane & 15)) * kRowBytes + uint32_t(lane >> 4) * 16u;
  const uint4* qrow = reinterpret_cast<const uint4*>(Qf + g * kR8QPitch) + t;  // + 4 b
  int slot = 0;
  uint32_t phase = 0;

  #pragma unroll 1
  for (int tile = 0; tile < n_tiles; ++tile) {
    if (producer) {
      // refill the slots every warp has released; block only for this tile
      while (issued < n_tiles && issued < tile + S && !*abort_flag) {
        const uint32_t bar = smem_addr(&empty[issued % S]);
        const uint32_t parity = uint32_t(issued / S - 1) & 1u;
        if (issued > tile) {
          if (!mbar_test_wait(bar, parity)) break;
        } else if (!mbar_wait_or_abort(bar, parity, a.err, abort_flag)) {
          break;
        }
        issue(issued++);
      }
    }
    __syncwarp();
    const int t0 = t_begin + tile * TT;
    const int n_tok = min(TT, t_end - t0);
    mbar_wait_or_abort(smem_addr(&full[slot]), phase, a.err, abort_flag);
    const uint8_t* Kt = ring + size_t(slot) * kR8StageBytes;
    const uint8_t* Vt = Kt + TT * kRowBytes;
    if (tok0 < n_tok) {
      const uint32_t Kt_addr = smem_addr(Kt), Vt_addr = smem_addr(Vt);
      // ---- scores S^T (tokens tok0 + g, tok0 + g + 8; rows 2t, 2t + 1)
      float s[4] = {0.f, 0.f, 0.f, 0.f};
      const uint8_t* da_p = Kt + (tok0 + g) * kRowBytes + 128;
      const uint8_t* db_p = da_p + 8 * kRowBytes;
      #pragma unroll
      for (int b = 0; b < 8; b += 2) {
        uint32_t w0a, w0b, w1a, w1b;
        ldsm_x4(Kt_addr + lrow + uint32_t(b) * 16u, w0a, w0b, w1a, w1b);
        const float2 dA = __half22float2(*reinterpret_cast<const __half2*>(da_p + 2 * b));
        const float2 dB = __half22float2(*reinterpret_cast<const __half2*>(db_p + 2 * b));
        #pragma unroll
        for (int bb = 0; bb < 2; ++bb) {
          uint32_t qa[4], qb[4];
          k_pairs(bb ? w1a : w0a, qa);
          k_pairs(bb ? w1b : w0b, qb);
          const uint4 qv = qrow[4 * (b + bb)];
          float c[4] = {0.f, 0.f, 0.f, 0.f};
          mma_f16(c, qa[0], qb[0], qa[1], qb[1], qv.x, qv.y);
          mma_f16(c, qa[2], qb[2], qa[3], qb[3], qv.z, qv.w);
          const float da = bb ? dA.y : dA.x, db = bb ? dB.y : dB.x;
          s[0] = fmaf(da, c[0], s[0]);
          s[1] = fmaf(da, c[1], s[1]);
          s[2] = fmaf(db, c[2], s[2]);
          s[3] = fmaf(db, c[3], s[3]);
        }
      }
      // ---- warp-local online softmax (base 2)
      const int ta = tok0 + g, tb = ta + 8;
      float alpha[2];
      #pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int pos = row_pos[e];
        s[e] = (ta < n_tok && t0 + ta <= pos) ? s[e] * a.scale_log2 : -INFINITY;
        s[2 + e] = (tb < n_tok && t0 + tb <= pos) ? s[2 + e] * a.scale_log2 : -INFINITY;
        float mx = fmaxf(s[e], s[2 + e]);
        mx = fmaxf(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, 4));
        mx = fmaxf(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, 8));
        mx = fmaxf(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, 16));
        const float m_new = fmaxf(m_run[e], mx);
        // a row with no visible token so far (or a padding row) keeps
        // m = -inf, weight 0 and alpha = 1: nothing to rescale
        const float m_use = m_new == -INFINITY ? 0.f : m_new;
        alpha[e] = m_new == -INFINITY ? 1.f : ex2(m_run[e] - m_use);
        m_run[e] = m_new;
        s[e] = ex2(s[e] - m_use);
        s[2 + e] = ex2(s[2 + e] - m_use);
      }
      const uint32_t pa = pack_f16x2(s[0], s[1]);  // token ta, rows 2t, 2t + 1
      const uint32_t pb = pack_f16x2(s[2], s[3]);  // token tb
      {
        const float2 fa = __half22float2(*reinterpret_cast<const __half2*>(&pa));
        const float2 fb = __half22float2(*reinterpret_cast<const __half2*>(&pb));
        l_run[0] = l_run[0] * alpha[0] + fa.x + fb.x;
        l_run[1] = l_run[1] * alpha[1] + fa.y + fb.y;
      }
      // P^T B fragments: (tokens 2t, 2t + 1; row g) and (tokens 2t + 8, 2t + 9; row g)
      const uint32_t B0 = movmatrix_trans(pa), B1 = movmatrix_trans(pb);
      if (__any_sync(0xFFFFFFFFu, alpha[0] != 1.f || alpha[1] != 1.f)) {
        #pragma unroll
        for (int b = 0; b < 8; ++b)
          #pragma unroll
          for (int d = 0; d < 2; ++d) {
            o[b][d][0] *= alpha[0];
            o[b][d][1] *= alpha[1];
            o[b][d][2] *= alpha[0];
            o[b][d][3] *= alpha[1];
          }
      }
      // ---- V block scales of tokens 2t, 2t + 1, 2t + 8, 2t + 9 (all 8
      // blocks, as fp16 pairs (d_2i, d_2i+1)); zero past the tile end
      uint4 dw[4];
      #pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int tk = tok0 + 2 * t + (i & 1) + (i >> 1) * 8;
        dw[i] = *reinterpret_cast<const uint4*>(Vt + tk * kRowBytes + 128);
        if (tok0 + 16 > n_tok && tk >= n_tok) dw[i] = make_uint4(0u, 0u, 0u, 0u);
      }
      // ---- O^T[dims][rows] += (q - 8)^T (P^T d) over this warp's 16 tokens
      #pragma unroll
      for (int b = 0; b < 8; b += 2) {
        uint32_t v0, v1, v2, v3;  // blocks b (v0, v1) and b + 1 (v2, v3)
        ldsm_x4_trans(Vt_addr + lrow + uint32_t(b) * 16u, v0, v1, v2, v3);
        #pragma unroll
        for (int bb = 0; bb < 2; ++bb) {
          const uint32_t ra = bb ? v2 : v0, rb = bb ? v3 : v1;
          const int wd = (b + bb) >> 1;
          const uint32_t sel = ((b + bb) & 1) ? 0x7632u : 0x5410u;
          const uint32_t x0 = wd == 0 ? dw[0].x : wd == 1 ? dw[0].y : wd == 2 ? dw[0].z : dw[0].w;
          const uint32_t x1 = wd == 0 ? dw[1].x : wd == 1 ? dw[1].y : wd == 2 ? dw[1].z : dw[1].w;
          const uint32_t x2 = wd == 0 ? dw[2].x : wd == 1 ? dw[2].y : wd == 2 ? dw[2].z : dw[2].w;
          const uint32_t x3 = wd == 0 ? dw[3].x : wd == 1 ? dw[3].y : wd == 2 ? dw[3].z : dw[3].w;
          const uint32_t p0 = f16x2_mul(B0, prmt(x0, x1, sel));
          const uint32_t p1 = f16x2_mul(B1, prmt(x2, x3, sel));
          mma_f16(o[b + bb][0], q8_pair<true>(ra), q8_pair<false>(ra), q8_pair<true>(rb),
                  q8_pair<false>(rb), p0, p1);
          mma_f16(o[b + bb][1], q8_pair<true>(ra >> 8), q8_pair<false>(ra >> 8),
                  q8_pair<true>(rb >> 8), q8_pair<false>(rb >> 8), p0, p1);
        }
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(smem_addr(&empty[slot]));
    if (++slot == S) {
      slot = 0;
      phase ^= 1u;
    }
  }

  // After a time-out: wait (bounded) for the copies still in flight -- the
  // last tile issued into each slot -- before the ring is reused below and
  // before the CTA exits.
  if (producer && *abort_flag)
    for (int tile = max(0, issued - S); tile < issued; ++tile)
      mbar_wait(smem_addr(&full[tile % S]), uint32_t(tile / S) & 1u, a.err);

  // ---- combine the warps: per-row maxima and sums, then O^T parked in the
  // (now idle) ring as [warp][row][dim] and summed in warp order
  #pragma unroll
  for (int e = 0; e < 2; ++e) {
    float l = l_run[e];
    l += __shfl_xor_sync(0xFFFFFFFFu, l, 4);
    l += __shfl_xor_sync(0xFFFFFFFFu, l, 8);
    l += __shfl_xor_sync(0xFFFFFFFFu, l, 16);
    if (g == 0) {
      wml[(warp * 8 + 2 * t + e) * 2 + 0] = m_run[e];
      wml[(warp * 8 + 2 * t + e) * 2 + 1] = l;
    }
  }
  __syncthreads();
  float cw[2];
  #pragma unroll
  for (int e = 0; e < 2; ++e) {
    const int r = 2 * t + e;
    float M = -INFINITY;
    for (int w = 0; w < kR8Warps; ++w) M = fmaxf(M, wml[(w * 8 + r) * 2]);
    const float m_use = M == -INFINITY ? 0.f : M;
    cw[e] = ex2(m_run[e] - m_use);
    if (warp == 0 && g == 0) {
      float L = 0.f;
      for (int w = 0; w < kR8Warps; ++w)
        L += wml[(w * 8 + r) * 2 + 1] * ex2(wml[(w * 8 + r) * 2] - m_use);
      rml[r * 2 + 0] = M;
      rml[r * 2 + 1] = L;
    }
  }
  float* park = reinterpret_cast<float*>(ring) + warp * 8 * kHeadDim;
  #pragma unroll
  for (int b = 0; b < 8; ++b)
    #pragma unroll
    for (int d = 0; d < 2; ++d)
      #pragma unroll
      for (int k = 0; k < 4; ++k)
        park[(2 * t + (k & 1)) * kHeadDim + 32 * b + 2 * g + d + (k >= 2 ? 16 : 0)] =
            o[b][d][k] * cw[k & 1];
  __syncthreads();
  const float* parked = reinterpret_cast<const float*>(ring);
  const size_t rows_total = size_t(a.M) * a.n_q;
  for (int i = tid; i < R * kHeadDim; i += kR8Threads) {
    const int r = i / kHeadDim, dim = i - r * kHeadDim;
    float acc = 0.f;
    #pragma unroll
    for (int w = 0; w < kR8Warps; ++w) acc += parked[(w * 8 + r) * kHeadDim + dim];
    const int rr = row0 + r, m = rr / a.g, j = rr - m * a.g;
    const size_t row = size_t(m) * a.n_q + kh * a.g + j;
    if (a.n_splits == 1) {
      if (out_row_in_range(a, row)) a.out[row * kHeadDim + dim] = acc / rml[r * 2 + 1];
    } else if (state_in_range(a, split, row)) {
      a.ws_o[(size_t(split) * rows_total + row) * kHeadDim + dim] = acc;
      if (dim == 0) {
        a.ws_ml[(size_t(split) * rows_total + row) * 2 + 0] = rml[r * 2 + 0];
        a.ws_ml[(size_t(split) * rows_total + row) * 2 + 1] = rml[r * 2 + 1];
      }
    }
  }
}

// Log-sum-exp merge of the per-split states (base 2); one CTA of eight warps
// per (draft row, head).  Launched so that its CTAs may start while the split
// kernel still runs (programmatic dependent launch): they read the split
// states only once that kernel has completed.  Every warp finds the global maximum and the total
// weight itself; warp w then adds splits w, w + 8, ... for all 256
// dimensions (two float4 per lane), and the eight partial vectors are summed
// in warp order.
__global__ void __launch_bounds__(256) q4kv_attn_merge_kernel(const AttnArgs a) {
  const int row = blockIdx.x;  // m * n_q + h
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (tid == 0) griddep_launch_dependents();
  griddep_wait();  // the split kernel has finished: its states are visible
  const size_t rows = size_t(a.M) * a.n_q;
  if (!state_in_range(a, a.n_splits - 1, row)) return;  // every split's state of this row
  __shared__ float part[8 * kHeadDim];
  const int n = a.n_splits;
  float mx = -INFINITY;
  for (int c = lane; c < n; c += 32) mx = fmaxf(mx, a.ws_ml[(c * rows + row) * 2]);
  #pragma unroll
  for (int off = 16; off >= 1; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, off));
  float L = 0.f;
  for (int c = lane; c < n; c += 32) {
    const float mc = a.ws_ml[(c * rows + row) * 2];
    if (mc != -INFINITY) L += a.ws_ml[(c * rows + row) * 2 + 1] * ex2(mc - mx);
  }
  #pragma unroll
  for (int off = 16; off >= 1; off >>= 1) L += __shfl_xor_sync(0xFFFFFFFFu, L, off);
  float4 acc0 = make_float4(0.f, 0.f, 0.f, 0.f), acc1 = acc0;
  #pragma unroll 4
  for (int c = warp; c < n; c += 8) {
    const float mc = a.ws_ml[(c * rows + row) * 2];
    const float wc = mc == -INFINITY ? 0.f : ex2(mc - mx);
    const float4* src = reinterpret_cast<const float4*>(a.ws_o + (c * rows + row) * kHeadDim);
    const float4 v0 = src[lane], v1 = src[32 + lane];
    acc0.x = fmaf(wc, v0.x, acc0.x);
    acc0.y = fmaf(wc, v0.y, acc0.y);
    acc0.z = fmaf(wc, v0.z, acc0.z);
    acc0.w = fmaf(wc, v0.w, acc0.w);
    acc1.x = fmaf(wc, v1.x, acc1.x);
    acc1.y = fmaf(wc, v1.y, acc1.y);
    acc1.z = fmaf(wc, v1.z, acc1.z);
    acc1.w = fmaf(wc, v1.w, acc1.w);
  }
  reinterpret_cast<float4*>(part + warp * kHeadDim)[lane] = acc0;
  reinterpret_cast<float4*>(part + warp * kHeadDim)[32 + lane] = acc1;
  __syncthreads();
  float sum = 0.f;
  #pragma unroll
  for (int w = 0; w < 8; ++w) sum += part[w * kHeadDim + tid];
  if (out_row_in_range(a, row)) a.out[size_t(row) * kHeadDim + tid] = sum / L;
}

}  // namespace q4d
