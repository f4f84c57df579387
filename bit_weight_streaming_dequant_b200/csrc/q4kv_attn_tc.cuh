// Causal GQA flash-decode attention over the Q4_0 K/V cache on the
// 5th-generation tensor cores (tcgen05, tensor memory).
//
// The same computation as the split kernels in q4kv_attn.cuh ("Qwen3.8-27B at
// 256K on a 24GB RTX PRO 4000 SFF (432 GB/s): 50 tok/s with MTP", paragraphs
// on the 16 full-attention layers and on the 432 GB/s ceiling), organised so
// that the multiply-adds leave the SM's issue slots (one thread issues every
// MMA, the tensor core runs them asynchronously) and the remaining per-element
// work runs as a pipeline of warp roles over 128-token tiles:
//  * K warps (4): unpack their token's K row with the block scale folded in
//    (fp16 d * (q - 8), one rounding) into tensor memory, one token per lane;
//  * MMA warp: S^T = Khat Q^T, one chain of M = 128 (tokens) x N (query rows)
//    x K = 16 MMAs with A in tensor memory and Q (fp16, in the unpacked
//    element order) in shared memory; then O^T += Vhat^T P^T, two M = 128
//    (dimensions) x N x K = 16 chains per 16 tokens, operands in shared
//    memory;
//  * softmax warps (4): scores in base 2, exact per-tile row maxima (warp
//    maxima by redux.sync, four warps combined in shared memory), O^T
//    rescaled in tensor memory when a row maximum grows, P rounded to fp16
//    (the row sums add the rounded values), P^T stored N-major in one of two
//    buffers, so that the softmax of a tile overlaps the P.V of the last;
//  * V warps (4): the unpacked V tile (fp16 d * (q - 8), M-major, dimensions
//    in the unpacked order), one half of the dimensions at a time so that
//    each half is rewritten as soon as its P.V chain has read it;
//  * producer warp: K and V tiles through a ring of bulk copies.
// The split states use the workspace layout of the other split kernels, so the
// same merge kernel finishes the job.  Every wait is bounded in time.
//
// The same kernel serves the 8-bit cache variant (Q8: 272-byte super-blocks
// of 256 int8 values and 8 fp16 scales, the `--cache-type-k/v q8_0` cache of
// "Running Qwen3.8-27B on an RTX 4090"): only the row size and the unpack
// (fp16 d * q, elements in their natural order) change.
#pragma once

#include <climits>

#include "q4dec_device.cuh"
#include "q4kv_attn.cuh"

namespace q4d {

constexpr int kTcaRoleWarps = 4;                       // warps per role: one per TMEM lane quadrant
constexpr int kTcaProducerWarp = 3 * kTcaRoleWarps;    // warps 0-3 softmax, 4-7 K, 8-11 V
constexpr int kTcaMmaWarp = kTcaProducerWarp + 1;
constexpr int kTcaThreads = (kTcaMmaWarp + 1) * 32;
constexpr int kTcaTile = 128;                          // tokens per tile (TMEM lanes)
constexpr uint32_t kTcaVBytes = 256u * kTcaTile * 2u;  // unpacked V tile, fp16

// Bytes of one token row (one super-block) of the cache, and of a ring stage
// (a K tile and a V tile).
__host__ __device__ constexpr uint32_t tca_row_bytes(bool q8) { return q8 ? 272u : 144u; }
__host__ __device__ constexpr uint32_t tca_stage_bytes(bool q8) {
  return 2u * kTcaTile * tca_row_bytes(q8);
}
constexpr int kTcaBarriers = 12;                       // besides the ring's 2 per stage

// Element (within its 32-element block) that K position kk (0..31) of the
// unpacked register order holds: column c = kk / 2 of a block holds pair
// i = c % 4 of word t = c / 4, its low (kk even) or high half; pair i of word
// t: i = 0 -> (4t, 4t+2), 1 -> (16+4t, 18+4t), 2 -> (4t+1, 4t+3),
// 3 -> (17+4t, 19+4t).
__host__ __device__ constexpr int unpacked_element(int kk) {
  return ((((kk >> 1) & 3) & 1) ? 16 : 0) + 4 * ((kk >> 1) >> 2) + (((kk >> 1) & 3) >> 1) +
         2 * (kk & 1);
}

// Shared memory for NR (16 or 32) MMA columns of query rows, S stages and PB
// (1 or 2) P^T buffers: ring, Q, V tile, P^T, row statistics ([4][32] +
// 5 x [32]), flags, barriers.
__host__ __device__ constexpr size_t tca_smem_bytes(int NR, int stages, bool q8, int PB) {
  return size_t(stages) * tca_stage_bytes(q8) + size_t(512) * NR + kTcaVBytes +
         size_t(NR) * 256 * PB +
         4 * 32 * 4 + 5 * 32 * 4 + 16 + size_t(2 * stages + kTcaBarriers) * 8 + 8;
}

// 8 dimensions (word t of a block, the unpacked order) of fp16 d * (q - 8).
__device__ __forceinline__ uint4 tca_scaled_word(uint32_t w, uint32_t d2) {
  return make_uint4(f16x2_mul(q8_pair<true>(w), d2), f16x2_mul(q8_pair<false>(w), d2),
                    f16x2_mul(q8_pair<true>(w >> 8), d2), f16x2_mul(q8_pair<false>(w >> 8), d2));
}

// Q8: fp16 pairs d * q of the four int8 values of w, (byte 0, byte 1) and
// (byte 2, byte 3).  q ^ 0x80 = q + 128 is the low byte of the fp16 value
// 1024 + q + 128 (high byte 0x64); subtracting 1152 leaves q exactly; one
// multiply rounds d * q once.
__device__ __forceinline__ void tca_scaled_q8_word(uint32_t w, uint32_t d2, uint32_t& lo,
                                                   uint32_t& hi) {
  const uint32_t x = w ^ 0x80808080u;
  lo = f16x2_mul(f16x2_fma(prmt(x, 0x64646464u, 0x4140u), 0x3C003C00u, 0xE480E480u), d2);
  hi = f16x2_mul(f16x2_fma(prmt(x, 0x64646464u, 0x4342u), 0x3C003C00u, 0xE480E480u), d2);
}

// The 16 fp16 pairs (d folded) of block b of a token row, in tensor-memory
// column order: Q4 in the unpacked element order, Q8 in element order.
template <bool Q8>
__device__ __forceinline__ void tca_block(const uint8_t* row, int b, uint32_t d2,
                                          uint32_t (&o)[16]) {
  if constexpr (!Q8) {
    const uint4 w = *reinterpret_cast<const uint4*>(row + 16 * b);
    const uint32_t w4[4] = {w.x, w.y, w.z, w.w};
    #pragma unroll
    for (int t = 0; t < 4; ++t) {
      const uint4 v = tca_scaled_word(w4[t], d2);
      o[4 * t + 0] = v.x;
      o[4 * t + 1] = v.y;
      o[4 * t + 2] = v.z;
      o[4 * t + 3] = v.w;
    }
  } else {
    const uint4 w0 = *reinterpret_cast<const uint4*>(row + 32 * b);
    const uint4 w1 = *reinterpret_cast<const uint4*>(row + 32 * b + 16);
    const uint32_t w8[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
    #pragma unroll
    for (int i = 0; i < 8; ++i) tca_scaled_q8_word(w8[i], d2, o[2 * i], o[2 * i + 1]);
  }
}

// Element of a block that position kk (0..31) of the column order holds.
template <bool Q8>
__host__ __device__ constexpr int tca_element(int kk) {
  return Q8 ? kk : unpacked_element(kk);
}

// fp16 scale of block b (0..7) from the row's 16 scale bytes, in both halves
// (0 for a token past the end of the tile's data).
__device__ __forceinline__ uint32_t tca_scale2(const uint4& dv, int b, bool live) {
  const uint32_t w = (b < 2) ? dv.x : (b < 4) ? dv.y : (b < 6) ? dv.z : dv.w;
  return live ? prmt(w, 0u, (b & 1) ? 0x3232u : 0x1010u) : 0u;
}

// NR: MMA columns of query rows (16 or 32); Q8: the 8-bit cache; PB: P^T
// buffers (2 lets the softmax of a tile overlap the previous P.V; 1 when
// shared memory holds no more).
template <int NR, bool Q8, int PB>
__global__ void __launch_bounds__(kTcaThreads, 1) q4kv_attn_tc_kernel(const AttnArgs a) {
  static_assert(NR == 16 || NR == 32, "query rows per CTA: 16 or 32 MMA columns");
  static_assert(PB == 1 || PB == 2, "one or two P^T buffers");
  constexpr int TT = kTcaTile;
  constexpr uint32_t RB = tca_row_bytes(Q8);           // bytes per token row
  constexpr uint32_t kStage = tca_stage_bytes(Q8);
  constexpr uint32_t kScales = Q8 ? 256u : 128u;       // offset of the 8 fp16 scales
  constexpr uint32_t kIdescQK = idesc_f16(128, NR, 0, 0);
  constexpr uint32_t kIdescPV = idesc_f16(128, NR, 1, 1);
  extern __shared__ __align__(128) uint8_t smem[];
  const int S = a.stages;
  uint8_t* ring = smem;
  uint8_t* Qs = ring + size_t(S) * kStage;
  uint8_t* Vs = Qs + 512 * NR;
  uint8_t* Ps = Vs + kTcaVBytes;
  float* wred = reinterpret_cast<float*>(Ps + NR * 256 * PB);   // [4][32]; P^T [PB][NR * 256]
  float* m_run = wred + 4 * 32;
  float* m_use = m_run + 32;
  float* alph = m_use + 32;
  float* lsum = alph + 32;
  int* rpos = reinterpret_cast<int*>(lsum + 32);            // causal limit of each row
  int* flags = rpos + 32;          // [0] some row's maximum grew, [1] abort
  // set by the first wait that times out: from then on no wait blocks and no
  // further copy is issued (the results are void; the error word says so)
  volatile int* abort_flag = flags + 1;
  uint64_t* full = reinterpret_cast<uint64_t*>(flags + 4);
  uint64_t* empty = full + S;
  uint64_t* kready = empty + S;   // [2] K tile in tensor memory
  uint64_t* sdone = kready + 2;   // [2] S^T written
  uint64_t* pready = sdone + 2;   // [2] P^T buffer stored (and O^T rescaled)
  uint64_t* pfree = pready + 2;   // [2] P^T buffer read by its P.V
  uint64_t* vready = pfree + 2;   // [2] V half stored
  uint64_t* pvdone = vready + 2;  // [2] P.V half finished
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(pvdone + 2);

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int split = blockIdx.x, kh = blockIdx.y, rgrp = blockIdx.z;
  const int row0 = rgrp * a.rows_per_cta;
  const int R = min(a.rows_per_cta, a.g * a.M - row0);
  const int t_begin = split * a.split_tokens;
  const int t_end = min(a.ctx_len, t_begin + a.split_tokens);
  const int n_tiles = (t_end - t_begin + TT - 1) / TT;
  // every token up to this one is visible to every row of the CTA
  const int all_visible = a.ctx_len - a.M + row0 / a.g;

  if (tid == 0) {
    griddep_launch_dependents();
    for (int s = 0; s < S; ++s) {
      mbar_init(smem_addr(&full[s]), 1);
      mbar_init(smem_addr(&empty[s]), 2 * kTcaRoleWarps);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(smem_addr(&kready[i]), kTcaRoleWarps * 32);
      mbar_init(smem_addr(&sdone[i]), 1);
      mbar_init(smem_addr(&vready[i]), kTcaRoleWarps * 32);
      mbar_init(smem_addr(&pvdone[i]), 1);
      mbar_init(smem_addr(&pready[i]), kTcaRoleWarps * 32);
      mbar_init(smem_addr(&pfree[i]), 1);
    }
    flags[1] = 0;
    mbar_init_fence();
  }
  // Q in the unpacked element order, K-major canonical layout (core matrices
  // of 8 rows x 8 elements); rows >= R are zero: their scores are 0 and their
  // outputs are never written
  for (int i = tid; i < NR * 256; i += kTcaThreads) {
    const int n = i >> 8, kp = i & 255;
    float v = 0.f;
    if (n < R) {
      const int rr = row0 + n, m = rr / a.g, j = rr - m * a.g;
      const int e = (kp & ~31) + tca_element<Q8>(kp & 31);
      if (query_in_range(a, m, kh * a.g + j))
        v = bf16_bits_to_float(a.Q[(size_t(m) * a.n_q + kh * a.g + j) * kHeadDim + e]);
    }
    *reinterpret_cast<__half*>(Qs + (kp >> 3) * (NR * 16) + (n >> 3) * 128 + (n & 7) * 16 +
                               (kp & 7) * 2) = __float2half_rn(v);
  }
  if (tid < 32) {
    m_run[tid] = -INFINITY;
    rpos[tid] = tid < R ? a.ctx_len - a.M + (row0 + tid) / a.g : INT_MAX;
  }
  if (warp == kTcaProducerWarp) {
    tmem_alloc(smem_addr(tmem_slot), 512);
    tmem_relinquish();
  }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // tensor memory columns: K tiles [2][128], S^T [2][NR], O^T halves [2][NR]
  const uint32_t tm_ak = tmem, tm_s = tmem + 256u, tm_o = tmem + 256u + 2u * NR;
  const int quad = warp & 3;
  const int k = 32 * quad + lane;                      // token of the tile (TMEM lane)
  const uint32_t lane_base = uint32_t(32 * quad) << 16;

  if (warp == kTcaProducerWarp) {
    // ------------------------------ producer ------------------------------
    if (lane == 0) {
      const uint8_t* Kh = a.K + size_t(kh) * a.kv_stride * RB;
      const uint8_t* Vh = a.V + size_t(kh) * a.kv_stride * RB;
      const uint64_t pol = l2_evict_first_policy();
      int issued = 0;
      for (int tile = 0; tile < n_tiles; ++tile) {
        const int slot = tile % S;
        if (tile >= S && !mbar_wait_or_abort(smem_addr(&empty[slot]), uint32_t(tile / S - 1) & 1u,
                                             a.err, abort_flag))
          break;  // no further copies after a time-out
        int t0 = t_begin + tile * TT, n = min(TT, t_end - t0);
        const uint8_t *kp = Kh, *vp = Vh;
        if (!kv_rows_in_range(a, kh, t0, n)) {  // copy rows of the first head instead
          kp = a.K;
          vp = a.V;
          t0 = 0;
          n = max(1, min(n, a.ctx_len));
        }
        const uint32_t bytes = uint32_t(n) * RB;
        const uint32_t bar = smem_addr(&full[slot]);
        const uint32_t dk = smem_addr(ring + size_t(slot) * kStage);
        mbar_arrive_expect_tx(bar, 2 * bytes);
        bulk_g2s(dk, kp + size_t(t0) * RB, bytes, bar, pol);
        bulk_g2s(dk + TT * RB, vp + size_t(t0) * RB, bytes, bar, pol);
        issued = tile + 1;
      }
      // after a time-out: wait (bounded) for the copies still in flight, the
      // last tile issued into each slot, before the CTA can exit
      if (*abort_flag)
        for (int tile = max(0, issued - S); tile < issued; ++tile)
          mbar_wait(smem_addr(&full[tile % S]), uint32_t(tile / S) & 1u, a.err);
    }
  } else if (warp == kTcaMmaWarp) {
    // ------------------------------ MMA issuer -----------------------------
    if (lane == 0) {
      auto qk = [&](int tile) {
        const int b = tile & 1;
        // S^T[b] is free: the P.V of tile - 2, issued before, waited for the
        // softmax warps to have read it (they read S^T before storing P^T)
        mbar_wait_or_abort(smem_addr(&kready[b]), uint32_t(tile >> 1) & 1u, a.err, abort_flag);
        tc_fence_after();
        const uint32_t qs = smem_addr(Qs);
        #pragma unroll
        for (int s = 0; s < 16; ++s)  // K = 256: 16 steps of 16, 8 TMEM columns each
          tc_mma_ts(tm_s + uint32_t(b * NR), tm_ak + uint32_t(b * 128 + 8 * s),
                    smem_desc(qs + uint32_t(s) * (NR * 32), NR * 16, 128), kIdescQK, uint32_t(s));
        tc_commit(smem_addr(&sdone[b]));
      };
      if (n_tiles > 0) qk(0);
      const uint32_t vs = smem_addr(Vs), ps = smem_addr(Ps);
      for (int tile = 0; tile < n_tiles; ++tile) {
        if (tile + 1 < n_tiles) qk(tile + 1);
        const int pb = tile % PB;
        mbar_wait_or_abort(smem_addr(&pready[pb]), uint32_t(tile / PB) & 1u, a.err, abort_flag);
        const uint32_t psb = ps + uint32_t(pb) * (NR * 256);
        #pragma unroll
        for (int h = 0; h < 2; ++h) {
          mbar_wait_or_abort(smem_addr(&vready[h]), uint32_t(tile) & 1u, a.err, abort_flag);
          tc_fence_after();
          #pragma unroll
          for (int j = 0; j < 8; ++j)  // 16 tokens per step
            tc_mma_ss(tm_o + uint32_t(h * NR),
                      smem_desc(vs + uint32_t(h) * (kTcaVBytes / 2) + uint32_t(j) * 256u, 128, 2048),
                      smem_desc(psb + uint32_t(j) * 256u, 128, 2048), kIdescPV,
                      (tile > 0 || j > 0) ? 1u : 0u);
          tc_commit(smem_addr(&pvdone[h]));
        }
        tc_commit(smem_addr(&pfree[pb]));
      }
      // every MMA issued has completed (the last commit tracks them all)
      // before tensor memory is read by the epilogue and freed -- also after a
      // time-out, when the waits above no longer hold the chain back
      if (n_tiles > 0)
        mbar_wait(smem_addr(&pfree[(n_tiles - 1) % PB]), uint32_t((n_tiles - 1) / PB) & 1u, a.err);
    }
  } else if (warp >= kTcaRoleWarps && warp < 2 * kTcaRoleWarps) {
    // ------------------------------ K warps --------------------------------
    for (int tile = 0; tile < n_tiles; ++tile) {
      const int slot = tile % S;
      mbar_wait_or_abort(smem_addr(&full[slot]), uint32_t(tile / S) & 1u, a.err, abort_flag);
      // K buffer (tile & 1) was last read by QK(tile - 2)
      if (tile >= 2) mbar_wait_or_abort(smem_addr(&sdone[tile & 1]), uint32_t((tile - 2) >> 1) & 1u, a.err, abort_flag);
      __syncwarp();  // the tensor-memory stores below are warp-collective
      tc_fence_after();
      const uint8_t* row = ring + size_t(slot) * kStage + k * RB;
      const bool live = k < t_end - (t_begin + tile * TT);
      const uint4 dv = *reinterpret_cast<const uint4*>(row + kScales);
      #pragma unroll 1
      for (int c = 0; c < 4; ++c) {  // blocks 2c, 2c + 1: 32 tensor-memory columns
        uint32_t r[32];
        #pragma unroll
        for (int bb = 0; bb < 2; ++bb) {
          const int b = 2 * c + bb;
          uint32_t o[16];
          tca_block<Q8>(row, b, tca_scale2(dv, b, live), o);
          #pragma unroll
          for (int i = 0; i < 16; ++i) r[16 * bb + i] = o[i];
        }
        tc_st32(tm_ak + lane_base + uint32_t((tile & 1) * 128 + 32 * c), r);
      }
      tc_wait_st();
      tc_fence_before();
      mbar_arrive(smem_addr(&kready[tile & 1]));
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_addr(&empty[slot]));
    }
  } else if (warp >= 2 * kTcaRoleWarps && warp < kTcaProducerWarp) {
    // ------------------------------ V warps --------------------------------
    for (int tile = 0; tile < n_tiles; ++tile) {
      const int slot = tile % S;
      mbar_wait_or_abort(smem_addr(&full[slot]), uint32_t(tile / S) & 1u, a.err, abort_flag);
      const uint8_t* row = ring + size_t(slot) * kStage + (TT + k) * RB;
      const bool live = k < t_end - (t_begin + tile * TT);
      const uint4 dv = *reinterpret_cast<const uint4*>(row + kScales);
      #pragma unroll 1
      for (int h = 0; h < 2; ++h) {
        // half h of the V tile was last read by the P.V chain of tile - 1
        if (tile > 0) mbar_wait_or_abort(smem_addr(&pvdone[h]), uint32_t(tile - 1) & 1u, a.err, abort_flag);
        #pragma unroll
        for (int bb = 0; bb < 4; ++bb) {
          const int b = 4 * h + bb;
          uint32_t o[16];
          tca_block<Q8>(row, b, tca_scale2(dv, b, live), o);
          #pragma unroll
          for (int t = 0; t < 4; ++t)  // 8 dimensions: one 16-byte chunk of the M-major tile
            *reinterpret_cast<uint4*>(Vs + (4 * b + t) * 2048 + (k >> 3) * 128 + (k & 7) * 16) =
                make_uint4(o[4 * t], o[4 * t + 1], o[4 * t + 2], o[4 * t + 3]);
        }
        fence_proxy_async_smem();
        mbar_arrive(smem_addr(&vready[h]));
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_addr(&empty[slot]));  // K and V of this tile are consumed
    }
  } else {
    // ------------------------------ softmax warps ---------------------------
    float l_part[NR];
    #pragma unroll
    for (int i = 0; i < NR; ++i) l_part[i] = 0.f;
    #pragma unroll 1
    for (int tile = 0; tile < n_tiles; ++tile) {
      const int t0 = t_begin + tile * TT;
      const int n_tok = min(TT, t_end - t0);
      mbar_wait_or_abort(smem_addr(&sdone[tile & 1]), uint32_t(tile >> 1) & 1u, a.err, abort_flag);
      __syncwarp();
      tc_fence_after();
      float s[NR];
      {
        uint32_t v[NR];
        if constexpr (NR == 32) {
          tc_ld32(tm_s + lane_base + uint32_t((tile & 1) * NR), v);
        } else {
          tc_ld16(tm_s + lane_base + uint32_t((tile & 1) * NR), v);
        }
        tc_wait_ld();
        #pragma unroll
        for (int i = 0; i < NR; ++i) s[i] = __uint_as_float(v[i]) * a.scale_log2;
      }
      if (n_tok < TT || t0 + TT - 1 > all_visible) {  // stale tokens, causal limits
        #pragma unroll
        for (int i = 0; i < NR; ++i)
          if (k >= n_tok || t0 + k > rpos[i]) s[i] = -INFINITY;
      }
      #pragma unroll
      for (int i = 0; i < NR; ++i) {
        const float mx = redux_max_f32(s[i]);
        if (lane == 0) wred[quad * 32 + i] = mx;
      }
      asm volatile("bar.sync 1, %0;" ::"n"(kTcaRoleWarps * 32) : "memory");
      if (tid < NR) {  // row tid: tile maximum, running maximum, rescale factor
        const float tmax = fmaxf(fmaxf(wred[tid], wred[32 + tid]), fmaxf(wred[64 + tid], wred[96 + tid]));
        const float mo = m_run[tid];
        const float mn = fmaxf(mo, tmax);
        const float mu = mn == -INFINITY ? 0.f : mn;
        const float al = mn == -INFINITY ? 1.f : ex2(mo - mu);
        m_run[tid] = mn;
        m_use[tid] = mu;
        alph[tid] = al;
        const int any = __any_sync(NR == 32 ? 0xFFFFFFFFu : 0x0000FFFFu, al != 1.f);
        if (tid == 0) flags[0] = any;
      }
      asm volatile("bar.sync 1, %0;" ::"n"(kTcaRoleWarps * 32) : "memory");
      const bool rescale = flags[0] != 0;
      uint32_t pp[NR / 2];
      #pragma unroll
      for (int i = 0; i < NR; i += 4) {
        const float4 mu4 = *reinterpret_cast<const float4*>(m_use + i);
        const float4 al4 = *reinterpret_cast<const float4*>(alph + i);
        pp[i / 2] = pack_f16x2(ex2(s[i] - mu4.x), ex2(s[i + 1] - mu4.y));
        pp[i / 2 + 1] = pack_f16x2(ex2(s[i + 2] - mu4.z), ex2(s[i + 3] - mu4.w));
        const float2 f0 = __half22float2(*reinterpret_cast<const __half2*>(&pp[i / 2]));
        const float2 f1 = __half22float2(*reinterpret_cast<const __half2*>(&pp[i / 2 + 1]));
        l_part[i] = fmaf(l_part[i], al4.x, f0.x);
        l_part[i + 1] = fmaf(l_part[i + 1], al4.y, f0.y);
        l_part[i + 2] = fmaf(l_part[i + 2], al4.z, f1.x);
        l_part[i + 3] = fmaf(l_part[i + 3], al4.w, f1.y);
      }
      // P^T buffer (tile % PB) is free once the P.V of tile - PB has read it;
      // O^T may be rescaled only after the P.V of tile - 1 has finished
      if (tile >= PB)
        mbar_wait_or_abort(smem_addr(&pfree[tile % PB]), uint32_t((tile - PB) / PB) & 1u, a.err, abort_flag);
      if (rescale && tile > 0) {
        mbar_wait_or_abort(smem_addr(&pvdone[1]), uint32_t(tile - 1) & 1u, a.err, abort_flag);
        __syncwarp();
        tc_fence_after();
        {
          // O^T column n (query row n) *= alpha[n], this warp's lanes, both halves
          #pragma unroll
          for (int c0 = 0; c0 < 2 * NR; c0 += 16) {
            uint32_t o[16];
            tc_ld16(tm_o + lane_base + uint32_t(c0), o);
            tc_wait_ld();
            #pragma unroll
            for (int i = 0; i < 16; ++i)
              o[i] = __float_as_uint(__uint_as_float(o[i]) * alph[(c0 + i) % NR]);
            tc_st16(tm_o + lane_base + uint32_t(c0), o);
          }
          tc_wait_st();
        }
      }
      uint8_t* Pb = Ps + (tile % PB) * (NR * 256);
      #pragma unroll
      for (int c = 0; c < NR / 8; ++c)  // rows 8c .. 8c + 7 of token k
        *reinterpret_cast<uint4*>(Pb + c * 2048 + (k >> 3) * 128 + (k & 7) * 16) =
            make_uint4(pp[4 * c], pp[4 * c + 1], pp[4 * c + 2], pp[4 * c + 3]);
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(smem_addr(&pready[tile % PB]));
    }
    // ---- split totals: row sums of the rounded P (after the last P.V)
    if (n_tiles > 0) {
      mbar_wait_or_abort(smem_addr(&pfree[(n_tiles - 1) % PB]), uint32_t((n_tiles - 1) / PB) & 1u, a.err, abort_flag);
      __syncwarp();
    }
    #pragma unroll
    for (int i = 0; i < NR; ++i) {
      float l = l_part[i];
      #pragma unroll
      for (int off = 16; off >= 1; off >>= 1) l += __shfl_xor_sync(0xFFFFFFFFu, l, off);
      if (lane == 0) wred[quad * 32 + i] = l;
    }
    asm volatile("bar.sync 1, %0;" ::"n"(kTcaRoleWarps * 32) : "memory");
    if (tid < NR) lsum[tid] = wred[tid] + wred[32 + tid] + wred[64 + tid] + wred[96 + tid];
  }

  // ---- epilogue: O^T half 0 by the softmax warps, half 1 by the K warps
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp < 2 * kTcaRoleWarps) {
    const int half = warp / kTcaRoleWarps;
    const int mm = 128 * half + k;                      // lane = unpacked dimension position
    const int dim = (mm & ~31) + tca_element<Q8>(mm & 31);
    const size_t rows_total = size_t(a.M) * a.n_q;
    #pragma unroll
    for (int c0 = 0; c0 < NR; c0 += 16) {
      uint32_t o[16];
      tc_ld16(tm_o + lane_base + uint32_t(half * NR + c0), o);
      tc_wait_ld();
      #pragma unroll
      for (int i = 0; i < 16; ++i) {
        const int n = c0 + i;
        if (n >= R) continue;
        const int rr = row0 + n, m = rr / a.g, j = rr - m * a.g;
        const size_t orow = size_t(m) * a.n_q + kh * a.g + j;
        const float ov = __uint_as_float(o[i]);
        if (a.n_splits == 1) {
          if (out_row_in_range(a, orow)) a.out[orow * kHeadDim + dim] = ov / lsum[n];
        } else if (state_in_range(a, split, orow)) {
          a.ws_o[(size_t(split) * rows_total + orow) * kHeadDim + dim] = ov;
          if (mm == 0) {
            a.ws_ml[(size_t(split) * rows_total + orow) * 2 + 0] = m_run[n];
            a.ws_ml[(size_t(split) * rows_total + orow) * 2 + 1] = lsum[n];
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == kTcaProducerWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace q4d
