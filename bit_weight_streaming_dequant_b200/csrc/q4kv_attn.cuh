// Causal GQA flash-decode attention over a Q4_0 K/V cache (CUDA cores).
//
// What it computes: for draft row m at position p_m = ctx_len - M + m and
// query head h, softmax over tokens t <= p_m of s = scale * Q . Khat, applied
// to Vhat -- the K/V read that grows with context ("Qwen3.8-27B at 256K on a
// 24GB RTX PRO 4000 SFF (432 GB/s): 50 tok/s with MTP", paragraphs on the 16
// full-attention layers and on the 432 GB/s ceiling).
//
// Design:
//  * Grid = (context split, KV head, query-row group).  One CTA holds every
//    query row that reads its KV head (g grouped heads x M draft rows, up to
//    32), so each K/V byte of its split is read from HBM exactly once.
//  * K and V tiles of 64 tokens stream through a shared-memory ring with
//    cp.async.bulk completing on mbarriers (bounded waits).
//  * Per tile: scores (thread = token x row group, block scale applied once
//    per 32-element block), online softmax (warp per query row), then P.V
//    (thread = output dimension, nibble dequantised in registers).
//  * Each split writes its running (max, sum, unnormalised o); a second kernel
//    merges the splits with log-sum-exp weights.  A single split writes the
//    normalised output directly.
#pragma once

#include "q4dec_device.cuh"

namespace q4d {

constexpr int kAttnThreads = 256;
constexpr int kAttnTileTokens = 64;
constexpr int kAttnMaxRows = 32;
constexpr int kHeadDim = 256;
constexpr int kRowBytes = 144;  // one super-block per token

struct AttnArgs {
  const uint16_t* Q;   // bf16 bits [M][n_q][256]
  const uint8_t* K;    // [n_kv][kv_stride] super-blocks
  const uint8_t* V;
  float* out;          // [M][n_q][256]
  float* ws_o;         // [n_splits][M*n_q][256]
  float* ws_ml;        // [n_splits][M*n_q][2]
  unsigned* err;
  int ctx_len, n_q, n_kv, M, g, kv_stride;
  float scale;
  int n_splits, split_tokens, rows_per_cta, stages;
};

__device__ __forceinline__ float nib_minus8(uint32_t q) {
  return __uint_as_float(0x4B000000u | q) - 8388616.0f;  // (2^23 + q) - (2^23 + 8)
}

__global__ void __launch_bounds__(kAttnThreads, 2) q4kv_attn_split_kernel(const AttnArgs a) {
  constexpr int TT = kAttnTileTokens, RM = kAttnMaxRows;
  extern __shared__ __align__(128) uint8_t smem[];
  float* Qs = reinterpret_cast<float*>(smem);                       // [RM][256]
  uint8_t* ring = smem + RM * kHeadDim * 4;                          // [stages][2][TT*144]
  float* Ps = reinterpret_cast<float*>(ring + size_t(a.stages) * 2 * TT * kRowBytes);  // [TT][RM]
  float* m_run = Ps + TT * RM;
  float* l_run = m_run + RM;
  float* alpha = l_run + RM;
  uint64_t* bars = reinterpret_cast<uint64_t*>(alpha + RM);

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int split = blockIdx.x, kh = blockIdx.y, rgrp = blockIdx.z;
  const int R_all = a.g * a.M;
  const int row0 = rgrp * a.rows_per_cta;
  const int R = min(a.rows_per_cta, R_all - row0);
  const int t_begin = split * a.split_tokens;
  const int t_end = min(a.ctx_len, t_begin + a.split_tokens);
  const int n_tiles = (t_end - t_begin + TT - 1) / TT;
  const uint8_t* Kh = a.K + size_t(kh) * a.kv_stride * kRowBytes;
  const uint8_t* Vh = a.V + size_t(kh) * a.kv_stride * kRowBytes;

  if (tid == 0) {
    for (int s = 0; s < a.stages; ++s) mbar_init(smem_addr(&bars[s]), 1);
    mbar_init_fence();
  }
  __syncthreads();

  const uint64_t pol = l2_evict_first_policy();
  auto issue = [&](int tile) {
    const int slot = tile % a.stages;
    const int t0 = t_begin + tile * TT;
    const uint32_t bytes = uint32_t(min(TT, t_end - t0)) * kRowBytes;
    const uint32_t bar = smem_addr(&bars[slot]);
    const uint32_t dk = smem_addr(ring + size_t(slot) * 2 * TT * kRowBytes);
    mbar_arrive_expect_tx(bar, 2 * bytes);
    bulk_g2s(dk, Kh + size_t(t0) * kRowBytes, bytes, bar, pol);
    bulk_g2s(dk + TT * kRowBytes, Vh + size_t(t0) * kRowBytes, bytes, bar, pol);
  };
  if (tid == 0) {
    const int pre = min(a.stages, n_tiles);
    for (int t = 0; t < pre; ++t) issue(t);
  }

  // Stage the queries (scaled) as fp32, rows r = m*g + j of this row group.
  for (int i = tid; i < RM * kHeadDim; i += kAttnThreads) {
    const int r = i / kHeadDim, c = i - r * kHeadDim;
    float q = 0.f;
    if (r < R) {
      const int rr = row0 + r, m = rr / a.g, j = rr - m * a.g;
      const int h = kh * a.g + j;
      q = bf16_bits_to_float(a.Q[(size_t(m) * a.n_q + h) * kHeadDim + c]) * a.scale;
    }
    Qs[i] = q;
  }
  if (tid < RM) {
    m_run[tid] = -INFINITY;
    l_run[tid] = 0.f;
  }
  __syncthreads();

  // score-phase mapping: token st, rows sr0 + 4*i
  const int st = tid & (TT - 1);
  const int sr0 = tid >> 6;
  // PV-phase mapping: output dimension pd (block pb, byte pj, high nibble?)
  const int pd = tid;
  const int pb = pd >> 5, pe = pd & 31, pj = pe & 15;
  const bool phi = pe >= 16;

  float o[RM];
  #pragma unroll
  for (int r = 0; r < RM; ++r) o[r] = 0.f;

  for (int tile = 0; tile < n_tiles; ++tile) {
    const int slot = tile % a.stages;
    const int t0 = t_begin + tile * TT;
    const int n_tok = min(TT, t_end - t0);
    mbar_wait(smem_addr(&bars[slot]), uint32_t(tile / a.stages) & 1u, a.err);
    const uint8_t* Kt = ring + size_t(slot) * 2 * TT * kRowBytes;
    const uint8_t* Vt = Kt + TT * kRowBytes;

    // ---- scores
    {
      float s[RM / 4];
      #pragma unroll
      for (int i = 0; i < RM / 4; ++i) s[i] = 0.f;
      if (st < n_tok) {
        const uint8_t* krow = Kt + st * kRowBytes;
        #pragma unroll 1
        for (int b = 0; b < 8; ++b) {
          const uint4 nb = *reinterpret_cast<const uint4*>(krow + 16 * b);
          const float db = half_bits_to_float(*reinterpret_cast<const uint16_t*>(krow + 128 + 2 * b));
          const uint32_t wd[4] = {nb.x, nb.y, nb.z, nb.w};
          float kv[32];
          #pragma unroll
          for (int j = 0; j < 16; ++j) {
            const uint32_t byte = (wd[j >> 2] >> (8 * (j & 3))) & 0xFFu;
            kv[j] = nib_minus8(byte & 0xFu);
            kv[j + 16] = nib_minus8(byte >> 4);
          }
          #pragma unroll
          for (int i = 0; i < RM / 4; ++i) {
            const int r = sr0 + 4 * i;
            if (r < R) {
              const float4* q4 = reinterpret_cast<const float4*>(Qs + r * kHeadDim + 32 * b);
              float dot = 0.f;
              #pragma unroll
              for (int e = 0; e < 8; ++e) {
                const float4 qv = q4[e];
                dot = fmaf(kv[4 * e + 0], qv.x, dot);
                dot = fmaf(kv[4 * e + 1], qv.y, dot);
                dot = fmaf(kv[4 * e + 2], qv.z, dot);
                dot = fmaf(kv[4 * e + 3], qv.w, dot);
              }
              s[i] = fmaf(db, dot, s[i]);
            }
          }
        }
      }
      const int t_abs = t0 + st;
      #pragma unroll
      for (int i = 0; i < RM / 4; ++i) {
        const int r = sr0 + 4 * i;
        if (r < R) {
          const int m = (row0 + r) / a.g;
          const bool vis = st < n_tok && t_abs <= a.ctx_len - a.M + m;
          Ps[st * RM + r] = vis ? s[i] : -INFINITY;
        }
      }
    }
    __syncthreads();

    // ---- online softmax, one warp per query row
    for (int r = warp; r < R; r += kAttnThreads / 32) {
      const float s0 = Ps[lane * RM + r], s1 = Ps[(lane + 32) * RM + r];
      float mx = fmaxf(s0, s1);
      #pragma unroll
      for (int off = 16; off >= 1; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, off));
      const float m_old = m_run[r];
      const float m_new = fmaxf(m_old, mx);
      float p0 = 0.f, p1 = 0.f, al = 1.f;
      if (m_new != -INFINITY) {
        al = __expf(m_old - m_new);
        p0 = __expf(s0 - m_new);
        p1 = __expf(s1 - m_new);
      }
      float ps = p0 + p1;
      #pragma unroll
      for (int off = 16; off >= 1; off >>= 1) ps += __shfl_xor_sync(0xFFFFFFFFu, ps, off);
      Ps[lane * RM + r] = p0;
      Ps[(lane + 32) * RM + r] = p1;
      __syncwarp();
      if (lane == 0) {
        m_run[r] = m_new;
        l_run[r] = al * l_run[r] + ps;
        alpha[r] = al;
      }
    }
    __syncthreads();

    // ---- o = alpha * o + P V, thread per output dimension
    {
      #pragma unroll
      for (int r = 0; r < RM; ++r)
        if (r < R) o[r] *= alpha[r];
      #pragma unroll 2
      for (int t = 0; t < n_tok; ++t) {
        const uint8_t* vrow = Vt + t * kRowBytes;
        const uint32_t byte = vrow[16 * pb + pj];
        const float dv = half_bits_to_float(*reinterpret_cast<const uint16_t*>(vrow + 128 + 2 * pb));
        const float v = dv * nib_minus8(phi ? (byte >> 4) : (byte & 0xFu));
        const float4* p4 = reinterpret_cast<const float4*>(Ps + t * RM);
        #pragma unroll
        for (int q = 0; q < RM / 4; ++q) {
          if (4 * q < R) {
            const float4 pv = p4[q];
            o[4 * q + 0] = fmaf(pv.x, v, o[4 * q + 0]);
            o[4 * q + 1] = fmaf(pv.y, v, o[4 * q + 1]);
            o[4 * q + 2] = fmaf(pv.z, v, o[4 * q + 2]);
            o[4 * q + 3] = fmaf(pv.w, v, o[4 * q + 3]);
          }
        }
      }
    }
    __syncthreads();
    if (tid == 0 && tile + a.stages < n_tiles) issue(tile + a.stages);
  }

  // ---- write this split's state (or the final output for a single split)
  #pragma unroll
  for (int r = 0; r < RM; ++r) {
    if (r < R) {
      const int rr = row0 + r, m = rr / a.g, j = rr - m * a.g;
      const int row = m * a.n_q + kh * a.g + j;  // (m, h) flattened
      if (a.n_splits == 1) {
        a.out[size_t(row) * kHeadDim + pd] = o[r] / l_run[r];
      } else {
        a.ws_o[(size_t(split) * a.M * a.n_q + row) * kHeadDim + pd] = o[r];
        if (pd == 0) {
          a.ws_ml[(size_t(split) * a.M * a.n_q + row) * 2 + 0] = m_run[r];
          a.ws_ml[(size_t(split) * a.M * a.n_q + row) * 2 + 1] = l_run[r];
        }
      }
    }
  }
}

// Log-sum-exp merge of the per-split states; one CTA per (draft row, head).
__global__ void __launch_bounds__(kHeadDim) q4kv_attn_merge_kernel(const AttnArgs a) {
  const int row = blockIdx.x;  // m * n_q + h
  const int d = threadIdx.x;
  const size_t rows = size_t(a.M) * a.n_q;
  float mx = -INFINITY;
  for (int c = 0; c < a.n_splits; ++c) mx = fmaxf(mx, a.ws_ml[(c * rows + row) * 2]);
  float L = 0.f, acc = 0.f;
  for (int c = 0; c < a.n_splits; ++c) {
    const float mc = a.ws_ml[(c * rows + row) * 2];
    const float w = (mc == -INFINITY) ? 0.f : __expf(mc - mx);
    L = fmaf(a.ws_ml[(c * rows + row) * 2 + 1], w, L);
    acc = fmaf(a.ws_o[(c * rows + row) * kHeadDim + d], w, acc);
  }
  a.out[size_t(row) * kHeadDim + d] = acc / L;
}

}  // namespace q4d
