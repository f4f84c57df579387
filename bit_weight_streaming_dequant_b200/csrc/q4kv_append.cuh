// K/V cache append: quantise the new K and V rows of the M verified tokens
// into the Q4_0 cache (one 144-byte super-block per token per KV head).  The
// cache is Q4 ("Qwen3.8-27B at 256K on a 24GB RTX PRO 4000 SFF (432 GB/s):
// 50 tok/s with MTP", paragraph on the 16 full-attention layers); the
// quantiser is the signed-amax rule: amax = element of largest magnitude
// (first on ties), d = fp16(amax / -8), q = clamp(floor(v / d + 8.5), 0, 15)
// with the division and the addition rounded to nearest in fp32; a zero d
// stores +0 and q = 8.
//
// Work: one CTA per (token, KV head, K or V), one warp per 32-element block,
// one lane per element; a warp argmax finds amax, lanes 0..15 pack their
// element with the one 16 places later into a byte.
#pragma once

#include <cuda_fp16.h>

#include "q4dec_device.cuh"

namespace q4d {

struct AppendArgs {
  uint8_t* K;          // [n_kv][kv_stride] super-blocks
  uint8_t* V;
  const float* k_new;  // [M][n_kv][256]
  const float* v_new;
  unsigned* err;       // device error record (index checks of a Q4D_DEBUG build)
  int n_kv, kv_stride, pos, M;
};

__global__ void __launch_bounds__(256) q4kv_append_kernel(const AppendArgs a) {
  const int lane = threadIdx.x & 31, blk = threadIdx.x >> 5;
  const int row = blockIdx.x;                 // m * n_kv + h
  const int m = row / a.n_kv, h = row - m * a.n_kv;
  const bool is_v = blockIdx.y != 0;
  if (threadIdx.x == 0) griddep_launch_dependents();
  const float v = (is_v ? a.v_new : a.k_new)[size_t(row) * 256 + blk * 32 + lane];
  // argmax of |v| over the block, first index on ties
  float best = fabsf(v);
  int bi = lane;
  #pragma unroll
  for (int off = 16; off >= 1; off >>= 1) {
    const float ob = __shfl_xor_sync(0xFFFFFFFFu, best, off);
    const int oi = __shfl_xor_sync(0xFFFFFFFFu, bi, off);
    if (ob > best || (ob == best && oi < bi)) {
      best = ob;
      bi = oi;
    }
  }
  const float amax = __shfl_sync(0xFFFFFFFFu, v, bi);
  __half d16 = __float2half_rn(amax * -0.125f);   // amax / -8, exact before the fp16 rounding
  int q = 8;
  const float d = __half2float(d16);
  if (d != 0.f) {
    q = int(floorf(__fadd_rn(__fdiv_rn(v, d), 8.5f)));
    q = min(15, max(0, q));
  } else {
    d16 = __float2half_rn(0.f);                    // +0 for a zero scale
  }
  const int q_hi = __shfl_down_sync(0xFFFFFFFFu, q, 16);
  uint8_t* sb = (is_v ? a.V : a.K) + (size_t(h) * a.kv_stride + a.pos + m) * 144;
  if (!Q4D_CHECK(m < a.M && h < a.n_kv && a.pos >= 0 && a.pos + m < a.kv_stride, a.err,
                 kSiteAppend, (long long)h * a.kv_stride + a.pos + m))
    return;
  if (lane < 16) sb[blk * 16 + lane] = uint8_t(q | (q_hi << 4));
  if (lane == 0) *reinterpret_cast<__half*>(sb + 128 + 2 * blk) = d16;
}

}  // namespace q4d
