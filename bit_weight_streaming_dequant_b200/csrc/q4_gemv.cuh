// Dequant-fused Q4_0 GEMV / skinny GEMM for M = 1..5 rows on CUDA cores.
//
// What it computes: y[m][n] = sum_k d(n,k) * (q(n,k) - 8) * x[m][k], the weight
// stream that dominates a decode step ("Qwen3.8-27B at 256K on a 24GB RTX PRO
// 4000 SFF (432 GB/s): 50 tok/s with MTP", paragraph beginning "NVIDIA quotes
// 432 GB/s"), with M = 2..5 rows sharing one pass over the weights when the
// target model verifies a drafted block ("Qwen3.8-27B on RTX 4090: 5,000 tok/s
// Prefill Reproduced", section "MTP helps ordinary prose ...").
//
// Design (B200):
//  * Each thread owns a fixed slice of K (W 32-bit nibble words = 8*W
//    elements) for the whole kernel, so its activations live in registers for
//    every row it touches; rows stream past it.  The activations are stored
//    pre-scaled so that the nibble -> float conversion is one LOP3 (nibble
//    OR'd into the mantissa of 2^23) plus one packed subtraction, and the
//    products use packed fp32 FMA (FFMA2) -- both exact.
//  * Each CTA (one per SM) owns a contiguous range of rows and pulls them
//    through a shared-memory ring with cp.async.bulk, completing on an
//    mbarrier; with an evict-first L2 policy since each weight is read once.
//  * Per-thread partial dot products of RSR rows are combined by a warp
//    reduce-scatter, then across the warps of a row stream in a fixed order
//    (deterministic, no atomics).
//  * If K is long relative to the thread budget, or there are fewer rows than
//    SMs, K is split into ranges whose fp32 partials are summed in a fixed
//    order by a second small kernel.
#pragma once

#include "q4dec_device.cuh"

namespace q4d {

constexpr int kGemvMaxThreads = 640;

struct GemvArgs {
  const uint8_t* W;    // super-blocks, N rows of nsb
  const uint16_t* x;   // bf16 bits [M][K]
  float* out;          // y [M][N] or partials [k_splits][M][N]
  unsigned* err;       // device error word
  int N, K, nsb;
  int k_splits, sb_base, sb_rem;
  int row_streams, tpr, stages, grid_rows;
  uint32_t slot_bytes;
};

constexpr int next_pow2(int v) { return v <= 1 ? 1 : 2 * next_pow2((v + 1) / 2); }

// Scale applied to nibble position p (0..7) of a word by the extraction below:
// positions 0..4 are used in place (bits 4p..4p+3), positions 5..7 from the
// word shifted right by 12 (bits 4p-12..4p-9).
__device__ __forceinline__ constexpr float nib_scale(int p) {
  return p <= 4 ? float(1u << (4 * p)) : float(1u << (4 * p - 12));
}

// Word -> 8 floats equal to (q_p - 8) * nib_scale(p).  The nibble placed in
// the low mantissa bits of 2^23 gives 2^23 + q*scale exactly; subtracting
// 2^23 + 8*scale (exact) leaves (q - 8) * scale.
__device__ __forceinline__ void dequant_word(uint32_t w, float2 (&t)[4]) {
  const uint32_t w12 = w >> 12;
  const float f0 = __uint_as_float(0x4B000000u | (w & 0x0000000Fu));
  const float f1 = __uint_as_float(0x4B000000u | (w & 0x000000F0u));
  const float f2 = __uint_as_float(0x4B000000u | (w & 0x00000F00u));
  const float f3 = __uint_as_float(0x4B000000u | (w & 0x0000F000u));
  const float f4 = __uint_as_float(0x4B000000u | (w & 0x000F0000u));
  const float f5 = __uint_as_float(0x4B000000u | (w12 & 0x00000F00u));
  const float f6 = __uint_as_float(0x4B000000u | (w12 & 0x0000F000u));
  const float f7 = __uint_as_float(0x4B000000u | (w12 & 0x000F0000u));
  constexpr float c23 = 8388608.0f;
  t[0] = __fadd2_rn(make_float2(f0, f1),
                    make_float2(-(c23 + 8.0f * nib_scale(0)), -(c23 + 8.0f * nib_scale(1))));
  t[1] = __fadd2_rn(make_float2(f2, f3),
                    make_float2(-(c23 + 8.0f * nib_scale(2)), -(c23 + 8.0f * nib_scale(3))));
  t[2] = __fadd2_rn(make_float2(f4, f5),
                    make_float2(-(c23 + 8.0f * nib_scale(4)), -(c23 + 8.0f * nib_scale(5))));
  t[3] = __fadd2_rn(make_float2(f6, f7),
                    make_float2(-(c23 + 8.0f * nib_scale(6)), -(c23 + 8.0f * nib_scale(7))));
}

template <int W>
__device__ __forceinline__ void load_words(const uint8_t* p, uint32_t (&wv)[W]) {
  if constexpr (W == 4) {
    const uint4 v = *reinterpret_cast<const uint4*>(p);
    wv[0] = v.x; wv[1] = v.y; wv[2] = v.z; wv[3] = v.w;
  } else if constexpr (W == 2) {
    const uint2 v = *reinterpret_cast<const uint2*>(p);
    wv[0] = v.x; wv[1] = v.y;
  } else {
    wv[0] = *reinterpret_cast<const uint32_t*>(p);
  }
}

// M: activation rows, W: nibble words per thread per row, RSR: rows each
// row stream handles per pipeline stage.
template <int M, int W, int RSR>
__global__ void __launch_bounds__(kGemvMaxThreads, 1) q4_gemv_kernel(const GemvArgs a) {
  constexpr int TPS = 32 / W;                 // threads per super-block
  constexpr int VPAD = next_pow2(RSR * M);    // reduce-scatter width (<= 32)
  static_assert(VPAD <= 32, "reduce-scatter holds at most one value per lane");

  extern __shared__ __align__(128) uint8_t smem[];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int nwarps = blockDim.x >> 5;
  const int ks = blockIdx.y;

  const int sb_count = a.sb_base + (ks < a.sb_rem ? 1 : 0);
  const int sb0 = ks * a.sb_base + min(ks, a.sb_rem);
  const uint32_t seg_bytes = uint32_t(sb_count) * 144u;

  const int row_begin = int((long long)a.N * blockIdx.x / a.grid_rows);
  const int row_end = int((long long)a.N * (blockIdx.x + 1) / a.grid_rows);
  const int rows_per_stage = a.row_streams * RSR;
  const int n_stages = (row_end - row_begin + rows_per_stage - 1) / rows_per_stage;

  uint8_t* slots = smem;
  float* red = reinterpret_cast<float*>(smem + size_t(a.stages) * a.slot_bytes);
  uint64_t* bars = reinterpret_cast<uint64_t*>(red + 2 * nwarps * VPAD);

  const int stream = tid / a.tpr;
  const int idx = tid - stream * a.tpr;
  const int sb_local = idx / TPS;
  const int word0 = (idx % TPS) * W;
  const int blk = word0 >> 2;
  const bool active = sb_local < sb_count;

  if (tid == 0) {
    for (int s = 0; s < a.stages; ++s) mbar_init(smem_addr(&bars[s]), 1);
    mbar_init_fence();
  }
  __syncthreads();

  const uint64_t pol = l2_evict_first_policy();
  auto issue = [&](int st) {
    const int slot = st % a.stages;
    const int r0 = row_begin + st * rows_per_stage;
    const int nr = min(rows_per_stage, row_end - r0);
    const uint32_t bar = smem_addr(&bars[slot]);
    const uint32_t dst = smem_addr(slots + size_t(slot) * a.slot_bytes);
    mbar_arrive_expect_tx(bar, uint32_t(nr) * seg_bytes);
    if (a.k_splits == 1) {
      bulk_g2s(dst, a.W + size_t(r0) * a.nsb * 144u, uint32_t(nr) * seg_bytes, bar, pol);
    } else {
      for (int r = 0; r < nr; ++r)
        bulk_g2s(dst + uint32_t(r) * seg_bytes,
                 a.W + (size_t(r0 + r) * a.nsb + sb0) * 144u, seg_bytes, bar, pol);
    }
  };
  if (tid == 0) {
    const int pre = min(a.stages, n_stages);
    for (int st = 0; st < pre; ++st) issue(st);
  }

  // Activations of my words, pre-divided by the extraction scale.
  float2 xr[M][W][4];
  #pragma unroll
  for (int m = 0; m < M; ++m)
    #pragma unroll
    for (int w = 0; w < W; ++w)
      #pragma unroll
      for (int i = 0; i < 4; ++i) xr[m][w][i] = make_float2(0.f, 0.f);
  if (active) {
    const int kb = (sb0 + sb_local) * 256 + blk * 32;
    #pragma unroll
    for (int w = 0; w < W; ++w) {
      const int klo = kb + 4 * ((word0 + w) & 3);
      #pragma unroll
      for (int m = 0; m < M; ++m) {
        const uint2 lo = *reinterpret_cast<const uint2*>(a.x + size_t(m) * a.K + klo);
        const uint2 hi = *reinterpret_cast<const uint2*>(a.x + size_t(m) * a.K + klo + 16);
        const uint32_t lv[4] = {lo.x & 0xFFFFu, lo.x >> 16, lo.y & 0xFFFFu, lo.y >> 16};
        const uint32_t hv[4] = {hi.x & 0xFFFFu, hi.x >> 16, hi.y & 0xFFFFu, hi.y >> 16};
        #pragma unroll
        for (int c = 0; c < 4; ++c) {
          // byte c: low nibble = position 2c (element klo+c), high = 2c+1 (klo+16+c)
          const float xl = bf16_bits_to_float(lv[c]) * (1.0f / nib_scale(2 * c));
          const float xh = bf16_bits_to_float(hv[c]) * (1.0f / nib_scale(2 * c + 1));
          if (c == 0) xr[m][w][0] = make_float2(xl, xh);
          if (c == 1) xr[m][w][1] = make_float2(xl, xh);
          if (c == 2) xr[m][w][2] = make_float2(xl, xh);
          if (c == 3) xr[m][w][3] = make_float2(xl, xh);
        }
      }
    }
  }

  const uint32_t word_off = uint32_t(sb_local) * 144u + uint32_t(word0) * 4u;
  const uint32_t scale_off = uint32_t(sb_local) * 144u + 128u + uint32_t(blk) * 2u;
  const int wps = a.tpr >> 5;  // warps per row stream

  for (int st = 0; st < n_stages; ++st) {
    const int slot = st % a.stages;
    mbar_wait(smem_addr(&bars[slot]), uint32_t(st / a.stages) & 1u, a.err);
    const uint8_t* sl = slots + size_t(slot) * a.slot_bytes;
    const int r0 = row_begin + st * rows_per_stage;
    const int nr = min(rows_per_stage, row_end - r0);

    float v[VPAD];
    #pragma unroll
    for (int i = 0; i < VPAD; ++i) v[i] = 0.f;
    #pragma unroll
    for (int r = 0; r < RSR; ++r) {
      const int lr = stream * RSR + r;
      if (active && lr < nr) {
        const uint8_t* rowp = sl + uint32_t(lr) * seg_bytes;
        uint32_t wv[W];
        load_words<W>(rowp + word_off, wv);
        const float dsc = half_bits_to_float(*reinterpret_cast<const uint16_t*>(rowp + scale_off));
        float2 acc[M];
        #pragma unroll
        for (int m = 0; m < M; ++m) acc[m] = make_float2(0.f, 0.f);
        #pragma unroll
        for (int w = 0; w < W; ++w) {
          float2 t[4];
          dequant_word(wv[w], t);
          #pragma unroll
          for (int i = 0; i < 4; ++i)
            #pragma unroll
            for (int m = 0; m < M; ++m) acc[m] = __ffma2_rn(t[i], xr[m][w][i], acc[m]);
        }
        #pragma unroll
        for (int m = 0; m < M; ++m) v[r * M + m] = dsc * (acc[m].x + acc[m].y);
      }
    }

    // Warp reduce-scatter: after it, lane L holds the warp sum of value
    // L / (32 / VPAD); lanes with L % (32 / VPAD) == 0 publish it.
    #pragma unroll
    for (int it = 0; it < 5; ++it) {
      const int off = 16 >> it;
      const int width = (VPAD >> it) > 1 ? (VPAD >> it) : 1;
      if (width > 1) {
        const bool upper = (lane & off) != 0;
        #pragma unroll
        for (int i = 0; i < width / 2; ++i) {
          const float send = upper ? v[i] : v[i + width / 2];
          const float keep = upper ? v[i + width / 2] : v[i];
          v[i] = keep + __shfl_xor_sync(0xFFFFFFFFu, send, off);
        }
      } else {
        v[0] += __shfl_xor_sync(0xFFFFFFFFu, v[0], off);
      }
    }
    float* redb = red + (st & 1) * nwarps * VPAD;
    if ((lane % (32 / VPAD)) == 0) redb[warp * VPAD + lane / (32 / VPAD)] = v[0];
    __syncthreads();

    if (tid == 0 && st + a.stages < n_stages) issue(st + a.stages);

    // Combine the warps of each row stream in a fixed order and store.
    if (tid < rows_per_stage * M) {
      const int lr = tid / M, m = tid - (tid / M) * M;
      if (lr < nr) {
        const int s = lr / RSR, r = lr - s * RSR;
        float sum = 0.f;
        for (int w = 0; w < wps; ++w) sum += redb[(s * wps + w) * VPAD + r * M + m];
        a.out[(size_t(ks) * M + m) * a.N + r0 + lr] = sum;
      }
    }
  }
}

// y[i] = sum over k ranges of the partials, in range order.
__global__ void q4_gemv_splitk_reduce(const float* __restrict__ ws, float* __restrict__ y,
                                      long long mn, int k_splits) {
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < mn;
       i += (long long)gridDim.x * blockDim.x) {
    float s = 0.f;
    for (int k = 0; k < k_splits; ++k) s += ws[k * mn + i];
    y[i] = s;
  }
}

}  // namespace q4d
