// Q4_0 GEMV / skinny GEMM for M = 1..5 rows with register dequantisation
// feeding mma.sync (m16n8k16, bf16 in, fp32 accumulate).
//
// Why tensor-core instructions for a bandwidth-bound GEMV: on B200 the
// logic/integer pipe runs at half the FP32 rate, and unpacking nibbles plus
// one FMA per weight per row keeps the SM issue-bound well below HBM speed
// (the CUDA-core formulation measured ~4.8 thread instructions per weight at
// M = 1).  Letting mma.sync do the multiply-adds leaves ~2 instructions per
// weight -- the unpack -- for every M up to 8, so M = 2..5 verification rows
// ("Qwen3.8-27B on RTX 4090: 5,000 tok/s Prefill Reproduced", section "MTP
// helps ordinary prose ...") cost the same as plain decode.
//
// Exactness: q - 8 is an integer in [-8, 7], exact in bf16; x is bf16; their
// products are exact in fp32.  Each 32-element block gets its own fresh
// accumulator, multiplied by the block's fp16 scale d in fp32 and added to the
// row's fp32 sum -- the Q4_0 definition w = d * (q - 8) ("Qwen3.8-27B at 256K
// on a 24GB RTX PRO 4000 SFF (432 GB/s): 50 tok/s with MTP", paragraph on
// public GGUFs at 40K context names the format) with fp32 rounding only.
//
// Layout of the work:
//  * Weights are stored super-block-column-major: column s holds super-block
//    s of every row, so the rows a CTA owns form one contiguous piece of each
//    column -- every pipeline stage is a single contiguous bulk copy per
//    column, the access pattern that streams HBM fastest.
//  * CTA c owns rows [N*c/G, N*(c+1)/G) of one K range (k_splits > 1 only for
//    very few rows); rows are processed in passes of up to 8 m16 tiles; a
//    pass streams its K range KC super-block columns per stage.
//  * Warp specialisation: one producer warp issues the copies (bulk copy of
//    the weight piece, TMA box of the activations) into a ring of stages that
//    complete on "full" mbarriers; eight consumer warps compute and release
//    each stage on an "empty" mbarrier, so loads and math overlap with no
//    CTA-wide barrier per stage.  Every wait is bounded in time.
//  * Consumer warp w takes block w of each super-block; it builds the B
//    fragment (x) of its block once per column and applies it to every m-tile
//    of the pass.  At the end of a pass the eight warps' partial sums are
//    added in a fixed order through shared memory (deterministic).
//  * A-fragment k order: lane (g, t) dequantises word t of a block (bytes
//    4t..4t+3) of rows g and g+8; its four bf16 pairs (low nibbles of bytes
//    0/2, high nibbles of bytes 0/2, low of 1/3, high of 1/3) are the fragment
//    registers of the block's two k16 steps; the B fragment takes x in the
//    same element order, so the permutation cancels in the dot product.
//    Rows land at a 144-byte pitch, at which the 32 lanes' 4-byte nibble
//    loads hit 32 distinct banks.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>

#include "q4dec_device.cuh"

namespace q4d {

constexpr int kMmaMaxTiles = 8;  // m16 tiles per pass (128 rows)
constexpr int kMmaMaxStages = 16;

// Kernel parameters.  The tensor map describes x as a bf16 tensor [M][K]
// with boxes of [M][256] (one super-block column); passed as a
// __grid_constant__ so the TMA unit reads it from the parameter space.
struct alignas(64) GemvArgs {
  CUtensorMap xmap;
  const uint8_t* W;    // super-block-column-major weights, [K/256][N] x 144 B
  float* out;          // y [M][N] or partials [k_splits][M][N]
  unsigned* err;
  int out_bf16;        // 1: y (no K split) is stored as bf16 [M][N], rounded to nearest even
  int N;
  int sb_per_split;    // super-blocks per K range
  int rows_per_pass;   // multiple of 16, <= 128
  int grid_rows;
  int stages;
};

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, int x, int y,
                                            uint32_t bar, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      ".L2::cache_hint [%0], [%1, {%2, %3}], [%4], %5;" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar), "l"(policy)
      : "memory");
}

__device__ __forceinline__ void tma_load_2d_nohint(uint32_t dst, const CUtensorMap* map, int x,
                                                   int y, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar)
      : "memory");
}

constexpr uint32_t kSbBytes = 144;  // one super-block row piece in shared memory

// Bytes of one pipeline stage holding KC super-block columns: KC weight
// pieces (rows_per_pass x 144 bytes each, rounded up to 128) followed by KC
// activation boxes (M x 512 bytes each).
__host__ __device__ constexpr uint32_t gemv_wbox_bytes(int rows_per_pass) {
  return (uint32_t(rows_per_pass) * kSbBytes + 127u) / 128u * 128u;
}
__host__ __device__ constexpr uint32_t gemv_stage_bytes(int M, int KC, int rows_per_pass) {
  return uint32_t(KC) * (gemv_wbox_bytes(rows_per_pass) + uint32_t(M) * 512u);
}

// Element i of the output: fp32, or bf16 (round to nearest even) when the
// caller asked for bf16 outputs.  Partials of a K split are always fp32.
__device__ __forceinline__ void store_out(float* out, size_t i, float v, int bf16) {
  if (bf16)
    reinterpret_cast<__nv_bfloat16*>(out)[i] = __float2bfloat16_rn(v);
  else
    out[i] = v;
}

constexpr int kConsumerWarps = 8;
constexpr int kGemvThreads = (kConsumerWarps + 1) * 32;  // + one producer warp

__device__ __forceinline__ void consumer_sync() {
  asm volatile("bar.sync 1, %0;" ::"n"(kConsumerWarps * 32) : "memory");
}

// One m16 tile x one 32-element block: dequantise rows g (and g+8 when
// `second`), two MMAs against the block's x fragment, then add the tile's
// fresh accumulator times each row's block scale into acc.  Columns >= M
// of the accumulator stay zero and are not scaled.
template <int M>
__device__ __forceinline__ void gemv_tile(const uint8_t* pa, uint32_t woff, uint32_t doff,
                                          bool second, const uint32_t (&bx)[4],
                                          float (&acc)[4]) {
  const uint32_t mask = 0x000F000Fu, magic = 0x43004300u, c136 = 0x43084308u;  // bf16 136
  const uint8_t* pb = pa + 8u * kSbBytes;
  const uint32_t wa = *reinterpret_cast<const uint32_t*>(pa + woff);
  const uint32_t wb = second ? *reinterpret_cast<const uint32_t*>(pb + woff) : 0x88888888u;
  const float da = half_bits_to_float(*reinterpret_cast<const uint16_t*>(pa + doff));
  const float db = second ? half_bits_to_float(*reinterpret_cast<const uint16_t*>(pb + doff)) : 0.f;
  uint32_t qa[4], qb[4];
  dequant_pairs(wa, mask, magic, c136, qa);
  dequant_pairs(wb, mask, magic, c136, qb);
  float c[4] = {0.f, 0.f, 0.f, 0.f};
  mma_bf16(c, qa[0], qb[0], qa[1], qb[1], bx[0], bx[1]);
  mma_bf16(c, qa[2], qb[2], qa[3], qb[3], bx[2], bx[3]);
  acc[0] = fmaf(da, c[0], acc[0]);
  acc[2] = fmaf(db, c[2], acc[2]);
  if constexpr (M > 1) {
    acc[1] = fmaf(da, c[1], acc[1]);
    acc[3] = fmaf(db, c[3], acc[3]);
  }
}

// Everything a consumer warp needs to run the stages of one pass.
struct PassCtx {
  const uint8_t* ring;
  uint64_t* full;
  uint64_t* empty;
  unsigned* err;
  uint32_t stage_bytes, wbox, xoff, woff, doff;
  int S, n_chunks, warp, g, t, lane;
};

// One pass of T m-tiles (the last one using only rows 0..7 when HALF) over
// all chunks of the K range: wait for each stage, run every tile of every
// block fully unrolled (no per-tile guard, so the compiler interleaves the
// tiles' loads, unpacking and MMAs), then release the stage.  Rows beyond the
// pass's end hold stale shared memory; their results are never stored.
template <int M, int KC, int T, bool HALF>
__device__ __forceinline__ void gemv_pass(const PassCtx& c, int& slot, uint32_t& phase,
                                          float (&acc)[kMmaMaxTiles][4]) {
  #pragma unroll
  for (int p = 0; p < T; ++p) acc[p][0] = acc[p][1] = acc[p][2] = acc[p][3] = 0.f;
  for (int chunk = 0; chunk < c.n_chunks; ++chunk) {
    mbar_wait(smem_addr(&c.full[slot]), phase, c.err);
    const uint8_t* wst = c.ring + size_t(slot) * c.stage_bytes;
    #pragma unroll 1
    for (int j = 0; j < KC; ++j) {  // kept rolled: one copy of the tile code stays in the I-cache
      // B fragment (x) of this warp's block of column j for column g
      uint32_t bx[4] = {0u, 0u, 0u, 0u};
      if (c.g < M) {
        const uint8_t* xr = wst + c.xoff + (j * M + c.g) * 512 + (c.warp * 32 + 4 * c.t) * 2;
        const uint2 lo = *reinterpret_cast<const uint2*>(xr);
        const uint2 hi = *reinterpret_cast<const uint2*>(xr + 32);
        bx[0] = prmt(lo.x, lo.y, 0x5410);  // (x[4t+0], x[4t+2])
        bx[1] = prmt(hi.x, hi.y, 0x5410);  // (x[16+4t+0], x[16+4t+2])
        bx[2] = prmt(lo.x, lo.y, 0x7632);  // (x[4t+1], x[4t+3])
        bx[3] = prmt(hi.x, hi.y, 0x7632);  // (x[16+4t+1], x[16+4t+3])
      }
      const uint8_t* wj = wst + uint32_t(j) * c.wbox;
      #pragma unroll
      for (int p = 0; p < T; ++p)
        gemv_tile<M>(wj + 16u * p * kSbBytes, c.woff, c.doff, !(HALF && p == T - 1), bx, acc[p]);
    }
    __syncwarp();
    if (c.lane == 0) mbar_arrive(smem_addr(&c.empty[slot]));  // this warp is done with it
    if (++slot == c.S) {
      slot = 0;
      phase ^= 1u;
    }
  }
}

// M: activation rows (B fragment columns; columns M..7 are zero).
// KC: super-block columns per pipeline stage.
// Warps 0..7 consume: warp w takes block w of every super-block column and
// every m-tile of the pass.  Warp 8 produces: it refills a stage as soon as
// all eight consumers have released it.
// SWIGLU: the matrix holds gate / up row pairs (rows 2n, 2n + 1); CTAs own
// whole pairs and, without a K split, store h = silu(gate) * up per pair.
template <int M, int KC, bool SWIGLU>
__global__ void __launch_bounds__(kGemvThreads, 1)
    q4_gemv_kernel(const __grid_constant__ GemvArgs a) {
  extern __shared__ __align__(128) uint8_t smem[];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int ks = blockIdx.y;
  const int S = a.stages;

  const int unit = SWIGLU ? 2 : 1;  // rows per partition unit
  const int units = a.N / unit;
  const int row_begin = unit * int((long long)units * blockIdx.x / a.grid_rows);
  const int row_end = unit * int((long long)units * (blockIdx.x + 1) / a.grid_rows);
  const int n_rows = row_end - row_begin;
  const int R = a.rows_per_pass;
  const int n_passes = (n_rows + R - 1) / R;
  const int n_chunks = a.sb_per_split / KC;
  const int n_stages = n_passes * n_chunks;
  const int sb_split0 = ks * a.sb_per_split;
  const uint32_t wbox = gemv_wbox_bytes(R);
  const uint32_t stage_bytes = gemv_stage_bytes(M, KC, R);
  const uint32_t xoff = uint32_t(KC) * wbox;

  uint8_t* ring = smem;
  float4* red = reinterpret_cast<float4*>(smem + size_t(S) * stage_bytes);
  uint64_t* full = reinterpret_cast<uint64_t*>(red + kConsumerWarps * kMmaMaxTiles * 32);
  uint64_t* empty = full + S;

  if (tid == 0) {
    // the next kernel on the stream may start its own weight prefetch
    griddep_launch_dependents();
    for (int s = 0; s < S; ++s) {
      mbar_init(smem_addr(&full[s]), 1);
      mbar_init(smem_addr(&empty[s]), kConsumerWarps);
    }
    mbar_init_fence();
  }
  __syncthreads();

  if (warp == kConsumerWarps) {
    // ---------------- producer: one lane issues every copy ----------------
    if (lane == 0) {
      const uint64_t pol = l2_evict_first_policy();
      // First ring fill: the weights (no earlier kernel writes them) go out
      // before waiting on the previous kernel; the activations, which it may
      // produce, only after.  Under a plain launch the wait returns at once.
      const int pre = min(S, n_stages);
      for (int st = 0; st < pre; ++st) {
        const int ps = st / n_chunks, ch = st - ps * n_chunks;
        const int r0 = row_begin + ps * R;
        const int nr = min(R, row_end - r0);
        const int sb = sb_split0 + ch * KC;
        const uint32_t bar = smem_addr(&full[st]);
        const uint32_t dst = smem_addr(ring + size_t(st) * stage_bytes);
        mbar_arrive_expect_tx(bar, uint32_t(KC) * (uint32_t(nr) * kSbBytes + uint32_t(M) * 512u));
        #pragma unroll
        for (int j = 0; j < KC; ++j)
          bulk_g2s(dst + uint32_t(j) * wbox, a.W + (size_t(sb + j) * a.N + r0) * kSbBytes,
                   uint32_t(nr) * kSbBytes, bar, pol);
      }
      griddep_wait();
      for (int st = 0; st < pre; ++st) {
        const int sb = sb_split0 + (st % n_chunks) * KC;
        const uint32_t bar = smem_addr(&full[st]);
        const uint32_t dst = smem_addr(ring + size_t(st) * stage_bytes);
        #pragma unroll
        for (int j = 0; j < KC; ++j)
          tma_load_2d_nohint(dst + xoff + uint32_t(j) * uint32_t(M) * 512u, &a.xmap,
                             (sb + j) * 256, 0, bar);
      }
      int slot = 0, pass = pre / n_chunks, chunk = pre % n_chunks;
      uint32_t phase = pre == S ? 1u : 0u;
      for (int st = pre; st < n_stages; ++st) {
        mbar_wait(smem_addr(&empty[slot]), phase ^ 1u, a.err);
        const int r0 = row_begin + pass * R;
        const int nr = min(R, row_end - r0);
        const uint32_t bar = smem_addr(&full[slot]);
        const uint32_t dst = smem_addr(ring + size_t(slot) * stage_bytes);
        const int sb = sb_split0 + chunk * KC;
        mbar_arrive_expect_tx(bar, uint32_t(KC) * (uint32_t(nr) * kSbBytes + uint32_t(M) * 512u));
        #pragma unroll
        for (int j = 0; j < KC; ++j) {
          // rows r0 .. r0+nr of column sb+j are contiguous in the weight layout
          bulk_g2s(dst + uint32_t(j) * wbox, a.W + (size_t(sb + j) * a.N + r0) * kSbBytes,
                   uint32_t(nr) * kSbBytes, bar, pol);
          tma_load_2d_nohint(dst + xoff + uint32_t(j) * uint32_t(M) * 512u, &a.xmap,
                             (sb + j) * 256, 0, bar);
        }
        if (++slot == S) {
          slot = 0;
          phase ^= 1u;
        }
        if (++chunk == n_chunks) {
          chunk = 0;
          ++pass;
        }
      }
    }
    return;
  }

  // ---------------- consumers ----------------
  PassCtx c;
  c.ring = ring;
  c.full = full;
  c.empty = empty;
  c.err = a.err;
  c.stage_bytes = stage_bytes;
  c.wbox = wbox;
  c.xoff = xoff;
  c.warp = warp;
  c.lane = lane;
  c.g = lane >> 2;
  c.t = lane & 3;
  c.woff = uint32_t(c.g) * kSbBytes + uint32_t(warp) * 16u + uint32_t(c.t) * 4u;
  c.doff = uint32_t(c.g) * kSbBytes + 128u + uint32_t(warp) * 2u;
  c.S = S;
  c.n_chunks = n_chunks;
  float acc[kMmaMaxTiles][4];
  int slot = 0;
  uint32_t phase = 0;

  for (int pass = 0; pass < n_passes; ++pass) {
    const int nr = min(R, n_rows - pass * R);
    const int T = (nr + 15) >> 4;
    const bool half = (nr & 15) != 0 && (nr & 15) <= 8;
    switch (T * 2 + (half ? 1 : 0)) {
#define Q4D_PASS(TT)                                                   \
  case 2 * TT: gemv_pass<M, KC, TT, false>(c, slot, phase, acc); break; \
  case 2 * TT + 1: gemv_pass<M, KC, TT, true>(c, slot, phase, acc); break;
      Q4D_PASS(1) Q4D_PASS(2) Q4D_PASS(3) Q4D_PASS(4)
      Q4D_PASS(5) Q4D_PASS(6) Q4D_PASS(7) Q4D_PASS(8)
#undef Q4D_PASS
      default: break;
    }

    // Cross-warp sum of the pass, in a fixed order.
    #pragma unroll
    for (int p = 0; p < kMmaMaxTiles; ++p)
      if (16 * p < nr)
        red[(warp * kMmaMaxTiles + p) * 32 + lane] =
            make_float4(acc[p][0], acc[p][1], acc[p][2], acc[p][3]);
    consumer_sync();
    // out[m][row] = sum over the 8 warps; element (row r, column m) sits in
    // lane (r % 8) * 4 + m / 2 of tile r / 16, component (r >= 8 ? 2 : 0) + m % 2
    const int r0 = row_begin + pass * R;
    auto row_sum = [&](int r, int m) {
      const int p = r >> 4, rr = r & 15;
      const int ln = (rr & 7) * 4 + (m >> 1);
      const int comp = (rr >= 8 ? 2 : 0) + (m & 1);
      float s = 0.f;
      #pragma unroll
      for (int w = 0; w < kConsumerWarps; ++w) {
        const float4 v = red[(w * kMmaMaxTiles + p) * 32 + ln];
        s += comp == 0 ? v.x : comp == 1 ? v.y : comp == 2 ? v.z : v.w;
      }
      return s;
    };
    if (SWIGLU && gridDim.y == 1) {
      // h[m][n] = silu(g) * u for the pairs of this pass (passes hold whole pairs)
      for (int i = tid; i < (nr >> 1) * M; i += kConsumerWarps * 32) {
        const int j = i / M, m = i - (i / M) * M;
        const float g = row_sum(2 * j, m), u = row_sum(2 * j + 1, m);
        store_out(a.out, size_t(m) * (a.N >> 1) + ((r0 >> 1) + j), g / (1.f + __expf(-g)) * u,
                  a.out_bf16);
      }
    } else {
      for (int i = tid; i < nr * M; i += kConsumerWarps * 32) {
        const int r = i / M, m = i - (i / M) * M;
        store_out(a.out, (size_t(ks) * M + m) * a.N + r0 + r, row_sum(r, m), a.out_bf16);
      }
    }
    consumer_sync();  // red is rewritten at the next pass end
  }
}

// h[m][n] = silu(g) * u from the partials of the 2N gate / up rows, each
// summed over the K ranges in range order.
__global__ void q4_gemv_splitk_reduce_swiglu(const float* __restrict__ ws, float* __restrict__ h,
                                             int M, int N, int k_splits, int out_bf16) {
  if (threadIdx.x == 0) griddep_launch_dependents();
  const long long mn = (long long)M * N, rows = 2LL * N;
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < mn;
       i += (long long)gridDim.x * blockDim.x) {
    const long long m = i / N, n = i - m * N;
    float g = 0.f, u = 0.f;
    for (int k = 0; k < k_splits; ++k) {
      g += ws[(k * M + m) * rows + 2 * n];
      u += ws[(k * M + m) * rows + 2 * n + 1];
    }
    store_out(h, size_t(i), g / (1.f + __expf(-g)) * u, out_bf16);
  }
}

// y[i] = sum over K ranges of the partials, in range order.
__global__ void q4_gemv_splitk_reduce(const float* __restrict__ ws, float* __restrict__ y,
                                      long long mn, int k_splits, int out_bf16) {
  if (threadIdx.x == 0) griddep_launch_dependents();
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < mn;
       i += (long long)gridDim.x * blockDim.x) {
    float s = 0.f;
    for (int k = 0; k < k_splits; ++k) s += ws[k * mn + i];
    store_out(y, size_t(i), s, out_bf16);
  }
}

}  // namespace q4d
