// Q4_0 GEMV / skinny GEMM for M = 1..5 activation rows, one or many matrices
// per launch, with register dequantisation feeding mma.sync (m16n8k16, bf16
// in, fp32 accumulate).
//
// What it computes: y[m][n] = sum_k d * (q - 8) * x[m][k] over the Q4_0 blocks
// of weight row n -- the quantised weight stream that decode repeatedly
// reads ("Qwen3.8-27B at 256K on a 24GB RTX PRO 4000 SFF (432 GB/s): 50 tok/s
// with MTP", paragraph beginning "NVIDIA quotes 432 GB/s"); M = 2..5 rows are
// the target model verifying a drafted block, which shares one weight stream
// ("Qwen3.8-27B on RTX 4090: 5,000 tok/s Prefill Reproduced", section "MTP
// helps ordinary prose, but acceptance controls the gain").
//
// Exactness: q - 8 is an integer in [-8, 7], exact in bf16; x is bf16; their
// products are exact in fp32.  Each 32-element block gets its own fresh MMA
// accumulator, multiplied by the block's fp16 scale d in fp32 and added to the
// row's fp32 sum, so the only roundings are fp32 additions.
//
// Why tensor-core instructions for a bandwidth-bound GEMV: unpacking nibbles
// keeps the half-rate integer pipe busy (three shifts and four masks per eight
// weights, plus four bf16 subtractions on the fp16 pipe); letting mma.sync do
// the multiply-adds leaves that unpack as the only per-weight work, for every
// M up to 8.
//
// Work decomposition (stream-K):
//  * A matrix is cut into row blocks of 128 rows (8 m16 tiles) and, along K,
//    into units of two super-block columns (512 elements).  The units, row
//    block after row block, are shared out in equal contiguous ranges over the
//    CTAs (one CTA per SM), so every CTA streams the same number of bytes
//    whatever N and K are, and every pass keeps 8 tiles of independent work.
//    Where the units do not divide evenly, some CTAs get one more; a job's
//    CTA numbering is rotated by the units of the jobs before it, so that
//    over a batch those extra units land on different CTAs.
//  * A CTA's range covers the tail of one row block, whole row blocks and the
//    head of another.  A row block covered by one CTA is written directly.  A
//    row block shared by several CTAs has one slot of partial sums per
//    contributor, in K order; slot 0 belongs to the CTA whose range ends in
//    the row block, which reaches it last (the others reach it at the start
//    of their ranges or cover nothing else), so that CTA finishes it.  The
//    others write their slots, each entry one 64-bit word holding the fp32
//    value and the launch's 32-bit tag, so an entry is valid exactly when it
//    carries the tag (no flag, no fence, no round trip); the finisher reads
//    the entries until they are valid -- those of a partner that finished
//    early are read while its own sums are still being made -- adds the slots
//    in slot order, its own from registers, writes the rows and clears the
//    entries.  The workspace is handed over zero-filled, and the clearing
//    leaves it so after every launch; a cleared entry is never valid (tags
//    are non-zero), and replays of a captured launch (same tag) stay correct.
//  * Several matrices ("jobs") can run in one launch.  The producer keeps
//    streaming the next job's weights (they depend on nothing) while a job's
//    activations wait for the job they depend on: whichever epilogue warp
//    writes half of a row block in final form counts it on a per-job counter
//    (a release reduction), and a job's activation copies are issued only
//    once its prerequisite's count has reached twice that job's number of row
//    blocks (an acquire load).  These counters live in the launch descriptor,
//    which the host hands over zeroed; the last CTA to leave the launch sets
//    them back to zero.
//  * Weights are stored super-block-column-major: the 128 rows of a row block
//    are one contiguous piece of each column, so a unit is two bulk copies of
//    18 KB plus one copy of each activation row's 1 KB, issued by a producer
//    warp into a ring of stages that complete on "full" mbarriers.  Sixteen
//    consumer warps take one (column, block) task each per stage and release
//    it on an "empty" mbarrier.  At the end of each row block segment each
//    consumer warp of column 0 stores its partial sums into the slot of its
//    block index in a reduction buffer and signals it on an mbarrier; the
//    column-1 warp of the same block adds its sums to that slot, signals the
//    slot complete and goes on with the next stage -- no CTA-wide barrier;
//    two epilogue warps, each taking one half (64 rows) of every segment, add
//    the 8 slots in block order, release the buffer, write the sums out (y,
//    the partial slot, or the sum of the slots) and count the halves written
//    in final form for their job, so no global write or atomic stalls the
//    consumers, and a consumer warp waits at most for its column partner.
//  * Built with Q4D_DEBUG, every global access above is index-checked
//    against its buffer's extent (Q4D_CHECK): a failure is recorded in the
//    device error record and the access skipped, or a copy redirected to the
//    buffer's first bytes.
//  * Every wait is bounded in time.  A wait that runs out sets the device
//    error word and a per-CTA abort flag; from then on no wait blocks, the
//    producer issues no further copies and waits for the ones in flight, and
//    every role still runs its loop to the end, so the kernel terminates.
//
// A-fragment k order: lane (g, t) dequantises word t of a block (bytes
// 4t..4t+3) of rows g and g+8; its four bf16 pairs (low nibbles of bytes 0/2,
// high nibbles of bytes 0/2, low of 1/3, high of 1/3) are the fragment
// registers of the block's two k16 steps; the B fragment takes x in the same
// element order, so the permutation cancels in the dot product.  Rows land at
// a 144-byte pitch, at which the 32 lanes' 4-byte nibble loads hit 32
// distinct banks.
#pragma once

#include <cuda_bf16.h>

#include "q4dec_device.cuh"

namespace q4d {

constexpr int kGemvTiles = 8;                              // m16 tiles per row block
constexpr int kGemvRows = 16 * kGemvTiles;                 // 128 weight rows
constexpr int kGemvCols = 2;                               // super-block columns per unit
constexpr int kGemvConsumerWarps = 8 * kGemvCols;          // one (column, block) task each
constexpr int kGemvProducerWarp = kGemvConsumerWarps;      // bulk copies
constexpr int kGemvEpilogueWarps = 2;                      // output writes, flags, counts
constexpr int kGemvThreads = (kGemvConsumerWarps + 1 + kGemvEpilogueWarps) * 32;
constexpr int kGemvRedStride = kGemvRows + 4;              // floats per column of a slot (banks)
constexpr int kGemvMaxStages = 8;
constexpr uint32_t kSbBytes = 144;                         // one super-block
constexpr uint32_t kGemvWBox = kGemvRows * kSbBytes;       // one column of a row block
constexpr uint32_t kJobOutBf16 = 1u;                       // y stored as bf16 (RNE)
constexpr uint32_t kJobSwiglu = 2u;                        // rows are gate / up pairs

// Activation rows of a stage: two columns (1 KB) each, at a pitch of 1056
// bytes, so that the fragment loads of up to 8 rows (lanes g = row) fall on
// distinct banks.
constexpr uint32_t kGemvXPitch = kGemvCols * 512u + 32u;
// Reduction slots (consumers -> epilogue), [M][kGemvRedStride] fp32 each.  At
// M <= 3 one per consumer warp; at M >= 4 one per block index ("pair slots":
// the column-1 warp adds its sums to those the column-0 warp of its block
// stored), half the shared memory, which leaves room for a fifth ring stage.
// The epilogue adds, block index by block index, column 0 + column 1, then
// the block indices in order: the same roundings at every M.
__host__ __device__ constexpr bool gemv_pair_slots(int M) { return M >= 4; }
__host__ __device__ constexpr int gemv_red_slots(int M) { return gemv_pair_slots(M) ? 8 : 16; }
// One pipeline stage: the unit's two weight pieces, then M activation rows of
// two columns (the second half unused when the unit has one column), rounded
// up to 128 bytes, or to 16 (every bulk copy's alignment) with pair slots,
// so that five stages fit at M = 5 (a stage's bank pattern does not depend
// on where it starts: all its addresses shift alike).
__host__ __device__ constexpr uint32_t gemv_stage_bytes(int M) {
  return gemv_pair_slots(M)
             ? (kGemvCols * kGemvWBox + uint32_t(M) * kGemvXPitch + 15u) / 16u * 16u
             : (kGemvCols * kGemvWBox + uint32_t(M) * kGemvXPitch + 127u) / 128u * 128u;
}
// Reduction buffers: two for M <= 2, one otherwise.
__host__ __device__ constexpr int gemv_red_bufs(int M) { return M <= 2 ? 2 : 1; }
__host__ __device__ constexpr uint32_t gemv_red_bytes(int M) {
  return uint32_t(gemv_red_bufs(M)) * uint32_t(gemv_red_slots(M)) * uint32_t(M) * kGemvRedStride *
         4u;
}
// Reduction buffer b of the [bufs] at `red` (consumers and epilogue alike).
template <int M>
__device__ __forceinline__ float* gemv_red_buffer(float* red, int b) {
  return red + size_t(b) * gemv_red_slots(M) * M * kGemvRedStride;
}
// Shared memory: ring, reduction buffers, the abort flag (padded to 16), 2
// barriers per stage, 2 per reduction buffer and, with pair slots, one per
// slot of each buffer.
__host__ __device__ constexpr size_t gemv_smem_bytes(int M, int stages) {
  return size_t(stages) * gemv_stage_bytes(M) + gemv_red_bytes(M) + 16 + size_t(stages) * 16 +
         size_t(gemv_red_bufs(M)) * 16 +
         (gemv_pair_slots(M) ? size_t(gemv_red_bufs(M)) * gemv_red_slots(M) * 8 : 0);
}

// First unit of (job-local) CTA c when U units are shared out over G CTAs
// (G <= U), and the CTA whose range holds unit u.  32-bit arithmetic: the host
// accepts only U * G < 2^31.
__host__ __device__ __forceinline__ int unit_begin(int c, int U, int G) {
  return int(unsigned(c) * unsigned(U) / unsigned(G));
}
__host__ __device__ __forceinline__ int unit_owner(int u, int U, int G) {
  return int((unsigned(u + 1) * unsigned(G) - 1u) / unsigned(U));
}

// Everything the kernel needs to know about one matrix; the host planner
// fills it (the same for every M row count except the partial-slot size).
struct alignas(16) GemvJobDesc {
  const uint8_t* W;      // super-block-column-major weights
  const uint16_t* x;     // bf16 [M][K]
  void* y;               // fp32 or bf16 [M][N] ([M][N/2] for gate / up pairs)
  long long part_off;    // this job's partial slots: floats into the partial area
  int N;                 // weight rows
  int nsb;               // K / 256
  int flags;             // kJobOutBf16 | kJobSwiglu
  int wait_for;          // -1: x is ready at launch; j: x is read after job j finished
  int rbs;               // row blocks, ceil(N / 128)
  int upr;               // units per row block, ceil(nsb / 2)
  int units;             // rbs * upr
  int grid;              // CTAs that work on this job (min(launch grid, units))
  int slots;             // partial slots per row block (0: no row block is shared)
  int rot;               // job-local CTA index = (blockIdx.x + rot) mod launch grid
  long long w_bytes;     // extent of W that index checks allow (N * nsb * 144 or less)
};

struct GemvArgs {
  const GemvJobDesc* jobs;        // device array of n_jobs descriptors, or null: `job` below
  unsigned* sync;                 // [n_jobs] row blocks finished per job, [1] CTAs gone (zeroed)
  unsigned long long* partials;   // workspace: partial slots of {fp32 value, tag} entries
  unsigned* err;                  // device error word
  unsigned long long tag;         // this launch's tag (low 32 bits non-zero)
  int n_jobs;
  int grid;                       // CTAs of the launch
  int stages;                     // ring stages
  int pad_;
  long long ws_entries;           // entries of the partial area that index checks allow
  GemvJobDesc job;                // the single job of a one-matrix launch
};

__device__ __forceinline__ unsigned ld_acquire_gpu(const unsigned* p) {
  unsigned v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ unsigned long long ld_acquire_gpu_u64(const unsigned long long* p) {
  unsigned long long v;
  asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ void st_relaxed_gpu_u64(unsigned long long* p, unsigned long long v) {
  asm volatile("st.relaxed.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}

__device__ __forceinline__ unsigned long long ld_relaxed_gpu_u64(const unsigned long long* p) {
  unsigned long long v;
  asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
  return v;
}

// A partial-slot entry: the fp32 value's bits, the launch tag above them.
__device__ __forceinline__ unsigned long long slot_entry(float v, unsigned tag32) {
  return (static_cast<unsigned long long>(tag32) << 32) | __float_as_uint(v);
}

__device__ __forceinline__ void red_release_gpu_add(unsigned* p, unsigned v) {
  asm volatile("red.release.gpu.global.add.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

__device__ __forceinline__ void fence_acq_rel_gpu() {
  asm volatile("fence.acq_rel.gpu;" ::: "memory");
}

// Make generic-proxy writes of other CTAs (observed through an acquire) visible
// to this thread's subsequent bulk copies (async proxy) from global memory.
__device__ __forceinline__ void fence_proxy_async_global() {
  asm volatile("fence.proxy.async.global;" ::: "memory");
}

// Element i of an output: fp32, or bf16 (round to nearest even).
__device__ __forceinline__ void store_out(void* out, size_t i, float v, bool bf16) {
  if (bf16)
    reinterpret_cast<__nv_bfloat16*>(out)[i] = __float2bfloat16_rn(v);
  else
    reinterpret_cast<float*>(out)[i] = v;
}

// Wait for the barrier phase with the given parity, for at most kWaitLimitNs,
// unless the CTA has already given up (abort flag): then return false at
// once.  A wait that runs out sets the abort flag and the device error word.
__device__ __forceinline__ bool gemv_wait(uint32_t bar, uint32_t parity, unsigned* err,
                                          volatile int* abort_flag) {
  if (mbar_try_wait(bar, parity)) return true;
  if (*abort_flag) return false;
  const unsigned long long t0 = global_timer_ns();
  for (uint32_t polls = 1;; ++polls) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((polls & 255u) == 0) {
      if (*abort_flag) return false;
      if (global_timer_ns() - t0 > kWaitLimitNs) {
        *abort_flag = 1;
        atomicOr(err, kDevErrWaitTimeout);
        return false;
      }
    }
  }
}

__device__ __forceinline__ const GemvJobDesc* gemv_job(const GemvArgs& a, int i) {
  return a.jobs ? a.jobs + i : &a.job;
}

// This CTA's place in job J: its job-local index (-1 when it has no unit of
// the job) and its unit range [ub, ue).
struct JobRange {
  int cj, ub, ue;
};
__device__ __forceinline__ JobRange job_range(const GemvArgs& a, const GemvJobDesc* J) {
  JobRange r;
  int c = int(blockIdx.x) + J->rot;
  if (c >= a.grid) c -= a.grid;
  r.cj = c < J->grid ? c : -1;
  r.ub = r.cj < 0 ? 0 : unit_begin(r.cj, J->units, J->grid);
  r.ue = r.cj < 0 ? 0 : unit_begin(r.cj + 1, J->units, J->grid);
  return r;
}

// The sequence of units a CTA works through, job after job (jobs it has no
// units of are skipped), for the producer.  The row block rb and column pair
// cp of unit u are kept up to date incrementally (no division per unit).
struct UnitCursor {
  int job, u, ue, rb, cp;
  const uint8_t* W;
  const uint16_t* x;
  int N, nsb, upr, wait_for;
  unsigned wait_rbs;  // count of job wait_for once finished (row-block halves)
  long long w_bytes;
};

__device__ __forceinline__ void cursor_enter(UnitCursor& c, const GemvArgs& a, int i) {
  for (; i < a.n_jobs; ++i) {
    const GemvJobDesc* J = gemv_job(a, i);
    const JobRange r = job_range(a, J);
    if (r.cj < 0) continue;
    c.u = r.ub;
    c.ue = r.ue;
    c.rb = c.u / J->upr;
    c.cp = c.u - c.rb * J->upr;
    c.W = J->W;
    c.x = J->x;
    c.N = J->N;
    c.nsb = J->nsb;
    c.upr = J->upr;
    c.wait_for = J->wait_for;
    if (!Q4D_CHECK(c.wait_for < i, a.err, kSiteGemvCounters, c.wait_for)) c.wait_for = -1;
    c.w_bytes = J->w_bytes;
    c.wait_rbs = c.wait_for >= 0 ? unsigned(kGemvEpilogueWarps * gemv_job(a, c.wait_for)->rbs) : 0u;
    break;
  }
  c.job = i;
}

// Element offset in x of row m's columns [col0, col0 + kc) of 256 elements;
// a failed index check gives the first element instead (memory that exists).
template <int M>
__device__ __forceinline__ size_t x_offset_m(const UnitCursor& c, int m, int col0, int kc,
                                             unsigned* err) {
  const size_t o = (size_t(m) * c.nsb + col0) * 256;
  return Q4D_CHECK(m < M && o + size_t(kc) * 256 <= size_t(M) * c.nsb * 256, err,
                   kSiteGemvActivations, o)
             ? o
             : 0;
}

__device__ __forceinline__ void cursor_next(UnitCursor& c, const GemvArgs& a) {
  if (++c.u == c.ue) {
    cursor_enter(c, a, c.job + 1);
  } else if (++c.cp == c.upr) {
    c.cp = 0;
    ++c.rb;
  }
}

// Element k of lane `lane` in epilogue warp e's half of a segment: column
// m = k / 2 of the [M][128] layout, row r = 64 e + 32 (k % 2) + lane.
__device__ __forceinline__ int seg_row(int e, int lane, int k) { return 64 * e + 32 * (k & 1) + lane; }
__device__ __forceinline__ int seg_index(int e, int lane, int k) {
  return (k >> 1) * kGemvRows + seg_row(e, lane, k);
}

// Epilogue warp e's half of a row block, fully summed (v[k]: element k as
// above): write y (or, for gate / up pairs, h = silu(g) * u, pairing rows 2j
// and 2j + 1, held by neighbouring lanes).
template <int M>
__device__ __forceinline__ void gemv_store_rows(const GemvJobDesc* J, int rb, int e, int lane,
                                                unsigned* err, const float (&v)[2 * M]) {
  const bool bf16 = (J->flags & kJobOutBf16) != 0;
  const int r0 = rb * kGemvRows;
  if (J->flags & kJobSwiglu) {
    const int n_out = J->N >> 1;
    #pragma unroll
    for (int k = 0; k < 2 * M; ++k) {
      const int m = k >> 1, r = seg_row(e, lane, k);
      const float other = __shfl_down_sync(0xFFFFFFFFu, v[k], 1);
      const size_t i = size_t(m) * n_out + ((r0 + r) >> 1);
      if ((r & 1) == 0 && r0 + r + 1 < J->N &&
          Q4D_CHECK(i < size_t(M) * n_out, err, kSiteGemvOutput, i))
        store_out(J->y, i, v[k] / (1.f + expf(-v[k])) * other, bf16);
    }
  } else {
    #pragma unroll
    for (int k = 0; k < 2 * M; ++k) {
      const int m = k >> 1, r = seg_row(e, lane, k);
      const size_t i = size_t(m) * J->N + r0 + r;
      if (r0 + r < J->N && Q4D_CHECK(i < size_t(M) * J->N, err, kSiteGemvOutput, i))
        store_out(J->y, i, v[k], bf16);
    }
  }
}

// Who shares row block rb of job J, and this CTA's slot among them.
struct RowBlockShare {
  int n, my;
};
__device__ __forceinline__ RowBlockShare row_block_share(const GemvJobDesc* J, int cj, int rb) {
  const int first_u = rb * J->upr;
  const int c_first = unit_owner(first_u, J->units, J->grid);
  const int c_last = unit_owner(first_u + J->upr - 1, J->units, J->grid);
  return RowBlockShare{c_last - c_first + 1, cj - c_first};
}

// Entries of slot sl of row block rb ([M][128]; rows past N unused).
template <int M>
__device__ __forceinline__ unsigned long long* slot_entries(const GemvArgs& a,
                                                            const GemvJobDesc* J, int rb, int sl) {
  return a.partials + J->part_off + (size_t(rb) * J->slots + sl) * M * kGemvRows;
}

// Index check of slot sl of row block rb (always true without Q4D_DEBUG).
template <int M>
__device__ __forceinline__ bool slot_in_range(const GemvArgs& a, const GemvJobDesc* J, int rb,
                                              int sl) {
  return Q4D_CHECK(rb < J->rbs && sl < J->slots &&
                       J->part_off + ((long long)rb * J->slots + sl + 1) * M * kGemvRows <=
                           a.ws_entries,
                   a.err, kSiteGemvPartials,
                   J->part_off + ((long long)rb * J->slots + sl) * M * kGemvRows);
}

// Read this lane's entries (epilogue warp e's half) of a slot if they are all
// valid (tag): values into w.  Returns false (w unspecified) if any is not yet
// written.
template <int M>
__device__ __forceinline__ bool read_slot(const unsigned long long* s_e, int e, int lane,
                                          unsigned tag32, float (&w)[2 * M]) {
  unsigned long long r[2 * M];
  #pragma unroll
  for (int k = 0; k < 2 * M; ++k) r[k] = ld_relaxed_gpu_u64(s_e + seg_index(e, lane, k));
  bool ok = true;
  #pragma unroll
  for (int k = 0; k < 2 * M; ++k) {
    ok &= unsigned(r[k] >> 32) == tag32;
    w[k] = __uint_as_float(unsigned(r[k]));
  }
  return ok;
}

// This CTA's sums of a row block segment, epilogue side (warp e: rows [64 e,
// 64 e + 64)): the slots of reduction buffer `buf` added into v, block index
// by block index (column 0 + column 1: the sum a pair slot already holds),
// in block order; then the buffer is released (this warp's arrival).
template <int M>
__device__ __forceinline__ void gemv_segment_sum(const float* buf, uint64_t* buf_empty, int e,
                                                 int lane, float (&v)[2 * M]) {
  #pragma unroll
  for (int k = 0; k < 2 * M; ++k) {
    const float* col = buf + (k >> 1) * kGemvRedStride + seg_row(e, lane, k);
    float acc;
    if constexpr (gemv_pair_slots(M)) {
      acc = col[0];
      #pragma unroll
      for (int w = 1; w < 8; ++w) acc += col[w * M * kGemvRedStride];
    } else {
      constexpr int kCol1 = 8 * M * kGemvRedStride;     // the column-1 warps' slots
      acc = col[0] + col[kCol1];
      #pragma unroll
      for (int w = 1; w < 8; ++w)
        acc += col[w * M * kGemvRedStride] + col[kCol1 + w * M * kGemvRedStride];
    }
    v[k] = acc;
  }
  __syncwarp();
  if (lane == 0) mbar_arrive(smem_addr(buf_empty));  // this warp is done with the buffer
}

// End of a row block segment, epilogue side: warp e takes rows [64 e, 64 e +
// 64) of it, this CTA's sums in v.  Write the rows (row block covered by this
// CTA alone); or, in a shared row block, publish this CTA's slot (slots 1,
// 2, ...), or finish the row block (slot 0): read the other slots until valid
// (slot 1 may have been read already: pv, when `pre`), add the slots in slot
// order, write the rows and clear the slots read.  Returns whether this warp
// wrote final values.
template <int M>
__device__ __forceinline__ bool gemv_segment_write(const GemvArgs& a, const GemvJobDesc* J, int cj,
                                                   int rb, int e, int lane,
                                                   volatile int* abort_flag, bool pre,
                                                   const float (&pv)[2 * M], float (&v)[2 * M]) {
  const RowBlockShare sh = row_block_share(J, cj, rb);
  const unsigned tag32 = unsigned(a.tag);
  if (sh.n == 1) {
    gemv_store_rows<M>(J, rb, e, lane, a.err, v);
    return true;
  }
  if (sh.my != 0) {
    unsigned long long* s_e = slot_entries<M>(a, J, rb, sh.my);
    if (slot_in_range<M>(a, J, rb, sh.my)) {
      #pragma unroll
      for (int k = 0; k < 2 * M; ++k)
        st_relaxed_gpu_u64(s_e + seg_index(e, lane, k), slot_entry(v[k], tag32));
    }
    return false;
  }
  // the finisher: slot 0 (its own, from registers), then the others in order
  #pragma unroll
  for (int k = 0; k < 2 * M; ++k) v[k] = 0.f + v[k];
  for (int sl = 1; sl < sh.n; ++sl) {
    float w[2 * M];
    if (sl == 1 && pre) {
      #pragma unroll
      for (int k = 0; k < 2 * M; ++k) w[k] = pv[k];
    } else if (!slot_in_range<M>(a, J, rb, sl)) {
      #pragma unroll
      for (int k = 0; k < 2 * M; ++k) w[k] = 0.f;
    } else {
      const unsigned long long* s_e = slot_entries<M>(a, J, rb, sl);
      const unsigned long long t0 = global_timer_ns();
      while (!read_slot<M>(s_e, e, lane, tag32, w)) {  // bounded wait for the partner's entries
        if (*abort_flag) break;
        if (global_timer_ns() - t0 > kWaitLimitNs) {
          *abort_flag = 1;
          atomicOr(a.err, kDevErrWaitTimeout);
          break;
        }
        __nanosleep(32);
      }
    }
    #pragma unroll
    for (int k = 0; k < 2 * M; ++k) v[k] += w[k];
  }
  // clear the entries read, for the next launch with this tag (a replay),
  // which starts only after this one has ended
  for (int sl = 1; sl < sh.n; ++sl) {
    unsigned long long* s_e = slot_entries<M>(a, J, rb, sl);
    if (!slot_in_range<M>(a, J, rb, sl)) continue;
    #pragma unroll
    for (int k = 0; k < 2 * M; ++k) s_e[seg_index(e, lane, k)] = 0ull;
  }
  gemv_store_rows<M>(J, rb, e, lane, a.err, v);
  return true;
}

template <int M>
__global__ void __launch_bounds__(kGemvThreads, 1) q4_gemv_kernel(const __grid_constant__ GemvArgs a) {
  extern __shared__ __align__(128) uint8_t smem[];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int S = a.stages;
  constexpr uint32_t kStage = gemv_stage_bytes(M);
  constexpr uint32_t kXOff = kGemvCols * kGemvWBox;
  uint8_t* ring = smem;
  constexpr int kRedBufs = gemv_red_bufs(M);
  float* red = reinterpret_cast<float*>(smem + size_t(S) * kStage);  // [bufs][8 slots][M][stride]
  volatile int* abort_flag = reinterpret_cast<volatile int*>(red + gemv_red_bytes(M) / 4);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + size_t(S) * kStage + gemv_red_bytes(M) + 16);
  uint64_t* empty = full + S;
  uint64_t* red_full = empty + S;            // [bufs] every slot holds both columns' sums
  uint64_t* red_empty = red_full + kRedBufs; // [bufs] buffer read by both epilogue warps
  uint64_t* red_pair = red_empty + kRedBufs; // pair slots: [bufs][8] column 0's sums are in

  if (tid == 0) {
    griddep_launch_dependents();  // the next kernel on the stream may start its prologue
    for (int s = 0; s < S; ++s) {
      mbar_init(smem_addr(&full[s]), 1);
      mbar_init(smem_addr(&empty[s]), kGemvConsumerWarps);
    }
    for (int b = 0; b < kRedBufs; ++b) {
      mbar_init(smem_addr(&red_full[b]), gemv_red_slots(M));
      mbar_init(smem_addr(&red_empty[b]), kGemvEpilogueWarps);
      if constexpr (gemv_pair_slots(M))
        for (int k = 0; k < 8; ++k) mbar_init(smem_addr(&red_pair[b * 8 + k]), 1);
    }
    *abort_flag = 0;
    mbar_init_fence();
  }
  __syncthreads();

  if (warp == kGemvProducerWarp) {
    // ------------------------------ producer ------------------------------
    if (lane != 0) return;
    const uint64_t pol = l2_evict_first_policy();
    UnitCursor w, xs;   // next unit whose weights / whose activations to issue
    cursor_enter(w, a, 0);
    xs = w;
    int stw = 0, stx = 0, x_job_ready = -1;
    int w_slot = 0, x_slot = 0;
    uint32_t w_par = 0;  // parity of the ring pass of stage stw
    bool prior_grid_done = false;
    // Is the input of the job of the oldest stage without activations ready?
    auto x_ready = [&]() {
      if (x_job_ready == xs.job) return true;
      bool ready;
      if (xs.wait_for < 0) {
        if (!prior_grid_done) {
          griddep_wait();  // the kernel before this one has finished, its writes visible
          prior_grid_done = true;
        }
        ready = true;
      } else {
        ready = ld_acquire_gpu(a.sync + xs.wait_for) >= xs.wait_rbs;
      }
      if (ready) {
        fence_proxy_async_global();
        x_job_ready = xs.job;
      }
      return ready;
    };
    auto issue_x = [&]() {
      const uint32_t bar = smem_addr(&full[x_slot]);
      const uint32_t dst = smem_addr(ring + size_t(x_slot) * kStage) + kXOff;
      const int col0 = 2 * xs.cp;
      const int kc = min(kGemvCols, xs.nsb - col0);
      #pragma unroll
      for (int m = 0; m < M; ++m)
        bulk_g2s_nohint(dst + uint32_t(m) * kGemvXPitch,
                        xs.x + x_offset_m<M>(xs, m, col0, kc, a.err), uint32_t(kc) * 512u, bar);
      ++stx;
      if (++x_slot == S) x_slot = 0;
      cursor_next(xs, a);
    };
    unsigned long long dep_since = 0;
    while (xs.job < a.n_jobs && !*abort_flag) {
      // activations of every armed stage whose job's input is ready
      while (stx < stw && x_ready()) issue_x();
      if (w.job < a.n_jobs &&
          (stw < S || mbar_test_wait(smem_addr(&empty[w_slot]), w_par ^ 1u))) {
        // weights of the next unit: its ring slot is free
        const int col0 = 2 * w.cp;
        const int kc = min(kGemvCols, w.nsb - col0);
        const int rows = min(kGemvRows, w.N - w.rb * kGemvRows);
        const uint32_t bar = smem_addr(&full[w_slot]);
        const uint32_t dst = smem_addr(ring + size_t(w_slot) * kStage);
        mbar_arrive_expect_tx(bar, uint32_t(kc) * (uint32_t(rows) * kSbBytes + uint32_t(M) * 512u));
        for (int j = 0; j < kc; ++j) {
          size_t off = (size_t(col0 + j) * w.N + size_t(w.rb) * kGemvRows) * kSbBytes;
          // a failed check copies the matrix's first rows instead (memory that exists)
          if (!Q4D_CHECK(off + uint32_t(rows) * kSbBytes <= size_t(w.w_bytes), a.err,
                         kSiteGemvWeights, off))
            off = 0;
          bulk_g2s(dst + uint32_t(j) * kGemvWBox, w.W + off, uint32_t(rows) * kSbBytes, bar, pol);
        }
        ++stw;
        if (++w_slot == S) {
          w_slot = 0;
          w_par ^= 1u;
        }
        cursor_next(w, a);
        dep_since = 0;
        continue;
      }
      if (stx < stw) {
        // an armed stage waits for its job's input (another job of the launch)
        const unsigned long long now = global_timer_ns();
        if (dep_since == 0) {
          dep_since = now;
        } else if (now - dep_since > kWaitLimitNs) {
          *abort_flag = 1;
          atomicOr(a.err, kDevErrWaitTimeout);
        }
        __nanosleep(200);
      } else if (w.job < a.n_jobs) {
        // ring full, every armed stage complete: sleep until a slot is free
        gemv_wait(smem_addr(&empty[w_slot]), w_par ^ 1u, a.err, abort_flag);
      }
    }
    // After an abort: complete every armed stage with its activation copies
    // (valid memory, stale values: the results are void anyway), so that each
    // armed barrier phase can complete.
    for (; stx < stw; ++stx) {
      const uint32_t bar = smem_addr(&full[x_slot]);
      const uint32_t dst = smem_addr(ring + size_t(x_slot) * kStage) + kXOff;
      const int col0 = 2 * xs.cp;
      const int kc = min(kGemvCols, xs.nsb - col0);
      for (int m = 0; m < M; ++m)
        bulk_g2s_nohint(dst + uint32_t(m) * kGemvXPitch,
                        xs.x + x_offset_m<M>(xs, m, col0, kc, a.err), uint32_t(kc) * 512u, bar);
      if (++x_slot == S) x_slot = 0;
      cursor_next(xs, a);
    }
    // Wait for the copies still in flight (bounded), so that none lands after
    // the CTA has exited: the last stage issued into each slot.
    for (int k = 0; k < S && k < stw; ++k) {
      const int st = stw - 1 - k;
      const uint32_t bar = smem_addr(&full[st % S]);
      const unsigned long long t0 = global_timer_ns();
      while (!mbar_try_wait(bar, uint32_t(st / S) & 1u) && global_timer_ns() - t0 < kWaitLimitNs) {
      }
    }
    return;
  }

  if (warp > kGemvProducerWarp) {
    // ------------------------------ epilogue ------------------------------
    // Both warps take every segment, warp e rows [64 e, 64 e + 64) of it; each
    // half of a row block written in final form is counted for its job (a
    // release reduction, so that a CTA which sees the count complete also sees
    // the rows).  Nothing of the workspace or the outputs is touched before
    // the previous kernel on the stream is complete (it may still use the same
    // buffers).
    griddep_wait();
    const int e = warp - kGemvProducerWarp - 1;
    int seg = 0;
    for (int job = 0; job < a.n_jobs; ++job) {
      const GemvJobDesc* J = gemv_job(a, job);
      const JobRange r = job_range(a, J);
      for (int u = r.ub; u < r.ue;) {
        const int rb = u / J->upr;
        const int u_end = min(r.ue, (rb + 1) * J->upr);
        const int b = seg % kRedBufs;
        const uint32_t fb = smem_addr(&red_full[b]), fpar = uint32_t(seg / kRedBufs) & 1u;
        // Finishing a row block shared with one CTA, whose part came at the
        // start of its range: read that CTA's slot while this CTA's own sums
        // are still being made (it is usually written by then).
        bool pre = false;
        float pv[2 * M];
        const RowBlockShare sh = row_block_share(J, r.cj, rb);
        if (sh.n == 2 && sh.my == 0 && slot_in_range<M>(a, J, rb, 1)) {
          const unsigned long long* s_e = slot_entries<M>(a, J, rb, 1);
          while (!pre && !mbar_test_wait(fb, fpar) && !*abort_flag) {
            pre = read_slot<M>(s_e, e, lane, unsigned(a.tag), pv);
            if (!pre) __nanosleep(256);
          }
        }
        gemv_wait(fb, fpar, a.err, abort_flag);
        float v[2 * M];
        gemv_segment_sum<M>(gemv_red_buffer<M>(red, b), &red_empty[b], e, lane, v);
        const bool wrote =
            gemv_segment_write<M>(a, J, r.cj, rb, e, lane, abort_flag, pre, pv, v);
        if (wrote && a.n_jobs > 1) {
          __syncwarp();
          if (lane == 0) red_release_gpu_add(a.sync + job, 1u);
        }
        ++seg;
        u = u_end;
      }
    }
    if (a.n_jobs > 1) {
      // both epilogue warps are done; the last CTA to leave sets the per-job
      // counts back to zero (every count of every CTA is in by then)
      asm volatile("bar.sync 2, %0;" ::"n"(kGemvEpilogueWarps * 32) : "memory");
      if (e == 0 && lane == 0 && atomicAdd(a.sync + a.n_jobs, 1u) == unsigned(a.grid - 1)) {
        fence_acq_rel_gpu();
        for (int i = 0; i <= a.n_jobs; ++i) a.sync[i] = 0u;
      }
    }
    return;
  }

  // ------------------------------ consumers ------------------------------
  const int g = lane >> 2, t = lane & 3;
  const int task_col = warp >> 3, task_blk = warp & 7;
  const uint32_t mask = 0x000F000Fu, magic = 0x43004300u, c136 = 0x43084308u;  // bf16 136
  const uint32_t x_lane = kXOff + g * kGemvXPitch + task_col * 512 + (task_blk * 32 + 4 * t) * 2;
  const uint32_t w_lane = task_col * kGemvWBox + g * kSbBytes + task_blk * 16 + t * 4;
  const uint32_t d_lane = task_col * kGemvWBox + g * kSbBytes + 128 + task_blk * 2;
  int slot = 0, seg = 0;
  uint32_t phase = 0;
  for (int job = 0; job < a.n_jobs; ++job) {
    const GemvJobDesc* J = gemv_job(a, job);
    const JobRange r = job_range(a, J);
    const int upr = J->upr, nsb = J->nsb;
    for (int u = r.ub; u < r.ue;) {
      const int rb = u / upr;
      const int cp0 = u - rb * upr;
      const int n_units = min(r.ue, (rb + 1) * upr) - u;
      float acc[kGemvTiles][4];
      #pragma unroll
      for (int p = 0; p < kGemvTiles; ++p) acc[p][0] = acc[p][1] = acc[p][2] = acc[p][3] = 0.f;
      #pragma unroll 1
      for (int k = 0; k < n_units; ++k) {
        gemv_wait(smem_addr(&full[slot]), phase, a.err, abort_flag);
        const uint8_t* stage = ring + size_t(slot) * kStage;
        if (task_col < nsb - 2 * (cp0 + k)) {
          // B fragment (x) of this warp's block of its column, for column g
          uint32_t bx[4] = {0u, 0u, 0u, 0u};
          if (g < M) {
            const uint2 lo = *reinterpret_cast<const uint2*>(stage + x_lane);
            const uint2 hi = *reinterpret_cast<const uint2*>(stage + x_lane + 32);
            bx[0] = prmt(lo.x, lo.y, 0x5410);  // (x[4t+0], x[4t+2])
            bx[1] = prmt(hi.x, hi.y, 0x5410);  // (x[16+4t+0], x[16+4t+2])
            bx[2] = prmt(lo.x, lo.y, 0x7632);  // (x[4t+1], x[4t+3])
            bx[3] = prmt(hi.x, hi.y, 0x7632);  // (x[16+4t+1], x[16+4t+3])
          }
          // rows beyond the matrix's last row hold stale data; their sums are never stored
          #pragma unroll
          for (int p = 0; p < kGemvTiles; ++p) {
            const uint8_t* pa = stage + w_lane + 16 * p * kSbBytes;
            const uint8_t* pd = stage + d_lane + 16 * p * kSbBytes;
            const uint32_t wa = *reinterpret_cast<const uint32_t*>(pa);
            const uint32_t wb = *reinterpret_cast<const uint32_t*>(pa + 8 * kSbBytes);
            const float da = half_bits_to_float(*reinterpret_cast<const uint16_t*>(pd));
            const float db = half_bits_to_float(*reinterpret_cast<const uint16_t*>(pd + 8 * kSbBytes));
            uint32_t qa[4], qb[4];
            dequant_pairs(wa, mask, magic, c136, qa);
            dequant_pairs(wb, mask, magic, c136, qb);
            float cc[4] = {0.f, 0.f, 0.f, 0.f};
            mma_bf16(cc, qa[0], qb[0], qa[1], qb[1], bx[0], bx[1]);
            mma_bf16(cc, qa[2], qb[2], qa[3], qb[3], bx[2], bx[3]);
            acc[p][0] = fmaf(da, cc[0], acc[p][0]);
            acc[p][2] = fmaf(db, cc[2], acc[p][2]);
            if constexpr (M > 1) {
              acc[p][1] = fmaf(da, cc[1], acc[p][1]);
              acc[p][3] = fmaf(db, cc[3], acc[p][3]);
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
      // hand this warp's sums of the row block to the epilogue: its slot of
      // reduction buffer seg % bufs (released by the epilogue after segment
      // seg - bufs), element (m, row) at m * stride + row.  With pair slots
      // the column-0 warp stores its sums into the slot of its block index,
      // and the column-1 warp adds its own once they are there and reports
      // the slot complete.
      const int b = seg % kRedBufs;
      if (seg >= kRedBufs)
        gemv_wait(smem_addr(&red_empty[b]), uint32_t((seg - kRedBufs) / kRedBufs) & 1u, a.err,
                  abort_flag);
      constexpr bool kPair = gemv_pair_slots(M);
      float* slot =
          gemv_red_buffer<M>(red, b) + size_t(kPair ? task_blk : warp) * M * kGemvRedStride;
      const uint32_t pair = kPair ? smem_addr(&red_pair[b * 8 + task_blk]) : 0u;
      if (!kPair || task_col == 0) {
        #pragma unroll
        for (int p = 0; p < kGemvTiles; ++p)
          #pragma unroll
          for (int e = 0; e < 2; ++e)
            if (2 * t + e < M) {
              slot[(2 * t + e) * kGemvRedStride + 16 * p + g] = acc[p][e];
              slot[(2 * t + e) * kGemvRedStride + 16 * p + g + 8] = acc[p][2 + e];
            }
        __syncwarp();
        if (lane == 0) mbar_arrive(kPair ? pair : smem_addr(&red_full[b]));
      } else {
        gemv_wait(pair, uint32_t(seg / kRedBufs) & 1u, a.err, abort_flag);
        #pragma unroll
        for (int p = 0; p < kGemvTiles; ++p)
          #pragma unroll
          for (int e = 0; e < 2; ++e)
            if (2 * t + e < M) {
              slot[(2 * t + e) * kGemvRedStride + 16 * p + g] += acc[p][e];
              slot[(2 * t + e) * kGemvRedStride + 16 * p + g + 8] += acc[p][2 + e];
            }
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_addr(&red_full[b]));
      }
      ++seg;
      u += n_units;
    }
  }
}

}  // namespace q4d
