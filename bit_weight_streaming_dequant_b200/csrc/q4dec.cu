// libq4dec C ABI: argument validation, launch planning, workspace handling
// and kernel dispatch.  Declarations and the contract live in include/q4dec.h.
#include "q4dec.h"

#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <map>
#include <mutex>
#include <tuple>
#include <unordered_map>

#include "q4_gemv.cuh"
#include "q4kv_attn.cuh"
#include "q4kv_attn_tc.cuh"
#include "q4kv_append.cuh"

// Device error record: word 0 holds the bits (q4d::kDevErrWaitTimeout: a
// bounded wait ran out; q4d::kDevErrIndex: an index check of a Q4D_DEBUG
// build failed), words 1..3 the first failed check's site and index.
__device__ unsigned q4d_error_word[q4d::kDevErrRecordWords];

namespace {

constexpr int kMaxDevices = 64;
constexpr int kPlanFallbackSms = 148;
constexpr size_t kAttnSmemBudget = 224 * 1024;   // shared memory per attention CTA
// The 8-bit cache's 70 KB ring stages need the device's whole opt-in shared
// memory per block (227 KB on B200) for two stages next to the V tile.
constexpr size_t kAttnSmemMax = 227 * 1024;

struct DeviceState {
  std::atomic<bool> ready{false};
  int num_sms = 0;
  int smem_optin = 0;
  unsigned* err = nullptr;
  void* ws = nullptr;  // library-owned workspace of the plain attention entry point
  size_t ws_bytes = 0;
  void* gemv_ws = nullptr;  // library-owned workspace of the plain GEMV entry point
  size_t gemv_ws_bytes = 0;
};

std::mutex g_mu;
DeviceState g_dev[kMaxDevices];

q4d_status current_device(int* dev_out, DeviceState** st_out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    cudaGetLastError();
    return Q4D_ERR_CUDA;
  }
  DeviceState& s = g_dev[dev];
  if (!s.ready.load(std::memory_order_acquire)) {
    std::lock_guard<std::mutex> lk(g_mu);
    if (!s.ready.load(std::memory_order_relaxed)) {
      if (cudaDeviceGetAttribute(&s.num_sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
          cudaDeviceGetAttribute(&s.smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) !=
              cudaSuccess ||
          cudaGetSymbolAddress(reinterpret_cast<void**>(&s.err), q4d_error_word) != cudaSuccess) {
        cudaGetLastError();
        return Q4D_ERR_CUDA;
      }
      s.ready.store(true, std::memory_order_release);
    }
  }
  *dev_out = dev;
  *st_out = &s;
  return Q4D_OK;
}

// The end of a compute call.  In a debug build (Q4D_DEBUG) the call waits for
// its stream and reports the device error record -- a failed index check, or
// a bounded wait that ran out -- as its own status (the record stays set
// until q4d_device_error(1) clears it); work captured into a graph is not
// waited for.  In a release build it only returns the launch status.
q4d_status finish_call(cudaStream_t stream, const DeviceState& s) {
  if (cudaGetLastError() != cudaSuccess) return Q4D_ERR_CUDA;
#ifdef Q4D_DEBUG
  cudaStreamCaptureStatus capture = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(stream, &capture) != cudaSuccess) {
    cudaGetLastError();
    return Q4D_ERR_CUDA;
  }
  if (capture != cudaStreamCaptureStatusNone) return Q4D_OK;
  unsigned word = 0;
  if (cudaStreamSynchronize(stream) != cudaSuccess ||
      cudaMemcpy(&word, s.err, sizeof(word), cudaMemcpyDeviceToHost) != cudaSuccess) {
    cudaGetLastError();
    return Q4D_ERR_CUDA;
  }
  if (word & q4d::kDevErrIndex) return Q4D_ERR_DEVICE_INDEX;
  if (word) return Q4D_ERR_DEVICE_TIMEOUT;
#else
  (void)stream;
  (void)s;
#endif
  return Q4D_OK;
}

// Raise a kernel's dynamic shared-memory limit to the device maximum, once
// per (kernel, device).
template <typename Kernel>
q4d_status allow_smem(Kernel kernel, int dev, const DeviceState& s, std::atomic<bool>* done) {
  if (done[dev].load(std::memory_order_acquire)) return Q4D_OK;
  if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, s.smem_optin) !=
      cudaSuccess) {
    cudaGetLastError();
    return Q4D_ERR_CUDA;
  }
  done[dev].store(true, std::memory_order_release);
  return Q4D_OK;
}

q4d_status library_workspace(void*& buf, size_t& bytes, size_t need, void** ws) {
  if (need == 0) {
    *ws = nullptr;
    return Q4D_OK;
  }
  std::lock_guard<std::mutex> lk(g_mu);
  if (bytes < need) {
    if (buf) cudaFree(buf);
    buf = nullptr;
    bytes = 0;
    if (cudaMalloc(&buf, need) != cudaSuccess) {
      cudaGetLastError();
      return Q4D_ERR_CUDA;
    }
    // zero-filled, as the GEMV's partial slots require (launches keep it so)
    if (cudaMemset(buf, 0, need) != cudaSuccess) {
      cudaGetLastError();
      cudaFree(buf);
      buf = nullptr;
      return Q4D_ERR_CUDA;
    }
    bytes = need;
  }
  *ws = buf;
  return Q4D_OK;
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

int ceil_div(long long a, long long b) { return int((a + b - 1) / b); }
long long round_up(long long a, long long b) { return (a + b - 1) / b * b; }

q4d_status check_gemv_shape(int M, int N, int K) {
  if (N < 1 || K < 0) return Q4D_ERR_INVALID_ARG;
  if (M < 1 || M > 5 || K < 256 || K % 256 != 0) return Q4D_ERR_UNSUPPORTED_SHAPE;
  return Q4D_OK;
}

q4d_status check_attn_shape(int ctx_len, int n_q, int n_kv, int head_dim, int M, int kv_stride,
                            float scale) {
  if (ctx_len < 1 || n_q < 1 || n_kv < 1 || !std::isfinite(scale)) return Q4D_ERR_INVALID_ARG;
  if (head_dim != 256 || M < 1 || M > 5 || n_q % n_kv != 0 || ctx_len < M ||
      kv_stride < ctx_len)
    return Q4D_ERR_UNSUPPORTED_SHAPE;
  return Q4D_OK;
}

// ---------------------------------------------------------------------------
// GEMV planning (stream-K over row blocks of 128 rows and units of two
// super-block columns; see q4_gemv.cuh).

// Shape of one job's partition over G CTAs.
struct JobShape {
  int rbs, upr, units, grid, slots;
};

// Most CTAs that share one row block (0 when every row block has one CTA).
int max_contributors(int rbs, int upr, int units, int G) {
  int slots = 0;
  for (int rb = 0; rb < rbs; ++rb) {
    const int first = q4d::unit_owner(rb * upr, units, G);
    const int last = q4d::unit_owner(rb * upr + upr - 1, units, G);
    if (last > first) slots = std::max(slots, last - first + 1);
  }
  return slots;
}

std::mutex g_shape_mu;
std::map<std::tuple<int, int, int>, int> g_slots_cache;

// Row blocks x units per row block must stay below 2^31 / grid (the kernel's
// 32-bit partition arithmetic); true for any matrix below ~500 GB.
bool shape_fits(int rows, int nsb, int launch_grid) {
  const long long units = (long long)ceil_div(rows, q4d::kGemvRows) * ceil_div(nsb, q4d::kGemvCols);
  return units * (long long)launch_grid < (1ll << 31);
}

JobShape job_shape(int rows, int nsb, int launch_grid) {
  JobShape j;
  j.rbs = ceil_div(rows, q4d::kGemvRows);
  j.upr = ceil_div(nsb, q4d::kGemvCols);
  j.units = j.rbs * j.upr;
  j.grid = std::min(launch_grid, j.units);
  const auto key = std::make_tuple(rows, nsb, j.grid);
  {
    std::lock_guard<std::mutex> lk(g_shape_mu);
    auto it = g_slots_cache.find(key);
    if (it != g_slots_cache.end()) {
      j.slots = it->second;
      return j;
    }
  }
  j.slots = max_contributors(j.rbs, j.upr, j.units, j.grid);
  std::lock_guard<std::mutex> lk(g_shape_mu);
  if (g_slots_cache.size() > 4096) g_slots_cache.clear();
  g_slots_cache.emplace(key, j.slots);
  return j;
}

// Ring stages that fit next to the reduction and segment buffers in
// `smem_limit` bytes (at most kGemvMaxStages).
int gemv_stages(int M, size_t smem_limit) {
  int stages = 0;
  while (stages < q4d::kGemvMaxStages && q4d::gemv_smem_bytes(M, stages + 1) <= smem_limit)
    ++stages;
  return stages;
}

constexpr size_t kGemvEntryBytes = 8;     // one partial-slot entry: fp32 value + tag
constexpr int kSmemOptinB200 = 232448;    // planning default: B200's opt-in shared memory

size_t round_up16(size_t v) { return (v + 15) / 16 * 16; }

q4d_status plan_gemv_rows(int M, int rows, int K, int num_sms, int smem_optin,
                          q4d_gemv_plan* plan) {
  if (!plan || num_sms < 1) return Q4D_ERR_INVALID_ARG;
  q4d_status st = check_gemv_shape(M, rows, K);
  if (st != Q4D_OK) return st;
  if (!shape_fits(rows, K / 256, num_sms)) return Q4D_ERR_UNSUPPORTED_SHAPE;
  const JobShape j = job_shape(rows, K / 256, num_sms);
  plan->grid = j.grid;
  plan->threads = q4d::kGemvThreads;
  plan->row_blocks = j.rbs;
  plan->units_per_row_block = j.upr;
  plan->units = j.units;
  plan->slots = j.slots;
  plan->stages = gemv_stages(M, size_t(smem_optin));
  plan->reserved = 0;
  plan->smem_bytes = q4d::gemv_smem_bytes(M, plan->stages);
  // the partial slots: [row block][slot][M][128] entries
  plan->workspace_bytes = size_t(j.rbs) * j.slots * M * q4d::kGemvRows * kGemvEntryBytes;
  return Q4D_OK;
}

std::atomic<unsigned long long> g_gemv_tag{0};

// Weight extent that GEMV index checks allow, if a test has capped it
// (q4d_debug_limit_weights; 0: none): the true N * K / 256 * 144 bytes, or
// the cap when that is smaller.
std::atomic<unsigned long long> g_weight_limit{0};
long long declared_weight_bytes(int rows, int nsb) {
  const unsigned long long full = (unsigned long long)rows * nsb * 144ull;
  const unsigned long long cap = g_weight_limit.load(std::memory_order_relaxed);
  return (long long)((cap > 0 && cap < full) ? cap : full);
}

// A fresh tag for every launch; its low 32 bits, the ones partial-slot entries
// carry, are never 0 (a cleared entry is 0).
unsigned long long next_gemv_tag() {
  unsigned long long t = (g_gemv_tag.fetch_add(1, std::memory_order_relaxed) + 1) &
                         0xFFFFFFFFull;
  return t ? t : 1ull;
}

template <int M>
q4d_status launch_gemv_t(const q4d::GemvArgs& a, size_t smem, int dev, const DeviceState& s,
                         cudaStream_t stream, bool pdl) {
  static std::atomic<bool> smem_set[kMaxDevices];
  auto kernel = q4d::q4_gemv_kernel<M>;
  q4d_status st = allow_smem(kernel, dev, s, smem_set);
  if (st != Q4D_OK) return st;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(a.grid);
  cfg.blockDim = dim3(q4d::kGemvThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kernel, a) == cudaSuccess ? Q4D_OK : Q4D_ERR_CUDA;
}

q4d_status launch_gemv(int M, const q4d::GemvArgs& a, size_t smem, int dev, const DeviceState& s,
                       cudaStream_t stream, bool pdl) {
  switch (M) {
    case 1: return launch_gemv_t<1>(a, smem, dev, s, stream, pdl);
    case 2: return launch_gemv_t<2>(a, smem, dev, s, stream, pdl);
    case 3: return launch_gemv_t<3>(a, smem, dev, s, stream, pdl);
    case 4: return launch_gemv_t<4>(a, smem, dev, s, stream, pdl);
    default: return launch_gemv_t<5>(a, smem, dev, s, stream, pdl);
  }
}

// y = W x (N output rows), or with `swiglu` h[m][n] = silu(g) * u over the N
// gate / up row pairs of W (2N weight rows): one job in one launch.
q4d_status gemv_impl(const void* W_q4, const void* x, void* y, int M, int N, int K,
                     cudaStream_t stream, void* workspace, size_t workspace_bytes,
                     bool library_ws, bool pdl = false, bool swiglu = false,
                     bool out_bf16 = false) {
  if (swiglu && N > (1 << 29)) return Q4D_ERR_UNSUPPORTED_SHAPE;
  q4d_status st = check_gemv_shape(M, swiglu ? 2 * N : N, K);
  if (st != Q4D_OK) return st;
  if (!W_q4 || !x || !y) return Q4D_ERR_INVALID_ARG;
  if (!aligned(W_q4, 16) || !aligned(x, 16) || !aligned(y, out_bf16 ? 2 : 4))
    return Q4D_ERR_MISALIGNED;
  if (workspace && !aligned(workspace, 16)) return Q4D_ERR_MISALIGNED;

  int dev = 0;
  DeviceState* s = nullptr;
  if ((st = current_device(&dev, &s)) != Q4D_OK) return st;
  const int rows = swiglu ? 2 * N : N;
  q4d_gemv_plan p;
  if ((st = plan_gemv_rows(M, rows, K, s->num_sms, s->smem_optin, &p)) != Q4D_OK) return st;
  if (p.stages < 2) return Q4D_ERR_UNSUPPORTED_SHAPE;
  if (library_ws) {
    if ((st = library_workspace(s->gemv_ws, s->gemv_ws_bytes, p.workspace_bytes, &workspace)) !=
        Q4D_OK)
      return st;
  } else if (p.workspace_bytes > 0 && (!workspace || workspace_bytes < p.workspace_bytes)) {
    return Q4D_ERR_WORKSPACE;
  }

  q4d::GemvArgs a;
  std::memset(&a, 0, sizeof(a));
  a.jobs = nullptr;
  a.n_jobs = 1;
  a.grid = p.grid;
  a.stages = p.stages;
  a.err = s->err;
  a.tag = next_gemv_tag();
  if (p.workspace_bytes > 0) {
    a.partials = static_cast<unsigned long long*>(workspace);
  }
  a.ws_entries = (long long)(p.workspace_bytes / kGemvEntryBytes);
  q4d::GemvJobDesc& J = a.job;
  J.W = static_cast<const uint8_t*>(W_q4);
  J.x = static_cast<const uint16_t*>(x);
  J.y = y;
  J.part_off = 0;
  J.N = rows;
  J.nsb = K / 256;
  J.flags = (out_bf16 ? q4d::kJobOutBf16 : 0u) | (swiglu ? q4d::kJobSwiglu : 0u);
  J.wait_for = -1;
  J.rbs = p.row_blocks;
  J.upr = p.units_per_row_block;
  J.units = p.units;
  J.grid = p.grid;
  J.slots = p.slots;
  J.rot = 0;
  J.w_bytes = declared_weight_bytes(rows, K / 256);
  if ((st = launch_gemv(M, a, p.smem_bytes, dev, *s, stream, pdl)) != Q4D_OK) return st;
  return finish_call(stream, *s);
}

// The warp-local mma.sync kernel (at most 8 query rows per CTA).
q4d_status launch_attn_rows8(const q4d::AttnArgs& a, const q4d_attn_plan& p, int n_kv, int dev,
                             const DeviceState& s, cudaStream_t stream) {
  static std::atomic<bool> smem_set[kMaxDevices];
  q4d_status st = allow_smem(q4d::q4kv_attn_split_rows8_kernel, dev, s, smem_set);
  if (st != Q4D_OK) return st;
  dim3 grid(p.n_splits, n_kv, p.row_groups);
  q4d::q4kv_attn_split_rows8_kernel<<<grid, p.threads, p.smem_bytes, stream>>>(a);
  return Q4D_OK;
}

// The tensor-memory kernel with NR (16 or 32) MMA columns of query rows, the
// Q4 or Q8 cache and PB P^T buffers.
template <int NR, bool Q8, int PB>
q4d_status launch_attn_tc(const q4d::AttnArgs& a, const q4d_attn_plan& p, int n_kv, int dev,
                          const DeviceState& s, cudaStream_t stream) {
  static std::atomic<bool> smem_set[kMaxDevices];
  q4d_status st = allow_smem(q4d::q4kv_attn_tc_kernel<NR, Q8, PB>, dev, s, smem_set);
  if (st != Q4D_OK) return st;
  dim3 grid(p.n_splits, n_kv, p.row_groups);
  q4d::q4kv_attn_tc_kernel<NR, Q8, PB><<<grid, p.threads, p.smem_bytes, stream>>>(a);
  return Q4D_OK;
}

// P^T buffers of the tensor-memory kernel: two, except for the 8-bit cache
// with 32 MMA columns, whose shared memory holds only one next to two stages.
int tca_pbufs(int nr, bool q8) { return (q8 && nr == 32) ? 1 : 2; }

q4d_status plan_attn_impl(int ctx_len, int n_q_heads, int n_kv_heads, int head_dim, int M,
                          int num_sms, bool q8, q4d_attn_plan* plan);

q4d_status attn_impl(const void* Q, const void* Kq4, const void* Vq4, float* out, int ctx_len,
                     int n_q, int n_kv, int head_dim, int M, int kv_stride, float scale,
                     cudaStream_t stream, void* workspace, size_t workspace_bytes,
                     bool library_ws, bool q8 = false) {
  q4d_status st = check_attn_shape(ctx_len, n_q, n_kv, head_dim, M, kv_stride, scale);
  if (st != Q4D_OK) return st;
  if (!Q || !Kq4 || !Vq4 || !out) return Q4D_ERR_INVALID_ARG;
  if (!aligned(Q, 16) || !aligned(Kq4, 16) || !aligned(Vq4, 16) || !aligned(out, 4))
    return Q4D_ERR_MISALIGNED;
  if (workspace && !aligned(workspace, 16)) return Q4D_ERR_MISALIGNED;

  int dev = 0;
  DeviceState* s = nullptr;
  if ((st = current_device(&dev, &s)) != Q4D_OK) return st;
  q4d_attn_plan p;
  if ((st = plan_attn_impl(ctx_len, n_q, n_kv, head_dim, M, s->num_sms, q8, &p)) != Q4D_OK)
    return st;
  if (p.smem_bytes > size_t(s->smem_optin)) return Q4D_ERR_UNSUPPORTED_SHAPE;
  if (library_ws) {
    if ((st = library_workspace(s->ws, s->ws_bytes, p.workspace_bytes, &workspace)) != Q4D_OK)
      return st;
  } else if (p.workspace_bytes > 0 && (!workspace || workspace_bytes < p.workspace_bytes)) {
    return Q4D_ERR_WORKSPACE;
  }

  q4d::AttnArgs a;
  std::memset(&a, 0, sizeof(a));
  a.Q = static_cast<const uint16_t*>(Q);
  a.K = static_cast<const uint8_t*>(Kq4);
  a.V = static_cast<const uint8_t*>(Vq4);
  a.out = out;
  a.ws_o = static_cast<float*>(workspace);
  a.ws_ml = a.ws_o ? a.ws_o + size_t(p.n_splits) * M * n_q * 256 : nullptr;
  a.err = s->err;
  a.ctx_len = ctx_len;
  a.n_q = n_q;
  a.n_kv = n_kv;
  a.M = M;
  a.g = n_q / n_kv;
  a.kv_stride = kv_stride;
  a.scale_log2 = scale * 1.4426950408889634f;  // log2(e): the kernel works in base 2
  a.n_splits = p.n_splits;
  a.split_tokens = p.split_tokens;
  a.rows_per_cta = p.rows_per_cta;
  a.stages = p.stages;
  a.ws_floats = (long long)(p.workspace_bytes / 4);

  if (!q8 && p.rows_per_cta <= 8)
    st = launch_attn_rows8(a, p, n_kv, dev, *s, stream);
  else if (p.rows_per_cta <= 16)
    st = q8 ? launch_attn_tc<16, true, 2>(a, p, n_kv, dev, *s, stream)
            : launch_attn_tc<16, false, 2>(a, p, n_kv, dev, *s, stream);
  else
    st = q8 ? launch_attn_tc<32, true, 1>(a, p, n_kv, dev, *s, stream)
            : launch_attn_tc<32, false, 2>(a, p, n_kv, dev, *s, stream);
  if (st != Q4D_OK) return st;
  if (p.n_splits > 1) {
    // the merge may launch while the split kernel runs; it waits for it on
    // the device (griddepcontrol.wait) before reading the split states
    cudaLaunchConfig_t cfg;
    std::memset(&cfg, 0, sizeof(cfg));
    cfg.gridDim = dim3(unsigned(M * n_q));
    cfg.blockDim = dim3(256);
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, q4d::q4kv_attn_merge_kernel, a) != cudaSuccess) {
      cudaGetLastError();
      return Q4D_ERR_CUDA;
    }
  }
  return finish_call(stream, *s);
}

int planning_sms() {
  int dev = 0;
  DeviceState* s = nullptr;
  if (current_device(&dev, &s) != Q4D_OK) return kPlanFallbackSms;
  return s->num_sms;
}

}  // namespace

extern "C" {

int q4d_version(void) { return Q4D_VERSION; }

const char* q4d_status_string(int status) {
  switch (status) {
    case Q4D_OK: return "ok";
    case Q4D_ERR_INVALID_ARG: return "invalid argument";
    case Q4D_ERR_UNSUPPORTED_SHAPE: return "unsupported shape";
    case Q4D_ERR_MISALIGNED: return "misaligned pointer";
    case Q4D_ERR_WORKSPACE: return "workspace missing or too small";
    case Q4D_ERR_CUDA: return "CUDA runtime error";
    case Q4D_ERR_DEVICE_TIMEOUT: return "in-kernel wait timed out";
    case Q4D_ERR_DEVICE_INDEX: return "index check failed (debug build)";
    default: return "unknown status";
  }
}

q4d_status q4d_plan_gemv(int M, int N, int K, int num_sms, q4d_gemv_plan* plan) {
  return plan_gemv_rows(M, N, K, num_sms, kSmemOptinB200, plan);
}

q4d_status q4d_plan_attn(int ctx_len, int n_q_heads, int n_kv_heads, int head_dim, int M,
                         int num_sms, q4d_attn_plan* plan) {
  return plan_attn_impl(ctx_len, n_q_heads, n_kv_heads, head_dim, M, num_sms, false, plan);
}

q4d_status q8kv_plan_attn(int ctx_len, int n_q_heads, int n_kv_heads, int head_dim, int M,
                          int num_sms, q4d_attn_plan* plan) {
  return plan_attn_impl(ctx_len, n_q_heads, n_kv_heads, head_dim, M, num_sms, true, plan);
}

}  // extern "C"

namespace {

// Variant: warp-local mma.sync kernel (12 warps, 192-token tiles) for at
// most 8 rows per CTA of the Q4 cache, else the tensor-memory kernel (8 token
// warps, a producer warp and an MMA warp; 128-token tiles; 16 or 32 MMA
// columns), which also serves every row count of the Q8 cache.
q4d_status plan_attn_impl(int ctx_len, int n_q_heads, int n_kv_heads, int head_dim, int M,
                          int num_sms, bool q8, q4d_attn_plan* plan) {
  if (!plan || num_sms < 1) return Q4D_ERR_INVALID_ARG;
  q4d_status st = check_attn_shape(ctx_len, n_q_heads, n_kv_heads, head_dim, M, ctx_len, 1.0f);
  if (st != Q4D_OK) return st;
  const int rows_all = (n_q_heads / n_kv_heads) * M;
  const int row_groups = ceil_div(rows_all, q4d::kAttnMaxRows);
  const int rows_per_cta = ceil_div(rows_all, row_groups);
  const bool rows8 = !q8 && rows_per_cta <= 8;
  const int nr = rows_per_cta <= 16 ? 16 : 32;
  const int pb = tca_pbufs(nr, q8);
  const int TT = rows8 ? q4d::kR8Tile : q4d::kTcaTile;
  const size_t stage_bytes = rows8 ? q4d::kR8StageBytes : q4d::tca_stage_bytes(q8);
  // One CTA per SM (the K/V ring takes most of shared memory): enough context
  // splits that (splits x KV heads x row groups) fills the SMs once, each
  // split at least two tiles long and at most 256 splits (the merge kernel's
  // limit).
  const long long ctas_per_split = (long long)n_kv_heads * row_groups;
  int n_splits = int(std::max<long long>(1, (num_sms + ctas_per_split - 1) / ctas_per_split));
  n_splits = std::min(n_splits, std::max(1, ceil_div(ctx_len, 2 * TT)));
  n_splits = std::min(n_splits, 256);
  const int split_tokens = int(round_up(ceil_div(ctx_len, n_splits), TT));
  n_splits = ceil_div(ctx_len, split_tokens);
  // As many ring stages as fit next to the variant's fixed buffers, up to 8
  // (at least 2: the warp-local variant parks 96 KB in the ring at the end).
  const size_t fixed = rows8 ? q4d::attn_rows8_smem_bytes(0) : q4d::tca_smem_bytes(nr, 0, q8, pb);
  const size_t budget = q8 ? kAttnSmemMax : kAttnSmemBudget;
  int stages = int((budget - fixed) / (stage_bytes + 16));
  stages = std::max(2, std::min(8, stages));
  plan->n_splits = n_splits;
  plan->split_tokens = split_tokens;
  plan->tile_tokens = TT;
  plan->row_groups = row_groups;
  plan->rows_per_cta = rows_per_cta;
  plan->stages = stages;
  plan->threads = rows8 ? q4d::kR8Threads : q4d::kTcaThreads;
  plan->smem_bytes =
      rows8 ? q4d::attn_rows8_smem_bytes(stages) : q4d::tca_smem_bytes(nr, stages, q8, pb);
  plan->workspace_bytes =
      n_splits > 1 ? size_t(n_splits) * M * n_q_heads * (q4d::kHeadDim + 2) * 4 : 0;
  return Q4D_OK;
}

}  // namespace

extern "C" {

size_t q4d_gemv_workspace_bytes(int M, int N, int K) {
  q4d_gemv_plan p;
  int dev = 0;
  DeviceState* s = nullptr;
  const bool have = current_device(&dev, &s) == Q4D_OK;
  if (plan_gemv_rows(M, N, K, have ? s->num_sms : kPlanFallbackSms,
                     have ? s->smem_optin : kSmemOptinB200, &p) != Q4D_OK)
    return 0;
  return p.workspace_bytes;
}

size_t q4d_attn_workspace_bytes(int ctx_len, int n_q_heads, int n_kv_heads, int head_dim, int M) {
  q4d_attn_plan p;
  if (q4d_plan_attn(ctx_len, n_q_heads, n_kv_heads, head_dim, M, planning_sms(), &p) != Q4D_OK)
    return 0;
  return p.workspace_bytes;
}

size_t q8kv_attn_workspace_bytes(int ctx_len, int n_q_heads, int n_kv_heads, int head_dim, int M) {
  q4d_attn_plan p;
  if (q8kv_plan_attn(ctx_len, n_q_heads, n_kv_heads, head_dim, M, planning_sms(), &p) != Q4D_OK)
    return 0;
  return p.workspace_bytes;
}

q4d_status q4_gemv(const void* W_q4, const void* x, float* y, int M, int N, int K) {
  return gemv_impl(W_q4, x, y, M, N, K, nullptr, nullptr, 0, true);
}

q4d_status q4_gemv_ex(const void* W_q4, const void* x, float* y, int M, int N, int K,
                      void* stream, void* workspace, size_t workspace_bytes) {
  return gemv_impl(W_q4, x, y, M, N, K, static_cast<cudaStream_t>(stream), workspace,
                   workspace_bytes, false);
}

q4d_status q4_gemv_ex2(const void* W_q4, const void* x, void* y, int M, int N, int K,
                       void* stream, void* workspace, size_t workspace_bytes, unsigned flags) {
  if (flags & ~(Q4D_GEMV_WEIGHT_PREFETCH | Q4D_GEMV_OUT_BF16)) return Q4D_ERR_INVALID_ARG;
  return gemv_impl(W_q4, x, y, M, N, K, static_cast<cudaStream_t>(stream), workspace,
                   workspace_bytes, false, (flags & Q4D_GEMV_WEIGHT_PREFETCH) != 0, false,
                   (flags & Q4D_GEMV_OUT_BF16) != 0);
}

q4d_status q4_gemv_swiglu_ex(const void* W_gu, const void* x, void* h, int M, int N, int K,
                             void* stream, void* workspace, size_t workspace_bytes,
                             unsigned flags) {
  if (flags & ~(Q4D_GEMV_WEIGHT_PREFETCH | Q4D_GEMV_OUT_BF16)) return Q4D_ERR_INVALID_ARG;
  return gemv_impl(W_gu, x, h, M, N, K, static_cast<cudaStream_t>(stream), workspace,
                   workspace_bytes, false, (flags & Q4D_GEMV_WEIGHT_PREFETCH) != 0, true,
                   (flags & Q4D_GEMV_OUT_BF16) != 0);
}

size_t q4d_gemv_swiglu_workspace_bytes(int M, int N, int K) {
  if (N < 1 || N > (1 << 29)) return 0;
  return q4d_gemv_workspace_bytes(M, 2 * N, K);
}

// ---- GEMV batches: many matrices in one launch
namespace {

constexpr uint32_t kBatchMagic = 0x42443451u;  // "Q4DB"
constexpr size_t kBatchHeader = 64;

struct BatchHeader {
  uint32_t magic;
  int n_jobs, M, num_sms, grid;
  int pad_;
  size_t workspace_bytes;
  size_t reserved_;
};
static_assert(sizeof(BatchHeader) <= kBatchHeader, "batch header");
static_assert(sizeof(q4d::GemvJobDesc) % 16 == 0, "job descriptor alignment");

}  // namespace

// Descriptor: header, the jobs, then the per-job completion counters and the
// exit counter (zero when handed to the device; each launch leaves them zero).
size_t batch_sync_offset(int n_jobs) {
  return kBatchHeader + size_t(n_jobs) * sizeof(q4d::GemvJobDesc);
}

size_t q4d_gemv_batch_desc_bytes(int n_jobs) {
  if (n_jobs < 1 || n_jobs > (1 << 20)) return 0;
  return batch_sync_offset(n_jobs) + round_up16(size_t(n_jobs + 1) * 4);
}

q4d_status q4d_gemv_batch_prepare(const q4d_gemv_job* jobs, int n_jobs, int M, int num_sms,
                                  void* desc, size_t desc_bytes, size_t* workspace_bytes) {
  if (!jobs || !desc || n_jobs < 1 || n_jobs > (1 << 20) || num_sms < 1 || num_sms > 65535)
    return Q4D_ERR_INVALID_ARG;
  if (M < 1 || M > 5) return Q4D_ERR_UNSUPPORTED_SHAPE;
  if (desc_bytes < q4d_gemv_batch_desc_bytes(n_jobs)) return Q4D_ERR_INVALID_ARG;
  // grid: one CTA per SM, fewer if no job has that many units
  int grid = 1;
  for (int i = 0; i < n_jobs; ++i) {
    const q4d_gemv_job& j = jobs[i];
    const bool swiglu = (j.flags & Q4D_GEMV_SWIGLU) != 0;
    if (j.flags & ~(Q4D_GEMV_OUT_BF16 | Q4D_GEMV_SWIGLU)) return Q4D_ERR_INVALID_ARG;
    if (swiglu && j.N > (1 << 29)) return Q4D_ERR_UNSUPPORTED_SHAPE;
    q4d_status st = check_gemv_shape(M, swiglu ? 2 * j.N : j.N, j.K);
    if (st != Q4D_OK) return st;
    if (!j.W_q4 || !j.x || !j.y) return Q4D_ERR_INVALID_ARG;
    if (!aligned(j.W_q4, 16) || !aligned(j.x, 16) ||
        !aligned(j.y, (j.flags & Q4D_GEMV_OUT_BF16) ? 2 : 4))
      return Q4D_ERR_MISALIGNED;
    if (j.wait_for < -1 || j.wait_for >= i) return Q4D_ERR_INVALID_ARG;
    if (!shape_fits(swiglu ? 2 * j.N : j.N, j.K / 256, num_sms)) return Q4D_ERR_UNSUPPORTED_SHAPE;
    const JobShape sh = job_shape(swiglu ? 2 * j.N : j.N, j.K / 256, num_sms);
    grid = std::max(grid, sh.grid);
  }
  q4d::GemvJobDesc* out =
      reinterpret_cast<q4d::GemvJobDesc*>(static_cast<uint8_t*>(desc) + kBatchHeader);
  size_t partials = 0;  // partial-slot entries
  long long units_before = 0;  // rotates each job's CTA numbering (balance across the batch)
  for (int i = 0; i < n_jobs; ++i) {
    const q4d_gemv_job& j = jobs[i];
    const bool swiglu = (j.flags & Q4D_GEMV_SWIGLU) != 0;
    const int rows = swiglu ? 2 * j.N : j.N;
    const JobShape sh = job_shape(rows, j.K / 256, grid);
    q4d::GemvJobDesc d;
    std::memset(&d, 0, sizeof(d));
    d.W = static_cast<const uint8_t*>(j.W_q4);
    d.x = static_cast<const uint16_t*>(j.x);
    d.y = j.y;
    d.N = rows;
    d.nsb = j.K / 256;
    d.flags = ((j.flags & Q4D_GEMV_OUT_BF16) ? q4d::kJobOutBf16 : 0u) |
              (swiglu ? q4d::kJobSwiglu : 0u);
    d.wait_for = j.wait_for;
    d.rbs = sh.rbs;
    d.upr = sh.upr;
    d.units = sh.units;
    d.grid = sh.grid;
    d.slots = sh.slots;
    d.part_off = (long long)partials;
    d.rot = int(units_before % grid);
    d.w_bytes = declared_weight_bytes(rows, j.K / 256);
    units_before += sh.units;
    if (sh.slots > 0) {
      partials += size_t(sh.rbs) * sh.slots * M * q4d::kGemvRows;
    }
    std::memcpy(out + i, &d, sizeof(d));
  }
  BatchHeader h;
  std::memset(&h, 0, sizeof(h));
  h.magic = kBatchMagic;
  h.n_jobs = n_jobs;
  h.M = M;
  h.num_sms = num_sms;
  h.grid = grid;
  h.workspace_bytes = partials * kGemvEntryBytes;
  std::memset(desc, 0, kBatchHeader);
  std::memcpy(desc, &h, sizeof(h));
  std::memset(static_cast<uint8_t*>(desc) + batch_sync_offset(n_jobs), 0,
              q4d_gemv_batch_desc_bytes(n_jobs) - batch_sync_offset(n_jobs));
  if (workspace_bytes) *workspace_bytes = h.workspace_bytes;
  return Q4D_OK;
}

q4d_status q4_gemv_batch_ex(const void* desc_host, void* desc_dev, void* stream,
                            void* workspace, size_t workspace_bytes, unsigned flags) {
  if (!desc_host || !desc_dev) return Q4D_ERR_INVALID_ARG;
  if (flags & ~Q4D_GEMV_WEIGHT_PREFETCH) return Q4D_ERR_INVALID_ARG;
  BatchHeader h;
  std::memcpy(&h, desc_host, sizeof(h));
  if (h.magic != kBatchMagic || h.n_jobs < 1 || h.M < 1 || h.M > 5 || h.grid < 1)
    return Q4D_ERR_INVALID_ARG;
  if (!aligned(desc_dev, 16) || (workspace && !aligned(workspace, 16))) return Q4D_ERR_MISALIGNED;
  if (h.workspace_bytes > 0 && (!workspace || workspace_bytes < h.workspace_bytes))
    return Q4D_ERR_WORKSPACE;
  int dev = 0;
  DeviceState* s = nullptr;
  q4d_status st = current_device(&dev, &s);
  if (st != Q4D_OK) return st;
  if (h.num_sms != s->num_sms) return Q4D_ERR_INVALID_ARG;  // prepared for another device
  const int stages = gemv_stages(h.M, size_t(s->smem_optin));
  if (stages < 2) return Q4D_ERR_UNSUPPORTED_SHAPE;
  q4d::GemvArgs a;
  std::memset(&a, 0, sizeof(a));
  a.jobs = reinterpret_cast<const q4d::GemvJobDesc*>(static_cast<const uint8_t*>(desc_dev) +
                                                      kBatchHeader);
  a.sync = reinterpret_cast<unsigned*>(static_cast<uint8_t*>(desc_dev) +
                                       batch_sync_offset(h.n_jobs));
  a.n_jobs = h.n_jobs;
  a.grid = h.grid;
  a.stages = stages;
  a.err = s->err;
  a.tag = next_gemv_tag();
  a.partials = static_cast<unsigned long long*>(workspace);
  a.ws_entries = (long long)(h.workspace_bytes / kGemvEntryBytes);
  if ((st = launch_gemv(h.M, a, q4d::gemv_smem_bytes(h.M, stages), dev, *s,
                        static_cast<cudaStream_t>(stream), (flags & Q4D_GEMV_WEIGHT_PREFETCH) != 0)) !=
      Q4D_OK)
    return st;
  return finish_call(static_cast<cudaStream_t>(stream), *s);
}

q4d_status q4kv_attn_decode(const void* Q, const void* Kq4, const void* Vq4, float* out,
                            int ctx_len, int n_q_heads, int n_kv_heads, int head_dim, int M) {
  return attn_impl(Q, Kq4, Vq4, out, ctx_len, n_q_heads, n_kv_heads, head_dim, M, ctx_len, 1.0f,
                   nullptr, nullptr, 0, true);
}

q4d_status q4kv_attn_decode_ex(const void* Q, const void* Kq4, const void* Vq4, float* out,
                               int ctx_len, int n_q_heads, int n_kv_heads, int head_dim, int M,
                               int kv_stride_tokens, float softmax_scale, void* stream,
                               void* workspace, size_t workspace_bytes) {
  return attn_impl(Q, Kq4, Vq4, out, ctx_len, n_q_heads, n_kv_heads, head_dim, M,
                   kv_stride_tokens, softmax_scale, static_cast<cudaStream_t>(stream), workspace,
                   workspace_bytes, false);
}

q4d_status q8kv_attn_decode_ex(const void* Q, const void* Kq8, const void* Vq8, float* out,
                               int ctx_len, int n_q_heads, int n_kv_heads, int head_dim, int M,
                               int kv_stride_tokens, float softmax_scale, void* stream,
                               void* workspace, size_t workspace_bytes) {
  return attn_impl(Q, Kq8, Vq8, out, ctx_len, n_q_heads, n_kv_heads, head_dim, M,
                   kv_stride_tokens, softmax_scale, static_cast<cudaStream_t>(stream), workspace,
                   workspace_bytes, false, true);
}

}  // extern "C"

// ---- K/V append
extern "C" q4d_status q4kv_append(void* Kq4, void* Vq4, const float* k_new, const float* v_new,
                                  int n_kv_heads, int kv_stride_tokens, int pos, int M,
                                  void* stream) {
  if (!Kq4 || !Vq4 || !k_new || !v_new || n_kv_heads < 1 || M < 1 || pos < 0 ||
      kv_stride_tokens < 1)
    return Q4D_ERR_INVALID_ARG;
  if ((long long)pos + M > kv_stride_tokens) return Q4D_ERR_UNSUPPORTED_SHAPE;
  if (!aligned(Kq4, 16) || !aligned(Vq4, 16) || !aligned(k_new, 4) || !aligned(v_new, 4))
    return Q4D_ERR_MISALIGNED;
  int dev = 0;
  DeviceState* s = nullptr;
  q4d_status st = current_device(&dev, &s);
  if (st != Q4D_OK) return st;
  q4d::AppendArgs a;
  a.K = static_cast<uint8_t*>(Kq4);
  a.V = static_cast<uint8_t*>(Vq4);
  a.k_new = k_new;
  a.v_new = v_new;
  a.n_kv = n_kv_heads;
  a.kv_stride = kv_stride_tokens;
  a.pos = pos;
  a.M = M;
  a.err = s->err;
  q4d::q4kv_append_kernel<<<dim3(M * n_kv_heads, 2), 256, 0, static_cast<cudaStream_t>(stream)>>>(a);
  return finish_call(static_cast<cudaStream_t>(stream), *s);
}

// ---- host layout helpers: canonical 18-byte blocks <-> 144-byte super-blocks
namespace {
q4d_status check_pack_args(const void* a, const void* b, int rows, int K) {
  if (!a || !b || rows < 1 || K < 0) return Q4D_ERR_INVALID_ARG;
  if (K < 256 || K % 256 != 0) return Q4D_ERR_UNSUPPORTED_SHAPE;
  return Q4D_OK;
}
// super-block index of (row r, column s) in either layout
size_t sb_index(bool column_major, int rows, int nsb, int r, int s) {
  return column_major ? size_t(s) * rows + r : size_t(r) * nsb + s;
}
q4d_status pack_impl(const void* blocks18, void* out, int rows, int K, bool column_major) {
  q4d_status st = check_pack_args(blocks18, out, rows, K);
  if (st != Q4D_OK) return st;
  const int nsb = K / 256;
  const uint8_t* in = static_cast<const uint8_t*>(blocks18);
  uint8_t* o = static_cast<uint8_t*>(out);
  for (int r = 0; r < rows; ++r)
    for (int s = 0; s < nsb; ++s) {
      uint8_t* sb = o + sb_index(column_major, rows, nsb, r, s) * 144;
      for (int b = 0; b < 8; ++b) {
        const uint8_t* blk = in + (size_t(r) * (K / 32) + size_t(s) * 8 + b) * 18;
        std::memcpy(sb + 16 * b, blk + 2, 16);     // nibbles
        std::memcpy(sb + 128 + 2 * b, blk, 2);     // fp16 scale
      }
    }
  return Q4D_OK;
}
q4d_status unpack_impl(const void* in_q4, void* blocks18, int rows, int K, bool column_major) {
  q4d_status st = check_pack_args(in_q4, blocks18, rows, K);
  if (st != Q4D_OK) return st;
  const int nsb = K / 256;
  const uint8_t* in = static_cast<const uint8_t*>(in_q4);
  uint8_t* o = static_cast<uint8_t*>(blocks18);
  for (int r = 0; r < rows; ++r)
    for (int s = 0; s < nsb; ++s) {
      const uint8_t* sb = in + sb_index(column_major, rows, nsb, r, s) * 144;
      for (int b = 0; b < 8; ++b) {
        uint8_t* blk = o + (size_t(r) * (K / 32) + size_t(s) * 8 + b) * 18;
        std::memcpy(blk, sb + 128 + 2 * b, 2);
        std::memcpy(blk + 2, sb + 16 * b, 16);
      }
    }
  return Q4D_OK;
}
}  // namespace

extern "C" {
q4d_status q4d_pack_q4_0_weights(const void* blocks18, void* W_q4, int N, int K) {
  return pack_impl(blocks18, W_q4, N, K, true);
}
q4d_status q4d_unpack_q4_0_weights(const void* W_q4, void* blocks18, int N, int K) {
  return unpack_impl(W_q4, blocks18, N, K, true);
}
q4d_status q4d_pack_q4_0_rows(const void* blocks18, void* rows_q4, int rows, int K) {
  return pack_impl(blocks18, rows_q4, rows, K, false);
}
q4d_status q4d_unpack_q4_0_rows(const void* rows_q4, void* blocks18, int rows, int K) {
  return unpack_impl(rows_q4, blocks18, rows, K, false);
}
}  // extern "C"

extern "C" {
q4d_status q4d_device_error_record(unsigned* record, int reset) {
  int dev = 0;
  DeviceState* s = nullptr;
  q4d_status st = current_device(&dev, &s);
  if (st != Q4D_OK) return st;
  unsigned rec[q4d::kDevErrRecordWords] = {0u, 0u, 0u, 0u};
  if (cudaDeviceSynchronize() != cudaSuccess ||
      cudaMemcpy(rec, s->err, sizeof(rec), cudaMemcpyDeviceToHost) != cudaSuccess) {
    cudaGetLastError();
    return Q4D_ERR_CUDA;
  }
  if (record) std::memcpy(record, rec, sizeof(rec));
  if (reset && (rec[0] | rec[1] | rec[2] | rec[3])) {
    const unsigned zero[q4d::kDevErrRecordWords] = {0u, 0u, 0u, 0u};
    if (cudaMemcpy(s->err, zero, sizeof(zero), cudaMemcpyHostToDevice) != cudaSuccess)
      return Q4D_ERR_CUDA;
  }
  if (rec[0] & q4d::kDevErrIndex) return Q4D_ERR_DEVICE_INDEX;
  return rec[0] ? Q4D_ERR_DEVICE_TIMEOUT : Q4D_OK;
}

q4d_status q4d_device_error(int reset) { return q4d_device_error_record(nullptr, reset); }

int q4d_debug_build(void) {
#ifdef Q4D_DEBUG
  return 1;
#else
  return 0;
#endif
}

q4d_status q4d_debug_limit_weights(unsigned long long bytes) {
#ifdef Q4D_DEBUG
  g_weight_limit.store(bytes, std::memory_order_relaxed);
  return Q4D_OK;
#else
  (void)bytes;
  return Q4D_ERR_INVALID_ARG;
#endif
}

}  // extern "C"

// ----------------------------------------------------------------------------
// Allocation-free attention (q4kv_attn_decode_noalloc): the split states live
// in this file-scope device array instead of a caller or library allocation.
// In host code the name below is only a host-side stand-in; kernels get the
// device address looked up per device with cudaGetSymbolAddress.
static __device__ __align__(256) unsigned char q4d_noalloc_scratch[Q4D_NOALLOC_SCRATCH_BYTES];

namespace {

struct NoAllocScratch {
  std::atomic<bool> ready{false};
  void* ptr = nullptr;
};
NoAllocScratch g_noalloc[kMaxDevices];
std::mutex g_noalloc_mu;

// Device address of the scratch array on the current device, looked up once.
q4d_status noalloc_scratch(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    cudaGetLastError();
    return Q4D_ERR_CUDA;
  }
  NoAllocScratch& s = g_noalloc[dev];
  if (!s.ready.load(std::memory_order_acquire)) {
    std::lock_guard<std::mutex> lk(g_noalloc_mu);
    if (!s.ready.load(std::memory_order_relaxed)) {
      void* p = nullptr;
      if (cudaGetSymbolAddress(&p, q4d_noalloc_scratch) != cudaSuccess || p == nullptr) {
        cudaGetLastError();
        return Q4D_ERR_CUDA;
      }
      s.ptr = p;
      s.ready.store(true, std::memory_order_release);
    }
  }
  *out = s.ptr;
  return Q4D_OK;
}

}  // namespace

extern "C" q4d_status q4kv_attn_decode_noalloc(const void* Q, const void* Kq4, const void* Vq4,
                                               float* out, int ctx_len, int n_q_heads,
                                               int n_kv_heads, int head_dim, int M,
                                               int kv_stride_tokens, float softmax_scale,
                                               void* stream) {
  // Reject bad arguments before touching CUDA, as the other entry points do.
  q4d_status st = check_attn_shape(ctx_len, n_q_heads, n_kv_heads, head_dim, M,
                                   kv_stride_tokens, softmax_scale);
  if (st != Q4D_OK) return st;
  if (!Q || !Kq4 || !Vq4 || !out) return Q4D_ERR_INVALID_ARG;
  if (!aligned(Q, 16) || !aligned(Kq4, 16) || !aligned(Vq4, 16) || !aligned(out, 4))
    return Q4D_ERR_MISALIGNED;
  void* scratch = nullptr;
  if ((st = noalloc_scratch(&scratch)) != Q4D_OK) return st;
  // The workspace path never allocates; a plan needing more than the array
  // holds comes back as Q4D_ERR_WORKSPACE before any launch.
  return attn_impl(Q, Kq4, Vq4, out, ctx_len, n_q_heads, n_kv_heads, head_dim, M,
                   kv_stride_tokens, softmax_scale, static_cast<cudaStream_t>(stream), scratch,
                   Q4D_NOALLOC_SCRATCH_BYTES, false);
}
