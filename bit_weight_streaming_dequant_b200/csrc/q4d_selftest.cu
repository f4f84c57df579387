// Self-tests of the library's two failure reports.  First the bounded
// in-kernel wait that every pipeline of the library relies on to terminate:
// one CTA waits, by phase parity, on an mbarrier that (unless asked to)
// nobody arrives on, with the same try-wait and wall-clock check the kernels
// use but a caller-chosen limit.  When the limit runs out the kernel records
// it in a caller-owned word and returns normally, so the CUDA context stays
// usable.  Then the record of a failed index check (below).  Nothing here
// faults, traps or spins without a bound.
#include <cuda_runtime.h>

#include "q4dec.h"
#include "q4dec_device.cuh"

namespace {

__global__ void q4d_wait_selftest_kernel(unsigned* word, unsigned long long limit_ns,
                                         int arrive) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    q4d::mbar_init(q4d::smem_addr(&bar), 1);
    q4d::mbar_init_fence();
  }
  __syncthreads();
  if (threadIdx.x != 0) return;
  const uint32_t b = q4d::smem_addr(&bar);
  if (arrive) q4d::mbar_arrive(b);  // completes phase 0: the wait below succeeds at once
  const unsigned long long t0 = q4d::global_timer_ns();
  for (;;) {
    if (q4d::mbar_try_wait(b, 0u)) {
      atomicOr(word, 2u);  // the phase completed
      return;
    }
    if (q4d::global_timer_ns() - t0 > limit_ns) {
      atomicOr(word, q4d::kDevErrWaitTimeout);  // gave up: report and terminate
      return;
    }
  }
}

}  // namespace

extern "C" q4d_status q4d_wait_selftest(unsigned* word, unsigned limit_us, int arrive,
                                        void* stream) {
  if (!word || limit_us == 0 || limit_us > 10u * 1000u * 1000u) return Q4D_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(word) % 4) return Q4D_ERR_MISALIGNED;
  q4d_wait_selftest_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(
      word, 1000ull * limit_us, arrive ? 1 : 0);
  return cudaGetLastError() == cudaSuccess ? Q4D_OK : Q4D_ERR_CUDA;
}

// Self-test of the index-check record: the first n_fail of 64 threads fail a
// check (site kSiteSelftest, index base + thread), through Q4D_CHECK in a
// debug build and through the recording function itself in a release build
// (whose Q4D_CHECK is the constant true).  A check that does not return its
// condition ORs 4 into word 0.
namespace {

__global__ void q4d_index_check_selftest_kernel(unsigned* record, long long base, int n_fail) {
  const int t = threadIdx.x;
  const bool ok = t >= n_fail;
#ifdef Q4D_DEBUG
  const bool seen = Q4D_CHECK(ok, record, q4d::kSiteSelftest, base + t);
#else
  const bool seen = ok || (q4d::index_check_failed(record, q4d::kSiteSelftest, base + t), false);
#endif
  if (seen != ok) atomicOr(record, 4u);
}

}  // namespace

extern "C" q4d_status q4d_index_check_selftest(unsigned* record, long long base, int n_fail,
                                               void* stream) {
  if (!record || n_fail < 0 || n_fail > 64) return Q4D_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(record) % 4) return Q4D_ERR_MISALIGNED;
  q4d_index_check_selftest_kernel<<<1, 64, 0, static_cast<cudaStream_t>(stream)>>>(record, base,
                                                                                  n_fail);
  return cudaGetLastError() == cudaSuccess ? Q4D_OK : Q4D_ERR_CUDA;
}
