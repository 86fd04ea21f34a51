// Self-test of the bounded waits: a kernel whose mbarriers nothing ever
// arrives at, so that every wait in it runs out.  It exercises the three wait
// forms the library's kernels use (one thread with mbar_wait, one thread with
// the shared give-up flag, a whole warp with the warp-uniform form) and
// records, in the library's device error word and in a caller's word, which
// of them gave up.  Each wait ends by its own limit (about a second), so the
// kernel always returns and the context stays usable.

#include <cuda_runtime.h>

#include "rbq.h"
#include "rbq_internal.h"
#include "rbq_sm100.cuh"

namespace rbq {
namespace {

using namespace sm100;

// Bits of the caller's word: which waits returned false.
constexpr unsigned kSingle = 1u;      // warp 0, lane 0: mbar_wait
constexpr unsigned kShared = 2u;      // warp 1, lane 0: mbar_wait_or_abort
constexpr unsigned kWarp = 4u;        // warp 2, all lanes: mbar_warp_wait
constexpr unsigned kAbortSeen = 8u;   // the shared give-up flag was raised
constexpr unsigned kErrBit = 1u << 12;  // device error word bit for this kernel

__global__ void __launch_bounds__(96, 1) wait_limit_kernel(unsigned int* err, unsigned int* out) {
  __shared__ __align__(8) uint64_t bar[3];
  __shared__ volatile uint32_t abort_flag;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int i = 0; i < 3; ++i) mbar_init(&bar[i], 1);
    abort_flag = 0u;
    mbar_fence_init();
  }
  __syncthreads();
  unsigned gave_up = 0;
  if (warp == 0) {
    if (lane == 0 && !mbar_wait(&bar[0], 0)) gave_up = kSingle;
  } else if (warp == 1) {
    if (lane == 0 && !mbar_wait_or_abort(&bar[1], 0, &abort_flag)) gave_up = kShared;
  } else {
    if (!mbar_warp_wait(&bar[2], 0, &abort_flag) && lane == 0) gave_up = kWarp;
  }
  if (gave_up) {
    atomicOr(out, gave_up);
    atomicOr(err, kErrBit);
  }
  __syncthreads();
  if (threadIdx.x == 0 && abort_flag) atomicOr(out, kAbortSeen);
}

}  // namespace
}  // namespace rbq

extern "C" int rbq_selftest_wait_limit(unsigned int* out, void* stream) {
  if (!out) return RBQ_EINVAL;
  if (reinterpret_cast<uintptr_t>(out) % alignof(unsigned int)) return RBQ_EALIGN;
  unsigned int* err = nullptr;
  int rc = rbq::device_error_word_ptr(&err);
  if (rc != RBQ_OK) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaMemsetAsync(out, 0, sizeof(unsigned int), st);
  if (e != cudaSuccess) return rbq::cuda_fail(e);
  rbq::wait_limit_kernel<<<1, 96, 0, st>>>(err, out);
  e = cudaGetLastError();
  if (e != cudaSuccess) return rbq::cuda_fail(e);
  return RBQ_OK;
}
