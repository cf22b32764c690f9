// kda_selftest.cu — self-tests of the failure detection (include/kda_selftest.h).
//
// Bounded waits: one block waits on an mbarrier phase that nothing completes, through the same
// bounded wait (sm100::mbar_wait) that every pipeline of the library uses; the wait gives up after
// its limit, sets the timeout bit of the status word and the block exits. Bounds checks (the
// bounds-checked build only): one thread tests an access just past a registered extent with the
// kernels' own check, which skips the access and sets the bounds bit. Nothing faults, traps or
// spins without a bound.
#include "kda_selftest.h"

#include "kda_common.cuh"
#include "kda_internal.h"
#include "kda_sm100.cuh"

namespace kda {

__global__ void selftest_wait_kernel(uint64_t limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    sm100::mbar_init(&bar, 1);
    sm100::fence_mbar_init();
  }
  __syncthreads();
  // no thread ever arrives on `bar`: its phase 0 cannot complete
  if (threadIdx.x == 0) sm100::mbar_wait(&bar, 0, limit_ns);
}

// tests, without performing it, an access of 4 bytes at `base + offset` against the extent of
// role kBufO
__global__ void selftest_bounds_kernel(const char* base, unsigned long long offset) {
  if (threadIdx.x == 0) (void)KDA_IN_BOUNDS(kBufO, base + offset, 4);
}

}  // namespace kda

extern "C" {

kda_status_t kda_selftest_wait_timeout(uint64_t limit_ns, kda_stream_t stream) {
  if (limit_ns < 1 || limit_ns > 1000000000ull) return KDA_ERR_INVALID_ARG;
  kda::selftest_wait_kernel<<<1, 32, 0, (cudaStream_t)stream>>>(limit_ns);
  return cudaGetLastError() == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
}

kda_status_t kda_selftest_bounds(const void* buffer, size_t bytes, kda_stream_t stream_) {
  if (!kda::kBoundsChecked) return KDA_ERR_UNSUPPORTED;
  if (!buffer || bytes == 0) return KDA_ERR_INVALID_ARG;
  cudaStream_t stream = (cudaStream_t)stream_;
  kda::BoundsTable t = {};
  t.base[kda::kBufO] = buffer;
  t.bytes[kda::kBufO] = bytes;
  if (kda::register_bounds(t, stream) != cudaSuccess) return KDA_ERR_CUDA;
  kda::selftest_bounds_kernel<<<1, 32, 0, stream>>>(static_cast<const char*>(buffer),
                                                    (unsigned long long)bytes);
  return cudaGetLastError() == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
}

}  // extern "C"