// kda_noalloc.cu — kda_chunk_fwd_noalloc: chunkwise prefill with library-owned scratch.
//
// For callers that cannot give the library a workspace (their framework owns all device memory,
// or they avoid cudaMalloc/cudaFree on a latency-critical path), the prefill scratch lives in a
// file-scope device array. Host code cannot use the array's name as a device address, so the
// address is looked up once per device with cudaGetSymbolAddress and cached. No allocating call
// is made. Calls on one device share the array; overlapping calls race (see include/kda.h).
#include <mutex>

#include "kda_internal.h"

namespace kda {

static __device__ __align__(256) unsigned char g_noalloc_scratch[KDA_NOALLOC_SCRATCH_BYTES];

namespace {
constexpr int kNoallocMaxDevices = 64;
std::mutex g_noalloc_mu;
void* g_noalloc_addr[kNoallocMaxDevices] = {};

// Device address of g_noalloc_scratch on the current device (set-up on first use).
kda_status_t noalloc_scratch(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return KDA_ERR_CUDA;
  if (dev < 0 || dev >= kNoallocMaxDevices) return KDA_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (g_noalloc_addr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr)
      return KDA_ERR_CUDA;
    g_noalloc_addr[dev] = p;
  }
  *out = g_noalloc_addr[dev];
  return KDA_OK;
}
}  // namespace

}  // namespace kda

extern "C" kda_status_t kda_chunk_fwd_noalloc(const void* q, const void* k, const void* v,
                                              kda_dtype_t dt, const float* log_alpha,
                                              const float* beta, const float* initial_state,
                                              const int32_t* cu_seqlens, int32_t N, int32_t B,
                                              int32_t T, int32_t H, int32_t Dk, int32_t Dv,
                                              int32_t C, void* o, float* final_state,
                                              kda_stream_t stream) {
  void* scratch = nullptr;
  const kda_status_t st = kda::noalloc_scratch(&scratch);
  if (st != KDA_OK) return st;
  // kda_chunk_fwd rejects, with KDA_ERR_WORKSPACE and before any launch, a call that needs more
  // than the array holds.
  return kda_chunk_fwd(q, k, v, dt, log_alpha, beta, initial_state, cu_seqlens, N, B, T, H, Dk,
                       Dv, C, o, final_state, scratch, KDA_NOALLOC_SCRATCH_BYTES, stream);
}
