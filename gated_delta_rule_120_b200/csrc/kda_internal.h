// kda_internal.h — host-side declarations shared by the C-ABI layer and the kernel files.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "kda.h"

namespace kda {

struct SeqGeometry;

// RAII bracket of one kernel launch for kda_profile_* (no-op unless profiling is enabled).
class ProfileScope {
 public:
  ProfileScope(const char* name, cudaStream_t stream);
  ~ProfileScope();
  ProfileScope(const ProfileScope&) = delete;
  ProfileScope& operator=(const ProfileScope&) = delete;

 private:
  const char* name_;
  cudaStream_t stream_;
  cudaEvent_t start_ = nullptr, stop_ = nullptr;
  bool active_ = false;
};

// Prologue fusion (see kda_fusion_t): in-kernel q/k L2 normalisation and the log-space gate.
struct Fusion {
  int l2 = 0;
  float eps = 0.f;
  const float* A_log = nullptr;    // [H]; non-null: the decay input is the raw gate
  const float* dt_bias = nullptr;  // [H, Dk] or null
  int onorm = 0;                   // output epilogue: head-wise RMSNorm x sigmoid gate
  float oeps = 0.f;
  const float* ow = nullptr;       // [Dv] norm weight or null (ones)
  const void* og = nullptr;        // gate in o's layout and dtype, or null
};

// Arguments of one kda_chunk_fwd call after host validation.
struct PrefillArgs {
  const void* q;
  const void* k;
  const void* v;
  kda_dtype_t dtype;
  const float* log_alpha;
  const float* beta;
  const float* initial_state;
  const int32_t* cu_seqlens;
  int N, B, T, H, Dk, Dv, C;
  void* o;
  float* final_state;
  Fusion fz;
};

// Per (chunk, head) record of the fp32 CUDA-core path, in floats:
//   W [C][Dk], U [C][Dv], Kt [C][Dk], Qt [C][Dk], A_qk [C][C], gamma_C [Dk]
//   (+ for the backward pass: T = (I + A_kk)^{-1} [C][C] and the strictly lower
//    B[r][i] = sum_c k_r[c] k_i[c] gamma_r[c]/gamma_i[c] [C][C], i.e. A_kk without Diag(beta))
struct SimtRecord {
  static constexpr size_t kNone = ~(size_t)0;
  size_t record_floats;
  size_t off_w, off_u, off_kt, off_qt, off_aqk, off_gam;
  size_t off_t = kNone, off_b = kNone;

  static SimtRecord make(int C, int Dk, int Dv, bool for_backward = false) {
    SimtRecord r;
    size_t o = 0;
    if (for_backward) {
      r.off_t = o;
      o += (size_t)C * C;
      r.off_b = o;
      o += (size_t)C * C;
    }
    r.off_w = o;
    o += (size_t)C * Dk;
    r.off_u = o;
    o += (size_t)C * Dv;
    r.off_kt = o;
    o += (size_t)C * Dk;
    r.off_qt = o;
    o += (size_t)C * Dk;
    r.off_aqk = o;
    o += (size_t)C * C;
    r.off_gam = o;
    o += (size_t)Dk;
    r.record_floats = (o + 63) / 64 * 64;  // 256-byte records
    return r;
  }
};

// bytes of one (chunk, head) record of the bf16 tensor-core path (d = 128, C = 64)
constexpr size_t TcRecordBytes = 74240;

// Bounds-checked build: the call's buffer extents into the device table, on `stream` (a no-op
// returning cudaSuccess in the normal build).
struct BoundsTable;
cudaError_t register_bounds(const BoundsTable& t, cudaStream_t stream);

cudaError_t launch_prefill_tc(const PrefillArgs& a, const SeqGeometry& geo, int max_chunks,
                              uint8_t* records, cudaStream_t stream);
size_t tc_local_smem_bytes();
size_t tc_state_smem_bytes();

cudaError_t launch_decode_step(const void* q, const void* k, const void* v, kda_dtype_t dt,
                               const float* log_alpha, const float* beta, float* state, void* o,
                               int N, int H, int Dk, int Dv, const Fusion* fz,
                               cudaStream_t stream);

cudaError_t launch_recurrent_multi(const void* q, const void* k, const void* v, kda_dtype_t dt,
                                   const float* log_alpha, const float* beta, float* pool,
                                   const int32_t* idx, void* o, int N, int T, int H, int Dk,
                                   int Dv, int P, const Fusion& fz, cudaStream_t stream);

cudaError_t launch_chunk_map(const int32_t* cu, int N, int total, int C, int32_t* chunk_off,
                             int32_t* valid, int32_t* order, cudaStream_t stream);

cudaError_t launch_prefill_simt(const PrefillArgs& a, const SeqGeometry& geo, int max_chunks,
                                float* records, const SimtRecord& rec, cudaStream_t stream);

// The fp32 chunk kernels run for the backward pass: records with T and B, and the state at the
// start of every chunk (states [chunks, H, Dk, Dv]) instead of the output.
cudaError_t launch_forward_for_backward(const PrefillArgs& a, const SeqGeometry& geo,
                                        int max_chunks, float* records, const SimtRecord& rec,
                                        float* states, cudaStream_t stream);

// Arguments of one kda_chunk_bwd call after host validation.
struct BackwardArgs {
  PrefillArgs fwd;          // inputs, geometry sizes; fwd.o unused, fwd.C = backward chunk
  const void* d_o;          // [B,T,H,Dv], input dtype
  const float* d_final;     // [N,H,Dk,Dv] or null
  void* dq;                 // [B,T,H,Dk], input dtype
  void* dk;
  void* dv;                 // [B,T,H,Dv]
  float* dlog_alpha;        // [B,T,H,Dk]
  float* dbeta;             // [B,T,H]
  float* d_initial;         // [N,H,Dk,Dv] or null
};
cudaError_t launch_chunk_bwd(const BackwardArgs& b, const SeqGeometry& geo, int max_chunks,
                             float* records, const SimtRecord& rec, float* states,
                             float* dstates, float* dvp, cudaStream_t stream);

size_t simt_local_smem_bytes(int C, int Dk, int Dv);

// The output epilogue as its own in-place pass over o (rows = token-head pairs); cu_end (device,
// may be null) bounds the rows to cu_seqlens[N] * H.
cudaError_t launch_output_norm_gate(void* o, kda_dtype_t dt, const Fusion& fz, long long rows,
                                    int H, int Dv, const int32_t* cu_end, cudaStream_t stream);
size_t simt_state_smem_bytes(int C, int Dk);

}  // namespace kda
