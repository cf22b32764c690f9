// kda_epilogue.cu — the output epilogue (head-wise RMSNorm x sigmoid gate) as a pass of its own,
// for the fp32 CUDA-core prefill path. The bf16 tensor-core path and the recurrent kernels apply
// the same epilogue inside their output stores.
//
// "Kimi Linear: An Expressive, Efficient Attention Architecture" (paper-graph-ui walkthrough,
// §3.4 "Neural Parameterization", the output-gate equation): every (token, head) row o of the
// operator's output becomes sigmoid(gate) * weight * o / sqrt(mean(o^2) + eps).
#include "kda_common.cuh"
#include "kda_internal.h"

namespace kda {

constexpr int kEpiRowsPerBlock = 8;  // one warp per row

template <typename T>
__global__ void __launch_bounds__(32 * kEpiRowsPerBlock)
    output_norm_gate_kernel(T* __restrict__ o, const T* __restrict__ gate,
                            const float* __restrict__ weight, float eps, long long rows, int H,
                            int Dv, const int32_t* __restrict__ cu_end) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long row = (long long)blockIdx.x * kEpiRowsPerBlock + warp;
  // varlen: tokens past the last sequence end are not the operator's output
  const long long limit = (cu_end KDA_AND_IN_BOUNDS(kBufCuSeqlens, cu_end, 4))
                              ? min(rows, (long long)(*cu_end) * H)
                              : rows;
  if (row >= limit) return;
  T* orow = o + row * Dv;
#ifdef KDA_BOUNDS_CHECK
  if (!(in_bounds(kBufO, orow, Dv * sizeof(T)) &&
        (!gate || in_bounds(kBufGate, gate + row * Dv, Dv * sizeof(T))) &&
        (!weight || in_bounds(kBufNormW, weight, Dv * 4ull))))
    return;  // (uniform in the warp that owns the row)
#endif
  float x[4];
  float ss = 0.f;
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const int c = lane + 32 * j;
    x[j] = c < Dv ? to_f32(orow[c]) : 0.f;
    ss += x[j] * x[j];
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
  const float inv = rsqrtf(ss / (float)Dv + eps);
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const int c = lane + 32 * j;
    if (c >= Dv) continue;
    float y = x[j] * inv;
    if (weight) y *= weight[c];
    if (gate) y *= sigmoid_f(to_f32(gate[row * Dv + c]));
    orow[c] = from_f32<T>(y);
  }
}

cudaError_t launch_output_norm_gate(void* o, kda_dtype_t dt, const Fusion& fz, long long rows,
                                    int H, int Dv, const int32_t* cu_end, cudaStream_t stream) {
  if (rows <= 0) return cudaSuccess;
  const unsigned blocks = (unsigned)((rows + kEpiRowsPerBlock - 1) / kEpiRowsPerBlock);
  ProfileScope prof("output_norm_gate", stream);
  if (dt == KDA_DTYPE_BF16)
    output_norm_gate_kernel<__nv_bfloat16><<<blocks, 32 * kEpiRowsPerBlock, 0, stream>>>(
        (__nv_bfloat16*)o, (const __nv_bfloat16*)fz.og, fz.ow, fz.oeps, rows, H, Dv, cu_end);
  else
    output_norm_gate_kernel<float><<<blocks, 32 * kEpiRowsPerBlock, 0, stream>>>(
        (float*)o, (const float*)fz.og, fz.ow, fz.oeps, rows, H, Dv, cu_end);
  return cudaGetLastError();
}

}  // namespace kda
