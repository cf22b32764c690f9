// kda_decode.cu — single-token recurrent decode step of KDA (HBM-streaming, sm_100a).
//
// Operation ("Kimi Linear: An Expressive, Efficient Attention Architecture", paper-graph-ui
// walkthrough, §3.4: Eq. 1 in the gradient-step form of "Online Learning Interpretation", and the
// recurrent kernel of "FLOPs Accounting and Inference Strategy"):
//     S' = Diag(alpha) S                      alpha = exp(log_alpha), per key channel (row)
//     e  = S'^T k,   p = S'^T q               two reductions over the key channels
//     u  = beta (v - e)
//     S  = S' + k u^T                         = (I - beta k k^T) Diag(alpha) S + beta k v^T
//     o  = S^T q = p + (k . q) u              so both reductions share ONE pass over S
//
// One CTA per (sequence, head); 8 warps; warp w owns rows [16w, 16w+16) of the 128 x 128 fp32
// state and lane l owns columns [4l, 4l+4), so every row is read and written as one 512-byte
// coalesced float4 transaction per warp. The state is loaded once into registers (64 floats a
// thread), reduced, updated and stored once: 2 x 64 KiB of HBM traffic per head, nothing else
// of note. Loads and stores use the streaming cache hint: the state of a decode batch is larger
// than L2 and is not reused within the step.
#include "kda_common.cuh"
#include "kda_internal.h"

namespace kda {

constexpr int kDecThreads = 256;
constexpr int kDecRowsPerWarp = 16;

template <typename Tin>
__global__ void __launch_bounds__(kDecThreads, 2)
    decode_step_kernel(const Tin* __restrict__ q, const Tin* __restrict__ k,
                       const Tin* __restrict__ v, const float* __restrict__ log_alpha,
                       const float* __restrict__ beta, float* __restrict__ state,
                       Tin* __restrict__ o, int Dk, int Dv) {
  __shared__ float s_a[128], s_k[128], s_q[128];
  __shared__ float4 s_e[8][32], s_p[8][32];
  __shared__ float s_kq[4];

  const int nh = blockIdx.x;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const size_t vec_off = (size_t)nh * Dk;

  // key-side vectors: alpha, k, q, and k . q
  float kq_part = 0.f;
  if (tid < 128) {
    float a = 1.f, kk = 0.f, qq = 0.f;
    if (tid < Dk) {
      a = expf(log_alpha[vec_off + tid]);
      kk = to_f32(k[vec_off + tid]);
      qq = to_f32(q[vec_off + tid]);
    }
    s_a[tid] = a;
    s_k[tid] = kk;
    s_q[tid] = qq;
    kq_part = kk * qq;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) kq_part += __shfl_xor_sync(0xffffffffu, kq_part, off);
    if (lane == 0) s_kq[warp] = kq_part;
  }

  // stream this thread's 16 rows x 4 columns of S into registers
  const int col = lane * 4;
  const bool col_ok = col < Dv;  // Dv is a multiple of 4
  float4* Srow = reinterpret_cast<float4*>(state + (size_t)nh * Dk * Dv) + (col >> 2);
  const int row0 = warp * kDecRowsPerWarp;
  const int vstride = Dv >> 2;
  float4 s[kDecRowsPerWarp];
#pragma unroll
  for (int i = 0; i < kDecRowsPerWarp; ++i) {
    const int r = row0 + i;
    s[i] = (col_ok && r < Dk) ? __ldcs(Srow + (size_t)r * vstride) : make_float4(0.f, 0.f, 0.f, 0.f);
  }
  __syncthreads();

  // decay and partial reductions over this warp's rows
  float4 e = make_float4(0.f, 0.f, 0.f, 0.f), p = e;
#pragma unroll
  for (int i = 0; i < kDecRowsPerWarp; ++i) {
    const int r = row0 + i;
    const float a = s_a[r], kr = s_k[r], qr = s_q[r];  // rows >= Dk hold a=1, k=q=0
    s[i].x *= a;
    s[i].y *= a;
    s[i].z *= a;
    s[i].w *= a;
    e.x += s[i].x * kr;
    e.y += s[i].y * kr;
    e.z += s[i].z * kr;
    e.w += s[i].w * kr;
    p.x += s[i].x * qr;
    p.y += s[i].y * qr;
    p.z += s[i].z * qr;
    p.w += s[i].w * qr;
  }
  s_e[warp][lane] = e;
  s_p[warp][lane] = p;
  __syncthreads();
  e = make_float4(0.f, 0.f, 0.f, 0.f);
  p = e;
#pragma unroll
  for (int w = 0; w < 8; ++w) {
    const float4 ew = s_e[w][lane], pw = s_p[w][lane];
    e.x += ew.x;
    e.y += ew.y;
    e.z += ew.z;
    e.w += ew.w;
    p.x += pw.x;
    p.y += pw.y;
    p.z += pw.z;
    p.w += pw.w;
  }

  // u = beta (v - e)
  const float b = beta[nh];
  float4 u = make_float4(0.f, 0.f, 0.f, 0.f);
  if (col_ok) {
    const Tin* vp = v + (size_t)nh * Dv + col;
    u.x = b * (to_f32(vp[0]) - e.x);
    u.y = b * (to_f32(vp[1]) - e.y);
    u.z = b * (to_f32(vp[2]) - e.z);
    u.w = b * (to_f32(vp[3]) - e.w);
  }

  // S = S' + k u^T, streamed back
#pragma unroll
  for (int i = 0; i < kDecRowsPerWarp; ++i) {
    const int r = row0 + i;
    if (col_ok && r < Dk) {
      const float kr = s_k[r];
      float4 t = s[i];
      t.x += kr * u.x;
      t.y += kr * u.y;
      t.z += kr * u.z;
      t.w += kr * u.w;
      __stcs(Srow + (size_t)r * vstride, t);
    }
  }

  // o = p + (k . q) u
  if (warp == 0 && col_ok) {
    const float kq = s_kq[0] + s_kq[1] + s_kq[2] + s_kq[3];
    Tin* op = o + (size_t)nh * Dv + col;
    op[0] = from_f32<Tin>(p.x + kq * u.x);
    op[1] = from_f32<Tin>(p.y + kq * u.y);
    op[2] = from_f32<Tin>(p.z + kq * u.z);
    op[3] = from_f32<Tin>(p.w + kq * u.w);
  }
}

cudaError_t launch_decode_step(const void* q, const void* k, const void* v, kda_dtype_t dt,
                               const float* log_alpha, const float* beta, float* state, void* o,
                               int N, int H, int Dk, int Dv, cudaStream_t stream) {
  const long long heads = (long long)N * H;
  if (heads == 0) return cudaSuccess;
  dim3 grid((unsigned)heads), block(kDecThreads);
  ProfileScope prof("decode_step", stream);
  if (dt == KDA_DTYPE_BF16) {
    decode_step_kernel<__nv_bfloat16><<<grid, block, 0, stream>>>(
        (const __nv_bfloat16*)q, (const __nv_bfloat16*)k, (const __nv_bfloat16*)v, log_alpha, beta,
        state, (__nv_bfloat16*)o, Dk, Dv);
  } else {
    decode_step_kernel<float><<<grid, block, 0, stream>>>((const float*)q, (const float*)k,
                                                          (const float*)v, log_alpha, beta, state,
                                                          (float*)o, Dk, Dv);
  }
  return cudaGetLastError();
}

}  // namespace kda
