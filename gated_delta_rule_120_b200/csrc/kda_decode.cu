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
#include <atomic>

#include "kda_common.cuh"
#include "kda_internal.h"
#include "kda_sm100.cuh"

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

// ---------------------------------------------------------------------------------------------
// Multi-token recurrent variant: one CTA per (sequence, head) applies T tokens to a state that
// stays in registers (same thread layout as above); the next token's vectors are fetched while
// the current one is processed. Two block-wide barriers per token (cross-warp reductions).
// ---------------------------------------------------------------------------------------------
template <typename Tin>
__global__ void __launch_bounds__(kDecThreads, 2)
    recurrent_multi_kernel(const Tin* __restrict__ q, const Tin* __restrict__ k,
                           const Tin* __restrict__ v, const float* __restrict__ log_alpha,
                           const float* __restrict__ beta, float* __restrict__ pool,
                           const int32_t* __restrict__ state_indices, Tin* __restrict__ o, int T,
                           int H, int Dk, int Dv, int P, Fusion fz) {
  __shared__ float s_a[128], s_k[128], s_q[128];
  __shared__ float4 s_e[8][32], s_p[8][32];
  __shared__ float s_kq[4], s_ssk[4], s_ssq[4];

  const int nh = blockIdx.x;
  const int n = nh / H, h = nh - n * H;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  int slot = state_indices ? state_indices[n] : n;
  if (slot < 0) return;  // padding entry of the batch
  if (slot >= P) {
    if (tid == 0) raise_status(kStatusBadSeqlens);
    return;
  }

  const int col = lane * 4;
  const bool col_ok = col < Dv;
  float4* Srow = reinterpret_cast<float4*>(pool + ((size_t)slot * H + h) * Dk * Dv) + (col >> 2);
  const int row0 = warp * kDecRowsPerWarp;
  const int vstride = Dv >> 2;
  float4 s[kDecRowsPerWarp];
#pragma unroll
  for (int i = 0; i < kDecRowsPerWarp; ++i) {
    const int r = row0 + i;
    s[i] = (col_ok && r < Dk) ? Srow[(size_t)r * vstride] : make_float4(0.f, 0.f, 0.f, 0.f);
  }

  // per-token vectors: threads 0..127 hold one key channel, lanes hold 4 value columns
  auto vec_base = [&](int t) { return (((size_t)n * T + t) * H + h); };
  float la_n = 0.f, k_n = 0.f, q_n = 0.f, b_n = 0.f;
  float4 v_n = make_float4(0.f, 0.f, 0.f, 0.f);
  const float neg_a = fz.A_log ? -expf(fz.A_log[h]) : 0.f;
  const float bias_c = (fz.A_log && fz.dt_bias && tid < Dk) ? fz.dt_bias[h * Dk + tid] : 0.f;
  auto fetch = [&](int t) {
    const size_t base = vec_base(t);
    if (tid < Dk) {
      la_n = log_alpha[base * Dk + tid];
      if (fz.A_log) la_n = neg_a * softplus_f(la_n + bias_c);  // fused gate
      k_n = to_f32(k[base * Dk + tid]);
      q_n = to_f32(q[base * Dk + tid]);
    }
    if (col_ok) {
      const Tin* vp = v + base * Dv + col;
      v_n = make_float4(to_f32(vp[0]), to_f32(vp[1]), to_f32(vp[2]), to_f32(vp[3]));
    }
    b_n = beta[base];
  };
  if (T > 0) fetch(0);
  for (int t = 0; t < T; ++t) {
    const float la_c = la_n, k_c = k_n, q_c = q_n, b = b_n;
    const float4 vc = v_n;
    if (tid < 128) {
      const bool in = tid < Dk;
      s_a[tid] = in ? expf(la_c) : 1.f;
      s_k[tid] = in ? k_c : 0.f;
      s_q[tid] = in ? q_c : 0.f;
      float kq = in ? k_c * q_c : 0.f;
      float ssk = in ? k_c * k_c : 0.f, ssq = in ? q_c * q_c : 0.f;
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) {
        kq += __shfl_xor_sync(0xffffffffu, kq, off);
        ssk += __shfl_xor_sync(0xffffffffu, ssk, off);
        ssq += __shfl_xor_sync(0xffffffffu, ssq, off);
      }
      if (lane == 0) {
        s_kq[warp] = kq;
        s_ssk[warp] = ssk;
        s_ssq[warp] = ssq;
      }
    }
    if (t + 1 < T) fetch(t + 1);  // in flight while this token is processed
    __syncthreads();
    float4 e = make_float4(0.f, 0.f, 0.f, 0.f), p = e;
#pragma unroll
    for (int i = 0; i < kDecRowsPerWarp; ++i) {
      const int r = row0 + i;
      const float a = s_a[r], kr = s_k[r], qr = s_q[r];
      s[i].x *= a; s[i].y *= a; s[i].z *= a; s[i].w *= a;
      e.x += s[i].x * kr; e.y += s[i].y * kr; e.z += s[i].z * kr; e.w += s[i].w * kr;
      p.x += s[i].x * qr; p.y += s[i].y * qr; p.z += s[i].z * qr; p.w += s[i].w * qr;
    }
    s_e[warp][lane] = e;
    s_p[warp][lane] = p;
    __syncthreads();
    e = make_float4(0.f, 0.f, 0.f, 0.f);
    p = e;
#pragma unroll
    for (int w = 0; w < 8; ++w) {
      const float4 ew = s_e[w][lane], pw = s_p[w][lane];
      e.x += ew.x; e.y += ew.y; e.z += ew.z; e.w += ew.w;
      p.x += pw.x; p.y += pw.y; p.z += pw.z; p.w += pw.w;
    }
    float kq = s_kq[0] + s_kq[1] + s_kq[2] + s_kq[3];
    float ik = 1.f;
    if (fz.l2) {  // fused L2 norm, applied to the reductions rather than to the state pass
      ik = rsqrtf(s_ssk[0] + s_ssk[1] + s_ssk[2] + s_ssk[3] + fz.eps);
      const float iq = rsqrtf(s_ssq[0] + s_ssq[1] + s_ssq[2] + s_ssq[3] + fz.eps);
      e.x *= ik; e.y *= ik; e.z *= ik; e.w *= ik;
      p.x *= iq; p.y *= iq; p.z *= iq; p.w *= iq;
      kq *= ik * iq;
    }
    float4 u = make_float4(0.f, 0.f, 0.f, 0.f);
    if (col_ok) {
      u.x = b * (vc.x - e.x); u.y = b * (vc.y - e.y); u.z = b * (vc.z - e.z); u.w = b * (vc.w - e.w);
    }
#pragma unroll
    for (int i = 0; i < kDecRowsPerWarp; ++i) {
      const float kr = s_k[row0 + i] * ik;
      s[i].x += kr * u.x; s[i].y += kr * u.y; s[i].z += kr * u.z; s[i].w += kr * u.w;
    }
    if (warp == 0) {
      float4 y = make_float4(p.x + kq * u.x, p.y + kq * u.y, p.z + kq * u.z, p.w + kq * u.w);
      if (fz.onorm) {  // output epilogue: head-wise RMSNorm x sigmoid gate over the Dv columns
        float ss = col_ok ? y.x * y.x + y.y * y.y + y.z * y.z + y.w * y.w : 0.f;
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
        const float inv = rsqrtf(ss / (float)Dv + fz.oeps);
        if (col_ok) {
          float4 wv = (fz.ow && KDA_IN_BOUNDS(kBufNormW, fz.ow + col, 16))
                          ? *reinterpret_cast<const float4*>(fz.ow + col)
                            : make_float4(1.f, 1.f, 1.f, 1.f);
          if (fz.og) {
            const Tin* gp = reinterpret_cast<const Tin*>(fz.og) + vec_base(t) * Dv + col;
            wv.x *= sigmoid_f(to_f32(gp[0]));
            wv.y *= sigmoid_f(to_f32(gp[1]));
            wv.z *= sigmoid_f(to_f32(gp[2]));
            wv.w *= sigmoid_f(to_f32(gp[3]));
          }
          y = make_float4(y.x * inv * wv.x, y.y * inv * wv.y, y.z * inv * wv.z, y.w * inv * wv.w);
        }
      }
      if (col_ok) {
        Tin* op = o + vec_base(t) * Dv + col;
        op[0] = from_f32<Tin>(y.x);
        op[1] = from_f32<Tin>(y.y);
        op[2] = from_f32<Tin>(y.z);
        op[3] = from_f32<Tin>(y.w);
      }
    }
    __syncthreads();  // s_a / s_k / s_q / s_e / s_p are rewritten by the next token
  }
#pragma unroll
  for (int i = 0; i < kDecRowsPerWarp; ++i) {
    const int r = row0 + i;
    if (col_ok && r < Dk) Srow[(size_t)r * vstride] = s[i];
  }
}

static cudaError_t launch_recurrent_blockwise(const void* q, const void* k, const void* v,
                                              kda_dtype_t dt, const float* log_alpha,
                                              const float* beta, float* pool, const int32_t* idx,
                                              void* o, int N, int T, int H, int Dk, int Dv, int P,
                                              const Fusion& fz, cudaStream_t stream) {
  const long long heads = (long long)N * H;
  if (heads == 0 || T == 0) return cudaSuccess;
  ProfileScope prof("recurrent_multi", stream);
  if (dt == KDA_DTYPE_BF16)
    recurrent_multi_kernel<__nv_bfloat16><<<(unsigned)heads, kDecThreads, 0, stream>>>(
        (const __nv_bfloat16*)q, (const __nv_bfloat16*)k, (const __nv_bfloat16*)v, log_alpha, beta,
        pool, idx, (__nv_bfloat16*)o, T, H, Dk, Dv, P, fz);
  else
    recurrent_multi_kernel<float><<<(unsigned)heads, kDecThreads, 0, stream>>>(
        (const float*)q, (const float*)k, (const float*)v, log_alpha, beta, pool, idx, (float*)o,
        T, H, Dk, Dv, P, fz);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------------------------
// Streaming variant (used whenever the per-head vectors allow 16-byte bulk copies): one
// persistent CTA per SM walks its heads through a three-stage shared-memory ring. A producer warp
// bulk-loads a head's whole state plus its q, k, v and log-decay vectors ahead of use and bulk-
// stores the updated state back, so HBM reads of later heads overlap the compute and the write
// of earlier ones; eight compute warps do the same one-pass update as above on the staged copy.
// ---------------------------------------------------------------------------------------------
constexpr int kDsStages = 3;
constexpr int kDsCompute = 256;                // 8 compute warps
constexpr int kDsThreads = kDsCompute + 32;    // + producer warp

struct DsLayout {
  uint32_t state_bytes, la_off, q_off, k_off, v_off, stage_bytes, vec_tx;
  uint32_t og_off, bias_off;  // fused step: output gate row and the head's dt_bias row
  uint32_t og_bytes, bias_bytes;  // 0 when the fused step has no such input
};

__host__ __device__ inline uint32_t align16u(uint32_t x) { return (x + 15u) & ~15u; }

static DsLayout make_ds_layout(int Dk, int Dv, int es, bool gate_row = false,
                               bool bias_row = false) {
  DsLayout L;
  L.state_bytes = (uint32_t)Dk * Dv * 4;
  L.la_off = L.state_bytes;
  L.q_off = L.la_off + align16u((uint32_t)Dk * 4);
  L.k_off = L.q_off + align16u((uint32_t)Dk * es);
  L.v_off = L.k_off + align16u((uint32_t)Dk * es);
  L.og_off = L.v_off + align16u((uint32_t)Dv * es);
  L.og_bytes = gate_row ? (uint32_t)Dv * es : 0u;
  L.bias_off = L.og_off + align16u(L.og_bytes);
  L.bias_bytes = bias_row ? (uint32_t)Dk * 4 : 0u;
  L.stage_bytes = (L.bias_off + align16u(L.bias_bytes) + 127u) & ~127u;
  L.vec_tx = (uint32_t)Dk * 4 + 2u * Dk * es + (uint32_t)Dv * es + L.og_bytes + L.bias_bytes;
  return L;
}

__device__ __forceinline__ bool block_all(bool pred, uint32_t bar_id, uint32_t nthreads) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.and.pred q, %2, %3, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)pred), "r"(bar_id), "r"(nthreads)
      : "memory");
  return r != 0;
}

// kFused: the prologue and epilogue of kda_fusion_t (log_alpha holds the raw gate when A_log is
// given; q and k normalised through the reductions; output RMSNorm x sigmoid gate in warp 0).
template <typename Tin, bool kFused>
__global__ void __launch_bounds__(kDsThreads, 1)
    decode_stream_kernel(const Tin* __restrict__ q, const Tin* __restrict__ k,
                         const Tin* __restrict__ v, const float* __restrict__ log_alpha,
                         const float* __restrict__ beta, float* __restrict__ state,
                         Tin* __restrict__ o, int NH, int Dk, int Dv, DsLayout lay, int H,
                         Fusion fz) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = smem_raw + ((128 - (sm100::smem_u32(smem_raw) & 127)) & 127);
  uint8_t* stages = sm;
  float4* s_e = reinterpret_cast<float4*>(sm + kDsStages * lay.stage_bytes);  // [8][32]
  float4* s_p = s_e + 8 * 32;                                                 // [8][32]
  float* s_kq = reinterpret_cast<float*>(s_p + 8 * 32);                        // [8]
  float* s_ss = s_kq + 8;                                                      // [2][8] (fused)
  uint64_t* full = reinterpret_cast<uint64_t*>(s_kq + 24);                     // [kDsStages]
  uint64_t* computed = full + kDsStages;                                       // [kDsStages]

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int first = blockIdx.x, stride = gridDim.x;
  const int count = first < NH ? (NH - first + stride - 1) / stride : 0;
  const uint32_t es = sizeof(Tin);

  if (tid == 0) {
    for (int i = 0; i < kDsStages; ++i) {
      sm100::mbar_init(full + i, 1);
      sm100::mbar_init(computed + i, 1);
    }
    sm100::fence_mbar_init();
  }
  __syncthreads();

  if (warp == kDsCompute / 32) {
    // ---------------------------------------------------------------- producer warp
    if (lane == 0) {
      auto issue_load = [&](int it) {
        const int s = it % kDsStages;
        const size_t head = (size_t)first + (size_t)it * stride;
        uint8_t* st = stages + (size_t)s * lay.stage_bytes;
        if (kBoundsChecked &&
            !(KDA_IN_BOUNDS(kBufState, state + head * Dk * Dv, lay.state_bytes) &&
              KDA_IN_BOUNDS(kBufLogAlpha, log_alpha + head * Dk, Dk * 4ull) &&
              KDA_IN_BOUNDS(kBufQ, q + head * Dk, (size_t)Dk * es) &&
              KDA_IN_BOUNDS(kBufK, k + head * Dk, (size_t)Dk * es) &&
              KDA_IN_BOUNDS(kBufV, v + head * Dv, (size_t)Dv * es) &&
              (!(kFused && lay.og_bytes) ||
               KDA_IN_BOUNDS(kBufGate, reinterpret_cast<const Tin*>(fz.og) + head * Dv,
                             lay.og_bytes)) &&
              (!(kFused && lay.bias_bytes) ||
               KDA_IN_BOUNDS(kBufDtBias, fz.dt_bias + (head % (size_t)H) * Dk,
                             lay.bias_bytes)))) {
          sm100::mbar_arrive(full + s);  // nothing copied: the phase completes on a stale stage
          return;
        }
        sm100::mbar_arrive_expect_tx(full + s, lay.state_bytes + lay.vec_tx);
        sm100::bulk_g2s(st, state + head * Dk * Dv, lay.state_bytes, full + s);
        sm100::bulk_g2s(st + lay.la_off, log_alpha + head * Dk, Dk * 4, full + s);
        sm100::bulk_g2s(st + lay.q_off, q + head * Dk, Dk * es, full + s);
        sm100::bulk_g2s(st + lay.k_off, k + head * Dk, Dk * es, full + s);
        sm100::bulk_g2s(st + lay.v_off, v + head * Dv, Dv * es, full + s);
        if (kFused && lay.og_bytes)
          sm100::bulk_g2s(st + lay.og_off, reinterpret_cast<const Tin*>(fz.og) + head * Dv,
                          lay.og_bytes, full + s);
        if (kFused && lay.bias_bytes)
          sm100::bulk_g2s(st + lay.bias_off, fz.dt_bias + (head % (size_t)H) * Dk,
                          lay.bias_bytes, full + s);
      };
      for (int it = 0; it < count && it < kDsStages; ++it) issue_load(it);
      for (int it = 0; it < count; ++it) {
        const int s = it % kDsStages;
        if (!sm100::mbar_wait(computed + s, (it / kDsStages) & 1)) break;
        const size_t head = (size_t)first + (size_t)it * stride;
        if (KDA_IN_BOUNDS(kBufState, state + head * Dk * Dv, lay.state_bytes)) {
          sm100::bulk_s2g(state + head * Dk * Dv, stages + (size_t)s * lay.stage_bytes,
                          lay.state_bytes);
          sm100::bulk_commit();
        }
        if (it + kDsStages < count) {
          sm100::bulk_wait_read_all();  // the stage is free once its store has read it
          issue_load(it + kDsStages);
        }
      }
      sm100::bulk_wait_all();
      // loads that were issued but never consumed (only after a timeout) must land first
      for (int it = 0; it < count && it < kDsStages; ++it) {
        const int last = count - 1 - it;
        if (last >= 0) sm100::mbar_wait(full + last % kDsStages, (last / kDsStages) & 1, 100000000ull);
      }
    }
  } else {
    // ---------------------------------------------------------------- compute warps
    const int col = lane * 4;
    const bool col_ok = col < Dv;
    const int row0 = warp * kDecRowsPerWarp;
    float b_next = (count > 0 && KDA_IN_BOUNDS(kBufBeta, beta + first, 4)) ? beta[first] : 0.f;
    // fused gate: -exp(A_log[h]) of the next head, fetched a head ahead like beta
    float na_next = (kFused && fz.A_log && count > 0) ? -expf(fz.A_log[first % H]) : 0.f;
    for (int it = 0; it < count; ++it) {
      const int s = it % kDsStages;
      const size_t head = (size_t)first + (size_t)it * stride;
      const float b = b_next;
      if (it + 1 < count)
        b_next = KDA_IN_BOUNDS(kBufBeta, beta + head + stride, 4) ? beta[head + stride] : 0.f;
      const float neg_a = na_next;
      if (kFused && fz.A_log && it + 1 < count)
        na_next = -expf(fz.A_log[(head + stride) % (size_t)H]);
      const bool ok = sm100::mbar_wait(full + s, (it / kDsStages) & 1);
      if (!block_all(ok, 1, kDsCompute)) break;
      uint8_t* st = stages + (size_t)s * lay.stage_bytes;
      const float* la = reinterpret_cast<const float*>(st + lay.la_off);
      const Tin* qv = reinterpret_cast<const Tin*>(st + lay.q_off);
      const Tin* kv = reinterpret_cast<const Tin*>(st + lay.k_off);
      const Tin* vv = reinterpret_cast<const Tin*>(st + lay.v_off);
      // decay of this warp's 16 rows: lanes 0..15 evaluate one each, shuffled to the warp
      const int rl = row0 + (lane & 15);
      float la_mine = (rl < Dk) ? la[rl] : 0.f;
      if (kFused && fz.A_log && rl < Dk) {  // fused gate: raw gate -> log decay
        const float bias = lay.bias_bytes ? reinterpret_cast<const float*>(st + lay.bias_off)[rl]
                                          : 0.f;
        la_mine = neg_a * softplus_f(la_mine + bias);
      }
      const float a_mine = (rl < Dk) ? expf(la_mine) : 1.f;
      float4* Srow = reinterpret_cast<float4*>(st) + (col >> 2);
      const int vstride = Dv >> 2;
      float4 sreg[kDecRowsPerWarp];
#pragma unroll
      for (int i = 0; i < kDecRowsPerWarp; ++i) {
        const int r = row0 + i;
        sreg[i] = (col_ok && r < Dk) ? Srow[r * vstride] : make_float4(0.f, 0.f, 0.f, 0.f);
      }
      float4 e = make_float4(0.f, 0.f, 0.f, 0.f), p = e;
      float kq = 0.f, ssk = 0.f, ssq = 0.f;
      float kr_[kDecRowsPerWarp];
#pragma unroll
      for (int i = 0; i < kDecRowsPerWarp; ++i) {
        const int r = row0 + i;
        const float a = __shfl_sync(0xffffffffu, a_mine, i);
        const float kr = (r < Dk) ? to_f32(kv[r]) : 0.f;
        const float qr = (r < Dk) ? to_f32(qv[r]) : 0.f;
        kr_[i] = kr;
        kq += kr * qr;
        if (kFused) {
          ssk += kr * kr;
          ssq += qr * qr;
        }
        sreg[i].x *= a; sreg[i].y *= a; sreg[i].z *= a; sreg[i].w *= a;
        e.x += sreg[i].x * kr; e.y += sreg[i].y * kr; e.z += sreg[i].z * kr; e.w += sreg[i].w * kr;
        p.x += sreg[i].x * qr; p.y += sreg[i].y * qr; p.z += sreg[i].z * qr; p.w += sreg[i].w * qr;
      }
      s_e[warp * 32 + lane] = e;
      s_p[warp * 32 + lane] = p;
      if (lane == 0) {
        s_kq[warp] = kq;
        if (kFused) {
          s_ss[warp] = ssk;
          s_ss[8 + warp] = ssq;
        }
      }
      sm100::named_barrier_sync(1, kDsCompute);
      e = make_float4(0.f, 0.f, 0.f, 0.f);
      p = e;
      kq = 0.f;
#pragma unroll
      for (int w = 0; w < 8; ++w) {
        const float4 ew = s_e[w * 32 + lane], pw = s_p[w * 32 + lane];
        e.x += ew.x; e.y += ew.y; e.z += ew.z; e.w += ew.w;
        p.x += pw.x; p.y += pw.y; p.z += pw.z; p.w += pw.w;
        kq += s_kq[w];
      }
      float ik = 1.f;
      if (kFused && fz.l2) {  // fused L2 norm, applied to the reductions and to the update
        float sk = 0.f, sq = 0.f;
#pragma unroll
        for (int w = 0; w < 8; ++w) {
          sk += s_ss[w];
          sq += s_ss[8 + w];
        }
        ik = rsqrtf(sk + fz.eps);
        const float iq = rsqrtf(sq + fz.eps);
        e.x *= ik; e.y *= ik; e.z *= ik; e.w *= ik;
        p.x *= iq; p.y *= iq; p.z *= iq; p.w *= iq;
        kq *= ik * iq;
      }
      float4 u = make_float4(0.f, 0.f, 0.f, 0.f);
      if (col_ok) {
        u.x = b * (to_f32(vv[col]) - e.x);
        u.y = b * (to_f32(vv[col + 1]) - e.y);
        u.z = b * (to_f32(vv[col + 2]) - e.z);
        u.w = b * (to_f32(vv[col + 3]) - e.w);
      }
#pragma unroll
      for (int i = 0; i < kDecRowsPerWarp; ++i) {
        const int r = row0 + i;
        if (col_ok && r < Dk) {
          const float kn = kr_[i] * ik;
          float4 t = sreg[i];
          t.x += kn * u.x; t.y += kn * u.y; t.z += kn * u.z; t.w += kn * u.w;
          Srow[r * vstride] = t;
        }
      }
      if (warp == 0) {
        float4 y = make_float4(p.x + kq * u.x, p.y + kq * u.y, p.z + kq * u.z, p.w + kq * u.w);
        if (kFused && fz.onorm) {  // output epilogue: head-wise RMSNorm x sigmoid gate
          float ss = col_ok ? y.x * y.x + y.y * y.y + y.z * y.z + y.w * y.w : 0.f;
#pragma unroll
          for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
          const float inv = rsqrtf(ss / (float)Dv + fz.oeps);
          if (col_ok) {
            float4 wv = (fz.ow && KDA_IN_BOUNDS(kBufNormW, fz.ow + col, 16))
                          ? *reinterpret_cast<const float4*>(fz.ow + col)
                              : make_float4(1.f, 1.f, 1.f, 1.f);
            if (lay.og_bytes) {  // the output gate row staged with the head's vectors
              const Tin* gp = reinterpret_cast<const Tin*>(st + lay.og_off) + col;
              wv.x *= sigmoid_f(to_f32(gp[0]));
              wv.y *= sigmoid_f(to_f32(gp[1]));
              wv.z *= sigmoid_f(to_f32(gp[2]));
              wv.w *= sigmoid_f(to_f32(gp[3]));
            }
            y = make_float4(y.x * inv * wv.x, y.y * inv * wv.y, y.z * inv * wv.z,
                            y.w * inv * wv.w);
          }
        }
        if (col_ok && KDA_IN_BOUNDS(kBufO, o + head * Dv + col, 4ull * sizeof(Tin))) {
          Tin* op = o + head * Dv + col;
          op[0] = from_f32<Tin>(y.x);
          op[1] = from_f32<Tin>(y.y);
          op[2] = from_f32<Tin>(y.z);
          op[3] = from_f32<Tin>(y.w);
        }
      }
      sm100::fence_proxy_async_smem();
      sm100::named_barrier_sync(1, kDsCompute);
      if (tid == 0) sm100::mbar_arrive(computed + s);
    }
  }
  __syncthreads();
}

// ---------------------------------------------------------------------------------------------
// Streaming multi-token variant of the recurrent mode (T <= kRsMaxT tokens per sequence): one
// persistent CTA per SM walks its (sequence, head) items through a two-stage ring. The producer
// warp bulk-loads the item's state (from the pool row given by the state index) and all T
// tokens' vectors at once, and bulk-stores the state back after the last token; the eight compute
// warps keep the state in registers across the T tokens (two block reductions per token), so
// no token waits on global memory and the state crosses HBM once per call.
// ---------------------------------------------------------------------------------------------
constexpr int kRsStages = 2;
constexpr int kRsMaxT = 32;

struct RsLayout {
  uint32_t state_bytes, la_off, q_off, k_off, v_off, og_off, bias_off, stage_bytes;
  uint32_t la_row, qk_row, v_row, og_row;  // bytes of one token's row in the stage
  uint32_t bias_bytes, vec_tx;
};

static RsLayout make_rs_layout(int T, int Dk, int Dv, int es, bool gate_rows, bool bias_row) {
  RsLayout L;
  L.state_bytes = (uint32_t)Dk * Dv * 4;
  L.la_row = align16u((uint32_t)Dk * 4);
  L.qk_row = align16u((uint32_t)Dk * es);
  L.v_row = align16u((uint32_t)Dv * es);
  L.og_row = gate_rows ? L.v_row : 0u;
  L.la_off = L.state_bytes;
  L.q_off = L.la_off + (uint32_t)T * L.la_row;
  L.k_off = L.q_off + (uint32_t)T * L.qk_row;
  L.v_off = L.k_off + (uint32_t)T * L.qk_row;
  L.og_off = L.v_off + (uint32_t)T * L.v_row;
  L.bias_off = L.og_off + (uint32_t)T * L.og_row;
  L.bias_bytes = bias_row ? (uint32_t)Dk * 4 : 0u;
  L.stage_bytes = (L.bias_off + L.bias_bytes + 127u) & ~127u;
  L.vec_tx = (uint32_t)T * ((uint32_t)Dk * 4 + 2u * Dk * es + (uint32_t)Dv * es +
                            (gate_rows ? (uint32_t)Dv * es : 0u)) +
             L.bias_bytes;
  return L;
}

template <typename Tin, bool kFused>
__global__ void __launch_bounds__(kDsThreads, 1)
    recurrent_stream_kernel(const Tin* __restrict__ q, const Tin* __restrict__ k,
                            const Tin* __restrict__ v, const float* __restrict__ log_alpha,
                            const float* __restrict__ beta, float* __restrict__ pool,
                            const int32_t* __restrict__ state_indices, Tin* __restrict__ o,
                            int NH, int T, int H, int Dk, int Dv, int P, RsLayout lay, Fusion fz) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = smem_raw + ((128 - (sm100::smem_u32(smem_raw) & 127)) & 127);
  uint8_t* stages = sm;
  float4* s_e = reinterpret_cast<float4*>(sm + kRsStages * lay.stage_bytes);  // [8][32]
  float4* s_p = s_e + 8 * 32;                                                 // [8][32]
  float* s_kq = reinterpret_cast<float*>(s_p + 8 * 32);                        // [8]
  float* s_ss = s_kq + 8;                                                      // [2][8]
  float* s_beta = s_ss + 16;                                   // [2][kRsMaxT + 1] (+ -exp(A_log))
  uint64_t* full = reinterpret_cast<uint64_t*>(s_beta + 2 * (kRsMaxT + 2));    // [kRsStages]
  uint64_t* computed = full + kRsStages;                                       // [kRsStages]

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int first = blockIdx.x, stride = gridDim.x;
  const int count = first < NH ? (NH - first + stride - 1) / stride : 0;
  const uint32_t es = sizeof(Tin);
  // pool row of an item, -1 to skip it (padding entry or an index past the pool)
  auto slot_of = [&](int it) -> int {
    const int item = first + it * stride, n = item / H;
    const int sl = state_indices ? state_indices[n] : n;
    return (sl >= 0 && sl < P) ? sl : -1;
  };

  if (tid == 0) {
    for (int i = 0; i < kRsStages; ++i) {
      sm100::mbar_init(full + i, 1);
      sm100::mbar_init(computed + i, 1);
    }
    sm100::fence_mbar_init();
  }
  __syncthreads();

  if (warp == kDsCompute / 32) {
    // ---------------------------------------------------------------- producer warp
    auto issue_load = [&](int it, int slot) {
      const int s = it % kRsStages;
      if (slot < 0) {  // nothing to load: complete the phase so the compute warps move on
        if (lane == 0) sm100::mbar_arrive(full + s);
        return;
      }
      const int item = first + it * stride, n = item / H, h = item - n * H;
      uint8_t* st = stages + (size_t)s * lay.stage_bytes;
      if (lane == 0) {
        sm100::mbar_arrive_expect_tx(full + s, lay.state_bytes + lay.vec_tx);
        sm100::bulk_g2s(st, pool + ((size_t)slot * H + h) * Dk * Dv, lay.state_bytes, full + s);
        if (kFused && lay.bias_bytes)
          sm100::bulk_g2s(st + lay.bias_off, fz.dt_bias + (size_t)h * Dk, lay.bias_bytes,
                          full + s);
      }
      for (int t = lane; t < T; t += 32) {  // one token's rows per lane
        const size_t base = ((size_t)n * T + t) * H + h;
        sm100::bulk_g2s(st + lay.la_off + t * lay.la_row, log_alpha + base * Dk, Dk * 4,
                        full + s);
        sm100::bulk_g2s(st + lay.q_off + t * lay.qk_row, q + base * Dk, Dk * es, full + s);
        sm100::bulk_g2s(st + lay.k_off + t * lay.qk_row, k + base * Dk, Dk * es, full + s);
        sm100::bulk_g2s(st + lay.v_off + t * lay.v_row, v + base * Dv, Dv * es, full + s);
        if (kFused && lay.og_row)
          sm100::bulk_g2s(st + lay.og_off + t * lay.og_row,
                          reinterpret_cast<const Tin*>(fz.og) + base * Dv, Dv * es, full + s);
      }
    };
    int slot_cur[kRsStages];
    for (int it = 0; it < count && it < kRsStages; ++it) {
      slot_cur[it] = slot_of(it);
      issue_load(it, slot_cur[it]);
    }
    for (int it = 0; it < count; ++it) {
      const int s = it % kRsStages;
      bool ok = sm100::mbar_wait(computed + s, (it / kRsStages) & 1);
      if (!__all_sync(0xffffffffu, ok)) break;
      if (lane == 0 && slot_cur[s] >= 0) {
        const int item = first + it * stride, h = item % H;
        sm100::bulk_s2g(pool + ((size_t)slot_cur[s] * H + h) * Dk * Dv,
                        stages + (size_t)s * lay.stage_bytes, lay.state_bytes);
        sm100::bulk_commit();
      }
      if (it + kRsStages < count) {
        if (lane == 0) sm100::bulk_wait_read_all();  // the stage is free once its store read it
        __syncwarp();
        slot_cur[s] = slot_of(it + kRsStages);
        issue_load(it + kRsStages, slot_cur[s]);
      }
    }
    if (lane == 0) {
      sm100::bulk_wait_all();
      // loads that were issued but never consumed (only after a timeout) must land first
      for (int it = 0; it < count && it < kRsStages; ++it) {
        const int last = count - 1 - it;
        if (last >= 0)
          sm100::mbar_wait(full + last % kRsStages, (last / kRsStages) & 1, 100000000ull);
      }
    }
  } else {
    // ---------------------------------------------------------------- compute warps
    const int col = lane * 4;
    const bool col_ok = col < Dv;
    const int row0 = warp * kDecRowsPerWarp;
    // per-token beta (and -exp(A_log[h]) for the fused gate) of an item, one item ahead
    auto stage_scalars = [&](int it) {
      float* dst = s_beta + (it & 1) * (kRsMaxT + 2);
      const int item = first + it * stride, n = item / H, h = item - n * H;
      if (tid < T) dst[tid] = beta[((size_t)n * T + tid) * H + h];
      if (kFused && tid == 32 && fz.A_log) dst[kRsMaxT] = -expf(fz.A_log[h]);
    };
    if (count > 0) stage_scalars(0);
    sm100::named_barrier_sync(1, kDsCompute);
    for (int it = 0; it < count; ++it) {
      const int s = it % kRsStages;
      const int item = first + it * stride, n = item / H;
      const int slot_raw = state_indices ? state_indices[n] : n;
      const bool ok = sm100::mbar_wait(full + s, (it / kRsStages) & 1);
      if (!block_all(ok, 1, kDsCompute)) break;
      if (it + 1 < count) stage_scalars(it + 1);  // read after this item's barriers
      if (slot_raw < 0 || slot_raw >= P) {
        if (slot_raw >= P && tid == 0) raise_status(kStatusBadSeqlens);
        sm100::named_barrier_sync(1, kDsCompute);
        if (tid == 0) sm100::mbar_arrive(computed + s);
        continue;
      }
      uint8_t* st = stages + (size_t)s * lay.stage_bytes;
      const float* sb = s_beta + (it & 1) * (kRsMaxT + 2);
      float4* Srow = reinterpret_cast<float4*>(st) + (col >> 2);
      const int vstride = Dv >> 2;
      float4 sreg[kDecRowsPerWarp];
#pragma unroll
      for (int i = 0; i < kDecRowsPerWarp; ++i) {
        const int r = row0 + i;
        sreg[i] = (col_ok && r < Dk) ? Srow[r * vstride] : make_float4(0.f, 0.f, 0.f, 0.f);
      }
      const int rl = row0 + (lane & 15);
      const float bias_r = (kFused && fz.A_log && lay.bias_bytes && rl < Dk)
                               ? reinterpret_cast<const float*>(st + lay.bias_off)[rl]
                               : 0.f;
      for (int t = 0; t < T; ++t) {
        const float* la = reinterpret_cast<const float*>(st + lay.la_off + t * lay.la_row);
        const Tin* qv = reinterpret_cast<const Tin*>(st + lay.q_off + t * lay.qk_row);
        const Tin* kv = reinterpret_cast<const Tin*>(st + lay.k_off + t * lay.qk_row);
        const Tin* vv = reinterpret_cast<const Tin*>(st + lay.v_off + t * lay.v_row);
        float la_mine = (rl < Dk) ? la[rl] : 0.f;
        if (kFused && fz.A_log && rl < Dk) la_mine = sb[kRsMaxT] * softplus_f(la_mine + bias_r);
        const float a_mine = (rl < Dk) ? expf(la_mine) : 1.f;
        float4 e = make_float4(0.f, 0.f, 0.f, 0.f), p = e;
        float kq = 0.f, ssk = 0.f, ssq = 0.f;
        float kr_[kDecRowsPerWarp];
#pragma unroll
        for (int i = 0; i < kDecRowsPerWarp; ++i) {
          const int r = row0 + i;
          const float a = __shfl_sync(0xffffffffu, a_mine, i);
          const float kr = (r < Dk) ? to_f32(kv[r]) : 0.f;
          const float qr = (r < Dk) ? to_f32(qv[r]) : 0.f;
          kr_[i] = kr;
          kq += kr * qr;
          if (kFused) {
            ssk += kr * kr;
            ssq += qr * qr;
          }
          sreg[i].x *= a; sreg[i].y *= a; sreg[i].z *= a; sreg[i].w *= a;
          e.x += sreg[i].x * kr; e.y += sreg[i].y * kr; e.z += sreg[i].z * kr; e.w += sreg[i].w * kr;
          p.x += sreg[i].x * qr; p.y += sreg[i].y * qr; p.z += sreg[i].z * qr; p.w += sreg[i].w * qr;
        }
        s_e[warp * 32 + lane] = e;
        s_p[warp * 32 + lane] = p;
        if (lane == 0) {
          s_kq[warp] = kq;
          if (kFused) {
            s_ss[warp] = ssk;
            s_ss[8 + warp] = ssq;
          }
        }
        sm100::named_barrier_sync(1, kDsCompute);
        e = make_float4(0.f, 0.f, 0.f, 0.f);
        p = e;
        kq = 0.f;
#pragma unroll
        for (int w = 0; w < 8; ++w) {
          const float4 ew = s_e[w * 32 + lane], pw = s_p[w * 32 + lane];
          e.x += ew.x; e.y += ew.y; e.z += ew.z; e.w += ew.w;
          p.x += pw.x; p.y += pw.y; p.z += pw.z; p.w += pw.w;
          kq += s_kq[w];
        }
        float ik = 1.f;
        if (kFused && fz.l2) {
          float sk = 0.f, sq = 0.f;
#pragma unroll
          for (int w = 0; w < 8; ++w) {
            sk += s_ss[w];
            sq += s_ss[8 + w];
          }
          ik = rsqrtf(sk + fz.eps);
          const float iq = rsqrtf(sq + fz.eps);
          e.x *= ik; e.y *= ik; e.z *= ik; e.w *= ik;
          p.x *= iq; p.y *= iq; p.z *= iq; p.w *= iq;
          kq *= ik * iq;
        }
        const float b = sb[t];
        float4 u = make_float4(0.f, 0.f, 0.f, 0.f);
        if (col_ok) {
          u.x = b * (to_f32(vv[col]) - e.x);
          u.y = b * (to_f32(vv[col + 1]) - e.y);
          u.z = b * (to_f32(vv[col + 2]) - e.z);
          u.w = b * (to_f32(vv[col + 3]) - e.w);
        }
#pragma unroll
        for (int i = 0; i < kDecRowsPerWarp; ++i) {
          const float kn = kr_[i] * ik;
          sreg[i].x += kn * u.x; sreg[i].y += kn * u.y; sreg[i].z += kn * u.z; sreg[i].w += kn * u.w;
        }
        if (warp == 0) {
          float4 y = make_float4(p.x + kq * u.x, p.y + kq * u.y, p.z + kq * u.z, p.w + kq * u.w);
          if (kFused && fz.onorm) {
            float ss = col_ok ? y.x * y.x + y.y * y.y + y.z * y.z + y.w * y.w : 0.f;
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
            const float inv = rsqrtf(ss / (float)Dv + fz.oeps);
            if (col_ok) {
              float4 wv = (fz.ow && KDA_IN_BOUNDS(kBufNormW, fz.ow + col, 16))
                          ? *reinterpret_cast<const float4*>(fz.ow + col)
                                : make_float4(1.f, 1.f, 1.f, 1.f);
              if (lay.og_row) {
                const Tin* gp = reinterpret_cast<const Tin*>(st + lay.og_off + t * lay.og_row) + col;
                wv.x *= sigmoid_f(to_f32(gp[0]));
                wv.y *= sigmoid_f(to_f32(gp[1]));
                wv.z *= sigmoid_f(to_f32(gp[2]));
                wv.w *= sigmoid_f(to_f32(gp[3]));
              }
              y = make_float4(y.x * inv * wv.x, y.y * inv * wv.y, y.z * inv * wv.z,
                              y.w * inv * wv.w);
            }
          }
          if (col_ok) {
            Tin* op = o + (((size_t)n * T + t) * H + (item - n * H)) * Dv + col;
            op[0] = from_f32<Tin>(y.x);
            op[1] = from_f32<Tin>(y.y);
            op[2] = from_f32<Tin>(y.z);
            op[3] = from_f32<Tin>(y.w);
          }
        }
        sm100::named_barrier_sync(1, kDsCompute);  // s_e / s_p are rewritten by the next token
      }
#pragma unroll
      for (int i = 0; i < kDecRowsPerWarp; ++i) {
        const int r = row0 + i;
        if (col_ok && r < Dk) Srow[r * vstride] = sreg[i];
      }
      sm100::fence_proxy_async_smem();
      sm100::named_barrier_sync(1, kDsCompute);
      if (tid == 0) sm100::mbar_arrive(computed + s);
    }
  }
  __syncthreads();
}

// ---------------------------------------------------------------------------------------------
// Column-layout variant of the streaming recurrent mode (d_k = d_v = 128, T tokens that fit the
// shared-memory budget): the same producer warp and two-stage ring, eight compute warps, each
// owning 16 columns of the state over all 128 rows: lane = (row group rg of 16 rows, column quad
// cq), so a thread holds a 16 x 4 tile in registers, as packed fp32 pairs of adjacent rows: the
// decay, the two reductions and the update each take one fma/mul .f32x2 per row pair and column,
// with the rows' decays, keys and queries read from shared memory as pairs. For T <= 16, an item
// whose rows decay by less than e^-60 over the call runs in the running-decay form: with D_t the
// product of the row's decays from the item start, S_t = Diag(D_t) Shat_t, so
// e = Shat^T (D_t k), p = Shat^T (D_t q) and Shat += (k / D_t) (beta (v - e))^T need no per-token
// decay of the state; D_t k, D_t q and k / D_t are formed once per token before the loop and the
// state is scaled by D_T after it (fp32 throughout: every term keeps its relative precision).
// A token's reductions
// e_j = sum_i S'[i][j] k_i and p_j = sum_i S'[i][j] q_i then end in three lane exchanges inside
// the warp instead of a block-wide reduction, so the token loop has no barrier. The per-token decays exp(log alpha),
// k.q, the norms and beta are computed for all T tokens of an item in one pass before it, and
// the outputs (with the head-wise norm and gate when fused) are written by one pass after it.
// ---------------------------------------------------------------------------------------------
constexpr int kRcCompute = 256;                // 8 compute warps
// the running-decay form keeps 1 / D_t below e^60: its terms stay far inside fp32's range
constexpr float kRcLazyLimit = 60.f;

// Position of row r inside a token's per-row vector in shared memory (the decays, or the scaled
// keys and queries): the 4-row chunks of each 16-row group are permuted by ((r >> 5) & 3), so the
// eight row groups of a warp, which read one chunk each at a time, hit eight distinct bank groups.
__device__ __forceinline__ int rc_row(int r) {
  return (r & ~15) | ((((r >> 2) & 3) ^ ((r >> 5) & 3)) << 2) | (r & 3);
}
constexpr int kRcThreads = kRcCompute + 32;    // + producer warp
constexpr int kRcD = 128;

__device__ __forceinline__ void load8_f32(const float* p, float (&x)[8]) {
  const float4 a = reinterpret_cast<const float4*>(p)[0], b = reinterpret_cast<const float4*>(p)[1];
  x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w; x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
}
__device__ __forceinline__ void load8_in(const float* p, float (&x)[8]) { load8_f32(p, x); }
__device__ __forceinline__ void load8_in(const __nv_bfloat16* p, float (&x)[8]) {
  const uint4 u = *reinterpret_cast<const uint4*>(p);
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    x[2 * i] = __uint_as_float(w[i] << 16);
    x[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
  }
}

template <typename Tin, bool kFused>
__global__ void __launch_bounds__(kRcThreads, 1)
    recurrent_cols_kernel(const Tin* __restrict__ q, const Tin* __restrict__ k,
                          const Tin* __restrict__ v, const float* __restrict__ log_alpha,
                          const float* __restrict__ beta, float* __restrict__ pool,
                          const int32_t* __restrict__ state_indices, Tin* __restrict__ o, int NH,
                          int T, int H, int P, RsLayout lay, Fusion fz) {
  constexpr int D = kRcD;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = smem_raw + ((128 - (sm100::smem_u32(smem_raw) & 127)) & 127);
  uint8_t* stages = sm;
  float* s_alpha = reinterpret_cast<float*>(sm + kRsStages * lay.stage_bytes);  // [kRsMaxT][D]
  float* s_y = s_alpha + kRsMaxT * D;                                           // [kRsMaxT][D]
  float4* s_tok = reinterpret_cast<float4*>(s_y + kRsMaxT * D);  // [kRsMaxT]: kq, 1/|k|, 1/|q|, beta
  float* s_beta = reinterpret_cast<float*>(s_tok + kRsMaxT);     // [2][kRsMaxT + 2]
  uint64_t* full = reinterpret_cast<uint64_t*>(s_beta + 2 * (kRsMaxT + 2));  // [kRsStages]
  uint64_t* computed = full + kRsStages;                                     // [kRsStages]
  // running-decay form (T <= kRsMaxT / 2): D_t k, D_t q in the decay area, k / D_t beside the
  // outputs; D_T per row and the item's form flag after the barriers
  float* s_dT = reinterpret_cast<float*>(computed + kRsStages);  // [D]
  int* s_lazy = reinterpret_cast<int*>(s_dT + D);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int first = blockIdx.x, stride = gridDim.x;
  const int count = first < NH ? (NH - first + stride - 1) / stride : 0;
  const uint32_t es = sizeof(Tin);
  auto slot_of = [&](int it) -> int {
    const int item = first + it * stride, n = item / H;
    const int sl = state_indices ? (KDA_IN_BOUNDS(kBufIndices, state_indices + n, 4)
                                        ? state_indices[n] : -1)
                                 : n;
    return (sl >= 0 && sl < P) ? sl : -1;
  };

  if (tid == 0) {
    for (int i = 0; i < kRsStages; ++i) {
      sm100::mbar_init(full + i, 1);
      sm100::mbar_init(computed + i, 1);
    }
    sm100::fence_mbar_init();
  }
  __syncthreads();

  if (warp == kRcCompute / 32) {
    // ---------------------------------------------------------------- producer warp
    // issues the item's loads and returns the pool row its state came from (-1: none loaded)
    auto issue_load = [&](int it, int slot) -> int {
      const int s = it % kRsStages;
      const int item = first + it * stride, n = item / H, h = item - n * H;
      if (slot >= 0 && kBoundsChecked) {  // every copy of the item inside its buffer, or none
        bool ok =
            KDA_IN_BOUNDS(kBufState, pool + ((size_t)slot * H + h) * D * D, lay.state_bytes) &&
            (!(kFused && lay.bias_bytes) ||
             KDA_IN_BOUNDS(kBufDtBias, fz.dt_bias + (size_t)h * D, lay.bias_bytes));
        for (int t = lane; t < T; t += 32) {
          const size_t base = ((size_t)n * T + t) * H + h;
          ok = ok && KDA_IN_BOUNDS(kBufLogAlpha, log_alpha + base * D, D * 4ull) &&
               KDA_IN_BOUNDS(kBufQ, q + base * D, (size_t)D * es) &&
               KDA_IN_BOUNDS(kBufK, k + base * D, (size_t)D * es) &&
               KDA_IN_BOUNDS(kBufV, v + base * D, (size_t)D * es) &&
               (!(kFused && lay.og_row) ||
                KDA_IN_BOUNDS(kBufGate, reinterpret_cast<const Tin*>(fz.og) + base * D,
                              (size_t)D * es));
        }
        if (!__all_sync(0xffffffffu, ok)) slot = -1;
      }
      if (slot < 0) {
        if (lane == 0) sm100::mbar_arrive(full + s);
        return -1;
      }
      uint8_t* st = stages + (size_t)s * lay.stage_bytes;
      if (lane == 0) {
        sm100::mbar_arrive_expect_tx(full + s, lay.state_bytes + lay.vec_tx);
        sm100::bulk_g2s(st, pool + ((size_t)slot * H + h) * D * D, lay.state_bytes, full + s);
        if (kFused && lay.bias_bytes)
          sm100::bulk_g2s(st + lay.bias_off, fz.dt_bias + (size_t)h * D, lay.bias_bytes, full + s);
      }
      for (int t = lane; t < T; t += 32) {
        const size_t base = ((size_t)n * T + t) * H + h;
        sm100::bulk_g2s(st + lay.la_off + t * lay.la_row, log_alpha + base * D, D * 4, full + s);
        sm100::bulk_g2s(st + lay.q_off + t * lay.qk_row, q + base * D, D * es, full + s);
        sm100::bulk_g2s(st + lay.k_off + t * lay.qk_row, k + base * D, D * es, full + s);
        sm100::bulk_g2s(st + lay.v_off + t * lay.v_row, v + base * D, D * es, full + s);
        if (kFused && lay.og_row)
          sm100::bulk_g2s(st + lay.og_off + t * lay.og_row,
                          reinterpret_cast<const Tin*>(fz.og) + base * D, D * es, full + s);
      }
      return slot;
    };
    int slot_cur[kRsStages];
    for (int it = 0; it < count && it < kRsStages; ++it) slot_cur[it] = issue_load(it, slot_of(it));
    for (int it = 0; it < count; ++it) {
      const int s = it % kRsStages;
      bool ok = sm100::mbar_wait(computed + s, (it / kRsStages) & 1);
      if (!__all_sync(0xffffffffu, ok)) break;
      if (lane == 0 && slot_cur[s] >= 0) {  // (a row inside the pool: issue_load checked it)
        const int item = first + it * stride, h = item % H;
        sm100::bulk_s2g(pool + ((size_t)slot_cur[s] * H + h) * D * D,
                        stages + (size_t)s * lay.stage_bytes, lay.state_bytes);
        sm100::bulk_commit();
      }
      if (it + kRsStages < count) {
        if (lane == 0) sm100::bulk_wait_read_all();  // the stage is free once its store read it
        __syncwarp();
        slot_cur[s] = issue_load(it + kRsStages, slot_of(it + kRsStages));
      }
    }
    if (lane == 0) {
      sm100::bulk_wait_all();
      for (int it = 0; it < count && it < kRsStages; ++it) {
        const int last = count - 1 - it;
        if (last >= 0)
          sm100::mbar_wait(full + last % kRsStages, (last / kRsStages) & 1, 100000000ull);
      }
    }
  } else {
    // ---------------------------------------------------------------- compute warps
    const int rg = lane >> 2, cq = lane & 3;
    const int r0 = 16 * rg, c0 = 16 * warp + 4 * cq;  // rows r0 .. r0 + 15, columns c0 .. c0 + 3
    auto stage_scalars = [&](int it) {  // beta (and -exp(A_log[h])) of an item, one item ahead
      float* dst = s_beta + (it & 1) * (kRsMaxT + 2);
      const int item = first + it * stride, n = item / H, h = item - n * H;
      if (tid < T)
        dst[tid] = KDA_IN_BOUNDS(kBufBeta, beta + ((size_t)n * T + tid) * H + h, 4)
                       ? beta[((size_t)n * T + tid) * H + h]
                       : 0.f;
      if (kFused && tid == 32 && fz.A_log)
        dst[kRsMaxT] = KDA_IN_BOUNDS(kBufALog, fz.A_log + h, 4) ? -expf(fz.A_log[h]) : 0.f;
    };
    if (count > 0) stage_scalars(0);
    sm100::named_barrier_sync(1, kRcCompute);
    for (int it = 0; it < count; ++it) {
      const int s = it % kRsStages;
      const int item = first + it * stride, n = item / H, h = item - n * H;
      const int slot_raw =
          state_indices ? (KDA_IN_BOUNDS(kBufIndices, state_indices + n, 4) ? state_indices[n] : -1)
                        : n;
      const bool ok = sm100::mbar_wait(full + s, (it / kRsStages) & 1);
      if (!block_all(ok, 1, kRcCompute)) break;
      const float* sb = s_beta + (it & 1) * (kRsMaxT + 2);
      if (slot_raw < 0 || slot_raw >= P) {
        if (slot_raw >= P && tid == 0) raise_status(kStatusBadSeqlens);
        if (it + 1 < count) stage_scalars(it + 1);
        sm100::named_barrier_sync(1, kRcCompute);
        if (tid == 0) sm100::mbar_arrive(computed + s);
        continue;
      }
      uint8_t* st = stages + (size_t)s * lay.stage_bytes;
      // pre-pass: the running log decay of every row over the item decides the form; then either
      // every token's decays (token form) or the scaled keys and queries (running-decay form);
      // k.q, inverse norms and beta per token (one warp each)
      float* s_khat = s_alpha;
      float* s_qhat = s_alpha + T * D;
      float* s_ktil = s_y + (kRsMaxT / 2) * D;
      if (tid == 0) *s_lazy = T <= kRsMaxT / 2;
      sm100::named_barrier_sync(1, kRcCompute);
      if (tid < D) {
        float G = 0.f;
        for (int t = 0; t < T; ++t) {
          float la = reinterpret_cast<const float*>(st + lay.la_off + t * lay.la_row)[tid];
          if (kFused && fz.A_log) {
            const float bias = lay.bias_bytes
                                   ? reinterpret_cast<const float*>(st + lay.bias_off)[tid]
                                   : 0.f;
            la = sb[kRsMaxT] * softplus_f(la + bias);
          }
          G += la;
        }
        s_dT[tid] = expf(G);
        if (!(G >= -kRcLazyLimit)) *s_lazy = 0;
      }
      sm100::named_barrier_sync(1, kRcCompute);
      const bool lazy = *s_lazy != 0;
      if (lazy) {
        if (tid < D) {  // row tid: D_t = exp(sum of the decays up to t)
          float G = 0.f;
          for (int t = 0; t < T; ++t) {
            float la = reinterpret_cast<const float*>(st + lay.la_off + t * lay.la_row)[tid];
            if (kFused && fz.A_log) {
              const float bias = lay.bias_bytes
                                     ? reinterpret_cast<const float*>(st + lay.bias_off)[tid]
                                     : 0.f;
              la = sb[kRsMaxT] * softplus_f(la + bias);
            }
            G += la;
            const float Dt = expf(G), Di = expf(-G);
            const float kx = to_f32(reinterpret_cast<const Tin*>(st + lay.k_off + t * lay.qk_row)[tid]);
            const float qx = to_f32(reinterpret_cast<const Tin*>(st + lay.q_off + t * lay.qk_row)[tid]);
            s_khat[t * D + rc_row(tid)] = Dt * kx;
            s_qhat[t * D + rc_row(tid)] = Dt * qx;
            s_ktil[t * D + rc_row(tid)] = Di * kx;
          }
        }
      } else {
        for (int e = tid; e < T * D; e += kRcCompute) {
          const int t = e >> 7, i = e & (D - 1);
          float la = reinterpret_cast<const float*>(st + lay.la_off + t * lay.la_row)[i];
          if (kFused && fz.A_log) {
            const float bias = lay.bias_bytes
                                   ? reinterpret_cast<const float*>(st + lay.bias_off)[i]
                                   : 0.f;
            la = sb[kRsMaxT] * softplus_f(la + bias);
          }
          s_alpha[t * D + rc_row(i)] = expf(la);
        }
      }
      for (int t = warp; t < T; t += kRcCompute / 32) {
        float kx[4], qx[4];
        const Tin* kv = reinterpret_cast<const Tin*>(st + lay.k_off + t * lay.qk_row) + 4 * lane;
        const Tin* qv = reinterpret_cast<const Tin*>(st + lay.q_off + t * lay.qk_row) + 4 * lane;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          kx[c] = to_f32(kv[c]);
          qx[c] = to_f32(qv[c]);
        }
        float kq = 0.f, ssk = 0.f, ssq = 0.f;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          kq = fmaf(kx[c], qx[c], kq);
          ssk = fmaf(kx[c], kx[c], ssk);
          ssq = fmaf(qx[c], qx[c], ssq);
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
          kq += __shfl_xor_sync(0xffffffffu, kq, off);
          ssk += __shfl_xor_sync(0xffffffffu, ssk, off);
          ssq += __shfl_xor_sync(0xffffffffu, ssq, off);
        }
        if (lane == 0) {
          float ik = 1.f, iq = 1.f;
          if (kFused && fz.l2) {
            ik = rsqrtf(ssk + fz.eps);
            iq = rsqrtf(ssq + fz.eps);
          }
          s_tok[t] = make_float4(kq * ik * iq, ik, iq, sb[t]);
        }
      }
      if (it + 1 < count) stage_scalars(it + 1);  // the other buffer; read after this barrier
      sm100::named_barrier_sync(1, kRcCompute);

      // the thread's 16 x 4 state tile as 8 row pairs x 4 columns: SP[4 jr + c] holds
      // (S[r0 + 2 jr][c0 + c], S[r0 + 2 jr + 1][c0 + c]), so the per-row decays, keys and queries
      // enter the packed products as adjacent pairs straight from shared memory
      f32x2 SP[32];
      float* Sst = reinterpret_cast<float*>(st);
#pragma unroll
      for (int jr = 0; jr < 8; ++jr) {
        const float4 lo = *reinterpret_cast<const float4*>(Sst + (r0 + 2 * jr) * D + c0);
        const float4 hi = *reinterpret_cast<const float4*>(Sst + (r0 + 2 * jr + 1) * D + c0);
        SP[4 * jr + 0] = f2_pack(lo.x, hi.x);
        SP[4 * jr + 1] = f2_pack(lo.y, hi.y);
        SP[4 * jr + 2] = f2_pack(lo.z, hi.z);
        SP[4 * jr + 3] = f2_pack(lo.w, hi.w);
      }
      for (int t = 0; t < T; ++t) {
        f32x2 kp[8];  // (k_r, k_r+1) pairs for the update: k / D_t (running form) or k
        f32x2 ep[4], pp[4];  // per column: partial sums over the even and the odd rows
#pragma unroll
        for (int c = 0; c < 4; ++c) ep[c] = pp[c] = 0ull;
        if (lazy) {
          const int sw = (rg >> 1) & 3;  // this row group's chunk permutation (rc_row)
#pragma unroll
          for (int m = 0; m < 4; ++m) {
            const int o4 = t * D + r0 + 4 * (m ^ sw);
            const float4 a = *reinterpret_cast<const float4*>(s_khat + o4);
            const float4 b = *reinterpret_cast<const float4*>(s_qhat + o4);
            const float4 c4 = *reinterpret_cast<const float4*>(s_ktil + o4);
#pragma unroll
            for (int hlf = 0; hlf < 2; ++hlf) {
              const int jr = 2 * m + hlf;
              const f32x2 khp = hlf ? f2_pack(a.z, a.w) : f2_pack(a.x, a.y);
              const f32x2 qhp = hlf ? f2_pack(b.z, b.w) : f2_pack(b.x, b.y);
              kp[jr] = hlf ? f2_pack(c4.z, c4.w) : f2_pack(c4.x, c4.y);
#pragma unroll
              for (int c = 0; c < 4; ++c) {
                ep[c] = f2_fma(SP[4 * jr + c], khp, ep[c]);
                pp[c] = f2_fma(SP[4 * jr + c], qhp, pp[c]);
              }
            }
          }
        } else {
        const float* al = s_alpha + t * D + r0;
        const Tin* kv = reinterpret_cast<const Tin*>(st + lay.k_off + t * lay.qk_row) + r0;
        const Tin* qv = reinterpret_cast<const Tin*>(st + lay.q_off + t * lay.qk_row) + r0;
        const int sw = (rg >> 1) & 3;  // this row group's chunk permutation (rc_row)
#pragma unroll
        for (int i8 = 0; i8 < 2; ++i8) {  // S' = Diag(alpha) S; e, p over this thread's rows
          float a[8], kk[8], qv8[8];
          {
            const float4 a0 = *reinterpret_cast<const float4*>(al + 4 * ((2 * i8) ^ sw));
            const float4 a1 = *reinterpret_cast<const float4*>(al + 4 * ((2 * i8 + 1) ^ sw));
            a[0] = a0.x; a[1] = a0.y; a[2] = a0.z; a[3] = a0.w;
            a[4] = a1.x; a[5] = a1.y; a[6] = a1.z; a[7] = a1.w;
          }
          load8_in(kv + 8 * i8, kk);
          load8_in(qv + 8 * i8, qv8);
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const int jr = 4 * i8 + u;
            const f32x2 ap = f2_pack(a[2 * u], a[2 * u + 1]);
            kp[jr] = f2_pack(kk[2 * u], kk[2 * u + 1]);
            const f32x2 qp = f2_pack(qv8[2 * u], qv8[2 * u + 1]);
#pragma unroll
            for (int c = 0; c < 4; ++c) {
              SP[4 * jr + c] = f2_mul(SP[4 * jr + c], ap);
              ep[c] = f2_fma(SP[4 * jr + c], kp[jr], ep[c]);
              pp[c] = f2_fma(SP[4 * jr + c], qp, pp[c]);
            }
          }
        }
        }
        float4 e, p;
        {
          const float2 e0 = f2_unpack(ep[0]), e1 = f2_unpack(ep[1]), e2 = f2_unpack(ep[2]),
                       e3 = f2_unpack(ep[3]);
          const float2 p0 = f2_unpack(pp[0]), p1 = f2_unpack(pp[1]), p2 = f2_unpack(pp[2]),
                       p3 = f2_unpack(pp[3]);
          e = make_float4(e0.x + e0.y, e1.x + e1.y, e2.x + e2.y, e3.x + e3.y);
          p = make_float4(p0.x + p0.y, p1.x + p1.y, p2.x + p2.y, p3.x + p3.y);
        }
#pragma unroll
        for (int off = 4; off < 32; off <<= 1) {  // over the eight row groups of the warp
          e.x += __shfl_xor_sync(0xffffffffu, e.x, off);
          e.y += __shfl_xor_sync(0xffffffffu, e.y, off);
          e.z += __shfl_xor_sync(0xffffffffu, e.z, off);
          e.w += __shfl_xor_sync(0xffffffffu, e.w, off);
          p.x += __shfl_xor_sync(0xffffffffu, p.x, off);
          p.y += __shfl_xor_sync(0xffffffffu, p.y, off);
          p.z += __shfl_xor_sync(0xffffffffu, p.z, off);
          p.w += __shfl_xor_sync(0xffffffffu, p.w, off);
        }
        const float4 tk = s_tok[t];  // k.q (normalised), 1/|k|, 1/|q|, beta
        const Tin* vv = reinterpret_cast<const Tin*>(st + lay.v_off + t * lay.v_row) + c0;
        const float4 u = make_float4(tk.w * (to_f32(vv[0]) - e.x * tk.y),
                                     tk.w * (to_f32(vv[1]) - e.y * tk.y),
                                     tk.w * (to_f32(vv[2]) - e.z * tk.y),
                                     tk.w * (to_f32(vv[3]) - e.w * tk.y));
        if (rg == 0)  // o_t = S'^T q + (k.q) beta (v - e)
          *reinterpret_cast<float4*>(s_y + t * D + c0) =
              make_float4(p.x * tk.z + tk.x * u.x, p.y * tk.z + tk.x * u.y,
                          p.z * tk.z + tk.x * u.z, p.w * tk.z + tk.x * u.w);
        const f32x2 ku[4] = {f2_pack(tk.y * u.x, tk.y * u.x), f2_pack(tk.y * u.y, tk.y * u.y),
                             f2_pack(tk.y * u.z, tk.y * u.z), f2_pack(tk.y * u.w, tk.y * u.w)};
#pragma unroll
        for (int jr = 0; jr < 8; ++jr)  // S = S' + k (beta (v - e))^T
#pragma unroll
          for (int c = 0; c < 4; ++c) SP[4 * jr + c] = f2_fma(kp[jr], ku[c], SP[4 * jr + c]);
      }
      if (lazy) {  // S = Diag(D_T) Shat
#pragma unroll
        for (int jr = 0; jr < 8; ++jr) {
          const f32x2 dp = f2_pack(s_dT[r0 + 2 * jr], s_dT[r0 + 2 * jr + 1]);
#pragma unroll
          for (int c = 0; c < 4; ++c) SP[4 * jr + c] = f2_mul(SP[4 * jr + c], dp);
        }
      }
#pragma unroll
      for (int jr = 0; jr < 8; ++jr) {
        const float2 s0 = f2_unpack(SP[4 * jr + 0]), s1 = f2_unpack(SP[4 * jr + 1]);
        const float2 s2 = f2_unpack(SP[4 * jr + 2]), s3 = f2_unpack(SP[4 * jr + 3]);
        *reinterpret_cast<float4*>(Sst + (r0 + 2 * jr) * D + c0) = make_float4(s0.x, s1.x, s2.x, s3.x);
        *reinterpret_cast<float4*>(Sst + (r0 + 2 * jr + 1) * D + c0) = make_float4(s0.y, s1.y, s2.y, s3.y);
      }
      sm100::named_barrier_sync(1, kRcCompute);  // s_y complete
      // outputs: one warp per token row, four columns per lane (head-wise norm x gate if fused)
      for (int t = warp; t < T; t += kRcCompute / 32) {
        float4 y = reinterpret_cast<const float4*>(s_y + t * D)[lane];
        if (kFused && fz.onorm) {
          float ss = y.x * y.x + y.y * y.y + y.z * y.z + y.w * y.w;
#pragma unroll
          for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
          const float inv = rsqrtf(ss * (1.f / D) + fz.oeps);
          float4 wv = (fz.ow && KDA_IN_BOUNDS(kBufNormW, fz.ow + 4 * lane, 16))
                          ? reinterpret_cast<const float4*>(fz.ow)[lane]
                          : make_float4(1.f, 1.f, 1.f, 1.f);
          if (lay.og_row) {
            const Tin* gp = reinterpret_cast<const Tin*>(st + lay.og_off + t * lay.og_row) + 4 * lane;
            wv.x *= sigmoid_f(to_f32(gp[0]));
            wv.y *= sigmoid_f(to_f32(gp[1]));
            wv.z *= sigmoid_f(to_f32(gp[2]));
            wv.w *= sigmoid_f(to_f32(gp[3]));
          }
          y = make_float4(y.x * inv * wv.x, y.y * inv * wv.y, y.z * inv * wv.z, y.w * inv * wv.w);
        }
        Tin* op = o + (((size_t)n * T + t) * H + h) * D + 4 * lane;
        if (KDA_IN_BOUNDS(kBufO, op, 4ull * sizeof(Tin))) {
          op[0] = from_f32<Tin>(y.x);
          op[1] = from_f32<Tin>(y.y);
          op[2] = from_f32<Tin>(y.z);
          op[3] = from_f32<Tin>(y.w);
        }
      }
      sm100::fence_proxy_async_smem();
      sm100::named_barrier_sync(1, kRcCompute);
      if (tid == 0) sm100::mbar_arrive(computed + s);
    }
  }
  __syncthreads();
}

template <typename Tin, bool kFused>
static cudaError_t launch_rc_typed(const void* q, const void* k, const void* v,
                                   const float* log_alpha, const float* beta, float* pool,
                                   const int32_t* idx, void* o, int heads, int T, int H, int P,
                                   const RsLayout& lay, int grid, size_t smem, const Fusion& fz,
                                   cudaStream_t stream) {
  cudaError_t err = cudaFuncSetAttribute(recurrent_cols_kernel<Tin, kFused>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (err != cudaSuccess) return err;
  recurrent_cols_kernel<Tin, kFused><<<grid, kRcThreads, smem, stream>>>(
      (const Tin*)q, (const Tin*)k, (const Tin*)v, log_alpha, beta, pool, idx, (Tin*)o, heads, T,
      H, P, lay, fz);
  return cudaGetLastError();
}

template <typename Tin, bool kFused>
static cudaError_t launch_rs_typed(const void* q, const void* k, const void* v,
                                   const float* log_alpha, const float* beta, float* pool,
                                   const int32_t* idx, void* o, int heads, int T, int H, int Dk,
                                   int Dv, int P, const RsLayout& lay, int grid, size_t smem,
                                   const Fusion& fz, cudaStream_t stream) {
  cudaError_t err = cudaFuncSetAttribute(recurrent_stream_kernel<Tin, kFused>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (err != cudaSuccess) return err;
  recurrent_stream_kernel<Tin, kFused><<<grid, kDsThreads, smem, stream>>>(
      (const Tin*)q, (const Tin*)k, (const Tin*)v, log_alpha, beta, pool, idx, (Tin*)o, heads, T,
      H, Dk, Dv, P, lay, fz);
  return cudaGetLastError();
}

// SM count of each device (0 until first asked); calls from several host threads may fill an
// entry concurrently, all with the same value.
static std::atomic<int> g_num_sms[64];

static int num_sms_cached() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  int nsm = (dev >= 0 && dev < 64) ? g_num_sms[dev].load(std::memory_order_relaxed) : 0;
  if (nsm == 0) {
    if (cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
    if (dev >= 0 && dev < 64) g_num_sms[dev].store(nsm, std::memory_order_relaxed);
  }
  return nsm;
}

cudaError_t launch_recurrent_multi(const void* q, const void* k, const void* v, kda_dtype_t dt,
                                   const float* log_alpha, const float* beta, float* pool,
                                   const int32_t* idx, void* o, int N, int T, int H, int Dk,
                                   int Dv, int P, const Fusion& fz, cudaStream_t stream) {
  const long long heads = (long long)N * H;
  if (heads == 0 || T == 0) return cudaSuccess;
  if (recurrent_chunk_applies(dt, T, Dk, Dv, q, k, v, log_alpha, pool, o, fz))
    return launch_recurrent_chunk(q, k, v, dt, log_alpha, beta, pool, idx, o, heads, T, H, P, fz,
                                  stream);
  const int es = dt == KDA_DTYPE_BF16 ? 2 : 4;
  auto al16 = [](const void* p) { return ((uintptr_t)p & 15u) == 0; };
  const bool fused = fz.l2 || fz.A_log || fz.onorm;
  const bool gate_rows = fz.onorm && fz.og, bias_row = fz.A_log && fz.dt_bias;
  const RsLayout lay = make_rs_layout(T, Dk, Dv, es, gate_rows, bias_row);
  const size_t smem = (size_t)kRsStages * lay.stage_bytes + 2 * 8 * 32 * sizeof(float4) +
                      (24 + 2 * (kRsMaxT + 2)) * sizeof(float) +
                      2 * kRsStages * sizeof(uint64_t) + 128;
  const bool streamable = T <= kRsMaxT && (Dk * es) % 16 == 0 && (Dv * es) % 16 == 0 &&
                          (Dk * 4) % 16 == 0 && al16(q) && al16(k) && al16(v) &&
                          al16(log_alpha) && al16(pool) && (!gate_rows || al16(fz.og)) &&
                          (!bias_row || al16(fz.dt_bias)) && smem <= 227u * 1024u &&
                          heads <= INT32_MAX;
  if (!streamable)
    return launch_recurrent_blockwise(q, k, v, dt, log_alpha, beta, pool, idx, o, N, T, H, Dk,
                                      Dv, P, fz, stream);
  const int nsm = num_sms_cached();
  if (nsm <= 0) return cudaErrorUnknown;
  const int grid = (int)(heads < nsm ? heads : nsm);
  // d = 128: the column layout, when its per-item buffers fit beside the two stages
  const size_t smem_cols = (size_t)kRsStages * lay.stage_bytes +
                           2 * (size_t)kRsMaxT * kRcD * sizeof(float) + kRsMaxT * sizeof(float4) +
                           2 * (kRsMaxT + 2) * sizeof(float) + 2 * kRsStages * sizeof(uint64_t) +
                           (kRcD + 4) * sizeof(float) + 128;
  if (Dk == kRcD && Dv == kRcD && (!fz.ow || al16(fz.ow)) && smem_cols <= 227u * 1024u) {
    ProfileScope prof(fused ? "recurrent_cols_fused" : "recurrent_cols", stream);
    if (dt == KDA_DTYPE_BF16)
      return fused ? launch_rc_typed<__nv_bfloat16, true>(q, k, v, log_alpha, beta, pool, idx, o,
                                                          (int)heads, T, H, P, lay, grid,
                                                          smem_cols, fz, stream)
                   : launch_rc_typed<__nv_bfloat16, false>(q, k, v, log_alpha, beta, pool, idx,
                                                           o, (int)heads, T, H, P, lay, grid,
                                                           smem_cols, fz, stream);
    return fused ? launch_rc_typed<float, true>(q, k, v, log_alpha, beta, pool, idx, o,
                                                (int)heads, T, H, P, lay, grid, smem_cols, fz,
                                                stream)
                 : launch_rc_typed<float, false>(q, k, v, log_alpha, beta, pool, idx, o,
                                                 (int)heads, T, H, P, lay, grid, smem_cols, fz,
                                                 stream);
  }
  ProfileScope prof(fused ? "recurrent_stream_fused" : "recurrent_stream", stream);
  if (dt == KDA_DTYPE_BF16)
    return fused ? launch_rs_typed<__nv_bfloat16, true>(q, k, v, log_alpha, beta, pool, idx, o,
                                                        (int)heads, T, H, Dk, Dv, P, lay, grid,
                                                        smem, fz, stream)
                 : launch_rs_typed<__nv_bfloat16, false>(q, k, v, log_alpha, beta, pool, idx, o,
                                                         (int)heads, T, H, Dk, Dv, P, lay, grid,
                                                         smem, fz, stream);
  return fused ? launch_rs_typed<float, true>(q, k, v, log_alpha, beta, pool, idx, o, (int)heads,
                                              T, H, Dk, Dv, P, lay, grid, smem, fz, stream)
               : launch_rs_typed<float, false>(q, k, v, log_alpha, beta, pool, idx, o,
                                               (int)heads, T, H, Dk, Dv, P, lay, grid, smem, fz,
                                               stream);
}

template <typename Tin, bool kFused>
static cudaError_t launch_stream_typed(const void* q, const void* k, const void* v,
                                       const float* log_alpha, const float* beta, float* state,
                                       void* o, int heads, int Dk, int Dv, const DsLayout& lay,
                                       int grid, size_t smem, int H, const Fusion& fz,
                                       cudaStream_t stream) {
  cudaError_t err = cudaFuncSetAttribute(decode_stream_kernel<Tin, kFused>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (err != cudaSuccess) return err;
  decode_stream_kernel<Tin, kFused><<<grid, kDsThreads, smem, stream>>>(
      (const Tin*)q, (const Tin*)k, (const Tin*)v, log_alpha, beta, state, (Tin*)o, heads, Dk,
      Dv, lay, H, fz);
  return cudaGetLastError();
}

cudaError_t launch_decode_step(const void* q, const void* k, const void* v, kda_dtype_t dt,
                               const float* log_alpha, const float* beta, float* state, void* o,
                               int N, int H, int Dk, int Dv, const Fusion* fz,
                               cudaStream_t stream) {
  const long long heads = (long long)N * H;
  if (heads == 0) return cudaSuccess;
  const int es = dt == KDA_DTYPE_BF16 ? 2 : 4;
  auto al16 = [](const void* p) { return ((uintptr_t)p & 15u) == 0; };
  const bool streamable = (Dk * es) % 16 == 0 && (Dv * es) % 16 == 0 && (Dk * 4) % 16 == 0 &&
                          al16(q) && al16(k) && al16(v) && al16(log_alpha) && al16(state) &&
                          (!fz || ((!fz->onorm || !fz->og || al16(fz->og)) &&
                                   (!fz->A_log || !fz->dt_bias || al16(fz->dt_bias))));
  if (fz && !streamable)  // the fused step on other shapes: the token-by-token kernel with T = 1
    return launch_recurrent_multi(q, k, v, dt, log_alpha, beta, state, nullptr, o, N, 1, H, Dk,
                                  Dv, N, *fz, stream);
  if (streamable) {
    const int nsm = num_sms_cached();
    if (nsm <= 0) return cudaErrorUnknown;
    const DsLayout lay = make_ds_layout(Dk, Dv, es, fz && fz->onorm && fz->og,
                                        fz && fz->A_log && fz->dt_bias);
    const size_t smem = (size_t)kDsStages * lay.stage_bytes + 2 * 8 * 32 * sizeof(float4) +
                        24 * sizeof(float) + 2 * kDsStages * sizeof(uint64_t) + 128;
    const int grid = (int)(heads < nsm ? heads : nsm);
    const Fusion none;
    ProfileScope prof(fz ? "decode_stream_fused" : "decode_stream", stream);
    if (dt == KDA_DTYPE_BF16)
      return fz ? launch_stream_typed<__nv_bfloat16, true>(q, k, v, log_alpha, beta, state, o,
                                                           (int)heads, Dk, Dv, lay, grid, smem,
                                                           H, *fz, stream)
                : launch_stream_typed<__nv_bfloat16, false>(q, k, v, log_alpha, beta, state, o,
                                                            (int)heads, Dk, Dv, lay, grid, smem,
                                                            H, none, stream);
    return fz ? launch_stream_typed<float, true>(q, k, v, log_alpha, beta, state, o, (int)heads,
                                                 Dk, Dv, lay, grid, smem, H, *fz, stream)
              : launch_stream_typed<float, false>(q, k, v, log_alpha, beta, state, o,
                                                  (int)heads, Dk, Dv, lay, grid, smem, H, none,
                                                  stream);
  }
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
