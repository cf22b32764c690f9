// kda_chunk_bwd.cu — backward pass of the chunkwise KDA operator (fp32 arithmetic, CUDA cores).
//
// Reverse-mode derivative of the chunk form of "Kimi Linear: An Expressive, Efficient Attention
// Architecture" (paper-graph-ui walkthrough, §3.4 "Chunkwise Parallelization": the UT transform,
// Eq. 8 and Eq. 9), for gradients of L = <dO, O> + <dS_T, S_T>. Per chunk, with the chunk-start
// state S, the notation of the forward kernels (g cumulative log decay, Qt = Gamma.Q,
// Kt = (gamma_C / gamma_i) k_i, P = Tril((Gamma.Q)(K/Gamma)^T), A = StrictTril(Diag(beta) B),
// B = (Gamma.K)(K/Gamma)^T, T = (I + A)^{-1}, M = T Diag(beta), W = M Gamma.K, U = M V,
// V' = U - W S) and dS' the cotangent of the state leaving the chunk:
//
//   state pass, sequential over chunks backwards (chunk_state_bwd):
//       dV' = P^T dO + Kt dS'          dS = Qt^T dO + Diag(gamma_C) dS' - W^T dV'
//   chunk-local pass, all chunks in parallel (chunk_local_bwd):
//       dQt = dO S^T    dW = -dV' S^T    dKt = V' dS'^T    dgamma_C = rowsum(dS' . S)
//       dP = Tril(dO V'^T)               dM = Tril(dW (Gamma.K)^T + dV' V^T)
//       dbeta += colsum(dM . T)          dT = dM Diag(beta)     dA = -StrictTril(T^T dT T^T)
//       dbeta += rowsum(dA . B)          d(Gamma.K) = M^T dW     dV = M^T dV'
//   and the products through A and P are differentiated in ratio form, exp(g_r - g_i) <= 1 for
//   i <= r, so no factor overflows for any decay:
//       dk_r += sum_i dA_ri beta_r k_i e_ri      dk_i += sum_r (dA_ri beta_r k_r + dP_ri q_r) e_ri
//       dq_r += sum_i dP_ri k_i e_ri             dg_r += s_ri,  dg_i -= s_ri,
//       s_ri = (dA_ri beta_r k_r + dP_ri q_r) k_i e_ri     (per key channel, elementwise)
//   then the elementwise maps of Qt, Gamma.K, Kt, gamma_C onto q, k, g, and d log_alpha as the
//   reverse cumulative sum of dg inside the chunk.
//
// The forward quantities come from the fp32 chunk kernels run first (records with T and B, and
// the state entering every chunk). The backward pass uses chunks of 32 tokens whatever the
// forward pass used (the result does not depend on the chunk size).
#include "kda_common.cuh"
#include "kda_internal.h"
#include "kda_items.cuh"

namespace kda {

constexpr int kBwdThreads = 256;
constexpr int kBwSlice = 32;  // value columns per CTA of the state pass

__device__ __forceinline__ float4 ld4(const float* p) { return *reinterpret_cast<const float4*>(p); }
__device__ __forceinline__ void st4(float* p, float4 v) { *reinterpret_cast<float4*>(p) = v; }
__device__ __forceinline__ float dot4(float4 a, float4 b, float acc) {
  return fmaf(a.x, b.x, fmaf(a.y, b.y, fmaf(a.z, b.z, fmaf(a.w, b.w, acc))));
}
// acc += s b on packed pairs (each lane rounded as fmaf rounds it)
__device__ __forceinline__ void fma4(float s, float4 b, float4& acc) {
  const f32x2 ss = f2_pack(s, s);
  const float2 lo = f2_unpack(f2_fma(ss, f2_pack(b.x, b.y), f2_pack(acc.x, acc.y)));
  const float2 hi = f2_unpack(f2_fma(ss, f2_pack(b.z, b.w), f2_pack(acc.z, acc.w)));
  acc = make_float4(lo.x, lo.y, hi.x, hi.y);
}


// ----------------------------------------------------------------------------------------------
// state pass: one CTA per (sequence, head, 32-column slice of d_v), chunks in reverse order
// ----------------------------------------------------------------------------------------------
constexpr int kBwdC = 32;  // chunk of the backward pass (both passes)
constexpr int kDoPerThread = kBwdC * kBwSlice / kBwdThreads;

// Each chunk step has two phases, dV' (reads Kt, P, dO, dS') and dS (reads Qt, W, gamma, dO, dV').
// The record sections are fetched with cp.async in two groups, each a phase ahead of its use:
// group A (W, Qt, gamma of chunk c) is issued when step c starts and lands during its dV' phase;
// group B (Kt, P of chunk c - 1) is issued when the dV' phase of step c ends and lands during its
// dS phase. The dO slice of chunk c - 1 is loaded into registers in the same place and stored to
// shared memory when step c - 1 starts. The chain then waits on global memory only at its start.
template <typename Tin>
__global__ void __launch_bounds__(kBwdThreads, 2)
    chunk_state_bwd_kernel(const float* __restrict__ ws, SimtRecord rec, SeqGeometry geo, int H,
                           int Dk, int Dv, const Tin* __restrict__ d_o,
                           const float* __restrict__ d_final, float* __restrict__ d_initial,
                           float* __restrict__ dstates, float* __restrict__ dvp) {
  extern __shared__ __align__(16) float smem[];
  constexpr int C = kBwdC;
  float* sdS = smem;                 // [Dk][32] cotangent of the state leaving the chunk
  float* sW = sdS + Dk * kBwSlice;   // [C][Dk]
  float* sKt = sW + C * Dk;          // [C][Dk]
  float* sQt = sKt + C * Dk;         // [C][Dk]
  float* sP = sQt + C * Dk;          // [C][C] P[r][i] (read for r >= i only)
  float* sGam = sP + C * C;          // [Dk]
  float* sdO = sGam + Dk;            // [C][32]
  float* sdV = sdO + C * kBwSlice;   // [C][32]

  if (!geo.ok()) return;
  const int n = blockIdx.x, h = blockIdx.y, j0 = blockIdx.z * kBwSlice;
  const int NV = min(kBwSlice, Dv - j0);
  const int tid = threadIdx.x, nt = blockDim.x;
  const size_t sbase = ((size_t)n * H + h) * Dk * Dv;
  const int tb = geo.seq_begin(n), te = geo.seq_end(n);
  const int c_first = geo.first_chunk(n);
  const int nchunks = te > tb ? ceil_div(te - tb, C) : 0;
#ifdef KDA_BOUNDS_CHECK
  {  // the chain's records, dO and dV' rows, cotangent slices and chunk-end cotangents
    const size_t rf = rec.record_floats, st = (size_t)Dk * Dv, rv = (size_t)H * Dv;
    const bool ok =
        rows_in_bounds(kBufWork, ws + h * rf, c_first, c_first + nchunks, H * rf, rf) &&
        rows_in_bounds(kBufDO, d_o + (size_t)h * Dv + j0, tb, te, rv, NV) &&
        rows_in_bounds(kBufWork, dvp + (size_t)h * Dv + j0, tb, te, rv, NV) &&
        rows_in_bounds(kBufWork, dstates + h * st, c_first, c_first + nchunks, H * st, st) &&
        (!d_final || rows_in_bounds(kBufDFinal, d_final + sbase + j0, 0, Dk, Dv, NV)) &&
        (!d_initial || rows_in_bounds(kBufDInitial, d_initial + sbase + j0, 0, Dk, Dv, NV));
    if (!ok) return;  // (uniform: the whole CTA leaves)
  }
#endif

  // record sections are 16-byte aligned (d_k multiple of 4, C multiple of 16)
  auto record = [&](int c) { return ws + rec.record_floats * ((size_t)c * H + h); };
  auto issue_a = [&](int c) {
    const float* r_ = record(c);
    for (int idx = tid; idx < C * Dk / 4; idx += nt) {
      cp_async_16B(sW + 4 * idx, r_ + rec.off_w + 4 * idx);
      cp_async_16B(sQt + 4 * idx, r_ + rec.off_qt + 4 * idx);
    }
    for (int idx = tid; idx < Dk / 4; idx += nt) cp_async_16B(sGam + 4 * idx, r_ + rec.off_gam + 4 * idx);
    cp_async_commit();
  };
  auto issue_b = [&](int c) {
    const float* r_ = record(c);
    for (int idx = tid; idx < C * Dk / 4; idx += nt)
      cp_async_16B(sKt + 4 * idx, r_ + rec.off_kt + 4 * idx);
    for (int idx = tid; idx < C * C / 4; idx += nt) cp_async_16B(sP + 4 * idx, r_ + rec.off_aqk + 4 * idx);
    cp_async_commit();
  };
  float dnext[kDoPerThread];  // the dO slice of the next chunk (element tid + m * nt)
  auto load_do = [&](int ci) {
    const int t0 = tb + ci * C, L = min(C, te - t0);
#pragma unroll
    for (int m = 0; m < kDoPerThread; ++m) {
      const int idx = tid + m * kBwdThreads, r = idx / kBwSlice, jj = idx - r * kBwSlice;
      dnext[m] = (r < L && jj < NV)
                     ? to_f32(d_o[((size_t)(t0 + r) * H + h) * Dv + j0 + jj])
                     : 0.f;
    }
  };

  for (int idx = tid; idx < Dk * kBwSlice; idx += nt) {
    const int a = idx / kBwSlice, jj = idx - a * kBwSlice;
    sdS[idx] = (d_final && jj < NV) ? d_final[sbase + (size_t)a * Dv + j0 + jj] : 0.f;
  }
  if (nchunks > 0) {
    issue_b(c_first + nchunks - 1);
    load_do(nchunks - 1);
  }
  __syncthreads();
  for (int ci = nchunks - 1; ci >= 0; --ci) {
    const int c = c_first + ci;
    const int t0 = tb + ci * C;
    const int L = min(C, te - t0);
#pragma unroll
    for (int m = 0; m < kDoPerThread; ++m) sdO[tid + m * kBwdThreads] = dnext[m];
    issue_a(c);
    {  // the cotangent entering from the right of this chunk, for the chunk-local pass
      float* dst = dstates + ((size_t)c * H + h) * Dk * Dv;
      for (int idx = tid; idx < Dk * kBwSlice / 4; idx += nt) {
        const int a = idx / (kBwSlice / 4), q = idx - a * (kBwSlice / 4);
        if (4 * q < NV)
          *reinterpret_cast<float4*>(dst + (size_t)a * Dv + j0 + 4 * q) =
              reinterpret_cast<const float4*>(sdS)[idx];
      }
    }
    cp_async_wait<1>();  // group B of this chunk has landed (group A may be in flight)
    __syncthreads();
    // dV'[i][j] = sum_r P[r][i] dO[r][j] + sum_a Kt[i][a] dS'[a][j] (P[r][i] = 0 for r < i):
    // 2 x 4 tiles (rows i0, i0 + 1; columns 4 jq .. 4 jq + 3), the d_k part split between the two
    // thread halves
    {
      const float4* Kt4 = reinterpret_cast<const float4*>(sKt);
      const float4* S4 = reinterpret_cast<const float4*>(sdS);  // [Dk][8]
      const float4* O4 = reinterpret_cast<const float4*>(sdO);  // [C][8]
      constexpr int split = 64 / C;
      const int dq = Dk >> 2;
      const int ip = (tid >> 3) % (C >> 1), jq = tid & 7, sp = tid / (4 * C);
      const int i0 = 2 * ip, i1 = i0 + 1;
      static_assert(split == 2, "the dV' phase splits its d_k part between two thread halves");
      // the first half also runs the A_qk part (about C / 5 float4 groups' worth of work), so it
      // takes that many fewer d_k groups
      const int qs = max(0, (dq - C / 5) / 2), q0 = sp == 0 ? 0 : qs, q1 = sp == 0 ? qs : dq;
      float4 acc[2] = {make_float4(0.f, 0.f, 0.f, 0.f), make_float4(0.f, 0.f, 0.f, 0.f)};
      for (int q = q0; q < q1; ++q) {
        const float4 x0 = Kt4[i0 * dq + q], x1 = Kt4[i1 * dq + q];
        const float xa[4] = {x0.x, x0.y, x0.z, x0.w}, xb[4] = {x1.x, x1.y, x1.z, x1.w};
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const float4 sv = S4[(4 * q + k) * 8 + jq];
          fma4(xa[k], sv, acc[0]);
          fma4(xb[k], sv, acc[1]);
        }
      }
      if (sp == 0) {  // the A_qk part (contraction over the chunk rows r >= i)
        for (int r = i0; r < C; ++r) {
          const float4 ov = O4[r * 8 + jq];
          fma4(sP[r * C + i0], ov, acc[0]);
          if (r >= i1) fma4(sP[r * C + i1], ov, acc[1]);
        }
      }
      float4* sRed = reinterpret_cast<float4*>(sdV + C * kBwSlice);  // [split][C][8]
      if (split > 1) {
        sRed[(sp * C + i0) * 8 + jq] = acc[0];
        sRed[(sp * C + i1) * 8 + jq] = acc[1];
        __syncthreads();
        if (sp == 0)
          for (int s2 = 1; s2 < split; ++s2)
#pragma unroll
            for (int u = 0; u < 2; ++u) {
              const float4 p = sRed[(s2 * C + i0 + u) * 8 + jq];
              acc[u].x += p.x; acc[u].y += p.y; acc[u].z += p.z; acc[u].w += p.w;
            }
      }
      if (sp == 0) {
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          const int i = i0 + u;
          const float4 val = acc[u];
          reinterpret_cast<float4*>(sdV)[i * 8 + jq] = val;
          if (i < L && 4 * jq < NV)
            *reinterpret_cast<float4*>(dvp + ((size_t)(t0 + i) * H + h) * Dv + j0 + 4 * jq) = val;
        }
      }
    }
    __syncthreads();  // dV' complete; Kt and P are free for the next chunk
    if (ci > 0) {
      issue_b(c - 1);
      load_do(ci - 1);
      cp_async_wait<1>();  // group A of this chunk has landed
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();
    // dS = Qt^T dO + Diag(gamma_C) dS' - W^T dV': 4 x 4 tiles (rows 4 aq .. 4 aq + 3), each
    // thread rewrites only its own tile
    {
      const float4* Q4 = reinterpret_cast<const float4*>(sQt);
      const float4* W4 = reinterpret_cast<const float4*>(sW);
      const float4* O4 = reinterpret_cast<const float4*>(sdO);
      const float4* V4 = reinterpret_cast<const float4*>(sdV);
      float4* S4 = reinterpret_cast<float4*>(sdS);
      const int dq = Dk >> 2;
      for (int t = tid; t < dq * 8; t += nt) {
        const int aq = t >> 3, jq = t & 7;
        float4 acc[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float g = sGam[4 * aq + e];
          const float4 sv = S4[(4 * aq + e) * 8 + jq];
          acc[e] = make_float4(g * sv.x, g * sv.y, g * sv.z, g * sv.w);
        }
        for (int r = 0; r < C; ++r) {
          const float4 qv = Q4[r * dq + aq], wv = W4[r * dq + aq];
          const float4 ov = O4[r * 8 + jq], dv = V4[r * 8 + jq];
          const float qx[4] = {qv.x, qv.y, qv.z, qv.w}, wx[4] = {wv.x, wv.y, wv.z, wv.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            fma4(qx[e], ov, acc[e]);
            fma4(-wx[e], dv, acc[e]);
          }
        }
#pragma unroll
        for (int e = 0; e < 4; ++e) S4[(4 * aq + e) * 8 + jq] = acc[e];
      }
    }
    __syncthreads();  // dS complete; W, Qt, gamma and dO are free
  }
  if (d_initial) {
    for (int idx = tid; idx < Dk * kBwSlice; idx += nt) {
      const int a = idx / kBwSlice, jj = idx - a * kBwSlice;
      if (jj < NV) d_initial[sbase + (size_t)a * Dv + j0 + jj] = sdS[idx];
    }
  }
}

// ----------------------------------------------------------------------------------------------
// chunk-local pass: one CTA per (chunk, head); chunk = 32 tokens
// ----------------------------------------------------------------------------------------------

// Shared-memory rows are padded by four floats (ld = D + 4): rows stay 16-byte aligned for
// float4 accesses, and consecutive rows start 4 banks apart. The products are register-tiled:
// a thread owns output rows {tm, tm + 16} and, along the other dimension, either columns
// {tn, tn + 16} (contractions over d_k / d_v of two row-major operands, float4 along the
// contraction) or two float4 column groups {4 tn .. 4 tn + 3, 64 + 4 tn .. 64 + 4 tn + 3}
// (contractions over the chunk rows). Requires Dk, Dv multiples of 4.
struct BwdSmem {  // float offsets of the chunk-local pass (C = 32)
  int ldk, ldv, ldm, ldc;
  int K, Q, G, V, dO, dV, X1, X2, X3, X4, Y1, Y2, T, B, dP, dM, X, beta, dgam, db, total;
  __host__ __device__ static BwdSmem make(int Dk, int Dv) {
    const int C = kBwdC, Dm = Dk > Dv ? Dk : Dv;
    BwdSmem s;
    s.ldk = Dk + 4;
    s.ldv = Dv + 4;
    s.ldm = Dm + 4;
    s.ldc = C + 4;
    int o = 0;
    s.K = o; o += C * s.ldk;
    s.Q = o; o += C * s.ldk;
    s.G = o; o += C * s.ldk;
    s.V = o; o += C * s.ldv;
    s.dO = o; o += C * s.ldv;
    s.dV = o; o += C * s.ldv;
    s.X1 = o; o += C * s.ldm;   // V' (ldv), then dg (ldk)
    s.X2 = o; o += C * s.ldk;   // dQt, then dq
    s.X3 = o; o += C * s.ldk;   // dW, then dk
    s.X4 = o; o += C * s.ldk;   // W, then dKt
    s.Y1 = o; o += C * s.ldm;   // chunk-start state rows (ldv), then Gamma.K (ldk)
    s.Y2 = o; o += C * s.ldm;   // cotangent rows (ldv), then d(Gamma.K) (ldk)
    s.T = o; o += C * s.ldc;
    s.B = o; o += C * s.ldc;
    s.dP = o; o += C * s.ldc;
    s.dM = o; o += C * s.ldc;   // dM, then dT, then dA
    s.X = o; o += C * s.ldc;
    s.beta = o; o += C;
    s.dgam = o; o += Dk;
    s.db = o; o += C;
    s.total = o;
    return s;
  }
};

// A [kBwdC][D] tile of Tin rows (row r at src + r * stride; rows >= L read as zeros; D <= 128 a
// multiple of kPer; 16-byte aligned rows) moved into fp32 shared-memory rows as 16-byte vectors:
// load() issues every load of the thread, store() converts them once they have been issued.
template <typename Tin>
struct RowVec {
  static constexpr int kPer = 16 / sizeof(Tin);                    // elements per vector
  static constexpr int kMax = kBwdC * 128 / kPer / kBwdThreads;  // vectors per thread
  uint4 x[kMax];
  __device__ __forceinline__ void load(const Tin* src, size_t stride, int L, int D) {
    const int vpr = D / kPer;
#pragma unroll
    for (int m = 0; m < kMax; ++m) {
      const int idx = threadIdx.x + m * kBwdThreads, r = idx / vpr, c = idx - r * vpr;
      x[m] = r < L ? __ldg(reinterpret_cast<const uint4*>(src + r * stride + c * kPer))
                   : make_uint4(0u, 0u, 0u, 0u);
    }
  }
  __device__ __forceinline__ void store(float* dst, int ld, int D) const {
    const int vpr = D / kPer;
#pragma unroll
    for (int m = 0; m < kMax; ++m) {
      const int idx = threadIdx.x + m * kBwdThreads, r = idx / vpr, c = idx - r * vpr;
      if (r < kBwdC) store_vec(dst + r * ld + c * kPer, x[m], Tin());
    }
  }
};

// Factored ratio-form sums of one key channel over the rows r = kParity, kParity + 2, ... of the
// chunk (i <= r; dA and dP are zero for i >= r and i > r, so whole float4 groups are read):
//   row r:     s1 = sum_i dA_ri kF_i, s2 = sum_i dP_ri kF_i  ->  dk_r += beta_r E_r s1,
//              dq_r += E_r s2, dg_r += beta_r k_r E_r s1 + q_r E_r s2
//   column i:  cacc_i += dA_ri beta_r k_r E_r + dP_ri q_r E_r   (scaled by F_i by the caller)
// with e_ri = E_r F_i, E_r = exp(g_r - m), F_i = exp(m - g_i), kF_i = k_i F_i.
template <int kParity>
__device__ __forceinline__ void ratio_rows(const float* sdA, const float* sdP, int ldc,
                                           const float* sK, const float* sQ, const float* sG,
                                           const float* sbeta, int ldk, int a, float m,
                                           const float (&kF)[kBwdC], float (&cacc)[kBwdC],
                                           float* dk, float* dq, float* dg) {
#pragma unroll
  for (int r = kParity; r < kBwdC; r += 2) {
    const float Er = expf(sG[r * ldk + a] - m);
    const float bE = sbeta[r] * Er;
    const float bkE = bE * sK[r * ldk + a], qE = sQ[r * ldk + a] * Er;
    float s1 = 0.f, s2 = 0.f;
#pragma unroll
    for (int i4 = 0; i4 <= r / 4; ++i4) {
      const float4 da = ld4(sdA + r * ldc + 4 * i4), dp = ld4(sdP + r * ldc + 4 * i4);
      const float xa[4] = {da.x, da.y, da.z, da.w}, xp[4] = {dp.x, dp.y, dp.z, dp.w};
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int i = 4 * i4 + u;
        s1 = fmaf(xa[u], kF[i], s1);
        s2 = fmaf(xp[u], kF[i], s2);
        cacc[i] = fmaf(xa[u], bkE, fmaf(xp[u], qE, cacc[i]));
      }
    }
    dk[r * ldk + a] += bE * s1;
    dq[r * ldk + a] += Er * s2;
    dg[r * ldk + a] += bkE * s1 + qE * s2;
  }
}

// acc[u][w] += sum_{k < K} X[(tm + 16u) * ldx + k] * Y[(tn + 16w) * ldy + k]  (K multiple of 4),
// on packed pairs: the even and the odd k are summed apart and added at the end
__device__ __forceinline__ void abt_2x2(const float* X, int ldx, const float* Y, int ldy, int K,
                                        int tm, int tn, float (&acc)[2][2]) {
  const float* x0 = X + tm * ldx;
  const float* x1 = X + (tm + 16) * ldx;
  const float* y0 = Y + tn * ldy;
  const float* y1 = Y + (tn + 16) * ldy;
  f32x2 p[2][2];
#pragma unroll
  for (int u = 0; u < 2; ++u)
#pragma unroll
    for (int w = 0; w < 2; ++w) p[u][w] = f2_pack(0.f, 0.f);
  for (int k = 0; k < K; k += 4) {
    const float4 a0 = ld4(x0 + k), a1 = ld4(x1 + k), b0 = ld4(y0 + k), b1 = ld4(y1 + k);
    const f32x2 al[2] = {f2_pack(a0.x, a0.y), f2_pack(a1.x, a1.y)};
    const f32x2 ah[2] = {f2_pack(a0.z, a0.w), f2_pack(a1.z, a1.w)};
    const f32x2 bl[2] = {f2_pack(b0.x, b0.y), f2_pack(b1.x, b1.y)};
    const f32x2 bh[2] = {f2_pack(b0.z, b0.w), f2_pack(b1.z, b1.w)};
#pragma unroll
    for (int u = 0; u < 2; ++u)
#pragma unroll
      for (int w = 0; w < 2; ++w) p[u][w] = f2_fma(ah[u], bh[w], f2_fma(al[u], bl[w], p[u][w]));
  }
#pragma unroll
  for (int u = 0; u < 2; ++u)
#pragma unroll
    for (int w = 0; w < 2; ++w) {
      const float2 v = f2_unpack(p[u][w]);
      acc[u][w] += v.x + v.y;
    }
}

// Two products sharing the right operand: accA[u][w] += X1 row . Y row, accB[u][w] += X2 row .
// Y row, with abt_2x2's tiles and packed pairs (each Y row read once for both).
__device__ __forceinline__ void abt_2x2_dual(const float* XA, const float* XB, int ldx,
                                             const float* Y, int ldy, int K, int tm, int tn,
                                             float (&accA)[2][2], float (&accB)[2][2]) {
  const float* y0 = Y + tn * ldy;
  const float* y1 = Y + (tn + 16) * ldy;
  f32x2 pa[2][2], pb[2][2];
#pragma unroll
  for (int u = 0; u < 2; ++u)
#pragma unroll
    for (int w = 0; w < 2; ++w) pa[u][w] = pb[u][w] = f2_pack(0.f, 0.f);
  for (int k = 0; k < K; k += 4) {
    const float4 b0 = ld4(y0 + k), b1 = ld4(y1 + k);
    const f32x2 bl[2] = {f2_pack(b0.x, b0.y), f2_pack(b1.x, b1.y)};
    const f32x2 bh[2] = {f2_pack(b0.z, b0.w), f2_pack(b1.z, b1.w)};
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const float4 a = ld4(XA + (tm + 16 * u) * ldx + k), c = ld4(XB + (tm + 16 * u) * ldx + k);
      const f32x2 al = f2_pack(a.x, a.y), ah = f2_pack(a.z, a.w);
      const f32x2 cl = f2_pack(c.x, c.y), ch = f2_pack(c.z, c.w);
#pragma unroll
      for (int w = 0; w < 2; ++w) {
        pa[u][w] = f2_fma(ah, bh[w], f2_fma(al, bl[w], pa[u][w]));
        pb[u][w] = f2_fma(ch, bh[w], f2_fma(cl, bl[w], pb[u][w]));
      }
    }
  }
#pragma unroll
  for (int u = 0; u < 2; ++u)
#pragma unroll
    for (int w = 0; w < 2; ++w) {
      const float2 va = f2_unpack(pa[u][w]), vb = f2_unpack(pb[u][w]);
      accA[u][w] += va.x + va.y;
      accB[u][w] += vb.x + vb.y;
    }
}

template <typename Tin>
__global__ void __launch_bounds__(kBwdThreads, 1)
    chunk_local_bwd_kernel(const Tin* __restrict__ q, const Tin* __restrict__ k,
                           const Tin* __restrict__ v, const float* __restrict__ log_alpha,
                           const float* __restrict__ beta, SeqGeometry geo, int H, int Dk, int Dv,
                           const float* __restrict__ ws, SimtRecord rec,
                           const float* __restrict__ states, const float* __restrict__ dstates,
                           const float* __restrict__ dvp, const Tin* __restrict__ d_o,
                           Tin* __restrict__ dq, Tin* __restrict__ dk, Tin* __restrict__ dv,
                           float* __restrict__ dla, float* __restrict__ dbeta) {
  extern __shared__ __align__(16) float smem[];
  constexpr int C = kBwdC;
  const BwdSmem L_ = BwdSmem::make(Dk, Dv);
  const int ldk = L_.ldk, ldv = L_.ldv, ldc = L_.ldc;
  float* sK = smem + L_.K;
  float* sQ = smem + L_.Q;
  float* sG = smem + L_.G;
  float* sV = smem + L_.V;
  float* sdO = smem + L_.dO;
  float* sdV = smem + L_.dV;
  float* X1 = smem + L_.X1;
  float* X2 = smem + L_.X2;
  float* X3 = smem + L_.X3;
  float* X4 = smem + L_.X4;
  float* Y1 = smem + L_.Y1;
  float* Y2 = smem + L_.Y2;
  float* sT = smem + L_.T;
  float* sB = smem + L_.B;
  float* sdP = smem + L_.dP;
  float* sdM = smem + L_.dM;
  float* sX = smem + L_.X;
  float* sbeta = smem + L_.beta;
  float* sdgam = smem + L_.dgam;
  float* sdb = smem + L_.db;

  if (!geo.ok()) return;
  const ChunkItem item = chunk_item();
  const int c = item.c, h = item.h;
  if (c >= geo.num_chunks_total()) return;
  const int n = geo.seq_of_chunk(c);
  const int t0 = geo.seq_begin(n) + (c - geo.first_chunk(n)) * C;
  const int L = min(C, geo.seq_end(n) - t0);
  const int tid = threadIdx.x, nt = blockDim.x;
  const int tm = tid >> 4, tn = tid & 15;  // register-tile coordinates
  const float* r_ = ws + rec.record_floats * ((size_t)c * H + h);
  const float* S0 = states + ((size_t)c * H + h) * Dk * Dv;   // state entering the chunk
  const float* dS1 = dstates + ((size_t)c * H + h) * Dk * Dv; // cotangent of the state leaving it
  const int Dv4 = Dv >> 2;
#ifdef KDA_BOUNDS_CHECK
  {  // every access of the item lies in its record and states and in rows t0 .. t0 + L - 1
    const size_t rk = (size_t)H * Dk, rv = (size_t)H * Dv, hk = (size_t)h * Dk, hv = (size_t)h * Dv;
    const bool ok =
        in_bounds(kBufWork, r_, rec.record_floats * sizeof(float)) &&
        in_bounds(kBufWork, S0, (size_t)Dk * Dv * 4) && in_bounds(kBufWork, dS1, (size_t)Dk * Dv * 4) &&
        rows_in_bounds(kBufWork, dvp + hv, t0, t0 + L, rv, Dv) &&
        rows_in_bounds(kBufQ, q + hk, t0, t0 + L, rk, Dk) &&
        rows_in_bounds(kBufK, k + hk, t0, t0 + L, rk, Dk) &&
        rows_in_bounds(kBufV, v + hv, t0, t0 + L, rv, Dv) &&
        rows_in_bounds(kBufLogAlpha, log_alpha + hk, t0, t0 + L, rk, Dk) &&
        rows_in_bounds(kBufBeta, beta + h, t0, t0 + L, H, 1) &&
        rows_in_bounds(kBufDO, d_o + hv, t0, t0 + L, rv, Dv) &&
        rows_in_bounds(kBufDQ, dq + hk, t0, t0 + L, rk, Dk) &&
        rows_in_bounds(kBufDK, dk + hk, t0, t0 + L, rk, Dk) &&
        rows_in_bounds(kBufDV, dv + hv, t0, t0 + L, rv, Dv) &&
        rows_in_bounds(kBufDLogAlpha, dla + hk, t0, t0 + L, rk, Dk) &&
        rows_in_bounds(kBufDBeta, dbeta + h, t0, t0 + L, H, 1);
    if (!ok) return;  // (uniform: the whole CTA leaves)
  }
#endif

  // ---- P0: inputs, record, cumulative decay. With 16-byte aligned input rows every copy is
  // issued before any is used: the record, dV' and log_alpha by cp.async, the Tin inputs as
  // 16-byte vectors converted once all are in flight (the record and dV' rows are always aligned).
  const bool vec = ((reinterpret_cast<uintptr_t>(q) | reinterpret_cast<uintptr_t>(k) |
                     reinterpret_cast<uintptr_t>(v) | reinterpret_cast<uintptr_t>(d_o) |
                     reinterpret_cast<uintptr_t>(log_alpha)) & 15) == 0 &&
                   Dk % RowVec<Tin>::kPer == 0 && Dv % RowVec<Tin>::kPer == 0;
  if (vec) {
    const size_t rowk = (size_t)H * Dk, rowv = (size_t)H * Dv;  // token strides
    const size_t bk = ((size_t)t0 * H + h) * Dk, bv = ((size_t)t0 * H + h) * Dv;
    const float4 zero4 = make_float4(0.f, 0.f, 0.f, 0.f);
    RowVec<Tin> xk, xq, xv, xo;
    xk.load(k + bk, rowk, L, Dk);
    xq.load(q + bk, rowk, L, Dk);
    xv.load(v + bv, rowv, L, Dv);
    xo.load(d_o + bv, rowv, L, Dv);
    for (int idx = tid; idx < C * (Dk / 4); idx += nt) {
      const int r = idx / (Dk / 4), a = 4 * (idx - r * (Dk / 4));
      cp_async_16B(X4 + r * ldk + a, r_ + rec.off_w + r * Dk + a);
      if (r < L)
        cp_async_16B(sG + r * ldk + a, log_alpha + bk + r * rowk + a);
      else
        st4(sG + r * ldk + a, zero4);
    }
    for (int idx = tid; idx < C * (Dv / 4); idx += nt) {
      const int r = idx / (Dv / 4), jj = 4 * (idx - r * (Dv / 4));
      if (r < L)
        cp_async_16B(sdV + r * ldv + jj, dvp + bv + r * rowv + jj);
      else
        st4(sdV + r * ldv + jj, zero4);
    }
    for (int idx = tid; idx < C * (C / 4); idx += nt) {
      const int r = idx / (C / 4), i = 4 * (idx - r * (C / 4));
      cp_async_16B(sT + r * ldc + i, r_ + rec.off_t + r * C + i);
      cp_async_16B(sB + r * ldc + i, r_ + rec.off_b + r * C + i);
    }
    cp_async_commit();
    xk.store(sK, ldk, Dk);
    xq.store(sQ, ldk, Dk);
    xv.store(sV, ldv, Dv);
    xo.store(sdO, ldv, Dv);
    cp_async_wait<0>();
  } else {
    for (int idx = tid; idx < C * Dk; idx += nt) {
      const int r = idx / Dk, a = idx - r * Dk;
      const bool in = r < L;
      const size_t gi = ((size_t)(t0 + r) * H + h) * Dk + a;
      sK[r * ldk + a] = in ? to_f32(k[gi]) : 0.f;
      sQ[r * ldk + a] = in ? to_f32(q[gi]) : 0.f;
      sG[r * ldk + a] = in ? log_alpha[gi] : 0.f;
      X4[r * ldk + a] = r_[rec.off_w + idx];
    }
    for (int idx = tid; idx < C * Dv; idx += nt) {
      const int r = idx / Dv, jj = idx - r * Dv;
      const bool in = r < L;
      const size_t gi = ((size_t)(t0 + r) * H + h) * Dv + jj;
      sV[r * ldv + jj] = in ? to_f32(v[gi]) : 0.f;
      sdO[r * ldv + jj] = in ? to_f32(d_o[gi]) : 0.f;
      sdV[r * ldv + jj] = in ? dvp[gi] : 0.f;
    }
    for (int idx = tid; idx < C * C; idx += nt) {
      const int r = idx / C, i = idx - r * C;
      sT[r * ldc + i] = r_[rec.off_t + idx];
      sB[r * ldc + i] = r_[rec.off_b + idx];
    }
  }
  for (int r = tid; r < C; r += nt) sbeta[r] = r < L ? beta[(size_t)(t0 + r) * H + h] : 0.f;
  __syncthreads();
  for (int a = tid; a < Dk; a += nt) {
    float acc = 0.f;
    for (int r = 0; r < C; ++r) {
      acc += sG[r * ldk + a];
      sG[r * ldk + a] = acc;
    }
  }

  // ---- P1: products with the chunk-start state S, its rows streamed in slices of 32: slice s of
  // S in Y1 / Y2 alternately and of dS' in X1 (free until V' is stored), slice s + 1 fetched while
  // slice s is used; the last step fetches P2's first slice of dS' instead.
  // V' = U - W S: this thread's rows {tm, tm + 16}, column groups {4 tn, 64 + 4 tn}
  float4 vp[2][2];
#pragma unroll
  for (int u = 0; u < 2; ++u)
#pragma unroll
    for (int w = 0; w < 2; ++w) {
      const int j = 4 * tn + 64 * w;
      vp[u][w] = j < Dv ? ld4(r_ + rec.off_u + (tm + 16 * u) * Dv + j)
                        : make_float4(0.f, 0.f, 0.f, 0.f);
    }
  const int nsl = (Dk + 31) / 32;
  auto sbuf = [&](int i) { return (i & 1) ? Y2 : Y1; };  // the two slice buffers
  auto fetch_rows = [&](float* dst, const float* src, int a0) {  // (state rows: 16-byte aligned)
    const int na = min(32, Dk - a0);
    for (int idx = tid; idx < na * Dv4; idx += nt) {
      const int aa = idx / Dv4, j4 = idx - aa * Dv4;
      cp_async_16B(dst + aa * ldv + 4 * j4, src + (size_t)(a0 + aa) * Dv + 4 * j4);
    }
  };
  fetch_rows(Y1, S0, 0);
  fetch_rows(X1, dS1, 0);
  cp_async_commit();
  for (int sl = 0; sl < nsl; ++sl) {
    const int a0 = 32 * sl, na = min(32, Dk - a0);
    const float* Ys = sbuf(sl);
    cp_async_wait<0>();
    __syncthreads();  // slice sl landed; slice sl - 1 consumed (the first time: the cumsum done)
    {  // dgamma_C = rowsum(dS' . S): eight lanes per row, each over every eighth float4
      const int aa = tid >> 3, part = tid & 7;
      float s = 0.f;
      if (aa < na)
        for (int j = 4 * part; j < Dv; j += 32)
          s = dot4(ld4(X1 + aa * ldv + j), ld4(Ys + aa * ldv + j), s);
      s += __shfl_xor_sync(0xffffffffu, s, 1);
      s += __shfl_xor_sync(0xffffffffu, s, 2);
      s += __shfl_xor_sync(0xffffffffu, s, 4);
      if (aa < na && part == 0) sdgam[a0 + aa] = s;
    }
    __syncthreads();  // X1 and the other slice buffer are free
    if (sl + 1 < nsl) {
      fetch_rows(sbuf(sl + 1), S0, a0 + 32);
      fetch_rows(X1, dS1, a0 + 32);
    } else {
      fetch_rows(sbuf(sl + 1), dS1, 0);
    }
    cp_async_commit();
    for (int a4 = 0; a4 < na; a4 += 4) {  // (na is a multiple of 4)
      const float4 w04 = ld4(X4 + tm * ldk + a0 + a4), w14 = ld4(X4 + (tm + 16) * ldk + a0 + a4);
      const float w0s[4] = {w04.x, w04.y, w04.z, w04.w}, w1s[4] = {w14.x, w14.y, w14.z, w14.w};
#pragma unroll
      for (int e = 0; e < 4; ++e)
#pragma unroll
        for (int w = 0; w < 2; ++w) {
          const int j = 4 * tn + 64 * w;
          if (j < Dv) {
            const float4 sv = ld4(Ys + (a4 + e) * ldv + j);
            fma4(-w0s[e], sv, vp[0][w]);
            fma4(-w1s[e], sv, vp[1][w]);
          }
        }
    }
    if (tn < na || tn + 16 < na) {  // dQt = dO S^T, dW = -dV' S^T over this slice's columns
      float a1[2][2] = {{0.f, 0.f}, {0.f, 0.f}}, a2[2][2] = {{0.f, 0.f}, {0.f, 0.f}};
      abt_2x2_dual(sdO, sdV, ldv, Ys, ldv, Dv, tm, tn, a1, a2);
#pragma unroll
      for (int u = 0; u < 2; ++u)
#pragma unroll
        for (int w = 0; w < 2; ++w) {
          const int aa = tn + 16 * w;
          if (aa < na) {
            X2[(tm + 16 * u) * ldk + a0 + aa] = a1[u][w];
            X3[(tm + 16 * u) * ldk + a0 + aa] = -a2[u][w];
          }
        }
    }
  }
#pragma unroll
  for (int u = 0; u < 2; ++u)
#pragma unroll
    for (int w = 0; w < 2; ++w) {
      const int j = 4 * tn + 64 * w;
      if (j < Dv) st4(X1 + (tm + 16 * u) * ldv + j, vp[u][w]);
    }
  // ---- P2: dKt = V' dS'^T over slices of dS' rows in the same two buffers, slice s + 1 fetched
  // while slice s is used (W is dead: its buffer takes dKt)
  for (int sl = 0; sl < nsl; ++sl) {
    const int a0 = 32 * sl, na = min(32, Dk - a0);
    const float* Ys = sbuf(nsl + sl);
    cp_async_wait<0>();
    __syncthreads();  // slice sl landed; V' stored; slice sl - 1 consumed
    if (sl + 1 < nsl) {
      fetch_rows(sbuf(nsl + sl + 1), dS1, a0 + 32);
      cp_async_commit();
    }
    if (tn < na || tn + 16 < na) {
      float acc[2][2] = {{0.f, 0.f}, {0.f, 0.f}};
      abt_2x2(X1, ldv, Ys, ldv, Dv, tm, tn, acc);
#pragma unroll
      for (int u = 0; u < 2; ++u)
#pragma unroll
        for (int w = 0; w < 2; ++w) {
          const int aa = tn + 16 * w;
          if (aa < na) X4[(tm + 16 * u) * ldk + a0 + aa] = acc[u][w];
        }
    }
  }
  __syncthreads();
  // ---- P3: C x C products
  for (int idx = tid; idx < C * Dk; idx += nt) {  // Gamma.K
    const int r = idx / Dk, a = idx - r * Dk;
    Y1[r * ldk + a] = sK[r * ldk + a] * expf(sG[r * ldk + a]);
  }
  {  // dP = Tril(dO V'^T)
    float acc[2][2] = {{0.f, 0.f}, {0.f, 0.f}};
    abt_2x2(sdO, ldv, X1, ldv, Dv, tm, tn, acc);
#pragma unroll
    for (int u = 0; u < 2; ++u)
#pragma unroll
      for (int w = 0; w < 2; ++w) {
        const int r = tm + 16 * u, i = tn + 16 * w;
        sdP[r * ldc + i] = i <= r ? acc[u][w] : 0.f;
      }
  }
  __syncthreads();
  {  // dM = Tril(dW (Gamma.K)^T + dV' V^T)
    float acc[2][2] = {{0.f, 0.f}, {0.f, 0.f}};
    abt_2x2(X3, ldk, Y1, ldk, Dk, tm, tn, acc);
    abt_2x2(sdV, ldv, sV, ldv, Dv, tm, tn, acc);
#pragma unroll
    for (int u = 0; u < 2; ++u)
#pragma unroll
      for (int w = 0; w < 2; ++w) {
        const int r = tm + 16 * u, i = tn + 16 * w;
        sdM[r * ldc + i] = i <= r ? acc[u][w] : 0.f;
      }
  }
  __syncthreads();
  for (int i = tid; i < C; i += nt) {  // dbeta from M = T Diag(beta)
    float s = 0.f;
    for (int r = i; r < C; ++r) s += sdM[r * ldc + i] * sT[r * ldc + i];
    sdb[i] = s;
  }
  __syncthreads();
  for (int idx = tid; idx < C * C; idx += nt) {  // dT
    const int r = idx / C, i = idx - r * C;
    sdM[r * ldc + i] *= sbeta[i];
  }
  __syncthreads();
  {  // X = dT T^T
    float acc[2][2] = {{0.f, 0.f}, {0.f, 0.f}};
    abt_2x2(sdM, ldc, sT, ldc, C, tm, tn, acc);
#pragma unroll
    for (int u = 0; u < 2; ++u)
#pragma unroll
      for (int w = 0; w < 2; ++w) sX[(tm + 16 * u) * ldc + tn + 16 * w] = acc[u][w];
  }
  __syncthreads();
  for (int idx = tid; idx < C * C; idx += nt) {  // dA = -StrictTril(T^T X)
    const int r = idx / C, i = idx - r * C;
    float s = 0.f;
    if (i < r)
      for (int p = r; p < C; ++p) s += sT[p * ldc + r] * sX[p * ldc + i];
    sdM[r * ldc + i] = -s;
  }
  __syncthreads();
  for (int r = tid; r < C; r += nt) {  // dbeta from A = StrictTril(Diag(beta) B)
    float s = 0.f;
    for (int i = 0; i < r; ++i) s += sdM[r * ldc + i] * sB[r * ldc + i];
    sdb[r] += s;
  }
  // ---- P4: d(Gamma.K) = M^T dW, dV = M^T dV' (rows {tm, tm + 16}, column groups)
  {
    float4 gk[2][2], gv[2][2];
#pragma unroll
    for (int u = 0; u < 2; ++u)
#pragma unroll
      for (int w = 0; w < 2; ++w)
        gk[u][w] = gv[u][w] = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int r = tm; r < C; ++r) {  // M[r][i] = 0 for r < i: rows below tm only
      const float m0 = sT[r * ldc + tm];
      const float m1 = r >= tm + 16 ? sT[r * ldc + tm + 16] : 0.f;
#pragma unroll
      for (int w = 0; w < 2; ++w) {
        const int a = 4 * tn + 64 * w;
        if (a < Dk) {
          const float4 x = ld4(X3 + r * ldk + a);
          fma4(m0, x, gk[0][w]);
          fma4(m1, x, gk[1][w]);
        }
        if (a < Dv) {
          const float4 x = ld4(sdV + r * ldv + a);
          fma4(m0, x, gv[0][w]);
          fma4(m1, x, gv[1][w]);
        }
      }
    }
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int i = tm + 16 * u;
      const float b = sbeta[i];
#pragma unroll
      for (int w = 0; w < 2; ++w) {
        const int a = 4 * tn + 64 * w;
        if (a < Dk)
          st4(Y2 + i * ldk + a, make_float4(gk[u][w].x * b, gk[u][w].y * b, gk[u][w].z * b,
                                            gk[u][w].w * b));
        if (a < Dv && i < L) {
          Tin* dst = dv + ((size_t)(t0 + i) * H + h) * Dv + a;
          dst[0] = from_f32<Tin>(gv[u][w].x * b);
          dst[1] = from_f32<Tin>(gv[u][w].y * b);
          dst[2] = from_f32<Tin>(gv[u][w].z * b);
          dst[3] = from_f32<Tin>(gv[u][w].w * b);
        }
      }
    }
  }
  __syncthreads();
  // ---- P5: elementwise maps of Qt, Gamma.K, Kt onto q, k, g
  for (int idx = tid; idx < C * Dk; idx += nt) {
    const int r = idx / Dk, a = idx - r * Dk;
    const int x = r * ldk + a;
    const float g = sG[x], e = expf(g), et = expf(sG[(C - 1) * ldk + a] - g);
    const float dqt = X2[x], dkg = Y2[x], dkt = X4[x];
    X1[x] = dqt * sQ[x] * e + dkg * Y1[x] - dkt * sK[x] * et;  // dg
    X2[x] = dqt * e;                                           // dq
    X3[x] = dkg * e + dkt * et;                                // dk
  }
  __syncthreads();
  // ratio-form products through A and P, per key channel, each pair (r >= i) weighed by
  // e_ri = exp(g_r - g_i) <= 1. When every channel's cumulative decay spans at most 2 x 40 nats
  // over the chunk, e_ri is taken as E_r F_i around the channel's midpoint m (every factor within
  // e^+-40, so each product keeps fp32 relative precision): two threads per channel (even and odd
  // rows), 64 exponentials per channel instead of one per pair, four FMAs per pair. Otherwise
  // threads [0, Dk) accumulate along rows (row r over i <= r) into the dk / dq / dg buffers and
  // threads [128, 128 + Dk) along columns (column i over r >= i), one exponential per pair.
  // Column sums go to the dead Gamma.K / d(Gamma.K) buffers either way.
  bool span_ok = true;
  float gmid = 0.f;
  if ((tid & 127) < Dk) {
    const int a = tid & 127;
    float gmin = sG[a], gmax = gmin;
    for (int r = 1; r < C; ++r) {
      const float g = sG[r * ldk + a];
      gmin = fminf(gmin, g);
      gmax = fmaxf(gmax, g);
    }
    span_ok = gmax - gmin <= 80.f;  // false for NaN or infinite decays
    gmid = 0.5f * (gmax + gmin);
  }
  if (__syncthreads_and(span_ok)) {
    const int a = tid & 127, half = tid >> 7;
    float F[C], kF[C], cacc[C];
    if (a < Dk) {
#pragma unroll
      for (int i = 0; i < C; ++i) {
        F[i] = expf(gmid - sG[i * ldk + a]);
        kF[i] = sK[i * ldk + a] * F[i];
        cacc[i] = 0.f;
      }
      if (half == 0)
        ratio_rows<0>(sdM, sdP, ldc, sK, sQ, sG, sbeta, ldk, a, gmid, kF, cacc, X3, X2, X1);
      else
        ratio_rows<1>(sdM, sdP, ldc, sK, sQ, sG, sbeta, ldk, a, gmid, kF, cacc, X3, X2, X1);
      if (half == 0) {
#pragma unroll
        for (int i = 0; i < C; ++i) {
          Y1[i * ldk + a] = F[i] * cacc[i];
          Y2[i * ldk + a] = -kF[i] * cacc[i];
        }
      }
    }
    __syncthreads();
    if (a < Dk && half == 1) {
#pragma unroll
      for (int i = 0; i < C; ++i) {
        Y1[i * ldk + a] += F[i] * cacc[i];
        Y2[i * ldk + a] -= kF[i] * cacc[i];
      }
    }
  } else if (tid < Dk) {
    const int a = tid;
    for (int r = 0; r < C; ++r) {
      const float kr = sK[r * ldk + a], qr = sQ[r * ldk + a], gr = sG[r * ldk + a];
      const float br = sbeta[r];
      float dk_r = 0.f, dq_r = 0.f, dg_r = 0.f;
      for (int i = 0; i <= r; ++i) {
        const float e = __expf(gr - sG[i * ldk + a]);
        const float pa = sdP[r * ldc + i];
        const float aa = i < r ? sdM[r * ldc + i] * br : 0.f;
        const float t1 = e * sK[i * ldk + a];
        dk_r = fmaf(aa, t1, dk_r);
        dq_r = fmaf(pa, t1, dq_r);
        dg_r = fmaf(fmaf(aa, kr, pa * qr), t1, dg_r);
      }
      X3[r * ldk + a] += dk_r;
      X2[r * ldk + a] += dq_r;
      X1[r * ldk + a] += dg_r;
    }
  } else if (tid >= 128 && tid - 128 < Dk) {
    const int a = tid - 128;
    for (int i = 0; i < C; ++i) {
      const float ki = sK[i * ldk + a], gi = sG[i * ldk + a];
      float dk_i = 0.f, dg_i = 0.f;
      for (int r = i; r < C; ++r) {
        const float e = __expf(sG[r * ldk + a] - gi);
        const float pa = sdP[r * ldc + i];
        const float aa = i < r ? sdM[r * ldc + i] * sbeta[r] : 0.f;
        const float w = fmaf(aa, sK[r * ldk + a], pa * sQ[r * ldk + a]) * e;
        dk_i += w;
        dg_i = fmaf(-w, ki, dg_i);
      }
      Y1[i * ldk + a] = dk_i;
      Y2[i * ldk + a] = dg_i;
    }
  }
  __syncthreads();
  for (int idx = tid; idx < C * Dk; idx += nt) {
    const int r = idx / Dk, a = idx - r * Dk;
    X3[r * ldk + a] += Y1[r * ldk + a];
    X1[r * ldk + a] += Y2[r * ldk + a];
  }
  __syncthreads();
  for (int a = tid; a < Dk; a += nt) {
    // g_C enters Kt and gamma_C
    const float gc = sG[(C - 1) * ldk + a];
    float dgc = sdgam[a] * expf(gc);
    for (int i = 0; i < C; ++i)
      dgc += X4[i * ldk + a] * sK[i * ldk + a] * expf(gc - sG[i * ldk + a]);
    X1[(C - 1) * ldk + a] += dgc;
    float acc = 0.f;  // d log_alpha_j = sum_{r >= j} dg_r
    for (int r = C - 1; r >= 0; --r) {
      acc += X1[r * ldk + a];
      X1[r * ldk + a] = acc;
    }
  }
  __syncthreads();
  // ---- P6: outputs
  for (int idx = tid; idx < C * Dk; idx += nt) {
    const int r = idx / Dk, a = idx - r * Dk;
    if (r < L) {
      const size_t gi = ((size_t)(t0 + r) * H + h) * Dk + a;
      const int x = r * ldk + a;
      dq[gi] = from_f32<Tin>(X2[x]);
      dk[gi] = from_f32<Tin>(X3[x]);
      dla[gi] = X1[x];
    }
  }
  for (int r = tid; r < L; r += nt) dbeta[(size_t)(t0 + r) * H + h] = sdb[r];
}

size_t bwd_state_smem_bytes(int C, int Dk) {
  // + the split-contraction partial sums of dV' ([64 / C][C][32])
  return sizeof(float) * ((size_t)Dk * kBwSlice + 3 * (size_t)C * Dk + (size_t)C * C + Dk +
                          2 * (size_t)C * kBwSlice + 64 * (size_t)kBwSlice);
}
size_t bwd_local_smem_bytes(int Dk, int Dv) {
  return sizeof(float) * (size_t)BwdSmem::make(Dk, Dv).total;
}

template <typename Tin>
static cudaError_t launch_bwd_typed(const BackwardArgs& b, const SeqGeometry& geo, int max_chunks,
                                    float* records, const SimtRecord& rec, float* states,
                                    float* dstates, float* dvp, cudaStream_t stream) {
  const PrefillArgs& a = b.fwd;
  if (a.C != kBwdC || geo.C != kBwdC) return cudaErrorInvalidValue;
  cudaError_t err =
      launch_forward_for_backward(a, geo, max_chunks, records, rec, states, stream);
  if (err != cudaSuccess) return err;
  const size_t sm3 = bwd_state_smem_bytes(a.C, a.Dk), sm4 = bwd_local_smem_bytes(a.Dk, a.Dv);
  err = cudaFuncSetAttribute(chunk_state_bwd_kernel<Tin>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm3);
  if (err != cudaSuccess) return err;
  err = cudaFuncSetAttribute(chunk_local_bwd_kernel<Tin>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm4);
  if (err != cudaSuccess) return err;
  {
    ProfileScope prof("chunk_state_bwd", stream);
    chunk_state_bwd_kernel<Tin><<<dim3(a.N, a.H, ceil_div(a.Dv, kBwSlice)), kBwdThreads, sm3,
                                  stream>>>(records, rec, geo, a.H, a.Dk, a.Dv,
                                            (const Tin*)b.d_o, b.d_final, b.d_initial, dstates,
                                            dvp);
    err = cudaGetLastError();
    if (err != cudaSuccess) return err;
  }
  if (max_chunks == 0) return cudaSuccess;
  ProfileScope prof("chunk_local_bwd", stream);
  chunk_local_bwd_kernel<Tin><<<item_grid(max_chunks, a.H), kBwdThreads, sm4, stream>>>(
      (const Tin*)a.q, (const Tin*)a.k, (const Tin*)a.v, a.log_alpha, a.beta, geo, a.H, a.Dk,
      a.Dv, records, rec, states, dstates, dvp, (const Tin*)b.d_o, (Tin*)b.dq, (Tin*)b.dk,
      (Tin*)b.dv, b.dlog_alpha, b.dbeta);
  return cudaGetLastError();
}

cudaError_t launch_chunk_bwd(const BackwardArgs& b, const SeqGeometry& geo, int max_chunks,
                             float* records, const SimtRecord& rec, float* states,
                             float* dstates, float* dvp, cudaStream_t stream) {
  if (b.fwd.dtype == KDA_DTYPE_BF16)
    return launch_bwd_typed<__nv_bfloat16>(b, geo, max_chunks, records, rec, states, dstates,
                                           dvp, stream);
  return launch_bwd_typed<float>(b, geo, max_chunks, records, rec, states, dstates, dvp, stream);
}

}  // namespace kda
