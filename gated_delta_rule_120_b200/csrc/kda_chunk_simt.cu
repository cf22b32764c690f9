// kda_chunk_simt.cu — fp32 CUDA-core chunkwise prefill of KDA (any Dk, Dv <= 128; C in 16/32/64).
//
// This is the exact-fp32 path (tensor cores in bf16 or tf32 cannot hold the 1e-4 relative state
// error that fp32 inputs ask for). It follows the chunkwise algorithm of "Kimi Linear: An
// Expressive, Efficient Attention Architecture" (paper-graph-ui walkthrough, §3.4 "Chunkwise
// Parallelization"), split in two kernels:
//
//   K1  chunk_local   one CTA per (chunk, head), all chunks in parallel:
//         g      = cumulative log decay inside the chunk (Gamma in log space)
//         A_kk   = StrictTril(Diag(beta)(Gamma.K)(K/Gamma)^T),  A_qk = Tril((Gamma.Q)(K/Gamma)^T)
//                  with every ratio gamma_r/gamma_i formed as exp(g_r - g_i) <= 1 (no 1/Gamma)
//         M      = (I + A_kk)^{-1} Diag(beta)                     (forward substitution, fp32)
//         W      = M (Gamma.K),  U = M V                           (the UT transform)
//         Kt     = (gamma_C / gamma_i) k_i,  Qt = gamma_r q_r,  gamma_C
//       written to the caller's workspace.
//   K2  chunk_state   one CTA per (sequence, head, 32-column slice of d_v), sequential in chunks:
//         V' = U - W S;  O = Qt S + A_qk V' (Eq. 9);  S = Diag(gamma_C) S + Kt^T V' (Eq. 8)
//       The d_v columns of S evolve independently (Eq. 1 mixes key channels only), so slices
//       need no communication. The state slice stays in shared memory for the whole sequence.
//
// Padded rows of a partial last chunk act as identity steps (log_alpha = 0, beta = 0, k = q = v
// = 0): they add nothing and their outputs are not written.
#include "kda_common.cuh"
#include "kda_internal.h"

namespace kda {

constexpr int kSimtThreads = 256;

// ----------------------------------------------------------------------------------------------
// chunk map for packed variable-length batches: chunk_off[n] = sum_{m<n} ceil(len_m / C).
// Validates cu_seqlens (cu[0] == 0, non-decreasing, cu[N] <= total) and records the verdict in
// `valid`; the other kernels do nothing when it is 0 and the per-device status word is raised.
// With `order` it also writes the sequences by decreasing chunk count (ties by index) for up to
// blockDim.x sequences, the identity beyond that.
// ----------------------------------------------------------------------------------------------
__global__ void chunk_map_kernel(const int32_t* __restrict__ cu, int N, int total, int C,
                                 int32_t* __restrict__ chunk_off, int32_t* __restrict__ valid,
                                 int32_t* __restrict__ order) {
  __shared__ int s_sum[1024];
  __shared__ int s_cnt[1024];
  __shared__ int s_bad;
  const int tid = threadIdx.x, nt = blockDim.x;
  if (tid == 0) s_bad = (cu[0] != 0 || cu[N] > total) ? 1 : 0;
  const int per = (N + nt - 1) / nt;
  const int lo = min(N, tid * per), hi = min(N, lo + per);
  int local = 0, bad = 0;
  for (int n = lo; n < hi; ++n) {
    const int len = cu[n + 1] - cu[n];
    if (len < 0) bad = 1;
    local += len > 0 ? (len + C - 1) / C : 0;
  }
  s_sum[tid] = local;
  __syncthreads();
  if (bad) atomicOr(&s_bad, 1);
  // inclusive scan over the per-thread sums (Hillis-Steele, nt <= 1024)
  for (int off = 1; off < nt; off <<= 1) {
    const int x = tid >= off ? s_sum[tid - off] : 0;
    __syncthreads();
    s_sum[tid] += x;
    __syncthreads();
  }
  int run = s_sum[tid] - local;  // exclusive prefix
  for (int n = lo; n < hi; ++n) {
    chunk_off[n] = run;
    const int len = cu[n + 1] - cu[n];
    run += len > 0 ? (len + C - 1) / C : 0;
  }
  if (tid == nt - 1) chunk_off[N] = s_sum[nt - 1];
  if (order) {
    if (N <= nt) {  // rank = number of sequences ahead of this one
      const int len = tid < N ? cu[tid + 1] - cu[tid] : 0;
      const int cnt = len > 0 ? (len + C - 1) / C : 0;
      s_cnt[tid] = cnt;
      __syncthreads();
      if (tid < N) {
        int rank = 0;
        for (int m = 0; m < N; ++m) {
          const int cm = s_cnt[m];
          rank += (cm > cnt || (cm == cnt && m < tid)) ? 1 : 0;
        }
        order[rank] = tid;
      }
    } else {
      for (int n = tid; n < N; n += nt) order[n] = n;
    }
  }
  __syncthreads();
  if (tid == 0) {
    *valid = s_bad ? 0 : 1;
    if (s_bad) raise_status(kStatusBadSeqlens);
  }
}

cudaError_t launch_chunk_map(const int32_t* cu, int N, int total, int C, int32_t* chunk_off,
                             int32_t* valid, int32_t* order, cudaStream_t stream) {
  ProfileScope prof("chunk_map", stream);
  chunk_map_kernel<<<1, 1024, 0, stream>>>(cu, N, total, C, chunk_off, valid, order);
  return cudaGetLastError();
}

// ----------------------------------------------------------------------------------------------
// K1: chunk-local UT transform (fp32, CUDA cores)
// ----------------------------------------------------------------------------------------------
template <typename Tin>
__global__ void __launch_bounds__(kSimtThreads)
    chunk_local_simt_kernel(const Tin* __restrict__ q, const Tin* __restrict__ k,
                            const Tin* __restrict__ v, const float* __restrict__ log_alpha,
                            const float* __restrict__ beta, SeqGeometry geo, int H, int Dk, int Dv,
                            float* __restrict__ ws, SimtRecord rec, Fusion fz) {
  extern __shared__ float smem[];
  const int C = geo.C;
  float* sk = smem;            // [C][Dk]  k, later Gamma.K
  float* sq = sk + C * Dk;     // [C][Dk]
  float* sv = sq + C * Dk;     // [C][Dv]
  float* sg = sv + C * Dv;     // [C][Dk]  cumulative log decay
  float* sA = sg + C * Dk;     // [C][C]   A_kk (strict lower), then M
  float* sT = sA + C * C;      // [C][C]   (I + A)^{-1}
  float* sb = sT + C * C;      // [C]

  if (!geo.ok()) return;
  const int c = blockIdx.x, h = blockIdx.y;
  if (c >= geo.num_chunks_total()) return;
  const int n = geo.seq_of_chunk(c);
  const int t0 = geo.seq_begin(n) + (c - geo.first_chunk(n)) * C;
  const int L = min(C, geo.seq_end(n) - t0);
  const int tid = threadIdx.x, nt = blockDim.x, lane = tid & 31, warp = tid >> 5;
  float* out = ws + rec.record_floats * ((size_t)c * H + h);

  const float neg_a = fz.A_log ? -expf(fz.A_log[h]) : 0.f;
  for (int idx = tid; idx < C * Dk; idx += nt) {
    const int r = idx / Dk, cc = idx - r * Dk;
    const size_t gi = ((size_t)(t0 + r) * H + h) * Dk + cc;
    const bool in = r < L;
    sk[idx] = in ? to_f32(k[gi]) : 0.f;
    sq[idx] = in ? to_f32(q[gi]) : 0.f;
    float la = in ? log_alpha[gi] : 0.f;
    if (fz.A_log && in)  // fused gate: raw gate -> log decay
      la = neg_a * softplus_f(la + (fz.dt_bias ? fz.dt_bias[h * Dk + cc] : 0.f));
    sg[idx] = la;
  }
  for (int idx = tid; idx < C * Dv; idx += nt) {
    const int r = idx / Dv, cc = idx - r * Dv;
    sv[idx] = r < L ? to_f32(v[((size_t)(t0 + r) * H + h) * Dv + cc]) : 0.f;
  }
  for (int r = tid; r < C; r += nt) sb[r] = r < L ? beta[(size_t)(t0 + r) * H + h] : 0.f;
  __syncthreads();
  if (fz.l2) {  // fused L2 norm of q and k rows (one warp per row)
    for (int r = warp; r < C; r += nt / 32) {
      float ssk = 0.f, ssq = 0.f;
      for (int cc = lane; cc < Dk; cc += 32) {
        ssk += sk[r * Dk + cc] * sk[r * Dk + cc];
        ssq += sq[r * Dk + cc] * sq[r * Dk + cc];
      }
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) {
        ssk += __shfl_xor_sync(0xffffffffu, ssk, off);
        ssq += __shfl_xor_sync(0xffffffffu, ssq, off);
      }
      const float ik = rsqrtf(ssk + fz.eps), iq = rsqrtf(ssq + fz.eps);
      for (int cc = lane; cc < Dk; cc += 32) {
        sk[r * Dk + cc] *= ik;
        sq[r * Dk + cc] *= iq;
      }
    }
    __syncthreads();
  }

  // g_r = sum_{j<=r} log alpha_j, per key channel
  for (int cc = tid; cc < Dk; cc += nt) {
    float acc = 0.f;
    for (int r = 0; r < C; ++r) {
      acc += sg[r * Dk + cc];
      sg[r * Dk + cc] = acc;
    }
  }
  __syncthreads();

  // A_kk and A_qk: one warp per (r, i) pair with i <= r, lanes over key channels
  float* gAqk = out + rec.off_aqk;
  const int npairs = C * (C + 1) / 2;
  for (int p = warp; p < npairs; p += nt / 32) {
    int r = (int)((sqrtf(8.f * p + 1.f) - 1.f) * 0.5f);
    while ((r + 1) * (r + 2) / 2 <= p) ++r;
    while (r * (r + 1) / 2 > p) --r;
    const int i = p - r * (r + 1) / 2;
    float akk = 0.f, aqk = 0.f;
    for (int cc = lane; cc < Dk; cc += 32) {
      const float f = expf(sg[r * Dk + cc] - sg[i * Dk + cc]);  // gamma_r / gamma_i <= 1
      const float ki = sk[i * Dk + cc] * f;
      akk += sk[r * Dk + cc] * ki;
      aqk += sq[r * Dk + cc] * ki;
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      akk += __shfl_xor_sync(0xffffffffu, akk, off);
      aqk += __shfl_xor_sync(0xffffffffu, aqk, off);
    }
    if (lane == 0) {
      sA[r * C + i] = (i < r) ? sb[r] * akk : 0.f;
      gAqk[r * C + i] = aqk;
      if (rec.off_b != SimtRecord::kNone) out[rec.off_b + r * C + i] = (i < r) ? akk : 0.f;
    }
  }
  for (int idx = tid; idx < C * C; idx += nt) {  // upper triangles
    const int r = idx / C, i = idx - r * C;
    if (i > r) {
      sA[idx] = 0.f;
      gAqk[idx] = 0.f;
      if (rec.off_b != SimtRecord::kNone) out[rec.off_b + idx] = 0.f;
    }
  }
  __syncthreads();

  // (I + A)^{-1} by forward substitution: row r = e_r - sum_{j<r} A[r][j] row j
  for (int r = 0; r < C; ++r) {
    for (int cc = tid; cc < C; cc += nt) {
      float val = 0.f;
      if (cc <= r) {
        val = (cc == r) ? 1.f : 0.f;
        for (int j = cc; j < r; ++j) val -= sA[r * C + j] * sT[j * C + cc];
      }
      sT[r * C + cc] = val;
    }
    __syncthreads();
  }
  // M = (I + A)^{-1} Diag(beta)  (the backward pass keeps (I + A)^{-1} itself)
  for (int idx = tid; idx < C * C; idx += nt) {
    if (rec.off_t != SimtRecord::kNone) out[rec.off_t + idx] = sT[idx];
    sT[idx] *= sb[idx % C];
  }

  // Kt = (gamma_C/gamma_i) k_i, Qt = gamma_r q_r, gamma_C; then sk <- Gamma.K
  const float* gC = sg + (C - 1) * Dk;
  for (int idx = tid; idx < C * Dk; idx += nt) {
    const int cc = idx % Dk;
    const float g = sg[idx];
    const float kk = sk[idx];
    out[rec.off_kt + idx] = kk * expf(gC[cc] - g);
    out[rec.off_qt + idx] = sq[idx] * expf(g);
    sk[idx] = kk * expf(g);
  }
  for (int cc = tid; cc < Dk; cc += nt) out[rec.off_gam + cc] = expf(gC[cc]);
  __syncthreads();

  // W = M (Gamma.K), U = M V
  const int wu = Dk + Dv;
  for (int idx = tid; idx < C * wu; idx += nt) {
    const int r = idx / wu, cc = idx - r * wu;
    float acc = 0.f;
    if (cc < Dk) {
      for (int i = 0; i <= r; ++i) acc += sT[r * C + i] * sk[i * Dk + cc];
      out[rec.off_w + r * Dk + cc] = acc;
    } else {
      const int cv = cc - Dk;
      for (int i = 0; i <= r; ++i) acc += sT[r * C + i] * sv[i * Dv + cv];
      out[rec.off_u + r * Dv + cv] = acc;
    }
  }
}

// ----------------------------------------------------------------------------------------------
// K2: sequential inter-chunk state propagation and output (fp32, CUDA cores)
// ----------------------------------------------------------------------------------------------
constexpr int kSlice = 32;

template <typename Tin>
__global__ void __launch_bounds__(kSimtThreads)
    chunk_state_simt_kernel(const float* __restrict__ ws, SimtRecord rec, SeqGeometry geo, int H,
                            int Dk, int Dv, const float* __restrict__ initial_state,
                            float* __restrict__ final_state, Tin* __restrict__ o,
                            float* __restrict__ states_out) {
  extern __shared__ float smem[];
  const int C = geo.C;
  float* sS = smem;               // [Dk][32] state slice
  float* sW = sS + Dk * kSlice;   // [C][Dk]
  float* sKt = sW + C * Dk;       // [C][Dk]
  float* sQt = sKt + C * Dk;      // [C][Dk]
  float* sU = sQt + C * Dk;       // [C][32]
  float* sVp = sU + C * kSlice;   // [C][32]
  float* sAq = sVp + C * kSlice;  // [C][C]
  float* sGam = sAq + C * C;      // [Dk]

  if (!geo.ok()) return;
  const int n = blockIdx.x, h = blockIdx.y, j0 = blockIdx.z * kSlice;
  const int NV = min(kSlice, Dv - j0);
  const int tid = threadIdx.x, nt = blockDim.x, j = tid & 31, rg = tid >> 5;
  const int ng = nt >> 5;
  const size_t sbase = ((size_t)n * H + h) * Dk * Dv;

  for (int idx = tid; idx < Dk * kSlice; idx += nt) {
    const int cc = idx / kSlice, jj = idx - cc * kSlice;
    sS[idx] = (initial_state && jj < NV) ? initial_state[sbase + (size_t)cc * Dv + j0 + jj] : 0.f;
  }

  const int tb = geo.seq_begin(n), te = geo.seq_end(n);
  const int c_first = geo.first_chunk(n);
  const int nchunks = te > tb ? ceil_div(te - tb, C) : 0;
  for (int ci = 0; ci < nchunks; ++ci) {
    const int c = c_first + ci;
    const int t0 = tb + ci * C;
    const int L = min(C, te - t0);
    const float* r_ = ws + rec.record_floats * ((size_t)c * H + h);
    __syncthreads();  // previous chunk done with the staging buffers
    for (int idx = tid; idx < C * Dk; idx += nt) {
      sW[idx] = r_[rec.off_w + idx];
      sKt[idx] = r_[rec.off_kt + idx];
      sQt[idx] = r_[rec.off_qt + idx];
    }
    for (int idx = tid; idx < C * kSlice; idx += nt) {
      const int r = idx / kSlice, jj = idx - r * kSlice;
      sU[idx] = jj < NV ? r_[rec.off_u + r * Dv + j0 + jj] : 0.f;
    }
    for (int idx = tid; idx < C * C; idx += nt) sAq[idx] = r_[rec.off_aqk + idx];
    for (int cc = tid; cc < Dk; cc += nt) sGam[cc] = r_[rec.off_gam + cc];
    if (states_out) {  // the state entering this chunk, for the backward pass
      float* so = states_out + ((size_t)c * H + h) * Dk * Dv;
      for (int idx = tid; idx < Dk * kSlice; idx += nt) {
        const int cc = idx / kSlice, jj = idx - cc * kSlice;
        if (jj < NV) so[(size_t)cc * Dv + j0 + jj] = sS[idx];
      }
    }
    __syncthreads();

    // V' = U - W S  and  O_inter = Qt S
    float o1[8];
#pragma unroll
    for (int m = 0; m < 8; ++m) {
      const int r = rg + m * ng;
      float aw = 0.f, aq = 0.f;
      if (r < C) {
        if (o) {
          for (int cc = 0; cc < Dk; ++cc) {
            const float s = sS[cc * kSlice + j];
            aw += sW[r * Dk + cc] * s;
            aq += sQt[r * Dk + cc] * s;
          }
        } else {  // only the states are wanted
          for (int cc = 0; cc < Dk; ++cc) aw += sW[r * Dk + cc] * sS[cc * kSlice + j];
        }
        sVp[r * kSlice + j] = sU[r * kSlice + j] - aw;
      }
      o1[m] = aq;
    }
    __syncthreads();

    // O = O_inter + Tril(A_qk) V'  (Eq. 9)
#pragma unroll
    for (int m = 0; m < 8; ++m) {
      const int r = rg + m * ng;
      if (o && r < C) {
        float acc = o1[m];
        for (int i = 0; i <= r; ++i) acc += sAq[r * C + i] * sVp[i * kSlice + j];
        if (o && r < L && j < NV) o[((size_t)(t0 + r) * H + h) * Dv + j0 + j] = from_f32<Tin>(acc);
      }
    }
    // S = Diag(gamma_C) S + Kt^T V'  (Eq. 8); each thread owns its (cc, j) elements
    for (int cc = rg; cc < Dk; cc += ng) {
      float acc = sGam[cc] * sS[cc * kSlice + j];
      for (int i = 0; i < C; ++i) acc += sKt[i * Dk + cc] * sVp[i * kSlice + j];
      sS[cc * kSlice + j] = acc;
    }
  }
  __syncthreads();
  if (final_state) {
    for (int idx = tid; idx < Dk * kSlice; idx += nt) {
      const int cc = idx / kSlice, jj = idx - cc * kSlice;
      if (jj < NV) final_state[sbase + (size_t)cc * Dv + j0 + jj] = sS[idx];
    }
  }
}

size_t simt_local_smem_bytes(int C, int Dk, int Dv) {
  return sizeof(float) * ((size_t)3 * C * Dk + (size_t)C * Dv + 2 * (size_t)C * C + C);
}
size_t simt_state_smem_bytes(int C, int Dk) {
  return sizeof(float) *
         ((size_t)Dk * kSlice + 3 * (size_t)C * Dk + 2 * (size_t)C * kSlice + (size_t)C * C + Dk);
}

template <typename Tin>
static cudaError_t launch_simt_typed(const PrefillArgs& a, const SeqGeometry& geo, int max_chunks,
                                     float* records, const SimtRecord& rec, cudaStream_t stream) {
  const size_t sm1 = simt_local_smem_bytes(a.C, a.Dk, a.Dv);
  const size_t sm2 = simt_state_smem_bytes(a.C, a.Dk);
  cudaError_t err;
  err = cudaFuncSetAttribute(chunk_local_simt_kernel<Tin>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm1);
  if (err != cudaSuccess) return err;
  err = cudaFuncSetAttribute(chunk_state_simt_kernel<Tin>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm2);
  if (err != cudaSuccess) return err;
  if (max_chunks > 0) {
    dim3 g1(max_chunks, a.H);
    ProfileScope prof("chunk_local_simt", stream);
    chunk_local_simt_kernel<Tin><<<g1, kSimtThreads, sm1, stream>>>(
        (const Tin*)a.q, (const Tin*)a.k, (const Tin*)a.v, a.log_alpha, a.beta, geo, a.H, a.Dk,
        a.Dv, records, rec, a.fz);
    err = cudaGetLastError();
    if (err != cudaSuccess) return err;
  }
  dim3 g2(a.N, a.H, ceil_div(a.Dv, kSlice));
  ProfileScope prof("chunk_state_simt", stream);
  chunk_state_simt_kernel<Tin><<<g2, kSimtThreads, sm2, stream>>>(
      records, rec, geo, a.H, a.Dk, a.Dv, a.initial_state, a.final_state, (Tin*)a.o, nullptr);
  err = cudaGetLastError();
  if (err != cudaSuccess || !a.fz.onorm) return err;
  return launch_output_norm_gate(a.o, a.dtype, a.fz, (long long)a.B * a.T * a.H, a.H, a.Dv,
                                 a.cu_seqlens ? a.cu_seqlens + a.N : nullptr, stream);
}

template <typename Tin>
static cudaError_t launch_fwd_for_bwd_typed(const PrefillArgs& a, const SeqGeometry& geo,
                                            int max_chunks, float* records, const SimtRecord& rec,
                                            float* states, cudaStream_t stream) {
  const size_t sm1 = simt_local_smem_bytes(a.C, a.Dk, a.Dv);
  const size_t sm2 = simt_state_smem_bytes(a.C, a.Dk);
  cudaError_t err;
  err = cudaFuncSetAttribute(chunk_local_simt_kernel<Tin>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm1);
  if (err != cudaSuccess) return err;
  err = cudaFuncSetAttribute(chunk_state_simt_kernel<Tin>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm2);
  if (err != cudaSuccess) return err;
  if (max_chunks > 0) {
    ProfileScope prof("bwd_chunk_local_fwd", stream);
    chunk_local_simt_kernel<Tin><<<dim3(max_chunks, a.H), kSimtThreads, sm1, stream>>>(
        (const Tin*)a.q, (const Tin*)a.k, (const Tin*)a.v, a.log_alpha, a.beta, geo, a.H, a.Dk,
        a.Dv, records, rec, a.fz);
    err = cudaGetLastError();
    if (err != cudaSuccess) return err;
  }
  ProfileScope prof("bwd_chunk_state_fwd", stream);
  chunk_state_simt_kernel<Tin><<<dim3(a.N, a.H, ceil_div(a.Dv, kSlice)), kSimtThreads, sm2,
                                 stream>>>(records, rec, geo, a.H, a.Dk, a.Dv, a.initial_state,
                                           nullptr, (Tin*)nullptr, states);
  return cudaGetLastError();
}

cudaError_t launch_forward_for_backward(const PrefillArgs& a, const SeqGeometry& geo,
                                        int max_chunks, float* records, const SimtRecord& rec,
                                        float* states, cudaStream_t stream) {
  if (a.dtype == KDA_DTYPE_BF16)
    return launch_fwd_for_bwd_typed<__nv_bfloat16>(a, geo, max_chunks, records, rec, states,
                                                   stream);
  return launch_fwd_for_bwd_typed<float>(a, geo, max_chunks, records, rec, states, stream);
}

cudaError_t launch_prefill_simt(const PrefillArgs& a, const SeqGeometry& geo, int max_chunks,
                                float* records, const SimtRecord& rec, cudaStream_t stream) {
  if (a.dtype == KDA_DTYPE_BF16)
    return launch_simt_typed<__nv_bfloat16>(a, geo, max_chunks, records, rec, stream);
  return launch_simt_typed<float>(a, geo, max_chunks, records, rec, stream);
}

}  // namespace kda
