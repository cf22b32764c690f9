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
#include "kda_items.cuh"

namespace kda {

constexpr int kSimtThreads = 256;

// ----------------------------------------------------------------------------------------------
// chunk map for packed variable-length batches: chunk_off[n] = sum_{m<n} ceil(len_m / C).
// Validates cu_seqlens (cu[0] == 0, non-decreasing, cu[N] <= total) and records the outcome in
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
  if (!KDA_IN_BOUNDS(kBufCuSeqlens, cu, (N + 1) * 4ull) || !KDA_IN_BOUNDS(kBufWork, valid, 4) ||
      !KDA_IN_BOUNDS(kBufWork, chunk_off, (N + 1) * 4ull) ||
      (order && !KDA_IN_BOUNDS(kBufWork, order, N * 4ull)))
    return;  // (uniform: the whole block leaves)
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
  if (kBoundsChecked) {  // a map that skips its accesses leaves the call's kernels disabled
    const cudaError_t err = cudaMemsetAsync(valid, 0, sizeof(int32_t), stream);
    if (err != cudaSuccess) return err;
  }
  ProfileScope prof("chunk_map", stream);
  chunk_map_kernel<<<1, 1024, 0, stream>>>(cu, N, total, C, chunk_off, valid, order);
  return cudaGetLastError();
}

// ----------------------------------------------------------------------------------------------
// K1: chunk-local UT transform (fp32, CUDA cores)
// ----------------------------------------------------------------------------------------------

// Column cc of T = (I + A)^{-1} (A strictly lower, C <= kMaxC rows), held in registers:
// T[r][cc] = [r == cc] - sum_{cc <= j < r} A[r][j] T[j][cc] (col[j] = 0 for j < cc). Up to 32 rows
// each row's sum runs as four partial sums (float4 groups of A's row, then the rest), so mostly
// the newest column entries are on the dependency chain; 64 rows keep one sum (register budget).
template <int kMaxC>
__device__ __forceinline__ void forward_subst(const float* sA, float* sT, int C, int cc) {
  float col[kMaxC];
#pragma unroll
  for (int r = 0; r < kMaxC; ++r) {
    if (r < C) {
      float val;
      if (kMaxC <= 32) {
        float acc[4] = {(r == cc) ? 1.f : 0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int j4 = 0; j4 < r / 4; ++j4) {
          const float4 a = *reinterpret_cast<const float4*>(sA + r * C + 4 * j4);
          acc[0] = fmaf(-a.x, col[4 * j4], acc[0]);
          acc[1] = fmaf(-a.y, col[4 * j4 + 1], acc[1]);
          acc[2] = fmaf(-a.z, col[4 * j4 + 2], acc[2]);
          acc[3] = fmaf(-a.w, col[4 * j4 + 3], acc[3]);
        }
#pragma unroll
        for (int jj = 4 * (r / 4); jj < r; ++jj)
          acc[jj & 3] = fmaf(-sA[r * C + jj], col[jj], acc[jj & 3]);
        val = (acc[0] + acc[1]) + (acc[2] + acc[3]);
      } else {
        val = (r == cc) ? 1.f : 0.f;
#pragma unroll
        for (int jj = 0; jj < r; ++jj) val -= sA[r * C + jj] * col[jj];
      }
      col[r] = r >= cc ? val : 0.f;
      sT[r * C + cc] = col[r];
    }
  }
}
template <typename Tin>
__global__ void __launch_bounds__(kSimtThreads, 3)
    chunk_local_simt_kernel(const Tin* __restrict__ q, const Tin* __restrict__ k,
                            const Tin* __restrict__ v, const float* __restrict__ log_alpha,
                            const float* __restrict__ beta, SeqGeometry geo, int H, int Dk, int Dv,
                            float* __restrict__ ws, SimtRecord rec, Fusion fz) {
  extern __shared__ __align__(16) float smem[];
  const int C = geo.C;
  const int ldk = Dk + 4;      // row pitch of sk: rows of one float4 column hit distinct banks
  float* sk = smem;            // [C][ldk] k (k F in the factored form), later Gamma.K
  float* sq = sk + C * ldk;    // [C][Dk]
  float* sv = sq + C * Dk;     // [C][Dv]
  float* sg = sv + C * Dv;     // [C][Dk]  cumulative log decay (E in the factored form)
  float* sA = sg + C * Dk;     // [C][C]   A_kk (strict lower), then M
  float* sT = sA + C * C;      // [C][C]   (I + A)^{-1}
  float* sb = sT + C * C;      // [C]
  float* smid = sb + C;        // [Dk]     per-channel midpoint m of g (factored form)

  if (!geo.ok()) return;
  const ChunkItem item = chunk_item();
  const int c = item.c, h = item.h;
  if (c >= geo.num_chunks_total()) return;
  const int n = geo.seq_of_chunk(c);
  const int t0 = geo.seq_begin(n) + (c - geo.first_chunk(n)) * C;
  const int L = min(C, geo.seq_end(n) - t0);
  const int tid = threadIdx.x, nt = blockDim.x, lane = tid & 31, warp = tid >> 5;
  float* out = ws + rec.record_floats * ((size_t)c * H + h);
#ifdef KDA_BOUNDS_CHECK
  {  // every access of the item lies in its record and in rows t0 .. t0 + L - 1 of head h
    const size_t rk = (size_t)H * Dk, rv = (size_t)H * Dv;
    const bool ok =
        in_bounds(kBufWork, out, rec.record_floats * sizeof(float)) &&
        rows_in_bounds(kBufK, k + (size_t)h * Dk, t0, t0 + L, rk, Dk) &&
        rows_in_bounds(kBufQ, q + (size_t)h * Dk, t0, t0 + L, rk, Dk) &&
        rows_in_bounds(kBufV, v + (size_t)h * Dv, t0, t0 + L, rv, Dv) &&
        rows_in_bounds(kBufLogAlpha, log_alpha + (size_t)h * Dk, t0, t0 + L, rk, Dk) &&
        rows_in_bounds(kBufBeta, beta + h, t0, t0 + L, H, 1) &&
        (!fz.A_log || in_bounds(kBufALog, fz.A_log + h, 4)) &&
        (!fz.A_log || !fz.dt_bias || in_bounds(kBufDtBias, fz.dt_bias + (size_t)h * Dk, Dk * 4ull));
    if (!ok) return;  // (uniform: the whole CTA leaves)
  }
#endif

  const float neg_a = fz.A_log ? -expf(fz.A_log[h]) : 0.f;
  constexpr int kPer = 16 / sizeof(Tin);
  const bool vec_in = ((reinterpret_cast<uintptr_t>(q) | reinterpret_cast<uintptr_t>(k) |
                        reinterpret_cast<uintptr_t>(v)) & 15) == 0 &&
                      Dk % kPer == 0 && Dv % kPer == 0;
  const bool vec_la = !fz.A_log && (reinterpret_cast<uintptr_t>(log_alpha) & 15) == 0 &&
                      Dk % 4 == 0;
  const size_t bk = ((size_t)t0 * H + h) * Dk, bv = ((size_t)t0 * H + h) * Dv;
  if (vec_in) {  // 16-byte vectors, several in flight per thread
    stage_rows_f32<Tin>(sk, ldk, k + bk, (size_t)H * Dk, C, L, Dk, tid, nt);
    stage_rows_f32<Tin>(sq, Dk, q + bk, (size_t)H * Dk, C, L, Dk, tid, nt);
    stage_rows_f32<Tin>(sv, Dv, v + bv, (size_t)H * Dv, C, L, Dv, tid, nt);
  } else {
    for (int idx = tid; idx < C * Dk; idx += nt) {
      const int r = idx / Dk, cc = idx - r * Dk;
      const size_t gi = bk + (size_t)r * H * Dk + cc;
      const bool in = r < L;
      sk[r * ldk + cc] = in ? to_f32(k[gi]) : 0.f;
      sq[idx] = in ? to_f32(q[gi]) : 0.f;
    }
    for (int idx = tid; idx < C * Dv; idx += nt) {
      const int r = idx / Dv, cc = idx - r * Dv;
      sv[idx] = r < L ? to_f32(v[bv + (size_t)r * H * Dv + cc]) : 0.f;
    }
  }
  if (vec_la) {
    stage_rows_f32<float>(sg, Dk, log_alpha + bk, (size_t)H * Dk, C, L, Dk, tid, nt);
  } else {
    for (int idx = tid; idx < C * Dk; idx += nt) {
      const int r = idx / Dk, cc = idx - r * Dk;
      const bool in = r < L;
      float la = in ? log_alpha[bk + (size_t)r * H * Dk + cc] : 0.f;
      if (fz.A_log && in)  // fused gate: raw gate -> log decay
        la = neg_a * softplus_f(la + (fz.dt_bias ? fz.dt_bias[h * Dk + cc] : 0.f));
      sg[idx] = la;
    }
  }
  for (int r = tid; r < C; r += nt) sb[r] = r < L ? beta[(size_t)(t0 + r) * H + h] : 0.f;
  __syncthreads();
  if (fz.l2) {  // fused L2 norm of q and k rows (one warp per row)
    for (int r = warp; r < C; r += nt / 32) {
      float ssk = 0.f, ssq = 0.f;
      for (int cc = lane; cc < Dk; cc += 32) {
        ssk += sk[r * ldk + cc] * sk[r * ldk + cc];
        ssq += sq[r * Dk + cc] * sq[r * Dk + cc];
      }
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) {
        ssk += __shfl_xor_sync(0xffffffffu, ssk, off);
        ssq += __shfl_xor_sync(0xffffffffu, ssq, off);
      }
      const float ik = rsqrtf(ssk + fz.eps), iq = rsqrtf(ssq + fz.eps);
      for (int cc = lane; cc < Dk; cc += 32) {
        sk[r * ldk + cc] *= ik;
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

  // A_kk and A_qk. With d_k a multiple of 4 and every key channel's cumulative decay spanning at
  // most 80 nats over the chunk, exp(g_r - g_i) = E_r F_i around the channel's midpoint m
  // (E = exp(g - m), F = exp(m - g), each factor within e^+-40, so every term keeps fp32 relative
  // precision): sk <- k F, sg <- E, and A_kk = (k F E^2)(k F)^T, A_qk = (q E)(k F)^T are
  // register-tiled products over d_k (2 x 2 tiles: rows {rp, rp + C/2}, columns {ip, ip + C/2};
  // sk's padded pitch spreads a warp's 16 columns over the banks). Otherwise one warp per (r, i)
  // pair with lanes over key channels, one exponential per term.
  float* gAqk = out + rec.off_aqk;
  float* sgC = smid + Dk;  // [Dk] g of the chunk's last row (gamma_C), kept in the factored form
  bool span_ok = (Dk & 3) == 0;
  for (int cc = tid; cc < Dk; cc += nt) {
    float gmin = sg[cc], gmax = gmin;
    for (int r = 1; r < C; ++r) {
      const float g = sg[r * Dk + cc];
      gmin = fminf(gmin, g);
      gmax = fmaxf(gmax, g);
    }
    span_ok = span_ok && gmax - gmin <= 80.f;  // false for NaN or infinite decays
    smid[cc] = 0.5f * (gmax + gmin);
    sgC[cc] = sg[(C - 1) * Dk + cc];
  }
  const bool factored = __syncthreads_and(span_ok) != 0;
  if (factored) {
    for (int idx = tid; idx < C * Dk; idx += nt) {
      const int r = idx / Dk, cc = idx - r * Dk;
      const float d = sg[idx] - smid[cc];
      sk[r * ldk + cc] *= expf(-d);
      sg[idx] = expf(d);
    }
    __syncthreads();
    for (int cc = tid; cc < Dk; cc += nt) smid[cc] = expf(smid[cc]);  // e^m, read after the inverse
    const int half = C >> 1, dq = Dk >> 2;
    for (int t = tid; t < half * half; t += nt) {
      const int rp = t / half, ip = t - rp * half;
      const int rr[2] = {rp, rp + half}, ii[2] = {ip, ip + half};
      f32x2 pk[2][2], pq[2][2];
#pragma unroll
      for (int u = 0; u < 2; ++u)
#pragma unroll
        for (int w = 0; w < 2; ++w) pk[u][w] = pq[u][w] = f2_pack(0.f, 0.f);
      for (int c4 = 0; c4 < dq; ++c4) {
        f32x2 bl[2], bh[2];
#pragma unroll
        for (int w = 0; w < 2; ++w) {
          const float4 b = *reinterpret_cast<const float4*>(sk + ii[w] * ldk + 4 * c4);
          bl[w] = f2_pack(b.x, b.y);
          bh[w] = f2_pack(b.z, b.w);
        }
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          const float4 kf = *reinterpret_cast<const float4*>(sk + rr[u] * ldk + 4 * c4);
          const float4 e = *reinterpret_cast<const float4*>(sg + rr[u] * Dk + 4 * c4);
          const float4 qv = *reinterpret_cast<const float4*>(sq + rr[u] * Dk + 4 * c4);
          const f32x2 el = f2_pack(e.x, e.y), eh = f2_pack(e.z, e.w);
          const f32x2 kel = f2_mul(f2_mul(f2_pack(kf.x, kf.y), el), el);
          const f32x2 keh = f2_mul(f2_mul(f2_pack(kf.z, kf.w), eh), eh);
          const f32x2 qel = f2_mul(f2_pack(qv.x, qv.y), el), qeh = f2_mul(f2_pack(qv.z, qv.w), eh);
#pragma unroll
          for (int w = 0; w < 2; ++w) {
            pk[u][w] = f2_fma(keh, bh[w], f2_fma(kel, bl[w], pk[u][w]));
            pq[u][w] = f2_fma(qeh, bh[w], f2_fma(qel, bl[w], pq[u][w]));
          }
        }
      }
#pragma unroll
      for (int u = 0; u < 2; ++u)
#pragma unroll
        for (int w = 0; w < 2; ++w) {
          const int r = rr[u], i = ii[w];
          const float2 a2 = f2_unpack(pk[u][w]), q2 = f2_unpack(pq[u][w]);
          const float akk = a2.x + a2.y, aqk = q2.x + q2.y;
          sA[r * C + i] = (i < r) ? sb[r] * akk : 0.f;
          gAqk[r * C + i] = (i <= r) ? aqk : 0.f;
          if (rec.off_b != SimtRecord::kNone) out[rec.off_b + r * C + i] = (i < r) ? akk : 0.f;
        }
    }
  } else {
    const int npairs = C * (C + 1) / 2;
    for (int p = warp; p < npairs; p += nt / 32) {
      int r = (int)((sqrtf(8.f * p + 1.f) - 1.f) * 0.5f);
      while ((r + 1) * (r + 2) / 2 <= p) ++r;
      while (r * (r + 1) / 2 > p) --r;
      const int i = p - r * (r + 1) / 2;
      float akk = 0.f, aqk = 0.f;
      for (int cc = lane; cc < Dk; cc += 32) {
        // gamma_r / gamma_i <= 1; the fast exponential's relative error (a few 1e-7 plus the
        // argument's rounding, < 1e-5 for any argument above -87) is far below fp32 parity needs
        const float f = __expf(sg[r * Dk + cc] - sg[i * Dk + cc]);
        const float ki = sk[i * ldk + cc] * f;
        akk += sk[r * ldk + cc] * ki;
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
  }
  __syncthreads();

  // (I + A)^{-1} by forward substitution, one lane per column of the inverse (warps 0 and 1
  // for C = 64)
  if (tid < C) {
    if (C <= 32)
      forward_subst<32>(sA, sT, C, tid);
    else
      forward_subst<64>(sA, sT, C, tid);
  }
  __syncthreads();
  // M = (I + A)^{-1} Diag(beta)  (the backward pass keeps (I + A)^{-1} itself)
  for (int idx = tid; idx < C * C; idx += nt) {
    if (rec.off_t != SimtRecord::kNone) out[rec.off_t + idx] = sT[idx];
    sT[idx] *= sb[idx % C];
  }

  // Kt = (gamma_C/gamma_i) k_i, Qt = gamma_r q_r, gamma_C; then sk <- Gamma.K. In the factored
  // form (sk = k F, sg = E, smid = e^m): Kt = k F E_C, Qt = q E e^m, Gamma.K = k F E^2 e^m.
  if (factored) {
    const float* EC = sg + (C - 1) * Dk;
    for (int idx = tid; idx < C * Dk; idx += nt) {
      const int r = idx / Dk, cc = idx - r * Dk;
      const float e = sg[idx], em = smid[cc], kf = sk[r * ldk + cc];
      out[rec.off_kt + idx] = kf * EC[cc];
      out[rec.off_qt + idx] = sq[idx] * e * em;
      sk[r * ldk + cc] = kf * e * e * em;
    }
  } else {
    const float* gC = sg + (C - 1) * Dk;
    for (int idx = tid; idx < C * Dk; idx += nt) {
      const int r = idx / Dk, cc = idx - r * Dk;
      const float g = sg[idx];
      const float kk = sk[r * ldk + cc];
      const float eg = __expf(g);  // operand scales (arguments <= 0); gamma_C uses expf
      out[rec.off_kt + idx] = kk * __expf(gC[cc] - g);
      out[rec.off_qt + idx] = sq[idx] * eg;
      sk[r * ldk + cc] = kk * eg;
    }
  }
  for (int cc = tid; cc < Dk; cc += nt) out[rec.off_gam + cc] = expf(sgC[cc]);
  __syncthreads();

  // W = M (Gamma.K), U = M V
  if ((Dk & 3) == 0 && (Dv & 3) == 0) {  // 2 x 4 register tiles, float4 rows and record stores
    const int dq = Dk >> 2, vq = Dv >> 2;
    const float4* k4 = reinterpret_cast<const float4*>(sk);  // rows of ldk / 4 float4
    const float4* v4 = reinterpret_cast<const float4*>(sv);
    for (int t = tid; t < (C >> 1) * (dq + vq); t += nt) {
      const int rp = t / (dq + vq), cq = t - rp * (dq + vq);
      const int r0 = 2 * rp, r1 = r0 + 1;
      float a0[4] = {0.f, 0.f, 0.f, 0.f}, a1[4] = {0.f, 0.f, 0.f, 0.f};
      for (int i = 0; i <= r1; ++i) {  // M is lower triangular: M[r0][r1] = 0
        const float m0 = sT[r0 * C + i], m1 = sT[r1 * C + i];
        const float4 x = cq < dq ? k4[i * (dq + 1) + cq] : v4[i * vq + (cq - dq)];
        fma_s4(m0, x, a0);
        fma_s4(m1, x, a1);
      }
      float* dst = cq < dq ? out + rec.off_w + 4 * cq : out + rec.off_u + 4 * (cq - dq);
      const int ld = cq < dq ? Dk : Dv;
      *reinterpret_cast<float4*>(dst + r0 * ld) = make_float4(a0[0], a0[1], a0[2], a0[3]);
      *reinterpret_cast<float4*>(dst + r1 * ld) = make_float4(a1[0], a1[1], a1[2], a1[3]);
    }
    return;
  }
  const int wu = Dk + Dv;
  for (int idx = tid; idx < C * wu; idx += nt) {
    const int r = idx / wu, cc = idx - r * wu;
    float acc = 0.f;
    if (cc < Dk) {
      for (int i = 0; i <= r; ++i) acc += sT[r * C + i] * sk[i * ldk + cc];
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

constexpr int kSimtRedFloats = 4096;  // split-contraction partial sums of the tiled step

// The state chain with register tiles (d_k, d_v multiples of 4; C in {16, 32, 64};
// kSimtThreads threads). Shared memory as in chunk_state_simt_kernel plus kSimtRedFloats.
// Per chunk:
//   V' = U - W S and O_inter = Qt S: 2 x 4 output tiles, the d_k contraction split 64 / C ways;
//   O = O_inter + Tril(A_qk) V' (Eq. 9): 2 x 4 tiles;  S = Diag(gamma_C) S + Kt^T V' (Eq. 8):
//   4 x 4 tiles of the state slice, updated in place.
// The record sections arrive by cp.async in two groups, each issued a phase ahead of its use:
// group A (W, Qt, the U slice: the first phase) of chunk c + 1 while chunk c computes its output
// and state update, group B (A_qk, Kt, gamma_C: the output and the update) of chunk c while chunk
// c computes its first phase.
template <typename Tin>
__device__ __forceinline__ void state_chain_tiled(const float* __restrict__ ws,
                                                  const SimtRecord& rec, int c_first, int nchunks,
                                                  int tb, int te, int C, int H, int h, int Dk,
                                                  int Dv, int j0, int NV, float* smem, Tin* o,
                                                  float* states_out) {
  const int tid = threadIdx.x;
  const int dq = Dk >> 2;  // float4 columns of a d_k row
  float4* sS = reinterpret_cast<float4*>(smem);  // [Dk][8]
  float4* sW = sS + Dk * (kSlice / 4);           // [C][dq]
  float4* sKt = sW + C * dq;
  float4* sQt = sKt + C * dq;
  float4* sU = sQt + C * dq;     // [C][8]
  float4* sVp = sU + C * 8;      // [C][8]
  float* sAq = reinterpret_cast<float*>(sVp + C * 8);  // [C][C]
  float* sGam = sAq + C * C;                            // [Dk]
  float4* sRed = reinterpret_cast<float4*>(sGam + Dk);  // [split][2][C][8]
  // record sections are 16-byte aligned (d_k, d_v multiples of 4; C multiple of 16)
  auto record = [&](int c) {
    return reinterpret_cast<const float4*>(ws + rec.record_floats * ((size_t)c * H + h));
  };
  auto issue_a = [&](int c) {
    const float4* r4 = record(c);
    for (int i = tid; i < C * dq; i += kSimtThreads) {
      cp_async_16B(sW + i, r4 + rec.off_w / 4 + i);
      if (o) cp_async_16B(sQt + i, r4 + rec.off_qt / 4 + i);
    }
    for (int i = tid; i < C * 8; i += kSimtThreads) {
      const int r = i >> 3, q = i & 7;
      if (4 * q < NV)
        cp_async_16B(sU + i, r4 + (rec.off_u + (size_t)r * Dv + j0) / 4 + q);
      else
        sU[i] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
    cp_async_commit();
  };
  auto issue_b = [&](int c) {
    const float4* r4 = record(c);
    for (int i = tid; i < C * dq; i += kSimtThreads) cp_async_16B(sKt + i, r4 + rec.off_kt / 4 + i);
    for (int i = tid; i < C * C / 4; i += kSimtThreads)
      cp_async_16B(reinterpret_cast<float4*>(sAq) + i, r4 + rec.off_aqk / 4 + i);
    for (int i = tid; i < dq; i += kSimtThreads)
      cp_async_16B(reinterpret_cast<float4*>(sGam) + i, r4 + rec.off_gam / 4 + i);
    cp_async_commit();
  };

  const int split = 64 / C;
  const int rp = (tid >> 3) % (C >> 1), jq = tid & 7, sp = tid / (4 * C);
  const int kq = (dq + split - 1) / split, q0 = sp * kq, q1 = min(dq, q0 + kq);
  const int r0 = 2 * rp, r1 = r0 + 1;

  if (nchunks > 0) issue_a(c_first);
  __syncthreads();  // the initial state slice is in place
  for (int ci = 0; ci < nchunks; ++ci) {
    const int c = c_first + ci;
    const int t0 = tb + ci * C;
    const int L = min(C, te - t0);
    issue_b(c);
    if (states_out) {  // the state entering this chunk, for the backward pass
      float* so = states_out + ((size_t)c * H + h) * Dk * Dv;
      for (int i = tid; i < Dk * 8; i += kSimtThreads) {
        const int cc = i >> 3, q = i & 7;
        if (4 * q < NV) *reinterpret_cast<float4*>(so + (size_t)cc * Dv + j0 + 4 * q) = sS[i];
      }
    }
    cp_async_wait<1>();  // group A of this chunk has landed (group B may be in flight)
    __syncthreads();

    // V' and O_inter: tile (rows 2 rp, 2 rp + 1; columns 4 jq .. 4 jq + 3), d_k split `split` ways
    float aw[2][4] = {}, aq[2][4] = {};
    // acc[a] += X[row a] S over this thread's share of d_k, for X = W and (with o) X = Qt
    auto contract = [&](const float4* X, float (&acc)[2][4]) {
      for (int q = q0; q < q1; ++q) {
        const float4 x0 = X[r0 * dq + q], x1 = X[r1 * dq + q];
        const float xa[4] = {x0.x, x0.y, x0.z, x0.w}, xb[4] = {x1.x, x1.y, x1.z, x1.w};
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const float4 sv = sS[(4 * q + k) * 8 + jq];
          fma_s4(xa[k], sv, acc[0]);
          fma_s4(xb[k], sv, acc[1]);
        }
      }
    };
    contract(sW, aw);
    if (o) contract(sQt, aq);
    if (split > 1) {  // partial sums of the split contraction, summed by the sp == 0 threads
      sRed[((sp * 2 + 0) * C + r0) * 8 + jq] = make_float4(aw[0][0], aw[0][1], aw[0][2], aw[0][3]);
      sRed[((sp * 2 + 0) * C + r1) * 8 + jq] = make_float4(aw[1][0], aw[1][1], aw[1][2], aw[1][3]);
      if (o) {
        sRed[((sp * 2 + 1) * C + r0) * 8 + jq] =
            make_float4(aq[0][0], aq[0][1], aq[0][2], aq[0][3]);
        sRed[((sp * 2 + 1) * C + r1) * 8 + jq] =
            make_float4(aq[1][0], aq[1][1], aq[1][2], aq[1][3]);
      }
      __syncthreads();
      if (sp == 0) {
        for (int s2 = 1; s2 < split; ++s2) {
#pragma unroll
          for (int a = 0; a < 2; ++a) {
            const float4 pw = sRed[((s2 * 2 + 0) * C + r0 + a) * 8 + jq];
            aw[a][0] += pw.x; aw[a][1] += pw.y; aw[a][2] += pw.z; aw[a][3] += pw.w;
            if (o) {
              const float4 pq = sRed[((s2 * 2 + 1) * C + r0 + a) * 8 + jq];
              aq[a][0] += pq.x; aq[a][1] += pq.y; aq[a][2] += pq.z; aq[a][3] += pq.w;
            }
          }
        }
      }
    }
    if (sp == 0) {
#pragma unroll
      for (int a = 0; a < 2; ++a) {
        const float4 u = sU[(r0 + a) * 8 + jq];
        sVp[(r0 + a) * 8 + jq] =
            make_float4(u.x - aw[a][0], u.y - aw[a][1], u.z - aw[a][2], u.w - aw[a][3]);
      }
    }
    __syncthreads();  // V' complete; W, Qt and U are free for the next chunk
    if (ci + 1 < nchunks) {
      issue_a(c + 1);
      cp_async_wait<1>();  // group B of this chunk has landed
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();

    // O = O_inter + Tril(A_qk) V' (Eq. 9)
    if (o && sp == 0) {
      for (int i = 0; i <= r1; ++i) {
        const float4 v = sVp[i * 8 + jq];
        const float a0 = i <= r0 ? sAq[r0 * C + i] : 0.f, a1 = sAq[r1 * C + i];
        fma_s4(a0, v, aq[0]);
        fma_s4(a1, v, aq[1]);
      }
#pragma unroll
      for (int a = 0; a < 2; ++a) {
        const int r = r0 + a;
        if (r < L)
#pragma unroll
          for (int e = 0; e < 4; ++e)
            if (4 * jq + e < NV)
              o[((size_t)(t0 + r) * H + h) * Dv + j0 + 4 * jq + e] = from_f32<Tin>(aq[a][e]);
      }
    }
    // S = Diag(gamma_C) S + Kt^T V' (Eq. 8): 4 x 4 tiles (rows 4 cq .. 4 cq + 3)
    for (int t = tid; t < dq * 8; t += kSimtThreads) {
      const int cq = t >> 3, jj = t & 7;
      float acc[4][4];
#pragma unroll
      for (int a = 0; a < 4; ++a) {
        const float g = sGam[4 * cq + a];
        const float4 sv = sS[(4 * cq + a) * 8 + jj];
        acc[a][0] = g * sv.x; acc[a][1] = g * sv.y; acc[a][2] = g * sv.z; acc[a][3] = g * sv.w;
      }
      for (int i = 0; i < C; ++i) {
        const float4 kv = sKt[i * dq + cq], v = sVp[i * 8 + jj];
        const float kx[4] = {kv.x, kv.y, kv.z, kv.w};
#pragma unroll
        for (int a = 0; a < 4; ++a) fma_s4(kx[a], v, acc[a]);
      }
#pragma unroll
      for (int a = 0; a < 4; ++a)
        sS[(4 * cq + a) * 8 + jj] = make_float4(acc[a][0], acc[a][1], acc[a][2], acc[a][3]);
    }
    __syncthreads();  // the state update is complete; A_qk, Kt and gamma_C are free
  }
}

template <typename Tin>
__global__ void __launch_bounds__(kSimtThreads)
    chunk_state_simt_kernel(const float* __restrict__ ws, SimtRecord rec, SeqGeometry geo, int H,
                            int Dk, int Dv, const float* __restrict__ initial_state,
                            float* __restrict__ final_state, Tin* __restrict__ o,
                            float* __restrict__ states_out) {
  extern __shared__ __align__(16) float smem[];
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
  const int tb = geo.seq_begin(n), te = geo.seq_end(n);
  const int c_first = geo.first_chunk(n);
  const int nchunks = te > tb ? ceil_div(te - tb, C) : 0;
#ifdef KDA_BOUNDS_CHECK
  {  // the chain's records, o rows, state slices and chunk-start states
    const size_t rf = rec.record_floats, st = (size_t)Dk * Dv;
    const bool ok =
        rows_in_bounds(kBufWork, ws + h * rf, c_first, c_first + nchunks, H * rf, rf) &&
        (!o || rows_in_bounds(kBufO, o + (size_t)h * Dv + j0, tb, te, (size_t)H * Dv, NV)) &&
        (!initial_state || rows_in_bounds(kBufInitial, initial_state + sbase + j0, 0, Dk, Dv, NV)) &&
        (!final_state || rows_in_bounds(kBufFinal, final_state + sbase + j0, 0, Dk, Dv, NV)) &&
        (!states_out ||
         rows_in_bounds(kBufWork, states_out + h * st, c_first, c_first + nchunks, H * st, st));
    if (!ok) return;  // (uniform: the whole CTA leaves)
  }
#endif

  for (int idx = tid; idx < Dk * kSlice; idx += nt) {
    const int cc = idx / kSlice, jj = idx - cc * kSlice;
    sS[idx] = (initial_state && jj < NV) ? initial_state[sbase + (size_t)cc * Dv + j0 + jj] : 0.f;
  }

  // d_k and d_v multiples of 4: 16-byte record sections and float4 register tiles
  const bool tiled = (Dk & 3) == 0 && (Dv & 3) == 0 && nt == kSimtThreads &&
                     (C == 16 || C == 32 || C == 64);
  if (tiled) {
    state_chain_tiled<Tin>(ws, rec, c_first, nchunks, tb, te, C, H, h, Dk, Dv, j0, NV, smem, o,
                           states_out);
  } else {
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
  return sizeof(float) * ((size_t)C * (Dk + 4) + 2 * (size_t)C * Dk + (size_t)C * Dv +
                          2 * (size_t)C * C + C + 2 * (size_t)Dk);
}
size_t simt_state_smem_bytes(int C, int Dk) {
  return sizeof(float) * ((size_t)Dk * kSlice + 3 * (size_t)C * Dk + 2 * (size_t)C * kSlice +
                          (size_t)C * C + Dk + kSimtRedFloats);
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
    const dim3 g1 = item_grid(max_chunks, a.H);
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
    chunk_local_simt_kernel<Tin><<<item_grid(max_chunks, a.H), kSimtThreads, sm1, stream>>>(
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
