// kda_recurrent_chunk.cu — the recurrent mode (a few tokens per sequence against pooled states) in
// the chunk form, fp32, one CTA per (sequence, head).
//
// The tokens are taken in chunks of 16 of the chunkwise form ("Kimi Linear: An Expressive,
// Efficient Attention Architecture", paper-graph-ui walkthrough, §3.4 "Chunkwise
// Parallelization"): with g_t the cumulative log decay of token t from the chunk's start and S the
// state entering the chunk,
//   A_kk[r][i] = sum_c k_r[c] k_i[c] exp(g_r[c] - g_i[c])  (i < r),  A_qk likewise with q_r (i <= r)
//   M  = (I + StrictTril(Diag(beta) A_kk))^{-1} Diag(beta)
//   W  = M (exp(g) . K),  U = M V,  V' = U - W S
//   O  = (exp(g) . Q) S + A_qk V'
//   S' = Diag(exp(g_T)) S + (K . exp(g_T - g))^T V'
// The token-by-token kernels spend most of an item in per-token reductions across the state's
// rows; here the state is read once into shared memory and enters two products, [W; Q~] S and
// K~^T V', evaluated as register-tiled fp32 products on packed pairs. The ratios exp(g_r - g_i)
// are factored around each channel's midpoint, or formed exactly per term when a channel's decay
// spans too far for the factors, so any finite decay is safe.
// The state is read from its pool row once, stays in shared memory across the chunks and is
// written back once; everything else stays on chip.

#include "kda_common.cuh"
#include "kda_internal.h"
#include "kda_sm100.cuh"

namespace kda {
namespace rchunk {

constexpr int kT = 16;         // tokens per chunk
constexpr int kD = 128;        // d_k = d_v
constexpr int kThreads = 256;  // 8 warps
constexpr float kLog2e = 1.4426950408889634f;

// shared memory (fp32 words)
constexpr int kOffS = 0;                   // S [128][128], row-major
constexpr int kOffK = kOffS + kD * kD;     // k [16][128], k exp(g - m), then K~
constexpr int kOffQ = kOffK + kT * kD;     // q, q exp(g - m) } later [W; Q~]^T [128][32]
constexpr int kOffG = kOffQ + kT * kD;     // g log2e or k exp(m - g) }  (swizzled)
constexpr int kOffV = kOffG + kT * kD;     // v, then U, then V' [16][128]
constexpr int kOffKG = kOffV + kT * kD;    // exp(g) . k [16][128]
constexpr int kOffAkk = kOffKG + kT * kD;  // Diag(beta) A_kk strict lower [16][16]
constexpr int kOffAqk = kOffAkk + kT * kT; // A_qk lower [16][16]
constexpr int kOffM = kOffAqk + kT * kT;   // M [16][16]
constexpr int kOffBeta = kOffM + kT * kT;  // beta [16]
constexpr int kOffGam = kOffBeta + kT;     // exp(g_T) [128]
constexpr int kWords = kOffGam + kD;
constexpr size_t kSmemBytes = (size_t)kWords * 4;
static_assert(kSmemBytes <= 113 * 1024, "two CTAs per SM");

// [W; Q~]^T: row = key channel (128), 32 columns (W rows 0..15, Q~ rows 16..31) in groups of four,
// the group index XOR-ed by (row % 8) so that a column of rows spreads over the banks
__device__ __forceinline__ int at_idx(int row, int col) {
  return row * 32 + ((((col >> 2) ^ (row & 7)) << 2) | (col & 3));
}

template <typename Tin>
__device__ __forceinline__ void load_row8(float* dst, const Tin* src);
template <>
__device__ __forceinline__ void load_row8<__nv_bfloat16>(float* dst, const __nv_bfloat16* src) {
  store_vec(dst, __ldg(reinterpret_cast<const uint4*>(src)), __nv_bfloat16());
}
template <>
__device__ __forceinline__ void load_row8<float>(float* dst, const float* src) {
  store_vec(dst, __ldg(reinterpret_cast<const uint4*>(src)), float());
  store_vec(dst + 4, __ldg(reinterpret_cast<const uint4*>(src) + 1), float());
}

template <typename Tin>
__device__ __forceinline__ void load8(const Tin* src, float (&f)[8]);
template <>
__device__ __forceinline__ void load8<__nv_bfloat16>(const __nv_bfloat16* src, float (&f)[8]) {
  const uint4 u = __ldg(reinterpret_cast<const uint4*>(src));
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    f[2 * j] = __uint_as_float(w[j] << 16);
    f[2 * j + 1] = __uint_as_float(w[j] & 0xffff0000u);
  }
}
template <>
__device__ __forceinline__ void load8<float>(const float* src, float (&f)[8]) {
  const float4 a = __ldg(reinterpret_cast<const float4*>(src));
  const float4 b = __ldg(reinterpret_cast<const float4*>(src) + 1);
  f[0] = a.x; f[1] = a.y; f[2] = a.z; f[3] = a.w;
  f[4] = b.x; f[5] = b.y; f[6] = b.z; f[7] = b.w;
}

template <typename Tin>
__device__ __forceinline__ void store4(Tin* dst, const float (&v)[4]);
template <>
__device__ __forceinline__ void store4<float>(float* dst, const float (&v)[4]) {
  *reinterpret_cast<float4*>(dst) = make_float4(v[0], v[1], v[2], v[3]);
}
template <>
__device__ __forceinline__ void store4<__nv_bfloat16>(__nv_bfloat16* dst, const float (&v)[4]) {
  *reinterpret_cast<uint2*>(dst) =
      make_uint2(sm100::pack_bf16(v[0], v[1]), sm100::pack_bf16(v[2], v[3]));
}

// kFused: the prologue and epilogue of kda_fusion_t — q and k L2-normalised per token, the log
// decay formed from the raw gate, the output rows normalised and gated before the store.
template <typename Tin, bool kFused>
__global__ void __launch_bounds__(kThreads, 2)
    recurrent_chunk_kernel(const Tin* __restrict__ q, const Tin* __restrict__ k,
                           const Tin* __restrict__ v, const float* __restrict__ log_alpha,
                           const float* __restrict__ beta, float* __restrict__ pool,
                           const int32_t* __restrict__ state_indices, Tin* __restrict__ o, int Tn,
                           int H, int P, Fusion fz) {
  extern __shared__ float4 smem4[];
  float* sm = reinterpret_cast<float*>(smem4);
  float* sS = sm + kOffS;
  float* sK = sm + kOffK;
  float* sQ = sm + kOffQ;
  float* sG = sm + kOffG;
  float* sAT = sm + kOffQ;  // aliases q and g once the A products have read them
  float* sV = sm + kOffV;
  float* sKG = sm + kOffKG;
  float* sAkk = sm + kOffAkk;
  float* sAqk = sm + kOffAqk;
  float* sM = sm + kOffM;
  float* sBeta = sm + kOffBeta;
  float* sGam = sm + kOffGam;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int item = blockIdx.x, n = item / H, h = item - n * H;
  const int slot = state_indices ? (KDA_IN_BOUNDS(kBufIndices, state_indices + n, 4)
                                        ? state_indices[n]
                                        : -1)
                                 : n;
  if (slot < 0) return;  // a skipped sequence: no state update, o untouched
  if (slot >= P) {
    if (tid == 0) raise_status(kStatusBadSeqlens);
    return;
  }
  float* state = pool + ((size_t)slot * H + h) * kD * kD;
  const size_t row0 = ((size_t)n * Tn) * H + h;  // the sequence's first token row
#ifdef KDA_BOUNDS_CHECK
  {
    const size_t rs = (size_t)H;
    bool ok = in_bounds(kBufState, state, (size_t)kD * kD * 4) &&
              rows_in_bounds(kBufQ, q + row0 * kD, 0, Tn, rs * kD, kD) &&
              rows_in_bounds(kBufK, k + row0 * kD, 0, Tn, rs * kD, kD) &&
              rows_in_bounds(kBufV, v + row0 * kD, 0, Tn, rs * kD, kD) &&
              rows_in_bounds(kBufLogAlpha, log_alpha + row0 * kD, 0, Tn, rs * kD, kD) &&
              rows_in_bounds(kBufBeta, beta + row0, 0, Tn, rs, 1) &&
              rows_in_bounds(kBufO, o + row0 * kD, 0, Tn, rs * kD, kD);
    if (kFused) {
      const Tin* og = reinterpret_cast<const Tin*>(fz.og);
      ok = ok && (!fz.A_log || in_bounds(kBufALog, fz.A_log + h, 4)) &&
           (!(fz.A_log && fz.dt_bias) ||
            in_bounds(kBufDtBias, fz.dt_bias + (size_t)h * kD, kD * 4)) &&
           (!(fz.onorm && fz.ow) || in_bounds(kBufNormW, fz.ow, kD * 4)) &&
           (!(fz.onorm && og) || rows_in_bounds(kBufGate, og + row0 * kD, 0, Tn, rs * kD, kD));
    }
    if (__syncthreads_or(!ok)) return;
  }
#endif

  // the state by cp.async, once for all chunks (needed from phase 5 on)
#pragma unroll
  for (int j = 0; j < (kD * kD / 4) / kThreads; ++j) {
    const int i4 = tid + j * kThreads;
    cp_async_16B(sS + 4 * i4, reinterpret_cast<const float4*>(state) + i4);
  }
  cp_async_commit();

  // the tokens in chunks of kT; the state stays in shared memory from one chunk to the next
  for (int cs = 0; cs < Tn; cs += kT) {
    const int T = min(kT, Tn - cs);             // tokens of this chunk
    const size_t rowc = row0 + (size_t)cs * H;  // its first token row
    const bool last = cs + kT >= Tn;
    // ---- phase 1: the token rows as fp32 -------------------------------------------------------
    {
      const int t = tid >> 4, c8 = (tid & 15) * 8;  // token row t, channels c8 .. c8 + 7
      if (kFused) {  // rows through registers: L2 norms over the row's 16 lanes, gate per channel
        float kx[8], qx[8], gx[8];
        const size_t r = (rowc + (size_t)t * H) * kD + c8;
        if (t < T) {
          load8<Tin>(k + r, kx);
          load8<Tin>(q + r, qx);
          load8<float>(log_alpha + r, gx);
          load_row8<Tin>(sV + t * kD + c8, v + r);
        } else {
#pragma unroll
          for (int j = 0; j < 8; ++j) kx[j] = qx[j] = gx[j] = sV[t * kD + c8 + j] = 0.f;
        }
        if (fz.l2) {
          float ssk = 0.f, ssq = 0.f;
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            ssk = fmaf(kx[j], kx[j], ssk);
            ssq = fmaf(qx[j], qx[j], ssq);
          }
#pragma unroll
          for (int off = 8; off > 0; off >>= 1) {  // the 16 lanes of this row
            ssk += __shfl_xor_sync(0xffffffffu, ssk, off);
            ssq += __shfl_xor_sync(0xffffffffu, ssq, off);
          }
          const float ik = rsqrtf(ssk + fz.eps), iq = rsqrtf(ssq + fz.eps);
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            kx[j] *= ik;
            qx[j] *= iq;
          }
        }
        if (fz.A_log && t < T) {  // log alpha = -exp(A_log[h]) softplus(g + dt_bias[h])
          const float neg_a = -expf(fz.A_log[h]);
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const float bias = fz.dt_bias ? fz.dt_bias[(size_t)h * kD + c8 + j] : 0.f;
            gx[j] = neg_a * softplus_f(gx[j] + bias);
          }
        }
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          sK[t * kD + c8 + j] = kx[j];
          sQ[t * kD + c8 + j] = qx[j];
          sG[t * kD + c8 + j] = gx[j];
        }
      } else if (t < T) {
        const size_t r = (rowc + (size_t)t * H) * kD + c8;
        load_row8<Tin>(sK + t * kD + c8, k + r);
        load_row8<Tin>(sQ + t * kD + c8, q + r);
        load_row8<Tin>(sV + t * kD + c8, v + r);
        load_row8<float>(sG + t * kD + c8, log_alpha + r);
      } else {  // padding rows: no key, no decay
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          sK[t * kD + c8 + j] = 0.f;
          sQ[t * kD + c8 + j] = 0.f;
          sV[t * kD + c8 + j] = 0.f;
          sG[t * kD + c8 + j] = 0.f;
        }
      }
      if (tid < kT) sBeta[tid] = tid < T ? beta[rowc + (size_t)tid * H] : 0.f;
      for (int i = tid; i < 2 * kT * kT; i += kThreads) sAkk[i] = 0.f;  // A_kk and A_qk
    }
    __syncthreads();

    // ---- phase 2: cumulative decay per channel; exp(g) . k; Q~ and K~ kept in registers ---------
    // The A products take each channel's ratios exp(g_r - g_i) as k_r exp(g_r - m) times
    // k_i exp(m - g_i) around the midpoint m of the channel's range of g, both factors within
    // 2^(span / 2) (span = that range in log2 units). An item with a channel spanning more than
    // kSpanMax takes every ratio exactly instead (slower).
    constexpr float kSpanMax = 200.f;
    // thread = channel c and half of the tokens (8 half .. + 7); both halves run the channel's scan
    const int c = tid & (kD - 1), th0 = 8 * (tid >> 7);
    float qt[8], kt[8], gl[kT], gmid;
    bool wide;
    {
      float run = 0.f;
#pragma unroll
      for (int t = 0; t < kT; ++t) {
        run += sG[t * kD + c];
        gl[t] = run * kLog2e;
      }
      if (th0 == 0) sGam[c] = exp2f(gl[kT - 1]);
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int t = th0 + j;
        const float gt = th0 ? gl[8 + j] : gl[j];  // (constant indices: gl stays in registers)
        const float e = exp2f(gt), kv = sK[t * kD + c];
        sKG[t * kD + c] = kv * e;
        qt[j] = sQ[t * kD + c] * e;
        kt[j] = kv * exp2f(gl[kT - 1] - gt);
      }
      float lo = gl[0], hi = gl[0];  // (log decays are <= 0, so g falls; any sign is handled)
#pragma unroll
      for (int t = 1; t < kT; ++t) {
        lo = fminf(lo, gl[t]);
        hi = fmaxf(hi, gl[t]);
      }
      wide = !(hi - lo <= kSpanMax);  // (a NaN decay takes the exact form too)
      gmid = 0.5f * (lo + hi);
    }
    wide = __syncthreads_or(wide) != 0;  // the item's form, known to every thread
    if (wide) {
#pragma unroll
      for (int j = 0; j < 8; ++j) sG[(th0 + j) * kD + c] = th0 ? gl[8 + j] : gl[j];
    } else {  // k exp(g - m), q exp(g - m) in place of k, q; k exp(m - g) in place of g
      const float m = gmid;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int t = th0 + j;
        const float gt = th0 ? gl[8 + j] : gl[j];
        const float ep = exp2f(gt - m), em = exp2f(m - gt);
        const float kv = sK[t * kD + c];
        sK[t * kD + c] = kv * ep;
        sQ[t * kD + c] = sQ[t * kD + c] * ep;
        sG[t * kD + c] = kv * em;
      }
    }
    __syncthreads();

    // ---- phase 3: A_kk, A_qk ---------------------------------------------------------------
    if (!wide) {  // thread = pair (r, i); channels rotated by i so the 16 rows i spread over banks
      const int r = tid >> 4, i = tid & 15;
      float akk = 0.f, aqk = 0.f;
#pragma unroll 8
      for (int j = 0; j < kD / 4; ++j) {
        const int c4 = 4 * ((j + i) & (kD / 4 - 1));
        const float4 kr = *reinterpret_cast<const float4*>(sK + r * kD + c4);
        const float4 qr = *reinterpret_cast<const float4*>(sQ + r * kD + c4);
        const float4 ki = *reinterpret_cast<const float4*>(sG + i * kD + c4);
        akk = fmaf(kr.x, ki.x, fmaf(kr.y, ki.y, fmaf(kr.z, ki.z, fmaf(kr.w, ki.w, akk))));
        aqk = fmaf(qr.x, ki.x, fmaf(qr.y, ki.y, fmaf(qr.z, ki.z, fmaf(qr.w, ki.w, aqk))));
      }
      if (r < T) {
        if (i < r) sAkk[r * kT + i] = sBeta[r] * akk;
        if (i <= r) sAqk[r * kT + i] = aqk;
      }
    } else {  // exact ratios: warp = pairs (r, i), lane = four channels
      const int c4 = 4 * lane;
      for (int p = warp; p < kT * (kT + 1) / 2; p += kThreads / 32) {
        int r = 0;
        while ((r + 1) * (r + 2) / 2 <= p) ++r;
        const int i = p - r * (r + 1) / 2;
        if (r >= T) continue;  // warp-uniform: padding rows stay zero
        const float4 kr = *reinterpret_cast<const float4*>(sK + r * kD + c4);
        const float4 ki = *reinterpret_cast<const float4*>(sK + i * kD + c4);
        const float4 qr = *reinterpret_cast<const float4*>(sQ + r * kD + c4);
        const float4 gr = *reinterpret_cast<const float4*>(sG + r * kD + c4);
        const float4 gi = *reinterpret_cast<const float4*>(sG + i * kD + c4);
        const float e0 = exp2f(gr.x - gi.x), e1 = exp2f(gr.y - gi.y);
        const float e2 = exp2f(gr.z - gi.z), e3 = exp2f(gr.w - gi.w);
        const float b0 = ki.x * e0, b1 = ki.y * e1, b2 = ki.z * e2, b3 = ki.w * e3;
        float akk = kr.x * b0 + kr.y * b1 + kr.z * b2 + kr.w * b3;
        float aqk = qr.x * b0 + qr.y * b1 + qr.z * b2 + qr.w * b3;
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
          akk += __shfl_xor_sync(0xffffffffu, akk, off);
          aqk += __shfl_xor_sync(0xffffffffu, aqk, off);
        }
        if (lane == 0) {
          if (i < r) sAkk[r * kT + i] = sBeta[r] * akk;
          sAqk[r * kT + i] = aqk;
        }
      }
    }
    __syncthreads();

    // ---- phase 4: Q~ and K~ out of the registers (q and g are dead); M by forward substitution --
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      sAT[at_idx(c, kT + th0 + j)] = qt[j];
      sK[(th0 + j) * kD + c] = kt[j];
    }
    if (warp == 0 && lane < kT) {  // column `lane` of (I + A)^{-1}, then M = T Diag(beta)
      float col[kT];
#pragma unroll
      for (int i = 0; i < kT; ++i) {
        float val = (i == lane) ? 1.f : 0.f;
#pragma unroll
        for (int m = 0; m < i; ++m) val -= sAkk[i * kT + m] * col[m];
        col[i] = val;
      }
      const float bj = sBeta[lane];
#pragma unroll
      for (int i = 0; i < kT; ++i) sM[i * kT + lane] = col[i] * bj;
    }
    __syncthreads();

    // ---- phase 5: W = M (exp(g) . K) into [W; Q~]^T, U = M V over V (rows 8 half .. + 7) -------
    {
      const int c = tid & (kD - 1), half = tid >> 7;
      float w[8], u[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) w[j] = u[j] = 0.f;
#pragma unroll
      for (int t = 0; t < kT; ++t) {
        const float kg = sKG[t * kD + c], vv = sV[t * kD + c];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const float m = sM[(8 * half + j) * kT + t];  // zero for t > row
          w[j] = fmaf(m, kg, w[j]);
          u[j] = fmaf(m, vv, u[j]);
        }
      }
#pragma unroll
      for (int j = 0; j < 8; ++j) sAT[at_idx(c, 8 * half + j)] = w[j];
      __syncthreads();  // every thread has read V
#pragma unroll
      for (int j = 0; j < 8; ++j) sV[(8 * half + j) * kD + c] = u[j];
    }
    cp_async_wait<0>();
    __syncthreads();
    if (kFused && fz.onorm && fz.og) {  // the chunk's output-gate rows into the dead exp(g) . k
      // buffer, in flight under the [W; Q~] S product
      constexpr int kPerRow = kD * (int)sizeof(Tin) / 16;  // 16-byte words per row
      const Tin* og = reinterpret_cast<const Tin*>(fz.og);
      for (int w = tid; w < kT * kPerRow; w += kThreads) {
        const int t = w / kPerRow, c16 = w - t * kPerRow;
        if (t < T)
          cp_async_16B(reinterpret_cast<Tin*>(sKG) + t * kD + c16 * (16 / (int)sizeof(Tin)),
                       og + (rowc + (size_t)t * H) * kD + c16 * (16 / (int)sizeof(Tin)));
      }
      cp_async_commit();
    }

    // ---- phase 6: [W; Q~] S; V' = U - W S; O = Q~ S + A_qk V' -----------------------------------
    // warp = 16 state columns, lane = 4 rows (mg) x 4 columns (cg) of the 32 x 128 product; the
    // accumulators stay packed pairs of adjacent columns
    {
      const int mg = lane >> 2, cg = lane & 3, col = 16 * warp + 4 * cg;
      f32x2 acc[4][2];
#pragma unroll
      for (int a = 0; a < 4; ++a) acc[a][0] = acc[a][1] = f2_pack(0.f, 0.f);
#pragma unroll 32
      for (int kk = 0; kk < kD; ++kk) {
        const float4 a = *reinterpret_cast<const float4*>(sAT + kk * 32 + ((mg ^ (kk & 7)) << 2));
        const float4 sv = *reinterpret_cast<const float4*>(sS + kk * kD + col);
        const f32x2 s01 = f2_pack(sv.x, sv.y), s23 = f2_pack(sv.z, sv.w);
        const float av[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
        for (int r = 0; r < 4; ++r) {
          const f32x2 ar = f2_pack(av[r], av[r]);
          acc[r][0] = f2_fma(ar, s01, acc[r][0]);
          acc[r][1] = f2_fma(ar, s23, acc[r][1]);
        }
      }
      if (mg < 4) {  // rows 4 mg .. + 3 of W S: V' in place of U
#pragma unroll
        for (int r = 0; r < 4; ++r) {
          float4* up = reinterpret_cast<float4*>(sV + (4 * mg + r) * kD + col);
          const float4 uu = *up;
          const float2 lo = f2_unpack(acc[r][0]), hi = f2_unpack(acc[r][1]);
          *up = make_float4(uu.x - lo.x, uu.y - lo.y, uu.z - hi.x, uu.w - hi.y);
        }
      }
      __syncwarp();  // this warp's 16 columns of V' are complete
      const int t0 = 4 * (mg - 4);  // output rows t0 .. t0 + 3 (lanes with mg >= 4)
      if (mg >= 4) {
#pragma unroll
        for (int tau = 0; tau < kT; ++tau) {
          const float4 vp = *reinterpret_cast<const float4*>(sV + tau * kD + col);
          const f32x2 v01 = f2_pack(vp.x, vp.y), v23 = f2_pack(vp.z, vp.w);
#pragma unroll
          for (int r = 0; r < 4; ++r) {
            const float aq = sAqk[(t0 + r) * kT + tau];
            const f32x2 ar = f2_pack(aq, aq);
            acc[r][0] = f2_fma(ar, v01, acc[r][0]);
            acc[r][1] = f2_fma(ar, v23, acc[r][1]);
          }
        }
      }
      float y[4][4];
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        const float2 lo = f2_unpack(acc[r][0]), hi = f2_unpack(acc[r][1]);
        y[r][0] = lo.x;
        y[r][1] = lo.y;
        y[r][2] = hi.x;
        y[r][3] = hi.y;
      }
      if (kFused && fz.onorm) {  // y = sigmoid(gate) weight o / RMS over the row's 128 columns
        float* sPart = sAkk;     // [8 warps][16 rows] partial sums of squares (A_kk is dead)
#pragma unroll
        for (int r = 0; r < 4; ++r) {
          float ss = y[r][0] * y[r][0] + y[r][1] * y[r][1] + y[r][2] * y[r][2] + y[r][3] * y[r][3];
          ss += __shfl_xor_sync(0xffffffffu, ss, 1);  // the four lanes of this row's 16 columns
          ss += __shfl_xor_sync(0xffffffffu, ss, 2);
          if (mg >= 4 && cg == 0) sPart[warp * kT + t0 + r] = ss;
        }
        cp_async_wait<0>();  // this thread's gate-row copies
        __syncthreads();
        if (mg >= 4) {
          const Tin* sOg = reinterpret_cast<const Tin*>(sKG);  // the staged gate rows
#pragma unroll
          for (int r = 0; r < 4; ++r) {
            const int t = t0 + r;
            float tot = 0.f;
#pragma unroll
            for (int w = 0; w < kThreads / 32; ++w) tot += sPart[w * kT + t];
            const float inv = rsqrtf(tot * (1.f / kD) + fz.oeps);
#pragma unroll
            for (int c = 0; c < 4; ++c) {
              float f = inv * (fz.ow ? fz.ow[col + c] : 1.f);
              if (fz.og && t < T) f *= sigmoid_f(to_f32(sOg[t * kD + col + c]));
              y[r][c] *= f;
            }
          }
        }
      }
      if (mg >= 4) {
#pragma unroll
        for (int r = 0; r < 4; ++r) {
          const int t = t0 + r;
          if (t < T) store4<Tin>(o + (rowc + (size_t)t * H) * kD + col, y[r]);
        }
      }
    }
    __syncthreads();

    // ---- phase 7: S' = Diag(exp(g_T)) S + K~^T V', into the pool row after the last chunk -----
    // warp = 16 state rows, lane = 4 columns (two packed pairs)
    {
      const int r0 = 16 * warp, c4 = 4 * lane;
      f32x2 acc[16][2];
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const float4 sv = *reinterpret_cast<const float4*>(sS + (r0 + i) * kD + c4);
        const float g = sGam[r0 + i];
        const f32x2 gg = f2_pack(g, g);
        acc[i][0] = f2_mul(gg, f2_pack(sv.x, sv.y));
        acc[i][1] = f2_mul(gg, f2_pack(sv.z, sv.w));
      }
      for (int t = 0; t < T; ++t) {
        const float4 vp = *reinterpret_cast<const float4*>(sV + t * kD + c4);
        const f32x2 v01 = f2_pack(vp.x, vp.y), v23 = f2_pack(vp.z, vp.w);
#pragma unroll
        for (int i4 = 0; i4 < 4; ++i4) {
          const float4 kk = *reinterpret_cast<const float4*>(sK + t * kD + r0 + 4 * i4);
          const float kv[4] = {kk.x, kk.y, kk.z, kk.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const f32x2 kr = f2_pack(kv[e], kv[e]);
            acc[4 * i4 + e][0] = f2_fma(kr, v01, acc[4 * i4 + e][0]);
            acc[4 * i4 + e][1] = f2_fma(kr, v23, acc[4 * i4 + e][1]);
          }
        }
      }
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const float2 lo = f2_unpack(acc[i][0]), hi = f2_unpack(acc[i][1]);
        const float4 sv = make_float4(lo.x, lo.y, hi.x, hi.y);
        if (last)
          *reinterpret_cast<float4*>(state + (size_t)(r0 + i) * kD + c4) = sv;
        else  // (each thread rewrites only the elements it read)
          *reinterpret_cast<float4*>(sS + (r0 + i) * kD + c4) = sv;
      }
    }
    __syncthreads();  // the token buffers and S are rewritten by the next chunk
  }
}

}  // namespace rchunk

// The recurrent mode through the chunk-form kernel: T >= 2, d_k = d_v = 128, 16-byte aligned rows.
// Returns false (nothing launched) when the call does not qualify.
static bool recurrent_chunk_applies(kda_dtype_t dt, int T, int Dk, int Dv, const void* q,
                                    const void* k, const void* v, const float* log_alpha,
                                    const float* pool, const void* o, const Fusion& fz) {
  auto al16 = [](const void* p) { return ((uintptr_t)p & 15u) == 0; };
  return T >= 2 && Dk == rchunk::kD && Dv == rchunk::kD &&
         (dt == KDA_DTYPE_BF16 || dt == KDA_DTYPE_F32) && al16(q) && al16(k) && al16(v) &&
         al16(log_alpha) && al16(pool) && ((uintptr_t)o & (dt == KDA_DTYPE_BF16 ? 7u : 15u)) == 0 &&
         (!(fz.onorm && fz.og) || al16(fz.og));
}

template <typename Tin, bool kFused>
static cudaError_t launch_rchunk_typed(const void* q, const void* k, const void* v,
                                       const float* log_alpha, const float* beta, float* pool,
                                       const int32_t* idx, void* o, long long heads, int T, int H,
                                       int P, const Fusion& fz, cudaStream_t stream) {
  const int smem = (int)rchunk::kSmemBytes;
  cudaError_t err = cudaFuncSetAttribute(rchunk::recurrent_chunk_kernel<Tin, kFused>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (err == cudaSuccess)  // two CTAs per SM: the whole unified array as shared memory
    err = cudaFuncSetAttribute(rchunk::recurrent_chunk_kernel<Tin, kFused>,
                               cudaFuncAttributePreferredSharedMemoryCarveout, 100);
  if (err != cudaSuccess) return err;
  rchunk::recurrent_chunk_kernel<Tin, kFused><<<(unsigned)heads, rchunk::kThreads, smem, stream>>>(
      (const Tin*)q, (const Tin*)k, (const Tin*)v, log_alpha, beta, pool, idx, (Tin*)o, T, H, P,
      fz);
  return cudaGetLastError();
}

static cudaError_t launch_recurrent_chunk(const void* q, const void* k, const void* v,
                                          kda_dtype_t dt, const float* log_alpha,
                                          const float* beta, float* pool, const int32_t* idx,
                                          void* o, long long heads, int T, int H, int P,
                                          const Fusion& fz, cudaStream_t stream) {
  if (heads > INT32_MAX) return cudaErrorInvalidConfiguration;
  const bool fused = fz.l2 || fz.A_log || fz.onorm;
  ProfileScope prof(fused ? "recurrent_chunk_fused" : "recurrent_chunk", stream);
  if (dt == KDA_DTYPE_BF16)
    return fused ? launch_rchunk_typed<__nv_bfloat16, true>(q, k, v, log_alpha, beta, pool, idx,
                                                             o, heads, T, H, P, fz, stream)
                 : launch_rchunk_typed<__nv_bfloat16, false>(q, k, v, log_alpha, beta, pool, idx,
                                                              o, heads, T, H, P, fz, stream);
  return fused ? launch_rchunk_typed<float, true>(q, k, v, log_alpha, beta, pool, idx, o, heads,
                                                  T, H, P, fz, stream)
               : launch_rchunk_typed<float, false>(q, k, v, log_alpha, beta, pool, idx, o, heads,
                                                   T, H, P, fz, stream);
}

}  // namespace kda
