// kda_chunk_tc.cu — tensor-core (tcgen05) chunkwise prefill of KDA for bf16 q/k/v, d = 128, C = 64.
//
// Same two-kernel structure as the fp32 CUDA-core path, following "Kimi Linear: An Expressive,
// Efficient Attention Architecture" (paper-graph-ui walkthrough, §3.4 "Chunkwise
// Parallelization"), with every dense chunk contraction on the fifth-generation tensor cores:
//
//   K1 chunk_local_tc  one CTA per (chunk, head):
//        g = cumulative log decay (fp32); Kg = Gamma.K, Ki = K/Gamma, Qg = Gamma.Q (bf16 tiles)
//        A_kk = Kg Ki^T, A_qk = Qg Ki^T                      (tcgen05, fp32 in TMEM)
//        M = (I + StrictTril(Diag(beta) A_kk))^{-1} Diag(beta)  (blocked forward substitution, fp32)
//        W = M Kg, U = M V                                   (tcgen05)
//      and writes one bf16 record per (chunk, head): W, Qt = Qg, Kt = (gamma_C/gamma_i) k_i, the
//      masked A_qk, U, gamma_C — every tile already in the tensor-core operand layout, so K2 moves
//      it with plain bulk copies.
//   K2 chunk_state_tc  one CTA per (sequence, head, 64-column half of d_v), sequential in chunks:
//        D1 = W S, D2 = Qt S  ->  V' = U - D1  ->  D3 = Kt^T V', D2 += A_qk V'
//        S = Diag(gamma_C) S + D3 (Eq. 8, fp32 in registers),  O = D2 (Eq. 9)
//      Warp roles: a bulk-copy producer (double-buffered records), a single MMA-issuing thread,
//      8 epilogue warps, 32 columns of S each (one row of S per thread, in fp32 registers).
//
// The ratio exp(g_r - g_i) inside A_kk and A_qk is split into two bf16 factors around a reference
// log decay, and each factor must stay inside bf16 range. Three cases per (chunk, head):
//   fast   every channel decays by less than exp(-L) over the chunk: one reference (the chunk
//          start), K/Gamma = k * exp(-g), one pair of MMAs;
//   blocks some channel decays harder, but none by more than exp(-L) within any 16-row block:
//          row block R takes the reference g at the end of block R-1, so the row factor
//          k_r exp(g_r - ref_R) is <= 1 and the column factor k_i exp(ref_R - g_i) is <= 1 for
//          earlier blocks and <= exp(L) inside block R; three rounds of MMAs cover the four row
//          blocks (the column tile is rebuilt per reference);
//   exact  otherwise: a CUDA-core evaluation of every product with ratios exp(g_r - g_i) <= 1.
#include "kda_common.cuh"
#include "kda_internal.h"
#include "kda_sm100.cuh"

namespace kda {
namespace tc {

using namespace sm100;

constexpr int kC = 64;
constexpr int kD = 128;
// Log-decay range bound L of one bf16 factorisation: the factors k exp(+-g) stay below
// |k| exp(L) inside bf16's range. L = 80 when the keys are L2-normalised in the kernel
// (|k| <= 1; the discarded upper triangle of A_kk may overflow in its fp32 accumulator without
// being read), L = 60 for caller-provided keys (any |k| below ~1e12).
constexpr float kDecayLimitNormalisedKeys = 80.f;
constexpr float kDecayLimitRawKeys = 60.f;
constexpr int kModeFast = 0, kModeBlocks = 1, kModeExact = 2;

// record layout (bytes) of one (chunk, head). QW is a [128 x 128] tile (64-column blocks
// 16 KiB apart): rows 0..63 hold Qt = Gamma.Q, rows 64..127 hold W, so one M = 128 MMA
// computes [Qt; W] S.
constexpr uint32_t kRecQW = 0;
constexpr uint32_t kRecKt = 32768;
constexpr uint32_t kRecAqk = 49152;
constexpr uint32_t kRecU = 57344;
constexpr uint32_t kRecGam = 73728;
constexpr uint32_t kRecBytes = 74240;
__device__ __forceinline__ uint32_t qw_chunk_off(int row128, int c8) {
  return tile_chunk_off(row128, c8, 16384);
}
// exact-fallback scratch for the cumulative decay g (fp32 [64][128]) inside the record: the W
// half of QW (rows 0..31) and U (rows 32..63), both written only after g is consumed
__device__ __forceinline__ uint32_t g_scratch_off(int r) {
  return r < 16 ? kRecQW + 8192u + (uint32_t)r * 512u
                : (r < 32 ? kRecQW + 24576u + (uint32_t)(r - 16) * 512u
                          : kRecU + (uint32_t)(r - 32) * 512u);
}
static_assert(kRecBytes == TcRecordBytes, "record size mismatch");

// ============================================================================================
// K1
// ============================================================================================
constexpr int kK1Threads = 256;
constexpr int kK1Tmem = 128;  // A_kk | A_qk, then W, then U

// shared-memory map of K1 (offsets from a 1024-aligned base). Three CTAs fit on an SM.
constexpr uint32_t kS1Kg = 0;         // [64 x 128] bf16: raw k, then Gamma.K
constexpr uint32_t kS1Ki = 16384;     // [64 x 128] bf16: scan partials, then K/Gamma, then fp32 A
constexpr uint32_t kS1Qg = 32768;     // [64 x 128] bf16: raw q, then Gamma.Q, then fp32 T
constexpr uint32_t kS1V = 49152;      // [64 x 128] bf16 v
constexpr uint32_t kS1M = 65536;      // [64 x 64] bf16 M (the level products X alias it first)
constexpr uint32_t kS1Inv = kS1M;     // fp32 [2][64] inverse norms of k and q, until phase 4
constexpr uint32_t kS1Ref = kS1M + 1024;  // fp32 [4][128] g at rows 15, 31, 47, 63 (row 3 = g_C)
constexpr uint32_t kS1Beta = 73728;   // fp32 [64]
constexpr uint32_t kS1Bar = 73984;    // mbarrier
constexpr uint32_t kS1Tmem = 73992;   // TMEM base address
constexpr uint32_t kS1Bytes = 74000;

// fp32 64 x 64 matrices (A, T) are stored row-major with column bits 2..5 XOR-ed by (row % 16):
// groups of four consecutive columns stay contiguous (128-bit accesses) while sixteen consecutive
// rows of one column group spread over the banks.
__device__ __forceinline__ int sidx(int r, int c) { return r * 64 + (c ^ ((r & 15) << 2)); }
__device__ __forceinline__ float4 lds4(const float* base, int r, int c4) {  // cols 4*c4 .. +3
  return *reinterpret_cast<const float4*>(base + sidx(r, 4 * c4));
}
__device__ __forceinline__ void sts4(float* base, int r, int c4, float4 v) {
  *reinterpret_cast<float4*>(base + sidx(r, 4 * c4)) = v;
}
// the level product Y (fp32 32 x 32) of the inverse: column groups of four XOR-ed by (row % 8),
// so that eight consecutive rows of one group, or eight groups of one row, hit distinct banks
__device__ __forceinline__ int yidx(int r, int c4) { return r * 32 + 4 * (c4 ^ (r & 7)); }

__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint4 v) {
  asm volatile("st.shared.v4.b32 [%0], {%1,%2,%3,%4};" ::"r"(addr), "r"(v.x), "r"(v.y), "r"(v.z),
               "r"(v.w)
               : "memory");
}
__device__ __forceinline__ uint4 ld_shared_v4(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.b32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(addr)
               : "memory");
  return v;
}
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() {
  asm volatile("cp.async.commit_group;\n\tcp.async.wait_group 0;" ::: "memory");
}

__device__ __forceinline__ void unpack8(uint4 u, float (&f)[8]) {
  float2 a = unpack_bf16(u.x), b = unpack_bf16(u.y), c = unpack_bf16(u.z), d = unpack_bf16(u.w);
  f[0] = a.x; f[1] = a.y; f[2] = b.x; f[3] = b.y; f[4] = c.x; f[5] = c.y; f[6] = d.x; f[7] = d.y;
}
__device__ __forceinline__ uint4 pack8(const float (&f)[8]) {
  return make_uint4(pack_bf16(f[0], f[1]), pack_bf16(f[2], f[3]), pack_bf16(f[4], f[5]),
                    pack_bf16(f[6], f[7]));
}

// TMEM [0, 128) of an M = 64 accumulator -> bf16 record tile rows (lanes 0..15 of each warp of
// warps 0..3 own rows 16*warp + lane; warps 4..7 take the upper 64 columns).
__device__ __forceinline__ void readout_rows_bf16(uint32_t tmem, int warp, int lane,
                                                  uint8_t* dst_tile, int row_off,
                                                  uint32_t block_bytes) {
  const int sp = warp & 3, half = warp >> 2;
  const int r = sp * 16 + (lane & 15);
  float va[32];
#pragma unroll
  for (int part = 0; part < 2; ++part) {
    const int col0 = half * 64 + part * 32;
    tmem_ld32(tmem_at(tmem, sp * 32, col0), va);
    tmem_ld_wait();
    if (lane < 16) {
#pragma unroll
      for (int c8 = 0; c8 < 4; ++c8) {
        float f[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) f[j] = va[c8 * 8 + j];
        *reinterpret_cast<uint4*>(dst_tile +
                                  tile_chunk_off(r + row_off, (col0 >> 3) + c8, block_bytes)) =
            pack8(f);
      }
    }
  }
}

// softplus for the in-kernel gate of this bf16 path: max(x, 0) + log(1 + exp(-|x|)) with the
// hardware exp2/log2 approximations. Its absolute error (below 1e-6 per token) is far under what
// the bf16 operands' rounding does to the decays; the fp32 paths keep the accurate form.
__device__ __forceinline__ float softplus_approx(float x) {
  return fmaxf(x, 0.f) + __logf(1.f + __expf(-fabsf(x)));
}

// The reference of a channel in the shifted fast mode: half its decay over the chunk when that
// exceeds exp(-L), else the chunk start.
__device__ __forceinline__ float shift_ref(float g_c, float limit) {
  return g_c < -limit ? 0.5f * g_c : 0.f;
}

// kGate: the instance for calls with the in-kernel decay gate (A_log given). It forms the log
// decays from the raw gates and has the shifted fast mode for the strong decays such gates give;
// the instance for caller-given log decays has neither (the extra code slowed its common path).
template <bool kGate>
__global__ void __launch_bounds__(kK1Threads, 3)
    chunk_local_tc_kernel(const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k,
                          const __nv_bfloat16* __restrict__ v, const float* __restrict__ log_alpha,
                          const float* __restrict__ beta, SeqGeometry geo, int H,
                          uint8_t* __restrict__ ws_records, Fusion fz) {
  extern __shared__ uint8_t smem_raw[];
  if (!geo.ok()) return;
  const int c = blockIdx.x, h = blockIdx.y;
  if (c >= geo.num_chunks_total()) return;

  uint8_t* sm = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
  const uint32_t sb = smem_u32(sm);
  float* sA = reinterpret_cast<float*>(sm + kS1Ki);
  float* sT = reinterpret_cast<float*>(sm + kS1Qg);
  float* sX = reinterpret_cast<float*>(sm + kS1M);
  float* sBeta = reinterpret_cast<float*>(sm + kS1Beta);
  float* sScan = reinterpret_cast<float*>(sm + kS1Ki);  // [16][128], before K/Gamma exists
  float* sInv = reinterpret_cast<float*>(sm + kS1Inv);
  float* sRef = reinterpret_cast<float*>(sm + kS1Ref);
  const float* sGC = sRef + 3 * kD;  // the chunk's cumulative log decay g_C
  uint64_t* bar = reinterpret_cast<uint64_t*>(sm + kS1Bar);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + kS1Tmem);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int n = geo.seq_of_chunk(c);
  const int t0 = geo.seq_begin(n) + (c - geo.first_chunk(n)) * kC;
  const int L = min(kC, geo.seq_end(n) - t0);
  uint8_t* rec = ws_records + (size_t)kRecBytes * ((size_t)c * H + h);
#ifdef KDA_BOUNDS_CHECK
  if (!KDA_IN_BOUNDS(kBufWork, rec, kRecBytes)) return;  // (uniform: the whole CTA leaves)
#endif

  // ---- phase 1: raw k, q, v straight into their operand tiles; log decay into registers ------
  const int cg = tid & 15, rg = tid >> 4;  // thread = 8 channels (one 16-byte chunk) x 4 rows
  float g[4][8];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int r = rg * 4 + i;
    const uint32_t off = tile_chunk_off(r, cg, 8192);
    if (r < L KDA_AND_IN_BOUNDS(kBufK, k + ((size_t)(t0 + r) * H + h) * kD + cg * 8, 16)
              KDA_AND_IN_BOUNDS(kBufQ, q + ((size_t)(t0 + r) * H + h) * kD + cg * 8, 16)
              KDA_AND_IN_BOUNDS(kBufV, v + ((size_t)(t0 + r) * H + h) * kD + cg * 8, 16)
              KDA_AND_IN_BOUNDS(kBufLogAlpha,
                                log_alpha + ((size_t)(t0 + r) * H + h) * kD + cg * 8, 32)) {
      const size_t row = (size_t)(t0 + r) * H + h;
      cp_async16(sb + kS1Kg + off, reinterpret_cast<const uint4*>(k + row * kD) + cg);
      cp_async16(sb + kS1Qg + off, reinterpret_cast<const uint4*>(q + row * kD) + cg);
      cp_async16(sb + kS1V + off, reinterpret_cast<const uint4*>(v + row * kD) + cg);
      const float4* lp = reinterpret_cast<const float4*>(log_alpha + row * kD) + 2 * cg;
      const float4 a0 = __ldg(lp), a1 = __ldg(lp + 1);
      g[i][0] = a0.x; g[i][1] = a0.y; g[i][2] = a0.z; g[i][3] = a0.w;
      g[i][4] = a1.x; g[i][5] = a1.y; g[i][6] = a1.z; g[i][7] = a1.w;
    } else {  // identity padding: log alpha = 0, k = q = v = 0
      const uint4 z = make_uint4(0, 0, 0, 0);
      st_shared_v4(sb + kS1Kg + off, z);
      st_shared_v4(sb + kS1Qg + off, z);
      st_shared_v4(sb + kS1V + off, z);
#pragma unroll
      for (int j = 0; j < 8; ++j) g[i][j] = 0.f;
    }
  }
  if (tid < kC)
    sBeta[tid] = (tid < L KDA_AND_IN_BOUNDS(kBufBeta, beta + (size_t)(t0 + tid) * H + h, 4))
                     ? beta[(size_t)(t0 + tid) * H + h]
                     : 0.f;
  // the tensor memory and the barrier are first used in phase 3: set them up while the loads
  // above are in flight
  if (warp == 7) {
    tmem_alloc(tmem_slot, kK1Tmem);
    tmem_relinquish();
    tc_fence_before();
  }
  if (tid == 224) {
    mbar_init(bar, 1);
    fence_mbar_init();
  }
  if (kGate && fz.A_log) {  // fused gate: the loaded values are raw gates; valid rows become log
                            // decays
#ifdef KDA_BOUNDS_CHECK
    const float neg_a = KDA_IN_BOUNDS(kBufALog, fz.A_log + h, 4) ? -expf(fz.A_log[h]) : 0.f;
    const bool bias_ok =
        fz.dt_bias && KDA_IN_BOUNDS(kBufDtBias, fz.dt_bias + h * kD + cg * 8, 32);
#else
    const float neg_a = -expf(fz.A_log[h]);
    const bool bias_ok = fz.dt_bias != nullptr;
#endif
    float bias[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) bias[j] = bias_ok ? fz.dt_bias[h * kD + cg * 8 + j] : 0.f;
#pragma unroll
    for (int i = 0; i < 4; ++i)
      if (rg * 4 + i < L)
#pragma unroll
        for (int j = 0; j < 8; ++j) g[i][j] = neg_a * softplus_approx(g[i][j] + bias[j]);
  }
#pragma unroll
  for (int i = 1; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 8; ++j) g[i][j] += g[i - 1][j];
  {  // 128-bit accesses: eight lanes of a row segment cover all 32 banks once
    float4* sc = reinterpret_cast<float4*>(sScan + rg * kD + cg * 8);
    sc[0] = make_float4(g[3][0], g[3][1], g[3][2], g[3][3]);
    sc[1] = make_float4(g[3][4], g[3][5], g[3][6], g[3][7]);
  }
  __syncthreads();
  if (tid < kD) {  // exclusive prefix over the 16 row groups in place, one channel per thread
    float acc = 0.f;
#pragma unroll
    for (int r2 = 0; r2 < 16; ++r2) {
      const float x = sScan[r2 * kD + tid];
      sScan[r2 * kD + tid] = acc;
      acc += x;
    }
  }
  __syncthreads();
  {
    const float4* sc = reinterpret_cast<const float4*>(sScan + rg * kD + cg * 8);
    const float4 a = sc[0], b = sc[1];
    const float pre[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 8; ++j) g[i][j] += pre[j];
  }
  if ((rg & 3) == 3) {  // the last row of each 16-row block: the block references and g_C
    float4* gcp = reinterpret_cast<float4*>(sRef + (rg >> 2) * kD + cg * 8);
    gcp[0] = make_float4(g[3][0], g[3][1], g[3][2], g[3][3]);
    gcp[1] = make_float4(g[3][4], g[3][5], g[3][6], g[3][7]);
  }
  cp_async_wait_all();
  // the threads of the chunk's last rows hold g_C: fast mode iff every channel's is above -L
  const float decay_limit = fz.l2 ? kDecayLimitNormalisedKeys : kDecayLimitRawKeys;
  float gmin = 0.f;
#pragma unroll
  for (int j = 0; j < 8; ++j) gmin = fminf(gmin, g[3][j]);
  const bool fast = __syncthreads_and(rg != 15 || gmin >= -decay_limit) != 0;
  // Up to exp(-2L) over the chunk the fast evaluation still holds around a per-channel reference
  // m = g_C / 2 (for the channels with g_C < -L): the factors k exp(g - m), k exp(m - g) then stay
  // within e^+-L. Gamma.Q for the record and Gamma.K for W are rescaled by e^m.
  bool shifted = false;
  if constexpr (kGate)
    shifted = !fast && __syncthreads_and(rg != 15 || gmin >= -2.f * decay_limit) != 0;
  float egc[8];
  {
    const float4* gcp = reinterpret_cast<const float4*>(sGC + cg * 8);
    const float4 a = gcp[0], b = gcp[1];
    const float gcv[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
    if constexpr (kGate) {
#pragma unroll
      for (int j = 0; j < 8; ++j) egc[j] = __expf(gcv[j] - shift_ref(sGC[cg * 8 + j], decay_limit));
    } else {
#pragma unroll
      for (int j = 0; j < 8; ++j)
        egc[j] = __expf(gcv[j]);  // only scales a bf16 operand; the carried gamma_C uses expf
    }
  }
  int mode = kModeFast;
  if (!fast && !shifted) {
    bool blocks_ok = true;  // every channel's decay within every 16-row block
    if (tid < kD) {
      float prev = 0.f;
#pragma unroll
      for (int R = 0; R < 4; ++R) {
        const float next = sRef[R * kD + tid];
        blocks_ok = blocks_ok && (prev - next <= decay_limit);
        prev = next;
      }
    }
    mode = __syncthreads_and(blocks_ok) ? kModeBlocks : kModeExact;
  }
  if (tid < kD) reinterpret_cast<float*>(rec + kRecGam)[tid] = expf(sGC[tid]);

  // ---- phase 2: scale in place (each thread rewrites only the chunks it staged) --------------
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int r = rg * 4 + i;
    const uint32_t off = tile_chunk_off(r, cg, 8192);
    float kf[8], qf[8];
    unpack8(ld_shared_v4(sb + kS1Kg + off), kf);
    unpack8(ld_shared_v4(sb + kS1Qg + off), qf);
    if (fz.l2) {  // fused L2 norm: the 16 lanes holding this row reduce its sums of squares
      float ssk = 0.f, ssq = 0.f;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        ssk += kf[j] * kf[j];
        ssq += qf[j] * qf[j];
      }
#pragma unroll
      for (int off2 = 1; off2 < 16; off2 <<= 1) {
        ssk += __shfl_xor_sync(0xffffffffu, ssk, off2);
        ssq += __shfl_xor_sync(0xffffffffu, ssq, off2);
      }
      const float ik = rsqrtf(ssk + fz.eps), iq = rsqrtf(ssq + fz.eps);
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        kf[j] *= ik;
        qf[j] *= iq;
      }
      if (cg == 0) {  // for the exact fallback, which re-reads k and q from global memory
        sInv[r] = ik;
        sInv[64 + r] = iq;
      }
    }
    if (mode == kModeFast) {
      if constexpr (kGate) {
        if (shifted) {  // the factors around the reference m (the record's Q~ is rewritten below)
#pragma unroll
          for (int j = 0; j < 8; ++j) g[i][j] -= shift_ref(sGC[cg * 8 + j], decay_limit);
        }
      }
      float kg[8], ki[8], kt[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const float e = __expf(g[i][j]);
        kg[j] = kf[j] * e;
        qf[j] *= e;
        ki[j] = kf[j] * __expf(-g[i][j]);
        kt[j] = ki[j] * egc[j];
      }
      const uint4 qgv = pack8(qf);
      st_shared_v4(sb + kS1Kg + off, pack8(kg));
      st_shared_v4(sb + kS1Ki + off, pack8(ki));
      st_shared_v4(sb + kS1Qg + off, qgv);
      *reinterpret_cast<uint4*>(rec + kRecQW + qw_chunk_off(r, cg)) = qgv;
      *reinterpret_cast<uint4*>(rec + kRecKt + off) = pack8(kt);
    } else {
      const int R = rg >> 2;
      {
        float kt[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) kt[j] = kf[j] * __expf(sGC[cg * 8 + j] - g[i][j]);
        *reinterpret_cast<uint4*>(rec + kRecKt + off) = pack8(kt);
      }
      if (mode == kModeBlocks) {
        float qr[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const float er = R > 0 ? __expf(g[i][j] - sRef[(R - 1) * kD + cg * 8 + j]) : __expf(g[i][j]);
          kf[j] *= er;
          qr[j] = qf[j] * er;
        }
        st_shared_v4(sb + kS1Kg + off, pack8(kf));
        st_shared_v4(sb + kS1Qg + off, pack8(qr));
      }
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const float e = __expf(g[i][j]);
        if (mode != kModeBlocks) kf[j] *= e;
        qf[j] *= e;
      }
      if (mode != kModeBlocks) st_shared_v4(sb + kS1Kg + off, pack8(kf));
      *reinterpret_cast<uint4*>(rec + kRecQW + qw_chunk_off(r, cg)) = pack8(qf);
      float* gp = reinterpret_cast<float*>(rec + g_scratch_off(r));
      *reinterpret_cast<float4*>(gp + cg * 8) = make_float4(g[i][0], g[i][1], g[i][2], g[i][3]);
      *reinterpret_cast<float4*>(gp + cg * 8 + 4) = make_float4(g[i][4], g[i][5], g[i][6], g[i][7]);
    }
  }
  fence_proxy_async_smem();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  // ---- phase 3: A_kk = Kg Ki^T (cols 0..63), A_qk = Qg Ki^T (cols 64..127) -------------------
  bool alive = true;
  uint32_t nwait = 0;  // completed phases of `bar`
  if (mode == kModeFast) {
    if (tid == 0) {
      const uint32_t id = idesc_bf16_f32(64, 64, 0, 0);
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        const uint32_t koff = (kk >> 2) * 8192 + (kk & 3) * 32;
        const uint64_t bdesc = smem_desc_sw128(sb + kS1Ki + koff, 16, 1024);
        mma_bf16(tmem + 0, smem_desc_sw128(sb + kS1Kg + koff, 16, 1024), bdesc, id, kk > 0);
        mma_bf16(tmem + 64, smem_desc_sw128(sb + kS1Qg + koff, 16, 1024), bdesc, id, kk > 0);
      }
      mma_commit(bar);
    }
    alive = __syncthreads_and(mbar_wait(bar, 0)) != 0;
    nwait = 1;
    tc_fence_after();
    // K/Gamma and Gamma.Q are dead from here: A (fp32) takes the K/Gamma area
    const int sp = warp & 3, half = warp >> 2;
    const int r = sp * 16 + (lane & 15);
    float va[32];
#pragma unroll
    for (int part = 0; part < 2; ++part) {
      tmem_ld32(tmem_at(tmem, sp * 32, half * 64 + part * 32), va);
      tmem_ld_wait();
      if (lane < 16) {
        if (half == 0) {  // the inverse reads only the strictly lower triangle: no mask
          const float br = sBeta[r];
#pragma unroll
          for (int j4 = 0; j4 < 8; ++j4)
            sts4(sA, r, part * 8 + j4,
                 make_float4(br * va[4 * j4], br * va[4 * j4 + 1], br * va[4 * j4 + 2],
                             br * va[4 * j4 + 3]));
        } else {
#pragma unroll
          for (int c8 = 0; c8 < 4; ++c8) {
            float f[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) {
              const int i = part * 32 + c8 * 8 + j;
              f[j] = (i <= r) ? va[c8 * 8 + j] : 0.f;
            }
            *reinterpret_cast<uint4*>(rec + kRecAqk + tile_chunk_off(r, part * 4 + c8, 8192)) =
                pack8(f);
          }
        }
      }
    }
    if constexpr (kGate) {
      if (shifted) {  // the A products have read their tiles: rescale this thread's chunks by
        // e^m, Gamma.K in place for W and Gamma.Q into the record
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int r = rg * 4 + i;
          const uint32_t off = tile_chunk_off(r, cg, 8192);
          float kg[8], qg[8];
          unpack8(ld_shared_v4(sb + kS1Kg + off), kg);
          unpack8(ld_shared_v4(sb + kS1Qg + off), qg);
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const float em = __expf(shift_ref(sGC[cg * 8 + j], decay_limit));
            kg[j] *= em;
            qg[j] *= em;
          }
          st_shared_v4(sb + kS1Kg + off, pack8(kg));
          *reinterpret_cast<uint4*>(rec + kRecQW + qw_chunk_off(r, cg)) = pack8(qg);
        }
      }
    }
  } else if (mode == kModeBlocks) {
    // Three rounds; round `rho` serves row blocks {3}, {2, 0}, {1}. A piece (R, ts) puts the
    // column tile of row block R (rows i < 16R + 16, factor k_i exp(ref_R - g_i)) at rows
    // [ts, ts + 16R + 16) of the v area and its products at TMEM columns [ts, ...) (A_kk) and
    // [64 + ts, ...) (A_qk); only the 16 rows of block R (lanes 0..15 of TMEM sub-partition R)
    // are read back. The K/Gamma area receives A (fp32) row block by row block.
#pragma unroll 1
    for (int rho = 0; rho < 3 && alive; ++rho) {
#pragma unroll
      for (int ii = 0; ii < 4; ++ii) {
        const int t = rg * 4 + ii;
        const bool second = (rho == 1 && t >= 48);
        const int R = rho == 0 ? 3 : (rho == 1 ? (second ? 0 : 2) : 1);
        const int i = second ? t - 48 : t;
        if (i >= 16 * R + 16) continue;
        float kc[8];
        if (i < L KDA_AND_IN_BOUNDS(kBufK, k + ((size_t)(t0 + i) * H + h) * kD + cg * 8, 16)) {
          unpack8(*(reinterpret_cast<const uint4*>(k + ((size_t)(t0 + i) * H + h) * kD) + cg), kc);
          const float sc = fz.l2 ? sInv[i] : 1.f;
          const float* gi = reinterpret_cast<const float*>(rec + g_scratch_off(i)) + cg * 8;
          const float4 ga = *reinterpret_cast<const float4*>(gi);
          const float4 gb = *reinterpret_cast<const float4*>(gi + 4);
          const float gv[8] = {ga.x, ga.y, ga.z, ga.w, gb.x, gb.y, gb.z, gb.w};
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const float ref = R > 0 ? sRef[(R - 1) * kD + cg * 8 + j] : 0.f;
            kc[j] = kc[j] * sc * __expf(ref - gv[j]);
          }
        } else {
#pragma unroll
          for (int j = 0; j < 8; ++j) kc[j] = 0.f;
        }
        st_shared_v4(sb + kS1V + tile_chunk_off(t, cg, 8192), pack8(kc));
      }
      fence_proxy_async_smem();
      __syncthreads();
      tc_fence_after();
      const int npieces = rho == 1 ? 2 : 1;
      if (tid == 0) {
        for (int pc = 0; pc < npieces; ++pc) {
          const int R = rho == 0 ? 3 : (rho == 1 ? (pc == 0 ? 2 : 0) : 1);
          const int ts = pc == 1 ? 48 : 0;
          const uint32_t id = idesc_bf16_f32(64, 16 * R + 16, 0, 0);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint32_t koff = (kk >> 2) * 8192 + (kk & 3) * 32;
            const uint64_t bdesc = smem_desc_sw128(sb + kS1V + koff + ts * 128, 16, 1024);
            mma_bf16(tmem + ts, smem_desc_sw128(sb + kS1Kg + koff, 16, 1024), bdesc, id, kk > 0);
            mma_bf16(tmem + 64 + ts, smem_desc_sw128(sb + kS1Qg + koff, 16, 1024), bdesc, id,
                     kk > 0);
          }
        }
        mma_commit(bar);
      }
      alive = __syncthreads_and(mbar_wait(bar, nwait & 1)) != 0;
      ++nwait;
      tc_fence_after();
      {
        const int R = warp & 3, half = warp >> 2;
        const bool mine = rho == 0 ? R == 3 : (rho == 1 ? (R == 2 || R == 0) : R == 1);
        if (mine) {
          const int ts = (rho == 1 && R == 0) ? 48 : 0, N = 16 * R + 16;
          const int r = 16 * R + (lane & 15);
          const float br = sBeta[r];
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            float va[16];
            if (16 * u < N) {
              tmem_ld16(tmem_at(tmem, 32 * R, half * 64 + ts + 16 * u), va);
              tmem_ld_wait();
            } else {
#pragma unroll
              for (int j = 0; j < 16; ++j) va[j] = 0.f;
            }
            if (lane < 16) {
              if (half == 0) {  // only the strictly lower triangle is read: no mask
#pragma unroll
                for (int j4 = 0; j4 < 4; ++j4)
                  sts4(sA, r, 4 * u + j4,
                       make_float4(br * va[4 * j4], br * va[4 * j4 + 1], br * va[4 * j4 + 2],
                                   br * va[4 * j4 + 3]));
              } else {
#pragma unroll
                for (int c8 = 0; c8 < 2; ++c8) {
                  float f[8];
#pragma unroll
                  for (int j = 0; j < 8; ++j) {
                    const int i = 16 * u + 8 * c8 + j;
                    f[j] = (i <= r) ? va[8 * c8 + j] : 0.f;
                  }
                  *reinterpret_cast<uint4*>(rec + kRecAqk +
                                            tile_chunk_off(r, 2 * u + c8, 8192)) = pack8(f);
                }
              }
            }
          }
        }
      }
      tc_fence_before();
      __syncthreads();  // TMEM read and the v area free before the next round
    }
    // the row tiles and column tiles are dead: Gamma.K back into its area for W, v reloaded
#pragma unroll
    for (int ii = 0; ii < 4; ++ii) {
      const int r = rg * 4 + ii;
      const uint32_t off = tile_chunk_off(r, cg, 8192);
      if (r < L KDA_AND_IN_BOUNDS(kBufV, v + ((size_t)(t0 + r) * H + h) * kD + cg * 8, 16)
                KDA_AND_IN_BOUNDS(kBufK, k + ((size_t)(t0 + r) * H + h) * kD + cg * 8, 16)) {
        const size_t row = (size_t)(t0 + r) * H + h;
        cp_async16(sb + kS1V + off, reinterpret_cast<const uint4*>(v + row * kD) + cg);
        float kf[8];
        unpack8(*(reinterpret_cast<const uint4*>(k + row * kD) + cg), kf);
        const float sc = fz.l2 ? sInv[r] : 1.f;
        const float* gr = reinterpret_cast<const float*>(rec + g_scratch_off(r)) + cg * 8;
        const float4 ga = *reinterpret_cast<const float4*>(gr);
        const float4 gb = *reinterpret_cast<const float4*>(gr + 4);
        const float gv[8] = {ga.x, ga.y, ga.z, ga.w, gb.x, gb.y, gb.z, gb.w};
#pragma unroll
        for (int j = 0; j < 8; ++j) kf[j] = kf[j] * sc * __expf(gv[j]);
        st_shared_v4(sb + kS1Kg + off, pack8(kf));
      } else {
        const uint4 z = make_uint4(0, 0, 0, 0);
        st_shared_v4(sb + kS1V + off, z);
        st_shared_v4(sb + kS1Kg + off, z);
      }
    }
  } else {
    // exact fallback: one warp per (r, i) pair, ratios exp(g_r - g_i) <= 1, fp32
    for (int p = warp; p < kC * (kC + 1) / 2; p += kK1Threads / 32) {
      int r = (int)((sqrtf(8.f * p + 1.f) - 1.f) * 0.5f);
      while ((r + 1) * (r + 2) / 2 <= p) ++r;
      while (r * (r + 1) / 2 > p) --r;
      const int i = p - r * (r + 1) / 2;
      float akk = 0.f, aqk = 0.f;
      if (r < L KDA_AND_IN_BOUNDS(kBufK, k + ((size_t)(t0 + r) * H + h) * kD, 256)
                KDA_AND_IN_BOUNDS(kBufK, k + ((size_t)(t0 + i) * H + h) * kD, 256)
                KDA_AND_IN_BOUNDS(kBufQ, q + ((size_t)(t0 + r) * H + h) * kD, 256)) {
        const float* gr = reinterpret_cast<const float*>(rec + g_scratch_off(r));
        const float* gi = reinterpret_cast<const float*>(rec + g_scratch_off(i));
        const size_t rowr = (size_t)(t0 + r) * H + h, rowi = (size_t)(t0 + i) * H + h;
        for (int cc = lane; cc < kD; cc += 32) {
          const float f = __expf(gr[cc] - gi[cc]);
          const float kk = __bfloat162float(k[rowi * kD + cc]) * f;
          akk += __bfloat162float(k[rowr * kD + cc]) * kk;
          aqk += __bfloat162float(q[rowr * kD + cc]) * kk;
        }
      }
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) {
        akk += __shfl_xor_sync(0xffffffffu, akk, off);
        aqk += __shfl_xor_sync(0xffffffffu, aqk, off);
      }
      if (fz.l2) {
        akk *= sInv[r] * sInv[i];
        aqk *= sInv[64 + r] * sInv[i];
      }
      if (lane == 0) {
        sA[sidx(r, i)] = (i < r) ? sBeta[r] * akk : 0.f;
        reinterpret_cast<__nv_bfloat16*>(rec + kRecAqk + tile_off(r, i, 8192))[0] =
            __float2bfloat16_rn(aqk);
      }
    }
    for (int idx = tid; idx < kC * kC; idx += kK1Threads) {
      const int r = idx >> 6, i = idx & 63;
      if (i > r) {
        sA[sidx(r, i)] = 0.f;
        reinterpret_cast<__nv_bfloat16*>(rec + kRecAqk + tile_off(r, i, 8192))[0] =
            __float2bfloat16_rn(0.f);
      }
    }
  }
  tc_fence_before();
  __syncthreads();

  // ---- phase 4: T = (I + A)^{-1} in fp32 (16 x 16 blocks), T in the Gamma.Q area ------------
  // Only the lower triangle of T is ever read (the M build masks the rest), so T is not cleared.
  if (warp < 4 && lane < 16) {  // diagonal blocks by forward substitution: lane = column of T_bb
    const int b = warp, cidx = lane;
    float col[16];  // col[i] = T_bb[i][cidx]; entries above the diagonal come out as 0
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      float val = (i == cidx) ? 1.f : 0.f;
#pragma unroll
      for (int j4 = 0; j4 < 4; ++j4) {
        if (4 * j4 < i) {
          const float4 a = lds4(sA, 16 * b + i, 4 * b + j4);
          if (4 * j4 + 0 < i) val -= a.x * col[4 * j4 + 0];
          if (4 * j4 + 1 < i) val -= a.y * col[4 * j4 + 1];
          if (4 * j4 + 2 < i) val -= a.z * col[4 * j4 + 2];
          if (4 * j4 + 3 < i) val -= a.w * col[4 * j4 + 3];
        }
      }
      col[i] = val;
    }
#pragma unroll
    for (int i = 0; i < 16; ++i) sT[sidx(16 * b + i, 16 * b + cidx)] = col[i];
  }
  __syncthreads();
  // Off-diagonal blocks by the 2 x 2 block rule (I + A)^{-1} = [[T11, 0], [-T22 A21 T11, T22]]:
  //   32 x 32 halves first (t_{b+1,b} = -t_{b+1} a_{b+1,b} t_b for b = 0, 2), then the lower-left
  //   32 x 32 block T21 = -T22 (A21 T11). Threads own 1 x 4 strips; entries of T above the
  //   diagonal outside the diagonal blocks are never read.
  {
    // stage 2: X_b = a_{b+1,b} t_b for b = 0, 2 (two 16 x 16 products, 128 strips)
    const int b2 = (tid >> 6) & 1, rr = (tid >> 2) & 15, cq = tid & 3;
    const int bb = 2 * b2;  // b = 0 or 2
    if (tid < 128) {
      float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int k4 = 0; k4 < 4; ++k4) {
        if (k4 < cq) continue;  // t_b[k][c] = 0 for k < c
        const float4 a = lds4(sA, 16 * (bb + 1) + rr, 4 * bb + k4);
        const float4 t0 = lds4(sT, 16 * bb + 4 * k4 + 0, 4 * bb + cq);
        const float4 t1 = lds4(sT, 16 * bb + 4 * k4 + 1, 4 * bb + cq);
        const float4 t2 = lds4(sT, 16 * bb + 4 * k4 + 2, 4 * bb + cq);
        const float4 t3 = lds4(sT, 16 * bb + 4 * k4 + 3, 4 * bb + cq);
        acc.x += a.x * t0.x + a.y * t1.x + a.z * t2.x + a.w * t3.x;
        acc.y += a.x * t0.y + a.y * t1.y + a.z * t2.y + a.w * t3.y;
        acc.z += a.x * t0.z + a.y * t1.z + a.z * t2.z + a.w * t3.z;
        acc.w += a.x * t0.w + a.y * t1.w + a.z * t2.w + a.w * t3.w;
      }
      *reinterpret_cast<float4*>(sX + b2 * 256 + rr * 16 + 4 * cq) = acc;
    }
    __syncthreads();
    // t_{b+1,b} = -t_{b+1} X_b
    if (tid < 128) {
      float4 t = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int m4 = 0; m4 < 4; ++m4) {
        if (4 * m4 > rr) continue;  // t_{b+1}[rr][m] = 0 for m > rr
        const float4 a = lds4(sT, 16 * (bb + 1) + rr, 4 * (bb + 1) + m4);
        const float4* xr = reinterpret_cast<const float4*>(sX + b2 * 256 + (4 * m4) * 16 + 4 * cq);
        const float4 x0 = xr[0], x1 = xr[4], x2 = xr[8], x3 = xr[12];
        t.x += a.x * x0.x + a.y * x1.x + a.z * x2.x + a.w * x3.x;
        t.y += a.x * x0.y + a.y * x1.y + a.z * x2.y + a.w * x3.y;
        t.z += a.x * x0.z + a.y * x1.z + a.z * x2.z + a.w * x3.z;
        t.w += a.x * x0.w + a.y * x1.w + a.z * x2.w + a.w * x3.w;
      }
      sts4(sT, 16 * (bb + 1) + rr, 4 * bb + cq, make_float4(-t.x, -t.y, -t.z, -t.w));
    }
    __syncthreads();
    // stage 3: Y = A21 T11 (32 x 32, K over k >= c); warp = column group (so the triangular
    // extent of the sum is the same across the warp), lane = row
    {
      const int c3w = warp, r3w = lane;
      float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int k4 = 0; k4 < 8; ++k4) {
        if (k4 < c3w) continue;
        const float4 a = lds4(sA, 32 + r3w, k4);
        const float4 t0 = lds4(sT, 4 * k4 + 0, c3w), t1 = lds4(sT, 4 * k4 + 1, c3w);
        const float4 t2 = lds4(sT, 4 * k4 + 2, c3w), t3 = lds4(sT, 4 * k4 + 3, c3w);
        acc.x += a.x * t0.x + a.y * t1.x + a.z * t2.x + a.w * t3.x;
        acc.y += a.x * t0.y + a.y * t1.y + a.z * t2.y + a.w * t3.y;
        acc.z += a.x * t0.z + a.y * t1.z + a.z * t2.z + a.w * t3.z;
        acc.w += a.x * t0.w + a.y * t1.w + a.z * t2.w + a.w * t3.w;
      }
      *reinterpret_cast<float4*>(sX + yidx(r3w, c3w)) = acc;
    }
    __syncthreads();
    const int r3 = tid >> 3, c3 = tid & 7;
    // T21 = -T22 Y (K over k <= r)
    {
      float4 t = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int k4 = 0; k4 < 8; ++k4) {
        if (4 * k4 > r3) continue;
        const float4 a = lds4(sT, 32 + r3, 8 + k4);
        const float4 y0 = *reinterpret_cast<const float4*>(sX + yidx(4 * k4 + 0, c3));
        const float4 y1 = *reinterpret_cast<const float4*>(sX + yidx(4 * k4 + 1, c3));
        const float4 y2 = *reinterpret_cast<const float4*>(sX + yidx(4 * k4 + 2, c3));
        const float4 y3 = *reinterpret_cast<const float4*>(sX + yidx(4 * k4 + 3, c3));
        t.x += a.x * y0.x + a.y * y1.x + a.z * y2.x + a.w * y3.x;
        t.y += a.x * y0.y + a.y * y1.y + a.z * y2.y + a.w * y3.y;
        t.z += a.x * y0.z + a.y * y1.z + a.z * y2.z + a.w * y3.z;
        t.w += a.x * y0.w + a.y * y1.w + a.z * y2.w + a.w * y3.w;
      }
      sts4(sT, 32 + r3, c3, make_float4(-t.x, -t.y, -t.z, -t.w));
    }
    __syncthreads();
  }
  // M = T Diag(beta) -> bf16 operand tile (the level products are dead)
  for (int e = tid; e < kC * 8; e += kK1Threads) {
    const int r = e >> 3, c8 = e & 7;
    const float4 ta = lds4(sT, r, 2 * c8), tb = lds4(sT, r, 2 * c8 + 1);
    const float4 ba = *reinterpret_cast<const float4*>(sBeta + 8 * c8);
    const float4 bb = *reinterpret_cast<const float4*>(sBeta + 8 * c8 + 4);
    const int i0 = 8 * c8;
    float f[8] = {ta.x * ba.x, ta.y * ba.y, ta.z * ba.z, ta.w * ba.w,
                  tb.x * bb.x, tb.y * bb.y, tb.z * bb.z, tb.w * bb.w};
#pragma unroll
    for (int j = 0; j < 8; ++j) f[j] = (i0 + j <= r) ? f[j] : 0.f;
    st_shared_v4(sb + kS1M + tile_chunk_off(r, c8, 8192), pack8(f));
  }
  cp_async_wait_all();  // the reloaded v of the block mode
  fence_proxy_async_smem();
  __syncthreads();
  tc_fence_after();

  // ---- phase 5: W = M Kg, then U = M V, through TMEM [0, 128) -------------------------------
  // the state kernel launched after this one may start its set-up now; it waits for this grid's
  // completion before it reads any record
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  uint32_t phase = nwait & 1;
#pragma unroll 1
  for (int which = 0; which < 2 && alive; ++which) {
    if (tid == 0) {
      const uint32_t id = idesc_bf16_f32(64, 128, 0, 1);
      const uint32_t src = which == 0 ? kS1Kg : kS1V;
#pragma unroll
      for (int kk = 0; kk < 4; ++kk)
        mma_bf16(tmem, smem_desc_sw128(sb + kS1M + kk * 32, 16, 1024),
                 smem_desc_sw128(sb + src + kk * 2048, 8192, 1024), id, kk > 0);
      mma_commit(bar);
    }
    alive = __syncthreads_and(mbar_wait(bar, phase)) != 0;
    phase ^= 1;
    tc_fence_after();
    if (which == 0)
      readout_rows_bf16(tmem, warp, lane, rec + kRecQW, 64, 16384);  // W: rows 64..127 of QW
    else
      readout_rows_bf16(tmem, warp, lane, rec + kRecU, 0, 8192);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 7) {  // the allocating warp frees
    tc_fence_after();
    tmem_dealloc(tmem, kK1Tmem);
  }
}

// ============================================================================================
// K2
// ============================================================================================
constexpr int kEpiWarps = 8;                       // two per TMEM sub-partition, 32 columns each
constexpr int kK2Threads = 64 + 32 * kEpiWarps;    // warp 0 producer, warp 1 MMA, then epilogue
// stage: QW [128 x 128] | AZ [128 x 64] = A_qk rows 0..63, zero rows 64..127 | Kt [64 x 128] |
//        U (this CTA's 64-column block) [64 x 64] | gamma_C fp32 [128]
constexpr uint32_t kStQW = 0, kStAZ = 32768, kStKt = 49152, kStU = 65536, kStGam = 73728;
constexpr uint32_t kStageTx = 32768 + 8192 + 16384 + 8192 + 512;
constexpr int kStages = 2;
constexpr uint32_t kS2Stage0 = 0;
constexpr int kNumBars2 = 2 * kStages + 5;
constexpr int kOutWarps = 4;

// shared-memory map of K2; the output epilogue (head-wise RMSNorm x sigmoid gate) adds, because
// the two column halves of one (sequence, head) run as a cluster of two CTAs that exchange per-row
// sums of squares of their 64 columns, the exchange buffers
template <bool kNorm>
struct K2Smem {
  static constexpr uint32_t stage = 74752;         // 1024-aligned stages
  static constexpr uint32_t S = kStages * stage;   // [128 x 64] bf16 state tile (B operand)
  static constexpr uint32_t Vp = S + 16384;        // [64 x 64] bf16 pseudo-value tile
  static constexpr uint32_t Bar = Vp + 8192;
  static constexpr uint32_t Tmem = Bar + 8 * kNumBars2;
  static constexpr uint32_t Flags = Tmem + 4;
  static constexpr uint32_t Part = (Flags + 12 + 15) & ~15u;  // fp32 [2 parity][2 half][64 rows]
  static constexpr uint32_t Peer = Part + 1024;    // fp32 [2 parity][64]: the peer's row sums
  static constexpr uint32_t W = Peer + 512;        // fp32 [64] norm weight of this CTA's columns
  static constexpr uint32_t NBar = W + 256;        // mbarriers: part (local), norm[2] (peer)
  static constexpr uint32_t bytes = kNorm ? NBar + 24 : Flags + 12;
};
// TMEM columns: [Qt; W] S accumulators (double buffer) [0,64) / [64,128); Kt^T V' [128,192)
constexpr uint32_t kTmD12 = 0, kTmD3 = 128;

template <bool kNorm>
__global__ void __launch_bounds__(kK2Threads, 1)
    chunk_state_tc_kernel(const uint8_t* __restrict__ ws_records, SeqGeometry geo, int H,
                          const float* __restrict__ initial_state, float* __restrict__ final_state,
                          __nv_bfloat16* __restrict__ o, Fusion fz) {
  extern __shared__ uint8_t smem_raw[];
  if (!geo.ok()) return;
  using SM = K2Smem<kNorm>;
  constexpr uint32_t kStageBytes = SM::stage;
  constexpr uint32_t kS2S = SM::S, kS2Vp = SM::Vp;
  uint8_t* sm = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
  const uint32_t sb = smem_u32(sm);
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + SM::Bar);
  uint64_t* full = bars + 0;           // [kStages] record copied
  uint64_t* empty = bars + kStages;    // [kStages] record consumed by the tensor cores
  uint64_t* d12 = bars + 2 * kStages;  // [Qt; W] S done
  uint64_t* d3 = d12 + 1;              // Kt^T V' done (state update can proceed)
  uint64_t* d2done = d12 + 2;          // A_qk V' accumulated (output can be read)
  uint64_t* vp_ready = d12 + 3;        // V' tile written (one arrival per epilogue warp)
  uint64_t* s_ready = d12 + 4;         // state tile written (one arrival per epilogue warp)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + SM::Tmem);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + SM::Flags);

  // one CTA per (sequence, head, 64-column half), linear in that order with the sequence slowest:
  // the longest sequences' chains are dispatched first
  const int n = geo.seq_at_rank((int)(blockIdx.x / (2u * (unsigned)H)));
  const int h = (int)((blockIdx.x >> 1) % (unsigned)H), j0 = (int)(blockIdx.x & 1u) * 64;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int tb = geo.seq_begin(n), te = geo.seq_end(n);
  const int nchunks = te > tb ? ceil_div(te - tb, kC) : 0;
  const int c_first = geo.first_chunk(n);

  if (warp == 0) {
    tmem_alloc(tmem_slot, 256);
    tmem_relinquish();
    tc_fence_before();
  }
  if (tid == 0) {
    for (int i = 0; i < 2 * kStages; ++i) mbar_init(bars + i, 1);
    mbar_init(d12, 1);
    mbar_init(d3, 1);
    mbar_init(d2done, 1);
    mbar_init(vp_ready, kEpiWarps);
    mbar_init(s_ready, kEpiWarps);
    *abort_flag = 0;
    if (kNorm) {
      uint64_t* nb = reinterpret_cast<uint64_t*>(sm + SM::NBar);
      mbar_init(nb, kOutWarps);  // this CTA's out warps wrote their partial sums
      mbar_init(nb + 1, 1);      // the peer's 64 row sums landed (256 transaction bytes), even
      mbar_init(nb + 2, 1);      // chunk index / odd; the one arrival is this CTA's expect_tx
    }
    fence_mbar_init();
  }
  if (kNorm && tid < 64)
    reinterpret_cast<float*>(sm + SM::W)[tid] =
        (fz.ow && KDA_IN_BOUNDS(kBufNormW, fz.ow + j0 + tid, 4)) ? fz.ow[j0 + tid] : 1.f;
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  if (kNorm) cluster_sync();  // the peer's barriers are initialised before any remote arrival

  if (warp == 0) {
    // ------------------------------------------------------------------ producer
    // launched as a programmatic dependent of the chunk-local kernel: the records are complete
    // and visible only after this wait (the set-up above overlapped that kernel's tail)
    if (lane == 0) asm volatile("griddepcontrol.wait;" ::: "memory");
    if (lane == 0) {
      for (int ci = 0; ci < nchunks; ++ci) {
        const int st = ci % kStages;
        if (!((ci < kStages || mbar_wait(empty + st, ((ci / kStages) - 1) & 1)) &&
              !*abort_flag)) {
          *abort_flag = 1;
          break;
        }
        uint8_t* stage = sm + kS2Stage0 + st * kStageBytes;
        const uint8_t* rec = ws_records + (size_t)kRecBytes * ((size_t)(c_first + ci) * H + h);
        if (!KDA_IN_BOUNDS(kBufWork, rec, kRecBytes)) {
          mbar_arrive(full + st);  // nothing copied: the phase completes on the stale stage
        } else {
          mbar_arrive_expect_tx(full + st, kStageTx);
          bulk_g2s(stage + kStQW, rec + kRecQW, 32768, full + st);
          bulk_g2s(stage + kStAZ, rec + kRecAqk, 8192, full + st);
          bulk_g2s(stage + kStKt, rec + kRecKt, 16384, full + st);
          bulk_g2s(stage + kStU, rec + kRecU + (j0 >> 6) * 8192, 8192, full + st);
          bulk_g2s(stage + kStGam, rec + kRecGam, 512, full + st);
        }
      }
      // the last copies must land before the CTA may exit
      for (int ci = nchunks > kStages ? nchunks - kStages : 0; ci < nchunks; ++ci)
        mbar_wait(full + ci % kStages, (ci / kStages) & 1);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t id_qw = idesc_bf16_f32(128, 64, 0, 1);  // K-major A, MN-major B
      const uint32_t id_kt = idesc_bf16_f32(128, 64, 1, 1);  // MN-major A and B
      // descriptors are built once; the start-address field (bits 0..13, >> 4) is advanced by
      // plain addition, which never carries out of the field inside shared memory
      const uint64_t dqw = smem_desc_sw128(sb + kS2Stage0 + kStQW, 16, 1024);
      const uint64_t daz = smem_desc_sw128(sb + kS2Stage0 + kStAZ, 16, 1024);
      const uint64_t dkt = smem_desc_sw128(sb + kS2Stage0 + kStKt, 8192, 1024);
      const uint64_t ds = smem_desc_sw128(sb + kS2S, 8192, 1024);
      const uint64_t dvp = smem_desc_sw128(sb + kS2Vp, 8192, 1024);
      for (int ci = 0; ci < nchunks; ++ci) {
        const int st = ci % kStages;
        if (!mbar_wait(full + st, (ci / kStages) & 1) || !mbar_wait(s_ready, ci & 1)) {
          *abort_flag = 1;
          break;
        }
        tc_fence_after();
        const uint32_t d12t = tmem + kTmD12 + (ci & 1) * 64;
        const uint64_t soff = (uint64_t)((st * kStageBytes) >> 4);
        const uint64_t aqw = dqw + soff, aaz = daz + soff, akt = dkt + soff;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)  // [Qt; W] S
          mma_bf16(d12t, aqw + (uint64_t)((((kk >> 2) * 16384) + (kk & 3) * 32) >> 4),
                   ds + (uint64_t)((kk * 2048) >> 4), id_qw, kk > 0);
        mma_commit(d12);
        if (!mbar_wait(vp_ready, ci & 1)) {
          *abort_flag = 1;
          break;
        }
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)  // Kt^T V'
          mma_bf16(tmem + kTmD3, akt + (uint64_t)((kk * 2048) >> 4),
                   dvp + (uint64_t)((kk * 2048) >> 4), id_kt, kk > 0);
        mma_commit(d3);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)  // [A_qk; 0] V' accumulated onto the output rows
          mma_bf16(d12t, aaz + (uint64_t)((kk * 32) >> 4), dvp + (uint64_t)((kk * 2048) >> 4),
                   id_qw, true);
        mma_commit(d2done);
        mma_commit(empty + st);
      }
    }
  } else {
    // ------------------------------------------------------------------ epilogue (8 warps)
    // thread = TMEM lane = row, warp pair = column half: rows 0..63 of D12 are the chunk output
    // O, rows 64..127 are W S; every row is a row of the state slice for D3.
    const int ew = warp - 2;
    const int sp = warp & 3;
    const int chalf = ew >> 2;       // columns [32 chalf, 32 chalf + 32) of the 64-column slice
    const int row = sp * 32 + lane;
    const bool out_warp = sp < 2;    // reads O (rows 0..63); the others compute V'
    const int r = row & 63;
    // the zero rows of every stage's [A_qk; 0] operand
    for (int st = 0; st < kStages; ++st)
      for (int i = tid - 64; i < 512; i += 32 * kEpiWarps)
        st_shared_v4(sb + kS2Stage0 + st * kStageBytes + kStAZ + 8192 + i * 16,
                     make_uint4(0, 0, 0, 0));
    float S[32];
    const size_t sbase = (((size_t)n * H + h) * kD + row) * kD + j0 + 32 * chalf;
    if (initial_state && KDA_IN_BOUNDS(kBufInitial, initial_state + sbase, 128)) {
      const float4* src = reinterpret_cast<const float4*>(initial_state + sbase);
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const float4 x = src[j];
        S[4 * j] = x.x; S[4 * j + 1] = x.y; S[4 * j + 2] = x.z; S[4 * j + 3] = x.w;
      }
    } else {
#pragma unroll
      for (int j = 0; j < 32; ++j) S[j] = 0.f;
    }
    auto write_state_tile = [&]() {
#pragma unroll
      for (int q8 = 0; q8 < 4; ++q8) {
        float f[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) f[j] = S[q8 * 8 + j];
        st_shared_v4(sb + kS2S + tile_chunk_off(row, 4 * chalf + q8, 16384), pack8(f));
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(s_ready);
    };
    write_state_tile();

    // the output-gate row of this thread's chunk row (its 32 columns, 64 bytes), loaded from
    // global memory a chunk ahead of its use
    uint4 graw[4] = {};
    const __nv_bfloat16* g0 = reinterpret_cast<const __nv_bfloat16*>(fz.og);
    auto load_gate = [&](int ci) {
      if (kNorm && out_warp && g0 && ci < nchunks && tb + ci * kC + r < te) {
        const __nv_bfloat16* gp = g0 + ((size_t)(tb + ci * kC + r) * H + h) * kD + j0 + 32 * chalf;
        if (KDA_IN_BOUNDS(kBufGate, gp, 64)) {
#pragma unroll
          for (int q8 = 0; q8 < 4; ++q8) graw[q8] = __ldg(reinterpret_cast<const uint4*>(gp) + q8);
        }
      }
    };
    load_gate(0);
    float va[32];
    for (int ci = 0; ci < nchunks; ++ci) {
      const int st = ci % kStages;
      const uint32_t stage = sb + kS2Stage0 + st * kStageBytes;
      const int t0 = tb + ci * kC;
      const int L = min(kC, te - t0);
      const uint32_t d12c = kTmD12 + (ci & 1) * 64 + 32 * chalf;
      bool ok = !*abort_flag && mbar_wait(full + st, (ci / kStages) & 1);
      if (!__all_sync(0xffffffffu, ok)) {  // warp-uniform exit: tcgen05.ld is warp-collective
        *abort_flag = 1;
        break;
      }
      const float gam = reinterpret_cast<const float*>(sm + st * kStageBytes + kStGam)[row];
      if (!out_warp) {  // V' = U - W S for chunk row r, this warp's 32 columns
        float u[32];
#pragma unroll
        for (int q8 = 0; q8 < 4; ++q8) {
          float f[8];
          unpack8(ld_shared_v4(stage + kStU + tile_chunk_off(r, 4 * chalf + q8, 8192)), f);
#pragma unroll
          for (int j = 0; j < 8; ++j) u[q8 * 8 + j] = f[j];
        }
        ok = mbar_wait(d12, ci & 1);
        if (!__all_sync(0xffffffffu, ok)) {
          *abort_flag = 1;
          break;
        }
        tc_fence_after();
        tmem_ld32(tmem_at(tmem, sp * 32, d12c), va);
        tmem_ld_wait();
#pragma unroll
        for (int q8 = 0; q8 < 4; ++q8) {
          float f[8];
#pragma unroll
          for (int j = 0; j < 8; ++j) f[j] = u[q8 * 8 + j] - va[q8 * 8 + j];
          st_shared_v4(sb + kS2Vp + tile_chunk_off(r, 4 * chalf + q8, 8192), pack8(f));
        }
        fence_proxy_async_smem();
        tc_fence_before();
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(vp_ready);
      // S = Diag(gamma_C) S + Kt^T V'
      ok = mbar_wait(d3, ci & 1);
      if (!__all_sync(0xffffffffu, ok)) {
        *abort_flag = 1;
        break;
      }
      tc_fence_after();
      tmem_ld32(tmem_at(tmem, sp * 32, kTmD3 + 32 * chalf), va);
      tmem_ld_wait();
#pragma unroll
      for (int j = 0; j < 32; ++j) S[j] = fmaf(gam, S[j], va[j]);
      write_state_tile();
      if (out_warp) {  // O = Qt S + A_qk V' (Eq. 9), off the state chain
        ok = mbar_wait(d2done, ci & 1);
        if (!__all_sync(0xffffffffu, ok)) {
          *abort_flag = 1;
          break;
        }
        tc_fence_after();
        tmem_ld32(tmem_at(tmem, sp * 32, d12c), va);
        tmem_ld_wait();
        if (kNorm) {  // y = sigmoid(gate) * weight * O / RMS over all 128 columns of the row
          const int b = ci & 1;
          float* sPart = reinterpret_cast<float*>(sm + SM::Part) + b * 128;
          const float* sPeer = reinterpret_cast<const float*>(sm + SM::Peer) + b * 64;
          uint64_t* nb = reinterpret_cast<uint64_t*>(sm + SM::NBar);
          const bool gated = fz.og && r < L;
          float ss = 0.f;
#pragma unroll
          for (int j = 0; j < 32; ++j) ss = fmaf(va[j], va[j], ss);
          sPart[chalf * 64 + r] = ss;
          __syncwarp();
          if (lane == 0) mbar_arrive(nb);
          ok = mbar_wait(nb, ci & 1);
          if (ok && chalf == 0) {  // send this CTA's 64-column sum of the row to the peer
            const uint32_t peer = cluster_ctarank() ^ 1u;
            if (sp == 0 && lane == 0) mbar_arrive_expect_tx(nb + 1 + b, 64 * 4);
            st_async_remote_f32(mapa_shared(smem_u32(sPeer + r), peer), ss + sPart[64 + r],
                                mapa_shared(smem_u32(nb + 1 + b), peer));
          }
          ok = ok && mbar_wait(nb + 1 + b, (ci >> 1) & 1);
          if (!__all_sync(0xffffffffu, ok)) {
            *abort_flag = 1;
            break;
          }
          const float inv =
              rsqrtf((sPart[r] + sPart[64 + r] + sPeer[r]) * (1.f / kD) + fz.oeps);
          const float* sW = reinterpret_cast<const float*>(sm + SM::W) + 32 * chalf;
          float gt[32];
          if (gated) {  // the gate row loaded a chunk ahead: 32 columns of row r
#pragma unroll
            for (int q8 = 0; q8 < 4; ++q8) {
              float f[8];
              unpack8(graw[q8], f);
#pragma unroll
              for (int j = 0; j < 8; ++j)  // sigmoid(x) = (1 + tanh(x / 2)) / 2: one MUFU op
                gt[q8 * 8 + j] = fmaf(0.5f, tanh_approx(0.5f * f[j]), 0.5f);
            }
          } else {
#pragma unroll
            for (int j = 0; j < 32; ++j) gt[j] = 1.f;
          }
          load_gate(ci + 1);
#pragma unroll
          for (int j = 0; j < 32; ++j) va[j] = va[j] * inv * sW[j] * gt[j];
        }
        if (r < L && KDA_IN_BOUNDS(kBufO, o + ((size_t)(t0 + r) * H + h) * kD + j0 + 32 * chalf,
                                   64)) {
          uint4* dst = reinterpret_cast<uint4*>(o + ((size_t)(t0 + r) * H + h) * kD + j0 +
                                                32 * chalf);
#pragma unroll
          for (int q8 = 0; q8 < 4; ++q8) {
            float f[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) f[j] = va[q8 * 8 + j];
            dst[q8] = pack8(f);
          }
        }
      }
    }
    if (final_state && !*abort_flag && KDA_IN_BOUNDS(kBufFinal, final_state + sbase, 128)) {
      float4* dst = reinterpret_cast<float4*>(final_state + sbase);
#pragma unroll
      for (int j = 0; j < 8; ++j)
        dst[j] = make_float4(S[4 * j], S[4 * j + 1], S[4 * j + 2], S[4 * j + 3]);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
  if (kNorm) cluster_sync();  // no CTA leaves while its peer may still write into it
}

}  // namespace tc

size_t tc_local_smem_bytes() { return tc::kS1Bytes + 1024; }
size_t tc_state_smem_bytes() { return tc::K2Smem<false>::bytes + 1024; }

cudaError_t launch_prefill_tc(const PrefillArgs& a, const SeqGeometry& geo, int max_chunks,
                              uint8_t* records, cudaStream_t stream) {
  const bool norm = a.fz.onorm != 0;
  const int sm1 = (int)tc_local_smem_bytes();
  const int sm2 = (int)(norm ? tc::K2Smem<true>::bytes + 1024 : tc_state_smem_bytes());
  auto* k1 = a.fz.A_log ? tc::chunk_local_tc_kernel<true> : tc::chunk_local_tc_kernel<false>;
  cudaError_t err = cudaFuncSetAttribute(k1, cudaFuncAttributeMaxDynamicSharedMemorySize, sm1);
  if (err != cudaSuccess) return err;
  err = cudaFuncSetAttribute(norm ? tc::chunk_state_tc_kernel<true>
                                  : tc::chunk_state_tc_kernel<false>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, sm2);
  if (err != cudaSuccess) return err;
  if (max_chunks > 0) {
    ProfileScope prof("chunk_local_tc", stream);
    k1<<<dim3(max_chunks, a.H), tc::kK1Threads, sm1, stream>>>(
        (const __nv_bfloat16*)a.q, (const __nv_bfloat16*)a.k, (const __nv_bfloat16*)a.v,
        a.log_alpha, a.beta, geo, a.H, records, a.fz);
    err = cudaGetLastError();
    if (err != cudaSuccess) return err;
  }
  if (2LL * a.N * a.H > INT32_MAX) return cudaErrorInvalidConfiguration;
  // programmatic dependent launch: the state kernel's set-up (tensor memory, barriers, initial
  // state) overlaps the chunk-local kernel's last wave; its producer waits for the records
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2u * (unsigned)a.N * (unsigned)a.H);
  cfg.blockDim = dim3(tc::kK2Threads);
  cfg.dynamicSmemBytes = (size_t)sm2;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (!norm) {
    ProfileScope prof("chunk_state_tc", stream);
    return cudaLaunchKernelEx(&cfg, tc::chunk_state_tc_kernel<false>, (const uint8_t*)records, geo,
                              (int)a.H, a.initial_state, a.final_state, (__nv_bfloat16*)a.o, a.fz);
  }
  // the two column halves of a (sequence, head) form one cluster
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = 2;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.numAttrs = 2;
  ProfileScope prof("chunk_state_tc_norm", stream);
  return cudaLaunchKernelEx(&cfg, tc::chunk_state_tc_kernel<true>, (const uint8_t*)records, geo,
                            (int)a.H, a.initial_state, a.final_state, (__nv_bfloat16*)a.o, a.fz);
}

}  // namespace kda
