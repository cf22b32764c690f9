// kda_api.cu — the C ABI of the KDA library: argument validation, workspace layout, dispatch.
// Every argument error is caught here, on the host, before anything is launched.
#include <stdint.h>
#include <string.h>

#include "kda_common.cuh"
#include "kda_internal.h"

namespace kda {

namespace {

inline bool aligned(const void* p, size_t a) { return ((uintptr_t)p % a) == 0; }

// Workspace layout of one prefill call:
//   [0, 256)                 header: int32 `valid` flag written by the chunk-map kernel
//   [256, 256 + off_bytes)   int32 chunk_off[N+1], then int32 order[N] (the sequences longest
//                            first), for packed varlen batches only
//   [rec_base, ...)          per (chunk, head) records of the kernel path
struct WsLayout {
  size_t chunk_off_base;
  size_t rec_base;
  size_t rec_bytes;  // bytes of one record
  long long max_chunks;
  size_t total;
};

bool is_tc_path(kda_dtype_t dt) { return dt == KDA_DTYPE_BF16; }

// Upper bound on the chunks of one call: every sequence may end in a partial chunk.
long long max_chunks_of(int32_t B, int32_t T, int32_t C, int32_t N, bool varlen) {
  const long long tokens = (long long)B * T;
  return varlen ? (tokens + C - 1) / C + N : (long long)B * ((T + C - 1) / C);
}

// Launch-grid limits of the chunk kernels: the head index is a grid y extent (<= 65535) in the
// chunk-state kernels, and chunk x head items and 2 x sequence x head chains are counted in int.
// Bounding the items also keeps every workspace size far inside size_t.
bool grid_limits_ok(int32_t B, int32_t T, int32_t H, int32_t C, int32_t N, bool varlen) {
  if (H > 65535) return false;
  return max_chunks_of(B, T, C, N, varlen) * H <= INT32_MAX && 2LL * N * H <= INT32_MAX;
}

kda_status_t check_prefill_shape(int32_t B, int32_t T, int32_t H, int32_t Dk, int32_t Dv,
                                 int32_t C, int32_t N, kda_dtype_t dt, bool varlen) {
  if (B < 0 || T < 0 || H <= 0 || Dk <= 0 || Dv <= 0 || N < 0 || C <= 0)
    return KDA_ERR_INVALID_ARG;
  if (dt != KDA_DTYPE_F32 && dt != KDA_DTYPE_BF16) return KDA_ERR_INVALID_ARG;
  if (varlen) {
    if (B != 1 && !(B == 0 && T == 0)) return KDA_ERR_INVALID_ARG;
  } else if (N != B) {
    return KDA_ERR_INVALID_ARG;
  }
  if (dt == KDA_DTYPE_BF16) {
    if (Dk != 128 || Dv != 128 || C != 64) return KDA_ERR_UNSUPPORTED;
  } else {
    if (Dk > 128 || Dv > 128) return KDA_ERR_UNSUPPORTED;
    if (C != 16 && C != 32 && C != 64) return KDA_ERR_UNSUPPORTED;
  }
  const long long tokens = (long long)B * T;
  const long long elems = tokens * H * (long long)(Dk > Dv ? Dk : Dv);
  if (tokens > INT32_MAX || elems > (1LL << 40)) return KDA_ERR_UNSUPPORTED;
  if (!grid_limits_ok(B, T, H, C, N, varlen)) return KDA_ERR_UNSUPPORTED;
  return KDA_OK;
}

WsLayout prefill_layout(int32_t B, int32_t T, int32_t H, int32_t Dk, int32_t Dv, int32_t C,
                        int32_t N, bool varlen, kda_dtype_t dt) {
  WsLayout w;
  w.max_chunks = max_chunks_of(B, T, C, N, varlen);
  w.chunk_off_base = 256;
  const size_t off_bytes = varlen ? align_up(sizeof(int32_t) * (2 * (size_t)N + 1), 256) : 0;
  w.rec_base = w.chunk_off_base + off_bytes;
  w.rec_bytes = is_tc_path(dt) ? TcRecordBytes
                               : SimtRecord::make(C, Dk, Dv).record_floats * sizeof(float);
  w.total = w.rec_base + (size_t)w.max_chunks * H * w.rec_bytes;
  return w;
}

kda_status_t from_cuda(cudaError_t e) { return e == cudaSuccess ? KDA_OK : KDA_ERR_CUDA; }

// one entry of a call's bounds table (bytes = 0 leaves the role empty: any access is reported)
inline void set_extent(BoundsTable& t, BufRole role, const void* base, size_t bytes) {
  t.base[role] = bytes ? base : nullptr;
  t.bytes[role] = bytes;
}

// the extents of the fusion descriptor's buffers
void fusion_extents(BoundsTable& t, const Fusion& fz, size_t gate_bytes, int32_t H, int32_t Dk,
                    int32_t Dv) {
  set_extent(t, kBufALog, fz.A_log, fz.A_log ? (size_t)H * 4 : 0);
  set_extent(t, kBufDtBias, fz.dt_bias, fz.dt_bias ? (size_t)H * Dk * 4 : 0);
  set_extent(t, kBufGate, fz.og, fz.og ? gate_bytes : 0);
  set_extent(t, kBufNormW, fz.ow, fz.ow ? (size_t)Dv * 4 : 0);
}

// Backward pass: chunk of 32 tokens, fp32 arithmetic for both input dtypes.
constexpr int32_t kBwdChunk = 32;

kda_status_t check_backward_shape(int32_t B, int32_t T, int32_t H, int32_t Dk, int32_t Dv,
                                  int32_t N, kda_dtype_t dt, bool varlen) {
  if (B < 0 || T < 0 || H <= 0 || Dk <= 0 || Dv <= 0 || N < 0) return KDA_ERR_INVALID_ARG;
  if (dt != KDA_DTYPE_F32 && dt != KDA_DTYPE_BF16) return KDA_ERR_INVALID_ARG;
  if (varlen) {
    if (B != 1 && !(B == 0 && T == 0)) return KDA_ERR_INVALID_ARG;
  } else if (N != B) {
    return KDA_ERR_INVALID_ARG;
  }
  if (Dk > 128 || Dv > 128 || Dk % 4 != 0 || Dv % 4 != 0) return KDA_ERR_UNSUPPORTED;
  const long long tokens = (long long)B * T;
  const long long elems = tokens * H * (long long)(Dk > Dv ? Dk : Dv);
  if (tokens > INT32_MAX || elems > (1LL << 40)) return KDA_ERR_UNSUPPORTED;
  if (!grid_limits_ok(B, T, H, kBwdChunk, N, varlen)) return KDA_ERR_UNSUPPORTED;
  return KDA_OK;
}

// Workspace layout of one backward call:
//   header | chunk_off | fp32 records (with T and B) | states entering every chunk |
//   cotangents of the states leaving every chunk | dV' [B*T, H, Dv]
struct BwdLayout {
  size_t chunk_off_base, rec_base, states_base, dstates_base, dvp_base, total;
  long long max_chunks;
};

BwdLayout backward_layout(int32_t B, int32_t T, int32_t H, int32_t Dk, int32_t Dv, int32_t N,
                          bool varlen) {
  BwdLayout w;
  const long long tokens = (long long)B * T;
  w.max_chunks = max_chunks_of(B, T, kBwdChunk, N, varlen);
  w.chunk_off_base = 256;
  const size_t off_bytes = varlen ? align_up(sizeof(int32_t) * ((size_t)N + 1), 256) : 0;
  w.rec_base = w.chunk_off_base + off_bytes;
  const size_t rec_bytes = SimtRecord::make(kBwdChunk, Dk, Dv, true).record_floats * sizeof(float);
  const size_t state_bytes = (size_t)Dk * Dv * sizeof(float);
  w.states_base = w.rec_base + (size_t)w.max_chunks * H * rec_bytes;
  w.dstates_base = align_up(w.states_base + (size_t)w.max_chunks * H * state_bytes, 256);
  w.dvp_base = align_up(w.dstates_base + (size_t)w.max_chunks * H * state_bytes, 256);
  w.total = align_up(w.dvp_base + (size_t)tokens * H * Dv * sizeof(float), 256);
  return w;
}

}  // namespace

cudaError_t register_bounds(const BoundsTable& t, cudaStream_t stream) {
#ifdef KDA_BOUNDS_CHECK
  set_bounds_kernel<<<1, 1, 0, stream>>>(t);
  return cudaGetLastError();
#else
  (void)t;
  (void)stream;
  return cudaSuccess;
#endif
}

}  // namespace kda

using namespace kda;

extern "C" {

const char* kda_status_string(kda_status_t s) {
  switch (s) {
    case KDA_OK: return "KDA_OK";
    case KDA_ERR_INVALID_ARG: return "KDA_ERR_INVALID_ARG: invalid argument";
    case KDA_ERR_UNSUPPORTED: return "KDA_ERR_UNSUPPORTED: unsupported size or dtype";
    case KDA_ERR_CUDA: return "KDA_ERR_CUDA: CUDA runtime error";
    case KDA_ERR_TIMEOUT: return "KDA_ERR_TIMEOUT: a bounded device wait gave up";
    case KDA_ERR_WORKSPACE: return "KDA_ERR_WORKSPACE: workspace missing, small or misaligned";
  }
  return "KDA_ERR_UNKNOWN";
}

const char* kda_version(void) { return "0.2.0"; }

kda_status_t kda_chunk_fwd_workspace_size(int32_t B, int32_t T, int32_t H, int32_t Dk, int32_t Dv,
                                          int32_t chunk, int32_t num_seqs, kda_dtype_t dt,
                                          size_t* bytes) {
  if (!bytes) return KDA_ERR_INVALID_ARG;
  // the size query cannot know whether cu_seqlens will be passed: size for the larger (varlen)
  // layout whenever B == 1, which also covers the fixed-length layout
  const bool varlen = (B == 1);
  kda_status_t st = check_prefill_shape(B, T, H, Dk, Dv, chunk, varlen ? num_seqs : B, dt, varlen);
  if (st != KDA_OK) return st;
  *bytes = prefill_layout(B, T, H, Dk, Dv, chunk, varlen ? num_seqs : B, varlen, dt).total;
  return KDA_OK;
}

kda_status_t kda_chunk_bwd_workspace_size(int32_t B, int32_t T, int32_t H, int32_t Dk, int32_t Dv,
                                          int32_t num_seqs, kda_dtype_t dt, size_t* bytes) {
  if (!bytes) return KDA_ERR_INVALID_ARG;
  const bool varlen = (B == 1);
  kda_status_t st = check_backward_shape(B, T, H, Dk, Dv, varlen ? num_seqs : B, dt, varlen);
  if (st != KDA_OK) return st;
  *bytes = backward_layout(B, T, H, Dk, Dv, varlen ? num_seqs : B, varlen).total;
  return KDA_OK;
}

kda_status_t kda_chunk_bwd(const void* q, const void* k, const void* v, kda_dtype_t dt,
                           const float* log_alpha, const float* beta, const float* initial_state,
                           const int32_t* cu_seqlens, int32_t N, int32_t B, int32_t T, int32_t H,
                           int32_t Dk, int32_t Dv, const void* d_o, const float* d_final_state,
                           void* dq, void* dk, void* dv, float* dlog_alpha, float* dbeta,
                           float* d_initial_state, void* workspace, size_t workspace_bytes,
                           kda_stream_t stream_) {
  const bool varlen = cu_seqlens != nullptr;
  kda_status_t st = check_backward_shape(B, T, H, Dk, Dv, N, dt, varlen);
  if (st != KDA_OK) return st;
  const long long tokens = (long long)B * T;
  const size_t es = dt == KDA_DTYPE_BF16 ? 2 : 4;
  if (tokens > 0) {
    if (!q || !k || !v || !log_alpha || !beta || !d_o || !dq || !dk || !dv || !dlog_alpha ||
        !dbeta)
      return KDA_ERR_INVALID_ARG;
    if (!aligned(q, es) || !aligned(k, es) || !aligned(v, es) || !aligned(d_o, es) ||
        !aligned(dq, es) || !aligned(dk, es) || !aligned(dv, es) || !aligned(log_alpha, 4) ||
        !aligned(beta, 4) || !aligned(dlog_alpha, 4) || !aligned(dbeta, 4))
      return KDA_ERR_INVALID_ARG;
  }
  if ((initial_state && !aligned(initial_state, 4)) ||
      (d_final_state && !aligned(d_final_state, 4)) ||
      (d_initial_state && !aligned(d_initial_state, 4)) || (varlen && !aligned(cu_seqlens, 4)))
    return KDA_ERR_INVALID_ARG;
  if (N == 0) return KDA_OK;
  const BwdLayout lay = backward_layout(B, T, H, Dk, Dv, N, varlen);
  if (!workspace || !aligned(workspace, 256) || workspace_bytes < lay.total)
    return KDA_ERR_WORKSPACE;

  cudaStream_t stream = (cudaStream_t)stream_;
  if (kBoundsChecked) {
    BoundsTable t = {};
    const size_t th = (size_t)tokens * H, states = (size_t)N * H * Dk * Dv * 4;
    set_extent(t, kBufQ, q, th * Dk * es);
    set_extent(t, kBufK, k, th * Dk * es);
    set_extent(t, kBufV, v, th * Dv * es);
    set_extent(t, kBufLogAlpha, log_alpha, th * Dk * 4);
    set_extent(t, kBufBeta, beta, th * 4);
    set_extent(t, kBufInitial, initial_state, initial_state ? states : 0);
    set_extent(t, kBufDO, d_o, th * Dv * es);
    set_extent(t, kBufDFinal, d_final_state, d_final_state ? states : 0);
    set_extent(t, kBufDQ, dq, th * Dk * es);
    set_extent(t, kBufDK, dk, th * Dk * es);
    set_extent(t, kBufDV, dv, th * Dv * es);
    set_extent(t, kBufDLogAlpha, dlog_alpha, th * Dk * 4);
    set_extent(t, kBufDBeta, dbeta, th * 4);
    set_extent(t, kBufDInitial, d_initial_state, d_initial_state ? states : 0);
    set_extent(t, kBufWork, workspace, workspace_bytes);
    set_extent(t, kBufCuSeqlens, cu_seqlens, varlen ? ((size_t)N + 1) * 4 : 0);
    st = from_cuda(register_bounds(t, stream));
    if (st != KDA_OK) return st;
  }
  char* ws = (char*)workspace;
  int32_t* valid = (int32_t*)ws;
  int32_t* chunk_off = (int32_t*)(ws + lay.chunk_off_base);
  if (varlen) {
    st = from_cuda(
        launch_chunk_map(cu_seqlens, N, (int)tokens, kBwdChunk, chunk_off, valid, nullptr,
                         stream));
    if (st != KDA_OK) return st;
  }
  SeqGeometry geo;
  geo.cu_seqlens = cu_seqlens;
  geo.chunk_off = chunk_off;
  geo.valid = valid;
  geo.N = N;
  geo.T = T;
  geo.C = kBwdChunk;

  BackwardArgs b;
  PrefillArgs& a = b.fwd;
  a.q = q;
  a.k = k;
  a.v = v;
  a.dtype = dt;
  a.log_alpha = log_alpha;
  a.beta = beta;
  a.initial_state = initial_state;
  a.cu_seqlens = cu_seqlens;
  a.N = N;
  a.B = B;
  a.T = T;
  a.H = H;
  a.Dk = Dk;
  a.Dv = Dv;
  a.C = kBwdChunk;
  a.o = nullptr;
  a.final_state = nullptr;
  b.d_o = d_o;
  b.d_final = d_final_state;
  b.dq = dq;
  b.dk = dk;
  b.dv = dv;
  b.dlog_alpha = dlog_alpha;
  b.dbeta = dbeta;
  b.d_initial = d_initial_state;
  const SimtRecord rec = SimtRecord::make(kBwdChunk, Dk, Dv, true);
  return from_cuda(launch_chunk_bwd(b, geo, (int)lay.max_chunks, (float*)(ws + lay.rec_base), rec,
                                    (float*)(ws + lay.states_base),
                                    (float*)(ws + lay.dstates_base), (float*)(ws + lay.dvp_base),
                                    stream));
}

}  // extern "C"

namespace kda {
namespace {

// Validates a fusion descriptor (NULL = no fusion) and converts it.
kda_status_t to_fusion(const kda_fusion_t* f, Fusion* out) {
  *out = Fusion();
  if (!f) return KDA_OK;
  if (f->qk_l2norm && !(f->qk_l2norm_eps >= 0.f)) return KDA_ERR_INVALID_ARG;
  if ((f->A_log && !aligned(f->A_log, 4)) || (f->dt_bias && !aligned(f->dt_bias, 4)))
    return KDA_ERR_INVALID_ARG;
  out->l2 = f->qk_l2norm ? 1 : 0;
  out->eps = f->qk_l2norm_eps;
  out->A_log = f->A_log;
  out->dt_bias = f->A_log ? f->dt_bias : nullptr;
  if (f->out_norm) {
    if (!(f->out_norm_eps >= 0.f) || (f->out_norm_weight && !aligned(f->out_norm_weight, 4)))
      return KDA_ERR_INVALID_ARG;
    out->onorm = 1;
    out->oeps = f->out_norm_eps;
    out->ow = f->out_norm_weight;
    out->og = f->out_gate;
  }
  return KDA_OK;
}

kda_status_t chunk_fwd_impl(const void* q, const void* k, const void* v, kda_dtype_t dt,
                            const float* log_alpha, const float* beta, const float* initial_state,
                            const int32_t* cu_seqlens, int32_t N, int32_t B, int32_t T, int32_t H,
                            int32_t Dk, int32_t Dv, int32_t C, void* o, float* final_state,
                            void* workspace, size_t workspace_bytes, const Fusion& fz,
                            kda_stream_t stream_) {
  const bool varlen = cu_seqlens != nullptr;
  kda_status_t st = check_prefill_shape(B, T, H, Dk, Dv, C, N, dt, varlen);
  if (st != KDA_OK) return st;
  const long long tokens = (long long)B * T;
  if (tokens > 0) {
    if (!q || !k || !v || !log_alpha || !beta || !o) return KDA_ERR_INVALID_ARG;
    if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16) ||
        !aligned(log_alpha, 16) || !aligned(beta, 4))
      return KDA_ERR_INVALID_ARG;
  }
  if ((initial_state && !aligned(initial_state, 16)) || (final_state && !aligned(final_state, 16)))
    return KDA_ERR_INVALID_ARG;
  if (varlen && !aligned(cu_seqlens, 4)) return KDA_ERR_INVALID_ARG;
  if (fz.onorm && fz.og && tokens > 0 && !aligned(fz.og, 16)) return KDA_ERR_INVALID_ARG;
  if (N == 0) return KDA_OK;

  const WsLayout lay = prefill_layout(B, T, H, Dk, Dv, C, N, varlen, dt);
  if (!workspace || !aligned(workspace, 256) || workspace_bytes < lay.total)
    return KDA_ERR_WORKSPACE;

  cudaStream_t stream = (cudaStream_t)stream_;
  if (kBoundsChecked) {
    BoundsTable t = {};
    const size_t es = dt == KDA_DTYPE_BF16 ? 2 : 4, th = (size_t)tokens * H;
    const size_t states = (size_t)N * H * Dk * Dv * 4;
    set_extent(t, kBufQ, q, th * Dk * es);
    set_extent(t, kBufK, k, th * Dk * es);
    set_extent(t, kBufV, v, th * Dv * es);
    set_extent(t, kBufO, o, th * Dv * es);
    set_extent(t, kBufLogAlpha, log_alpha, th * Dk * 4);
    set_extent(t, kBufBeta, beta, th * 4);
    set_extent(t, kBufInitial, initial_state, initial_state ? states : 0);
    set_extent(t, kBufFinal, final_state, final_state ? states : 0);
    set_extent(t, kBufWork, workspace, workspace_bytes);
    set_extent(t, kBufCuSeqlens, cu_seqlens, varlen ? ((size_t)N + 1) * 4 : 0);
    fusion_extents(t, fz, th * Dv * es, H, Dk, Dv);
    st = from_cuda(register_bounds(t, stream));
    if (st != KDA_OK) return st;
  }
  char* ws = (char*)workspace;
  int32_t* valid = (int32_t*)ws;
  int32_t* chunk_off = (int32_t*)(ws + lay.chunk_off_base);
  if (varlen) {
    st = from_cuda(launch_chunk_map(cu_seqlens, N, (int)tokens, C, chunk_off, valid,
                                    chunk_off + N + 1, stream));
    if (st != KDA_OK) return st;
  }
  SeqGeometry geo;
  if (varlen) geo.order = chunk_off + N + 1;
  geo.cu_seqlens = cu_seqlens;
  geo.chunk_off = chunk_off;
  geo.valid = valid;
  geo.N = N;
  geo.T = T;
  geo.C = C;

  PrefillArgs a;
  a.q = q;
  a.k = k;
  a.v = v;
  a.dtype = dt;
  a.log_alpha = log_alpha;
  a.beta = beta;
  a.initial_state = initial_state;
  a.cu_seqlens = cu_seqlens;
  a.N = N;
  a.B = B;
  a.T = T;
  a.H = H;
  a.Dk = Dk;
  a.Dv = Dv;
  a.C = C;
  a.o = o;
  a.final_state = final_state;
  a.fz = fz;

  if (is_tc_path(dt))
    return from_cuda(launch_prefill_tc(a, geo, (int)lay.max_chunks, (uint8_t*)(ws + lay.rec_base),
                                       stream));
  const SimtRecord rec = SimtRecord::make(C, Dk, Dv);
  return from_cuda(launch_prefill_simt(a, geo, (int)lay.max_chunks,
                                       (float*)(ws + lay.rec_base), rec, stream));
}

kda_status_t recurrent_step_impl(const void* q, const void* k, const void* v, kda_dtype_t dt,
                                 const float* log_alpha, const float* beta, float* state, void* o,
                                 int32_t N, int32_t H, int32_t Dk, int32_t Dv, const Fusion* fz,
                                 kda_stream_t stream) {
  if (N < 0 || H < 0 || Dk <= 0 || Dv <= 0) return KDA_ERR_INVALID_ARG;
  if (dt != KDA_DTYPE_F32 && dt != KDA_DTYPE_BF16) return KDA_ERR_INVALID_ARG;
  if (Dk > 128 || Dv > 128 || Dv % 4 != 0) return KDA_ERR_UNSUPPORTED;
  if ((long long)N * H > INT32_MAX) return KDA_ERR_UNSUPPORTED;
  if ((long long)N * H == 0) return KDA_OK;
  if (!q || !k || !v || !log_alpha || !beta || !state || !o) return KDA_ERR_INVALID_ARG;
  const size_t es = dt == KDA_DTYPE_BF16 ? 2 : 4;  // q, k, v, o need element alignment only
  if (!aligned(state, 16) || !aligned(q, es) || !aligned(k, es) || !aligned(v, es) ||
      !aligned(o, es) || !aligned(log_alpha, 4) || !aligned(beta, 4))
    return KDA_ERR_INVALID_ARG;
  if (fz && fz->onorm && ((fz->og && !aligned(fz->og, es)) || (fz->ow && !aligned(fz->ow, 16))))
    return KDA_ERR_INVALID_ARG;
  if (kBoundsChecked) {
    BoundsTable t = {};
    const size_t nh = (size_t)N * H;
    set_extent(t, kBufQ, q, nh * Dk * es);
    set_extent(t, kBufK, k, nh * Dk * es);
    set_extent(t, kBufV, v, nh * Dv * es);
    set_extent(t, kBufO, o, nh * Dv * es);
    set_extent(t, kBufLogAlpha, log_alpha, nh * Dk * 4);
    set_extent(t, kBufBeta, beta, nh * 4);
    set_extent(t, kBufState, state, nh * Dk * Dv * 4);
    if (fz) fusion_extents(t, *fz, nh * Dv * es, H, Dk, Dv);
    const kda_status_t st = from_cuda(register_bounds(t, (cudaStream_t)stream));
    if (st != KDA_OK) return st;
  }
  return from_cuda(launch_decode_step(q, k, v, dt, log_alpha, beta, state, o, N, H, Dk, Dv, fz,
                                      (cudaStream_t)stream));
}

kda_status_t recurrent_fwd_impl(const void* q, const void* k, const void* v, kda_dtype_t dt,
                                const float* log_alpha, const float* beta, float* pool,
                                const int32_t* state_indices, void* o, int32_t N, int32_t T,
                                int32_t H, int32_t Dk, int32_t Dv, int32_t P, const Fusion& fz,
                                kda_stream_t stream) {
  if (N < 0 || T < 0 || H < 0 || Dk <= 0 || Dv <= 0 || P < 0) return KDA_ERR_INVALID_ARG;
  if (dt != KDA_DTYPE_F32 && dt != KDA_DTYPE_BF16) return KDA_ERR_INVALID_ARG;
  if (Dk > 128 || Dv > 128 || Dv % 4 != 0) return KDA_ERR_UNSUPPORTED;
  if ((long long)N * H > INT32_MAX || (long long)N * T * H * (Dk > Dv ? Dk : Dv) > (1LL << 40))
    return KDA_ERR_UNSUPPORTED;
  if ((long long)N * H * T == 0) return KDA_OK;
  if (!state_indices && P < N) return KDA_ERR_INVALID_ARG;
  if (!q || !k || !v || !log_alpha || !beta || !pool || !o) return KDA_ERR_INVALID_ARG;
  const size_t es = dt == KDA_DTYPE_BF16 ? 2 : 4;
  if (!aligned(pool, 16) || !aligned(q, es) || !aligned(k, es) || !aligned(v, es) ||
      !aligned(o, es) || !aligned(log_alpha, 4) || !aligned(beta, 4) ||
      (state_indices && !aligned(state_indices, 4)) || (fz.onorm && fz.og && !aligned(fz.og, es)) ||
      (fz.onorm && fz.ow && !aligned(fz.ow, 16)))
    return KDA_ERR_INVALID_ARG;
  if (kBoundsChecked) {
    BoundsTable t = {};
    const size_t nth = (size_t)N * T * H;
    set_extent(t, kBufQ, q, nth * Dk * es);
    set_extent(t, kBufK, k, nth * Dk * es);
    set_extent(t, kBufV, v, nth * Dv * es);
    set_extent(t, kBufO, o, nth * Dv * es);
    set_extent(t, kBufLogAlpha, log_alpha, nth * Dk * 4);
    set_extent(t, kBufBeta, beta, nth * 4);
    set_extent(t, kBufState, pool, (size_t)P * H * Dk * Dv * 4);
    set_extent(t, kBufIndices, state_indices, state_indices ? (size_t)N * 4 : 0);
    fusion_extents(t, fz, nth * Dv * es, H, Dk, Dv);
    const kda_status_t st = from_cuda(register_bounds(t, (cudaStream_t)stream));
    if (st != KDA_OK) return st;
  }
  return from_cuda(launch_recurrent_multi(q, k, v, dt, log_alpha, beta, pool, state_indices, o, N,
                                          T, H, Dk, Dv, P, fz, (cudaStream_t)stream));
}

}  // namespace
}  // namespace kda

extern "C" {

kda_status_t kda_chunk_fwd(const void* q, const void* k, const void* v, kda_dtype_t dt,
                           const float* log_alpha, const float* beta, const float* initial_state,
                           const int32_t* cu_seqlens, int32_t N, int32_t B, int32_t T, int32_t H,
                           int32_t Dk, int32_t Dv, int32_t C, void* o, float* final_state,
                           void* workspace, size_t workspace_bytes, kda_stream_t stream) {
  return chunk_fwd_impl(q, k, v, dt, log_alpha, beta, initial_state, cu_seqlens, N, B, T, H, Dk,
                        Dv, C, o, final_state, workspace, workspace_bytes, Fusion(), stream);
}

kda_status_t kda_chunk_fwd_fused(const void* q, const void* k, const void* v, kda_dtype_t dt,
                                 const float* log_alpha_or_gate, const float* beta,
                                 const float* initial_state, const int32_t* cu_seqlens, int32_t N,
                                 int32_t B, int32_t T, int32_t H, int32_t Dk, int32_t Dv,
                                 int32_t C, void* o, float* final_state, void* workspace,
                                 size_t workspace_bytes, const kda_fusion_t* fusion,
                                 kda_stream_t stream) {
  Fusion fz;
  const kda_status_t st = to_fusion(fusion, &fz);
  if (st != KDA_OK) return st;
  return chunk_fwd_impl(q, k, v, dt, log_alpha_or_gate, beta, initial_state, cu_seqlens, N, B, T,
                        H, Dk, Dv, C, o, final_state, workspace, workspace_bytes, fz, stream);
}

kda_status_t kda_recurrent_step(const void* q, const void* k, const void* v, kda_dtype_t dt,
                                const float* log_alpha, const float* beta, float* state, void* o,
                                int32_t N, int32_t H, int32_t Dk, int32_t Dv,
                                kda_stream_t stream) {
  return recurrent_step_impl(q, k, v, dt, log_alpha, beta, state, o, N, H, Dk, Dv, nullptr,
                             stream);
}

kda_status_t kda_recurrent_step_fused(const void* q, const void* k, const void* v,
                                      kda_dtype_t dt, const float* log_alpha_or_gate,
                                      const float* beta, float* state, void* o, int32_t N,
                                      int32_t H, int32_t Dk, int32_t Dv,
                                      const kda_fusion_t* fusion, kda_stream_t stream) {
  Fusion fz;
  const kda_status_t st = to_fusion(fusion, &fz);
  if (st != KDA_OK) return st;
  return recurrent_step_impl(q, k, v, dt, log_alpha_or_gate, beta, state, o, N, H, Dk, Dv,
                             fusion ? &fz : nullptr, stream);
}

kda_status_t kda_recurrent_fwd(const void* q, const void* k, const void* v, kda_dtype_t dt,
                               const float* log_alpha, const float* beta, float* pool,
                               const int32_t* state_indices, void* o, int32_t N, int32_t T,
                               int32_t H, int32_t Dk, int32_t Dv, int32_t P,
                               kda_stream_t stream) {
  return recurrent_fwd_impl(q, k, v, dt, log_alpha, beta, pool, state_indices, o, N, T, H, Dk, Dv,
                            P, Fusion(), stream);
}

kda_status_t kda_recurrent_fwd_fused(const void* q, const void* k, const void* v, kda_dtype_t dt,
                                     const float* log_alpha_or_gate, const float* beta,
                                     float* pool, const int32_t* state_indices, void* o,
                                     int32_t N, int32_t T, int32_t H, int32_t Dk, int32_t Dv,
                                     int32_t P, const kda_fusion_t* fusion, kda_stream_t stream) {
  Fusion fz;
  const kda_status_t st = to_fusion(fusion, &fz);
  if (st != KDA_OK) return st;
  return recurrent_fwd_impl(q, k, v, dt, log_alpha_or_gate, beta, pool, state_indices, o, N, T, H,
                            Dk, Dv, P, fz, stream);
}

kda_status_t kda_last_device_error(kda_stream_t stream) {
  cudaError_t e = cudaStreamSynchronize((cudaStream_t)stream);
  if (e != cudaSuccess) return KDA_ERR_CUDA;
  unsigned int bits = 0;
  e = cudaMemcpyFromSymbol(&bits, g_status, sizeof(bits));
  if (e != cudaSuccess) return KDA_ERR_CUDA;
  if (bits) {
    const unsigned int zero = 0;
    e = cudaMemcpyToSymbol(g_status, &zero, sizeof(zero));
    if (e != cudaSuccess) return KDA_ERR_CUDA;
  }
  if (bits & kStatusTimeout) return KDA_ERR_TIMEOUT;
  if (bits & (kStatusBadSeqlens | kStatusBounds)) return KDA_ERR_INVALID_ARG;
  return KDA_OK;
}

}  // extern "C"
