/*
 * kda.h — C ABI of the Kimi Delta Attention (KDA) operator for NVIDIA B200 (sm_100a).
 *
 * KDA is the channel-wise gated delta rule
 *     S_t = (I - beta_t k_t k_t^T) Diag(alpha_t) S_{t-1} + beta_t k_t v_t^T,      o_t = S_t^T q_t
 * ("Kimi Linear: An Expressive, Efficient Attention Architecture", paper-graph-ui walkthrough,
 *  §3.4 "The KDA State Update Equation", Eq. 1 and the output read that follows it).
 * S is d_k x d_v (rows indexed by key channels), alpha_t = exp(log_alpha_t) in (0,1]^{d_k},
 * beta_t in [0,1]. No query scale is applied: o_t reads the updated state S_t.
 *
 * Conventions shared by every entry point
 *   - All tensor pointers are DEVICE pointers owned by the caller. Nothing is allocated inside
 *     the calls: prefill scratch is the caller's `workspace`.
 *   - Calls are asynchronous and stream-ordered on `stream` (NULL = legacy default stream).
 *     They return once the kernels are enqueued.
 *   - Argument errors (null pointers, unsupported sizes, misaligned pointers, workspace too
 *     small) are detected on the host before anything is launched; nothing is written then.
 *   - Faults that only the device can see (a cu_seqlens array that is not monotone or that runs
 *     past T) set a per-device status word; the kernels then skip their work and
 *     kda_last_device_error() reports it.
 *   - No C++ exception crosses this boundary.
 *
 * Layouts (row-major, innermost dimension last):
 *   q, k          [B, T, H, Dk]   dtype = qkv_dtype (bf16 or fp32)
 *   v, o          [B, T, H, Dv]   dtype = qkv_dtype
 *   log_alpha     [B, T, H, Dk]   fp32, finite and <= 0 (log of the per-channel decay alpha)
 *   beta          [B, T, H]       fp32
 *   states        [N, H, Dk, Dv]  fp32 (N = number of sequences)
 * For packed variable-length input, B = 1, T = total tokens and cu_seqlens holds N+1 offsets.
 */
#ifndef KDA_H_
#define KDA_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define KDA_API __attribute__((visibility("default")))
#else
#define KDA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* kda_stream_t; /* identical to cudaStream_t */

typedef enum {
  KDA_OK = 0,
  KDA_ERR_INVALID_ARG = 1, /* null pointer, negative size, misalignment, bad cu_seqlens */
  KDA_ERR_UNSUPPORTED = 2, /* a size or dtype combination the library has no kernel for */
  KDA_ERR_CUDA = 3,        /* a CUDA runtime call failed (launch error, no device, ...) */
  KDA_ERR_TIMEOUT = 4,     /* a bounded device-side wait gave up */
  KDA_ERR_WORKSPACE = 5    /* workspace missing, too small or not 256-byte aligned */
} kda_status_t;

typedef enum { KDA_DTYPE_F32 = 0, KDA_DTYPE_BF16 = 1 } kda_dtype_t;

/* Human-readable name of a status code. Never returns NULL. */
KDA_API const char* kda_status_string(kda_status_t status);

/* Library version, "major.minor.patch". */
KDA_API const char* kda_version(void);

/*
 * kda_chunk_fwd_workspace_size — bytes of device scratch that kda_chunk_fwd needs.
 *
 * Chunkwise prefill keeps, per chunk and head, the UT-transform products of the walkthrough's
 * §3.4 "Chunkwise Parallelization" (W, U, the decayed keys and queries, the causal
 * query-key matrix and the chunk decay). The figure is an upper bound valid for any
 * cu_seqlens with `num_seqs` sequences totalling B*T tokens.
 *   B, T, H, Dk, Dv, chunk, num_seqs : as for kda_chunk_fwd; qkv_dtype selects the kernel path.
 *   bytes (out, host pointer)         : required size, a multiple of 256.
 * Returns KDA_ERR_INVALID_ARG / KDA_ERR_UNSUPPORTED for sizes kda_chunk_fwd would reject.
 */
KDA_API kda_status_t kda_chunk_fwd_workspace_size(int32_t B, int32_t T, int32_t H, int32_t Dk, int32_t Dv,
                                          int32_t chunk, int32_t num_seqs, kda_dtype_t qkv_dtype,
                                          size_t* bytes);

/*
 * kda_chunk_fwd — chunkwise-parallel prefill (the walkthrough's §3.4 "Chunkwise
 * Parallelization": UT transform, chunk state update Eq. 8, chunk output Eq. 9).
 *
 *   q, k, v         device, layouts above, dtype qkv_dtype; 16-byte aligned.
 *   log_alpha       device fp32 [B,T,H,Dk]; finite, <= 0. 16-byte aligned.
 *   beta            device fp32 [B,T,H].
 *   initial_state   device fp32 [N,H,Dk,Dv], or NULL for zero states. May alias final_state.
 *   cu_seqlens      device int32 [N+1] with cu_seqlens[0] = 0, non-decreasing,
 *                   cu_seqlens[N] <= B*T; or NULL, then the B rows are N = B sequences of T.
 *                   When non-NULL, B must be 1. Sequences may be empty.
 *   num_seqs        N (must equal B when cu_seqlens is NULL).
 *   chunk           chunk length C: 64 on the bf16 path; 16, 32 or 64 on the fp32 path.
 *   o               device [B,T,H,Dv], dtype qkv_dtype (rounded to nearest-even for bf16).
 *   final_state     device fp32 [N,H,Dk,Dv], or NULL to skip it.
 *   workspace       device scratch of at least kda_chunk_fwd_workspace_size() bytes,
 *                   256-byte aligned; its contents on entry are ignored.
 * Supported: qkv_dtype BF16 with Dk = Dv = 128, chunk = 64 (tensor-core path); qkv_dtype F32
 * with 1 <= Dk, Dv <= 128 and Dv a multiple of 4 (CUDA-core fp32 path).
 * Size limits (else KDA_ERR_UNSUPPORTED, before any launch): B*T <= INT32_MAX tokens,
 * B*T*H*max(Dk, Dv) <= 2^40 elements, H <= 65535, (chunks + N) * H <= INT32_MAX and
 * 2 * N * H <= INT32_MAX (chunks = ceil(B*T / chunk); the same limits hold for kda_chunk_bwd
 * with chunk = 32).
 * Tokens past cu_seqlens[N] are neither read nor written.
 */
KDA_API kda_status_t kda_chunk_fwd(const void* q, const void* k, const void* v, kda_dtype_t qkv_dtype,
                           const float* log_alpha, const float* beta, const float* initial_state,
                           const int32_t* cu_seqlens, int32_t num_seqs, int32_t B, int32_t T,
                           int32_t H, int32_t Dk, int32_t Dv, int32_t chunk, void* o,
                           float* final_state, void* workspace, size_t workspace_bytes,
                           kda_stream_t stream);

/*
 * kda_chunk_fwd_noalloc — kda_chunk_fwd for callers that must not allocate device memory.
 *
 * The pages have no counterpart to this entry point; it exists only for deployment. Some callers
 * cannot hand the library a workspace: a serving engine that reserves nearly all of HBM for its
 * caches up front and hands out no side buffers, a plugin whose host framework owns every
 * device allocation, or a latency-critical loop that avoids cudaMalloc/cudaFree because they can
 * synchronise the whole device. This variant takes the same arguments as kda_chunk_fwd minus the
 * workspace and uses instead a scratch array of KDA_NOALLOC_SCRATCH_BYTES that lives in the
 * library's own device image (every GPU that loads the library holds it until the process
 * exits). It calls no cudaMalloc, cudaFree or other allocating routine.
 *
 *   - Limit: a call whose workspace (kda_chunk_fwd_workspace_size) exceeds
 *     KDA_NOALLOC_SCRATCH_BYTES is rejected with KDA_ERR_WORKSPACE before anything is launched.
 *   - Set-up: the first call on a device looks up the device address of the scratch array (with
 *     that device current), so make that first call before any stream capture; the current
 *     device must be the one that owns the pointers. The address is kept for the life of the
 *     process: resetting the device (cudaDeviceReset, or anything else that destroys and
 *     re-creates its primary context) leaves it stale, so do not call this entry point on a
 *     device after resetting it in the same process.
 *   - Sharing: all calls on a device share the one array and it keeps the last call's contents.
 *     Nothing in it needs clearing (every byte a call reads was written earlier in that call),
 *     but calls that overlap on the GPU (different streams, or different host threads) race on
 *     it: serialise them.
 */
#define KDA_NOALLOC_SCRATCH_BYTES ((size_t)64 << 20)

KDA_API kda_status_t kda_chunk_fwd_noalloc(const void* q, const void* k, const void* v,
                                           kda_dtype_t qkv_dtype, const float* log_alpha,
                                           const float* beta, const float* initial_state,
                                           const int32_t* cu_seqlens, int32_t num_seqs, int32_t B,
                                           int32_t T, int32_t H, int32_t Dk, int32_t Dv,
                                           int32_t chunk, void* o, float* final_state,
                                           kda_stream_t stream);

/*
 * kda_recurrent_step — one decode token per sequence, state updated in place (the
 * walkthrough's §3.4 "FLOPs Accounting and Inference Strategy": the recurrent kernel used for
 * generation; the update is Eq. 1 in its online-gradient form of "Online Learning
 * Interpretation": S' = Diag(alpha) S, S = S' - beta k (S'^T k - v)^T).
 *
 *   q, k            device [N,H,Dk], dtype qkv_dtype.
 *   v               device [N,H,Dv], dtype qkv_dtype.
 *   log_alpha       device fp32 [N,H,Dk]; beta device fp32 [N,H].
 *   state           device fp32 [N,H,Dk,Dv], read and overwritten; 16-byte aligned.
 *   o               device [N,H,Dv], dtype qkv_dtype: o = S_new^T q.
 * q, k, v and o need the alignment of their element type; log_alpha and beta 4 bytes.
 * Supported: 1 <= Dk <= 128, 4 <= Dv <= 128 (Dv % 4 == 0), either dtype, N * H <= INT32_MAX
 * (else KDA_ERR_UNSUPPORTED). The state is streamed once from HBM and written once.
 */
KDA_API kda_status_t kda_recurrent_step(const void* q, const void* k, const void* v, kda_dtype_t qkv_dtype,
                                const float* log_alpha, const float* beta, float* state, void* o,
                                int32_t N, int32_t H, int32_t Dk, int32_t Dv, kda_stream_t stream);

/*
 * kda_recurrent_fwd — token-by-token KDA over short sequences (the recurrent mode the walkthrough's
 * §3.4 "FLOPs Accounting and Inference Strategy" uses for generation; the model card's code picks
 * it for query lengths up to 64) with states taken from a pool, as a serving cache holds them.
 * For each sequence n the T tokens are applied in order to state pool[state_indices[n]] (Eq. 1,
 * o_t = S_t^T q_t); that state is read once, kept on chip for all T tokens and written once.
 *
 *   q, k            device [N, T, H, Dk], dtype qkv_dtype.
 *   v, o            device [N, T, H, Dv], dtype qkv_dtype.
 *   log_alpha       device fp32 [N, T, H, Dk]; beta device fp32 [N, T, H].
 *   state_pool      device fp32 [P, H, Dk, Dv], updated in place; 16-byte aligned.
 *   state_indices   device int32 [N]: pool row of sequence n. A negative entry skips the sequence
 *                   (no state update, its o is left untouched). Entries must be distinct; an
 *                   entry >= P is skipped too and reported as KDA_ERR_INVALID_ARG through
 *                   kda_last_device_error(). NULL means pool row n (then P >= N is required).
 * Supported: as kda_recurrent_step, T >= 0 and N * T * H * max(Dk, Dv) <= 2^40.
 * For longer sequences kda_chunk_fwd is the faster path.
 */
KDA_API kda_status_t kda_recurrent_fwd(const void* q, const void* k, const void* v,
                                       kda_dtype_t qkv_dtype, const float* log_alpha,
                                       const float* beta, float* state_pool,
                                       const int32_t* state_indices, void* o, int32_t N, int32_t T,
                                       int32_t H, int32_t Dk, int32_t Dv, int32_t P,
                                       kda_stream_t stream);

/*
 * Fusion of the steps around the operator in the model ("Kimi Linear: An Expressive, Efficient
 * Attention Architecture", paper-graph-ui walkthrough, §3.4 "Neural Parameterization").
 *
 * Prologue: q, k = L2Norm(...) and alpha = f(low-rank gate); the L2 Deep Distill page's
 * implementation notes put the L2 normalisation of q and k inside the kernel and fuse the decay
 * gate with A_log and a bias. The pages leave f unspecified beyond "similar to GDN and Mamba2, in
 * log space"; this library reads it as
 *     log alpha[t, h, c] = -exp(A_log[h]) * softplus(g[t, h, c] + dt_bias[h, c]).
 *
 * Epilogue: the output-gate equation of the same section applies, per (token, head), a head-wise
 * RMSNorm and a sigmoid gate to the operator's output (the module table of the L2 Deep Distill
 * page names it FusedRMSNormGated: the sigmoid gate inside the RMSNorm). With out_norm set the
 * library stores, instead of o,
 *     y[t, h, c] = sigmoid(out_gate[t, h, c]) * out_norm_weight[c] * o[t, h, c]
 *                  / sqrt(mean_c' o[t, h, c']^2 + out_norm_eps)
 * where o is the fp32 result before rounding. The output projection W_o that follows is a plain
 * GEMM and stays with the caller.
 */
typedef struct {
  int32_t qk_l2norm;     /* nonzero: q and k are divided by sqrt(sum x^2 + qk_l2norm_eps) per
                            (token, head) inside the kernels */
  float qk_l2norm_eps;   /* e.g. 1e-6 */
  const float* A_log;    /* device fp32 [H], or NULL. Non-NULL: the log_alpha argument holds the
                            raw gate g (same layout) and the decay is computed as above */
  const float* dt_bias;  /* device fp32 [H, Dk], or NULL for a zero bias; used only with A_log */
  int32_t out_norm;      /* nonzero: the output epilogue above replaces o by y */
  float out_norm_eps;    /* e.g. 1e-5; must be >= 0 */
  const float* out_norm_weight; /* device fp32 [Dv] (16-byte aligned), or NULL for ones */
  const void* out_gate;  /* device, o's layout and dtype ([B,T,H,Dv] / [N,T,H,Dv]), or NULL for
                            no gate; used only with out_norm. 16-byte aligned for bf16 prefill */
} kda_fusion_t;

/* kda_chunk_fwd with the fusion above; fusion == NULL is exactly kda_chunk_fwd. With out_norm on
 * the bf16 path, the state kernel runs as clusters of two CTAs (the two column halves of one
 * (sequence, head)) that exchange per-row sums of squares through distributed shared memory. */
KDA_API kda_status_t kda_chunk_fwd_fused(const void* q, const void* k, const void* v,
                                         kda_dtype_t qkv_dtype, const float* log_alpha_or_gate,
                                         const float* beta, const float* initial_state,
                                         const int32_t* cu_seqlens, int32_t num_seqs, int32_t B,
                                         int32_t T, int32_t H, int32_t Dk, int32_t Dv,
                                         int32_t chunk, void* o, float* final_state,
                                         void* workspace, size_t workspace_bytes,
                                         const kda_fusion_t* fusion, kda_stream_t stream);

/* kda_recurrent_step with the fusion above (the serving decode step with the layer's prologue
 * and epilogue); fusion == NULL is exactly kda_recurrent_step. The streaming kernel runs it when
 * the shapes and pointers allow 16-byte bulk copies, the token-by-token kernel otherwise. */
KDA_API kda_status_t kda_recurrent_step_fused(const void* q, const void* k, const void* v,
                                              kda_dtype_t qkv_dtype, const float* log_alpha_or_gate,
                                              const float* beta, float* state, void* o, int32_t N,
                                              int32_t H, int32_t Dk, int32_t Dv,
                                              const kda_fusion_t* fusion, kda_stream_t stream);

/* kda_recurrent_fwd with the fusion above; fusion == NULL is exactly kda_recurrent_fwd. */
KDA_API kda_status_t kda_recurrent_fwd_fused(const void* q, const void* k, const void* v,
                                             kda_dtype_t qkv_dtype, const float* log_alpha_or_gate,
                                             const float* beta, float* state_pool,
                                             const int32_t* state_indices, void* o, int32_t N,
                                             int32_t T, int32_t H, int32_t Dk, int32_t Dv,
                                             int32_t P, const kda_fusion_t* fusion,
                                             kda_stream_t stream);

/*
 * kda_chunk_bwd — backward pass of the operator (reverse-mode derivative of kda_chunk_fwd).
 *
 * The pages motivate it through training ("Kimi Linear: An Expressive, Efficient Attention
 * Architecture", paper-graph-ui walkthrough, §3.4 "Chunkwise Parallelization": the UT transform
 * is what makes the chunk form trainable; "FLOPs Accounting and Inference Strategy": training
 * FLOPs). Computes the gradients of L = <d_o, o> + <d_final_state, final_state> with respect to
 * every input of the same call of kda_chunk_fwd (same q, k, v, log_alpha, beta, initial_state,
 * cu_seqlens, num_seqs, B, T, H, Dk, Dv; no prologue or epilogue fusion).
 *
 *   d_o             device, o's layout [B,T,H,Dv] and q's dtype: the output cotangent
 *   d_final_state   device fp32 [N,H,Dk,Dv], or NULL for zero
 *   dq, dk          device [B,T,H,Dk], q's dtype (written for every token of a sequence)
 *   dv              device [B,T,H,Dv], q's dtype
 *   dlog_alpha      device fp32 [B,T,H,Dk]
 *   dbeta           device fp32 [B,T,H]
 *   d_initial_state device fp32 [N,H,Dk,Dv], or NULL (not computed)
 *   workspace       device, >= kda_chunk_bwd_workspace_size(...) bytes, 256-byte aligned
 *
 * The pass runs the fp32 chunk kernels forward once more (chunks of 32 tokens, whatever chunk
 * the forward call used; the result does not depend on it), keeping the state entering every
 * chunk, then a sequential backward state pass and a parallel chunk-local pass; all arithmetic
 * is fp32 on CUDA cores, for fp32 and bf16 inputs alike. Supported: Dk, Dv multiples of 4 in
 * [4, 128] (anything else: KDA_ERR_UNSUPPORTED). Tokens
 * outside every sequence (varlen) are not written. Arguments are checked on the host (pointers
 * aligned to their element size); a bad cu_seqlens is reported by kda_last_device_error().
 */
KDA_API kda_status_t kda_chunk_bwd_workspace_size(int32_t B, int32_t T, int32_t H, int32_t Dk,
                                                  int32_t Dv, int32_t num_seqs,
                                                  kda_dtype_t qkv_dtype, size_t* bytes);
KDA_API kda_status_t kda_chunk_bwd(const void* q, const void* k, const void* v,
                                   kda_dtype_t qkv_dtype, const float* log_alpha,
                                   const float* beta, const float* initial_state,
                                   const int32_t* cu_seqlens, int32_t num_seqs, int32_t B,
                                   int32_t T, int32_t H, int32_t Dk, int32_t Dv, const void* d_o,
                                   const float* d_final_state, void* dq, void* dk, void* dv,
                                   float* dlog_alpha, float* dbeta, float* d_initial_state,
                                   void* workspace, size_t workspace_bytes, kda_stream_t stream);

/*
 * kda_last_device_error — read and clear the per-device status word that the kernels set
 * (KDA_ERR_INVALID_ARG for a bad cu_seqlens, KDA_ERR_TIMEOUT for a bounded wait that gave up).
 * Synchronises `stream`. Returns KDA_OK when no kernel reported a fault.
 */
KDA_API kda_status_t kda_last_device_error(kda_stream_t stream);

/*
 * Kernel-level timing (tracing). While enabled, every kernel the library launches on the calling
 * host thread is bracketed by a pair of CUDA events recorded on its stream. kda_profile_read
 * synchronises those events, returns per-kernel launch counts and summed device milliseconds
 * (entries sorted by total time, descending) and forgets them. Events are host-side objects: no
 * device memory is allocated. Disabled by default; enabling adds two event records per launch.
 */
typedef struct {
  char name[48];
  int32_t launches;
  double total_ms;
} kda_profile_entry_t;

KDA_API kda_status_t kda_profile_enable(int32_t enable);
KDA_API kda_status_t kda_profile_read(kda_profile_entry_t* entries, int32_t capacity,
                                      int32_t* count);

#ifdef __cplusplus
}
#endif

#endif /* KDA_H_ */
