/*
 * kda_oracle.c — fp64 CPU oracle of the Kimi Delta Attention operator.
 *
 * TEST INFRASTRUCTURE ONLY. Nothing on the product path may call, link or load this file: only
 * the tests, the package smoke check and the benchmark's CPU-baseline leg use it. It shares no
 * code, header, table or helper with the CUDA library.
 *
 * Sources ("Kimi Linear: An Expressive, Efficient Attention Architecture"):
 *   [W]  paper-graph-ui walkthrough, §3.4 "Detailed, Sentence-Based Technical Breakdown":
 *        "The KDA State Update Equation" (Eq. 1 and the output read o_t = S_t^T q_t),
 *        "Online Learning Interpretation" (the gradient-step form of Eq. 1),
 *        "Chunkwise Parallelization" (chunk notation, WY/UT transform, Eq. 8, Eq. 9).
 *   [D]  zhaifeiyue "L2 Deep Distill", §4 "6 项最低检查" item 2: the state at the end of a chunk
 *        is the initial state of the next one.
 *
 * Everything is fp64 and written for readability, not speed. Layouts are packed:
 *   q, k, log_alpha [T_total, H, Dk]; v, o [T_total, H, Dv]; beta [T_total, H];
 *   states [N, H, Dk, Dv]; cu_seqlens [N+1] (int64) gives sequence n = tokens
 *   cu_seqlens[n] .. cu_seqlens[n+1]-1.
 *
 * Parity pins (tests/test_oracle_pins.py): closed forms for beta = 0 and alpha = 1, exact
 * key-to-value retrieval with orthonormal keys, delta-rule overwrite, the scalar-gate (Gated
 * DeltaNet) special case, the chunk hand-off invariant, brute-force transition products, and
 * agreement between kda_oracle_recurrent and kda_oracle_chunked (two independent
 * formulations of [W]) for several chunk sizes.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

#define IDX3(t, h, c, H, D) ((((int64_t)(t)) * (H) + (h)) * (D) + (c))

static void set_threads(int nthreads) {
#ifdef _OPENMP
  if (nthreads > 0) omp_set_num_threads(nthreads);
#else
  (void)nthreads;
#endif
}

/* Number of OpenMP threads a parallel region would use (1 without OpenMP). */
int kda_oracle_max_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

/*
 * Token-by-token recurrence — the plain definition ([W] Eq. 1 and o_t = S_t^T q_t), evaluated
 * in the gradient-step form of [W] "Online Learning Interpretation":
 *     S~ = Diag(alpha_t) S_{t-1}
 *     e  = S~^T k_t                       (prediction for key k_t)
 *     S_t = S~ - beta_t k_t (e - v_t)^T   (= (I - beta k k^T) S~ + beta k v^T)
 *     o_t = S_t^T q_t                     (reads the UPDATED state)
 * alpha_t = exp(log_alpha_t) per key channel (row of S). No query scale.
 * initial_state may be NULL (zero state); final_state may be NULL.
 */
int kda_oracle_recurrent(const double* q, const double* k, const double* v, const double* log_alpha,
                         const double* beta, const double* initial_state, const int64_t* cu_seqlens,
                         int64_t N, int64_t H, int64_t Dk, int64_t Dv, double* o,
                         double* final_state, int nthreads) {
  if (!q || !k || !v || !log_alpha || !beta || !cu_seqlens || !o) return 1;
  if (N < 0 || H <= 0 || Dk <= 0 || Dv <= 0) return 1;
  set_threads(nthreads);
  int bad = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : bad)
  for (int64_t nh = 0; nh < N * H; ++nh) {
    const int64_t n = nh / H, h = nh % H;
    double* S = (double*)malloc(sizeof(double) * Dk * Dv);
    double* e = (double*)malloc(sizeof(double) * Dv);
    if (!S || !e) {
      bad |= 1;
      free(S);
      free(e);
      continue;
    }
    const double* S0 = initial_state ? initial_state + nh * Dk * Dv : NULL;
    for (int64_t i = 0; i < Dk * Dv; ++i) S[i] = S0 ? S0[i] : 0.0;
    for (int64_t t = cu_seqlens[n]; t < cu_seqlens[n + 1]; ++t) {
      const double* kt = k + IDX3(t, h, 0, H, Dk);
      const double* qt = q + IDX3(t, h, 0, H, Dk);
      const double* vt = v + IDX3(t, h, 0, H, Dv);
      const double* lat = log_alpha + IDX3(t, h, 0, H, Dk);
      const double bt = beta[t * H + h];
      /* S~ = Diag(alpha) S : row i of S is key channel i */
      for (int64_t i = 0; i < Dk; ++i) {
        const double a = exp(lat[i]);
        for (int64_t j = 0; j < Dv; ++j) S[i * Dv + j] *= a;
      }
      /* e = S~^T k */
      for (int64_t j = 0; j < Dv; ++j) e[j] = 0.0;
      for (int64_t i = 0; i < Dk; ++i)
        for (int64_t j = 0; j < Dv; ++j) e[j] += S[i * Dv + j] * kt[i];
      /* S = S~ - beta k (e - v)^T */
      for (int64_t i = 0; i < Dk; ++i)
        for (int64_t j = 0; j < Dv; ++j) S[i * Dv + j] -= bt * kt[i] * (e[j] - vt[j]);
      /* o = S^T q */
      double* ot = o + IDX3(t, h, 0, H, Dv);
      for (int64_t j = 0; j < Dv; ++j) {
        double acc = 0.0;
        for (int64_t i = 0; i < Dk; ++i) acc += S[i * Dv + j] * qt[i];
        ot[j] = acc;
      }
    }
    if (final_state)
      for (int64_t i = 0; i < Dk * Dv; ++i) final_state[nh * Dk * Dv + i] = S[i];
    free(S);
    free(e);
  }
  return bad;
}

/*
 * (I + A)^{-1} for a strictly lower-triangular C x C matrix A, by forward substitution row by
 * row ([W] "The UT transform": the inverse of the unit lower-triangular matrix is obtained by
 * forward substitution instead of a general inverse). Row r of X = (I + A)^{-1} satisfies
 *     X[r,:] = e_r - sum_{j<r} A[r,j] X[j,:]
 * because (I + A) X = I. Row-major, A and X must not overlap.
 */
void kda_oracle_unit_lower_inverse(const double* A, int64_t C, double* X) {
  for (int64_t r = 0; r < C; ++r) {
    for (int64_t c = 0; c < C; ++c) X[r * C + c] = (r == c) ? 1.0 : 0.0;
    for (int64_t j = 0; j < r; ++j) {
      const double a = A[r * C + j];
      if (a == 0.0) continue;
      for (int64_t c = 0; c < C; ++c) X[r * C + c] -= a * X[j * C + c];
    }
  }
}

/*
 * Chunkwise WY/UT evaluation of the same operator, following [W] "Chunkwise Parallelization"
 * step by step, in fp64, for one chunk length `chunk` (any C >= 1). Test-only: it pins the chunk
 * algebra against the recurrence. For each sequence and head, chunk [t] holds rows r = 1..Cc
 * (the last chunk of a sequence may be shorter):
 *   Gamma_r      = prod_{j<=r} alpha_j            (cumulative decay from the chunk start,
 *                                                 inclusive of r; kept in log space g_r)
 *   A            = StrictTril(Diag(beta) (Gamma . K) (K / Gamma)^T)
 *   M            = (I + A)^{-1} Diag(beta)         (forward substitution)
 *   W = M (Gamma . K),   U = M V
 *   V'           = U - W S                         (pseudo-value)
 *   O            = (Gamma . Q) S + Tril((Gamma . Q)(K / Gamma)^T) V'        (Eq. 9, Tril inclusive)
 *   S_next       = Diag(gamma_C) S + (Gamma_{i->C} . K)^T V'                  (Eq. 8)
 * with Gamma_{i->C} = gamma_C / gamma_i (decay strictly after position i up to the chunk end;
 * the walkthrough's product printed from j = i is read as starting at j = i+1, which is the
 * only reading under which its WY recurrences and its matrix form agree).
 * The ratios gamma_r / gamma_i are formed as exp(g_r - g_i), which is the literal entry of
 * (Gamma . K)(K / Gamma)^T without the fp64 overflow of 1/gamma_i for long chunks.
 */
int kda_oracle_chunked(const double* q, const double* k, const double* v, const double* log_alpha,
                       const double* beta, const double* initial_state, const int64_t* cu_seqlens,
                       int64_t N, int64_t H, int64_t Dk, int64_t Dv, int64_t chunk, double* o,
                       double* final_state, int nthreads) {
  if (!q || !k || !v || !log_alpha || !beta || !cu_seqlens || !o) return 1;
  if (N < 0 || H <= 0 || Dk <= 0 || Dv <= 0 || chunk <= 0) return 1;
  set_threads(nthreads);
  const int64_t C = chunk;
  int bad = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : bad)
  for (int64_t nh = 0; nh < N * H; ++nh) {
    const int64_t n = nh / H, h = nh % H;
    double* S = (double*)calloc((size_t)(Dk * Dv), sizeof(double));
    double* Snew = (double*)calloc((size_t)(Dk * Dv), sizeof(double));
    double* g = (double*)calloc((size_t)(C * Dk), sizeof(double));
    double* A = (double*)calloc((size_t)(C * C), sizeof(double));
    double* Tinv = (double*)calloc((size_t)(C * C), sizeof(double));
    double* M = (double*)calloc((size_t)(C * C), sizeof(double));
    double* W = (double*)calloc((size_t)(C * Dk), sizeof(double));
    double* U = (double*)calloc((size_t)(C * Dv), sizeof(double));
    double* Vp = (double*)calloc((size_t)(C * Dv), sizeof(double));
    double* Aqk = (double*)calloc((size_t)(C * C), sizeof(double));
    if (!S || !Snew || !g || !A || !Tinv || !M || !W || !U || !Vp || !Aqk) {
      bad |= 1;
    } else {
      if (initial_state)
        for (int64_t i = 0; i < Dk * Dv; ++i) S[i] = initial_state[nh * Dk * Dv + i];
      const int64_t t_begin = cu_seqlens[n], t_end = cu_seqlens[n + 1];
      for (int64_t c0 = t_begin; c0 < t_end; c0 += C) {
        const int64_t Cc = (t_end - c0 < C) ? (t_end - c0) : C;
#define Kr(r, c) k[IDX3(c0 + (r), h, (c), H, Dk)]
#define Qr(r, c) q[IDX3(c0 + (r), h, (c), H, Dk)]
#define Vr(r, c) v[IDX3(c0 + (r), h, (c), H, Dv)]
#define Br(r) beta[(c0 + (r)) * H + h]
        /* g_r = log gamma_r = sum_{j<=r} log alpha_j (per key channel) */
        for (int64_t c = 0; c < Dk; ++c) {
          double acc = 0.0;
          for (int64_t r = 0; r < Cc; ++r) {
            acc += log_alpha[IDX3(c0 + r, h, c, H, Dk)];
            g[r * Dk + c] = acc;
          }
        }
        /* A = StrictTril(Diag(beta)(Gamma.K)(K/Gamma)^T) and Aqk = Tril((Gamma.Q)(K/Gamma)^T) */
        for (int64_t r = 0; r < Cc; ++r)
          for (int64_t i = 0; i < Cc; ++i) {
            double akk = 0.0, aqk = 0.0;
            if (i <= r)
              for (int64_t c = 0; c < Dk; ++c) {
                const double ratio = exp(g[r * Dk + c] - g[i * Dk + c]); /* gamma_r / gamma_i */
                akk += Kr(r, c) * Kr(i, c) * ratio;
                aqk += Qr(r, c) * Kr(i, c) * ratio;
              }
            A[r * Cc + i] = (i < r) ? Br(r) * akk : 0.0;
            Aqk[r * Cc + i] = (i <= r) ? aqk : 0.0;
          }
        /* M = (I + A)^{-1} Diag(beta) */
        kda_oracle_unit_lower_inverse(A, Cc, Tinv);
        for (int64_t r = 0; r < Cc; ++r)
          for (int64_t i = 0; i < Cc; ++i) M[r * Cc + i] = Tinv[r * Cc + i] * Br(i);
        /* W = M (Gamma.K), U = M V */
        for (int64_t r = 0; r < Cc; ++r) {
          for (int64_t c = 0; c < Dk; ++c) {
            double acc = 0.0;
            for (int64_t i = 0; i < Cc; ++i) acc += M[r * Cc + i] * exp(g[i * Dk + c]) * Kr(i, c);
            W[r * Dk + c] = acc;
          }
          for (int64_t c = 0; c < Dv; ++c) {
            double acc = 0.0;
            for (int64_t i = 0; i < Cc; ++i) acc += M[r * Cc + i] * Vr(i, c);
            U[r * Dv + c] = acc;
          }
        }
        /* V' = U - W S */
        for (int64_t r = 0; r < Cc; ++r)
          for (int64_t j = 0; j < Dv; ++j) {
            double acc = 0.0;
            for (int64_t c = 0; c < Dk; ++c) acc += W[r * Dk + c] * S[c * Dv + j];
            Vp[r * Dv + j] = U[r * Dv + j] - acc;
          }
        /* Eq. 9: O = (Gamma.Q) S + Tril(...) V' */
        for (int64_t r = 0; r < Cc; ++r) {
          double* orow = o + IDX3(c0 + r, h, 0, H, Dv);
          for (int64_t j = 0; j < Dv; ++j) {
            double acc = 0.0;
            for (int64_t c = 0; c < Dk; ++c) acc += exp(g[r * Dk + c]) * Qr(r, c) * S[c * Dv + j];
            for (int64_t i = 0; i <= r; ++i) acc += Aqk[r * Cc + i] * Vp[i * Dv + j];
            orow[j] = acc;
          }
        }
        /* Eq. 8: S_next = Diag(gamma_C) S + (Gamma_{i->C}.K)^T V' */
        const double* gC = g + (Cc - 1) * Dk;
        for (int64_t c = 0; c < Dk; ++c)
          for (int64_t j = 0; j < Dv; ++j) {
            double acc = exp(gC[c]) * S[c * Dv + j];
            for (int64_t i = 0; i < Cc; ++i)
              acc += exp(gC[c] - g[i * Dk + c]) * Kr(i, c) * Vp[i * Dv + j];
            Snew[c * Dv + j] = acc;
          }
        memcpy(S, Snew, sizeof(double) * Dk * Dv);
#undef Kr
#undef Qr
#undef Vr
#undef Br
      }
      if (final_state)
        for (int64_t i = 0; i < Dk * Dv; ++i) final_state[nh * Dk * Dv + i] = S[i];
    }
    free(S);
    free(Snew);
    free(g);
    free(A);
    free(Tinv);
    free(M);
    free(W);
    free(U);
    free(Vp);
    free(Aqk);
  }
  return bad;
}

/*
 * Reverse-mode derivative of kda_oracle_recurrent (the backward pass of the operator; the pages
 * motivate it through training: [W] §3.4 "Chunkwise Parallelization" calls the UT transform
 * central to training, and "FLOPs Accounting and Inference Strategy" counts training FLOPs).
 *
 * Given the output cotangent d_o [T_total, H, Dv] and the final-state cotangent d_final
 * [N, H, Dk, Dv] (NULL = 0), returns the gradients of L = <d_o, o> + <d_final, S_T> with respect
 * to q, k (d_q, d_k [T_total, H, Dk]), v (d_v), log_alpha (d_log_alpha), beta (d_beta [T_total,
 * H]) and the initial state (d_initial [N, H, Dk, Dv]; may be NULL). Tokens outside every
 * sequence get zero gradients.
 *
 * The forward step, with S' = Diag(alpha) S_{t-1}, e = S'^T k, u = beta (v - e),
 * S_t = S' + k u^T, o_t = S_t^T q, is walked backwards with the running cotangent dS of S_t:
 *     dS   += q d_o^T              d_q = S_t d_o
 *     du    = dS^T k               d_k = dS u
 *     d_beta = du . (v - e)        d_v = beta du            de = -beta du
 *     dS'   = dS + k de^T          d_k += S' de
 *     d_log_alpha[a] = sum_j dS'[a, j] S'[a, j]             dS_{t-1} = Diag(alpha) dS'
 * The states of each sequence are recomputed forward from checkpoints every `seg` tokens.
 */
int kda_oracle_recurrent_bwd(const double* q, const double* k, const double* v,
                             const double* log_alpha, const double* beta,
                             const double* initial_state, const int64_t* cu_seqlens, int64_t N,
                             int64_t H, int64_t Dk, int64_t Dv, const double* d_o,
                             const double* d_final, double* d_q, double* d_k, double* d_v,
                             double* d_log_alpha, double* d_beta, double* d_initial,
                             int nthreads) {
  if (!q || !k || !v || !log_alpha || !beta || !cu_seqlens || !d_o || !d_q || !d_k || !d_v ||
      !d_log_alpha || !d_beta)
    return 1;
  if (N < 0 || H <= 0 || Dk <= 0 || Dv <= 0) return 1;
  const int64_t T_total = cu_seqlens[N];
  memset(d_q, 0, sizeof(double) * T_total * H * Dk);
  memset(d_k, 0, sizeof(double) * T_total * H * Dk);
  memset(d_log_alpha, 0, sizeof(double) * T_total * H * Dk);
  memset(d_v, 0, sizeof(double) * T_total * H * Dv);
  memset(d_beta, 0, sizeof(double) * T_total * H);
  set_threads(nthreads);
  const int64_t seg = 32;
  const int64_t SS = Dk * Dv;
  int bad = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : bad)
  for (int64_t nh = 0; nh < N * H; ++nh) {
    const int64_t n = nh / H, h = nh % H;
    const int64_t t_begin = cu_seqlens[n], len = cu_seqlens[n + 1] - cu_seqlens[n];
    const int64_t nseg = (len + seg - 1) / seg;
    /* checkpoints: state before each segment; states: S_{t0 - 1}, ..., S_{t0 + seg - 1} */
    double* ckpt = (double*)malloc(sizeof(double) * SS * (nseg + 1));
    double* S = (double*)malloc(sizeof(double) * SS);
    double* states = (double*)malloc(sizeof(double) * SS * (seg + 1));
    double* dS = (double*)malloc(sizeof(double) * SS);
    double* Sp = (double*)malloc(sizeof(double) * SS);
    double* e = (double*)malloc(sizeof(double) * Dv);
    double* u = (double*)malloc(sizeof(double) * Dv);
    double* du = (double*)malloc(sizeof(double) * Dv);
    double* de = (double*)malloc(sizeof(double) * Dv);
    if (!ckpt || !S || !states || !dS || !Sp || !e || !u || !du || !de) {
      bad |= 1;
      free(ckpt); free(S); free(states); free(dS); free(Sp); free(e); free(u); free(du); free(de);
      continue;
    }
    /* forward pass over the sequence, keeping the state before every segment */
    for (int64_t x = 0; x < SS; ++x) S[x] = initial_state ? initial_state[nh * SS + x] : 0.0;
    for (int64_t t = 0; t < len; ++t) {
      if (t % seg == 0) memcpy(ckpt + (t / seg) * SS, S, sizeof(double) * SS);
      const int64_t tt = t_begin + t;
      for (int64_t a = 0; a < Dk; ++a) {
        const double al = exp(log_alpha[IDX3(tt, h, a, H, Dk)]);
        for (int64_t j = 0; j < Dv; ++j) S[a * Dv + j] *= al;
      }
      for (int64_t j = 0; j < Dv; ++j) {
        double acc = 0.0;
        for (int64_t a = 0; a < Dk; ++a) acc += S[a * Dv + j] * k[IDX3(tt, h, a, H, Dk)];
        u[j] = beta[tt * H + h] * (v[IDX3(tt, h, j, H, Dv)] - acc);
      }
      for (int64_t a = 0; a < Dk; ++a)
        for (int64_t j = 0; j < Dv; ++j) S[a * Dv + j] += k[IDX3(tt, h, a, H, Dk)] * u[j];
    }
    for (int64_t x = 0; x < SS; ++x) dS[x] = d_final ? d_final[nh * SS + x] : 0.0;
    for (int64_t sg = nseg - 1; sg >= 0; --sg) {
      const int64_t s0 = sg * seg, s1 = (s0 + seg < len) ? s0 + seg : len;
      /* recompute S_{s0-1} .. S_{s1-1} into states[0 .. s1-s0] */
      memcpy(states, ckpt + sg * SS, sizeof(double) * SS);
      for (int64_t t = s0; t < s1; ++t) {
        const int64_t tt = t_begin + t;
        const double* P = states + (t - s0) * SS;
        double* Q = states + (t - s0 + 1) * SS;
        for (int64_t a = 0; a < Dk; ++a) {
          const double al = exp(log_alpha[IDX3(tt, h, a, H, Dk)]);
          for (int64_t j = 0; j < Dv; ++j) Q[a * Dv + j] = al * P[a * Dv + j];
        }
        for (int64_t j = 0; j < Dv; ++j) {
          double acc = 0.0;
          for (int64_t a = 0; a < Dk; ++a) acc += Q[a * Dv + j] * k[IDX3(tt, h, a, H, Dk)];
          u[j] = beta[tt * H + h] * (v[IDX3(tt, h, j, H, Dv)] - acc);
        }
        for (int64_t a = 0; a < Dk; ++a)
          for (int64_t j = 0; j < Dv; ++j) Q[a * Dv + j] += k[IDX3(tt, h, a, H, Dk)] * u[j];
      }
      /* reverse steps */
      for (int64_t t = s1 - 1; t >= s0; --t) {
        const int64_t tt = t_begin + t;
        const double* Sprev = states + (t - s0) * SS;
        const double* Scur = states + (t - s0 + 1) * SS;
        const double b = beta[tt * H + h];
        for (int64_t a = 0; a < Dk; ++a) {
          const double al = exp(log_alpha[IDX3(tt, h, a, H, Dk)]);
          for (int64_t j = 0; j < Dv; ++j) Sp[a * Dv + j] = al * Sprev[a * Dv + j];
        }
        for (int64_t j = 0; j < Dv; ++j) {
          double acc = 0.0;
          for (int64_t a = 0; a < Dk; ++a) acc += Sp[a * Dv + j] * k[IDX3(tt, h, a, H, Dk)];
          e[j] = acc;
          u[j] = b * (v[IDX3(tt, h, j, H, Dv)] - acc);
        }
        /* o_t = S_t^T q_t */
        for (int64_t a = 0; a < Dk; ++a) {
          double acc = 0.0;
          for (int64_t j = 0; j < Dv; ++j) {
            dS[a * Dv + j] += q[IDX3(tt, h, a, H, Dk)] * d_o[IDX3(tt, h, j, H, Dv)];
            acc += Scur[a * Dv + j] * d_o[IDX3(tt, h, j, H, Dv)];
          }
          d_q[IDX3(tt, h, a, H, Dk)] = acc;
        }
        /* S_t = S' + k u^T */
        for (int64_t j = 0; j < Dv; ++j) {
          double acc = 0.0;
          for (int64_t a = 0; a < Dk; ++a) acc += dS[a * Dv + j] * k[IDX3(tt, h, a, H, Dk)];
          du[j] = acc;
        }
        double db = 0.0;
        for (int64_t j = 0; j < Dv; ++j) {
          db += du[j] * (v[IDX3(tt, h, j, H, Dv)] - e[j]);
          d_v[IDX3(tt, h, j, H, Dv)] = b * du[j];
          de[j] = -b * du[j];
        }
        d_beta[tt * H + h] = db;
        for (int64_t a = 0; a < Dk; ++a) {
          double acc = 0.0;
          for (int64_t j = 0; j < Dv; ++j) acc += dS[a * Dv + j] * u[j] + Sp[a * Dv + j] * de[j];
          d_k[IDX3(tt, h, a, H, Dk)] = acc;
        }
        /* e = S'^T k: dS' = dS + k de^T; S' = Diag(alpha) S_{t-1} */
        for (int64_t a = 0; a < Dk; ++a) {
          const double ka = k[IDX3(tt, h, a, H, Dk)];
          const double al = exp(log_alpha[IDX3(tt, h, a, H, Dk)]);
          double acc = 0.0;
          for (int64_t j = 0; j < Dv; ++j) {
            const double dsp = dS[a * Dv + j] + ka * de[j];
            acc += dsp * Sp[a * Dv + j];
            dS[a * Dv + j] = al * dsp;
          }
          d_log_alpha[IDX3(tt, h, a, H, Dk)] = acc;
        }
      }
    }
    if (d_initial) memcpy(d_initial + nh * SS, dS, sizeof(double) * SS);
    free(ckpt); free(S); free(states); free(dS); free(Sp); free(e); free(u); free(du); free(de);
  }
  return bad ? 1 : 0;
}
