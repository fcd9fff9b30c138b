/*
 * Gated delta rule: slow, obviously correct fp64 CPU oracle.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path links, loads or
 * calls this file; only the tests, the smoke check and the CPU-baseline leg
 * of the benchmark do.  It shares no code, header or constant with the CUDA
 * library.
 *
 * What it computes (per sequence, per value head, token by token, no
 * chunking, no reordering):
 *
 *   - "Qwen3.8-Flash-Next: architecture, efficiency and technical lineage"
 *     (technical-report-notes analysis page), section 03 "Gated DeltaNet",
 *     the four update equations:
 *         S~    = alpha_t * S_{t-1}
 *         e_t   = v_t - S~^T k_t
 *         S_t   = S~ + beta_t * k_t e_t^T
 *         y_t   = S_t^T q_t
 *     with alpha, beta in (0,1) (the "Decay alpha" / "Write beta" boxes).
 *   - "On the Design of Qwen3.8-Next Architecture ... (close reading)",
 *     section 4.1 "token mixing": the product form
 *         S_t = alpha_t (I - beta_t k_t k_t^T) S_{t-1} + beta_t k_t v_t^T,
 *     and q/k L2-normalised before the rule.  Evaluated separately by
 *     gdn_oracle_product_form (used only to pin the error form).
 *   - same analysis page, section 03, "what Qwen changed on the original
 *     GDN": zero-centred RMSNorm, then a sigmoid output gate; the paper
 *     summary page (hyper.ai, "Method") fixes the order: head outputs are
 *     normalised, then modulated by the gate.
 *
 * Readings where the pages are silent (each is listed in the design notes):
 *   alpha enters as log(alpha) (fp32, <= 0) and alpha = exp(log alpha);
 *   alpha and beta are one scalar per token per value head;
 *   y_t reads the updated state S_t (inclusive of token t);
 *   scale multiplies y (default 1; the pages write none);
 *   L2 norm: x / sqrt(sum x^2 + eps_l2);
 *   value head h reads QK head h / (H_v / H_qk) (contiguous groups);
 *   epilogue: y / sqrt(mean_j y_j^2 + eps_norm) * (1 + w_j) * sigmoid(g_j),
 *   mean over d_v, w of shape [d_v] shared by all heads;
 *   every sequence of a packed batch starts from its own initial state.
 *
 * Inputs are fp32 arrays (bf16 values are exactly representable in fp32);
 * all arithmetic is fp64.  Layouts are dense row-major:
 *   q, k        [total_T, H_qk, d_k]
 *   v, g, y     [total_T, H_v, d_v]
 *   log_alpha, beta [total_T, H_v]
 *   norm_w      [d_v]
 *   states      [n_seq, H_v, d_k, d_v]   (S[i][j], i over d_k, j over d_v)
 *   cu_seqlens  [n_seq + 1], cu[0] = 0, non-decreasing, cu[n_seq] = total_T
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* One (sequence, value head) pair through the error-form recurrence. */
static void run_pair(const float* q, const float* k, const float* v,
                     const float* log_alpha, const float* beta,
                     const float* g, const float* norm_w,
                     const float* s0, int64_t t0, int64_t t1, int h, int Hqk,
                     int Hv, int dk, int dv, int l2norm, double eps_l2,
                     double eps_norm, double scale, double* y, double* s_out,
                     double* S, double* kh, double* qh, double* e,
                     double* yt) {
  const int group = Hv / Hqk;
  const int hq = h / group;
  if (s0) {
    for (int i = 0; i < dk * dv; ++i) S[i] = (double)s0[i];
  } else {
    memset(S, 0, sizeof(double) * (size_t)dk * dv);
  }
  for (int64_t t = t0; t < t1; ++t) {
    const float* kt = k + ((size_t)t * Hqk + hq) * dk;
    const float* qt = q + ((size_t)t * Hqk + hq) * dk;
    const float* vt = v + ((size_t)t * Hv + h) * dv;
    double nk = 0.0, nq = 0.0;
    for (int i = 0; i < dk; ++i) {
      kh[i] = (double)kt[i];
      qh[i] = (double)qt[i];
      nk += kh[i] * kh[i];
      nq += qh[i] * qh[i];
    }
    if (l2norm) {
      const double rk = 1.0 / sqrt(nk + eps_l2);
      const double rq = 1.0 / sqrt(nq + eps_l2);
      for (int i = 0; i < dk; ++i) {
        kh[i] *= rk;
        qh[i] *= rq;
      }
    }
    const double alpha = exp((double)log_alpha[(size_t)t * Hv + h]);
    const double b = (double)beta[(size_t)t * Hv + h];
    /* S~ = alpha * S */
    for (int i = 0; i < dk * dv; ++i) S[i] *= alpha;
    /* e = v - S~^T k */
    for (int j = 0; j < dv; ++j) e[j] = (double)vt[j];
    for (int i = 0; i < dk; ++i) {
      const double ki = kh[i];
      const double* Si = S + (size_t)i * dv;
      for (int j = 0; j < dv; ++j) e[j] -= Si[j] * ki;
    }
    /* S = S~ + beta k e^T */
    for (int i = 0; i < dk; ++i) {
      const double bk = b * kh[i];
      double* Si = S + (size_t)i * dv;
      for (int j = 0; j < dv; ++j) Si[j] += bk * e[j];
    }
    /* y = scale * S^T q */
    for (int j = 0; j < dv; ++j) yt[j] = 0.0;
    for (int i = 0; i < dk; ++i) {
      const double qi = qh[i];
      const double* Si = S + (size_t)i * dv;
      for (int j = 0; j < dv; ++j) yt[j] += Si[j] * qi;
    }
    for (int j = 0; j < dv; ++j) yt[j] *= scale;
    double* yo = y + ((size_t)t * Hv + h) * dv;
    if (g) {
      /* normalise the head output, then gate it */
      const float* gt = g + ((size_t)t * Hv + h) * dv;
      double ms = 0.0;
      for (int j = 0; j < dv; ++j) ms += yt[j] * yt[j];
      ms /= (double)dv;
      const double r = 1.0 / sqrt(ms + eps_norm);
      for (int j = 0; j < dv; ++j) {
        const double w = norm_w ? (double)norm_w[j] : 0.0;
        const double sg = 1.0 / (1.0 + exp(-(double)gt[j]));
        yo[j] = yt[j] * r * (1.0 + w) * sg;
      }
    } else {
      for (int j = 0; j < dv; ++j) yo[j] = yt[j];
    }
  }
  if (s_out) memcpy(s_out, S, sizeof(double) * (size_t)dk * dv);
}

/*
 * Error-form recurrence over a packed batch.  Returns 0 on success, -1 on a
 * bad argument.  n_threads <= 0 means "OpenMP default".  y must hold
 * [total_T, H_v, d_v] doubles; final_state (may be NULL) [n_seq, H_v, d_k, d_v].
 */
int gdn_oracle_recurrence(const float* q, const float* k, const float* v,
                          const float* log_alpha, const float* beta,
                          const float* g, const float* norm_w,
                          const float* initial_state,
                          const int64_t* cu_seqlens, int64_t n_seq,
                          int64_t total_T, int Hqk, int Hv, int dk, int dv,
                          int l2norm, double eps_l2, double eps_norm,
                          double scale, double* y, double* final_state,
                          int n_threads) {
  if (!q || !k || !v || !log_alpha || !beta || !y || !cu_seqlens) return -1;
  if (Hqk <= 0 || Hv <= 0 || Hv % Hqk != 0 || dk <= 0 || dv <= 0) return -1;
  if (n_seq < 0 || cu_seqlens[0] != 0 || cu_seqlens[n_seq] != total_T) return -1;
  for (int64_t s = 0; s < n_seq; ++s)
    if (cu_seqlens[s + 1] < cu_seqlens[s]) return -1;
  const int64_t pairs = n_seq * (int64_t)Hv;
#ifdef _OPENMP
  if (n_threads > 0) omp_set_num_threads(n_threads);
#else
  (void)n_threads;
#endif
  int bad = 0;
#pragma omp parallel
  {
    double* S = (double*)malloc(sizeof(double) * (size_t)dk * dv);
    double* kh = (double*)malloc(sizeof(double) * (size_t)dk);
    double* qh = (double*)malloc(sizeof(double) * (size_t)dk);
    double* e = (double*)malloc(sizeof(double) * (size_t)dv);
    double* yt = (double*)malloc(sizeof(double) * (size_t)dv);
    if (!S || !kh || !qh || !e || !yt) {
#pragma omp atomic write
      bad = 1;
    } else {
#pragma omp for schedule(dynamic, 1)
      for (int64_t p = 0; p < pairs; ++p) {
        const int64_t s = p / Hv;
        const int h = (int)(p % Hv);
        const size_t st = ((size_t)s * Hv + h) * (size_t)dk * dv;
        run_pair(q, k, v, log_alpha, beta, g, norm_w,
                 initial_state ? initial_state + st : NULL, cu_seqlens[s],
                 cu_seqlens[s + 1], h, Hqk, Hv, dk, dv, l2norm, eps_l2,
                 eps_norm, scale, y, final_state ? final_state + st : NULL, S,
                 kh, qh, e, yt);
      }
    }
    free(S);
    free(kh);
    free(qh);
    free(e);
    free(yt);
  }
  return bad ? -1 : 0;
}

/*
 * Product form S_t = alpha_t (I - beta_t k k^T) S_{t-1} + beta_t k v^T for one
 * sequence and one head (H_qk = H_v = 1), inputs already in fp64 and k, q
 * used as given (no normalisation).  Forms the d_k x d_k transition matrix
 * explicitly each step.  y[t] = S_t^T q_t.  Used to pin the error form.
 */
int gdn_oracle_product_form(const double* q, const double* k, const double* v,
                            const double* alpha, const double* beta,
                            const double* s0, int64_t T, int dk, int dv,
                            double* y, double* s_out) {
  if (!q || !k || !v || !alpha || !beta || !y || dk <= 0 || dv <= 0) return -1;
  double* S = (double*)calloc((size_t)dk * dv, sizeof(double));
  double* Sn = (double*)calloc((size_t)dk * dv, sizeof(double));
  double* M = (double*)calloc((size_t)dk * dk, sizeof(double));
  if (!S || !Sn || !M) {
    free(S);
    free(Sn);
    free(M);
    return -1;
  }
  if (s0) memcpy(S, s0, sizeof(double) * (size_t)dk * dv);
  for (int64_t t = 0; t < T; ++t) {
    const double* kt = k + (size_t)t * dk;
    const double* qt = q + (size_t)t * dk;
    const double* vt = v + (size_t)t * dv;
    const double a = alpha[t], b = beta[t];
    for (int i = 0; i < dk; ++i)
      for (int l = 0; l < dk; ++l)
        M[(size_t)i * dk + l] = a * ((i == l ? 1.0 : 0.0) - b * kt[i] * kt[l]);
    for (int i = 0; i < dk; ++i)
      for (int j = 0; j < dv; ++j) {
        double acc = b * kt[i] * vt[j];
        for (int l = 0; l < dk; ++l) acc += M[(size_t)i * dk + l] * S[(size_t)l * dv + j];
        Sn[(size_t)i * dv + j] = acc;
      }
    memcpy(S, Sn, sizeof(double) * (size_t)dk * dv);
    for (int j = 0; j < dv; ++j) {
      double acc = 0.0;
      for (int i = 0; i < dk; ++i) acc += S[(size_t)i * dv + j] * qt[i];
      y[(size_t)t * dv + j] = acc;
    }
  }
  if (s_out) memcpy(s_out, S, sizeof(double) * (size_t)dk * dv);
  free(S);
  free(Sn);
  free(M);
  return 0;
}

/* Number of threads an OpenMP parallel region would use. */
int gdn_oracle_max_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}
