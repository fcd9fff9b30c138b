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

/*
 * Backward of the error-form recurrence (the adjoint of run_pair), for one
 * (sequence, value head) pair.  The forward result is differentiated by
 * hand, step by step in reverse token order; for each token, with S' =
 * alpha S_{t-1}, e = v - S'^T k, S_t = S' + beta k e^T, o = scale S_t^T q:
 *
 *     dS     += scale q do^T             dq   = scale S_t do
 *     de      = beta dS^T k              dv   = de
 *     dbeta   = k^T dS e                 dk   = beta dS e - S' de
 *     dS'     = dS - k de^T              dlog alpha = <dS', S'>
 *     dS_{t-1} = alpha dS'
 *
 * where dS is the gradient with respect to S_t.  With the epilogue
 * y = n (1 + w) sigmoid(g), n = o / sqrt(mean o^2 + eps_norm), the gradient
 * do comes from dy by the chain rule through the gate and the RMS norm.  The
 * L2 norm of q and k is differentiated afterwards (by the caller), once the
 * gradients of the value heads sharing a QK head are summed.
 *
 * States are recomputed from checkpoints taken every kCk tokens of the
 * forward pass; the recomputation repeats the forward arithmetic exactly.
 * dqh/dkh receive the gradients with respect to the normalised q and k of
 * this value head, [total_T, H_v, d_k]; dw (may be NULL) receives this
 * pair's share of the norm-weight gradient, [d_v].
 */
enum { kCk = 64 };

static void l2_unit(const float* x, int n, int l2norm, double eps, double* xh) {
  double s = 0.0;
  for (int i = 0; i < n; ++i) {
    xh[i] = (double)x[i];
    s += xh[i] * xh[i];
  }
  if (l2norm) {
    const double r = 1.0 / sqrt(s + eps);
    for (int i = 0; i < n; ++i) xh[i] *= r;
  }
}

static void step_state(const double* Sp, const double* kh, const float* vt,
                       double alpha, double b, int dk, int dv, double* Sn,
                       double* e) {
  /* Sn = S' + b k e^T with S' = alpha Sp and e = v - S'^T k */
  for (int i = 0; i < dk * dv; ++i) Sn[i] = alpha * Sp[i];
  for (int j = 0; j < dv; ++j) e[j] = (double)vt[j];
  for (int i = 0; i < dk; ++i)
    for (int j = 0; j < dv; ++j) e[j] -= Sn[(size_t)i * dv + j] * kh[i];
  for (int i = 0; i < dk; ++i)
    for (int j = 0; j < dv; ++j) Sn[(size_t)i * dv + j] += b * kh[i] * e[j];
}

static int backward_pair(const float* q, const float* k, const float* v,
                         const float* log_alpha, const float* beta,
                         const float* g, const float* norm_w, const float* s0,
                         const float* dy, const float* dsT, int64_t t0,
                         int64_t t1, int h, int Hqk, int Hv, int dk, int dv,
                         int l2norm, double eps_l2, double eps_norm,
                         double scale, double* dqh, double* dkh, double* dv_out,
                         double* dla, double* dbeta, double* dg, double* dw,
                         double* ds0) {
  const int group = Hv / Hqk;
  const int hq = h / group;
  const size_t SS = (size_t)dk * dv;
  const int64_t T = t1 - t0;
  const int64_t nck = (T + kCk - 1) / kCk;
  double* ck = (double*)malloc(sizeof(double) * SS * (size_t)(nck > 0 ? nck : 1));
  double* St = (double*)malloc(sizeof(double) * SS * (kCk + 1));
  double* dS = (double*)malloc(sizeof(double) * SS);
  double* Sp = (double*)malloc(sizeof(double) * SS);
  double* kh = (double*)malloc(sizeof(double) * dk);
  double* qh = (double*)malloc(sizeof(double) * dk);
  double* e = (double*)malloc(sizeof(double) * dv);
  double* o = (double*)malloc(sizeof(double) * dv);
  double* dO = (double*)malloc(sizeof(double) * dv);
  double* de = (double*)malloc(sizeof(double) * dv);
  double* tmp = (double*)malloc(sizeof(double) * (dk > dv ? dk : dv));
  int ok = ck && St && dS && Sp && kh && qh && e && o && dO && de && tmp;
  if (ok) {
    /* forward pass: the state entering every kCk-token block */
    double* S = St;
    if (s0) {
      for (size_t i = 0; i < SS; ++i) S[i] = (double)s0[i];
    } else {
      memset(S, 0, sizeof(double) * SS);
    }
    for (int64_t t = t0; t < t1; ++t) {
      if ((t - t0) % kCk == 0) memcpy(ck + SS * (size_t)((t - t0) / kCk), S, sizeof(double) * SS);
      l2_unit(k + ((size_t)t * Hqk + hq) * dk, dk, l2norm, eps_l2, kh);
      const double alpha = exp((double)log_alpha[(size_t)t * Hv + h]);
      const double b = (double)beta[(size_t)t * Hv + h];
      step_state(S, kh, v + ((size_t)t * Hv + h) * dv, alpha, b, dk, dv, Sp, e);
      memcpy(S, Sp, sizeof(double) * SS);
    }
    /* reverse pass, one block at a time */
    if (dsT) {
      for (size_t i = 0; i < SS; ++i) dS[i] = (double)dsT[i];
    } else {
      memset(dS, 0, sizeof(double) * SS);
    }
    for (int64_t blk = nck - 1; blk >= 0; --blk) {
      const int64_t b0 = t0 + blk * kCk;
      const int64_t b1 = (b0 + kCk < t1) ? b0 + kCk : t1;
      /* St[m] = state entering token b0 + m; St[b1 - b0] = state after the block */
      memcpy(St, ck + SS * (size_t)blk, sizeof(double) * SS);
      for (int64_t t = b0; t < b1; ++t) {
        l2_unit(k + ((size_t)t * Hqk + hq) * dk, dk, l2norm, eps_l2, kh);
        const double alpha = exp((double)log_alpha[(size_t)t * Hv + h]);
        const double b = (double)beta[(size_t)t * Hv + h];
        step_state(St + SS * (size_t)(t - b0), kh, v + ((size_t)t * Hv + h) * dv, alpha, b,
                   dk, dv, St + SS * (size_t)(t - b0 + 1), e);
      }
      for (int64_t t = b1 - 1; t >= b0; --t) {
        const double* Sprev = St + SS * (size_t)(t - b0);
        const double* Snew = St + SS * (size_t)(t - b0 + 1);
        l2_unit(k + ((size_t)t * Hqk + hq) * dk, dk, l2norm, eps_l2, kh);
        l2_unit(q + ((size_t)t * Hqk + hq) * dk, dk, l2norm, eps_l2, qh);
        const double alpha = exp((double)log_alpha[(size_t)t * Hv + h]);
        const double b = (double)beta[(size_t)t * Hv + h];
        const size_t row = (size_t)t * Hv + h;
        /* S' and e of this token */
        for (size_t i = 0; i < SS; ++i) Sp[i] = alpha * Sprev[i];
        for (int j = 0; j < dv; ++j) e[j] = (double)v[row * dv + j];
        for (int i = 0; i < dk; ++i)
          for (int j = 0; j < dv; ++j) e[j] -= Sp[(size_t)i * dv + j] * kh[i];
        /* o = scale S_t^T q, then do from dy */
        for (int j = 0; j < dv; ++j) {
          double acc = 0.0;
          for (int i = 0; i < dk; ++i) acc += Snew[(size_t)i * dv + j] * qh[i];
          o[j] = scale * acc;
        }
        const float* dyt = dy + row * dv;
        if (g) {
          const float* gt = g + row * dv;
          double ms = 0.0;
          for (int j = 0; j < dv; ++j) ms += o[j] * o[j];
          const double r = 1.0 / sqrt(ms / (double)dv + eps_norm);
          double dot = 0.0;
          for (int j = 0; j < dv; ++j) {
            const double w = norm_w ? (double)norm_w[j] : 0.0;
            const double sg = 1.0 / (1.0 + exp(-(double)gt[j]));
            const double n = o[j] * r;
            const double dyj = (double)dyt[j];
            dg[row * dv + j] = dyj * n * (1.0 + w) * sg * (1.0 - sg);
            if (dw) dw[j] += dyj * n * sg;
            dO[j] = dyj * (1.0 + w) * sg; /* gradient w.r.t. n */
            dot += dO[j] * n;
          }
          dot /= (double)dv;
          for (int j = 0; j < dv; ++j) dO[j] = r * (dO[j] - o[j] * r * dot);
        } else {
          for (int j = 0; j < dv; ++j) dO[j] = (double)dyt[j];
        }
        /* read-out: dq = scale S_t do, dS += scale q do^T */
        for (int i = 0; i < dk; ++i) {
          double acc = 0.0;
          for (int j = 0; j < dv; ++j) acc += Snew[(size_t)i * dv + j] * dO[j];
          dqh[row * dk + i] = scale * acc;
        }
        for (int i = 0; i < dk; ++i)
          for (int j = 0; j < dv; ++j) dS[(size_t)i * dv + j] += scale * qh[i] * dO[j];
        /* write: de = beta dS^T k, dbeta = k^T dS e, dk = beta dS e - S' de */
        for (int j = 0; j < dv; ++j) {
          double acc = 0.0;
          for (int i = 0; i < dk; ++i) acc += dS[(size_t)i * dv + j] * kh[i];
          de[j] = b * acc;
          dv_out[row * dv + j] = de[j];
        }
        double db = 0.0;
        for (int i = 0; i < dk; ++i) {
          double dse = 0.0, spde = 0.0;
          for (int j = 0; j < dv; ++j) {
            dse += dS[(size_t)i * dv + j] * e[j];
            spde += Sp[(size_t)i * dv + j] * de[j];
          }
          db += kh[i] * dse;
          tmp[i] = b * dse - spde;
        }
        dbeta[row] = db;
        for (int i = 0; i < dk; ++i) dkh[row * dk + i] = tmp[i];
        /* dS' = dS - k de^T; dlog alpha = <dS', S'>; dS_{t-1} = alpha dS' */
        double dl = 0.0;
        for (int i = 0; i < dk; ++i)
          for (int j = 0; j < dv; ++j) {
            const size_t x = (size_t)i * dv + j;
            dS[x] -= kh[i] * de[j];
            dl += dS[x] * Sp[x];
            dS[x] *= alpha;
          }
        dla[row] = dl;
      }
    }
    memcpy(ds0, dS, sizeof(double) * SS);
  }
  free(ck);
  free(St);
  free(dS);
  free(Sp);
  free(kh);
  free(qh);
  free(e);
  free(o);
  free(dO);
  free(de);
  free(tmp);
  return ok ? 0 : -1;
}

/*
 * Backward over a packed batch.  Inputs as gdn_oracle_recurrence plus
 * dy [total_T, H_v, d_v] (the gradient of the loss with respect to y, after
 * the epilogue when g is given) and d_final_state [n_seq, H_v, d_k, d_v] (may
 * be NULL = zeros).  Outputs, all fp64 and written in full:
 *   dq, dk          [total_T, H_qk, d_k]  (through the L2 norm when l2norm)
 *   dv              [total_T, H_v, d_v]
 *   dlog_alpha, dbeta [total_T, H_v]
 *   dg              [total_T, H_v, d_v]  (only when g is given; may be NULL)
 *   dnorm_w         [d_v]                (only when g is given; may be NULL)
 *   d_initial_state [n_seq, H_v, d_k, d_v]
 * Returns 0 on success, -1 on a bad argument or an allocation failure.
 */
int gdn_oracle_backward(const float* q, const float* k, const float* v,
                        const float* log_alpha, const float* beta,
                        const float* g, const float* norm_w,
                        const float* initial_state, const int64_t* cu_seqlens,
                        int64_t n_seq, int64_t total_T, int Hqk, int Hv,
                        int dk, int dv, int l2norm, double eps_l2,
                        double eps_norm, double scale, const float* dy,
                        const float* d_final_state, double* dq, double* dk_out,
                        double* dv_out, double* dlog_alpha, double* dbeta,
                        double* dg, double* dnorm_w, double* d_initial_state,
                        int n_threads) {
  if (!q || !k || !v || !log_alpha || !beta || !dy || !cu_seqlens) return -1;
  if (!dq || !dk_out || !dv_out || !dlog_alpha || !dbeta || !d_initial_state) return -1;
  if (g && !dg) return -1;
  if (Hqk <= 0 || Hv <= 0 || Hv % Hqk != 0 || dk <= 0 || dv <= 0) return -1;
  if (n_seq < 0 || cu_seqlens[0] != 0 || cu_seqlens[n_seq] != total_T) return -1;
  for (int64_t s = 0; s < n_seq; ++s)
    if (cu_seqlens[s + 1] < cu_seqlens[s]) return -1;
  const int64_t pairs = n_seq * (int64_t)Hv;
  const size_t nq = (size_t)total_T * Hv * dk;
  double* dqh = (double*)calloc(nq ? nq : 1, sizeof(double));
  double* dkh = (double*)calloc(nq ? nq : 1, sizeof(double));
  double* dwp = (double*)calloc((size_t)(pairs ? pairs : 1) * dv, sizeof(double));
  if (!dqh || !dkh || !dwp) {
    free(dqh);
    free(dkh);
    free(dwp);
    return -1;
  }
#ifdef _OPENMP
  if (n_threads > 0) omp_set_num_threads(n_threads);
#else
  (void)n_threads;
#endif
  int bad = 0;
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t p = 0; p < pairs; ++p) {
    const int64_t s = p / Hv;
    const int h = (int)(p % Hv);
    const size_t st = ((size_t)s * Hv + h) * (size_t)dk * dv;
    if (backward_pair(q, k, v, log_alpha, beta, g, norm_w,
                      initial_state ? initial_state + st : NULL, dy,
                      d_final_state ? d_final_state + st : NULL, cu_seqlens[s],
                      cu_seqlens[s + 1], h, Hqk, Hv, dk, dv, l2norm, eps_l2,
                      eps_norm, scale, dqh, dkh, dv_out, dlog_alpha, dbeta, dg,
                      g ? dwp + (size_t)p * dv : NULL, d_initial_state + st) != 0) {
#pragma omp atomic write
      bad = 1;
    }
  }
  if (!bad) {
    /* sum the value heads of each QK group, then differentiate the L2 norm:
       for x^ = x r, r = 1/sqrt(|x|^2 + eps): dx = r (dx^ - x^ (x^ . dx^)) */
    const int group = Hv / Hqk;
    double* xh = (double*)malloc(sizeof(double) * dk);
    double* gq = (double*)malloc(sizeof(double) * dk);
    if (!xh || !gq) bad = 1;
    for (int64_t t = 0; t < total_T && !bad; ++t)
      for (int hq = 0; hq < Hqk; ++hq)
        for (int which = 0; which < 2; ++which) {
          const float* x = (which ? k : q) + ((size_t)t * Hqk + hq) * dk;
          const double* part = which ? dkh : dqh;
          double* out = (which ? dk_out : dq) + ((size_t)t * Hqk + hq) * dk;
          for (int i = 0; i < dk; ++i) gq[i] = 0.0;
          for (int m = 0; m < group; ++m) {
            const double* pr = part + ((size_t)t * Hv + (size_t)hq * group + m) * dk;
            for (int i = 0; i < dk; ++i) gq[i] += pr[i];
          }
          if (l2norm) {
            double ss = 0.0;
            for (int i = 0; i < dk; ++i) ss += (double)x[i] * (double)x[i];
            const double r = 1.0 / sqrt(ss + eps_l2);
            double dot = 0.0;
            for (int i = 0; i < dk; ++i) {
              xh[i] = (double)x[i] * r;
              dot += xh[i] * gq[i];
            }
            for (int i = 0; i < dk; ++i) out[i] = r * (gq[i] - xh[i] * dot);
          } else {
            for (int i = 0; i < dk; ++i) out[i] = gq[i];
          }
        }
    free(xh);
    free(gq);
    if (g && dnorm_w) {
      for (int j = 0; j < dv; ++j) dnorm_w[j] = 0.0;
      for (int64_t p = 0; p < pairs; ++p)
        for (int j = 0; j < dv; ++j) dnorm_w[j] += dwp[(size_t)p * dv + j];
    }
  }
  free(dqh);
  free(dkh);
  free(dwp);
  return bad ? -1 : 0;
}

/*
 * Front end of the mixer: short depthwise causal convolution of kernel 4
 * over time, then SiLU ("Qwen3.8-Flash-Next: architecture, efficiency and
 * technical lineage", section 02 module table, GDN row: Q/K/V pass a short
 * causal conv of kernel 4; hyper.ai summary, "Method": projections followed
 * by short depthwise causal convolutions; "On the Design of Qwen3.8-Next
 * Architecture ... close reading", section 4.1: short conv + SiLU + L2 norm).
 *
 * x [total_T, C] (C channels of one token side by side), w [C, 4] with w[c][3]
 * the weight of the current token and w[c][3 - j] that of the token j steps
 * back; no bias.  For each sequence s and channel c:
 *     u_t = sum_{j=0..3} w[c][3 - j] * x_{t - j}
 * where x_{t - j} before the sequence's first token comes from state_in[s]
 * ([3, C]; row m holds the input m - 3 tokens before the start, row 2 the
 * last one) or is 0 when state_in is NULL.  y_t = silu ? u_t / (1 + e^-u_t)
 * : u_t.  state_out[s] (may be NULL) receives the three inputs the next
 * segment of the sequence would need: rows 0..2 = the inputs 3, 2, 1 tokens
 * before the end (taken from state_in, or 0, for short sequences).
 * Returns 0, or -1 on a bad argument.
 */
int gdn_oracle_conv(const float* x, int64_t total_T, int C, const float* w,
                    const float* state_in, const int64_t* cu_seqlens,
                    int64_t n_seq, int silu, double* y, double* state_out) {
  if (!x && total_T > 0) return -1;
  if (!w || !y || !cu_seqlens || C <= 0 || n_seq < 0) return -1;
  if (cu_seqlens[0] != 0 || cu_seqlens[n_seq] != total_T) return -1;
  for (int64_t s = 0; s < n_seq; ++s)
    if (cu_seqlens[s + 1] < cu_seqlens[s]) return -1;
  for (int64_t s = 0; s < n_seq; ++s) {
    const int64_t t0 = cu_seqlens[s], t1 = cu_seqlens[s + 1];
    const float* st = state_in ? state_in + (size_t)s * 3 * C : NULL;
    for (int c = 0; c < C; ++c) {
      /* the input `back` tokens before token t of this sequence */
#define XIN(t, back)                                                        \
  (((t) - (back) >= t0) ? (double)x[(size_t)((t) - (back)) * C + c]         \
   : (st ? (double)st[(size_t)(3 - ((back) - ((t) - t0))) * C + c] : 0.0))
      for (int64_t t = t0; t < t1; ++t) {
        double u = 0.0;
        for (int j = 0; j < 4; ++j) u += (double)w[(size_t)c * 4 + 3 - j] * XIN(t, j);
        y[(size_t)t * C + c] = silu ? u / (1.0 + exp(-u)) : u;
      }
      if (state_out) {
        for (int m = 0; m < 3; ++m)
          state_out[((size_t)s * 3 + m) * C + c] = XIN(t1, 3 - m);
      }
#undef XIN
    }
  }
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
