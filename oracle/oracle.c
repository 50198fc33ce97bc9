/*
 * oracle.c -- plain, slow fp64 CPU oracle for masked softmax attention,
 * forward and backward.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may link, load or
 * call this file: only the test suite, the smoke check and the CPU-baseline
 * leg of the benchmark use it.  It shares no code with the CUDA library.
 *
 * What it computes (per batch b, head h, query row i, key j):
 *
 *   s_ij = scale * sum_d Q_id K_jd + bias_h(i, j) + A[b,h,i,j]
 *          -- "FlashAttentionScore fusion operator replacement guide", sec. 2
 *             (the attention formula) and sec. 4 step 1 (matmul * scale,
 *             then the additive mask, softmax, matmul with V).
 *   bias_h(i, j) = -slope_h * |i - j|   (ALiBi position bias, the optional
 *             `pse` input of sec. 3.2 of the same guide), or 0 without pse.
 *   A[b,h,i,j] = a dense additive term (the general `pse` tensor of sec. 3.2,
 *             or a float `atten_mask` added to the scores as in sec. 4 step
 *             1), broadcast over b and h by zero strides, or 0 without one.
 *             Its values are finite or -inf; an s_ij of -inf counts as a
 *             disallowed pair below (the same as masked_fill with -inf).
 *   allowed(i, j) = AND of the active rules
 *        causal   : j <= i             (lower-triangular `tril` mask,
 *                                       CogVLM page, "attention mask mechanism")
 *        padding  : j < kv_len[b]      (document padding mask on the key axis,
 *                                       retrieval page, layer 2 SemanticModeler)
 *        bool     : mask[b,h,i,j] != 0 (True = may attend; multimodal page,
 *                                       layer 2 create_cross_modal_mask)
 *        modality : allow[id_i][id_j] || (allow_diag && i == j)
 *                                      (cross-modal rule of the same page,
 *                                       generalised to a 2x2 table)
 *   Disallowed scores are -inf (masked_fill with -inf, multimodal page,
 *   layer 2 flash_attention_with_mask).
 *   m_i = max_allowed s_ij ; L_i = sum_allowed exp(s_ij - m_i)
 *   p_ij = exp(s_ij - m_i) / L_i  (0 where not allowed)
 *   O_i = sum_j p_ij V_j ; LSE_i = m_i + ln L_i
 *   A row with no allowed key: O_i = 0, LSE_i = -inf (the pages are silent;
 *   this is the reading that keeps the result finite and exact).
 *
 * Backward, from the same explicit P (the pages only say the gradient is
 * produced without storing the N x N matrix; the gradient itself is the
 * derivative of the forward definition above):
 *   dV_j = sum_i p_ij dO_i
 *   dP_ij = dO_i . V_j
 *   Dl_i  = sum_j p_ij dP_ij
 *   dS_ij = p_ij (dP_ij - Dl_i)
 *   dQ_i  = scale * sum_j dS_ij K_j
 *   dK_j  = scale * sum_i dS_ij Q_i
 *
 * All arrays are fp64 in BNSD order ([B][N][S][D], D contiguous); lse is
 * [B][N][Sq].  The score matrix of one (b, h) is materialised explicitly --
 * this is the unfused "discrete" algorithm, deliberately.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

typedef struct {
  int causal;
  const int32_t* kv_len;   /* [B] or NULL */
  const uint8_t* mask;     /* bool mask or NULL; element (b,h,i,j) at
                              b*msb + h*msh + i*msq + j */
  int64_t msb, msh, msq;
  const int32_t* ids;      /* [B][S] modality ids (0/1) or NULL; Sq == Sk */
  int allow00, allow01, allow10, allow11, allow_diag;
  const double* add;       /* dense additive term or NULL; element (b,h,i,j)
                              at b*asb + h*ash + i*asq + j */
  int64_t asb, ash, asq;
} oracle_mask;

static int oracle_threads = 0;

void oracle_set_threads(int n) { oracle_threads = n; }

int oracle_get_threads(void) {
#ifdef _OPENMP
  return oracle_threads > 0 ? oracle_threads : omp_get_max_threads();
#else
  return 1;
#endif
}

static int is_allowed(const oracle_mask* m, int b, int h, int Sq, int Sk,
                      int i, int j) {
  (void)Sq;
  if (!m) return 1;
  if (m->causal && j > i) return 0;
  if (m->kv_len && j >= m->kv_len[b]) return 0;
  if (m->mask && m->mask[b * m->msb + h * m->msh + i * m->msq + j] == 0)
    return 0;
  if (m->ids) {
    int a = m->ids[(int64_t)b * Sk + i];
    int c = m->ids[(int64_t)b * Sk + j];
    int ok;
    if (a == 0 && c == 0) ok = m->allow00;
    else if (a == 0 && c == 1) ok = m->allow01;
    else if (a == 1 && c == 0) ok = m->allow10;
    else ok = m->allow11;
    if (m->allow_diag && i == j) ok = 1;
    if (!ok) return 0;
  }
  return 1;
}

/* P for one (b, h): p[i*Sk + j], plus lse[i].  Returns nothing; rows with no
 * allowed key get p = 0 and lse = -inf. */
static void probs_one_head(int b, int h, int Sq, int Sk, int D,
                           const double* q, const double* k,
                           const double* slopes, const oracle_mask* m,
                           double scale, double* s, double* p, double* lse) {
  for (int i = 0; i < Sq; ++i) {
    double mx = -INFINITY;
    int any = 0;
    for (int j = 0; j < Sk; ++j) {
      double* sij = &s[(int64_t)i * Sk + j];
      if (!is_allowed(m, b, h, Sq, Sk, i, j)) {
        *sij = -INFINITY;
        continue;
      }
      double dot = 0.0;
      for (int d = 0; d < D; ++d)
        dot += q[(int64_t)i * D + d] * k[(int64_t)j * D + d];
      double val = scale * dot;
      if (slopes) val += -slopes[h] * fabs((double)(i - j));
      if (m && m->add) val += m->add[b * m->asb + h * m->ash + (int64_t)i * m->asq + j];
      if (val == -INFINITY) { /* an additive -inf masks the pair */
        *sij = -INFINITY;
        continue;
      }
      *sij = val;
      if (!any || val > mx) mx = val;
      any = 1;
    }
    if (!any) {
      for (int j = 0; j < Sk; ++j) p[(int64_t)i * Sk + j] = 0.0;
      lse[i] = -INFINITY;
      continue;
    }
    double sum = 0.0;
    for (int j = 0; j < Sk; ++j) {
      double sij = s[(int64_t)i * Sk + j];
      double e = (sij == -INFINITY) ? 0.0 : exp(sij - mx);
      p[(int64_t)i * Sk + j] = e;
      sum += e;
    }
    for (int j = 0; j < Sk; ++j) p[(int64_t)i * Sk + j] /= sum;
    lse[i] = mx + log(sum);
  }
}

int oracle_fwd(int B, int N, int Sq, int Sk, int D, const double* q,
               const double* k, const double* v, const double* slopes,
               const oracle_mask* m, double scale, double* out, double* lse) {
  if (B < 0 || N < 0 || Sq < 0 || Sk < 0 || D <= 0) return 1;
  int64_t BN = (int64_t)B * N;
  int fail = 0;
#pragma omp parallel for schedule(dynamic) num_threads(oracle_get_threads())
  for (int64_t bh = 0; bh < BN; ++bh) {
    int b = (int)(bh / N), h = (int)(bh % N);
    const double* qh = q + bh * Sq * D;
    const double* kh = k + bh * Sk * D;
    const double* vh = v + bh * Sk * D;
    double* oh = out + bh * Sq * D;
    double* s = (double*)malloc(sizeof(double) * ((size_t)Sq * Sk + 1));
    double* p = (double*)malloc(sizeof(double) * ((size_t)Sq * Sk + 1));
    if (!s || !p) {
      free(s); free(p);
#pragma omp atomic write
      fail = 1;
      continue;
    }
    probs_one_head(b, h, Sq, Sk, D, qh, kh, slopes, m, scale, s, p,
                   lse + bh * Sq);
    for (int i = 0; i < Sq; ++i)
      for (int d = 0; d < D; ++d) {
        double acc = 0.0;
        for (int j = 0; j < Sk; ++j)
          acc += p[(int64_t)i * Sk + j] * vh[(int64_t)j * D + d];
        oh[(int64_t)i * D + d] = acc;
      }
    free(s);
    free(p);
  }
  return fail ? 2 : 0;
}

int oracle_bwd(int B, int N, int Sq, int Sk, int D, const double* q,
               const double* k, const double* v, const double* dout,
               const double* slopes, const oracle_mask* m, double scale,
               double* dq, double* dk, double* dv) {
  if (B < 0 || N < 0 || Sq < 0 || Sk < 0 || D <= 0) return 1;
  int64_t BN = (int64_t)B * N;
  int fail = 0;
#pragma omp parallel for schedule(dynamic) num_threads(oracle_get_threads())
  for (int64_t bh = 0; bh < BN; ++bh) {
    int b = (int)(bh / N), h = (int)(bh % N);
    const double* qh = q + bh * Sq * D;
    const double* kh = k + bh * Sk * D;
    const double* vh = v + bh * Sk * D;
    const double* doh = dout + bh * Sq * D;
    double* dqh = dq + bh * Sq * D;
    double* dkh = dk + bh * Sk * D;
    double* dvh = dv + bh * Sk * D;
    size_t ss = (size_t)Sq * Sk + 1;
    double* s = (double*)malloc(sizeof(double) * ss);
    double* p = (double*)malloc(sizeof(double) * ss);
    double* ds = (double*)malloc(sizeof(double) * ss);
    double* lse = (double*)malloc(sizeof(double) * ((size_t)Sq + 1));
    if (!s || !p || !ds || !lse) {
      free(s); free(p); free(ds); free(lse);
#pragma omp atomic write
      fail = 1;
      continue;
    }
    probs_one_head(b, h, Sq, Sk, D, qh, kh, slopes, m, scale, s, p, lse);
    /* dV_j = sum_i p_ij dO_i */
    for (int j = 0; j < Sk; ++j)
      for (int d = 0; d < D; ++d) {
        double acc = 0.0;
        for (int i = 0; i < Sq; ++i)
          acc += p[(int64_t)i * Sk + j] * doh[(int64_t)i * D + d];
        dvh[(int64_t)j * D + d] = acc;
      }
    /* dP_ij = dO_i . V_j ; Dl_i = sum_j p_ij dP_ij ; dS = p (dP - Dl) */
    for (int i = 0; i < Sq; ++i) {
      double dl = 0.0;
      for (int j = 0; j < Sk; ++j) {
        double dp = 0.0;
        for (int d = 0; d < D; ++d)
          dp += doh[(int64_t)i * D + d] * vh[(int64_t)j * D + d];
        ds[(int64_t)i * Sk + j] = dp; /* holds dP for now */
        dl += p[(int64_t)i * Sk + j] * dp;
      }
      for (int j = 0; j < Sk; ++j) {
        double pij = p[(int64_t)i * Sk + j];
        ds[(int64_t)i * Sk + j] = pij * (ds[(int64_t)i * Sk + j] - dl);
      }
    }
    /* dQ_i = scale * sum_j dS_ij K_j */
    for (int i = 0; i < Sq; ++i)
      for (int d = 0; d < D; ++d) {
        double acc = 0.0;
        for (int j = 0; j < Sk; ++j)
          acc += ds[(int64_t)i * Sk + j] * kh[(int64_t)j * D + d];
        dqh[(int64_t)i * D + d] = scale * acc;
      }
    /* dK_j = scale * sum_i dS_ij Q_i */
    for (int j = 0; j < Sk; ++j)
      for (int d = 0; d < D; ++d) {
        double acc = 0.0;
        for (int i = 0; i < Sq; ++i)
          acc += ds[(int64_t)i * Sk + j] * qh[(int64_t)i * D + d];
        dkh[(int64_t)j * D + d] = scale * acc;
      }
    free(s); free(p); free(ds); free(lse);
  }
  return fail ? 2 : 0;
}

/* Explicit probability matrix of one (b, h), for tests that inspect P
 * (row sums, closed forms).  p is [Sq][Sk]. */
int oracle_probs(int B, int N, int Sq, int Sk, int D, int b, int h,
                 const double* q, const double* k, const double* slopes,
                 const oracle_mask* m, double scale, double* p, double* lse) {
  if (b < 0 || b >= B || h < 0 || h >= N) return 1;
  int64_t bh = (int64_t)b * N + h;
  double* s = (double*)malloc(sizeof(double) * ((size_t)Sq * Sk + 1));
  if (!s) return 2;
  probs_one_head(b, h, Sq, Sk, D, q + bh * Sq * D, k + bh * Sk * D, slopes, m,
                 scale, s, p, lse);
  free(s);
  return 0;
}
