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
 *   Dropout (the guide's keep_prob, sec. 3.1/3.2; the unfused softmax ->
 *   dropout -> matmul of sec. 1): p'_ij = p_ij * keep_ij / keep_prob with
 *   keep_ij = [u_ij < round(keep_prob * 65536)], u_ij a 16-bit field of
 *   Philox-4x32-10 (Salmon, Moraes, Dror, Shaw, "Parallel Random Numbers:
 *   As Easy as 1, 2, 3", SC'11) with key (seed mod 2^32, seed / 2^32) and
 *   counter words (c0, c1) = offset + j / 8 (a 64-bit block index, mod 2^64),
 *   c2 = i, c3 = (b * N + h) mod 2^32; field j mod 8 is word (j mod 8) / 2,
 *   bits 16 * (j mod 2).
 *   The pages fix only the retention probability; the generator, the
 *   counter layout and the 16-bit threshold are this implementation's
 *   reading.  O_i = sum_j p'_ij V_j; LSE is that of p (before dropout).
 *   m_i = max_allowed s_ij ; L_i = sum_allowed exp(s_ij - m_i)
 *   p_ij = exp(s_ij - m_i) / L_i  (0 where not allowed)
 *   O_i = sum_j p_ij V_j ; LSE_i = m_i + ln L_i
 *   A row with no allowed key: O_i = 0, LSE_i = -inf (the pages are silent;
 *   this is the reading that keeps the result finite and exact).
 *
 * Backward, from the same explicit P (the pages only say the gradient is
 * produced without storing the N x N matrix; the gradient itself is the
 * derivative of the forward definition above; f_ij = keep_ij / keep_prob
 * with dropout, else 1):
 *   dV_j = sum_i p_ij f_ij dO_i
 *   dP_ij = f_ij (dO_i . V_j)
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
  int dropout;             /* 1: apply dropout with keep_prob, seed, offset */
  double keep_prob;
  uint64_t seed, offset;
} oracle_mask;

/* Philox-4x32-10 (Salmon et al., SC'11): ten rounds of two 32x32->64
 * multiplies by the round multipliers, the high halves xored with the other
 * counter words and the key, the key bumped by the Weyl constants between
 * rounds. */
static void philox4x32_10(const uint32_t ctr[4], const uint32_t key[2], uint32_t out[4]) {
  const uint32_t M0 = 0xD2511F53u, M1 = 0xCD9E8D57u;
  const uint32_t W0 = 0x9E3779B9u, W1 = 0xBB67AE85u;
  uint32_t x0 = ctr[0], x1 = ctr[1], x2 = ctr[2], x3 = ctr[3];
  uint32_t k0 = key[0], k1 = key[1];
  for (int r = 0; r < 10; ++r) {
    uint64_t p0 = (uint64_t)M0 * x0;
    uint64_t p1 = (uint64_t)M1 * x2;
    uint32_t hi0 = (uint32_t)(p0 >> 32), lo0 = (uint32_t)p0;
    uint32_t hi1 = (uint32_t)(p1 >> 32), lo1 = (uint32_t)p1;
    x0 = hi1 ^ x1 ^ k0;
    x1 = lo1;
    x2 = hi0 ^ x3 ^ k1;
    x3 = lo0;
    k0 += W0;
    k1 += W1;
  }
  out[0] = x0; out[1] = x1; out[2] = x2; out[3] = x3;
}

void oracle_philox4x32(const uint32_t* ctr, const uint32_t* key, uint32_t* out) {
  philox4x32_10(ctr, key, out);
}

/* keep_ij of the dropout definition in the header (1 = kept). */
static int dropout_keep(const oracle_mask* m, int N, int b, int h, int i, int j) {
  uint64_t block = m->offset + (uint64_t)(j / 8);
  uint64_t bh = (uint64_t)b * N + h;
  uint32_t ctr[4] = {(uint32_t)block, (uint32_t)(block >> 32), (uint32_t)i, (uint32_t)bh};
  uint32_t key[2] = {(uint32_t)m->seed, (uint32_t)(m->seed >> 32)};
  uint32_t w[4];
  philox4x32_10(ctr, key, w);
  int f = j % 8;
  uint32_t u = (w[f / 2] >> (16 * (f % 2))) & 0xFFFFu;
  double t = floor(m->keep_prob * 65536.0 + 0.5);
  return (double)u < t;
}

/* f_ij = keep_ij / keep_prob with dropout, 1 without, for one (b, h). */
static void dropout_factors(const oracle_mask* m, int N, int b, int h, int Sq, int Sk,
                            double* f) {
  for (int i = 0; i < Sq; ++i)
    for (int j = 0; j < Sk; ++j)
      f[(int64_t)i * Sk + j] =
          (m && m->dropout) ? (dropout_keep(m, N, b, h, i, j) ? 1.0 / m->keep_prob : 0.0) : 1.0;
}

/* keep[b][h][i][j] (1 = kept) for tests. */
int oracle_dropout_mask(int B, int N, int Sq, int Sk, const oracle_mask* m, uint8_t* keep) {
  if (!m || !m->dropout) return 1;
  for (int b = 0; b < B; ++b)
    for (int h = 0; h < N; ++h)
      for (int i = 0; i < Sq; ++i)
        for (int j = 0; j < Sk; ++j)
          keep[(((int64_t)b * N + h) * Sq + i) * Sk + j] = (uint8_t)dropout_keep(m, N, b, h, i, j);
  return 0;
}

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
    if (m && m->dropout) {   /* p' = p * f, kept in p (s is free now) */
      dropout_factors(m, N, b, h, Sq, Sk, s);
      for (int64_t e = 0; e < (int64_t)Sq * Sk; ++e) p[e] *= s[e];
    }
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
    double* f = s;   /* the dropout factors f_ij (1 without dropout) */
    dropout_factors(m, N, b, h, Sq, Sk, f);
    /* dV_j = sum_i p_ij f_ij dO_i */
    for (int j = 0; j < Sk; ++j)
      for (int d = 0; d < D; ++d) {
        double acc = 0.0;
        for (int i = 0; i < Sq; ++i)
          acc += p[(int64_t)i * Sk + j] * f[(int64_t)i * Sk + j] * doh[(int64_t)i * D + d];
        dvh[(int64_t)j * D + d] = acc;
      }
    /* dP_ij = f_ij dO_i . V_j ; Dl_i = sum_j p_ij dP_ij ; dS = p (dP - Dl) */
    for (int i = 0; i < Sq; ++i) {
      double dl = 0.0;
      for (int j = 0; j < Sk; ++j) {
        double dp = 0.0;
        for (int d = 0; d < D; ++d)
          dp += doh[(int64_t)i * D + d] * vh[(int64_t)j * D + d];
        dp *= f[(int64_t)i * Sk + j];
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
