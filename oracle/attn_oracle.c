/*
 * Exact attention oracle: plain, slow, float64, CPU.
 *
 * TEST INFRASTRUCTURE.  Only the tests, the smoke check and the benchmark's
 * CPU-baseline leg may load or call this file.  It shares no code, header,
 * table or helper with the CUDA library, and the CUDA library never calls it.
 *
 * What it computes is the definition of attention, written out:
 *
 *   O = softmax(Q K^T * scale + mask) V
 *
 *   - "FlashAttention ... Transformer optimization" (page 2, first paragraph of
 *     the technical deep dive) gives Softmax(QK^T / sqrt(d)) V; scale defaults
 *     to 1/sqrt(d) and is otherwise the caller's softmax_scale (the
 *     integration example on the FlashAttention-2 page passes it explicitly).
 *   - The tiled method reaches this same result (page 4, definition: "exact
 *     attention"; page 5: the result is unchanged by tiling), so the oracle is
 *     the untiled definition: explicit scores, a two-pass softmax (row max,
 *     then row sum), explicit masks.
 *   - Masks (FlashAttention-2 page, section 3 "more flexible masks" and the
 *     sparse-attention extension): causal and sliding-window.  Reading taken:
 *     key j is visible from query i iff
 *         j <= i + off                       (causal)
 *         j >= i + off - window_left         (window_left  >= 0)
 *         j <= i + off + window_right        (window_right >= 0)
 *     with off = seqlen_k - seqlen_q (bottom-right alignment), bounds
 *     inclusive, -1 meaning unbounded.
 *   - Grouped-query attention (page 5, hardware/dtype section, MQA/GQA):
 *     query head h reads kv head h / (nheads / nheads_kv).
 *   - Positional bias from per-head slopes (the alibi_slopes argument named
 *     on the FlashAttention-2 page, FAQ Q2, and on page 5's backend list;
 *     neither gives the formula).  Reading taken: when slopes are given,
 *         S_ij += -slope_h * |i + off - j|
 *     on the scaled scores, with the masks' bottom-right alignment; no
 *     slopes (NULL) means no bias.
 *   - LSE_i = m_i + ln(l_i), natural log, of the scaled scores.  A row with
 *     no visible key gets O = 0 and LSE = -inf.
 *   - Dropout on the attention probabilities (named as a supported feature
 *     on page 5, hardware/dtype section: the backward's head-dim limit
 *     "without dropout" and the backends that offer dropout; no formula is
 *     given).  Reading taken: inverted dropout,
 *         O_i = sum_j P_ij z_ij V_j,   z_ij = 0 (dropped) or 1 / (1 - p'),
 *     with P, m, l and LSE those of the undropped scores.  The drop
 *     decisions come from a counter-based generator so that any program can
 *     reproduce them: Philox4x32-10 (Salmon, Moraes, Dror and Shaw,
 *     "Parallel random numbers: as easy as 1, 2, 3", SC 2011) with key
 *     (seed low word, seed high word) and, for element (b, h, i, j) of the
 *     score matrix, counter (j / 4, i / 4, b * H + h, offset); its output
 *     word i mod 4, byte j mod 4 (bits 8 (j mod 4) and up) is the element's
 *     random byte u, and the element is dropped iff u < t for the threshold
 *     t = round(256 p) in [0, 255]; p' = t / 256.  t = 0 is no dropout.
 *     Backward through the same mask: dP_ij = z_ij dO_i . V_j and
 *     dV_j = sum_i P_ij z_ij dO_i; the dS formula below is unchanged.
 *   - Backward (page 2, item 2: the backward pass recomputes the score
 *     matrix; the arithmetic is the analytic gradient of the definition):
 *         dV = P^T dO,  dP = dO V^T,
 *         dS = P o (dP - rowsum(P o dP)),
 *         dQ = scale * dS K,  dK = scale * dS^T Q,
 *     with dK and dV summed over the query heads that share a kv head.
 *
 * Layouts: q, o, dout, dq (B, Nq, H, d); k, v, dk, dv (B, Nk, Hkv, d);
 * lse (B, H, Nq).  All float64, contiguous.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

typedef struct {
  int64_t batch, seqlen_q, seqlen_k, nheads, nheads_kv, headdim;
  double softmax_scale;
  int64_t causal, window_left, window_right;
  const double *alibi_slopes; /* nheads slopes, or NULL */
  int64_t dropout_threshold;  /* t in [0, 255]; 0 = no dropout */
  uint64_t dropout_seed;
  int64_t dropout_offset;     /* the counter's last word (32 bits) */
  int64_t batch_base;         /* counter batch index of this call's batch 0 */
} oracle_params;

/* Philox4x32-10 (the SC 2011 paper above).  One round: the 64-bit products
 * of counter words 0 and 2 with the two multipliers; the new words are
 * (high half of product 2) ^ word 1 ^ key 0, low half of product 2,
 * (high half of product 0) ^ word 3 ^ key 1, low half of product 0.  The key
 * advances by the two Weyl constants after every round; ten rounds. */
void oracle_philox4x32_10(const uint32_t ctr[4], const uint32_t key[2], uint32_t out[4]) {
  const uint32_t m0 = 0xD2511F53u, m1 = 0xCD9E8D57u, w0 = 0x9E3779B9u, w1 = 0xBB67AE85u;
  uint32_t x0 = ctr[0], x1 = ctr[1], x2 = ctr[2], x3 = ctr[3], k0 = key[0], k1 = key[1];
  for (int r = 0; r < 10; ++r) {
    const uint64_t p0 = (uint64_t)m0 * x0, p1 = (uint64_t)m1 * x2;
    const uint32_t y0 = (uint32_t)(p1 >> 32) ^ x1 ^ k0;
    const uint32_t y2 = (uint32_t)(p0 >> 32) ^ x3 ^ k1;
    x1 = (uint32_t)p1;
    x3 = (uint32_t)p0;
    x0 = y0;
    x2 = y2;
    k0 += w0;
    k1 += w1;
  }
  out[0] = x0; out[1] = x1; out[2] = x2; out[3] = x3;
}

/* Dropout factor z of score element (b, h, i, j): 1 without dropout, else 0
 * (dropped) or 256 / (256 - t) (the counter layout stated above). */
static double keep_scale(const oracle_params *p, int64_t b, int64_t h, int64_t i, int64_t j) {
  if (p->dropout_threshold <= 0) return 1.0;
  const uint32_t ctr[4] = {(uint32_t)(j >> 2), (uint32_t)(i >> 2),
                           (uint32_t)((p->batch_base + b) * p->nheads + h),
                           (uint32_t)p->dropout_offset};
  const uint32_t key[2] = {(uint32_t)p->dropout_seed, (uint32_t)(p->dropout_seed >> 32)};
  uint32_t out[4];
  oracle_philox4x32_10(ctr, key, out);
  const uint32_t u = (out[i & 3] >> (8 * (j & 3))) & 0xFFu;
  if (u < (uint32_t)p->dropout_threshold) return 0.0;
  return 256.0 / (256.0 - (double)p->dropout_threshold);
}

/* Visibility of key j from query i (the mask reading stated above). */
static int visible(const oracle_params *p, int64_t i, int64_t j) {
  int64_t ii = i + (p->seqlen_k - p->seqlen_q);
  if (p->causal && j > ii) return 0;
  if (p->window_left >= 0 && j < ii - p->window_left) return 0;
  if (p->window_right >= 0 && j > ii + p->window_right) return 0;
  return 1;
}

static const double *qrow(const oracle_params *p, const double *q, int64_t b, int64_t i, int64_t h) {
  return q + ((b * p->seqlen_q + i) * p->nheads + h) * p->headdim;
}
static const double *krow(const oracle_params *p, const double *k, int64_t b, int64_t j, int64_t g) {
  return k + ((b * p->seqlen_k + j) * p->nheads_kv + g) * p->headdim;
}
static int64_t kv_head(const oracle_params *p, int64_t h) {
  return h / (p->nheads / p->nheads_kv);
}

static double dot(const double *a, const double *b, int64_t n) {
  double acc = 0.0;
  for (int64_t c = 0; c < n; ++c) acc += a[c] * b[c];
  return acc;
}

/*
 * Scores of one query row and its softmax statistics (two passes).
 * s[j] = scale * q_i . k_j for visible j, -inf otherwise.
 * *m = max_j s[j]; *l = sum_j exp(s[j] - *m).  No visible key: *l = 0.
 */
/* Score of query i (head h, row qi) against key j (row kj): the scaled dot
 * product plus the positional bias when slopes are given. */
static double score(const oracle_params *p, const double *qi, const double *kj, int64_t h,
                    int64_t i, int64_t j) {
  double sij = p->softmax_scale * dot(qi, kj, p->headdim);
  if (p->alibi_slopes)
    sij -= p->alibi_slopes[h] * fabs((double)(i + p->seqlen_k - p->seqlen_q - j));
  return sij;
}

static void row_scores(const oracle_params *p, const double *q, const double *k,
                       int64_t b, int64_t h, int64_t i, double *s, double *m, double *l) {
  const int64_t g = kv_head(p, h);
  const double *qi = qrow(p, q, b, i, h);
  double mx = -INFINITY;
  int64_t count = 0;
  for (int64_t j = 0; j < p->seqlen_k; ++j) {
    if (!visible(p, i, j)) { s[j] = -INFINITY; continue; }
    s[j] = score(p, qi, krow(p, k, b, j, g), h, i, j);
    if (s[j] > mx) mx = s[j];
    ++count;
  }
  double sum = 0.0;
  if (count > 0)
    for (int64_t j = 0; j < p->seqlen_k; ++j)
      if (s[j] != -INFINITY) sum += exp(s[j] - mx);
  *m = mx;
  *l = sum;
}

/* Probability P_ij from the row's score and statistics. */
static double prob(double s, double m, double l) {
  return (s == -INFINITY || l == 0.0) ? 0.0 : exp(s - m) / l;
}

/* One forward row: o_out[0..d) and *lse_out. */
static void fwd_row(const oracle_params *p, const double *q, const double *k, const double *v,
                    int64_t b, int64_t h, int64_t i, double *s, double *o_out, double *lse_out) {
  const int64_t d = p->headdim, g = kv_head(p, h);
  double m, l;
  row_scores(p, q, k, b, h, i, s, &m, &l);
  for (int64_t c = 0; c < d; ++c) o_out[c] = 0.0;
  if (l == 0.0) { *lse_out = -INFINITY; return; }
  for (int64_t j = 0; j < p->seqlen_k; ++j) {
    double pij = prob(s[j], m, l);
    if (pij == 0.0) continue;
    const double zij = keep_scale(p, b, h, i, j);
    const double *vj = krow(p, v, b, j, g);
    for (int64_t c = 0; c < d; ++c) o_out[c] += pij * zij * vj[c];
  }
  *lse_out = m + log(l);
}

static int valid(const oracle_params *p) {
  return p && p->batch >= 0 && p->seqlen_q >= 0 && p->seqlen_k >= 0 && p->nheads > 0 &&
         p->nheads_kv > 0 && p->nheads % p->nheads_kv == 0 && p->headdim > 0 &&
         p->dropout_threshold >= 0 && p->dropout_threshold <= 255 && p->batch_base >= 0;
}

int oracle_num_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

void oracle_set_num_threads(int n) {
#ifdef _OPENMP
  if (n > 0) omp_set_num_threads(n);
#else
  (void)n;
#endif
}

/*
 * Forward for a list of query positions `rows` (nrows of them, each in
 * [0, Nq)), for every batch and head.  Outputs: o (B, nrows, H, d) and
 * lse (B, H, nrows).  rows == NULL means all rows in order (nrows = Nq).
 * Returns 0, or -1 on invalid arguments.
 */
int oracle_attn_fwd_rows(const oracle_params *p, const double *q, const double *k, const double *v,
                         const int64_t *rows, int64_t nrows, double *o, double *lse) {
  if (!valid(p)) return -1;
  if (!rows) nrows = p->seqlen_q;
  const int64_t B = p->batch, H = p->nheads, d = p->headdim;
  const int64_t total = B * H * nrows;
  int bad = 0;
#pragma omp parallel
  {
    double *s = (double *)malloc(sizeof(double) * (size_t)(p->seqlen_k > 0 ? p->seqlen_k : 1));
    if (!s) {
#pragma omp atomic write
      bad = 1;
    }
#pragma omp for schedule(dynamic, 4)
    for (int64_t t = 0; t < total; ++t) {
      if (!s) continue;
      const int64_t r = t % nrows, h = (t / nrows) % H, b = t / (nrows * H);
      const int64_t i = rows ? rows[r] : r;
      if (i < 0 || i >= p->seqlen_q) {
#pragma omp atomic write
        bad = 1;
        continue;
      }
      fwd_row(p, q, k, v, b, h, i, s, o + ((b * nrows + r) * H + h) * d, lse + (b * H + h) * nrows + r);
    }
    free(s);
  }
  return bad ? -1 : 0;
}

int oracle_attn_fwd(const oracle_params *p, const double *q, const double *k, const double *v,
                    double *o, double *lse) {
  return oracle_attn_fwd_rows(p, q, k, v, NULL, 0, o, lse);
}

/*
 * Full backward.  dq (B, Nq, H, d); dk, dv (B, Nk, Hkv, d).
 * Parallel over (batch, kv head) so that the sums into dk/dv over the heads
 * of a group and over query rows stay within one thread.
 */
int oracle_attn_bwd(const oracle_params *p, const double *q, const double *k, const double *v,
                    const double *dout, double *dq, double *dk, double *dv) {
  if (!valid(p)) return -1;
  const int64_t B = p->batch, H = p->nheads, Hkv = p->nheads_kv, d = p->headdim;
  const int64_t Nq = p->seqlen_q, Nk = p->seqlen_k, group = H / Hkv;
  memset(dk, 0, sizeof(double) * (size_t)(B * Nk * Hkv * d));
  memset(dv, 0, sizeof(double) * (size_t)(B * Nk * Hkv * d));
  int bad = 0;
#pragma omp parallel
  {
    const size_t n = (size_t)(Nk > 0 ? Nk : 1);
    double *s = (double *)malloc(sizeof(double) * n);
    double *pr = (double *)malloc(sizeof(double) * n);
    double *dp = (double *)malloc(sizeof(double) * n);
    double *zr = (double *)malloc(sizeof(double) * n);
    if (!s || !pr || !dp || !zr) {
#pragma omp atomic write
      bad = 1;
    }
#pragma omp for schedule(dynamic, 1)
    for (int64_t t = 0; t < B * Hkv; ++t) {
      if (!s || !pr || !dp || !zr) continue;
      const int64_t b = t / Hkv, g = t % Hkv;
      for (int64_t h = g * group; h < (g + 1) * group; ++h) {
        for (int64_t i = 0; i < Nq; ++i) {
          double m, l;
          const double *qi = qrow(p, q, b, i, h);
          const double *doi = qrow(p, dout, b, i, h);
          double *dqi = dq + ((b * Nq + i) * H + h) * d;
          row_scores(p, q, k, b, h, i, s, &m, &l);
          double rowsum = 0.0; /* sum_j P_ij dP_ij */
          for (int64_t j = 0; j < Nk; ++j) {
            pr[j] = prob(s[j], m, l);
            zr[j] = (pr[j] != 0.0) ? keep_scale(p, b, h, i, j) : 0.0;
            dp[j] = (pr[j] != 0.0) ? zr[j] * dot(doi, krow(p, v, b, j, g), d) : 0.0;
            rowsum += pr[j] * dp[j];
          }
          for (int64_t c = 0; c < d; ++c) dqi[c] = 0.0;
          for (int64_t j = 0; j < Nk; ++j) {
            if (pr[j] == 0.0) continue;
            const double ds = pr[j] * (dp[j] - rowsum);
            const double *kj = krow(p, k, b, j, g);
            double *dkj = dk + ((b * Nk + j) * Hkv + g) * d;
            double *dvj = dv + ((b * Nk + j) * Hkv + g) * d;
            for (int64_t c = 0; c < d; ++c) {
              dqi[c] += p->softmax_scale * ds * kj[c];
              dkj[c] += p->softmax_scale * ds * qi[c];
              dvj[c] += pr[j] * zr[j] * doi[c];
            }
          }
        }
      }
    }
    free(s); free(pr); free(dp); free(zr);
  }
  return bad ? -1 : 0;
}

/*
 * Backward on sampled rows.
 *   dq rows:  query positions qrows[0..nq) -> dq (B, nq, H, d)
 *   dk/dv rows: key positions krows[0..nk) -> dk, dv (B, nk, Hkv, d)
 * The dk/dv rows need every query row's softmax statistics and rowsum(P o dP),
 * which are computed first for all (b, h, i); the sums over i and over the
 * heads of a group then run for the sampled keys only.
 */
int oracle_attn_bwd_rows(const oracle_params *p, const double *q, const double *k, const double *v,
                         const double *dout, const int64_t *qrows, int64_t nq, double *dq,
                         const int64_t *krows, int64_t nk, double *dk, double *dv) {
  if (!valid(p)) return -1;
  const int64_t B = p->batch, H = p->nheads, Hkv = p->nheads_kv, d = p->headdim;
  const int64_t Nq = p->seqlen_q, Nk = p->seqlen_k, group = H / Hkv;
  int bad = 0;
  for (int64_t r = 0; r < nq; ++r) if (qrows[r] < 0 || qrows[r] >= Nq) return -1;
  for (int64_t r = 0; r < nk; ++r) if (krows[r] < 0 || krows[r] >= Nk) return -1;

  /* dq rows: each is independent. */
#pragma omp parallel
  {
    const size_t n = (size_t)(Nk > 0 ? Nk : 1);
    double *s = (double *)malloc(sizeof(double) * n);
    double *pr = (double *)malloc(sizeof(double) * n);
    double *dp = (double *)malloc(sizeof(double) * n);
    if (!s || !pr || !dp) {
#pragma omp atomic write
      bad = 1;
    }
#pragma omp for schedule(dynamic, 2)
    for (int64_t t = 0; t < B * H * nq; ++t) {
      if (!s || !pr || !dp) continue;
      const int64_t r = t % nq, h = (t / nq) % H, b = t / (nq * H);
      const int64_t i = qrows[r], g = kv_head(p, h);
      const double *doi = qrow(p, dout, b, i, h);
      double *dqi = dq + ((b * nq + r) * H + h) * d;
      double m, l;
      row_scores(p, q, k, b, h, i, s, &m, &l);
      double rowsum = 0.0;
      for (int64_t j = 0; j < Nk; ++j) {
        pr[j] = prob(s[j], m, l);
        dp[j] = (pr[j] != 0.0) ? keep_scale(p, b, h, i, j) * dot(doi, krow(p, v, b, j, g), d)
                               : 0.0;
        rowsum += pr[j] * dp[j];
      }
      for (int64_t c = 0; c < d; ++c) dqi[c] = 0.0;
      for (int64_t j = 0; j < Nk; ++j) {
        if (pr[j] == 0.0) continue;
        const double ds = pr[j] * (dp[j] - rowsum);
        const double *kj = krow(p, k, b, j, g);
        for (int64_t c = 0; c < d; ++c) dqi[c] += p->softmax_scale * ds * kj[c];
      }
    }
    free(s); free(pr); free(dp);
  }
  if (bad || nk == 0) return bad ? -1 : 0;

  /* Row statistics of every query row: max, sum and rowsum(P o dP). */
  const int64_t nrow_all = B * H * Nq;
  double *M = (double *)malloc(sizeof(double) * (size_t)(nrow_all > 0 ? nrow_all : 1));
  double *L = (double *)malloc(sizeof(double) * (size_t)(nrow_all > 0 ? nrow_all : 1));
  double *R = (double *)malloc(sizeof(double) * (size_t)(nrow_all > 0 ? nrow_all : 1));
  if (!M || !L || !R) { free(M); free(L); free(R); return -1; }
#pragma omp parallel
  {
    const size_t n = (size_t)(Nk > 0 ? Nk : 1);
    double *s = (double *)malloc(sizeof(double) * n);
    if (!s) {
#pragma omp atomic write
      bad = 1;
    }
#pragma omp for schedule(dynamic, 4)
    for (int64_t t = 0; t < nrow_all; ++t) {
      if (!s) continue;
      const int64_t i = t % Nq, h = (t / Nq) % H, b = t / (Nq * H), g = kv_head(p, h);
      const double *doi = qrow(p, dout, b, i, h);
      double m, l, rowsum = 0.0;
      row_scores(p, q, k, b, h, i, s, &m, &l);
      for (int64_t j = 0; j < Nk; ++j) {
        const double pij = prob(s[j], m, l);
        if (pij != 0.0)
          rowsum += pij * keep_scale(p, b, h, i, j) * dot(doi, krow(p, v, b, j, g), d);
      }
      M[t] = m; L[t] = l; R[t] = rowsum;
    }
    free(s);
  }
  if (bad) { free(M); free(L); free(R); return -1; }

  /* dk/dv of the sampled keys: sums over the group's heads and all rows. */
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t t = 0; t < B * Hkv * nk; ++t) {
    const int64_t r = t % nk, g = (t / nk) % Hkv, b = t / (nk * Hkv);
    const int64_t j = krows[r];
    const double *kj = krow(p, k, b, j, g), *vj = krow(p, v, b, j, g);
    double *dkj = dk + ((b * nk + r) * Hkv + g) * d;
    double *dvj = dv + ((b * nk + r) * Hkv + g) * d;
    for (int64_t c = 0; c < d; ++c) { dkj[c] = 0.0; dvj[c] = 0.0; }
    for (int64_t h = g * group; h < (g + 1) * group; ++h) {
      for (int64_t i = 0; i < Nq; ++i) {
        if (!visible(p, i, j)) continue;
        const int64_t row = (b * H + h) * Nq + i;
        const double *qi = qrow(p, q, b, i, h), *doi = qrow(p, dout, b, i, h);
        const double sij = score(p, qi, kj, h, i, j);
        const double pij = prob(sij, M[row], L[row]);
        if (pij == 0.0) continue;
        const double zij = keep_scale(p, b, h, i, j);
        const double ds = pij * (zij * dot(doi, vj, d) - R[row]);
        for (int64_t c = 0; c < d; ++c) {
          dkj[c] += p->softmax_scale * ds * qi[c];
          dvj[c] += pij * zij * doi[c];
        }
      }
    }
  }
  free(M); free(L); free(R);
  return 0;
}

/*
 * The dropout keep mask: keep (B, H, Nq, Nk), 1 where element (b, h, i, j)
 * is kept, 0 where dropped, for every element whether masked or not (the
 * decision does not depend on the mask).  Returns 0, or -1 on invalid
 * arguments.
 */
int oracle_dropout_keep(const oracle_params *p, uint8_t *keep) {
  if (!valid(p)) return -1;
  const int64_t B = p->batch, H = p->nheads, Nq = p->seqlen_q, Nk = p->seqlen_k;
#pragma omp parallel for schedule(static)
  for (int64_t t = 0; t < B * H * Nq; ++t) {
    const int64_t i = t % Nq, h = (t / Nq) % H, b = t / (Nq * H);
    for (int64_t j = 0; j < Nk; ++j) keep[t * Nk + j] = keep_scale(p, b, h, i, j) != 0.0;
  }
  return 0;
}

/*
 * Merge of partial results over disjoint key sets (split-KV decoding,
 * sequence-parallel partials).  The exact identity behind the online softmax
 * (the tiled, exact computation described on "FlashAttention ... Transformer
 * optimization", items 1-2, and the FlashAttention-2 page's online softmax):
 * for query row r with parts s computed over disjoint key sets,
 *     LSE_r = log sum_s exp(LSE_s,r)
 *     O_r   = sum_s exp(LSE_s,r - LSE_r) O_s,r
 * and a row whose parts all have LSE = -inf (no key) gets O = 0, LSE = -inf.
 * Layouts: o_parts (splits, B, Nq, H, d), lse_parts (splits, B, H, Nq); o
 * (B, Nq, H, d), lse (B, H, Nq).
 */
int oracle_attn_merge(int64_t splits, int64_t B, int64_t Nq, int64_t H, int64_t d,
                      const double *o_parts, const double *lse_parts, double *o, double *lse) {
  if (splits < 1 || B < 0 || Nq < 0 || H < 1 || d < 1) return -1;
  const int64_t rows = B * Nq * H, lrows = B * H * Nq;
#pragma omp parallel for schedule(static)
  for (int64_t r = 0; r < rows; ++r) {
    const int64_t h = r % H, i = (r / H) % Nq, b = r / (H * Nq);
    const int64_t lr = (b * H + h) * Nq + i;
    double m = -INFINITY;
    for (int64_t s = 0; s < splits; ++s)
      if (lse_parts[s * lrows + lr] > m) m = lse_parts[s * lrows + lr];
    double *orow = o + r * d;
    for (int64_t c = 0; c < d; ++c) orow[c] = 0.0;
    if (m == -INFINITY) {
      lse[lr] = -INFINITY;
      continue;
    }
    double z = 0.0;
    for (int64_t s = 0; s < splits; ++s) z += exp(lse_parts[s * lrows + lr] - m);
    const double total = m + log(z);
    for (int64_t s = 0; s < splits; ++s) {
      const double w = exp(lse_parts[s * lrows + lr] - total);
      const double *op = o_parts + s * rows * d + r * d;
      for (int64_t c = 0; c < d; ++c) orow[c] += w * op[c];
    }
    lse[lr] = total;
  }
  return 0;
}

/*
 * E4M3, the 8-bit float of FP8 attention (FlashAttention-3's FP8 forward,
 * named on page 5's hardware/dtype section): sign bit, 4 exponent bits with
 * bias 7, 3 mantissa bits.  Exponent field 0 holds subnormals m/8 * 2^-6;
 * there are no infinities; S.1111.111 is NaN, so the largest finite value
 * is 1.75 * 2^8 = 448.
 */
double oracle_e4m3_value(uint8_t c) {
  const int s = c >> 7, e = (c >> 3) & 15, m = c & 7;
  if (e == 15 && m == 7) return NAN;
  const double mag = e == 0 ? ldexp(m / 8.0, -6) : ldexp(1.0 + m / 8.0, e - 7);
  return s ? -mag : mag;
}

/* The code nearest to x among all finite codes of x's sign (a search over
 * the table above); a tie goes to the code with an even mantissa (round to
 * nearest even); magnitudes beyond 448 give +-448 (saturation), NaN gives
 * 0x7F. */
uint8_t oracle_e4m3_code(double x) {
  if (isnan(x)) return 0x7F;
  const uint8_t sign = signbit(x) ? 0x80 : 0x00;
  const double a = fabs(x);
  int best = 0;
  double best_err = INFINITY;
  for (int c = 0; c < 0x7F; ++c) {
    const double err = fabs(oracle_e4m3_value((uint8_t)c) - a);
    if (err < best_err || (err == best_err && (c & 1) == 0)) {
      best = c;
      best_err = err;
    }
  }
  return (uint8_t)(sign | best);
}

/* codes[i] = e4m3 code of x[i] / scale (per-tensor scale: x ~ scale * code). */
void oracle_e4m3_quantize(const double *x, int64_t n, double scale, uint8_t *codes) {
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < n; ++i) codes[i] = oracle_e4m3_code(x[i] / scale);
}
