/*
 * Plain CPU oracle for the batched speculative-sampling verification step.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may call, link or
 * load this file: only the test suite, the smoke check and the benchmark's
 * CPU-baseline leg use it.  It shares no code, header or constant with the
 * CUDA library.
 *
 * Sources (page title, section):
 *   [P2] "Speculative decoding - the small model writes first and the big
 *        model checks" (blog.mna-game.duckdns.org, deep-learning post 46),
 *        section 1 (the verify rule and its notation p, q, t, k),
 *        section 3 (tokens per step = accepted + 1), section 4 (exactness).
 *   [P3] "Speculative decoding: how to run big models fast" (ai-trend.me),
 *        section "How it works: draft -> parallel verification ->
 *        accept/correct" (the four steps of a round, the 1..gamma+1 output
 *        guarantee, temperature as sampling from an adjusted distribution).
 *
 * What it computes, for each sequence b of the batch, in the pages' order:
 *   1. q_j = softmax(target_logits[b, j, :] / T) for j = 0..gamma and
 *      p_j = softmax(draft_logits[b, j, :] / T) for j = 0..gamma-1
 *      ([P2] sec. 1 notation; [P3] "how it works", temperature remark).
 *   2. Left to right over j = 0..gamma-1 with t = draft_tokens[b, j]: accept
 *      when u_accept[b, j] < q_j(t) / p_j(t), i.e. with probability
 *      min(1, q/p); stop at the first rejection ([P2] sec. 1 rule; [P3]
 *      "how it works", third step).  n = number accepted.
 *   3. If n < gamma: draw from max(0, q_n - p_n) / ||max(0, q_n - p_n)||_1
 *      ([P2] sec. 1 rule; [P3] fourth step).
 *   4. If n == gamma: draw one bonus token from q_gamma ([P3] fourth step,
 *      last sentence).
 *   Emit the n accepted drafts and the drawn token: 1..gamma+1 tokens
 *   ([P3] "how it works", guarantee paragraph; [P2] sec. 3).
 *
 * Readings where the pages leave a step open (each one restated in the
 * design notes of the repository):
 *   - acceptance test is the strict comparison u < ratio with u in [0, 1);
 *     q(t) == 0 gives ratio 0, p(t) == 0 < q(t) gives ratio +inf;
 *   - the draw in steps 3/4 is the inverse CDF of the unnormalised mass r
 *     with the caller's uniform u: the smallest index i with
 *     C_i = sum_{k<=i} r_k  >  u * Z, Z = sum_k r_k; if rounding leaves no
 *     such index, the last index with r_i > 0;
 *   - Z == 0 at a rejection (only reachable through rounding) falls back to
 *     a draw from q_n and raises the ZERO_MASS warning;
 *   - a draft token outside [0, V), or any row of the sequence holding NaN
 *     or +inf or no finite entry, is a data error: the sequence emits
 *     nothing (num_accepted 0, all tokens -1) and carries the error code;
 *   - output positions after the drawn token are padded with -1.
 *
 * Everything is computed in double precision with sequential loops.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_DTYPE_F32 0
#define ORACLE_DTYPE_BF16 1
#define ORACLE_DTYPE_F64 2 /* logits computed exactly from an output layer */

#define ORACLE_OK 0
#define ORACLE_ERR_TOKEN_RANGE 16
#define ORACLE_ERR_NONFINITE 17
#define ORACLE_WARN_ZERO_MASS 18

/* Inputs of one verification call (host memory). */
typedef struct {
  int batch;                 /* B */
  int gamma;                 /* number of draft positions */
  int vocab;                 /* V */
  int dtype;                 /* ORACLE_DTYPE_F32 or ORACLE_DTYPE_BF16 (raw bits) */
  const void *target_logits; /* [B, gamma+1, V] */
  const void *draft_logits;  /* [B, gamma, V] */
  const int32_t *draft_tokens; /* [B, gamma] */
  const float *u_accept;     /* [B, gamma] */
  const float *u_resample;   /* [B] */
  double temperature;        /* T > 0 */
} oracle_problem;

/* Outputs.  Every pointer except out_tokens / out_num_accepted may be NULL. */
typedef struct {
  int32_t *out_tokens;       /* [B, gamma+1] */
  int32_t *out_num_accepted; /* [B] */
  int32_t *seq_status;       /* [B] ORACLE_* code per sequence */
  double *target_max;        /* [B, gamma+1]  max_i x_i (raw logits) */
  double *target_sum;        /* [B, gamma+1]  sum_i exp((x_i - max)/T) */
  double *draft_max;         /* [B, gamma] */
  double *draft_sum;         /* [B, gamma] */
  double *q_tok;             /* [B, gamma]  q_j(t_j) */
  double *p_tok;             /* [B, gamma]  p_j(t_j) */
  double *ratio;             /* [B, gamma]  q_j(t_j)/p_j(t_j) */
  double *accept_margin;     /* [B, gamma]  |u - ratio| at tested positions, NaN after */
  double *resid_mass;        /* [B]  Z of the drawn-from distribution */
  double *cdf_margin_mass;   /* [B]  distance of u*Z to the chosen interval's ends */
  double *cdf_margin_norm;   /* [B]  the same divided by Z */
  int32_t *sampled;          /* [B]  the drawn token (residual or bonus) */
} oracle_result;

/* bf16 is the upper half of an IEEE binary32 word. */
static double oracle_bf16_to_double(uint16_t bits) {
  uint32_t w = ((uint32_t)bits) << 16;
  float f;
  memcpy(&f, &w, sizeof f);
  return (double)f;
}

static double oracle_load(const void *base, int dtype, size_t index) {
  if (dtype == ORACLE_DTYPE_BF16)
    return oracle_bf16_to_double(((const uint16_t *)base)[index]);
  if (dtype == ORACLE_DTYPE_F64) return ((const double *)base)[index];
  return (double)((const float *)base)[index];
}

/*
 * Softmax of one row at temperature T ([P2] sec. 1 notation, [P3] temperature
 * remark): y_i = x_i / T, m = max y, e_i = exp(y_i - m), S = sum e_i,
 * prob_i = e_i / S.  Returns 0 when the row is valid, ORACLE_ERR_NONFINITE
 * when it holds NaN or +inf or no finite entry.  *raw_max receives max_i x_i
 * and *sum receives S.
 */
int oracle_softmax_row(const void *base, int dtype, size_t offset, int V,
                       double T, double *prob, double *raw_max, double *sum) {
  int i;
  double mx = -INFINITY;
  for (i = 0; i < V; ++i) {
    double x = oracle_load(base, dtype, offset + (size_t)i);
    if (isnan(x) || (isinf(x) && x > 0)) return ORACLE_ERR_NONFINITE;
    if (x > mx) mx = x;
  }
  if (!isfinite(mx)) return ORACLE_ERR_NONFINITE; /* every entry is -inf */
  /* x/T is monotone in x for T > 0, so max_i (x_i/T) == (max_i x_i)/T */
  double m = mx / T;
  double S = 0.0;
  for (i = 0; i < V; ++i) {
    double y = oracle_load(base, dtype, offset + (size_t)i) / T;
    double e = exp(y - m);
    prob[i] = e;
    S += e;
  }
  for (i = 0; i < V; ++i) prob[i] = prob[i] / S;
  if (raw_max) *raw_max = mx;
  if (sum) *sum = S;
  return ORACLE_OK;
}

/*
 * Inverse-CDF draw from the unnormalised mass r[0..V-1] with uniform u:
 * the smallest i with C_i > u * Z; if rounding leaves none, the last i with
 * r_i > 0.  Also reports Z and the distance of u*Z to the chosen interval's
 * ends (in mass and divided by Z).
 */
static int oracle_draw(const double *r, int V, double u, double *Z_out,
                       double *margin_mass, double *margin_norm) {
  int i;
  double Z = 0.0;
  for (i = 0; i < V; ++i) Z += r[i];
  double target = u * Z;
  double C = 0.0;
  int chosen = -1;
  double lo = 0.0, hi = 0.0;
  for (i = 0; i < V; ++i) {
    double before = C;
    C += r[i];
    if (r[i] > 0.0 && C > target) {
      chosen = i;
      lo = before;
      hi = C;
      break;
    }
  }
  if (chosen < 0) {
    C = 0.0;
    for (i = 0; i < V; ++i) {
      if (r[i] > 0.0) {
        chosen = i;
        lo = C;
        hi = C + r[i];
      }
      C += r[i];
    }
  }
  double mm = fmin(fabs(target - lo), fabs(hi - target));
  if (Z_out) *Z_out = Z;
  if (margin_mass) *margin_mass = mm;
  if (margin_norm) *margin_norm = (Z > 0.0) ? mm / Z : 0.0;
  return chosen;
}

static void put(double *arr, size_t idx, double v) {
  if (arr) arr[idx] = v;
}

/*
 * Verify sequences b in [b_begin, b_end).  Returns the number of sequences
 * that carry a data error (ORACLE_ERR_*), or -1 on allocation failure.
 */
int oracle_verify(const oracle_problem *P, const oracle_result *R, int b_begin,
                  int b_end) {
  const int G = P->gamma, V = P->vocab;
  const double T = P->temperature;
  int errors = 0;
  double *q = (double *)malloc(sizeof(double) * (size_t)(G + 1) * (size_t)V);
  double *p = (double *)malloc(sizeof(double) * (size_t)(G > 0 ? G : 1) * (size_t)V);
  double *r = (double *)malloc(sizeof(double) * (size_t)V);
  if (!q || !p || !r) {
    free(q); free(p); free(r);
    return -1;
  }
  for (int b = b_begin; b < b_end; ++b) {
    int status = ORACLE_OK;
    int j;
    /* Step 1: all softmaxes of the sequence. */
    for (j = 0; j <= G; ++j) {
      double mx = NAN, sm = NAN;
      size_t off = ((size_t)b * (size_t)(G + 1) + (size_t)j) * (size_t)V;
      int st = oracle_softmax_row(P->target_logits, P->dtype, off, V, T,
                                  q + (size_t)j * V, &mx, &sm);
      if (st != ORACLE_OK) status = st;
      put(R->target_max, (size_t)b * (G + 1) + j, mx);
      put(R->target_sum, (size_t)b * (G + 1) + j, sm);
    }
    for (j = 0; j < G; ++j) {
      double mx = NAN, sm = NAN;
      size_t off = ((size_t)b * (size_t)G + (size_t)j) * (size_t)V;
      int st = oracle_softmax_row(P->draft_logits, P->dtype, off, V, T,
                                  p + (size_t)j * V, &mx, &sm);
      if (st != ORACLE_OK) status = st;
      put(R->draft_max, (size_t)b * G + j, mx);
      put(R->draft_sum, (size_t)b * G + j, sm);
    }
    for (j = 0; j < G; ++j) {
      int t = P->draft_tokens[(size_t)b * G + j];
      if (t < 0 || t >= V) status = ORACLE_ERR_TOKEN_RANGE;
    }
    for (j = 0; j < G; ++j) {
      put(R->q_tok, (size_t)b * G + j, NAN);
      put(R->p_tok, (size_t)b * G + j, NAN);
      put(R->ratio, (size_t)b * G + j, NAN);
      put(R->accept_margin, (size_t)b * G + j, NAN);
    }
    int32_t *toks = R->out_tokens + (size_t)b * (G + 1);
    for (j = 0; j <= G; ++j) toks[j] = -1;
    if (status != ORACLE_OK) {
      R->out_num_accepted[b] = 0;
      if (R->seq_status) R->seq_status[b] = status;
      put(R->resid_mass, b, NAN);
      put(R->cdf_margin_mass, b, NAN);
      put(R->cdf_margin_norm, b, NAN);
      if (R->sampled) R->sampled[b] = -1;
      ++errors;
      continue;
    }
    /* Step 2: left-to-right acceptance, stop at the first rejection. */
    int n = G;
    for (j = 0; j < G; ++j) {
      int t = P->draft_tokens[(size_t)b * G + j];
      double qt = q[(size_t)j * V + t];
      double pt = p[(size_t)j * V + t];
      double ratio;
      if (qt == 0.0) ratio = 0.0;
      else if (pt == 0.0) ratio = INFINITY;
      else ratio = qt / pt;
      double u = (double)P->u_accept[(size_t)b * G + j];
      put(R->q_tok, (size_t)b * G + j, qt);
      put(R->p_tok, (size_t)b * G + j, pt);
      put(R->ratio, (size_t)b * G + j, ratio);
      put(R->accept_margin, (size_t)b * G + j, fabs(u - ratio));
      if (u < ratio) {
        toks[j] = t;
      } else {
        n = j;
        break;
      }
    }
    /* Steps 3/4: residual draw at the rejection, else the bonus draw. */
    int i;
    if (n < G) {
      for (i = 0; i < V; ++i) {
        double d = q[(size_t)n * V + i] - p[(size_t)n * V + i];
        r[i] = d > 0.0 ? d : 0.0;
      }
    } else {
      for (i = 0; i < V; ++i) r[i] = q[(size_t)G * V + i];
    }
    double Z = 0.0;
    for (i = 0; i < V; ++i) Z += r[i];
    if (!(Z > 0.0)) {
      /* only reachable at a rejection through rounding: draw from q_n */
      for (i = 0; i < V; ++i) r[i] = q[(size_t)n * V + i];
      status = ORACLE_WARN_ZERO_MASS;
    }
    double mm = NAN, mn = NAN;
    double u = (double)P->u_resample[b];
    int tok = oracle_draw(r, V, u, &Z, &mm, &mn);
    toks[n] = tok;
    R->out_num_accepted[b] = n;
    if (R->seq_status) R->seq_status[b] = status;
    put(R->resid_mass, b, Z);
    put(R->cdf_margin_mass, b, mm);
    put(R->cdf_margin_norm, b, mn);
    if (R->sampled) R->sampled[b] = tok;
  }
  free(q);
  free(p);
  free(r);
  return errors;
}
