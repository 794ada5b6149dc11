/*
 * Plain CPU oracle for the verification step under sampling variants: greedy
 * (argmax), top-k, nucleus (top-p) and a temperature per sequence.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may call, link or
 * load this file: only the test suite, the smoke check and the benchmark's
 * CPU-baseline leg use it.  It shares no code, header or constant with the
 * CUDA library.
 *
 * Source (page, section): "Speculative decoding: how to run big models fast"
 * (ai-trend.me), section "How it works", guarantee paragraph: argmax, top-k,
 * nucleus and temperature sampling can all be written as standard sampling
 * from an adjusted distribution, so the same verification rule handles them.
 * The rule itself is the one of "Speculative decoding - the small model
 * writes first and the big model checks" (blog.mna-game.duckdns.org, post
 * 46), section 1, applied to the adjusted q and p.
 *
 * The adjusted distribution of a row x (V logits) for temperature T, top_k and
 * top_p (readings of what the pages leave open, each listed in the design
 * notes):
 *   T == 0 (greedy): the point mass on the first index of the largest logit;
 *     top_k and top_p do not change it.
 *   T > 0:
 *     1. w_i = exp(x_i / T) (relative to the row maximum), the temperature
 *        softmax;
 *     2. top_k in (0, V): keep the entries with x_i >= the k-th largest logit
 *        (counted with multiplicity; entries tied with it are kept too);
 *     3. top_p in (0, 1): over the entries kept by step 2, renormalised, go
 *        through the distinct logit values from the largest down and stop at
 *        the first value v whose cumulative mass (all entries >= v) reaches
 *        top_p; keep the entries >= v.  Ties at v are all kept;
 *     4. the adjusted distribution is w restricted to the kept entries and
 *        renormalised.
 *   The same T, top_k and top_p adjust the draft rows p_j and the target rows
 *   q_j of the sequence.
 * Then, as in the plain step: accept t_j when u_accept < q_j(t_j) / p_j(t_j)
 * (q(t) == 0 gives 0, p(t) == 0 < q(t) gives +inf), stop at the first
 * rejection n, draw from max(0, q_n - p_n) (or from q_gamma when every draft
 * is accepted) as the smallest index whose cumulative mass exceeds
 * u_resample times the total, falling back to the last positive index, and
 * to q_n with a warning when the residual has no mass.
 *
 * Errors (the sequence emits nothing): a draft token outside [0, V), a row
 * holding NaN or +inf or no finite entry, a temperature that is negative or
 * not finite (status 21).
 *
 * Everything is computed in double precision with sequential loops; the only
 * library step is qsort.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define SAMP_OK 0
#define SAMP_ERR_TOKEN_RANGE 16
#define SAMP_ERR_NONFINITE 17
#define SAMP_WARN_ZERO_MASS 18
#define SAMP_ERR_TEMPERATURE 21

typedef struct {
  int batch, gamma, vocab;
  int dtype;                   /* 0: float32, 1: bf16 bits */
  const void *target_logits;   /* [B, gamma+1, V] */
  const void *draft_logits;    /* [B, gamma, V] */
  const int32_t *draft_tokens; /* [B, gamma] */
  const float *u_accept;       /* [B, gamma] */
  const float *u_resample;     /* [B] */
  const float *temperature;    /* [B] */
  int top_k;                   /* 0 or >= V: off */
  double top_p;                /* >= 1: off */
} samp_problem;

/* Every pointer except out_tokens / out_num_accepted may be NULL. */
typedef struct {
  int32_t *out_tokens;         /* [B, gamma+1] */
  int32_t *out_num_accepted;   /* [B] */
  int32_t *seq_status;         /* [B] */
  double *q_tok;               /* [B, gamma] adjusted q_j(t_j) of tested positions, else NaN */
  double *p_tok;               /* [B, gamma] */
  double *accept_margin;       /* [B, gamma] |u - ratio| of tested positions */
  double *resid_mass;          /* [B] mass of the drawn-from vector (sums to 1 for q) */
  double *cdf_margin_norm;     /* [B] distance of u to the drawn token's CDF interval ends */
  int32_t *kept_target;        /* [B, gamma+1] entries kept by the filters */
  int32_t *kept_draft;         /* [B, gamma] */
  double *filter_margin;       /* [B] smallest top-p boundary margin over the sequence's rows */
} samp_result;

static double samp_value(const void *base, int dtype, size_t i) {
  if (dtype == 1) {
    uint32_t bits = (uint32_t)((const uint16_t *)base)[i] << 16;
    float f;
    memcpy(&f, &bits, sizeof f);
    return (double)f;
  }
  return (double)((const float *)base)[i];
}

typedef struct {
  double x;
  int i;
} samp_entry;

/* descending by logit, ties by ascending index */
static int samp_cmp(const void *a, const void *b) {
  const samp_entry *p = (const samp_entry *)a, *q = (const samp_entry *)b;
  if (p->x > q->x) return -1;
  if (p->x < q->x) return 1;
  return (p->i > q->i) - (p->i < q->i);
}

/*
 * The adjusted distribution of one row into prob[V].  Returns SAMP_OK or
 * SAMP_ERR_NONFINITE; *kept = entries with prob > 0 or kept by the filters;
 * *margin = top-p boundary margin (+inf when top-p does not apply).
 */
static int samp_row(const void *base, int dtype, size_t off, int V, double T, int top_k,
                    double top_p, double *prob, samp_entry *work, int *kept, double *margin) {
  *margin = INFINITY;
  double mx = -INFINITY;
  int arg = -1;
  for (int i = 0; i < V; ++i) {
    const double x = samp_value(base, dtype, off + (size_t)i);
    if (isnan(x) || x == INFINITY) return SAMP_ERR_NONFINITE;
    if (x > mx) {
      mx = x;
      arg = i;
    }
  }
  if (arg < 0 || mx == -INFINITY) return SAMP_ERR_NONFINITE;
  if (T == 0.0) {
    for (int i = 0; i < V; ++i) prob[i] = 0.0;
    prob[arg] = 1.0;
    *kept = 1;
    return SAMP_OK;
  }
  /* step 1: temperature weights */
  for (int i = 0; i < V; ++i) {
    const double x = samp_value(base, dtype, off + (size_t)i);
    prob[i] = exp((x - mx) / T);
  }
  /* step 2: the k-th largest logit */
  double theta = -INFINITY;
  const int use_k = top_k > 0 && top_k < V;
  const int use_p = top_p < 1.0;
  if (use_k || use_p) {
    for (int i = 0; i < V; ++i) {
      work[i].x = samp_value(base, dtype, off + (size_t)i);
      work[i].i = i;
    }
    qsort(work, (size_t)V, sizeof(samp_entry), samp_cmp);
  }
  if (use_k) theta = work[top_k - 1].x;
  /* step 3: nucleus over the entries >= theta, by distinct values */
  if (use_p) {
    double Z = 0.0;
    for (int i = 0; i < V; ++i)
      if (work[i].x >= theta) Z += prob[work[i].i];
    double above = 0.0; /* mass of the values strictly above the current one */
    int a = 0;
    while (a < V && work[a].x >= theta) {
      int e = a;
      double group = 0.0;
      while (e < V && work[e].x == work[a].x) group += prob[work[e++].i];
      const double before = above / Z, after = (above + group) / Z;
      if (after >= top_p || e >= V || work[e].x < theta) {
        theta = work[a].x;
        const double m1 = top_p - before, m2 = after - top_p;
        *margin = m1 < m2 ? m1 : m2;
        break;
      }
      above += group;
      a = e;
    }
  }
  /* step 4: restrict and renormalise */
  double Z = 0.0;
  int n = 0;
  for (int i = 0; i < V; ++i) {
    const double x = samp_value(base, dtype, off + (size_t)i);
    if (x >= theta && x != -INFINITY) {
      Z += prob[i];
      ++n;
    } else {
      prob[i] = 0.0;
    }
  }
  for (int i = 0; i < V; ++i) prob[i] /= Z;
  *kept = n;
  return SAMP_OK;
}

/* smallest i with C_i > u Z, else the last positive index; -1 if Z == 0 */
static int samp_draw(const double *r, int V, double u, double *Z_out, double *margin) {
  double Z = 0.0;
  for (int i = 0; i < V; ++i) Z += r[i];
  *Z_out = Z;
  *margin = NAN;
  if (!(Z > 0.0)) return -1;
  const double target = u * Z;
  double C = 0.0;
  int last = -1;
  for (int i = 0; i < V; ++i) {
    if (r[i] > 0.0) last = i;
    const double before = C;
    C += r[i];
    if (r[i] > 0.0 && C > target) {
      const double lo = fabs(u - before / Z), hi = fabs(C / Z - u);
      *margin = lo < hi ? lo : hi;
      return i;
    }
  }
  *margin = 0.0;
  return last;
}

static void samp_put(double *a, size_t i, double v) {
  if (a) a[i] = v;
}

int oracle_verify_sampling(const samp_problem *P, const samp_result *R, int b_begin, int b_end) {
  const int G = P->gamma, V = P->vocab;
  int errors = 0;
  double *q = (double *)malloc(sizeof(double) * (size_t)V * (size_t)(G + 1));
  double *p = (double *)malloc(sizeof(double) * (size_t)V * (size_t)(G > 0 ? G : 1));
  double *r = (double *)malloc(sizeof(double) * (size_t)V);
  samp_entry *work = (samp_entry *)malloc(sizeof(samp_entry) * (size_t)V);
  if (!q || !p || !r || !work) {
    free(q);
    free(p);
    free(r);
    free(work);
    return -1;
  }
  for (int b = b_begin; b < b_end; ++b) {
    const double T = (double)P->temperature[b];
    int status = SAMP_OK;
    double fmargin = INFINITY;
    for (int j = 0; j < G; ++j) {
      samp_put(R->q_tok, (size_t)b * G + j, NAN);
      samp_put(R->p_tok, (size_t)b * G + j, NAN);
      samp_put(R->accept_margin, (size_t)b * G + j, NAN);
    }
    if (!(T >= 0.0) || isinf(T)) status = SAMP_ERR_TEMPERATURE;
    /* the adjusted distributions of every row of the sequence */
    for (int j = 0; status == SAMP_OK && j <= G; ++j) {
      int kept;
      double m;
      const int st = samp_row(P->target_logits, P->dtype, ((size_t)b * (G + 1) + j) * (size_t)V,
                              V, T, P->top_k, P->top_p, q + (size_t)j * V, work, &kept, &m);
      if (st != SAMP_OK) status = st;
      if (R->kept_target) R->kept_target[(size_t)b * (G + 1) + j] = st == SAMP_OK ? kept : 0;
      if (m < fmargin) fmargin = m;
    }
    for (int j = 0; status == SAMP_OK && j < G; ++j) {
      int kept;
      double m;
      const int st = samp_row(P->draft_logits, P->dtype, ((size_t)b * G + j) * (size_t)V, V, T,
                              P->top_k, P->top_p, p + (size_t)j * V, work, &kept, &m);
      if (st != SAMP_OK) status = st;
      if (R->kept_draft) R->kept_draft[(size_t)b * G + j] = st == SAMP_OK ? kept : 0;
      if (m < fmargin) fmargin = m;
    }
    for (int j = 0; status == SAMP_OK && j < G; ++j) {
      const int t = P->draft_tokens[(size_t)b * G + j];
      if (t < 0 || t >= V) status = SAMP_ERR_TOKEN_RANGE;
    }
    if (R->filter_margin) R->filter_margin[b] = fmargin;
    if (status != SAMP_OK && status != SAMP_WARN_ZERO_MASS) {
      for (int j = 0; j <= G; ++j) R->out_tokens[(size_t)b * (G + 1) + j] = -1;
      R->out_num_accepted[b] = 0;
      if (R->seq_status) R->seq_status[b] = status;
      samp_put(R->resid_mass, (size_t)b, NAN);
      samp_put(R->cdf_margin_norm, (size_t)b, NAN);
      ++errors;
      continue;
    }
    /* left-to-right acceptance */
    int n = G;
    for (int j = 0; j < G; ++j) {
      const int t = P->draft_tokens[(size_t)b * G + j];
      const double qt = q[(size_t)j * V + t], pt = p[(size_t)j * V + t];
      double ratio;
      if (qt == 0.0) ratio = 0.0;
      else if (pt == 0.0) ratio = INFINITY;
      else ratio = qt / pt;
      const double u = (double)P->u_accept[(size_t)b * G + j];
      samp_put(R->q_tok, (size_t)b * G + j, qt);
      samp_put(R->p_tok, (size_t)b * G + j, pt);
      samp_put(R->accept_margin, (size_t)b * G + j, fabs(u - ratio));
      if (!(u < ratio)) {
        n = j;
        break;
      }
    }
    /* residual or bonus draw */
    const double *qn = q + (size_t)n * V;
    if (n < G) {
      const double *pn = p + (size_t)n * V;
      for (int i = 0; i < V; ++i) r[i] = qn[i] > pn[i] ? qn[i] - pn[i] : 0.0;
    } else {
      for (int i = 0; i < V; ++i) r[i] = qn[i];
    }
    double Z, cm;
    const double u = (double)P->u_resample[b];
    int s = samp_draw(r, V, u, &Z, &cm);
    if (s < 0) {
      status = SAMP_WARN_ZERO_MASS;
      for (int i = 0; i < V; ++i) r[i] = qn[i];
      s = samp_draw(r, V, u, &Z, &cm);
    }
    for (int j = 0; j < n; ++j)
      R->out_tokens[(size_t)b * (G + 1) + j] = P->draft_tokens[(size_t)b * G + j];
    R->out_tokens[(size_t)b * (G + 1) + n] = s;
    for (int j = n + 1; j <= G; ++j) R->out_tokens[(size_t)b * (G + 1) + j] = -1;
    R->out_num_accepted[b] = n;
    if (R->seq_status) R->seq_status[b] = status;
    samp_put(R->resid_mass, (size_t)b, Z);
    samp_put(R->cdf_margin_norm, (size_t)b, cm);
  }
  free(q);
  free(p);
  free(r);
  free(work);
  return errors;
}
