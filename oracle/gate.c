/*
 * Plain CPU oracle for the multi-branch fold gate (hidden-state difference
 * test, fold provenance, packing of the positions to recompute).
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may call, link or
 * load this file: only the test suite, the smoke check and the benchmark's
 * CPU-baseline leg use it.  It shares no code, header or constant with the
 * CUDA library.
 *
 * Source (page, section): the SpecFold explainer (blog.ontle.kr, post 356):
 *   - the observation paragraph: child and parent candidates are compared by
 *     the relative difference ||H_child - H_parent|| / ||H_parent|| of their
 *     hidden states, measured at the input of the same layer and position;
 *   - the per-position path (measure, reuse the parent, keep the own
 *     difference, recompute when needed) and the paragraph after it: the
 *     positions whose difference exceeds the threshold tau are gathered from
 *     all branches into one packed batch, so the heavy layer runs once;
 *   - the implementer's note: the gate kernel measures the cross-branch
 *     hidden-state difference and records where each folded position comes
 *     from; a resolution step follows the fold chain to the real parent state.
 *
 * What it computes for hidden states H [branches, positions, dim] and a
 * parent index per branch (-1: the branch has no parent):
 *   1. A branch is valid when its parent is -1, or in [0, branches), not the
 *      branch itself, and following parents from it reaches -1 within
 *      `branches` steps.  An invalid branch is treated as a branch without a
 *      parent and raises ORACLE_GATE_ERR_PARENT.
 *   2. For each row (c, j), with P = parent of c:
 *        no parent:  d = +inf;
 *        otherwise:  d = ||H[c, j] - H[P, j]||_2 / ||H[P, j]||_2, with
 *                    0/0 read as 0 and x/0 (x > 0) as +inf.
 *      A row without a parent is always recomputed; any other row is
 *      recomputed unless d <= tau (so NaN recomputes).
 *   3. provenance(c, j) = P * positions + j for a folded row, -1 for a
 *      recomputed one; source(c, j) = the recomputed row reached by
 *      following provenance (the row itself when recomputed).
 *   4. packed = the recomputed rows in ascending row order, and their count.
 *   Also returned: margin(c, j) = |d - tau| / tau (relative distance of the
 *   decision from the threshold; +inf for rows without a parent).
 *
 * Readings where the page is silent or garbled: the row order of the packed
 * batch (ascending), the handling of invalid parents and of zero or
 * non-finite norms (above), and the use of the immediate parent's state at
 * the same position as the comparison partner.  The "keep the own difference"
 * step is garbled on the page and is not part of the gate.
 *
 * Everything is computed in double precision with sequential loops.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_GATE_OK 0
#define ORACLE_GATE_ERR_PARENT 20

typedef struct {
  int branches;          /* number of candidate branches */
  int positions;         /* positions per branch */
  int dim;               /* hidden size */
  int dtype;             /* 0: float32, 1: bf16 bits */
  const void *hidden;    /* [branches, positions, dim] */
  const int32_t *parent; /* [branches] */
  double tau;            /* threshold, >= 0 */
} oracle_gate_problem;

/* Every pointer may be NULL except packed and n_packed. */
typedef struct {
  double *rel_diff;      /* [rows] */
  double *margin;        /* [rows] */
  int32_t *recompute;    /* [rows] 0 / 1 */
  int32_t *provenance;   /* [rows] */
  int32_t *source;       /* [rows] */
  int32_t *packed;       /* [rows], first n_packed entries used */
  int32_t *n_packed;     /* [1] */
  int32_t *parent_used;  /* [branches] parent after validation (-1 for invalid) */
} oracle_gate_result;

static double gate_value(const void *base, int dtype, size_t index) {
  if (dtype == 1) {
    uint32_t bits = (uint32_t)((const uint16_t *)base)[index] << 16;
    float f;
    memcpy(&f, &bits, sizeof f);
    return (double)f;
  }
  return (double)((const float *)base)[index];
}

/* Returns ORACLE_GATE_OK, or ORACLE_GATE_ERR_PARENT if some parent entry was
 * invalid (the outputs are complete either way), or -1 if out of memory. */
int oracle_gate(const oracle_gate_problem *P, const oracle_gate_result *R) {
  const int nb = P->branches, np = P->positions, D = P->dim;
  const long rows = (long)nb * np;
  int status = ORACLE_GATE_OK;
  int32_t *par = (int32_t *)malloc(sizeof(int32_t) * (size_t)(nb > 0 ? nb : 1));
  int32_t *rec = (int32_t *)malloc(sizeof(int32_t) * (size_t)(rows > 0 ? rows : 1));
  int32_t *prov = (int32_t *)malloc(sizeof(int32_t) * (size_t)(rows > 0 ? rows : 1));
  if (!par || !rec || !prov) {
    free(par);
    free(rec);
    free(prov);
    return -1;
  }

  /* step 1: validate the parent of every branch by walking its chain */
  for (int c = 0; c < nb; ++c) {
    int ok = 1, at = c, steps = 0;
    while (P->parent[at] != -1) {
      const int nx = P->parent[at];
      if (nx < 0 || nx >= nb || nx == at || ++steps > nb) {
        ok = 0;
        break;
      }
      at = nx;
    }
    if (!ok) status = ORACLE_GATE_ERR_PARENT;
    par[c] = ok ? P->parent[c] : -1;
    if (R->parent_used) R->parent_used[c] = par[c];
  }

  /* steps 2-3: the difference test and the immediate provenance of each row */
  for (int c = 0; c < nb; ++c) {
    for (int j = 0; j < np; ++j) {
      const long row = (long)c * np + j;
      double d;
      if (par[c] < 0) {
        d = INFINITY;
      } else {
        const size_t oc = (size_t)row * (size_t)D;
        const size_t op = ((size_t)par[c] * (size_t)np + (size_t)j) * (size_t)D;
        double num = 0.0, den = 0.0;
        for (int k = 0; k < D; ++k) {
          const double hc = gate_value(P->hidden, P->dtype, oc + (size_t)k);
          const double hp = gate_value(P->hidden, P->dtype, op + (size_t)k);
          num += (hc - hp) * (hc - hp);
          den += hp * hp;
        }
        if (den == 0.0) d = (num == 0.0) ? 0.0 : INFINITY;
        else d = sqrt(num) / sqrt(den);
      }
      rec[row] = (par[c] < 0) || !(d <= P->tau);
      prov[row] = rec[row] ? -1 : (int32_t)((long)par[c] * np + j);
      if (R->rel_diff) R->rel_diff[row] = d;
      if (R->margin) {
        if (isinf(d) || isnan(d)) R->margin[row] = INFINITY;
        else R->margin[row] = (P->tau > 0.0) ? fabs(d - P->tau) / P->tau : fabs(d - P->tau);
      }
      if (R->recompute) R->recompute[row] = rec[row];
      if (R->provenance) R->provenance[row] = prov[row];
    }
  }

  /* step 3: follow the fold chain of every folded row to a recomputed row */
  if (R->source) {
    for (long row = 0; row < rows; ++row) {
      long at = row;
      while (!rec[at]) at = prov[at];
      R->source[row] = (int32_t)at;
    }
  }

  /* step 4: the recomputed rows, ascending */
  int32_t n = 0;
  for (long row = 0; row < rows; ++row)
    if (rec[row]) R->packed[n++] = (int32_t)row;
  *R->n_packed = n;

  free(par);
  free(rec);
  free(prov);
  return status;
}
