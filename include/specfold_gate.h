/*
 * specfold_gate: the multi-branch fold gate on NVIDIA B200 (sm_100a).
 *
 * The operation (page and section that define it): the SpecFold explainer
 * (blog.ontle.kr, post 356).  Candidate branches that are verified together
 * differ from their parent branch in a few positions only.  Per layer, the
 * gate compares each branch's hidden state at the layer input with its
 * parent's at the same position by the relative difference
 *     d = ||H_child - H_parent||_2 / ||H_parent||_2
 * (the observation paragraph), reuses the parent's result where d is at most
 * the threshold tau, and gathers the positions above tau from all branches
 * into one packed batch so the heavy layer runs once on them (the per-position
 * path and the paragraph after it).  The gate records where every folded
 * position comes from, and a resolution step follows the fold chain to the
 * real parent state (the implementer's note).
 *
 * For hidden states H [branches, positions, dim] (row (c, j) = c * positions
 * + j) and parent[c] in {-1} U [0, branches):
 *   - branch c is valid if following parents from c reaches -1 within
 *     `branches` steps with every link in range and no self link; an invalid
 *     branch is handled as a branch without a parent and sets status bit 1;
 *   - d(c, j) = +inf for a branch without a parent, else the relative
 *     difference above with 0/0 = 0 and x/0 = +inf (x > 0);
 *   - a row of a branch without a parent is always recomputed; any other
 *     row (c, j) is recomputed unless d <= tau (NaN recomputes);
 *   - provenance(c, j) = parent[c] * positions + j for a folded row, -1 for
 *     a recomputed row;
 *   - source(c, j) = the recomputed row reached by following provenance (the
 *     row itself when it is recomputed);
 *   - packed_rows = the recomputed rows in ascending row order, n_packed their
 *     count; packed_hidden[k] = H row packed_rows[k] (the packed batch).
 * Sums of squares are accumulated in fp32 per lane and combined in fp64; the
 * decision d <= tau is taken in fp64.
 *
 * Memory: the caller owns every input and output.  A handle owns a small
 * device workspace (per-branch validated parents, per-row flags, provenance
 * and packed slots, a status word).  Errors: argument
 * errors return before anything is enqueued; a bad parent array never traps:
 * it sets status bit 1, read (and cleared) by specfold_gate_get_status.  On
 * 16-byte aligned rows of at most 50 KB the difference test streams row pairs
 * into shared memory by bulk copies; its waits are bounded (2 s), and a wait
 * that gives up (it never should) sets status bit 2 instead of hanging.
 */
#ifndef SPECFOLD_GATE_H
#define SPECFOLD_GATE_H

#include <stdint.h>

#include "specverify.h"

#ifdef __cplusplus
extern "C" {
#endif

typedef struct specfold_gate_ctx *specfold_gate_t;

/*
 * Create a gate handle for `branches` x `positions` rows of `dim` hidden
 * values stored as `dtype`, on CUDA device `device`.  1 <= branches <= 16384,
 * 1 <= positions, branches * positions < 2^31, 1 <= dim <= 2^20.  The
 * caller's current device is left unchanged.
 */
sv_status specfold_gate_create(specfold_gate_t *out, int branches, int positions, int dim,
                               sv_dtype dtype, int device);

/*
 * Enqueue one gate pass on `stream` (device pointers):
 *   hidden         [branches, positions, dim] dtype, row-major, contiguous
 *   parent         int32 [branches]
 *   tau            host value, >= 0 (may be +inf; not NaN)
 *   rel_diff       float [branches, positions] (written; may be NULL)
 *   provenance     int32 [branches, positions] (written; may be NULL)
 *   source         int32 [branches, positions] (written; may be NULL)
 *   packed_rows    int32 [branches * positions] (first n_packed entries written)
 *   n_packed       int32 [1] (written)
 *   packed_hidden  [branches * positions, dim] dtype (first n_packed rows
 *                  written; may be NULL)
 * `hidden` and `packed_hidden` must be aligned to the element size; 16-byte
 * alignment with dim * sizeof(dtype) a multiple of 16 takes 128-bit loads.
 * The call is asynchronous.
 */
sv_status specfold_gate_run(specfold_gate_t h, const void *hidden, const int32_t *parent,
                            float tau, float *rel_diff, int32_t *provenance, int32_t *source,
                            int32_t *packed_rows, int32_t *n_packed, void *packed_hidden,
                            void *stream);

/* Wait for `stream`, read and clear the status word: SV_ERR_PIPELINE if a
 * bounded wait of the difference test gave up since the last call, else
 * SV_ERR_PARENT if some parent entry was invalid, else SV_OK.  `*bits` (may
 * be NULL) receives the raw bits (1: invalid parent, 2: a wait gave up). */
sv_status specfold_gate_get_status(specfold_gate_t h, void *stream, uint32_t *bits);

/* Record CUDA events around each of the next `max_runs` runs' kernels
 * (0 stops recording). */
sv_status specfold_gate_profile_begin(specfold_gate_t h, int max_runs);

/* Wait for the recorded runs and return the mean device milliseconds per run
 * of the difference kernel (`rows_ms`) and of the slot scan plus the packing
 * kernel (`pack_ms`),
 * and the number of runs averaged. */
sv_status specfold_gate_profile_end(specfold_gate_t h, float *rows_ms, float *pack_ms, int *runs);

/* Free the handle (waits for its device work).  NULL is ignored. */
void specfold_gate_destroy(specfold_gate_t h);

#ifdef __cplusplus
}
#endif

#endif /* SPECFOLD_GATE_H */
