/*
 * specverify_lmhead: the verification step fused with the LM head, on the
 * tensor cores of NVIDIA B200 (sm_100a).
 *
 * The operation is the one of specverify.h ("Speculative decoding - the small
 * model writes first and the big model checks", section 1; "Speculative
 * decoding: how to run big models fast", section "How it works") with the
 * logits produced by the models' output layer:
 *   target_logits[b, j, :] = target_hidden[b, j, :] . target_weight^T,  j = 0..gamma
 *   draft_logits[b, j, :]  = draft_hidden[b, j, :]  . draft_weight^T,   j = 0..gamma-1
 * (bf16 inputs, fp32 accumulation on tcgen05 tensor cores).  The page's
 * bandwidth argument for verification (one read of the parameters scores many
 * positions) is what the fusion exploits: the softmax statistics and the
 * draft tokens' logits are taken from each 128 x 256 accumulator tile in
 * tensor memory.  The draw needs the fp32 logits of two rows per sequence
 * (its target and draft rows at the first rejection, or the bonus row), known
 * only after the decision.  Two forms (specverify_lmhead_set_keep_logits):
 * kept logits (the default when the buffer takes at most 16 GB): the
 * statistics GEMMs also store every row's fp32 logits, which the GEMM's
 * tensor-bound time leaves the memory bandwidth to write, and the draw reads
 * its rows there; recomputed: nothing but the statistics leaves tensor
 * memory, and a second GEMM over the output layer recomputes the drawn rows.
 *
 * Shapes: hidden is a multiple of 64 (<= 65536); vocab <= 65535 x 256.  Layouts
 * (device pointers, 16-byte aligned, row-major, contiguous):
 *   target_hidden [batch, gamma+1, hidden] bf16;  target_weight [vocab, hidden] bf16
 *   draft_hidden  [batch, gamma, hidden]   bf16;  draft_weight  [vocab, hidden] bf16
 *   draft_tokens, u_accept, u_resample, out_tokens, out_num_accepted as in
 *   specverify_run; temperature a host float, finite and > 0.
 * The two weights may be the same buffer (a shared output layer).
 *
 * Memory: the handle owns a workspace of per-(row, 256-column tile) partial
 * statistics (16 B each), the picked-out logits, the plain step's decision
 * records, 2 x batch x (hidden x 2 + vocab x 4) bytes for the drawn rows, and
 * with kept logits batch x (2 gamma + 1) x vocab x 4 bytes.
 * Errors: argument errors return before anything is enqueued; data errors set
 * the status word as in specverify.h; a tensor-core pipeline wait that gives
 * up (it never should) sets SV_ERR_PIPELINE instead of hanging.
 */
#ifndef SPECVERIFY_LMHEAD_H
#define SPECVERIFY_LMHEAD_H

#include <stdint.h>

#include "specverify.h"

#ifdef __cplusplus
extern "C" {
#endif

typedef struct specverify_lmhead_ctx *specverify_lmhead_t;

/* Create a handle for (batch, gamma, vocab, hidden) on `device`. */
sv_status specverify_lmhead_create(specverify_lmhead_t *out, int batch, int gamma, int vocab,
                                   int hidden, int device);

/* Kept logits (nonzero, allocating their buffer if the handle has none;
 * SV_ERR_OOM if that fails) or the recomputing form (zero).  Results are the
 * same: the drawn rows' logits come from the same tensor-core arithmetic.
 * Not stream-ordered: change it only while no run of the handle is in
 * flight. */
sv_status specverify_lmhead_set_keep_logits(specverify_lmhead_t h, int keep);
sv_status specverify_lmhead_get_keep_logits(specverify_lmhead_t h, int *keep);

/* Enqueue one fused step on `stream` (asynchronous). */
sv_status specverify_lmhead_run(specverify_lmhead_t h, const void *target_hidden,
                                const void *target_weight, const void *draft_hidden,
                                const void *draft_weight, const int32_t *draft_tokens,
                                const float *u_accept, const float *u_resample,
                                float temperature, int32_t *out_tokens,
                                int32_t *out_num_accepted, void *stream);

/* Diagnostic: the GEMM alone, out_logits [rows, vocab] fp32 = hidden_rows
 * [rows, hidden] bf16 . weight [vocab, hidden]^T (16-byte aligned pointers). */
sv_status specverify_lmhead_logits(specverify_lmhead_t h, const void *hidden_rows, int rows,
                                   const void *weight, float *out_logits, void *stream);

/* Wait for `stream`, read and clear the status: SV_ERR_PIPELINE, then the
 * data errors of specverify_get_status.  `*bits`: the data-error bits, plus 32
 * for a pipeline error. */
sv_status specverify_lmhead_get_status(specverify_lmhead_t h, void *stream, uint32_t *bits);

/* Wait for `stream`; copy log sum exp(x/T) of every target [batch, gamma+1]
 * and draft [batch, gamma] row, q(t) and p(t) of every draft position, and the
 * drawn-from mass per sequence into host arrays (any may be NULL). */
sv_status specverify_lmhead_readback(specverify_lmhead_t h, double *target_lse,
                                     double *draft_lse, double *q_tok, double *p_tok,
                                     double *resid_mass, void *stream);

/* CUDA-event timing of the next `max_runs` runs: the statistics GEMMs, and
 * the rest (decision, and the draw; without kept logits also the row gather
 * and the logit GEMMs), mean ms per run. */
sv_status specverify_lmhead_profile_begin(specverify_lmhead_t h, int max_runs);
sv_status specverify_lmhead_profile_end(specverify_lmhead_t h, float *stats_ms, float *rest_ms,
                                        int *runs);

/* Free the handle (waits for its device work).  NULL is ignored. */
void specverify_lmhead_destroy(specverify_lmhead_t h);

#ifdef __cplusplus
}
#endif

#endif /* SPECVERIFY_LMHEAD_H */
