/*
 * specverify: batched speculative-sampling verification on NVIDIA B200 (sm_100a).
 *
 * The operation (page title and section that define it):
 *   "Speculative decoding - the small model writes first and the big model
 *   checks" (blog.mna-game.duckdns.org, deep-learning post 46), section 1:
 *   accept a draft token t with probability min(1, q(t)/p(t)); on rejection
 *   draw again from max(0, q - p) / ||max(0, q - p)||_1.
 *   "Speculative decoding: how to run big models fast" (ai-trend.me), section
 *   "How it works": check the drafts left to right, stop at the first rejection
 *   and discard the rest, append one token drawn from q at position gamma+1
 *   when every draft is accepted, so each call emits 1 .. gamma+1 tokens;
 *   temperature is handled as sampling from an adjusted distribution.
 *
 * For every sequence b of a batch of B:
 *   q_j = softmax(target_logits[b, j, :] / T),  j = 0 .. gamma
 *   p_j = softmax(draft_logits[b, j, :] / T),   j = 0 .. gamma-1
 *   n   = first j with  u_accept[b, j] >= q_j(t_j) / p_j(t_j)  (t_j =
 *         draft_tokens[b, j]), or gamma if there is none
 *   if n < gamma: r = max(0, q_n - p_n)   else: r = q_gamma
 *   s   = smallest i with  sum_{k<=i} r_k  >  u_resample[b] * sum_k r_k
 *   out_tokens[b, :] = t_0 .. t_{n-1}, s, -1, ..., -1     (gamma+1 entries)
 *   out_num_accepted[b] = n
 *
 * Conventions that the pages leave open:
 *   - the acceptance comparison is strict (u < ratio); q(t) == 0 gives ratio 0
 *     and p(t) == 0 < q(t) gives ratio +inf;
 *   - one uniform per sequence serves both the residual draw and the bonus
 *     draw, because exactly one of the two happens;
 *   - if rounding leaves no index with cumulative mass above u * Z, the draw
 *     returns the last index with r_i > 0; zero-mass tokens are never drawn;
 *   - if the residual mass is zero at a rejection, the draw falls back to q_n
 *     and the status word records SV_WARN_ZERO_MASS.  With draft tokens drawn
 *     from p, as the method requires, this is reachable only through rounding
 *     when q and p agree; a token that p gives no mass can also reach it (for
 *     instance under greedy sampling, a token that is not the draft's argmax
 *     while the two argmaxes agree);
 *   - a sequence with a draft token outside [0, V), or with any logit row
 *     holding NaN or +inf or no finite entry, emits nothing:
 *     out_num_accepted[b] = 0 and out_tokens[b, :] = -1, and the status word
 *     records SV_ERR_TOKEN_RANGE or SV_ERR_NONFINITE.  -inf logits are legal
 *     (masked vocabulary entries carry zero probability).
 *
 * Memory: the caller owns every input and output buffer.  A handle owns a
 * small device workspace (per-row statistics, per-position decisions, one
 * ticket per sequence, the status word), allocated by specverify_create and
 * freed by specverify_destroy.  Device buffers must be device memory of the
 * handle's device.  A handle may be used by one stream at a time.
 *
 * Errors: argument errors are reported before anything is enqueued.  Data
 * errors found on the device never trap or stall: they set bits of the
 * handle's status word, read back (and cleared) by specverify_get_status.
 *
 * Streams: `stream` is a cudaStream_t passed as void* (NULL is the legacy
 * default stream).  specverify_run only enqueues work and returns.
 */
#ifndef SPECVERIFY_H
#define SPECVERIFY_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct specverify_ctx *specverify_t;

typedef enum {
  SV_DTYPE_F32 = 0,  /* IEEE binary32 logits */
  SV_DTYPE_BF16 = 1  /* bfloat16 logits */
} sv_dtype;

typedef enum {
  SV_OK = 0,
  SV_ERR_INVALID_ARG = 1,  /* bad size, pointer, alignment, temperature or handle */
  SV_ERR_CUDA = 2,         /* a CUDA runtime call failed; see specverify_last_error() */
  SV_ERR_OOM = 3,          /* device or host allocation failed */
  SV_ERR_UNSUPPORTED = 4,  /* the device is not an sm_100 (B200-class) GPU */
  SV_ERR_TOKEN_RANGE = 16, /* device: some draft token was outside [0, V) */
  SV_ERR_NONFINITE = 17,   /* device: some logit row held NaN/+inf or only -inf */
  SV_WARN_ZERO_MASS = 18,  /* device: a residual had zero mass; drew from q_n instead */
  SV_ERR_ROW_INDEX = 19,   /* device: a row map entry was outside the rows given */
  SV_ERR_PARENT = 20,      /* device (fold gate): a parent entry out of range, a self link or a cycle */
  SV_ERR_TEMPERATURE = 21, /* device (sampling variants): a temperature < 0, NaN or infinite */
  SV_ERR_PIPELINE = 22,    /* device: a bounded wait gave up (LM-head pipeline, single-launch step) */
  SV_ERR_BOUNDS = 23       /* device, debug builds only (libspecverify_debug.so, compiled with
                              -DSV_DEBUG_BOUNDS=1): an index the kernels derived fell outside its
                              buffer; the access was skipped */
} sv_status;

/*
 * Create a handle for batches of `batch` sequences with `gamma` draft tokens
 * over a vocabulary of `vocab` entries stored as `dtype`, on CUDA device
 * `device`.  0 <= batch, 0 <= gamma <= 255, 1 <= vocab <= 2^30.
 * Allocates the workspace (per position: up to 64 partial statistics of
 * 32 bytes plus about 64 bytes; per sequence 16 bytes per 32 groups of 16
 * bytes of a row) and chooses a default launch shape.  The caller's current device is left
 * unchanged.  Returns SV_OK and stores the handle in *out, or an error and
 * leaves *out NULL.
 */
sv_status specverify_create(specverify_t *out, int batch, int gamma, int vocab,
                            sv_dtype dtype, int device);

/*
 * Enqueue one verification step on `stream` (device pointers):
 *   target_logits    [batch, gamma+1, vocab]  dtype, row-major, contiguous
 *   draft_logits     [batch, gamma,   vocab]  dtype, row-major, contiguous
 *   draft_tokens     int32 [batch, gamma], expected in [0, vocab)
 *   u_accept         float [batch, gamma], uniforms in [0, 1)
 *   u_resample       float [batch],        uniforms in [0, 1)
 *   temperature      host value, finite and > 0 (divides both logit tensors)
 *   out_tokens       int32 [batch, gamma+1] (written)
 *   out_num_accepted int32 [batch]          (written)
 * Logit pointers must be aligned to their element size; 16-byte aligned
 * pointers together with vocab * sizeof(dtype) a multiple of 16 take the
 * vectorised (128-bit load) path, anything else a scalar-load path.
 * Draft pointers may be NULL when gamma == 0; everything may be NULL when
 * batch == 0 (nothing is enqueued).  The call is asynchronous.
 */
sv_status specverify_run(specverify_t h, const void *target_logits,
                         const void *draft_logits, const int32_t *draft_tokens,
                         const float *u_accept, const float *u_resample,
                         float temperature, int32_t *out_tokens,
                         int32_t *out_num_accepted, void *stream);

/*
 * The same step on HOST buffers with the shapes of specverify_run (pinned
 * host memory gives full copy bandwidth).  Copies the inputs to a device
 * staging area owned by the handle (allocated on first use, freed by
 * specverify_destroy), runs the step, copies both outputs back and waits for
 * `stream`.  Returns after the outputs are in host memory.
 */
sv_status specverify_run_host(specverify_t h, const void *target_logits,
                              const void *draft_logits, const int32_t *draft_tokens,
                              const float *u_accept, const float *u_resample,
                              float temperature, int32_t *out_tokens,
                              int32_t *out_num_accepted, void *stream);

/*
 * The step under sampling variants.  Argmax, top-k, nucleus and temperature
 * sampling are standard sampling from an adjusted distribution, so the same
 * rule verifies them ("Speculative decoding: how to run big models fast",
 * section "How it works", guarantee paragraph).  Every target row q_j and draft
 * row p_j of sequence b is replaced by its adjusted distribution:
 *   temperatures[b] == 0: the point mass on the first index of the row's
 *     largest logit (greedy; top_k and top_p do not change it);
 *   temperatures[b] > 0: softmax(x / T) restricted to the entries with
 *     x >= the k-th largest logit (top_k in [1, vocab); entries tied with it
 *     are kept), then, within those, to the entries >= the largest logit value
 *     v whose cumulative mass (all kept entries >= v) reaches top_p of the
 *     kept mass (top_p in (0, 1); ties at v are kept), and renormalised.
 * top_k == 0 or >= vocab and top_p >= 1 switch the filters off.  Then the
 * rule of specverify_run: accept while u_accept < q(t)/p(t) (q(t) == 0 gives
 * 0, p(t) == 0 < q(t) gives +inf), draw from max(0, q_n - p_n) at the first
 * rejection or from q_gamma, by the inverse CDF with u_resample.
 * Arguments as specverify_run, plus
 *   temperatures  float [batch] device array, one per sequence
 *   top_k         host value >= 0
 *   top_p         host value in (0, inf); values >= 1 switch it off
 * A sequence with a temperature < 0, NaN or infinite emits nothing and sets
 * status bit 16 (SV_ERR_TEMPERATURE).  Each row is read several times (the
 * threshold search); the kernels are separate from the plain step's.
 */
sv_status specverify_run_sampling(specverify_t h, const void *target_logits,
                                  const void *draft_logits, const int32_t *draft_tokens,
                                  const float *u_accept, const float *u_resample,
                                  const float *temperatures, int top_k, float top_p,
                                  int32_t *out_tokens, int32_t *out_num_accepted, void *stream);

/*
 * After specverify_run_sampling: wait for `stream` and copy the number of
 * entries each row's adjusted distribution keeps ([batch, gamma+1] and
 * [batch, gamma] int32 host arrays; either may be NULL).  Diagnostic.
 */
sv_status specverify_debug_kept(specverify_t h, int32_t *kept_target, int32_t *kept_draft,
                                void *stream);

/*
 * Multi-branch verification over shared logit rows.  Where many candidate
 * branches of one sequence share a prefix, their target and draft rows at the
 * shared positions are the same rows; the SpecFold explainer (blog.ontle.kr,
 * post 356: the multi-branch paragraph and the implementer's note, where the
 * shared cache is read through a strided view instead of a per-branch copy)
 * describes that reuse.  This entry point takes each distinct row once and a
 * map from every (branch, position) to its row, so the step reads
 * (n_target_rows + n_draft_rows) rows of V logits instead of B (2 gamma + 1):
 *   target_rows   [n_target_rows, vocab] dtype, 1 <= n_target_rows <= batch (gamma+1)
 *   target_map    int32 [batch, gamma+1]: row of target_rows of each position
 *   draft_rows    [n_draft_rows, vocab]  dtype, 1 <= n_draft_rows <= batch gamma
 *   draft_map     int32 [batch, gamma]: row of draft_rows of each draft position
 * and the rest as specverify_run.  Every branch is a sequence b of the batch;
 * the result equals specverify_run on the rows the maps pick out
 * (target_logits[b, j] = target_rows[target_map[b, j]], likewise for drafts).
 * Each distinct row's softmax statistics are computed once and shared by
 * every position mapped to it.  All pointers are device pointers; the maps
 * must be 4-byte aligned.  When gamma == 0 the draft arguments are ignored.
 * A map entry outside [0, n rows) makes that sequence emit nothing (as a
 * data error does) and records SV_ERR_ROW_INDEX in the status word.
 */
sv_status specverify_run_mapped(specverify_t h, const void *target_rows, int n_target_rows,
                                const int32_t *target_map, const void *draft_rows,
                                int n_draft_rows, const int32_t *draft_map,
                                const int32_t *draft_tokens, const float *u_accept,
                                const float *u_resample, float temperature,
                                int32_t *out_tokens, int32_t *out_num_accepted,
                                void *stream);

/* Free the handle and everything it owns.  NULL is ignored.  Waits for the
 * device work of the handle to finish first. */
void specverify_destroy(specverify_t h);

/*
 * Wait for `stream`, read and clear the handle's device status word.
 * Returns the most severe condition seen since the last call:
 * SV_ERR_ROW_INDEX, then SV_ERR_TOKEN_RANGE, then SV_ERR_NONFINITE, then
 * SV_WARN_ZERO_MASS, else SV_OK.  `*bits` (may be NULL) receives the raw bit
 * set (1: token range, 2: non-finite row, 4: zero residual mass, 8: row map
 * entry out of range).
 */
sv_status specverify_get_status(specverify_t h, void *stream, uint32_t *bits);

/*
 * Test and debug readback of the last step's intermediate values (waits for
 * `stream`; host pointers, any may be NULL):
 *   target_lse  double [batch, gamma+1]  log sum_i exp(x_i / T) of each target row
 *   draft_lse   double [batch, gamma]    the same for each draft row
 *   q_tok       double [batch, gamma]    q_j(t_j)
 *   p_tok       double [batch, gamma]    p_j(t_j)
 *   ratio       double [batch, gamma]    q_j(t_j) / p_j(t_j) as tested
 *   resid_mass  double [batch]           mass Z of the distribution drawn from
 * Positions that the device did not need keep their previous contents.
 */
sv_status specverify_debug_readback(specverify_t h, double *target_lse, double *draft_lse,
                                   double *q_tok, double *p_tok, double *ratio,
                                   double *resid_mass, void *stream);

/*
 * Launch shape.  The statistics kernel (the one that streams every logit)
 * splits each logit row over `slices` thread blocks of `threads` threads
 * (128, 256 or 512); 1 <= slices <= min(64, ceil(vocab / group) / 128),
 * group = 8 bf16 or 4 fp32 entries.  The draw kernel spreads the rows drawn
 * from over `draw_slices` blocks per sequence (1..64, at most one per four
 * 32-group tiles of a row; 0 or less restores the default).  Invalid values
 * return SV_ERR_INVALID_ARG.  specverify_create picks a shape from the
 * problem size and the SM count; this call overrides it for later runs
 * (results do not depend on the shape beyond the rounding of partial sums).
 * Not stream-ordered: change it only while no run of the handle is in flight.
 */
sv_status specverify_set_launch(specverify_t h, int slices, int threads, int draw_slices);

/* Current shape and the largest `slices` this handle accepts (any pointer may be NULL). */
sv_status specverify_get_launch(specverify_t h, int *slices, int *threads, int *max_slices,
                                int *draw_slices);

/*
 * Number of kernels one run of the handle enqueues (`mapped` nonzero: a run
 * of specverify_run_mapped): statistics, decide and draw (3); one for an
 * aligned unmapped run in the single-launch form (specverify_set_fused); none
 * for an empty batch.
 */
sv_status specverify_kernels_per_run(specverify_t h, int mapped, int *kernels);

/*
 * Single-launch form of the step (default off).  With `enable` nonzero, a run
 * of specverify_run (or specverify_run_host) whose logit pointers are 16-byte
 * aligned with vocab * sizeof(dtype) a multiple of 16 is one persistent
 * kernel: its warps take statistics units (runs of `unit_groups` 16-byte
 * groups of one row, 128 .. 2^20, with at most `max_slices` units per row;
 * 0 picks 1024) and draw chunks (`chunk_tiles` tiles of 64 groups of the
 * rows drawn from; 0 picks 8) from one ordered list, sequence by sequence,
 * the draw chunks of a sequence `lag` sequences after its statistics (-1
 * derives it from the grid).  The warp that finishes a sequence's statistics
 * decides it; the rows drawn from are then re-read from L2 while later
 * sequences stream.  Results equal the three-kernel form's up to the rounding
 * of partial sums.  Waits between warps are bounded; one that runs out (it
 * never should) makes specverify_get_status return SV_ERR_PIPELINE and reset
 * the form's control words.  `enable` zero: three kernels (statistics,
 * decide, draw) as for unaligned or mapped runs.  Invalid values return
 * SV_ERR_INVALID_ARG.  Not stream-ordered: change it only while no run of
 * the handle is in flight.
 */
sv_status specverify_set_fused(specverify_t h, int enable, int unit_groups, int chunk_tiles,
                               int lag);

/* Whether an aligned unmapped run takes the single launch, and its shape
 * (the lag as derived); any pointer may be NULL. */
sv_status specverify_get_fused(specverify_t h, int *enabled, int *unit_groups, int *chunk_tiles,
                               int *lag);

/*
 * Per-kernel timing of the next `max_runs` runs of the handle: each run then
 * records CUDA events on its stream around its two kernels (the statistics
 * kernel, which streams every logit, and the decide-and-draw kernel; a
 * single-launch run records its one kernel as the statistics time and zero
 * for the other).  Waits for the device first; re-arming discards earlier
 * records.
 */
sv_status specverify_profile_begin(specverify_t h, int max_runs);

/*
 * Wait for the last recorded run, store the mean device time per run of each
 * kernel in milliseconds (any pointer may be NULL) and the number of runs
 * recorded, and stop recording.
 */
sv_status specverify_profile_end(specverify_t h, float *stats_ms, float *draw_ms, int *runs);

/*
 * The verification step without a handle and without allocating: for
 * callers that cannot call cudaMalloc (code inside a captured graph region
 * that must not allocate, embedders whose device memory belongs to a pool
 * they cannot reach from here, serving paths that forbid allocation).  The
 * pages have no counterpart; this is an interface of this library only.
 *
 * Arguments and results are those of specverify_create + specverify_run,
 * on the CURRENT device (its buffers and `stream` must belong to it), with
 * the default launch shape.  The workspace is one static device array of
 * 16 MiB that every GPU loading this library holds until the process exits;
 * a batch whose workspace does not fit returns SV_ERR_INVALID_ARG with the
 * needed size in specverify_last_error() and enqueues nothing.  The first
 * call on a device looks up the array's address (and the SM count); make it
 * before any stream capture.  The entry point calls no cudaMalloc or
 * cudaFree.  Every call shares the one array: calls whose work overlaps on
 * the GPU (other streams, other threads) race and must be serialised by the
 * caller.  Each call clears what must start at zero.  Data errors show only
 * in the outputs (num_accepted 0, tokens -1): the status word is not kept.
 */
sv_status specverify_run_noalloc(int batch, int gamma, int vocab, sv_dtype dtype,
                                 const void *target_logits, const void *draft_logits,
                                 const int32_t *draft_tokens, const float *u_accept,
                                 const float *u_resample, float temperature,
                                 int32_t *out_tokens, int32_t *out_num_accepted, void *stream);

/* Static text for a status code. */
const char *specverify_status_string(sv_status s);

/* Text of the last CUDA runtime error seen by this thread ("" if none). */
const char *specverify_last_error(void);

#ifdef __cplusplus
}
#endif

#endif /* SPECVERIFY_H */
