// Single-launch verification step for sm_100a.
//
// The three phases of the step (softmax statistics, decide, draw) run in one
// persistent kernel whose warps are independent workers.  The work of a batch
// is one ordered list of tasks that the warps take from a global counter:
//
//   statistics unit  one warp streams a contiguous run of 16-byte groups of
//                    one logit row (eight 128-bit loads in flight per lane)
//                    and writes its (offset, sum) partial;
//   draw chunk       one warp computes the residual (or target) masses of a
//                    run of tiles of the rows a sequence draws from.
//
// Tasks are ordered sequence by sequence: all statistics units of sequence b
// (its gamma+1 target rows and gamma draft rows), and after them the draw
// chunks of sequence b - D.  The warp that finishes the last statistics unit
// of a sequence (an atomic count per sequence) takes its decision (steps 2
// and 3: ratio tests and the first rejection, the same warp routine as the
// three-kernel form) and publishes it with a release flag.  A warp that takes
// a draw chunk waits (bounded) for that flag; by construction the sequence's
// statistics units were handed out D sequences earlier, so the flag is
// normally set already.  The lag D is chosen so that the rows a sequence draws
// from were streamed only a few microseconds before its draw chunks run: they
// are read from L2, not HBM, and the draw's arithmetic overlaps the streaming
// of later sequences instead of following the whole batch.  The warp that
// finishes the last draw chunk of a sequence (a second count) locates u * Z
// in the tile-mass table and writes the drawn token (step 4).
//
// Progress: a warp that waits holds no other task, and a warp holds at most
// the task it runs and the one it took next.  The unfinished task with the
// smallest index is therefore always held by a warp that runs it, and a draw
// chunk waits only for statistics units with smaller indices, so the launch
// cannot deadlock, whether or not every block is resident.
// Every wait is bounded (kWaitIters polls and 2 s of the global timer); a
// wait that runs out sets the kStatWait status bit and skips its chunk.
//
// The control words (task counter, exit count, per-sequence counts and flags)
// are zero between launches: each per-sequence word is cleared by the warp
// that uses it last, the task counter and the exit count by the last warp to
// leave, so consecutive launches (or graph replays) need no memset.
//
// Pages (title, section): "Speculative decoding - the small model writes first
// and the big model checks", section 1 (the rule); "Speculative decoding: how
// to run big models fast", section "How it works" (one verification pass per
// round, the bonus token).
#pragma once

#include "verify_kernel.cuh"

namespace specverify {

struct FusedParams {
  unsigned* task_next;   // [1] next task to hand out
  unsigned* exit_count;  // [1] warps that have left the task loop
  unsigned* stats_done;  // [B] statistics units finished per sequence
  unsigned* ready;       // [B] 1 once the sequence's decision is published
  unsigned* draw_done;   // [B] draw chunks finished per sequence
  unsigned total_tasks;  // B * (units_per_seq + chunks_per_seq)
  unsigned total_warps;  // warps in the grid
  int units_per_row;     // statistics units per logit row
  int groups_per_unit;   // 16-byte groups per unit (a row's last unit may be shorter)
  int units_per_seq;     // (2 gamma + 1) * units_per_row
  int chunk_tiles;       // tiles of the mass table per draw chunk
  int chunks_per_seq;    // ceil(tiles per row / chunk_tiles)
  int lag;               // D: sequences between a sequence's statistics and its draw chunks
};

constexpr int kFusedThreads = 128;
constexpr int kFusedWarps = kFusedThreads / kWarp;
constexpr int kFusedBlocksPerSM = 8;
constexpr int kFusedLoads = 8;  // 16-byte loads in flight per lane in a statistics unit
constexpr int kFusedStages = 3;  // ring stages of a draw chunk
constexpr size_t kFusedSmem = sizeof(uint4) * kStageU4 * kFusedStages * kFusedWarps;
constexpr unsigned kWaitIters = 1u << 24;
constexpr unsigned long long kWaitNs = 2000000000ull;

enum : int { kTaskStats = 0, kTaskDraw = 1 };

struct Task {
  int kind;
  int b;    // sequence
  int idx;  // unit of the sequence (statistics) or chunk (draw)
};

// Task t of the ordered list: the statistics units of sequences 0 .. D-1,
// then per sequence s = D .. B-1 its statistics units followed by the draw
// chunks of sequence s - D, then the draw chunks of the last D sequences.
__device__ __forceinline__ Task decode_task(const FusedParams& F, int B, unsigned t) {
  const long U = F.units_per_seq, C = F.chunks_per_seq, D = F.lag;
  long r = t;
  const long head = D * U;
  if (r < head) return Task{kTaskStats, static_cast<int>(r / U), static_cast<int>(r % U)};
  r -= head;
  const long mid = (static_cast<long>(B) - D) * (U + C);
  if (r < mid) {
    const long s = r / (U + C), w = r - s * (U + C);
    if (w < U) return Task{kTaskStats, static_cast<int>(D + s), static_cast<int>(w)};
    return Task{kTaskDraw, static_cast<int>(s), static_cast<int>(w - U)};
  }
  r -= mid;
  return Task{kTaskDraw, static_cast<int>(B - D + r / C), static_cast<int>(r % C)};
}

__device__ __forceinline__ unsigned ld_acquire_u32(const unsigned* p) {
  unsigned v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// atomic add with release semantics at GPU scope: the calling thread's
// earlier writes are visible to whoever observes the new count
__device__ __forceinline__ unsigned atom_add_release(unsigned* p, unsigned v) {
  unsigned old;
  asm volatile("atom.add.release.gpu.global.u32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
  return old;
}

__device__ __forceinline__ void st_release_u32(unsigned* p, unsigned v) {
  asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

__device__ __forceinline__ unsigned long long global_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// Waits (calling lane only) until *flag is nonzero; at most kWaitIters polls
// and kWaitNs of the global timer.  Returns false (and sets kStatWait) if the
// wait ran out.
__device__ __noinline__ bool wait_flag(const unsigned* flag, unsigned* status) {
  if (ld_acquire_u32(flag) != 0u) return true;
  const unsigned long long t0 = global_ns();
  unsigned sleep = 32;
  for (unsigned it = 0; it < kWaitIters; ++it) {
    __nanosleep(sleep);
    if (sleep < 512) sleep <<= 1;
    if (ld_acquire_u32(flag) != 0u) return true;
    if (global_ns() - t0 > kWaitNs) break;
  }
  atomicOr(status, kStatWait);
  return false;
}

// Statistics of groups [lo, hi) of one 16-byte aligned row by the calling
// warp: lane l streams groups lo + l + 32 i, kL loads in flight per round,
// into a running (o, s); the warp's partial is (max o, sum s 2^(o - max o)),
// the sum in fp64.  Valid in every lane.
template <typename T, int kL>
__device__ __forceinline__ RowPartial warp_unit_stats(const T* row, long lo, long hi, float c_hi,
                                                      float c_lo) {
  const int lane = threadIdx.x & (kWarp - 1);
  const uint4* g4 = reinterpret_cast<const uint4*>(row);
  float o = -INFINITY, s = 0.f;
  long g = lo + lane;
  for (; g + static_cast<long>(kWarp) * (kL - 1) < hi; g += static_cast<long>(kWarp) * kL) {
    uint4 v[kL];
#pragma unroll
    for (int u = 0; u < kL; ++u) v[u] = ld_stream(g4 + g + static_cast<long>(u) * kWarp);
#pragma unroll
    for (int u = 0; u < kL; ++u) accumulate_group<T>(v[u], o, s, c_hi, c_lo);
  }
  if (g < hi) {
    uint4 v[kL];
#pragma unroll
    for (int u = 0; u < kL; ++u)
      if (g + static_cast<long>(u) * kWarp < hi) v[u] = ld_stream(g4 + g + static_cast<long>(u) * kWarp);
#pragma unroll
    for (int u = 0; u < kL; ++u)
      if (g + static_cast<long>(u) * kWarp < hi) accumulate_group<T>(v[u], o, s, c_hi, c_lo);
  }
  const float O = warp_max(o);
  // a lane with o = -inf holds s = 0 (or NaN, which must propagate)
  const float f = (o == -INFINITY) ? 0.f : ex2(o - O);
  const double S = warp_sum(static_cast<double>(s) * static_cast<double>(f));
  return RowPartial{S, O, 0};
}

// Copies the sequence's partials (its gamma+1 target rows, then its gamma
// draft rows, nu per row: two contiguous runs of the table) into the calling
// warp's shared memory with every load in flight at once; returns false if
// they do not fit in `cap` entries.
__device__ __forceinline__ bool stage_partials(const Params& P, int b, int nu, RowPartial* smem,
                                               int cap) {
  const int lane = threadIdx.x & (kWarp - 1);
  const int G = P.gamma;
  const long nt = static_cast<long>(G + 1) * nu, nd = static_cast<long>(G) * nu;
  if (nt + nd > cap) return false;
  const uint4* srcT = reinterpret_cast<const uint4*>(P.partial + static_cast<long>(b) * (G + 1) * nu);
  const uint4* srcD =
      reinterpret_cast<const uint4*>(P.partial + (P.target_rows + static_cast<long>(b) * G) * nu);
  uint4* dst = reinterpret_cast<uint4*>(smem);
  constexpr int kU = 8;
  for (long e0 = lane; e0 < nt + nd; e0 += static_cast<long>(kWarp) * kU) {
    uint4 v[kU];
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      const long e = e0 + static_cast<long>(u) * kWarp;
      if (e < nt + nd) v[u] = (e < nt) ? __ldcg(srcT + e) : __ldcg(srcD + (e - nt));
    }
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      const long e = e0 + static_cast<long>(u) * kWarp;
      if (e < nt + nd) dst[e] = v[u];
    }
  }
  __syncwarp();
  return true;
}

// The decision of sequence b by the calling warp, then its publication (a
// separate function: its registers are not live across the streaming loop).
template <typename T>
__device__ __noinline__ void decide_and_publish(const Params* Pp, const FusedParams* Fp, int b,
                                                uint4* ring) {
  const Params& P = *Pp;
  const FusedParams& F = *Fp;
  const int lane = threadIdx.x & (kWarp - 1);
  __threadfence();  // the other warps' partials, seen through the count
  RowPartial* staged = reinterpret_cast<RowPartial*>(ring);
  constexpr int kCap = static_cast<int>(kStageU4 * kFusedStages * sizeof(uint4) / sizeof(RowPartial));
  if (stage_partials(P, b, F.units_per_row, staged, kCap))
    decide_sequence<T, true>(P, b, staged);
  else
    decide_sequence<T, true>(P, b);
  __syncwarp();  // the ring is reused by this warp's next draw chunk
  __threadfence();  // every lane's writes before the flag
  __syncwarp();
  if (lane == 0) {
    F.stats_done[b] = 0u;  // no unit of this sequence is left
    st_release_u32(F.ready + b, 1u);
  }
}

// One statistics unit; the warp that completes its sequence decides it and
// publishes the decision.
template <typename T>
__device__ __forceinline__ void run_stats_unit(const Params& P, const FusedParams& F, int b, int w,
                                               uint4* ring) {
  constexpr int kVec = Elem<T>::kVec;
  const int lane = threadIdx.x & (kWarp - 1);
  const int V = P.vocab, G = P.gamma, nu = F.units_per_row;
  const int r = w / nu, k = w - r * nu;
  const T* row;
  long prow;  // row of the partial table
  if (r <= G) {
    const long tr = static_cast<long>(b) * (G + 1) + r;
    row = static_cast<const T*>(P.target) + tr * V;
    prow = tr;
  } else {
    const long dr = static_cast<long>(b) * G + (r - G - 1);
    row = static_cast<const T*>(P.draft) + dr * V;
    prow = P.target_rows + dr;
  }
  const long ngroups = (static_cast<long>(V) + kVec - 1) / kVec;
  const long lo = static_cast<long>(k) * F.groups_per_unit;
  const long hi = (lo + F.groups_per_unit < ngroups) ? lo + F.groups_per_unit : ngroups;
  const RowPartial part = warp_unit_stats<T, kFusedLoads>(row, lo, hi, P.c_hi, P.c_lo);
  unsigned last = 0;
  if (lane == 0) {
    P.partial[prow * nu + k] = part;
    __threadfence();
    const unsigned old = atomicAdd(F.stats_done + b, 1u);
    last = (old + 1u == static_cast<unsigned>(F.units_per_seq));
  }
  last = __shfl_sync(0xffffffffu, last, 0);
  if (last) decide_and_publish<T>(&P, &F, b, ring);
}

// One draw chunk (its sequence's decision already published): tile masses
// of tiles [chunk * CT, ...) of the rows sequence b draws from; the warp that
// completes the sequence's chunks locates the token and clears the
// sequence's words.
template <typename T>
__device__ __noinline__ void run_draw_chunk(const Params* Pp, const FusedParams* Fp, int b,
                                            int chunk, uint4* ring) {
  const Params& P = *Pp;
  const FusedParams& F = *Fp;
  constexpr int kVec = Elem<T>::kVec;
  const int lane = threadIdx.x & (kWarp - 1);
  const int V = P.vocab;
  // the decision was written by another warp of this launch: read it from L2
  const SeqDecision* dp = P.decision + b;
  const int mode = __ldcg(&dp->mode);
  const long ngroups = (static_cast<long>(V) + kVec - 1) / kVec;
  const long ntiles = P.draw_tiles;
  DrawConsts k;
  k.c_hi = P.c_hi;
  k.c_lo = P.c_lo;
  const T* rowT = nullptr;
  const T* rowD = nullptr;
  int n = 0;
  if (mode != kDrawNone) {
    n = __ldcg(&dp->n);
    k.lt_hi = __ldcg(&dp->lt_hi);
    k.k_hi = __ldcg(&dp->k_hi);
    k.k_lo = __ldcg(&dp->k_lo);
    k.fT = __ldcg(&dp->fT);
    rowT = static_cast<const T*>(P.target) + __ldcg(&dp->trow) * V;
    if (mode == kDrawResidual) rowD = static_cast<const T*>(P.draft) + __ldcg(&dp->drow) * V;
    const long t0 = static_cast<long>(chunk) * F.chunk_tiles;
    const long t1 = (t0 + F.chunk_tiles < ntiles) ? t0 + F.chunk_tiles : ntiles;
    double* table = P.draw_mass + static_cast<long>(b) * ntiles;
    if (mode == kDrawResidual)
      tile_masses_ring<T, kDrawResidual, kFusedStages>(rowT, rowD, k, t0, t1, ngroups, table, ring);
    else
      tile_masses_ring<T, kDrawTarget, kFusedStages>(rowT, rowD, k, t0, t1, ngroups, table, ring);
  }
  unsigned last = 0;
  if (lane == 0) {
    __threadfence();
    const unsigned old = atomicAdd(F.draw_done + b, 1u);
    last = (old + 1u == static_cast<unsigned>(F.chunks_per_seq));
  }
  last = __shfl_sync(0xffffffffu, last, 0);
  if (!last) return;
  __threadfence();  // every lane reads the other warps' table entries after the count
  if (mode != kDrawNone) locate<T, true>(&P, b, n, mode, rowT, rowD, k, ntiles, ngroups);
  if (lane == 0) {
    F.draw_done[b] = 0u;
    F.ready[b] = 0u;  // every chunk of this sequence has read the flag
  }
}

// The whole step in one launch (16-byte aligned rows, unmapped layout:
// target [B, G+1, V], draft [B, G, V]).  Grid: at most the resident blocks.
template <typename T>
__global__ void __launch_bounds__(kFusedThreads, kFusedBlocksPerSM)
    fused_kernel(const __grid_constant__ Params P, const __grid_constant__ FusedParams F) {
  extern __shared__ uint4 fused_smem[];
  uint4* ring = fused_smem + (threadIdx.x >> 5) * (kStageU4 * kFusedStages);  // this warp's ring
  const int lane = threadIdx.x & (kWarp - 1);
  unsigned next = 0;
  if (lane == 0) next = atomicAdd(F.task_next, 1u);
  next = __shfl_sync(0xffffffffu, next, 0);
  while (next < F.total_tasks) {
    const Task t = decode_task(F, P.batch, next);
    // A draw chunk first waits for its sequence's decision, holding no other
    // task meanwhile; then the following task is taken before this one runs,
    // so the atomic's latency overlaps it.
    unsigned ok = 1;
    if (t.kind == kTaskDraw && lane == 0) ok = wait_flag(F.ready + t.b, P.status) ? 1u : 0u;
    if (lane == 0) next = atomicAdd(F.task_next, 1u);
    ok = __shfl_sync(0xffffffffu, ok, 0);
    if (t.kind == kTaskStats) run_stats_unit<T>(P, F, t.b, t.idx, ring);
    else if (ok) run_draw_chunk<T>(&P, &F, t.b, t.idx, ring);
    // (a wait that ran out set kStatWait: that sequence's draw is incomplete)
    next = __shfl_sync(0xffffffffu, next, 0);
  }
  if (lane == 0) {
    const unsigned old = atomicAdd(F.exit_count, 1u);
    if (old + 1u == F.total_warps) {
      // every warp has taken its last task index: ready for the next launch
      *F.task_next = 0u;
      *F.exit_count = 0u;
    }
  }
}

// Host: the fused launch's task layout for a batch.
struct FusedShape {
  int units_per_row, groups_per_unit, units_per_seq, chunk_tiles, chunks_per_seq, lag;
  long total_tasks;
};

inline FusedShape fused_shape(long batch, int gamma, long ngroups, long ntiles, int unit_groups,
                              int chunk_tiles, int lag, long total_warps) {
  FusedShape s;
  const long nu = (ngroups + unit_groups - 1) / unit_groups;
  s.units_per_row = static_cast<int>(nu < 1 ? 1 : nu);
  s.groups_per_unit = static_cast<int>((ngroups + s.units_per_row - 1) / s.units_per_row);
  s.units_per_seq = (2 * gamma + 1) * s.units_per_row;
  s.chunk_tiles = chunk_tiles;
  s.chunks_per_seq = static_cast<int>((ntiles + chunk_tiles - 1) / chunk_tiles);
  if (lag < 0) {
    // about three grids' worth of tasks between a sequence's statistics and
    // its draw: its last unit is then finished and decided before its chunks
    // run
    const long per = s.units_per_seq + s.chunks_per_seq;
    lag = static_cast<int>((3 * total_warps + per - 1) / per) + 1;
  }
  if (lag > batch) lag = static_cast<int>(batch);
  s.lag = lag;
  s.total_tasks = batch * static_cast<long>(s.units_per_seq + s.chunks_per_seq);
  return s;
}

}  // namespace specverify
