// C ABI of the speculative-sampling verification library (see specverify.h).
//
// Host side only: argument checks, the workspace, the launch shapes, the
// three stream-ordered launches of one step, host-buffer staging, readbacks.
#include "specverify.h"

#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <new>
#include <vector>

#include "fused_kernel.cuh"
#include "host_common.h"
#include "sampling_kernel.cuh"
#include "verify_kernel.cuh"

using specverify::RowPartial;
using specverify::Params;
using specverify::PosInfo;
using specverify::RowStat;
using specverify::SeqDecision;

struct specverify_ctx {
  int device = 0;
  int batch = 0, gamma = 0, vocab = 0;
  sv_dtype dtype = SV_DTYPE_F32;
  int slices = 1, threads = 128;
  int max_slices = 1;  // the partial-statistics workspace holds this many per position
  int draw_slices = 64; // at most this many draw blocks per sequence
  int num_sms = 148;
  // tapered statistics grid (0: every row in `slices` slices): all but the
  // last taper_tail rows of a run in taper_slices long slices
  long taper_tail = 0;
  int taper_slices = 0;
  void* ws = nullptr;  // one device allocation for the whole workspace
  RowPartial* partial = nullptr;
  RowStat* tstat = nullptr;
  RowStat* dstat = nullptr;
  PosInfo* pos = nullptr;
  SeqDecision* decision = nullptr;
  double* draw_mass = nullptr;
  unsigned* draw_ticket = nullptr;
  double* resid = nullptr;
  unsigned* status = nullptr;
  specsamp::SampRow* samp_rows = nullptr;          // sampling variants: per-row filter
  // single-launch step (fused_kernel): used for 16-byte aligned, unmapped
  // runs when `fused` is set; its own partial table and control words
  int fused = 0;  // off by default (specverify_set_fused)
  int fused_unit_groups = 1024;  // 16-byte groups per statistics unit
  int fused_chunk_tiles = 8;     // mass-table tiles per draw chunk
  int fused_lag = -1;            // sequences between statistics and draw (-1: derived)
  int fused_blocks_per_sm = 0;   // resident blocks of fused_kernel per SM
  unsigned* fctl = nullptr;      // task counter, exit count, then 3 words per sequence
  specsamp::SampDecision* samp_decision = nullptr; // sampling variants: per sequence
  void* stage = nullptr;  // device staging for host-buffer runs
  size_t stage_bytes = 0;
  // optional per-kernel timing: 3 events per recorded run
  std::vector<cudaEvent_t> events;
  int prof_capacity = 0;
  int prof_runs = 0;
};

namespace svhost {

thread_local char g_last_error[256] = "";

sv_status cuda_fail(cudaError_t e) {
  std::snprintf(g_last_error, sizeof g_last_error, "%s: %s", cudaGetErrorName(e),
                cudaGetErrorString(e));
  return (e == cudaErrorMemoryAllocation) ? SV_ERR_OOM : SV_ERR_CUDA;
}

}  // namespace svhost

namespace {

using svhost::cuda_fail;
using svhost::DeviceScope;
using svhost::g_last_error;
using svhost::round_up;

size_t elem_size(sv_dtype d) { return d == SV_DTYPE_BF16 ? 2 : 4; }
int group_elems(sv_dtype d) { return d == SV_DTYPE_BF16 ? 8 : 4; }

long num_groups(const specverify_ctx* h) {
  const int ve = group_elems(h->dtype);
  return (static_cast<long>(h->vocab) + ve - 1) / ve;
}

// Tapered grid: rows in long slices first, then about one wave of short
// blocks (kTaperShort slices per row) at the end of the grid.
constexpr int kTaperLong = 2;
constexpr int kTaperShort = 8;
constexpr double kTaperWaves = 1.0;

// Default launch shape of the statistics kernel: 128 threads per block,
// every logit row split over `slices` blocks (at most 8) so that the grid
// holds about four waves of blocks where the batch allows (the last, partial
// wave then costs little; more, smaller blocks only add per-block overhead),
// with at least one 16-byte group per thread.  Batches of several waves of
// rows of 64 KB or more take the tapered grid instead: long blocks (less
// start-up per byte) with the short ones dispatched last, so that the SMs
// run out of work together.
void default_shape(specverify_ctx* h) {
  const int threads = 128;
  const long rows = static_cast<long>(h->batch) * (2L * h->gamma + 1);
  const long slots = static_cast<long>(h->num_sms) * (1024 / threads);
  const long ngroups = num_groups(h);
  int best = 1;
  // more than 8 slices only lengthens the decision kernel's combine
  const int cap = h->max_slices < 8 ? h->max_slices : 8;
  for (int c = 1; c <= cap; ++c) {
    if (ngroups / c < threads && c > 1) break;
    best = c;
    if (rows * c >= 4 * slots) break;
  }
  h->slices = best;
  h->threads = threads;
  h->taper_tail = 0;
  h->taper_slices = 0;
  const int shortS = cap < kTaperShort ? cap : kTaperShort;
  const long tail = static_cast<long>(kTaperWaves * static_cast<double>(slots) / shortS + 0.999);
  if (shortS > kTaperLong && ngroups >= 4096 && rows >= 2 * tail &&
      (rows - tail) * kTaperLong + tail * shortS >= 2 * slots) {
    h->slices = shortS;
    h->taper_slices = kTaperLong;
    h->taper_tail = tail;
  }
}

// Draw blocks per sequence, at most: the draw kernel's grid is also capped at
// one resident wave and at one warp per tile, so the default only bounds it.
int draw_shape(const specverify_ctx*) { return 64; }

long draw_tiles(const specverify_ctx* h) {
  return specverify::draw_tiles_per_row(h->vocab, group_elems(h->dtype));
}

unsigned draw_blocks(const specverify_ctx* h) {
  return specverify::draw_grid(h->batch, draw_tiles(h), h->draw_slices, h->num_sms);
}

template <typename K, typename PP>
cudaError_t launch_pdl(K kernel, unsigned blocks, unsigned threads, cudaStream_t s, const PP& p) {
  // programmatic dependent launch: the kernel may be scheduled before its
  // predecessor on the stream has finished; it waits in a grid-dependency
  // barrier before it reads the predecessor's results
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(blocks, 1, 1);
  cfg.blockDim = dim3(threads, 1, 1);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, p);
}

// The statistics kernel is a programmatic dependent of whatever precedes it
// on the stream: its blocks may become resident during the predecessor's
// tail and wait for it to complete before their first load.
template <typename T, int NT, bool A>
cudaError_t launch_stats_nt(const Params& p, long blocks, cudaStream_t s) {
  return launch_pdl(specverify::stats_kernel<T, NT, A>, static_cast<unsigned>(blocks), NT, s, p);
}

// One step: statistics, decide, draw.  events[0..2] (may be null): before
// stats, after stats, after draw.
template <typename T, bool A>
cudaError_t launch_step(const Params& p, int NT, unsigned draw_blocks, cudaStream_t s,
                        cudaEvent_t* ev) {
  const long rows = p.target_rows + p.draft_rows;
  const long blocks = p.taper_rows * p.taper_slices + (rows - p.taper_rows) * p.slices;
  cudaError_t e = cudaSuccess;
  if (ev) e = cudaEventRecord(ev[0], s);
  if (e != cudaSuccess) return e;
  switch (NT) {
    case 128: e = launch_stats_nt<T, 128, A>(p, blocks, s); break;
    case 256: e = launch_stats_nt<T, 256, A>(p, blocks, s); break;
    case 512: e = launch_stats_nt<T, 512, A>(p, blocks, s); break;
    default: return cudaErrorInvalidValue;
  }
  if (e == cudaSuccess && ev) e = cudaEventRecord(ev[1], s);
  if (e != cudaSuccess) return e;
  const int per = specverify::kDecideThreads / specverify::kWarp;
  e = launch_pdl(specverify::decide_kernel<T>, static_cast<unsigned>((p.batch + per - 1) / per),
                 specverify::kDecideThreads, s, p);
  if (e != cudaSuccess) return e;
  e = specverify::launch_draw<T, A>(p, draw_blocks, s, true);
  if (e == cudaSuccess && ev) e = cudaEventRecord(ev[2], s);
  return e;
}

template <typename T>
cudaError_t launch_dtype(const Params& p, int NT, unsigned draw_blocks, bool aligned,
                         cudaStream_t s, cudaEvent_t* ev) {
  return aligned ? launch_step<T, true>(p, NT, draw_blocks, s, ev)
                 : launch_step<T, false>(p, NT, draw_blocks, s, ev);
}

bool aligned_to(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// the sampling-variant step: select (one block per row), decide, draw
// events (may be null): before select, after select, after draw
template <typename T, bool A>
cudaError_t launch_sampling(const specsamp::SampParams& p, long rows, int per, cudaStream_t s,
                            cudaEvent_t* ev) {
  cudaError_t e = cudaFuncSetAttribute(specsamp::select_kernel<T, A>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       specsamp::kCandSmem);
  if (e == cudaSuccess && ev) e = cudaEventRecord(ev[0], s);
  if (e != cudaSuccess) return e;
  specsamp::select_kernel<T, A><<<static_cast<unsigned>(rows), specsamp::kSelThreads,
                                  static_cast<size_t>(p.cand_cap) * 8, s>>>(p);
  e = cudaGetLastError();
  if (e == cudaSuccess && ev) e = cudaEventRecord(ev[1], s);
  if (e == cudaSuccess)
    e = launch_pdl(specsamp::decide_kernel<T>, static_cast<unsigned>((p.batch + per - 1) / per),
                   specsamp::kDecideThreads, s, p);
  if (e == cudaSuccess)
    e = launch_pdl(specsamp::draw_kernel<T>, static_cast<unsigned>(p.batch),
                   specsamp::kDrawThreads, s, p);
  if (e == cudaSuccess && ev) e = cudaEventRecord(ev[2], s);
  return e;
}

// The single-launch step's task layout for this handle's batch.
specverify::FusedShape fused_shape_of(const specverify_ctx* h) {
  const long warps = static_cast<long>(h->num_sms) * h->fused_blocks_per_sm * specverify::kFusedWarps;
  return specverify::fused_shape(h->batch, h->gamma, num_groups(h), draw_tiles(h),
                                 h->fused_unit_groups, h->fused_chunk_tiles, h->fused_lag, warps);
}

// Whether an (aligned) run of the handle takes the single launch: the fused
// mode is on, the rows are not mapped, and the task list fits its counters.
bool use_fused(const specverify_ctx* h, const int32_t* target_map) {
  if (!h->fused || target_map || !h->fctl || h->fused_blocks_per_sm < 1) return false;
  const specverify::FusedShape fs = fused_shape_of(h);
  return fs.units_per_row <= h->max_slices && fs.total_tasks < (1L << 31);
}

// The single-launch step.  events (may be null): [0] before, [1] and [2]
// after the kernel (the whole step is reported as the statistics time).
template <typename T>
cudaError_t launch_fused(const specverify_ctx* h, Params p, cudaStream_t s, cudaEvent_t* ev) {
  const specverify::FusedShape fs = fused_shape_of(h);
  p.slices = fs.units_per_row;  // the partial table holds max_slices >= this per row
  p.taper_rows = 0;
  specverify::FusedParams f;
  f.task_next = h->fctl;
  f.exit_count = h->fctl + 1;
  f.stats_done = h->fctl + 2;
  f.ready = h->fctl + 2 + h->batch;
  f.draw_done = h->fctl + 2 + 2L * h->batch;
  f.total_tasks = static_cast<unsigned>(fs.total_tasks);
  f.units_per_row = fs.units_per_row;
  f.groups_per_unit = fs.groups_per_unit;
  f.units_per_seq = fs.units_per_seq;
  f.chunk_tiles = fs.chunk_tiles;
  f.chunks_per_seq = fs.chunks_per_seq;
  f.lag = fs.lag;
  long blocks = static_cast<long>(h->num_sms) * h->fused_blocks_per_sm;
  const long need = (fs.total_tasks + specverify::kFusedWarps - 1) / specverify::kFusedWarps;
  if (blocks > need) blocks = need;
  if (blocks < 1) blocks = 1;
  f.total_warps = static_cast<unsigned>(blocks * specverify::kFusedWarps);
  cudaError_t e = cudaSuccess;
  if (ev) e = cudaEventRecord(ev[0], s);
  if (e != cudaSuccess) return e;
  specverify::fused_kernel<T><<<static_cast<unsigned>(blocks), specverify::kFusedThreads,
                                specverify::kFusedSmem, s>>>(p, f);
  e = cudaGetLastError();
  if (e == cudaSuccess && ev) e = cudaEventRecord(ev[1], s);
  if (e == cudaSuccess && ev) e = cudaEventRecord(ev[2], s);
  return e;
}

// Row maps null: the logit buffers hold one row per position, [B, G+1, V] and
// [B, G, V].  Otherwise `target_rows` / `draft_rows` rows that the maps index.
// Every argument check of a verification call: null and alignment tests,
// the temperature and log2(e)/T range.  Runs before anything is enqueued.
sv_status check_args(const specverify_ctx* h, const void* target, const void* draft,
                     const int32_t* tokens, const float* u_accept, const float* u_resample,
                     float temperature, const int32_t* out_tokens,
                     const int32_t* out_num_accepted, const int32_t* target_map,
                     const int32_t* draft_map) {
  const int G = h->gamma;
  const size_t es = elem_size(h->dtype);
  if (!target || !u_resample || !out_tokens || !out_num_accepted) return SV_ERR_INVALID_ARG;
  if (G > 0 && (!draft || !tokens || !u_accept)) return SV_ERR_INVALID_ARG;
  if (!aligned_to(target_map, 4) || !aligned_to(draft_map, 4)) return SV_ERR_INVALID_ARG;
  if (!aligned_to(target, es) || (G > 0 && !aligned_to(draft, es))) return SV_ERR_INVALID_ARG;
  if (!aligned_to(tokens, 4) || !aligned_to(u_accept, 4) || !aligned_to(u_resample, 4) ||
      !aligned_to(out_tokens, 4) || !aligned_to(out_num_accepted, 4))
    return SV_ERR_INVALID_ARG;
  if (!std::isfinite(temperature) || !(temperature > 0.f)) return SV_ERR_INVALID_ARG;
  const double c = 1.4426950408889634074 / static_cast<double>(temperature);
  if (!(c < 1e30)) return SV_ERR_INVALID_ARG;
  return SV_OK;
}

sv_status enqueue(specverify_t h, const void* target, const void* draft, const int32_t* tokens,
                  const float* u_accept, const float* u_resample, float temperature,
                  int32_t* out_tokens, int32_t* out_num_accepted, cudaStream_t stream,
                  const int32_t* target_map = nullptr, const int32_t* draft_map = nullptr,
                  long target_rows = -1, long draft_rows = -1) {
  const int G = h->gamma;
  const sv_status chk = check_args(h, target, draft, tokens, u_accept, u_resample, temperature,
                                   out_tokens, out_num_accepted, target_map, draft_map);
  if (chk != SV_OK) return chk;
  const size_t es = elem_size(h->dtype);
  if (target_rows < 0) target_rows = static_cast<long>(h->batch) * (G + 1);
  if (draft_rows < 0) draft_rows = static_cast<long>(h->batch) * G;

  // log2(e)/T = c_hi + c_lo with c_hi rounded toward zero, so c_lo >= 0;
  // c_lo is kept a normal positive float so that -inf * c_lo stays -inf
  const double c = 1.4426950408889634074 / static_cast<double>(temperature);
  float c_hi = static_cast<float>(c);
  if (static_cast<double>(c_hi) > c) c_hi = std::nextafter(c_hi, 0.f);
  float c_lo = static_cast<float>(c - static_cast<double>(c_hi));
  if (!(c_lo >= 1e-30f)) c_lo = 1e-30f;

  Params p;
  p.target = target;
  p.draft = draft;
  p.target_map = target_map;
  p.draft_map = draft_map;
  p.target_rows = target_rows;
  p.draft_rows = draft_rows;
  p.tokens = tokens;
  p.u_accept = u_accept;
  p.u_resample = u_resample;
  p.out_tokens = out_tokens;
  p.out_num_accepted = out_num_accepted;
  p.partial = h->partial;
  p.tstat = h->tstat;
  p.dstat = h->dstat;
  p.pos = h->pos;
  p.decision = h->decision;
  p.draw_mass = h->draw_mass;
  p.draw_ticket = h->draw_ticket;
  p.resid_mass = h->resid;
  p.status = h->status;
  p.batch = h->batch;
  p.gamma = G;
  p.vocab = h->vocab;
  const long ngroups = num_groups(h);
  p.slices = h->slices;
  p.groups_per_slice = static_cast<int>((ngroups + h->slices - 1) / h->slices);
  const long rows = target_rows + draft_rows;
  p.taper_rows = (h->taper_slices > 0 && rows > h->taper_tail) ? rows - h->taper_tail : 0;
  p.taper_slices = h->taper_slices;
  p.taper_groups = h->taper_slices > 0
                       ? static_cast<int>((ngroups + h->taper_slices - 1) / h->taper_slices)
                       : 0;
  p.draw_tiles = draw_tiles(h);
  const unsigned nd = draw_blocks(h);
  p.c_hi = c_hi;
  p.c_lo = c_lo;
  p.c = static_cast<double>(c_hi) + static_cast<double>(c_lo);
  p.gathered_target = nullptr;
  p.gathered_draft = nullptr;
  p.draw_compact = 0;

  const bool aligned = aligned_to(target, 16) && (G == 0 || aligned_to(draft, 16)) &&
                       (static_cast<size_t>(h->vocab) * es) % 16 == 0;
  cudaEvent_t* ev = nullptr;
  if (h->prof_runs < h->prof_capacity) ev = h->events.data() + 3 * (h->prof_runs++);
  if (aligned && use_fused(h, target_map)) {
    const cudaError_t fe = (h->dtype == SV_DTYPE_BF16)
                               ? launch_fused<__nv_bfloat16>(h, p, stream, ev)
                               : launch_fused<float>(h, p, stream, ev);
    if (fe != cudaSuccess) return cuda_fail(fe);
    return SV_OK;
  }
  cudaError_t e = (h->dtype == SV_DTYPE_BF16)
                      ? launch_dtype<__nv_bfloat16>(p, h->threads, nd, aligned, stream, ev)
                      : launch_dtype<float>(p, h->threads, nd, aligned, stream, ev);
  if (e != cudaSuccess) return cuda_fail(e);
  return SV_OK;
}

}  // namespace

extern "C" {

sv_status specverify_create(specverify_t* out, int batch, int gamma, int vocab, sv_dtype dtype,
                            int device) {
  if (!out) return SV_ERR_INVALID_ARG;
  *out = nullptr;
  if (batch < 0 || gamma < 0 || gamma > specverify::kMaxGamma || vocab < 1 || vocab > (1 << 30))
    return SV_ERR_INVALID_ARG;
  if (dtype != SV_DTYPE_F32 && dtype != SV_DTYPE_BF16) return SV_ERR_INVALID_ARG;
  const long positions = static_cast<long>(batch) * (gamma + 1);
  if (positions * specverify::kMaxSlices > 0x7fffffffL) return SV_ERR_INVALID_ARG;
  int ndev = 0;
  cudaError_t e = cudaGetDeviceCount(&ndev);
  if (e != cudaSuccess) return cuda_fail(e);
  if (device < 0 || device >= ndev) return SV_ERR_INVALID_ARG;
  cudaDeviceProp prop;
  e = cudaGetDeviceProperties(&prop, device);
  if (e != cudaSuccess) return cuda_fail(e);
  if (prop.major != 10 || prop.minor != 0) {
    std::snprintf(g_last_error, sizeof g_last_error,
                  "device %d is sm_%d%d; this library is built for sm_100a only", device,
                  prop.major, prop.minor);
    return SV_ERR_UNSUPPORTED;
  }
  DeviceScope scope(device);
  if (!scope.ok()) return SV_ERR_CUDA;

  specverify_ctx* h = new (std::nothrow) specverify_ctx;
  if (!h) return SV_ERR_OOM;
  h->device = device;
  h->batch = batch;
  h->gamma = gamma;
  h->vocab = vocab;
  h->dtype = dtype;
  h->num_sms = prop.multiProcessorCount;
  {
    // at most one slice per 128 groups (2 KB of bf16 logits) and 64 in all
    const long cap = num_groups(h) / 128;
    h->max_slices = static_cast<int>(cap < 1 ? 1 : (cap > specverify::kMaxSlices ? specverify::kMaxSlices : cap));
  }
  default_shape(h);

  const size_t nT = static_cast<size_t>(batch) * (gamma + 1);
  const size_t nD = static_cast<size_t>(batch) * gamma;
  const size_t nB = static_cast<size_t>(batch);
  h->draw_slices = draw_shape(h);
  const size_t nPart = (nT + nD) * static_cast<size_t>(h->max_slices);
  const size_t nDraw = nB * static_cast<size_t>(draw_tiles(h));
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t at = off;
    off = round_up(off + bytes, 256);
    return at;
  };
  const size_t offA = take(nPart * sizeof(RowPartial));
  const size_t offT = take(nT * sizeof(RowStat));
  const size_t offD = take(nD * sizeof(RowStat));
  const size_t offP = take(nD * sizeof(PosInfo));
  const size_t offC = take(nB * sizeof(SeqDecision));
  const size_t offW = take(nDraw * sizeof(double));
  const size_t offK = take(nB * sizeof(unsigned));
  const size_t offR = take(nB * sizeof(double));
  const size_t offS = take(sizeof(unsigned));
  const size_t offSR = take((nT + nD) * sizeof(specsamp::SampRow));
  const size_t offSD = take(nB * sizeof(specsamp::SampDecision));
  const size_t offF = take((2 + 3 * nB) * sizeof(unsigned));
  const size_t total = off;
  e = cudaMalloc(&h->ws, total);
  if (e != cudaSuccess) {
    delete h;
    return cuda_fail(e);
  }
  char* base = static_cast<char*>(h->ws);
  h->partial = reinterpret_cast<RowPartial*>(base + offA);
  h->tstat = reinterpret_cast<RowStat*>(base + offT);
  h->dstat = reinterpret_cast<RowStat*>(base + offD);
  h->pos = reinterpret_cast<PosInfo*>(base + offP);
  h->decision = reinterpret_cast<SeqDecision*>(base + offC);
  h->draw_mass = reinterpret_cast<double*>(base + offW);
  h->draw_ticket = reinterpret_cast<unsigned*>(base + offK);
  h->resid = reinterpret_cast<double*>(base + offR);
  h->status = reinterpret_cast<unsigned*>(base + offS);
  h->samp_rows = reinterpret_cast<specsamp::SampRow*>(base + offSR);
  h->samp_decision = reinterpret_cast<specsamp::SampDecision*>(base + offSD);
  h->fctl = reinterpret_cast<unsigned*>(base + offF);
  {
    // resident blocks of the single-launch kernel (its grid is one wave)
    int nb = 0;
    e = (dtype == SV_DTYPE_BF16)
            ? cudaOccupancyMaxActiveBlocksPerMultiprocessor(
                  &nb, specverify::fused_kernel<__nv_bfloat16>, specverify::kFusedThreads,
                  specverify::kFusedSmem)
            : cudaOccupancyMaxActiveBlocksPerMultiprocessor(
                  &nb, specverify::fused_kernel<float>, specverify::kFusedThreads,
                  specverify::kFusedSmem);
    if (e != cudaSuccess) {
      cudaFree(h->ws);
      delete h;
      return cuda_fail(e);
    }
    h->fused_blocks_per_sm = nb;
    h->fused = 0;  // opt-in: the three kernels are faster on every measured batch
    long ug = 1024;
    while ((num_groups(h) + ug - 1) / ug > h->max_slices) ug *= 2;
    h->fused_unit_groups = static_cast<int>(ug);
  }
  e = cudaMemset(h->ws, 0, total);
  if (e == cudaSuccess) e = cudaDeviceSynchronize();
  if (e != cudaSuccess) {
    cudaFree(h->ws);
    delete h;
    return cuda_fail(e);
  }
  *out = h;
  return SV_OK;
}

sv_status specverify_run(specverify_t h, const void* target_logits, const void* draft_logits,
                         const int32_t* draft_tokens, const float* u_accept,
                         const float* u_resample, float temperature, int32_t* out_tokens,
                         int32_t* out_num_accepted, void* stream) {
  svhost::NvtxRange nvtx_range("specverify_run");
  if (!h) return SV_ERR_INVALID_ARG;
  if (h->batch == 0) return SV_OK;
  DeviceScope scope(h->device);
  if (!scope.ok()) return SV_ERR_CUDA;
  return enqueue(h, target_logits, draft_logits, draft_tokens, u_accept, u_resample,
                 temperature, out_tokens, out_num_accepted, static_cast<cudaStream_t>(stream));
}

sv_status specverify_run_sampling(specverify_t h, const void* target_logits,
                                  const void* draft_logits, const int32_t* draft_tokens,
                                  const float* u_accept, const float* u_resample,
                                  const float* temperatures, int top_k, float top_p,
                                  int32_t* out_tokens, int32_t* out_num_accepted, void* stream) {
  svhost::NvtxRange nvtx_range("specverify_run_sampling");
  if (!h) return SV_ERR_INVALID_ARG;
  if (h->batch == 0) return SV_OK;
  const int G = h->gamma;
  const size_t es = elem_size(h->dtype);
  if (!target_logits || !u_resample || !temperatures || !out_tokens || !out_num_accepted)
    return SV_ERR_INVALID_ARG;
  if (G > 0 && (!draft_logits || !draft_tokens || !u_accept)) return SV_ERR_INVALID_ARG;
  if (!aligned_to(target_logits, es) || (G > 0 && !aligned_to(draft_logits, es)))
    return SV_ERR_INVALID_ARG;
  if (!aligned_to(draft_tokens, 4) || !aligned_to(u_accept, 4) || !aligned_to(u_resample, 4) ||
      !aligned_to(temperatures, 4) || !aligned_to(out_tokens, 4) ||
      !aligned_to(out_num_accepted, 4))
    return SV_ERR_INVALID_ARG;
  if (top_k < 0 || std::isnan(top_p) || !(top_p > 0.f)) return SV_ERR_INVALID_ARG;
  DeviceScope scope(h->device);
  if (!scope.ok()) return SV_ERR_CUDA;
  specsamp::SampParams p;
  p.target = target_logits;
  p.draft = draft_logits;
  p.tokens = draft_tokens;
  p.u_accept = u_accept;
  p.u_resample = u_resample;
  p.temperature = temperatures;
  p.out_tokens = out_tokens;
  p.out_num_accepted = out_num_accepted;
  p.rows = h->samp_rows;
  p.decision = h->samp_decision;
  p.tstat = h->tstat;
  p.dstat = h->dstat;
  p.pos = h->pos;
  p.resid_mass = h->resid;
  p.status = h->status;
  p.batch = h->batch;
  p.gamma = G;
  p.vocab = h->vocab;
  p.top_k = (top_k >= h->vocab) ? 0 : top_k;
  p.top_p = (top_p >= 1.f) ? 1.0 : static_cast<double>(top_p);
  // Candidate room (dynamic shared memory, so blocks per SM): a small top-k
  // set or no filter fits in the small one; a nucleus cut alone takes the
  // room of the band histograms; a larger top-k set, room for its k entries
  // and a band or so beyond them.
  const bool small_k = p.top_k > 0 && p.top_k <= specsamp::kSelThreads;
  if (small_k || (p.top_k == 0 && p.top_p >= 1.0)) {
    p.cand_cap = specsamp::kCandSmall;
  } else {
    const int want = p.top_k > 0 ? static_cast<int>(svhost::round_up(static_cast<size_t>(p.top_k) + p.top_k / 4 + 256, 1024)) : 0;
    p.cand_cap = std::min(specsamp::kCand, std::max(specsamp::kBandCap, want));
  }
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const long rows = static_cast<long>(h->batch) * (2L * G + 1);
  const int per = specsamp::kDecideThreads / specsamp::kWarp;
  cudaError_t e;
  const bool aligned = aligned_to(target_logits, 16) && (G == 0 || aligned_to(draft_logits, 16)) &&
                       (static_cast<size_t>(h->vocab) * es) % 16 == 0;
  cudaEvent_t* ev = nullptr;
  if (h->prof_runs < h->prof_capacity) ev = h->events.data() + 3 * (h->prof_runs++);
  if (h->dtype == SV_DTYPE_BF16)
    e = aligned ? launch_sampling<__nv_bfloat16, true>(p, rows, per, s, ev)
                : launch_sampling<__nv_bfloat16, false>(p, rows, per, s, ev);
  else
    e = aligned ? launch_sampling<float, true>(p, rows, per, s, ev)
                : launch_sampling<float, false>(p, rows, per, s, ev);
  if (e != cudaSuccess) return cuda_fail(e);
  return SV_OK;
}

sv_status specverify_debug_kept(specverify_t h, int32_t* kept_target, int32_t* kept_draft,
                                void* stream) {
  if (!h) return SV_ERR_INVALID_ARG;
  DeviceScope scope(h->device);
  if (!scope.ok()) return SV_ERR_CUDA;
  const size_t nT = static_cast<size_t>(h->batch) * (h->gamma + 1);
  const size_t nD = static_cast<size_t>(h->batch) * h->gamma;
  std::vector<RowStat> ts(nT), ds(nD);
  cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
  if (e == cudaSuccess && nT) e = cudaMemcpy(ts.data(), h->tstat, nT * sizeof(RowStat), cudaMemcpyDeviceToHost);
  if (e == cudaSuccess && nD) e = cudaMemcpy(ds.data(), h->dstat, nD * sizeof(RowStat), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(e);
  for (size_t i = 0; i < nT; ++i)
    if (kept_target) kept_target[i] = ts[i].pad;
  for (size_t i = 0; i < nD; ++i)
    if (kept_draft) kept_draft[i] = ds[i].pad;
  return SV_OK;
}

sv_status specverify_run_mapped(specverify_t h, const void* target_rows, int n_target_rows,
                                const int32_t* target_map, const void* draft_rows,
                                int n_draft_rows, const int32_t* draft_map,
                                const int32_t* draft_tokens, const float* u_accept,
                                const float* u_resample, float temperature, int32_t* out_tokens,
                                int32_t* out_num_accepted, void* stream) {
  svhost::NvtxRange nvtx_range("specverify_run_mapped");
  if (!h) return SV_ERR_INVALID_ARG;
  if (h->batch == 0) return SV_OK;
  const int G = h->gamma;
  const long nT = static_cast<long>(h->batch) * (G + 1);
  const long nD = static_cast<long>(h->batch) * G;
  if (!target_map || n_target_rows < 1 || n_target_rows > nT) return SV_ERR_INVALID_ARG;
  if (G > 0 && (!draft_map || n_draft_rows < 1 || n_draft_rows > nD)) return SV_ERR_INVALID_ARG;
  if (G == 0) n_draft_rows = 0;
  DeviceScope scope(h->device);
  if (!scope.ok()) return SV_ERR_CUDA;
  return enqueue(h, target_rows, draft_rows, draft_tokens, u_accept, u_resample, temperature,
                 out_tokens, out_num_accepted, static_cast<cudaStream_t>(stream), target_map,
                 G > 0 ? draft_map : nullptr, n_target_rows, n_draft_rows);
}

sv_status specverify_run_host(specverify_t h, const void* target_logits,
                              const void* draft_logits, const int32_t* draft_tokens,
                              const float* u_accept, const float* u_resample, float temperature,
                              int32_t* out_tokens, int32_t* out_num_accepted, void* stream) {
  svhost::NvtxRange nvtx_range("specverify_run_host");
  if (!h) return SV_ERR_INVALID_ARG;
  if (h->batch == 0) return SV_OK;
  const int G = h->gamma;
  if (!target_logits || !u_resample || !out_tokens || !out_num_accepted) return SV_ERR_INVALID_ARG;
  if (G > 0 && (!draft_logits || !draft_tokens || !u_accept)) return SV_ERR_INVALID_ARG;
  DeviceScope scope(h->device);
  if (!scope.ok()) return SV_ERR_CUDA;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const size_t B = static_cast<size_t>(h->batch);
  const size_t es = elem_size(h->dtype);
  const size_t bT = B * (G + 1) * h->vocab * es;
  const size_t bD = B * G * h->vocab * es;
  const size_t bK = B * G * sizeof(int32_t);
  const size_t bUA = B * G * sizeof(float);
  const size_t bUR = B * sizeof(float);
  const size_t bOT = B * (G + 1) * sizeof(int32_t);
  const size_t bON = B * sizeof(int32_t);
  const size_t oT = 0, oD = round_up(oT + bT, 256), oK = round_up(oD + bD, 256),
               oUA = round_up(oK + bK, 256), oUR = round_up(oUA + bUA, 256),
               oOT = round_up(oUR + bUR, 256), oON = round_up(oOT + bOT, 256),
               total = round_up(oON + bON, 256);
  cudaError_t e;
  if (h->stage_bytes < total) {
    if (h->stage) {
      e = cudaStreamSynchronize(s);
      if (e != cudaSuccess) return cuda_fail(e);
      cudaFree(h->stage);
      h->stage = nullptr;
      h->stage_bytes = 0;
    }
    e = cudaMalloc(&h->stage, total);
    if (e != cudaSuccess) return cuda_fail(e);
    h->stage_bytes = total;
  }
  char* d = static_cast<char*>(h->stage);
  e = cudaMemcpyAsync(d + oT, target_logits, bT, cudaMemcpyHostToDevice, s);
  if (e == cudaSuccess && G > 0) e = cudaMemcpyAsync(d + oD, draft_logits, bD, cudaMemcpyHostToDevice, s);
  if (e == cudaSuccess && G > 0) e = cudaMemcpyAsync(d + oK, draft_tokens, bK, cudaMemcpyHostToDevice, s);
  if (e == cudaSuccess && G > 0) e = cudaMemcpyAsync(d + oUA, u_accept, bUA, cudaMemcpyHostToDevice, s);
  if (e == cudaSuccess) e = cudaMemcpyAsync(d + oUR, u_resample, bUR, cudaMemcpyHostToDevice, s);
  if (e != cudaSuccess) return cuda_fail(e);
  sv_status st = enqueue(h, d + oT, d + oD, reinterpret_cast<int32_t*>(d + oK),
                         reinterpret_cast<float*>(d + oUA), reinterpret_cast<float*>(d + oUR),
                         temperature, reinterpret_cast<int32_t*>(d + oOT),
                         reinterpret_cast<int32_t*>(d + oON), s);
  if (st != SV_OK) return st;
  e = cudaMemcpyAsync(out_tokens, d + oOT, bOT, cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaMemcpyAsync(out_num_accepted, d + oON, bON, cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_fail(e);
  return SV_OK;
}

void specverify_destroy(specverify_t h) {
  if (!h) return;
  {
    DeviceScope scope(h->device);
    if (scope.ok()) {
      cudaDeviceSynchronize();
      for (cudaEvent_t ev : h->events) cudaEventDestroy(ev);
      if (h->stage) cudaFree(h->stage);
      if (h->ws) cudaFree(h->ws);
    }
  }
  delete h;
}

sv_status specverify_get_status(specverify_t h, void* stream, uint32_t* bits) {
  if (!h) return SV_ERR_INVALID_ARG;
  DeviceScope scope(h->device);
  if (!scope.ok()) return SV_ERR_CUDA;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  unsigned v = 0;
  cudaError_t e = cudaMemcpyAsync(&v, h->status, sizeof v, cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaMemsetAsync(h->status, 0, sizeof(unsigned), s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_fail(e);
  if (bits) *bits = v;
  if (v & specverify::kStatWait) {
    // a wait of the single launch ran out: its control words may be left
    // nonzero; clear them so that the next run starts clean
    e = cudaMemsetAsync(h->fctl, 0, (2 + 3 * static_cast<size_t>(h->batch)) * sizeof(unsigned), s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return cuda_fail(e);
    return SV_ERR_PIPELINE;
  }
  if (v & specverify::kStatBounds) return SV_ERR_BOUNDS;
  if (v & specverify::kStatRowIndex) return SV_ERR_ROW_INDEX;
  if (v & specsamp::kStatTemperature) return SV_ERR_TEMPERATURE;
  if (v & specverify::kStatTokenRange) return SV_ERR_TOKEN_RANGE;
  if (v & specverify::kStatNonFinite) return SV_ERR_NONFINITE;
  if (v & specverify::kStatZeroMass) return SV_WARN_ZERO_MASS;
  return SV_OK;
}

sv_status specverify_debug_readback(specverify_t h, double* target_lse, double* draft_lse,
                                   double* q_tok, double* p_tok, double* ratio,
                                   double* resid_mass, void* stream) {
  if (!h) return SV_ERR_INVALID_ARG;
  DeviceScope scope(h->device);
  if (!scope.ok()) return SV_ERR_CUDA;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const size_t nT = static_cast<size_t>(h->batch) * (h->gamma + 1);
  const size_t nD = static_cast<size_t>(h->batch) * h->gamma;
  std::vector<RowStat> ts(nT), ds(nD);
  std::vector<PosInfo> ps(nD);
  std::vector<double> rm(h->batch);
  cudaError_t e = cudaStreamSynchronize(s);
  if (e == cudaSuccess && nT) e = cudaMemcpy(ts.data(), h->tstat, nT * sizeof(RowStat), cudaMemcpyDeviceToHost);
  if (e == cudaSuccess && nD) e = cudaMemcpy(ds.data(), h->dstat, nD * sizeof(RowStat), cudaMemcpyDeviceToHost);
  if (e == cudaSuccess && nD) e = cudaMemcpy(ps.data(), h->pos, nD * sizeof(PosInfo), cudaMemcpyDeviceToHost);
  if (e == cudaSuccess && h->batch) e = cudaMemcpy(rm.data(), h->resid, h->batch * sizeof(double), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(e);
  const double ln2 = 0.69314718055994530942;
  for (size_t i = 0; i < nT; ++i)
    if (target_lse) target_lse[i] = ts[i].lse2 * ln2;
  for (size_t i = 0; i < nD; ++i) {
    if (draft_lse) draft_lse[i] = ds[i].lse2 * ln2;
    if (q_tok) q_tok[i] = ps[i].q_tok;
    if (p_tok) p_tok[i] = ps[i].p_tok;
    if (ratio) ratio[i] = ps[i].ratio;
  }
  if (resid_mass)
    for (int b = 0; b < h->batch; ++b) resid_mass[b] = rm[b];
  return SV_OK;
}

sv_status specverify_set_launch(specverify_t h, int slices, int threads, int draw_slices) {
  if (!h) return SV_ERR_INVALID_ARG;
  if (slices < 1 || slices > h->max_slices) return SV_ERR_INVALID_ARG;
  if (threads != 128 && threads != 256 && threads != 512) return SV_ERR_INVALID_ARG;
  if (draw_slices > 64) return SV_ERR_INVALID_ARG;
  h->slices = slices;
  h->threads = threads;
  h->taper_tail = 0;  // an explicit shape cuts every row alike
  h->taper_slices = 0;
  h->draw_slices = (draw_slices >= 1) ? draw_slices : draw_shape(h);
  return SV_OK;
}

sv_status specverify_get_launch(specverify_t h, int* slices, int* threads, int* max_slices,
                                int* draw_slices) {
  if (!h) return SV_ERR_INVALID_ARG;
  if (max_slices) *max_slices = h->max_slices;
  if (slices) *slices = h->slices;
  if (threads) *threads = h->threads;
  if (draw_slices) *draw_slices = h->draw_slices;
  return SV_OK;
}

sv_status specverify_kernels_per_run(specverify_t h, int mapped, int* kernels) {
  if (!h || !kernels) return SV_ERR_INVALID_ARG;
  // statistics, decide, draw; one launch for an unmapped run in fused mode
  // (the count for 16-byte aligned logits with vocab * sizeof(dtype) a
  // multiple of 16)
  if (h->batch == 0) *kernels = 0;
  else if (!mapped && use_fused(h, nullptr)) *kernels = 1;
  else *kernels = 3;
  return SV_OK;
}

sv_status specverify_set_fused(specverify_t h, int enable, int unit_groups, int chunk_tiles,
                               int lag) {
  if (!h) return SV_ERR_INVALID_ARG;
  if (unit_groups != 0) {
    if (unit_groups < 128 || unit_groups > (1 << 20)) return SV_ERR_INVALID_ARG;
    const long nu = (num_groups(h) + unit_groups - 1) / unit_groups;
    if (nu > h->max_slices) return SV_ERR_INVALID_ARG;
  }
  if (chunk_tiles < 0 || chunk_tiles > 4096) return SV_ERR_INVALID_ARG;
  if (lag < -1) return SV_ERR_INVALID_ARG;
  if (enable && h->fused_blocks_per_sm < 1) return SV_ERR_UNSUPPORTED;
  h->fused = enable ? 1 : 0;
  if (unit_groups != 0) h->fused_unit_groups = unit_groups;
  else {
    // default: 1024 groups (16 KB), fewer units if the table has no room
    long ug = 1024;
    while ((num_groups(h) + ug - 1) / ug > h->max_slices) ug *= 2;
    h->fused_unit_groups = static_cast<int>(ug);
  }
  h->fused_chunk_tiles = chunk_tiles ? chunk_tiles : 8;
  h->fused_lag = lag;
  return SV_OK;
}

sv_status specverify_get_fused(specverify_t h, int* enabled, int* unit_groups, int* chunk_tiles,
                               int* lag) {
  if (!h) return SV_ERR_INVALID_ARG;
  const specverify::FusedShape fs = fused_shape_of(h);
  if (enabled) *enabled = use_fused(h, nullptr) ? 1 : 0;
  if (unit_groups) *unit_groups = h->fused_unit_groups;
  if (chunk_tiles) *chunk_tiles = h->fused_chunk_tiles;
  if (lag) *lag = fs.lag;
  return SV_OK;
}

sv_status specverify_profile_begin(specverify_t h, int max_runs) {
  if (!h || max_runs < 0 || max_runs > (1 << 20)) return SV_ERR_INVALID_ARG;
  DeviceScope scope(h->device);
  if (!scope.ok()) return SV_ERR_CUDA;
  cudaError_t e = cudaDeviceSynchronize();
  if (e != cudaSuccess) return cuda_fail(e);
  for (cudaEvent_t ev : h->events) cudaEventDestroy(ev);
  h->events.clear();
  h->prof_runs = 0;
  h->prof_capacity = 0;
  for (int i = 0; i < 3 * max_runs; ++i) {
    cudaEvent_t ev;
    e = cudaEventCreate(&ev);
    if (e != cudaSuccess) return cuda_fail(e);
    h->events.push_back(ev);
  }
  h->prof_capacity = max_runs;
  return SV_OK;
}

sv_status specverify_profile_end(specverify_t h, float* stats_ms, float* draw_ms, int* runs) {
  if (!h) return SV_ERR_INVALID_ARG;
  DeviceScope scope(h->device);
  if (!scope.ok()) return SV_ERR_CUDA;
  const int n = h->prof_runs;
  double t[2] = {0.0, 0.0};
  cudaError_t e = cudaSuccess;
  if (n > 0) e = cudaEventSynchronize(h->events[3 * (n - 1) + 2]);
  for (int r = 0; r < n && e == cudaSuccess; ++r) {
    for (int k = 0; k < 2 && e == cudaSuccess; ++k) {
      float ms = 0.f;
      e = cudaEventElapsedTime(&ms, h->events[3 * r + k], h->events[3 * r + k + 1]);
      t[k] += ms;
    }
  }
  for (cudaEvent_t ev : h->events) cudaEventDestroy(ev);
  h->events.clear();
  h->prof_capacity = 0;
  h->prof_runs = 0;
  if (e != cudaSuccess) return cuda_fail(e);
  if (stats_ms) *stats_ms = n ? static_cast<float>(t[0] / n) : 0.f;
  if (draw_ms) *draw_ms = n ? static_cast<float>(t[1] / n) : 0.f;
  if (runs) *runs = n;
  return SV_OK;
}

const char* specverify_status_string(sv_status s) {
  switch (s) {
    case SV_OK: return "ok";
    case SV_ERR_INVALID_ARG: return "invalid argument";
    case SV_ERR_CUDA: return "CUDA runtime error";
    case SV_ERR_OOM: return "out of memory";
    case SV_ERR_UNSUPPORTED: return "unsupported device (needs sm_100)";
    case SV_ERR_TOKEN_RANGE: return "draft token outside [0, vocab)";
    case SV_ERR_NONFINITE: return "logit row with NaN/+inf or no finite entry";
    case SV_WARN_ZERO_MASS: return "zero residual mass; drew from the target distribution";
    case SV_ERR_ROW_INDEX: return "row map entry outside the logit rows given";
    case SV_ERR_PARENT: return "parent index out of range, self link or cycle";
    case SV_ERR_TEMPERATURE: return "temperature negative, NaN or infinite";
    case SV_ERR_BOUNDS: return "device: a bounds check of a debug build failed";
    case SV_ERR_PIPELINE: return "a bounded device wait gave up (tensor-core pipeline or single-launch step)";
  }
  return "unknown status";
}

const char* specverify_last_error(void) { return g_last_error; }

}  // extern "C"

// ---------------------------------------------------------------------------
// Allocation-free entry point
//
// For callers that cannot allocate device memory: code running inside a
// captured CUDA graph region that must not call cudaMalloc, embedders whose
// device memory is owned by a pool or allocator they cannot reach from this
// library, and runtimes that forbid allocation on their serving path.  The
// workspace then lives in one file-scope device array; only its address is
// looked up, once per device.
// ---------------------------------------------------------------------------

namespace {

constexpr size_t kNoAllocScratchBytes = size_t{16} << 20;  // 16 MiB on every device
constexpr int kNoAllocMaxDevices = 64;

// Device storage of the allocation-free path.  Host code must never pass
// this name to a kernel: on the host it only stands for the symbol, so its
// device address is taken with cudaGetSymbolAddress below.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

std::mutex g_noalloc_mutex;
char* g_noalloc_base[kNoAllocMaxDevices] = {};  // device address, per device
int g_noalloc_sms[kNoAllocMaxDevices] = {};

// First call on the current device: look up the array's device address
// (with that device current) and the SM count.
sv_status noalloc_setup(int dev, char** base, int* sms) {
  std::lock_guard<std::mutex> lock(g_noalloc_mutex);
  if (!g_noalloc_base[dev]) {
    int major = 0, minor = 0, count = 0;
    cudaError_t e = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&count, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return cuda_fail(e);
    if (major != 10 || minor != 0) {
      std::snprintf(g_last_error, sizeof g_last_error,
                    "device %d is sm_%d%d; this library is built for sm_100a only", dev, major,
                    minor);
      return SV_ERR_UNSUPPORTED;
    }
    void* ptr = nullptr;
    e = cudaGetSymbolAddress(&ptr, g_noalloc_scratch);
    if (e != cudaSuccess) return cuda_fail(e);
    g_noalloc_sms[dev] = count;
    g_noalloc_base[dev] = static_cast<char*>(ptr);
  }
  *base = g_noalloc_base[dev];
  *sms = g_noalloc_sms[dev];
  return SV_OK;
}

}  // namespace

extern "C" sv_status specverify_run_noalloc(int batch, int gamma, int vocab, sv_dtype dtype,
                                            const void* target_logits, const void* draft_logits,
                                            const int32_t* draft_tokens, const float* u_accept,
                                            const float* u_resample, float temperature,
                                            int32_t* out_tokens, int32_t* out_num_accepted,
                                            void* stream) {
  svhost::NvtxRange nvtx_range("specverify_run_noalloc");
  if (batch < 0 || gamma < 0 || gamma > specverify::kMaxGamma || vocab < 1 || vocab > (1 << 30))
    return SV_ERR_INVALID_ARG;
  if (dtype != SV_DTYPE_F32 && dtype != SV_DTYPE_BF16) return SV_ERR_INVALID_ARG;
  if (batch == 0) return SV_OK;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e);
  if (dev < 0 || dev >= kNoAllocMaxDevices) return SV_ERR_UNSUPPORTED;
  char* base = nullptr;
  int sms = 0;
  sv_status st = noalloc_setup(dev, &base, &sms);
  if (st != SV_OK) return st;

  // the same launch shape and workspace layout a handle would use, carved
  // out of the static array (a host-side record only: nothing is allocated)
  specverify_ctx h;
  h.device = dev;
  h.batch = batch;
  h.gamma = gamma;
  h.vocab = vocab;
  h.dtype = dtype;
  h.num_sms = sms;
  {
    const long cap = num_groups(&h) / 128;
    h.max_slices = static_cast<int>(cap < 1 ? 1 : (cap > specverify::kMaxSlices ? specverify::kMaxSlices : cap));
  }
  default_shape(&h);
  h.draw_slices = draw_shape(&h);
  const size_t nT = static_cast<size_t>(batch) * (gamma + 1);
  const size_t nD = static_cast<size_t>(batch) * gamma;
  const size_t nB = static_cast<size_t>(batch);
  const size_t nDraw = nB * static_cast<size_t>(draw_tiles(&h));
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t at = off;
    off = round_up(off + bytes, 256);
    return at;
  };
  const size_t offA = take((nT + nD) * static_cast<size_t>(h.slices) * sizeof(RowPartial));
  const size_t offT = take(nT * sizeof(RowStat));
  const size_t offD = take(nD * sizeof(RowStat));
  const size_t offP = take(nD * sizeof(PosInfo));
  const size_t offC = take(nB * sizeof(SeqDecision));
  const size_t offW = take(nDraw * sizeof(double));
  const size_t offK = take(nB * sizeof(unsigned));
  const size_t offR = take(nB * sizeof(double));
  const size_t offS = take(sizeof(unsigned));
  if (off > kNoAllocScratchBytes) {
    std::snprintf(g_last_error, sizeof g_last_error,
                  "specverify_run_noalloc: this batch needs %zu bytes of scratch; the "
                  "allocation-free entry point has %zu",
                  off, kNoAllocScratchBytes);
    return SV_ERR_INVALID_ARG;
  }
  h.partial = reinterpret_cast<RowPartial*>(base + offA);
  h.tstat = reinterpret_cast<RowStat*>(base + offT);
  h.dstat = reinterpret_cast<RowStat*>(base + offD);
  h.pos = reinterpret_cast<PosInfo*>(base + offP);
  h.decision = reinterpret_cast<SeqDecision*>(base + offC);
  h.draw_mass = reinterpret_cast<double*>(base + offW);
  h.draw_ticket = reinterpret_cast<unsigned*>(base + offK);
  h.resid = reinterpret_cast<double*>(base + offR);
  h.status = reinterpret_cast<unsigned*>(base + offS);

  // a rejected call enqueues nothing: every argument check runs before the
  // array is touched
  const sv_status chk = check_args(&h, target_logits, draft_logits, draft_tokens, u_accept,
                                   u_resample, temperature, out_tokens, out_num_accepted,
                                   nullptr, nullptr);
  if (chk != SV_OK) return chk;

  // the array keeps the previous call's contents: the draw tickets and the
  // status word must start at zero
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  e = cudaMemsetAsync(h.draw_ticket, 0, nB * sizeof(unsigned), s);
  if (e == cudaSuccess) e = cudaMemsetAsync(h.status, 0, sizeof(unsigned), s);
  if (e != cudaSuccess) return cuda_fail(e);
  return enqueue(&h, target_logits, draft_logits, draft_tokens, u_accept, u_resample,
                 temperature, out_tokens, out_num_accepted, s);
}
