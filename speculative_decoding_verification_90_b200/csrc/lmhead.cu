// C ABI of the verification step fused with the LM head (see specverify_lmhead.h).
//
// Host side only: argument checks, the workspace, the TMA tensor maps, and the
// stream-ordered launches of one step:
//   1. statistics GEMMs (target rows, then draft rows): per-(row, vocabulary
//      tile) softmax partials and the logits at the draft tokens; with kept
//      logits (the default) every row's fp32 logits are stored as well;
//   2. the per-tile partials folded to one per row, and the decide kernel of
//      the plain step on them;
//   3. without kept logits: a gather of the two hidden rows each sequence
//      draws from, and logit GEMMs for those rows (fp32, [batch, vocab] each);
//   4. the draw kernel of the plain step on the rows drawn from.
#include "specverify_lmhead.h"

#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <new>
#include <vector>

#include "host_common.h"
#include "lmhead_kernel.cuh"
#include "verify_kernel.cuh"

using specverify::Params;
using specverify::PosInfo;
using specverify::RowPartial;
using specverify::RowStat;
using specverify::SeqDecision;
using svhost::cuda_fail;
using svhost::DeviceScope;
using svhost::g_last_error;
using svhost::round_up;

struct specverify_lmhead_ctx {
  int device = 0;
  int batch = 0, gamma = 0, vocab = 0, hidden = 0;
  int ntiles = 0;
  int num_sms = 148;
  int draw_slices = 1;  // the draw kernel's grid (blocks)
  long draw_tiles = 1;  // tiles per fp32 row drawn from
  void* ws = nullptr;
  RowPartial* partial = nullptr;   // [(nT + nD) * ntiles] one per row and 256-column tile
  RowPartial* combined = nullptr;  // [nT + nD] one per row
  float* gathered = nullptr;   // [nT + nD]
  RowStat* tstat = nullptr;
  RowStat* dstat = nullptr;
  PosInfo* pos = nullptr;
  SeqDecision* decision = nullptr;
  double* draw_mass = nullptr;
  unsigned* draw_ticket = nullptr;
  double* resid = nullptr;
  unsigned* status = nullptr;
  unsigned* gemm_error = nullptr;
  __nv_bfloat16* xt = nullptr;  // [B, hidden] the rows drawn from
  __nv_bfloat16* xd = nullptr;
  float* lt = nullptr;          // [B, vocab] their logits
  float* ld = nullptr;
  // kept logits: every row's fp32 logits [nT + nD, vocab] (target rows, then
  // draft rows), written by the statistics GEMMs; the draw reads its rows
  // there instead of recomputing them
  int keep_logits = 0;
  float* all_logits = nullptr;
  std::vector<cudaEvent_t> events;  // 3 per recorded run
  int prof_capacity = 0;
  int prof_runs = 0;
};

namespace {

using EncodeTiled = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                 const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                 const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                 CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiled encode_fn() {
  static EncodeTiled fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiled>(p);
  });
  return fn;
}

// a row-major [rows, cols] bf16 matrix, loaded in boxes of box_rows x 64
// (128-byte rows, 128-byte swizzle); rows past the end read as zeros
bool make_map(CUtensorMap* map, const void* base, long rows, int cols, int box_rows) {
  EncodeTiled fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(cols) * 2};
  const cuuint32_t box[2] = {static_cast<cuuint32_t>(lmhead::kBK), static_cast<cuuint32_t>(box_rows)};
  const cuuint32_t estr[2] = {1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool aligned16(const void* p) { return reinterpret_cast<uintptr_t>(p) % 16 == 0; }

// ma: the first hidden tensor (p.rows rows); ma2: the second (p.rows2 rows,
// statistics mode only; pass ma again when there is none); mb: the weight
template <int kMode>
cudaError_t launch_gemm(const CUtensorMap& ma, const CUtensorMap& ma2, const CUtensorMap& mb,
                        const lmhead::LmParams& p, cudaStream_t s) {
  cudaError_t e = cudaFuncSetAttribute(lmhead::gemm_kernel<kMode>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       lmhead::kSmemBytes);
  if (e != cudaSuccess) return e;
  const long tiles = static_cast<long>((p.rows + lmhead::kBM - 1) / lmhead::kBM +
                                       (p.rows2 + lmhead::kBM - 1) / lmhead::kBM) *
                     p.ntiles;
  const long grid = tiles < p.num_sms ? tiles : p.num_sms;  // persistent: one CTA per SM
  lmhead::gemm_kernel<kMode><<<static_cast<unsigned>(grid), lmhead::kPThreads,
                               lmhead::kSmemBytes, s>>>(ma, ma2, mb, p);
  return cudaGetLastError();
}

// the rows each sequence draws from: target row n and draft row n
__global__ void gather_rows_kernel(const __nv_bfloat16* ht, const __nv_bfloat16* hd,
                                   const SeqDecision* decision, int gamma, int hidden,
                                   __nv_bfloat16* xt, __nv_bfloat16* xd) {
  const int b = blockIdx.x;
  const SeqDecision d = decision[b];
  const int n = (d.mode == specverify::kDrawNone) ? 0 : d.n;
  const uint4* st = reinterpret_cast<const uint4*>(ht + (static_cast<long>(b) * (gamma + 1) + n) * hidden);
  uint4* dt = reinterpret_cast<uint4*>(xt + static_cast<long>(b) * hidden);
  const int groups = hidden / 8;
  for (int g = threadIdx.x; g < groups; g += blockDim.x) dt[g] = st[g];
  if (gamma > 0) {
    const int nd = n < gamma ? n : gamma - 1;
    const uint4* sd = reinterpret_cast<const uint4*>(hd + (static_cast<long>(b) * gamma + nd) * hidden);
    uint4* dd = reinterpret_cast<uint4*>(xd + static_cast<long>(b) * hidden);
    for (int g = threadIdx.x; g < groups; g += blockDim.x) dd[g] = sd[g];
  }
}

// one warp per row: the row's per-tile partials (o_t, s_t) folded into one,
// O = max o_t, S = sum s_t 2^(o_t - O) in fp64 (a NaN partial stays visible)
__global__ void __launch_bounds__(256) combine_rows_kernel(const RowPartial* in, int ntiles,
                                                           long rows, RowPartial* out) {
  const int lane = threadIdx.x & 31;
  const long r = static_cast<long>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  cudaGridDependencySynchronize();  // the GEMM's partials (programmatic dependent launch)
  if (r >= rows) return;
  const RowPartial* p = in + r * ntiles;
  float O = -INFINITY;
  for (int t = lane; t < ntiles; t += 32) O = fmaxf(O, p[t].o);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) O = fmaxf(O, __shfl_xor_sync(0xffffffffu, O, o));
  double S = 0.0;
  for (int t = lane; t < ntiles; t += 32) {
    const RowPartial q = p[t];
    S += (q.o == -INFINITY) ? q.s * 0.0 : q.s * exp2(static_cast<double>(q.o) - O);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) S += __shfl_xor_sync(0xffffffffu, S, o);
  if (lane == 0) out[r] = RowPartial{S, O, 0};
}

// a launch that may start before its predecessor on the stream has finished
// (programmatic dependent launch); the kernel waits in a grid-dependency
// barrier before it reads the predecessor's results
template <typename K, typename... A>
cudaError_t launch_pdl(K kernel, unsigned grid, unsigned block, cudaStream_t s, A... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid, 1, 1);
  cfg.blockDim = dim3(block, 1, 1);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, args...);
}

// the kept-logits buffer is allocated by default up to this size
constexpr size_t kKeepDefaultBytes = size_t{16} << 30;

void split_c(float temperature, float& c_hi, float& c_lo, double& c) {
  const double cd = 1.4426950408889634074 / static_cast<double>(temperature);
  c_hi = static_cast<float>(cd);
  if (static_cast<double>(c_hi) > cd) c_hi = std::nextafter(c_hi, 0.f);
  c_lo = static_cast<float>(cd - static_cast<double>(c_hi));
  if (!(c_lo >= 1e-30f)) c_lo = 1e-30f;
  c = static_cast<double>(c_hi) + static_cast<double>(c_lo);
}

}  // namespace

extern "C" {

sv_status specverify_lmhead_create(specverify_lmhead_t* out, int batch, int gamma, int vocab,
                                   int hidden, int device) {
  if (!out) return SV_ERR_INVALID_ARG;
  *out = nullptr;
  if (batch < 1 || gamma < 0 || gamma > specverify::kMaxGamma || vocab < 1 ||
      vocab > 65535 * lmhead::kBN || hidden < lmhead::kBK || hidden % lmhead::kBK != 0 || hidden > (1 << 16))
    return SV_ERR_INVALID_ARG;
  const long nT = static_cast<long>(batch) * (gamma + 1), nD = static_cast<long>(batch) * gamma;
  if (nT + nD > (1L << 30)) return SV_ERR_INVALID_ARG;
  int ndev = 0;
  cudaError_t e = cudaGetDeviceCount(&ndev);
  if (e != cudaSuccess) return cuda_fail(e);
  if (device < 0 || device >= ndev) return SV_ERR_INVALID_ARG;
  int major = 0, minor = 0, sms = 0;
  e = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, device);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, device);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, device);
  if (e != cudaSuccess) return cuda_fail(e);
  if (major != 10 || minor != 0) {
    std::snprintf(g_last_error, sizeof g_last_error,
                  "device %d is sm_%d%d; this library is built for sm_100a only", device, major,
                  minor);
    return SV_ERR_UNSUPPORTED;
  }
  if (!encode_fn()) {
    std::snprintf(g_last_error, sizeof g_last_error, "cuTensorMapEncodeTiled is not available");
    return SV_ERR_UNSUPPORTED;
  }
  DeviceScope scope(device);
  if (!scope.ok()) return SV_ERR_CUDA;
  specverify_lmhead_ctx* h = new (std::nothrow) specverify_lmhead_ctx;
  if (!h) return SV_ERR_OOM;
  h->device = device;
  h->batch = batch;
  h->gamma = gamma;
  h->vocab = vocab;
  h->hidden = hidden;
  h->num_sms = sms;
  h->ntiles = (vocab + lmhead::kBN - 1) / lmhead::kBN;
  // the draw on fp32 rows: the plain step's grid rule (one resident wave at
  // most, one warp per tile at least)
  h->draw_tiles = specverify::draw_tiles_per_row(vocab, 4);
  h->draw_slices = static_cast<int>(specverify::draw_grid(batch, h->draw_tiles, 64, sms));
  const size_t nB = static_cast<size_t>(batch);
  const size_t tiles32 = static_cast<size_t>(h->draw_tiles);
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t at = off;
    off = round_up(off + bytes, 256);
    return at;
  };
  const size_t oP = take(static_cast<size_t>(nT + nD) * h->ntiles * sizeof(RowPartial));
  const size_t oM = take(static_cast<size_t>(nT + nD) * sizeof(RowPartial));
  const size_t oG = take(static_cast<size_t>(nT + nD) * sizeof(float));
  const size_t oT = take(static_cast<size_t>(nT) * sizeof(RowStat));
  const size_t oD = take(static_cast<size_t>(nD > 0 ? nD : 1) * sizeof(RowStat));
  const size_t oQ = take(static_cast<size_t>(nD > 0 ? nD : 1) * sizeof(PosInfo));
  const size_t oC = take(nB * sizeof(SeqDecision));
  const size_t oW = take(nB * tiles32 * sizeof(double));
  const size_t oK = take(nB * sizeof(unsigned));
  const size_t oR = take(nB * sizeof(double));
  const size_t oS = take(sizeof(unsigned));
  const size_t oE = take(sizeof(unsigned));
  // the drawn rows: the B target rows then the B draft rows, contiguous, so
  // that with one output layer a single GEMM tile holds both rows of a
  // sequence pair (hidden states bf16, logits fp32)
  const size_t oXT = take(2 * nB * hidden * 2);
  const size_t oLT = take(2 * nB * static_cast<size_t>(vocab) * 4);
  e = cudaMalloc(&h->ws, off);
  if (e != cudaSuccess) {
    delete h;
    return cuda_fail(e);
  }
  char* b = static_cast<char*>(h->ws);
  h->partial = reinterpret_cast<RowPartial*>(b + oP);
  h->combined = reinterpret_cast<RowPartial*>(b + oM);
  h->gathered = reinterpret_cast<float*>(b + oG);
  h->tstat = reinterpret_cast<RowStat*>(b + oT);
  h->dstat = reinterpret_cast<RowStat*>(b + oD);
  h->pos = reinterpret_cast<PosInfo*>(b + oQ);
  h->decision = reinterpret_cast<SeqDecision*>(b + oC);
  h->draw_mass = reinterpret_cast<double*>(b + oW);
  h->draw_ticket = reinterpret_cast<unsigned*>(b + oK);
  h->resid = reinterpret_cast<double*>(b + oR);
  h->status = reinterpret_cast<unsigned*>(b + oS);
  h->gemm_error = reinterpret_cast<unsigned*>(b + oE);
  h->xt = reinterpret_cast<__nv_bfloat16*>(b + oXT);
  h->xd = h->xt + nB * hidden;
  h->lt = reinterpret_cast<float*>(b + oLT);
  h->ld = h->lt + nB * static_cast<size_t>(vocab);
  e = cudaMemset(h->ws, 0, off);
  if (e == cudaSuccess) e = cudaDeviceSynchronize();
  if (e != cudaSuccess) {
    cudaFree(h->ws);
    delete h;
    return cuda_fail(e);
  }
  // kept logits by default when they take at most kKeepDefaultBytes; an
  // allocation that fails leaves the recomputing form (no error)
  const size_t keep_bytes = static_cast<size_t>(nT + nD) * static_cast<size_t>(vocab) * 4;
  if (keep_bytes <= kKeepDefaultBytes) {
    void* kl = nullptr;
    if (cudaMalloc(&kl, keep_bytes) == cudaSuccess) {
      h->all_logits = static_cast<float*>(kl);
      h->keep_logits = 1;
    } else {
      (void)cudaGetLastError();
    }
  }
  *out = h;
  return SV_OK;
}

sv_status specverify_lmhead_set_keep_logits(specverify_lmhead_t h, int keep) {
  if (!h) return SV_ERR_INVALID_ARG;
  if (keep && !h->all_logits) {
    DeviceScope scope(h->device);
    if (!scope.ok()) return SV_ERR_CUDA;
    const size_t bytes = static_cast<size_t>(h->batch) * (2L * h->gamma + 1) *
                         static_cast<size_t>(h->vocab) * 4;
    void* kl = nullptr;
    const cudaError_t e = cudaMalloc(&kl, bytes);
    if (e != cudaSuccess) return cuda_fail(e);
    h->all_logits = static_cast<float*>(kl);
  }
  h->keep_logits = keep ? 1 : 0;
  return SV_OK;
}

sv_status specverify_lmhead_get_keep_logits(specverify_lmhead_t h, int* keep) {
  if (!h || !keep) return SV_ERR_INVALID_ARG;
  *keep = h->keep_logits;
  return SV_OK;
}

sv_status specverify_lmhead_logits(specverify_lmhead_t h, const void* hidden_rows, int rows,
                                   const void* weight, float* out_logits, void* stream) {
  if (!h || !hidden_rows || !weight || !out_logits || rows < 1) return SV_ERR_INVALID_ARG;
  if (!aligned16(hidden_rows) || !aligned16(weight) || !aligned16(out_logits))
    return SV_ERR_INVALID_ARG;
  DeviceScope scope(h->device);
  if (!scope.ok()) return SV_ERR_CUDA;
  CUtensorMap ma, mb;
  if (!make_map(&ma, hidden_rows, rows, h->hidden, lmhead::kBM) ||
      !make_map(&mb, weight, h->vocab, h->hidden, lmhead::kBN))
    return SV_ERR_INVALID_ARG;
  lmhead::LmParams p{};
  p.rows = rows;
  p.vocab = h->vocab;
  p.hidden = h->hidden;
  p.ntiles = h->ntiles;
  p.num_sms = h->num_sms;
  p.logits = out_logits;
  p.error = h->gemm_error;
  cudaError_t e = launch_gemm<lmhead::kModeLogits>(ma, ma, mb, p, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e);
  return SV_OK;
}

sv_status specverify_lmhead_run(specverify_lmhead_t h, const void* target_hidden,
                                const void* target_weight, const void* draft_hidden,
                                const void* draft_weight, const int32_t* draft_tokens,
                                const float* u_accept, const float* u_resample, float temperature,
                                int32_t* out_tokens, int32_t* out_num_accepted, void* stream) {
  svhost::NvtxRange nvtx_range("specverify_lmhead_run");
  if (!h) return SV_ERR_INVALID_ARG;
  const int B = h->batch, G = h->gamma, V = h->vocab, D = h->hidden;
  if (!target_hidden || !target_weight || !u_resample || !out_tokens || !out_num_accepted)
    return SV_ERR_INVALID_ARG;
  if (G > 0 && (!draft_hidden || !draft_weight || !draft_tokens || !u_accept))
    return SV_ERR_INVALID_ARG;
  if (!aligned16(target_hidden) || !aligned16(target_weight) ||
      (G > 0 && (!aligned16(draft_hidden) || !aligned16(draft_weight))))
    return SV_ERR_INVALID_ARG;
  if (!std::isfinite(temperature) || !(temperature > 0.f)) return SV_ERR_INVALID_ARG;
  DeviceScope scope(h->device);
  if (!scope.ok()) return SV_ERR_CUDA;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const long nT = static_cast<long>(B) * (G + 1), nD = static_cast<long>(B) * G;

  float c_hi, c_lo;
  double c;
  split_c(temperature, c_hi, c_lo, c);
  if (!(c < 1e30)) return SV_ERR_INVALID_ARG;

  CUtensorMap mht, mwt, mhd, mwd, mxt, mxd, mx2;
  if (!make_map(&mht, target_hidden, nT, D, lmhead::kBM) ||
      !make_map(&mwt, target_weight, V, D, lmhead::kBN) ||
      !make_map(&mxt, h->xt, B, D, lmhead::kBM) ||
      !make_map(&mx2, h->xt, 2L * B, D, lmhead::kBM))
    return SV_ERR_INVALID_ARG;
  if (G > 0 && (!make_map(&mhd, draft_hidden, nD, D, lmhead::kBM) ||
                !make_map(&mwd, draft_weight, V, D, lmhead::kBN) ||
                !make_map(&mxd, h->xd, B, D, lmhead::kBM)))
    return SV_ERR_INVALID_ARG;

  cudaEvent_t* ev = nullptr;
  if (h->prof_runs < h->prof_capacity) ev = h->events.data() + 3 * (h->prof_runs++);
  cudaError_t e = ev ? cudaEventRecord(ev[0], s) : cudaSuccess;

  // 1. statistics GEMMs
  lmhead::LmParams g{};
  g.vocab = V;
  g.hidden = D;
  g.ntiles = h->ntiles;
  g.num_sms = h->num_sms;
  g.partial = h->partial;
  g.tokens = draft_tokens;
  g.token_stride = G;
  g.gathered = h->gathered;
  g.c_hi = c_hi;
  g.c_lo = c_lo;
  g.error = h->gemm_error;
  g.rows = static_cast<int>(nT);
  g.row_offset = 0;
  g.positions = G + 1;
  g.rows2 = 0;
  const bool keep = h->keep_logits && h->all_logits;
  g.logits = keep ? h->all_logits : nullptr;  // every row's logits, indexed by row_offset + r
  g.logits2 = g.logits;
  if (G > 0 && draft_weight == target_weight) {
    // one output layer: target and draft rows in one launch, the weight read once
    g.rows2 = static_cast<int>(nD);
    g.row_offset2 = nT;
    g.positions2 = G;
    if (e == cudaSuccess) e = launch_gemm<lmhead::kModeStats>(mht, mhd, mwt, g, s);
  } else {
    if (e == cudaSuccess) e = launch_gemm<lmhead::kModeStats>(mht, mht, mwt, g, s);
    if (G > 0) {
      g.rows = static_cast<int>(nD);
      g.row_offset = nT;
      g.positions = G;
      if (e == cudaSuccess) e = launch_gemm<lmhead::kModeStats>(mhd, mhd, mwd, g, s);
    }
  }
  if (e == cudaSuccess && ev) e = cudaEventRecord(ev[1], s);

  // 2. the decision, on the partials (one per 256-column tile of each row)
  Params p{};
  // the rows drawn from: with kept logits, rows of the [nT + nD, vocab]
  // buffer (unmapped layout); else the compact rows written in step 3
  p.target = keep ? h->all_logits : h->lt;
  p.draft = keep ? h->all_logits + nT * static_cast<long>(V) : h->ld;
  p.target_map = nullptr;
  p.draft_map = nullptr;
  p.target_rows = nT;
  p.draft_rows = nD;
  p.tokens = draft_tokens;
  p.u_accept = u_accept;
  p.u_resample = u_resample;
  p.out_tokens = out_tokens;
  p.out_num_accepted = out_num_accepted;
  p.partial = h->combined;
  p.tstat = h->tstat;
  p.dstat = h->dstat;
  p.pos = h->pos;
  p.decision = h->decision;
  p.draw_mass = h->draw_mass;
  p.draw_ticket = h->draw_ticket;
  p.resid_mass = h->resid;
  p.status = h->status;
  p.batch = B;
  p.gamma = G;
  p.vocab = V;
  p.slices = 1;  // the per-tile partials are folded first
  p.groups_per_slice = 0;
  p.draw_tiles = h->draw_tiles;
  p.c_hi = c_hi;
  p.c_lo = c_lo;
  p.c = c;
  p.gathered_target = h->gathered;
  p.gathered_draft = h->gathered + nT;
  p.draw_compact = keep ? 0 : 1;
  if (e == cudaSuccess)
    e = launch_pdl(combine_rows_kernel, static_cast<unsigned>((nT + nD + 7) / 8), 256u, s,
                   static_cast<const RowPartial*>(h->partial), h->ntiles, nT + nD, h->combined);
  const int per = specverify::kDecideThreads / specverify::kWarp;
  if (e == cudaSuccess)
    e = launch_pdl(specverify::decide_kernel<float>, static_cast<unsigned>((B + per - 1) / per),
                   static_cast<unsigned>(specverify::kDecideThreads), s, p);

  // 3. without kept logits: the two rows each sequence draws from, and their logits
  if (e == cudaSuccess && !keep) {
    gather_rows_kernel<<<B, 256, 0, s>>>(static_cast<const __nv_bfloat16*>(target_hidden),
                                         static_cast<const __nv_bfloat16*>(draft_hidden),
                                         h->decision, G, D, h->xt, h->xd);
    e = cudaGetLastError();
  }
  lmhead::LmParams l{};
  l.rows = B;
  l.vocab = V;
  l.hidden = D;
  l.ntiles = h->ntiles;
  l.num_sms = h->num_sms;
  l.error = h->gemm_error;
  l.logits = h->lt;
  if (keep) {
    // the rows drawn from are in the kept logits
  } else if (G > 0 && draft_weight == target_weight) {
    // one output layer: the 2B drawn rows (target rows, then draft rows, one
    // tensor) as one GEMM, so each weight tile is read once for both
    l.rows = 2 * B;
    l.rows2 = 0;
    if (e == cudaSuccess) e = launch_gemm<lmhead::kModeLogits>(mx2, mx2, mwt, l, s);
  } else {
    if (e == cudaSuccess) e = launch_gemm<lmhead::kModeLogits>(mxt, mxt, mwt, l, s);
    if (G > 0) {
      l.logits = h->ld;
      if (e == cudaSuccess) e = launch_gemm<lmhead::kModeLogits>(mxd, mxd, mwd, l, s);
    }
  }

  // 4. the draw on fp32 rows
  const bool aligned = (static_cast<size_t>(V) * 4) % 16 == 0;
  if (e == cudaSuccess)
    e = aligned ? specverify::launch_draw<float, true>(p, static_cast<unsigned>(h->draw_slices), s, true)
                : specverify::launch_draw<float, false>(p, static_cast<unsigned>(h->draw_slices), s, true);
  if (e == cudaSuccess && ev) e = cudaEventRecord(ev[2], s);
  if (e != cudaSuccess) return cuda_fail(e);
  return SV_OK;
}

sv_status specverify_lmhead_get_status(specverify_lmhead_t h, void* stream, uint32_t* bits) {
  if (!h) return SV_ERR_INVALID_ARG;
  DeviceScope scope(h->device);
  if (!scope.ok()) return SV_ERR_CUDA;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  unsigned v[2] = {0, 0};
  cudaError_t e = cudaMemcpyAsync(&v[0], h->status, sizeof(unsigned), cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaMemcpyAsync(&v[1], h->gemm_error, sizeof(unsigned), cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaMemsetAsync(h->status, 0, sizeof(unsigned), s);
  if (e == cudaSuccess) e = cudaMemsetAsync(h->gemm_error, 0, sizeof(unsigned), s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_fail(e);
  const unsigned all = v[0] | (v[1] ? 32u : 0u);
  if (bits) *bits = all;
  if (v[1]) return SV_ERR_PIPELINE;
  if (v[0] & specverify::kStatTokenRange) return SV_ERR_TOKEN_RANGE;
  if (v[0] & specverify::kStatNonFinite) return SV_ERR_NONFINITE;
  if (v[0] & specverify::kStatZeroMass) return SV_WARN_ZERO_MASS;
  return SV_OK;
}

sv_status specverify_lmhead_readback(specverify_lmhead_t h, double* target_lse,
                                     double* draft_lse, double* q_tok, double* p_tok,
                                     double* resid_mass, void* stream) {
  if (!h) return SV_ERR_INVALID_ARG;
  DeviceScope scope(h->device);
  if (!scope.ok()) return SV_ERR_CUDA;
  const size_t nT = static_cast<size_t>(h->batch) * (h->gamma + 1);
  const size_t nD = static_cast<size_t>(h->batch) * h->gamma;
  std::vector<RowStat> ts(nT), ds(nD);
  std::vector<PosInfo> ps(nD);
  std::vector<double> rm(h->batch);
  cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
  if (e == cudaSuccess) e = cudaMemcpy(ts.data(), h->tstat, nT * sizeof(RowStat), cudaMemcpyDeviceToHost);
  if (e == cudaSuccess && nD) e = cudaMemcpy(ds.data(), h->dstat, nD * sizeof(RowStat), cudaMemcpyDeviceToHost);
  if (e == cudaSuccess && nD) e = cudaMemcpy(ps.data(), h->pos, nD * sizeof(PosInfo), cudaMemcpyDeviceToHost);
  if (e == cudaSuccess) e = cudaMemcpy(rm.data(), h->resid, h->batch * sizeof(double), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(e);
  const double ln2 = 0.69314718055994530942;
  for (size_t i = 0; i < nT; ++i)
    if (target_lse) target_lse[i] = ts[i].lse2 * ln2;
  for (size_t i = 0; i < nD; ++i) {
    if (draft_lse) draft_lse[i] = ds[i].lse2 * ln2;
    if (q_tok) q_tok[i] = ps[i].q_tok;
    if (p_tok) p_tok[i] = ps[i].p_tok;
  }
  if (resid_mass)
    for (int b = 0; b < h->batch; ++b) resid_mass[b] = rm[b];
  return SV_OK;
}

sv_status specverify_lmhead_profile_begin(specverify_lmhead_t h, int max_runs) {
  if (!h || max_runs < 0 || max_runs > (1 << 20)) return SV_ERR_INVALID_ARG;
  DeviceScope scope(h->device);
  if (!scope.ok()) return SV_ERR_CUDA;
  cudaError_t e = cudaDeviceSynchronize();
  if (e != cudaSuccess) return cuda_fail(e);
  for (cudaEvent_t ev : h->events) cudaEventDestroy(ev);
  h->events.clear();
  h->prof_capacity = 0;
  h->prof_runs = 0;
  for (int i = 0; i < 3 * max_runs; ++i) {
    cudaEvent_t ev;
    e = cudaEventCreate(&ev);
    if (e != cudaSuccess) return cuda_fail(e);
    h->events.push_back(ev);
  }
  h->prof_capacity = max_runs;
  return SV_OK;
}

sv_status specverify_lmhead_profile_end(specverify_lmhead_t h, float* stats_ms, float* rest_ms,
                                        int* runs) {
  if (!h) return SV_ERR_INVALID_ARG;
  DeviceScope scope(h->device);
  if (!scope.ok()) return SV_ERR_CUDA;
  double a = 0.0, c = 0.0;
  for (int r = 0; r < h->prof_runs; ++r) {
    cudaEvent_t* ev = h->events.data() + 3 * r;
    float t1 = 0.f, t2 = 0.f;
    cudaError_t e = cudaEventSynchronize(ev[2]);
    if (e == cudaSuccess) e = cudaEventElapsedTime(&t1, ev[0], ev[1]);
    if (e == cudaSuccess) e = cudaEventElapsedTime(&t2, ev[1], ev[2]);
    if (e != cudaSuccess) return cuda_fail(e);
    a += t1;
    c += t2;
  }
  const int n = h->prof_runs;
  if (stats_ms) *stats_ms = n ? static_cast<float>(a / n) : 0.f;
  if (rest_ms) *rest_ms = n ? static_cast<float>(c / n) : 0.f;
  if (runs) *runs = n;
  for (cudaEvent_t ev : h->events) cudaEventDestroy(ev);
  h->events.clear();
  h->prof_capacity = 0;
  h->prof_runs = 0;
  return SV_OK;
}

void specverify_lmhead_destroy(specverify_lmhead_t h) {
  if (!h) return;
  {
    DeviceScope scope(h->device);
    if (scope.ok()) {
      cudaDeviceSynchronize();
      for (cudaEvent_t ev : h->events) cudaEventDestroy(ev);
      if (h->ws) cudaFree(h->ws);
      if (h->all_logits) cudaFree(h->all_logits);
    }
  }
  delete h;
}

}  // extern "C"
