// C ABI of the speculative-sampling verification library (see specverify.h).
//
// Host side only: argument checks, the workspace, the launch shape, the
// cluster launch of the fused kernel, host-buffer staging and readbacks.
#include "specverify.h"

#include <cuda_runtime.h>

#include <cmath>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <new>
#include <vector>

#include "verify_kernel.cuh"

using specverify::Params;
using specverify::PosInfo;
using specverify::RowStat;

struct specverify_ctx {
  int device = 0;
  int batch = 0, gamma = 0, vocab = 0;
  sv_dtype dtype = SV_DTYPE_F32;
  int cluster = 1, threads = 256;
  int num_sms = 148;
  void* ws = nullptr;  // one device allocation for the whole workspace
  RowStat* tstat = nullptr;
  RowStat* dstat = nullptr;
  PosInfo* pos = nullptr;
  double* resid = nullptr;
  unsigned* ticket = nullptr;
  unsigned* status = nullptr;
  void* stage = nullptr;  // device staging for host-buffer runs
  size_t stage_bytes = 0;
};

namespace {

thread_local char g_last_error[256] = "";

sv_status cuda_fail(cudaError_t e) {
  std::snprintf(g_last_error, sizeof g_last_error, "%s: %s", cudaGetErrorName(e),
                cudaGetErrorString(e));
  return (e == cudaErrorMemoryAllocation) ? SV_ERR_OOM : SV_ERR_CUDA;
}

// makes the handle's device current for the scope, restores the caller's
class DeviceScope {
 public:
  explicit DeviceScope(int dev) {
    ok_ = cudaGetDevice(&prev_) == cudaSuccess;
    if (ok_ && prev_ != dev) ok_ = cudaSetDevice(dev) == cudaSuccess;
    switched_ = ok_ && prev_ != dev;
  }
  ~DeviceScope() {
    if (switched_) cudaSetDevice(prev_);
  }
  bool ok() const { return ok_; }

 private:
  int prev_ = 0;
  bool ok_ = false;
  bool switched_ = false;
};

size_t elem_size(sv_dtype d) { return d == SV_DTYPE_BF16 ? 2 : 4; }
int group_elems(sv_dtype d) { return d == SV_DTYPE_BF16 ? 8 : 4; }
size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

long num_groups(const specverify_ctx* h) {
  const int ve = group_elems(h->dtype);
  return (static_cast<long>(h->vocab) + ve - 1) / ve;
}

// Default launch shape.  A position's rows are split over `cluster` CTAs;
// aim for at least eight waves of CTAs over the SMs (so the last partial
// wave costs little) while keeping every thread at two or more 16-byte
// groups per row.
void default_shape(specverify_ctx* h) {
  const int threads = 256;
  const long positions = static_cast<long>(h->batch) * (h->gamma + 1);
  const long slots = static_cast<long>(h->num_sms) * (2048 / threads);
  const long ngroups = num_groups(h);
  int best = 1;
  for (int c = 1; c <= specverify::kMaxCluster; ++c) {
    if (ngroups / c < 2L * threads && c > 1) break;
    best = c;
    if (positions * c >= 8 * slots) break;
  }
  h->cluster = best;
  h->threads = threads;
}

template <typename T, int NT, bool A>
cudaError_t launch_shape(const Params& p, int C, long positions, cudaStream_t s) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(positions * C), 1, 1);
  cfg.blockDim = dim3(NT, 1, 1);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = static_cast<unsigned>(C);
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, specverify::verify_kernel<T, NT, A>, p);
}

template <typename T, bool A>
cudaError_t launch_threads(const Params& p, int C, int NT, long positions, cudaStream_t s) {
  switch (NT) {
    case 128: return launch_shape<T, 128, A>(p, C, positions, s);
    case 256: return launch_shape<T, 256, A>(p, C, positions, s);
    case 512: return launch_shape<T, 512, A>(p, C, positions, s);
    default: return cudaErrorInvalidValue;
  }
}

template <typename T>
cudaError_t launch_dtype(const Params& p, int C, int NT, bool aligned, long positions,
                         cudaStream_t s) {
  return aligned ? launch_threads<T, true>(p, C, NT, positions, s)
                 : launch_threads<T, false>(p, C, NT, positions, s);
}

bool aligned_to(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

sv_status enqueue(specverify_t h, const void* target, const void* draft, const int32_t* tokens,
                  const float* u_accept, const float* u_resample, float temperature,
                  int32_t* out_tokens, int32_t* out_num_accepted, cudaStream_t stream) {
  const int G = h->gamma;
  const size_t es = elem_size(h->dtype);
  if (!target || !u_resample || !out_tokens || !out_num_accepted) return SV_ERR_INVALID_ARG;
  if (G > 0 && (!draft || !tokens || !u_accept)) return SV_ERR_INVALID_ARG;
  if (!aligned_to(target, es) || (G > 0 && !aligned_to(draft, es))) return SV_ERR_INVALID_ARG;
  if (!aligned_to(tokens, 4) || !aligned_to(u_accept, 4) || !aligned_to(u_resample, 4) ||
      !aligned_to(out_tokens, 4) || !aligned_to(out_num_accepted, 4))
    return SV_ERR_INVALID_ARG;
  if (!std::isfinite(temperature) || !(temperature > 0.f)) return SV_ERR_INVALID_ARG;

  // log2(e)/T = c_hi + c_lo with c_hi rounded toward zero, so c_lo >= 0;
  // c_lo is kept a normal positive float so that -inf * c_lo stays -inf
  const double c = 1.4426950408889634074 / static_cast<double>(temperature);
  if (!(c < 1e30)) return SV_ERR_INVALID_ARG;
  float c_hi = static_cast<float>(c);
  if (static_cast<double>(c_hi) > c) c_hi = std::nextafter(c_hi, 0.f);
  float c_lo = static_cast<float>(c - static_cast<double>(c_hi));
  if (!(c_lo >= 1e-30f)) c_lo = 1e-30f;

  Params p;
  p.target = target;
  p.draft = draft;
  p.tokens = tokens;
  p.u_accept = u_accept;
  p.u_resample = u_resample;
  p.out_tokens = out_tokens;
  p.out_num_accepted = out_num_accepted;
  p.tstat = h->tstat;
  p.dstat = h->dstat;
  p.pos = h->pos;
  p.resid_mass = h->resid;
  p.ticket = h->ticket;
  p.status = h->status;
  p.batch = h->batch;
  p.gamma = G;
  p.vocab = h->vocab;
  const long ngroups = num_groups(h);
  p.groups_per_cta = static_cast<int>((ngroups + h->cluster - 1) / h->cluster);
  p.c_hi = c_hi;
  p.c_lo = c_lo;
  p.c = c;

  const bool aligned = aligned_to(target, 16) && (G == 0 || aligned_to(draft, 16)) &&
                       (static_cast<size_t>(h->vocab) * es) % 16 == 0;
  const long positions = static_cast<long>(h->batch) * (G + 1);
  cudaError_t e = (h->dtype == SV_DTYPE_BF16)
                      ? launch_dtype<__nv_bfloat16>(p, h->cluster, h->threads, aligned,
                                                    positions, stream)
                      : launch_dtype<float>(p, h->cluster, h->threads, aligned, positions, stream);
  if (e != cudaSuccess) return cuda_fail(e);
  return SV_OK;
}

}  // namespace

extern "C" {

sv_status specverify_create(specverify_t* out, int batch, int gamma, int vocab, sv_dtype dtype,
                            int device) {
  if (!out) return SV_ERR_INVALID_ARG;
  *out = nullptr;
  if (batch < 0 || gamma < 0 || gamma > 4096 || vocab < 1 || vocab > (1 << 30))
    return SV_ERR_INVALID_ARG;
  if (dtype != SV_DTYPE_F32 && dtype != SV_DTYPE_BF16) return SV_ERR_INVALID_ARG;
  const long positions = static_cast<long>(batch) * (gamma + 1);
  if (positions * specverify::kMaxCluster > 0x7fffffffL) return SV_ERR_INVALID_ARG;
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
  default_shape(h);

  const size_t nT = static_cast<size_t>(batch) * (gamma + 1);
  const size_t nD = static_cast<size_t>(batch) * gamma;
  const size_t offT = 0;
  const size_t offD = round_up(offT + nT * sizeof(RowStat), 256);
  const size_t offP = round_up(offD + nD * sizeof(RowStat), 256);
  const size_t offR = round_up(offP + nD * sizeof(PosInfo), 256);
  const size_t offK = round_up(offR + static_cast<size_t>(batch) * sizeof(double), 256);
  const size_t offS = round_up(offK + static_cast<size_t>(batch) * sizeof(unsigned), 256);
  const size_t total = offS + 256;
  e = cudaMalloc(&h->ws, total);
  if (e != cudaSuccess) {
    delete h;
    return cuda_fail(e);
  }
  char* base = static_cast<char*>(h->ws);
  h->tstat = reinterpret_cast<RowStat*>(base + offT);
  h->dstat = reinterpret_cast<RowStat*>(base + offD);
  h->pos = reinterpret_cast<PosInfo*>(base + offP);
  h->resid = reinterpret_cast<double*>(base + offR);
  h->ticket = reinterpret_cast<unsigned*>(base + offK);
  h->status = reinterpret_cast<unsigned*>(base + offS);
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
  if (!h) return SV_ERR_INVALID_ARG;
  if (h->batch == 0) return SV_OK;
  DeviceScope scope(h->device);
  if (!scope.ok()) return SV_ERR_CUDA;
  return enqueue(h, target_logits, draft_logits, draft_tokens, u_accept, u_resample,
                 temperature, out_tokens, out_num_accepted, static_cast<cudaStream_t>(stream));
}

sv_status specverify_run_host(specverify_t h, const void* target_logits,
                              const void* draft_logits, const int32_t* draft_tokens,
                              const float* u_accept, const float* u_resample, float temperature,
                              int32_t* out_tokens, int32_t* out_num_accepted, void* stream) {
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
  if (v & specverify::kStatTokenRange) return SV_ERR_TOKEN_RANGE;
  if (v & specverify::kStatNonFinite) return SV_ERR_NONFINITE;
  if (v & specverify::kStatZeroMass) return SV_WARN_ZERO_MASS;
  return SV_OK;
}

sv_status specverify_debug_readback(specverify_t h, float* target_max, double* target_sum,
                                   float* draft_max, double* draft_sum, double* q_tok,
                                   double* p_tok, double* ratio, double* resid_mass,
                                   void* stream) {
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
  for (size_t i = 0; i < nT; ++i) {
    if (target_max) target_max[i] = ts[i].max;
    if (target_sum) target_sum[i] = ts[i].sum;
  }
  for (size_t i = 0; i < nD; ++i) {
    if (draft_max) draft_max[i] = ds[i].max;
    if (draft_sum) draft_sum[i] = ds[i].sum;
    if (q_tok) q_tok[i] = ps[i].q_tok;
    if (p_tok) p_tok[i] = ps[i].p_tok;
    if (ratio) ratio[i] = ps[i].ratio;
  }
  if (resid_mass)
    for (int b = 0; b < h->batch; ++b) resid_mass[b] = rm[b];
  return SV_OK;
}

sv_status specverify_set_launch(specverify_t h, int cluster_ctas, int threads) {
  if (!h) return SV_ERR_INVALID_ARG;
  if (cluster_ctas < 1 || cluster_ctas > specverify::kMaxCluster) return SV_ERR_INVALID_ARG;
  if (threads != 128 && threads != 256 && threads != 512) return SV_ERR_INVALID_ARG;
  h->cluster = cluster_ctas;
  h->threads = threads;
  return SV_OK;
}

sv_status specverify_get_launch(specverify_t h, int* cluster_ctas, int* threads) {
  if (!h) return SV_ERR_INVALID_ARG;
  if (cluster_ctas) *cluster_ctas = h->cluster;
  if (threads) *threads = h->threads;
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
  }
  return "unknown status";
}

const char* specverify_last_error(void) { return g_last_error; }

}  // extern "C"
