// C ABI of the multi-branch fold gate (see specfold_gate.h).
//
// Host side only: argument checks, the workspace, the three stream-ordered
// launches of one pass, per-kernel event timing.
#include "specfold_gate.h"

#include <cuda_runtime.h>

#include <cmath>
#include <cstdio>
#include <new>
#include <vector>

#include "gate_kernel.cuh"
#include "host_common.h"

using specfold::GateParams;
using svhost::cuda_fail;
using svhost::DeviceScope;
using svhost::g_last_error;
using svhost::round_up;

struct specfold_gate_ctx {
  int device = 0;
  int branches = 0, positions = 0, dim = 0;
  long rows = 0;
  int blocks = 0;       // difference kernel (persistent)
  int bulk_stages = 0;  // bulk-copy difference kernel: ring stages (0: register form only)
  int bulk_consumers = 0;  // its consumer warps (bulk_stages is a multiple)
  int bulk_parts = 1;      // stage loads per row pair (2: half rows)
  int bulk_blocks = 0;  // its grid: one block per SM
  int pack_blocks = 0;  // packing kernel
  sv_dtype dtype = SV_DTYPE_F32;
  void* ws = nullptr;
  int32_t* eff_parent = nullptr;
  uint8_t* flag = nullptr;
  int32_t* rank = nullptr;
  int32_t* prov = nullptr;
  unsigned* status = nullptr;
  // optional timing: 3 events per recorded run (before rows, after rows, after pack)
  std::vector<cudaEvent_t> events;
  int prof_capacity = 0;
  int prof_runs = 0;
};

namespace {

size_t gate_elem_size(sv_dtype d) { return d == SV_DTYPE_BF16 ? 2 : 4; }
bool gate_aligned(const void* p, size_t a) { return reinterpret_cast<uintptr_t>(p) % a == 0; }

template <typename K>
cudaError_t launch_pdl(K kernel, unsigned grid, unsigned block, size_t smem, cudaStream_t s,
                       const GateParams& p) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(block);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, p);
}

template <typename T, bool A>
cudaError_t launch_pass(const GateParams& p, int bulk_blocks, cudaStream_t s, cudaEvent_t* ev) {
  const size_t smem = 2 * sizeof(int32_t) * static_cast<size_t>(p.branches);
  cudaError_t e = cudaSuccess;
  specfold::tree_kernel<<<1, specfold::kTreeThreads, smem, s>>>(p);
  e = cudaGetLastError();
  if (e == cudaSuccess && ev) e = cudaEventRecord(ev[0], s);
  if (e == cudaSuccess) {
    if (A && p.bulk_stages > 0)
      e = launch_pdl(specfold::rows_bulk_kernel<T>, static_cast<unsigned>(bulk_blocks),
                     static_cast<unsigned>(p.bulk_consumers * specfold::kWarp),
                     static_cast<size_t>(p.bulk_stages) * 2 * sizeof(T) * p.dim / p.bulk_parts, s,
                     p);
    else
      e = launch_pdl(specfold::rows_kernel<T, A>, static_cast<unsigned>(p.blocks),
                     specfold::kThreads, 0, s, p);
  }
  if (e == cudaSuccess && ev) e = cudaEventRecord(ev[1], s);
  if (e == cudaSuccess)
    e = launch_pdl(specfold::scan_kernel, 1u, specfold::kSlotThreads, 0, s, p);
  if (e == cudaSuccess)
    e = launch_pdl(specfold::pack_kernel<T, A>, static_cast<unsigned>(p.pack_blocks),
                   specfold::kThreads, 0, s, p);
  if (e == cudaSuccess && ev) e = cudaEventRecord(ev[2], s);
  return e;
}

}  // namespace

extern "C" {

sv_status specfold_gate_create(specfold_gate_t* out, int branches, int positions, int dim,
                               sv_dtype dtype, int device) {
  if (!out) return SV_ERR_INVALID_ARG;
  *out = nullptr;
  if (branches < 1 || branches > specfold::kMaxBranches || positions < 1 || dim < 1 ||
      dim > (1 << 20))
    return SV_ERR_INVALID_ARG;
  const long rows = static_cast<long>(branches) * positions;
  if (rows >= 0x7fffffffL) return SV_ERR_INVALID_ARG;
  if (dtype != SV_DTYPE_F32 && dtype != SV_DTYPE_BF16) return SV_ERR_INVALID_ARG;
  int ndev = 0;
  cudaError_t e = cudaGetDeviceCount(&ndev);
  if (e != cudaSuccess) return cuda_fail(e);
  if (device < 0 || device >= ndev) return SV_ERR_INVALID_ARG;
  int major = 0, minor = 0;
  e = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, device);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, device);
  if (e != cudaSuccess) return cuda_fail(e);
  if (major != 10 || minor != 0) {
    std::snprintf(g_last_error, sizeof g_last_error,
                  "device %d is sm_%d%d; this library is built for sm_100a only", device, major,
                  minor);
    return SV_ERR_UNSUPPORTED;
  }
  DeviceScope scope(device);
  if (!scope.ok()) return SV_ERR_CUDA;

  specfold_gate_ctx* h = new (std::nothrow) specfold_gate_ctx;
  if (!h) return SV_ERR_OOM;
  h->device = device;
  h->branches = branches;
  h->positions = positions;
  h->dim = dim;
  h->rows = rows;
  h->pack_blocks = static_cast<int>((rows + specfold::kRowsPerBlock - 1) / specfold::kRowsPerBlock);
  h->dtype = dtype;
  // the difference kernel is persistent: as many blocks as fit on the GPU at
  // once (its registers set the limit), never more than there are rows
  {
    int sms = 0, occ = 0;
    e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, device);
    const void* k = (dtype == SV_DTYPE_BF16)
                        ? reinterpret_cast<const void*>(specfold::rows_kernel<__nv_bfloat16, true>)
                        : reinterpret_cast<const void*>(specfold::rows_kernel<float, true>);
    if (e == cudaSuccess)
      e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, k, specfold::kThreads, 0);
    if (e != cudaSuccess) {
      delete h;
      return cuda_fail(e);
    }
    const long want = static_cast<long>(sms) * (occ > 0 ? occ : 1);
    h->blocks = static_cast<int>(want < rows ? want : rows);
    // rows of 16-byte multiples up to a quarter of the ring take the
    // bulk-copy form on aligned inputs: one block per SM, as many stages of
    // (child, parent) row pairs as the ring holds (at most kBulkMaxStages).
    // Each warp that takes rows owns S / C stages.  A warp's reduction of a
    // row pair is one long dependent chain per lane, so the most warps with
    // one stage each beat fewer warps with deeper rings (measured on the
    // 4096-wide bf16 rows: 12 warps x 1 stage 49.9 us, 8 x 1 53.5 us,
    // 6 x 2 65.0 us, 4 x 3 74.1 us, 3 x 4 94.4 us; 24 warps of half rows
    // 50.7 us).  Where the ring holds fewer than 12 whole row pairs and a row
    // has a multiple of 64 groups, a stage holds half of each row instead
    // (twice the warps).
    const long rb = static_cast<long>(dim) * static_cast<long>(gate_elem_size(dtype));
    if (rb % 16 == 0 && rb <= specfold::kBulkMaxRowBytes) {
      int parts = 1;
      long smax = specfold::kBulkRingBytes / (2 * rb);  // >= 2
      if (smax < specfold::kBulkMaxStages / 2 && (rb / 16) % 64 == 0) {
        parts = 2;
        smax = specfold::kBulkRingBytes / rb;
      }
      if (smax > specfold::kBulkMaxStages) smax = specfold::kBulkMaxStages;
      long cons = smax;
      if (cons > specfold::kBulkWarps) cons = specfold::kBulkWarps;
      h->bulk_parts = parts;
      h->bulk_stages = static_cast<int>(cons * (smax / cons));
      h->bulk_consumers = static_cast<int>(cons);
      h->bulk_blocks = static_cast<int>(sms < rows ? sms : rows);
      // the attribute is per function, shared by all handles: the ring's maximum
      const void* kb = (dtype == SV_DTYPE_BF16)
                           ? reinterpret_cast<const void*>(specfold::rows_bulk_kernel<__nv_bfloat16>)
                           : reinterpret_cast<const void*>(specfold::rows_bulk_kernel<float>);
      e = cudaFuncSetAttribute(kb, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               specfold::kBulkRingBytes);
      if (e != cudaSuccess) {
        delete h;
        return cuda_fail(e);
      }
    }
  }

  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t at = off;
    off = round_up(off + bytes, 256);
    return at;
  };
  const size_t oE = take(sizeof(int32_t) * branches);
  const size_t oF = take(static_cast<size_t>(rows) + 4);  // + padding for 4-byte reads
  const size_t oR = take(sizeof(int32_t) * rows);
  const size_t oP = take(sizeof(int32_t) * rows);
  const size_t oS = take(sizeof(unsigned));
  e = cudaMalloc(&h->ws, off);
  if (e != cudaSuccess) {
    delete h;
    return cuda_fail(e);
  }
  char* b = static_cast<char*>(h->ws);
  h->eff_parent = reinterpret_cast<int32_t*>(b + oE);
  h->flag = reinterpret_cast<uint8_t*>(b + oF);
  h->rank = reinterpret_cast<int32_t*>(b + oR);
  h->prov = reinterpret_cast<int32_t*>(b + oP);
  h->status = reinterpret_cast<unsigned*>(b + oS);
  // the attribute is per function, shared by all handles: allow the largest tree
  e = cudaFuncSetAttribute(specfold::tree_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(2 * sizeof(int32_t) * specfold::kMaxBranches));
  if (e == cudaSuccess) e = cudaMemset(h->ws, 0, off);
  if (e == cudaSuccess) e = cudaDeviceSynchronize();
  if (e != cudaSuccess) {
    cudaFree(h->ws);
    delete h;
    return cuda_fail(e);
  }
  *out = h;
  return SV_OK;
}

sv_status specfold_gate_run(specfold_gate_t h, const void* hidden, const int32_t* parent,
                            float tau, float* rel_diff, int32_t* provenance, int32_t* source,
                            int32_t* packed_rows, int32_t* n_packed, void* packed_hidden,
                            void* stream) {
  svhost::NvtxRange nvtx_range("specfold_gate_run");
  if (!h) return SV_ERR_INVALID_ARG;
  if (!hidden || !parent || !packed_rows || !n_packed) return SV_ERR_INVALID_ARG;
  if (std::isnan(tau) || !(tau >= 0.f)) return SV_ERR_INVALID_ARG;
  const size_t es = gate_elem_size(h->dtype);
  if (!gate_aligned(hidden, es) || (packed_hidden && !gate_aligned(packed_hidden, es)))
    return SV_ERR_INVALID_ARG;
  if (!gate_aligned(parent, 4) || !gate_aligned(rel_diff, 4) || !gate_aligned(provenance, 4) ||
      !gate_aligned(source, 4) || !gate_aligned(packed_rows, 4) || !gate_aligned(n_packed, 4))
    return SV_ERR_INVALID_ARG;
  DeviceScope scope(h->device);
  if (!scope.ok()) return SV_ERR_CUDA;

  GateParams p;
  p.hidden = hidden;
  p.parent = parent;
  p.tau = static_cast<double>(tau);
  p.branches = h->branches;
  p.positions = h->positions;
  p.dim = h->dim;
  p.rows = h->rows;
  p.blocks = h->blocks;
  p.bulk_stages = h->bulk_stages;
  p.bulk_consumers = h->bulk_consumers;
  p.bulk_parts = h->bulk_parts;
  p.pack_blocks = h->pack_blocks;
  p.rel_diff = rel_diff;
  p.provenance = provenance;
  p.source = source;
  p.packed = packed_rows;
  p.n_packed = n_packed;
  p.packed_hidden = packed_hidden;
  p.eff_parent = h->eff_parent;
  p.flag = h->flag;
  p.rank = h->rank;
  p.prov = h->prov;
  p.status = h->status;

  const bool aligned = gate_aligned(hidden, 16) && (!packed_hidden || gate_aligned(packed_hidden, 16)) &&
                       (static_cast<size_t>(h->dim) * es) % 16 == 0;
  cudaEvent_t* ev = nullptr;
  if (h->prof_runs < h->prof_capacity) ev = h->events.data() + 3 * (h->prof_runs++);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e;
  if (h->dtype == SV_DTYPE_BF16)
    e = aligned ? launch_pass<__nv_bfloat16, true>(p, h->bulk_blocks, s, ev)
                : launch_pass<__nv_bfloat16, false>(p, h->bulk_blocks, s, ev);
  else
    e = aligned ? launch_pass<float, true>(p, h->bulk_blocks, s, ev)
                : launch_pass<float, false>(p, h->bulk_blocks, s, ev);
  if (e != cudaSuccess) return cuda_fail(e);
  return SV_OK;
}

sv_status specfold_gate_get_status(specfold_gate_t h, void* stream, uint32_t* bits) {
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
  if (v & specfold::kStatWait) return SV_ERR_PIPELINE;
  return (v & specfold::kStatParent) ? SV_ERR_PARENT : SV_OK;
}

sv_status specfold_gate_profile_begin(specfold_gate_t h, int max_runs) {
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

sv_status specfold_gate_profile_end(specfold_gate_t h, float* rows_ms, float* pack_ms, int* runs) {
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
  if (rows_ms) *rows_ms = n ? static_cast<float>(a / n) : 0.f;
  if (pack_ms) *pack_ms = n ? static_cast<float>(c / n) : 0.f;
  if (runs) *runs = n;
  for (cudaEvent_t ev : h->events) cudaEventDestroy(ev);
  h->events.clear();
  h->prof_capacity = 0;
  h->prof_runs = 0;
  return SV_OK;
}

void specfold_gate_destroy(specfold_gate_t h) {
  if (!h) return;
  {
    DeviceScope scope(h->device);
    if (scope.ok()) {
      cudaDeviceSynchronize();
      for (cudaEvent_t ev : h->events) cudaEventDestroy(ev);
      if (h->ws) cudaFree(h->ws);
    }
  }
  delete h;
}

}  // extern "C"
