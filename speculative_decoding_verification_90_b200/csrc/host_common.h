// Host-side helpers shared by the C-ABI translation units of the library.
#pragma once

#include <cuda_runtime.h>
#include <nvtx3/nvToolsExt.h>

#include <cstddef>

#include "specverify.h"

namespace svhost {

// the calling thread's last error message (specverify_last_error)
extern thread_local char g_last_error[256];

// records `e` in g_last_error; returns SV_ERR_OOM or SV_ERR_CUDA
sv_status cuda_fail(cudaError_t e);

// makes a device current for the scope, restores the caller's on exit
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
  DeviceScope(const DeviceScope&) = delete;
  DeviceScope& operator=(const DeviceScope&) = delete;
  bool ok() const { return ok_; }

 private:
  int prev_ = 0;
  bool ok_ = false;
  bool switched_ = false;
};

inline size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// An NVTX range around the host side of one entry point (the enqueue, not the
// kernels' device time): named ranges in a profiler's timeline.  NVTX v3 is
// header-only; without a profiler attached each push / pop is a no-op call.
class NvtxRange {
 public:
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
  NvtxRange(const NvtxRange&) = delete;
  NvtxRange& operator=(const NvtxRange&) = delete;
};

}  // namespace svhost
