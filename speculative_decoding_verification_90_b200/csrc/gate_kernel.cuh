// Kernels of the multi-branch fold gate (include/specfold_gate.h).
//
// SpecFold explainer (blog.ontle.kr, post 356): the observation paragraph
// (relative hidden-state difference of a child and its parent at the same
// layer input), the per-position path and the paragraph after it (positions
// above tau from all branches are packed into one batch), the implementer's
// note (the gate records provenance; a resolution step follows fold chains).
//
// Three stream-ordered kernels per pass:
//   tree_kernel  one block: validates every branch's parent chain by pointer
//                jumping in shared memory;
//   rows_kernel  one warp per row (c, j): streams H[c, j] and H[parent, j]
//                with 128-bit loads, sum of squares in fp32 per lane, fp64
//                across the warp; decides recompute = !(d <= tau); ranks the
//                recomputed rows of the block; the block that takes the last
//                ticket turns the per-block counts into offsets;
//   pack_kernel  one warp per row: writes the packed row index, follows the
//                fold chain to the source row, copies recomputed rows into the
//                packed batch.
// The only hand-off inside a kernel is the ticket (the last arriver proceeds);
// nothing waits on another block.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace specfold {

constexpr int kWarp = 32;
constexpr int kRowsPerBlock = 8;  // one warp per row
constexpr int kThreads = kRowsPerBlock * kWarp;
constexpr int kTreeThreads = 1024;
constexpr int kMaxBranches = 16384;
constexpr int kScanThreads = kThreads;

enum : unsigned { kStatParent = 1u };

struct GateParams {
  const void* hidden;       // [branches, positions, dim]
  const int32_t* parent;    // [branches]
  double tau;
  int branches, positions, dim;
  long rows;
  int blocks;               // rows_kernel / pack_kernel grid
  // outputs (rel_diff, provenance, source, packed_hidden may be null)
  float* rel_diff;
  int32_t* provenance;
  int32_t* source;
  int32_t* packed;
  int32_t* n_packed;
  void* packed_hidden;
  // workspace
  int32_t* eff_parent;      // [branches] parent after validation, -1 if none
  uint8_t* flag;            // [rows] 1: recompute
  uint8_t* rank;            // [rows] rank among the recomputed rows of its block
  int32_t* prov;            // [rows] provenance (always kept for the chain walk)
  int32_t* block_count;     // [blocks]
  int32_t* block_offset;    // [blocks]
  unsigned* ticket;
  unsigned* status;
};

// ---------------------------------------------------------------------------
// loads
// ---------------------------------------------------------------------------

__device__ __forceinline__ uint4 ld_v4(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

template <typename T>
struct HElem;

template <>
struct HElem<float> {
  static constexpr int kPerVec = 4;
  __device__ static float scalar(const float* p, long i) { return __ldg(p + i); }
  // d += (c - p)^2, n += p^2 over one 16-byte group of each row
  __device__ static void accumulate(uint4 c, uint4 p, float& d0, float& d1, float& n0, float& n1) {
    const float c0 = __uint_as_float(c.x), c1 = __uint_as_float(c.y);
    const float c2 = __uint_as_float(c.z), c3 = __uint_as_float(c.w);
    const float p0 = __uint_as_float(p.x), p1 = __uint_as_float(p.y);
    const float p2 = __uint_as_float(p.z), p3 = __uint_as_float(p.w);
    float e;
    e = c0 - p0; d0 = fmaf(e, e, d0); n0 = fmaf(p0, p0, n0);
    e = c1 - p1; d1 = fmaf(e, e, d1); n1 = fmaf(p1, p1, n1);
    e = c2 - p2; d0 = fmaf(e, e, d0); n0 = fmaf(p2, p2, n0);
    e = c3 - p3; d1 = fmaf(e, e, d1); n1 = fmaf(p3, p3, n1);
  }
};

template <>
struct HElem<__nv_bfloat16> {
  static constexpr int kPerVec = 8;
  __device__ static float scalar(const __nv_bfloat16* p, long i) {
    const unsigned short b = __ldg(reinterpret_cast<const unsigned short*>(p) + i);
    return __uint_as_float(static_cast<unsigned>(b) << 16);
  }
  __device__ static void pair(unsigned c, unsigned p, float& d0, float& d1, float& n0, float& n1) {
    const float cl = __uint_as_float(c << 16), ch = __uint_as_float(c & 0xffff0000u);
    const float pl = __uint_as_float(p << 16), ph = __uint_as_float(p & 0xffff0000u);
    float e;
    e = cl - pl; d0 = fmaf(e, e, d0); n0 = fmaf(pl, pl, n0);
    e = ch - ph; d1 = fmaf(e, e, d1); n1 = fmaf(ph, ph, n1);
  }
  __device__ static void accumulate(uint4 c, uint4 p, float& d0, float& d1, float& n0, float& n1) {
    pair(c.x, p.x, d0, d1, n0, n1);
    pair(c.y, p.y, d0, d1, n0, n1);
    pair(c.z, p.z, d0, d1, n0, n1);
    pair(c.w, p.w, d0, d1, n0, n1);
  }
};

// ---------------------------------------------------------------------------
// kernel 1: parent validation by pointer jumping
// ---------------------------------------------------------------------------

// cur[c] = an ancestor of c (>= 0), or -1 (the chain reached a branch without
// a parent: valid) or -2 (it met a link out of range or a self link).  Each
// round replaces the ancestor by the ancestor's ancestor, so after
// ceil(log2(branches)) + 1 rounds every finite chain has ended; entries still
// >= 0 lie on or lead into a cycle.
__global__ void __launch_bounds__(kTreeThreads) tree_kernel(const GateParams P) {
  extern __shared__ int32_t anc[];  // 2 * branches
  const int nb = P.branches;
  int32_t* cur = anc;
  int32_t* nxt = anc + nb;
  for (int c = threadIdx.x; c < nb; c += blockDim.x) {
    const int p = P.parent[c];
    cur[c] = (p == -1) ? -1 : ((p < 0 || p >= nb || p == c) ? -2 : p);
  }
  __syncthreads();
  int rounds = 1;
  while ((1 << (rounds - 1)) < nb) ++rounds;
  for (int r = 0; r < rounds; ++r) {
    for (int c = threadIdx.x; c < nb; c += blockDim.x) {
      const int a = cur[c];
      nxt[c] = (a >= 0) ? cur[a] : a;
    }
    __syncthreads();
    int32_t* t = cur;
    cur = nxt;
    nxt = t;
  }
  bool bad = false;
  for (int c = threadIdx.x; c < nb; c += blockDim.x) {
    const bool ok = cur[c] == -1;
    P.eff_parent[c] = ok ? P.parent[c] : -1;
    bad |= !ok;
  }
  if (__syncthreads_or(bad) && threadIdx.x == 0) atomicOr(P.status, kStatParent);
}

// ---------------------------------------------------------------------------
// kernel 2: difference test
// ---------------------------------------------------------------------------

template <typename T, bool kAligned>
__device__ __forceinline__ void row_sums(const T* hc, const T* hp, int dim, double& num,
                                         double& den) {
  const int lane = threadIdx.x & (kWarp - 1);
  float d0 = 0.f, d1 = 0.f, n0 = 0.f, n1 = 0.f;
  if constexpr (kAligned) {
    constexpr int kU = 4;
    const int groups = dim / HElem<T>::kPerVec;
    const uint4* gc = reinterpret_cast<const uint4*>(hc);
    const uint4* gp = reinterpret_cast<const uint4*>(hp);
    int g = lane;
    for (; g + (kU - 1) * kWarp < groups; g += kU * kWarp) {
      uint4 c[kU], p[kU];
#pragma unroll
      for (int u = 0; u < kU; ++u) {
        c[u] = ld_v4(gc + g + u * kWarp);
        p[u] = ld_v4(gp + g + u * kWarp);
      }
#pragma unroll
      for (int u = 0; u < kU; ++u) HElem<T>::accumulate(c[u], p[u], d0, d1, n0, n1);
    }
    for (; g < groups; g += kWarp) HElem<T>::accumulate(ld_v4(gc + g), ld_v4(gp + g), d0, d1, n0, n1);
  } else {
    for (int k = lane; k < dim; k += kWarp) {
      const float c = HElem<T>::scalar(hc, k), p = HElem<T>::scalar(hp, k);
      const float e = c - p;
      d0 = fmaf(e, e, d0);
      n0 = fmaf(p, p, n0);
    }
  }
  num = static_cast<double>(d0) + static_cast<double>(d1);
  den = static_cast<double>(n0) + static_cast<double>(n1);
#pragma unroll
  for (int o = kWarp / 2; o > 0; o >>= 1) {
    num += __shfl_xor_sync(0xffffffffu, num, o);
    den += __shfl_xor_sync(0xffffffffu, den, o);
  }
}

template <typename T, bool kAligned>
__global__ void __launch_bounds__(kThreads) rows_kernel(const GateParams P) {
  __shared__ unsigned s_flags;
  __shared__ bool s_last;
  const int warp = threadIdx.x / kWarp, lane = threadIdx.x & (kWarp - 1);
  const long row = static_cast<long>(blockIdx.x) * kRowsPerBlock + warp;
  if (threadIdx.x == 0) s_flags = 0u;

  // the validated parents come from the tree kernel
  cudaGridDependencySynchronize();
  __syncthreads();
  bool rec = false;
  if (row < P.rows) {
    const int c = static_cast<int>(row / P.positions);
    const int j = static_cast<int>(row - static_cast<long>(c) * P.positions);
    const int par = P.eff_parent[c];
    double d = INFINITY;
    if (par >= 0) {
      const T* base = static_cast<const T*>(P.hidden);
      const T* hc = base + row * P.dim;
      const T* hp = base + (static_cast<long>(par) * P.positions + j) * P.dim;
      double num, den;
      row_sums<T, kAligned>(hc, hp, P.dim, num, den);
      d = (den == 0.0) ? ((num == 0.0) ? 0.0 : INFINITY) : sqrt(num / den);
    }
    rec = par < 0 || !(d <= P.tau);
    if (lane == 0) {
      const int32_t prov = rec ? -1 : static_cast<int32_t>(static_cast<long>(par) * P.positions + j);
      P.prov[row] = prov;
      P.flag[row] = rec ? 1 : 0;
      if (P.provenance) P.provenance[row] = prov;
      if (P.rel_diff) P.rel_diff[row] = static_cast<float>(d);
      if (rec) atomicOr(&s_flags, 1u << warp);
    }
  }
  __syncthreads();
  const unsigned flags = s_flags;
  if (row < P.rows && lane == 0)
    P.rank[row] = static_cast<uint8_t>(__popc(flags & ((1u << warp) - 1u)));
  if (threadIdx.x == 0) {
    P.block_count[blockIdx.x] = __popc(flags);
    __threadfence();
    // atomicInc wraps to 0 at the last block, so the ticket resets itself
    s_last = atomicInc(P.ticket, static_cast<unsigned>(P.blocks - 1)) ==
             static_cast<unsigned>(P.blocks - 1);
  }
  __syncthreads();
  if (!s_last) return;

  // last block: exclusive prefix sum of the per-block counts
  __threadfence();
  __shared__ int32_t s_warp[kScanThreads / kWarp];
  __shared__ int32_t s_carry;
  if (threadIdx.x == 0) s_carry = 0;
  __syncthreads();
  for (int base = 0; base < P.blocks; base += kScanThreads) {
    const int i = base + threadIdx.x;
    const int v = (i < P.blocks) ? __ldcg(P.block_count + i) : 0;
    int x = v;
#pragma unroll
    for (int o = 1; o < kWarp; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    if (lane == kWarp - 1) s_warp[warp] = x;
    __syncthreads();
    if (warp == 0) {
      int w = (lane < kScanThreads / kWarp) ? s_warp[lane] : 0;
#pragma unroll
      for (int o = 1; o < kWarp; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, w, o);
        if (lane >= o) w += y;
      }
      if (lane < kScanThreads / kWarp) s_warp[lane] = w;  // inclusive over warps
    }
    __syncthreads();
    const int before = s_carry + (warp > 0 ? s_warp[warp - 1] : 0) + x - v;
    if (i < P.blocks) P.block_offset[i] = before;
    __syncthreads();
    if (threadIdx.x == 0) s_carry += s_warp[kScanThreads / kWarp - 1];
    __syncthreads();
  }
  if (threadIdx.x == 0) *P.n_packed = s_carry;
}

// ---------------------------------------------------------------------------
// kernel 3: packing and fold-chain resolution
// ---------------------------------------------------------------------------

template <typename T, bool kAligned>
__global__ void __launch_bounds__(kThreads) pack_kernel(const GateParams P) {
  const int warp = threadIdx.x / kWarp, lane = threadIdx.x & (kWarp - 1);
  const long row = static_cast<long>(blockIdx.x) * kRowsPerBlock + warp;
  cudaGridDependencySynchronize();
  if (row >= P.rows) return;
  const bool rec = __ldcg(P.flag + row) != 0;
  long slot = 0;
  if (rec) slot = static_cast<long>(__ldcg(P.block_offset + blockIdx.x)) + __ldcg(P.rank + row);
  if (lane == 0) {
    if (rec) P.packed[slot] = static_cast<int32_t>(row);
    if (P.source) {
      // a folded row's chain ends at a recomputed row within `branches` steps,
      // because validated parents form a forest
      long at = row;
      int steps = 0;
      while (!__ldcg(P.flag + at) && steps <= P.branches) {
        at = __ldcg(P.prov + at);
        ++steps;
      }
      P.source[row] = static_cast<int32_t>(at);
    }
  }
  if (rec && P.packed_hidden) {
    const T* src = static_cast<const T*>(P.hidden) + row * P.dim;
    T* dst = static_cast<T*>(P.packed_hidden) + slot * P.dim;
    if constexpr (kAligned) {
      const int groups = P.dim / HElem<T>::kPerVec;
      const uint4* gs = reinterpret_cast<const uint4*>(src);
      uint4* gd = reinterpret_cast<uint4*>(dst);
      for (int g = lane; g < groups; g += kWarp) __stcs(gd + g, ld_v4(gs + g));
    } else {
      for (int k = lane; k < P.dim; k += kWarp) dst[k] = src[k];
    }
  }
}

}  // namespace specfold
