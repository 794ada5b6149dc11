// Kernels of the multi-branch fold gate (include/specfold_gate.h).
//
// SpecFold explainer (blog.ontle.kr, post 356): the observation paragraph
// (relative hidden-state difference of a child and its parent at the same
// layer input), the per-position path and the paragraph after it (positions
// above tau from all branches are packed into one batch), the implementer's
// note (the gate records provenance; a resolution step follows fold chains).
//
// Four stream-ordered kernels per pass:
//   tree_kernel  one block: validates every branch's parent chain by pointer
//                jumping in shared memory;
//   rows_kernel  persistent warps, global warp w taking rows w, w + W, ...;
//                each warp streams its rows' H[c, j] and H[parent, j] through
//                a ring of cp.async stages, sums squares in fp32 per lane and
//                fp64 across the warp, and decides recompute = !(d <= tau);
//   scan_kernel  one block: the packed slot of every recomputed row (an
//                exclusive prefix sum of the flags) and their count;
//   pack_kernel  one warp per row: writes the packed row index, follows the
//                fold chain to the source row, copies recomputed rows into the
//                packed batch.
// Nothing waits on another block inside a kernel.
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

enum : unsigned { kStatParent = 1u };

struct GateParams {
  const void* hidden;       // [branches, positions, dim]
  const int32_t* parent;    // [branches]
  double tau;
  int branches, positions, dim;
  long rows;
  int blocks;               // rows_kernel grid (persistent warps)
  int pack_blocks;          // pack_kernel grid (8 rows per block)
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
  int32_t* rank;            // [rows] packed slot of each recomputed row
  int32_t* prov;            // [rows] provenance (always kept for the chain walk)
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

constexpr int kStages = 8;  // cp.async stages in flight per warp
constexpr int kStageBytes = kWarp * 32;  // one 16-byte group of child and parent per lane
constexpr int kRowsSmem = kStages * kStageBytes * (kThreads / kWarp);

__device__ __forceinline__ void cp_async16(void* smem, const void* gmem, bool valid) {
  const unsigned dst = static_cast<unsigned>(__cvta_generic_to_shared(smem));
  const int n = valid ? 16 : 0;  // 0: fill with zeros, read nothing
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(gmem), "r"(n));
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;"); }
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(kStages - 1));
}

// lane 0's per-row epilogue: the decision and its records
__device__ __forceinline__ bool finish_row(const GateParams& P, long row, int par, int j,
                                           double num, double den) {
  double d = INFINITY;
  if (par >= 0) d = (den == 0.0) ? ((num == 0.0) ? 0.0 : INFINITY) : sqrt(num / den);
  const bool rec = par < 0 || !(d <= P.tau);
  const int32_t prov = rec ? -1 : static_cast<int32_t>(static_cast<long>(par) * P.positions + j);
  P.prov[row] = prov;
  P.flag[row] = rec ? 1 : 0;
  if (P.provenance) P.provenance[row] = prov;
  if (P.rel_diff) P.rel_diff[row] = static_cast<float>(d);
  return rec;
}

// Persistent warps: global warp w takes rows w, w + W, w + 2W, ... (W warps
// in the grid), so all warps move through the tensor together and a parent
// row, a few hundred rows before its children, is still in L2 when they read
// it.  With 128-bit rows a warp streams its rows' (child, parent) groups
// through a ring of kStages cp.async stages in shared memory, so loads stay in
// flight across row boundaries without holding registers.
template <typename T, bool kAligned>
__global__ void __launch_bounds__(kThreads) rows_kernel(const GateParams P) {
  extern __shared__ uint4 ring[];  // [warps][kStages][2][kWarp]
  const int warp = threadIdx.x / kWarp, lane = threadIdx.x & (kWarp - 1);
  const long W = static_cast<long>(gridDim.x) * (kThreads / kWarp);
  const long r0 = static_cast<long>(blockIdx.x) * (kThreads / kWarp) + warp;
  const long r1 = P.rows;
  const T* base = static_cast<const T*>(P.hidden);
  cudaGridDependencySynchronize();  // validated parents

  // rows without a parent are decided without reading anything
  auto parent_of = [&](long row) -> int { return P.eff_parent[row / P.positions]; };
  if (lane == 0)
    for (long row = r0; row < r1; row += W)
      if (parent_of(row) < 0) finish_row(P, row, -1, 0, 0.0, 0.0);
  // next row at or after `row` (in this warp's sequence) that has a parent
  auto next_row = [&](long row) -> long {
    while (row < r1 && parent_of(row) < 0) row += W;
    return row;
  };

  if constexpr (kAligned) {
    constexpr int kVec = HElem<T>::kPerVec;
    const int groups = P.dim / kVec;
    const int chunks = (groups + kWarp - 1) / kWarp;  // units per row
    uint4* my = ring + static_cast<long>(warp) * kStages * 2 * kWarp;
    // issue pointer: the row being fetched, its two group pointers (this
    // lane's group of chunk 0) and the chunk; all set once per row
    long irow = next_row(r0);
    int ichunk = 0;
    const uint4* igc = nullptr;  // this lane's next group of the child row
    const uint4* igp = nullptr;  // and of the parent row
    const uint4* rc = nullptr;   // first group of each row: the (unread) source
    const uint4* rp = nullptr;   // address of a zero-filling copy
    auto set_issue_row = [&]() {
      if (irow < r1) {
        const int par = parent_of(irow);
        const long j = irow - (irow / P.positions) * P.positions;
        rc = reinterpret_cast<const uint4*>(base + irow * P.dim);
        rp = reinterpret_cast<const uint4*>(base + (static_cast<long>(par) * P.positions + j) * P.dim);
        igc = rc + lane;
        igp = rp + lane;
      }
    };
    set_issue_row();
    int g_left = groups - lane;  // groups of the row at or after this lane's
    auto issue = [&](int slot) {
      if (irow < r1) {
        const bool ok = g_left > 0;
        cp_async16(my + (slot * 2 + 0) * kWarp + lane, ok ? igc : rc, ok);
        cp_async16(my + (slot * 2 + 1) * kWarp + lane, ok ? igp : rp, ok);
        igc += kWarp;
        igp += kWarp;
        g_left -= kWarp;
        if (++ichunk == chunks) {
          ichunk = 0;
          g_left = groups - lane;
          irow = next_row(irow + W);
          set_issue_row();
        }
      }
      cp_async_commit();  // an empty group keeps the wait count uniform
    };
#pragma unroll 1
    for (int st = 0; st < kStages - 1; ++st) issue(st);
    long crow = next_row(r0);
    int cchunk = 0, slot = 0;
    float d0 = 0.f, d1 = 0.f, n0 = 0.f, n1 = 0.f;
    while (crow < r1) {
      issue(slot == 0 ? kStages - 1 : slot - 1);
      cp_async_wait();
      const uint4 c = my[(slot * 2 + 0) * kWarp + lane];
      const uint4 p = my[(slot * 2 + 1) * kWarp + lane];
      HElem<T>::accumulate(c, p, d0, d1, n0, n1);
      slot = (slot == kStages - 1) ? 0 : slot + 1;
      if (++cchunk == chunks) {
        double num = static_cast<double>(d0) + static_cast<double>(d1);
        double den = static_cast<double>(n0) + static_cast<double>(n1);
#pragma unroll
        for (int o = kWarp / 2; o > 0; o >>= 1) {
          num += __shfl_xor_sync(0xffffffffu, num, o);
          den += __shfl_xor_sync(0xffffffffu, den, o);
        }
        if (lane == 0)
          finish_row(P, crow, parent_of(crow), static_cast<int>(crow % P.positions), num, den);
        d0 = d1 = n0 = n1 = 0.f;
        cchunk = 0;
        crow = next_row(crow + W);
      }
    }
    asm volatile("cp.async.wait_all;");
  } else {
    for (long row = next_row(r0); row < r1; row = next_row(row + W)) {
      const int par = parent_of(row);
      const int j = static_cast<int>(row % P.positions);
      const T* hc = base + row * P.dim;
      const T* hp = base + (static_cast<long>(par) * P.positions + j) * P.dim;
      float dd = 0.f, nn = 0.f;
      for (int k = lane; k < P.dim; k += kWarp) {
        const float c = HElem<T>::scalar(hc, k), p = HElem<T>::scalar(hp, k);
        const float e = c - p;
        dd = fmaf(e, e, dd);
        nn = fmaf(p, p, nn);
      }
      double num = dd, den = nn;
#pragma unroll
      for (int o = kWarp / 2; o > 0; o >>= 1) {
        num += __shfl_xor_sync(0xffffffffu, num, o);
        den += __shfl_xor_sync(0xffffffffu, den, o);
      }
      if (lane == 0) finish_row(P, row, par, j, num, den);
    }
  }

}

// ---------------------------------------------------------------------------
// kernel 3: the packed slots (one block): exclusive prefix sum of the flags
// ---------------------------------------------------------------------------

// each thread owns a contiguous chunk of rows: its count, one block-wide
// exclusive scan of the counts, then its slots in row order
constexpr int kSlotThreads = 1024;

__global__ void __launch_bounds__(kSlotThreads) scan_kernel(const GateParams P) {
  __shared__ int32_t s_warp[kSlotThreads / kWarp];
  const int warp = threadIdx.x / kWarp, lane = threadIdx.x & (kWarp - 1);
  cudaGridDependencySynchronize();
  // chunks of a multiple of 4 rows: the flags are read four per 32-bit load
  // (the flag array is 256-byte aligned and padded to a multiple of 4)
  const long chunk = ((P.rows + kSlotThreads - 1) / kSlotThreads + 3) & ~3L;
  const long lo = min(P.rows, chunk * threadIdx.x), hi = min(P.rows, lo + chunk);
  int v = 0;
  for (long i = lo; i < hi; i += 4) {
    const unsigned w = __ldcg(reinterpret_cast<const unsigned*>(P.flag + i));
    // bytes past `hi` (the next chunk's rows, or padding past the last row)
    // are masked off
    const long left = hi - i;
    const unsigned keep = left >= 4 ? 0xffffffffu : ((1u << (8 * left)) - 1u);
    v += __popc(w & keep & 0x01010101u);
  }
  int x = v;
#pragma unroll
  for (int o = 1; o < kWarp; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == kWarp - 1) s_warp[warp] = x;
  __syncthreads();
  if (warp == 0) {
    int w = s_warp[lane];  // kSlotThreads / kWarp == kWarp warps
#pragma unroll
    for (int o = 1; o < kWarp; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += y;
    }
    s_warp[lane] = w;  // inclusive over warps
  }
  __syncthreads();
  int slot = (warp > 0 ? s_warp[warp - 1] : 0) + x - v;
  for (long i = lo; i < hi; ++i)
    if (__ldcg(P.flag + i) != 0) P.rank[i] = slot++;
  if (threadIdx.x == kSlotThreads - 1) *P.n_packed = s_warp[kWarp - 1];
}

// ---------------------------------------------------------------------------
// kernel 4: packing and fold-chain resolution
// ---------------------------------------------------------------------------

// one warp per row; the row's slot comes from the scan
template <typename T, bool kAligned>
__global__ void __launch_bounds__(kThreads) pack_kernel(const GateParams P) {
  const int warp = threadIdx.x / kWarp, lane = threadIdx.x & (kWarp - 1);
  const long row = static_cast<long>(blockIdx.x) * kRowsPerBlock + warp;
  cudaGridDependencySynchronize();
  if (row >= P.rows) return;
  const bool rec = __ldcg(P.flag + row) != 0;
  long slot = 0;
  if (rec) slot = __ldcg(P.rank + row);
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
