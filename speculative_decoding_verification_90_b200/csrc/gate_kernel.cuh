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
//                each warp streams its rows' H[c, j] and H[parent, j] with
//                128-bit loads, eight in flight per lane, sums squares with
//                packed fp32 pairs per lane and in fp64 across the warp, and
//                decides recompute = !(d <= tau); on 16-byte aligned rows
//                of at most 50 KB the bulk-copy form rows_bulk_kernel does
//                the same test from shared memory (one block per SM);
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
  int bulk_stages;          // > 0: rows_bulk_kernel with this many ring stages
  int bulk_consumers;       // its consumer warps that take rows (bulk_stages is a multiple)
  int bulk_parts;           // stage loads per row pair: 1, or 2 (halves of the rows)
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
  // d += (c - p)^2, n += p^2 on pairs of entries (packed fp32 instructions)
  __device__ static void accumulate2(uint4 c, uint4 p, float2& d, float2& n) {
    const float2 m1 = make_float2(-1.f, -1.f);
    float2 cc = make_float2(__uint_as_float(c.x), __uint_as_float(c.y));
    float2 pp = make_float2(__uint_as_float(p.x), __uint_as_float(p.y));
    float2 e = __ffma2_rn(pp, m1, cc);
    d = __ffma2_rn(e, e, d);
    n = __ffma2_rn(pp, pp, n);
    cc = make_float2(__uint_as_float(c.z), __uint_as_float(c.w));
    pp = make_float2(__uint_as_float(p.z), __uint_as_float(p.w));
    e = __ffma2_rn(pp, m1, cc);
    d = __ffma2_rn(e, e, d);
    n = __ffma2_rn(pp, pp, n);
  }
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
  __device__ static void pair2(unsigned c, unsigned p, float2& d, float2& n) {
    const float2 cc = make_float2(__uint_as_float(c << 16), __uint_as_float(c & 0xffff0000u));
    const float2 pp = make_float2(__uint_as_float(p << 16), __uint_as_float(p & 0xffff0000u));
    const float2 e = __ffma2_rn(pp, make_float2(-1.f, -1.f), cc);  // exact: bf16 differences
    d = __ffma2_rn(e, e, d);
    n = __ffma2_rn(pp, pp, n);
  }
  // d += (c - p)^2, n += p^2 on pairs of entries (packed fp32 instructions)
  __device__ static void accumulate2(uint4 c, uint4 p, float2& d, float2& n) {
    pair2(c.x, p.x, d, n);
    pair2(c.y, p.y, d, n);
    pair2(c.z, p.z, d, n);
    pair2(c.w, p.w, d, n);
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

constexpr int kRowUnroll = 4;  // 16-byte groups of each row in flight per lane
constexpr int kRowsBlocksPerSM = 4;

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
// it.  With 128-bit rows each lane keeps kRowUnroll groups of the child row
// and kRowUnroll of the parent row in flight (the statistics kernel's load
// scheme: independent non-coherent 16-byte loads, coalesced across the warp).
template <typename T, bool kAligned>
__global__ void __launch_bounds__(kThreads, kRowsBlocksPerSM) rows_kernel(const GateParams P) {
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
    for (long row = next_row(r0); row < r1; row = next_row(row + W)) {
      const int par = parent_of(row);
      const int j = static_cast<int>(row % P.positions);
      const uint4* hc = reinterpret_cast<const uint4*>(base + row * P.dim);
      const uint4* hp = reinterpret_cast<const uint4*>(base + (static_cast<long>(par) * P.positions + j) * P.dim);
      float2 d = make_float2(0.f, 0.f), n = make_float2(0.f, 0.f);
      for (int g0 = lane; g0 < groups; g0 += kWarp * kRowUnroll) {
        uint4 c[kRowUnroll], q[kRowUnroll];
#pragma unroll
        for (int u = 0; u < kRowUnroll; ++u) {
          const int g = g0 + u * kWarp;
          if (g < groups) {
            c[u] = ld_v4(hc + g);
            q[u] = ld_v4(hp + g);
          } else {
            c[u] = make_uint4(0u, 0u, 0u, 0u);
            q[u] = c[u];
          }
        }
#pragma unroll
        for (int u = 0; u < kRowUnroll; ++u) HElem<T>::accumulate2(c[u], q[u], d, n);
      }
      double num = static_cast<double>(d.x) + static_cast<double>(d.y);
      double den = static_cast<double>(n.x) + static_cast<double>(n.y);
#pragma unroll
      for (int o = kWarp / 2; o > 0; o >>= 1) {
        num += __shfl_xor_sync(0xffffffffu, num, o);
        den += __shfl_xor_sync(0xffffffffu, den, o);
      }
      if (lane == 0) finish_row(P, row, par, j, num, den);
    }
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
// kernel 2, bulk-copy form (16-byte aligned rows of at most kBulkMaxRowBytes)
// ---------------------------------------------------------------------------
//
// One persistent block per SM (C warps) takes rows blockIdx.x + k G (G
// blocks), as the register form's warps do, so every block moves through the
// tensor with the others and a parent row is still in L2 when its children
// read it.  The warps take the block's rows k = c, c + C, ... (warp c) that have a
// parent; each warp streams its rows through a private ring of R stages of
// shared memory, every stage one (child row, parent row) pair brought in by
// two 1-D bulk copies (the copy engine generates the addresses: one
// instruction per row) whose completion the stage's mbarrier counts in bytes.
// A warp reduces the pair of its oldest stage and refills that stage with
// its load R ahead.  The reduction of a pair is one dependent chain per lane,
// so the most warps with one stage each do best; where whole row pairs would
// leave fewer than 12 stages, a stage holds half of each row (the two halves
// of a row go through the same warp, one after the other).  With hidden size
// 4096, bf16: 12 warps of one 16 KB stage, 96 KB of child rows per SM in
// flight or being reduced, where the register form keeps about 64 KB of
// child rows in flight at its full occupancy.  A stage only ever holds its own
// warp's rows, in order, so no wait can run a phase ahead of its barrier (a
// parity wait could not tell two phases apart) and no stage needs a release
// barrier.  The parents of a warp's rows are looked up 32 at a time, one
// lane per row, with the next 32 in flight.  Each lane adds the groups lane,
// lane + 32, ... of both rows in the register form's order (a half row holds
// a multiple of 32 groups), so the sums are the same bits.  Every wait is bounded (2 s of the global timer): a wait
// that runs out sets kStatWait, and the warp waits (bounded) for the copies
// it issued before it leaves.

constexpr int kBulkWarps = 24;  // warps per block at most; the launch has P.bulk_consumers
constexpr int kBulkThreads = kBulkWarps * kWarp;
constexpr int kBulkMaxStages = 24;
constexpr int kBulkRingBytes = 200 * 1024;                  // dynamic shared memory, at most
constexpr long kBulkMaxRowBytes = kBulkRingBytes / 4;       // at least 2 whole-row stages
constexpr unsigned long long kBulkWaitNs = 2000000000ull;  // 2 s

__device__ __forceinline__ unsigned smem_u32(const void* p) {
  return static_cast<unsigned>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ unsigned long long global_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
__device__ __forceinline__ void mbar_init(uint64_t* bar, unsigned count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ void mbar_arrive_tx(uint64_t* bar, unsigned bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}
__device__ __forceinline__ bool mbar_test(uint64_t* bar, unsigned parity) {
  unsigned ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
// wait for the phase of `parity` to complete; false after 2 s
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, unsigned parity) {
  if (mbar_test(bar, parity)) return true;
  const unsigned long long t0 = global_ns();
  while (!mbar_test(bar, parity))
    if (global_ns() - t0 > kBulkWaitNs) return false;
  return true;
}
// bytes from global to this block's shared memory (both 16-byte aligned,
// bytes a multiple of 16), counted on `bar`; no multicast
__device__ __forceinline__ void bulk_load(void* dst, const void* src, unsigned bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

enum : unsigned { kStatWait = 2u };

template <typename T>
__global__ void __launch_bounds__(kBulkThreads, 1) rows_bulk_kernel(const GateParams P) {
  extern __shared__ __align__(128) unsigned char ring[];  // C rings of R (child row, parent row) stages
  __shared__ uint64_t full[kBulkMaxStages];
  __shared__ int item_row[kBulkMaxStages], item_par[kBulkMaxStages], item_part[kBulkMaxStages];
  const int warp = threadIdx.x / kWarp, lane = threadIdx.x & (kWarp - 1);
  const int C = P.bulk_consumers;      // warps that take rows, 1 .. kBulkWarps
  const int R = P.bulk_stages / C;     // stages per warp (bulk_stages is a multiple of C)
  const int parts = P.bulk_parts;      // 1 or 2 stage loads per row pair
  const long G = gridDim.x;
  const unsigned rb = static_cast<unsigned>(P.dim * sizeof(T));  // a multiple of 16
  const unsigned pb = rb / parts;      // bytes of one row per stage: a multiple of 512 when parts = 2
  const T* base = static_cast<const T*>(P.hidden);
  if (threadIdx.x == 0) {
    for (int s = 0; s < C * R; ++s) mbar_init(&full[s], 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  __syncthreads();
  cudaGridDependencySynchronize();  // validated parents

  // the block's rows are blockIdx.x + k G, k = 0 .. nk - 1 (rows < 2^31)
  const int nk = static_cast<int>((P.rows - blockIdx.x + G - 1) / G);
  auto row_of = [&](int k) -> int { return static_cast<int>(blockIdx.x + static_cast<long>(k) * G); };
  // rows without a parent are decided without reading anything, lane by lane
  // across all warps of the block
  const int nwarps = static_cast<int>(blockDim.x) / kWarp;
  for (int k = warp + nwarps * lane; k < nk; k += nwarps * kWarp) {
    const int row = row_of(k);
    if (P.eff_parent[row / P.positions] < 0) finish_row(P, row, -1, 0, 0.0, 0.0);
  }
  const int c = warp;
  if (c >= C) return;

  // warp c's rows: m-th = k = c + m C, m = 0 .. mc - 1; lane l looks up the
  // parent of m = m0 + l, the next 32 lookups in flight
  const int mc = (nk > c) ? (nk - c + C - 1) / C : 0;
  auto lookup = [&](int m) -> int {
    return (m < mc) ? P.eff_parent[row_of(c + m * C) / P.positions] : -1;
  };
  int m0 = 0;
  int par_cur = lookup(lane);
  int par_next = lookup(kWarp + lane);
  unsigned todo = __ballot_sync(0xffffffffu, par_cur >= 0);
  // the next row of the warp that has a parent (warp-uniform); false at the end
  auto next_item = [&](int& row, int& par) -> bool {
    while (todo == 0u) {
      if (m0 + kWarp >= mc) return false;
      m0 += kWarp;
      par_cur = par_next;
      par_next = lookup(m0 + kWarp + lane);
      todo = __ballot_sync(0xffffffffu, par_cur >= 0);
    }
    const int bit = __ffs(todo) - 1;
    todo &= todo - 1u;
    par = __shfl_sync(0xffffffffu, par_cur, bit);
    row = row_of(c + (m0 + bit) * C);
    return true;
  };
  uint64_t* bar = full + c * R;
  unsigned char* mine = ring + static_cast<size_t>(c) * R * 2 * pb;
  // the stage loads of a warp: part h = 0 .. parts - 1 of each of its rows
  // with a parent, in order (warp-uniform); false at the end
  int cur_row = 0, cur_par = 0, cur_part = parts;
  auto next_load = [&](int& row, int& par, int& part) -> bool {
    if (cur_part == parts) {
      if (!next_item(cur_row, cur_par)) return false;
      cur_part = 0;
    }
    row = cur_row;
    par = cur_par;
    part = cur_part++;
    return true;
  };
  // the copies of part h of (row, par) into stage s of this warp's ring (lane 0)
  auto issue = [&](int s, int row, int par, int part) {
    if (lane == 0) {
      item_row[c * R + s] = row;
      item_par[c * R + s] = par;
      item_part[c * R + s] = part;
      const int j = row % P.positions;
      unsigned char* dst = mine + static_cast<size_t>(s) * 2 * pb;
      const char* child = reinterpret_cast<const char*>(base + static_cast<long>(row) * P.dim);
      const char* parent =
          reinterpret_cast<const char*>(base + (static_cast<long>(par) * P.positions + j) * P.dim);
      // the warp's generic reads of this stage (synchronised by the caller)
      // come before the copy engine's writes
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      mbar_arrive_tx(&bar[s], 2 * pb);
      bulk_load(dst, child + static_cast<size_t>(part) * pb, pb, &bar[s]);
      bulk_load(dst + pb, parent + static_cast<size_t>(part) * pb, pb, &bar[s]);
    }
  };

  int issued = 0;
  bool more = true;
  while (issued < R) {
    int row, par, part;
    if (!(more = next_load(row, par, part))) break;
    issue(issued, row, par, part);
    ++issued;
  }
  // a part holds groups/parts groups, a multiple of 32 when parts = 2, so
  // each lane meets its groups lane, lane + 32, ... of the row in order
  const int pgroups = static_cast<int>(pb / 16);
  int t = 0, s = 0;
  unsigned ph = 0;
  bool ok = true;
  float2 d = make_float2(0.f, 0.f), n = make_float2(0.f, 0.f);
  for (; t < issued; ++t) {
    // every lane waits; the warp leaves together if any lane's wait gave up
    if (!__all_sync(0xffffffffu, mbar_wait(&bar[s], ph))) {
      ok = false;
      break;
    }
    __syncwarp();
    const int row = item_row[c * R + s];
    const int par = item_par[c * R + s];
    const int part = item_part[c * R + s];
    const uint4* hc = reinterpret_cast<const uint4*>(mine + static_cast<size_t>(s) * 2 * pb);
    const uint4* hp = hc + pgroups;
#pragma unroll 4
    for (int g = lane; g < pgroups; g += kWarp) HElem<T>::accumulate2(hc[g], hp[g], d, n);
    __syncwarp();  // every lane's reads of the stage are done
    if (more) {
      int r2, p2, h2;
      if ((more = next_load(r2, p2, h2))) {
        issue(s, r2, p2, h2);
        ++issued;
      }
    }
    if (part == parts - 1) {
      double num = static_cast<double>(d.x) + static_cast<double>(d.y);
      double den = static_cast<double>(n.x) + static_cast<double>(n.y);
#pragma unroll
      for (int o = kWarp / 2; o > 0; o >>= 1) {
        num += __shfl_xor_sync(0xffffffffu, num, o);
        den += __shfl_xor_sync(0xffffffffu, den, o);
      }
      if (lane == 0) finish_row(P, row, par, row % P.positions, num, den);
      d = make_float2(0.f, 0.f);
      n = make_float2(0.f, 0.f);
    }
    if (++s == R) {
      s = 0;
      ph ^= 1u;
    }
  }
  if (!ok) {
    if (lane == 0) {
      atomicOr(P.status, kStatWait);
      // the copies still in flight must land before the warp leaves
      for (int u = t; u < issued; ++u)
        if (!mbar_wait(&bar[u % R], static_cast<unsigned>((u / R) & 1))) break;
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
  // kW words (4 flags each) loaded together, so a thread's chunk costs one
  // memory round trip per 4 kW rows in each of the two passes
  constexpr int kW = 8;
  const unsigned* fw = reinterpret_cast<const unsigned*>(P.flag);
  int v = 0;
  for (long i0 = lo; i0 < hi; i0 += 4 * kW) {
    unsigned w[kW];
#pragma unroll
    for (int k = 0; k < kW; ++k) w[k] = (i0 + 4 * k < hi) ? __ldcg(fw + (i0 + 4 * k) / 4) : 0u;
#pragma unroll
    for (int k = 0; k < kW; ++k) {
      // bytes past `hi` (the next chunk's rows, or padding past the last
      // row) are masked off
      const long left = hi - (i0 + 4 * k);
      const unsigned keep = left >= 4 ? 0xffffffffu : (left > 0 ? ((1u << (8 * left)) - 1u) : 0u);
      v += __popc(w[k] & keep & 0x01010101u);
    }
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
  for (long i0 = lo; i0 < hi; i0 += 4 * kW) {
    unsigned w[kW];
#pragma unroll
    for (int k = 0; k < kW; ++k) w[k] = (i0 + 4 * k < hi) ? __ldcg(fw + (i0 + 4 * k) / 4) : 0u;
#pragma unroll
    for (int k = 0; k < kW; ++k)
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const long i = i0 + 4 * k + q;
        if (i < hi && ((w[k] >> (8 * q)) & 0xffu) != 0u) P.rank[i] = slot++;
      }
  }
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
