// Kernels of the verification step under sampling variants: greedy (T = 0),
// top-k, nucleus (top-p) and a temperature per sequence.
//
// "Speculative decoding: how to run big models fast" (ai-trend.me), section
// "How it works", guarantee paragraph: argmax, top-k, nucleus and temperature
// sampling are standard sampling from an adjusted distribution, so the
// verification rule of "Speculative decoding - the small model writes first
// and the big model checks" (section 1) applies to the adjusted q and p.
//
// Adjusted distribution of a row (T > 0): the temperature softmax restricted
// to the entries whose sortable key is >= a per-row threshold theta, which is
// the larger of the top-k threshold (the k-th largest logit) and the nucleus
// threshold (the largest logit value v whose mass of entries >= v, within
// the top-k set, reaches top_p of that set's mass).  T = 0: the point mass on
// the first index of the largest logit.
//
// Three stream-ordered kernels:
//   select_kernel  one block per row: one scan for the maximum, the first
//                  argmax and (top-k <= 256) each thread's four largest values,
//                  which hold the top-k set whenever no thread's fourth value
//                  reaches the cut.  Otherwise a band histogram: one scan
//                  counts (top-k) or weighs (top-p alone) the entries in bands
//                  of their distance below the maximum, and a second gathers
//                  the bands that hold the cut as candidates.  The cuts
//                  themselves are binary searches over keys on the candidates'
//                  counts and double-precision masses.  A count radix select
//                  and a mass-histogram digit descent remain as fallbacks
//                  (candidates that do not fit; a cut outside them).  Last,
//                  the log-normaliser of the kept entries.
//   decide_kernel  one warp per sequence, one lane per position: adjusted
//                  q(t), p(t), the acceptance test and the first rejection by
//                  ballot; greedy sequences emit the argmax here.
//   draw_kernel    one block per sequence: the masked residual max(0, q - p)
//                  (or q for the bonus draw) in tiles, then the inverse CDF.
#pragma once

#include "verify_kernel.cuh"

namespace specsamp {

using specverify::Elem;
using specverify::ex2;
using specverify::kWarp;

constexpr int kSelThreads = 256;
constexpr int kSelWarps = kSelThreads / kWarp;
constexpr int kCand = 12288;         // most candidates kept in shared memory (large top-k sets)
constexpr int kCandSmem = kCand * 8; // their keys and weights (dynamic shared memory)
constexpr int kCandSmall = 2048;     // the candidate room of a call whose cuts need no more
constexpr int kDrawThreads = 512;
constexpr int kDecideThreads = 128;

// status bits (shared meaning with the plain step's status word)
enum : unsigned {
  kStatTokenRange = 1u,
  kStatNonFinite = 2u,
  kStatZeroMass = 4u,
  kStatTemperature = 16u
};

enum : int { kModeResidual = 0, kModeTarget = 1, kModeNone = 2, kModeGreedy = 3 };

struct SampRow {
  double l2;         // log2 sum over kept entries of 2^(x c)
  unsigned theta;    // kept iff key(x) >= theta
  int argmax;        // first index of the largest logit
  int valid;         // 0: NaN / +inf / no finite entry / bad temperature
  int kept;          // entries kept (diagnostic)
  float margin;      // top-p boundary margin (diagnostic; +inf when unused)
  int pad;
};

struct SampDecision {
  double lT, lD;
  unsigned thT, thD;
  int n, mode;
};

struct SampParams {
  const void* target;        // [B, G+1, V]
  const void* draft;         // [B, G, V]
  const int32_t* tokens;     // [B, G]
  const float* u_accept;     // [B, G]
  const float* u_resample;   // [B]
  const float* temperature;  // [B]
  int32_t* out_tokens;       // [B, G+1]
  int32_t* out_num_accepted; // [B]
  SampRow* rows;             // [B(G+1) + BG]: target rows, then draft rows
  SampDecision* decision;    // [B]
  specverify::RowStat* tstat;  // [B(G+1)] readback copies: log2 normaliser, valid, kept
  specverify::RowStat* dstat;  // [BG]
  specverify::PosInfo* pos;    // [BG] readback copies: q(t), p(t), ratio
  double* resid_mass;        // [B]
  unsigned* status;
  int batch, gamma, vocab;
  int top_k;                 // 0: off
  double top_p;              // >= 1: off
  int cand_cap;              // candidates that fit in the launch's dynamic shared memory
};

// ---------------------------------------------------------------------------
// helpers
// ---------------------------------------------------------------------------

// order-preserving unsigned key of a float (NaN excluded by the callers)
__device__ __forceinline__ unsigned fkey(float x) {
  const unsigned u = __float_as_uint(x);
  // negative: all bits flipped; otherwise the sign bit set
  return u ^ (static_cast<unsigned>(static_cast<int>(u) >> 31) | 0x80000000u);
}

__device__ __forceinline__ float key_value(unsigned k) {
  const unsigned u = (k & 0x80000000u) ? (k & 0x7fffffffu) : ~k;
  return __uint_as_float(u);
}

// log2(e)/T = c_hi + c_lo with c_hi rounded toward zero, c_lo a small positive
// normal float (so that -inf * c_lo stays -inf)
__device__ __forceinline__ void temp_consts(float T, float& c_hi, float& c_lo, double& c) {
  const double cd = 1.4426950408889634074 / static_cast<double>(T);
  c_hi = static_cast<float>(cd);
  if (static_cast<double>(c_hi) > cd) c_hi = nextafterf(c_hi, 0.f);
  c_lo = static_cast<float>(cd - static_cast<double>(c_hi));
  if (!(c_lo >= 1e-30f)) c_lo = 1e-30f;
  c = static_cast<double>(c_hi) + static_cast<double>(c_lo);
}

__device__ __forceinline__ bool temp_ok(float T) { return T >= 0.f && T < INFINITY; }

template <typename T>
__device__ __forceinline__ float elem(const T* row, long i) {
  return Elem<T>::load1(row, i);
}

// block reductions over kSelThreads (or kDrawThreads; both 512) threads
template <int NT>
__device__ __forceinline__ double block_sum(double v, double* sm) {
  const int lane = threadIdx.x & (kWarp - 1), warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  __syncthreads();
  if (lane == 0) sm[warp] = v;
  __syncthreads();
  double t = 0.0;
#pragma unroll
  for (int w = 0; w < NT / kWarp; ++w) t += sm[w];
  return t;
}

template <int NT>
__device__ __forceinline__ unsigned block_max_u(unsigned v, unsigned* sm) {
  const int lane = threadIdx.x & (kWarp - 1), warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = max(v, __shfl_xor_sync(0xffffffffu, v, o));
  __syncthreads();
  if (lane == 0) sm[warp] = v;
  __syncthreads();
  unsigned t = 0;
#pragma unroll
  for (int w = 0; w < NT / kWarp; ++w) t = max(t, sm[w]);
  return t;
}

template <int NT>
__device__ __forceinline__ int block_min_i(int v, int* sm) {
  const int lane = threadIdx.x & (kWarp - 1), warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = min(v, __shfl_xor_sync(0xffffffffu, v, o));
  __syncthreads();
  if (lane == 0) sm[warp] = v;
  __syncthreads();
  int t = 0x7fffffff;
#pragma unroll
  for (int w = 0; w < NT / kWarp; ++w) t = min(t, sm[w]);
  return t;
}

template <int NT>
__device__ __forceinline__ int block_max_i(int v, int* sm) {
  const int lane = threadIdx.x & (kWarp - 1), warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = max(v, __shfl_xor_sync(0xffffffffu, v, o));
  __syncthreads();
  if (lane == 0) sm[warp] = v;
  __syncthreads();
  int t = -1;
#pragma unroll
  for (int w = 0; w < NT / kWarp; ++w) t = max(t, sm[w]);
  return t;
}

// Row scans.  With 16-byte aligned rows a thread reads one 16-byte group per
// step (consecutive threads, consecutive groups); otherwise one element.
// `f(x, i)` sees every element once.  The loop count is the same for all
// threads of the block, so `f` may use warp collectives when `kUniform`.
template <typename T, bool kAligned, bool kUniform, typename F>
__device__ __forceinline__ void scan_row(const T* row, int V, F&& f) {
  if constexpr (kAligned) {
    // four groups per thread in flight per round
    constexpr int kVec = Elem<T>::kVec;
    constexpr int kU = 4;
    const long groups = V / kVec;
    const uint4* g4 = reinterpret_cast<const uint4*>(row);
    const long stride = static_cast<long>(blockDim.x) * kU;
    const long end = kUniform ? ((groups + stride - 1) / stride) * stride : groups;
    for (long g0 = threadIdx.x; g0 < end; g0 += stride) {
      uint4 v[kU];
#pragma unroll
      for (int u = 0; u < kU; ++u) {
        const long g = g0 + static_cast<long>(u) * blockDim.x;
        if (g < groups) v[u] = __ldg(g4 + g);
      }
#pragma unroll
      for (int u = 0; u < kU; ++u) {
        const long g = g0 + static_cast<long>(u) * blockDim.x;
        const bool in = g < groups;
        if (!kUniform && !in) break;
        float x[kVec];
        if (in) {
          Elem<T>::unpack(v[u], x);
        } else {
#pragma unroll
          for (int e = 0; e < kVec; ++e) x[e] = NAN;
        }
#pragma unroll
        for (int e = 0; e < kVec; ++e) f(x[e], in ? g * kVec + e : -1L);
      }
    }
  } else {
    const long end = kUniform ? ((static_cast<long>(V) + blockDim.x - 1) / blockDim.x) * blockDim.x : V;
    for (long i = threadIdx.x; i < end; i += blockDim.x) {
      const bool in = i < V;
      f(in ? elem<T>(row, i) : NAN, in ? i : -1L);
    }
  }
}

// The count-based radix select: the `rank`-th largest key (1-based) among the
// row's entries with key >= `floor_key`, for keys whose low `low_bits` bits are
// zero (bf16 values widened to float).  Histograms of 256 bins per 8-bit digit
// in shared memory; each warp adds a bin's lanes once (match_any).  Returns the
// key, and in *count_eq the number of entries equal to it.
template <typename T, bool kAligned>
__device__ unsigned radix_select(const T* row, int V, unsigned floor_key, long rank, int low_bits,
                                 int* hist, int* count_eq) {
  // hist: kSelWarps private histograms of 256 bins (plain shared atomics; a
  // warp's lanes that share a bin are serialised by the hardware)
  const int warp = threadIdx.x >> 5;
  __shared__ unsigned s_prefix, s_mask;
  __shared__ long s_rank;
  __shared__ int s_eq;
  if (threadIdx.x == 0) {
    s_prefix = 0u;
    s_mask = 0u;
    s_rank = rank;
    s_eq = 0;
  }
  __syncthreads();
  int* mine = hist + warp * 256;
  for (int shift = 24; shift >= low_bits; shift -= 8) {
    for (int i = threadIdx.x; i < 256 * kSelWarps; i += blockDim.x) hist[i] = 0;
    __syncthreads();
    const unsigned prefix = s_prefix, mask = s_mask;
    scan_row<T, kAligned, false>(row, V, [&](float x, long) {
      const unsigned k = fkey(x);
      if (k >= floor_key && (k & mask) == prefix) atomicAdd(&mine[(k >> shift) & 255u], 1);
    });
    __syncthreads();
    // totals into the first histogram
    for (int bin = threadIdx.x; bin < 256; bin += blockDim.x) {
      int t = 0;
      for (int w = 0; w < kSelWarps; ++w) t += hist[w * 256 + bin];
      hist[bin] = t;
    }
    __syncthreads();
    if (threadIdx.x < kWarp) {
      // the bin holding the rank-th largest: warp scan from the top bin down
      const int lane = threadIdx.x;
      long need = s_rank;
      long cum = 0;
      int sel = -1;
      for (int base = 255; base >= 0 && sel < 0; base -= kWarp) {
        const int bin = base - lane;
        long c = hist[bin];
        long incl = c;
#pragma unroll
        for (int o = 1; o < kWarp; o <<= 1) {
          const long y = __shfl_up_sync(0xffffffffu, incl, o);
          if (lane >= o) incl += y;
        }
        const unsigned hit = __ballot_sync(0xffffffffu, cum + incl >= need);
        if (hit) {
          const int l = __ffs(hit) - 1;
          const long before = __shfl_sync(0xffffffffu, incl - c, l);
          sel = base - l;
          cum += before;
        } else {
          cum += __shfl_sync(0xffffffffu, incl, kWarp - 1);
        }
      }
      if (lane == 0) {
        if (sel < 0) sel = 0;
        s_rank = need - cum;
        s_prefix = prefix | (static_cast<unsigned>(sel) << shift);
        s_mask = mask | (255u << shift);
        s_eq = hist[sel];
      }
    }
    __syncthreads();
  }
  *count_eq = s_eq;
  return s_prefix;
}

// The nucleus cut below the candidates: the largest key v in [lo, hi) with
// above + M(lo <= key, v <= key < hi) >= goal, where M sums the fp32 weights
// 2^(x c - o).  An 8-bit digit descent over the key with per-warp mass
// histograms in shared memory (one pass per digit).  Returns v, and the masses
// at or above v and strictly above v (both including `above`).
template <typename T, bool kAligned>
__device__ unsigned mass_descent(const T* row, int V, unsigned lo, unsigned hi, double above,
                                 double goal, int low_bits, float c_hi, float c_lo, float o,
                                 float* histw, double* m_ge, double* m_gt) {
  const int warp = threadIdx.x >> 5;
  __shared__ unsigned d_prefix, d_mask;
  __shared__ double d_above, d_bin;
  if (threadIdx.x == 0) {
    d_prefix = 0u;
    d_mask = 0u;
    d_above = above;
    d_bin = 0.0;
  }
  __syncthreads();
  float* mine = histw + warp * 256;
  for (int shift = 24; shift >= low_bits; shift -= 8) {
    for (int i = threadIdx.x; i < 256 * kSelWarps; i += blockDim.x) histw[i] = 0.f;
    __syncthreads();
    const unsigned prefix = d_prefix, mask = d_mask;
    scan_row<T, kAligned, false>(row, V, [&](float x, long) {
      const unsigned k = fkey(x);
      if (k >= lo && k < hi && (k & mask) == prefix)
        atomicAdd(&mine[(k >> shift) & 255u], ex2(specverify::arg2(x, c_hi, c_lo, o)));
    });
    __syncthreads();
    if (threadIdx.x < kWarp) {
      // bins from the top down, 32 at a time: the first whose cumulative mass
      // (after everything above it) reaches the goal
      const int lane = threadIdx.x;
      double cum = d_above;
      int sel = -1;
      double sel_mass = 0.0;
      for (int base = 255; base >= 0 && sel < 0; base -= kWarp) {
        const int bin = base - lane;
        double m = 0.0;
        for (int w = 0; w < kSelWarps; ++w) m += static_cast<double>(histw[w * 256 + bin]);
        double incl = m;
#pragma unroll
        for (int off = 1; off < kWarp; off <<= 1) {
          const double y = __shfl_up_sync(0xffffffffu, incl, off);
          if (lane >= off) incl += y;
        }
        const unsigned hit = __ballot_sync(0xffffffffu, cum + incl >= goal);
        if (hit) {
          const int l = __ffs(hit) - 1;
          sel = base - l;
          sel_mass = __shfl_sync(0xffffffffu, m, l);
          cum += __shfl_sync(0xffffffffu, incl - m, l);
        } else {
          cum += __shfl_sync(0xffffffffu, incl, kWarp - 1);
        }
      }
      if (lane == 0) {
        if (sel < 0) {  // rounding: the goal is not reached; take the lowest bin
          sel = 0;
          sel_mass = 0.0;
        }
        d_above = cum;
        d_bin = sel_mass;
        d_prefix = prefix | (static_cast<unsigned>(sel) << shift);
        d_mask = mask | (255u << shift);
      }
    }
    __syncthreads();
  }
  *m_gt = d_above;
  *m_ge = d_above + d_bin;
  return d_prefix;
}

// Bands of an entry's distance below the row maximum gmx: j = the nearest
// integer to min(max((gmx - x) s, 0), kBands - 1), with (gmx - x) s formed as
// one fused multiply-add and the rounding done by adding 2^23.  Every step is
// monotone, so j never increases with x and a run of bands is a run of keys;
// -inf lands in the last band.  s = kBandsPerUnit for counts (bands of 1/32
// logit) and kBandsPerUnit log2(e)/T for masses (1/32 of a factor 2 in weight).
constexpr int kBands = 4 * kSelThreads;  // 1024
constexpr float kBandsPerUnit = 32.f;
constexpr int kBandCap = kBands * kSelWarps / 2;  // candidate room whose area holds the histograms
constexpr double kBandSlack = 4e-6;      // relative room around the nucleus goal

__device__ __forceinline__ int band_of(float x, float s, float gs) {
  const float d = fminf(fmaxf(fmaf(-x, s, gs), 0.f), static_cast<float>(kBands - 1));
  return __float_as_int(d + 8388608.f) - 0x4b000000;
}

// Row scan by groups: `f(x, n, i0)` sees the n (0 past the end) elements
// i0 .. i0 + n - 1 in x[0 .. n); the loop count is the same for every thread
// of the block, so `f` may use warp collectives.
template <typename T, bool kAligned>
struct Groups {
  static constexpr int kN = kAligned ? Elem<T>::kVec : 1;
};

template <typename T, bool kAligned, typename F>
__device__ __forceinline__ void scan_groups(const T* row, int V, F&& f) {
  constexpr int kN = Groups<T, kAligned>::kN;
  if constexpr (kAligned) {
    constexpr int kU = 4;
    const long groups = V / kN;
    const uint4* g4 = reinterpret_cast<const uint4*>(row);
    const long stride = static_cast<long>(blockDim.x) * kU;
    const long end = ((groups + stride - 1) / stride) * stride;
    for (long g0 = threadIdx.x; g0 < end; g0 += stride) {
      uint4 v[kU];
#pragma unroll
      for (int u = 0; u < kU; ++u) {
        const long g = g0 + static_cast<long>(u) * blockDim.x;
        if (g < groups) v[u] = __ldg(g4 + g);
      }
#pragma unroll
      for (int u = 0; u < kU; ++u) {
        const long g = g0 + static_cast<long>(u) * blockDim.x;
        float x[kN];
        int n = 0;
        if (g < groups) {
          Elem<T>::unpack(v[u], x);
          n = kN;
        } else {
#pragma unroll
          for (int e = 0; e < kN; ++e) x[e] = 0.f;
        }
        f(x, n, g * kN);
      }
    }
  } else {
    const long end = ((static_cast<long>(V) + blockDim.x - 1) / blockDim.x) * blockDim.x;
    for (long i = threadIdx.x; i < end; i += blockDim.x) {
      const int n = i < V ? 1 : 0;
      float x[1] = {n ? elem<T>(row, i) : 0.f};
      f(x, n, i);
    }
  }
}

struct BandCut {
  int lo, hi;         // the bands holding the cut (lo = -1: none found)
  double end;         // running total (count or mass) through band hi
  double head, tail;  // mass: of the bands before lo, and after hi
  unsigned k_lo;      // smallest key in a band <= hi
  unsigned k_head;    // mass: smallest key in a band < lo (kmax + step when lo = 0);
                      // count: kmax + step (every band down to hi is wanted)
};

// Smallest key K in [key(-inf), kmax] with band_of(K) <= j, by warp 0 (every
// lane calls it): each round probes 32 evenly spaced keys of the remaining
// range, whose predicate runs false ... true since the band never increases
// with the key, and band(kmax) = 0.  (Should the rounding of gs put the
// maximum in a later band, no lane votes and lo only grows, so the loop still
// ends, at kmax.)  Rounded up to a multiple of `step`,
// which selects the same entries when every key is such a multiple.
__device__ __forceinline__ unsigned band_floor_key(int j, float s, float gs, unsigned kmax,
                                                   unsigned step) {
  const int lane = threadIdx.x & (kWarp - 1);
  unsigned lo = 0x007fffffu, hi = kmax;  // key(-inf) .. key(max): no NaN in between
  while (lo < hi) {
    const unsigned w = (hi - lo) / kWarp + 1u;
    const unsigned p = min(hi, lo + (static_cast<unsigned>(lane) + 1u) * w - 1u);
    const unsigned ok = __ballot_sync(0xffffffffu, band_of(key_value(p), s, gs) <= j);
    const int l = __ffs(ok) - 1;  // lane 31 probes hi, whose band is <= j
    const unsigned p_hit = __shfl_sync(0xffffffffu, p, l);
    const unsigned p_before = __shfl_sync(0xffffffffu, p, max(l - 1, 0));
    lo = (l == 0) ? lo : p_before + 1u;
    hi = p_hit;
  }
  return ((lo + step - 1u) / step) * step;
}

// One scan: per-warp histograms over bands of the entry count (kMass false)
// or of the fp32 weight 2^(x c - o) (kMass true), in `smem` (kSelWarps x
// kBands words); then warp 0 walks the bands from the largest values down,
// each lane over kBands / 32 consecutive bands, and takes the first band where
// the running total reaches the goal: `goal` entries (count), or `goal` times
// the row's mass (mass).  With kMass the range spans the bands holding the
// goal -/+ kBandSlack of the mass (the cut itself is settled later on
// double-precision candidate weights), and the masses before and after it
// come from the same histogram.
template <typename T, bool kAligned, bool kMass>
__device__ BandCut band_cut(const T* row, int V, float s, float gs, float c_hi, float c_lo,
                            float o, double goal, unsigned kmax, unsigned step, unsigned* smem) {
  float* hw = reinterpret_cast<float*>(smem);
  int* hc = reinterpret_cast<int*>(smem);
  const int warp = threadIdx.x >> 5;
  for (int i = threadIdx.x; i < kBands * kSelWarps; i += blockDim.x) smem[i] = 0u;
  __syncthreads();
  float* hwm = hw + warp * kBands;
  int* hcm = hc + warp * kBands;
  // the last band (everything far below the maximum; most of the row at a
  // low temperature) is summed in registers, not by atomics on one word
  float last_w = 0.f;
  int last_c = 0;
  scan_row<T, kAligned, false>(row, V, [&](float x, long) {
    const int j = band_of(x, s, gs);
    if constexpr (kMass) {
      const float w = ex2(specverify::arg2(x, c_hi, c_lo, o));
      if (j == kBands - 1) last_w += w;
      else atomicAdd(hwm + j, w);
    } else {
      if (j == kBands - 1) ++last_c;
      else atomicAdd(hcm + j, 1);
    }
  });
  if constexpr (kMass) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) last_w += __shfl_xor_sync(0xffffffffu, last_w, off);
    if ((threadIdx.x & (kWarp - 1)) == 0) atomicAdd(hwm + kBands - 1, last_w);
  } else {
    last_c = __reduce_add_sync(0xffffffffu, last_c);
    if ((threadIdx.x & (kWarp - 1)) == 0) atomicAdd(hcm + kBands - 1, last_c);
  }
  __syncthreads();
  // totals over the warps (fp64) into the first kBands doubles of `smem`
  constexpr int kPerT = kBands / kSelThreads;
  const int b0 = kPerT * threadIdx.x;
  double a[kPerT];
#pragma unroll
  for (int e = 0; e < kPerT; ++e) {
    a[e] = 0.0;
#pragma unroll
    for (int w = 0; w < kSelWarps; ++w)
      a[e] += kMass ? static_cast<double>(hw[w * kBands + b0 + e])
                    : static_cast<double>(hc[w * kBands + b0 + e]);
  }
  __syncthreads();
  double* tot = reinterpret_cast<double*>(smem);
#pragma unroll
  for (int e = 0; e < kPerT; ++e) tot[b0 + e] = a[e];
  __syncthreads();
  __shared__ BandCut s_bc;
  if (threadIdx.x < kWarp) {
    constexpr int kPer = kBands / kWarp;
    const int lane = threadIdx.x;
    const double* mine = tot + lane * kPer;
    double sl = 0.0;
#pragma unroll 8
    for (int i = 0; i < kPer; ++i) sl += mine[i];
    double incl = sl;
#pragma unroll
    for (int off = 1; off < kWarp; off <<= 1) {
      const double y = __shfl_up_sync(0xffffffffu, incl, off);
      if (lane >= off) incl += y;
    }
    // each lane's bands run from the previous lane's end to its own, so the
    // lanes' intervals chain and cover (0, total]
    double start = __shfl_up_sync(0xffffffffu, incl, 1);
    if (lane == 0) start = 0.0;
    const double total = __shfl_sync(0xffffffffu, incl, kWarp - 1);
    const double g = kMass ? goal * total : goal;
    const double slack = kMass ? kBandSlack * total : 0.0;
    // first band j with end(j - 1) < h <= end(j); its start and end
    auto find = [&](double h, double* s_out, double* e_out) -> int {
      int found = -1;
      double fs = 0.0, fe = 0.0, cum = start;
      for (int i = 0; i < kPer; ++i) {
        const double nxt = (i == kPer - 1) ? incl : cum + mine[i];
        if (found < 0 && cum < h && h <= nxt) {
          found = lane * kPer + i;
          fs = cum;
          fe = nxt;
        }
        cum = nxt;
      }
      const unsigned m = __ballot_sync(0xffffffffu, found >= 0);
      if (!m) return -1;
      const int l = __ffs(m) - 1;
      *s_out = __shfl_sync(0xffffffffu, fs, l);
      *e_out = __shfl_sync(0xffffffffu, fe, l);
      return __shfl_sync(0xffffffffu, found, l);
    };
    double s_lo = 0.0, e_lo = 0.0, s_hi = 0.0, e_hi = 0.0;
    const double h_lo = g - slack;
    int lo = h_lo <= 0.0 ? 0 : find(h_lo, &s_lo, &e_lo);
    const int hi = find(fmin(g + slack, total), &s_hi, &e_hi);
    if (hi < 0 || lo > hi) lo = -1;
    unsigned k_lo = 0u, k_head = 0u;
    if (lo >= 0) {
      k_lo = band_floor_key(hi, s, gs, kmax, step);
      k_head = (kMass && lo > 0) ? band_floor_key(lo - 1, s, gs, kmax, step) : kmax + step;
    }
    if (lane == 0) s_bc = BandCut{lo, hi, e_hi, s_lo, fmax(total - e_hi, 0.0), k_lo, k_head};
  }
  __syncthreads();
  return s_bc;
}

// Candidates: the entries with k_lo <= key < k_head (exactly the entries of
// the bands holding the cut), keys into shared memory and then their weights
// in double precision (rounded to float); the count in the return value (may
// exceed the room).  With kHead also the number of entries with key >= k_head
// (the earlier bands) in *nhead.  One vote per group of elements: where a lane
// holds candidates, one warp scan of the lanes' counts and one shared atomic
// per warp place them.
template <typename T, bool kAligned, bool kHead>
__device__ int gather_range(const T* row, int V, unsigned k_lo, unsigned k_head, double c,
                            double od, unsigned* cand_key, float* cand_w, int* cand_n, double* smd,
                            double* nhead, int cap) {
  constexpr int kN = Groups<T, kAligned>::kN;
  const int lane = threadIdx.x & (kWarp - 1);
  if (threadIdx.x == 0) *cand_n = 0;
  __syncthreads();
  int nh = 0;
  scan_groups<T, kAligned>(row, V, [&](const float* x, int n, long) {
    unsigned tmask = 0u;
    if (n == kN) {
#pragma unroll
      for (int e = 0; e < kN; ++e) {
        const unsigned key = fkey(x[e]);
        const bool above_lo = key >= k_lo;
        const bool in_head = key >= k_head;
        tmask |= static_cast<unsigned>(above_lo && !in_head) << e;
        if constexpr (kHead) nh += in_head;
      }
    }
    if (__any_sync(0xffffffffu, tmask != 0u)) {
      const int cnt = __popc(tmask);
      int incl = cnt;
#pragma unroll
      for (int off = 1; off < kWarp; off <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += y;
      }
      int base = 0;
      if (lane == kWarp - 1) base = atomicAdd(cand_n, incl);
      int slot = __shfl_sync(0xffffffffu, base, kWarp - 1) + incl - cnt;
#pragma unroll
      for (int e = 0; e < kN; ++e) {
        if ((tmask >> e) & 1u) {
          if (slot < cap) cand_key[slot] = fkey(x[e]);
          ++slot;
        }
      }
    }
  });
  __syncthreads();
  const int nc = *cand_n;
  for (int i = threadIdx.x; i < min(nc, cap); i += blockDim.x)
    cand_w[i] = static_cast<float>(exp2(static_cast<double>(key_value(cand_key[i])) * c - od));
  *nhead = kHead ? block_sum<kSelThreads>(static_cast<double>(nh), smd) : 0.0;
  return nc;
}

// What the candidate stage needs besides the candidates of a band cut
// (kept in shared memory: read only after the scans).
struct BandSide {
  unsigned kmax;     // a key at or above every candidate
  unsigned hkmin;    // smallest key above the candidates' bands
  double head, nhead;  // mass (fp64 weights 2^(x c - od)) and count of those entries
};

// ---------------------------------------------------------------------------
// kernel 1: per-row adjusted distribution
// ---------------------------------------------------------------------------

__device__ __forceinline__ void put_row(const SampParams& P, long r, long nT, const SampRow& v) {
  P.rows[r] = v;
  const specverify::RowStat st{v.l2, v.valid, v.kept};
  if (r < nT) P.tstat[r] = st;
  else P.dstat[r - nT] = st;
}

// Candidates: entries gathered into shared memory (key, weight in double
// precision rounded to float) when their key is above `above` and at least
// `floor_key`; the count may exceed the room `cap` (then only the first `cap`
// are kept and the caller falls back).  Entries equal to `above` are counted
// in *n_eq.
template <typename T, bool kAligned, bool kTail>
__device__ int gather(const T* row, int V, unsigned above, unsigned floor_key, double c, double od,
                      unsigned* cand_key, float* cand_w, int* cand_n, float c_hi, float c_lo,
                      float o, double* sm, double* n_eq_out, double* tail_out, int cap) {
  const int lane = threadIdx.x & (kWarp - 1);
  if (threadIdx.x == 0) *cand_n = 0;
  __syncthreads();
  int n_eq = 0;
  float tail = 0.f;  // entries floor_key <= key < above
  scan_row<T, kAligned, true>(row, V, [&](float x, long i) {
    const unsigned k = fkey(x);
    const bool valid = i >= 0;
    const bool take = valid && k > above && k >= floor_key;
    n_eq += (valid && k == above && k >= floor_key);
    if (kTail && valid && k < above && k >= floor_key) tail += ex2(specverify::arg2(x, c_hi, c_lo, o));
    const unsigned m = __ballot_sync(0xffffffffu, take);
    if (m) {
      int at = 0;
      if (lane == __ffs(m) - 1) at = atomicAdd(cand_n, __popc(m));
      at = __shfl_sync(0xffffffffu, at, __ffs(m) - 1);
      if (take) {
        const int slot = at + __popc(m & ((1u << lane) - 1u));
        if (slot < cap) cand_key[slot] = k;
      }
    }
  });
  __syncthreads();
  const int n = *cand_n;
  // the candidates' weights in double precision (rounded to float), after the
  // scan so that no lane waits on another's exp2
  for (int i = threadIdx.x; i < min(n, cap); i += blockDim.x)
    cand_w[i] = static_cast<float>(exp2(static_cast<double>(key_value(cand_key[i])) * c - od));
  *n_eq_out = block_sum<kSelThreads>(static_cast<double>(n_eq), sm);
  *tail_out = block_sum<kSelThreads>(static_cast<double>(tail), sm) * exp2(static_cast<double>(o) - od);
  return n;
}

// A reduction over either warp 0 alone (kW) or the whole block.
template <bool kW>
struct Red {
  double* sm;
  __device__ __forceinline__ double sum(double v) const {
    if constexpr (kW) return specverify::warp_sum(v);
    else return block_sum<kSelThreads>(v, sm);
  }
  __device__ __forceinline__ int first() const { return kW ? (threadIdx.x & (kWarp - 1)) : threadIdx.x; }
  __device__ __forceinline__ int stride() const { return kW ? kWarp : static_cast<int>(blockDim.x); }
};

constexpr int kWarpCands = 2048;  // candidate sets up to this size: warp 0 alone

struct CandSet {
  const unsigned* key;
  const float* w;   // weights 2^(x c - od), double-precision exp2 rounded to float
  int n;
  unsigned above;   // every entry with key > above is a candidate
  double n_eq;      // entries equal to `above` (not stored; one weight)
  double w_above;
  double tail;      // mass of the entries theta <= key < above
  unsigned kmax, step;  // largest candidate key; spacing of keys
  double head, nhead;   // mass and count of entries above every candidate (not stored)
};

struct StageOut {
  unsigned theta;
  float margin;
  double Z, kept;   // mass (when z_valid) and count (when kept_valid) of the kept set
  double Zk, goal, m0;  // for the whole-row fallback, when below
  int z_valid, kept_valid;
  int below;        // 1: the nucleus cut lies below the candidates; 2: above them
};

// The top-k cut (when `do_k`: the k-th largest candidate key, searched from
// `theta` = a lower bound) and the nucleus cut (when `do_p`) over the
// candidates; run by warp 0 alone or by the whole block.  Thread 0 writes *out.
template <bool kW>
__device__ void cand_stage(const Red<kW>& R, const CandSet& cs, bool do_k, int top_k, bool do_p,
                           double top_p, unsigned theta, StageOut* out) {
  const int f = R.first(), st = R.stride();
  const unsigned step = cs.step;
  if (do_k) {
    unsigned lo = theta, hi = cs.kmax;
    while (lo < hi) {
      const unsigned mid = lo + (((hi - lo) / step + 1) / 2) * step;
      double cnt = 0.0;
      for (int i = f; i < cs.n; i += st) cnt += cs.key[i] >= mid ? 1.0 : 0.0;
      if (R.sum(cnt) >= top_k) lo = mid;
      else hi = mid - step;
    }
    theta = lo;
  }
  // M(>= v) for v up to the largest candidate: candidates >= max(v, theta),
  // the group at `above`, and the entries above every candidate
  auto mass_ge = [&](unsigned v) -> double {
    double sv = 0.0;
    for (int i = f; i < cs.n; i += st)
      if (cs.key[i] >= v && cs.key[i] >= theta) sv += static_cast<double>(cs.w[i]);
    double t = R.sum(sv) + cs.head;
    if (v <= cs.above && cs.above >= theta) t += cs.n_eq * cs.w_above;
    return t;
  };
  StageOut o{theta, INFINITY, 0.0, 0.0, 0.0, 0.0, 0.0, 0, 0, 0};
  if (do_p) {
    const unsigned v0 = max(theta, cs.above);
    const double m0 = mass_ge(v0);
    const double Zk = cs.tail + m0;  // mass of the entries >= theta
    const double goal = top_p * Zk;
    o.Zk = Zk;
    o.goal = goal;
    o.m0 = m0;
    if (cs.head > 0.0 && cs.head >= goal) {
      o.below = 2;
    } else if (m0 >= goal) {
      unsigned lo = v0, hi = cs.kmax;
      while (lo < hi) {
        const unsigned mid = lo + (((hi - lo) / step + 1) / 2) * step;
        if (mass_ge(mid) >= goal) lo = mid;
        else hi = mid - step;
      }
      const double m_ge = mass_ge(lo);
      const double m_gt = (lo >= cs.kmax) ? cs.head : mass_ge(lo + step);
      o.margin = static_cast<float>(fmin(top_p - m_gt / Zk, m_ge / Zk - top_p));
      o.theta = max(theta, lo);
    } else {
      o.below = 1;
    }
  }
  // the kept set's mass and size, when every kept entry is a candidate or
  // above them
  if (!o.below && (o.theta > cs.above || (o.theta == cs.above && cs.n_eq == 0.0))) {
    double sv = 0.0, cnt = 0.0;
    for (int i = f; i < cs.n; i += st)
      if (cs.key[i] >= o.theta && key_value(cs.key[i]) != -INFINITY) {
        sv += static_cast<double>(cs.w[i]);
        cnt += 1.0;
      }
    o.Z = R.sum(sv) + cs.head;
    o.kept = R.sum(cnt) + cs.nhead;
    o.z_valid = 1;
    o.kept_valid = 1;
  } else if (!o.below && do_p) {
    o.Z = mass_ge(o.theta);  // includes the group at `above`; the count comes from a pass
    o.z_valid = 1;
  }
  if (threadIdx.x == 0) *out = o;
}

struct PassA {
  float mx;     // largest value of the thread's entries
  long am;      // its first index
  bool bad;     // a NaN or +inf entry
  float t[4];   // the thread's four largest values, descending (-inf: empty)
  float o, s;   // with kSum: s = sum 2^(x c - o) over the thread's entries
  int ninf;     // with kSum: entries equal to -inf
};

// One scan of the row: each thread's maximum, first argmax and invalid
// entries; with kTrack also its four largest values, inserted only when a
// 16-byte group's maximum beats the fourth (rare after the first groups).
template <typename T, bool kAligned, bool kTrack, bool kSum>
__device__ __forceinline__ PassA pass_a(const T* row, int V, float c_hi, float c_lo) {
  PassA a{-INFINITY, 0x7fffffff, false, {-INFINITY, -INFINITY, -INFINITY, -INFINITY},
          -INFINITY, 0.f, 0};
  auto insert = [&](float x) {
    if (x > a.t[3]) {  // old values on the right
      a.t[3] = fmaxf(a.t[3], fminf(a.t[2], x));
      a.t[2] = fmaxf(a.t[2], fminf(a.t[1], x));
      a.t[1] = fmaxf(a.t[1], fminf(a.t[0], x));
      a.t[0] = fmaxf(a.t[0], x);
    }
  };
  if constexpr (kAligned) {
    constexpr int kVec = Elem<T>::kVec;
    constexpr int kU = 4;
    const long groups = V / kVec;
    const uint4* g4 = reinterpret_cast<const uint4*>(row);
    const long stride = static_cast<long>(blockDim.x) * kU;
    for (long g0 = threadIdx.x; g0 < groups; g0 += stride) {
      uint4 v[kU];
#pragma unroll
      for (int u = 0; u < kU; ++u) {
        const long g = g0 + static_cast<long>(u) * blockDim.x;
        if (g < groups) v[u] = __ldg(g4 + g);
      }
#pragma unroll
      for (int u = 0; u < kU; ++u) {
        const long g = g0 + static_cast<long>(u) * blockDim.x;
        if (g >= groups) break;
        float x[kVec];
        Elem<T>::unpack(v[u], x);
        float gm = x[0];
        bool gb = (x[0] != x[0]) || x[0] == INFINITY;
#pragma unroll
        for (int e = 1; e < kVec; ++e) {
          gm = fmaxf(gm, x[e]);
          gb |= (x[e] != x[e]) || x[e] == INFINITY;
        }
        a.bad |= gb;
        if (gm > a.mx) {  // the first index of the group's maximum
          a.mx = gm;
#pragma unroll
          for (int e = kVec - 1; e >= 0; --e)
            if (x[e] == gm) a.am = g * kVec + e;
        }
        if (kTrack && gm > a.t[3]) {
#pragma unroll
          for (int e = 0; e < kVec; ++e) insert(x[e]);
        }
        if constexpr (kSum) {
          const float on = gm * c_hi;
          if (on > a.o) {  // raise the offset (a.o = -inf: a.s is 0 and stays so)
            a.s *= ex2(a.o - on);
            a.o = on;
          }
#pragma unroll
          for (int e = 0; e < kVec; ++e) {
            a.s += ex2(specverify::arg2(x[e], c_hi, c_lo, a.o));
            a.ninf += x[e] == -INFINITY;
          }
        }
      }
    }
  } else {
    for (long i = threadIdx.x; i < V; i += blockDim.x) {
      const float x = elem<T>(row, i);
      a.bad |= (x != x) || x == INFINITY;
      if (x > a.mx) {
        a.mx = x;
        a.am = i;
      }
      if (kTrack) insert(x);
      if constexpr (kSum) {
        const float on = x * c_hi;
        if (on > a.o) {
          a.s *= ex2(a.o - on);
          a.o = on;
        }
        a.s += ex2(specverify::arg2(x, c_hi, c_lo, a.o));
        a.ninf += x == -INFINITY;
      }
    }
  }
  return a;
}

// ---------------------------------------------------------------------------
// bf16 rows: the cuts in one scan, over exact values
// ---------------------------------------------------------------------------
//
// A bf16 logit takes one of at most 65536 values, and the entries near the
// row maximum hold the mass that top-k and top-p cut.  One scan counts, per
// value, the entries of every value in a window of kXBins consecutive bf16
// values (counts in shared memory), placed from a sample of the row: kXAbove
// values above the sample's maximum, the rest below it.  Entries below the
// window only add to a per-thread fp32 mass (a nucleus cut alone needs the
// row's total); an entry above it means the sample missed the maximum by
// more than the window allows, and the row takes the general path.  After
// the scan every value of the window has an exact count, so its mass
// count * 2^(x c - od) is exact in fp64, and the cuts are walks over the
// window from the largest value down: the k-th largest value (cumulative
// counts), then the first value whose cumulative mass reaches top_p of the
// kept set's mass (or the row's): the walk over distinct values, ties
// included, that defines the cut.  A cut that would fall below the window
// takes the general path too, and so does a row holding NaN or +inf (an
// entry above the window) or no entry in the window (the general path also
// reports the invalid rows).  The row maximum is the largest value with a
// count; the first argmax is not needed (only greedy rows use it, and they do
// not come here).

constexpr int kXBins = 4096;                   // values in the window (16 KB of counts)
constexpr int kXAbove = 1024;                  // of which above the sample's maximum
constexpr int kXPer = kXBins / kSelThreads;    // window values per thread in the walks
constexpr unsigned kKeyNegInf = 0x007fu;       // 16-bit key of -inf
constexpr unsigned kKeyPosInf = 0xff80u;       // 16-bit key of +inf (NaN keys lie outside both)

// order-preserving 16-bit key of a bf16 value (its bits in the low half of h):
// the top half of fkey of the value widened to float
__device__ __forceinline__ unsigned bf16_key(unsigned h) {
  return (h & 0x8000u) ? (~h & 0xffffu) : (h | 0x8000u);
}
__device__ __forceinline__ float key16_value(unsigned k) {
  const unsigned h = (k & 0x8000u) ? (k & 0x7fffu) : (~k & 0xffffu);
  return __uint_as_float(h << 16);
}

struct XState {
  unsigned kmax2 = 0u;            // per 16-bit half: the largest key seen
  unsigned kmin2 = 0xffffffffu;   // per 16-bit half: the smallest key seen
  float2 tail = make_float2(0.f, 0.f);  // kTail: sum 2^(x c - o) below the window (per half)
};

// One 32-bit word of two bf16 entries, branch-free: both keys in one register
// (each half h -> h ^ 0x8000 for a positive value, ~h for a negative one);
// a key in the window [klo, klo + span] adds 1 to its count (a shared
// reduction at index key - klo, predicated in the instruction itself); the
// largest and smallest keys of both halves are kept with packed 16-bit
// max / min, which after the scan flag a key above the window, +inf or NaN
// of either sign; the mass below the window is an ex2 of -inf where it does
// not apply.  hb: the shared-memory address of the count of key 0.
template <bool kTail>
__device__ __forceinline__ void x_word(unsigned w, unsigned klo, unsigned span, unsigned hb,
                                       float c_hi, float c_lo, float o, XState& st) {
  const unsigned neg = (w >> 15) & 0x00010001u;              // sign of each half
  const unsigned k2 = w ^ (0x80008000u | (neg * 0x7fffu));   // both keys
  asm("max.u16x2 %0, %0, %1;" : "+r"(st.kmax2) : "r"(k2));
  asm("min.u16x2 %0, %0, %1;" : "+r"(st.kmin2) : "r"(k2));
  unsigned idx[2];
#pragma unroll
  for (int half = 0; half < 2; ++half) {
    const unsigned k = half ? (k2 >> 16) : (k2 & 0xffffu);
    idx[half] = k - klo;
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.le.u32 p, %0, %1;\n\t@p red.shared.add.u32 [%2], 1;\n\t}"
        ::"r"(idx[half]), "r"(span), "r"(hb + 4u * k));
  }
  if constexpr (kTail) {
    // both halves' exponents with the packed fp32x2 instructions (x c - o
    // as two FMAs each, as everywhere); ex2 of -inf for entries in the window
    const float2 x = make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
    const float2 y = __ffma2_rn(x, make_float2(c_lo, c_lo),
                                __ffma2_rn(x, make_float2(c_hi, c_hi), make_float2(-o, -o)));
    const float2 e = make_float2(ex2(idx[0] <= span ? -INFINITY : y.x),
                                 ex2(idx[1] <= span ? -INFINITY : y.y));
    st.tail = __fadd2_rn(st.tail, e);
  }
}

// Returns true when the row's adjusted distribution is settled (and written),
// false when the general path must take the row.  Every thread of the block
// calls it and gets the same answer.
template <bool kTail>
__device__ bool exact_select(const SampParams& P, long r, long nT, const __nv_bfloat16* row, int V,
                             float c_hi, float c_lo, double c, bool use_k, bool use_p,
                             unsigned* hist) {
  __shared__ double smd[kSelWarps];
  __shared__ unsigned smu[kSelWarps];
  __shared__ int s_cut;        // window value of the cut (-1: the general path)
  __shared__ double s_zcut;    // mass through it
  __shared__ double s_ncut;    // entries through it
  __shared__ float s_margin;
  const int tid = threadIdx.x;
  const long groups = V / 8;
  const uint4* g4 = reinterpret_cast<const uint4*>(row);

  // the window: from the largest finite key among the row's first kSelThreads groups
  unsigned ks = 0u;
  if (tid < groups) {
    const uint4 v = __ldg(g4 + tid);
    const unsigned w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const unsigned k0 = bf16_key(w[q] & 0xffffu), k1 = bf16_key(w[q] >> 16);
      if (k0 < kKeyPosInf) ks = max(ks, k0);
      if (k1 < kKeyPosInf) ks = max(ks, k1);
    }
  }
  for (int i = tid; i < kXBins; i += kSelThreads) hist[i] = 0u;
  ks = block_max_u<kSelThreads>(ks, smu);  // (barriers inside: hist is clear after it)
  if (ks <= kKeyNegInf) ks = 0x8000u;      // no finite entry sampled: centre on 0
  const int khi = min(static_cast<int>(ks) + kXAbove, static_cast<int>(kKeyPosInf) - 1);
  // the window: keys klo .. khi (never the key of -inf); count index = key - klo
  const int klo = max(khi - kXBins + 1, static_cast<int>(kKeyNegInf) + 1);
  const unsigned span = static_cast<unsigned>(khi - klo);
  // the count of key k lives at hist[k - klo] (only keys in the window are counted)
  const unsigned hb = static_cast<unsigned>(__cvta_generic_to_shared(hist)) - 4u * static_cast<unsigned>(klo);
  const float o = key16_value(ks) * c_hi;  // weights of the entries below the window

  XState st;
  {
    constexpr int kU = 8;  // 16-byte loads in flight per thread
    const long stride = static_cast<long>(kSelThreads) * kU;
    for (long g0 = tid; g0 < groups; g0 += stride) {
      uint4 v[kU];
#pragma unroll
      for (int u = 0; u < kU; ++u) {
        const long g = g0 + static_cast<long>(u) * kSelThreads;
        if (g < groups) v[u] = __ldg(g4 + g);
      }
#pragma unroll
      for (int u = 0; u < kU; ++u) {
        const long g = g0 + static_cast<long>(u) * kSelThreads;
        if (g >= groups) break;
        x_word<kTail>(v[u].x, static_cast<unsigned>(klo), span, hb, c_hi, c_lo, o, st);
        x_word<kTail>(v[u].y, static_cast<unsigned>(klo), span, hb, c_hi, c_lo, o, st);
        x_word<kTail>(v[u].z, static_cast<unsigned>(klo), span, hb, c_hi, c_lo, o, st);
        x_word<kTail>(v[u].w, static_cast<unsigned>(klo), span, hb, c_hi, c_lo, o, st);
      }
    }
  }
  // rows with an entry above the window, NaN or +inf go to the general path
  // (which also reports the invalid ones); a key below that of -inf is a
  // negative NaN
  const unsigned kmx = max(st.kmax2 & 0xffffu, st.kmax2 >> 16);
  const unsigned kmn = min(st.kmin2 & 0xffffu, st.kmin2 >> 16);
  const bool off = kmx > static_cast<unsigned>(khi) || kmn < kKeyNegInf;
  if (__syncthreads_or(off)) return false;
  const double tail_o =
      kTail ? block_sum<kSelThreads>(static_cast<double>(st.tail.x) + static_cast<double>(st.tail.y), smd)
            : 0.0;
  // the window in descending order: rank q = khi - key, count hist[span - q]
  // (ranks past span lie below the window: no count); the row maximum is the
  // first rank with a count (none: every entry is below the window or -inf,
  // and the general path takes the row)
  const int b0 = tid * kXPer;
  auto count_at = [&](int q) -> unsigned {
    return q <= static_cast<int>(span) ? hist[static_cast<int>(span) - q] : 0u;
  };
  unsigned first = 0xffffffffu;
  for (int i = kXPer - 1; i >= 0; --i)
    if (count_at(b0 + i)) first = static_cast<unsigned>(b0 + i);
  first = 0xffffffffu - block_max_u<kSelThreads>(0xffffffffu - first, smu);
  if (first == 0xffffffffu) return false;
  const unsigned kmax = static_cast<unsigned>(khi) - first;
  SampRow out{0.0, 0u, -1, 1, V, INFINITY, 0};

  // exact masses of the window's values, relative to the maximum
  const double od = static_cast<double>(key16_value(kmax)) * c;
  double cnt_t = 0.0, mass_t = 0.0;
#pragma unroll 4
  for (int i = 0; i < kXPer; ++i) {
    const unsigned n = count_at(b0 + i);
    if (n) {
      const double x = key16_value(static_cast<unsigned>(khi - (b0 + i)));
      cnt_t += n;
      mass_t += n * exp2(x * c - od);
    }
  }
  double c_in, c_ex, c_tot, m_in, m_ex, m_tot;
  specverify::block_scan<kSelThreads>(cnt_t, c_in, c_ex, c_tot);
  specverify::block_scan<kSelThreads>(mass_t, m_in, m_ex, m_tot);
  if (tid == 0) {
    s_cut = -1;
    s_margin = INFINITY;
  }
  __syncthreads();
  // top-k: the window value where the cumulative count reaches k
  int kcut = kXBins - 1;
  double zk = m_tot;
  if (use_k) {
    const double k = static_cast<double>(P.top_k);
    if (c_ex < k && k <= c_in) {
      double cc = c_ex, mm = m_ex;
      for (int i = 0; i < kXPer; ++i) {
        const unsigned n = count_at(b0 + i);
        if (!n) continue;
        cc += n;
        mm += n * exp2(static_cast<double>(key16_value(static_cast<unsigned>(khi - (b0 + i)))) * c - od);
        if (cc >= k) {
          s_cut = b0 + i;
          s_zcut = mm;
          s_ncut = cc;
          break;
        }
      }
    }
    __syncthreads();
    if (s_cut < 0) return false;  // the k-th largest lies below the window
    kcut = s_cut;
    zk = s_zcut;
  }
  if (use_p) {
    // the row's mass (nucleus alone, with the entries below the window) or
    // the top-k set's; the first window value whose cumulative mass, divided
    // by it, reaches top_p, and never past the top-k cut
    const double Z = use_k ? zk : m_tot + tail_o * exp2(static_cast<double>(o) - od);
    const double tp = P.top_p;
    __syncthreads();
    if (tid == 0) s_cut = -1;
    __syncthreads();
    const bool mine = b0 <= kcut && (m_ex / Z < tp || b0 == 0) &&
                      (m_in / Z >= tp || (b0 <= kcut && kcut < b0 + kXPer));
    if (mine) {
      double cc = c_ex, mm = m_ex;
      for (int i = 0; i < kXPer && b0 + i <= kcut; ++i) {
        const unsigned n = count_at(b0 + i);
        if (!n) continue;
        const double before = mm;
        cc += n;
        mm += n * exp2(static_cast<double>(key16_value(static_cast<unsigned>(khi - (b0 + i)))) * c - od);
        if (mm / Z >= tp || b0 + i == kcut) {
          if (atomicCAS(&s_cut, -1, b0 + i) == -1) {
            s_zcut = mm;
            s_ncut = cc;
            s_margin = static_cast<float>(fmin(tp - before / Z, mm / Z - tp));
          }
          break;
        }
      }
    }
    __syncthreads();
    if (s_cut < 0) return false;  // the nucleus reaches below the window
  }
  if (tid == 0) {
    const int cut = s_cut;
    out.theta = fkey(key16_value(static_cast<unsigned>(khi - cut)));
    out.l2 = od + log2(s_zcut);
    out.kept = static_cast<int>(s_ncut);
    out.margin = s_margin;
    put_row(P, r, nT, out);
  }
  return true;
}

template <typename T, bool kAligned>
__global__ void __launch_bounds__(kSelThreads, 4) select_kernel(const SampParams P) {
  __shared__ double smd[kSelWarps];
  __shared__ unsigned smu[kSelWarps];
  __shared__ int smi[kSelWarps];
  __shared__ unsigned s_tmax[kSelThreads];
  extern __shared__ unsigned cand_smem[];  // cap keys, then cap weights
  const int kCap = P.cand_cap;
  unsigned* cand_key = cand_smem;
  float* cand_w = reinterpret_cast<float*>(cand_smem + kCap);
  // the radix select's per-warp histograms reuse the candidate area: every
  // radix select runs before the candidates it serves are gathered
  int* hist = reinterpret_cast<int*>(cand_smem);
  __shared__ int cand_n;

  const int G = P.gamma, V = P.vocab;
  const long nT = static_cast<long>(P.batch) * (G + 1);
  const long r = blockIdx.x;
  const bool is_t = r < nT;
  const int b = is_t ? static_cast<int>(r / (G + 1)) : static_cast<int>((r - nT) / G);
  const T* row = is_t ? static_cast<const T*>(P.target) + r * V
                      : static_cast<const T*>(P.draft) + (r - nT) * V;
  const float temp = P.temperature[b];
  const int low_bits = sizeof(T) == 2 ? 16 : 0;
  const unsigned step = 1u << low_bits;

  // bf16 rows with a filter: the one-scan cut over exact values first
  if constexpr (sizeof(T) == 2 && kAligned) {
    const bool filter = (P.top_k > 0 && P.top_k < V) || P.top_p < 1.0;
    // (a top-k cut of at most kSelThreads keeps the per-thread lists below:
    // one lighter scan settles it)
    const bool lists = P.top_k > 0 && P.top_k <= kSelThreads && P.top_k < V;
    if (filter && !lists && temp > 0.f && temp_ok(temp)) {
      float xc_hi, xc_lo;
      double xc;
      temp_consts(temp, xc_hi, xc_lo, xc);
      const bool uk = P.top_k > 0 && P.top_k < V, up = P.top_p < 1.0;
      const bool done =
          (up && !uk) ? exact_select<true>(P, r, nT, row, V, xc_hi, xc_lo, xc, uk, up, cand_smem)
                      : exact_select<false>(P, r, nT, row, V, xc_hi, xc_lo, xc, uk, up, cand_smem);
      if (done) return;
      __syncthreads();  // the general path reuses the candidate area
    }
  }

  // pass A: maximum, first argmax, invalid entries, and (for a top-k cut)
  // each thread's four largest values
  PassA a;
  float c_hi = 0.f, c_lo = 0.f;
  double c = 0.0;
  if (temp_ok(temp) && temp > 0.f) temp_consts(temp, c_hi, c_lo, c);
  const bool any_filter = (P.top_k > 0 && P.top_k < V) || P.top_p < 1.0;
  if (P.top_k > 0 && P.top_k <= kSelThreads && P.top_k < V && temp > 0.f)
    a = pass_a<T, kAligned, true, false>(row, V, c_hi, c_lo);
  else if (!any_filter && temp > 0.f && temp_ok(temp))
    a = pass_a<T, kAligned, false, true>(row, V, c_hi, c_lo);  // the normaliser in the same scan
  else
    a = pass_a<T, kAligned, false, false>(row, V, c_hi, c_lo);
  const float mx = a.mx;
  const long am = a.am;
  const bool bad = a.bad;
  const unsigned t0 = fkey(a.t[0]), t1 = fkey(a.t[1]), t2 = fkey(a.t[2]), t3 = fkey(a.t[3]);
  s_tmax[threadIdx.x] = fkey(mx);
  const unsigned kmax = block_max_u<kSelThreads>(bad ? 0u : fkey(mx), smu);
  const bool any_bad = __syncthreads_or(bad);
  const float gmx = key_value(kmax);
  const int arg = block_min_i<kSelThreads>(mx == gmx ? static_cast<int>(am) : 0x7fffffff, smi);
  SampRow out{0.0, 0u, arg, 1, V, INFINITY, 0};
  if (!temp_ok(temp)) {
    out.valid = 0;
    out.kept = 0;
    if (threadIdx.x == 0) {
      put_row(P, r, nT, out);
      atomicOr(P.status, kStatTemperature);
    }
    return;
  }
  if (any_bad || gmx == -INFINITY) {
    out.valid = 0;
    out.kept = 0;
    if (threadIdx.x == 0) put_row(P, r, nT, out);
    return;
  }
  if (temp == 0.f) {  // greedy: the point mass on the first argmax
    out.theta = kmax;
    out.kept = 1;
    if (threadIdx.x == 0) put_row(P, r, nT, out);
    return;
  }
  if (!any_filter) {
    // no filter: the normaliser of the whole row from pass A
    const float O = key_value(block_max_u<kSelThreads>(a.o == -INFINITY ? 0u : fkey(a.o), smu));
    const double S = block_sum<kSelThreads>(
        a.o == -INFINITY ? 0.0 : static_cast<double>(a.s) * exp2(static_cast<double>(a.o) - O), smd);
    const double ninf = block_sum<kSelThreads>(static_cast<double>(a.ninf), smd);
    if (threadIdx.x == 0) {
      out.l2 = static_cast<double>(O) + log2(S);
      out.theta = 0u;
      out.kept = V - static_cast<int>(ninf);
      put_row(P, r, nT, out);
    }
    return;
  }
  const float o = gmx * c_hi;                       // fp32 weights 2^(x c - o)
  const double od = static_cast<double>(gmx) * c;   // fp64 weights 2^(x c - od)
  const bool use_k = P.top_k > 0 && P.top_k < V;
  const bool use_p = P.top_p < 1.0;

  // The candidate set in shared memory: every entry with key > `above` (and
  // >= theta), plus the group of entries equal to `above`, all of one weight.
  __shared__ StageOut s_st;
  unsigned theta = 0u;
  unsigned above = 0u;
  int nc = -1;  // candidates gathered (-1: none)
  double n_eq = 0.0, tail = 0.0;
  int eq = 0;
  if (use_k && P.top_k <= kSelThreads) {
    // The threads' four largest keys hold every entry >= their k-th largest
    // value theta4 when no thread's fourth key reaches theta4 (a thread with
    // more entries >= theta4 would have its fourth key >= theta4).  Then
    // theta4 is the row's k-th largest key and the lists are the candidates.
    cand_key[4 * threadIdx.x + 0] = t0;
    cand_key[4 * threadIdx.x + 1] = t1;
    cand_key[4 * threadIdx.x + 2] = t2;
    cand_key[4 * threadIdx.x + 3] = t3;
    __syncthreads();
    __shared__ unsigned s_t4;
    __shared__ int s_t4_ok;
    if (threadIdx.x < kWarp) {
      unsigned lo = 0u, hi = kmax, m3 = 0u;
      while (lo < hi) {
        const unsigned mid = lo + (((hi - lo) / step + 1) / 2) * step;
        int cnt = 0;
        for (int i = threadIdx.x; i < 4 * kSelThreads; i += kWarp) cnt += cand_key[i] >= mid;
        if (__reduce_add_sync(0xffffffffu, cnt) >= P.top_k) lo = mid;
        else hi = mid - step;
      }
      for (int i = threadIdx.x; i < kSelThreads; i += kWarp) m3 = max(m3, cand_key[4 * i + 3]);
      m3 = __reduce_max_sync(0xffffffffu, m3);
      if (threadIdx.x == 0) {
        s_t4 = lo;
        s_t4_ok = (m3 < lo) && lo > fkey(-INFINITY);  // empty places are -inf
      }
    }
    __syncthreads();
    if (s_t4_ok) {
      const unsigned t4 = s_t4;
      for (int i = threadIdx.x; i < 4 * kSelThreads; i += blockDim.x) {
        const unsigned k = cand_key[i];
        cand_w[i] = (k >= t4) ? static_cast<float>(exp2(static_cast<double>(key_value(k)) * c - od)) : 0.f;
      }
      __syncthreads();
      nc = 4 * kSelThreads;
      above = t4 - 1u;  // every entry >= t4 is in the lists
      theta = t4;
      n_eq = 0.0;
      tail = 0.0;
    }
  }
  if (use_k && P.top_k <= kSelThreads && nc < 0) {
    // a lower bound on the k-th largest: the k-th largest of the threads'
    // maxima (k distinct entries are at or above it); a short row is
    // gathered whole.  Warp 0 searches the kSelThreads maxima.
    __shared__ unsigned s_lb;
    if (threadIdx.x < kWarp) {
      unsigned lo = 0u, hi = (V > kCap) ? kmax : 0u;
      while (lo < hi) {
        const unsigned mid = lo + (((hi - lo) / step + 1) / 2) * step;
        int cnt = 0;
        for (int i = threadIdx.x; i < kSelThreads; i += kWarp) cnt += s_tmax[i] >= mid;
        if (__reduce_add_sync(0xffffffffu, cnt) >= P.top_k) lo = mid;
        else hi = mid - step;
      }
      if (threadIdx.x == 0) s_lb = lo;
    }
    __syncthreads();
    const unsigned lb = s_lb;
    const unsigned lb_floor = lb > 0u ? lb - 1u : 0u;  // gather keys >= lb
    const int n = gather<T, kAligned, false>(row, V, lb_floor, 0u, c, od, cand_key, cand_w, &cand_n,
                                             c_hi, c_lo, o, smd, &n_eq, &tail, kCap);
    if (n <= kCap) {
      nc = n;
      above = lb_floor;
      theta = lb;    // raised to the k-th largest candidate below
      n_eq = 0.0;    // the candidates hold every entry >= lb
      tail = 0.0;
    }
  }
  // Band histograms (when the candidate room holds them).  A top-k cut the
  // lists did not settle: every entry down to the band holding the k-th
  // largest is a candidate.  A nucleus cut alone: the candidates are the
  // bands around the cut, the masses above and below them from the histogram.
  __shared__ BandSide s_bs;
  if (threadIdx.x == 0) s_bs = BandSide{kmax, 0u, 0.0, 0.0};
  // (gs must be finite for the bands to follow the keys: an overflow there
  // means logits beyond 1e37, left to the fallbacks)
  if (use_k && nc < 0 && P.top_k <= kCap && kCap >= kBandCap && isfinite(gmx * kBandsPerUnit)) {
    const float sb = kBandsPerUnit;
    const float gs = gmx * sb;
    const BandCut bc = band_cut<T, kAligned, false>(row, V, sb, gs, c_hi, c_lo, o,
                                                   static_cast<double>(P.top_k), kmax, step,
                                                   cand_smem);
    if (bc.lo >= 0 && bc.end <= kCap) {
      double unused;
      const int n = gather_range<T, kAligned, false>(row, V, bc.k_lo, kmax + step, c, od,
                                                     cand_key, cand_w, &cand_n, smd, &unused, kCap);
      if (n > 0 && n <= kCap) {
        nc = n;
        above = bc.k_lo;  // the candidates hold every entry >= k_lo, at least k of them
        theta = bc.k_lo;
        n_eq = 0.0;
        tail = 0.0;
      }
    }
  }
  const float sb_p = fminf(kBandsPerUnit * c_hi, 1e30f);
  if (use_p && !use_k && nc < 0 && kCap >= kBandCap && isfinite(gmx * sb_p)) {
    const float sb = sb_p;
    const float gs = gmx * sb;
    const BandCut bc = band_cut<T, kAligned, true>(row, V, sb, gs, c_hi, c_lo, o, P.top_p, kmax,
                                                  step, cand_smem);
    if (bc.lo >= 0) {
      double nh = 0.0;
      const int n = gather_range<T, kAligned, true>(row, V, bc.k_lo, bc.k_head, c, od, cand_key,
                                                    cand_w, &cand_n, smd, &nh, kCap);
      if (n > 0 && n <= kCap) {
        // histogram masses are relative to o; the candidates' to od
        const double sc = exp2(static_cast<double>(o) - od);
        nc = n;
        above = bc.k_lo;   // entries below k_lo: the later bands (mass `tail`);
        n_eq = 0.0;        // entries from k_head on: the earlier bands (head)
        tail = bc.tail * sc;
        if (threadIdx.x == 0)
          s_bs = BandSide{bc.lo > 0 ? bc.k_head - step : kmax, bc.k_head, bc.head * sc, nh};
      }
    }
  }
  if (use_k && nc < 0) theta = radix_select<T, kAligned>(row, V, 0u, P.top_k, low_bits, hist, &eq);
  const bool k_in_cands = use_k && nc >= 0;

  if (use_p && nc < 0) {
    // candidate key: the kCap-th largest key >= theta (theta itself when
    // fewer entries are kept)
    unsigned vc = theta;
    double nd = V;  // without a top-k cut every entry is >= theta = 0
    if (theta > 0u) {
      int n_ge = 0;
      scan_row<T, kAligned, false>(row, V, [&](float x, long) { n_ge += fkey(x) >= theta; });
      nd = block_sum<kSelThreads>(static_cast<double>(n_ge), smd);
    }
    int eq_c = 0;
    if (nd > kCap) vc = radix_select<T, kAligned>(row, V, theta, kCap, low_bits, hist, &eq_c);
    nc = min(gather<T, kAligned, true>(row, V, vc, theta, c, od, cand_key, cand_w, &cand_n, c_hi,
                                       c_lo, o, smd, &n_eq, &tail, kCap),
             kCap);
    above = vc;
  }

  float margin = INFINITY;
  double Z_kept = -1.0;  // from the candidates when they hold the kept set
  double nk = -1.0;
  if (nc >= 0 && (k_in_cands || use_p)) {
    // (no entry equals `above` when every entry is a candidate: it may then
    // be a key that decodes to no finite value)
    const float xv = key_value(above);
    const double w_above = (n_eq > 0.0 && xv != -INFINITY) ? exp2(static_cast<double>(xv) * c - od) : 0.0;
    __syncthreads();
    CandSet cs{cand_key, cand_w, nc, above, n_eq, w_above, tail, s_bs.kmax, step, s_bs.head, s_bs.nhead};
    if (nc <= kWarpCands) {
      if (threadIdx.x < kWarp)
        cand_stage(Red<true>{smd}, cs, k_in_cands, P.top_k, use_p, P.top_p, theta, &s_st);
    } else {
      cand_stage(Red<false>{smd}, cs, k_in_cands, P.top_k, use_p, P.top_p, theta, &s_st);
    }
    __syncthreads();
    const StageOut st = s_st;
    theta = st.theta;
    if (st.below) {
      // the nucleus boundary lies outside the candidates: a mass descent over
      // the keys in [theta, v0), everything at or above v0 (mass m0) counted
      // (below), or over the keys above every candidate (above); fp32 weights
      // relative to o, the candidates' room holds the histograms
      const double sc = exp2(static_cast<double>(o) - od);
      const double Zk = st.Zk;
      const bool up = st.below == 2;
      const unsigned lo_key = up ? s_bs.hkmin : theta;
      const unsigned hi_key = up ? 0xffffffffu : max(theta, above);
      double m_ge, m_gt;
      const unsigned lo = mass_descent<T, kAligned>(
          row, V, lo_key, hi_key, up ? 0.0 : st.m0 / sc, st.goal / sc, low_bits, c_hi, c_lo, o,
          reinterpret_cast<float*>(cand_smem), &m_ge, &m_gt);
      m_ge *= sc;
      m_gt *= sc;
      margin = static_cast<float>(fmin(P.top_p - m_gt / Zk, m_ge / Zk - P.top_p));
      theta = max(lo, lo_key);  // (a goal missed by rounding keeps the whole range)
      Z_kept = m_ge;
    } else {
      margin = st.margin;
      if (st.z_valid) Z_kept = st.Z;
      if (st.kept_valid) nk = st.kept;
    }
  }

  // log-normaliser and size of the kept set, when the candidates do not hold it
  double Z = Z_kept;
  if (nk < 0.0) {
    float sf = 0.f;
    int kept = 0;
    scan_row<T, kAligned, false>(row, V, [&](float x, long) {
      if (fkey(x) >= theta && x != -INFINITY) {
        sf += ex2(specverify::arg2(x, c_hi, c_lo, o));
        ++kept;
      }
    });
    const double zs = block_sum<kSelThreads>(static_cast<double>(sf), smd) * exp2(static_cast<double>(o) - od);
    nk = block_sum<kSelThreads>(static_cast<double>(kept), smd);
    if (Z < 0.0) Z = zs;
  }
  if (threadIdx.x == 0) {
    // log2 sum 2^(x c): the double-precision candidate masses where they hold
    // the kept set, else the streaming pass
    out.l2 = od + log2(Z);
    out.theta = theta;
    out.kept = static_cast<int>(nk);
    out.margin = margin;
    put_row(P, r, nT, out);
  }
  (void)eq;
}

// ---------------------------------------------------------------------------
// kernel 2: acceptance test and first rejection
// ---------------------------------------------------------------------------

template <typename T>
__global__ void __launch_bounds__(kDecideThreads) decide_kernel(const SampParams P) {
  const int G = P.gamma, V = P.vocab;
  const int lane = threadIdx.x & (kWarp - 1);
  const int b = blockIdx.x * (kDecideThreads / kWarp) + (threadIdx.x >> 5);
  cudaGridDependencySynchronize();
  if (b >= P.batch) return;
  const long nT = static_cast<long>(P.batch) * (G + 1);
  const float temp = P.temperature[b];
  const bool greedy = temp == 0.f;
  float c_hi = 0.f, c_lo = 0.f;
  double c = 0.0;
  if (!greedy && temp_ok(temp)) temp_consts(temp, c_hi, c_lo, c);
  int n = G;
  unsigned bits = temp_ok(temp) ? 0u : kStatTemperature;
  for (int base = 0; base <= G; base += kWarp) {
    const int j = base + lane;
    bool tok_bad = false, row_bad = false, rej = false;
    if (j <= G) {
      const long position = static_cast<long>(b) * (G + 1) + j;
      const SampRow rt = P.rows[position];
      row_bad = !rt.valid;
      if (j < G) {
        const long pj = static_cast<long>(b) * G + j;
        const SampRow rd = P.rows[nT + pj];
        row_bad |= !rd.valid;
        const int t = P.tokens[pj];
        tok_bad = t < 0 || t >= V;
        if (!tok_bad && !row_bad) {
          const float xt = Elem<T>::load1(static_cast<const T*>(P.target) + position * V, t);
          const float xd = Elem<T>::load1(static_cast<const T*>(P.draft) + pj * V, t);
          const float u = P.u_accept[pj];
          double q, p;
          if (greedy) {
            q = (t == rt.argmax) ? 1.0 : 0.0;
            p = (t == rd.argmax) ? 1.0 : 0.0;
          } else {
            const bool kq = fkey(xt) >= rt.theta && xt != -INFINITY;
            const bool kp = fkey(xd) >= rd.theta && xd != -INFINITY;
            q = kq ? exp2(static_cast<double>(xt) * c - rt.l2) : 0.0;
            p = kp ? exp2(static_cast<double>(xd) * c - rd.l2) : 0.0;
          }
          double ratio;
          if (q == 0.0) ratio = 0.0;
          else if (p == 0.0) ratio = INFINITY;
          else if (greedy) ratio = 1.0;
          else ratio = exp2((static_cast<double>(xt) * c - rt.l2) -
                            (static_cast<double>(xd) * c - rd.l2));
          rej = !(static_cast<double>(u) < ratio);
          P.pos[pj] = specverify::PosInfo{q, p, ratio, rej ? 0 : 1, 0};
        }
      }
    }
    if (__ballot_sync(0xffffffffu, tok_bad)) bits |= kStatTokenRange;
    if (__ballot_sync(0xffffffffu, row_bad)) bits |= kStatNonFinite;
    const unsigned rm = __ballot_sync(0xffffffffu, j < G && rej);
    if (n == G && rm) n = base + __ffs(rm) - 1;
  }
  const long bo = static_cast<long>(b) * (G + 1);
  if (bits) {
    for (int q = lane; q <= G; q += kWarp) P.out_tokens[bo + q] = -1;
    if (lane == 0) {
      P.out_num_accepted[b] = 0;
      P.resid_mass[b] = NAN;
      P.decision[b] = SampDecision{0.0, 0.0, 0u, 0u, 0, kModeNone};
      atomicOr(P.status, bits);
    }
    return;
  }
  for (int q = lane; q <= G; q += kWarp) {
    if (q < n) P.out_tokens[bo + q] = P.tokens[static_cast<long>(b) * G + q];
    else if (q > n) P.out_tokens[bo + q] = -1;
  }
  if (lane == 0) {
    const SampRow rt = P.rows[bo + n];
    P.out_num_accepted[b] = n;
    if (greedy) {
      // the residual of two point masses, and the bonus draw, are the target's
      // point mass (a zero residual falls back to q_n): its argmax
      P.out_tokens[bo + n] = rt.argmax;
      if (n < G && P.rows[nT + static_cast<long>(b) * G + n].argmax == rt.argmax)
        atomicOr(P.status, kStatZeroMass);
      P.resid_mass[b] = 1.0;
      P.decision[b] = SampDecision{0.0, 0.0, 0u, 0u, n, kModeGreedy};
    } else {
      SampDecision d{rt.l2, 0.0, rt.theta, 0u, n, n < G ? kModeResidual : kModeTarget};
      if (n < G) {
        const SampRow rd = P.rows[nT + static_cast<long>(b) * G + n];
        d.lD = rd.l2;
        d.thD = rd.theta;
      }
      P.decision[b] = d;
    }
  }
}

// ---------------------------------------------------------------------------
// kernel 3: residual / bonus draw
// ---------------------------------------------------------------------------

// r_i of one element: q_i (target mode) or max(0, q_i - p_i), with the
// filters' masks; q and p from the logit difference as in the plain draw
__device__ __forceinline__ float resid_elem(float xt, float xd, int mode, const SampDecision& d,
                                            float c_hi, float c_lo, float lt_hi, float lt_lo,
                                            float k_hi, float k_lo) {
  if (!(fkey(xt) >= d.thT) || xt == -INFINITY) return 0.f;
  const float q = ex2(specverify::arg2l(xt, c_hi, c_lo, lt_hi, lt_lo));
  if (mode == kModeTarget) return q;
  if (!(fkey(xd) >= d.thD) || xd == -INFINITY) return q;
  const float dx = xt - xd;
  const float L = fmaf(dx, c_hi, -k_hi) + fmaf(dx, c_lo, -k_lo);
  const float p = q * ex2(-L);
  float t = specverify::kA5;
  t = fmaf(t, L, specverify::kA4);
  t = fmaf(t, L, specverify::kA3);
  t = fmaf(t, L, specverify::kA2);
  t = fmaf(t, L, specverify::kA1);
  const float small = p * (t * L);
  const float res = (L > 0.f && L < 0.125f) ? small : q - p;
  return fmaxf(res, 0.f);
}

constexpr int kDrawChunk = 8;    // consecutive elements per thread and tile
constexpr int kMaxTiles = 512;   // tiles per row (a tile grows for longer rows)

template <typename T>
__global__ void __launch_bounds__(kDrawThreads) draw_kernel(const SampParams P) {
  constexpr int kNW = kDrawThreads / kWarp;
  __shared__ float s_part[kMaxTiles][kNW];
  __shared__ double s_tile[kMaxTiles];
  __shared__ double smd[kNW];
  __shared__ int smi[kNW];
  __shared__ int s_k;
  __shared__ double s_before;
  const int G = P.gamma, V = P.vocab;
  const int b = blockIdx.x;
  const int lane = threadIdx.x & (kWarp - 1), warp = threadIdx.x >> 5;
  cudaGridDependencySynchronize();
  const SampDecision d = P.decision[b];
  if (d.mode == kModeNone || d.mode == kModeGreedy) return;
  const int n = d.n;
  const long bo = static_cast<long>(b) * (G + 1);
  const T* rowT = static_cast<const T*>(P.target) + (bo + n) * V;
  const T* rowD = static_cast<const T*>(P.draft) + (static_cast<long>(b) * G + n) * V;
  float c_hi, c_lo;
  double c;
  temp_consts(P.temperature[b], c_hi, c_lo, c);
  (void)c;
  float lt_hi, lt_lo, k_hi, k_lo;
  specverify::split2(d.lT, lt_hi, lt_lo);
  specverify::split2(d.lT - d.lD, k_hi, k_lo);

  // a thread's chunk: L consecutive elements; a tile: kDrawThreads chunks
  const long per_tile_min = static_cast<long>(kDrawThreads) * kDrawChunk;
  const long tiles_min = (V + per_tile_min - 1) / per_tile_min;
  const int m = static_cast<int>((tiles_min + kMaxTiles - 1) / kMaxTiles);
  const int L = kDrawChunk * m;
  const long E = static_cast<long>(kDrawThreads) * L;
  const int ntiles = static_cast<int>((V + E - 1) / E);
  int mode = d.mode;

  auto chunk_sum = [&](int tile, int md, int* last) -> float {
    const long i0 = static_cast<long>(tile) * E + static_cast<long>(threadIdx.x) * L;
    float s = 0.f;
    for (int e = 0; e < L; ++e) {
      const long i = i0 + e;
      if (i >= V) break;
      const float xt = elem<T>(rowT, i);
      const float xd = (md == kModeResidual) ? elem<T>(rowD, i) : 0.f;
      const float rv = resid_elem(xt, xd, md, d, c_hi, c_lo, lt_hi, lt_lo, k_hi, k_lo);
      s += rv;
      if (rv > 0.f) *last = static_cast<int>(i);
    }
    return s;
  };

  // 16-byte aligned rows with one chunk of kDrawChunk elements per thread
  // and tile: the chunks are read as kQ 16-byte loads per row, four tiles'
  // loads in flight together (the same elements, sums and order as
  // chunk_sum)
  constexpr int kVec = specverify::Elem<T>::kVec;
  constexpr int kQ = kDrawChunk / kVec;  // 16-byte loads per row and chunk
  constexpr int kTB = 4;                 // tiles whose loads are in flight together
  const bool vec = L == kDrawChunk && (static_cast<long>(V) * sizeof(T)) % 16 == 0 &&
                   reinterpret_cast<uintptr_t>(rowT) % 16 == 0 &&
                   (G == 0 || reinterpret_cast<uintptr_t>(rowD) % 16 == 0);
  auto load_chunk = [&](int tile, int md, uint4 (&vt)[kQ], uint4 (&vd)[kQ]) {
    const long i0 = static_cast<long>(tile) * E + static_cast<long>(threadIdx.x) * L;
#pragma unroll
    for (int q = 0; q < kQ; ++q) {
      const long i = i0 + q * kVec;
      if (i < V) {  // V is a multiple of kVec here: the group is whole
        vt[q] = __ldg(reinterpret_cast<const uint4*>(rowT + i));
        if (md == kModeResidual) vd[q] = __ldg(reinterpret_cast<const uint4*>(rowD + i));
      }
    }
  };
  auto chunk_sum_vec = [&](int tile, int md, const uint4 (&vt)[kQ], const uint4 (&vd)[kQ],
                           int* last) -> float {
    const long i0 = static_cast<long>(tile) * E + static_cast<long>(threadIdx.x) * L;
    float s = 0.f;
#pragma unroll
    for (int q = 0; q < kQ; ++q) {
      if (i0 + q * kVec >= V) break;
      float xt[kVec], xd[kVec];
      specverify::Elem<T>::unpack(vt[q], xt);
      if (md == kModeResidual) specverify::Elem<T>::unpack(vd[q], xd);
#pragma unroll
      for (int e = 0; e < kVec; ++e) {
        const float rv = resid_elem(xt[e], md == kModeResidual ? xd[e] : 0.f, md, d, c_hi, c_lo,
                                    lt_hi, lt_lo, k_hi, k_lo);
        s += rv;
        if (rv > 0.f) *last = static_cast<int>(i0 + q * kVec + e);
      }
    }
    return s;
  };

  // pass 1: the mass of every tile (warp partials, no barrier in the loop)
  double Z = 0.0;
  int last_pos = -1;
  for (int attempt = 0; attempt < 2; ++attempt) {
    int lp = -1;
    if (vec) {
      for (int t0 = 0; t0 < ntiles; t0 += kTB) {
        uint4 vt[kTB][kQ], vd[kTB][kQ];
#pragma unroll
        for (int j = 0; j < kTB; ++j)
          if (t0 + j < ntiles) load_chunk(t0 + j, mode, vt[j], vd[j]);
#pragma unroll
        for (int j = 0; j < kTB; ++j) {
          if (t0 + j >= ntiles) break;
          float s = chunk_sum_vec(t0 + j, mode, vt[j], vd[j], &lp);
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
          if (lane == 0) s_part[t0 + j][warp] = s;
        }
      }
    } else {
      for (int t = 0; t < ntiles; ++t) {
        float s = chunk_sum(t, mode, &lp);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
        if (lane == 0) s_part[t][warp] = s;
      }
    }
    __syncthreads();
    double zt = 0.0;
    for (int t = threadIdx.x; t < ntiles; t += blockDim.x) {
      double tm = 0.0;
      for (int w = 0; w < kNW; ++w) tm += static_cast<double>(s_part[t][w]);
      s_tile[t] = tm;
      zt += tm;
    }
    Z = block_sum<kDrawThreads>(zt, smd);
    last_pos = block_max_i<kDrawThreads>(lp, smi);
    if (Z > 0.0 || mode == kModeTarget) break;
    // a residual without mass (q and p agree up to rounding): draw from q_n
    mode = kModeTarget;
    if (threadIdx.x == 0) atomicOr(P.status, kStatZeroMass);
    __syncthreads();
  }
  const double goal = static_cast<double>(P.u_resample[b]) * Z;

  // the tile holding the goal, by a walk over the tile masses
  if (threadIdx.x == 0) {
    double before = 0.0;
    int k = -1;
    for (int t = 0; t < ntiles; ++t) {
      if (before + s_tile[t] > goal) {
        k = t;
        break;
      }
      before += s_tile[t];
    }
    s_k = k;
    s_before = before;
  }
  __syncthreads();
  const int k = s_k;
  int found = 0x7fffffff;
  if (k >= 0) {
    // inside the tile: a block scan over the chunks, then the chunk's elements
    int dummy = -1;
    const float cs = chunk_sum(k, mode, &dummy);
    double incl, excl, total;
    specverify::block_scan<kDrawThreads>(static_cast<double>(cs), incl, excl, total);
    const double before = s_before;
    if (cs > 0.f && before + excl <= goal && before + incl > goal) {
      const long i0 = static_cast<long>(k) * E + static_cast<long>(threadIdx.x) * L;
      double cum = before + excl;
      for (int e = 0; e < L; ++e) {
        const long i = i0 + e;
        if (i >= V) break;
        const float xt = elem<T>(rowT, i);
        const float xd = (mode == kModeResidual) ? elem<T>(rowD, i) : 0.f;
        const float rv = resid_elem(xt, xd, mode, d, c_hi, c_lo, lt_hi, lt_lo, k_hi, k_lo);
        cum += rv;
        if (rv > 0.f && cum > goal) {
          found = static_cast<int>(i);
          break;
        }
      }
    }
  }
  found = block_min_i<kDrawThreads>(found, smi);
  if (threadIdx.x == 0) {
    P.out_tokens[bo + n] = (found != 0x7fffffff) ? found : last_pos;
    P.resid_mass[b] = Z;
  }
}

}  // namespace specsamp
