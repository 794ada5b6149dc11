// Speculative-sampling verification kernels for sm_100a.
//
// One verification step is three stream-ordered kernels (each later one
// launched early through programmatic dependent launch and waiting for its
// predecessor with a grid-dependency barrier):
//
//   stats   S blocks per logit row (every target row, then every draft
//           row), each streaming its contiguous 1/S of the row with 128-bit
//           coalesced loads, eight in flight per thread; each thread keeps a
//           running sum of 2^(x c - o) against a lazily raised offset o; the
//           block writes its (o, sum) partial (step 1 of the round: softmax
//           statistics).  No atomics, no waits, the same work in every block:
//           this is the kernel that moves all of the logit bytes.
//   decide  one warp per sequence, one lane per position: the lane combines
//           the position's partials into log2 sum_i 2^(x_i c), forms q(t),
//           p(t) and the ratio, and a warp ballot finds the first rejection n
//           (steps 2 and 3); writes the accepted prefix and what to draw from.
//   draw    the grid's warps split every tile of every sequence's rows drawn
//           from (n < gamma: max(0, q_n - p_n) from target and draft row n;
//           n == gamma: q of target row gamma) into even contiguous runs,
//           write each tile's mass, and the warp that completes a sequence's
//           tiles (an atomic ticket) locates u * Z by a warp scan over the
//           tile masses and one re-read tile (step 4).
//
// No thread ever waits for another block (the only hand-off inside a kernel
// is an atomic ticket, never a spin).
//
// Pages (title, section): "Speculative decoding - the small model writes first
// and the big model checks", section 1 (rule); "Speculative decoding: how to
// run big models fast", section "How it works" (steps, bonus token, 1..gamma+1
// tokens per call, temperature).
//
// Numerics.  c = log2(e)/T is carried as two floats c_hi + c_lo (c_lo > 0).
// Every exponent argument is x c_hi - o + x c_lo, two FMAs whose only
// rounding is relative to the (small) result, so no rounding of c or of a
// large offset ever becomes a systematic factor on the probabilities.  The
// offset o of a thread is any float near its largest x c seen so far; it is
// raised only when a group's sum leaves [0, 2^100), so the streaming loop has
// no max pass.  Per-thread sums are fp32; everything above a thread (warp,
// block, position, ratio, CDF positions) is fp64.  In the residual q - p is
// formed as p (2^L - 1) with L = log2(q/p) taken from the logit difference,
// which keeps it accurate where q and p nearly cancel.  Data errors set bits
// of a status word; nothing traps.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cfloat>
#include <cstdint>

namespace specverify {

constexpr int kWarp = 32;
constexpr int kMaxSlices = 64;

// per-position decision flags
enum : int { kFlagReject = 0, kFlagAccept = 1, kFlagTokenRange = 2, kFlagNonFinite = 3 };
// status word bits
// (16 is the sampling variants' temperature bit; 32: a bounded wait of the
// single-launch step gave up; 64: a bounds check of a debug build failed)
enum : unsigned {
  kStatTokenRange = 1u,
  kStatNonFinite = 2u,
  kStatZeroMass = 4u,
  kStatRowIndex = 8u,
  kStatWait = 32u,
  kStatBounds = 64u
};

// Debug builds (compiled with -DSV_DEBUG_BOUNDS=1) check the indices that
// the kernels derive from launch geometry and from decisions before they
// touch the workspace or the outputs: a failed check sets kStatBounds in the
// status word and the access is skipped (nothing traps).  In normal builds
// every check is the constant true.
#ifndef SV_DEBUG_BOUNDS
#define SV_DEBUG_BOUNDS 0
#endif
__device__ __forceinline__ bool bounds_ok(long i, long n, unsigned* status) {
#if SV_DEBUG_BOUNDS
  if (i >= 0 && i < n) return true;
  atomicOr(status, kStatBounds);
  return false;
#else
  (void)i;
  (void)n;
  (void)status;
  return true;
#endif
}
// what the draw kernel draws from
enum : int { kDrawResidual = 0, kDrawTarget = 1, kDrawNone = 2 };

struct RowStat {
  double lse2;  // log2 sum_i 2^(x_i c) = log2 sum_i exp(x_i / T) / ln 2
  int valid;    // 1 if the row is finite with at least one finite entry
  int pad;
};

struct PosInfo {
  double q_tok;
  double p_tok;
  double ratio;
  int flag;
  int pad;
};

// one block's partial statistics of its slice of one row: sum_i 2^(x_i c - o)
// against the offset o
struct __align__(16) RowPartial {
  double s;
  float o;
  int pad;
};

// per sequence, from the decide kernel to the draw kernel
struct SeqDecision {
  double lT, lD;       // log2 sum 2^(x c) of the rows drawn from
  long trow, drow;     // the rows drawn from, as rows of the logit buffers
  int n;               // accepted drafts
  int mode;            // kDraw*
  unsigned stat_bits;  // data errors found
  // the draw's float constants (see DrawConsts), formed once in fp64
  float lt_hi, k_hi, k_lo, fT;
};

struct Params {
  const void* target;        // [target_rows, V] logit rows ([B, G+1, V] when unmapped)
  const void* draft;         // [draft_rows, V] logit rows ([B, G, V] when unmapped)
  const int32_t* target_map; // [B, G+1] row of `target` of each position, or null (identity)
  const int32_t* draft_map;  // [B, G] row of `draft` of each draft position, or null
  long target_rows, draft_rows;
  const int32_t* tokens;     // [B, G]
  const float* u_accept;     // [B, G]
  const float* u_resample;   // [B]
  int32_t* out_tokens;       // [B, G+1]
  int32_t* out_num_accepted; // [B]
  RowPartial* partial;       // [(target_rows + draft_rows) * S]: target rows, then draft rows
  RowStat* tstat;            // [B*(G+1)]
  RowStat* dstat;            // [B*G]
  PosInfo* pos;              // [B*G]
  SeqDecision* decision;     // [B]
  double* draw_mass;         // [B * tiles of a row] mass of each 32-group tile of the draw
  unsigned* draw_ticket;     // [B], zero between launches
  double* resid_mass;        // [B]
  unsigned* status;          // [1]
  int batch, gamma, vocab;
  int slices;                // S stats blocks per position
  int groups_per_slice;      // 16-byte groups of the vocabulary per stats block
  long draw_tiles;           // tiles of kTile groups per row drawn from
  float c_hi, c_lo;          // log2(e)/T = c_hi + c_lo, c_lo > 0
  double c;                  // c_hi + c_lo, exactly
  // fused LM-head form: the logits at the draft tokens were picked out by the
  // GEMM ([target_rows] and [draft_rows] floats; null: read the logit rows),
  // and the draw reads row b of compact [B, V] logit buffers
  const float* gathered_target;
  const float* gathered_draft;
  int draw_compact;
  // tapered slicing of the statistics grid: the first taper_rows rows are
  // cut into taper_slices slices of taper_groups groups each, the remaining
  // rows into `slices` slices of groups_per_slice groups, so that the blocks
  // dispatched last are short and the grid's last wave ends together.  The
  // partial table keeps `slices` entries per row; a tapered row fills its
  // entries past taper_slices with empty partials.  taper_rows 0: every row
  // alike.
  long taper_rows;
  int taper_slices, taper_groups;
};

// ---------------------------------------------------------------------------
// element access: a "group" is 16 bytes of one row (8 bf16 or 4 fp32)
// ---------------------------------------------------------------------------

template <typename T>
struct Elem;

template <>
struct Elem<float> {
  static constexpr int kVec = 4;
  static __device__ __forceinline__ float load1(const float* row, long i) { return __ldg(row + i); }
  static __device__ __forceinline__ void unpack(const uint4& v, float (&x)[4]) {
    x[0] = __uint_as_float(v.x);
    x[1] = __uint_as_float(v.y);
    x[2] = __uint_as_float(v.z);
    x[3] = __uint_as_float(v.w);
  }
  // scalar path: pack up to 4 in-range values, -inf beyond the row end
  static __device__ __forceinline__ uint4 fetch_scalar(const float* row, long g, int V) {
    const unsigned ninf = 0xff800000u;
    long i = g * 4;
    uint4 v;
    v.x = (i + 0 < V) ? __float_as_uint(__ldg(row + i + 0)) : ninf;
    v.y = (i + 1 < V) ? __float_as_uint(__ldg(row + i + 1)) : ninf;
    v.z = (i + 2 < V) ? __float_as_uint(__ldg(row + i + 2)) : ninf;
    v.w = (i + 3 < V) ? __float_as_uint(__ldg(row + i + 3)) : ninf;
    return v;
  }
};

template <>
struct Elem<__nv_bfloat16> {
  static constexpr int kVec = 8;
  static __device__ __forceinline__ float load1(const __nv_bfloat16* row, long i) {
    unsigned short bits = __ldg(reinterpret_cast<const unsigned short*>(row) + i);
    return __uint_as_float(static_cast<unsigned>(bits) << 16);
  }
  // bf16 is the upper half of a binary32 word: widening is a shift / mask
  static __device__ __forceinline__ void unpack(const uint4& v, float (&x)[8]) {
    x[0] = __uint_as_float(v.x << 16);
    x[1] = __uint_as_float(v.x & 0xffff0000u);
    x[2] = __uint_as_float(v.y << 16);
    x[3] = __uint_as_float(v.y & 0xffff0000u);
    x[4] = __uint_as_float(v.z << 16);
    x[5] = __uint_as_float(v.z & 0xffff0000u);
    x[6] = __uint_as_float(v.w << 16);
    x[7] = __uint_as_float(v.w & 0xffff0000u);
  }
  static __device__ __forceinline__ uint4 fetch_scalar(const __nv_bfloat16* row, long g, int V) {
    const unsigned short* r = reinterpret_cast<const unsigned short*>(row);
    const unsigned ninf = 0xff80u;
    long i = g * 8;
    unsigned w[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) w[k] = (i + k < V) ? static_cast<unsigned>(__ldg(r + i + k)) : ninf;
    return make_uint4(w[0] | (w[1] << 16), w[2] | (w[3] << 16), w[4] | (w[5] << 16),
                      w[6] | (w[7] << 16));
  }
};

// streaming 128-bit load: read-only path, no L1 allocation
__device__ __forceinline__ uint4 ld_stream(const uint4* p) {
  uint4 v;
  asm("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
      : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
      : "l"(p));
  return v;
}

template <typename T, bool kAligned>
__device__ __forceinline__ uint4 fetch_group(const T* row, long g, int V) {
  if constexpr (kAligned) {
    return ld_stream(reinterpret_cast<const uint4*>(row) + g);
  } else {
    return Elem<T>::fetch_scalar(row, g, V);
  }
}

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// x c - o with c = c_hi + c_lo: two FMAs; x = -inf gives -inf (c_lo > 0, so
// never inf * 0), and the rounding is relative to the result only
__device__ __forceinline__ float arg2(float x, float c_hi, float c_lo, float o) {
  return fmaf(x, c_lo, fmaf(x, c_hi, -o));
}

// x c - (l_hi + l_lo), for an offset known to double precision
__device__ __forceinline__ float arg2l(float x, float c_hi, float c_lo, float l_hi, float l_lo) {
  return fmaf(x, c_hi, -l_hi) + fmaf(x, c_lo, -l_lo);
}

// ---------------------------------------------------------------------------
// phase 1: streaming softmax statistics
// ---------------------------------------------------------------------------

constexpr float kGroupSumLimit = 1.2676506e30f;  // 2^100

// Adds one group to (o, s): s = sum 2^(x c - o).  The fast path is two FMAs,
// one ex2 and one add per element; the offset is raised (and the group
// recomputed) only when the group's sum is not in [0, 2^100): the first
// group (o = -inf), a much larger logit, +inf or NaN.
template <typename T>
__device__ __forceinline__ void accumulate_group(const uint4& v, float& o, float& s, float c_hi,
                                                 float c_lo) {
  constexpr int kVec = Elem<T>::kVec;
  float x[kVec];
  Elem<T>::unpack(v, x);
  float sg = 0.f;
#pragma unroll
  for (int k = 0; k < kVec; ++k) sg += ex2(arg2(x[k], c_hi, c_lo, o));
  if (!(sg < kGroupSumLimit)) {
    float gm = -INFINITY;
    bool nan = false;
#pragma unroll
    for (int k = 0; k < kVec; ++k) {
      gm = fmaxf(gm, x[k]);
      nan |= (x[k] != x[k]);
    }
    if (nan || gm == INFINITY) {
      sg = NAN;  // the row is invalid; the NaN marks it through every sum
    } else if (gm == -INFINITY) {
      sg = 0.f;  // the group has no mass
    } else {
      const float on = gm * c_hi;
      if (on > o) {
        s *= ex2(o - on);  // o = -inf: s is 0 (or NaN) and stays so
        o = on;
      }
      sg = 0.f;
#pragma unroll
      for (int k = 0; k < kVec; ++k) sg += ex2(arg2(x[k], c_hi, c_lo, o));
    }
  }
  s += sg;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

__device__ __forceinline__ double warp_sum(double v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ int warp_maxi(int v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = max(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// contiguous group range [lo, hi) of warp `w` inside the range [clo, chi)
__device__ __forceinline__ void warp_range(long clo, long chi, int w, int nwarps, long& lo,
                                           long& hi) {
  long n = chi - clo;
  long per = (n + nwarps - 1) / nwarps;
  lo = clo + per * w;
  hi = lo + per;
  if (lo > chi) lo = chi;
  if (hi > chi) hi = chi;
}

// ---------------------------------------------------------------------------
// phase 4 helpers: residual mass of one group
// ---------------------------------------------------------------------------

struct DrawConsts {
  float c_hi, c_lo;
  float lt_hi;   // log2 sum 2^(x c) of the target row, rounded to float
  float k_hi, k_lo;  // K = lT - lD, two-float
  float fT;      // 2^(-lt_lo): applied to every sum of group masses
};

// Taylor coefficients of 2^L - 1 = sum_k (ln 2)^k L^k / k!, k = 1..5
constexpr float kA1 = 0.6931471805599453f;
constexpr float kA2 = 0.2402265069591007f;
constexpr float kA3 = 0.055504108664821576f;
constexpr float kA4 = 0.009618129107628477f;
constexpr float kA5 = 0.0013333558146428441f;

__device__ __forceinline__ void split2(double v, float& hi, float& lo) {
  hi = static_cast<float>(v);
  lo = static_cast<float>(v - static_cast<double>(hi));
}

// ---------------------------------------------------------------------------
// block-level helpers
// ---------------------------------------------------------------------------

// Streaming statistics of one block's slice [glo, ghi) of one row, reduced to
// the block (offset = the block's largest thread offset); valid in thread 0.
template <typename T, int NT, bool kAligned, int kUnroll>
__device__ __forceinline__ RowPartial slice_stats(const T* row, long glo, long ghi, int V,
                                                  float c_hi, float c_lo) {
  constexpr int kNW = NT / kWarp;
  __shared__ float sm_off[kNW];
  __shared__ double sm_sum[kNW];
  const int tid = threadIdx.x, lane = tid & (kWarp - 1), warp = tid >> 5;

  float o = -INFINITY, s = 0.f;
  // consecutive threads read consecutive 16-byte groups: each warp-wide load
  // is 512 contiguous bytes; kUnroll groups are in flight per thread
  long g0 = glo + tid;
  for (; g0 + static_cast<long>(NT) * (kUnroll - 1) < ghi; g0 += static_cast<long>(NT) * kUnroll) {
    uint4 v[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) v[u] = fetch_group<T, kAligned>(row, g0 + static_cast<long>(u) * NT, V);
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) accumulate_group<T>(v[u], o, s, c_hi, c_lo);
  }
  if (g0 < ghi) {
    // the last, partial round: all of its loads in flight together
    uint4 v[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const long g = g0 + static_cast<long>(u) * NT;
      if (g < ghi) v[u] = fetch_group<T, kAligned>(row, g, V);
    }
#pragma unroll
    for (int u = 0; u < kUnroll; ++u)
      if (g0 + static_cast<long>(u) * NT < ghi) accumulate_group<T>(v[u], o, s, c_hi, c_lo);
  }

  // the block's offset is its largest thread offset; each thread rescales
  const float wo = warp_max(o);
  if (lane == 0) sm_off[warp] = wo;
  __syncthreads();
  float O = sm_off[0];
#pragma unroll
  for (int w = 1; w < kNW; ++w) O = fmaxf(O, sm_off[w]);
  // a thread with o = -inf holds s = 0 (or NaN, which must propagate)
  const float f = (o == -INFINITY) ? 0.f : ex2(o - O);
  const double z = warp_sum(static_cast<double>(s) * static_cast<double>(f));
  if (lane == 0) sm_sum[warp] = z;
  __syncthreads();
  RowPartial out{0.0, O, 0};
  if (tid == 0) {
    for (int w = 0; w < kNW; ++w) out.s += sm_sum[w];
  }
  return out;
}

// (o, s) pairs combined: O = max o, S = sum s 2^(o - O)
__device__ __forceinline__ void combine_into(float& O, double& S, float o, double s) {
  if (o == -INFINITY) {
    S += s * 0.0;  // keeps a NaN partial visible
    return;
  }
  if (o > O) {
    S = (O == -INFINITY) ? S : S * exp2(static_cast<double>(O) - o);
    O = o;
  }
  S += s * exp2(static_cast<double>(o) - O);
}

// block-wide scan of one double per thread: inclusive, exclusive, total
template <int NT>
__device__ __forceinline__ void block_scan(double v, double& incl, double& excl, double& total) {
  constexpr int kNW = NT / kWarp;
  __shared__ double sm_w[kNW];
  const int tid = threadIdx.x, lane = tid & (kWarp - 1), warp = tid >> 5;
  double x = v;
#pragma unroll
  for (int o = 1; o < kWarp; o <<= 1) {
    const double y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  const double prev = __shfl_up_sync(0xffffffffu, x, 1);
  if (lane == kWarp - 1) sm_w[warp] = x;
  __syncthreads();
  double wpre = 0.0;
  total = 0.0;
  for (int w = 0; w < kNW; ++w) {
    if (w < warp) wpre += sm_w[w];
    total += sm_w[w];
  }
  __syncthreads();  // sm_w is reused by the next call
  incl = wpre + x;
  excl = (lane == 0) ? wpre : wpre + prev;
  (void)tid;
}

// ---------------------------------------------------------------------------
// steps 2 and 3: the decision of one sequence (one warp, one lane per position)
// ---------------------------------------------------------------------------

constexpr int kDecideThreads = 128;
constexpr int kMaxGamma = 255;

// (o, s) partials of one row combined in two passes, so that the fp64
// exponentials of the second pass are independent of one another.  kCg: the
// partials were written by other warps of the same launch, so they are read
// through L2 (ld.global.cg), never from a possibly stale L1 line.
template <bool kCg>
__device__ __forceinline__ double row_lse2(const RowPartial* parts, int S, int& valid) {
  if (S <= 8) {
    // every partial's 16-byte record loaded at once (one memory round trip);
    // then the same two passes, in the same order, as the general loop
    float o[8];
    double s[8];
#pragma unroll
    for (int r = 0; r < 8; ++r) {
      if (r < S) {
        const uint4 v = kCg ? __ldcg(reinterpret_cast<const uint4*>(parts) + r)
                            : *(reinterpret_cast<const uint4*>(parts) + r);
        s[r] = __hiloint2double(static_cast<int>(v.y), static_cast<int>(v.x));
        o[r] = __uint_as_float(v.z);
      }
    }
    float O = -INFINITY;
#pragma unroll
    for (int r = 0; r < 8; ++r)
      if (r < S) O = fmaxf(O, o[r]);
    double sum = 0.0;
#pragma unroll
    for (int r = 0; r < 8; ++r)
      if (r < S) sum += (o[r] == -INFINITY) ? s[r] * 0.0 : s[r] * exp2(static_cast<double>(o[r]) - O);
    valid = (O != -INFINITY) && isfinite(sum) && sum > 0.0;
    return static_cast<double>(O) + log2(sum);
  }
  float O = -INFINITY;
  for (int r = 0; r < S; ++r) O = fmaxf(O, kCg ? __ldcg(&parts[r].o) : parts[r].o);
  double sum = 0.0;
  for (int r = 0; r < S; ++r) {
    const float o = kCg ? __ldcg(&parts[r].o) : parts[r].o;
    const double s = kCg ? __ldcg(&parts[r].s) : parts[r].s;
    sum += (o == -INFINITY) ? s * 0.0 : s * exp2(static_cast<double>(o) - O);  // NaN survives
  }
  valid = (O != -INFINITY) && isfinite(sum) && sum > 0.0;
  return static_cast<double>(O) + log2(sum);  // log2 sum_i 2^(x_i c)
}

// What lane j of a deciding warp reads from the caller's buffers for position
// j of sequence b (j <= gamma): its rows, the drafted token, its uniform and
// the two logits at the token.  None of it comes from this library's kernels,
// so a programmatic dependent may load it before its grid-dependency wait.
struct LaneInputs {
  long tr, dr;  // rows of the logit buffers that hold the position
  int t;        // drafted token
  float u, xt, xd;
  bool tok_bad, map_bad;
};

template <typename T>
__device__ __forceinline__ LaneInputs lane_inputs(const Params& P, int b, int j) {
  const int G = P.gamma, V = P.vocab;
  LaneInputs in{0, 0, 0, 0.f, 0.f, 0.f, false, false};
  if (j > G) return in;
  const long position = static_cast<long>(b) * (G + 1) + j;
  const long pj = static_cast<long>(b) * G + j;
  const bool has_draft = j < G;
  in.tr = P.target_map ? static_cast<long>(P.target_map[position]) : position;
  in.dr = has_draft ? (P.draft_map ? static_cast<long>(P.draft_map[pj]) : pj) : 0;
  in.map_bad = in.tr < 0 || in.tr >= P.target_rows ||
               (has_draft && (in.dr < 0 || in.dr >= P.draft_rows));
  if (has_draft) {
    in.t = P.tokens[pj];
    in.u = P.u_accept[pj];
    in.tok_bad = (in.t < 0 || in.t >= V);
    if (!in.tok_bad && !in.map_bad) {
      in.xt = P.gathered_target ? P.gathered_target[in.tr]
                                : Elem<T>::load1(static_cast<const T*>(P.target) + in.tr * V, in.t);
      in.xd = P.gathered_draft ? P.gathered_draft[in.dr]
                               : Elem<T>::load1(static_cast<const T*>(P.draft) + in.dr * V, in.t);
    }
  }
  return in;
}

// The decision of sequence b by the calling warp (all 32 lanes): lane j
// combines the partials of position j's rows, forms q(t), p(t) and the ratio
// in fp64 and tests u < ratio (step 2); a warp ballot finds the first
// rejection n (step 3).  Returns what the draw draws from (in every lane).
// write: also writes the accepted prefix, the padding, the count, the
// per-position readback records, the status bits and the decision record
// (exactly one warp per sequence writes; others only use the result).
// kCg: the partials come from other warps of the same launch (see row_lse2).
// staged (unmapped rows only): the sequence's partials were copied to shared
// memory, its gamma+1 target rows then its gamma draft rows, S per row.
// pre (may be null): this lane's lane_inputs for positions 0 .. 31, loaded
// earlier.
template <typename T, bool kCg = false>
__device__ __forceinline__ SeqDecision decide_sequence(const Params& P, int b,
                                                       const RowPartial* staged = nullptr,
                                                       bool write = true,
                                                       const LaneInputs* pre = nullptr) {
  const int lane = threadIdx.x & (kWarp - 1);
  const int G = P.gamma, S = P.slices;
  const double c = P.c;
  int n = G;          // first rejection, gamma if none
  unsigned bits = 0;  // data errors of the sequence
  double lT_n = 0.0, lD_n = 0.0;
  long tr_n = 0, dr_n = 0;
  for (int base = 0; base <= G; base += kWarp) {
    const int j = base + lane;
    int flag = kFlagAccept;
    bool tok_bad = false, row_bad = false, map_bad = false;
    double lT = 0.0, lD = 0.0;
    long tr = 0, dr = 0;
    if (j <= G) {
      const long position = static_cast<long>(b) * (G + 1) + j;
      const long pj = static_cast<long>(b) * G + j;
      const bool has_draft = j < G;
      // the acceptance test's inputs first: their loads overlap the combine
      const LaneInputs in = (pre && base == 0) ? *pre : lane_inputs<T>(P, b, j);
      tr = in.tr;
      dr = in.dr;
      map_bad = in.map_bad;
      tok_bad = in.tok_bad;
      const float u = in.u, xt = in.xt, xd = in.xd;
      int validT = 0, validD = 1;
      if (!map_bad) {
        if (staged) {
          lT = row_lse2<false>(staged + static_cast<long>(j) * S, S, validT);
          if (has_draft) lD = row_lse2<false>(staged + static_cast<long>(G + 1 + j) * S, S, validD);
        } else {
          lT = row_lse2<kCg>(P.partial + tr * S, S, validT);
          if (has_draft) lD = row_lse2<kCg>(P.partial + (P.target_rows + dr) * S, S, validD);
        }
      }
      if (write) {
        P.tstat[position] = RowStat{lT, validT, 0};
        if (has_draft) P.dstat[pj] = RowStat{lD, validD, 0};
      }
      row_bad = !map_bad && (!validT || !validD);
      if (has_draft) {
        PosInfo info{0.0, 0.0, 0.0, kFlagReject, 0};
        if (tok_bad) {
          info.flag = kFlagTokenRange;
        } else if (row_bad || map_bad) {
          info.flag = kFlagNonFinite;
        } else {
          const double lq = static_cast<double>(xt) * c - lT;  // log2 q(t)
          const double lp = static_cast<double>(xd) * c - lD;  // log2 p(t)
          info.q_tok = exp2(lq);
          info.p_tok = exp2(lp);
          if (!(info.q_tok > 0.0)) info.ratio = 0.0;
          else if (!(info.p_tok > 0.0)) info.ratio = INFINITY;
          else info.ratio = exp2(lq - lp);
          info.flag = (static_cast<double>(u) < info.ratio) ? kFlagAccept : kFlagReject;
        }
        if (write) P.pos[pj] = info;
        flag = info.flag;
      }
    }
    const unsigned rej = __ballot_sync(0xffffffffu, j < G && flag == kFlagReject);
    if (__ballot_sync(0xffffffffu, tok_bad)) bits |= kStatTokenRange;
    if (__ballot_sync(0xffffffffu, row_bad)) bits |= kStatNonFinite;
    if (__ballot_sync(0xffffffffu, map_bad)) bits |= kStatRowIndex;
    // the statistics the draw needs live in lane (n - base) of this chunk
    const int first = rej ? base + __ffs(rej) - 1 : G;
    const bool here = (n == G) && (first < G || G < base + kWarp);
    if (n == G) n = first;
    const int src = (n - base) & (kWarp - 1);
    const double lTs = __shfl_sync(0xffffffffu, lT, src);
    const double lDs = __shfl_sync(0xffffffffu, lD, src);
    const long trs = __shfl_sync(0xffffffffu, tr, src);
    const long drs = __shfl_sync(0xffffffffu, dr, src);
    if (here) {
      lT_n = lTs;
      lD_n = lDs;
      tr_n = trs;
      dr_n = drs;
    }
  }
  const long bo = static_cast<long>(b) * (G + 1);
  SeqDecision d{0.0, 0.0, 0, 0, 0, kDrawNone, bits, 0.f, 0.f, 0.f, 1.f};
  if (!bits) {
    d = SeqDecision{lT_n, lD_n, P.draw_compact ? b : tr_n, P.draw_compact ? b : dr_n, n,
                    (n < G) ? kDrawResidual : kDrawTarget, 0u, 0.f, 0.f, 0.f, 1.f};
    float lt_lo;
    split2(lT_n, d.lt_hi, lt_lo);
    split2(lT_n - lD_n, d.k_hi, d.k_lo);
    d.fT = static_cast<float>(exp2(-static_cast<double>(lt_lo)));
  }
  if (!write) return d;
  if (bits) {
    for (int q = lane; q <= G; q += kWarp) P.out_tokens[bo + q] = -1;
    if (lane == 0) {
      P.out_num_accepted[b] = 0;
      P.resid_mass[b] = NAN;
      P.decision[b] = d;
      atomicOr(P.status, bits);
    }
  } else {
    // accepted prefix and padding; the drawn token at n is the draw kernel's
    for (int q = lane; q <= G; q += kWarp) {
      if (q < n) P.out_tokens[bo + q] = P.tokens[static_cast<long>(b) * G + q];
      else if (q > n) P.out_tokens[bo + q] = -1;
    }
    if (lane == 0) {
      P.out_num_accepted[b] = n;
      P.decision[b] = d;
    }
  }
  return d;
}

// ---------------------------------------------------------------------------
// kernel 1: streaming statistics
// ---------------------------------------------------------------------------

template <int NT>
constexpr int min_blocks() {
  return 1024 / NT;  // caps registers at 64 per thread
}

template <typename T, int NT, bool kAligned>
__global__ void __launch_bounds__(NT, min_blocks<NT>()) stats_kernel(const Params P) {
  constexpr int kVec = Elem<T>::kVec;
  // the logits may be the previous kernel's output (programmatic launch):
  // the block may be resident before it completes, and waits for it here
  cudaGridDependencySynchronize();
  // From here every input of the caller is complete, so the next kernel may
  // be scheduled: it reads the caller's inputs at once, and this grid's
  // results only after its own grid-dependency wait.
  cudaTriggerProgrammaticLaunchCompletion();
  const int V = P.vocab, S = P.slices;
  // one unit = one block = one slice of one row; the target tensor's rows
  // come first, then the draft tensor's, so the grid walks memory in order
  // (the tapered rows first, in long slices)
  const long unit = blockIdx.x;
  const long uA = P.taper_rows * P.taper_slices;
  long r, slice, gps, Sr;
  if (unit < uA) {
    r = unit / P.taper_slices;
    slice = unit - r * P.taper_slices;
    gps = P.taper_groups;
    Sr = P.taper_slices;
  } else {
    const long u2 = unit - uA;
    const long q = u2 / S;
    r = P.taper_rows + q;
    slice = u2 - q * S;
    gps = P.groups_per_slice;
    Sr = S;
  }
  const long nT = P.target_rows;
  if (!bounds_ok(r, nT + P.draft_rows, P.status)) return;  // (block-uniform)
  const T* row = (r < nT) ? static_cast<const T*>(P.target) + r * V
                          : static_cast<const T*>(P.draft) + (r - nT) * V;
  const long ngroups = (static_cast<long>(V) + kVec - 1) / kVec;
  long glo = slice * gps;
  long ghi = glo + gps;
  if (glo > ngroups) glo = ngroups;
  if (ghi > ngroups) ghi = ngroups;
  const RowPartial part = slice_stats<T, NT, kAligned, 8>(row, glo, ghi, V, P.c_hi, P.c_lo);
  if (threadIdx.x == 0) {
    P.partial[r * S + slice] = part;
    // a tapered row's table entries past its slices: empty partials
    if (slice == 0)
      for (long j = Sr; j < S; ++j) P.partial[r * S + j] = RowPartial{0.0, -INFINITY, 0};
  }
}

// ---------------------------------------------------------------------------
// kernel 2: decide (one warp per sequence)
// ---------------------------------------------------------------------------

// The caller's inputs to a decision (tokens, uniforms, row maps, the logits
// at the tokens) are loaded before the grid-dependency wait: the statistics
// kernel lets this one be scheduled only once they are complete.  Logits
// gathered by an earlier kernel of this library are read after the wait.
// The draw kernel reads nothing before its own wait, so it may be scheduled
// at once.
template <typename T>
__global__ void __launch_bounds__(kDecideThreads) decide_kernel(const Params P) {
  const int b = blockIdx.x * (kDecideThreads / kWarp) + (threadIdx.x >> 5);
  const bool early = b < P.batch && !P.gathered_target && !P.gathered_draft;
  LaneInputs pre{0, 0, 0, 0.f, 0.f, 0.f, false, false};
  if (early) pre = lane_inputs<T>(P, b, threadIdx.x & (kWarp - 1));
  cudaTriggerProgrammaticLaunchCompletion();
  // the statistics of the previous kernel must be complete and visible
  cudaGridDependencySynchronize();
  if (b < P.batch) decide_sequence<T>(P, b, nullptr, true, early ? &pre : nullptr);  // warp-uniform
}

// ---------------------------------------------------------------------------
// kernel 3: draw (step 4)
// ---------------------------------------------------------------------------
//
// The rows drawn from are cut into tiles of kTile 16-byte groups: lane l of a
// warp takes groups k * 32 + l of the tile, k = 0 .. kDrawK - 1 (every load
// instruction of the warp reads 512 contiguous bytes).  All tiles of the
// batch, sequence by sequence, form one index range that the grid's warps
// split into contiguous runs, so the work is even whatever mix of residual
// draws (two rows), bonus draws (one row) and error outcomes (none) the batch
// holds.  A warp streams its run through a private ring of kStages tiles in
// shared memory filled by asynchronous 16-byte copies (cp.async; each lane
// copies and later reads only its own slots), so about three tiles per warp
// are in flight while one is reduced, without holding them in registers.  It
// writes the fp64 mass of each tile of its run to the sequence's table, then
// adds the number of tiles it finished to the sequence's ticket; the warp
// that completes the count locates u * Z: a warp scan over the table finds
// the tile, and a re-read of that one tile finds the index.

constexpr int kDrawThreads = 256;
constexpr int kDrawWarps = kDrawThreads / kWarp;
constexpr int kDrawK = 2;                 // groups per lane per tile
constexpr int kTile = kWarp * kDrawK;     // groups per tile of the mass table
constexpr int kDrawBlocksPerSM = 2;
constexpr int kStages = 4;                          // ring depth per warp
constexpr int kStageU4 = 2 * kDrawK * kWarp;        // 16-byte slots per warp per stage
constexpr size_t kDrawSmem = sizeof(uint4) * kStageU4 * kStages * kDrawWarps;

// tiles of one row of V entries stored `vec` to a 16-byte group
inline long draw_tiles_per_row(long V, int vec) {
  const long groups = (V + vec - 1) / vec;
  return (groups + kTile - 1) / kTile;
}

// Grid of the draw kernel: at most `draw_blocks` blocks per sequence, at most
// one resident wave, and at least one tile per warp.
inline unsigned draw_grid(long batch, long tiles_per_row, int draw_blocks, int num_sms) {
  long g = batch * static_cast<long>(draw_blocks);
  const long wave = static_cast<long>(num_sms) * kDrawBlocksPerSM;
  const long by_tiles = (batch * tiles_per_row + kDrawWarps - 1) / kDrawWarps;
  if (g > wave) g = wave;
  if (g > by_tiles) g = by_tiles;
  if (g < 1) g = 1;
  return static_cast<unsigned>(g);
}

// r (in units of 1/fT) for the kVec elements of one group: residual
// max(0, q - p) or target q.  Pairs of elements go through the packed fp32
// instructions (two lanes of arithmetic per instruction); the exponentials
// are one MUFU ex2 each.  L = log2(q/p) comes from the logit difference
// (exact for bf16 inputs) and p = q 2^-L.  L < 1/8 takes p (2^L - 1) from its
// Taylor series in L to L^5 (truncation below 7e-9 relative on (0, 1/8); for
// L <= 0 the series factor stays above 0.31, so the product is <= 0 and the
// final max(., 0) makes it 0); L >= 1/8 takes q - p (q >= 1.09 p: at most 3.6
// bits cancel).  Infinite logits need no test: a draft logit of -inf gives
// L = +inf, p = 0 and r = q; a target logit of -inf gives q = 0 and r = 0
// (the NaN of 0 * 2^inf is discarded by the final max).
template <typename T, int kMode>
__device__ __forceinline__ void group_r(const uint4& vt, const uint4& vd, const DrawConsts& k,
                                        float (&r)[Elem<T>::kVec]) {
  constexpr int kVec = Elem<T>::kVec;
  float xt[kVec];
  Elem<T>::unpack(vt, xt);
  const float2 chi = make_float2(k.c_hi, k.c_hi), clo = make_float2(k.c_lo, k.c_lo);
  const float2 mlt = make_float2(-k.lt_hi, -k.lt_hi);
  if constexpr (kMode == kDrawTarget) {
#pragma unroll
    for (int e = 0; e < kVec; e += 2) {
      const float2 x = make_float2(xt[e], xt[e + 1]);
      const float2 y = __ffma2_rn(x, clo, __ffma2_rn(x, chi, mlt));
      r[e] = ex2(y.x);
      r[e + 1] = ex2(y.y);
    }
  } else {
    float xd[kVec];
    Elem<T>::unpack(vd, xd);
    const float2 mkhi = make_float2(-k.k_hi, -k.k_hi), mklo = make_float2(-k.k_lo, -k.k_lo);
    const float2 one_neg = make_float2(-1.f, -1.f);
    const float2 a1 = make_float2(kA1, kA1), a2 = make_float2(kA2, kA2);
    const float2 a3 = make_float2(kA3, kA3), a4 = make_float2(kA4, kA4);
    const float2 a5 = make_float2(kA5, kA5);
#pragma unroll
    for (int e = 0; e < kVec; e += 2) {
      const float2 x = make_float2(xt[e], xt[e + 1]);
      const float2 xdp = make_float2(xd[e], xd[e + 1]);
      const float2 y = __ffma2_rn(x, clo, __ffma2_rn(x, chi, mlt));
      float2 q;
      q.x = ex2(y.x);
      q.y = ex2(y.y);
      const float2 dx = __ffma2_rn(xdp, one_neg, x);  // xt - xd, exact for bf16
      const float2 L = __fadd2_rn(__ffma2_rn(dx, chi, mkhi), __ffma2_rn(dx, clo, mklo));
      float2 w;
      w.x = ex2(-L.x);
      w.y = ex2(-L.y);
      const float2 p = __fmul2_rn(q, w);
      float2 t = __ffma2_rn(a5, L, a4);
      t = __ffma2_rn(t, L, a3);
      t = __ffma2_rn(t, L, a2);
      t = __ffma2_rn(t, L, a1);
      const float2 small = __fmul2_rn(p, __fmul2_rn(t, L));
      const float2 big = __ffma2_rn(p, one_neg, q);  // q - p
      r[e] = fmaxf((L.x < 0.125f) ? small.x : big.x, 0.f);
      r[e + 1] = fmaxf((L.y < 0.125f) ? small.y : big.y, 0.f);
    }
  }
}

// fp32 sum of a group's r, pairwise
template <int kVec>
__device__ __forceinline__ float group_sum(const float (&r)[kVec]) {
  float2 acc = make_float2(r[0], r[1]);
#pragma unroll
  for (int e = 2; e < kVec; e += 2) acc = __fadd2_rn(acc, make_float2(r[e], r[e + 1]));
  return acc.x + acc.y;
}

// One tile's loads for the calling lane: its kDrawK groups of the target row
// (and of the draft row for a residual draw); groups past the row end are
// not read.
template <typename T, bool kAligned, int kMode>
__device__ __forceinline__ void load_tile(const T* rowT, const T* rowD, long tile, long ngroups,
                                          int V, uint4 (&vt)[kDrawK], uint4 (&vd)[kDrawK]) {
  const int lane = threadIdx.x & (kWarp - 1);
#pragma unroll
  for (int kk = 0; kk < kDrawK; ++kk) {
    const long g = tile * kTile + kk * kWarp + lane;
    if (g < ngroups) {
      vt[kk] = fetch_group<T, kAligned>(rowT, g, V);
      if constexpr (kMode == kDrawResidual) vd[kk] = fetch_group<T, kAligned>(rowD, g, V);
    }
  }
}

// fp64 mass (times fT) of one tile whose loads are in vt / vd, valid in every lane
template <typename T, int kMode>
__device__ __forceinline__ double tile_mass_of(const uint4 (&vt)[kDrawK], const uint4 (&vd)[kDrawK],
                                               const DrawConsts& k, long tile, long ngroups) {
  constexpr int kVec = Elem<T>::kVec;
  const int lane = threadIdx.x & (kWarp - 1);
  double m = 0.0;
#pragma unroll
  for (int kk = 0; kk < kDrawK; ++kk) {
    const long g = tile * kTile + kk * kWarp + lane;
    if (g < ngroups) {
      float r[kVec];
      group_r<T, kMode>(vt[kk], vd[kk], k, r);
      m += static_cast<double>(group_sum<kVec>(r));
    }
  }
  return warp_sum(m) * static_cast<double>(k.fT);
}

// Masses of tiles [t0, t1) of one row into table[t0 .. t1) (lane 0 stores),
// software-pipelined: the next tile's loads are in flight while the current
// tile is reduced (two register buffers, alternated).
template <typename T, bool kAligned, int kMode>
__device__ __forceinline__ void tile_masses_mode(const T* rowT, const T* rowD, const DrawConsts& k,
                                                 long t0, long t1, long ngroups, int V,
                                                 double* table) {
  const int lane = threadIdx.x & (kWarp - 1);
  uint4 at[kDrawK], ad[kDrawK], bt[kDrawK], bd[kDrawK];
  long t = t0;
  if (t < t1) load_tile<T, kAligned, kMode>(rowT, rowD, t, ngroups, V, at, ad);
  while (t < t1) {
    if (t + 1 < t1) load_tile<T, kAligned, kMode>(rowT, rowD, t + 1, ngroups, V, bt, bd);
    const double za = tile_mass_of<T, kMode>(at, ad, k, t, ngroups);
    if (lane == 0) table[t] = za;
    if (++t >= t1) break;
    if (t + 1 < t1) load_tile<T, kAligned, kMode>(rowT, rowD, t + 1, ngroups, V, at, ad);
    const double zb = tile_mass_of<T, kMode>(bt, bd, k, t, ngroups);
    if (lane == 0) table[t] = zb;
    ++t;
  }
}

__device__ __forceinline__ void cp_async16(uint4* smem, const uint4* gmem) {
  const unsigned sa = static_cast<unsigned>(__cvta_generic_to_shared(smem));
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(sa), "l"(gmem) : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// One tile's copies into a ring slot: target groups at [kk * 32 + lane],
// draft groups at [(kDrawK + kk) * 32 + lane]; groups past the row end are
// not copied (and not read).
template <int kMode>
__device__ __forceinline__ void issue_tile(uint4* slot, const uint4* rowT, const uint4* rowD,
                                           long tile, long ngroups) {
  const int lane = threadIdx.x & (kWarp - 1);
#pragma unroll
  for (int kk = 0; kk < kDrawK; ++kk) {
    const long g = tile * kTile + kk * kWarp + lane;
    if (g < ngroups) {
      cp_async16(slot + kk * kWarp + lane, rowT + g);
      if constexpr (kMode == kDrawResidual) cp_async16(slot + (kDrawK + kk) * kWarp + lane, rowD + g);
    }
  }
}

// Masses of tiles [t0, t1) of one row (16-byte aligned rows) into table,
// through the calling warp's ring of NS stages: NS - 1 tiles are in flight
// while one is reduced.  Every iteration commits one copy group (possibly
// empty), so waiting until at most NS - 1 groups are pending means the
// oldest tile has landed.  Returns with no copy in flight.
template <typename T, int kMode, int NS = kStages>
__device__ __forceinline__ void tile_masses_ring(const T* rowT, const T* rowD, const DrawConsts& k,
                                                 long t0, long t1, long ngroups, double* table,
                                                 uint4* ring) {
  const int lane = threadIdx.x & (kWarp - 1);
  const uint4* gT = reinterpret_cast<const uint4*>(rowT);
  const uint4* gD = reinterpret_cast<const uint4*>(rowD);
  const long n = t1 - t0;
#pragma unroll
  for (int i = 0; i < NS - 1; ++i) {
    if (i < n) issue_tile<kMode>(ring + i * kStageU4, gT, gD, t0 + i, ngroups);
    cp_async_commit();
  }
  for (long i = 0; i < n; ++i) {
    const long nx = i + NS - 1;
    if (nx < n) issue_tile<kMode>(ring + (nx % NS) * kStageU4, gT, gD, t0 + nx, ngroups);
    cp_async_commit();
    cp_async_wait<NS - 1>();
    const uint4* slot = ring + (i % NS) * kStageU4;
    uint4 vt[kDrawK], vd[kDrawK];
#pragma unroll
    for (int kk = 0; kk < kDrawK; ++kk) {
      vt[kk] = slot[kk * kWarp + lane];
      if constexpr (kMode == kDrawResidual) vd[kk] = slot[(kDrawK + kk) * kWarp + lane];
    }
    const double z = tile_mass_of<T, kMode>(vt, vd, k, t0 + i, ngroups);
    if (lane == 0) table[t0 + i] = z;
  }
  cp_async_wait<0>();
}

template <typename T, bool kAligned>
__device__ __forceinline__ void tile_masses(int mode, const T* rowT, const T* rowD,
                                            const DrawConsts& k, long t0, long t1, long ngroups,
                                            int V, double* table) {
  if (mode == kDrawResidual)
    tile_masses_mode<T, kAligned, kDrawResidual>(rowT, rowD, k, t0, t1, ngroups, V, table);
  else
    tile_masses_mode<T, kAligned, kDrawTarget>(rowT, rowD, k, t0, t1, ngroups, V, table);
}

// The index inside `tile` where the running mass first exceeds tl_mass (in
// table units); else the tile's last index with mass (rounding between the
// table's sum and this scan's); else -1.  The calling warp re-reads the
// tile: lane l's groups k * 32 + l, scanned in index order (k, then lane,
// then element).
template <typename T, bool kAligned, int kMode>
__device__ __forceinline__ int scan_tile(const T* rowT, const T* rowD, const DrawConsts& k,
                                         long tile, long ngroups, int V, double tl_mass) {
  constexpr int kVec = Elem<T>::kVec;
  const int lane = threadIdx.x & (kWarp - 1);
  const double tl = tl_mass / static_cast<double>(k.fT);  // in the units of group_r
  uint4 vt[kDrawK], vd[kDrawK];
  load_tile<T, kAligned, kMode>(rowT, rowD, tile, ngroups, V, vt, vd);
  double base = 0.0;
  int mylast = -1;
#pragma unroll
  for (int kk = 0; kk < kDrawK; ++kk) {
    const long g = tile * kTile + kk * kWarp + lane;
    float r[kVec];
#pragma unroll
    for (int e = 0; e < kVec; ++e) r[e] = 0.f;
    if (g < ngroups) group_r<T, kMode>(vt[kk], vd[kk], k, r);
    const double v = static_cast<double>(group_sum<kVec>(r));
#pragma unroll
    for (int e = 0; e < kVec; ++e)
      if (r[e] > 0.f) mylast = static_cast<int>(g * kVec + e);
    double incl = v;
#pragma unroll
    for (int o = 1; o < kWarp; o <<= 1) {
      const double y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    double excl = __shfl_up_sync(0xffffffffu, incl, 1);
    if (lane == 0) excl = 0.0;
    const unsigned hit =
        __ballot_sync(0xffffffffu, v > 0.0 && base + excl <= tl && base + incl > tl);
    if (hit) {
      const int Ln = __ffs(hit) - 1;
      int token = -1;
      if (lane == Ln) {
        double acc = base + excl;
        int last = -1;
#pragma unroll
        for (int e = 0; e < kVec; ++e) {
          if (r[e] > 0.f) {
            acc += static_cast<double>(r[e]);
            last = static_cast<int>(g * kVec + e);
            if (token < 0 && acc > tl) token = last;
          }
        }
        if (token < 0) token = last;  // rounding between the two sums
      }
      return __shfl_sync(0xffffffffu, token, Ln);
    }
    base += __shfl_sync(0xffffffffu, incl, kWarp - 1);
  }
  return warp_maxi(mylast);  // rounding past the tile's end
}

constexpr int kLocRun = 10;  // table entries per lane per round of the scans below

// Sum of table[0 .. ntiles) by the calling warp: each lane loads a contiguous
// run of kLocRun entries per round (all loads of a round in flight together)
// and adds it in index order; lane sums are combined across the warp.
__device__ __forceinline__ double table_total(const double* table, long ntiles) {
  const int lane = threadIdx.x & (kWarp - 1);
  double tot = 0.0;
  for (long r0 = 0; r0 < ntiles; r0 += static_cast<long>(kWarp) * kLocRun) {
    const long a = r0 + static_cast<long>(lane) * kLocRun;
    double v[kLocRun];
#pragma unroll
    for (int q = 0; q < kLocRun; ++q) v[q] = (a + q < ntiles) ? __ldcg(table + a + q) : 0.0;
    double sm = 0.0;
#pragma unroll
    for (int q = 0; q < kLocRun; ++q) sm += v[q];
    tot += warp_sum(sm);
  }
  return tot;
}

// The first entry i of table[0 .. ntiles) with positive mass whose running
// sum in index order passes `target` (found = i, tl = target minus the mass
// before i), by the calling warp: per round, lane runs as in table_total, a
// warp scan of the lane sums picks the lane and that lane walks its run.  If
// rounding leaves no such entry, the last entry with mass and tl = +inf.
__device__ __forceinline__ void find_in_table(const double* table, long ntiles, double target,
                                              long& found, double& tl) {
  const int lane = threadIdx.x & (kWarp - 1);
  double base = 0.0;
  long last_mass = -1;
  found = -1;
  tl = INFINITY;
  for (long r0 = 0; r0 < ntiles; r0 += static_cast<long>(kWarp) * kLocRun) {
    const long a = r0 + static_cast<long>(lane) * kLocRun;
    double v[kLocRun];
#pragma unroll
    for (int q = 0; q < kLocRun; ++q) v[q] = (a + q < ntiles) ? __ldcg(table + a + q) : 0.0;
    double sm = 0.0;
    long mylast = -1;
#pragma unroll
    for (int q = 0; q < kLocRun; ++q) {
      sm += v[q];
      if (v[q] > 0.0) mylast = a + q;
    }
    double incl = sm;
#pragma unroll
    for (int o = 1; o < kWarp; o <<= 1) {
      const double y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    double excl = __shfl_up_sync(0xffffffffu, incl, 1);
    if (lane == 0) excl = 0.0;
    long lm = mylast;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) lm = max(lm, __shfl_xor_sync(0xffffffffu, lm, o));
    if (lm >= 0) last_mass = lm;
    const unsigned hit =
        __ballot_sync(0xffffffffu, sm > 0.0 && base + excl <= target && base + incl > target);
    if (hit) {
      const int Ln = __ffs(hit) - 1;
      long f = -1;
      double t = INFINITY;
      if (lane == Ln) {
        double acc = base + excl;
#pragma unroll
        for (int q = 0; q < kLocRun; ++q) {
          if (f < 0 && v[q] > 0.0 && acc + v[q] > target) {
            f = a + q;
            t = target - acc;
          }
          acc += v[q];
        }
        if (f < 0) f = mylast;  // rounding between the lane sum and this walk
      }
      found = __shfl_sync(0xffffffffu, f, Ln);
      tl = __shfl_sync(0xffffffffu, t, Ln);
      return;
    }
    base += __shfl_sync(0xffffffffu, incl, kWarp - 1);
  }
  found = last_mass;  // rounding past the table's end
  tl = INFINITY;
}

// find_in_table for a table of at most kWarp * kLocRun entries, with the
// total computed from the same loads; returns Z (found = -1 if Z is 0).
__device__ __forceinline__ double locate_one_round(const double* table, long ntiles, double u,
                                                   long& found, double& tl) {
  const int lane = threadIdx.x & (kWarp - 1);
  const long a = static_cast<long>(lane) * kLocRun;
  double v[kLocRun];
#pragma unroll
  for (int q = 0; q < kLocRun; ++q) v[q] = (a + q < ntiles) ? __ldcg(table + a + q) : 0.0;
  double sm = 0.0;
  long mylast = -1;
#pragma unroll
  for (int q = 0; q < kLocRun; ++q) {
    sm += v[q];
    if (v[q] > 0.0) mylast = a + q;
  }
  double incl = sm;
#pragma unroll
  for (int o = 1; o < kWarp; o <<= 1) {
    const double y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  double excl = __shfl_up_sync(0xffffffffu, incl, 1);
  if (lane == 0) excl = 0.0;
  const double Z = __shfl_sync(0xffffffffu, incl, kWarp - 1);
  found = -1;
  tl = INFINITY;
  if (!(Z > 0.0)) return Z;
  const double target = u * Z;
  const unsigned hit = __ballot_sync(0xffffffffu, sm > 0.0 && excl <= target && incl > target);
  if (hit) {
    const int Ln = __ffs(hit) - 1;
    long f = -1;
    double t = INFINITY;
    if (lane == Ln) {
      double acc = excl;
#pragma unroll
      for (int q = 0; q < kLocRun; ++q) {
        if (f < 0 && v[q] > 0.0 && acc + v[q] > target) {
          f = a + q;
          t = target - acc;
        }
        acc += v[q];
      }
      if (f < 0) f = mylast;  // rounding between the lane sum and this walk
    }
    found = __shfl_sync(0xffffffffu, f, Ln);
    tl = __shfl_sync(0xffffffffu, t, Ln);
  } else {
    long lm = mylast;  // rounding past the table's end: the last entry with mass
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) lm = max(lm, __shfl_xor_sync(0xffffffffu, lm, o));
    found = lm;
  }
  return Z;
}

// Step 4's last part for sequence b, by the warp that finished its table:
// Z = sum of the tile masses; the tile holding u * Z (a warp scan over the
// table in index order); the index inside it.  Z = 0 at a rejection: the
// warp recomputes the table for q_n and draws from it (ZERO_MASS warning).
template <typename T, bool kAligned>
__device__ __noinline__ void locate(const Params* Pp, int b, int n, int mode, const T* rowT,
                                    const T* rowD, const DrawConsts k, long ntiles,
                                    long ngroups) {
  const Params& P = *Pp;
  const int lane = threadIdx.x & (kWarp - 1);
  const int V = P.vocab, G = P.gamma;
  double* table = P.draw_mass + static_cast<long>(b) * ntiles;
  unsigned extra_bits = 0;
  const double u = static_cast<double>(P.u_resample[b]);
  long found = -1;
  double tl = INFINITY, Z = 0.0;
  // a table of at most one round of lane runs is read once: Z and the place
  // of u * Z come from the same loads
  const bool one_round = ntiles <= static_cast<long>(kWarp) * kLocRun;
  if (one_round) Z = locate_one_round(table, ntiles, u, found, tl);
  else Z = table_total(table, ntiles);
  if (!(Z > 0.0) && mode == kDrawResidual) {
    mode = kDrawTarget;
    extra_bits |= kStatZeroMass;
    tile_masses<T, kAligned>(mode, rowT, rowD, k, 0, ntiles, ngroups, V, table);
    __syncwarp();
    if (one_round) Z = locate_one_round(table, ntiles, u, found, tl);
    else Z = table_total(table, ntiles);
  }
  if (!one_round) find_in_table(table, ntiles, u * Z, found, tl);
  int token = -1;
  if (found >= 0 && bounds_ok(found, ntiles, P.status)) {
    token = (mode == kDrawResidual)
                ? scan_tile<T, kAligned, kDrawResidual>(rowT, rowD, k, found, ngroups, V, tl)
                : scan_tile<T, kAligned, kDrawTarget>(rowT, rowD, k, found, ngroups, V, tl);
  }
  if (lane == 0) {
    if (bounds_ok(n, G + 1, P.status)) P.out_tokens[static_cast<long>(b) * (G + 1) + n] = token;
    P.resid_mass[b] = Z;
    if (extra_bits) atomicOr(P.status, extra_bits);
    P.draw_ticket[b] = 0u;  // ready for the next launch
  }
}

template <typename T, bool kAligned>
__global__ void __launch_bounds__(kDrawThreads, kDrawBlocksPerSM) draw_kernel(const __grid_constant__ Params P) {
  constexpr int kVec = Elem<T>::kVec;
  extern __shared__ uint4 draw_smem[];
  uint4* ring = draw_smem + (threadIdx.x >> 5) * (kStageU4 * kStages);  // this warp's ring
  const int lane = threadIdx.x & (kWarp - 1);
  const int V = P.vocab;
  const long ngroups = (static_cast<long>(V) + kVec - 1) / kVec;
  const long ntiles = P.draw_tiles;
  const long total = static_cast<long>(P.batch) * ntiles;
  const long W = static_cast<long>(gridDim.x) * kDrawWarps;
  const long w = static_cast<long>(blockIdx.x) * kDrawWarps + (threadIdx.x >> 5);
  const long lo = total * w / W, hi = total * (w + 1) / W;
  cudaGridDependencySynchronize();  // the decisions of the previous kernel
  for (long t = lo; t < hi;) {
    const int b = static_cast<int>(t / ntiles);
    const long row0 = static_cast<long>(b) * ntiles;
    const long end = (hi < row0 + ntiles) ? hi : row0 + ntiles;
    const SeqDecision d = P.decision[b];
    // (a debug build skips a sequence whose rows drawn from lie outside the
    // logit buffers, in every warp alike, so its ticket stays untouched)
    const bool rows_ok = d.mode == kDrawNone ||
                         (bounds_ok(d.trow, P.target_rows, P.status) &&
                          (d.mode != kDrawResidual || bounds_ok(d.drow, P.draft_rows, P.status)));
    if (d.mode != kDrawNone && rows_ok) {
      const T* rowT = static_cast<const T*>(P.target) + d.trow * V;
      const T* rowD = (d.mode == kDrawResidual) ? static_cast<const T*>(P.draft) + d.drow * V
                                                : nullptr;
      DrawConsts k;
      k.c_hi = P.c_hi;
      k.c_lo = P.c_lo;
      k.lt_hi = d.lt_hi;
      k.k_hi = d.k_hi;
      k.k_lo = d.k_lo;
      k.fT = d.fT;
      double* table = P.draw_mass + row0;
      if constexpr (kAligned) {
        if (d.mode == kDrawResidual)
          tile_masses_ring<T, kDrawResidual>(rowT, rowD, k, t - row0, end - row0, ngroups, table, ring);
        else
          tile_masses_ring<T, kDrawTarget>(rowT, rowD, k, t - row0, end - row0, ngroups, table, ring);
      } else {
        tile_masses<T, kAligned>(d.mode, rowT, rowD, k, t - row0, end - row0, ngroups, V, table);
      }
      // publish this run's tiles; the warp that completes the row locates
      unsigned last = 0;
      if (lane == 0) {
        __threadfence();
        const unsigned cnt = static_cast<unsigned>(end - t);
        const unsigned old = atomicAdd(P.draw_ticket + b, cnt);
        last = (old + cnt == static_cast<unsigned>(ntiles));
        if (last) __threadfence();
      }
      last = __shfl_sync(0xffffffffu, last, 0);
      if (last) {
        __threadfence();  // every lane reads the other warps' tiles after the ticket
        locate<T, kAligned>(&P, b, d.n, d.mode, rowT, rowD, k, ntiles, ngroups);
      }
    }
    t = end;
  }
}

// Host: launch the draw kernel (its ring needs more than the default 48 KB of
// dynamic shared memory per block), optionally as a programmatic dependent
// launch of the previous kernel on the stream.
template <typename T, bool kAligned>
inline cudaError_t launch_draw(const Params& p, unsigned grid, cudaStream_t s, bool pdl) {
  const size_t smem = kAligned ? kDrawSmem : 0;
  cudaError_t e = cudaSuccess;
  if (kAligned)
    e = cudaFuncSetAttribute(draw_kernel<T, kAligned>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid, 1, 1);
  cfg.blockDim = dim3(kDrawThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, draw_kernel<T, kAligned>, p);
}

}  // namespace specverify
