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
//   draw    S' blocks per sequence over the rows drawn from (n < gamma:
//           max(0, q_n - p_n) from target and draft row n; n == gamma: q of
//           target row gamma); each block publishes the mass of every
//           32-group tile of its share, and the block that takes the
//           sequence's ticket last finds, by a block-wide prefix scan over
//           the tile masses, the tile that holds u * Z and scans it one group
//           per lane in index order (step 4).
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
enum : unsigned { kStatTokenRange = 1u, kStatNonFinite = 2u, kStatZeroMass = 4u, kStatRowIndex = 8u };
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
  int draw_slices;           // S2 draw blocks per sequence
  int groups_per_draw;       // groups per draw block (whole 32-group tiles)
  float c_hi, c_lo;          // log2(e)/T = c_hi + c_lo, c_lo > 0
  double c;                  // c_hi + c_lo, exactly
  // fused LM-head form: the logits at the draft tokens were picked out by the
  // GEMM ([target_rows] and [draft_rows] floats; null: read the logit rows),
  // and the draw reads row b of compact [B, V] logit buffers
  const float* gathered_target;
  const float* gathered_draft;
  int draw_compact;
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

// r / fT for the VEC elements of one group: residual max(0, q - p) or target
// q; the caller multiplies sums of r by fT.  L = log2(q/p) comes from the
// logit difference (exact for bf16 inputs) and p = q 2^-L.  L >= 1/8 gives
// q - p (q >= 1.09 p: at most 3.6 bits cancel); 0 < L < 1/8 gives
// p (2^L - 1) from its Taylor series in L (to L^5, truncation below 7e-9
// relative); L <= 0 gives q - p <= 0, which the final max(., 0) turns into 0.
// The infinite cases need no test: a draft logit of -inf gives L = +inf,
// p = 0 and r = q; a target logit of -inf gives q = 0, L = -inf and r = 0
// (the NaN of 0 * 2^inf is discarded by the selects).
template <typename T, int kMode>
__device__ __forceinline__ void group_mass(const uint4& vt, const uint4& vd, const DrawConsts& k,
                                           float (&r)[Elem<T>::kVec]) {
  constexpr int kVec = Elem<T>::kVec;
  float xt[kVec];
  Elem<T>::unpack(vt, xt);
  if constexpr (kMode == kDrawTarget) {
#pragma unroll
    for (int e = 0; e < kVec; ++e) r[e] = ex2(arg2(xt[e], k.c_hi, k.c_lo, k.lt_hi));
  } else {
    float xd[kVec];
    Elem<T>::unpack(vd, xd);
#pragma unroll
    for (int e = 0; e < kVec; ++e) {
      const float q = ex2(arg2(xt[e], k.c_hi, k.c_lo, k.lt_hi));
      const float dx = xt[e] - xd[e];
      const float L = fmaf(dx, k.c_hi, -k.k_hi) + fmaf(dx, k.c_lo, -k.k_lo);
      const float p = q * ex2(-L);
      float t = kA5;
      t = fmaf(t, L, kA4);
      t = fmaf(t, L, kA3);
      t = fmaf(t, L, kA2);
      t = fmaf(t, L, kA1);
      const float small = p * (t * L);
      const float res = (L > 0.f && L < 0.125f) ? small : q - p;
      r[e] = fmaxf(res, 0.f);  // NaN (0 * inf) becomes 0 here
    }
  }
}

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
// kernel 1: streaming statistics
// ---------------------------------------------------------------------------

template <int NT>
constexpr int min_blocks() {
  return 1024 / NT;  // caps registers at 64 per thread
}

template <typename T, int NT, bool kAligned>
__global__ void __launch_bounds__(NT, min_blocks<NT>()) stats_kernel(const Params P) {
  constexpr int kVec = Elem<T>::kVec;
  const int G = P.gamma, V = P.vocab, S = P.slices;
  // one unit = one block = one slice of one row; the target tensor's rows
  // come first, then the draft tensor's, so the grid walks memory in order
  const long unit = blockIdx.x;
  const long r = unit / S;
  const int slice = static_cast<int>(unit - r * S);
  const long nT = P.target_rows;
  const T* row = (r < nT) ? static_cast<const T*>(P.target) + r * V
                          : static_cast<const T*>(P.draft) + (r - nT) * V;
  (void)G;
  const long ngroups = (static_cast<long>(V) + kVec - 1) / kVec;
  long glo = static_cast<long>(slice) * P.groups_per_slice;
  long ghi = glo + P.groups_per_slice;
  if (glo > ngroups) glo = ngroups;
  if (ghi > ngroups) ghi = ngroups;
  const RowPartial part = slice_stats<T, NT, kAligned, 8>(row, glo, ghi, V, P.c_hi, P.c_lo);
  if (threadIdx.x == 0) P.partial[unit] = part;
  cudaTriggerProgrammaticLaunchCompletion();
}

// ---------------------------------------------------------------------------
// kernel 2: decide (one warp per sequence, one lane per position)
// ---------------------------------------------------------------------------

constexpr int kDecideThreads = 128;
constexpr int kMaxGamma = 255;

// (o, s) partials of one row combined in two passes, so that the fp64
// exponentials of the second pass are independent of one another
__device__ __forceinline__ double row_lse2(const RowPartial* parts, int S, int& valid) {
  float O = -INFINITY;
  for (int r = 0; r < S; ++r) O = fmaxf(O, parts[r].o);
  double sum = 0.0;
  for (int r = 0; r < S; ++r) {
    const float o = parts[r].o;
    const double s = parts[r].s;
    sum += (o == -INFINITY) ? s * 0.0 : s * exp2(static_cast<double>(o) - O);  // NaN survives
  }
  valid = (O != -INFINITY) && isfinite(sum) && sum > 0.0;
  return static_cast<double>(O) + log2(sum);  // log2 sum_i 2^(x_i c)
}

template <typename T>
__global__ void __launch_bounds__(kDecideThreads) decide_kernel(const Params P) {
  // the statistics of the previous kernel must be complete and visible
  cudaGridDependencySynchronize();
  const int lane = threadIdx.x & (kWarp - 1);
  const int b = blockIdx.x * (kDecideThreads / kWarp) + (threadIdx.x >> 5);
  if (b < P.batch) {  // warp-uniform
    const int G = P.gamma, V = P.vocab, S = P.slices;
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
        // rows of the logit buffers that hold this position
        tr = P.target_map ? static_cast<long>(P.target_map[position]) : position;
        dr = has_draft ? (P.draft_map ? static_cast<long>(P.draft_map[pj]) : pj) : 0;
        map_bad = tr < 0 || tr >= P.target_rows || (has_draft && (dr < 0 || dr >= P.draft_rows));
        // the acceptance test's inputs first: their loads overlap the combine
        int t = 0;
        float u = 0.f, xt = 0.f, xd = 0.f;
        if (has_draft) {
          t = P.tokens[pj];
          u = P.u_accept[pj];
          tok_bad = (t < 0 || t >= V);
          if (!tok_bad && !map_bad) {
            xt = P.gathered_target ? P.gathered_target[tr]
                                   : Elem<T>::load1(static_cast<const T*>(P.target) + tr * V, t);
            xd = P.gathered_draft ? P.gathered_draft[dr]
                                  : Elem<T>::load1(static_cast<const T*>(P.draft) + dr * V, t);
          }
        }
        int validT = 0, validD = 1;
        if (!map_bad) {
          lT = row_lse2(P.partial + tr * S, S, validT);
          if (has_draft) lD = row_lse2(P.partial + (P.target_rows + dr) * S, S, validD);
        }
        P.tstat[position] = RowStat{lT, validT, 0};
        if (has_draft) P.dstat[pj] = RowStat{lD, validD, 0};
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
          P.pos[pj] = info;
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
    if (bits) {
      for (int q = lane; q <= G; q += kWarp) P.out_tokens[bo + q] = -1;
      if (lane == 0) {
        P.out_num_accepted[b] = 0;
        P.resid_mass[b] = NAN;
        P.decision[b] = SeqDecision{0.0, 0.0, 0, 0, 0, kDrawNone, bits, 0.f, 0.f, 0.f, 1.f};
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
        SeqDecision d{lT_n, lD_n, P.draw_compact ? b : tr_n, P.draw_compact ? b : dr_n, n,
                      (n < G) ? kDrawResidual : kDrawTarget, 0u, 0.f, 0.f, 0.f, 1.f};
        float lt_lo;
        split2(lT_n, d.lt_hi, lt_lo);
        split2(lT_n - lD_n, d.k_hi, d.k_lo);
        d.fT = static_cast<float>(exp2(-static_cast<double>(lt_lo)));
        P.decision[b] = d;
      }
    }
  }
  cudaTriggerProgrammaticLaunchCompletion();
}

// ---------------------------------------------------------------------------
// kernel 3: draw
// ---------------------------------------------------------------------------

constexpr int kDrawThreads = 128;
constexpr int kDrawWarps = kDrawThreads / kWarp;
constexpr int kTile = 32;  // groups per tile of the draw's mass table

// Mass of each 32-group tile of [tlo, thi) (tiles of the row, warp w takes
// tiles w, w + 4, ...); lane 0 of the warp stores the tile's mass in `table`.
// Software-pipelined: the next two tiles' loads are in flight while the
// current two are reduced.
template <typename T, bool kAligned>
__device__ __forceinline__ void tile_masses(int mode, const T* drawT, const T* drawD,
                                            const DrawConsts& k, long tlo, long thi,
                                            long ngroups, int V, double* table) {
  constexpr int kVec = Elem<T>::kVec;
  constexpr int kPair = 2;  // tiles per pipeline stage
  const int lane = threadIdx.x & (kWarp - 1), warp = threadIdx.x >> 5;
  const long first = tlo + warp;
  if (first >= thi) return;
  const long count = (thi - first + kDrawWarps - 1) / kDrawWarps;  // this warp's tiles
  auto load = [&](long kk, uint4 (&vt)[kPair], uint4 (&vd)[kPair]) {
#pragma unroll
    for (int u = 0; u < kPair; ++u) {
      const long g = (first + (kk + u) * kDrawWarps) * kTile + lane;
      if (kk + u < count && g < ngroups) {
        vt[u] = fetch_group<T, kAligned>(drawT, g, V);
        vd[u] = (mode == kDrawResidual) ? fetch_group<T, kAligned>(drawD, g, V) : vt[u];
      }
    }
  };
  uint4 ct[kPair], cd[kPair];
  load(0, ct, cd);
  for (long kk = 0; kk < count; kk += kPair) {
    uint4 nt[kPair], nd[kPair];
    load(kk + kPair, nt, nd);
#pragma unroll
    for (int u = 0; u < kPair; ++u) {
      if (kk + u < count) {  // warp-uniform
        const long tile = first + (kk + u) * kDrawWarps;
        const long g = tile * kTile + lane;
        float gs = 0.f;
        if (g < ngroups) {
          float r[kVec];
          if (mode == kDrawResidual) group_mass<T, kDrawResidual>(ct[u], cd[u], k, r);
          else group_mass<T, kDrawTarget>(ct[u], cd[u], k, r);
#pragma unroll
          for (int e = 0; e < kVec; ++e) gs += r[e];
        }
        const double z = warp_sum(static_cast<double>(gs)) * k.fT;
        if (lane == 0) table[tile] = z;
      }
    }
#pragma unroll
    for (int u = 0; u < kPair; ++u) {
      ct[u] = nt[u];
      cd[u] = nd[u];
    }
  }
}

// The masses of the 32 groups of `tile`, one per lane of the calling warp:
// returns the index where the running mass first exceeds tl, else the
// tile's last index with mass (rounding), else -1 (no mass in the tile).
template <typename T, bool kAligned>
__device__ __forceinline__ int scan_tile(int mode, const T* drawT, const T* drawD,
                                         const DrawConsts& k, long tile, long ngroups, int V,
                                         double tl_mass) {
  const double tl = tl_mass / static_cast<double>(k.fT);  // in the units of group_mass
  constexpr int kVec = Elem<T>::kVec;
  const int lane = threadIdx.x & (kWarp - 1);
  const long g = tile * kTile + lane;
  float r[kVec];
#pragma unroll
  for (int e = 0; e < kVec; ++e) r[e] = 0.f;
  if (g < ngroups) {
    const uint4 vt = fetch_group<T, kAligned>(drawT, g, V);
    const uint4 vd = (mode == kDrawResidual) ? fetch_group<T, kAligned>(drawD, g, V) : vt;
    if (mode == kDrawResidual) group_mass<T, kDrawResidual>(vt, vd, k, r);
    else group_mass<T, kDrawTarget>(vt, vd, k, r);
  }
  float gs = 0.f;
  int mylast = -1;
#pragma unroll
  for (int e = 0; e < kVec; ++e) {
    gs += r[e];
    if (r[e] > 0.f) mylast = static_cast<int>(g * kVec + e);
  }
  const double ls = static_cast<double>(gs);
  double incl = ls;
#pragma unroll
  for (int o = 1; o < kWarp; o <<= 1) {
    const double y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  double excl = __shfl_up_sync(0xffffffffu, incl, 1);
  if (lane == 0) excl = 0.0;
  const unsigned hit = __ballot_sync(0xffffffffu, excl <= tl && incl > tl);
  if (hit) {
    const int L = __ffs(hit) - 1;
    int token = -1;
    if (lane == L) {
      double acc = excl;
#pragma unroll
      for (int e = 0; e < kVec; ++e) {
        if (r[e] > 0.f) {
          acc += static_cast<double>(r[e]);
          if (token < 0 && acc > tl) token = static_cast<int>(g * kVec + e);
        }
      }
      if (token < 0) token = mylast;  // rounding between the two sums
    }
    return __shfl_sync(0xffffffffu, token, L);
  }
  return warp_maxi(mylast);  // rounding past the tile's end
}

template <typename T, bool kAligned>
__global__ void __launch_bounds__(kDrawThreads, 8) draw_kernel(const Params P) {
  constexpr int kVec = Elem<T>::kVec;
  const int tid = threadIdx.x;
  const int G = P.gamma, V = P.vocab, S2 = P.draw_slices;
  const int b = blockIdx.x / S2;
  const int s2 = blockIdx.x - b * S2;
  cudaGridDependencySynchronize();  // the decisions of the previous kernel
  const SeqDecision d = P.decision[b];
  if (d.mode == kDrawNone) return;  // the decide kernel wrote the error outcome
  const int n = d.n;
  const long bo = static_cast<long>(b) * (G + 1);

  // ---- step 4: residual (n < gamma) or bonus (n == gamma) draw ----
  int mode = d.mode;
  const T* drawT = static_cast<const T*>(P.target) + d.trow * V;
  const T* drawD = (mode == kDrawResidual) ? static_cast<const T*>(P.draft) + d.drow * V : nullptr;
  DrawConsts k;
  k.c_hi = P.c_hi;
  k.c_lo = P.c_lo;
  k.lt_hi = d.lt_hi;
  k.k_hi = d.k_hi;
  k.k_lo = d.k_lo;
  k.fT = d.fT;

  const long ngroups = (static_cast<long>(V) + kVec - 1) / kVec;
  const long ntiles = (ngroups + kTile - 1) / kTile;
  const long tiles_per = P.groups_per_draw / kTile;
  long tlo = static_cast<long>(s2) * tiles_per;
  long thi = tlo + tiles_per;
  if (tlo > ntiles) tlo = ntiles;
  if (thi > ntiles) thi = ntiles;
  double* table = P.draw_mass + static_cast<long>(b) * ntiles;
  tile_masses<T, kAligned>(mode, drawT, drawD, k, tlo, thi, ngroups, V, table);
  __threadfence();  // this block's tiles are published before its ticket
  __syncthreads();
  __shared__ int sm_last;
  if (tid == 0) {
    const unsigned old = atomicAdd(P.draw_ticket + b, 1u);
    sm_last = (old == static_cast<unsigned>(S2 - 1));
    if (sm_last) __threadfence();
  }
  __syncthreads();
  if (!sm_last) return;

  // ---- the block that finishes the sequence locates u * Z ----
  __shared__ long sm_tile;
  __shared__ double sm_tl, sm_Z;
  unsigned extra_bits = 0;
  for (int attempt = 0; attempt < 2; ++attempt) {
    // each thread owns a contiguous run of up to kRun tiles per round, loaded
    // together (independent loads), summed in index order
    constexpr int kRun = 8;
    const long per_round = static_cast<long>(kDrawThreads) * kRun;
    double base = 0.0;  // mass of the rounds before this one
    long found_tile = -1;
    double found_tl = 0.0;
    bool have_last = false;
    long last_tile = -1;
    const double target0 = static_cast<double>(P.u_resample[b]);
    // pass 1: Z (all rounds)
    double Z = 0.0;
    for (long r0 = 0; r0 < ntiles; r0 += per_round) {
      const long a0 = r0 + static_cast<long>(tid) * kRun;
      double v[kRun];
#pragma unroll
      for (int q = 0; q < kRun; ++q) v[q] = (a0 + q < ntiles) ? __ldcg(&table[a0 + q]) : 0.0;
      double mine = 0.0;
#pragma unroll
      for (int q = 0; q < kRun; ++q) mine += v[q];
      double incl, excl, tot;
      block_scan<kDrawThreads>(mine, incl, excl, tot);
      Z += tot;
    }
    if (Z > 0.0 || mode != kDrawResidual) {
      const double target = target0 * Z;
      // pass 2: the round, thread and tile holding u * Z
      for (long r0 = 0; r0 < ntiles; r0 += per_round) {
        const long a0 = r0 + static_cast<long>(tid) * kRun;
        double v[kRun];
#pragma unroll
        for (int q = 0; q < kRun; ++q) v[q] = (a0 + q < ntiles) ? __ldcg(&table[a0 + q]) : 0.0;
        double mine = 0.0;
#pragma unroll
        for (int q = 0; q < kRun; ++q) mine += v[q];
        double incl, excl, tot;
        block_scan<kDrawThreads>(mine, incl, excl, tot);
        if (base + excl <= target && base + incl > target) {
          double acc = base + excl;
#pragma unroll
          for (int q = 0; q < kRun; ++q) {
            if (found_tile < 0 && v[q] > 0.0 && acc + v[q] > target) {
              found_tile = a0 + q;
              found_tl = target - acc;
            }
            acc += v[q];
          }
        }
        // remember the last tile with mass (rounding fallback)
#pragma unroll
        for (int q = 0; q < kRun; ++q)
          if (v[q] > 0.0) {
            have_last = true;
            last_tile = a0 + q;
          }
        base += tot;
      }
      // publish: the owning tile, else the last tile with mass
      __shared__ long sm_found, sm_lastt[kDrawThreads / kWarp];
      if (tid == 0) sm_found = -1;
      __syncthreads();
      if (found_tile >= 0) {
        sm_found = found_tile;
        sm_tl = found_tl;
      }
      const long wl = have_last ? last_tile : -1;
      long m = wl;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, o));
      if ((tid & (kWarp - 1)) == 0) sm_lastt[tid >> 5] = m;
      __syncthreads();
      if (tid == 0) {
        sm_Z = Z;
        if (sm_found >= 0) {
          sm_tile = sm_found;
        } else {
          long lt = -1;
          for (int w = 0; w < kDrawThreads / kWarp; ++w) lt = max(lt, sm_lastt[w]);
          sm_tile = lt;
          sm_tl = INFINITY;  // the tile's last index with mass
        }
      }
      __syncthreads();
      break;
    }
    // zero residual mass (reachable only through rounding): draw from q_n,
    // this block alone recomputing the row's tiles
    mode = kDrawTarget;
    extra_bits |= kStatZeroMass;
    tile_masses<T, kAligned>(mode, drawT, drawD, k, 0, ntiles, ngroups, V, table);
    __threadfence();
    __syncthreads();
  }

  // the owning tile: one group per lane, warp 0 scans it in index order
  if (tid < kWarp) {
    const long tile = sm_tile;
    const int token = (tile >= 0) ? scan_tile<T, kAligned>(mode, drawT, drawD, k, tile, ngroups, V, sm_tl)
                                  : -1;
    if (tid == 0) {
      P.out_tokens[bo + n] = token;
      P.resid_mass[b] = sm_Z;
      if (extra_bits) atomicOr(P.status, extra_bits);
      P.draw_ticket[b] = 0u;  // ready for the next launch
    }
  }
}

}  // namespace specverify
