// Fused speculative-sampling verification kernel for sm_100a.
//
// One thread-block cluster of C CTAs owns one position (b, j), j = 0..gamma,
// of one sequence: target row (b, j) and, for j < gamma, draft row (b, j).
// Each CTA owns a contiguous slice of the vocabulary of both rows.
//
//   phase 1  single streaming pass over the slice with 128-bit coalesced
//            loads; online (max, sum of exp) per thread, reduced per CTA and
//            combined across the cluster through distributed shared memory
//            ("softmax statistics", step 1 of the round);
//   phase 2  rank 0 forms q(t), p(t) and the ratio for the position's draft
//            token and records accept / reject (step 2, min(1, q/p));
//   phase 3  an atomic ticket per sequence elects the cluster that finishes
//            last; it scans the gamma decisions with a warp ballot to find
//            the first rejection n (step 3);
//   phase 4  that cluster re-reads one row pair (n < gamma: max(0, q_n - p_n))
//            or one row (n == gamma: q_gamma) - rows that the sequence's other
//            clusters have just streamed, so they come from L2 - sums the
//            mass per warp and per CTA, exchanges the CTA sums through
//            distributed shared memory, and the CTA and warp that hold
//            u * Z locate the drawn token with a warp prefix scan (step 4).
//
// Pages (title, section): "Speculative decoding - the small model writes first
// and the big model checks", section 1 (rule); "Speculative decoding: how to
// run big models fast", section "How it works" (steps, bonus token, 1..gamma+1
// tokens per call, temperature).
//
// Numerics: exponentials are base 2 with log2(e)/T split into two floats
// (c_hi + c_lo, c_lo > 0) so that the argument d * c carries no systematic
// rounding of the constant; per-thread sums are fp32, everything above a
// thread (warp, CTA, cluster, ratio, CDF positions) is fp64.  In the residual
// q - p is formed as p * (2^L - 1) with L = log2(q/p) computed from the logit
// difference, which keeps it accurate where q and p nearly cancel.
//
// No thread ever waits on another cluster: cross-cluster hand-off is a ticket
// (atomicAdd), never a spin.  Data errors set bits of a status word.
#pragma once

#include <cooperative_groups.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cfloat>
#include <cstdint>

namespace specverify {

namespace cg = cooperative_groups;

constexpr int kWarp = 32;
constexpr int kMaxCluster = 8;

// per-position decision flags
enum : int { kFlagReject = 0, kFlagAccept = 1, kFlagTokenRange = 2, kFlagNonFinite = 3 };
// status word bits
enum : unsigned { kStatTokenRange = 1u, kStatNonFinite = 2u, kStatZeroMass = 4u };
// what the finishing cluster draws from
enum : int { kDrawResidual = 0, kDrawTarget = 1, kDrawNone = 2 };

struct RowStat {
  double sum;  // sum_i 2^((x_i - max) * c)
  float max;   // max_i x_i
  int valid;   // 1 if the row is finite with at least one finite entry
};

struct PosInfo {
  double q_tok;
  double p_tok;
  double ratio;
  int flag;
  int pad;
};

struct Params {
  const void* target;        // [B, G+1, V]
  const void* draft;         // [B, G, V]
  const int32_t* tokens;     // [B, G]
  const float* u_accept;     // [B, G]
  const float* u_resample;   // [B]
  int32_t* out_tokens;       // [B, G+1]
  int32_t* out_num_accepted; // [B]
  RowStat* tstat;            // [B*(G+1)]
  RowStat* dstat;            // [B*G]
  PosInfo* pos;              // [B*G]
  double* resid_mass;        // [B]
  unsigned* ticket;          // [B], zero between launches
  unsigned* status;          // [1]
  int batch, gamma, vocab;
  int groups_per_cta;        // 16-byte groups of the vocabulary per CTA
  float c_hi, c_lo;          // log2(e)/T = c_hi + c_lo, c_lo > 0
  double c;                  // log2(e)/T
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

// d * log2(e)/T with the constant carried in two parts; c_lo > 0 keeps
// d = -inf mapping to -inf (never inf * 0)
__device__ __forceinline__ float scaled(float d, float c_hi, float c_lo) {
  return fmaf(d, c_hi, d * c_lo);
}

// ---------------------------------------------------------------------------
// phase 1: online softmax statistics
// ---------------------------------------------------------------------------

template <typename T>
__device__ __forceinline__ void accumulate_group(const uint4& v, float& m, float& s, float c_hi,
                                                 float c_lo) {
  constexpr int kVec = Elem<T>::kVec;
  float x[kVec];
  Elem<T>::unpack(v, x);
  float cm = x[0];
#pragma unroll
  for (int k = 1; k < kVec; ++k) cm = fmaxf(cm, x[k]);
  if (cm > m) {
    // (m - cm) is -inf while m is -inf: the factor is 0 and s stays 0 (or NaN)
    s *= ex2(scaled(m - cm, c_hi, c_lo));
    m = cm;
  }
  const float ms = (m == -INFINITY) ? 0.f : m;
  float acc = 0.f;
#pragma unroll
  for (int k = 0; k < kVec; ++k) acc += ex2(scaled(x[k] - ms, c_hi, c_lo));
  s += acc;
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

// contiguous group range [lo, hi) of warp `w` inside the CTA range [clo, chi)
__device__ __forceinline__ void warp_range(long clo, long chi, int w, int nwarps, long& lo,
                                           long& hi) {
  long n = chi - clo;
  long per = (n + nwarps - 1) / nwarps;
  lo = clo + per * w;
  hi = lo + per;
  if (lo > chi) lo = chi;
  if (hi > chi) hi = chi;
}

struct __align__(16) CtaStats {
  double sT, sD;
  float mT, mD;
  int pad[2];
};

struct __align__(16) Bcast {
  double sT, sD;       // row sums of the rows drawn from
  float mT, mD;        // row maxima
  int last;            // this cluster finishes the sequence
  int n;               // accepted drafts
  int mode;            // kDraw*
  int trow, drow;      // target / draft position of the draw (drow < 0: none)
  unsigned stat_bits;  // status bits to raise
  int pad[2];
};

struct __align__(16) CtaMass {
  double z;     // residual mass of the CTA slice
  int last_pos; // last index with r > 0 in the slice, -1 if none
  int pad;
};

// ---------------------------------------------------------------------------
// phase 4 helpers: residual mass of one group
// ---------------------------------------------------------------------------

struct DrawConsts {
  float c_hi, c_lo;
  float mT, mD;      // row maxima
  float invST, invSD;
  float k_hi, k_lo;  // K = (mT - mD) * c + log2(sT / sD), two-float
};

// r for the VEC elements of one group: residual max(0, q - p) or target q
template <typename T, int kMode>
__device__ __forceinline__ void group_mass(const uint4& vt, const uint4& vd, const DrawConsts& k,
                                           float (&r)[Elem<T>::kVec]) {
  constexpr int kVec = Elem<T>::kVec;
  float xt[kVec];
  Elem<T>::unpack(vt, xt);
  if constexpr (kMode == kDrawTarget) {
#pragma unroll
    for (int e = 0; e < kVec; ++e) r[e] = ex2(scaled(xt[e] - k.mT, k.c_hi, k.c_lo)) * k.invST;
  } else {
    float xd[kVec];
    Elem<T>::unpack(vd, xd);
#pragma unroll
    for (int e = 0; e < kVec; ++e) {
      const float q = ex2(scaled(xt[e] - k.mT, k.c_hi, k.c_lo)) * k.invST;
      const float p = ex2(scaled(xd[e] - k.mD, k.c_hi, k.c_lo)) * k.invSD;
      float res;
      if (!(q > 0.f)) {
        res = 0.f;                     // target gives the token no mass
      } else if (xd[e] == -INFINITY) {
        res = q;                       // draft gives it none: all of q is residual
      } else {
        // L = log2(q/p) from the logit difference (exact for bf16 inputs)
        const float dx = xt[e] - xd[e];
        const float L = fmaf(dx, k.c_hi, -k.k_hi) + fmaf(dx, k.c_lo, -k.k_lo);
        if (!(L > 0.f)) {
          res = 0.f;
        } else if (L >= 1.f) {
          res = q - p;                 // q >= 2p: no cancellation
        } else {
          // 2^L - 1 = e^y - 1, y = L ln 2 in (0, 0.694): Taylor series to y^10
          const float y = L * 0.69314718055994531f;
          float t = 2.755731922398589e-7f;           // 1/10!
          t = fmaf(t, y, 2.755731922398589e-6f);     // 1/9!
          t = fmaf(t, y, 2.480158730158730e-5f);     // 1/8!
          t = fmaf(t, y, 1.984126984126984e-4f);     // 1/7!
          t = fmaf(t, y, 1.388888888888889e-3f);     // 1/6!
          t = fmaf(t, y, 8.333333333333333e-3f);     // 1/5!
          t = fmaf(t, y, 4.166666666666667e-2f);     // 1/4!
          t = fmaf(t, y, 1.666666666666667e-1f);     // 1/3!
          t = fmaf(t, y, 0.5f);                      // 1/2!
          t = fmaf(t, y, 1.0f);                      // 1/1!
          res = p * (t * y);
        }
      }
      r[e] = res;
    }
  }
}

// ---------------------------------------------------------------------------
// the kernel
// ---------------------------------------------------------------------------

template <typename T, int NT, bool kAligned>
__global__ void __launch_bounds__(NT) verify_kernel(const Params P) {
  constexpr int kVec = Elem<T>::kVec;
  constexpr int kNW = NT / kWarp;
  constexpr int kUnroll = 4;

  cg::cluster_group cluster = cg::this_cluster();
  const int C = static_cast<int>(cluster.num_blocks());
  const int rank = static_cast<int>(cluster.block_rank());
  const int tid = threadIdx.x;
  const int lane = tid & (kWarp - 1);
  const int warp = tid >> 5;

  const int G = P.gamma;
  const int V = P.vocab;
  const long position = static_cast<long>(blockIdx.x) / C;  // b * (G+1) + j
  const int b = static_cast<int>(position / (G + 1));
  const int j = static_cast<int>(position - static_cast<long>(b) * (G + 1));
  const bool has_draft = j < G;

  const T* rowT = static_cast<const T*>(P.target) + position * V;
  const T* rowD = has_draft
                      ? static_cast<const T*>(P.draft) + (static_cast<long>(b) * G + j) * V
                      : nullptr;

  const long ngroups = (static_cast<long>(V) + kVec - 1) / kVec;
  long clo = static_cast<long>(rank) * P.groups_per_cta;
  long chi = clo + P.groups_per_cta;
  if (clo > ngroups) clo = ngroups;
  if (chi > ngroups) chi = ngroups;
  long wlo, whi;
  warp_range(clo, chi, warp, kNW, wlo, whi);

  __shared__ float sm_max[2][kNW];
  __shared__ double sm_sum[2][kNW];
  __shared__ CtaStats part;
  __shared__ Bcast bc;
  __shared__ CtaMass mass;
  __shared__ double sm_wz[kNW];
  __shared__ int sm_wlast[kNW];
  __shared__ int sm_owner_warp;
  __shared__ double sm_target_local;

  // ---------------- phase 1: streaming statistics ----------------
  const float c_hi = P.c_hi, c_lo = P.c_lo;
  float mT = -INFINITY, sT = 0.f, mD = -INFINITY, sD = 0.f;
  for (long g0 = wlo + lane; g0 < whi; g0 += static_cast<long>(kWarp) * kUnroll) {
    uint4 vt[kUnroll], vd[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const long g = g0 + static_cast<long>(u) * kWarp;
      if (g < whi) {
        vt[u] = fetch_group<T, kAligned>(rowT, g, V);
        if (has_draft) vd[u] = fetch_group<T, kAligned>(rowD, g, V);
      }
    }
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const long g = g0 + static_cast<long>(u) * kWarp;
      if (g < whi) {
        accumulate_group<T>(vt[u], mT, sT, c_hi, c_lo);
        if (has_draft) accumulate_group<T>(vd[u], mD, sD, c_hi, c_lo);
      }
    }
  }

  // CTA reduction: max first, then each thread rescales its sum to the CTA max
  {
    const float wT = warp_max(mT), wD = warp_max(mD);
    if (lane == 0) {
      sm_max[0][warp] = wT;
      sm_max[1][warp] = wD;
    }
    __syncthreads();
    float McT = sm_max[0][0], McD = sm_max[1][0];
#pragma unroll
    for (int w = 1; w < kNW; ++w) {
      McT = fmaxf(McT, sm_max[0][w]);
      McD = fmaxf(McD, sm_max[1][w]);
    }
    // s * 2^((m - M) c); a thread with m = -inf holds s = 0 (or NaN, which propagates)
    const float fT = (mT == -INFINITY) ? 0.f : ex2(scaled(mT - McT, c_hi, c_lo));
    const float fD = (mD == -INFINITY) ? 0.f : ex2(scaled(mD - McD, c_hi, c_lo));
    const double zT = warp_sum(static_cast<double>(sT) * static_cast<double>(fT));
    const double zD = warp_sum(static_cast<double>(sD) * static_cast<double>(fD));
    if (lane == 0) {
      sm_sum[0][warp] = zT;
      sm_sum[1][warp] = zD;
    }
    __syncthreads();
    if (tid == 0) {
      double a = 0.0, d = 0.0;
      for (int w = 0; w < kNW; ++w) {
        a += sm_sum[0][w];
        d += sm_sum[1][w];
      }
      part.sT = a;
      part.sD = d;
      part.mT = McT;
      part.mD = McD;
    }
  }
  cluster.sync();  // (1) every CTA's partial statistics are visible

  // ---------------- phases 2-3: rank 0 decides, takes the ticket ----------------
  if (rank == 0 && warp == 0) {
    int last = 0;
    if (lane == 0) {
      // combine the cluster's partials in rank order (fp64)
      double ST = 0.0, SD = 0.0;
      float MT = -INFINITY, MD = -INFINITY;
      for (int r = 0; r < C; ++r) {
        const CtaStats* pr = cluster.map_shared_rank(&part, r);
        MT = fmaxf(MT, pr->mT);
        MD = fmaxf(MD, pr->mD);
      }
      for (int r = 0; r < C; ++r) {
        const CtaStats* pr = cluster.map_shared_rank(&part, r);
        const float mt = pr->mT, md = pr->mD;
        const double st = pr->sT, sd = pr->sD;
        ST += (mt == -INFINITY) ? st * 0.0 : st * exp2((static_cast<double>(mt) - MT) * P.c);
        SD += (md == -INFINITY) ? sd * 0.0 : sd * exp2((static_cast<double>(md) - MD) * P.c);
      }
      const int validT = (MT != -INFINITY) && isfinite(ST) && ST > 0.0;
      P.tstat[position] = RowStat{ST, MT, validT};
      if (has_draft) {
        const long pj = static_cast<long>(b) * G + j;
        const int validD = (MD != -INFINITY) && isfinite(SD) && SD > 0.0;
        P.dstat[pj] = RowStat{SD, MD, validD};
        PosInfo info{0.0, 0.0, 0.0, kFlagReject, 0};
        const int t = P.tokens[pj];
        if (t < 0 || t >= V) {
          info.flag = kFlagTokenRange;
        } else if (!validT || !validD) {
          info.flag = kFlagNonFinite;
        } else {
          const double xt = static_cast<double>(Elem<T>::load1(rowT, t));
          const double xd = static_cast<double>(Elem<T>::load1(rowD, t));
          const double lq = (xt - MT) * P.c - log2(ST);  // log2 q(t)
          const double lp = (xd - MD) * P.c - log2(SD);  // log2 p(t)
          info.q_tok = exp2(lq);
          info.p_tok = exp2(lp);
          if (!(info.q_tok > 0.0)) info.ratio = 0.0;
          else if (!(info.p_tok > 0.0)) info.ratio = INFINITY;
          else info.ratio = exp2(lq - lp);
          const double u = static_cast<double>(P.u_accept[pj]);
          info.flag = (u < info.ratio) ? kFlagAccept : kFlagReject;
        }
        P.pos[pj] = info;
      }
      __threadfence();
      const unsigned old = atomicAdd(P.ticket + b, 1u);
      last = (old == static_cast<unsigned>(G)) ? 1 : 0;
      if (last) __threadfence();
    }
    last = __shfl_sync(0xffffffffu, last, 0);
    Bcast out{};
    out.last = last;
    if (last) {
      // first rejection and any data error, by warp ballot over the flags
      int n = G;
      unsigned stat_bits = 0;
      for (int base = 0; base < G; base += kWarp) {
        const int jj = base + lane;
        int f = kFlagAccept;
        if (jj < G) f = __ldcg(&P.pos[static_cast<long>(b) * G + jj].flag);
        const unsigned rej = __ballot_sync(0xffffffffu, f == kFlagReject);
        const unsigned tok = __ballot_sync(0xffffffffu, f == kFlagTokenRange);
        const unsigned bad = __ballot_sync(0xffffffffu, f == kFlagNonFinite);
        if (tok) stat_bits |= kStatTokenRange;
        if (bad) stat_bits |= kStatNonFinite;
        if (rej && n == G) n = base + __ffs(rej) - 1;
      }
      if (lane == 0) {
        if (!__ldcg(&P.tstat[static_cast<long>(b) * (G + 1) + G].valid)) stat_bits |= kStatNonFinite;
        out.n = n;
        out.stat_bits = stat_bits;
        if (stat_bits) {
          out.mode = kDrawNone;
        } else {
          const long tr = static_cast<long>(b) * (G + 1) + n;
          out.trow = n;
          out.mT = __ldcg(&P.tstat[tr].max);
          out.sT = __ldcg(&P.tstat[tr].sum);
          if (n < G) {
            const long dr = static_cast<long>(b) * G + n;
            out.mode = kDrawResidual;
            out.drow = n;
            out.mD = __ldcg(&P.dstat[dr].max);
            out.sD = __ldcg(&P.dstat[dr].sum);
          } else {
            out.mode = kDrawTarget;
            out.drow = -1;
          }
        }
      }
      // broadcast lane 0's decision to the other lanes
      out.n = __shfl_sync(0xffffffffu, out.n, 0);
      out.stat_bits = __shfl_sync(0xffffffffu, out.stat_bits, 0);
      out.mode = __shfl_sync(0xffffffffu, out.mode, 0);
      out.trow = __shfl_sync(0xffffffffu, out.trow, 0);
      out.drow = __shfl_sync(0xffffffffu, out.drow, 0);
      out.mT = __shfl_sync(0xffffffffu, out.mT, 0);
      out.mD = __shfl_sync(0xffffffffu, out.mD, 0);
      out.sT = __shfl_sync(0xffffffffu, out.sT, 0);
      out.sD = __shfl_sync(0xffffffffu, out.sD, 0);
    }
    // push the decision into every CTA of the cluster
    if (lane < C) *cluster.map_shared_rank(&bc, lane) = out;
  }
  cluster.sync();  // (2) the decision is in every CTA's shared memory

  if (!bc.last) return;  // cluster-uniform

  // ---------------- phase 4: the finishing cluster draws the token ----------------
  const float u_res = P.u_resample[b];
  int mode = bc.mode;
  const int n = bc.n;
  if (mode == kDrawNone) {
    if (rank == 0 && tid == 0) {
      int32_t* outt = P.out_tokens + static_cast<long>(b) * (G + 1);
      for (int k = 0; k <= G; ++k) outt[k] = -1;
      P.out_num_accepted[b] = 0;
      P.resid_mass[b] = NAN;
      atomicOr(P.status, bc.stat_bits);
      P.ticket[b] = 0u;
    }
    return;  // no CTA reads another's shared memory after barrier (2)
  }

  const T* drawT = static_cast<const T*>(P.target) + (static_cast<long>(b) * (G + 1) + bc.trow) * V;
  const T* drawD = (bc.drow >= 0)
                       ? static_cast<const T*>(P.draft) + (static_cast<long>(b) * G + bc.drow) * V
                       : nullptr;
  DrawConsts k;
  k.c_hi = c_hi;
  k.c_lo = c_lo;
  k.mT = bc.mT;
  k.mD = bc.mD;
  k.invST = static_cast<float>(1.0 / bc.sT);
  k.invSD = static_cast<float>(1.0 / bc.sD);
  {
    const double K = (static_cast<double>(bc.mT) - bc.mD) * P.c + log2(bc.sT / bc.sD);
    k.k_hi = static_cast<float>(K);
    k.k_lo = static_cast<float>(K - static_cast<double>(k.k_hi));
  }
  unsigned extra_bits = 0;
  double Z = 0.0, target = 0.0;
  int owner = -1, last_all = -1;
  double prefix_owner = 0.0;

  for (int attempt = 0; attempt < 2; ++attempt) {
    // pass A: mass per warp (contiguous warp ranges) and per CTA
    double lz = 0.0;
    int llast = -1;
    for (long g0 = wlo + lane; g0 < whi; g0 += static_cast<long>(kWarp) * kUnroll) {
      uint4 vt[kUnroll], vd[kUnroll];
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
        const long g = g0 + static_cast<long>(u) * kWarp;
        if (g < whi) {
          vt[u] = fetch_group<T, kAligned>(drawT, g, V);
          vd[u] = (mode == kDrawResidual) ? fetch_group<T, kAligned>(drawD, g, V) : vt[u];
        }
      }
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
        const long g = g0 + static_cast<long>(u) * kWarp;
        if (g < whi) {
          float r[kVec];
          if (mode == kDrawResidual) group_mass<T, kDrawResidual>(vt[u], vd[u], k, r);
          else group_mass<T, kDrawTarget>(vt[u], vd[u], k, r);
          float gs = 0.f;
#pragma unroll
          for (int e = 0; e < kVec; ++e) {
            gs += r[e];
            if (r[e] > 0.f) llast = static_cast<int>(g * kVec + e);
          }
          lz += static_cast<double>(gs);
        }
      }
    }
    const double wz = warp_sum(lz);
    const int wl = warp_maxi(llast);
    if (lane == 0) {
      sm_wz[warp] = wz;
      sm_wlast[warp] = wl;
    }
    __syncthreads();
    if (tid == 0) {
      double z = 0.0;
      int lp = -1;
      for (int w = 0; w < kNW; ++w) {
        z += sm_wz[w];
        lp = max(lp, sm_wlast[w]);
      }
      mass.z = z;
      mass.last_pos = lp;
    }
    cluster.sync();  // (3) CTA masses visible
    // every thread forms the same cluster totals in rank order
    Z = 0.0;
    last_all = -1;
    for (int r = 0; r < C; ++r) {
      const CtaMass* pr = cluster.map_shared_rank(&mass, r);
      Z += pr->z;
      last_all = max(last_all, pr->last_pos);
    }
    if (Z > 0.0 || mode != kDrawResidual) break;
    // zero residual mass (rounding only): draw from q_n instead
    mode = kDrawTarget;
    extra_bits |= kStatZeroMass;
    cluster.sync();  // (3b) nobody still reads the masses about to be rewritten
  }

  target = static_cast<double>(u_res) * Z;
  {
    double pre = 0.0;
    for (int r = 0; r < C; ++r) {
      const CtaMass* pr = cluster.map_shared_rank(&mass, r);
      if (pr->z > 0.0 && pre + pr->z > target) {
        owner = r;
        prefix_owner = pre;
        break;
      }
      pre += pr->z;
    }
  }

  if (owner == rank) {
    if (tid == 0) {
      const double tl = target - prefix_owner;
      double pre = 0.0;
      int ow = -1;
      for (int w = 0; w < kNW; ++w) {
        if (sm_wz[w] > 0.0 && pre + sm_wz[w] > tl) {
          ow = w;
          break;
        }
        pre += sm_wz[w];
      }
      sm_owner_warp = ow;
      sm_target_local = tl - pre;
    }
    __syncthreads();
    const int ow = sm_owner_warp;
    if (ow < 0) {
      if (tid == 0) P.out_tokens[static_cast<long>(b) * (G + 1) + n] = mass.last_pos;
    } else if (warp == ow) {
      // pass B: ordered scan of this warp's range
      const double tw = sm_target_local;
      double running = 0.0;
      int token = -1;
      for (long g0 = wlo; g0 < whi && token < 0; g0 += kWarp) {
        const long g = g0 + lane;
        float r[kVec];
#pragma unroll
        for (int e = 0; e < kVec; ++e) r[e] = 0.f;
        if (g < whi) {
          const uint4 vt = fetch_group<T, kAligned>(drawT, g, V);
          const uint4 vd = (mode == kDrawResidual) ? fetch_group<T, kAligned>(drawD, g, V) : vt;
          if (mode == kDrawResidual) group_mass<T, kDrawResidual>(vt, vd, k, r);
          else group_mass<T, kDrawTarget>(vt, vd, k, r);
        }
        float gs = 0.f;
#pragma unroll
        for (int e = 0; e < kVec; ++e) gs += r[e];
        const double ls = static_cast<double>(gs);
        double incl = ls;
#pragma unroll
        for (int o = 1; o < kWarp; o <<= 1) {
          const double y = __shfl_up_sync(0xffffffffu, incl, o);
          if (lane >= o) incl += y;
        }
        const double tot = __shfl_sync(0xffffffffu, incl, kWarp - 1);
        if (running + tot > tw) {
          const unsigned hit = __ballot_sync(0xffffffffu, ls > 0.0 && running + incl > tw);
          const int L = hit ? __ffs(hit) - 1 : kWarp - 1;
          int found = -1;
          if (lane == L) {
            double acc = running + (incl - ls);
            int lastpos = -1;
#pragma unroll
            for (int e = 0; e < kVec; ++e) {
              if (r[e] > 0.f) {
                lastpos = static_cast<int>(g * kVec + e);
                acc += static_cast<double>(r[e]);
                if (found < 0 && acc > tw) found = lastpos;
              }
            }
            if (found < 0) found = lastpos;  // rounding between the two sums
          }
          token = __shfl_sync(0xffffffffu, found, L);
        }
        running += tot;
      }
      if (token < 0) token = sm_wlast[ow];  // rounding: u * Z beyond this warp's scan
      if (lane == 0) P.out_tokens[static_cast<long>(b) * (G + 1) + n] = token;
    }
  }
  if (owner < 0 && rank == 0 && tid == 0) {
    P.out_tokens[static_cast<long>(b) * (G + 1) + n] = last_all;  // rounding: u * Z >= Z
  }
  if (rank == 0 && tid == 0) {
    int32_t* outt = P.out_tokens + static_cast<long>(b) * (G + 1);
    const int32_t* drafts = P.tokens + static_cast<long>(b) * G;
    for (int q = 0; q < n; ++q) outt[q] = drafts[q];
    for (int q = n + 1; q <= G; ++q) outt[q] = -1;
    P.out_num_accepted[b] = n;
    P.resid_mass[b] = Z;
    if (extra_bits) atomicOr(P.status, extra_bits);
    P.ticket[b] = 0u;  // ready for the next launch
  }
  cluster.sync();  // (4) keep shared memory alive until every remote read is done
}

}  // namespace specverify
