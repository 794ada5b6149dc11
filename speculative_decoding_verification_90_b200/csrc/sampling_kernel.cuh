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
//   select_kernel  one block per row: maximum and first argmax; count-based
//                  radix select of the top-k threshold; for top-p, the entries
//                  above a count-selected candidate key gathered into shared
//                  memory and a binary search over keys on their fp64 masses
//                  (whole-row passes when the boundary lies below the
//                  candidates); the log-normaliser of the kept entries.
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

constexpr int kSelThreads = 512;
constexpr int kSelWarps = kSelThreads / kWarp;
constexpr int kCand = 12288;         // top-p candidates kept in shared memory
constexpr int kCandSmem = kCand * 8; // their keys and weights (dynamic shared memory)
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
};

// ---------------------------------------------------------------------------
// helpers
// ---------------------------------------------------------------------------

// order-preserving unsigned key of a float (NaN excluded by the callers)
__device__ __forceinline__ unsigned fkey(float x) {
  const unsigned u = __float_as_uint(x);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
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

// The count-based radix select: the `rank`-th largest key (1-based) among the
// row's entries with key >= `floor_key`, for keys whose low `low_bits` bits are
// zero (bf16 values widened to float).  Histograms of 256 bins per 8-bit digit
// in shared memory; each warp adds a bin's lanes once (match_any).  Returns the
// key, and in *count_eq the number of entries equal to it.
template <typename T>
__device__ unsigned radix_select(const T* row, int V, unsigned floor_key, long rank, int low_bits,
                                 int* hist, int* count_eq) {
  const int lane = threadIdx.x & (kWarp - 1);
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
  for (int shift = 24; shift >= low_bits; shift -= 8) {
    for (int i = threadIdx.x; i < 256; i += blockDim.x) hist[i] = 0;
    __syncthreads();
    const unsigned prefix = s_prefix, mask = s_mask;
    const long nV = V;
    for (long base = 0; base < nV; base += blockDim.x) {
      const long i = base + threadIdx.x;
      bool in = false;
      unsigned bin = 0;
      if (i < nV) {
        const unsigned k = fkey(elem<T>(row, i));
        in = k >= floor_key && (k & mask) == prefix;
        bin = (k >> shift) & 255u;
      }
      const unsigned act = __ballot_sync(0xffffffffu, in);
      if (in) {
        const unsigned grp = __match_any_sync(act, bin);
        if (lane == __ffs(grp) - 1) atomicAdd(&hist[bin], __popc(grp));
      }
    }
    __syncthreads();
    if (threadIdx.x == 0) {
      long need = s_rank, cum = 0;
      int sel = 0;
      for (int b = 255; b >= 0; --b) {
        if (cum + hist[b] >= need) {
          sel = b;
          break;
        }
        cum += hist[b];
      }
      s_rank = need - cum;
      s_prefix = prefix | (static_cast<unsigned>(sel) << shift);
      s_mask = mask | (255u << shift);
      s_eq = hist[sel];
    }
    __syncthreads();
  }
  *count_eq = s_eq;
  return s_prefix;
}

// sum over the row of 2^(x c - o) for entries with key >= lo (and key < hi
// when hi != 0), per thread in fp32, over the block in fp64
template <typename T>
__device__ double masked_mass(const T* row, int V, unsigned lo, unsigned hi, float c_hi,
                              float c_lo, float o, double* sm) {
  float s = 0.f;
  for (long i = threadIdx.x; i < V; i += blockDim.x) {
    const float x = elem<T>(row, i);
    const unsigned k = fkey(x);
    if (k >= lo && (hi == 0u || k < hi)) s += ex2(specverify::arg2(x, c_hi, c_lo, o));
  }
  return block_sum<kSelThreads>(static_cast<double>(s), sm);
}

// ---------------------------------------------------------------------------
// kernel 1: per-row adjusted distribution
// ---------------------------------------------------------------------------

__device__ __forceinline__ void put_row(const SampParams& P, long r, long nT, const SampRow& v) {
  P.rows[r] = v;
  const specverify::RowStat st{v.l2, v.valid, v.kept};
  if (r < nT) P.tstat[r] = st;
  else P.dstat[r - nT] = st;
}

template <typename T>
__global__ void __launch_bounds__(kSelThreads) select_kernel(const SampParams P) {
  __shared__ int hist[256];
  __shared__ double smd[kSelWarps];
  __shared__ unsigned smu[kSelWarps];
  __shared__ int smi[kSelWarps];
  extern __shared__ unsigned cand_smem[];  // kCand keys, then kCand weights
  unsigned* cand_key = cand_smem;
  float* cand_w = reinterpret_cast<float*>(cand_smem + kCand);
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

  // pass A: maximum, first argmax, invalid entries
  float mx = -INFINITY;
  int am = 0x7fffffff;
  bool bad = false;
  for (long i = threadIdx.x; i < V; i += blockDim.x) {
    const float x = elem<T>(row, i);
    bad |= (x != x) || x == INFINITY;
    if (x > mx) {
      mx = x;
      am = static_cast<int>(i);
    }
  }
  const unsigned kmax = block_max_u<kSelThreads>(bad ? 0u : fkey(mx), smu);
  const bool any_bad = __syncthreads_or(bad);
  const float gmx = key_value(kmax);
  const int arg = block_min_i<kSelThreads>(mx == gmx ? am : 0x7fffffff, smi);
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
  float c_hi, c_lo;
  double c;
  temp_consts(temp, c_hi, c_lo, c);
  const float o = gmx * c_hi;  // weights 2^(x c - o) are at most about 1

  // top-k threshold
  unsigned theta = 0u;
  int eq = 0;
  if (P.top_k > 0 && P.top_k < V) theta = radix_select<T>(row, V, 0u, P.top_k, low_bits, hist, &eq);

  // nucleus threshold
  float margin = INFINITY;
  bool z_known = false;
  double Z_kept = 0.0;
  if (P.top_p < 1.0) {
    // candidate key vc: the kCand-th largest key >= theta (theta itself when
    // fewer entries are kept).  The entries strictly above vc (fewer than
    // kCand) go to shared memory with weights from the double-precision exp2;
    // the entries equal to vc form one group of equal weight.
    unsigned vc = theta;
    {
      int n_ge = 0;
      for (long i = threadIdx.x; i < V; i += blockDim.x) n_ge += fkey(elem<T>(row, i)) >= theta;
      const double nd = block_sum<kSelThreads>(static_cast<double>(n_ge), smd);
      int eq_c = 0;
      if (nd > kCand) vc = radix_select<T>(row, V, theta, kCand, low_bits, hist, &eq_c);
    }
    if (threadIdx.x == 0) cand_n = 0;
    __syncthreads();
    const int lane = threadIdx.x & (kWarp - 1);
    const double od = static_cast<double>(gmx) * c;
    int n_eq = 0;
    float tail = 0.f;  // entries theta <= key < vc (all lighter than every candidate)
    for (long base = 0; base < V; base += blockDim.x) {
      const long i = base + threadIdx.x;
      float x = -INFINITY;
      unsigned k = 0u;
      if (i < V) {
        x = elem<T>(row, i);
        k = fkey(x);
      }
      const bool take = i < V && k > vc && k >= theta;
      n_eq += (i < V && k == vc && k >= theta);
      if (i < V && k < vc && k >= theta) tail += ex2(specverify::arg2(x, c_hi, c_lo, o));
      const unsigned m = __ballot_sync(0xffffffffu, take);
      int at = 0;
      if (lane == 0 && m) at = atomicAdd(&cand_n, __popc(m));
      at = __shfl_sync(0xffffffffu, at, 0);
      if (take) {
        const int slot = at + __popc(m & ((1u << lane) - 1u));
        if (slot < kCand) {
          cand_key[slot] = k;
          cand_w[slot] = static_cast<float>(exp2(static_cast<double>(x) * c - od));
        }
      }
    }
    __syncthreads();
    const int nc = min(cand_n, kCand);
    const double n_vc = block_sum<kSelThreads>(static_cast<double>(n_eq), smd);
    const double z_tail = block_sum<kSelThreads>(static_cast<double>(tail), smd) *
                          exp2(static_cast<double>(o) - od);
    // (no entry equals vc when every entry is a candidate: vc may then be a key
    // that decodes to no finite value)
    const float xv = key_value(vc);
    const double w_vc = (n_vc > 0.0 && xv != -INFINITY) ? exp2(static_cast<double>(xv) * c - od) : 0.0;
    // M(>= v) for v >= vc: the candidates at or above v, plus the vc group
    auto mass_ge = [&](unsigned v) -> double {
      double sv = 0.0;
      for (int i = threadIdx.x; i < nc; i += blockDim.x)
        if (cand_key[i] >= v) sv += static_cast<double>(cand_w[i]);
      double t = block_sum<kSelThreads>(sv, smd);
      if (v <= vc) t += n_vc * w_vc;
      return t;
    };
    const double m_vc = mass_ge(vc);
    const double Zk = z_tail + m_vc;   // mass of the entries >= theta
    const double goal = P.top_p * Zk;
    const unsigned step = 1u << low_bits;
    unsigned lo, hi;  // the largest v in [lo, hi] with M(>= v) >= goal
    double m_ge, m_gt;
    if (m_vc >= goal) {
      lo = vc;
      hi = kmax;
      while (lo < hi) {
        const unsigned mid = lo + (((hi - lo) / step + 1) / 2) * step;
        if (mass_ge(mid) >= goal) lo = mid;
        else hi = mid - step;
      }
      m_ge = mass_ge(lo);
      m_gt = (lo >= kmax) ? 0.0 : mass_ge(lo + step);
      Z_kept = m_ge;
      z_known = true;
    } else {
      // the boundary lies below the candidates: whole-row passes (fp32 weights)
      const double sc = exp2(static_cast<double>(o) - od);
      lo = theta;
      hi = vc;
      while (lo < hi) {
        const unsigned mid = lo + (((hi - lo) / step + 1) / 2) * step;
        if (masked_mass<T>(row, V, mid, 0u, c_hi, c_lo, o, smd) * sc >= goal) lo = mid;
        else hi = mid - step;
      }
      m_ge = masked_mass<T>(row, V, lo, 0u, c_hi, c_lo, o, smd) * sc;
      m_gt = masked_mass<T>(row, V, lo + step, 0u, c_hi, c_lo, o, smd) * sc;
    }
    margin = static_cast<float>(fmin(P.top_p - m_gt / Zk, m_ge / Zk - P.top_p));
    theta = max(theta, lo);
  }

  // log-normaliser and size of the kept set
  float s = 0.f;
  int kept = 0;
  for (long i = threadIdx.x; i < V; i += blockDim.x) {
    const float x = elem<T>(row, i);
    if (fkey(x) >= theta && x != -INFINITY) {
      s += ex2(specverify::arg2(x, c_hi, c_lo, o));
      ++kept;
    }
  }
  const double Zs = block_sum<kSelThreads>(static_cast<double>(s), smd);
  const double nk = block_sum<kSelThreads>(static_cast<double>(kept), smd);
  if (threadIdx.x == 0) {
    // log2 sum 2^(x c): from the double-precision candidate masses when the
    // nucleus ends among them, else from this pass
    out.l2 = z_known ? static_cast<double>(gmx) * c + log2(Z_kept) : static_cast<double>(o) + log2(Zs);
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

  // pass 1: the mass of every tile (warp partials, no barrier in the loop)
  double Z = 0.0;
  int last_pos = -1;
  for (int attempt = 0; attempt < 2; ++attempt) {
    int lp = -1;
    for (int t = 0; t < ntiles; ++t) {
      float s = chunk_sum(t, mode, &lp);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
      if (lane == 0) s_part[t][warp] = s;
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
