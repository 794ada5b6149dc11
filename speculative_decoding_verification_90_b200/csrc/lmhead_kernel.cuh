// The LM-head GEMM of the fused verification step, on the 5th-generation
// tensor cores (tcgen05) of sm_100a.
//
// logits[r, v] = sum_k hidden[r, k] * weight[v, k]   (bf16 inputs, fp32 accumulation)
//
// Persistent CTAs (one per SM) walk 128 x 256 tiles of logits (rows x
// vocabulary): TMA loads 128 x 64 and 256 x 64 bf16 tiles (128-byte swizzle)
// into a 4-stage ring of shared memory; one thread issues tcgen05.mma (M = 128,
// N = 256, K = 16) into one of two 256-column accumulators in tensor memory;
// four epilogue warps read the other accumulator back with tcgen05.ld, 32
// columns at a time, each warp its 32 rows (TMEM lanes), while the next
// tile's MMAs run.  The epilogue either
//   - folds the tile into per-row softmax statistics (s = sum 2^(x c - o) with
//     a running offset o, as the streaming statistics kernel does), and picks
//     out the logit at the row's draft token when the token falls in the tile
//     (the logits never reach global memory), or
//   - writes the fp32 logits (the rows the draw needs).
//
// Every wait on an mbarrier is bounded in time (kWaitLimitNs of the global
// nanosecond timer): a wait that runs out sets the CTA's failure flag and its
// thread leaves its loop; the other roles see the flag and stop too.  Before
// the tensor memory is freed, a failed CTA drains what it still has in
// flight: the producer waits (bounded again) for every TMA load it issued
// that the MMA thread had not consumed, and the MMA thread commits its last
// MMAs to a drain barrier and waits for it (bounded).  Then warp 1 frees the
// tensor memory and the error flag reaches the host.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "verify_kernel.cuh"

namespace lmhead {

constexpr int kBM = 128;     // rows per tile (UMMA M)
constexpr int kBN = 256;     // vocabulary columns per tile (UMMA N)
constexpr int kBK = 64;      // K per stage: 64 bf16 = one 128-byte swizzle row
constexpr int kUK = 16;      // K per tcgen05.mma (bf16)
constexpr int kStages = 4;
constexpr int kABytes = kBM * kBK * 2;   // 16 KB
constexpr int kBBytes = kBN * kBK * 2;   // 32 KB
constexpr int kStageBytes = kABytes + kBBytes;
// the epilogue warps' staging buffers for the logits they store: 32 rows x
// kStageLd floats each (rows 16-byte aligned, conflict-free quarter warps)
constexpr int kStageLd = 36;
constexpr int kEpiStageBytes = 32 * kStageLd * 4;
constexpr int kSmemBytes = kStages * kStageBytes + 4 * kEpiStageBytes + 1024;  // + room to align to 1024
constexpr unsigned long long kWaitLimitNs = 2000000000ull;  // 2 s per wait

enum : int { kModeStats = 0, kModeLogits = 1 };

struct LmParams {
  int rows;                 // M: rows of hidden (the first segment)
  int rows2;                // rows of the second hidden tensor (statistics mode; 0: none)
  long row_offset2;         // its first row in the partial / gathered arrays
  int positions2;           // its positions per sequence (rows of one sequence)
  int vocab;                // N: rows of weight
  int hidden;               // K (a multiple of 64)
  int ntiles;               // vocabulary tiles = ceil(vocab / 256)
  int num_sms;              // persistent grid size
  // statistics mode
  specverify::RowPartial* partial;  // [(row_offset + rows) * ntiles]
  long row_offset;
  const int32_t* tokens;    // token whose logit is picked out for row r, or null
  int token_stride;         // row r -> tokens[(r / (G+1)) * G + r % (G+1)] via the two fields
  int positions;            // G + 1 for target rows (the last position has no token), G for draft
  float* gathered;          // [row_offset + rows] logit at the row's token
  float c_hi, c_lo;
  // logits mode; statistics mode: null, or [row_offset + rows, vocab] fp32
  // where the tile's logits are stored as well
  float* logits;            // [rows, vocab] fp32
  float* logits2;           // [rows2, vocab] fp32: the second hidden tensor's
  unsigned* error;          // set when a wait gives up
};

// ---------------------------------------------------------------------------
// PTX wrappers
// ---------------------------------------------------------------------------

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, unsigned count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, unsigned bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ unsigned long long global_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// wait for the phase with the given parity to complete; false once the wait
// has lasted kWaitLimitNs (the timer is read every 256 tries)
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, unsigned parity) {
  const uint32_t a = smem_u32(bar);
  unsigned long long t0 = 0;
  for (unsigned i = 0;; ++i) {
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(done)
        : "r"(a), "r"(parity)
        : "memory");
    if (done) return true;
    if ((i & 255u) == 0u) {
      const unsigned long long now = global_ns();
      if (i == 0u) t0 = now;
      else if (now - t0 > kWaitLimitNs) return false;
    }
  }
}

__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, uint64_t* bar, int x,
                                            int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cta.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], [%2];" ::
          "r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y)
      : "memory");
}

// K-major operand tile with 128-byte swizzle: rows of 128 bytes, 8-row groups
// 1024 bytes apart (stride byte offset), descriptor version 1, swizzle mode 2
__device__ __forceinline__ uint64_t umma_desc(uint32_t saddr) {
  return (static_cast<uint64_t>((saddr >> 4) & 0x3FFFu)) | (static_cast<uint64_t>(1) << 16) |
         (static_cast<uint64_t>(1024 >> 4) << 32) | (static_cast<uint64_t>(1) << 46) |
         (static_cast<uint64_t>(2) << 61);
}

// kind::f16 instruction descriptor: fp32 accumulator, bf16 A and B, both
// K-major, M = 128, N = 256
constexpr uint32_t kIdesc = (1u << 4) | (1u << 7) | (1u << 10) |
                            (static_cast<uint32_t>(kBN >> 3) << 17) |
                            (static_cast<uint32_t>(kBM >> 4) << 24);

__device__ __forceinline__ void umma_f16(uint32_t tmem_d, uint64_t da, uint64_t db, bool accum) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
      "l"(da), "l"(db), "r"(kIdesc), "r"(accum ? 1u : 0u));
}

// arrive on `bar` once every tcgen05.mma issued so far by this thread is done
__device__ __forceinline__ void umma_commit(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
          smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// 32 consecutive fp32 columns of this thread's TMEM lane
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
      "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

// ---------------------------------------------------------------------------
// the epilogue of one tile (one warp: its 32 TMEM lanes = rows q*32 .. q*32+31)
// ---------------------------------------------------------------------------

// The 32 x 32 chunk of fp32 logits of rows r0 .. r0+31 (lane l holds row
// r0 + l's values v[0..31]) and columns c .. c+31, stored to base[row *
// vocab + column] for the rows below nrows and the columns inside the
// vocabulary.  The chunk goes through the warp's staging buffer so that each
// store instruction writes whole 128-byte row segments (8 lanes per row, 4
// rows per instruction) instead of 16 bytes of 32 different rows.  16-byte
// stores when the vocabulary is a multiple of 4 (16-byte aligned rows), else
// one per column.  Streaming stores (evict-first in L2): the logits are read
// back at most once, later, and must not push the operand tiles that
// concurrent CTAs share out of L2.
__device__ __forceinline__ void store_chunk_staged(float* base, long r0, int nrows, int c,
                                                   int vocab, bool vec, const float (&v)[32],
                                                   float* stage) {
  const int lane = threadIdx.x & 31;
  float4* mine = reinterpret_cast<float4*>(stage + lane * kStageLd);
#pragma unroll
  for (int k = 0; k < 8; ++k) mine[k] = make_float4(v[4 * k], v[4 * k + 1], v[4 * k + 2], v[4 * k + 3]);
  __syncwarp();
  const int sub = lane >> 3, col = c + 4 * (lane & 7);
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int rr = 4 * i + sub;
    const float4 x = *reinterpret_cast<const float4*>(stage + rr * kStageLd + 4 * (lane & 7));
    if (rr < nrows) {
      float* out = base + (r0 + rr) * vocab + col;
      if (vec && col + 4 <= vocab) {
        __stcs(reinterpret_cast<float4*>(out), x);
      } else {
        if (col < vocab) __stcs(out, x.x);
        if (col + 1 < vocab) __stcs(out + 1, x.y);
        if (col + 2 < vocab) __stcs(out + 2, x.z);
        if (col + 3 < vocab) __stcs(out + 3, x.w);
      }
    }
  }
  __syncwarp();  // the buffer is rewritten by the next chunk
}

template <int kMode>
__device__ __forceinline__ void epilogue_tile(const LmParams& P, uint32_t acc_addr, int m0, int n0,
                                              int vt, int q, int lane, float* stage) {
  const int r = m0 + q * 32 + lane;
  const uint32_t lane_addr = acc_addr + (static_cast<uint32_t>(q * 32) << 16);
  if constexpr (kMode == kModeStats) {
    int t = -1;
    if (r < P.rows && P.tokens) {
      const int pos = r % P.positions, seq = r / P.positions;
      if (pos < P.token_stride) t = P.tokens[static_cast<long>(seq) * P.token_stride + pos];
    }
    float o = -INFINITY, sum = 0.f, xt = 0.f;
    const bool vec = (P.vocab % 4) == 0;
#pragma unroll 1
    for (int c0 = 0; c0 < kBN; c0 += 32) {
      float v[32];
      tmem_ld32(lane_addr + c0, v);
      if (P.logits)
        store_chunk_staged(P.logits + P.row_offset * P.vocab, m0 + q * 32, P.rows - (m0 + q * 32),
                           n0 + c0, P.vocab, vec, v, stage);
      float cm = -INFINITY;
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        const int col = n0 + c0 + i;
        if (col >= P.vocab) v[i] = -INFINITY;
        if (col == t) xt = v[i];
        cm = fmaxf(cm, v[i]);
      }
      const float on = cm * P.c_hi;
      if (cm != -INFINITY && on > o) {
        sum *= specverify::ex2(o - on);
        o = on;
      }
      if (o != -INFINITY) {
#pragma unroll
        for (int i = 0; i < 32; ++i) sum += specverify::ex2(specverify::arg2(v[i], P.c_hi, P.c_lo, o));
      }
    }
    if (r < P.rows) {
      P.partial[(P.row_offset + r) * P.ntiles + vt] =
          specverify::RowPartial{static_cast<double>(sum), o, 0};
      if (t >= n0 && t < n0 + kBN) P.gathered[P.row_offset + r] = xt;
    }
  } else {
    const bool vec = (P.vocab % 4) == 0;
#pragma unroll 1
    for (int c0 = 0; c0 < kBN; c0 += 32) {
      float v[32];
      tmem_ld32(lane_addr + c0, v);
      store_chunk_staged(P.logits, m0 + q * 32, P.rows - (m0 + q * 32), n0 + c0, P.vocab, vec, v,
                         stage);
    }
  }
}

// ---------------------------------------------------------------------------
// the kernel: persistent, one CTA per SM, tiles in the order (vocabulary tile,
// row tile) with row tiles fastest, so that concurrently running CTAs share a
// weight tile through L2
// ---------------------------------------------------------------------------
//
// warp 0 lane 0: TMA producer over a 4-stage ring, continuous across tiles
// warp 1: allocates 512 TMEM columns (two 256-column accumulators); lane 0
//         issues the MMAs of tile i into accumulator i % 2 once the epilogue of
//         tile i - 2 has released it
// warps 2-5: the epilogue; warp w reads TMEM lanes 32 (w % 4) .. + 31, so the
//         four cover the 128 rows, while the MMAs of the next tile run

constexpr int kPThreads = 192;
constexpr int kAccCols = 2 * kBN;

template <int kMode>
__global__ void __launch_bounds__(kPThreads, 1)
    gemm_kernel(const __grid_constant__ CUtensorMap tm_hidden,
                const __grid_constant__ CUtensorMap tm_hidden2,
                const __grid_constant__ CUtensorMap tm_weight, const LmParams P0) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t full_bar[kStages];
  __shared__ __align__(8) uint64_t empty_bar[kStages];
  __shared__ __align__(8) uint64_t tfull_bar[2];
  __shared__ __align__(8) uint64_t tempty_bar[2];
  __shared__ __align__(8) uint64_t drain_bar;
  __shared__ uint32_t tmem_base_s;
  __shared__ int s_failed;
  __shared__ long s_issued, s_consumed;  // TMA stage loads issued / waited for by the MMA thread

  const int warp = threadIdx.x / 32, lane = threadIdx.x & 31;
  const int tiles1 = (P0.rows + kBM - 1) / kBM;
  const int tiles2 = (P0.rows2 + kBM - 1) / kBM;
  const int n_rt = tiles1 + tiles2;
  const long n_tiles = static_cast<long>(n_rt) * P0.ntiles;
  const int nk = P0.hidden / kBK;
  volatile int* failed = &s_failed;
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull_bar[a], 1);
      mbar_init(&tempty_bar[a], 4);  // one arrival per epilogue warp
    }
    mbar_init(&drain_bar, 1);
    s_failed = 0;
    s_issued = 0;
    s_consumed = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(&tmem_base_s)),
                 "r"(kAccCols));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_s;

  if (warp == 0) {
    if (lane == 0) {
      long it = 0;
      for (long t = blockIdx.x; t < n_tiles && !*failed; t += gridDim.x) {
        const int rt = static_cast<int>(t % n_rt), vt = static_cast<int>(t / n_rt);
        const bool second = rt >= tiles1;
        const CUtensorMap* tm_a = second ? &tm_hidden2 : &tm_hidden;
        const int m0 = (second ? rt - tiles1 : rt) * kBM, n0 = vt * kBN;
        for (int kt = 0; kt < nk; ++kt, ++it) {
          const int s = static_cast<int>(it % kStages);
          if (it >= kStages && !mbar_wait(&empty_bar[s], static_cast<unsigned>((it / kStages) - 1) & 1)) {
            *failed = 1;
            break;
          }
          uint8_t* a = smem + s * kStageBytes;
          mbar_expect_tx(&full_bar[s], kStageBytes);
          tma_load_2d(a, tm_a, &full_bar[s], kt * kBK, m0);
          tma_load_2d(a + kABytes, &tm_weight, &full_bar[s], kt * kBK, n0);
          s_issued = it + 1;
        }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) {
      long it = 0;
      long i = 0;  // this CTA's tile count
      for (long t = blockIdx.x; t < n_tiles && !*failed; t += gridDim.x, ++i) {
        const int acc = static_cast<int>(i & 1);
        if (i >= 2 && !mbar_wait(&tempty_bar[acc], static_cast<unsigned>((i / 2) - 1) & 1)) {
          *failed = 1;
          break;
        }
        tc_fence_after();
        const uint32_t d = tmem + static_cast<uint32_t>(acc * kBN);
        for (int kt = 0; kt < nk; ++kt, ++it) {
          const int s = static_cast<int>(it % kStages);
          if (!mbar_wait(&full_bar[s], static_cast<unsigned>(it / kStages) & 1)) {
            *failed = 1;
            break;
          }
          s_consumed = it + 1;
          tc_fence_after();
          const uint32_t a = smem_u32(smem + s * kStageBytes);
          const uint32_t b = a + kABytes;
#pragma unroll
          for (int k = 0; k < kBK / kUK; ++k)
            umma_f16(d, umma_desc(a + k * kUK * 2), umma_desc(b + k * kUK * 2), kt > 0 || k > 0);
          umma_commit(&empty_bar[s]);  // the stage is free once these MMAs are done
        }
        umma_commit(&tfull_bar[acc]);  // accumulator `acc` holds tile t
      }
    }
    __syncwarp();
  } else {
    const int q = warp % 4;  // TMEM lane quarter of this warp
    float* stage = reinterpret_cast<float*>(smem + kStages * kStageBytes + (warp - 2) * kEpiStageBytes);
    long i = 0;
    for (long t = blockIdx.x; t < n_tiles; t += gridDim.x, ++i) {
      const int acc = static_cast<int>(i & 1);
      bool ok = mbar_wait(&tfull_bar[acc], static_cast<unsigned>(i / 2) & 1);
      ok = __all_sync(0xffffffffu, ok) && !*failed;
      if (!ok) {
        if (lane == 0) *failed = 1;
        break;
      }
      tc_fence_after();
      const int rt = static_cast<int>(t % n_rt), vt = static_cast<int>(t / n_rt);
      const bool second = rt >= tiles1;
      LmParams P = P0;
      if (second) {
        P.rows = P0.rows2;
        P.row_offset = P0.row_offset2;
        P.positions = P0.positions2;
        P.logits = P0.logits2;
      }
      epilogue_tile<kMode>(P, tmem + static_cast<uint32_t>(acc * kBN),
                           (second ? rt - tiles1 : rt) * kBM, vt * kBN, vt, q, lane, stage);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty_bar[acc]);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (*failed) {  // uniform: the flag is read after the barrier
    // drain before the shared memory and the tensor memory are given back:
    // the TMA loads the MMA thread never waited for, then the MMAs issued
    if (threadIdx.x == 0) {
      for (long j = s_consumed; j < s_issued; ++j)
        if (!mbar_wait(&full_bar[j % kStages], static_cast<unsigned>(j / kStages) & 1)) break;
    }
    if (warp == 1 && lane == 0) {
      umma_commit(&drain_bar);
      mbar_wait(&drain_bar, 0);
    }
    tc_fence_before();
    __syncthreads();
    if (threadIdx.x == 0) atomicOr(P0.error, 1u);
  }
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                 "r"(kAccCols));
  }
}

}  // namespace lmhead
