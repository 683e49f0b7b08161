// bsa_predict.cu -- online top-p block-mask prediction on the GPU, straight
// into the CRM form the forward reads.
//
// The block scores and the cut follow "ScalingAttention" Algorithm 1 (sort the
// block scores, accumulate, cut where the cumulative share reaches p: the
// Top-k(S, p) of Eq. 2), applied row by row as online top-p predictors do,
// with a top-p threshold per head (per-head top-p thresholds, as on the
// selective head globalization page).  The block score is the proxy of pooled
// queries and keys:
//   qbar_i = mean of the valid tokens of query block i (kbar_j alike)
//   s_ij = qbar_i . kbar_j / (sqrt(d) * tau_h),   p_ij = softmax_j(s_ij)
// Row i keeps the blocks taken in descending p (ties: lower j first) up to
// and including the one at which the cumulative sum reaches top_p[h]: at
// least one block, all of them if the sum never does.
//
// Launches:
//   1. pool:        one CTA per (b, h, block); fp32 means of the block's
//                   valid q and k rows into the workspace (HBM bound: q and k
//                   are read once).
//   2. score_mma:   one CTA per (b, h, 128 query blocks, 64 key blocks): the
//                   contraction qbar kbar^T on the tensor cores
//                   (tcgen05.mma kind::tf32, accumulator in TMEM).  Each mean
//                   is split into a tf32 part (its 13 low mantissa bits
//                   cleared) and the exact remainder, and the scores are the
//                   three products hi.hi + hi.lo + lo.hi, which carry
//                   fp32-level accuracy (the dropped lo.lo term and the tf32
//                   rounding of the remainders are below 2^-19 of each
//                   product).  TMA loads 32 dimensions at a time into a
//                   2-stage ring, where the CTA's threads split them in place;
//                   the scaled scores go through shared memory to a
//                   [B*H, nb, nb] fp32 buffer in the workspace (L2-resident at
//                   the workloads' sizes) in coalesced rows.
//   3. topp_rows:   one warp per row: max, exp, sum, and the cut found by
//                   bisection on the bit patterns of the (non-negative)
//                   exponentials -- the largest T with
//                   sum(e_j >= T) >= top_p * sum(e) -- over the whole row for
//                   the exponent bits, then over the values that share T's
//                   exponent only (compacted into shared memory); ties at T are
//                   taken in index order; the kept blocks are balloted into
//                   CRM words.
//   4-8. the tiled count sort and the kept-block lists shared with packing.
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "bsa.h"
#include "bsa_internal.h"
#include "sm100_ptx.cuh"

// BSA_ERR_TIMEOUT when a wait of the score kernel ran out (read and cleared by
// bsa_get_device_error through bsa::take_predict_device_error)
__device__ int g_predict_device_error = 0;

namespace {

using namespace sm100;

constexpr int kPoolThreads = 256;
constexpr int kScoreThreads = 256;
constexpr int kMaxBlocks = 2048;  // nb limit of the cut (score rows per warp in registers)

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// blockIdx.x = block i, blockIdx.y = b*H + h.  Threads: (d/8) column groups of
// 8 columns (one 16-byte load per token) x token groups; partial sums are
// combined in shared memory.  d is 64 or 128.
__global__ void __launch_bounds__(kPoolThreads)
    pool_kernel(const uint4* __restrict__ q, const uint4* __restrict__ k, int n_valid,
                int n_pad, int d, int block, float* __restrict__ qbar,
                float* __restrict__ kbar) {
  __shared__ float part[2][kPoolThreads * 8];  // [tensor][token group][column]
  const int vec = d / 8;                   // 16-byte pieces per row
  const int groups = kPoolThreads / vec;   // token groups
  const int cg = threadIdx.x % vec, tg = threadIdx.x / vec;
  const int i = blockIdx.x;
  const int64_t bh = blockIdx.y;
  const int first = i * block;
  const int count = min(block, n_valid - first);  // >= 1: n_pad - block < n_valid
  const uint4* qrow = q + (bh * n_pad + first) * vec + cg;
  const uint4* krow = k + (bh * n_pad + first) * vec + cg;
  float sq[8] = {0, 0, 0, 0, 0, 0, 0, 0}, sk[8] = {0, 0, 0, 0, 0, 0, 0, 0};
  for (int t = tg; t < count; t += groups) {
    const uint4 a = __ldcs(qrow + int64_t(t) * vec);
    const uint4 b = __ldcs(krow + int64_t(t) * vec);
    const uint32_t aw[4] = {a.x, a.y, a.z, a.w}, bw[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      sq[2 * u] += bf16_lo(aw[u]);
      sq[2 * u + 1] += bf16_hi(aw[u]);
      sk[2 * u] += bf16_lo(bw[u]);
      sk[2 * u + 1] += bf16_hi(bw[u]);
    }
  }
#pragma unroll
  for (int u = 0; u < 8; ++u) {
    part[0][tg * d + cg * 8 + u] = sq[u];
    part[1][tg * d + cg * 8 + u] = sk[u];
  }
  __syncthreads();
  const float inv = 1.0f / float(count);
  for (int c = threadIdx.x; c < 2 * d; c += kPoolThreads) {
    const int which = c / d, col = c - which * d;
    float s = 0.0f;
    for (int g = 0; g < groups; ++g) s += part[which][g * d + col];
    float* dst = which ? kbar : qbar;
    dst[(bh * (n_pad / block) + i) * d + col] = s * inv;
  }
}

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}
__device__ __forceinline__ float warp_max(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, o));
  return x;
}
__device__ __forceinline__ int warp_sum_int(int x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

// One row, one warp.  Lane l holds blocks l + 32 k (k < kPerLane) in
// registers; blocks past nb hold exp(-inf) = 0, which never counts.  The cut
// is the largest bit pattern T with sum(e_j >= T) >= top_p * sum(e) (the
// exponentials lie in [0, 1], so patterns order like values and bit 30 is
// never set), found by bisection from the top: bits 29..23 (the exponent)
// over the whole row; then the values with T's exponent are compacted into
// the warp's shared buffer `bucket` (kPerLane * 32 floats), those above it
// summed once, and bits 22..0 bisect over the bucket alone.  Blocks above T
// are kept and ties at T join in index order until the cumulative sum reaches
// the target.  If the total never reaches it (top_p >= 1, or rounding) every
// block is kept.  Block j = l + 32 k is bit l of CRM word k.
template <int kPerLane>
__device__ __forceinline__ void top_p_row(const float* __restrict__ s_row, int nb, float p_h,
                                          uint32_t* __restrict__ out,
                                          int32_t* __restrict__ count,
                                          float* __restrict__ bucket) {
  const int lane = threadIdx.x & 31;
  const uint32_t below = (1u << lane) - 1u;
  float e[kPerLane];
  float m = -INFINITY;
#pragma unroll
  for (int k = 0; k < kPerLane; ++k) {
    const int j = lane + 32 * k;
    e[k] = j < nb ? s_row[j] : -INFINITY;
    m = fmaxf(m, e[k]);
  }
  m = warp_max(m);
  float l = 0.0f;
#pragma unroll
  for (int k = 0; k < kPerLane; ++k) {
    e[k] = expf(e[k] - m);
    l += e[k];
  }
  l = warp_sum(l);
  const float target = p_h * l;
  uint32_t T = 0;
  for (int bit = 29; bit >= 23; --bit) {
    const uint32_t cand = T | (1u << bit);
    float sum = 0.0f;
#pragma unroll
    for (int k = 0; k < kPerLane; ++k) sum += __float_as_uint(e[k]) >= cand ? e[k] : 0.0f;
    if (warp_sum(sum) >= target) T = cand;
  }
  // values above T's exponent always count; those sharing it go to the bucket
  const uint32_t next_exp = T + (1u << 23);
  float hi_sum = 0.0f;
  int n_b = 0;
#pragma unroll
  for (int k = 0; k < kPerLane; ++k) {
    const uint32_t eb = __float_as_uint(e[k]);
    hi_sum += eb >= next_exp ? e[k] : 0.0f;
    const bool in = eb >= T && eb < next_exp && lane + 32 * k < nb;
    const uint32_t m = __ballot_sync(0xffffffffu, in);
    if (in) bucket[n_b + __popc(m & below)] = e[k];
    n_b += __popc(m);
  }
  hi_sum = warp_sum(hi_sum);
  __syncwarp();
  for (int bit = 22; bit >= 0; --bit) {
    const uint32_t cand = T | (1u << bit);
    float sum = 0.0f;
    for (int i = lane; i < n_b; i += 32) {
      const float v = bucket[i];
      sum += __float_as_uint(v) >= cand ? v : 0.0f;
    }
    if (hi_sum + warp_sum(sum) >= target) T = cand;
  }
  const bool keep_all = !(l >= target);
  float above = 0.0f;
  int ties = 0;
#pragma unroll
  for (int k = 0; k < kPerLane; ++k) {
    const uint32_t eb = __float_as_uint(e[k]);
    above += eb > T ? e[k] : 0.0f;
    ties += (eb == T) & (lane + 32 * k < nb);
  }
  above = warp_sum(above);
  ties = warp_sum_int(ties);
  const float e_t = __uint_as_float(T);
  int need = 0;
  for (float acc = above; need < ties && acc < target; ++need) acc += e_t;
  const int words = (nb + 31) / 32;
  int total = 0, tie_rank = 0;
#pragma unroll
  for (int k = 0; k < kPerLane; ++k) {
    if (k < words) {  // uniform
      const int j = lane + 32 * k;
      const uint32_t eb = __float_as_uint(e[k]);
      const bool tie = j < nb && eb == T;
      const uint32_t tie_mask = __ballot_sync(0xffffffffu, tie);
      const bool keep = j < nb && (keep_all || eb > T ||
                                   (tie && tie_rank + __popc(tie_mask & below) < need));
      tie_rank += __popc(tie_mask);
      const uint32_t word = __ballot_sync(0xffffffffu, keep);
      if (lane == 0) out[k] = word;
      total += __popc(word);
    }
  }
  if (lane == 0) *count = total;
}

// Scores on the tensor cores: one CTA of 128 threads per (b, h, 128 query
// blocks i0.., 64 key blocks j0..), two CTAs per SM (97 KB of shared memory
// each), so that one CTA's loads and stores overlap the other's products.
// Thread 0 issues the TMA loads of the means, 32 dimensions (one 128-byte
// swizzle atom per row) per stage: query means 16 KB, key means 8 KB.  All
// 128 threads then split each value in place into its tf32 part and write
// the remainder at the same offset of a parallel region (the split is
// elementwise, so the swizzle carries over).  Thread 32 issues per stage 4
// steps of K = 8, each three tcgen05.mma kind::tf32 products into one
// 128 x 64 fp32 accumulator in TMEM (hi.hi, hi.lo, lo.hi).  All four warps
// then move the accumulator (one query block per TMEM lane) through shared
// memory to the score rows.  Rows or keys past nb (the next head's, or the
// zero fill past the last head) are computed and not stored.
constexpr int kMmaThreads = 128;
constexpr int kTileK = 64;                                // key blocks per CTA
constexpr uint32_t kQPart = 128u * 128u;                  // 128 query rows x 32 fp32
constexpr uint32_t kKPart = uint32_t(kTileK) * 128u;     // 64 key rows x 32 fp32
constexpr uint32_t kLoaded = kQPart + kKPart;             // q, k as loaded
constexpr uint32_t kStageBytes = 2u * kLoaded;            // q hi, k hi, q lo, k lo
constexpr int kMmaStages = 2;
constexpr int kOutStride = kTileK + 1;                    // floats per staged output row
constexpr uint64_t kScoreTimeoutNs = 2000000000ull;

struct ScoreBars {
  uint64_t full[kMmaStages], split[kMmaStages], empty[kMmaStages], done;
  uint32_t tmem_base;
  int abort;
};
constexpr size_t kScoreMmaSmem = size_t(kMmaStages) * kStageBytes + 256 + 1024;
static_assert(size_t(128) * kOutStride * 4 <= size_t(kMmaStages) * kStageBytes, "output staging");
static_assert(kQPart % 1024 == 0 && kLoaded % 1024 == 0, "1024-byte aligned swizzled tiles");

// D[tmem] (+)= A[smem] * B[smem]^T, kind::tf32 (fp32 containers, fp32 accumulate)
__device__ __forceinline__ void mma_ss_tf32(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                            uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::tf32 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Instruction descriptor, kind::tf32: fp32 accumulator (bits 4-5 = 1), tf32 A
// and B (bits 7-9 = 2, bits 10-12 = 2), both K-major, N >> 3 at bits 17-22,
// M >> 4 at bits 24-28.
constexpr uint32_t idesc_tf32_f32(int M, int N) {
  return (1u << 4) | (2u << 7) | (2u << 10) | (uint32_t(N >> 3) << 17) | (uint32_t(M >> 4) << 24);
}

// Bounded wait: true once the phase of `parity` completed; false after about
// two seconds (records BSA_ERR_TIMEOUT) or, with abort != nullptr, when
// another thread of the CTA gave up.
__device__ __noinline__ bool score_wait(uint32_t bar, uint32_t parity, volatile int* abort) {
  const uint64_t t0 = global_timer_ns();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 63u) == 0) {
      if (abort && *abort) return false;
      if (global_timer_ns() - t0 > kScoreTimeoutNs) {
        if (abort) *abort = 1;
        atomicExch(&g_predict_device_error, int(BSA_ERR_TIMEOUT));
        return false;
      }
    }
  }
}

__global__ void __launch_bounds__(kMmaThreads, 1)
    score_mma_kernel(const __grid_constant__ CUtensorMap tm_q,
                     const __grid_constant__ CUtensorMap tm_k, int H, int nb, int d,
                     const float* __restrict__ tau, float* __restrict__ scores) {
  extern __shared__ __align__(1024) uint8_t score_smem_raw[];
  // 128-byte swizzle atoms need 1024-byte aligned tiles
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(score_smem_raw) + 1023) & ~uintptr_t(1023));
  ScoreBars* bars = reinterpret_cast<ScoreBars*>(smem + size_t(kMmaStages) * kStageBytes);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int j0 = blockIdx.x * kTileK, i0 = blockIdx.y * 128;
  const int bh = blockIdx.z;
  const int n_st = d / 32;  // stages of 32 dimensions
  volatile int* abort = &bars->abort;
  const uint32_t s0 = smem_addr(smem);

  if (threadIdx.x == 0) {
    for (int i = 0; i < kMmaStages; ++i) {
      mbar_init(smem_addr(&bars->full[i]), 1);
      mbar_init(smem_addr(&bars->split[i]), kMmaThreads);
      mbar_init(smem_addr(&bars->empty[i]), 1);
    }
    mbar_init(smem_addr(&bars->done), 1);
    bars->abort = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_addr(&bars->tmem_base), kTileK);
    tmem_relinquish();
  }
  if (threadIdx.x == 0) {
    prefetch_tensormap(&tm_q);
    prefetch_tensormap(&tm_k);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;

  // Per stage st (slot st % kMmaStages): thread 0 loads it (the first
  // kMmaStages up front, stage st + kMmaStages once the products of stage st
  // have released the slot); every thread splits it once it has landed and
  // arrives on `split`; thread 32 issues its products once all 128 have.
  constexpr uint32_t idesc = idesc_tf32_f32(128, kTileK);
  auto load_stage = [&](int st) {
    const int slot = st % kMmaStages;
    const uint32_t fbar = smem_addr(&bars->full[slot]);
    mbar_arrive_expect_tx(fbar, kLoaded);
    const uint32_t base = s0 + slot * kStageBytes;
    tma_load_2d(base, &tm_q, fbar, st * 32, bh * nb + i0);
    tma_load_2d(base + kQPart, &tm_k, fbar, st * 32, bh * nb + j0);
  };
  int issued = 0;  // stages loaded (thread 0)
  if (threadIdx.x == 0)
    for (; issued < n_st && issued < kMmaStages; ++issued) load_stage(issued);
  bool ok = true;
  for (int st = 0; st < n_st; ++st) {
    const int slot = st % kMmaStages;
    const uint32_t par = (st / kMmaStages) & 1;
    // ---------------------------------------------------------- split
    // the stage's 24 KB of means -> tf32 parts in place, exact remainders
    // 24 KB further
    ok = ok && score_wait(smem_addr(&bars->full[slot]), par, abort);
    if (ok) {
      uint4* v = reinterpret_cast<uint4*>(smem + size_t(slot) * kStageBytes);
      uint4* lo = v + kLoaded / 16;
      for (int e = threadIdx.x; e < int(kLoaded / 16); e += kMmaThreads) {
        const uint4 x = v[e];
        uint4 h, r;
        h.x = x.x & 0xFFFFE000u; r.x = __float_as_uint(__uint_as_float(x.x) - __uint_as_float(h.x));
        h.y = x.y & 0xFFFFE000u; r.y = __float_as_uint(__uint_as_float(x.y) - __uint_as_float(h.y));
        h.z = x.z & 0xFFFFE000u; r.z = __float_as_uint(__uint_as_float(x.z) - __uint_as_float(h.z));
        h.w = x.w & 0xFFFFE000u; r.w = __float_as_uint(__uint_as_float(x.w) - __uint_as_float(h.w));
        v[e] = h;
        lo[e] = r;
      }
      // generic-proxy writes of shared memory become visible to the tensor core
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    }
    // arrive even after a failure, so that the MMA issuer's wait ends
    mbar_arrive(smem_addr(&bars->split[slot]));
    if (threadIdx.x == 32) {
      // -------------------------------------------------------- MMA issuer
      if (score_wait(smem_addr(&bars->split[slot]), par, nullptr)) {
        tc_fence_after();
        const uint32_t base = s0 + slot * kStageBytes;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {  // K = 8 (32 bytes) per product
          const uint32_t off = kk * 32;
          const uint64_t a_hi = smem_desc_sw128(base + off, 16, 1024);
          const uint64_t b_hi = smem_desc_sw128(base + kQPart + off, 16, 1024);
          const uint64_t a_lo = smem_desc_sw128(base + kLoaded + off, 16, 1024);
          const uint64_t b_lo = smem_desc_sw128(base + kLoaded + kQPart + off, 16, 1024);
          mma_ss_tf32(tmem, a_hi, b_hi, idesc, (st > 0 || kk > 0) ? 1u : 0u);
          mma_ss_tf32(tmem, a_hi, b_lo, idesc, 1u);
          mma_ss_tf32(tmem, a_lo, b_hi, idesc, 1u);
        }
      }
      mma_commit(smem_addr(&bars->empty[slot]));
      // everything issued completes before `done` (also after a failure)
      if (st == n_st - 1) mma_commit(smem_addr(&bars->done));
    }
    if (threadIdx.x == 0 && st + kMmaStages < n_st) {
      // ------------------------------------------------------ producer
      // the slot is free once stage st's products have read it
      if (score_wait(smem_addr(&bars->empty[slot]), par, nullptr)) {
        load_stage(st + kMmaStages);
        ++issued;
      }
    }
  }
  if (threadIdx.x == 0) {
    // every copy issued has landed before the ring is reused or the CTA exits
    // (already true unless a wait above ran out; bounded, ignores abort)
    for (int st = issued > kMmaStages ? issued - kMmaStages : 0; st < issued; ++st)
      score_wait(smem_addr(&bars->full[st % kMmaStages]), (st / kMmaStages) & 1, nullptr);
  }
  __syncwarp();

  // ------------------------------------------------------------ epilogue
  // lane l of warp w holds query block i0 + 32 w + l: its kTileK scores go
  // to shared memory (the ring is free: every product has read it), then
  // each warp writes 32 rows, one row per pass, lanes along the keys
  const bool good = __all_sync(0xffffffffu, score_wait(smem_addr(&bars->done), 0, nullptr));
  tc_fence_after();
  const float inv_denom = 1.0f / (sqrtf(float(d)) * __ldg(tau + (bh % H)));
  float* stage_out = reinterpret_cast<float*>(smem);
  __syncthreads();  // every split of the ring is over before it is reused
  if (good) {
    const uint32_t lane_base = uint32_t(warp * 32) << 16;
#pragma unroll
    for (int c0 = 0; c0 < kTileK; c0 += 32) {
      uint32_t r[32];
      tmem_load32(tmem + lane_base + c0, r);
#pragma unroll
      for (int c = 0; c < 32; ++c)
        stage_out[(warp * 32 + lane) * kOutStride + c0 + c] = __uint_as_float(r[c]) * inv_denom;
    }
  }
  __syncwarp();
  if (good) {
    const int ncols = min(kTileK, nb - j0);
    for (int rr = 0; rr < 32; ++rr) {
      const int row = warp * 32 + rr;
      if (i0 + row >= nb) break;
      float* dst = scores + (int64_t(bh) * nb + i0 + row) * nb + j0;
#pragma unroll
      for (int c = lane; c < kTileK; c += 32)
        if (c < ncols) dst[c] = stage_out[row * kOutStride + c];
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTileK);
  }
}

// The cut, one warp per row of the score buffer (kScoreThreads / 32 rows per CTA).
template <int kPerLane>
__global__ void __launch_bounds__(kScoreThreads)
    topp_rows_kernel(const float* __restrict__ scores, int H, int nb, int rows,
                     const float* __restrict__ top_p, uint32_t* __restrict__ bits,
                     int32_t* __restrict__ counts) {
  extern __shared__ float topp_bucket[];  // [warp][kPerLane * 32]
  const int r = blockIdx.x * (kScoreThreads / 32) + (threadIdx.x >> 5);
  if (r >= rows) return;
  const int h = (r / nb) % H;
  top_p_row<kPerLane>(scores + int64_t(r) * nb, nb, __ldg(top_p + h),
                      bits + int64_t(r) * ((nb + 31) / 32), counts + r,
                      topp_bucket + (threadIdx.x >> 5) * kPerLane * 32);
}

size_t scores_bytes(int64_t BH, int nb) {
  const size_t b = size_t(BH) * nb * nb * sizeof(float);
  return (b + 255) & ~size_t(255);
}

template <int kPerLane>
bsa_status launch_topp_rows(int rows, cudaStream_t s, const float* scores, int H, int nb,
                            const float* top_p, uint32_t* bits, int32_t* counts) {
  const int per_cta = kScoreThreads / 32;
  const int smem = per_cta * kPerLane * 32 * int(sizeof(float));
  if (cudaFuncSetAttribute(topp_rows_kernel<kPerLane>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           smem) != cudaSuccess)
    return BSA_ERR_LAUNCH;
  topp_rows_kernel<kPerLane><<<(rows + per_cta - 1) / per_cta, kScoreThreads, smem, s>>>(
      scores, H, nb, rows, top_p, bits, counts);
  return bsa::launch_status() == BSA_OK ? BSA_OK : BSA_ERR_LAUNCH;
}

size_t means_bytes(int64_t BH, int nb, int d) {
  const size_t b = size_t(BH) * nb * d * sizeof(float);
  return (b + 255) & ~size_t(255);
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// [rows, d] fp32 row-major, box = 32 columns (128 bytes) x box_rows rows,
// 128-byte swizzle; rows past the end read as zeros
bool make_means_map(CUtensorMap* map, const float* base, int64_t rows, int d, int box_rows) {
  static EncodeTiledFn enc = nullptr;
  if (!enc) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) !=
            cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return false;
    enc = reinterpret_cast<EncodeTiledFn>(ptr);
  }
  cuuint64_t dims[2] = {cuuint64_t(d), cuuint64_t(rows)};
  cuuint64_t strides[1] = {cuuint64_t(d) * 4};
  cuuint32_t box[2] = {32, cuuint32_t(box_rows)};
  cuuint32_t estr[2] = {1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<float*>(base), dims, strides,
             box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
         CUDA_SUCCESS;
}

}  // namespace

namespace bsa {
int take_predict_device_error() {
  int host = 0, zero = 0;
  if (cudaMemcpyFromSymbol(&host, g_predict_device_error, sizeof(int)) != cudaSuccess) return -1;
  if (cudaMemcpyToSymbol(g_predict_device_error, &zero, sizeof(int)) != cudaSuccess) return -1;
  return host;
}
}  // namespace bsa

extern "C" size_t bsa_predict_top_p_workspace(int B, int H, int n_pad, int d, int block) {
  if (B <= 0 || H <= 0 || n_pad <= 0 || d <= 0 || block <= 0 || n_pad % block != 0) return 0;
  const int nb = n_pad / block;
  const int64_t BH = int64_t(B) * H;
  return 2 * means_bytes(BH, nb, d) + scores_bytes(BH, nb) + bsa::pack_scratch_bytes(BH * nb, nb);
}

extern "C" bsa_status bsa_predict_top_p(const void* q, const void* k, int B, int H, int n_valid,
                                        int n_pad, int d, int block, const float* tau,
                                        const float* top_p, uint32_t* bits, int32_t* counts,
                                        int32_t* row_offsets, int32_t* col_idx,
                                        int32_t* schedule, void* workspace,
                                        size_t workspace_bytes, void* stream) {
  if (!q || !k || !tau || !top_p || !bits || !counts || !row_offsets || !schedule)
    return BSA_ERR_INVALID_ARG;
  if (B <= 0 || H <= 0 || d <= 0 || block <= 0 || n_pad <= 0) return BSA_ERR_INVALID_ARG;
  if (n_pad % block != 0 || n_valid <= n_pad - block || n_valid > n_pad)
    return BSA_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return BSA_ERR_UNSUPPORTED;
  const int nb = n_pad / block;
  if (nb > kMaxBlocks) return BSA_ERR_UNSUPPORTED;
  const int64_t BH = int64_t(B) * H;
  if (BH > 65535) return BSA_ERR_UNSUPPORTED;  // grid.y
  if (BH * nb * int64_t(nb) >= (int64_t(1) << 31) || BH * n_pad * int64_t(d) >= (int64_t(1) << 40))
    return BSA_ERR_OVERFLOW;
  if (!bsa::aligned16(q) || !bsa::aligned16(k) || !bsa::aligned4(tau) || !bsa::aligned4(top_p) ||
      !bsa::aligned4(bits) || !bsa::aligned4(counts) || !bsa::aligned4(row_offsets) ||
      !bsa::aligned4(schedule) || (col_idx && !bsa::aligned4(col_idx)))
    return BSA_ERR_MISALIGNED;
  if (!workspace || workspace_bytes < bsa_predict_top_p_workspace(B, H, n_pad, d, block))
    return BSA_ERR_WORKSPACE;
  if (!bsa::aligned16(workspace)) return BSA_ERR_MISALIGNED;
  if (bsa::num_sms() <= 0) return BSA_ERR_LAUNCH;

  cudaStream_t s = static_cast<cudaStream_t>(stream);
  char* ws = static_cast<char*>(workspace);
  // [q means][k means][scores][sort tables]
  const size_t mb = means_bytes(BH, nb, d);
  float* qbar = reinterpret_cast<float*>(ws);
  float* kbar = reinterpret_cast<float*>(ws + mb);
  float* scores = reinterpret_cast<float*>(ws + 2 * mb);
  void* scratch = ws + 2 * mb + scores_bytes(BH, nb);

  pool_kernel<<<dim3(unsigned(nb), unsigned(BH)), kPoolThreads, 0, s>>>(
      static_cast<const uint4*>(q), static_cast<const uint4*>(k), n_valid, n_pad, d, block, qbar,
      kbar);
  if (bsa::launch_status() != BSA_OK) return BSA_ERR_LAUNCH;
  CUtensorMap tq, tk;
  const int64_t mrows = BH * nb;
  if (!make_means_map(&tq, qbar, mrows, d, 128) || !make_means_map(&tk, kbar, mrows, d, kTileK))
    return BSA_ERR_LAUNCH;
  if (cudaFuncSetAttribute(score_mma_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           int(kScoreMmaSmem)) != cudaSuccess)
    return BSA_ERR_LAUNCH;
  score_mma_kernel<<<dim3(unsigned((nb + kTileK - 1) / kTileK), unsigned((nb + 127) / 128),
                         unsigned(BH)),
                     kMmaThreads, kScoreMmaSmem, s>>>(
      tq, tk, H, nb, d, tau, scores);
  if (bsa::launch_status() != BSA_OK) return BSA_ERR_LAUNCH;
  const int rows = int(BH * nb);
  const int per_lane = (nb + 31) / 32;
  bsa_status st;
  if (per_lane <= 8)
    st = launch_topp_rows<8>(rows, s, scores, H, nb, top_p, bits, counts);
  else if (per_lane <= 16)
    st = launch_topp_rows<16>(rows, s, scores, H, nb, top_p, bits, counts);
  else if (per_lane <= 20)
    st = launch_topp_rows<20>(rows, s, scores, H, nb, top_p, bits, counts);
  else if (per_lane <= 32)
    st = launch_topp_rows<32>(rows, s, scores, H, nb, top_p, bits, counts);
  else
    st = launch_topp_rows<64>(rows, s, scores, H, nb, top_p, bits, counts);
  if (st != BSA_OK) return st;
  return bsa::pack_finish(bits, counts, int(BH * nb), nb, nb, row_offsets, col_idx, schedule, scratch,
                          s);
}
