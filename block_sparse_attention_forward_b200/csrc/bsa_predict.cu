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
//   2. score_tile:  one CTA per (b, h, 32 query blocks).  Scores by fp32 FMA
//                   in 8 x 4 register tiles against key means staged in
//                   shared memory by cp.async, two slices deep, into a
//                   [B*H, nb, nb] fp32 buffer in the workspace (L2-resident at
//                   the workloads' sizes).
//   3. topp_rows:   one warp per row: max, exp, sum, and the cut found by
//                   bisection on the bit patterns of the (non-negative)
//                   exponentials -- the largest T with
//                   sum(e_j >= T) >= top_p * sum(e) -- then ties at T taken
//                   in index order; the kept blocks are balloted into CRM words.
//   4-8. the tiled count sort and the kept-block lists shared with packing.
#include <cuda_runtime.h>
#include <stdint.h>

#include "bsa.h"
#include "bsa_internal.h"

namespace {

constexpr int kPoolThreads = 256;
constexpr int kKeyChunk = 256;   // key blocks per pass
constexpr int kDSlice = 32;      // dimensions of the key means staged at a time
constexpr int kKsStride = kDSlice + 4;  // padded row (16-byte aligned, conflict-free)
constexpr int kScoreThreads = 256;
constexpr int kMaxBlocks = 2048;  // nb limit: the score rows live in shared memory

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
// exponentials are >= 0, so patterns order like values), found by bisection
// from the top bit over the registers (measured faster than bisecting the
// exponent first and then only the blocks sharing it); blocks above T are kept and ties at T join in index
// order until the cumulative sum reaches the target.  If the total never
// reaches it (top_p >= 1, or rounding) every block is kept.  Block j = l + 32 k
// is bit l of CRM word k.
template <int kPerLane>
__device__ __forceinline__ void top_p_row(const float* __restrict__ s_row, int nb, float p_h,
                                          uint32_t* __restrict__ out,
                                          int32_t* __restrict__ count) {
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
  for (int bit = 30; bit >= 0; --bit) {
    const uint32_t cand = T | (1u << bit);
    float sum = 0.0f;
#pragma unroll
    for (int k = 0; k < kPerLane; ++k) sum += __float_as_uint(e[k]) >= cand ? e[k] : 0.0f;
    if (warp_sum(sum) >= target) T = cand;
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

// Scores alone, written to a global [B*H, nb, nb] buffer (L2-resident at the
// workloads' sizes): one CTA per (b, h, 32 query blocks), each thread an
// 8-row x 4-key register tile (rows 8 (t / 64) + a, keys (t % 64) + 64 b of
// each pass of kKeyChunk keys), so that one 16-byte vector of key means (a
// quarter warp's in distinct banks) feeds 8 FMA chains and one broadcast
// vector of query means feeds 4: 12 vector loads per 128 FMAs.  The key means
// are staged 32 dimensions at a time, the next slice's cp.async copies in
// flight while this slice's FMAs run.  88 KB of shared memory: two CTAs per SM.
constexpr int kRowsTile = 32;
constexpr int kSliceFloats = kKeyChunk * kKsStride;  // one staged slice of key means

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src),
               "r"(src_bytes)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

__global__ void __launch_bounds__(kScoreThreads)
    score_tile_kernel(const float* __restrict__ qbar, const float* __restrict__ kbar, int H,
                      int nb, int d, const float* __restrict__ tau, float* __restrict__ scores) {
  extern __shared__ float4 score_smem4[];
  float* qs = reinterpret_cast<float*>(score_smem4);  // [kRowsTile][d]
  float* ks = qs + kRowsTile * d;                     // [2][kKeyChunk][kKsStride]
  const int64_t bh = blockIdx.y;
  const int h = int(bh % H);
  const int i0 = blockIdx.x * kRowsTile;
  const int rows = min(kRowsTile, nb - i0);
  const float inv_denom = 1.0f / (sqrtf(float(d)) * __ldg(tau + h));
  const int slices_per_chunk = d / kDSlice;
  const int n_slices = ((nb + kKeyChunk - 1) / kKeyChunk) * slices_per_chunk;

  // slice sl = (key chunk sl / slices_per_chunk, dims 32 (sl % slices_per_chunk))
  // into buffer sl & 1: 256 keys x 8 vectors, 8 per thread; keys past nb read
  // zeros (source size 0)
  auto stage = [&](int sl) {
    const int j0 = (sl / slices_per_chunk) * kKeyChunk;
    const int c0 = (sl % slices_per_chunk) * kDSlice;
    float* buf = ks + (sl & 1) * kSliceFloats;
    for (int e = threadIdx.x; e < kKeyChunk * (kDSlice / 4); e += kScoreThreads) {
      const int key = e / (kDSlice / 4), part = e - key * (kDSlice / 4);
      const bool in = j0 + key < nb;
      const float* src = kbar + ((bh * nb + (in ? j0 + key : 0)) * d + c0 + part * 4);
      cp_async16(static_cast<uint32_t>(__cvta_generic_to_shared(buf + key * kKsStride + part * 4)),
                 src, in ? 16u : 0u);
    }
    cp_async_commit();
  };

  stage(0);
  for (int e = threadIdx.x; e < kRowsTile * d; e += kScoreThreads) {
    const int r = e / d, c = e - r * d;
    qs[e] = r < rows ? qbar[(bh * nb + i0 + r) * d + c] : 0.0f;
  }
  const int rg = threadIdx.x / 64, kg = threadIdx.x % 64;
  float acc[8][4];
#pragma unroll
  for (int a = 0; a < 8; ++a)
#pragma unroll
    for (int b = 0; b < 4; ++b) acc[a][b] = 0.0f;
  for (int sl = 0; sl < n_slices; ++sl) {
    if (sl + 1 < n_slices) {
      stage(sl + 1);
      cp_async_wait<1>();  // this slice has landed (the next may be in flight)
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();
    const int c0 = (sl % slices_per_chunk) * kDSlice;
    const float* buf = ks + (sl & 1) * kSliceFloats;
#pragma unroll
    for (int c4 = 0; c4 < kDSlice / 4; ++c4) {
      float4 qv[8], kv[4];
#pragma unroll
      for (int a = 0; a < 8; ++a)
        qv[a] = *reinterpret_cast<const float4*>(qs + (rg * 8 + a) * d + c0 + c4 * 4);
#pragma unroll
      for (int b = 0; b < 4; ++b)
        kv[b] = *reinterpret_cast<const float4*>(buf + (kg + 64 * b) * kKsStride + c4 * 4);
#pragma unroll
      for (int a = 0; a < 8; ++a)
#pragma unroll
        for (int b = 0; b < 4; ++b) {
          acc[a][b] = fmaf(qv[a].x, kv[b].x, acc[a][b]);
          acc[a][b] = fmaf(qv[a].y, kv[b].y, acc[a][b]);
          acc[a][b] = fmaf(qv[a].z, kv[b].z, acc[a][b]);
          acc[a][b] = fmaf(qv[a].w, kv[b].w, acc[a][b]);
        }
    }
    if (sl % slices_per_chunk == slices_per_chunk - 1) {  // a key chunk is complete
      const int j0 = (sl / slices_per_chunk) * kKeyChunk;
#pragma unroll
      for (int a = 0; a < 8; ++a) {
        const int r = rg * 8 + a;
#pragma unroll
        for (int b = 0; b < 4; ++b) {
          const int key = j0 + kg + 64 * b;
          if (r < rows && key < nb) scores[(bh * nb + i0 + r) * nb + key] = acc[a][b] * inv_denom;
          acc[a][b] = 0.0f;
        }
      }
    }
    __syncthreads();  // every thread is done with this buffer before it is refilled
  }
}

// The cut, one warp per row of the score buffer (kScoreThreads / 32 rows per CTA).
template <int kPerLane>
__global__ void __launch_bounds__(kScoreThreads)
    topp_rows_kernel(const float* __restrict__ scores, int H, int nb, int rows,
                     const float* __restrict__ top_p, uint32_t* __restrict__ bits,
                     int32_t* __restrict__ counts) {
  const int r = blockIdx.x * (kScoreThreads / 32) + (threadIdx.x >> 5);
  if (r >= rows) return;
  const int h = (r / nb) % H;
  top_p_row<kPerLane>(scores + int64_t(r) * nb, nb, __ldg(top_p + h),
                      bits + int64_t(r) * ((nb + 31) / 32), counts + r);
}

size_t score_tile_smem_bytes(int d) {
  return sizeof(float) * (size_t(kRowsTile) * d + 2 * size_t(kSliceFloats));
}

size_t scores_bytes(int64_t BH, int nb) {
  const size_t b = size_t(BH) * nb * nb * sizeof(float);
  return (b + 255) & ~size_t(255);
}

template <int kPerLane>
bsa_status launch_topp_rows(int rows, cudaStream_t s, const float* scores, int H, int nb,
                            const float* top_p, uint32_t* bits, int32_t* counts) {
  const int per_cta = kScoreThreads / 32;
  topp_rows_kernel<kPerLane><<<(rows + per_cta - 1) / per_cta, kScoreThreads, 0, s>>>(
      scores, H, nb, rows, top_p, bits, counts);
  return bsa::launch_status() == BSA_OK ? BSA_OK : BSA_ERR_LAUNCH;
}

size_t means_bytes(int64_t BH, int nb, int d) {
  const size_t b = size_t(BH) * nb * d * sizeof(float);
  return (b + 255) & ~size_t(255);
}

}  // namespace

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
  float* qbar = reinterpret_cast<float*>(ws);
  float* kbar = reinterpret_cast<float*>(ws + means_bytes(BH, nb, d));
  float* scores = reinterpret_cast<float*>(ws + 2 * means_bytes(BH, nb, d));
  void* scratch = ws + 2 * means_bytes(BH, nb, d) + scores_bytes(BH, nb);

  pool_kernel<<<dim3(unsigned(nb), unsigned(BH)), kPoolThreads, 0, s>>>(
      static_cast<const uint4*>(q), static_cast<const uint4*>(k), n_valid, n_pad, d, block, qbar,
      kbar);
  if (bsa::launch_status() != BSA_OK) return BSA_ERR_LAUNCH;
  const size_t smem = score_tile_smem_bytes(d);
  if (cudaFuncSetAttribute(score_tile_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           int(smem)) != cudaSuccess)
    return BSA_ERR_LAUNCH;
  score_tile_kernel<<<dim3(unsigned((nb + kRowsTile - 1) / kRowsTile), unsigned(BH)),
                      kScoreThreads, smem, s>>>(qbar, kbar, H, nb, d, tau, scores);
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
