// bsa_threshold.cu -- resize of a per-head threshold map to another block grid
// ("ScalingAttention", Sec. 4.3.1, Eq. 7: conservative bilinear interpolation
// with a ceiling rule, so that any overlap with an active region survives).
//
// The map is sampled at (u / s_h, v / s_w) with s_h = tq / sq and s_w = tk / sk.
// Read on the active-region indicator 1(T <= p), the ceiling of a bilinear mix
// is 1 exactly when a source block with a nonzero weight is active; for every
// p at once this is the minimum threshold over those source blocks.  Along
// each axis they are floor(u * sq / tq) and, when the division leaves a
// remainder (a nonzero weight), the next block, clamped to the last one.  The
// sample position is exact integer arithmetic here.
//
// One warp per target row (h, u) (the grid has a warp for every row).  The
// row's two source rows a0, a1 are found once; when the source has at most
// kStagedCols columns the warp first writes their element-wise minimum to
// shared memory (coalesced reads), so each output is the minimum of two shared
// words; wider sources read the four global words per output directly.  Each
// lane takes v = lane + 32 k and keeps kResizeRun outputs in flight before it
// stores them (coalesced).  Along v the sample position advances by
// 32 * sk / tk per step, kept as an exact quotient and remainder, with no
// division in the loop.  Block counts are limited to 65535 per axis so that
// every product fits in 32 bits.
#include <cuda_runtime.h>
#include <stdint.h>

#include "bsa.h"
#include "bsa_internal.h"

namespace {

constexpr int kMaxBlocksPerAxis = 65535;

__device__ __forceinline__ void support(uint32_t u, uint32_t n_src, uint32_t n_dst, uint32_t* lo,
                                        uint32_t* hi) {
  const uint32_t num = u * n_src;  // < 2^32: both factors are below 2^16
  const uint32_t a = num / n_dst;
  *lo = a;
  *hi = (a * n_dst != num && a + 1 < n_src) ? a + 1 : a;
}

constexpr int kResizeRun = 8;
constexpr int kResizeWarps = 8;
constexpr int kStagedCols = 1024;

template <bool kStaged>
__global__ void __launch_bounds__(256)
    threshold_resize_kernel(const float* __restrict__ src, int H, int sq, int sk,
                            float* __restrict__ dst, int tq, int tk) {
  __shared__ float colmin[kStaged ? kResizeWarps : 1][kStaged ? kStagedCols : 1];
  const uint32_t lane = threadIdx.x & 31;
  const uint32_t wib = threadIdx.x >> 5;  // warp in block
  const uint32_t rows = uint32_t(H) * uint32_t(tq);  // < 2^31, checked on the host
  const uint32_t warp = blockIdx.x * kResizeWarps + wib;  // < 2^31
  const uint32_t n_warps = gridDim.x * kResizeWarps;
  const uint32_t utk = uint32_t(tk), usk = uint32_t(sk);
  const uint32_t step_q = (32u * usk) / utk, step_r = (32u * usk) % utk;
  const uint32_t lane_q = (lane * usk) / utk, lane_r = (lane * usk) % utk;
  for (uint32_t row = warp; row < rows; row += n_warps) {
    const uint32_t h = row / uint32_t(tq);
    const uint32_t u = row - h * uint32_t(tq);
    uint32_t a0, a1;
    support(u, sq, tq, &a0, &a1);
    const float* r0 = src + (size_t(h) * sq + a0) * sk;
    const float* r1 = src + (size_t(h) * sq + a1) * sk;
    float* cm = colmin[kStaged ? wib : 0];
    if (kStaged) {
      __syncwarp();  // the previous row's reads of cm are done
#pragma unroll 8
      for (uint32_t b = lane; b < usk; b += 32) cm[b] = fminf(__ldg(r0 + b), __ldg(r1 + b));
      __syncwarp();
    }
    float* out = dst + size_t(row) * tk;
    uint32_t q = lane_q, rem = lane_r;  // v * sk = q * tk + rem for v = lane
    for (uint32_t v0 = 0; v0 < utk; v0 += 32u * kResizeRun) {
      float m[kResizeRun];
#pragma unroll
      for (int k = 0; k < kResizeRun; ++k) {
        const uint32_t v = v0 + 32u * k + lane;
        m[k] = 0.0f;
        if (v < utk) {
          const uint32_t b0 = q, b1 = (rem != 0 && q + 1 < usk) ? q + 1 : q;
          // a block repeated (no second neighbour on an axis) changes nothing;
          // fminf returns the other operand when one is NaN, NaN only when
          // both are, so NaN thresholds are skipped
          if (kStaged)
            m[k] = fminf(cm[b0], cm[b1]);
          else
            m[k] = fminf(fminf(__ldg(r0 + b0), __ldg(r0 + b1)),
                         fminf(__ldg(r1 + b0), __ldg(r1 + b1)));
        }
        q += step_q;
        rem += step_r;
        if (rem >= utk) {
          rem -= utk;
          ++q;
        }
      }
#pragma unroll
      for (int k = 0; k < kResizeRun; ++k) {
        const uint32_t v = v0 + 32u * k + lane;
        if (v < utk) out[v] = m[k];
      }
    }
  }
}

}  // namespace

extern "C" bsa_status bsa_threshold_resize(const float* src, int H, int sq, int sk, float* dst,
                                           int tq, int tk, void* stream) {
  if (!src || !dst) return BSA_ERR_INVALID_ARG;
  if (H <= 0 || sq <= 0 || sk <= 0 || tq <= 0 || tk <= 0) return BSA_ERR_INVALID_ARG;
  if (sq > kMaxBlocksPerAxis || sk > kMaxBlocksPerAxis || tq > kMaxBlocksPerAxis ||
      tk > kMaxBlocksPerAxis)
    return BSA_ERR_UNSUPPORTED;
  if (!bsa::aligned4(src) || !bsa::aligned4(dst)) return BSA_ERR_MISALIGNED;
  if (int64_t(H) * tq >= (int64_t(1) << 31)) return BSA_ERR_OVERFLOW;
  const int sms = bsa::num_sms();
  if (sms <= 0) return BSA_ERR_LAUNCH;
  // kResizeWarps warps per block, one row per warp: blocks turn over as rows finish
  const int grid = int((int64_t(H) * tq + kResizeWarps - 1) / kResizeWarps);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (sk <= kStagedCols)
    threshold_resize_kernel<true><<<grid, 256, 0, s>>>(src, H, sq, sk, dst, tq, tk);
  else
    threshold_resize_kernel<false><<<grid, 256, 0, s>>>(src, H, sq, sk, dst, tq, tk);
  return bsa::launch_status();
}
