// bsa_permute.cu -- 3-D tile gather kernels (token permutation of
// "ScalingAttention" Sec. 5.4-5.5, in the tile form: frame-major T x H x W
// tokens <-> contiguous spatio-temporal tiles, edge tiles clipped and
// concatenated with no holes, zero tail up to n_pad).
//
// Both directions are output-driven gathers, so every store is coalesced.  A
// CTA owns a chunk of kChunk output positions: it maps each position to its
// source position once (the index arithmetic is amortised over all B*H heads
// that share the permutation), keeps the map in shared memory, then moves the
// 16-byte pieces of every row of that chunk for each (b, h) in turn.
#include <cuda_runtime.h>
#include <stdint.h>

#include "bsa.h"
#include "bsa_internal.h"

namespace {

constexpr int kChunk = 64;     // output positions per CTA
constexpr int kThreads = 256;  // threads per CTA

struct Grid3 {
  int T, Hs, Ws, tt, th, tw;
};

// tile-major position p (< T*Hs*Ws) -> frame-major index.  Slabs of tt frames
// are contiguous; inside a slab, rows of tiles (th rows of the grid) are
// contiguous; inside such a row, tiles; inside a tile, (t, y, x) row-major.
__device__ __forceinline__ int64_t tile_to_frame(int64_t p, const Grid3& g) {
  const int64_t plane = int64_t(g.Hs) * g.Ws;
  const int64_t a = p / (int64_t(g.tt) * plane);
  int64_t r = p - a * g.tt * plane;
  const int ct = min(g.tt, g.T - int(a) * g.tt);
  const int64_t tile_row = int64_t(ct) * g.th * g.Ws;
  const int64_t b = r / tile_row;
  r -= b * tile_row;
  const int cy = min(g.th, g.Hs - int(b) * g.th);
  const int64_t tile_sz = int64_t(ct) * cy * g.tw;
  const int64_t c = r / tile_sz;
  r -= c * tile_sz;
  const int cx = min(g.tw, g.Ws - int(c) * g.tw);
  const int64_t t_in = r / (int64_t(cy) * cx);
  const int64_t rem = r - t_in * cy * cx;
  const int64_t y_in = rem / cx;
  const int64_t x_in = rem - y_in * cx;
  const int64_t t = a * g.tt + t_in, y = b * g.th + y_in, x = c * g.tw + x_in;
  return (t * g.Hs + y) * g.Ws + x;
}

// frame-major index f -> tile-major position (the inverse of tile_to_frame).
__device__ __forceinline__ int64_t frame_to_tile(int64_t f, const Grid3& g) {
  const int64_t plane = int64_t(g.Hs) * g.Ws;
  const int64_t t = f / plane;
  const int64_t rem = f - t * plane;
  const int64_t y = rem / g.Ws, x = rem - (rem / g.Ws) * g.Ws;
  const int64_t a = t / g.tt, b = y / g.th, c = x / g.tw;
  const int ct = min(g.tt, g.T - int(a) * g.tt);
  const int cy = min(g.th, g.Hs - int(b) * g.th);
  const int cx = min(g.tw, g.Ws - int(c) * g.tw);
  return a * g.tt * plane + int64_t(ct) * (b * g.th) * g.Ws + int64_t(ct) * cy * (c * g.tw) +
         ((t - a * g.tt) * cy + (y - b * g.th)) * cx + (x - c * g.tw);
}

// kForward: in [BH, n, row] -> out [BH, n_pad, row] (tile-major, zero tail).
// !kForward: in [BH, n_pad, row] -> out [BH, n, row] (frame-major).
template <bool kForward>
__global__ void __launch_bounds__(kThreads) tile_gather_kernel(const uint4* __restrict__ in,
                                                                uint4* __restrict__ out, int BH,
                                                                int64_t n, int64_t n_pad,
                                                                int vec_per_row, Grid3 g) {
  __shared__ int64_t src_pos[kChunk];
  const int64_t n_out = kForward ? n_pad : n;
  const int64_t n_in = kForward ? n : n_pad;
  const int64_t pos0 = int64_t(blockIdx.x) * kChunk;
  const int64_t left = n_out - pos0;
  const int rows_here = left < kChunk ? int(left) : kChunk;
  if (threadIdx.x < rows_here) {
    const int64_t p = pos0 + threadIdx.x;
    int64_t s;
    if (kForward) s = p < n ? tile_to_frame(p, g) : -1;
    else s = frame_to_tile(p, g);
    src_pos[threadIdx.x] = s;
  }
  __syncthreads();

  const int per_bh = rows_here * vec_per_row;
  for (int bh = 0; bh < BH; ++bh) {
    const uint4* src_base = in + int64_t(bh) * n_in * vec_per_row;
    uint4* dst_base = out + (int64_t(bh) * n_out + pos0) * vec_per_row;
    // 4 independent 16-byte moves in flight per thread
    for (int i0 = threadIdx.x; i0 < per_bh; i0 += 4 * kThreads) {
      uint4 val[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int i = i0 + u * kThreads;
        val[u] = make_uint4(0u, 0u, 0u, 0u);
        if (i < per_bh) {
          const int row = i / vec_per_row, col = i - row * vec_per_row;
          const int64_t s = src_pos[row];
          if (s >= 0) val[u] = __ldcs(src_base + s * vec_per_row + col);
        }
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int i = i0 + u * kThreads;
        if (i < per_bh) dst_base[i] = val[u];
      }
    }
  }
}

bsa_status check_permute_args(const void* in, const void* out, int B, int H, int T, int Hs,
                              int Ws, int d, int tt, int th, int tw, int n_pad) {
  if (!in || !out) return BSA_ERR_INVALID_ARG;
  if (B <= 0 || H <= 0 || T <= 0 || Hs <= 0 || Ws <= 0 || d <= 0 || tt <= 0 || th <= 0 ||
      tw <= 0)
    return BSA_ERR_INVALID_ARG;
  if (d % 8 != 0) return BSA_ERR_UNSUPPORTED;
  const int64_t n = int64_t(T) * Hs * Ws;
  if (n_pad < n) return BSA_ERR_INVALID_ARG;
  if (int64_t(B) * H * n_pad * d >= (int64_t(1) << 40)) return BSA_ERR_OVERFLOW;
  if (int64_t(B) * H >= (int64_t(1) << 31)) return BSA_ERR_OVERFLOW;
  if (!bsa::aligned16(in) || !bsa::aligned16(out)) return BSA_ERR_MISALIGNED;
  return BSA_OK;
}

template <bool kForward>
bsa_status launch_gather(const void* in, void* out, int B, int H, int T, int Hs, int Ws, int d,
                         int tt, int th, int tw, int n_pad, void* stream) {
  bsa_status st = check_permute_args(in, out, B, H, T, Hs, Ws, d, tt, th, tw, n_pad);
  if (st != BSA_OK) return st;
  const int64_t n = int64_t(T) * Hs * Ws;
  const int64_t n_out = kForward ? int64_t(n_pad) : n;
  const int64_t grid = (n_out + kChunk - 1) / kChunk;
  if (grid >= (int64_t(1) << 31)) return BSA_ERR_OVERFLOW;
  Grid3 g{T, Hs, Ws, tt, th, tw};
  tile_gather_kernel<kForward><<<unsigned(grid), kThreads, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<const uint4*>(in), static_cast<uint4*>(out), B * H, n, n_pad, d / 8, g);
  return bsa::launch_status();
}

}  // namespace

extern "C" bsa_status bsa_tile_permute(const void* in, void* out, int B, int H, int T, int Hs,
                                       int Ws, int d, int tt, int th, int tw, int n_pad,
                                       void* stream) {
  return launch_gather<true>(in, out, B, H, T, Hs, Ws, d, tt, th, tw, n_pad, stream);
}

extern "C" bsa_status bsa_tile_unpermute(const void* in, void* out, int B, int H, int T, int Hs,
                                         int Ws, int d, int tt, int th, int tw, int n_pad,
                                         void* stream) {
  return launch_gather<false>(in, out, B, H, T, Hs, Ws, d, tt, th, tw, n_pad, stream);
}
