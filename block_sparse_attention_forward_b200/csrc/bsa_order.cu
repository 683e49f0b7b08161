// bsa_order.cu -- token orders other than the 3-D tile order, and the row
// gather that applies any order given as a table.
//
// The pages compose block-sparse attention with token reorderings that
// cluster related tokens into the same 128-token block ("ScalingAttention",
// Sec. 5.4-5.5: token permutation eases the 128 x 128 granularity
// bottleneck), and name two more layouts: DFSAttn's Hilbert-curve token
// reordering and Veda's head-aware tiling, where heads use differently shaped
// tiles.  Both are fixed per grid shape, so they are built once on the host
// as tables (a plan), and every step applies them with one gather kernel:
//   out[b, h, i, :] = in[b, h, src[i], :]   (src[i] outside [0, n_in) -> zeros)
// with one table shared by all heads or one table per head.
#include <cuda_runtime.h>
#include <stdint.h>

#include <algorithm>
#include <utility>
#include <vector>

#include "bsa.h"
#include "bsa_internal.h"

namespace {

constexpr int kChunk = 64;     // output positions per CTA
constexpr int kThreads = 256;  // threads per CTA

// blockIdx.y is the table; a shared table serves all B*H heads, a per-head
// table serves the B heads (b, h = blockIdx.y).  The chunk's source rows are
// read once into shared memory, then 16-byte pieces move with 4 loads in
// flight per thread; every store is coalesced.
__global__ void __launch_bounds__(kThreads)
    table_gather_kernel(const uint4* __restrict__ in, uint4* __restrict__ out, int B, int H,
                        int64_t n_in, int64_t n_out, int vec_per_row,
                        const int32_t* __restrict__ src, int per_head) {
  __shared__ int64_t src_pos[kChunk];
  const int table = blockIdx.y;
  const int64_t pos0 = int64_t(blockIdx.x) * kChunk;
  const int64_t left = n_out - pos0;
  const int rows_here = left < kChunk ? int(left) : kChunk;
  if (threadIdx.x < rows_here) {
    const int64_t s = __ldg(src + int64_t(table) * n_out + pos0 + threadIdx.x);
    src_pos[threadIdx.x] = (s >= 0 && s < n_in) ? s : -1;
  }
  __syncthreads();

  const int per_bh = rows_here * vec_per_row;
  const int heads_here = per_head ? B : B * H;
  for (int k = 0; k < heads_here; ++k) {
    const int64_t bh = per_head ? int64_t(k) * H + table : k;
    const uint4* src_base = in + bh * n_in * vec_per_row;
    uint4* dst_base = out + (bh * n_out + pos0) * vec_per_row;
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

// Hilbert index of the point (c[0], c[1], c[2]) = (t, y, x) on the curve over
// the cube of side 2^bits: Skilling's transpose method ("Programming the
// Hilbert curve", AIP Conf. Proc. 707, 2004) -- undo the excess work of the
// inverse map level by level (inversions and exchanges of the low bits), Gray
// encode across the axes, then read the index off the transposed bits, most
// significant level first, axis 0 first.
uint64_t hilbert_index3(uint32_t c0, uint32_t c1, uint32_t c2, int bits) {
  uint32_t c[3] = {c0, c1, c2};
  const uint32_t top = 1u << (bits - 1);
  for (uint32_t q = top; q > 1; q >>= 1) {
    const uint32_t low = q - 1;
    for (int i = 0; i < 3; ++i) {
      if (c[i] & q) {
        c[0] ^= low;
      } else {
        const uint32_t swap = (c[0] ^ c[i]) & low;
        c[0] ^= swap;
        c[i] ^= swap;
      }
    }
  }
  c[1] ^= c[0];
  c[2] ^= c[1];
  uint32_t fold = 0;
  for (uint32_t q = top; q > 1; q >>= 1)
    if (c[2] & q) fold ^= q - 1;
  for (int i = 0; i < 3; ++i) c[i] ^= fold;
  uint64_t index = 0;
  for (int level = bits - 1; level >= 0; --level)
    for (int i = 0; i < 3; ++i) index = (index << 1) | ((c[i] >> level) & 1u);
  return index;
}

bool valid_grid(int T, int Hs, int Ws) {
  return T > 0 && Hs > 0 && Ws > 0 && int64_t(T) * Hs * Ws < (int64_t(1) << 31);
}

}  // namespace

extern "C" bsa_status bsa_hilbert_order(int T, int Hs, int Ws, int32_t* order) {
  if (!order || !valid_grid(T, Hs, Ws)) return BSA_ERR_INVALID_ARG;
  const int side = std::max(T, std::max(Hs, Ws));
  int bits = 1;
  while ((1 << bits) < side) ++bits;
  if (bits > 21) return BSA_ERR_UNSUPPORTED;  // 3 * bits must fit in 64
  const int64_t n = int64_t(T) * Hs * Ws;
  std::vector<std::pair<uint64_t, int32_t>> keyed(static_cast<size_t>(n));
  for (int t = 0; t < T; ++t)
    for (int y = 0; y < Hs; ++y)
      for (int x = 0; x < Ws; ++x) {
        const int32_t f = int32_t((int64_t(t) * Hs + y) * Ws + x);
        keyed[size_t(f)] = {hilbert_index3(t, y, x, bits), f};
      }
  std::sort(keyed.begin(), keyed.end());  // keys are distinct: a bijection on the cube
  for (int64_t i = 0; i < n; ++i) order[i] = keyed[size_t(i)].second;
  return BSA_OK;
}

extern "C" bsa_status bsa_tile_order(int T, int Hs, int Ws, int tt, int th, int tw,
                                     int32_t* order) {
  if (!order || !valid_grid(T, Hs, Ws) || tt <= 0 || th <= 0 || tw <= 0)
    return BSA_ERR_INVALID_ARG;
  int64_t p = 0;
  for (int t0 = 0; t0 < T; t0 += tt)
    for (int y0 = 0; y0 < Hs; y0 += th)
      for (int x0 = 0; x0 < Ws; x0 += tw) {
        const int t1 = std::min(T, t0 + tt), y1 = std::min(Hs, y0 + th),
                  x1 = std::min(Ws, x0 + tw);
        for (int t = t0; t < t1; ++t)
          for (int y = y0; y < y1; ++y)
            for (int x = x0; x < x1; ++x) order[p++] = int32_t((int64_t(t) * Hs + y) * Ws + x);
      }
  return BSA_OK;
}

extern "C" bsa_status bsa_order_tables(const int32_t* order, int n, int n_pad, int32_t* fwd,
                                       int32_t* inv) {
  if (!order || !fwd || !inv || n <= 0 || n_pad < n) return BSA_ERR_INVALID_ARG;
  std::vector<char> seen(static_cast<size_t>(n), 0);
  for (int i = 0; i < n; ++i) {
    const int32_t f = order[i];
    if (f < 0 || f >= n || seen[size_t(f)]) return BSA_ERR_INVALID_ARG;  // not a permutation
    seen[size_t(f)] = 1;
  }
  for (int i = 0; i < n; ++i) {
    fwd[i] = order[i];
    inv[order[i]] = i;
  }
  for (int i = n; i < n_pad; ++i) fwd[i] = -1;
  return BSA_OK;
}

extern "C" bsa_status bsa_gather_rows(const void* in, void* out, int B, int H, int n_in,
                                      int n_out, int d, const int32_t* src, int per_head,
                                      void* stream) {
  if (!in || !out || !src) return BSA_ERR_INVALID_ARG;
  if (B <= 0 || H <= 0 || n_in <= 0 || n_out <= 0 || d <= 0) return BSA_ERR_INVALID_ARG;
  if (per_head != 0 && per_head != 1) return BSA_ERR_INVALID_ARG;
  if (d % 8 != 0) return BSA_ERR_UNSUPPORTED;
  if (int64_t(B) * H * std::max(n_in, n_out) * d >= (int64_t(1) << 40)) return BSA_ERR_OVERFLOW;
  if (int64_t(B) * H >= (int64_t(1) << 31) || (per_head && H > 65535)) return BSA_ERR_OVERFLOW;
  if (!bsa::aligned16(in) || !bsa::aligned16(out) || !bsa::aligned4(src))
    return BSA_ERR_MISALIGNED;
  const int64_t chunks = (int64_t(n_out) + kChunk - 1) / kChunk;
  const dim3 grid(unsigned(chunks), per_head ? unsigned(H) : 1u);
  table_gather_kernel<<<grid, kThreads, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<const uint4*>(in), static_cast<uint4*>(out), B, H, n_in, n_out, d / 8, src,
      per_head);
  return bsa::launch_status();
}
