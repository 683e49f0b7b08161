// bsa_pack.cu -- dense per-head block masks -> CRM rows, counts, row offsets,
// ascending key-block lists and the count-ordered schedule.
//
// CRM layout ("ScalingAttention", Sec. 4.3.2 and Appendix E, Algorithm 2): one
// row of uint32 words per query block; bit j of word w is key block 32*w + j
// (the iterator's base grows by 32 per word and the index is base + CTZ).
//
// Three launches on the caller's stream:
//   1. pack_rows:   one warp per row; a coalesced 32-byte read of the dense row
//                   per word, __ballot_sync builds the word, popcounts sum.
//   2. scan_sort:   one CTA; exclusive prefix of counts -> row_offsets, and a
//                   stable counting sort of rows by count (descending) with
//                   per-warp histograms kept in the caller's workspace.
//   3. write_lists: one warp per row; each lane takes one word, a warp scan of
//                   popcounts gives its output offset, set bits are written in
//                   ascending order.
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>

#include "bsa.h"
#include "bsa_internal.h"

namespace {

constexpr int kSortThreads = 1024;
constexpr int kSortWarps = kSortThreads / 32;

__global__ void __launch_bounds__(256) pack_rows_kernel(const uint8_t* __restrict__ dense,
                                                        int64_t rows, int nb_k, int words,
                                                        uint32_t* __restrict__ bits,
                                                        int32_t* __restrict__ counts) {
  const int lane = threadIdx.x & 31;
  const int64_t warp = (int64_t(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t n_warps = (int64_t(gridDim.x) * blockDim.x) >> 5;
  for (int64_t r = warp; r < rows; r += n_warps) {
    const uint8_t* row = dense + r * nb_k;
    uint32_t* out = bits + r * words;
    int total = 0;
    for (int w = 0; w < words; ++w) {
      const int j = w * 32 + lane;
      const bool kept = (j < nb_k) && (row[j] != 0);
      const uint32_t word = __ballot_sync(0xffffffffu, kept);
      if (lane == 0) out[w] = word;
      total += __popc(word);
    }
    if (lane == 0) counts[r] = total;
  }
}

// Block-wide exclusive scan of one value per thread; returns the prefix and
// writes the block total to *total.  `smem` holds kSortWarps ints.
__device__ __forceinline__ int block_exclusive_scan(int x, int* smem, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int incl = x;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    int y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) smem[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    int v = smem[lane];
    int vi = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      int y = __shfl_up_sync(0xffffffffu, vi, o);
      if (lane >= o) vi += y;
    }
    smem[lane] = vi - v;  // exclusive prefix of warp totals
    if (lane == 31) smem[32] = vi;
  }
  __syncthreads();
  const int result = smem[warp] + incl - x;
  *total = smem[32];
  __syncthreads();
  return result;
}

// hist: kSortWarps * (nb_k + 1) ints of workspace, laid out [count desc][warp]
// so that one flat exclusive scan yields every (warp, count) output base.
__global__ void __launch_bounds__(kSortThreads, 1)
    scan_sort_kernel(const int32_t* __restrict__ counts, int rows, int nb_k,
                     int32_t* __restrict__ row_offsets, int32_t* __restrict__ schedule,
                     int32_t* __restrict__ hist) {
  __shared__ int scan_smem[33];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int n_bins = nb_k + 1;
  const int hist_len = kSortWarps * n_bins;

  // 1. row_offsets = exclusive prefix of counts
  int carry = 0;
  for (int base = 0; base < rows; base += kSortThreads) {
    const int r = base + tid;
    const int c = r < rows ? counts[r] : 0;
    int chunk_total;
    const int pre = block_exclusive_scan(c, scan_smem, &chunk_total);
    if (r < rows) row_offsets[r] = carry + pre;
    carry += chunk_total;
  }
  if (tid == 0) row_offsets[rows] = carry;

  // 2. per-warp histograms of counts over contiguous row segments
  // the histogram is touched through L2 only (atomics, __ldcg/__stcg)
  for (int i = tid; i < hist_len; i += kSortThreads) __stcg(hist + i, 0);
  __syncthreads();
  const int seg = (rows + kSortWarps - 1) / kSortWarps;
  const int seg_lo = min(rows, warp * seg), seg_hi = min(rows, seg_lo + seg);
  for (int r = seg_lo + lane; r < seg_hi; r += 32) {
    const int c = counts[r];
    atomicAdd(&hist[(nb_k - c) * kSortWarps + warp], 1);
  }
  __syncthreads();

  // 3. exclusive scan of hist in (count descending, warp ascending) order
  carry = 0;
  for (int base = 0; base < hist_len; base += kSortThreads) {
    const int i = base + tid;
    const int h = i < hist_len ? __ldcg(hist + i) : 0;
    int chunk_total;
    const int pre = block_exclusive_scan(h, scan_smem, &chunk_total);
    if (i < hist_len) __stcg(hist + i, carry + pre);
    carry += chunk_total;
  }
  __syncthreads();

  // 4. stable placement: each warp walks its segment in row order
  for (int base = seg_lo; base < seg_hi; base += 32) {
    const int r = base + lane;
    const bool active = r < seg_hi;
    const unsigned act = __ballot_sync(0xffffffffu, active);
    if (active) {
      const int c = counts[r];
      const unsigned peers = __match_any_sync(act, c);
      const int rank = __popc(peers & ((1u << lane) - 1u));
      int* slot = &hist[(nb_k - c) * kSortWarps + warp];
      const int pos = __ldcg(slot) + rank;
      schedule[pos] = r;
      __syncwarp(act);
      if (rank == 0) __stcg(slot, pos + __popc(peers));
    }
    __syncwarp();
  }
}

__global__ void __launch_bounds__(256) write_lists_kernel(const uint32_t* __restrict__ bits,
                                                          int64_t rows, int words,
                                                          const int32_t* __restrict__ row_offsets,
                                                          int32_t* __restrict__ col_idx) {
  const int lane = threadIdx.x & 31;
  const int64_t warp = (int64_t(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t n_warps = (int64_t(gridDim.x) * blockDim.x) >> 5;
  for (int64_t r = warp; r < rows; r += n_warps) {
    const uint32_t* row = bits + r * words;
    int out = row_offsets[r];
    for (int w0 = 0; w0 < words; w0 += 32) {
      const int w = w0 + lane;
      uint32_t word = w < words ? row[w] : 0u;
      const int pc = __popc(word);
      int incl = pc;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      int pos = out + incl - pc;
      while (word) {  // ascending: clear the lowest set bit each step
        col_idx[pos++] = w * 32 + (__ffs(word) - 1);
        word &= word - 1u;
      }
      out += __shfl_sync(0xffffffffu, incl, 31);
    }
  }
}

}  // namespace

extern "C" size_t bsa_pack_mask_workspace(int B, int H, int nb_q, int nb_k) {
  (void)B;
  (void)H;
  (void)nb_q;
  if (nb_k <= 0) return 0;
  size_t bytes = size_t(kSortWarps) * size_t(nb_k + 1) * sizeof(int32_t);
  return (bytes + 255) & ~size_t(255);
}

extern "C" bsa_status bsa_pack_mask(const uint8_t* dense, int B, int H, int nb_q, int nb_k,
                                    uint32_t* bits, int32_t* counts, int32_t* row_offsets,
                                    int32_t* col_idx, int32_t* schedule, void* workspace,
                                    size_t workspace_bytes, void* stream) {
  if (!dense || !bits || !counts || !row_offsets || !schedule) return BSA_ERR_INVALID_ARG;
  if (B <= 0 || H <= 0 || nb_q <= 0 || nb_k <= 0) return BSA_ERR_INVALID_ARG;
  const int64_t rows = int64_t(B) * H * nb_q;
  if (rows * int64_t(nb_k) >= (int64_t(1) << 31)) return BSA_ERR_OVERFLOW;
  if (!bsa::aligned4(bits) || !bsa::aligned4(counts) || !bsa::aligned4(row_offsets) ||
      !bsa::aligned4(schedule) || (col_idx && !bsa::aligned4(col_idx)))
    return BSA_ERR_MISALIGNED;
  const size_t need = bsa_pack_mask_workspace(B, H, nb_q, nb_k);
  if (!workspace || workspace_bytes < need) return BSA_ERR_WORKSPACE;
  if (!bsa::aligned16(workspace)) return BSA_ERR_MISALIGNED;
  const int sms = bsa::num_sms();
  if (sms <= 0) return BSA_ERR_LAUNCH;

  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int words = (nb_k + 31) / 32;
  const int64_t want_blocks = (rows + 7) / 8;  // 8 warps per block
  const int grid = int(want_blocks < int64_t(sms) * 8 ? want_blocks : int64_t(sms) * 8);
  pack_rows_kernel<<<grid, 256, 0, s>>>(dense, rows, nb_k, words, bits, counts);
  if (bsa::launch_status() != BSA_OK) return BSA_ERR_LAUNCH;
  scan_sort_kernel<<<1, kSortThreads, 0, s>>>(counts, int(rows), nb_k, row_offsets, schedule,
                                               static_cast<int32_t*>(workspace));
  if (bsa::launch_status() != BSA_OK) return BSA_ERR_LAUNCH;
  if (col_idx) {
    write_lists_kernel<<<grid, 256, 0, s>>>(bits, rows, words, row_offsets, col_idx);
    if (bsa::launch_status() != BSA_OK) return BSA_ERR_LAUNCH;
  }
  return BSA_OK;
}

// ---------------------------------------------------------------------------
// bsa_pack_mask_noalloc: the same three kernels as bsa_pack_mask, with the
// sort's scratch histogram in a fixed device array that this library owns,
// for callers that cannot allocate device memory.
//
// The array below lives in every GPU's memory from the moment the library is
// loaded on it until the process exits (512 KiB).  Host code cannot use the
// symbol's name as a device address, so the device address is fetched once per
// device with cudaGetSymbolAddress (with that device current) and cached.
// ---------------------------------------------------------------------------
namespace {

constexpr int kNoallocMaxNbK = 4095;  // key blocks per row the fixed scratch can sort
constexpr int kNoallocScratchInts = kSortWarps * (kNoallocMaxNbK + 1);
constexpr int kNoallocMaxDevices = 64;

static __device__ __align__(256) int32_t g_pack_scratch[kNoallocScratchInts];

std::mutex g_noalloc_mutex;
int32_t* g_noalloc_scratch_ptr[kNoallocMaxDevices] = {};

// Device address of g_pack_scratch on the current device (looked up on the
// first call per device), or null if the lookup failed.
int32_t* noalloc_scratch_for_current_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kNoallocMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lock(g_noalloc_mutex);
  if (!g_noalloc_scratch_ptr[dev]) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_pack_scratch) != cudaSuccess || !ptr) return nullptr;
    g_noalloc_scratch_ptr[dev] = static_cast<int32_t*>(ptr);
  }
  return g_noalloc_scratch_ptr[dev];
}

}  // namespace

extern "C" bsa_status bsa_pack_mask_noalloc(const uint8_t* dense, int B, int H, int nb_q,
                                            int nb_k, uint32_t* bits, int32_t* counts,
                                            int32_t* row_offsets, int32_t* col_idx,
                                            int32_t* schedule, void* stream) {
  if (!dense || !bits || !counts || !row_offsets || !schedule) return BSA_ERR_INVALID_ARG;
  if (B <= 0 || H <= 0 || nb_q <= 0 || nb_k <= 0) return BSA_ERR_INVALID_ARG;
  if (nb_k > kNoallocMaxNbK) return BSA_ERR_WORKSPACE;  // the fixed scratch is too small
  const int64_t rows = int64_t(B) * H * nb_q;
  if (rows * int64_t(nb_k) >= (int64_t(1) << 31)) return BSA_ERR_OVERFLOW;
  if (!bsa::aligned4(bits) || !bsa::aligned4(counts) || !bsa::aligned4(row_offsets) ||
      !bsa::aligned4(schedule) || (col_idx && !bsa::aligned4(col_idx)))
    return BSA_ERR_MISALIGNED;
  int32_t* scratch = noalloc_scratch_for_current_device();
  if (!scratch) return BSA_ERR_LAUNCH;
  const int sms = bsa::num_sms();
  if (sms <= 0) return BSA_ERR_LAUNCH;

  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int words = (nb_k + 31) / 32;
  const int64_t want_blocks = (rows + 7) / 8;  // 8 warps per block
  const int grid = int(want_blocks < int64_t(sms) * 8 ? want_blocks : int64_t(sms) * 8);
  pack_rows_kernel<<<grid, 256, 0, s>>>(dense, rows, nb_k, words, bits, counts);
  if (bsa::launch_status() != BSA_OK) return BSA_ERR_LAUNCH;
  // scan_sort_kernel zeroes the histogram part of the scratch it uses before
  // counting, so whatever an earlier call left there does not matter
  scan_sort_kernel<<<1, kSortThreads, 0, s>>>(counts, int(rows), nb_k, row_offsets, schedule,
                                               scratch);
  if (bsa::launch_status() != BSA_OK) return BSA_ERR_LAUNCH;
  if (col_idx) {
    write_lists_kernel<<<grid, 256, 0, s>>>(bits, rows, words, row_offsets, col_idx);
    if (bsa::launch_status() != BSA_OK) return BSA_ERR_LAUNCH;
  }
  return BSA_OK;
}
