// bsa_pack.cu -- per-head block masks -> CRM rows, counts, row offsets,
// ascending key-block lists and the schedule (the forward's work order).
//
// CRM layout ("ScalingAttention", Sec. 4.3.2 and Appendix E, Algorithm 2): one
// row of uint32 words per query block; bit j of word w is key block 32*w + j
// (the iterator's base grows by 32 per word and the index is base + CTZ).
//
// Seven launches on the caller's stream (five below one window of rows):
//   1. rows:        one warp per row; a coalesced read of the row per word,
//                   __ballot_sync builds the word, popcounts sum.  Two
//                   variants: a dense uint8 mask (bsa_pack_mask), or a
//                   per-head threshold map with one threshold per head,
//                   keeping block (u, v) when T(u, v) <= p_h (Sec. 4.1.2,
//                   M_p = 1(T <= p); Algorithm 1 picks p per layer, timestep
//                   and head; bsa_pack_mask_from_threshold).
//   2. tile_hist:   rows are cut into tiles of kTileRows; one CTA per tile
//                   histograms its counts in shared memory and sums them.
//   3. tile_scan:   one CTA; exclusive scan of the tile sums (row bases), and
//                   of the histograms in (count descending, tile ascending)
//                   order, which gives every (tile, count) its first slot in
//                   the schedule.
//   4. tile_place:  one CTA per tile; row_offsets from a block scan, then the
//                   tile's warps take turns placing their rows at their
//                   count's next slot -- in row order, so the sort is stable.
//   5. head_mix:    distinct heads per window of 148 entries of that order.
//   6. head_major:  if those heads' K and V, on average over the windows, do
//                   not fit in L2, the schedule becomes count-descending
//                   within each head, heads in order (a counting sort per
//                   head, one CTA each).
//   7. write_lists: one warp per row; words are taken one at a time and each
//                   lane writes its key block at the row's running offset, so
//                   each store instruction writes consecutive addresses.
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>

#include "bsa.h"
#include "bsa_internal.h"

namespace {

constexpr int kRowWarps = 8;  // warps (rows) per block of the row-parallel launches

// One row per warp.  `kept(j)` tells whether key block j (< nb_k) is kept.
// Words are built 32 at a time: for word k of the group every lane tests its
// key block and a ballot forms the word, which lane k keeps; the group is then
// stored with one coalesced write.  Loads of a partly filled last word are
// clamped to the row, and lanes past its end vote false.  (Unrolled by 8 at 32
// registers: measured faster than issuing all of a group's loads up front at
// 58-63 registers, where fewer warps fit on an SM.)
template <typename Kept>
__device__ __forceinline__ void pack_one_row(const Kept kept, int nb_k, int words,
                                             uint32_t* __restrict__ out, int32_t* count) {
  const int lane = threadIdx.x & 31;
  int total = 0;
  for (int w0 = 0; w0 < words; w0 += 32) {
    const int n = min(32, words - w0);
    uint32_t mine = 0;
#pragma unroll 8
    for (int k = 0; k < n; ++k) {
      const int j = (w0 + k) * 32 + lane;
      const bool keep = kept(min(j, nb_k - 1)) & (j < nb_k);
      const uint32_t word = __ballot_sync(0xffffffffu, keep);
      mine = lane == k ? word : mine;
    }
    if (lane < n) out[w0 + lane] = mine;
    total += __popc(mine);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) total += __shfl_xor_sync(0xffffffffu, total, o);
  if (lane == 0) *count = total;
}

// Row tests, passed by value so their state stays in registers.
struct DenseKept {
  const uint8_t* row;
  __device__ __forceinline__ bool operator()(int j) const { return __ldg(row + j) != 0; }
};
struct ThresholdKept {
  const float* row;
  float p;
  __device__ __forceinline__ bool operator()(int j) const { return __ldg(row + j) <= p; }
};

__global__ void __launch_bounds__(256) pack_rows_kernel(const uint8_t* __restrict__ dense,
                                                        int rows, int nb_k, int words,
                                                        uint32_t* __restrict__ bits,
                                                        int32_t* __restrict__ counts) {
  const int n_warps = gridDim.x * kRowWarps;
  for (int r = blockIdx.x * kRowWarps + (threadIdx.x >> 5); r < rows; r += n_warps) {
    const uint8_t* row = dense + size_t(r) * nb_k;
    pack_one_row(DenseKept{row}, nb_k, words, bits + size_t(r) * words, counts + r);
  }
}

// Threshold rows: row r = (b, h, u) reads map row (h, u), the same for every
// batch item (map_rows = H * nb_q).  A NaN threshold compares false: never kept.
__global__ void __launch_bounds__(256)
    pack_threshold_rows_kernel(const float* __restrict__ thr, const float* __restrict__ p,
                               int nb_q, int map_rows, int rows, int nb_k, int words,
                               uint32_t* __restrict__ bits, int32_t* __restrict__ counts) {
  const int n_warps = gridDim.x * kRowWarps;
  for (int r = blockIdx.x * kRowWarps + (threadIdx.x >> 5); r < rows; r += n_warps) {
    const int hu = r % map_rows;
    const float p_h = __ldg(p + hu / nb_q);
    const float* row = thr + size_t(hu) * nb_k;
    pack_one_row(ThresholdKept{row, p_h}, nb_k, words, bits + size_t(r) * words, counts + r);
  }
}

// ---------------------------------------------------------------------------
// Offsets and the stable count-descending schedule, over tiles of kTileRows
// rows (one thread per row in the tile launches).  The histograms are kept
// "count descending major": entry (d, t) with d = nb_k - count is at
// d * tiles + t, so that one contiguous exclusive scan gives every (count,
// tile) pair its first slot in the schedule.
// ---------------------------------------------------------------------------
constexpr int kTileRows = 1024;
constexpr int kTileWarps = kTileRows / 32;
constexpr int kScanRun = 8;  // values per thread in one pass of a chunked scan
// Dynamic shared memory any sort launch asks for, and so the largest per-count
// table a tile keeps there: nb_k + 1 ints.
constexpr size_t kMaxDynamicSmem = 196608;
constexpr int kMaxBins = int(kMaxDynamicSmem / sizeof(int32_t));

// Block-wide exclusive scan of one value per thread (kTileRows threads);
// returns the prefix and writes the block total to *total.  `smem` holds 33
// ints.  Starts and ends with a barrier's worth of ordering: shared-memory
// writes made before the call are visible to every thread after it.
__device__ __forceinline__ int block_exclusive_scan(int x, int* smem, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int incl = x;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) smem[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    const int v = smem[lane];
    int vi = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, vi, o);
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

// In-place exclusive scan of a[0..n) by one CTA of kTileRows threads, in
// chunks of kScanChunk values staged through shared memory `buf` (coalesced
// global reads and writes; each thread scans a contiguous run of kScanRun
// values of the chunk).  Rows of 32 values are padded by one word so that the
// runs of a warp fall in distinct banks.  Returns the total.
constexpr int kScanChunk = kTileRows * kScanRun;
constexpr int kScanBufInts = kScanChunk + kScanChunk / 32;
__device__ __forceinline__ int padded(int i) { return i + (i >> 5); }

__device__ __forceinline__ int cta_exclusive_scan_inplace(int32_t* a, int n, int* smem,
                                                          int* buf) {
  int carry = 0;
  for (int base = 0; base < n; base += kScanChunk) {
    const int m = min(kScanChunk, n - base);
    for (int i = threadIdx.x; i < kScanChunk; i += kTileRows)
      buf[padded(i)] = i < m ? a[base + i] : 0;
    __syncthreads();
    const int i0 = threadIdx.x * kScanRun;
    int v[kScanRun];
    int run = 0;
#pragma unroll
    for (int k = 0; k < kScanRun; ++k) {
      v[k] = buf[padded(i0 + k)];
      run += v[k];
    }
    int chunk_total;
    int pre = carry + block_exclusive_scan(run, smem, &chunk_total);
#pragma unroll
    for (int k = 0; k < kScanRun; ++k) {
      buf[padded(i0 + k)] = pre;
      pre += v[k];
    }
    __syncthreads();
    for (int i = threadIdx.x; i < m; i += kTileRows) a[base + i] = buf[padded(i)];
    __syncthreads();  // the next chunk reuses buf
    carry += chunk_total;
  }
  return carry;
}

// Lanes of `act` whose key equals this lane's key, for keys below 2^key_bits:
// one ballot per key bit, keeping the lanes that agree on every bit.  Every
// lane of `act` must call it.
__device__ __forceinline__ unsigned equal_keys(unsigned act, int key, int key_bits) {
  unsigned peers = act;
  for (int b = 0; b < key_bits; ++b) {
    const bool one = (key >> b) & 1;
    const unsigned ones = __ballot_sync(act, one);
    peers &= one ? ones : ~ones;
  }
  return peers;
}

// One CTA per tile: per-count histogram of the tile's rows and their count sum.
__global__ void __launch_bounds__(kTileRows)
    tile_hist_kernel(const int32_t* __restrict__ counts, int rows, int nb_k, int tiles,
                     int32_t* __restrict__ hist, int32_t* __restrict__ tile_sum) {
  extern __shared__ int32_t bins_smem[];  // nb_k + 1
  __shared__ int scan_smem[33];
  const int bins = nb_k + 1;
  for (int i = threadIdx.x; i < bins; i += kTileRows) bins_smem[i] = 0;
  __syncthreads();
  const int r = blockIdx.x * kTileRows + threadIdx.x;
  const int c = r < rows ? counts[r] : 0;
  if (r < rows) atomicAdd(&bins_smem[nb_k - c], 1);
  int total;
  block_exclusive_scan(c, scan_smem, &total);  // the tile's sum; orders the atomics
  for (int d = threadIdx.x; d < bins; d += kTileRows)
    hist[size_t(d) * tiles + blockIdx.x] = bins_smem[d];
  if (threadIdx.x == 0) tile_sum[blockIdx.x] = total;
}

// One CTA: tile sums -> tile row bases (and the grand total into
// row_offsets[rows]); histograms -> first schedule slot of every (count, tile).
__global__ void __launch_bounds__(kTileRows, 1)
    tile_scan_kernel(int rows, int nb_k, int tiles, int32_t* __restrict__ hist,
                     int32_t* __restrict__ tile_sum, int32_t* __restrict__ row_offsets,
                     int32_t* __restrict__ mix_sum) {
  __shared__ int scan_smem[33];
  __shared__ int buf[kScanBufInts];
  if (threadIdx.x == 0) *mix_sum = 0;  // summed by head_mix_kernel, two launches later
  const int total = cta_exclusive_scan_inplace(tile_sum, tiles, scan_smem, buf);
  if (threadIdx.x == 0) row_offsets[rows] = total;
  cta_exclusive_scan_inplace(hist, (nb_k + 1) * tiles, scan_smem, buf);
}

// One CTA per tile: row_offsets of the tile's rows, then stable placement of
// every row at its count's slot for this tile plus the number of rows of the
// tile before it with the same count.  Within a warp that number comes from
// equal-key lane masks; across warps (kParallelRanks) from per-warp counts per
// key, scanned over the warps -- shared memory for 33 tables of nb_k + 1 ints;
// otherwise the warps take turns, each advancing per-key counters in order.
template <bool kParallelRanks>
__global__ void __launch_bounds__(kTileRows)
    tile_place_kernel(const int32_t* __restrict__ counts, int rows, int nb_k, int tiles,
                      const int32_t* __restrict__ first, const int32_t* __restrict__ tile_base,
                      int32_t* __restrict__ row_offsets, int32_t* __restrict__ schedule) {
  extern __shared__ int32_t place_smem[];
  __shared__ int scan_smem[33];
  const int bins = nb_k + 1;
  int32_t* next_slot = place_smem;          // [bins], indexed by nb_k - count
  int32_t* warp_hist = place_smem + bins;  // [kTileWarps][bins] (kParallelRanks)
  const int t = blockIdx.x;
  for (int d = threadIdx.x; d < bins; d += kTileRows) next_slot[d] = first[size_t(d) * tiles + t];
  if (kParallelRanks)
    for (int i = threadIdx.x; i < kTileWarps * bins; i += kTileRows) warp_hist[i] = 0;
  const int r = t * kTileRows + threadIdx.x;
  const bool active = r < rows;
  const int c = active ? counts[r] : 0;
  int tile_total;
  const int pre = block_exclusive_scan(c, scan_smem, &tile_total);  // also publishes the tables
  if (active) row_offsets[r] = tile_base[t] + pre;

  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const unsigned below = (1u << lane) - 1u;
  const int key_bits = 32 - __clz(nb_k);  // keys d = nb_k - c lie in [0, nb_k]
  const unsigned act = __ballot_sync(0xffffffffu, active);
  const int d = nb_k - c;
  if (kParallelRanks) {
    unsigned peers = 0;
    if (active) {
      peers = equal_keys(act, d, key_bits);
      if ((peers & below) == 0) warp_hist[warp * bins + d] = __popc(peers);
    }
    __syncthreads();
    for (int k = threadIdx.x; k < bins; k += kTileRows) {  // exclusive scan over the warps
      int run = 0;
      for (int w = 0; w < kTileWarps; ++w) {
        const int x = warp_hist[w * bins + k];
        warp_hist[w * bins + k] = run;
        run += x;
      }
    }
    __syncthreads();
    if (active) schedule[next_slot[d] + warp_hist[warp * bins + d] + __popc(peers & below)] = r;
  } else {
    for (int w = 0; w < kTileWarps; ++w) {
      if (warp == w && active) {
        const unsigned peers = equal_keys(act, d, key_bits);
        const int rank = __popc(peers & below);
        const int pos = next_slot[d] + rank;
        schedule[pos] = r;
        __syncwarp(act);
        if (rank == 0) next_slot[d] = pos + __popc(peers);
      }
      __syncthreads();
    }
  }
}

// ---------------------------------------------------------------------------
// Head-major schedule.  The count order above interleaves heads wherever their
// rows have similar counts; then the query tiles in flight at one time read
// the K and V of many heads, which do not fit in L2 together (top-p masks at
// HunyuanVideo 768p: 20 of 24 heads per wave of 148 tiles, 139 GB of DRAM
// reads per forward).  So the mean number of distinct heads over the order's
// full windows of kMixWindow entries (one wave of a B200) is measured, and
// when that many heads' K and V -- nb_k key blocks of kKeyBlockBytes each --
// exceed the L2 capacity, the schedule becomes count-descending within each
// head, heads in order (ties by row id, as above).  The packing does not see
// the head dimension or the block size, so a key block is costed as 128
// tokens of K and V at d = 128 in bf16.
// ---------------------------------------------------------------------------
constexpr int kMixWindow = 148;
constexpr int64_t kKeyBlockBytes = 2 * 128 * 128 * 2;
constexpr int kMixMaxHeads = 8192;    // bitmap of one window: 1 KB of shared memory per warp
constexpr int kMixMaxRowsPerHead = 8192;
constexpr int kMixWarps = 8;

// One warp per window: the window's heads as bits of a shared-memory bitmap,
// their popcount added to *mix_sum.
__global__ void __launch_bounds__(kMixWarps * 32)
    head_mix_kernel(const int32_t* __restrict__ schedule, int nb_q, int heads, int windows,
                    int32_t* __restrict__ mix_sum) {
  __shared__ uint32_t seen[kMixWarps][kMixMaxHeads / 32];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int w = blockIdx.x * kMixWarps + warp;
  if (w >= windows) return;
  const int words = (heads + 31) / 32;
  uint32_t* bm = seen[warp];
  for (int i = lane; i < words; i += 32) bm[i] = 0u;
  __syncwarp();
  for (int i = lane; i < kMixWindow; i += 32) {
    const int h = schedule[w * kMixWindow + i] / nb_q;
    atomicOr(&bm[h >> 5], 1u << (h & 31));
  }
  __syncwarp();
  int distinct = 0;
  for (int i = lane; i < words; i += 32) distinct += __popc(bm[i]);
  for (int o = 16; o > 0; o >>= 1) distinct += __shfl_xor_sync(0xffffffffu, distinct, o);
  if (lane == 0) atomicAdd(mix_sum, distinct);
}

// One CTA per head (kTileRows threads), only when the windows' heads, on
// average, do not fit in L2 together: a counting sort of the head's rows by count,
// descending.  Histogram of keys d = nb_k - count in shared memory, exclusive
// scan of it (chunks of kTileRows bins), then the rows in order, a chunk of
// kTileRows at a time, the chunk's warps taking turns: each lane's slot is
// its key's next slot plus the lanes before it with the same key, so equal
// counts keep ascending row order.
__global__ void __launch_bounds__(kTileRows)
    head_major_kernel(const int32_t* __restrict__ counts, int nb_q, int nb_k, int windows,
                      int64_t l2_bytes, const int32_t* __restrict__ mix_sum,
                      int32_t* __restrict__ schedule) {
  // the count order's waves touch few enough heads: their K and V stay in L2
  if (int64_t(*mix_sum) * nb_k * kKeyBlockBytes <= int64_t(windows) * l2_bytes) return;
  extern __shared__ int32_t next_slot[];        // nb_k + 1 bins
  __shared__ int scan_smem[33];
  const int bins = nb_k + 1;
  const int64_t base = int64_t(blockIdx.x) * nb_q;
  for (int d = threadIdx.x; d < bins; d += kTileRows) next_slot[d] = 0;
  __syncthreads();
  for (int i = threadIdx.x; i < nb_q; i += kTileRows) atomicAdd(&next_slot[nb_k - counts[base + i]], 1);
  __syncthreads();
  int carry = 0;
  for (int d0 = 0; d0 < bins; d0 += kTileRows) {
    const int d = d0 + int(threadIdx.x);
    const int x = d < bins ? next_slot[d] : 0;
    int chunk_total;
    const int pre = block_exclusive_scan(x, scan_smem, &chunk_total);
    if (d < bins) next_slot[d] = carry + pre;
    carry += chunk_total;
  }
  __syncthreads();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const unsigned below = (1u << lane) - 1u;
  const int key_bits = 32 - __clz(nb_k);
  for (int i0 = 0; i0 < nb_q; i0 += kTileRows) {
    const int i = i0 + int(threadIdx.x);
    const bool active = i < nb_q;
    const unsigned act = __ballot_sync(0xffffffffu, active);
    const int d = active ? nb_k - counts[base + i] : 0;
    for (int w = 0; w < kTileWarps; ++w) {
      if (warp == w && active) {
        const unsigned peers = equal_keys(act, d, key_bits);
        const int rank = __popc(peers & below);
        const int pos = next_slot[d] + rank;
        schedule[base + pos] = int32_t(base + i);
        __syncwarp(act);
        if (rank == 0) next_slot[d] = pos + __popc(peers);
      }
      __syncthreads();
    }
  }
}

// One warp per row.  The row's words are loaded one per lane, then taken one
// at a time (broadcast by shuffle): lane j owns key block 32*w + j and, if the
// bit is set, writes it at the row's running offset plus the number of set
// bits below it, so each store instruction writes consecutive addresses.
__global__ void __launch_bounds__(256) write_lists_kernel(const uint32_t* __restrict__ bits,
                                                          int rows, int words,
                                                          const int32_t* __restrict__ row_offsets,
                                                          int32_t* __restrict__ col_idx) {
  const int lane = threadIdx.x & 31;
  const uint32_t below = (1u << lane) - 1u;
  const int n_warps = gridDim.x * kRowWarps;
  for (int r = blockIdx.x * kRowWarps + (threadIdx.x >> 5); r < rows; r += n_warps) {
    const uint32_t* row = bits + size_t(r) * words;
    int out = row_offsets[r];
    for (int w0 = 0; w0 < words; w0 += 32) {
      const uint32_t mine = w0 + lane < words ? row[w0 + lane] : 0u;
      const int n = min(32, words - w0);
      for (int k = 0; k < n; ++k) {
        const uint32_t word = __shfl_sync(0xffffffffu, mine, k);
        if ((word >> lane) & 1u) col_idx[out + __popc(word & below)] = (w0 + k) * 32 + lane;
        out += __popc(word);
      }
    }
  }
}

int num_tiles(int64_t rows) { return int((rows + kTileRows - 1) / kTileRows); }

// Workspace ints: the (count, tile) table, the tile sums and the head-mix sum.
int64_t workspace_ints(int64_t rows, int nb_k) {
  const int64_t tiles = num_tiles(rows);
  return (int64_t(nb_k) + 1) * tiles + tiles + 1;
}

// Grid of the row-parallel launches: kRowWarps warps per block, one row per
// warp, so that every row's loads are in flight at once and blocks turn over
// as rows finish (the kernels still stride over rows past the grid).
int row_grid(int64_t rows) {
  const int64_t want_blocks = (rows + kRowWarps - 1) / kRowWarps;
  return int(want_blocks < (int64_t(1) << 30) ? want_blocks : (int64_t(1) << 30));
}

// Checks shared by every packing entry point (before any CUDA call).
bsa_status check_pack_args(int B, int H, int nb_q, int nb_k, const void* bits,
                           const void* counts, const void* row_offsets, const void* col_idx,
                           const void* schedule) {
  if (!bits || !counts || !row_offsets || !schedule) return BSA_ERR_INVALID_ARG;
  if (B <= 0 || H <= 0 || nb_q <= 0 || nb_k <= 0) return BSA_ERR_INVALID_ARG;
  const int64_t rows = int64_t(B) * H * nb_q;
  if (rows * int64_t(nb_k) >= (int64_t(1) << 31)) return BSA_ERR_OVERFLOW;
  if (nb_k + 1 > kMaxBins) return BSA_ERR_UNSUPPORTED;
  if (!bsa::aligned4(bits) || !bsa::aligned4(counts) || !bsa::aligned4(row_offsets) ||
      !bsa::aligned4(schedule) || (col_idx && !bsa::aligned4(col_idx)))
    return BSA_ERR_MISALIGNED;
  return BSA_OK;
}

// Launches 2-5, after counts and bits of every row have been written.
// `scratch` holds workspace_ints(rows, nb_k) ints; its contents on entry do
// not matter (every entry is written before it is read).
bsa_status launch_offsets_schedule_lists(const uint32_t* bits, const int32_t* counts, int rows,
                                         int nb_q, int nb_k, int words, int32_t* row_offsets,
                                         int32_t* col_idx, int32_t* schedule, int32_t* scratch,
                                         cudaStream_t s) {
  const int tiles = num_tiles(rows);
  const int bins = nb_k + 1;
  int32_t* table = scratch;                       // [bins][tiles]
  int32_t* tile_sum = scratch + size_t(bins) * tiles;  // [tiles]
  int32_t* mix_sum = tile_sum + tiles;                 // [1]
  const size_t bins_bytes = size_t(bins) * sizeof(int32_t);
  const size_t ranks_bytes = size_t(kTileWarps + 1) * bins_bytes;
  const bool parallel_ranks = ranks_bytes <= kMaxDynamicSmem;
  const size_t place_bytes = parallel_ranks ? ranks_bytes : bins_bytes;
  if (cudaFuncSetAttribute(tile_hist_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           int(bins_bytes)) != cudaSuccess)
    return BSA_ERR_LAUNCH;
  const cudaError_t attr =
      parallel_ranks ? cudaFuncSetAttribute(tile_place_kernel<true>,
                                            cudaFuncAttributeMaxDynamicSharedMemorySize,
                                            int(place_bytes))
                     : cudaFuncSetAttribute(tile_place_kernel<false>,
                                            cudaFuncAttributeMaxDynamicSharedMemorySize,
                                            int(place_bytes));
  if (attr != cudaSuccess) return BSA_ERR_LAUNCH;
  tile_hist_kernel<<<tiles, kTileRows, bins_bytes, s>>>(counts, rows, nb_k, tiles, table,
                                                       tile_sum);
  if (bsa::launch_status() != BSA_OK) return BSA_ERR_LAUNCH;
  tile_scan_kernel<<<1, kTileRows, 0, s>>>(rows, nb_k, tiles, table, tile_sum, row_offsets,
                                           mix_sum);
  if (bsa::launch_status() != BSA_OK) return BSA_ERR_LAUNCH;
  if (parallel_ranks)
    tile_place_kernel<true><<<tiles, kTileRows, place_bytes, s>>>(
        counts, rows, nb_k, tiles, table, tile_sum, row_offsets, schedule);
  else
    tile_place_kernel<false><<<tiles, kTileRows, place_bytes, s>>>(
        counts, rows, nb_k, tiles, table, tile_sum, row_offsets, schedule);
  if (bsa::launch_status() != BSA_OK) return BSA_ERR_LAUNCH;
  const int heads = rows / nb_q, windows = rows / kMixWindow;
  if (windows > 0 && heads <= kMixMaxHeads && nb_q <= kMixMaxRowsPerHead) {
    head_mix_kernel<<<(windows + kMixWarps - 1) / kMixWarps, kMixWarps * 32, 0, s>>>(
        schedule, nb_q, heads, windows, mix_sum);
    if (bsa::launch_status() != BSA_OK) return BSA_ERR_LAUNCH;
    if (cudaFuncSetAttribute(head_major_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             int(bins_bytes)) != cudaSuccess)
      return BSA_ERR_LAUNCH;
    int dev = 0, l2 = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&l2, cudaDevAttrL2CacheSize, dev) != cudaSuccess || l2 <= 0)
      return BSA_ERR_LAUNCH;
    head_major_kernel<<<heads, kTileRows, bins_bytes, s>>>(counts, nb_q, nb_k, windows,
                                                          int64_t(l2), mix_sum, schedule);
    if (bsa::launch_status() != BSA_OK) return BSA_ERR_LAUNCH;
  }
  if (col_idx) {
    write_lists_kernel<<<row_grid(rows), 256, 0, s>>>(bits, rows, words, row_offsets, col_idx);
    if (bsa::launch_status() != BSA_OK) return BSA_ERR_LAUNCH;
  }
  return BSA_OK;
}

}  // namespace

static_assert(bsa::kPackMaxNbK + 1 == kMaxBins, "packing limit");

size_t bsa::pack_scratch_bytes(int64_t rows, int nb_k) {
  const size_t bytes = size_t(workspace_ints(rows, nb_k)) * sizeof(int32_t);
  return (bytes + 255) & ~size_t(255);
}

bsa_status bsa::pack_finish(const uint32_t* bits, const int32_t* counts, int rows, int nb_q,
                            int nb_k, int32_t* row_offsets, int32_t* col_idx, int32_t* schedule,
                            void* scratch, cudaStream_t s) {
  return launch_offsets_schedule_lists(bits, counts, rows, nb_q, nb_k, (nb_k + 31) / 32, row_offsets,
                                       col_idx, schedule, static_cast<int32_t*>(scratch), s);
}

extern "C" size_t bsa_pack_mask_workspace(int B, int H, int nb_q, int nb_k) {
  if (B <= 0 || H <= 0 || nb_q <= 0 || nb_k <= 0) return 0;
  return bsa::pack_scratch_bytes(int64_t(B) * H * nb_q, nb_k);
}

extern "C" bsa_status bsa_pack_mask(const uint8_t* dense, int B, int H, int nb_q, int nb_k,
                                    uint32_t* bits, int32_t* counts, int32_t* row_offsets,
                                    int32_t* col_idx, int32_t* schedule, void* workspace,
                                    size_t workspace_bytes, void* stream) {
  if (!dense) return BSA_ERR_INVALID_ARG;
  const bsa_status st = check_pack_args(B, H, nb_q, nb_k, bits, counts, row_offsets, col_idx,
                                        schedule);
  if (st != BSA_OK) return st;
  const size_t need = bsa_pack_mask_workspace(B, H, nb_q, nb_k);
  if (!workspace || workspace_bytes < need) return BSA_ERR_WORKSPACE;
  if (!bsa::aligned16(workspace)) return BSA_ERR_MISALIGNED;
  if (bsa::num_sms() <= 0) return BSA_ERR_LAUNCH;

  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int rows = B * H * nb_q;
  const int words = (nb_k + 31) / 32;
  pack_rows_kernel<<<row_grid(rows), 256, 0, s>>>(dense, rows, nb_k, words, bits, counts);
  if (bsa::launch_status() != BSA_OK) return BSA_ERR_LAUNCH;
  return launch_offsets_schedule_lists(bits, counts, rows, nb_q, nb_k, words, row_offsets, col_idx,
                                       schedule, static_cast<int32_t*>(workspace), s);
}

extern "C" bsa_status bsa_pack_mask_from_threshold(const float* thr, const float* p, int B,
                                                   int H, int nb_q, int nb_k, uint32_t* bits,
                                                   int32_t* counts, int32_t* row_offsets,
                                                   int32_t* col_idx, int32_t* schedule,
                                                   void* workspace, size_t workspace_bytes,
                                                   void* stream) {
  if (!thr || !p) return BSA_ERR_INVALID_ARG;
  const bsa_status st = check_pack_args(B, H, nb_q, nb_k, bits, counts, row_offsets, col_idx,
                                        schedule);
  if (st != BSA_OK) return st;
  if (!bsa::aligned4(thr) || !bsa::aligned4(p)) return BSA_ERR_MISALIGNED;
  const size_t need = bsa_pack_mask_workspace(B, H, nb_q, nb_k);
  if (!workspace || workspace_bytes < need) return BSA_ERR_WORKSPACE;
  if (!bsa::aligned16(workspace)) return BSA_ERR_MISALIGNED;
  if (bsa::num_sms() <= 0) return BSA_ERR_LAUNCH;

  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int rows = B * H * nb_q;
  const int words = (nb_k + 31) / 32;
  pack_threshold_rows_kernel<<<row_grid(rows), 256, 0, s>>>(thr, p, nb_q, H * nb_q, rows, nb_k,
                                                            words, bits, counts);
  if (bsa::launch_status() != BSA_OK) return BSA_ERR_LAUNCH;
  return launch_offsets_schedule_lists(bits, counts, rows, nb_q, nb_k, words, row_offsets, col_idx,
                                       schedule, static_cast<int32_t*>(workspace), s);
}

// ---------------------------------------------------------------------------
// bsa_pack_mask_noalloc: the same launches as bsa_pack_mask, with the sort's
// scratch in a fixed device array that this library owns, for callers that
// cannot allocate device memory.
//
// The array below lives in every GPU's memory from the moment the library is
// loaded on it until the process exits (512 KiB).  Host code cannot use the
// symbol's name as a device address, so the device address is fetched once per
// device with cudaGetSymbolAddress (with that device current) and cached.
// ---------------------------------------------------------------------------
namespace {

constexpr int kNoallocScratchInts = 131072;  // 512 KiB
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
  if (!dense) return BSA_ERR_INVALID_ARG;
  const bsa_status st = check_pack_args(B, H, nb_q, nb_k, bits, counts, row_offsets, col_idx,
                                        schedule);
  if (st != BSA_OK) return st;
  // the fixed scratch must hold the (count, tile) table and the tile sums
  if (workspace_ints(int64_t(B) * H * nb_q, nb_k) > kNoallocScratchInts) return BSA_ERR_WORKSPACE;
  int32_t* scratch = noalloc_scratch_for_current_device();
  if (!scratch) return BSA_ERR_LAUNCH;
  if (bsa::num_sms() <= 0) return BSA_ERR_LAUNCH;

  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int rows = B * H * nb_q;
  const int words = (nb_k + 31) / 32;
  pack_rows_kernel<<<row_grid(rows), 256, 0, s>>>(dense, rows, nb_k, words, bits, counts);
  if (bsa::launch_status() != BSA_OK) return BSA_ERR_LAUNCH;
  // every scratch entry the sort reads is written earlier in the same call, so
  // whatever an earlier call left there does not matter
  return launch_offsets_schedule_lists(bits, counts, rows, nb_q, nb_k, words, row_offsets, col_idx,
                                       schedule, scratch, s);
}
