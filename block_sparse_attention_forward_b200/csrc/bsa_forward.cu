// bsa_forward.cu -- block-sparse attention forward for sm_100a.
//
// What it computes ("ScalingAttention", Sec. 4.3.2): the FlashAttention
// forward whose dense key-block loop is replaced by the CRM forward iterator
// of Appendix E (Algorithm 2), so only the kept key blocks of each query block
// are visited; inside a kept tile the work is a dense tensor-core contraction,
// across tiles an fp32 online softmax.
//
// How (B200-first, not the pages' Hopper design):
//   * persistent grid, one CTA per SM, 192 threads in three roles:
//       warps 0-3  softmax: one query row per thread (TMEM lane = row), online
//                  max/sum in registers, P (bf16) written back into the S
//                  columns of TMEM, O rescaled in TMEM, epilogue;
//       warp  4    producer: walks the CRM words with the Algorithm 2 iterator
//                  and issues TMA loads of K_j, V_j per kept block j into a
//                  ring of shared-memory slots;
//       warp  5    MMA issuer: tcgen05.mma S = Q K_j^T into one of two TMEM S
//                  buffers and O += P V_j.  Q and P are A operands read from
//                  TMEM, so only K and V are read from shared memory (an M=128
//                  N=128 product with both operands in shared memory would
//                  need the whole 128 B/clk shared-memory port by itself).
//                  Per block n it waits for V_n and K_{n+2} first and for P(n)
//                  last, then issues P V_n and S(n+2) back to back: the path
//                  from the softmax's P(n) to the next products holds one
//                  barrier wait, and the tensor core gets sixteen products in
//                  one burst.
//   * TMEM (512 columns): S0 at 0, S1 at 128, O at 256, Q at 384 (bf16 pairs,
//     written by the softmax threads once per tile).  S(n+1) is computed
//     while the softmax works on S(n).
//   * work order: query tiles are taken from the count-descending schedule
//     (heaviest first) in rounds of one tile per CTA, alternating direction
//     (snake_tile)
//   * a tile is always 128 query rows; with 64-token query blocks it holds two
//     query blocks and walks the union of their CRM rows, each row masking the
//     key blocks its own query block did not keep.  Key blocks may be smaller
//     than query blocks (128-row query blocks over 64-key blocks: twice the
//     CRM bits per row, the finer key granularity Sec. 5.4 asks for below 40 %
//     density).  Such blocks are taken in pairs of consecutive kept blocks:
//     the producer loads the two 64-row K (and V) tiles into the two halves of
//     one 128-row ring slot, so every product and softmax pass covers 128
//     keys and the per-tile costs are paid once per pair; a lone last block
//     is loaded into both halves (the second half is masked), so every value
//     the tensor core reads is finite.
//   * the hot waits (every wait of the MMA issuer, the softmax's wait for S)
//     first test the phase inline (mbarrier.test_wait); only a phase still
//     open costs the call into the blocking loop.  Every wait is bounded
//     (about two seconds); a wait that runs out
//     records BSA_ERR_TIMEOUT in a device word, the CTA drains what it has in
//     flight and exits.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "bsa.h"
#include "bsa_internal.h"
#include "sm100_ptx.cuh"

__device__ int g_bsa_device_error = 0;

namespace {

using namespace sm100;

constexpr int kTileM = 128;  // query rows per tile = TMEM lanes
constexpr int kThreads = 192;
constexpr int kMaxStages = 8;  // K/V ring slots (as many as shared memory holds)
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kTmemS0 = 0, kTmemS1 = 128, kTmemO = 256, kTmemQ = 384;
constexpr uint64_t kTimeoutNs = 2000000000ull;
constexpr float kRescaleLog2 = 8.0f;  // lazy-rescale threshold (log2 units)
constexpr int kMaxListRounds = 2048;  // tiles per CTA for tiles of several query blocks

struct FwdParams {
  const __nv_bfloat16* q;   // [BH, n_pad, d]
  const uint32_t* bits;     // [BH, nb, words]
  const int32_t* schedule;  // [BH * nb_q] (used when one query block per tile)
  __nv_bfloat16* out;       // [BH, n_pad, d]
  float* lse;               // [BH, n_pad]
  int BH, nb_q, nb_k, words, n_valid, n_pad;
  int num_tiles, tiles_per_head;
  int use_list;  // tiles of several query blocks: taken in schedule order via a per-CTA list
  float scale_log2;
};

template <int D, int BQ, int BK>
struct Cfg {
  static constexpr int R = kTileM / BQ;                         // query blocks per tile
  static constexpr bool kPairs = BQ == 128 && BK == 64;         // two key blocks per S tile
  static constexpr int kTileN = kPairs ? 2 * BK : BK;           // keys per S tile and ring slot
  static constexpr int kRegions = D / 64;                       // 128-byte column groups
  static constexpr uint32_t kKVRegion = kTileN * 128;
  static constexpr uint32_t kSlotBytes = kRegions * kKVRegion;  // one K or V tile
  static constexpr uint32_t kMaxSmem = 227u * 1024u;
  // tiles of several query blocks keep this CTA's list of tiles in shared memory
  static constexpr int kListInts = R > 1 ? kMaxListRounds : 0;
  static constexpr uint32_t kListBytes = 4u * kListInts + (R > 1 ? 64u : 0u);
  static constexpr int kFitStages = int((kMaxSmem - 256 - kListBytes - 1024) / kSlotBytes);
  static constexpr int kStages = kFitStages > kMaxStages ? kMaxStages : kFitStages;
  static constexpr uint32_t kOffKV = 0;
  static constexpr uint32_t kOffBar = kOffKV + kStages * kSlotBytes;
  static constexpr uint32_t kOffList = kOffBar + 256;
  // + barriers + list + alignment slack; at least 120 KB so that a second CTA
  // never fits on the SM (each CTA owns all 512 TMEM columns)
  static constexpr uint32_t kSmemUsed = kOffList + kListBytes + 1024;
  static constexpr uint32_t kSmemBytes = kSmemUsed > 120u * 1024u ? kSmemUsed : 120u * 1024u;
  static constexpr uint32_t kIdescS = idesc_bf16_f32(kTileM, kTileN, false);
  static_assert(kSmemUsed <= kMaxSmem, "shared memory budget");
  // K(n+2) is waited for before V(n) is released
  static_assert(kStages >= 4, "ring too short for the MMA issue order");
  static constexpr uint32_t kIdescPV = idesc_bf16_f32(kTileM, D, true);
};

struct Barriers {
  uint64_t q_full;  // the softmax threads have written this tile's Q into TMEM
  uint64_t kv_full[kMaxStages], kv_empty[kMaxStages];
  uint64_t s_full[2], p_full[2];
  uint64_t o_done[2];  // PV(k) completes on o_done[k & 1]
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
};

// Bounded wait, slow path: spin until the phase of `parity` completed (true)
// or this CTA gives up (timeout here, or another role already aborted).  With
// abort == nullptr the wait ignores the other roles and ends only on the
// phase or the timeout: the drains use it, so that a CTA that is giving up
// still lets its copies land and its products finish before it frees TMEM
// and exits.
__device__ __noinline__ bool wait_barrier_slow(uint32_t bar, uint32_t parity, volatile int* abort,
                                               uint64_t timeout_ns = kTimeoutNs) {
  const uint64_t t0 = global_timer_ns();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 63u) == 0) {
      if (abort && *abort) return false;
      if (global_timer_ns() - t0 > timeout_ns) {
        if (abort) *abort = 1;
        atomicExch(&g_bsa_device_error, int(BSA_ERR_TIMEOUT));
        return false;
      }
    }
  }
}

// Bounded wait: true when the phase of `parity` completed, false if this CTA
// gave up.  Kept out of line: inlining it into the softmax loop measured slower.
__device__ __noinline__ bool wait_barrier(uint32_t bar, uint32_t parity, volatile int* abort) {
  if (mbar_try_wait(bar, parity)) return true;
  return wait_barrier_slow(bar, parity, abort);
}

// Bounded wait with an inline non-blocking test first: a phase that has
// already completed costs no call.
__device__ __forceinline__ bool wait_fast(uint32_t bar, uint32_t parity, volatile int* abort) {
  if (mbar_test_wait(bar, parity)) return true;
  return wait_barrier(bar, parity, abort);
}

// CRM forward iterator (Appendix E, Algorithm 2) over the OR of up to two CRM
// rows: Init loads the first nonzero word, Next clears the lowest set bit and
// skips empty words, Index is base + count-trailing-zeros or -1 at the end.
struct CrmIter {
  const uint32_t* row0;
  const uint32_t* row1;
  int w, words;
  uint32_t val;
  int base;
  __device__ __forceinline__ void advance() {
    while (val == 0u && w < words) {
      val = __ldg(row0 + w) | (row1 ? __ldg(row1 + w) : 0u);
      ++w;
      base += 32;
    }
  }
  __device__ __forceinline__ void init(const uint32_t* r0, const uint32_t* r1, int n_words) {
    row0 = r0;
    row1 = r1;
    words = n_words;
    w = 0;
    val = 0u;
    base = -32;
    advance();
  }
  __device__ __forceinline__ void next() {
    val &= val - 1u;
    if (val == 0u) advance();
  }
  __device__ __forceinline__ int index() const { return val == 0u ? -1 : base + __ffs(val) - 1; }
};

// Tile of round r for this CTA.  Tiles come in schedule order (most kept
// blocks first); rounds alternate direction (CTA b takes the b-th tile of an
// even round and the b-th from the end of an odd one), so the heavy and light
// ends of consecutive rounds pair up.  On the 720p workload the busiest CTA
// then carries 0.25 % more than the mean, against 0.54 % with a plain stride.
__device__ __forceinline__ int snake_tile(int r) {
  const int G = int(gridDim.x), b = int(blockIdx.x);
  return r * G + ((r & 1) ? G - 1 - b : b);
}

struct TileInfo {
  int bh, qb0;
  const uint32_t* row0;
  const uint32_t* row1;  // second query block's CRM row (two blocks per tile), or null
};

// The tile of round r for this CTA, as the flat row of its first query block;
// false when the CTA has no tile in this round.  One query block per tile:
// schedule position snake_tile(r).  Several: entry r of the CTA's list (the
// tiles in schedule order of their first row, dealt the same way), or, when
// the list does not fit, the tiles in head order.
template <int R>
__device__ __forceinline__ bool round_tile(const FwdParams& p, const int32_t* list, int r,
                                           int& row) {
  if (R > 1 && p.use_list) {
    row = list[r];
    return row >= 0;
  }
  const int tile = snake_tile(r);
  if (tile >= p.num_tiles) return false;
  if (R == 1) {
    row = __ldg(p.schedule + tile);
  } else {
    const int bh = tile / p.tiles_per_head;
    row = bh * p.nb_q + (tile - bh * p.tiles_per_head) * R;
  }
  return true;
}

template <int R>
__device__ __forceinline__ TileInfo tile_info(const FwdParams& p, int row) {
  TileInfo t;
  t.bh = row / p.nb_q;
  t.qb0 = row - t.bh * p.nb_q;
  t.row0 = p.bits + int64_t(row) * p.words;
  t.row1 = (R > 1 && t.qb0 + 1 < p.nb_q) ? t.row0 + p.words : nullptr;
  return t;
}

// Builds this CTA's list of tiles of R query blocks (all threads of the block
// take part): the rows whose query block starts a tile (qb % R == 0) in
// schedule order get ranks k = 0, 1, ...; rank k goes to round k / G, at index
// k % G of an even round and G - 1 - (k % G) of an odd one (as snake_tile).
template <int R>
__device__ void build_tile_list(const FwdParams& p, int32_t* list, int32_t* scan, int n_rounds) {
  const int G = int(gridDim.x), warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  constexpr int kWarps = kThreads / 32;
  for (int r = threadIdx.x; r < n_rounds; r += kThreads) list[r] = -1;
  const int rows = p.BH * p.nb_q;
  int base = 0;
  for (int c0 = 0; c0 < rows; c0 += kThreads * 8) {
    int vals[8];
    int cnt = 0;
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const int i = c0 + int(threadIdx.x) * 8 + e;
      const int row = i < rows ? __ldg(p.schedule + i) : -1;
      const bool first = row >= 0 && (row % p.nb_q) % R == 0;
      vals[e] = first ? row : -1;
      cnt += first ? 1 : 0;
    }
    int incl = cnt;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    __syncthreads();  // the previous chunk's reads of scan[] are done
    if (lane == 31) scan[warp] = incl;
    __syncthreads();
    int wbase = 0, total = 0;
    for (int w = 0; w < kWarps; ++w) {
      const int x = scan[w];
      wbase += w < warp ? x : 0;
      total += x;
    }
    int k = base + wbase + incl - cnt;
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      if (vals[e] < 0) continue;
      const int round = k / G, idx = k - round * G;
      const int owner = (round & 1) ? G - 1 - idx : idx;
      if (owner == int(blockIdx.x) && round < n_rounds) list[round] = vals[e];
      ++k;
    }
    base += total;
  }
}

__device__ __forceinline__ int union_count(const TileInfo& t, int words) {
  int c = 0;
  for (int w = 0; w < words; ++w)
    c += __popc(__ldg(t.row0 + w) | (t.row1 ? __ldg(t.row1 + w) : 0u));
  return c;
}

template <int D, int BQ, int BK>
__global__ void __launch_bounds__(kThreads, 1)
    bsa_forward_kernel(const __grid_constant__ CUtensorMap tm_k,
                       const __grid_constant__ CUtensorMap tm_v, const FwdParams p) {
  using C = Cfg<D, BQ, BK>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // 128-byte swizzle atoms need 1024-byte aligned shared-memory tiles
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  Barriers* bars = reinterpret_cast<Barriers*>(smem + C::kOffBar);
  int32_t* list = reinterpret_cast<int32_t*>(smem + C::kOffList);
  const uint32_t sKV = smem_addr(smem + C::kOffKV);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  volatile int* abort = &bars->abort;
  const int n_rounds = (p.num_tiles + int(gridDim.x) - 1) / int(gridDim.x);
  if constexpr (C::R > 1) {
    if (p.use_list) build_tile_list<C::R>(p, list, list + C::kListInts, n_rounds);
  }

  if (threadIdx.x == 0) {
    mbar_init(smem_addr(&bars->q_full), kTileM);
    for (int i = 0; i < C::kStages; ++i) {
      mbar_init(smem_addr(&bars->kv_full[i]), 1);
      mbar_init(smem_addr(&bars->kv_empty[i]), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(smem_addr(&bars->s_full[i]), 1);
      mbar_init(smem_addr(&bars->p_full[i]), kTileM);
    }
    mbar_init(smem_addr(&bars->o_done[0]), 1);
    mbar_init(smem_addr(&bars->o_done[1]), 1);
    mbar_init(smem_addr(&bars->drain), 1);
    bars->abort = 0;
    fence_barrier_init();
  }
  if (warp == 5) {
    tmem_alloc(smem_addr(&bars->tmem_base), kTmemCols);
    tmem_relinquish();
  }
  if (warp == 4 && lane == 0) {
    prefetch_tensormap(&tm_k);
    prefetch_tensormap(&tm_v);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;

  if (warp == 4) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      uint32_t item = 0;
      bool ok = true;
      for (int r = 0; r < n_rounds && ok; ++r) {
        int tile_row;
        if (!round_tile<C::R>(p, list, r, tile_row)) continue;
        const TileInfo t = tile_info<C::R>(p, tile_row);
        if (union_count(t, p.words) == 0) continue;
        CrmIter it;
        it.init(t.row0, t.row1, p.words);
        for (int j = it.index(); j >= 0;) {
          int j2 = -1;  // second key block of the pair (pairs only)
          if constexpr (C::kPairs) {
            it.next();
            j2 = it.index();
          }
          const int32_t kv_row = t.bh * p.n_pad + j * BK;
          const int32_t kv_row2 = t.bh * p.n_pad + (j2 >= 0 ? j2 : j) * BK;
#pragma unroll
          for (int kv = 0; kv < 2; ++kv) {  // K then V
            const uint32_t slot = item % C::kStages;
            if (item >= C::kStages &&
                !wait_barrier(smem_addr(&bars->kv_empty[slot]), ((item / C::kStages) + 1) & 1,
                              abort)) {
              ok = false;
              break;
            }
            const uint32_t fbar = smem_addr(&bars->kv_full[slot]);
            mbar_arrive_expect_tx(fbar, C::kSlotBytes);
            const uint32_t dst = sKV + slot * C::kSlotBytes;
#pragma unroll
            for (int r = 0; r < C::kRegions; ++r) {
              tma_load_2d(dst + r * C::kKVRegion, kv == 0 ? &tm_k : &tm_v, fbar, r * 64, kv_row);
              if constexpr (C::kPairs)  // rows BK.. of the slot: the pair's second block
                tma_load_2d(dst + r * C::kKVRegion + BK * 128, kv == 0 ? &tm_k : &tm_v, fbar,
                            r * 64, kv_row2);
            }
            ++item;
          }
          if (!ok) break;
          if (!C::kPairs || j2 >= 0) it.next();
          j = it.index();
        }
      }
      if (!ok) {
        // let the copies already issued land before the CTA exits (the wait
        // ignores the abort flag, which is set by now)
        const uint32_t first = item > C::kStages ? item - C::kStages : 0;
        for (uint32_t i = first; i < item; ++i)
          wait_barrier_slow(smem_addr(&bars->kv_full[i % C::kStages]), (i / C::kStages) & 1,
                            nullptr);
      }
    }
  } else if (warp == 5) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      uint32_t item = 0, g = 0, q_iter = 0;
      bool ok = true;
      // S(gi) = Q K^T into S buffer gi & 1 (K already waited for)
      auto mma_s = [&](uint32_t gi, uint32_t k_item) {
        const uint32_t slot = k_item % C::kStages;
        const uint32_t s_tmem = tmem + ((gi & 1) ? kTmemS1 : kTmemS0);
        // A = Q from TMEM (16 elements = 8 columns per step); B = K tile,
        // K-major: 16 elements (32 bytes) per step inside a 128-byte swizzle
        // atom, the next 64-column group C::kKVRegion further
        const uint32_t k_base = sKV + slot * C::kSlotBytes;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint64_t bdesc =
              smem_desc_sw128(k_base + (kk >> 2) * C::kKVRegion + (kk & 3) * 32, 16, 1024);
          mma_ts(s_tmem, tmem + kTmemQ + kk * 8, bdesc, C::kIdescS, kk > 0 ? 1u : 0u);
        }
        mma_commit(smem_addr(&bars->s_full[gi & 1]));
        mma_commit(smem_addr(&bars->kv_empty[slot]));
      };
      // O += P(gi) V (V already waited for)
      auto mma_pv = [&](uint32_t gi, uint32_t v_item, bool first) {
        const uint32_t slot = v_item % C::kStages;
        const uint32_t p_tmem = tmem + ((gi & 1) ? kTmemS1 : kTmemS0);
        // B = V tile, N (= head dim) contiguous: MN-major, 64-column groups
        // C::kKVRegion apart (LBO), 8-key groups 1024 bytes apart (SBO); 16
        // keys (2048 bytes) per step
        const uint32_t v_base = sKV + slot * C::kSlotBytes;
#pragma unroll
        for (int kk = 0; kk < C::kTileN / 16; ++kk) {
          const uint64_t bdesc = smem_desc_sw128(v_base + kk * 16 * 128, C::kKVRegion, 1024);
          mma_ts(tmem + kTmemO, p_tmem + kk * 8, bdesc, C::kIdescPV, (first && kk == 0) ? 0u : 1u);
        }
        mma_commit(smem_addr(&bars->kv_empty[slot]));
        mma_commit(smem_addr(&bars->o_done[gi & 1]));
      };
      auto kv_ready = [&](uint32_t it) {
        return wait_fast(smem_addr(&bars->kv_full[it % C::kStages]), (it / C::kStages) & 1,
                            abort);
      };
      for (int r = 0; r < n_rounds && ok; ++r) {
        int tile_row;
        if (!round_tile<C::R>(p, list, r, tile_row)) continue;
        const TileInfo t = tile_info<C::R>(p, tile_row);
        const int kept = union_count(t, p.words);
        if (kept == 0) continue;
        const int cnt = C::kPairs ? (kept + 1) / 2 : kept;  // S tiles of this query tile
        if (!wait_fast(smem_addr(&bars->q_full), q_iter & 1, abort)) {
          ok = false;
          break;
        }
        ++q_iter;
        // S(0), S(1); then per block n: P V(n) as soon as P(n) is in TMEM and
        // S(n+2) right behind it (it overwrites P(n), which the tensor core
        // reads first: products from one thread run in issue order).  The
        // K and V tiles are waited for before P(n), so only the softmax is
        // on the path from P(n) to the next products.
        const int pre = cnt < 2 ? cnt : 2;
        for (int n = 0; n < pre && ok; ++n) {
          if (!kv_ready(item + 2 * n)) {
            ok = false;
            break;
          }
          tc_fence_after();
          mma_s(g + n, item + 2 * n);
        }
        for (int n = 0; n < cnt && ok; ++n) {
          const uint32_t gi = g + n;
          if (!kv_ready(item + 2 * n + 1) || (n + 2 < cnt && !kv_ready(item + 2 * (n + 2))) ||
              !wait_fast(smem_addr(&bars->p_full[gi & 1]), (gi >> 1) & 1, abort)) {
            ok = false;
            break;
          }
          tc_fence_after();
          mma_pv(gi, item + 2 * n + 1, n == 0);
          if (n + 2 < cnt) mma_s(gi + 2, item + 2 * (n + 2));
        }
        if (!ok) break;
        item += 2 * cnt;
        g += cnt;
      }
      // drain: every MMA issued by this thread completes before TMEM is freed
      // (the wait ignores the abort flag: only the phase or the timeout ends it)
      mma_commit(smem_addr(&bars->drain));
      wait_barrier_slow(smem_addr(&bars->drain), 0, nullptr);
    }
  } else {
    // ------------------------------------------------------------ softmax (warps 0-3)
    const int row = threadIdx.x;  // TMEM lane and query row inside the tile
    const uint32_t lane_base = uint32_t(warp * 32) << 16;
    uint32_t g = 0;
    bool ok = true;
    const bool has_tail = p.n_valid < p.n_pad;
    for (int r = 0; r < n_rounds && ok; ++r) {
      int tile_row;
      if (!round_tile<C::R>(p, list, r, tile_row)) continue;
      const TileInfo t = tile_info<C::R>(p, tile_row);
      const int my_qb = t.qb0 + row / BQ;
      const bool row_in_head = my_qb < p.nb_q;
      const uint32_t* my_bits = p.bits + (int64_t(t.bh) * p.nb_q + my_qb) * p.words;
      const int64_t tok = int64_t(t.qb0) * BQ + row;  // token index inside the head
      float m_run = -INFINITY, l_run = 0.0f;

      if (union_count(t, p.words) > 0) {
        // this row of Q -> TMEM lane `row`, bf16 pairs (low half = even
        // element); every S product of the previous tile has completed (the
        // last one was waited for), so its Q may be overwritten
        uint32_t qr[D / 2];
        if (row_in_head) {
          const uint4* src = reinterpret_cast<const uint4*>(p.q + (int64_t(t.bh) * p.n_pad + tok) * D);
#pragma unroll
          for (int i = 0; i < D / 8; ++i) {
            const uint4 x = __ldg(src + i);
            qr[4 * i] = x.x;
            qr[4 * i + 1] = x.y;
            qr[4 * i + 2] = x.z;
            qr[4 * i + 3] = x.w;
          }
        } else {
#pragma unroll
          for (int i = 0; i < D / 2; ++i) qr[i] = 0u;
        }
        if constexpr (D == 128) tmem_store64(tmem + lane_base + kTmemQ, qr);
        else tmem_store32(tmem + lane_base + kTmemQ, qr);
        tmem_store_wait();
        tc_fence_before();
        mbar_arrive(smem_addr(&bars->q_full));
      }

      CrmIter it;
      it.init(t.row0, t.row1, p.words);
      int n = 0;
      for (int j = it.index(); j >= 0; ++n) {
        int j2 = -1;  // second key block of the pair (pairs only)
        if constexpr (C::kPairs) {
          it.next();
          j2 = it.index();
        }
        const uint32_t gi = g + n, sb = gi & 1;
        // tcgen05.ld/st below are warp-collective: agree on the outcome first
        if (!__all_sync(0xffffffffu, wait_fast(smem_addr(&bars->s_full[sb]), (gi >> 1) & 1,
                                                  abort))) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t s_tmem = tmem + lane_base + (sb ? kTmemS1 : kTmemS0);
        uint32_t sr[C::kTileN];  // raw fp32 scores of this row, one tcgen05.ld
        if constexpr (C::kTileN == 128) tmem_load128(s_tmem, sr);
        else tmem_load64(s_tmem, sr);
        bool member = row_in_head;
        if (C::R > 1 && member) member = (__ldg(my_bits + (j >> 5)) >> (j & 31)) & 1u;
        if constexpr (C::kPairs) {
          if (j2 < 0) {  // a lone block: its copy in the second half does not count
#pragma unroll
            for (int c = BK; c < 2 * BK; ++c) sr[c] = __float_as_uint(-INFINITY);
          }
          // the last key block, in whichever half it sits (static indices keep
          // sr in registers)
          const int valid = p.n_valid - (p.nb_k - 1) * BK;
          if (has_tail && j == p.nb_k - 1) {
#pragma unroll
            for (int c = 0; c < BK; ++c)
              if (c >= valid) sr[c] = __float_as_uint(-INFINITY);
          }
          if (has_tail && j2 == p.nb_k - 1) {
#pragma unroll
            for (int c = 0; c < BK; ++c)
              if (c >= valid) sr[BK + c] = __float_as_uint(-INFINITY);
          }
        } else if (has_tail && j == p.nb_k - 1) {
          const int valid = p.n_valid - j * BK;
#pragma unroll
          for (int c = 0; c < BK; ++c)
            if (c >= valid) sr[c] = __float_as_uint(-INFINITY);
        }
        float mx8[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) mx8[i] = __uint_as_float(sr[i]);
#pragma unroll
        for (int c = 8; c < C::kTileN; ++c) mx8[c & 7] = fmaxf(mx8[c & 7], __uint_as_float(sr[c]));
        const float mx = fmaxf(fmaxf(fmaxf(mx8[0], mx8[1]), fmaxf(mx8[2], mx8[3])),
                               fmaxf(fmaxf(mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7])));
        // Lazy rescale: the reference max only moves when the row max grows by
        // more than kRescaleLog2 (then O and l are scaled by alpha); otherwise
        // p = exp2(s - m_ref) stays below 2^kRescaleLog2.  O / l is the same
        // either way, since O and l always share one reference.
        const float mx_scaled = mx * p.scale_log2;
        bool rescale = false;
        float m_new = m_run;
        if (member) {
          if (m_run == -INFINITY) {
            m_new = mx_scaled;  // first kept block of this row: O and l are still 0
          } else if (mx_scaled > m_run + kRescaleLog2) {
            m_new = mx_scaled;
            rescale = true;
          }
        }
        const float alpha = rescale ? fast_exp2(m_run - m_new) : 1.0f;
        if (__any_sync(0xffffffffu, rescale)) {
          // O holds P(n-1) V(n-1) once that product has completed
          if (!__all_sync(0xffffffffu,
                          wait_barrier(smem_addr(&bars->o_done[(gi - 1) & 1]),
                                       ((gi - 1) >> 1) & 1, abort))) {
            ok = false;
          } else {
            tc_fence_after();
            const uint32_t o_tmem = tmem + lane_base + kTmemO;
#pragma unroll
            for (int c0 = 0; c0 < D; c0 += 32) {
              uint32_t r[32];
              tmem_load32(o_tmem + c0, r);
#pragma unroll
              for (int i = 0; i < 32; ++i) r[i] = __float_as_uint(__uint_as_float(r[i]) * alpha);
              tmem_store32(o_tmem + c0, r);
            }
          }
        }
        if (!ok) break;
        // a row outside this key block's CRM row gets p = 2^-inf = 0, with no
        // branch in the loop below (a predicated loop measured 35 % slower)
        const float neg_m = member ? -m_new : -INFINITY;
        const float sc = p.scale_log2;
        uint32_t pk[C::kTileN / 2];
        // x = s * scale - m and the row sums two columns per instruction
        const float2 sc2 = make_float2(sc, sc), nm2 = make_float2(neg_m, neg_m);
        float2 sum4[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) sum4[i] = make_float2(0.0f, 0.0f);
#pragma unroll
        for (int i = 0; i < C::kTileN / 2; ++i) {
          const float2 x =
              fma2(make_float2(__uint_as_float(sr[2 * i]), __uint_as_float(sr[2 * i + 1])), sc2, nm2);
          const float p0 = fast_exp2(x.x), p1 = fast_exp2(x.y);
          sum4[i & 3] = add2(sum4[i & 3], make_float2(p0, p1));
          __nv_bfloat162 h = __floats2bfloat162_rn(p0, p1);  // low half = even key
          pk[i] = *reinterpret_cast<uint32_t*>(&h);
        }
        // P overwrites the first half of this S buffer: packed bf16 pairs, one
        // 32-bit column per two keys
        if constexpr (C::kTileN == 128) tmem_store64(s_tmem, pk);
        else tmem_store32(s_tmem, pk);
        const float sum = ((sum4[0].x + sum4[1].x) + (sum4[2].x + sum4[3].x)) +
                          ((sum4[0].y + sum4[1].y) + (sum4[2].y + sum4[3].y));
        if (member) {
          l_run = l_run * alpha + sum;
          m_run = m_new;
        }
        tmem_store_wait();
        tc_fence_before();
        mbar_arrive(smem_addr(&bars->p_full[sb]));
        if (!C::kPairs || j2 >= 0) it.next();
        j = it.index();
      }
      if (!ok) break;

      // ---------------------------------------------------------- epilogue
      const bool write_row = row_in_head;
      const bool valid_row = tok < p.n_valid;
      __nv_bfloat16* out_row = p.out + (int64_t(t.bh) * p.n_pad + tok) * D;
      const float inv_l = (l_run > 0.0f) ? 1.0f / l_run : 0.0f;
      if (n > 0) {
        if (!__all_sync(0xffffffffu,
                        wait_barrier(smem_addr(&bars->o_done[(g + n - 1) & 1]),
                                     ((g + n - 1) >> 1) & 1, abort))) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t o_tmem = tmem + lane_base + kTmemO;
#pragma unroll
        for (int c0 = 0; c0 < D; c0 += 32) {
          uint32_t r[32];
          tmem_load32(o_tmem + c0, r);
          if (write_row) {
            uint32_t pk[16];
            const float sc = valid_row ? inv_l : 0.0f;
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              __nv_bfloat162 h = __floats2bfloat162_rn(__uint_as_float(r[2 * i]) * sc,
                                                       __uint_as_float(r[2 * i + 1]) * sc);
              pk[i] = *reinterpret_cast<uint32_t*>(&h);
            }
            uint4* dst = reinterpret_cast<uint4*>(out_row + c0);
#pragma unroll
            for (int i = 0; i < 4; ++i)
              dst[i] = make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
          }
        }
      } else if (write_row) {
        uint4* dst = reinterpret_cast<uint4*>(out_row);
#pragma unroll
        for (int i = 0; i < D / 8; ++i) dst[i] = make_uint4(0u, 0u, 0u, 0u);
      }
      if (write_row) {
        float lse = -INFINITY;
        if (valid_row && l_run > 0.0f) lse = (m_run + fast_log2(l_run)) * 0.69314718055994531f;
        p.lse[int64_t(t.bh) * p.n_pad + tok] = lse;
      }
      g += n;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// Failure-path check: one thread waits on an mbarrier that nothing arrives on,
// through the same bounded wait the forward uses; it gives up after
// timeout_ns, records BSA_ERR_TIMEOUT and returns.
__global__ void wait_timeout_check_kernel(uint64_t timeout_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort;
  if (threadIdx.x == 0) {
    mbar_init(smem_addr(&bar), 1);
    abort = 0;
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) wait_barrier_slow(smem_addr(&bar), 0, &abort, timeout_ns);
}

// ------------------------------------------------------------------ host side
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) !=
            cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return nullptr;
    fn = reinterpret_cast<EncodeTiledFn>(ptr);
  }
  return fn;
}

// [rows, d] bf16 row-major, box = 64 columns x box_rows rows, 128-byte swizzle
bool make_map(CUtensorMap* map, const void* base, int64_t rows, int d, int box_rows) {
  EncodeTiledFn enc = get_encode_fn();
  if (!enc) return false;
  cuuint64_t dims[2] = {cuuint64_t(d), cuuint64_t(rows)};
  cuuint64_t strides[1] = {cuuint64_t(d) * 2};
  cuuint32_t box[2] = {64, cuuint32_t(box_rows)};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims,
                   strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

template <int D, int BQ, int BK>
bsa_status launch_forward(const void* q, const void* k, const void* v, const bsa_mask* m,
                          void* out, float* lse, int BH, int n_valid, int n_pad, float scale,
                          cudaStream_t stream) {
  using C = Cfg<D, BQ, BK>;
  // set on every call: the attribute belongs to the current device, and one
  // process may launch on several
  if (cudaFuncSetAttribute(bsa_forward_kernel<D, BQ, BK>,
                           cudaFuncAttributeMaxDynamicSharedMemorySize,
                           int(C::kSmemBytes)) != cudaSuccess)
    return BSA_ERR_LAUNCH;
  const int64_t rows = int64_t(BH) * n_pad;
  CUtensorMap tk, tv;
  if (!make_map(&tk, k, rows, D, BK) || !make_map(&tv, v, rows, D, BK)) return BSA_ERR_LAUNCH;
  FwdParams p;
  p.q = static_cast<const __nv_bfloat16*>(q);
  p.bits = m->bits;
  p.schedule = m->schedule;
  p.out = static_cast<__nv_bfloat16*>(out);
  p.lse = lse;
  p.BH = BH;
  p.nb_q = n_pad / BQ;
  p.nb_k = n_pad / BK;
  p.words = (p.nb_k + 31) / 32;
  p.n_valid = n_valid;
  p.n_pad = n_pad;
  p.tiles_per_head = (p.nb_q + C::R - 1) / C::R;
  p.num_tiles = C::R == 1 ? BH * p.nb_q : BH * p.tiles_per_head;
  p.scale_log2 = scale * 1.4426950408889634f;
  const int sms = bsa::num_sms();
  if (sms <= 0) return BSA_ERR_LAUNCH;
  const int grid = p.num_tiles < sms ? p.num_tiles : sms;
  p.use_list = (C::R > 1 && (p.num_tiles + grid - 1) / grid <= C::kListInts) ? 1 : 0;
  bsa_forward_kernel<D, BQ, BK><<<grid, kThreads, C::kSmemBytes, stream>>>(tk, tv, p);
  return bsa::launch_status();
}

}  // namespace

extern "C" bsa_status bsa_forward_blocks(const void* q, const void* k, const void* v,
                                         const bsa_mask* mask, void* out, float* lse, int B,
                                         int H, int n_valid, int n_pad, int d, int block_q,
                                         int block_k, float softmax_scale, void* stream) {
  if (!q || !k || !v || !mask || !out || !lse) return BSA_ERR_INVALID_ARG;
  if (!mask->bits || !mask->schedule) return BSA_ERR_INVALID_ARG;
  if (B <= 0 || H <= 0 || n_pad <= 0 || n_valid <= 0 || block_q <= 0 || block_k <= 0 || d <= 0)
    return BSA_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return BSA_ERR_UNSUPPORTED;
  const bool same = block_q == block_k && (block_q == 64 || block_q == 128);
  const bool finer_keys = block_q == 128 && block_k == 64;
  if (!same && !finer_keys) return BSA_ERR_UNSUPPORTED;
  if (n_pad % block_q != 0 || n_pad % block_k != 0) return BSA_ERR_UNSUPPORTED;
  // only the last key block (and the last query block) may hold pad tokens
  if (n_valid > n_pad || n_valid <= n_pad - block_k) return BSA_ERR_INVALID_ARG;
  const int nb_q = n_pad / block_q, nb_k = n_pad / block_k;
  if (mask->B != B || mask->H != H || mask->nb_q != nb_q || mask->nb_k != nb_k ||
      mask->words != (nb_k + 31) / 32)
    return BSA_ERR_INVALID_ARG;
  if (int64_t(B) * H * n_pad >= (int64_t(1) << 31)) return BSA_ERR_OVERFLOW;
  if (!bsa::aligned16(q) || !bsa::aligned16(k) || !bsa::aligned16(v) || !bsa::aligned16(out) ||
      !bsa::aligned16(lse) || !bsa::aligned4(mask->bits) || !bsa::aligned4(mask->schedule))
    return BSA_ERR_MISALIGNED;
  const float scale = softmax_scale > 0.0f ? softmax_scale : 1.0f / sqrtf(float(d));
  const int BH = B * H;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (d == 128) {
    if (finer_keys)
      return launch_forward<128, 128, 64>(q, k, v, mask, out, lse, BH, n_valid, n_pad, scale, s);
    if (block_q == 128)
      return launch_forward<128, 128, 128>(q, k, v, mask, out, lse, BH, n_valid, n_pad, scale, s);
    return launch_forward<128, 64, 64>(q, k, v, mask, out, lse, BH, n_valid, n_pad, scale, s);
  }
  if (finer_keys)
    return launch_forward<64, 128, 64>(q, k, v, mask, out, lse, BH, n_valid, n_pad, scale, s);
  if (block_q == 128)
    return launch_forward<64, 128, 128>(q, k, v, mask, out, lse, BH, n_valid, n_pad, scale, s);
  return launch_forward<64, 64, 64>(q, k, v, mask, out, lse, BH, n_valid, n_pad, scale, s);
}

extern "C" bsa_status bsa_forward(const void* q, const void* k, const void* v,
                                  const bsa_mask* mask, void* out, float* lse, int B, int H,
                                  int n_valid, int n_pad, int d, int block, float softmax_scale,
                                  void* stream) {
  if (block != 64 && block != 128 && block > 0) return BSA_ERR_UNSUPPORTED;
  return bsa_forward_blocks(q, k, v, mask, out, lse, B, H, n_valid, n_pad, d, block, block,
                            softmax_scale, stream);
}

extern "C" bsa_status bsa_check_wait_timeout(unsigned timeout_us, void* stream) {
  if (timeout_us == 0 || timeout_us > 10000000u) return BSA_ERR_INVALID_ARG;
  wait_timeout_check_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(
      uint64_t(timeout_us) * 1000ull);
  return bsa::launch_status();
}

extern "C" bsa_status bsa_get_device_error(bsa_status* device_status) {
  if (!device_status) return BSA_ERR_INVALID_ARG;
  int host = 0, zero = 0;
  if (cudaDeviceSynchronize() != cudaSuccess) return BSA_ERR_LAUNCH;
  if (cudaMemcpyFromSymbol(&host, g_bsa_device_error, sizeof(int)) != cudaSuccess)
    return BSA_ERR_LAUNCH;
  if (cudaMemcpyToSymbol(g_bsa_device_error, &zero, sizeof(int)) != cudaSuccess)
    return BSA_ERR_LAUNCH;
  const int pred = bsa::take_predict_device_error();
  if (pred < 0) return BSA_ERR_LAUNCH;
  if (host == 0) host = pred;
  *device_status = host == 0 ? BSA_OK : bsa_status(host);
  return BSA_OK;
}

extern "C" int bsa_version(void) { return 100; }

extern "C" const char* bsa_status_string(bsa_status s) {
  switch (s) {
    case BSA_OK: return "BSA_OK";
    case BSA_ERR_INVALID_ARG: return "BSA_ERR_INVALID_ARG";
    case BSA_ERR_UNSUPPORTED: return "BSA_ERR_UNSUPPORTED";
    case BSA_ERR_MISALIGNED: return "BSA_ERR_MISALIGNED";
    case BSA_ERR_OVERFLOW: return "BSA_ERR_OVERFLOW";
    case BSA_ERR_LAUNCH: return "BSA_ERR_LAUNCH";
    case BSA_ERR_TIMEOUT: return "BSA_ERR_TIMEOUT";
    case BSA_ERR_WORKSPACE: return "BSA_ERR_WORKSPACE";
  }
  return "BSA_ERR_UNKNOWN";
}
