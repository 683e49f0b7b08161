/*
 * bsa.h -- C ABI of libbsa: bitmask-driven block-sparse attention forward for
 * B200 (sm_100a).
 *
 * The operations follow "ScalingAttention: Discovering Intrinsic Sparse
 * Attention Topology for Video Diffusion Transformers":
 *   - Sec. 4.3.2 (CRM Kernel): a per-head block mask is encoded as one bitmask
 *     row per query block (CRM), stored as aligned uint32 words, one bit per
 *     key block; the kernel walks the active key blocks of a row with bit scan
 *     and bit clear and runs the FlashAttention loop over them only.
 *   - Appendix E (Algorithm 2): the CRM forward iterator (Init / Advance /
 *     Next / Index).  Bit j of word w is key block 32*w + j.
 *   - Sec. 5.4-5.5: token permutation that clusters tokens into hardware-
 *     friendly blocks; here frame-major T x H x W tokens are gathered into
 *     contiguous 3-D tiles so that one attention block is one tile.
 *
 * Conventions shared by every call:
 *   - All data pointers are DEVICE pointers owned by the caller; the library
 *     allocates no device memory and frees nothing it did not create.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream).  Every call is asynchronous on that stream; none synchronises.
 *   - Arguments are checked on the host before any launch; a failed check
 *     returns an error status and launches nothing.  No call throws, exits or
 *     traps.  A launch failure returns BSA_ERR_LAUNCH.
 *   - bf16 tensors are raw IEEE bfloat16 (2 bytes), row-major, with the shape
 *     given beside each argument; the innermost index is contiguous.
 *   - A data pointer must be 16-byte aligned unless the call's description
 *     below asks for less (4-byte for the mask-packing and threshold-map
 *     calls), else BSA_ERR_MISALIGNED.
 */
#ifndef BSA_H_
#define BSA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  BSA_OK = 0,
  BSA_ERR_INVALID_ARG = 1, /* null pointer, non-positive size, inconsistent sizes */
  BSA_ERR_UNSUPPORTED = 2, /* valid but not implemented (e.g. head dim 96) */
  BSA_ERR_MISALIGNED = 3,  /* a data pointer is not 16-byte aligned */
  BSA_ERR_OVERFLOW = 4,    /* an index or offset would not fit in int32 */
  BSA_ERR_LAUNCH = 5,      /* the CUDA launch (or device query) failed */
  BSA_ERR_TIMEOUT = 6,     /* a kernel gave up waiting on a pipeline barrier */
  BSA_ERR_WORKSPACE = 7    /* workspace missing or smaller than required */
} bsa_status;

/* Device pointers produced by bsa_pack_mask and read by bsa_forward.  The
 * struct itself lives in host memory. */
typedef struct {
  const uint32_t* bits;        /* [B, H, nb_q, words] CRM rows, words = (nb_k + 31) / 32 */
  const int32_t* counts;       /* [B, H, nb_q] kept key blocks per query block */
  const int32_t* row_offsets;  /* [B*H*nb_q + 1] exclusive prefix of counts */
  const int32_t* col_idx;      /* [row_offsets[B*H*nb_q]] ascending kept key blocks per row */
  const int32_t* schedule;     /* [B*H*nb_q] flat row ids in work order (see bsa_pack_mask) */
  int B, H, nb_q, nb_k, words;
} bsa_mask;

/* Library version, major * 10000 + minor * 100 + patch. */
int bsa_version(void);

/* Human-readable name of a status code (static string, never NULL). */
const char* bsa_status_string(bsa_status status);

/* ---------------------------------------------------------------------------
 * bsa_pack_mask -- dense per-head block mask -> CRM rows + lists + schedule.
 *
 * Follows Sec. 4.3.2 (CRM representation: aligned uint32 rows, one bit per key
 * block) with the bit order of Appendix E, Algorithm 2 (bit j of word w is key
 * block 32*w + j; unused high bits of the last word are 0).
 *
 *   dense       [B, H, nb_q, nb_k] uint8; any nonzero byte marks a kept block.
 *   bits        out [B, H, nb_q, words] uint32, words = (nb_k + 31) / 32.
 *   counts      out [B*H*nb_q] int32, popcount of each row.
 *   row_offsets out [B*H*nb_q + 1] int32, exclusive prefix sum of counts over
 *               rows in (b, h, i) order; the last entry is the total.
 *   col_idx     out, room for B*H*nb_q*nb_k int32 (the worst case); row r's
 *               kept key blocks in ascending order at [row_offsets[r],
 *               row_offsets[r+1]).  May be NULL to skip the lists.
 *   schedule    out [B*H*nb_q] int32 flat row ids r = (b*H + h)*nb_q + i,
 *               ordered by counts descending; equal counts keep ascending r.
 *               Then the order is checked for how many heads it mixes: over
 *               its full windows of 148 consecutive entries (one wave of a
 *               B200), the distinct heads h' = r / nb_q (one per (b, h)) are
 *               counted; if that many heads' K and V (nb_k key blocks each,
 *               costed as 128 tokens at d = 128 in bf16: 64 KiB) exceed the
 *               device's L2 size on average, the schedule is instead ordered
 *               by head h' ascending, then counts descending, then r
 *               ascending.  (Query tiles taken together then share one head's
 *               K and V in L2; the check is skipped, keeping the count
 *               order, when B*H > 8192 or nb_q > 8192.)  Any order gives the
 *               same attention output; the forward only takes it as its work
 *               order.
 *   workspace   device scratch of at least bsa_pack_mask_workspace(...) bytes,
 *               16-byte aligned; its contents on entry do not matter.
 *
 * Alignment: dense needs no alignment; every other pointer must be 4-byte
 * aligned (16-byte for workspace).  Errors: BSA_ERR_INVALID_ARG (null output,
 * a size <= 0), BSA_ERR_OVERFLOW (B*H*nb_q*nb_k >= 2^31), BSA_ERR_UNSUPPORTED
 * (nb_k > 49151), BSA_ERR_WORKSPACE, BSA_ERR_LAUNCH.
 * ------------------------------------------------------------------------- */
size_t bsa_pack_mask_workspace(int B, int H, int nb_q, int nb_k);
bsa_status bsa_pack_mask(const uint8_t* dense, int B, int H, int nb_q, int nb_k, uint32_t* bits,
                         int32_t* counts, int32_t* row_offsets, int32_t* col_idx,
                         int32_t* schedule, void* workspace, size_t workspace_bytes,
                         void* stream);

/* ---------------------------------------------------------------------------
 * bsa_pack_mask_noalloc -- bsa_pack_mask without a caller-supplied workspace.
 *
 * The paper has no counterpart: this variant exists for callers that cannot
 * allocate device memory -- for example a plug-in host that hands a library
 * only its input and output buffers, or a runtime that reserves all device
 * memory up front and forbids later allocations (there cudaMalloc fails or
 * stalls the device).  It computes exactly what bsa_pack_mask computes, with
 * the same arguments minus the workspace, and allocates nothing: the sort's
 * scratch is a fixed 512 KiB array inside the library, present on every GPU
 * that loads it until the process exits.
 *
 * Limit: the built-in scratch holds 131072 ints and the call needs
 * (nb_k + 2) * ceil(B*H*nb_q / 1024) + 1 of them (e.g. every workload with up to
 * 40 heads of 1024 query blocks of 1024 key blocks, B = 1, fits); a larger
 * call returns BSA_ERR_WORKSPACE (use bsa_pack_mask).  The first call on each device
 * looks up the array's device address (cudaGetSymbolAddress) with that device
 * current, so make that first call before any stream capture; the address is
 * kept for the life of the process, so a device reset (cudaDeviceReset) or a
 * driver context other than the device's primary one is not supported.  All
 * calls share the one array, which keeps the last call's contents: calls whose
 * kernels overlap on a GPU (for example on two streams at once) race and give
 * wrong results; calls in order on one stream are safe, since each call writes
 * every scratch entry it reads before reading it.  Other errors as for
 * bsa_pack_mask; BSA_ERR_LAUNCH also if the address lookup fails.
 * ------------------------------------------------------------------------- */
bsa_status bsa_pack_mask_noalloc(const uint8_t* dense, int B, int H, int nb_q, int nb_k,
                                 uint32_t* bits, int32_t* counts, int32_t* row_offsets,
                                 int32_t* col_idx, int32_t* schedule, void* stream);

/* ---------------------------------------------------------------------------
 * bsa_pack_mask_from_threshold -- threshold map + per-head density threshold
 * -> CRM rows + lists + schedule, with no dense mask in between.
 *
 * Follows Sec. 4.1.2 (Eq. 2): the Threshold Map T records, per block (u, v),
 * the smallest sparsity threshold at which the block is active, and a mask for
 * a target threshold p is M_p = 1(T <= p).  Algorithm 1 (FAST, mask
 * instantiation) picks one p per layer, timestep and head, so p holds one
 * value per head and the map is shared by all batch items.  The result is
 * exactly bsa_pack_mask applied to the dense mask
 *     dense[b, h, u, v] = (thr[h, u, v] <= p[h]) ? 1 : 0
 * (fp32 comparison; a NaN threshold or a NaN p keeps nothing).
 *
 *   thr   [H, nb_q, nb_k] fp32 device array, 4-byte aligned.
 *   p     [H] fp32 device array, 4-byte aligned.
 *   bits, counts, row_offsets, col_idx, schedule, workspace: as for
 *         bsa_pack_mask (same shapes, same workspace size from
 *         bsa_pack_mask_workspace(B, H, nb_q, nb_k)).
 *
 * Errors: BSA_ERR_INVALID_ARG (null pointer, a size <= 0), BSA_ERR_MISALIGNED,
 * BSA_ERR_OVERFLOW (B*H*nb_q*nb_k >= 2^31), BSA_ERR_WORKSPACE, BSA_ERR_LAUNCH.
 * ------------------------------------------------------------------------- */
bsa_status bsa_pack_mask_from_threshold(const float* thr, const float* p, int B, int H, int nb_q,
                                        int nb_k, uint32_t* bits, int32_t* counts,
                                        int32_t* row_offsets, int32_t* col_idx,
                                        int32_t* schedule, void* workspace,
                                        size_t workspace_bytes, void* stream);

/* ---------------------------------------------------------------------------
 * bsa_threshold_resize -- resize a threshold map to another block grid
 * (Sec. 4.3.1, Eq. 7: the map of a base resolution is resized by conservative
 * bilinear interpolation with a ceiling rule, so that any overlap with an
 * active region is preserved; the topology is built once and reused at every
 * resolution).
 *
 * Target block (u, v) samples the source map at (u * sq / tq, v * sk / tk).
 * Along each axis the source blocks with a nonzero bilinear weight are
 * floor(u * sq / tq) and, when u * sq is not a multiple of tq, the next block
 * (clamped to sq - 1); likewise for v.  The ceiling of the bilinearly
 * resampled indicator 1(T <= p) is 1 exactly when one of those blocks is
 * active, for every p; so the target threshold is their minimum:
 *     dst[h, u, v] = min over those (a, c) of src[h, a, c]
 * NaN entries are skipped; if all are NaN the result is NaN; when +0 and -0
 * tie, the sign of the zero returned is unspecified (no mask can tell them
 * apart).  Exact (no arithmetic on the thresholds), so pack(resize(T), p)
 * equals the ceiling rule applied to pack(T, p) at every p.
 *
 *   src [H, sq, sk] fp32 device array, dst [H, tq, tk] fp32 device array;
 *   both 4-byte aligned, not overlapping.  Sizes 1 .. 65535 per axis (up- or
 *   downscale).
 *
 * Errors: BSA_ERR_INVALID_ARG (null pointer, a size <= 0), BSA_ERR_UNSUPPORTED
 * (a size above 65535), BSA_ERR_MISALIGNED, BSA_ERR_OVERFLOW (H*tq >= 2^31),
 * BSA_ERR_LAUNCH.
 * ------------------------------------------------------------------------- */
bsa_status bsa_threshold_resize(const float* src, int H, int sq, int sk, float* dst, int tq,
                                int tk, void* stream);

/* ---------------------------------------------------------------------------
 * bsa_tile_permute / bsa_tile_unpermute -- 3-D tile gather (Sec. 5.4-5.5,
 * token permutation into hardware-friendly blocks).
 *
 * Tokens of one (b, h) are frame-major: token (t, y, x) is at index
 * (t*Hs + y)*Ws + x, N = T*Hs*Ws.  The tile-major order enumerates tiles
 * (tile_t, tile_y, tile_x) row-major over a grid of tt x th x tw tiles; edge
 * tiles are clipped to the grid (ragged) and their tokens concatenated with no
 * holes; inside a tile tokens go (t, y, x) row-major.  Positions N..n_pad-1 are
 * padding.
 *
 *   bsa_tile_permute:   in  [B, H, N, d] bf16 frame-major
 *                       out [B, H, n_pad, d] bf16 tile-major, pad rows = 0.
 *   bsa_tile_unpermute: in  [B, H, n_pad, d] bf16 tile-major
 *                       out [B, H, N, d] bf16 frame-major (pad rows dropped).
 *
 * d must be a multiple of 8 (16-byte rows); n_pad >= N; in and out must not
 * overlap.  Errors: BSA_ERR_INVALID_ARG, BSA_ERR_MISALIGNED, BSA_ERR_OVERFLOW
 * (B*H*n_pad*d >= 2^40), BSA_ERR_LAUNCH.  Results are bit-exact copies.
 * ------------------------------------------------------------------------- */
bsa_status bsa_tile_permute(const void* in, void* out, int B, int H, int T, int Hs, int Ws, int d,
                            int tt, int th, int tw, int n_pad, void* stream);
bsa_status bsa_tile_unpermute(const void* in, void* out, int B, int H, int T, int Hs, int Ws,
                              int d, int tt, int th, int tw, int n_pad, void* stream);

/* ---------------------------------------------------------------------------
 * bsa_predict_top_p -- online top-p block mask from the (permuted) q and k,
 * straight to the CRM rows, lists and schedule that bsa_forward reads.
 *
 * The cut follows Algorithm 1 (sort the block scores, accumulate, cut where
 * the cumulative share reaches p: Top-k(S, p) of Eq. 2), applied per query
 * block with one top-p threshold per head, on the proxy scores of pooled
 * queries and keys:
 *   qbar_i = mean of the valid tokens of block i (kbar_j alike)
 *   s_ij = qbar_i . kbar_j / (sqrt(d) * tau[h]),  p_ij = softmax_j(s_ij)
 * Row i keeps the blocks in descending p (ties: lower j first) up to and
 * including the one where the cumulative sum reaches top_p[h]; at least one
 * block, all of them if the sum never reaches it.  Arithmetic: fp32 means;
 * scores on the tensor cores as three tf32 products per step (each mean split
 * into a tf32 part and its remainder: fp32-level accuracy), fp32 accumulation;
 * expf; the cumulative comparison is in fp32, so a block whose inclusion
 * changes the sum by less than fp32 rounding can go either way.
 *
 *   q, k      [B, H, n_pad, d] bf16 in block order (as given to bsa_forward).
 *   tau, top_p  [H] fp32 device arrays.
 *   bits, counts, row_offsets, col_idx, schedule: as for bsa_pack_mask with
 *             nb_q = nb_k = n_pad / block.
 *   workspace device scratch of bsa_predict_top_p_workspace(...) bytes,
 *             16-byte aligned (pooled means, the fp32 block scores
 *             [B*H, nb, nb] and the sort's tables).
 *
 * Supported: d in {64, 128}; n_pad % block == 0; n_pad - block < n_valid <=
 * n_pad; n_pad / block <= 2048; B*H <= 65535.  Errors: BSA_ERR_INVALID_ARG,
 * BSA_ERR_UNSUPPORTED, BSA_ERR_OVERFLOW, BSA_ERR_MISALIGNED (q, k,
 * workspace 16-byte; others 4-byte), BSA_ERR_WORKSPACE, BSA_ERR_LAUNCH.
 * ------------------------------------------------------------------------- */
size_t bsa_predict_top_p_workspace(int B, int H, int n_pad, int d, int block);
bsa_status bsa_predict_top_p(const void* q, const void* k, int B, int H, int n_valid, int n_pad,
                             int d, int block, const float* tau, const float* top_p,
                             uint32_t* bits, int32_t* counts, int32_t* row_offsets,
                             int32_t* col_idx, int32_t* schedule, void* workspace,
                             size_t workspace_bytes, void* stream);

/* ---------------------------------------------------------------------------
 * Token orders as tables, and the gather that applies them.
 *
 * Token permutation eases the 128 x 128 granularity bottleneck by clustering
 * related tokens into the same block (Sec. 5.4-5.5).  Besides the 3-D tile
 * order above, the pages name DFSAttn's Hilbert curve-based token reordering
 * and Veda's head-aware tiling (heads with differently shaped tiles).  An
 * order is fixed per grid shape, so it is built once on the HOST as a table
 * (these three calls take and fill host arrays, run on the calling thread and
 * touch no GPU); each step then applies it on the GPU with bsa_gather_rows.
 * An order lists, for each position p of the new order, the frame-major index
 * (t*Hs + y)*Ws + x of the token placed there.
 *
 * bsa_hilbert_order: order[N] (host) of the 3-D Hilbert curve over the cube of
 *   side 2^bits >= max(T, Hs, Ws), axes (t, y, x), points outside the grid
 *   skipped; the Hilbert index follows J. Skilling, "Programming the Hilbert
 *   curve" (2004).  Errors: BSA_ERR_INVALID_ARG (null, a size <= 0,
 *   N >= 2^31), BSA_ERR_UNSUPPORTED (a side above 2^21).
 * bsa_tile_order: order[N] (host) of bsa_tile_permute's tile order for one
 *   tile shape; with one shape per head it gives head-aware tilings.
 *   Errors: BSA_ERR_INVALID_ARG.
 * bsa_order_tables: from order[n] (host) build the gather tables (host)
 *   fwd[n_pad] (fwd[p] = order[p] for p < n, -1 for the zero tail) and
 *   inv[n] (inv[order[p]] = p).  BSA_ERR_INVALID_ARG if order is not a
 *   permutation of 0..n-1 or n_pad < n.
 * ------------------------------------------------------------------------- */
bsa_status bsa_hilbert_order(int T, int Hs, int Ws, int32_t* order);
bsa_status bsa_tile_order(int T, int Hs, int Ws, int tt, int th, int tw, int32_t* order);
bsa_status bsa_order_tables(const int32_t* order, int n, int n_pad, int32_t* fwd, int32_t* inv);

/* ---------------------------------------------------------------------------
 * bsa_gather_rows -- out[b, h, i, :] = in[b, h, src[i], :] on the GPU; a src
 * entry outside [0, n_in) writes a zero row (the tail pad).
 *
 *   in   [B, H, n_in, d] bf16 (any 2-byte rows, moved bit-exactly).
 *   out  [B, H, n_out, d], must not overlap in.
 *   src  device int32: [n_out] shared by every head (per_head = 0), or
 *        [H, n_out], table h for head h of every batch item (per_head = 1).
 * With fwd from bsa_order_tables (n_out = n_pad) this permutes; with inv
 * (n_in = n_pad, n_out = n) it restores frame-major order.  d % 8 == 0;
 * in/out 16-byte aligned, src 4-byte aligned.  Errors: BSA_ERR_INVALID_ARG,
 * BSA_ERR_UNSUPPORTED (d % 8 != 0), BSA_ERR_OVERFLOW (B*H*max(n_in,
 * n_out)*d >= 2^40, or per_head with H > 65535), BSA_ERR_MISALIGNED,
 * BSA_ERR_LAUNCH.  Bit-exact copies.
 * ------------------------------------------------------------------------- */
bsa_status bsa_gather_rows(const void* in, void* out, int B, int H, int n_in, int n_out, int d,
                           const int32_t* src, int per_head, void* stream);

/* ---------------------------------------------------------------------------
 * bsa_forward -- block-sparse attention forward (Sec. 4.3.2: the FlashAttention
 * forward whose key-block loop is replaced by the CRM iterator of Appendix E,
 * Algorithm 2; dense tensor-core work inside each kept tile).
 *
 * For each (b, h) and each valid query i < n_valid, with J the kept key blocks
 * of query block i / block and keys j < n_valid:
 *     s_j = scale * q_i . k_j   (j in a kept block; -inf otherwise)
 *     out_i = sum_j softmax(s)_j v_j,   lse_i = max_j s_j + ln sum_j exp(s_j - max)
 * Arithmetic: bf16 operands, fp32 accumulation and softmax, P rounded to bf16
 * for the P.V product.  Query rows with no kept valid key, and pad rows
 * i >= n_valid, get out = 0 and lse = -inf.
 *
 *   q, k, v  [B, H, n_pad, d] bf16 in tile-major order (see bsa_tile_permute).
 *   mask     host pointer to a bsa_mask from bsa_pack_mask with the same B, H
 *            and nb_q = nb_k = n_pad / block (bits and schedule are read).
 *   out      [B, H, n_pad, d] bf16.
 *   lse      [B, H, n_pad] fp32 (natural log, in units of the scaled logits).
 *   softmax_scale <= 0 selects 1/sqrt(d).
 *
 * Supported: d in {64, 128}; block in {64, 128}; n_pad % block == 0;
 * n_pad - block < n_valid <= n_pad.  Anything else: BSA_ERR_UNSUPPORTED or
 * BSA_ERR_INVALID_ARG.  q, k, v, out and lse must be 16-byte aligned.
 * A kernel that waits on a pipeline barrier for more than about two seconds
 * gives up, records BSA_ERR_TIMEOUT for bsa_get_device_error and returns.
 * ------------------------------------------------------------------------- */
bsa_status bsa_forward(const void* q, const void* k, const void* v, const bsa_mask* mask,
                       void* out, float* lse, int B, int H, int n_valid, int n_pad, int d,
                       int block, float softmax_scale, void* stream);

/* ---------------------------------------------------------------------------
 * bsa_forward_blocks -- bsa_forward with query blocks of block_q tokens and
 * key blocks of block_k tokens: query i and key j fall in blocks i / block_q
 * and j / block_k, and the mask (from bsa_pack_mask on a dense
 * [B, H, n_pad / block_q, n_pad / block_k] mask) has nb_q = n_pad / block_q
 * rows of nb_k = n_pad / block_k bits.  block_q = 128 with block_k = 64 halves
 * the key granularity: the 128 x 128 block is the granularity bottleneck the
 * pages name below 40 % density (Sec. 5.4), and finer key blocks keep fewer
 * unneeded keys per kept block.
 *
 * Supported (block_q, block_k): (128, 128), (64, 64), (128, 64); n_pad a
 * multiple of both; n_pad - block_k < n_valid <= n_pad.  bsa_forward(...,
 * block, ...) is bsa_forward_blocks(..., block, block, ...).  Arguments,
 * outputs and errors otherwise as for bsa_forward.
 * ------------------------------------------------------------------------- */
bsa_status bsa_forward_blocks(const void* q, const void* k, const void* v, const bsa_mask* mask,
                              void* out, float* lse, int B, int H, int n_valid, int n_pad, int d,
                              int block_q, int block_k, float softmax_scale, void* stream);

/* ---------------------------------------------------------------------------
 * bsa_attention_host -- the whole path from HOST buffers to HOST buffers:
 * bsa_pack_mask, bsa_tile_permute of q, k, v, bsa_forward and
 * bsa_tile_unpermute, with the host <-> device copies overlapped with the
 * kernels.
 *
 * Heads are independent (each has its own mask, token order and softmax), so
 * the B*H heads run in chunks of at most heads_per_chunk (<= 0: ceil(B*H / 16))
 * as a three-stage pipeline: chunk c + 1 is copied in and chunk c - 1 copied
 * out while chunk c computes on `stream`.  When heads_per_chunk > 1 and
 * B*H > 2, the first and the last chunk hold one head each, so the pipeline
 * fills and drains in one head's time.  Two auxiliary streams per device (made
 * on first use) carry the copies; they start after the work already queued on
 * `stream` and are joined back into it, so the call is ordered on `stream`
 * like any other.  Calls on one device from several host threads at once
 * share those streams and run one after the other.
 *
 *   q, k, v  HOST [B, H, N, d] bf16, frame-major (N = T*Hs*Ws).  Pinned
 *            (page-locked) memory lets the copies overlap; pageable memory
 *            works but copies synchronously.
 *   mask     HOST [B, H, nb, nb] uint8, nb = n_pad / block,
 *            n_pad = ceil(N / block) * block.
 *   out      HOST [B, H, N, d] bf16, frame-major (as bsa_tile_unpermute).
 *   lse      HOST [B, H, n_pad] fp32 in tile-major order (as bsa_forward).
 *   tt, th, tw, block, softmax_scale: as for bsa_tile_permute / bsa_forward.
 *   workspace  DEVICE scratch of bsa_attention_host_workspace(...) bytes,
 *            256-byte aligned (two chunks' buffers).
 *
 * The host buffers must stay valid until the work on `stream` completes.
 * Errors: BSA_ERR_INVALID_ARG, BSA_ERR_OVERFLOW, BSA_ERR_WORKSPACE,
 * BSA_ERR_MISALIGNED, BSA_ERR_LAUNCH, and any error of the calls above (for
 * example BSA_ERR_UNSUPPORTED for d = 96).  After an error part of the
 * pipeline may already be queued.
 * ------------------------------------------------------------------------- */
size_t bsa_attention_host_workspace(int B, int H, int T, int Hs, int Ws, int d, int block,
                                    int heads_per_chunk);
bsa_status bsa_attention_host(const void* q, const void* k, const void* v, const uint8_t* mask,
                              void* out, float* lse, int B, int H, int T, int Hs, int Ws, int d,
                              int tt, int th, int tw, int block, float softmax_scale,
                              int heads_per_chunk, void* workspace, size_t workspace_bytes,
                              void* stream);

/* Failure-path check (no counterpart in the paper): launches one thread that
 * waits on a pipeline barrier nothing will complete, through the same bounded
 * wait the forward kernel uses, so that the wait runs out after timeout_us
 * microseconds (1 .. 10^7) and records BSA_ERR_TIMEOUT for
 * bsa_get_device_error.  Nothing faults, traps or hangs: the kernel returns
 * and the context stays usable.  Errors: BSA_ERR_INVALID_ARG, BSA_ERR_LAUNCH. */
bsa_status bsa_check_wait_timeout(unsigned timeout_us, void* stream);

/* Reads and clears the device-side error word of the current device (set by a
 * kernel that timed out on a barrier).  Synchronises the current device.
 * Returns BSA_OK or BSA_ERR_TIMEOUT in *device_status; the return value is
 * BSA_ERR_LAUNCH if the read itself failed. */
bsa_status bsa_get_device_error(bsa_status* device_status);

#ifdef __cplusplus
}
#endif

#endif /* BSA_H_ */
