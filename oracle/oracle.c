/*
 * oracle.c -- plain fp64 CPU oracle for bitmask-driven block-sparse attention.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may call, link or
 * load this file: only tests/, the smoke check and the bench's CPU-baseline
 * leg use it.  It shares no code, header or constant with the CUDA library.
 *
 * What it computes, and where the pages define it:
 *
 *  - CRM (Compressed Row Mask): one bitmask row per query block, stored as
 *    uint32 words, one bit per key block ("ScalingAttention", Sec. 4.3.2).
 *    The bit order follows the forward iterator of Appendix E (Algorithm 2):
 *    the iterator's base starts at -32 and grows by 32 per word loaded, and
 *    the block index is base + count-trailing-zeros, so bit j of word w is
 *    key block 32*w + j.
 *  - The CRM forward iterator itself (Init / Advance / Next / Index,
 *    Appendix E, Algorithm 2), used here to list the kept key blocks of a row.
 *  - Masked softmax attention: the block-sparse FlashAttention forward of
 *    Sec. 4.3.2 computes, for every query, softmax over the keys of the kept
 *    blocks only; a masked block contributes exp(-inf) = 0.  We write out the
 *    plain definition: s = scale * q.k, -inf where the block is masked,
 *    m = max s, l = sum exp(s - m), o = sum exp(s - m) v / l, lse = m + ln l.
 *  - The 3-D tile permutation (token reordering, Sec. 5.4-5.5): tiles are
 *    enumerated (tile_t, tile_y, tile_x) row-major; inside a tile the tokens
 *    go (t, y, x) row-major over the tile's clipped extent; tokens are
 *    concatenated with no holes and the tail is zero-padded.
 *
 * Everything is fp64 except the inputs, which arrive as raw bf16 bits and are
 * widened exactly to double.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* ------------------------------------------------------------------ */
/* bf16 -> double, exact                                               */
/* ------------------------------------------------------------------ */
static double bf16_bits_to_double(uint16_t b) {
  uint32_t u = ((uint32_t)b) << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return (double)f;
}

int oracle_num_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

/* ------------------------------------------------------------------ */
/* CRM words per row: one uint32 holds the state of 32 key blocks      */
/* (ScalingAttention Sec. 4.3.2).                                      */
/* ------------------------------------------------------------------ */
int oracle_crm_words(int nb_k) { return (nb_k + 31) / 32; }

/* Dense 0/1 block mask rows -> CRM bit rows.  A nonzero byte is a kept
 * block.  rows = B*H*nb_q; dense is [rows, nb_k]; bits is [rows, words]. */
void oracle_pack_bits(const uint8_t* dense, int64_t rows, int nb_k, uint32_t* bits) {
  int words = oracle_crm_words(nb_k);
  for (int64_t r = 0; r < rows; ++r) {
    uint32_t* row_bits = bits + r * words;
    for (int w = 0; w < words; ++w) row_bits[w] = 0u;
    for (int j = 0; j < nb_k; ++j) {
      if (dense[r * (int64_t)nb_k + j] != 0) {
        row_bits[j / 32] |= (1u << (j % 32));
      }
    }
  }
}

/* ------------------------------------------------------------------ */
/* CRM forward iterator, ScalingAttention Appendix E (Algorithm 2).    */
/* State {ptr, end, val, base}.                                        */
/* ------------------------------------------------------------------ */
typedef struct {
  const uint32_t* ptr;
  const uint32_t* end;
  uint32_t val;
  int64_t base;
} crm_iterator;

/* Skip empty segments: load words until one is nonzero or the row ends. */
static void crm_advance(crm_iterator* s) {
  while (s->val == 0u && s->ptr != s->end) {
    s->val = *s->ptr;
    s->ptr += 1;
    s->base += 32;
  }
}

static void crm_init(crm_iterator* s, const uint32_t* row_ptr, int n_words) {
  s->ptr = row_ptr;
  s->end = row_ptr + n_words;
  s->val = 0u;
  s->base = -32;
  crm_advance(s); /* prefetch the first nonzero segment */
}

/* Consume the current active block: clear the lowest set bit. */
static void crm_next(crm_iterator* s) {
  s->val = s->val & (s->val - 1u);
  if (s->val == 0u) crm_advance(s);
}

static int count_trailing_zeros(uint32_t v) {
  int n = 0;
  while ((v & 1u) == 0u) {
    v >>= 1;
    n += 1;
  }
  return n;
}

/* Global key-block index of the current active block, -1 for the end-of-row
 * sentinel. */
static int64_t crm_index(const crm_iterator* s) {
  if (s->val == 0u) return -1;
  return s->base + count_trailing_zeros(s->val);
}

/* Walk every CRM row with the iterator: counts[r] = number of kept blocks,
 * row_offsets = exclusive prefix of counts (rows+1 entries), col_idx = the
 * kept block indices of each row in the order the iterator yields them.
 * col_idx may be NULL to only count.  Returns the total. */
int64_t oracle_crm_lists(const uint32_t* bits, int64_t rows, int n_words, int32_t* counts,
                         int64_t* row_offsets, int32_t* col_idx) {
  int64_t total = 0;
  for (int64_t r = 0; r < rows; ++r) {
    crm_iterator it;
    crm_init(&it, bits + r * n_words, n_words);
    int64_t c = 0;
    row_offsets[r] = total;
    for (int64_t j = crm_index(&it); j != -1; crm_next(&it), j = crm_index(&it)) {
      if (col_idx) col_idx[total + c] = (int32_t)j;
      c += 1;
    }
    counts[r] = (int32_t)c;
    total += c;
  }
  row_offsets[rows] = total;
  return total;
}

/* Schedule: row ids ordered by kept-block count, largest first; rows with
 * equal counts keep ascending row order (a stable sort).  Written as the
 * plainest counting order: for each count value from the largest down, list
 * its rows.  The pages are silent on the work order; this is the order the
 * load-balancing rule "most kept blocks first" names.  Any other work order
 * gives the same attention output. */
void oracle_schedule(const int32_t* counts, int64_t rows, int32_t* schedule) {
  int32_t max_count = 0;
  for (int64_t r = 0; r < rows; ++r)
    if (counts[r] > max_count) max_count = counts[r];
  int64_t pos = 0;
  for (int32_t c = max_count; c >= 0; --c)
    for (int64_t r = 0; r < rows; ++r)
      if (counts[r] == c) schedule[pos++] = (int32_t)r;
}

/* ------------------------------------------------------------------ */
/* 3-D tile permutation.  perm[p] = frame-major token index (t*H + y)*W */
/* + x of the token stored at tile-major position p, p < T*H*W.        */
/* ------------------------------------------------------------------ */
static int min_int(int a, int b) { return a < b ? a : b; }

void oracle_tile_order(int T, int Hs, int Ws, int tt, int th, int tw, int64_t* perm) {
  int64_t p = 0;
  for (int t0 = 0; t0 < T; t0 += tt)
    for (int y0 = 0; y0 < Hs; y0 += th)
      for (int x0 = 0; x0 < Ws; x0 += tw) {
        int t1 = min_int(t0 + tt, T), y1 = min_int(y0 + th, Hs), x1 = min_int(x0 + tw, Ws);
        for (int t = t0; t < t1; ++t)
          for (int y = y0; y < y1; ++y)
            for (int x = x0; x < x1; ++x) perm[p++] = ((int64_t)t * Hs + y) * Ws + x;
      }
}

/* Gather rows of d bf16 values: out[bh, p, :] = in[bh, perm[p], :] for
 * p < n, zero for n <= p < n_pad.  in is [BH, n, d], out is [BH, n_pad, d]. */
void oracle_permute(const uint16_t* in, uint16_t* out, int64_t BH, int64_t n, int64_t n_pad,
                    int d, const int64_t* perm) {
  for (int64_t bh = 0; bh < BH; ++bh)
    for (int64_t p = 0; p < n_pad; ++p) {
      uint16_t* dst = out + (bh * n_pad + p) * d;
      if (p < n) {
        const uint16_t* src = in + (bh * n + perm[p]) * d;
        memcpy(dst, src, (size_t)d * sizeof(uint16_t));
      } else {
        memset(dst, 0, (size_t)d * sizeof(uint16_t));
      }
    }
}

/* Inverse: out[bh, perm[p], :] = in[bh, p, :] for p < n; pad rows dropped. */
void oracle_unpermute(const uint16_t* in, uint16_t* out, int64_t BH, int64_t n, int64_t n_pad,
                      int d, const int64_t* perm) {
  for (int64_t bh = 0; bh < BH; ++bh)
    for (int64_t p = 0; p < n; ++p)
      memcpy(out + (bh * n + perm[p]) * d, in + (bh * n_pad + p) * d,
             (size_t)d * sizeof(uint16_t));
}

/* ------------------------------------------------------------------ */
/* Masked softmax attention in fp64.                                    */
/*                                                                      */
/* q, k, v: raw bf16 bits, [B*H, n_pad, d] in permuted token order.     */
/* mask: [B*H, nb, nb] bytes, nb = n_pad / block, nonzero = kept.       */
/* rows: the flat query ids (bh * n_pad + i) to compute, or NULL for    */
/* all B*H*n_pad of them; n_rows their number.                          */
/* dense_literal = 1: score every valid key and put -inf on masked      */
/* blocks (the definition, literally).  0: visit only kept blocks,      */
/* which is the same result because exp(-inf) = 0.                      */
/* Outputs: out [n_rows, d], lse [n_rows].  Rows with no valid kept key */
/* and pad rows (i >= n_valid) give out = 0, lse = -inf.                */
/* ------------------------------------------------------------------ */
/* Query blocks of block_q tokens and key blocks of block_k tokens: the mask is
 * [BH, n_pad / block_q, n_pad / block_k] and query i, key j are in blocks
 * i / block_q and j / block_k.  (Equal sizes are the method as the pages run
 * it; block_k = block_q / 2 is the finer key granularity they name as the
 * remedy for the 128 x 128 granularity bottleneck.) */
void oracle_attention_blocks(const uint16_t* q, const uint16_t* k, const uint16_t* v,
                             const uint8_t* mask, int64_t BH, int64_t n_valid, int64_t n_pad,
                             int d, int block_q, int block_k, double scale, const int64_t* rows,
                             int64_t n_rows, int dense_literal, double* out, double* lse) {
  const int64_t nb_q = n_pad / block_q, nb_k = n_pad / block_k;
  (void)nb_q;
  const int block = block_k; /* the key-side block, as the loops below walk keys */
  if (rows == NULL) n_rows = BH * n_pad;

#pragma omp parallel
  {
    double* s = (double*)malloc((size_t)n_valid * sizeof(double));
    double* qi = (double*)malloc((size_t)d * sizeof(double));
#pragma omp for schedule(dynamic, 16)
    for (int64_t r = 0; r < n_rows; ++r) {
      int64_t flat = rows ? rows[r] : r;
      int64_t bh = flat / n_pad, i = flat % n_pad;
      double* o = out + r * d;
      for (int c = 0; c < d; ++c) o[c] = 0.0;
      lse[r] = -INFINITY;
      if (i >= n_valid) continue; /* pad query row */

      const uint16_t* qrow = q + (bh * n_pad + i) * d;
      for (int c = 0; c < d; ++c) qi[c] = bf16_bits_to_double(qrow[c]);
      const uint8_t* mrow = mask + (bh * nb_q + i / block_q) * nb_k;

      /* scores s_j for j < n_valid; -inf where the key block is masked */
      double m = -INFINITY;
      for (int64_t j = 0; j < n_valid; ++j) {
        int kept = mrow[j / block] != 0;
        if (!kept) {
          s[j] = -INFINITY;
          if (!dense_literal) { /* skip the rest of this masked block */
            int64_t jend = (j / block + 1) * block;
            for (int64_t jj = j + 1; jj < jend && jj < n_valid; ++jj) s[jj] = -INFINITY;
            j = jend - 1;
          }
          continue;
        }
        const uint16_t* krow = k + (bh * n_pad + j) * d;
        double dot = 0.0;
        for (int c = 0; c < d; ++c) dot += qi[c] * bf16_bits_to_double(krow[c]);
        s[j] = scale * dot;
        if (s[j] > m) m = s[j];
      }
      if (m == -INFINITY) continue; /* no kept key: zero output, lse = -inf */

      double l = 0.0;
      for (int64_t j = 0; j < n_valid; ++j) {
        if (s[j] == -INFINITY) continue; /* exp(-inf - m) = 0 */
        double p = exp(s[j] - m);
        l += p;
        const uint16_t* vrow = v + (bh * n_pad + j) * d;
        for (int c = 0; c < d; ++c) o[c] += p * bf16_bits_to_double(vrow[c]);
      }
      for (int c = 0; c < d; ++c) o[c] /= l;
      lse[r] = m + log(l);
    }
    free(s);
    free(qi);
  }
}

/* One block size for queries and keys (mask [BH, nb, nb]). */
void oracle_attention(const uint16_t* q, const uint16_t* k, const uint16_t* v,
                      const uint8_t* mask, int64_t BH, int64_t n_valid, int64_t n_pad, int d,
                      int block, double scale, const int64_t* rows, int64_t n_rows,
                      int dense_literal, double* out, double* lse) {
  oracle_attention_blocks(q, k, v, mask, BH, n_valid, n_pad, d, block, block, scale, rows, n_rows,
                          dense_literal, out, lse);
}

/* ------------------------------------------------------------------ */
/* Threshold map -> block mask.                                        */
/*                                                                     */
/* ScalingAttention Sec. 4.1.2 (Eq. 2): T(u,v) is the smallest density */
/* threshold at which block (u,v) joins the union of active regions,   */
/* and a mask for any target density p is the comparison               */
/* M_p = 1(T <= p).  Algorithm 1 (FAST, mask instantiation) picks one  */
/* p* per layer, timestep and head, so here p holds one threshold per  */
/* head and the map is shared by every batch item.                     */
/*   thr   [H, nb_q, nb_k] float, p [H] float                          */
/*   dense [B, H, nb_q, nb_k] uint8, 1 where thr <= p[h] (a NaN        */
/*         threshold never compares true, so it is never kept)         */
/* ------------------------------------------------------------------ */
void oracle_threshold_mask(const float* thr, const float* p, int B, int H, int nb_q, int nb_k,
                           uint8_t* dense) {
  for (int b = 0; b < B; ++b)
    for (int h = 0; h < H; ++h)
      for (int u = 0; u < nb_q; ++u)
        for (int v = 0; v < nb_k; ++v) {
          const float t = thr[((int64_t)h * nb_q + u) * nb_k + v];
          const int64_t o = (((int64_t)b * H + h) * nb_q + u) * nb_k + v;
          dense[o] = (t <= p[h]) ? 1 : 0;
        }
}

/* ------------------------------------------------------------------ */
/* Threshold map resize, ScalingAttention Sec. 4.3.1 (Eq. 7).          */
/*                                                                     */
/* Eq. 7 samples the base map by bilinear interpolation at             */
/* (u / s_h, v / s_w) and applies a ceiling so that any overlap with   */
/* an active region survives.  Reading: s_h = tq / sq and s_w = tk / sk */
/* are the map's scale factors along its query and key axes, and the   */
/* ceiling acts on the interpolated active-region indicator 1(T <= p): */
/* the ceiling of a bilinear mix of 0/1 values is 1 exactly when some  */
/* source block with a nonzero interpolation weight is active.  For    */
/* every p at once that is the same as giving the target block the     */
/* minimum threshold over those source blocks, which is what we store. */
/* NaN thresholds (never active) are skipped; all-NaN gives NaN.       */
/*   src [H, sq, sk] float  ->  dst [H, tq, tk] float                  */
/* ------------------------------------------------------------------ */

/* Source blocks with a nonzero bilinear weight at sample x = u / s,
 * s = n_dst / n_src: floor(x) (weight 1 - frac, never 0) and floor(x) + 1
 * (weight frac) when frac > 0, clamped to the last block. */
static int bilinear_support(int u, int n_src, int n_dst, int* idx) {
  const double x = (double)u * (double)n_src / (double)n_dst;
  const double x0 = floor(x);
  const double frac = x - x0;
  int n = 0;
  idx[n++] = (int)x0;
  if (frac > 0.0) idx[n++] = ((int)x0 + 1 < n_src) ? (int)x0 + 1 : n_src - 1;
  return n;
}

void oracle_threshold_resize(const float* src, int H, int sq, int sk, float* dst, int tq,
                             int tk) {
  for (int h = 0; h < H; ++h)
    for (int u = 0; u < tq; ++u) {
      int rows[2], cols[2];
      const int nr = bilinear_support(u, sq, tq, rows);
      for (int v = 0; v < tk; ++v) {
        const int nc = bilinear_support(v, sk, tk, cols);
        float m = NAN;
        for (int a = 0; a < nr; ++a)
          for (int c = 0; c < nc; ++c) {
            const float t = src[((int64_t)h * sq + rows[a]) * sk + cols[c]];
            if (isnan(t)) continue;
            if (isnan(m) || t < m) m = t;
          }
        dst[((int64_t)h * tq + u) * tk + v] = m;
      }
    }
}

/* ------------------------------------------------------------------ */
/* Hilbert-curve token order (DFSAttn: Hilbert curve-based token       */
/* reordering; used with block-sparse attention as in ScalingAttention */
/* Sec. 5.4-5.5, token permutation into hardware-friendly blocks).     */
/*                                                                     */
/* The curve is the 3-D Hilbert curve over the cube of side 2^bits     */
/* that encloses the T x Hs x Ws grid, axes (t, y, x); grid points are */
/* taken in curve order and points outside the grid are skipped.  The  */
/* index of a point follows J. Skilling, "Programming the Hilbert      */
/* curve" (AIP Conf. Proc. 707, 2004): the axes are turned into the    */
/* "transpose" of the index by undoing, from the top level down, the   */
/* inversions and exchanges the inverse map would make, then Gray      */
/* coding across the axes; the index reads the transpose bit by bit,   */
/* top level first, axis t first.                                      */
/* ------------------------------------------------------------------ */
static uint64_t hilbert_key(const uint32_t axes_in[3], int bits) {
  uint32_t a[3] = {axes_in[0], axes_in[1], axes_in[2]};
  for (int level = bits - 1; level >= 1; --level) {
    const uint32_t bit = 1u << level;
    const uint32_t below = bit - 1u;
    for (int i = 0; i < 3; ++i) {
      if ((a[i] & bit) != 0) {
        a[0] ^= below; /* inversion of the low bits of axis 0 */
      } else {
        const uint32_t diff = (a[0] ^ a[i]) & below; /* exchange low bits of 0 and i */
        a[0] ^= diff;
        a[i] ^= diff;
      }
    }
  }
  for (int i = 1; i < 3; ++i) a[i] ^= a[i - 1]; /* Gray code across the axes */
  uint32_t flip = 0;
  for (int level = bits - 1; level >= 1; --level)
    if ((a[2] & (1u << level)) != 0) flip ^= (1u << level) - 1u;
  for (int i = 0; i < 3; ++i) a[i] ^= flip;
  uint64_t key = 0;
  for (int level = bits - 1; level >= 0; --level)
    for (int i = 0; i < 3; ++i) key = (key << 1) | (uint64_t)((a[i] >> level) & 1u);
  return key;
}

typedef struct {
  uint64_t key;
  int64_t frame;
} keyed_token;

static int cmp_keyed(const void* pa, const void* pb) {
  const keyed_token* a = (const keyed_token*)pa;
  const keyed_token* b = (const keyed_token*)pb;
  if (a->key < b->key) return -1;
  if (a->key > b->key) return 1;
  return 0;
}

/* Hilbert key of a point on the cube of side 2^bits (exposed for the pins). */
uint64_t oracle_hilbert_key(int t, int y, int x, int bits) {
  const uint32_t axes[3] = {(uint32_t)t, (uint32_t)y, (uint32_t)x};
  return hilbert_key(axes, bits);
}

/* perm[p] = frame-major index of the token at position p of the Hilbert order.
 * Returns the number of bits per axis of the enclosing cube. */
int oracle_hilbert_order(int T, int Hs, int Ws, int64_t* perm) {
  int side = T > Hs ? T : Hs;
  if (Ws > side) side = Ws;
  int bits = 1;
  while ((1 << bits) < side) ++bits;
  const int64_t n = (int64_t)T * Hs * Ws;
  keyed_token* tok = (keyed_token*)malloc((size_t)n * sizeof(keyed_token));
  if (!tok) return -1;
  for (int t = 0; t < T; ++t)
    for (int y = 0; y < Hs; ++y)
      for (int x = 0; x < Ws; ++x) {
        const int64_t f = ((int64_t)t * Hs + y) * Ws + x;
        tok[f].key = oracle_hilbert_key(t, y, x, bits);
        tok[f].frame = f;
      }
  qsort(tok, (size_t)n, sizeof(keyed_token), cmp_keyed);
  for (int64_t i = 0; i < n; ++i) perm[i] = tok[i].frame;
  free(tok);
  return bits;
}

/* ------------------------------------------------------------------ */
/* Online top-p block mask (dynamic block-sparse prediction).          */
/*                                                                     */
/* The block scores and the cut follow ScalingAttention Algorithm 1    */
/* (sort the block scores, accumulate, cut where the cumulative share  */
/* reaches p: the Top-k(S, p) of Eq. 2) applied row by row as online   */
/* top-p predictors do, with a top-p threshold per head (the selective */
/* head globalization page: per-head top-p thresholds).  The block     */
/* score is the proxy of pooled queries and keys:                      */
/*   qbar_i = mean of the valid tokens of query block i, kbar_j alike  */
/*   s_ij = qbar_i . kbar_j / (sqrt(d) * tau_h),  p_ij = softmax_j s_ij */
/* Row i keeps the blocks taken in descending p (ties: lower j first)  */
/* up to and including the one at which the cumulative sum reaches     */
/* top_p[h] (at least one block; all blocks if the sum never does).    */
/*   q, k   raw bf16 [B*H, n_pad, d] (tokens in block order)           */
/*   mask   out uint8 [B*H, nb, nb];  prob out double [B*H, nb, nb]    */
/*          (may be NULL)                                              */
/* ------------------------------------------------------------------ */
typedef struct {
  double p;
  int j;
} prob_entry;

static int cmp_prob_desc(const void* pa, const void* pb) {
  const prob_entry* a = (const prob_entry*)pa;
  const prob_entry* b = (const prob_entry*)pb;
  if (a->p > b->p) return -1;
  if (a->p < b->p) return 1;
  return (a->j > b->j) - (a->j < b->j);
}

static void block_means(const uint16_t* x, int64_t n_valid, int d, int block, int nb,
                        double* out /* [nb, d] */) {
  for (int i = 0; i < nb; ++i) {
    int64_t lo = (int64_t)i * block, hi = lo + block;
    if (hi > n_valid) hi = n_valid;
    for (int c = 0; c < d; ++c) out[(int64_t)i * d + c] = 0.0;
    for (int64_t t = lo; t < hi; ++t)
      for (int c = 0; c < d; ++c) out[(int64_t)i * d + c] += bf16_bits_to_double(x[t * d + c]);
    const double cnt = (double)(hi - lo);
    for (int c = 0; c < d; ++c) out[(int64_t)i * d + c] /= cnt;
  }
}

void oracle_top_p_mask(const uint16_t* q, const uint16_t* k, int64_t B, int64_t H,
                       int64_t n_valid, int64_t n_pad, int d, int block, const double* tau,
                       const double* top_p, uint8_t* mask, double* prob) {
  const int nb = (int)(n_pad / block);
#pragma omp parallel for schedule(dynamic)
  for (int64_t bh = 0; bh < B * H; ++bh) {
    const int64_t h = bh % H;
    double* qm = (double*)malloc(sizeof(double) * (size_t)nb * d);
    double* km = (double*)malloc(sizeof(double) * (size_t)nb * d);
    double* s = (double*)malloc(sizeof(double) * (size_t)nb);
    prob_entry* order = (prob_entry*)malloc(sizeof(prob_entry) * (size_t)nb);
    block_means(q + bh * n_pad * d, n_valid, d, block, nb, qm);
    block_means(k + bh * n_pad * d, n_valid, d, block, nb, km);
    const double denom = sqrt((double)d) * tau[h];
    for (int i = 0; i < nb; ++i) {
      double m = -INFINITY;
      for (int j = 0; j < nb; ++j) {
        double dot = 0.0;
        for (int c = 0; c < d; ++c) dot += qm[(int64_t)i * d + c] * km[(int64_t)j * d + c];
        s[j] = dot / denom;
        if (s[j] > m) m = s[j];
      }
      double l = 0.0;
      for (int j = 0; j < nb; ++j) l += exp(s[j] - m);
      uint8_t* row = mask + (bh * nb + i) * (int64_t)nb;
      for (int j = 0; j < nb; ++j) {
        order[j].p = exp(s[j] - m) / l;
        order[j].j = j;
        row[j] = 0;
        if (prob) prob[(bh * nb + i) * (int64_t)nb + j] = order[j].p;
      }
      qsort(order, (size_t)nb, sizeof(prob_entry), cmp_prob_desc);
      double cum = 0.0;
      for (int r = 0; r < nb; ++r) {
        row[order[r].j] = 1;
        cum += order[r].p;
        if (cum >= top_p[h]) break;
      }
    }
    free(qm);
    free(km);
    free(s);
    free(order);
  }
}
