"""Pins for the oracle's threshold-map functions, none of which re-types the oracle.

- ``threshold_mask`` follows "ScalingAttention", Sec. 4.1.2 (Eq. 2 and the
  instantiation M_p = 1(T <= p)) with one threshold per head (Algorithm 1,
  FAST mask instantiation).  It is pinned by properties that the definition
  fixes: an inclusive comparison (a block whose threshold equals p is kept),
  the exact count of kept blocks when the thresholds are distinct levels,
  monotonicity in p, the per-head choice of p, and copies per batch item.
- ``threshold_resize`` follows Sec. 4.3.1, Eq. 7.  It is pinned against a
  library routine: scipy's linear ``map_coordinates`` resamples each binary
  mask 1(T <= p) at (u * sq / tq, v * sk / tk), and the ceiling of the result
  must equal 1(resized T <= p) for every level p.  Closed forms for an
  integer upscale and the identity resize are also checked.
"""
import numpy as np
import pytest
from scipy import ndimage

import oracle



def _levels_map(H, nq, nk, seed):
    """Thresholds that are a random permutation of the distinct levels
    1/n, 2/n, ..., n/n per head (n = nq * nk)."""
    rng = np.random.default_rng(seed)
    n = nq * nk
    out = np.empty((H, nq, nk), dtype=np.float32)
    for h in range(H):
        out[h] = (rng.permutation(n) + 1).reshape(nq, nk).astype(np.float32) / np.float32(n)
    return out


def test_mask_keeps_a_block_whose_threshold_equals_p():
    # hand example: thresholds 0.125, 0.25, 0.375, 0.5 (exact in binary)
    thr = np.array([[[0.125, 0.25], [0.375, 0.5]]], dtype=np.float32)
    for p, want in ((0.25, [[1, 1], [0, 0]]), (0.2499, [[1, 0], [0, 0]]),
                    (0.5, [[1, 1], [1, 1]]), (0.0, [[0, 0], [0, 0]])):
        got = oracle.threshold_mask(thr, np.array([p], dtype=np.float32))
        assert got.tolist() == [[want]], p


def test_mask_count_is_exact_for_distinct_levels():
    H, nq, nk = 3, 7, 9
    thr = _levels_map(H, nq, nk, seed=11)
    n = nq * nk
    for k in (0, 1, 5, n // 2, n - 1, n):
        p = np.full(H, np.float32(k) / np.float32(n), dtype=np.float32)
        m = oracle.threshold_mask(thr, p)
        assert m.shape == (1, H, nq, nk)
        # level k/n is kept, so exactly k blocks per head
        assert m.reshape(H, -1).sum(axis=1).tolist() == [k] * H


def test_mask_is_monotone_in_p_and_per_head():
    H, nq, nk = 4, 6, 37
    rng = np.random.default_rng(5)
    thr = rng.random((H, nq, nk), dtype=np.float32)
    ps = np.sort(rng.random(6)).astype(np.float32)
    prev = None
    for p in ps:
        m = oracle.threshold_mask(thr, np.full(H, p, dtype=np.float32))
        if prev is not None:
            assert np.all(m >= prev)
        prev = m
    # a different p per head: head h's mask equals the mask of a shared p[h]
    p = np.array([0.1, 0.9, 0.4, 0.0], dtype=np.float32)
    m = oracle.threshold_mask(thr, p, B=3)
    for h in range(H):
        alone = oracle.threshold_mask(thr, np.full(H, p[h], dtype=np.float32))
        for b in range(3):
            assert np.array_equal(m[b, h], alone[0, h])


def test_mask_nan_never_kept_inf_always_dropped():
    thr = np.array([[[np.nan, np.inf, -np.inf, 0.0]]], dtype=np.float32)
    m = oracle.threshold_mask(thr, np.array([np.inf], dtype=np.float32))
    assert m.tolist() == [[[[0, 1, 1, 1]]]]
    m = oracle.threshold_mask(thr, np.array([np.nan], dtype=np.float32))
    assert m.tolist() == [[[[0, 0, 0, 0]]]]


def test_resize_identity():
    rng = np.random.default_rng(2)
    src = rng.random((2, 13, 17), dtype=np.float32)
    assert np.array_equal(oracle.threshold_resize(src, 13, 17), src)


def test_resize_integer_upscale_closed_form():
    rng = np.random.default_rng(3)
    src = rng.random((2, 5, 4), dtype=np.float32)
    dst = oracle.threshold_resize(src, 10, 8)
    for u in range(10):
        for v in range(8):
            a = [u // 2] + ([min(u // 2 + 1, 4)] if u % 2 else [])
            c = [v // 2] + ([min(v // 2 + 1, 3)] if v % 2 else [])
            for h in range(2):
                want = min(float(src[h, i, j]) for i in a for j in c)
                assert dst[h, u, v] == np.float32(want)


@pytest.mark.parametrize("sq,sk,tq,tk", [(8, 8, 19, 19), (16, 12, 37, 29), (21, 21, 9, 9),
                                         (256, 256, 591, 591), (7, 30, 7, 11)])
def test_resize_is_the_ceiling_of_bilinear_masks(sq, sk, tq, tk):
    # Eq. 7 read as: resample the active-region indicator bilinearly and take
    # the ceiling.  scipy's order-1 map_coordinates is the bilinear sampler;
    # mode "nearest" clamps the neighbour past the last block.
    H = 2
    levels = 11
    rng = np.random.default_rng(sq * 1000 + tq)
    src = (rng.integers(1, levels + 1, size=(H, sq, sk)) / levels).astype(np.float32)
    dst = oracle.threshold_resize(src, tq, tk)
    uu, vv = np.meshgrid(np.arange(tq, dtype=np.float64) * sq / tq,
                         np.arange(tk, dtype=np.float64) * sk / tk, indexing="ij")
    for h in range(H):
        for k in range(levels + 1):
            p = np.float32(k / levels)
            m = (src[h] <= p).astype(np.float64)
            interp = ndimage.map_coordinates(m, [uu, vv], order=1, mode="nearest")
            want = np.ceil(np.clip(interp, 0.0, 1.0) - 1e-12)
            got = (dst[h] <= p).astype(np.float64)
            assert np.array_equal(got, want), (h, k)


def test_resize_skips_nan_and_keeps_active_overlap():
    src = np.array([[[np.nan, 0.5], [np.nan, np.nan]]], dtype=np.float32)
    dst = oracle.threshold_resize(src, 4, 4)
    # (0, 0) samples only source (0, 0): NaN stays NaN
    assert np.isnan(dst[0, 0, 0])
    # (0, 1) samples (0, 0) and (0, 1): the NaN is skipped
    assert dst[0, 0, 1] == np.float32(0.5)
    # upscaling never loses an active block: density at p does not drop
    rng = np.random.default_rng(8)
    src = rng.random((3, 10, 10), dtype=np.float32)
    dst = oracle.threshold_resize(src, 23, 23)
    for p in (0.1, 0.3, 0.6):
        assert (dst <= p).mean() >= (src <= p).mean()
