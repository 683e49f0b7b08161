"""GPU parity of the threshold-map steps against the oracle, bit-exact:

- bsa_pack_mask_from_threshold: M_p = 1(T <= p_h) straight to CRM rows,
  counts, row offsets, kept-block lists and schedule ("ScalingAttention",
  Sec. 4.1.2 and Algorithm 1), compared with the oracle's threshold mask
  followed by the oracle's packing;
- bsa_threshold_resize: the conservative resize of Eq. 7 (Sec. 4.3.1),
  compared value by value with the oracle (NaN where the oracle has NaN);
- both composed, at the resolution change the pages describe (a map built at
  480p reused at 720p).

All of this is integer work or an exact minimum, so the comparison is exact."""
import numpy as np
import pytest
import torch

import oracle
from block_sparse_attention_forward_b200 import inputs as I
from tests.helpers import check_schedule

pytestmark = pytest.mark.gpu


def _oracle_pack(dense):
    bits = oracle.pack_bits(dense)
    counts, offsets, cols = oracle.crm_lists(bits)
    return bits, counts, offsets, cols, dense.shape[2:]


def _compare(pm, ref):
    bits, counts, offsets, cols, (nb_q, nb_k) = ref
    np.testing.assert_array_equal(pm.bits.cpu().numpy().view(np.uint32), bits)
    np.testing.assert_array_equal(pm.counts.cpu().numpy(), counts)
    np.testing.assert_array_equal(pm.row_offsets.cpu().numpy().astype(np.int64), offsets)
    total = int(offsets[-1])
    np.testing.assert_array_equal(pm.col_idx[:total].cpu().numpy(), cols)
    check_schedule(pm.schedule.cpu().numpy(), counts, nb_q, nb_k)


def _pack_threshold_and_compare(thr, p, B=1):
    import block_sparse_attention_forward_b200 as bsa
    pm = bsa.pack_mask_from_threshold(torch.from_numpy(thr).cuda(), torch.from_numpy(p).cuda(),
                                      B=B)
    torch.cuda.synchronize()
    _compare(pm, _oracle_pack(oracle.threshold_mask(thr, p, B=B)))
    return pm


@pytest.mark.parametrize("name", ["tiny", "wan13b_480p", "wan14b_480p", "wan14b_720p",
                                  "hunyuan_768p"])
def test_pack_from_threshold_workloads(cuda_ok, name):
    w = I.WORKLOADS[name]
    thr, p = I.gen_threshold(w)
    _pack_threshold_and_compare(thr, p, B=w.B)


@pytest.mark.parametrize("B,H,nbq,nbk", [(1, 1, 1, 1), (2, 3, 5, 33), (3, 2, 64, 64),
                                         (1, 4, 100, 65), (2, 1, 7, 4097), (1, 5, 31, 257)])
def test_pack_from_threshold_edge_shapes(cuda_ok, B, H, nbq, nbk):
    rng = np.random.default_rng(B * 1000 + nbk)
    thr = (rng.integers(1, 21, size=(H, nbq, nbk)) / 20).astype(np.float32)
    p = (rng.integers(0, 21, size=H) / 20).astype(np.float32)
    _pack_threshold_and_compare(thr, p, B=B)


def test_pack_from_threshold_special_values(cuda_ok):
    # NaN never kept, +inf kept only at p = +inf, -0 <= +0, equality kept;
    # p = -inf and p = NaN give empty rows (counts 0, schedule still valid)
    H, nbq, nbk = 6, 9, 40
    rng = np.random.default_rng(77)
    thr = rng.random((H, nbq, nbk)).astype(np.float32)
    thr[:, :, ::7] = np.nan
    thr[:, :, 3] = np.inf
    thr[:, 1, :] = -0.0
    thr[:, 2, 5] = np.float32(0.5)
    p = np.array([np.inf, -np.inf, np.nan, 0.5, 0.0, 1.0], dtype=np.float32)
    pm = _pack_threshold_and_compare(thr, p, B=2)
    counts = pm.counts.cpu().numpy().reshape(2, H, nbq)
    assert counts[:, 1].sum() == 0 and counts[:, 2].sum() == 0


def test_pack_from_threshold_matches_pack_mask(cuda_ok):
    # the same mask through both entry points gives the same bytes
    import block_sparse_attention_forward_b200 as bsa
    w = I.WORKLOADS["wan14b_720p"]
    thr, p = I.gen_threshold(w)
    a = bsa.pack_mask_from_threshold(torch.from_numpy(thr).cuda(), torch.from_numpy(p).cuda())
    b = bsa.pack_mask(torch.from_numpy(oracle.threshold_mask(thr, p)).cuda())
    torch.cuda.synchronize()
    for key in ("bits", "counts", "row_offsets", "schedule"):
        assert torch.equal(getattr(a, key), getattr(b, key)), key
    total = int(a.row_offsets[-1])
    assert torch.equal(a.col_idx[:total], b.col_idx[:total])


def _assert_same_thresholds(got, want):
    assert got.shape == want.shape
    nan = np.isnan(want)
    np.testing.assert_array_equal(np.isnan(got), nan)
    np.testing.assert_array_equal(got[~nan], want[~nan])


@pytest.mark.parametrize("H,sq,sk,tq,tk", [(2, 8, 8, 19, 19), (3, 16, 12, 37, 29),
                                           (2, 21, 21, 9, 9), (40, 256, 256, 591, 591),
                                           (1, 1, 1, 5, 7), (4, 7, 30, 7, 11), (2, 591, 591, 256, 256),
                                           (24, 256, 256, 990, 990), (2, 40, 1500, 33, 1700)])
def test_threshold_resize_matches_oracle(cuda_ok, H, sq, sk, tq, tk):
    import block_sparse_attention_forward_b200 as bsa
    rng = np.random.default_rng(H * 7 + sq + tq)
    src = (rng.integers(1, 21, size=(H, sq, sk)) / 20).astype(np.float32)
    src[rng.random(src.shape) < 0.05] = np.nan
    got = bsa.threshold_resize(torch.from_numpy(src).cuda(), tq, tk)
    torch.cuda.synchronize()
    _assert_same_thresholds(got.cpu().numpy(), oracle.threshold_resize(src, tq, tk))


def test_threshold_resize_zeros_and_all_nan(cuda_ok):
    import block_sparse_attention_forward_b200 as bsa
    src = np.array([[[np.nan, np.nan, 0.0], [np.nan, -0.0, 0.25], [0.5, 0.0, -0.0]]],
                   dtype=np.float32)
    got = bsa.threshold_resize(torch.from_numpy(src).cuda(), 7, 8).cpu().numpy()
    want = oracle.threshold_resize(src, 7, 8)
    # values agree (+0 == -0: the sign of a tied zero is unspecified, and no
    # mask 1(T <= p) can tell the two apart)
    _assert_same_thresholds(got, want)
    for p in (-0.0, 0.0, 0.25):
        np.testing.assert_array_equal(got <= np.float32(p), want <= np.float32(p))


def test_resize_then_pack_480p_map_at_720p(cuda_ok):
    # a map built once at the 480p block grid, reused at 720p (Sec. 4.3.1)
    import block_sparse_attention_forward_b200 as bsa
    base = I.WORKLOADS["wan14b_480p"]
    target = I.WORKLOADS["wan14b_720p"]
    thr, p = I.gen_threshold(base)
    thr_d, p_d = torch.from_numpy(thr).cuda(), torch.from_numpy(p).cuda()
    resized = bsa.threshold_resize(thr_d, target.nb, target.nb)
    pm = bsa.pack_mask_from_threshold(resized, p_d)
    torch.cuda.synchronize()
    ref_thr = oracle.threshold_resize(thr, target.nb, target.nb)
    _assert_same_thresholds(resized.cpu().numpy(), ref_thr)
    _compare(pm, _oracle_pack(oracle.threshold_mask(ref_thr, p)))
