"""GPU parity of the integer steps against the oracle, bit-exact: CRM
packing, kept-block lists (bsa_pack_mask) and the 3-D tile gather in both
directions (bsa_tile_permute / bsa_tile_unpermute).  The schedule has several
correct values (any work order gives the same attention output): it must be
a permutation of the rows in the oracle's count order or in that order taken
head by head, and the form must be the one the library's policy picks
(tests/helpers.py states the policy)."""
import numpy as np
import pytest
import torch

import oracle
from block_sparse_attention_forward_b200 import inputs as I
from tests.helpers import bf16_bits, check_schedule

pytestmark = pytest.mark.gpu


def _pack_and_compare(dense: np.ndarray):
    import block_sparse_attention_forward_b200 as bsa
    B, H, nbq, nbk = dense.shape
    pm = bsa.pack_mask(torch.from_numpy(dense).cuda())
    torch.cuda.synchronize()
    bits_ref = oracle.pack_bits(dense)
    counts_ref, offsets_ref, col_ref = oracle.crm_lists(bits_ref)
    np.testing.assert_array_equal(pm.bits.cpu().numpy().view(np.uint32), bits_ref)
    np.testing.assert_array_equal(pm.counts.cpu().numpy(), counts_ref)
    np.testing.assert_array_equal(pm.row_offsets.cpu().numpy().astype(np.int64), offsets_ref)
    total = int(offsets_ref[-1])
    np.testing.assert_array_equal(pm.col_idx[:total].cpu().numpy(), col_ref)
    return check_schedule(pm.schedule.cpu().numpy(), counts_ref, nbq, nbk)


@pytest.mark.parametrize("name", ["tiny", "wan13b_480p", "wan14b_480p", "wan14b_720p",
                                  "hunyuan_768p"])
def test_pack_mask_workloads(cuda_ok, name):
    w = I.WORKLOADS[name]
    _pack_and_compare(I.gen_mask(w))


def _mask_with_counts(counts_per_row: np.ndarray, nbk: int, seed: int) -> np.ndarray:
    """[1, H, nbq, nbk] mask whose row (h, i) keeps counts_per_row[h, i] random blocks."""
    rng = np.random.default_rng(seed)
    H, nbq = counts_per_row.shape
    dense = np.zeros((1, H, nbq, nbk), dtype=np.uint8)
    for h in range(H):
        for i in range(nbq):
            dense[0, h, i, rng.choice(nbk, size=int(counts_per_row[h, i]), replace=False)] = 1
    return dense


def test_pack_schedule_head_major_when_heads_mix(cuda_ok):
    # every head draws its counts from one distribution: the count order mixes
    # all 16 heads in every window of 148, so the policy goes head-major
    rng = np.random.default_rng(11)
    counts = rng.integers(0, 200, size=(16, 96))
    dense = _mask_with_counts(counts, 256, 12)
    assert _pack_and_compare(dense) == "head"


def test_pack_schedule_head_major_long_heads_and_batches(cuda_ok):
    # B = 2 (each (b, h) is its own head in the policy) and 1,500 rows per
    # head: more rows than one CTA's threads, so the head-major ranking loops
    rng = np.random.default_rng(14)
    B, H, nbq, nbk = 2, 5, 1500, 256
    dense = (rng.random((B, H, nbq, nbk)) < rng.uniform(0.1, 0.9, size=(B, H, nbq, 1))).astype(np.uint8)
    assert _pack_and_compare(dense) == "head"


def test_pack_schedule_stays_count_order_when_heads_separate(cuda_ok):
    # disjoint count ranges per head: about two heads per window, whose K and V
    # fit in L2, so the count order stays
    rng = np.random.default_rng(7)
    counts = np.stack([h * 20 + rng.integers(0, 15, size=96) for h in range(12)])
    dense = _mask_with_counts(counts, 256, 15)
    assert _pack_and_compare(dense) == "count"


@pytest.mark.parametrize("heads,form", [(8, "count"), (9, "head")])
def test_pack_schedule_mix_threshold(cuda_ok, heads, form):
    # row i of every head keeps 200 - i blocks: each count level lists all the
    # heads, so every window of 148 holds all of them; nb_k is chosen so that
    # this GPU's L2 holds the K and V of 8.5 heads: 8 heads per window stay in
    # count order, 9 turn head-major
    from tests.helpers import POLICY_KEY_BLOCK_BYTES, device_l2_bytes
    nbq = 148
    nbk = int(device_l2_bytes() / (8.5 * POLICY_KEY_BLOCK_BYTES))
    assert nbk >= 200
    counts = np.tile(200 - np.arange(nbq), (heads, 1))
    dense = _mask_with_counts(counts, nbk, 13)
    assert _pack_and_compare(dense) == form


@pytest.mark.parametrize("shape,density", [((1, 1, 1, 1), 1.0), ((1, 3, 5, 33), 0.3),
                                           ((2, 3, 64, 64), 0.0), ((1, 2, 100, 65), 0.9),
                                           ((1, 4, 990, 990), 0.12), ((3, 1, 7, 1100), 0.5),
                                           ((1, 2, 40, 2000), 0.4)])
def test_pack_mask_edge_shapes(cuda_ok, shape, density):
    rng = np.random.default_rng(sum(shape))
    dense = (rng.random(shape) < density).astype(np.uint8)
    dense[dense == 1] = rng.integers(1, 256, size=int(dense.sum()), dtype=np.uint8)
    _pack_and_compare(dense)


@pytest.mark.parametrize("name", ["tiny", "wan13b_480p", "wan14b_720p", "hunyuan_768p"])
def test_permute_roundtrip_workload_grids(cuda_ok, name):
    import block_sparse_attention_forward_b200 as bsa
    w = I.WORKLOADS[name]
    g = torch.Generator().manual_seed(w.seed)
    x = torch.randn((1, 2, w.n, w.d), generator=g).to(torch.bfloat16)
    grid, tile = (w.T, w.Hs, w.Ws), (w.tt, w.th, w.tw)
    y = bsa.tile_permute(x.cuda(), grid, tile, w.n_pad)
    z = bsa.tile_unpermute(y, grid, tile)
    torch.cuda.synchronize()
    perm = oracle.tile_order(w.T, w.Hs, w.Ws, w.tt, w.th, w.tw)
    ref = oracle.permute(bf16_bits(x).reshape(2, w.n, w.d), perm, w.n_pad)
    np.testing.assert_array_equal(bf16_bits(y).reshape(2, w.n_pad, w.d), ref)
    np.testing.assert_array_equal(bf16_bits(z), bf16_bits(x))


@pytest.mark.parametrize("grid,tile,d,n_extra", [((5, 7, 9), (2, 3, 4), 8, 3), ((1, 1, 1), (1, 1, 1), 64, 0),
                                                 ((3, 17, 33), (2, 8, 16), 136, 100),
                                                 ((4, 4, 4), (8, 8, 8), 128, 0)])
def test_permute_ragged_shapes(cuda_ok, grid, tile, d, n_extra):
    import block_sparse_attention_forward_b200 as bsa
    n = grid[0] * grid[1] * grid[2]
    n_pad = n + n_extra
    g = torch.Generator().manual_seed(n)
    x = torch.randn((2, 3, n, d), generator=g).to(torch.bfloat16)
    y = bsa.tile_permute(x.cuda(), grid, tile, n_pad)
    torch.cuda.synchronize()
    perm = oracle.tile_order(*grid, *tile)
    ref = oracle.permute(bf16_bits(x).reshape(6, n, d), perm, n_pad)
    np.testing.assert_array_equal(bf16_bits(y).reshape(6, n_pad, d), ref)
    z = bsa.tile_unpermute(y, grid, tile)
    np.testing.assert_array_equal(bf16_bits(z), bf16_bits(x))
