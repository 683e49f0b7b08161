"""The library's host-side order tables (no GPU needed) against the oracle,
exactly: the 3-D Hilbert order (bsa_hilbert_order), the tile order as a table
(bsa_tile_order), and the gather tables built from an order
(bsa_order_tables), which must reject anything that is not a permutation."""
import numpy as np
import pytest
import torch

import oracle
from block_sparse_attention_forward_b200 import inputs as I


@pytest.fixture(scope="module")
def bsa():
    from block_sparse_attention_forward_b200 import build
    build.build()
    import block_sparse_attention_forward_b200 as m
    return m


@pytest.mark.parametrize("grid", [(1, 1, 1), (2, 2, 2), (3, 5, 7), (4, 16, 16), (21, 30, 52),
                                  (21, 45, 80), (33, 48, 80), (64, 1, 3)])
def test_hilbert_order_matches_oracle(bsa, grid):
    np.testing.assert_array_equal(bsa.hilbert_order(*grid).numpy(), oracle.hilbert_order(*grid))


@pytest.mark.parametrize("name", ["tiny", "wan13b_480p", "wan14b_720p", "hunyuan_768p"])
def test_tile_order_table_matches_oracle(bsa, name):
    w = I.WORKLOADS[name]
    got = bsa.tile_order(w.T, w.Hs, w.Ws, w.tt, w.th, w.tw).numpy()
    np.testing.assert_array_equal(got, oracle.tile_order(w.T, w.Hs, w.Ws, w.tt, w.th, w.tw))


def test_order_tables_invert_and_pad(bsa):
    order = bsa.hilbert_order(3, 5, 7)
    fwd, inv = bsa.order_tables(order, 112)
    n = 105
    assert fwd[:n].tolist() == order.tolist() and fwd[n:].tolist() == [-1] * 7
    assert np.array_equal(inv.numpy()[order.numpy()], np.arange(n))


@pytest.mark.parametrize("bad", [[0, 1, 1], [0, 3, 1], [-1, 0, 1]])
def test_order_tables_reject_non_permutations(bsa, bad):
    with pytest.raises(bsa.BsaError):
        bsa.order_tables(torch.tensor(bad, dtype=torch.int32), 4)
