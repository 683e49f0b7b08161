"""GPU parity of bsa_gather_rows with the other token orders, bit-exact against
the oracle's permutation of the same tokens: the Hilbert-curve order
(DFSAttn's Hilbert curve-based token reordering) and head-aware tiling
(Veda: a tile shape per head), both ways, plus the zero rows of the tail and
of out-of-range table entries; and the attention forward on Hilbert-ordered
tokens against the oracle."""
import numpy as np
import pytest
import torch

import oracle
from block_sparse_attention_forward_b200 import inputs as I
from tests.helpers import bf16_bits

pytestmark = pytest.mark.gpu

HEAD_TILES = [(1, 8, 16), (2, 8, 8), (4, 4, 8), (1, 16, 8)]


def _x(B, H, n, d, seed):
    g = torch.Generator().manual_seed(seed)
    return torch.randn((B, H, n, d), generator=g).to(torch.bfloat16)


@pytest.mark.parametrize("grid,d,extra", [((4, 16, 16), 64, 0), ((21, 45, 80), 128, 48),
                                          ((3, 5, 7), 8, 23), ((33, 48, 80), 128, 0)])
def test_hilbert_gather_both_ways(cuda_ok, grid, d, extra):
    import block_sparse_attention_forward_b200 as bsa
    T, Hs, Ws = grid
    n = T * Hs * Ws
    n_pad = n + extra
    B, H = 1, 2
    x = _x(B, H, n, d, n)
    fwd, inv = bsa.order_tables(bsa.hilbert_order(T, Hs, Ws), n_pad)
    y = bsa.gather_rows(x.cuda(), fwd.cuda())
    z = bsa.gather_rows(y, inv.cuda())
    torch.cuda.synchronize()
    ref = oracle.permute(bf16_bits(x).reshape(B * H, n, d), oracle.hilbert_order(T, Hs, Ws), n_pad)
    np.testing.assert_array_equal(bf16_bits(y).reshape(B * H, n_pad, d), ref)
    np.testing.assert_array_equal(bf16_bits(z), bf16_bits(x))


@pytest.mark.parametrize("name", ["tiny", "wan14b_720p"])
def test_head_aware_tiles_both_ways(cuda_ok, name):
    import block_sparse_attention_forward_b200 as bsa
    w = I.WORKLOADS[name]
    B, H = 2, 4
    x = _x(B, H, w.n, w.d, 7)
    tabs = [bsa.order_tables(bsa.tile_order(w.T, w.Hs, w.Ws, *HEAD_TILES[h]), w.n_pad)
            for h in range(H)]
    fwd = torch.stack([f for f, _ in tabs]).cuda()
    inv = torch.stack([i for _, i in tabs]).cuda()
    y = bsa.gather_rows(x.cuda(), fwd)
    z = bsa.gather_rows(y, inv)
    torch.cuda.synchronize()
    xb = bf16_bits(x)
    yb = bf16_bits(y)
    for h in range(H):
        perm = oracle.tile_order(w.T, w.Hs, w.Ws, *HEAD_TILES[h])
        ref = oracle.permute(xb[:, h], perm, w.n_pad)
        np.testing.assert_array_equal(yb[:, h], ref)
    np.testing.assert_array_equal(bf16_bits(z), xb)


def test_out_of_range_entries_give_zero_rows(cuda_ok):
    import block_sparse_attention_forward_b200 as bsa
    x = _x(1, 3, 10, 16, 3)
    src = torch.tensor([9, -1, 0, 10, 123456, 5, -7, 2], dtype=torch.int32)
    y = bsa.gather_rows(x.cuda(), src.cuda()).cpu()
    for i, s in enumerate(src.tolist()):
        want = x[:, :, s] if 0 <= s < 10 else torch.zeros_like(x[:, :, 0])
        assert torch.equal(y[:, :, i], want), i


def test_forward_on_hilbert_ordered_tokens(cuda_ok):
    import block_sparse_attention_forward_b200 as bsa
    from tests.helpers import OUT_MAX_ABS, OUT_MEAN_ABS, LSE_ABS
    w = I.WORKLOADS["tiny"]
    q, k, v = I.gen_qkv(w)
    mask = I.gen_mask(w)
    fwd, inv = bsa.order_tables(bsa.hilbert_order(w.T, w.Hs, w.Ws), w.n_pad)
    fwd_d = fwd.cuda()
    qp, kp, vp = (bsa.gather_rows(t.cuda(), fwd_d) for t in (q, k, v))
    pm = bsa.pack_mask(torch.from_numpy(mask).cuda())
    out_p, lse = bsa.forward(qp, kp, vp, pm, w.n, w.block)
    torch.cuda.synchronize()
    BH = w.B * w.H
    perm = oracle.hilbert_order(w.T, w.Hs, w.Ws)
    qo, ko, vo = (oracle.permute(bf16_bits(t).reshape(BH, w.n, w.d), perm, w.n_pad)
                  for t in (q, k, v))
    ref, ref_lse = oracle.attention(qo, ko, vo, mask.reshape(BH, w.nb, w.nb), w.n, w.block)
    err = np.abs(out_p.float().cpu().numpy().reshape(-1, w.d) - ref)
    assert err.max() <= OUT_MAX_ABS and err.mean() <= OUT_MEAN_ABS
    lse_g = lse.cpu().numpy().reshape(-1)
    fin = np.isfinite(ref_lse)
    assert np.array_equal(np.isfinite(lse_g), fin)
    assert np.abs(lse_g[fin] - ref_lse[fin]).max() <= LSE_ABS
