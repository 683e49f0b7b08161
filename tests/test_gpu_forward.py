"""GPU parity of the whole hot path against the fp64 oracle.

Path under test (all on the GPU, through the C ABI): bsa_tile_permute of q, k, v
-> bsa_pack_mask -> bsa_forward -> bsa_tile_unpermute.  Oracle: the CPU tile
order and gather, then masked softmax attention in fp64.

Small cases are compared on every row; the full-size workloads on stratified
query blocks (most kept, least kept, tail block, block 0, seeded extras).
Tolerances: out max-abs 2e-2, mean-abs 2e-3; lse 1e-3; -inf rows exact.
"""
import numpy as np
import pytest
import torch

import oracle
from block_sparse_attention_forward_b200 import inputs as I
from tests.helpers import (LSE_ABS, OUT_MAX_ABS, OUT_MEAN_ABS, bf16_bits, compare_out,
                           stratified_query_blocks)

pytestmark = pytest.mark.gpu


def run_gpu_path(w, q, k, v, mask):
    import block_sparse_attention_forward_b200 as bsa
    grid, tile = (w.T, w.Hs, w.Ws), (w.tt, w.th, w.tw)
    qp = bsa.tile_permute(q.cuda(), grid, tile, w.n_pad)
    kp = bsa.tile_permute(k.cuda(), grid, tile, w.n_pad)
    vp = bsa.tile_permute(v.cuda(), grid, tile, w.n_pad)
    pm = bsa.pack_mask(torch.from_numpy(mask).cuda())
    out_p, lse = bsa.forward(qp, kp, vp, pm, w.n, w.block)
    out = bsa.tile_unpermute(out_p, grid, tile)
    torch.cuda.synchronize()
    assert bsa.device_error() == 0
    return out.cpu(), out_p.cpu(), lse.cpu()


def oracle_inputs(w, q, k, v):
    BH = w.B * w.H
    perm = oracle.tile_order(w.T, w.Hs, w.Ws, w.tt, w.th, w.tw)
    qp = oracle.permute(bf16_bits(q).reshape(BH, w.n, w.d), perm, w.n_pad)
    kp = oracle.permute(bf16_bits(k).reshape(BH, w.n, w.d), perm, w.n_pad)
    vp = oracle.permute(bf16_bits(v).reshape(BH, w.n, w.d), perm, w.n_pad)
    return perm, qp, kp, vp


def check_rows(w, q, k, v, mask, rows=None):
    out, out_p, lse = run_gpu_path(w, q, k, v, mask)
    BH = w.B * w.H
    perm, qp, kp, vp = oracle_inputs(w, q, k, v)
    ref_out, ref_lse = oracle.attention(qp, kp, vp, mask.reshape(BH, w.nb, w.nb), w.n, w.block,
                                        rows=rows)
    gpu_out_p = out_p.float().numpy().reshape(BH * w.n_pad, w.d)
    gpu_lse = lse.numpy().reshape(BH * w.n_pad)
    sel = np.arange(BH * w.n_pad) if rows is None else rows
    mx, mean, lse_err = compare_out(gpu_out_p[sel], ref_out, gpu_lse[sel], ref_lse)
    assert mx <= OUT_MAX_ABS, f"max abs {mx}"
    assert mean <= OUT_MEAN_ABS, f"mean abs {mean}"
    assert lse_err <= LSE_ABS, f"lse {lse_err}"
    # frame-major output after unpermute: row perm[p] of head bh is row p of the oracle
    bh, p = np.divmod(sel, w.n_pad)
    valid = p < w.n
    gpu_frame = out.float().numpy().reshape(BH, w.n, w.d)[bh[valid], perm[p[valid]]]
    diff = np.abs(gpu_frame - ref_out[valid])
    assert (diff.max() if diff.size else 0.0) <= OUT_MAX_ABS
    # pad rows: zero output and lse = -inf
    pad = ~valid
    if pad.any():
        assert np.all(gpu_out_p[sel[pad]] == 0)
        assert np.all(np.isneginf(gpu_lse[sel[pad]]))
    return mx, mean, lse_err


SMALL = [
    # name, B, H, d, T, Hs, Ws, tt, th, tw, block, seed, mask kind
    ("tiny", None),
    ("d128_b128_ragged", I.custom_workload("d128_b128_ragged", 1, 2, 128, 3, 30, 52, 1, 8, 16,
                                           128, 11, "bernoulli_half")),
    ("d64_b128", I.custom_workload("d64_b128", 1, 3, 64, 2, 20, 24, 1, 8, 8, 128, 12,
                                   "bernoulli_half")),
    ("d128_b64_odd_nb", I.custom_workload("d128_b64_odd_nb", 1, 2, 128, 3, 10, 19, 1, 4, 16, 64,
                                          13, "bernoulli_half")),
    ("d128_b128_ones", I.custom_workload("d128_b128_ones", 2, 1, 128, 2, 16, 40, 1, 8, 16, 128,
                                         14, "ones")),
    ("d128_b128_empty_rows", I.custom_workload("d128_b128_empty_rows", 1, 3, 128, 4, 24, 30, 1,
                                               8, 16, 128, 15, "bernoulli_sparse")),
    ("band_stripe_small", I.custom_workload("band_stripe_small", 1, 3, 128, 5, 30, 52, 1, 8, 16,
                                            128, 16, "band_stripe")),
    # 64-token blocks, 8 heads x 32 tiles of two blocks: more tiles than SMs, so every
    # CTA takes tiles from its schedule-ordered list over two rounds
    ("d64_b64_two_rounds", I.custom_workload("d64_b64_two_rounds", 1, 8, 64, 4, 32, 32, 1, 8, 8,
                                             64, 18, "bernoulli_half")),
]


@pytest.mark.parametrize("name,w", SMALL, ids=[s[0] for s in SMALL])
def test_forward_small_all_rows(cuda_ok, name, w):
    w = I.WORKLOADS["tiny"] if w is None else w
    q, k, v = I.gen_qkv(w)
    mask = I.gen_mask(w, q, k)
    check_rows(w, q, k, v, mask)


def test_forward_large_values_and_scale(cuda_ok):
    # outlier keys at 5x and a custom scale exercise the online rescale path
    import block_sparse_attention_forward_b200 as bsa
    w = I.custom_workload("outliers", 1, 2, 128, 2, 16, 32, 1, 8, 16, 128, 17, "bernoulli_half")
    q, k, v = I.gen_qkv(w)
    k = (k.float() * 3.0).to(torch.bfloat16)
    mask = I.gen_mask(w)
    grid, tile = (w.T, w.Hs, w.Ws), (w.tt, w.th, w.tw)
    qp = bsa.tile_permute(q.cuda(), grid, tile, w.n_pad)
    kp = bsa.tile_permute(k.cuda(), grid, tile, w.n_pad)
    vp = bsa.tile_permute(v.cuda(), grid, tile, w.n_pad)
    pm = bsa.pack_mask(torch.from_numpy(mask).cuda())
    out_p, lse = bsa.forward(qp, kp, vp, pm, w.n, w.block, softmax_scale=0.3)
    torch.cuda.synchronize()
    BH = w.B * w.H
    _, qo, ko, vo = oracle_inputs(w, q, k, v)
    ref_out, ref_lse = oracle.attention(qo, ko, vo, mask.reshape(BH, w.nb, w.nb), w.n, w.block,
                                        scale=0.3)
    mx, mean, lse_err = compare_out(out_p.float().cpu().numpy().reshape(-1, w.d), ref_out,
                                    lse.cpu().numpy().reshape(-1), ref_lse)
    assert mx <= OUT_MAX_ABS and mean <= OUT_MEAN_ABS and lse_err <= LSE_ABS


@pytest.mark.parametrize("name", ["wan13b_480p", "wan14b_480p", "wan14b_720p", "hunyuan_768p"])
def test_forward_full_size_sampled(cuda_ok, name):
    w = I.WORKLOADS[name]
    q, k, v = I.gen_qkv(w)
    mask = I.gen_mask(w, q, k)
    BH = w.B * w.H
    picks = stratified_query_blocks(mask, per_head=4, seed=w.seed)
    rng = np.random.default_rng(w.seed)
    heads = sorted(set(rng.choice(BH, size=min(BH, 10), replace=False).tolist()) |
                   {0, BH - 1})
    picks = [(bh, qb) for bh, qb in picks if bh in heads]
    rows = np.concatenate([bh * w.n_pad + qb * w.block + np.arange(w.block) for bh, qb in picks])
    check_rows(w, q, k, v, mask, rows=rows.astype(np.int64))
