"""GPU parity of the forward with 128-token query blocks over 64-token key
blocks (bsa_forward_blocks: finer key granularity, "ScalingAttention" Sec. 5.4's
granularity bottleneck) against the fp64 oracle with the same two block sizes.

Masks come from inputs.gen_mask_fine: the workload's mask with each kept key
block split in halves and 30 % of the halves dropped.  Small cases on every
row (ragged tails, d = 64, empty rows), the full-size workloads on stratified
query blocks.  Tolerances as for the forward: out max-abs 2e-2, mean-abs 2e-3,
lse 1e-3; -inf rows exact; pad rows zero."""
import numpy as np
import pytest
import torch

import oracle
from block_sparse_attention_forward_b200 import inputs as I
from tests.helpers import (LSE_ABS, OUT_MAX_ABS, OUT_MEAN_ABS, bf16_bits, compare_out,
                           stratified_query_blocks)

pytestmark = pytest.mark.gpu


def _check(w, q, k, v, mask, rows=None):
    import block_sparse_attention_forward_b200 as bsa
    grid, tile = (w.T, w.Hs, w.Ws), (w.tt, w.th, w.tw)
    qp = bsa.tile_permute(q.cuda(), grid, tile, w.n_pad)
    kp = bsa.tile_permute(k.cuda(), grid, tile, w.n_pad)
    vp = bsa.tile_permute(v.cuda(), grid, tile, w.n_pad)
    pm = bsa.pack_mask(torch.from_numpy(mask).cuda())
    out_p, lse = bsa.forward(qp, kp, vp, pm, w.n, w.block, block_k=w.block // 2)
    torch.cuda.synchronize()
    assert bsa.device_error() == 0
    BH = w.B * w.H
    perm = oracle.tile_order(w.T, w.Hs, w.Ws, w.tt, w.th, w.tw)
    qo, ko, vo = (oracle.permute(bf16_bits(t).reshape(BH, w.n, w.d), perm, w.n_pad)
                  for t in (q, k, v))
    ref, ref_lse = oracle.attention(qo, ko, vo, mask.reshape(BH, w.nb, 2 * w.nb), w.n, w.block,
                                    rows=rows, block_k=w.block // 2)
    gpu = out_p.float().cpu().numpy().reshape(BH * w.n_pad, w.d)
    gl = lse.cpu().numpy().reshape(BH * w.n_pad)
    sel = np.arange(BH * w.n_pad) if rows is None else rows
    mx, mean, lse_err = compare_out(gpu[sel], ref, gl[sel], ref_lse)
    assert mx <= OUT_MAX_ABS and mean <= OUT_MEAN_ABS and lse_err <= LSE_ABS, (mx, mean, lse_err)
    pad = (sel % w.n_pad) >= w.n
    if pad.any():
        assert np.all(gpu[sel[pad]] == 0) and np.all(np.isneginf(gl[sel[pad]]))


SMALL = [
    # n_pad - n < 64 in every case: only the last 64-key block holds pad
    I.custom_workload("fk_d128_ragged", 1, 2, 128, 3, 30, 52, 1, 8, 16, 128, 21, "bernoulli_half"),
    I.custom_workload("fk_d64", 1, 3, 64, 2, 16, 31, 1, 8, 8, 128, 22, "bernoulli_half"),
    I.custom_workload("fk_exact", 2, 1, 128, 2, 16, 32, 1, 8, 16, 128, 23, "band_stripe"),
    I.custom_workload("fk_empty_rows", 1, 2, 128, 4, 24, 29, 1, 8, 16, 128, 24,
                      "bernoulli_sparse"),
]


@pytest.mark.parametrize("w", SMALL, ids=[w.name for w in SMALL])
def test_finer_keys_small_all_rows(cuda_ok, w):
    assert w.n_pad - w.n < w.block // 2
    q, k, v = I.gen_qkv(w)
    mask = I.gen_mask_fine(w, q, k)
    if w.mask_kind == "bernoulli_sparse":  # rows with no kept half at all
        mask[:, :, 1::3] = 0
    _check(w, q, k, v, mask)


@pytest.mark.parametrize("name", ["wan13b_480p", "wan14b_720p", "hunyuan_768p"])
def test_finer_keys_full_size_sampled(cuda_ok, name):
    w = I.WORKLOADS[name]
    q, k, v = I.gen_qkv(w)
    mask = I.gen_mask_fine(w, q, k)
    BH = w.B * w.H
    picks = stratified_query_blocks(mask, per_head=4, seed=w.seed)
    rng = np.random.default_rng(w.seed)
    heads = sorted(set(rng.choice(BH, size=min(BH, 8), replace=False).tolist()) | {0, BH - 1})
    picks = [(bh, qb) for bh, qb in picks if bh in heads]
    rows = np.concatenate([bh * w.n_pad + qb * w.block + np.arange(w.block) for bh, qb in picks])
    _check(w, q, k, v, mask, rows=rows.astype(np.int64))


def test_refined_mask_matches_coarse_forward(cuda_ok):
    # a 128-granular mask written at 64-key granularity: same math, so the two
    # kernels agree to within bf16 rounding of P (different tile sizes)
    import block_sparse_attention_forward_b200 as bsa
    w = SMALL[0]
    q, k, v = I.gen_qkv(w)
    coarse = I.gen_mask(w, q, k)
    grid, tile = (w.T, w.Hs, w.Ws), (w.tt, w.th, w.tw)
    qp, kp, vp = (bsa.tile_permute(t.cuda(), grid, tile, w.n_pad) for t in (q, k, v))
    a, la = bsa.forward(qp, kp, vp, bsa.pack_mask(torch.from_numpy(coarse).cuda()), w.n, w.block)
    fine = np.repeat(coarse, 2, axis=3)
    b, lb = bsa.forward(qp, kp, vp, bsa.pack_mask(torch.from_numpy(fine).cuda()), w.n, w.block,
                        block_k=w.block // 2)
    torch.cuda.synchronize()
    assert (a.float() - b.float()).abs().max().item() <= OUT_MAX_ABS
    fin = torch.isfinite(la)
    assert torch.equal(fin, torch.isfinite(lb))
    assert (la[fin] - lb[fin]).abs().max().item() <= LSE_ABS
