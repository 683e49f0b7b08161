"""GPU parity of bsa_predict_top_p (online top-p block mask) against the oracle.

The mask is a floating-point decision: the GPU takes it in fp32 (means, FMA
scores, expf, fp32 cumulative comparison), the oracle in fp64.  Where the
decision is clear -- the oracle's cumulative share at the cut is more than
DELTA_SUM away from top_p on both sides, and the last kept and first dropped
probabilities differ by more than DELTA_P relative -- the GPU row must equal
the oracle's.  Elsewhere several rows are correct, so the GPU row is checked
for validity against the oracle's fp64 probabilities: kept blocks are at least
as probable as dropped ones (within DELTA_P relative), the kept share reaches
top_p and dropping the least probable kept block would not (within
DELTA_SUM).  DELTA_P = 1e-5 covers fp32 rounding of the means, scores and
exponentials; DELTA_SUM = 2e-5 covers fp32 sums of up to a thousand terms.
Most rows must match the oracle exactly.  The CRM words, counts, offsets,
lists and schedule that come with the GPU's mask must equal the oracle's
packing of that same mask."""
import dataclasses

import numpy as np
import pytest
import torch

import oracle
from block_sparse_attention_forward_b200 import inputs as I
from tests.helpers import bf16_bits, check_schedule

pytestmark = pytest.mark.gpu

DELTA_P = 1e-5    # relative, on probabilities
DELTA_SUM = 2e-5  # absolute, on cumulative shares


def _unpack(bits_words: np.ndarray, nb: int) -> np.ndarray:
    w = bits_words.view(np.uint32)
    j = np.arange(nb)
    return ((w[..., j // 32] >> (j % 32).astype(np.uint32)) & 1).astype(np.uint8)


def _check_rows(gpu_mask, ora_mask, prob, top_p_h):
    """Per row: exact where the oracle's decision is clear, else valid.
    Returns (rows equal to the oracle's, rows checked)."""
    equal = 0
    for i in range(prob.shape[0]):
        p = prob[i]
        g = gpu_mask[i].astype(bool)
        o = ora_mask[i].astype(bool)
        equal += int(np.array_equal(g, o))
        order = np.argsort(-p, kind="stable")
        cum = np.cumsum(p[order])
        n_keep = int(o.sum())
        clear = True
        if n_keep < len(p):
            before = cum[n_keep - 2] if n_keep >= 2 else 0.0
            last, nxt = p[order[n_keep - 1]], p[order[n_keep]]
            clear = (cum[n_keep - 1] - top_p_h > DELTA_SUM and top_p_h - before > DELTA_SUM
                     and last - nxt > DELTA_P * last)
        if clear:
            assert np.array_equal(g, o), i
            continue
        assert g.any(), i
        kept_p, drop_p = p[g], p[~g]
        if drop_p.size:
            assert kept_p.min() >= drop_p.max() * (1 - DELTA_P), i
            assert kept_p.sum() >= top_p_h - DELTA_SUM, i
        assert kept_p.sum() - kept_p.min() < top_p_h + DELTA_SUM, i
    return equal, prob.shape[0]


def _run(w, heads=None):
    import block_sparse_attention_forward_b200 as bsa
    if heads is not None:
        w = dataclasses.replace(w, H=heads)
    q, k, _ = I.gen_qkv(w)
    tau, top_p = I.gen_top_p_params(w)
    grid, tile = (w.T, w.Hs, w.Ws), (w.tt, w.th, w.tw)
    qp = bsa.tile_permute(q.cuda(), grid, tile, w.n_pad)
    kp = bsa.tile_permute(k.cuda(), grid, tile, w.n_pad)
    pm = bsa.predict_top_p(qp, kp, w.n, w.block, torch.from_numpy(tau).cuda(),
                           torch.from_numpy(top_p).cuda())
    torch.cuda.synchronize()
    BH = w.B * w.H
    ora, prob = oracle.top_p_mask(bf16_bits(qp).reshape(BH, w.n_pad, w.d),
                                  bf16_bits(kp).reshape(BH, w.n_pad, w.d), w.H, w.n, w.block,
                                  tau.astype(np.float64), top_p.astype(np.float64),
                                  with_prob=True)
    gpu = _unpack(pm.bits.cpu().numpy(), w.nb).reshape(BH, w.nb, w.nb)
    equal = checked = 0
    for bh in range(BH):
        e, c = _check_rows(gpu[bh], ora[bh], prob[bh], float(np.float64(top_p[bh % w.H])))
        equal += e
        checked += c
    # the packing of the GPU's own mask is integer work: exact
    bits_ref = oracle.pack_bits(gpu)
    counts_ref, offsets_ref, cols_ref = oracle.crm_lists(bits_ref)
    np.testing.assert_array_equal(pm.bits.cpu().numpy().view(np.uint32), bits_ref.reshape(pm.bits.shape))
    np.testing.assert_array_equal(pm.counts.cpu().numpy(), counts_ref)
    np.testing.assert_array_equal(pm.row_offsets.cpu().numpy().astype(np.int64), offsets_ref)
    total = int(offsets_ref[-1])
    np.testing.assert_array_equal(pm.col_idx[:total].cpu().numpy(), cols_ref)
    check_schedule(pm.schedule.cpu().numpy(), counts_ref, pm.nb_q, pm.nb_k)
    return equal, checked, gpu.mean()


@pytest.mark.parametrize("name,heads", [("tiny", None), ("wan13b_480p", 3), ("wan14b_720p", 2),
                                        ("hunyuan_768p", 2)])
def test_predict_top_p_matches_oracle(cuda_ok, name, heads):
    equal, checked, density = _run(I.WORKLOADS[name], heads)
    assert equal >= 0.9 * checked, (equal, checked)
    assert 0.02 < density < 0.98


# Tile edges of the tensor-core score kernel (128 query x 64 key blocks per
# CTA): several batches and heads whose tiles straddle head boundaries, a key
# count that is not a multiple of 64, d = 64 (two 32-dimension stages), and
# two query tiles over three key tiles with a ragged last one at d = 128.
@pytest.mark.parametrize("w", [
    I.custom_workload("pred_b2_d64_ragged", 2, 3, 64, 5, 24, 40, 1, 8, 8, 64, 31, "bernoulli_half"),
    I.custom_workload("pred_d128_two_row_tiles", 1, 2, 128, 9, 48, 48, 1, 8, 16, 128, 32,
                      "bernoulli_half"),
], ids=lambda w: w.name)
def test_predict_top_p_tile_edges(cuda_ok, w):
    equal, checked, density = _run(w)
    assert equal >= 0.9 * checked, (equal, checked)
    assert 0.02 < density < 0.98


def test_predict_top_p_edge_parameters(cuda_ok):
    # top_p = 1 keeps everything reachable, a tiny top_p keeps one block per
    # row, a huge temperature makes rows uniform (ceil(top_p * nb) lowest blocks)
    import block_sparse_attention_forward_b200 as bsa
    w = I.WORKLOADS["tiny"]
    q, k, _ = I.gen_qkv(w)
    grid, tile = (w.T, w.Hs, w.Ws), (w.tt, w.th, w.tw)
    qp = bsa.tile_permute(q.cuda(), grid, tile, w.n_pad)
    kp = bsa.tile_permute(k.cuda(), grid, tile, w.n_pad)
    tau = torch.tensor([0.01, 1e6], device="cuda")
    for top_p, want0, want1 in ((1.0, None, w.nb), (1e-6, 1, 1), (0.5, None, w.nb // 2)):
        pm = bsa.predict_top_p(qp, kp, w.n, w.block, tau,
                               torch.tensor([top_p, top_p], device="cuda"))
        counts = pm.counts.cpu().numpy().reshape(w.H, w.nb)
        if want0 is not None:
            assert np.all(counts[0] == want0)
        assert np.all(counts[1] >= want1 - 1) and np.all(counts[1] <= want1 + 1)
        assert np.all(counts >= 1)
