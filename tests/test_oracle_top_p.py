"""Pins for the oracle's online top-p block mask (pooled-query/key block scores,
row softmax, smallest descending-probability prefix whose cumulative share
reaches top_p, ties to the lower block; "ScalingAttention" Algorithm 1's
sort-and-accumulate cut applied per row with a per-head top_p).

Checked against closed forms and library routines, not by re-typing:
- equal scores: exactly ceil(top_p * nb) blocks, the lowest-indexed;
- a dominant block alone when its share reaches top_p;
- pooled means exclude pad tokens (garbage in the pad changes nothing);
- probabilities equal scipy's softmax of numpy block means and matmul;
- the kept set is the shortest prefix of numpy's stable descending sort;
- per-head tau and top_p are taken from that head.
"""
import numpy as np
import pytest
import torch
from scipy.special import softmax

import oracle


def _bits(x: torch.Tensor) -> np.ndarray:
    return x.contiguous().view(torch.int16).numpy().view(np.uint16)


def _rand(BH, n_pad, d, seed, scale=1.0):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn((BH, n_pad, d), generator=g) * scale).to(torch.bfloat16)


@pytest.mark.parametrize("nb,top_p,want", [(8, 0.5, 4), (8, 0.51, 5), (8, 1.0, 8), (8, 0.01, 1),
                                           (10, 0.35, 4), (16, 0.9, 15)])
def test_equal_scores_keep_lowest_ceil(nb, top_p, want):
    block, d = 4, 8
    q = torch.zeros((1, nb * block, d), dtype=torch.bfloat16)
    k = _rand(1, nb * block, d, 1)
    m = oracle.top_p_mask(_bits(q), _bits(k), 1, nb * block, block, [1.0], [top_p])
    for i in range(nb):
        assert m[0, i].tolist() == [1] * want + [0] * (nb - want), (i, m[0, i])


def test_dominant_block_alone():
    nb, block, d = 6, 4, 8
    q = torch.ones((1, nb * block, d), dtype=torch.bfloat16)
    k = torch.zeros((1, nb * block, d), dtype=torch.bfloat16)
    k[0, 3 * block:4 * block] = 4.0  # block 3: score 32/sqrt(8) over the rest at 0
    m, p = oracle.top_p_mask(_bits(q), _bits(k), 1, nb * block, block, [1.0], [0.9],
                             with_prob=True)
    assert p[0, 0, 3] > 0.99
    assert np.all(m[0] == np.eye(nb, dtype=np.uint8)[3])


def test_pad_tokens_do_not_count():
    n_valid, block, d = 50, 8, 16  # nb = 7, last block has 2 valid tokens
    q = _rand(2, 56, d, 2)
    k = _rand(2, 56, d, 3)
    q2, k2 = q.clone(), k.clone()
    q2[:, n_valid:] = 1e4
    k2[:, n_valid:] = -1e4
    a = oracle.top_p_mask(_bits(q), _bits(k), 2, n_valid, block, [0.05, 0.1], [0.7, 0.5])
    b = oracle.top_p_mask(_bits(q2), _bits(k2), 2, n_valid, block, [0.05, 0.1], [0.7, 0.5])
    assert np.array_equal(a, b)


def _reference_prob(q, k, n_valid, block, tau):
    """numpy block means over valid tokens, matmul, scipy softmax."""
    qf = q.float().numpy().astype(np.float64)
    kf = k.float().numpy().astype(np.float64)
    n_pad, d = qf.shape
    nb = n_pad // block
    cnt = np.array([min(block, n_valid - i * block) for i in range(nb)], dtype=np.float64)

    def means(x):
        return np.stack([x[i * block:i * block + int(cnt[i])].mean(axis=0) for i in range(nb)])
    s = means(qf) @ means(kf).T / (np.sqrt(d) * tau)
    return softmax(s, axis=1)


def test_probabilities_and_prefix_against_numpy():
    H, n_valid, n_pad, block, d = 3, 190, 192, 16, 32
    q = _rand(H, n_pad, d, 4, 3.0)
    k = _rand(H, n_pad, d, 5, 3.0)
    tau = np.array([0.02, 0.05, 0.3])
    top_p = np.array([0.9, 0.6, 0.95])
    m, p = oracle.top_p_mask(_bits(q), _bits(k), H, n_valid, block, tau, top_p, with_prob=True)
    for h in range(H):
        ref = _reference_prob(q[h], k[h], n_valid, block, tau[h])
        np.testing.assert_allclose(p[h], ref, rtol=1e-12, atol=1e-15)
        for i in range(ref.shape[0]):
            order = np.argsort(-ref[i], kind="stable")
            cum = np.cumsum(ref[i][order])
            n_keep = int(np.searchsorted(cum, top_p[h] - 1e-12)) + 1
            want = np.zeros(ref.shape[1], dtype=np.uint8)
            want[order[:min(n_keep, len(order))]] = 1
            assert np.array_equal(m[h, i], want), (h, i)


def test_per_head_parameters_and_monotone_top_p():
    H, n_pad, block, d = 2, 128, 16, 16
    q = _rand(H, n_pad, d, 6, 3.0)
    k = _rand(H, n_pad, d, 7, 3.0)
    a = oracle.top_p_mask(_bits(q), _bits(k), H, n_pad, block, [0.02, 0.2], [0.5, 0.9])
    # head h alone, with head h's parameters, gives the same rows
    for h, (t, p) in enumerate([(0.02, 0.5), (0.2, 0.9)]):
        solo = oracle.top_p_mask(_bits(q[h:h + 1]), _bits(k[h:h + 1]), 1, n_pad, block, [t], [p])
        assert np.array_equal(a[h], solo[0])
    prev = None
    for p in (0.3, 0.5, 0.8, 0.99):
        m = oracle.top_p_mask(_bits(q), _bits(k), H, n_pad, block, [0.05, 0.05], [p, p])
        if prev is not None:
            assert np.all(m >= prev)
        prev = m
