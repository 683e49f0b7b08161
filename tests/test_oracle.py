"""Pins for the fp64 CPU oracle: it is checked against what the pages and the
mathematics fix, never against itself or against the CUDA path.

Pins used (pages: "ScalingAttention", Sec. 4.3.2 and Appendix E, Algorithm 2):
- the worked CRM size (256k tokens, block 128 -> 64 words per row), a golden fixture;
- Algorithm 2's bit order and iteration against a naive scan of the dense mask;
- textbook attention (torch's scaled_dot_product_attention in fp64) for an all-ones mask,
  a single kept block, and the tail of valid keys;
- closed forms of a hand-worked 4-token example;
- invariants: rows of P sum to one, key/value permutation inside a kept block,
  permute/unpermute round trip, pad rows.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def bf16_bits(x: torch.Tensor) -> np.ndarray:
    return x.to(torch.bfloat16).contiguous().view(torch.int16).numpy().view(np.uint16)


def bits_to_f64(b: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(b.view(np.int16).copy()).view(torch.bfloat16).double()


# ---------------------------------------------------------------- CRM packing
def test_crm_words_worked_example():
    with open(os.path.join(GOLDEN, "crm_words_256k.json")) as f:
        g = json.load(f)
    nb = g["tokens"] // g["block"]
    assert oracle.crm_words(nb) == g["words_per_row"]


@pytest.mark.parametrize("nb_k", [1, 31, 32, 33, 64, 65, 591, 990])
def test_iterator_matches_naive_scan(nb_k):
    rng = np.random.default_rng(nb_k)
    for density in (0.0, 0.03, 0.5, 1.0):
        dense = (rng.random((7, nb_k)) < density).astype(np.uint8)
        dense[3, :] = 0  # an empty row
        dense[4, -1] = 1  # last block
        bits = oracle.pack_bits(dense)
        assert bits.shape == (7, (nb_k + 31) // 32)
        counts, offsets, col_idx = oracle.crm_lists(bits)
        for r in range(7):
            expect = np.nonzero(dense[r])[0]
            got = col_idx[offsets[r]:offsets[r + 1]]
            np.testing.assert_array_equal(got, expect)
            assert counts[r] == expect.size
        np.testing.assert_array_equal(offsets[1:] - offsets[:-1], counts)


def test_bit_order_single_blocks():
    # Algorithm 2: index = base + CTZ(word), base grows by 32 per word -> bit j of word w
    # is key block 32 w + j; unused high bits stay zero.
    nb_k = 70
    for j in range(nb_k):
        dense = np.zeros((1, nb_k), dtype=np.uint8)
        dense[0, j] = 1
        bits = oracle.pack_bits(dense)[0]
        expect = np.zeros(3, dtype=np.uint32)
        expect[j // 32] = np.uint32(1) << np.uint32(j % 32)
        np.testing.assert_array_equal(bits, expect)
    bits = oracle.pack_bits(np.ones((1, nb_k), dtype=np.uint8))[0]
    assert bits[2] == (1 << 6) - 1


def test_nonzero_bytes_count_as_kept():
    dense = np.array([[0, 2, 255, 0, 1]], dtype=np.uint8)
    bits = oracle.pack_bits(dense)
    assert bits[0, 0] == 0b10110


def test_schedule_is_stable_count_descending():
    rng = np.random.default_rng(5)
    counts = rng.integers(0, 9, size=500).astype(np.int32)
    sched = oracle.schedule(counts)
    expect = sorted(range(counts.size), key=lambda r: (-int(counts[r]), r))
    np.testing.assert_array_equal(sched, np.array(expect, dtype=np.int32))


def test_schedule_ties_keep_row_order_and_all_rows_appear():
    # all counts equal: the identity; strictly increasing counts: the reverse
    n = 300
    np.testing.assert_array_equal(oracle.schedule(np.full(n, 3, np.int32)), np.arange(n))
    np.testing.assert_array_equal(oracle.schedule(np.arange(n, dtype=np.int32)),
                                  np.arange(n)[::-1])
    rng = np.random.default_rng(9)
    counts = rng.integers(0, 5, size=1000).astype(np.int32)
    sched = oracle.schedule(counts)
    assert np.array_equal(np.sort(sched), np.arange(counts.size))
    assert np.all(np.diff(counts[sched]) <= 0)


@pytest.mark.parametrize("heads,form", [(8, "count"), (9, "head")])
def test_library_schedule_policy_boundary(heads, form):
    # the library's work-order policy (stated in tests/helpers.py, not part of
    # the oracle): row i of every head keeps 200 - i blocks, so each window of
    # 148 count-order entries holds every head.  With L2 sized for 8.5 heads'
    # K and V, 8 heads per window keep the count order and 9 turn head-major
    from tests.helpers import (POLICY_KEY_BLOCK_BYTES, head_major_order, policy_form,
                               schedule_form)
    nb_q, nb_k = 148, 240
    l2 = int(8.5 * nb_k * POLICY_KEY_BLOCK_BYTES)
    counts = np.tile(200 - np.arange(nb_q), heads).astype(np.int32)
    assert policy_form(counts, nb_q, nb_k, l2) == form
    assert schedule_form(head_major_order(counts, nb_q), counts, nb_q) == "head"
    assert schedule_form(oracle.schedule(counts), counts, nb_q) == "count"
    assert policy_form(counts[: 147], nb_q, nb_k, l2) == "count"  # no full window

def test_tile_order_divisible_matches_reshape():
    T, Hs, Ws, tt, th, tw = 4, 16, 16, 2, 8, 4
    perm = oracle.tile_order(T, Hs, Ws, tt, th, tw)
    ref = np.arange(T * Hs * Ws).reshape(T // tt, tt, Hs // th, th, Ws // tw, tw)
    ref = ref.transpose(0, 2, 4, 1, 3, 5).reshape(-1)
    np.testing.assert_array_equal(perm, ref)


def test_tile_order_ragged_hand_example():
    # 1x3x3 grid, 1x2x2 tiles: tiles (0,0) (0,1) (1,0) (1,1) with clipped extents
    perm = oracle.tile_order(1, 3, 3, 1, 2, 2)
    np.testing.assert_array_equal(perm, [0, 1, 3, 4, 2, 5, 6, 7, 8])


@pytest.mark.parametrize("grid,tile", [((21, 30, 52), (1, 8, 16)), ((21, 45, 80), (2, 8, 8)),
                                       ((5, 7, 9), (2, 3, 4))])
def test_tile_order_ragged_is_bijection_with_contiguous_tiles(grid, tile):
    T, Hs, Ws = grid
    tt, th, tw = tile
    perm = oracle.tile_order(T, Hs, Ws, tt, th, tw)
    assert np.array_equal(np.sort(perm), np.arange(T * Hs * Ws))
    t, rem = np.divmod(perm, Hs * Ws)
    y, x = np.divmod(rem, Ws)
    tile_id = ((t // tt) * (-(-Hs // th)) + (y // th)) * (-(-Ws // tw)) + (x // tw)
    # tiles appear in row-major order, each as one contiguous run
    assert np.all(np.diff(tile_id) >= 0)
    # inside a tile, tokens are (t, y, x) row-major
    key = (t * Hs + y) * Ws + x
    same = np.diff(tile_id) == 0
    assert np.all(np.diff(key)[same] > 0)


def test_permute_roundtrip_and_pad():
    rng = np.random.default_rng(1)
    T, Hs, Ws, tt, th, tw, d = 3, 5, 7, 2, 2, 4, 8
    n = T * Hs * Ws
    n_pad = 128
    x = rng.integers(0, 65535, size=(2, n, d), dtype=np.uint16)
    perm = oracle.tile_order(T, Hs, Ws, tt, th, tw)
    y = oracle.permute(x, perm, n_pad)
    assert np.all(y[:, n:] == 0)
    np.testing.assert_array_equal(y[:, :n], x[:, perm])
    np.testing.assert_array_equal(oracle.unpermute(y, perm, n), x)


# ---------------------------------------------------------------- attention
def make_case(BH, n_valid, n_pad, d, seed, scale_qk=1.0):
    g = torch.Generator().manual_seed(seed)
    q = torch.randn(BH, n_pad, d, generator=g) * scale_qk
    k = torch.randn(BH, n_pad, d, generator=g) * scale_qk
    v = torch.randn(BH, n_pad, d, generator=g)
    for t in (q, k, v):
        t[:, n_valid:] = 0
    return bf16_bits(q), bf16_bits(k), bf16_bits(v)


def sdpa(qb, kb, vb, keep=None, scale=None):
    """Textbook softmax attention in fp64 via torch (library routine)."""
    q, k, v = bits_to_f64(qb), bits_to_f64(kb), bits_to_f64(vb)
    d = q.shape[-1]
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    logits = scale * (q @ k.transpose(-1, -2))
    if keep is not None:
        logits = logits.masked_fill(~keep, float("-inf"))
    out = torch.nn.functional.scaled_dot_product_attention(q, k, v, attn_mask=keep, scale=scale)
    return out.numpy(), torch.logsumexp(logits, dim=-1).numpy()


@pytest.mark.parametrize("dense_literal", [True, False])
def test_all_ones_mask_is_full_attention(dense_literal):
    BH, n, block, d = 2, 192, 64, 32
    qb, kb, vb = make_case(BH, n, n, d, seed=3)
    mask = np.ones((BH, n // block, n // block), dtype=np.uint8)
    out, lse = oracle.attention(qb, kb, vb, mask, n, block, dense_literal=dense_literal)
    ref, ref_lse = sdpa(qb, kb, vb)
    np.testing.assert_allclose(out.reshape(BH, n, d), ref, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse.reshape(BH, n), ref_lse, rtol=0, atol=1e-12)


def test_single_kept_block_row_is_attention_over_that_block():
    BH, n, block, d = 1, 256, 64, 16
    qb, kb, vb = make_case(BH, n, n, d, seed=4)
    nb = n // block
    mask = np.zeros((BH, nb, nb), dtype=np.uint8)
    mask[0, 1, 2] = 1  # query block 1 keeps only key block 2
    rows = np.arange(block, 2 * block)
    out, lse = oracle.attention(qb, kb, vb, mask, n, block, rows=rows)
    sl = slice(2 * block, 3 * block)
    ref, ref_lse = sdpa(qb[:, rows], kb[:, sl], vb[:, sl])
    np.testing.assert_allclose(out, ref[0], rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, ref_lse[0], rtol=0, atol=1e-12)


def test_block_mask_matches_token_mask_sdpa_with_tail():
    BH, n_valid, n_pad, block, d = 2, 300, 320, 64, 32
    qb, kb, vb = make_case(BH, n_valid, n_pad, d, seed=6)
    nb = n_pad // block
    rng = np.random.default_rng(6)
    mask = (rng.random((BH, nb, nb)) < 0.5).astype(np.uint8)
    mask[:, np.arange(nb), np.arange(nb)] = 1
    out, lse = oracle.attention(qb, kb, vb, mask, n_valid, block)
    out = out.reshape(BH, n_pad, d)
    lse = lse.reshape(BH, n_pad)
    tok = np.arange(n_valid) // block
    keep = torch.from_numpy(mask[:, tok][:, :, tok].astype(bool))
    ref, ref_lse = sdpa(qb[:, :n_valid], kb[:, :n_valid], vb[:, :n_valid], keep=keep)
    np.testing.assert_allclose(out[:, :n_valid], ref, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse[:, :n_valid], ref_lse, rtol=0, atol=1e-12)
    # pad query rows: zero output, lse = -inf
    assert np.all(out[:, n_valid:] == 0)
    assert np.all(np.isneginf(lse[:, n_valid:]))


def test_dense_literal_equals_block_skip():
    BH, n, block, d = 3, 256, 64, 16
    qb, kb, vb = make_case(BH, n, n, d, seed=7)
    rng = np.random.default_rng(7)
    mask = (rng.random((BH, 4, 4)) < 0.4).astype(np.uint8)
    a = oracle.attention(qb, kb, vb, mask, n, block, dense_literal=True)
    b = oracle.attention(qb, kb, vb, mask, n, block, dense_literal=False)
    np.testing.assert_allclose(a[0], b[0], rtol=0, atol=1e-13)
    np.testing.assert_allclose(a[1], b[1], rtol=0, atol=1e-13)


def test_rows_of_p_sum_to_one():
    BH, n, block, d = 2, 256, 64, 16
    qb, kb, _ = make_case(BH, n, n, d, seed=8)
    vb = bf16_bits(torch.ones(BH, n, d))
    rng = np.random.default_rng(8)
    mask = (rng.random((BH, 4, 4)) < 0.5).astype(np.uint8)
    mask[:, np.arange(4), np.arange(4)] = 1
    out, _ = oracle.attention(qb, kb, vb, mask, n, block)
    np.testing.assert_allclose(out, 1.0, rtol=0, atol=1e-12)


def test_key_value_permutation_inside_kept_block():
    BH, n, block, d = 1, 256, 64, 16
    qb, kb, vb = make_case(BH, n, n, d, seed=9)
    mask = np.zeros((BH, 4, 4), dtype=np.uint8)
    mask[0, :, 1] = 1
    mask[0, :, 3] = 1
    a = oracle.attention(qb, kb, vb, mask, n, block)
    p = np.random.default_rng(9).permutation(block) + block  # shuffle keys of block 1
    kb2, vb2 = kb.copy(), vb.copy()
    kb2[:, block:2 * block] = kb[:, p]
    vb2[:, block:2 * block] = vb[:, p]
    b = oracle.attention(qb, kb2, vb2, mask, n, block)
    np.testing.assert_allclose(a[0], b[0], rtol=0, atol=1e-12)
    np.testing.assert_allclose(a[1], b[1], rtol=0, atol=1e-12)


def test_hand_worked_two_block_example():
    q = torch.tensor([[1, 0], [0, 1], [1, 1], [0, 0]], dtype=torch.float32)[None]
    k = torch.tensor([[1, 0], [0, 1], [1, 1], [-1, 0]], dtype=torch.float32)[None]
    v = torch.tensor([[1, 0], [0, 1], [2, 0], [0, 2]], dtype=torch.float32)[None]
    mask = np.array([[[1, 0], [1, 1]]], dtype=np.uint8)  # block 0 keeps {0}; block 1 keeps {0, 1}
    out, lse = oracle.attention(bf16_bits(q), bf16_bits(k), bf16_bits(v), mask, 4, 2, scale=1.0)
    e = math.e
    z2 = 2 * e + e * e + 1 / e
    expect_out = np.array([
        [e / (1 + e), 1 / (1 + e)],
        [1 / (1 + e), e / (1 + e)],
        [(e + 2 * e * e) / z2, (e + 2 / e) / z2],
        [0.75, 0.75],
    ])
    expect_lse = np.array([math.log(1 + e), math.log(1 + e), math.log(z2), math.log(4)])
    np.testing.assert_allclose(out, expect_out, rtol=0, atol=1e-14)
    np.testing.assert_allclose(lse, expect_lse, rtol=0, atol=1e-14)
    # the printed decimals of the closed forms
    np.testing.assert_allclose(out[2], [1.326137, 0.261799], atol=5e-7)
    np.testing.assert_allclose(lse[2], 2.579724, atol=5e-7)


def test_empty_row_gives_zero_and_neg_inf():
    BH, n, block, d = 1, 128, 64, 8
    qb, kb, vb = make_case(BH, n, n, d, seed=10)
    mask = np.zeros((BH, 2, 2), dtype=np.uint8)
    mask[0, 1, 0] = 1
    out, lse = oracle.attention(qb, kb, vb, mask, n, block)
    assert np.all(out[:block] == 0)
    assert np.all(np.isneginf(lse[:block]))
    assert np.all(np.isfinite(lse[block:]))


def test_default_scale_is_inverse_sqrt_d():
    BH, n, block, d = 1, 128, 64, 64
    qb, kb, vb = make_case(BH, n, n, d, seed=11)
    mask = np.ones((BH, 2, 2), dtype=np.uint8)
    a = oracle.attention(qb, kb, vb, mask, n, block)
    b = oracle.attention(qb, kb, vb, mask, n, block, scale=1.0 / 8.0)
    np.testing.assert_array_equal(a[0], b[0])
