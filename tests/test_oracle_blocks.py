"""Pins for the oracle with query blocks and key blocks of different sizes
(finer key blocks: "ScalingAttention" Sec. 5.4 names the fixed 128 x 128 block
as the granularity bottleneck below 40 % density).

- Refinement: a (128, 128) mask written at key granularity 64 (each key bit
  doubled) gives exactly the same output;
- half a block: keeping only one 64-key half equals torch's fp64 SDPA over
  exactly those keys;
- the query side keeps 128-row granularity: changing one mask row touches
  only the 128 queries of that block.
"""
import numpy as np
import torch

import oracle


def _qkv(BH, n_pad, d, seed):
    g = torch.Generator().manual_seed(seed)
    t = [torch.randn((BH, n_pad, d), generator=g).to(torch.bfloat16) for _ in range(3)]
    return t, [x.view(torch.int16).numpy().view(np.uint16) for x in t]


def test_refined_key_mask_is_identical():
    BH, n_pad, d, n_valid = 2, 512, 32, 500
    _, (qb, kb, vb) = _qkv(BH, n_pad, d, 1)
    rng = np.random.default_rng(0)
    m128 = (rng.random((BH, 4, 4)) < 0.6).astype(np.uint8)
    m128[:, np.arange(4), np.arange(4)] = 1
    m64 = np.repeat(m128, 2, axis=2)
    a = oracle.attention(qb, kb, vb, m128, n_valid, 128)
    b = oracle.attention(qb, kb, vb, m64, n_valid, 128, block_k=64)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])


def test_half_block_equals_sdpa_on_those_keys():
    BH, n_pad, d = 1, 256, 16
    (q, k, v), (qb, kb, vb) = _qkv(BH, n_pad, d, 2)
    m = np.zeros((BH, 2, 4), dtype=np.uint8)
    m[0, 0, 1] = 1  # query block 0 sees keys 64..127 only
    m[0, 1, [0, 3]] = 1  # query block 1 sees keys 0..63 and 192..255
    out, lse = oracle.attention(qb, kb, vb, m, n_pad, 128, block_k=64)
    qd, kd, vd = (x.double() for x in (q, k, v))
    allowed = torch.zeros((n_pad, n_pad), dtype=torch.bool)
    allowed[:128, 64:128] = True
    allowed[128:, :64] = True
    allowed[128:, 192:] = True
    ref = torch.nn.functional.scaled_dot_product_attention(qd, kd, vd, attn_mask=allowed[None])
    s = (qd @ kd.transpose(1, 2)) / np.sqrt(d)
    ref_lse = torch.logsumexp(s.masked_fill(~allowed[None], -float("inf")), dim=-1)
    np.testing.assert_allclose(out.reshape(BH, n_pad, d), ref.numpy(), rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse.reshape(BH, n_pad), ref_lse.numpy(), rtol=0, atol=1e-12)


def test_query_side_keeps_its_own_granularity():
    BH, n_pad, d = 1, 384, 16
    _, (qb, kb, vb) = _qkv(BH, n_pad, d, 3)
    rng = np.random.default_rng(4)
    m = (rng.random((BH, 3, 6)) < 0.5).astype(np.uint8)
    m[:, :, 0] = 1
    a, _ = oracle.attention(qb, kb, vb, m, n_pad, 128, block_k=64)
    m2 = m.copy()
    m2[0, 1] = 1 - m2[0, 1]
    m2[0, 1, 0] = 1
    b, _ = oracle.attention(qb, kb, vb, m2, n_pad, 128, block_k=64)
    a, b = a.reshape(n_pad, d), b.reshape(n_pad, d)
    assert np.array_equal(a[:128], b[:128]) and np.array_equal(a[256:], b[256:])
    assert not np.array_equal(a[128:256], b[128:256])
