"""bsa_attention_host: the whole path from host buffers to host buffers with the
copies overlapped with the kernels, chunked over heads.

Heads are independent problems and every kernel computes a head the same way
whatever else shares the launch, so the chunked pipeline must give exactly
the bytes of the device path on all heads at once (checked for several chunk
sizes, including a ragged last chunk, one head per chunk and one chunk for
all); and it must match the fp64 oracle on the small workload."""
import dataclasses

import numpy as np
import pytest
import torch

import oracle
from block_sparse_attention_forward_b200 import inputs as I
from tests.helpers import LSE_ABS, OUT_MAX_ABS, OUT_MEAN_ABS, bf16_bits, compare_out

pytestmark = pytest.mark.gpu


def _device_path(w, q, k, v, mask):
    import block_sparse_attention_forward_b200 as bsa
    grid, tile = (w.T, w.Hs, w.Ws), (w.tt, w.th, w.tw)
    qp, kp, vp = (bsa.tile_permute(t.cuda(), grid, tile, w.n_pad) for t in (q, k, v))
    pm = bsa.pack_mask(torch.from_numpy(mask).cuda())
    out_p, lse = bsa.forward(qp, kp, vp, pm, w.n, w.block)
    out = bsa.tile_unpermute(out_p, grid, tile)
    torch.cuda.synchronize()
    return out.cpu(), lse.cpu()


def _host_path(w, q, k, v, mask, heads_per_chunk, pinned=True):
    import block_sparse_attention_forward_b200 as bsa
    hq, hk, hv = (t.pin_memory() if pinned else t.clone() for t in (q, k, v))
    hm = torch.from_numpy(mask)
    hm = hm.pin_memory() if pinned else hm
    out, lse = bsa.attention_host(hq, hk, hv, hm, (w.T, w.Hs, w.Ws), (w.tt, w.th, w.tw), w.block,
                                  heads_per_chunk=heads_per_chunk)
    torch.cuda.synchronize()
    assert bsa.device_error() == 0
    return out, lse


def test_host_path_matches_oracle_tiny(cuda_ok):
    w = I.WORKLOADS["tiny"]
    q, k, v = I.gen_qkv(w)
    mask = I.gen_mask(w)
    out, lse = _host_path(w, q, k, v, mask, heads_per_chunk=1)
    BH = w.B * w.H
    perm = oracle.tile_order(w.T, w.Hs, w.Ws, w.tt, w.th, w.tw)
    qo, ko, vo = (oracle.permute(bf16_bits(t).reshape(BH, w.n, w.d), perm, w.n_pad)
                  for t in (q, k, v))
    ref, ref_lse = oracle.attention(qo, ko, vo, mask.reshape(BH, w.nb, w.nb), w.n, w.block)
    ref = ref.reshape(BH, w.n_pad, w.d)
    ref_frame = np.empty((BH, w.n, w.d))
    ref_frame[:, perm] = ref[:, :w.n]
    mx, mean, lse_err = compare_out(out.float().numpy().reshape(-1, w.d), ref_frame.reshape(-1, w.d),
                                    lse.numpy().reshape(-1), ref_lse)
    assert mx <= OUT_MAX_ABS and mean <= OUT_MEAN_ABS and lse_err <= LSE_ABS


@pytest.mark.parametrize("heads_per_chunk", [3, 1, 0, 64])
def test_host_path_equals_device_path(cuda_ok, heads_per_chunk):
    w = dataclasses.replace(I.WORKLOADS["wan14b_720p"], H=10)
    q, k, v = I.gen_qkv(w)
    mask = I.gen_mask(w)
    out_d, lse_d = _device_path(w, q, k, v, mask)
    out_h, lse_h = _host_path(w, q, k, v, mask, heads_per_chunk)
    assert torch.equal(out_h, out_d)
    assert torch.equal(lse_h.view(torch.int32), lse_d.view(torch.int32))


def test_host_path_pageable_memory(cuda_ok):
    w = dataclasses.replace(I.WORKLOADS["wan13b_480p"], H=3)
    q, k, v = I.gen_qkv(w)
    mask = I.gen_mask(w)
    out_d, lse_d = _device_path(w, q, k, v, mask)
    out_h, lse_h = _host_path(w, q, k, v, mask, heads_per_chunk=2, pinned=False)
    assert torch.equal(out_h, out_d)
    assert torch.equal(lse_h.view(torch.int32), lse_d.view(torch.int32))
