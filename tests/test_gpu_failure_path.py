"""Failure detection without a GPU fault: every pipeline wait in the forward is
bounded; a wait that runs out records BSA_ERR_TIMEOUT in a device word that the
host reads with bsa_get_device_error, and the kernel returns.  Here a wait on a
barrier nothing completes runs out after a short limit; the status must come
back, be cleared by the read, and leave the context usable (a forward on the
small workload still matches the oracle afterwards)."""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from block_sparse_attention_forward_b200 import inputs as I
from tests.helpers import LSE_ABS, OUT_MAX_ABS, OUT_MEAN_ABS, bf16_bits, compare_out

pytestmark = pytest.mark.gpu


def test_wait_that_runs_out_reports_timeout_and_context_survives(cuda_ok):
    import block_sparse_attention_forward_b200 as bsa
    from block_sparse_attention_forward_b200 import _ffi
    lib = _ffi.load()
    assert bsa.device_error() == 0  # starts clean
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    assert lib.bsa_check_wait_timeout(20000, stream) == 0  # 20 ms limit
    torch.cuda.synchronize()
    assert bsa.device_error() == 6  # BSA_ERR_TIMEOUT
    assert bsa.device_error() == 0  # the read cleared it
    assert lib.bsa_check_wait_timeout(0, stream) == 1  # argument check

    w = I.WORKLOADS["tiny"]
    q, k, v = I.gen_qkv(w)
    mask = I.gen_mask(w)
    grid, tile = (w.T, w.Hs, w.Ws), (w.tt, w.th, w.tw)
    qp, kp, vp = (bsa.tile_permute(t.cuda(), grid, tile, w.n_pad) for t in (q, k, v))
    out_p, lse = bsa.forward(qp, kp, vp, bsa.pack_mask(torch.from_numpy(mask).cuda()), w.n,
                             w.block)
    torch.cuda.synchronize()
    assert bsa.device_error() == 0
    BH = w.B * w.H
    perm = oracle.tile_order(w.T, w.Hs, w.Ws, w.tt, w.th, w.tw)
    qo, ko, vo = (oracle.permute(bf16_bits(t).reshape(BH, w.n, w.d), perm, w.n_pad)
                  for t in (q, k, v))
    ref, ref_lse = oracle.attention(qo, ko, vo, mask.reshape(BH, w.nb, w.nb), w.n, w.block)
    mx, mean, lse_err = compare_out(out_p.float().cpu().numpy().reshape(-1, w.d), ref,
                                    lse.cpu().numpy().reshape(-1), ref_lse)
    assert mx <= OUT_MAX_ABS and mean <= OUT_MEAN_ABS and lse_err <= LSE_ABS
