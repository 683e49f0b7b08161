"""bsa_pack_mask_noalloc, the entry point for callers that cannot allocate
device memory (a plug-in host that only passes its input and output buffers,
a runtime that reserved all device memory up front): it must give exactly what
bsa_pack_mask gives, call after call, although every call reuses one fixed
scratch array inside the library.  Packing is integer work, so the comparison
is exact.  This file is collected last on purpose."""
import ctypes

import numpy as np
import pytest
import torch

from block_sparse_attention_forward_b200 import inputs as I

pytestmark = pytest.mark.gpu


def _outputs(B, H, nb_q, nb_k, dev):
    words = (nb_k + 31) // 32
    rows = B * H * nb_q
    return {
        "bits": torch.empty((B, H, nb_q, words), dtype=torch.int32, device=dev),
        "counts": torch.empty(rows, dtype=torch.int32, device=dev),
        "row_offsets": torch.empty(rows + 1, dtype=torch.int32, device=dev),
        "col_idx": torch.full((rows * nb_k,), -7, dtype=torch.int32, device=dev),
        "schedule": torch.empty(rows, dtype=torch.int32, device=dev),
    }


def _via_existing(lib, dense, stream):
    B, H, nb_q, nb_k = dense.shape
    o = _outputs(B, H, nb_q, nb_k, dense.device)
    ws_bytes = lib.bsa_pack_mask_workspace(B, H, nb_q, nb_k)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dense.device)
    st = lib.bsa_pack_mask(dense.data_ptr(), B, H, nb_q, nb_k, o["bits"].data_ptr(),
                           o["counts"].data_ptr(), o["row_offsets"].data_ptr(),
                           o["col_idx"].data_ptr(), o["schedule"].data_ptr(), ws.data_ptr(),
                           ws_bytes, stream)
    assert st == 0
    return o


def _via_noalloc(lib, dense, stream):
    B, H, nb_q, nb_k = dense.shape
    o = _outputs(B, H, nb_q, nb_k, dense.device)
    st = lib.bsa_pack_mask_noalloc(dense.data_ptr(), B, H, nb_q, nb_k, o["bits"].data_ptr(),
                                   o["counts"].data_ptr(), o["row_offsets"].data_ptr(),
                                   o["col_idx"].data_ptr(), o["schedule"].data_ptr(), stream)
    assert st == 0
    return o


def test_noalloc_pack_matches_pack_mask_twice_in_a_row(cuda_ok):
    from block_sparse_attention_forward_b200 import _ffi
    lib = _ffi.load()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    # two different masks back to back: the second call finds the first call's
    # leftovers in the shared scratch array and must not be affected by them
    masks = [I.gen_mask(I.WORKLOADS["wan14b_720p"]), I.gen_mask(I.WORKLOADS["tiny"])]
    for m in masks:
        dense = torch.from_numpy(m).cuda()
        got = _via_noalloc(lib, dense, stream)
        ref = _via_existing(lib, dense, stream)
        torch.cuda.synchronize()
        for key in ("bits", "counts", "row_offsets", "col_idx", "schedule"):
            assert torch.equal(got[key], ref[key]), key
        total = int(ref["row_offsets"][-1])
        assert total == int(np.count_nonzero(m))


def test_noalloc_rejects_masks_larger_than_its_scratch(cuda_ok):
    # 262144 rows -> 256 tiles of 1024 rows, times (600 + 2) ints > 131072:
    # rejected on the host, before any launch (the pointers are never used)
    from block_sparse_attention_forward_b200 import _ffi
    lib = _ffi.load()
    P = ctypes.c_void_p
    fake = P(0x1000)
    assert lib.bsa_pack_mask_noalloc(fake, 1, 64, 4096, 600, fake, fake, fake, fake, fake,
                                     None) == 7  # BSA_ERR_WORKSPACE
