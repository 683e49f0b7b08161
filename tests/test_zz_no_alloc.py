"""bsa_pack_mask_noalloc, the entry point for callers that cannot allocate
device memory (a plug-in host that only passes its input and output buffers,
a runtime that reserved all device memory up front): it must give exactly what
bsa_pack_mask gives, call after call, although every call reuses one fixed
scratch array inside the library, and its CRM rows and lists must equal the
oracle's.  Packing is integer work, so the comparisons are exact.  This file is
collected last on purpose."""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from block_sparse_attention_forward_b200 import inputs as I
from tests.helpers import check_schedule

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
        _compare_with_oracle(got, m)


def _compare_with_oracle(got, m):
    bits_ref = oracle.pack_bits(m)
    counts_ref, offsets_ref, col_ref = oracle.crm_lists(bits_ref)
    np.testing.assert_array_equal(got["bits"].cpu().numpy().view(np.uint32), bits_ref)
    np.testing.assert_array_equal(got["counts"].cpu().numpy(), counts_ref)
    np.testing.assert_array_equal(got["row_offsets"].cpu().numpy().astype(np.int64), offsets_ref)
    total = int(offsets_ref[-1])
    np.testing.assert_array_equal(got["col_idx"][:total].cpu().numpy(), col_ref)
    check_schedule(got["schedule"].cpu().numpy(), counts_ref, m.shape[2], m.shape[3])


def test_noalloc_pack_at_the_largest_size_that_fits(cuda_ok):
    # scratch need (nb_k + 2) * ceil(rows / 1024) + 1 ints: 30 row tiles and
    # nb_k = 4367 need 131071, one int under the 131072 the array holds and the
    # most any accepted call can need (131072 itself would take
    # (nb_k + 2) * tiles = 131071, a prime: one tile of 131069 key blocks,
    # past the packing limit of 49151)
    from block_sparse_attention_forward_b200 import _ffi
    lib = _ffi.load()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    rng = np.random.default_rng(31)
    m = (rng.random((1, 30, 1024, 4367)) < 0.02).astype(np.uint8)
    dense = torch.from_numpy(m).cuda()
    for _ in range(2):
        got = _via_noalloc(lib, dense, stream)
        ref = _via_existing(lib, dense, stream)
        torch.cuda.synchronize()
        for key in ("bits", "counts", "row_offsets", "col_idx", "schedule"):
            assert torch.equal(got[key], ref[key]), key
    _compare_with_oracle(got, m)


@pytest.mark.parametrize("B,H,nb_q,nb_k", [(1, 64, 4096, 600),   # 256 tiles x 602 + 1
                                           (1, 1, 4096, 32766)])  # 4 x 32768 + 1 = 131073
def test_noalloc_rejects_masks_larger_than_its_scratch(cuda_ok, B, H, nb_q, nb_k):
    # rejected on the host, before any launch (the pointers are never used);
    # the second case needs exactly one int more than the array holds
    from block_sparse_attention_forward_b200 import _ffi
    lib = _ffi.load()
    P = ctypes.c_void_p
    fake = P(0x1000)
    assert lib.bsa_pack_mask_noalloc(fake, B, H, nb_q, nb_k, fake, fake, fake, fake, fake,
                                     None) == 7  # BSA_ERR_WORKSPACE
