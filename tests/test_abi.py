"""CPU-side checks of the C ABI: the library loads, exports every symbol that
include/bsa.h declares, and rejects bad arguments on the host before any CUDA
call (no GPU needed)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    with open(os.path.join(ROOT, "include", "bsa.h")) as f:
        text = f.read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(bsa_[a-z_]+)\s*\(", text)))


@pytest.fixture(scope="module")
def lib():
    from block_sparse_attention_forward_b200 import _ffi, build
    build.build()
    return _ffi.load()


def test_header_declarations_match_binding():
    from block_sparse_attention_forward_b200 import _ffi
    assert declared_functions() == sorted(_ffi.EXPORTED)


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name


def test_status_strings(lib):
    assert lib.bsa_status_string(0) == b"BSA_OK"
    assert lib.bsa_status_string(6) == b"BSA_ERR_TIMEOUT"
    assert lib.bsa_status_string(99) == b"BSA_ERR_UNKNOWN"
    assert lib.bsa_version() >= 100


def test_pack_mask_rejects_bad_args(lib):
    P = ctypes.c_void_p
    fake = P(0x1000)
    # null output
    assert lib.bsa_pack_mask(fake, 1, 1, 4, 4, None, fake, fake, fake, fake, fake, 4096, None) == 1
    # non-positive size
    assert lib.bsa_pack_mask(fake, 1, 0, 4, 4, fake, fake, fake, fake, fake, fake, 4096, None) == 1
    # int32 overflow of B*H*nb_q*nb_k
    assert lib.bsa_pack_mask(fake, 64, 64, 1024, 1024, fake, fake, fake, fake, fake, fake,
                             1 << 30, None) == 4
    # misaligned output
    assert lib.bsa_pack_mask(fake, 1, 1, 4, 4, P(0x1001), fake, fake, fake, fake, fake, 4096,
                             None) == 3
    # workspace too small
    assert lib.bsa_pack_mask_workspace(1, 1, 4, 4) > 0
    assert lib.bsa_pack_mask(fake, 1, 1, 4, 4, fake, fake, fake, fake, fake, fake, 1, None) == 7


def test_pack_from_threshold_rejects_bad_args(lib):
    P = ctypes.c_void_p
    f = P(0x1000)
    fn = lib.bsa_pack_mask_from_threshold
    # null threshold map, null p
    assert fn(None, f, 1, 1, 4, 4, f, f, f, f, f, f, 4096, None) == 1
    assert fn(f, None, 1, 1, 4, 4, f, f, f, f, f, f, 4096, None) == 1
    # non-positive batch
    assert fn(f, f, 0, 1, 4, 4, f, f, f, f, f, f, 4096, None) == 1
    # int32 overflow of B*H*nb_q*nb_k
    assert fn(f, f, 64, 64, 1024, 1024, f, f, f, f, f, f, 1 << 30, None) == 4
    # misaligned map or p
    assert fn(P(0x1002), f, 1, 1, 4, 4, f, f, f, f, f, f, 4096, None) == 3
    assert fn(f, P(0x1001), 1, 1, 4, 4, f, f, f, f, f, f, 4096, None) == 3
    # workspace too small
    assert fn(f, f, 1, 1, 4, 4, f, f, f, f, f, f, 1, None) == 7


def test_threshold_resize_rejects_bad_args(lib):
    P = ctypes.c_void_p
    a, b = P(0x1000), P(0x2000)
    fn = lib.bsa_threshold_resize
    assert fn(None, 1, 4, 4, b, 8, 8, None) == 1
    assert fn(a, 1, 4, 4, None, 8, 8, None) == 1
    assert fn(a, 1, 0, 4, b, 8, 8, None) == 1
    assert fn(a, 1, 4, 4, b, 8, -1, None) == 1
    assert fn(P(0x1001), 1, 4, 4, b, 8, 8, None) == 3
    assert fn(a, 1, 4, 4, b, 65536, 8, None) == 2  # more blocks per axis than supported
    assert fn(a, 1 << 20, 4, 4, b, 4096, 8, None) == 4  # H * tq >= 2^31


def test_gather_rows_rejects_bad_args(lib):
    P = ctypes.c_void_p
    a, b, t = P(0x1000), P(0x2000), P(0x3000)
    fn = lib.bsa_gather_rows
    assert fn(None, b, 1, 1, 8, 8, 8, t, 0, None) == 1
    assert fn(a, b, 1, 1, 8, 8, 8, None, 0, None) == 1
    assert fn(a, b, 1, 1, 8, 8, 8, t, 2, None) == 1       # per_head must be 0 or 1
    assert fn(a, b, 1, 1, 0, 8, 8, t, 0, None) == 1
    assert fn(a, b, 1, 1, 8, 8, 12, t, 0, None) == 2      # d % 8
    assert fn(P(0x1008), b, 1, 1, 8, 8, 8, t, 0, None) == 3
    assert fn(a, b, 1, 1, 8, 8, 8, P(0x3002), 0, None) == 3
    assert fn(a, b, 1, 70000, 8, 8, 8, t, 1, None) == 4   # per-head tables: H <= 65535


def test_host_orders_reject_bad_args(lib):
    P = ctypes.c_void_p
    buf = (ctypes.c_int32 * 8)()
    assert lib.bsa_hilbert_order(0, 2, 2, buf) == 1
    assert lib.bsa_hilbert_order(2, 2, 2, None) == 1
    assert lib.bsa_tile_order(2, 2, 2, 0, 1, 1, buf) == 1
    assert lib.bsa_order_tables(buf, 8, 7, buf, buf) == 1  # n_pad < n


def test_forward_blocks_rejects_bad_args(lib):
    from block_sparse_attention_forward_b200._ffi import BsaMask
    P = ctypes.c_void_p
    a = P(0x10000)
    fwd = lib.bsa_forward_blocks
    # 128-row query blocks over 64-key blocks: nb_q = 8, nb_k = 16, 1 word
    good = BsaMask(0x1000, 0x1000, 0x1000, 0x1000, 0x1000, 1, 2, 8, 16, 1)

    def call(m=good, bq=128, bk=64, n_valid=1000, n_pad=1024, d=128):
        return fwd(a, a, a, ctypes.byref(m), a, a, 1, 2, n_valid, n_pad, d, bq, bk, 0.0, None)
    assert call(bq=64, bk=128) == 2                      # finer queries than keys
    assert call(bq=128, bk=32) == 2
    assert call(n_valid=960) == 1                        # pad fills a whole 64-key block
    square = BsaMask(0x1000, 0x1000, 0x1000, 0x1000, 0x1000, 1, 2, 8, 8, 1)
    assert call(m=square) == 1                           # mask built for 128-key blocks
    assert call(d=96) == 2


def test_attention_host_rejects_bad_args(lib):
    P = ctypes.c_void_p
    a = P(0x10000)
    ws = P(0x100000)
    fn = lib.bsa_attention_host
    need = lib.bsa_attention_host_workspace(1, 2, 4, 16, 16, 64, 64, 0)
    assert need > 0

    def call(q=a, ws_ptr=ws, ws_bytes=need, d=64, block=64):
        return fn(q, a, a, a, a, a, 1, 2, 4, 16, 16, d, 1, 8, 8, block, 0.0, 0, ws_ptr, ws_bytes,
                  None)
    assert call(q=None) == 1
    assert call(ws_ptr=None) == 1
    assert call(ws_bytes=need - 1) == 7
    assert call(ws_ptr=P(0x100010)) == 3  # 256-byte alignment


def test_wait_timeout_check_rejects_bad_args(lib):
    assert lib.bsa_check_wait_timeout(0, None) == 1
    assert lib.bsa_check_wait_timeout(10000001, None) == 1


def test_permute_rejects_bad_args(lib):
    P = ctypes.c_void_p
    a, b = P(0x1000), P(0x2000)
    assert lib.bsa_tile_permute(None, b, 1, 1, 2, 2, 2, 8, 1, 1, 1, 8, None) == 1
    assert lib.bsa_tile_permute(a, b, 1, 1, 2, 2, 2, 8, 1, 1, 1, 7, None) == 1  # n_pad < N
    assert lib.bsa_tile_permute(a, b, 1, 1, 2, 2, 2, 6, 1, 1, 1, 8, None) == 2  # d % 8
    assert lib.bsa_tile_permute(P(0x1008), b, 1, 1, 2, 2, 2, 8, 1, 1, 1, 8, None) == 3
    assert lib.bsa_tile_unpermute(a, b, 1, 1, 2, 2, 0, 8, 1, 1, 1, 8, None) == 1


def test_forward_rejects_bad_args(lib):
    from block_sparse_attention_forward_b200._ffi import BsaMask
    P = ctypes.c_void_p
    a = P(0x10000)
    m = BsaMask(0x1000, 0x1000, 0x1000, 0x1000, 0x1000, 1, 2, 8, 8, 1)
    fwd = lib.bsa_forward
    ok = dict(B=1, H=2, n_valid=1000, n_pad=1024, d=128, block=128)

    def call(mask=m, q=a, out=a, **kw):
        args = dict(ok)
        args.update(kw)
        return fwd(q, a, a, ctypes.byref(mask), out, a, args["B"], args["H"], args["n_valid"],
                   args["n_pad"], args["d"], args["block"], 0.0, None)

    assert call(q=None) == 1
    assert call(d=96) == 2
    assert call(block=32) == 2
    assert call(n_pad=1000, n_valid=1000) == 2  # n_pad % block
    assert call(n_valid=1025) == 1
    assert call(n_valid=896) == 1  # a whole block of padding
    bad = BsaMask(0x1000, 0x1000, 0x1000, 0x1000, 0x1000, 1, 2, 8, 8, 2)  # wrong words
    assert call(mask=bad) == 1
    assert call(out=P(0x10004)) == 3


@pytest.mark.parametrize("B,H,nb_q,nb_k,expect", [(1, 1, 4096, 32766, 7),   # needs 131073 ints
                                                  (1, 64, 4096, 600, 7),
                                                  (1, 1, 1, 49152, 2)])     # past the packing cap
def test_pack_noalloc_rejects_oversize_on_the_host(lib, B, H, nb_q, nb_k, expect):
    # the built-in scratch holds 131072 ints; a call needing one more is
    # refused before any CUDA call (the pointers are never used)
    fake = ctypes.c_void_p(0x1000)
    assert lib.bsa_pack_mask_noalloc(fake, B, H, nb_q, nb_k, fake, fake, fake, fake, fake,
                                     None) == expect


def test_predict_top_p_workspace_and_host_checks(lib):
    # the workspace holds both block means, the fp32 scores and the sort's tables;
    # every rejection below happens on the host, before any CUDA call
    B, H, n_pad, d, block = 1, 2, 1024, 64, 64
    nb = n_pad // block
    need = lib.bsa_predict_top_p_workspace(B, H, n_pad, d, block)
    assert need >= 2 * B * H * nb * d * 4 + B * H * nb * nb * 4
    assert lib.bsa_predict_top_p_workspace(B, H, n_pad + 1, d, block) == 0  # n_pad % block
    assert lib.bsa_predict_top_p_workspace(0, H, n_pad, d, block) == 0
    P = ctypes.c_void_p
    f = P(0x1000)

    def call(q=f, B=B, H=H, n_valid=n_pad, n_pad=n_pad, d=d, block=block, ws=f, ws_bytes=need):
        return lib.bsa_predict_top_p(q, f, B, H, n_valid, n_pad, d, block, f, f, f, f, f, f, f,
                                     ws, ws_bytes, None)

    assert call(q=None) == 1                                  # null input
    assert call(n_valid=n_pad - block) == 1                   # last block would be empty
    assert call(d=96) == 2                                    # head dim
    assert call(n_pad=64 * 2049, n_valid=64 * 2049) == 2      # more than 2048 blocks per row
    assert call(q=P(0x1001)) == 3                             # misaligned q
    assert call(ws_bytes=need - 1) == 7                       # workspace too small
    assert call(ws=None) == 7
    assert call(ws=P(0x1008)) == 3                            # misaligned workspace
