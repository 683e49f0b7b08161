"""ctypes binding of libbsa (the C ABI in include/bsa.h).

Argument marshalling only: every step runs in the CUDA library.  There is no
CPU fallback; if libbsa.so is missing the first call raises.
"""
from __future__ import annotations

import ctypes
import os

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libbsa.so")

STATUS_NAMES = {
    0: "BSA_OK",
    1: "BSA_ERR_INVALID_ARG",
    2: "BSA_ERR_UNSUPPORTED",
    3: "BSA_ERR_MISALIGNED",
    4: "BSA_ERR_OVERFLOW",
    5: "BSA_ERR_LAUNCH",
    6: "BSA_ERR_TIMEOUT",
    7: "BSA_ERR_WORKSPACE",
}

# every symbol include/bsa.h declares
EXPORTED = (
    "bsa_version",
    "bsa_status_string",
    "bsa_pack_mask_workspace",
    "bsa_pack_mask",
    "bsa_pack_mask_noalloc",
    "bsa_pack_mask_from_threshold",
    "bsa_threshold_resize",
    "bsa_predict_top_p_workspace",
    "bsa_predict_top_p",
    "bsa_hilbert_order",
    "bsa_tile_order",
    "bsa_order_tables",
    "bsa_gather_rows",
    "bsa_tile_permute",
    "bsa_tile_unpermute",
    "bsa_forward",
    "bsa_forward_blocks",
    "bsa_attention_host_workspace",
    "bsa_attention_host",
    "bsa_check_wait_timeout",
    "bsa_get_device_error",
)


class BsaError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {STATUS_NAMES.get(status, status)}")


class BsaMask(ctypes.Structure):
    """Mirror of the C struct bsa_mask (device pointers + sizes)."""
    _fields_ = [
        ("bits", ctypes.c_void_p),
        ("counts", ctypes.c_void_p),
        ("row_offsets", ctypes.c_void_p),
        ("col_idx", ctypes.c_void_p),
        ("schedule", ctypes.c_void_p),
        ("B", ctypes.c_int),
        ("H", ctypes.c_int),
        ("nb_q", ctypes.c_int),
        ("nb_k", ctypes.c_int),
        ("words", ctypes.c_int),
    ]


_lib = None


def load() -> ctypes.CDLL:
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(
            f"libbsa.so not found at {LIB_PATH}; build it with "
            "`python -m block_sparse_attention_forward_b200.build` (no CPU fallback exists)")
    lib = ctypes.CDLL(LIB_PATH)
    P, I, SZ = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
    lib.bsa_version.restype = I
    lib.bsa_status_string.argtypes = [I]
    lib.bsa_status_string.restype = ctypes.c_char_p
    lib.bsa_pack_mask_workspace.argtypes = [I, I, I, I]
    lib.bsa_pack_mask_workspace.restype = SZ
    lib.bsa_pack_mask.argtypes = [P, I, I, I, I, P, P, P, P, P, P, SZ, P]
    lib.bsa_pack_mask.restype = I
    lib.bsa_pack_mask_noalloc.argtypes = [P, I, I, I, I, P, P, P, P, P, P]
    lib.bsa_pack_mask_noalloc.restype = I
    lib.bsa_pack_mask_from_threshold.argtypes = [P, P, I, I, I, I, P, P, P, P, P, P, SZ, P]
    lib.bsa_pack_mask_from_threshold.restype = I
    lib.bsa_threshold_resize.argtypes = [P, I, I, I, P, I, I, P]
    lib.bsa_threshold_resize.restype = I
    lib.bsa_predict_top_p_workspace.argtypes = [I, I, I, I, I]
    lib.bsa_predict_top_p_workspace.restype = SZ
    lib.bsa_predict_top_p.argtypes = [P, P, I, I, I, I, I, I, P, P, P, P, P, P, P, P, SZ, P]
    lib.bsa_predict_top_p.restype = I
    lib.bsa_hilbert_order.argtypes = [I, I, I, P]
    lib.bsa_hilbert_order.restype = I
    lib.bsa_tile_order.argtypes = [I, I, I, I, I, I, P]
    lib.bsa_tile_order.restype = I
    lib.bsa_order_tables.argtypes = [P, I, I, P, P]
    lib.bsa_order_tables.restype = I
    lib.bsa_gather_rows.argtypes = [P, P, I, I, I, I, I, P, I, P]
    lib.bsa_gather_rows.restype = I
    for name in ("bsa_tile_permute", "bsa_tile_unpermute"):
        fn = getattr(lib, name)
        fn.argtypes = [P, P, I, I, I, I, I, I, I, I, I, I, P]
        fn.restype = I
    lib.bsa_forward.argtypes = [P, P, P, ctypes.POINTER(BsaMask), P, P, I, I, I, I, I, I,
                                ctypes.c_float, P]
    lib.bsa_forward.restype = I
    lib.bsa_forward_blocks.argtypes = [P, P, P, ctypes.POINTER(BsaMask), P, P, I, I, I, I, I, I,
                                       I, ctypes.c_float, P]
    lib.bsa_forward_blocks.restype = I
    lib.bsa_attention_host_workspace.argtypes = [I, I, I, I, I, I, I, I]
    lib.bsa_attention_host_workspace.restype = SZ
    lib.bsa_attention_host.argtypes = [P, P, P, P, P, P, I, I, I, I, I, I, I, I, I, I,
                                       ctypes.c_float, I, P, SZ, P]
    lib.bsa_attention_host.restype = I
    lib.bsa_check_wait_timeout.argtypes = [ctypes.c_uint, P]
    lib.bsa_check_wait_timeout.restype = I
    lib.bsa_get_device_error.argtypes = [ctypes.POINTER(I)]
    lib.bsa_get_device_error.restype = I
    _lib = lib
    return lib


def check(status: int, where: str) -> None:
    if status != 0:
        raise BsaError(status, where)
