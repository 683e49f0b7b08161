"""fp64 CPU oracle for bitmask-driven block-sparse attention (test infrastructure).

TEST INFRASTRUCTURE ONLY: tests/, ``__graft_entry__.smoke()`` and the CPU
baseline leg of ``bench.py`` may import this package; the product path never
does.  It shares no code with the CUDA library: the arithmetic lives in
``oracle.c`` (plain loops, fp64) and this module only compiles it with gcc and
marshals numpy arrays.

Functions and the passages they follow (pages: "ScalingAttention: Discovering
Intrinsic Sparse Attention Topology for Video Diffusion Transformers"):

- ``crm_words``          -- Sec. 4.3.2, one uint32 holds 32 key blocks.
- ``pack_bits``          -- Sec. 4.3.2 (CRM bitmask rows), bit order from
                            Appendix E, Algorithm 2 (base + CTZ).
- ``crm_lists``          -- Appendix E, Algorithm 2 (Init/Advance/Next/Index).
- ``schedule``           -- rows by kept-block count, largest first, stable
                              (head-major when that order mixes many heads)
                            (the pages are silent; plainest reading).
- ``tile_order``, ``permute``, ``unpermute``
                         -- token reordering into 3-D tiles, Sec. 5.4 and 5.5.
- ``attention``          -- Sec. 4.3.2 block-sparse FlashAttention forward,
                            written as plain masked softmax attention in fp64;
                            query and key blocks may differ in size (finer key
                            blocks: Sec. 5.4, the granularity bottleneck).
- ``threshold_mask``     -- Sec. 4.1.2 (Eq. 2, M_p = 1(T <= p)) with one
                            threshold per head (Algorithm 1, FAST).
- ``threshold_resize``   -- Sec. 4.3.1, Eq. 7 (conservative bilinear resize of
                            the threshold map with the ceiling rule).
- ``hilbert_key``, ``hilbert_order``
                         -- DFSAttn's Hilbert-curve token reordering, as a 3-D
                            Hilbert curve over the enclosing power-of-two cube
                            (Skilling's transpose method), grid points in curve
                            order.
- ``top_p_mask``         -- online top-p block mask: pooled-query/key block
                            scores, row softmax, smallest descending prefix
                            reaching top_p (ScalingAttention Algorithm 1's
                            sort-and-accumulate cut, per row, per-head top-p).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile oracle.c into liboracle.so with gcc (-O2, OpenMP, fp64)."""
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    tmp = _LIB_PATH + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-fno-fast-math", "-fopenmp", "-shared", "-fPIC", "-std=c11",
           "-o", tmp, _SRC, "-lm"]
    subprocess.check_call(cmd)
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            P = ctypes.c_void_p
            I64 = ctypes.c_int64
            I = ctypes.c_int
            lib.oracle_num_threads.restype = I
            lib.oracle_crm_words.argtypes = [I]
            lib.oracle_crm_words.restype = I
            lib.oracle_pack_bits.argtypes = [P, I64, I, P]
            lib.oracle_crm_lists.argtypes = [P, I64, I, P, P, P]
            lib.oracle_crm_lists.restype = I64
            lib.oracle_schedule.argtypes = [P, I64, P]
            lib.oracle_tile_order.argtypes = [I, I, I, I, I, I, P]
            lib.oracle_permute.argtypes = [P, P, I64, I64, I64, I, P]
            lib.oracle_unpermute.argtypes = [P, P, I64, I64, I64, I, P]
            lib.oracle_attention.argtypes = [P, P, P, P, I64, I64, I64, I, I, ctypes.c_double,
                                             P, I64, I, P, P]
            lib.oracle_attention_blocks.argtypes = [P, P, P, P, I64, I64, I64, I, I, I,
                                                    ctypes.c_double, P, I64, I, P, P]
            lib.oracle_threshold_mask.argtypes = [P, P, I, I, I, I, P]
            lib.oracle_threshold_resize.argtypes = [P, I, I, I, P, I, I]
            lib.oracle_hilbert_key.argtypes = [I, I, I, I]
            lib.oracle_hilbert_key.restype = ctypes.c_uint64
            lib.oracle_hilbert_order.argtypes = [I, I, I, P]
            lib.oracle_hilbert_order.restype = I
            lib.oracle_top_p_mask.argtypes = [P, P, I64, I64, I64, I64, I, I, P, P, P, P]
            _lib = lib
    return _lib


def _ptr(a: np.ndarray):
    return ctypes.c_void_p(a.ctypes.data) if a is not None else None


def num_threads() -> int:
    return _load().oracle_num_threads()


def crm_words(nb_k: int) -> int:
    return _load().oracle_crm_words(int(nb_k))


def pack_bits(dense: np.ndarray) -> np.ndarray:
    """dense uint8 [..., nb_q, nb_k] -> CRM bits uint32 [..., nb_q, words]."""
    dense = np.ascontiguousarray(dense, dtype=np.uint8)
    nb_k = dense.shape[-1]
    rows = int(np.prod(dense.shape[:-1]))
    words = crm_words(nb_k)
    bits = np.zeros(dense.shape[:-1] + (words,), dtype=np.uint32)
    _load().oracle_pack_bits(_ptr(dense), rows, nb_k, _ptr(bits))
    return bits


def crm_lists(bits: np.ndarray):
    """Walk CRM rows with the Algorithm 2 iterator.

    Returns (counts int32 [rows], row_offsets int64 [rows+1], col_idx int32 [total]).
    """
    bits = np.ascontiguousarray(bits, dtype=np.uint32)
    words = bits.shape[-1]
    rows = int(np.prod(bits.shape[:-1]))
    counts = np.zeros(rows, dtype=np.int32)
    offsets = np.zeros(rows + 1, dtype=np.int64)
    lib = _load()
    total = lib.oracle_crm_lists(_ptr(bits), rows, words, _ptr(counts), _ptr(offsets), None)
    col_idx = np.zeros(max(total, 1), dtype=np.int32)
    lib.oracle_crm_lists(_ptr(bits), rows, words, _ptr(counts), _ptr(offsets), _ptr(col_idx))
    return counts, offsets, col_idx[:total]


def schedule(counts: np.ndarray) -> np.ndarray:
    """Work order of the rows: by kept-block count, largest first, ties by
    ascending row id (a stable sort)."""
    counts = np.ascontiguousarray(counts, dtype=np.int32)
    out = np.zeros(counts.size, dtype=np.int32)
    _load().oracle_schedule(_ptr(counts), counts.size, _ptr(out))
    return out


def tile_order(T: int, Hs: int, Ws: int, tt: int, th: int, tw: int) -> np.ndarray:
    """perm[p] = frame-major index of the token at tile-major position p."""
    perm = np.zeros(T * Hs * Ws, dtype=np.int64)
    _load().oracle_tile_order(T, Hs, Ws, tt, th, tw, _ptr(perm))
    return perm


def permute(x_bits: np.ndarray, perm: np.ndarray, n_pad: int) -> np.ndarray:
    """x_bits uint16 [BH, n, d] (raw bf16) -> [BH, n_pad, d] tile-major, zero tail."""
    x_bits = np.ascontiguousarray(x_bits, dtype=np.uint16)
    BH, n, d = x_bits.shape
    out = np.empty((BH, n_pad, d), dtype=np.uint16)
    perm = np.ascontiguousarray(perm, dtype=np.int64)
    _load().oracle_permute(_ptr(x_bits), _ptr(out), BH, n, n_pad, d, _ptr(perm))
    return out


def unpermute(y_bits: np.ndarray, perm: np.ndarray, n: int) -> np.ndarray:
    """y_bits uint16 [BH, n_pad, d] tile-major -> [BH, n, d] frame-major."""
    y_bits = np.ascontiguousarray(y_bits, dtype=np.uint16)
    BH, n_pad, d = y_bits.shape
    out = np.empty((BH, n, d), dtype=np.uint16)
    perm = np.ascontiguousarray(perm, dtype=np.int64)
    _load().oracle_unpermute(_ptr(y_bits), _ptr(out), BH, n, n_pad, d, _ptr(perm))
    return out


def attention(q_bits, k_bits, v_bits, mask, n_valid: int, block: int, scale: float | None = None,
              rows: np.ndarray | None = None, dense_literal: bool = False,
              block_k: int | None = None):
    """Masked softmax attention in fp64 over permuted tokens.

    q_bits/k_bits/v_bits: uint16 raw bf16, [BH, n_pad, d].  mask: uint8
    [BH, n_pad // block, n_pad // block_k] (block_k defaults to block).
    rows: optional int64 flat query ids (bh * n_pad + i).  Returns (out [R, d], lse [R])
    in float64, R = len(rows) or BH * n_pad.
    """
    q_bits = np.ascontiguousarray(q_bits, dtype=np.uint16)
    k_bits = np.ascontiguousarray(k_bits, dtype=np.uint16)
    v_bits = np.ascontiguousarray(v_bits, dtype=np.uint16)
    mask = np.ascontiguousarray(mask, dtype=np.uint8)
    BH, n_pad, d = q_bits.shape
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    if rows is None:
        n_rows = BH * n_pad
        rows_p = None
    else:
        rows = np.ascontiguousarray(rows, dtype=np.int64)
        n_rows = rows.size
        rows_p = _ptr(rows)
    out = np.zeros((n_rows, d), dtype=np.float64)
    lse = np.zeros(n_rows, dtype=np.float64)
    block_k = block if block_k is None else int(block_k)
    assert mask.shape == (BH, n_pad // block, n_pad // block_k), mask.shape
    _load().oracle_attention_blocks(_ptr(q_bits), _ptr(k_bits), _ptr(v_bits), _ptr(mask), BH,
                                    n_valid, n_pad, d, block, block_k, float(scale), rows_p,
                                    n_rows, int(dense_literal), _ptr(out), _ptr(lse))
    return out, lse


def threshold_mask(thr: np.ndarray, p: np.ndarray, B: int = 1) -> np.ndarray:
    """thr float32 [H, nb_q, nb_k], p float32 [H] -> dense uint8 [B, H, nb_q, nb_k]."""
    thr = np.ascontiguousarray(thr, dtype=np.float32)
    p = np.ascontiguousarray(p, dtype=np.float32)
    H, nb_q, nb_k = thr.shape
    assert p.shape == (H,)
    dense = np.zeros((B, H, nb_q, nb_k), dtype=np.uint8)
    _load().oracle_threshold_mask(_ptr(thr), _ptr(p), B, H, nb_q, nb_k, _ptr(dense))
    return dense


def threshold_resize(src: np.ndarray, tq: int, tk: int) -> np.ndarray:
    """src float32 [H, sq, sk] -> float32 [H, tq, tk] by Eq. 7 (min over the
    source blocks with a nonzero bilinear weight at (u*sq/tq, v*sk/tk))."""
    src = np.ascontiguousarray(src, dtype=np.float32)
    H, sq, sk = src.shape
    dst = np.empty((H, tq, tk), dtype=np.float32)
    _load().oracle_threshold_resize(_ptr(src), H, sq, sk, _ptr(dst), int(tq), int(tk))
    return dst


def hilbert_key(t: int, y: int, x: int, bits: int) -> int:
    """Index of (t, y, x) on the 3-D Hilbert curve over the cube of side 2**bits."""
    return int(_load().oracle_hilbert_key(int(t), int(y), int(x), int(bits)))


def hilbert_order(T: int, Hs: int, Ws: int) -> np.ndarray:
    """perm[p] = frame-major index of the token at position p of the Hilbert order."""
    perm = np.zeros(T * Hs * Ws, dtype=np.int64)
    if _load().oracle_hilbert_order(T, Hs, Ws, _ptr(perm)) < 0:
        raise MemoryError("oracle_hilbert_order")
    return perm


def top_p_mask(q_bits, k_bits, H: int, n_valid: int, block: int, tau, top_p,
               with_prob: bool = False):
    """q_bits/k_bits raw bf16 [B*H, n_pad, d] in block order; tau, top_p per head [H].
    Returns mask uint8 [B*H, nb, nb] (and the fp64 probabilities if with_prob)."""
    q_bits = np.ascontiguousarray(q_bits, dtype=np.uint16)
    k_bits = np.ascontiguousarray(k_bits, dtype=np.uint16)
    BH, n_pad, d = q_bits.shape
    assert k_bits.shape == q_bits.shape and BH % H == 0
    nb = n_pad // block
    tau = np.ascontiguousarray(tau, dtype=np.float64)
    top_p = np.ascontiguousarray(top_p, dtype=np.float64)
    assert tau.shape == (H,) and top_p.shape == (H,)
    mask = np.zeros((BH, nb, nb), dtype=np.uint8)
    prob = np.zeros((BH, nb, nb), dtype=np.float64) if with_prob else None
    _load().oracle_top_p_mask(_ptr(q_bits), _ptr(k_bits), BH // H, H, n_valid, n_pad, d, block,
                              _ptr(tau), _ptr(top_p), _ptr(mask), _ptr(prob))
    return (mask, prob) if with_prob else mask
