"""bitmask-driven block-sparse attention forward for B200 (sm_100a).

Torch-facing wrappers over the C ABI of libbsa (include/bsa.h).  PyTorch only
provides device memory and the current stream; each call checks dtypes,
devices and contiguity, then passes raw pointers to the library.

    mask = pack_mask(dense_u8)                     # CRM rows, lists, schedule
    mask = pack_mask_from_threshold(thr, p)        # or straight from a threshold map
    qp = tile_permute(q, grid, tile, n_pad)        # frame-major -> 3-D tiles
    out_p, lse = forward(qp, kp, vp, mask, n_valid, block)
    out = tile_unpermute(out_p, grid, tile)        # back to frame-major

Other token orders (Hilbert curve, one tile shape per head) are host-built
tables applied on the GPU by one gather:

    fwd, inv = order_tables(hilbert_order(T, Hs, Ws), n_pad)
    qp = gather_rows(q, fwd.cuda(), n_pad)         # and gather_rows(out_p, inv.cuda(), N)
"""
from __future__ import annotations

import ctypes
from dataclasses import dataclass

import torch

from . import _ffi
from ._ffi import BsaError, BsaMask

__all__ = ["BsaError", "PackedMask", "pack_mask", "pack_mask_from_threshold",
           "threshold_resize", "predict_top_p", "tile_permute", "tile_unpermute", "hilbert_order", "tile_order",
           "order_tables", "gather_rows", "forward", "attention_host", "device_error",
           "version"]


def _stream(device: torch.device) -> ctypes.c_void_p:
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _require_cuda(t: torch.Tensor, name: str, dtype: torch.dtype | None = None) -> None:
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")


def version() -> int:
    return _ffi.load().bsa_version()


@dataclass
class PackedMask:
    """Device tensors produced by bsa_pack_mask (see include/bsa.h)."""
    bits: torch.Tensor         # uint32 as int32 [B, H, nb_q, words]
    counts: torch.Tensor       # int32 [B*H*nb_q]
    row_offsets: torch.Tensor  # int32 [B*H*nb_q + 1]
    col_idx: torch.Tensor | None  # int32 [B*H*nb_q*nb_k] (valid prefix row_offsets[-1])
    schedule: torch.Tensor     # int32 [B*H*nb_q]
    B: int
    H: int
    nb_q: int
    nb_k: int

    @property
    def words(self) -> int:
        return (self.nb_k + 31) // 32

    def as_c(self) -> BsaMask:
        return BsaMask(self.bits.data_ptr(), self.counts.data_ptr(), self.row_offsets.data_ptr(),
                       self.col_idx.data_ptr() if self.col_idx is not None else None,
                       self.schedule.data_ptr(), self.B, self.H, self.nb_q, self.nb_k,
                       self.words)


def _packed_outputs(B, H, nb_q, nb_k, dev, with_lists):
    words = (nb_k + 31) // 32
    rows = B * H * nb_q
    return PackedMask(
        torch.empty((B, H, nb_q, words), dtype=torch.int32, device=dev),
        torch.empty(rows, dtype=torch.int32, device=dev),
        torch.empty(rows + 1, dtype=torch.int32, device=dev),
        torch.empty(max(rows * nb_k, 1), dtype=torch.int32, device=dev) if with_lists else None,
        torch.empty(rows, dtype=torch.int32, device=dev), B, H, nb_q, nb_k)


def _pack_pointers(pm: PackedMask):
    return (pm.bits.data_ptr(), pm.counts.data_ptr(), pm.row_offsets.data_ptr(),
            pm.col_idx.data_ptr() if pm.col_idx is not None else None, pm.schedule.data_ptr())


def pack_mask(dense: torch.Tensor, with_lists: bool = True) -> PackedMask:
    """dense uint8 [B, H, nb_q, nb_k] on the GPU -> PackedMask (bsa_pack_mask)."""
    _require_cuda(dense, "dense", torch.uint8)
    if dense.dim() != 4:
        raise ValueError("dense must be [B, H, nb_q, nb_k]")
    B, H, nb_q, nb_k = dense.shape
    lib = _ffi.load()
    dev = dense.device
    pm = _packed_outputs(B, H, nb_q, nb_k, dev, with_lists)
    ws_bytes = lib.bsa_pack_mask_workspace(B, H, nb_q, nb_k)
    ws = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device=dev)
    st = lib.bsa_pack_mask(dense.data_ptr(), B, H, nb_q, nb_k, *_pack_pointers(pm),
                           ws.data_ptr(), ws.numel(), _stream(dev))
    _ffi.check(st, "bsa_pack_mask")
    return pm


def pack_mask_from_threshold(thr: torch.Tensor, p: torch.Tensor, B: int = 1,
                             with_lists: bool = True) -> PackedMask:
    """Threshold map fp32 [H, nb_q, nb_k] and per-head thresholds fp32 [H], both on
    the GPU -> PackedMask of M_p = 1(thr <= p[h]) for B batch items
    (bsa_pack_mask_from_threshold)."""
    _require_cuda(thr, "thr", torch.float32)
    _require_cuda(p, "p", torch.float32)
    if thr.dim() != 3:
        raise ValueError("thr must be [H, nb_q, nb_k]")
    H, nb_q, nb_k = thr.shape
    if p.shape != (H,):
        raise ValueError("p must be [H]")
    lib = _ffi.load()
    dev = thr.device
    pm = _packed_outputs(int(B), H, nb_q, nb_k, dev, with_lists)
    ws_bytes = lib.bsa_pack_mask_workspace(int(B), H, nb_q, nb_k)
    ws = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device=dev)
    st = lib.bsa_pack_mask_from_threshold(thr.data_ptr(), p.data_ptr(), int(B), H, nb_q, nb_k,
                                          *_pack_pointers(pm), ws.data_ptr(), ws.numel(),
                                          _stream(dev))
    _ffi.check(st, "bsa_pack_mask_from_threshold")
    return pm


def threshold_resize(src: torch.Tensor, tq: int, tk: int,
                     out: torch.Tensor | None = None) -> torch.Tensor:
    """Threshold map fp32 [H, sq, sk] on the GPU -> fp32 [H, tq, tk] by the
    conservative resize of Eq. 7 (bsa_threshold_resize)."""
    _require_cuda(src, "src", torch.float32)
    if src.dim() != 3:
        raise ValueError("src must be [H, sq, sk]")
    H, sq, sk = src.shape
    if out is None:
        out = torch.empty((H, int(tq), int(tk)), dtype=torch.float32, device=src.device)
    _require_cuda(out, "out", torch.float32)
    if out.shape != (H, tq, tk):
        raise ValueError("out must be [H, tq, tk]")
    st = _ffi.load().bsa_threshold_resize(src.data_ptr(), H, sq, sk, out.data_ptr(), int(tq),
                                          int(tk), _stream(src.device))
    _ffi.check(st, "bsa_threshold_resize")
    return out


def _grid_args(grid, tile):
    T, Hs, Ws = (int(x) for x in grid)
    tt, th, tw = (int(x) for x in tile)
    return T, Hs, Ws, tt, th, tw


def tile_permute(x: torch.Tensor, grid, tile, n_pad: int, out: torch.Tensor | None = None):
    """[B, H, T*Hs*Ws, d] bf16 frame-major -> [B, H, n_pad, d] tile-major (bsa_tile_permute)."""
    _require_cuda(x, "x", torch.bfloat16)
    B, H, N, d = x.shape
    T, Hs, Ws, tt, th, tw = _grid_args(grid, tile)
    if N != T * Hs * Ws:
        raise ValueError("token count does not match the grid")
    if out is None:
        out = torch.empty((B, H, n_pad, d), dtype=x.dtype, device=x.device)
    _require_cuda(out, "out", torch.bfloat16)
    st = _ffi.load().bsa_tile_permute(x.data_ptr(), out.data_ptr(), B, H, T, Hs, Ws, d, tt, th,
                                      tw, n_pad, _stream(x.device))
    _ffi.check(st, "bsa_tile_permute")
    return out


def tile_unpermute(y: torch.Tensor, grid, tile, out: torch.Tensor | None = None):
    """[B, H, n_pad, d] bf16 tile-major -> [B, H, T*Hs*Ws, d] frame-major (bsa_tile_unpermute)."""
    _require_cuda(y, "y", torch.bfloat16)
    B, H, n_pad, d = y.shape
    T, Hs, Ws, tt, th, tw = _grid_args(grid, tile)
    if out is None:
        out = torch.empty((B, H, T * Hs * Ws, d), dtype=y.dtype, device=y.device)
    _require_cuda(out, "out", torch.bfloat16)
    st = _ffi.load().bsa_tile_unpermute(y.data_ptr(), out.data_ptr(), B, H, T, Hs, Ws, d, tt, th,
                                        tw, n_pad, _stream(y.device))
    _ffi.check(st, "bsa_tile_unpermute")
    return out


def predict_top_p(q: torch.Tensor, k: torch.Tensor, n_valid: int, block: int,
                  tau: torch.Tensor, top_p: torch.Tensor, with_lists: bool = True) -> PackedMask:
    """Online top-p block mask of block-ordered q, k [B, H, n_pad, d] bf16 with
    per-head tau and top_p (fp32 [H] on the GPU) -> PackedMask (bsa_predict_top_p)."""
    _require_cuda(q, "q", torch.bfloat16)
    _require_cuda(k, "k", torch.bfloat16)
    _require_cuda(tau, "tau", torch.float32)
    _require_cuda(top_p, "top_p", torch.float32)
    B, H, n_pad, d = q.shape
    if k.shape != q.shape:
        raise ValueError("q and k shapes differ")
    if tau.shape != (H,) or top_p.shape != (H,):
        raise ValueError("tau and top_p must be [H]")
    nb = n_pad // block
    lib = _ffi.load()
    pm = _packed_outputs(B, H, nb, nb, q.device, with_lists)
    ws_bytes = lib.bsa_predict_top_p_workspace(B, H, n_pad, d, block)
    ws = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device=q.device)
    st = lib.bsa_predict_top_p(q.data_ptr(), k.data_ptr(), B, H, int(n_valid), n_pad, d,
                               int(block), tau.data_ptr(), top_p.data_ptr(), *_pack_pointers(pm),
                               ws.data_ptr(), ws.numel(), _stream(q.device))
    _ffi.check(st, "bsa_predict_top_p")
    return pm


def _host_i32(n: int) -> torch.Tensor:
    return torch.empty(n, dtype=torch.int32)


def hilbert_order(T: int, Hs: int, Ws: int) -> torch.Tensor:
    """Host int32 [T*Hs*Ws]: frame-major token index at each position of the 3-D
    Hilbert-curve order (bsa_hilbert_order)."""
    order = _host_i32(T * Hs * Ws)
    _ffi.check(_ffi.load().bsa_hilbert_order(T, Hs, Ws, order.data_ptr()), "bsa_hilbert_order")
    return order


def tile_order(T: int, Hs: int, Ws: int, tt: int, th: int, tw: int) -> torch.Tensor:
    """Host int32 [T*Hs*Ws]: the tile order of bsa_tile_permute as a table (bsa_tile_order)."""
    order = _host_i32(T * Hs * Ws)
    _ffi.check(_ffi.load().bsa_tile_order(T, Hs, Ws, tt, th, tw, order.data_ptr()),
               "bsa_tile_order")
    return order


def order_tables(order: torch.Tensor, n_pad: int):
    """Host order int32 [n] -> host gather tables (fwd int32 [n_pad], inv int32 [n])
    (bsa_order_tables).  Stack per-head tables into [H, n_pad] for gather_rows."""
    order = order.to(torch.int32).contiguous()
    if order.is_cuda or order.dim() != 1:
        raise ValueError("order must be a 1-D host tensor")
    n = order.numel()
    fwd, inv = _host_i32(n_pad), _host_i32(n)
    _ffi.check(_ffi.load().bsa_order_tables(order.data_ptr(), n, int(n_pad), fwd.data_ptr(),
                                            inv.data_ptr()), "bsa_order_tables")
    return fwd, inv


def gather_rows(x: torch.Tensor, src: torch.Tensor, n_out: int | None = None,
                out: torch.Tensor | None = None) -> torch.Tensor:
    """[B, H, n_in, d] bf16 -> [B, H, n_out, d]: row i of each head is row src[i]
    (src [n_out] shared, or [H, n_out] per head, int32 on the GPU); entries
    outside [0, n_in) give zero rows (bsa_gather_rows)."""
    _require_cuda(x, "x", torch.bfloat16)
    _require_cuda(src, "src", torch.int32)
    B, H, n_in, d = x.shape
    per_head = 1 if src.dim() == 2 else 0
    if per_head and src.shape[0] != H:
        raise ValueError("a per-head table must be [H, n_out]")
    n_tab = src.shape[-1]
    n_out = n_tab if n_out is None else int(n_out)
    if n_out != n_tab:
        raise ValueError("n_out must match the table length")
    if out is None:
        out = torch.empty((B, H, n_out, d), dtype=x.dtype, device=x.device)
    _require_cuda(out, "out", torch.bfloat16)
    st = _ffi.load().bsa_gather_rows(x.data_ptr(), out.data_ptr(), B, H, n_in, n_out, d,
                                     src.data_ptr(), per_head, _stream(x.device))
    _ffi.check(st, "bsa_gather_rows")
    return out


def forward(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, mask: PackedMask, n_valid: int,
            block: int, softmax_scale: float | None = None, out: torch.Tensor | None = None,
            lse: torch.Tensor | None = None, block_k: int | None = None):
    """Block-sparse attention forward (bsa_forward, or bsa_forward_blocks when
    block_k differs from block) on tile-major q, k, v [B, H, n_pad, d] bf16.

    Returns (out bf16 [B, H, n_pad, d], lse fp32 [B, H, n_pad])."""
    for t, name in ((q, "q"), (k, "k"), (v, "v")):
        _require_cuda(t, name, torch.bfloat16)
    B, H, n_pad, d = q.shape
    if k.shape != q.shape or v.shape != q.shape:
        raise ValueError("q, k, v shapes differ")
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, H, n_pad), dtype=torch.float32, device=q.device)
    _require_cuda(out, "out", torch.bfloat16)
    _require_cuda(lse, "lse", torch.float32)
    cm = mask.as_c()
    lib = _ffi.load()
    if block_k is None or int(block_k) == int(block):
        st = lib.bsa_forward(q.data_ptr(), k.data_ptr(), v.data_ptr(), ctypes.byref(cm),
                             out.data_ptr(), lse.data_ptr(), B, H, int(n_valid), n_pad, d,
                             int(block), float(softmax_scale or 0.0), _stream(q.device))
        _ffi.check(st, "bsa_forward")
    else:
        st = lib.bsa_forward_blocks(q.data_ptr(), k.data_ptr(), v.data_ptr(), ctypes.byref(cm),
                                    out.data_ptr(), lse.data_ptr(), B, H, int(n_valid), n_pad, d,
                                    int(block), int(block_k), float(softmax_scale or 0.0),
                                    _stream(q.device))
        _ffi.check(st, "bsa_forward_blocks")
    return out, lse


def attention_host(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, mask: torch.Tensor, grid,
                   tile, block: int, softmax_scale: float | None = None,
                   heads_per_chunk: int = 0, out: torch.Tensor | None = None,
                   lse: torch.Tensor | None = None, device: torch.device | None = None):
    """The whole path from host tensors to host tensors on the current (or given)
    GPU, copies overlapped with the kernels (bsa_attention_host).

    q, k, v: host bf16 [B, H, T*Hs*Ws, d] frame-major (pinned for overlap);
    mask: host uint8 [B, H, nb, nb].  Returns (out host bf16 [B, H, N, d]
    frame-major, lse host fp32 [B, H, n_pad] tile-major); both are complete once
    the current stream has finished."""
    for t, name in ((q, "q"), (k, "k"), (v, "v")):
        if t.is_cuda or t.dtype != torch.bfloat16 or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous host bf16 tensor")
    if mask.is_cuda or mask.dtype != torch.uint8 or not mask.is_contiguous():
        raise ValueError("mask must be a contiguous host uint8 tensor")
    B, H, N, d = q.shape
    T, Hs, Ws, tt, th, tw = _grid_args(grid, tile)
    if N != T * Hs * Ws or k.shape != q.shape or v.shape != q.shape:
        raise ValueError("q, k, v must be [B, H, T*Hs*Ws, d]")
    n_pad = -(-N // block) * block
    dev = device if device is not None else torch.device("cuda", torch.cuda.current_device())
    if out is None:
        out = torch.empty_like(q, pin_memory=q.is_pinned())
    if lse is None:
        lse = torch.empty((B, H, n_pad), dtype=torch.float32, pin_memory=q.is_pinned())
    lib = _ffi.load()
    ws_bytes = lib.bsa_attention_host_workspace(B, H, T, Hs, Ws, d, int(block), int(heads_per_chunk))
    ws = torch.empty(max(ws_bytes, 256), dtype=torch.uint8, device=dev)
    st = lib.bsa_attention_host(q.data_ptr(), k.data_ptr(), v.data_ptr(), mask.data_ptr(),
                                out.data_ptr(), lse.data_ptr(), B, H, T, Hs, Ws, d, tt, th, tw,
                                int(block), float(softmax_scale or 0.0), int(heads_per_chunk),
                                ws.data_ptr(), ws.numel(), _stream(dev))
    _ffi.check(st, "bsa_attention_host")
    # the workspace must outlive the queued work: keep it until the stream drains
    ws.record_stream(torch.cuda.current_stream(dev))
    return out, lse


def device_error() -> int:
    """Reads and clears the device error word (BSA_ERR_TIMEOUT after a barrier timeout)."""
    code = ctypes.c_int(0)
    _ffi.check(_ffi.load().bsa_get_device_error(ctypes.byref(code)), "bsa_get_device_error")
    return code.value
