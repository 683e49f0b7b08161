"""Seeded synthetic inputs shaped like the pages' video-DiT workloads.

This module only draws random numbers and builds block masks: it holds none of
the attention, packing or permutation arithmetic, so both the CUDA path and the
CPU oracle can take their inputs from it.

Workloads (token grids from "ScalingAttention" Sec. 5.1 and PSA's 768x1280
HunyuanVideo setting):

- ``tiny``          B=1, H=2,  d=64,  grid 4x16x16,  tile 1x8x8,  block 64
- ``wan13b_480p``   B=1, H=12, d=128, grid 21x30x52, tile 1x8x16, block 128
- ``wan14b_480p``   B=1, H=40, d=128, grid 21x30x52, tile 1x8x16, block 128
- ``wan14b_720p``   B=1, H=40, d=128, grid 21x45x80, tile 2x8x8,  block 128
- ``hunyuan_768p``  B=1, H=24, d=128, grid 33x48x80, tile 1x8x16, block 128

Block coordinates used by the mask generators.  The blocks index the
tile-major (permuted) token order, where ragged edge tiles are concatenated,
so a block is not always one tile.  The generators therefore give block i the
coordinate (slab, spatial) with slab = floor(i * n_slabs / nb) (n_slabs =
ceil(T / tile_t)) and spatial = i - (first block of that slab).  The top-p
generator pools q and k over each block's tokens; its grid is a whole number
of block-sized tiles, so a reshape groups the frame-major tokens into those
tiles.  This only shapes the synthetic masks (both the kernels and the oracle
consume the same mask); the kernels treat every mask alike.
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import numpy as np
import torch


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    d: int
    T: int
    Hs: int
    Ws: int
    tt: int
    th: int
    tw: int
    block: int
    seed: int
    mask_kind: str

    @property
    def n(self) -> int:
        return self.T * self.Hs * self.Ws

    @property
    def n_pad(self) -> int:
        return -(-self.n // self.block) * self.block

    @property
    def nb(self) -> int:
        return self.n_pad // self.block

    @property
    def n_slabs(self) -> int:
        return -(-self.T // self.tt)


WORKLOADS = {
    "tiny": Workload("tiny", 1, 2, 64, 4, 16, 16, 1, 8, 8, 64, 20260001, "bernoulli_half"),
    "wan13b_480p": Workload("wan13b_480p", 1, 12, 128, 21, 30, 52, 1, 8, 16, 128, 20260002,
                            "band_stripe"),
    "wan14b_480p": Workload("wan14b_480p", 1, 40, 128, 21, 30, 52, 1, 8, 16, 128, 20260003,
                            "bernoulli_heads"),
    "wan14b_720p": Workload("wan14b_720p", 1, 40, 128, 21, 45, 80, 2, 8, 8, 128, 20260004,
                            "psa_stripes"),
    "hunyuan_768p": Workload("hunyuan_768p", 1, 24, 128, 33, 48, 80, 1, 8, 16, 128, 20260005,
                             "top_p"),
}


def custom_workload(name, B, H, d, T, Hs, Ws, tt, th, tw, block, seed, mask_kind) -> Workload:
    return Workload(name, B, H, d, T, Hs, Ws, tt, th, tw, block, seed, mask_kind)


# --------------------------------------------------------------------------
# Q, K, V
# --------------------------------------------------------------------------
def gen_qkv(w: Workload, seed: int | None = None):
    """Frame-major bf16 q, k, v of shape [B, H, N, d] on the CPU."""
    seed = w.seed if seed is None else seed
    g = torch.Generator(device="cpu").manual_seed(seed)
    shape = (w.B, w.H, w.n, w.d)
    out = []
    for name in ("q", "k", "v"):
        x = torch.randn(shape, generator=g, dtype=torch.float32)
        if w.mask_kind == "band_stripe" and name in ("q", "k"):
            x.mul_(0.5)  # Wan2.1-1.3B-shaped inputs: Q and K scaled by 0.5
        if w.mask_kind == "bernoulli_heads" and name == "k":
            # per-head outlier keys: 1 % of key positions at 5x scale
            n_out = max(1, w.n // 100)
            for b in range(w.B):
                for h in range(w.H):
                    pos = torch.randperm(w.n, generator=g)[:n_out]
                    x[b, h, pos] *= 5.0
        out.append(x.to(torch.bfloat16))
    return tuple(out)


# --------------------------------------------------------------------------
# Block masks, uint8 [B, H, nb, nb], 1 = kept
# --------------------------------------------------------------------------
def block_coords(nb: int, n_slabs: int):
    i = np.arange(nb, dtype=np.int64)
    slab = (i * n_slabs) // nb
    first = -((-slab * nb) // n_slabs)  # ceil(slab * nb / n_slabs)
    return slab, i - first


def _force_diag(m: np.ndarray) -> np.ndarray:
    idx = np.arange(m.shape[-1])
    m[..., idx, idx] = 1
    return m


def _mask_bernoulli_half(w: Workload, rng: np.random.Generator) -> np.ndarray:
    m = (rng.random((w.B, w.H, w.nb, w.nb)) < 0.5).astype(np.uint8)
    return _force_diag(m)


def _mask_band_stripe(w: Workload, rng: np.random.Generator) -> np.ndarray:
    """Diagonal + temporal band of width 3 + spatial stripes of stride 3."""
    slab, sp = block_coords(w.nb, w.n_slabs)
    dslab = slab[None, :] - slab[:, None]
    ds = sp[None, :] - sp[:, None]
    m = np.zeros((w.B, w.H, w.nb, w.nb), dtype=np.uint8)
    for h in range(w.H):
        o_h = h % 3
        keep = (np.abs(dslab) <= 1) | ((np.mod(ds, 3) == o_h) & (np.mod(dslab, 2) == 0))
        m[:, h] = keep.astype(np.uint8)
    return _force_diag(m)


def _mask_bernoulli_heads(w: Workload, rng: np.random.Generator) -> np.ndarray:
    """20 % of heads fully dense; the rest Bernoulli(rho_h), rho_h ~ U[0.10, 0.60]."""
    m = np.zeros((w.B, w.H, w.nb, w.nb), dtype=np.uint8)
    n_full = max(1, round(0.2 * w.H))
    full = set(rng.choice(w.H, size=n_full, replace=False).tolist())
    for b in range(w.B):
        for h in range(w.H):
            if h in full:
                m[b, h] = 1
            else:
                rho = rng.uniform(0.10, 0.60)
                m[b, h] = (rng.random((w.nb, w.nb)) < rho).astype(np.uint8)
    return _force_diag(m)


def _stripe(delta: np.ndarray, width: int, offset: int, stride: float) -> np.ndarray:
    """Keep where (delta - offset) mod stride lies in `width` consecutive residues
    centred on 0; an infinite stride is one band |delta - offset| <= width // 2."""
    x = delta - offset
    if math.isinf(stride):
        return np.abs(x) <= width // 2
    stride = int(stride)
    if width >= stride:
        return np.ones_like(x, dtype=bool)
    r = np.mod(x, stride)
    half = width // 2
    return (r <= half) | (r >= stride - (width - 1 - half))


def _mask_psa_stripes(w: Workload, rng: np.random.Generator) -> np.ndarray:
    """Per-head temporal band x spatial stripe, widths/strides from PSA's tables."""
    slab, sp = block_coords(w.nb, w.n_slabs)
    dslab = slab[None, :] - slab[:, None]
    ds = sp[None, :] - sp[:, None]
    best = None
    for _ in range(1000):
        m = np.zeros((w.B, w.H, w.nb, w.nb), dtype=np.uint8)
        for b in range(w.B):
            for h in range(w.H):
                tw_ = int(rng.choice([1, 5, 7]))
                sw_ = int(rng.choice([1, 3, 10]))
                ss_ = int(rng.choice([1, 3, 6]))
                keep = _stripe(dslab, tw_, 0, math.inf) & _stripe(ds, sw_, 0, ss_)
                m[b, h] = keep.astype(np.uint8)
        m = _force_diag(m)
        sparsity = 1.0 - m.mean()
        if 0.70 <= sparsity <= 0.80:
            return m
        if best is None or abs(sparsity - 0.75) < abs(1.0 - best.mean() - 0.75):
            best = m
    return best


def _tile_means(x: torch.Tensor, w: Workload) -> torch.Tensor:
    """Mean of each 3-D tile of a frame-major [T*Hs*Ws, d] tensor, tiles in
    (tile_t, tile_y, tile_x) row-major order: [nb, d] fp64.  Only for grids the
    tile divides, with one tile per block (a reshape groups the tokens)."""
    t = x.double().view(w.T // w.tt, w.tt, w.Hs // w.th, w.th, w.Ws // w.tw, w.tw, w.d)
    return t.mean(dim=(1, 3, 5)).reshape(-1, w.d)


def _mask_top_p(w: Workload, rng: np.random.Generator, q: torch.Tensor, k: torch.Tensor,
                p: float = 0.9) -> np.ndarray:
    """Top-p block masks from mean-pooled q/k block scores, temperature per head
    found by bisection so that the head's sparsity hits a target ~ U[0.80, 0.95].

    Pooling runs over the tokens of each attention block, that is over each
    3-D tile of the token grid (the blocks the kernels walk); the grid must be
    a whole number of tiles of `block` tokens each.
    """
    if (w.T % w.tt or w.Hs % w.th or w.Ws % w.tw or w.tt * w.th * w.tw != w.block):
        raise ValueError("top-p masks need a grid of whole tiles of one block each")
    m = np.zeros((w.B, w.H, w.nb, w.nb), dtype=np.uint8)
    nb = w.nb
    for b in range(w.B):
        for h in range(w.H):
            qbar = _tile_means(q[b, h], w)
            kbar = _tile_means(k[b, h], w)
            raw = (qbar @ kbar.T) / math.sqrt(w.d)
            target = rng.uniform(0.80, 0.95)

            def keep_for(tau):
                prob = torch.softmax(raw / tau, dim=1)
                order = torch.argsort(-prob, dim=1, stable=True)
                sorted_p = torch.gather(prob, 1, order)
                csum = torch.cumsum(sorted_p, dim=1)
                n_keep = (csum < p).sum(dim=1) + 1
                n_keep = torch.clamp(n_keep, 1, nb)
                ranks = torch.arange(nb).unsqueeze(0)
                sel = ranks < n_keep.unsqueeze(1)
                km = torch.zeros(nb, nb, dtype=torch.bool)
                km.scatter_(1, order, sel)
                return km

            lo, hi = -12.0, 6.0  # log2 of tau
            km = keep_for(2.0 ** hi)
            for _ in range(30):
                mid = 0.5 * (lo + hi)
                km = keep_for(2.0 ** mid)
                sparsity = 1.0 - km.float().mean().item()
                if sparsity > target:
                    lo = mid  # too sparse: flatten (raise tau)
                else:
                    hi = mid
            m[b, h] = km.numpy().astype(np.uint8)
    return m


def gen_mask(w: Workload, q: torch.Tensor | None = None, k: torch.Tensor | None = None,
             seed: int | None = None) -> np.ndarray:
    seed = (w.seed if seed is None else seed) + 1000
    rng = np.random.default_rng(seed)
    if w.mask_kind == "bernoulli_half":
        return _mask_bernoulli_half(w, rng)
    if w.mask_kind == "band_stripe":
        return _mask_band_stripe(w, rng)
    if w.mask_kind == "bernoulli_heads":
        return _mask_bernoulli_heads(w, rng)
    if w.mask_kind == "psa_stripes":
        return _mask_psa_stripes(w, rng)
    if w.mask_kind == "top_p":
        if q is None or k is None:
            q, k, _ = gen_qkv(w)
        return _mask_top_p(w, rng, q, k)
    if w.mask_kind == "ones":
        return np.ones((w.B, w.H, w.nb, w.nb), dtype=np.uint8)
    if w.mask_kind == "bernoulli_sparse":
        # 10 % density, no forced diagonal: exercises empty rows too
        return (rng.random((w.B, w.H, w.nb, w.nb)) < 0.10).astype(np.uint8)
    raise ValueError(f"unknown mask kind {w.mask_kind}")


THRESHOLD_LEVELS = 20  # candidate densities 0.05, 0.10, ..., 1.00


def gen_threshold(w: Workload, seed: int | None = None):
    """Synthetic per-head threshold map and per-head density thresholds.

    Stands in for the offline Threshold Map of "ScalingAttention" Sec. 4.1.2
    (Eq. 2; built there from calibration prompts on trained weights, which are
    not available here) and for FAST's per-head choice of p (Algorithm 1).
    Recipe: thresholds live on the candidate grid k/20; head h draws
    gamma_h ~ U[0.5, 2] and block (u, v) gets ceil(20 * min(1, U^gamma_h +
    0.03 * |slab(u) - slab(v)|)) / 20 with U ~ U[0, 1), so nearby slabs become
    active at lower thresholds; diagonal blocks get the lowest level, 0.05.
    p_h is drawn from the levels 0.20 .. 0.60.

    Returns (thr float32 [H, nb, nb], p float32 [H])."""
    seed = (w.seed if seed is None else seed) + 2000
    rng = np.random.default_rng(seed)
    slab, _ = block_coords(w.nb, w.n_slabs)
    dslab = np.abs(slab[:, None] - slab[None, :]).astype(np.float64)
    levels = THRESHOLD_LEVELS
    thr = np.empty((w.H, w.nb, w.nb), dtype=np.float32)
    for h in range(w.H):
        gamma = rng.uniform(0.5, 2.0)
        score = np.minimum(1.0, rng.random((w.nb, w.nb)) ** gamma + 0.03 * dslab)
        k = np.clip(np.ceil(score * levels), 1, levels)
        np.fill_diagonal(k, 1)
        thr[h] = (k / levels).astype(np.float32)
    p = (rng.integers(4, 13, size=w.H) / levels).astype(np.float32)
    return thr, p


def gen_top_p_params(w: Workload, seed: int | None = None):
    """Per-head temperature and top-p threshold for the online top-p predictor.

    The pooled-query/key score of N(0,1) tokens scales like 1 / (block * tau),
    so tau_h = c_h / block with c_h log-uniform on [0.35, 0.7] gives masks of
    roughly 15-40 % density; top_p_h ~ U[0.85, 0.95] (per-head top-p
    thresholds).  Returns (tau float32 [H], top_p float32 [H])."""
    seed = (w.seed if seed is None else seed) + 4000
    rng = np.random.default_rng(seed)
    c = np.exp(rng.uniform(np.log(0.35), np.log(0.7), size=w.H))
    tau = (c / w.block).astype(np.float32)
    top_p = rng.uniform(0.85, 0.95, size=w.H).astype(np.float32)
    return tau, top_p


FINE_DROP = 0.3  # share of the 64-key halves of kept blocks that a finer mask drops


def gen_mask_fine(w: Workload, q: torch.Tensor | None = None, k: torch.Tensor | None = None,
                  seed: int | None = None) -> np.ndarray:
    """Mask with key blocks of w.block // 2 tokens: [B, H, nb, 2 * nb].

    The workload's own mask at w.block granularity, each kept key block split
    into its two halves and each half dropped with probability FINE_DROP (a
    finer mask keeps fewer unneeded keys: the granularity the pages name as the
    bottleneck below 40 % density); both halves of the diagonal block stay."""
    coarse = gen_mask(w, q, k, seed)
    rng = np.random.default_rng((w.seed if seed is None else seed) + 6000)
    fine = np.repeat(coarse, 2, axis=3)
    fine[rng.random(fine.shape) < FINE_DROP] = 0
    i = np.arange(w.nb)
    fine[:, :, i, 2 * i] = 1
    fine[:, :, i, 2 * i + 1] = 1
    return fine


def kept_tiles(mask: np.ndarray) -> int:
    return int(np.count_nonzero(mask))


def effective_flops(w: Workload, mask: np.ndarray) -> float:
    """4 * d * block * block per kept (query-block, key-block) tile, summed over heads
    ("ScalingAttention" Sec. 5.1: density is the fraction of active blocks)."""
    return 4.0 * w.d * w.block * w.block * kept_tiles(mask)
