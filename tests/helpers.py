"""Shared test helpers: input conversion and the parity tolerances.

Tolerances (stated for bf16 outputs against the fp64 oracle): output max-abs
2e-2 and mean-abs 2e-3, log-sum-exp 1e-3 absolute; packing and permutation
bit-exact.
"""
import numpy as np
import torch

OUT_MAX_ABS = 2e-2
OUT_MEAN_ABS = 2e-3
LSE_ABS = 1e-3


def bf16_bits(x: torch.Tensor) -> np.ndarray:
    return x.detach().to("cpu", torch.bfloat16).contiguous().view(torch.int16).numpy().view(
        np.uint16)


def stratified_query_blocks(mask: np.ndarray, per_head: int, seed: int):
    """Query blocks to check per (b, h): the most-kept, the least-kept, the last
    (tail) block, block 0 and seeded random ones, as flat (bh, qb) pairs."""
    BH = mask.shape[0] * mask.shape[1]
    nb = mask.shape[-2]  # query blocks (key blocks may be finer)
    m = mask.reshape(BH, nb, mask.shape[-1])
    counts = m.sum(-1)
    rng = np.random.default_rng(seed)
    picks = []
    for bh in range(BH):
        chosen = {int(np.argmax(counts[bh])), int(np.argmin(counts[bh])), nb - 1, 0}
        extra = max(0, per_head - len(chosen))
        chosen.update(int(x) for x in rng.choice(nb, size=min(extra, nb), replace=False))
        picks.extend((bh, qb) for qb in sorted(chosen))
    return picks


def compare_out(gpu_out: np.ndarray, ref_out: np.ndarray, gpu_lse: np.ndarray, ref_lse: np.ndarray):
    """Returns (max_abs, mean_abs, lse_max_abs); -inf lse must match exactly."""
    diff = np.abs(gpu_out.astype(np.float64) - ref_out)
    neg_ref = np.isneginf(ref_lse)
    neg_gpu = np.isneginf(gpu_lse)
    assert np.array_equal(neg_ref, neg_gpu), "rows with lse = -inf differ"
    fin = ~neg_ref
    lse_err = float(np.max(np.abs(gpu_lse[fin].astype(np.float64) - ref_lse[fin]))) if fin.any() else 0.0
    return float(diff.max()) if diff.size else 0.0, float(diff.mean()) if diff.size else 0.0, lse_err
