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


# ---------------------------------------------------------------- schedule
# Any work order gives the same attention output, so the schedule has several
# correct values.  The oracle fixes one of them (count descending, ties by row
# id); the library may instead take that order head by head.  A schedule is
# valid when it is one of these two orders.  Which one the library picks is
# its own policy, stated here (and in the pack kernels) and tested as such.

def head_major_order(counts: np.ndarray, nb_q: int) -> np.ndarray:
    """Heads ascending; inside a head, count descending, ties by row id."""
    counts = np.asarray(counts).reshape(-1)
    order = sorted(range(counts.size), key=lambda r: (r // nb_q, -int(counts[r]), r))
    return np.array(order, dtype=np.int32)


def schedule_form(sched: np.ndarray, counts: np.ndarray, nb_q: int) -> str:
    """'count' or 'head' for a valid schedule; fails the test otherwise."""
    import oracle
    sched = np.asarray(sched).reshape(-1)
    counts = np.asarray(counts).reshape(-1)
    assert sched.size == counts.size
    assert np.array_equal(np.sort(sched), np.arange(counts.size)), "not a permutation of the rows"
    if np.array_equal(sched, oracle.schedule(counts)):
        return "count"
    assert np.array_equal(sched, head_major_order(counts, nb_q)), \
        "neither the count order nor the count order taken per head"
    return "head"


POLICY_WINDOW = 148      # one wave of a B200: one tile per SM
POLICY_KEY_BLOCK_BYTES = 2 * 128 * 128 * 2  # K and V of a 128-token key block, d = 128, bf16
POLICY_LIMIT = 8192      # heads and rows per head beyond which the check is skipped


def device_l2_bytes() -> int:
    import torch
    return int(torch.cuda.get_device_properties(torch.cuda.current_device()).L2_cache_size)


def policy_form(counts: np.ndarray, nb_q: int, nb_k: int, l2_bytes: int) -> str:
    """The library's rule: over the count order's full windows of 148 entries,
    count the distinct heads of each window; when that many heads' K and V
    (nb_k key blocks each) exceed the L2 capacity on average, take the order
    head by head."""
    import oracle
    counts = np.asarray(counts, dtype=np.int32).reshape(-1)
    heads = counts.size // nb_q
    windows = counts.size // POLICY_WINDOW
    if windows == 0 or heads > POLICY_LIMIT or nb_q > POLICY_LIMIT:
        return "count"
    order = oracle.schedule(counts)[: windows * POLICY_WINDOW].reshape(windows, POLICY_WINDOW)
    distinct = sum(len(set((row // nb_q).tolist())) for row in order)
    return ("head" if distinct * nb_k * POLICY_KEY_BLOCK_BYTES > windows * l2_bytes
            else "count")


def check_schedule(sched: np.ndarray, counts: np.ndarray, nb_q: int, nb_k: int,
                   l2_bytes: int | None = None) -> str:
    """Valid, and the form the library's policy picks (L2 size of the current
    device unless given)."""
    form = schedule_form(sched, counts, nb_q)
    l2 = device_l2_bytes() if l2_bytes is None else l2_bytes
    assert form == policy_form(counts, nb_q, nb_k, l2), (form, policy_form(counts, nb_q, nb_k, l2))
    return form
