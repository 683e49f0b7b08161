"""Benchmark of the block-sparse attention hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

One step = the whole hot path over one batch of synthetic, seeded inputs that
are already resident in HBM: bsa_pack_mask (CRM rows, lists, schedule),
bsa_tile_permute of q, k, v, bsa_forward, bsa_tile_unpermute of the output.

metric: effective TFLOPS = 4 * d * block^2 * (kept tiles) / time, with the
step time as denominator for `value` and the forward kernel's own time for
`roofline.achieved`.  Inputs (3 x 774 MB for the default workload) are larger
than L2, so no flush is needed between steps.  The forward is timed per launch
with CUDA events, so its roofline fraction is taken against the burst bf16
peak; the line also gives it against the sustained peak and against the burst
peak scaled to the median SM clock seen during the timed steps.

With N > 1 (torchrun), the ranks split ONE problem of the workload by flat
head index (sharding.head_range): every rank packs, permutes and attends its
own heads, with no exchange between ranks (the heads are independent), so
there is no collective on the data path; the step time is the max over ranks
and `value` counts the whole problem's kept tiles (strong scaling).

After the timed steps, `next_rows` reports further steps measured on their own
(L2 flushed before each call): bsa_tile_permute and bsa_tile_unpermute of one
tensor, bsa_pack_mask_from_threshold at the workload's block grid,
bsa_threshold_resize of a 480p-grid map to it, bsa_gather_rows applying the
Hilbert-curve order and head-aware tile orders to one tensor, the online top-p
predictor bsa_predict_top_p on the workload's q and k, the forward with 64-token
key blocks under 128-token query blocks, the forward on an all-ones mask (the
speedup of the workload's mask over it, and a density sweep), PyTorch's dense
SDPA on the same tensors as context, and `by_length`: the masked forward, the
all-ones forward and dense SDPA on each of the four full-size workloads
(32,760 to 126,720 tokens).

--impl reference times the fp64 CPU oracle on the host cores on a bounded
sample of query blocks of the same workload (rank 0 only).
"""
from __future__ import annotations

import argparse
import ctypes
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from block_sparse_attention_forward_b200 import inputs as I  # noqa: E402

METRIC = "effective TFLOPS of bsa_forward on kept tiles and % of B200 bf16 peak"
UNIT = "TFLOP/s"
DEFAULT_WORKLOAD = "wan14b_720p"  # the ~75 %-sparse 720p shape the target is quoted on


def load_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            pk = json.load(f)
        return pk, "measured"
    except OSError:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, "fallback"


class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons during a window."""

    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu_index = gpu_index
        self.proc = None
        self.lines = []
        self.thread = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.QUERY}", "--format=csv,noheader,nounits",
                 "-lms", "100", "-i", str(self.gpu_index)],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.time(), line.strip()))

    def stop(self):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            if self.thread is not None:
                self.thread.join(timeout=5)

    def summary(self, t0: float, t1: float):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ts, line in self.lines:
            if not (t0 <= ts <= t1):
                continue
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for name, val in zip(names, f[5:9]):
                if val.lower().startswith("active"):
                    reasons.add(name)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


def pack_launches(heads: int, nb_q: int) -> int:
    """Kernels one pack launches: rows, histogram, scan, placement, kept-block lists,
    plus the head-mix check and the head-major pass when the schedule has at least one
    full window of 148 rows (and at most 8192 heads and 8192 rows per head)."""
    rows = heads * nb_q
    return 5 + (2 if rows >= 148 and heads <= 8192 and nb_q <= 8192 else 0)


def forward_source_digest() -> str:
    """sha256 over the forward kernel's sources (ties a DRAM capture to the code it measured)."""
    import hashlib
    h = hashlib.sha256()
    for name in ("bsa_forward.cu", "sm100_ptx.cuh"):
        with open(os.path.join(ROOT, "block_sparse_attention_forward_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def recorded_traffic(workload: str):
    """DRAM bytes per forward launch from the committed ncu capture, or None when the
    capture is missing, for another workload, or older than the kernel sources."""
    path = os.path.join(ROOT, "profiles", "bsa_forward_dram.json")
    try:
        with open(path) as f:
            rec = json.load(f)
    except (OSError, ValueError):
        return None
    if rec.get("workload") != workload or rec.get("source_sha256") != forward_source_digest():
        return None
    return float(rec["dram_bytes_read"]) + float(rec["dram_bytes_write"])


def gpu_selector(dev: torch.device) -> str:
    """nvidia-smi -i argument for this device (PCI bus id, else the CUDA index)."""
    try:
        pr = torch.cuda.get_device_properties(dev)
        return f"{pr.pci_domain_id:08X}:{pr.pci_bus_id:02X}:{pr.pci_device_id:02X}.0"
    except Exception:  # noqa: BLE001 - older torch without PCI fields
        return str(dev.index or 0)


def dist_setup(n_gpus: int):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        torch.cuda.set_device(local)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device("cuda", local))
    return world, rank, local


def _bits(x: torch.Tensor) -> np.ndarray:
    return x.contiguous().view(torch.int16).numpy().view(np.uint16)


def oracle_sample(w, q, k, v, mask, budget_s: float, seed: int, gpu_out=None, gpu_lse=None):
    """Times the oracle on whole query blocks (all rows) of the workload until
    about budget_s of CPU work; returns (tflops_equivalent, seconds, blocks, cores,
    errors).  With the GPU's tile-major output and LSE ([B, H, n_pad, d] and
    [B, H, n_pad] on the host) the same rows are compared: errors = (max abs,
    mean abs, LSE max abs, rows), else None."""
    import oracle
    BH = w.B * w.H
    perm = oracle.tile_order(w.T, w.Hs, w.Ws, w.tt, w.th, w.tw)
    m = mask.reshape(BH, w.nb, w.nb)
    rng = np.random.default_rng(seed)
    heads = rng.choice(BH, size=min(BH, 4), replace=False)
    flat = [x.reshape(BH, w.n, w.d) for x in (q, k, v)]
    per_head = {}
    for bh in heads:
        bh = int(bh)
        per_head[bh] = tuple(oracle.permute(_bits(x[bh:bh + 1]), perm, w.n_pad) for x in flat)
    flops = 0.0
    spent = 0.0
    blocks = 0
    err_max = err_sum = lse_max = 0.0
    err_n = 0
    order = [(int(bh), int(qb)) for qb in rng.permutation(w.nb) for bh in heads]
    for bh, qb in order:
        qp, kp, vp = per_head[bh]
        rows = (qb * w.block + np.arange(w.block)).astype(np.int64)
        t0 = time.perf_counter()
        ref, ref_lse = oracle.attention(qp, kp, vp, m[bh:bh + 1], w.n, w.block, rows=rows)
        spent += time.perf_counter() - t0
        flops += 4.0 * w.d * w.block * w.block * float(m[bh, qb].sum())
        blocks += 1
        if gpu_out is not None:
            got = gpu_out.reshape(BH, w.n_pad, w.d)[bh, rows].astype(np.float64)
            diff = np.abs(got - ref)
            err_max = max(err_max, float(diff.max()))
            err_sum += float(diff.sum())
            err_n += diff.size
            gl = gpu_lse.reshape(BH, w.n_pad)[bh, rows].astype(np.float64)
            fin = np.isfinite(ref_lse)
            if fin.any():
                lse_max = max(lse_max, float(np.abs(gl[fin] - ref_lse[fin]).max()))
        if spent >= budget_s:
            break
    errors = ((err_max, err_sum / max(err_n, 1), lse_max, blocks * w.block)
              if gpu_out is not None else None)
    return flops / spent / 1e12, spent, blocks, oracle.num_threads(), errors


def run_reference(args, w):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    q, k, v = I.gen_qkv(w)
    mask = I.gen_mask(w, q, k)
    per_step = max(2.0, 60.0 / max(1, args.steps + args.warmup))
    vals = []
    for i in range(args.warmup + args.steps):
        tf, spent, blocks, cores, _ = oracle_sample(w, q, k, v, mask, per_step, seed=w.seed + i)
        if i >= args.warmup:
            vals.append((tf, spent, blocks))
    value = statistics.median([x[0] for x in vals])
    sample = (f"fp64 C oracle (OpenMP) on whole query blocks of 4 seeded heads, about "
              f"{per_step:.0f} s per step ({vals[0][2]} blocks of {w.block} rows in step 1)")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1000.0 * statistics.median([x[1] for x in vals]),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": workload_config(w, mask),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }
    print(json.dumps(line), flush=True)
    return 0


def time_device_us(fn, stream, flush: torch.Tensor, iters: int = 30, warmup: int = 10) -> float:
    """Median device time in microseconds of fn() on `stream`, CUDA events around
    each call, L2 flushed (a write larger than L2) before every call."""
    for _ in range(warmup):
        fn()
    times = []
    for _ in range(iters):
        flush.zero_()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        fn()
        e1.record(stream)
        times.append((e0, e1))
    torch.cuda.synchronize()
    return statistics.median(a.elapsed_time(b) for a, b in times) * 1e3


def measure_threshold_rows(w, dev, stream, hbm_gbs: float):
    """Threshold-map rows: bsa_pack_mask_from_threshold at the workload's block grid
    and bsa_threshold_resize of a map built at the 480p grid to this grid.  Both are
    HBM-bound; algorithmic bytes = every input byte read once + every output byte
    written once."""
    import dataclasses

    import block_sparse_attention_forward_b200 as bsa
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    thr, p = I.gen_threshold(w)
    thr_d, p_d = torch.from_numpy(thr).to(dev), torch.from_numpy(p).to(dev)
    pm = bsa.pack_mask_from_threshold(thr_d, p_d, B=w.B)
    torch.cuda.synchronize(dev)
    rows = w.B * w.H * w.nb
    words = (w.nb + 31) // 32
    kept = int(pm.row_offsets[-1])
    pack_bytes = (thr.nbytes + p.nbytes + 4 * (rows * words + rows + rows + 1 + rows + kept))
    pack_us = time_device_us(lambda: bsa.pack_mask_from_threshold(thr_d, p_d, B=w.B), stream,
                             flush)
    base_w = dataclasses.replace(I.WORKLOADS["wan14b_480p"], H=w.H)
    base, _ = I.gen_threshold(base_w)
    base_d = torch.from_numpy(base).to(dev)
    dst = torch.empty((w.H, w.nb, w.nb), dtype=torch.float32, device=dev)
    resize_bytes = base.nbytes + dst.numel() * 4
    resize_us = time_device_us(lambda: bsa.threshold_resize(base_d, w.nb, w.nb, out=dst), stream,
                               flush)
    del flush

    def entry(us, nbytes, **extra):
        gbs = nbytes / (us * 1e-6) / 1e9
        return {"us": us, "bytes": nbytes, "achieved_gbs": gbs, "frac_hbm": gbs / hbm_gbs,
                "bound": "hbm", "l2": "flushed before each call", **extra}

    return {
        "pack_mask_from_threshold": entry(
            pack_us, pack_bytes, launches=pack_launches(w.B * w.H, w.nb), map=[w.H, w.nb, w.nb],
            density=kept / (rows * w.nb)),
        "threshold_resize": entry(resize_us, resize_bytes, launches=1,
                                  src=[w.H, base_w.nb, base_w.nb], dst=[w.H, w.nb, w.nb]),
    }


HEAD_TILES = [(1, 8, 16), (2, 8, 8), (4, 4, 8), (1, 16, 8)]  # synthetic head-aware shapes


def measure_order_rows(w, dev, stream, hbm_gbs: float):
    """Other token orders, applied by bsa_gather_rows to one [B, H, N, d] bf16
    tensor of the workload: the Hilbert-curve order (one table) and head-aware
    tiles (head h uses HEAD_TILES[h % 4], one table per head).  HBM-bound;
    algorithmic bytes = N rows read + n_pad rows written per head (the tables,
    4 bytes per position, are not counted)."""
    import block_sparse_attention_forward_b200 as bsa
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    g = torch.Generator().manual_seed(w.seed + 3000)
    x = torch.randn((w.B, w.H, w.n, w.d), generator=g).to(torch.bfloat16).to(dev)
    out = torch.empty((w.B, w.H, w.n_pad, w.d), dtype=torch.bfloat16, device=dev)
    hil, _ = bsa.order_tables(bsa.hilbert_order(w.T, w.Hs, w.Ws), w.n_pad)
    hil = hil.to(dev)
    per_head = torch.stack([
        bsa.order_tables(bsa.tile_order(w.T, w.Hs, w.Ws, *HEAD_TILES[h % 4]), w.n_pad)[0]
        for h in range(w.H)]).to(dev)
    row_bytes = w.d * 2
    nbytes = w.B * w.H * (w.n + w.n_pad) * row_bytes
    res = {}
    for name, table in (("permute_hilbert", hil), ("permute_head_aware", per_head)):
        us = time_device_us(lambda: bsa.gather_rows(x, table, out=out), stream, flush)
        gbs = nbytes / (us * 1e-6) / 1e9
        res[name] = {"us": us, "bytes": nbytes, "achieved_gbs": gbs, "frac_hbm": gbs / hbm_gbs,
                     "bound": "hbm", "launches": 1,
                     "l2": "flushed before each call (the tensor is also larger than L2)"}
    res["permute_head_aware"]["tiles"] = [list(t) for t in HEAD_TILES]
    del flush, x, out
    return res


def measure_predict_row(w, dev, stream, hbm_gbs: float):
    """bsa_predict_top_p on the workload's block-ordered q and k (synthetic
    per-head tau and top_p).  Roofline: HBM, algorithmic bytes = q and k read
    once (the pooled means, 24 MB at 720p, and the mask outputs are counted
    too)."""
    import block_sparse_attention_forward_b200 as bsa
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    q, k, _ = I.gen_qkv(w, seed=w.seed + 5000)
    grid, tile = (w.T, w.Hs, w.Ws), (w.tt, w.th, w.tw)
    qp = bsa.tile_permute(q.to(dev), grid, tile, w.n_pad)
    kp = bsa.tile_permute(k.to(dev), grid, tile, w.n_pad)
    del q, k
    tau, top_p = I.gen_top_p_params(w)
    tau_d, top_d = torch.from_numpy(tau).to(dev), torch.from_numpy(top_p).to(dev)
    pm = bsa.predict_top_p(qp, kp, w.n, w.block, tau_d, top_d)
    torch.cuda.synchronize(dev)
    rows = w.B * w.H * w.nb
    kept = int(pm.row_offsets[-1])
    words = (w.nb + 31) // 32
    nbytes = (2 * w.B * w.H * w.n * w.d * 2 + 2 * rows * w.d * 4
              + 4 * (rows * words + 3 * rows + 1 + kept))
    us = time_device_us(lambda: bsa.predict_top_p(qp, kp, w.n, w.block, tau_d, top_d), stream,
                        flush)
    gbs = nbytes / (us * 1e-6) / 1e9
    del flush, qp, kp
    return {"predict_top_p": {"us": us, "bytes": nbytes, "achieved_gbs": gbs,
                              "frac_hbm": gbs / hbm_gbs, "bound": "hbm",
                              "launches": 1 + pack_launches(w.B * w.H, w.nb),
                              "density": kept / (rows * w.nb), "l2": "flushed before each call"}}


def measure_finer_keys_row(w, dev, stream, peak_tflops: float):
    """bsa_forward_blocks with 128-token query blocks over 64-token key blocks on
    the workload (mask from inputs.gen_mask_fine).  Roofline: tensor; algorithmic
    work 4 * d * 128 * 64 FLOP per kept (query block, key block) pair."""
    import block_sparse_attention_forward_b200 as bsa
    if w.block != 128 or (w.n_pad - w.n) >= 64:
        return {"forward_finer_keys": None}
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    q, k, v = I.gen_qkv(w, seed=w.seed + 7000)
    mask = I.gen_mask_fine(w, seed=w.seed + 7000)
    grid, tile = (w.T, w.Hs, w.Ws), (w.tt, w.th, w.tw)
    qp, kp, vp = (bsa.tile_permute(t.to(dev), grid, tile, w.n_pad) for t in (q, k, v))
    del q, k, v
    pm = bsa.pack_mask(torch.from_numpy(mask).to(dev))
    out = torch.empty_like(qp)
    lse = torch.empty((w.B, w.H, w.n_pad), dtype=torch.float32, device=dev)
    kept = I.kept_tiles(mask)
    flops = 4.0 * w.d * w.block * (w.block // 2) * kept
    us = time_device_us(lambda: bsa.forward(qp, kp, vp, pm, w.n, w.block, out=out, lse=lse,
                                            block_k=w.block // 2), stream, flush, iters=5,
                        warmup=3)
    if bsa.device_error() != 0:
        raise RuntimeError("device error in the finer-key forward")
    tf = flops / (us * 1e-6) / 1e12
    del flush, qp, kp, vp, out
    return {"forward_finer_keys": {"block_q": w.block, "block_k": w.block // 2, "us": us,
                                   "kept_pairs": kept,
                                   "density": kept / (w.B * w.H * w.nb * 2 * w.nb),
                                   "achieved_tflops": tf, "peak": peak_tflops,
                                   "frac": tf / peak_tflops, "bound": "tensor", "launches": 1}}


def measure_dense_rows(w, dev, stream, peak_tflops: float, sparse_fwd_ms: float | None):
    """The same forward on an all-ones mask (every tile kept) on the workload's
    shapes, the speedup of the workload's mask over it (the pages compare their
    kernel with dense FlashAttention the same way), and PyTorch's dense
    scaled_dot_product_attention on the same tensors as context only."""
    import block_sparse_attention_forward_b200 as bsa
    q, k, v = I.gen_qkv(w, seed=w.seed + 8000)
    grid, tile = (w.T, w.Hs, w.Ws), (w.tt, w.th, w.tw)
    qp, kp, vp = (bsa.tile_permute(t.to(dev), grid, tile, w.n_pad) for t in (q, k, v))
    del q, k, v
    ones = torch.ones((w.B, w.H, w.nb, w.nb), dtype=torch.uint8, device=dev)
    pm = bsa.pack_mask(ones)
    out = torch.empty_like(qp)
    lse = torch.empty((w.B, w.H, w.n_pad), dtype=torch.float32, device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    us = time_device_us(lambda: bsa.forward(qp, kp, vp, pm, w.n, w.block, out=out, lse=lse),
                        stream, flush, iters=3, warmup=2)
    if bsa.device_error() != 0:
        raise RuntimeError("device error in the dense forward")
    flops = 4.0 * w.d * w.block * w.block * w.B * w.H * w.nb * w.nb
    tf = flops / (us * 1e-6) / 1e12
    res = {"forward_all_ones": {"us": us, "achieved_tflops": tf, "peak": peak_tflops,
                                "frac": tf / peak_tflops, "bound": "tensor",
                                "speedup_of_mask": (us * 1e-3 / sparse_fwd_ms)
                                if sparse_fwd_ms else None}}
    # time against density on the same shapes (Bernoulli masks, diagonal kept):
    # the pages expect time to fall in proportion to the kept blocks
    rng = np.random.default_rng(w.seed + 9000)
    sweep = []
    for dens in (0.5, 0.25, 0.10, 0.05):
        m = (rng.random((w.B, w.H, w.nb, w.nb)) < dens).astype(np.uint8)
        idx = np.arange(w.nb)
        m[:, :, idx, idx] = 1
        pm_d = bsa.pack_mask(torch.from_numpy(m).to(dev))
        us_d = time_device_us(lambda: bsa.forward(qp, kp, vp, pm_d, w.n, w.block, out=out,
                                                  lse=lse), stream, flush, iters=3, warmup=2)
        kept = float(m.mean())
        sweep.append({"density": kept, "us": us_d, "speedup_vs_all_ones": us / us_d,
                      "time_over_density_x_all_ones": us_d / (kept * us),
                      "achieved_tflops": flops * kept / (us_d * 1e-6) / 1e12})
    res["density_sweep"] = sweep
    # context only: dense attention over the N valid tokens with PyTorch's SDPA
    qd, kd, vd = (t[:, :, :w.n] for t in (qp, kp, vp))
    try:
        sdpa = torch.nn.functional.scaled_dot_product_attention
        us_t = time_device_us(lambda: sdpa(qd, kd, vd), stream, flush, iters=3, warmup=2)
        tf_t = 4.0 * w.d * w.n * w.n * w.B * w.H / (us_t * 1e-6) / 1e12
        res["torch_sdpa_dense_context"] = {"us": us_t, "achieved_tflops": tf_t,
                                           "note": "context only, not ours"}
    except RuntimeError as e:  # e.g. no fused kernel for the shape
        res["torch_sdpa_dense_context"] = {"unavailable": str(e)[:120]}
    del flush, qp, kp, vp, out
    return res


def measure_permute_row(w, dev, stream, hbm_gbs: float, x_dev: torch.Tensor):
    """bsa_tile_permute and bsa_tile_unpermute of one [B, H, N, d] bf16 tensor of the
    workload, each launch timed alone with CUDA events, L2 flushed before each call.
    HBM-bound; algorithmic bytes = N rows read + n_pad rows written per head
    (permute) and n_pad rows read + N rows written (unpermute): one read and one
    write of the tensor."""
    import block_sparse_attention_forward_b200 as bsa
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    grid, tile = (w.T, w.Hs, w.Ws), (w.tt, w.th, w.tw)
    yp = torch.empty((w.B, w.H, w.n_pad, w.d), dtype=torch.bfloat16, device=dev)
    back = torch.empty_like(x_dev)
    nbytes = w.B * w.H * (w.n + w.n_pad) * w.d * 2
    res = {}
    for name, fn in (("tile_permute", lambda: bsa.tile_permute(x_dev, grid, tile, w.n_pad, out=yp)),
                     ("tile_unpermute", lambda: bsa.tile_unpermute(yp, grid, tile, out=back))):
        us = time_device_us(fn, stream, flush)
        gbs = nbytes / (us * 1e-6) / 1e9
        res[name] = {"us": us, "bytes": nbytes, "achieved_gbs": gbs, "frac_hbm": gbs / hbm_gbs,
                     "bound": "hbm", "launches": 1, "l2": "flushed before each call"}
    if not torch.equal(back, x_dev):
        raise RuntimeError("tile_unpermute(tile_permute(x)) != x")
    del flush, yp, back
    return {"permute": res}


def measure_by_length(dev, stream, peak_tflops: float, reuse=None):
    """The pages' kernel benchmark over sequence lengths: for each full-size
    workload, the masked forward (its own mask), the forward on an all-ones mask and
    PyTorch's dense SDPA (context, not ours) on the same permuted tensors, each a
    short loop with the L2 flushed before every call.  `reuse` = (workload name, qp,
    kp, vp, packed mask, mask) skips regenerating the timed workload's inputs."""
    import block_sparse_attention_forward_b200 as bsa
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    rows = []
    sdpa = torch.nn.functional.scaled_dot_product_attention
    for name in ("wan13b_480p", "wan14b_480p", "wan14b_720p", "hunyuan_768p"):
        w = I.WORKLOADS[name]
        if reuse is not None and reuse[0] == name:
            qp, kp, vp, pm, mask = reuse[1:]
        else:
            q, k, v = I.gen_qkv(w)
            mask = I.gen_mask(w, q, k)
            grid, tile = (w.T, w.Hs, w.Ws), (w.tt, w.th, w.tw)
            qp, kp, vp = (bsa.tile_permute(t.to(dev), grid, tile, w.n_pad) for t in (q, k, v))
            del q, k, v
            pm = bsa.pack_mask(torch.from_numpy(mask).to(dev))
        out = torch.empty_like(qp)
        lse = torch.empty((w.B, w.H, w.n_pad), dtype=torch.float32, device=dev)
        kept = I.kept_tiles(mask)
        tile_flop = 4.0 * w.d * w.block * w.block
        us_m = time_device_us(lambda: bsa.forward(qp, kp, vp, pm, w.n, w.block, out=out, lse=lse),
                              stream, flush, iters=5, warmup=2)
        ones = bsa.pack_mask(torch.ones((w.B, w.H, w.nb, w.nb), dtype=torch.uint8, device=dev))
        us_1 = time_device_us(lambda: bsa.forward(qp, kp, vp, ones, w.n, w.block, out=out,
                                                  lse=lse), stream, flush, iters=3, warmup=1)
        if bsa.device_error() != 0:
            raise RuntimeError(f"device error in the forward on {name}")
        qd, kd, vd = (t[:, :, :w.n] for t in (qp, kp, vp))
        try:
            us_s = time_device_us(lambda: sdpa(qd, kd, vd), stream, flush, iters=3, warmup=1)
        except RuntimeError:
            us_s = None
        dense_flop = tile_flop * w.B * w.H * w.nb * w.nb
        tf_m = tile_flop * kept / (us_m * 1e-6) / 1e12
        rows.append({
            "workload": name, "n_tokens": w.n, "heads": w.H, "density": kept / (w.B * w.H * w.nb * w.nb),
            "masked_us": us_m, "masked_tflops": tf_m, "masked_frac": tf_m / peak_tflops,
            "all_ones_us": us_1, "all_ones_tflops": dense_flop / (us_1 * 1e-6) / 1e12,
            "sdpa_us": us_s,
            "sdpa_tflops": (4.0 * w.d * w.n * w.n * w.B * w.H / (us_s * 1e-6) / 1e12) if us_s else None,
            "all_ones_over_sdpa": (us_1 / us_s) if us_s else None,
            "masked_speedup_vs_all_ones": us_1 / us_m,
        })
        del qp, kp, vp, pm, ones, out, lse, qd, kd, vd
        torch.cuda.empty_cache()
    del flush
    return {"by_length": rows, "by_length_peak": peak_tflops}


def measure_power_loops(w, dev, seconds: float = 6.0):
    """Power, SM clock and energy per FLOP of three kernels on the workload's
    tensors, each looped for `seconds` while nvidia-smi samples every 100 ms: the
    forward with the workload's mask, the forward with an all-ones mask, and
    PyTorch's dense SDPA (context, not ours).  Under the 1 kW cap the clock settles
    where the power meets the cap, so TFLOP/s per GHz and pJ per FLOP compare the
    kernels' work per clock and per joule."""
    import block_sparse_attention_forward_b200 as bsa
    q, k, v = I.gen_qkv(w)
    mask = I.gen_mask(w, q, k)
    grid, tile = (w.T, w.Hs, w.Ws), (w.tt, w.th, w.tw)
    qp, kp, vp = (bsa.tile_permute(t.to(dev), grid, tile, w.n_pad) for t in (q, k, v))
    del q, k, v
    pm = bsa.pack_mask(torch.from_numpy(mask).to(dev))
    ones = bsa.pack_mask(torch.ones((w.B, w.H, w.nb, w.nb), dtype=torch.uint8, device=dev))
    out = torch.empty_like(qp)
    lse = torch.empty((w.B, w.H, w.n_pad), dtype=torch.float32, device=dev)
    qd, kd, vd = (t[:, :, :w.n] for t in (qp, kp, vp))
    tile_flop = 4.0 * w.d * w.block * w.block
    cases = [
        ("forward_mask", lambda: bsa.forward(qp, kp, vp, pm, w.n, w.block, out=out, lse=lse),
         tile_flop * I.kept_tiles(mask)),
        ("forward_all_ones", lambda: bsa.forward(qp, kp, vp, ones, w.n, w.block, out=out, lse=lse),
         tile_flop * w.B * w.H * w.nb * w.nb),
        ("torch_sdpa_dense", lambda: torch.nn.functional.scaled_dot_product_attention(qd, kd, vd),
         4.0 * w.d * w.n * w.n * w.B * w.H),
    ]
    res = {}
    stream = torch.cuda.current_stream(dev)
    for name, fn, flops in cases:
        for _ in range(3):
            fn()
        torch.cuda.synchronize(dev)
        sampler = PowerSampler(gpu_selector(dev))
        sampler.start()
        time.sleep(0.5)
        t0 = time.time()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        n = 0
        while time.time() - t0 < seconds:
            fn()
            n += 1
            if n % 4 == 0:
                torch.cuda.synchronize(dev)
        e1.record(stream)
        torch.cuda.synchronize(dev)
        t1 = time.time()
        sampler.stop()
        ms = e0.elapsed_time(e1) / n
        sm, watts, capped = sampler.summary(t0 + 0.5, t1)
        tf = flops / (ms * 1e-3) / 1e12
        res[name] = {"ms": ms, "tflops": tf, "sm_mhz": sm, "watts": watts,
                     "pj_per_flop": (watts / (tf * 1e12) * 1e12) if watts else None,
                     "tflops_per_ghz": (tf / sm * 1e3) if sm else None,
                     "sw_power_cap_samples": capped, "calls": n}
    if bsa.device_error() != 0:
        raise RuntimeError("device error in the power loops")
    return res


class PowerSampler(ClockSampler):
    """SM clock, power draw and the power-cap flag, sampled during a window."""

    QUERY = "clocks.sm,power.draw,clocks_event_reasons.sw_power_cap"

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.QUERY}", "--format=csv,noheader,nounits",
                 "-lms", "100", "-i", str(self.gpu_index)],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def summary(self, t0: float, t1: float):
        sm, watts, capped = [], [], 0
        for ts, line in self.lines:
            if not (t0 <= ts <= t1):
                continue
            f = [x.strip() for x in line.split(",")]
            try:
                sm.append(float(f[0]))
                watts.append(float(f[1]))
                capped += f[2].lower().startswith("active")
            except (ValueError, IndexError):
                continue
        if not sm:
            return None, None, 0
        return statistics.median(sm), statistics.median(watts), capped


def workload_config(w, mask, world: int = 1):
    kept = I.kept_tiles(mask)
    total = w.B * w.H * w.nb * w.nb
    return {"workload": w.name, "B": w.B, "H": w.H, "d": w.d, "grid": [w.T, w.Hs, w.Ws],
            "tile": [w.tt, w.th, w.tw], "block": w.block, "n_tokens": w.n, "n_pad": w.n_pad,
            "kept_tiles": kept, "density": kept / total, "mask": w.mask_kind,
            "l2": "inputs larger than L2 (no flush)",
            "parallelism": (f"heads split over {world} ranks (head_range), no exchange"
                            if world > 1 else "one GPU, all heads")}


def shard_workload(w, q, k, v, mask, world: int, rank: int):
    """This rank's heads of one problem: flat heads [lo, hi) of B*H, as a workload
    with B = 1 and H = hi - lo (every head is an independent problem)."""
    import dataclasses

    from block_sparse_attention_forward_b200.sharding import head_range
    lo, hi = head_range(w.B * w.H, world, rank)

    def flat(x):
        y = x.reshape(1, w.B * w.H, *x.shape[2:])[:, lo:hi]
        return np.ascontiguousarray(y) if isinstance(y, np.ndarray) else y.contiguous()

    ws = dataclasses.replace(w, B=1, H=hi - lo)
    return ws, flat(q), flat(k), flat(v), flat(mask), (lo, hi)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(I.WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-next", action="store_true",
                    help="skip the threshold-map rows measured after the timed steps")
    ap.add_argument("--only-next", action="store_true",
                    help="measure only the threshold-map rows (a small case for profiling)")
    ap.add_argument("--no-by-length", action="store_true",
                    help="skip the forward / all-ones / SDPA comparison over the four workloads")
    ap.add_argument("--power-loops", action="store_true",
                    help="only loop the forward (mask, all-ones) and dense SDPA for a few seconds "
                         "each and report power, SM clock and energy per FLOP")
    ap.add_argument("--sdpa-only", action="store_true",
                    help="only run dense SDPA three times on the workload's tensors (a small case "
                         "for an ncu capture of its kernel)")
    ap.add_argument("--heads", type=int, default=0,
                    help="override the head count (smaller cases for profiling captures)")
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)
    w = I.WORKLOADS[args.workload]
    if args.heads > 0:
        import dataclasses
        w = dataclasses.replace(w, H=args.heads, name=f"{w.name}_h{args.heads}")
    if args.impl == "reference":
        return run_reference(args, w)

    import block_sparse_attention_forward_b200 as bsa
    from block_sparse_attention_forward_b200 import _ffi

    world, rank, local = dist_setup(args.gpus)
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    if args.power_loops:
        res = measure_power_loops(w, dev)
        if rank == 0:
            print(json.dumps({"workload": w.name, "power_loops": res}), flush=True)
        return 0
    if args.sdpa_only:
        g = torch.Generator().manual_seed(w.seed)
        q, k, v = (torch.randn((w.B, w.H, w.n, w.d), generator=g).to(torch.bfloat16).to(dev)
                   for _ in range(3))
        for _ in range(3):
            o = torch.nn.functional.scaled_dot_product_attention(q, k, v)
        torch.cuda.synchronize(dev)
        print(json.dumps({"workload": w.name, "sdpa_only": float(o.float().abs().mean())}))
        return 0
    if args.only_next:
        peaks, _ = load_peaks()
        rows = measure_threshold_rows(w, dev, torch.cuda.current_stream(dev),
                                      float(peaks["hbm_gbs"]))
        rows.update(measure_order_rows(w, dev, torch.cuda.current_stream(dev),
                                       float(peaks["hbm_gbs"])))
        rows.update(measure_predict_row(w, dev, torch.cuda.current_stream(dev),
                                        float(peaks["hbm_gbs"])))
        pk = float(peaks["bf16_tflops"])
        rows.update(measure_finer_keys_row(w, dev, torch.cuda.current_stream(dev), pk))
        rows.update(measure_dense_rows(w, dev, torch.cuda.current_stream(dev), pk, None))
        if rank == 0:
            print(json.dumps({"workload": w.name, "next_rows": rows}), flush=True)
        if world > 1:
            torch.distributed.destroy_process_group()
        return 0
    q_all, k_all, v_all = I.gen_qkv(w)
    mask_all = I.gen_mask(w, q_all, k_all)
    w_all = w
    w, q, k, v, mask, heads = shard_workload(w_all, q_all, k_all, v_all, mask_all, world, rank)
    del q_all, k_all, v_all
    flops = I.effective_flops(w, mask)
    grid, tile = (w.T, w.Hs, w.Ws), (w.tt, w.th, w.tw)

    qd, kd, vd = q.to(dev), k.to(dev), v.to(dev)
    maskd = torch.from_numpy(mask).to(dev)
    qp = torch.empty((w.B, w.H, w.n_pad, w.d), dtype=torch.bfloat16, device=dev)
    kp, vp, out_p = torch.empty_like(qp), torch.empty_like(qp), torch.empty_like(qp)
    out = torch.empty_like(qd)
    lse = torch.empty((w.B, w.H, w.n_pad), dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)
    fwd_ev = []

    def step(record_fwd: bool):
        pm = bsa.pack_mask(maskd)
        bsa.tile_permute(qd, grid, tile, w.n_pad, out=qp)
        bsa.tile_permute(kd, grid, tile, w.n_pad, out=kp)
        bsa.tile_permute(vd, grid, tile, w.n_pad, out=vp)
        if record_fwd:
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
        bsa.forward(qp, kp, vp, pm, w.n, w.block, out=out_p, lse=lse)
        if record_fwd:
            e1.record(stream)
            fwd_ev.append((e0, e1))
        bsa.tile_unpermute(out_p, grid, tile, out=out)
        return pm

    launches_per_step = pack_launches(w.B * w.H, w.nb) + 3 + 1 + 1  # pack, permute q/k/v, forward, unpermute

    for _ in range(args.warmup):
        step(False)
    torch.cuda.synchronize(dev)
    if bsa.device_error() != 0:
        raise RuntimeError("device error during warm-up")

    sampler = ClockSampler(gpu_selector(dev))
    sampler.start()
    time.sleep(0.3)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize(dev)
    t_wall0 = time.time()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ev0.record(stream)
    for _ in range(args.steps):
        step(True)
    ev1.record(stream)
    torch.cuda.synchronize(dev)
    t_wall1 = time.time()
    if world > 1:
        torch.distributed.barrier()
    sampler.stop()
    ms_total = ev0.elapsed_time(ev1)
    fwd_ms = statistics.mean(a.elapsed_time(b) for a, b in fwd_ev)
    if bsa.device_error() != 0:
        raise RuntimeError("device error during the timed region")

    fwd_ms_local = fwd_ms  # this rank's forward, for the kernel's roofline
    t = torch.tensor([ms_total, fwd_ms, flops], dtype=torch.float64, device=dev)
    total_flops = flops
    if world > 1:
        tmax = t[:2].clone()
        torch.distributed.all_reduce(tmax, op=torch.distributed.ReduceOp.MAX)
        tf = t[2:].clone()
        torch.distributed.all_reduce(tf, op=torch.distributed.ReduceOp.SUM)
        ms_total, fwd_ms = float(tmax[0]), float(tmax[1])
        total_flops = float(tf[0])
    ms_step = ms_total / args.steps
    value = total_flops / (ms_step * 1e-3) / 1e12

    # ---------------------------------------------------------------- e2e
    e2e = None
    if not args.no_e2e:
        lib = _ffi.load()
        h_q, h_k, h_v = q.pin_memory(), k.pin_memory(), v.pin_memory()
        h_mask = torch.from_numpy(mask).pin_memory()
        h_out = torch.empty_like(q).pin_memory()
        h_lse = torch.empty((w.B, w.H, w.n_pad), dtype=torch.float32).pin_memory()
        e_steps = max(2, min(args.steps, 5))
        sp = ctypes.c_void_p(stream.cuda_stream)

        def e2e_step():
            # the public host-to-host call: per head chunk, copy in, pack, permute,
            # forward, unpermute, copy out, pipelined over three streams
            bsa.attention_host(h_q, h_k, h_v, h_mask, grid, tile, w.block, out=h_out,
                               lse=h_lse, device=dev)

        e2e_step()
        torch.cuda.synchronize(dev)
        if world > 1:
            torch.distributed.barrier()
        a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a0.record(stream)
        for _ in range(e_steps):
            e2e_step()
        a1.record(stream)
        torch.cuda.synchronize(dev)
        e_ms = a0.elapsed_time(a1) / e_steps
        te = torch.tensor([e_ms], dtype=torch.float64, device=dev)
        if world > 1:
            torch.distributed.all_reduce(te, op=torch.distributed.ReduceOp.MAX)
        e_ms = float(te[0])
        h2d = sum(x.numel() * x.element_size() for x in (h_q, h_k, h_v, h_mask))
        d2h = h_out.numel() * h_out.element_size() + h_lse.numel() * h_lse.element_size()
        e2e = {"value": total_flops / (e_ms * 1e-3) / 1e12, "unit": UNIT, "ms_per_step": e_ms,
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
               "call": "bsa_attention_host (pinned host buffers, heads in chunks of "
                       f"{-(-w.B * w.H // 16)} with one-head first and last chunks, copies "
                       "overlapped with the kernels)",
               "bound": "host-to-device copy of q, k, v and mask (PCIe)"}
        del sp

    # ---------------------------------------------------------------- roofline
    peaks, peak_src = load_peaks()
    # the forward is timed per launch (CUDA events around each call), not as a
    # seconds-long loop: the burst peak is its denominator
    peak = float(peaks["bf16_tflops"])
    peak_sus = float(peaks.get("bf16_tflops_sustained", peak))
    clocks = sampler.summary(t_wall0, t_wall1)
    next_rows = None
    if not args.no_next and world == 1:  # extra rows only at N = 1: no GPU held longer
        hbm = float(peaks["hbm_gbs"])
        next_rows = measure_permute_row(w, dev, stream, hbm, qd)
        next_rows.update(measure_threshold_rows(w, dev, stream, hbm))
        next_rows.update(measure_order_rows(w, dev, stream, hbm))
        next_rows.update(measure_predict_row(w, dev, stream, hbm))
        next_rows.update(measure_finer_keys_row(w, dev, stream, peak))
        next_rows.update(measure_dense_rows(w, dev, stream, peak, fwd_ms_local))
        if not args.no_by_length:
            pm_main = bsa.pack_mask(maskd)
            next_rows.update(measure_by_length(dev, stream, peak,
                                               reuse=(w.name, qp, kp, vp, pm_main, mask)))
    fwd_tflops = flops / (fwd_ms_local * 1e-3) / 1e12
    sm_mhz, sm_max = clocks.get("sm_mhz"), clocks.get("sm_max_mhz") or peaks.get("sm_max_mhz")
    roofline = {"bound": "tensor", "achieved": fwd_tflops, "peak": peak, "unit": "TFLOP/s",
                "frac": fwd_tflops / peak, "traffic": recorded_traffic(w.name),
                "kernel": f"bsa_forward_kernel<{w.d},{w.block},{w.block}>",
                "peak_source": f"{peak_src} bf16_tflops (burst: dense bf16 cuBLAS, best of 10)",
                "frac_sustained": fwd_tflops / peak_sus, "peak_sustained": peak_sus,
                "frac_clock_normalised": (fwd_tflops / (peak * sm_mhz / sm_max)
                                          if sm_mhz and sm_max else None),
                "fwd_ms": fwd_ms_local}

    cpu = None
    parity = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        # the last timed step's tile-major output and LSE, compared on the sampled rows
        gpu_out = out_p.float().cpu().numpy()
        gpu_lse = lse.cpu().numpy()
        tf, spent, blocks, cores, errs = oracle_sample(w, q, k, v, mask, 15.0, seed=w.seed,
                                                       gpu_out=gpu_out, gpu_lse=gpu_lse)
        cpu = {"value": tf, "unit": UNIT, "cores": cores, "kind": "oracle",
               "sample": f"{blocks} whole query blocks ({w.block} rows each) of 4 seeded heads, "
                         f"{spent:.1f} s of fp64 OpenMP oracle"}
        parity = {"rows": errs[3], "out_max_abs": errs[0], "out_mean_abs": errs[1],
                  "lse_max_abs": errs[2],
                  "tolerance": {"out_max_abs": 2e-2, "out_mean_abs": 2e-3, "lse_max_abs": 1e-3},
                  "against": "fp64 oracle on the cpu_baseline sample, last timed step's output"}

    if world > 1:
        torch.distributed.barrier()
    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
            "scaling": "strong", "vs_baseline": None, "dtype": "bf16",
            "data": f"synthetic (seeded N(0,1) bf16 q/k/v, {w.mask_kind} masks)",
            "config": workload_config(w_all, mask_all, world), "roofline": roofline,
            "cpu_baseline": cpu, "e2e": e2e, "gpu_launches": launches_per_step * args.steps,
            "clocks": clocks,
            "peak_frac_step": value / peak,
            "parity": parity,
            "next_rows": next_rows,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        torch.distributed.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
