"""Multi-rank host logic on CPU (gloo, world size 2): heads shard with no
exchange.  Each rank computes its heads' attention with the oracle; gathering
the shards reproduces the single-process result exactly."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from block_sparse_attention_forward_b200.sharding import head_range


def test_head_range_partitions():
    for total in (1, 2, 7, 40):
        for world in (1, 2, 3, 8):
            got = [head_range(total, world, r) for r in range(world)]
            assert got[0][0] == 0 and got[-1][1] == total
            assert all(a[1] == b[0] for a, b in zip(got, got[1:]))
            sizes = [hi - lo for lo, hi in got]
            assert max(sizes) - min(sizes) <= 1


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _case():
    import oracle  # noqa: F401
    rng = np.random.default_rng(0)
    BH, n, d, block = 5, 256, 16, 64
    q = rng.integers(0, 2**16, size=(BH, n, d), dtype=np.uint16) & 0x3FFF  # small finite bf16
    k = rng.integers(0, 2**16, size=(BH, n, d), dtype=np.uint16) & 0x3FFF
    v = rng.integers(0, 2**16, size=(BH, n, d), dtype=np.uint16) & 0x3FFF
    mask = (rng.random((BH, n // block, n // block)) < 0.5).astype(np.uint8)
    return q, k, v, mask, n, block


def _worker(rank, world, port, out_path):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import oracle
        q, k, v, mask, n, block = _case()
        lo, hi = head_range(q.shape[0], world, rank)
        out, lse = oracle.attention(q[lo:hi], k[lo:hi], v[lo:hi], mask[lo:hi], n, block)
        pieces = [None] * world
        dist.all_gather_object(pieces, (lo, hi, out, lse))
        if rank == 0:
            np.save(out_path, np.concatenate([p[2] for p in sorted(pieces, key=lambda t: t[0])]))
    finally:
        dist.destroy_process_group()


def test_two_rank_head_sharding_matches_single_process(tmp_path):
    import oracle
    oracle.build()
    out_path = str(tmp_path / "gathered.npy")
    port = _free_port()
    mp.start_processes(_worker, args=(2, port, out_path), nprocs=2, join=True,
                       start_method="spawn")
    gathered = np.load(out_path)
    q, k, v, mask, n, block = _case()
    ref, _ = oracle.attention(q, k, v, mask, n, block)
    np.testing.assert_array_equal(gathered, ref)


@pytest.mark.parametrize("name", ["tiny", "wan13b_480p", "wan14b_480p", "wan14b_720p",
                                  "hunyuan_768p"])
def test_rank_slices_cover_every_head_once(name):
    # bench.py --gpus N splits one problem by flat head index: for each
    # workload shape and N in 1..8 the ranks' slices cover every (b, h) once
    from block_sparse_attention_forward_b200 import inputs as I
    w = I.WORKLOADS[name]
    for world in range(1, 9):
        seen = np.zeros(w.B * w.H, dtype=np.int64)
        for rank in range(world):
            lo, hi = head_range(w.B * w.H, world, rank)
            seen[lo:hi] += 1
        assert np.all(seen == 1), (name, world)


def test_bench_shard_workload_slices_reassemble():
    # bench.py --gpus N: each rank's slice of q, k, v and mask, concatenated in
    # rank order, is the whole problem
    import importlib.util
    from block_sparse_attention_forward_b200 import inputs as I
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    spec = importlib.util.spec_from_file_location("bench_mod", os.path.join(root, "bench.py"))
    bench = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(bench)
    w = I.custom_workload("shard", 2, 3, 64, 2, 8, 8, 1, 8, 8, 64, 5, "bernoulli_half")
    q, k, v = I.gen_qkv(w)
    mask = I.gen_mask(w)
    for world in (1, 2, 4):
        parts = [bench.shard_workload(w, q, k, v, mask, world, r) for r in range(world)]
        assert sum(p[0].H for p in parts) == w.B * w.H
        got_q = torch.cat([p[1] for p in parts], dim=1).reshape(q.shape)
        got_m = np.concatenate([p[4] for p in parts], axis=1).reshape(mask.shape)
        assert torch.equal(got_q, q)
        assert np.array_equal(got_m, mask)
