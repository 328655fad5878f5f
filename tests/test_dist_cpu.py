"""Multi-rank host logic on the CPU (gloo, world size 2): no GPU needed.

The W8A8 linear layer shards over tokens: the per-token quantizer and each
output row depend only on that token, so ranks that each process their own
tokens against a replicated weight need no data-path collective.  These
tests check that property on the CPU oracle across two gloo ranks, the
token split the benchmark uses, and the max-over-ranks reduction of the
timed region."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
import workloads


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out_dir):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import oracle
        wl = workloads.WORKLOADS["tiny"]
        # every rank: its own token batch, the same (replicated) weight
        d = workloads.make(wl, rows=bench.rank_token_rows(wl.M, rank))
        wq, sw = oracle.quantize_weight(d["w"])
        out, xq, sa, acc = oracle.linear(d["x"], wq, sw, d["bias"], nthreads=1)
        # gather only to check the result: the layer itself needs no exchange
        got = [torch.empty(out.shape, dtype=torch.int32) for _ in range(world)]
        dist.all_gather(got, torch.from_numpy(out.astype(np.int32)))
        t = bench.max_over_ranks(float(rank + 1) * 1.5)
        if rank == 0:
            np.save(os.path.join(out_dir, "gathered.npy"), torch.cat(got).numpy())
            np.save(os.path.join(out_dir, "tmax.npy"), np.array([t]))
    finally:
        dist.destroy_process_group()


def test_token_split_is_exact_partition():
    for M, world in [(4096, 2), (4096, 8), (9216, 3), (7, 4)]:
        rows = [workloads.shard_rows(M, world, r) for r in range(world)]
        covered = np.concatenate([np.arange(M)[s] for s in rows])
        assert np.array_equal(covered, np.arange(M))
        sizes = [s.stop - s.start for s in rows]
        assert max(sizes) - min(sizes) <= 1
    # the benchmark's weak-scaling batches are disjoint, contiguous token ranges
    assert bench.rank_token_rows(4096, 0) == slice(0, 4096)
    assert bench.rank_token_rows(4096, 3) == slice(12288, 16384)


def test_seeded_rows_do_not_depend_on_the_split():
    a = workloads.gen_activations(300, 64, 11)
    b = workloads.gen_activations(100, 64, 11, row_offset=200)
    assert np.array_equal(a[200:300], b)


def test_two_gloo_ranks_match_one_process(tmp_path):
    world = 2
    mp.spawn(_worker, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True)
    import oracle
    wl = workloads.WORKLOADS["tiny"]
    d = workloads.make(wl, rows=slice(0, world * wl.M))
    wq, sw = oracle.quantize_weight(d["w"])
    want, *_ = oracle.linear(d["x"], wq, sw, d["bias"], nthreads=1)
    got = np.load(tmp_path / "gathered.npy")
    assert np.array_equal(got.astype(np.uint16), want)
    assert float(np.load(tmp_path / "tmax.npy")[0]) == pytest.approx(3.0)
