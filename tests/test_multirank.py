"""Host-side multi-rank path of bench.py on two gloo ranks (CPU only).

The forward shards over independent (b, h) streams: every rank runs its own batch, and
the only collectives are the timing barrier and the max-over-ranks reduction.  These
tests run that rank logic as two spawned processes and check that sharding over streams
is exact: the union of the ranks' per-stream results equals one run over all streams.
"""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank: int, world: int, port: int, outdir: str):
    os.environ.update({"RANK": str(rank), "WORLD_SIZE": str(world), "LOCAL_RANK": str(rank),
                       "MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port)})
    sys.path.insert(0, ROOT)
    import torch.distributed as dist

    import bench
    import oracle
    import workloads

    r, n, local = bench.dist_setup("gloo")
    assert (r, n, local) == (rank, world, rank)
    # the slowest rank's time is what every rank reports
    assert bench.max_over_ranks(0.5 + r, n, device="cpu") == 0.5 + (n - 1)
    w, tokens = bench.rank_workload(r, n)
    assert tokens == bench.WORKLOAD.tokens * n
    seeds = [None] * n
    dist.all_gather_object(seeds, w.seed)
    assert len(set(seeds)) == n, "ranks must draw independent batches"

    # a small shard of each rank's streams through the oracle; gather to rank 0
    small = w.replace(B=1, H=2, T=96)
    inp = workloads.make_chunk_inputs(small)
    o, S_T = oracle.fwd(inp["q"], inp["k"], inp["v"], inp["beta"], inp["S0"], threads=1)
    shards = [None] * n
    dist.all_gather_object(shards, (small.seed, o, S_T))
    bench.barrier(n)
    if r == 0:
        np.save(os.path.join(outdir, "ok.npy"), np.array([1]))
        # the same streams in one batch of all ranks' inputs (stacked along H)
        parts = [workloads.make_chunk_inputs(small.replace(seed=s)) for s, _, _ in shards]
        cat = {k: torch.cat([p[k] for p in parts], dim=1) for k in ("q", "k", "v", "beta")}
        o_all, S_all = oracle.fwd(cat["q"], cat["k"], cat["v"], cat["beta"], None, threads=1)
        for i, (_, o_i, S_i) in enumerate(shards):
            assert np.array_equal(o_all[:, 2 * i:2 * i + 2], o_i)
            assert np.array_equal(S_all[:, 2 * i:2 * i + 2], S_i)
        np.save(os.path.join(outdir, "exact.npy"), np.array([1]))
    dist.destroy_process_group()


def test_two_gloo_ranks_shard_over_streams(tmp_path, oracle_lib):
    port = _free_port()
    mp.start_processes(_worker, args=(2, port, str(tmp_path)), nprocs=2, join=True,
                       start_method="spawn")
    assert (tmp_path / "ok.npy").exists()
    assert (tmp_path / "exact.npy").exists()


def test_single_rank_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    for k in ("RANK", "WORLD_SIZE", "LOCAL_RANK"):
        assert k not in os.environ or os.environ[k] in ("0", "1")
    assert bench.max_over_ranks(3.25, 1) == 3.25
    w, tokens = bench.rank_workload(0, 1)
    assert w == bench.WORKLOAD.replace(seed=bench.shard_seed(0))
    assert tokens == bench.WORKLOAD.tokens
