"""Multi-rank host logic on CPU (gloo, world size 2).

The path shards by batch with no exchange: every rank owns its own batch
(weak scaling).  These tests check the pieces bench.py uses across ranks --
distinct per-rank inputs, rank-independent results, max-over-ranks timing
and the whole-job aggregate -- without a GPU.
"""

import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
import oracle
from hadamard_rotation_bit_b200 import workloads as W


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        x = W.generate("c2", slice(0, 8), seed=W.rank_seed(rank))
        _, codes, scales = oracle.rotate_quant(W.bits_to_float64(x, "bf16"), 0, "int4", 128)
        digest = torch.tensor([int(codes.astype(np.int64).sum()), int(x.astype(np.int64).sum())], dtype=torch.int64)
        gathered = [torch.zeros_like(digest) for _ in range(world)]
        dist.all_gather(gathered, digest)
        t = bench.max_over_ranks(dist, 1.0 + rank)          # per-rank "elapsed" seconds
        np.save(os.path.join(out_dir, f"r{rank}.npy"),
                np.array([t] + [int(v) for g in gathered for v in g.tolist()], dtype=np.float64))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_rank_weak_scaling_logic(tmp_path):
    world, port = 2, _free_port()
    mp.start_processes(_worker, args=(world, port, str(tmp_path)), nprocs=world, start_method="spawn")
    r0 = np.load(tmp_path / "r0.npy")
    r1 = np.load(tmp_path / "r1.npy")
    assert r0[0] == r1[0] == 2.0                       # max over ranks, seen by every rank
    np.testing.assert_array_equal(r0[1:], r1[1:])      # same gathered digests on both ranks
    assert r0[2] != r0[4]                              # rank batches differ (distinct seeds)
    # each rank's result depends only on its own batch
    for rank in range(world):
        x = W.generate("c2", slice(0, 8), seed=W.rank_seed(rank))
        _, codes, _ = oracle.rotate_quant(W.bits_to_float64(x, "bf16"), 0, "int4", 128)
        assert int(codes.astype(np.int64).sum()) == r0[1 + 2 * rank]


def test_aggregate_is_total_bytes_over_slowest_rank():
    assert bench.aggregate_gbs(1e9, 10, 4, 2.0) == pytest.approx(20.0)
    assert bench.max_over_ranks(None, 3.5) == 3.5
