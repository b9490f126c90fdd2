"""The N>1 host path on CPU: two gloo ranks shard a global batch and reduce device times with MAX."""

import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from head_latent_attention_absorb_b200.shard import max_over_ranks, shard_range


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        start, count = shard_range(67, world, rank)
        got = max_over_ranks([float(rank), 10.0 - rank, float(count)])
        out[rank] = (start, count, got)
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_shard_range_partitions():
    for g in (0, 1, 5, 32, 67, 1000):
        for w in (1, 2, 3, 8):
            spans = [shard_range(g, w, r) for r in range(w)]
            assert sum(c for _, c in spans) == g
            pos = 0
            for s, c in spans:
                assert s == pos and c >= 0
                pos += c
            assert max(c for _, c in spans) - min(c for _, c in spans) <= 1
    with pytest.raises(ValueError):
        shard_range(4, 2, 2)


def test_two_gloo_ranks_shard_and_reduce():
    world, port = 2, _free_port()
    out = mp.get_context("spawn").Manager().dict()
    mp.start_processes(_worker, args=(world, port, out), nprocs=world, start_method="spawn", join=True)
    assert out[0][:2] == (0, 34) and out[1][:2] == (34, 33)
    for r in range(world):
        assert out[r][2] == [1.0, 10.0, 34.0]


def test_max_over_ranks_single_process():
    assert max_over_ranks([1.5, 2.0]) == [1.5, 2.0]
