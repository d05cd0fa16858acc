"""Expert parallelism on the CPU: world-size-2 gloo groups.

The layer's routed experts split into contiguous ranges, one per GPU, and the
GPUs' fp64 partial outputs are summed in rank order ("Comment exécuter un
réseau de neurones de 744 milliards de paramètres sur un ordinateur
ordinaire", devtrends.cc, "Les chiffres réels de vitesse": six GPUs hold the
experts in video memory).  Here the partition and the exchange -- all-gather,
then a sum in rank order that every rank computes identically -- run on gloo
ranks with partials whose fp64 sum depends on the order of addition.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import quantized_expert_ffn_noaux_b200 as qe


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.mark.parametrize("E,world", [(256, 2), (256, 3), (256, 6), (8, 3), (5, 8)])
def test_expert_ranges_partition_the_experts(E, world):
    ranges = [qe.expert_range(E, r, world) for r in range(world)]
    assert ranges[0][0] == 0 and ranges[-1][1] == E
    for (a, b), (c, d) in zip(ranges, ranges[1:]):
        assert b == c and a <= b
    sizes = [b - a for a, b in ranges]
    assert max(sizes) - min(sizes) <= 1 and sum(sizes) == E


def _partial(rank):
    # values whose fp64 sum depends on the order: 1e16 + 1 - 1e16 ...
    base = np.array([1e16, 1.0, -3.0, 0.5], np.float64)
    return torch.from_numpy(np.roll(base, rank) * (rank + 1))


def _worker(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        parts = qe.gather_partials(_partial(rank))
        total = parts[0].clone()
        for r in range(1, world):
            total += parts[r]
        out[rank] = (parts.numpy().tolist(), total.numpy().tolist())
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_partials_gathered_and_summed_in_rank_order():
    world = 2
    out = mp.Manager().dict()
    mp.spawn(_worker, args=(world, _free_port(), out), nprocs=world, join=True)
    want = [_partial(r).numpy() for r in range(world)]
    serial = want[0].copy()
    for r in range(1, world):
        serial = serial + want[r]
    for rank in range(world):
        parts, total = out[rank]
        np.testing.assert_array_equal(np.array(parts), np.stack(want))
        np.testing.assert_array_equal(np.array(total), serial)   # bit for bit, every rank
