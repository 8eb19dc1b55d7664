"""Host logic of the multi-GPU bench path on CPU: two gloo ranks, max-over-ranks timing and the
whole-job value (every rank runs an independent replica of the decode step)."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ms = 10.0 + 5.0 * rank                # each rank's own timing
        m = bench.max_over_ranks(ms, world)
        bench.barrier(world)
        out[rank] = m
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_two_gloo_ranks():
    world = 2
    out = mp.Manager().dict()
    mp.spawn(_worker, args=(world, _free_port(), out), nprocs=world, join=True)
    assert out[0] == out[1] == 15.0


def test_decode_bytes_per_step():
    layers = bench.decode_layers()
    assert len(layers) == 112
    # packed weights alone: 16 layers x 60.8M codes / 2 bytes
    assert sum(n * k for (_, n, k) in layers) // 2 == 486539264
    b = bench.decode_bytes(layers)
    assert 0.5e9 < b < 0.53e9
