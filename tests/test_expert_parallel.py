"""Expert parallelism on CPU ranks (gloo): every rank owns a contiguous range of experts, computes that
range's contribution to the MoE layer and the contributions are summed by an all-reduce.  The ranks'
local computation here is the oracle (a stand-in for the GPU range kernel, which needs a B200); the test
checks the split of the experts and the reduction against the oracle's whole layer."""
import os
import socket

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
from moe_linear_layers_b200 import q4, synth

T, H, I, E, TOPK, GROUP, SYM = 12, 128, 128, 7, 3, 64, False


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _layer():
    x = synth.activations(("ep", "x"), T, H)
    Wr, bias = synth.router(("ep",), E, H)
    stack = [oracle.quantize(synth.weights(("ep", nm), n, k), GROUP, SYM)
             for nm, n, k in (("g", E * I, H), ("u", E * I, H), ("d", E * H, I))]
    return x, Wr, bias, stack


def _slice(stack, e0, e1):
    out = []
    for (pk, sc, zr), rows in zip(stack, (I, I, H)):
        sl = slice(e0 * rows, e1 * rows)
        out.append((pk[sl], sc[sl], None if zr is None else zr[sl]))
    return tuple(out)


def _oracle_range(x, router_w, router_bias, topk, e0, e1, local, I_):
    """The contribution of experts e0 .. e1-1: the oracle layer over the slots routed into the range."""
    _, ids, w, _ = oracle.route(x, H, router_w.numpy(), router_bias.numpy(), topk)
    mine = (ids >= e0) & (ids < e1)
    y = oracle.moe_experts(x, H, np.where(mine, ids - e0, 0).astype(np.int32), np.where(mine, w, 0.0),
                           local[0], local[1], local[2], I_, GROUP, SYM)
    return torch.from_numpy(y)


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        x, Wr, bias, stack = _layer()
        e0, e1 = q4.expert_range(rank, world, E)
        y = q4.moe_q4_forward_expert_parallel(x, torch.from_numpy(Wr), torch.from_numpy(bias), TOPK,
                                              _slice(stack, e0, e1), I, range_fn=_oracle_range)
        out[rank] = (e0, e1, y.numpy())
    finally:
        dist.destroy_process_group()


def test_expert_ranges_partition_the_experts():
    for world in (1, 2, 3, 4, 7):
        ranges = [q4.expert_range(r, world, E) for r in range(world)]
        assert ranges[0][0] == 0 and ranges[-1][1] == E
        assert all(a[1] == b[0] for a, b in zip(ranges, ranges[1:]))
        assert all(e1 - e0 in (E // world, E // world + 1) for e0, e1 in ranges)


def test_expert_parallel_sum_equals_the_layer_on_gloo_ranks():
    x, Wr, bias, stack = _layer()
    _, ids, w, _ = oracle.route(x, H, Wr, bias, TOPK)
    ref = oracle.moe_experts(x, H, ids, w, stack[0], stack[1], stack[2], I, GROUP, SYM)
    for world in (2, 3):
        out = mp.get_context("spawn").Manager().dict()   # no fork of this threaded process
        mp.spawn(_worker, args=(world, _free_port(), out), nprocs=world, join=True)
        for r in range(world):
            e0, e1, y = out[r]
            assert (e0, e1) == q4.expert_range(r, world, E)
            np.testing.assert_allclose(y, ref, rtol=1e-12, atol=1e-13 * np.abs(ref).max())
