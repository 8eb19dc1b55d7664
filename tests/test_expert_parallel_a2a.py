"""Expert parallelism in its all-to-all form on CPU ranks (gloo): every rank holds its own tokens and the
weights of a contiguous range of experts; rows routed to another rank's experts go there in one
all-to-all and their results come back in the reverse one (q4.moe_q4_forward_ep).  The three device steps
(route + permute, the expert FFN on received rows, the combine) are the oracle here, a stand-in for the GPU
kernels, which need a B200; the test checks the exchange -- block sizes, the order of the rows both ways,
the ownership of experts -- against the oracle's whole layer on each rank's tokens."""
import os
import socket

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
from moe_linear_layers_b200 import q4, synth

T, H, I, E, TOPK, GROUP, SYM = 10, 128, 128, 7, 3, 64, False


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _layer():
    Wr, bias = synth.router(("ep-a2a",), E, H)
    stack = [oracle.quantize(synth.weights(("ep-a2a", nm), n, k), GROUP, SYM)
             for nm, n, k in (("g", E * I, H), ("u", E * I, H), ("d", E * H, I))]
    return Wr, bias, stack


def _tokens(rank):
    """Each rank's own tokens (different counts per rank, one rank with none at world 3)."""
    n = (T, T + 3, 0)[rank]
    return synth.activations(("ep-a2a", "x", rank), n, H) if n else np.zeros((0, H), np.uint16)


def _slice(stack, e0, e1):
    out = []
    for (pk, sc, zr), rows in zip(stack, (I, I, H)):
        sl = slice(e0 * rows, e1 * rows)
        out.append((pk[sl], sc[sl], None if zr is None else zr[sl]))
    return tuple(out)


def _bf16(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16)


def _oracle_fns(x, Wr, bias, local):
    """The route, rows and combine steps computed by the oracle on the host."""
    def route():
        n = x.shape[0]
        if n == 0:
            return {"topk_ids": torch.zeros((0, TOPK), dtype=torch.int32), "topk_w": torch.zeros((0, TOPK)),
                    "offsets": torch.zeros(E + 1, dtype=torch.int32), "pair_pos": torch.zeros(0, dtype=torch.int32),
                    "x_perm": torch.zeros((0, H), dtype=torch.bfloat16), "row_expert": torch.zeros(0, dtype=torch.int32)}
        _, ids, w, _ = oracle.route(x, H, Wr, bias, TOPK)
        offsets, perm = oracle.permute(ids, E)
        pair_pos = np.empty_like(perm)
        pair_pos[perm] = np.arange(perm.size, dtype=np.int32)
        return {"topk_ids": torch.from_numpy(ids), "topk_w": torch.from_numpy(w.astype(np.float32)),
                "offsets": torch.from_numpy(offsets), "pair_pos": torch.from_numpy(pair_pos),
                "x_perm": _bf16(x[perm // TOPK]), "row_expert": torch.from_numpy(ids.ravel()[perm].astype(np.int32))}

    def rows(x_rows, row_expert, e_base):
        R = x_rows.shape[0]
        if R == 0:
            return torch.zeros((0, H), dtype=torch.float32)
        bits = x_rows.contiguous().view(torch.int16).numpy().view(np.uint16)
        ids = (row_expert.numpy() - e_base).astype(np.int32)[:, None]
        y = oracle.moe_experts(bits, H, ids, np.ones((R, 1)), local[0], local[1], local[2], I, GROUP, SYM)
        return torch.from_numpy(y.astype(np.float32))

    def combine(o, pair_pos, w):
        n = w.shape[0]
        y = np.zeros((n, H))
        for t in range(n):
            for j in range(TOPK):
                y[t] += float(w[t, j]) * o[int(pair_pos[t * TOPK + j])].double().numpy()
        return torch.from_numpy(y)

    return {"route": route, "rows": rows, "combine": combine}


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        Wr, bias, stack = _layer()
        x = _tokens(rank)
        e0, e1 = q4.expert_range(rank, world, E)
        local = _slice(stack, e0, e1)
        y = q4.moe_q4_forward_ep(_bf16(x), torch.from_numpy(Wr), torch.from_numpy(bias), TOPK, local, I,
                                 fns=_oracle_fns(x, Wr, bias, local))
        out[rank] = y.numpy()
    finally:
        dist.destroy_process_group()


def test_expert_parallel_all_to_all_on_gloo_ranks():
    Wr, bias, stack = _layer()
    for world in (2, 3):
        out = mp.get_context("spawn").Manager().dict()   # no fork of this threaded process
        mp.spawn(_worker, args=(world, _free_port(), out), nprocs=world, join=True)
        for r in range(world):
            x = _tokens(r)
            if x.shape[0] == 0:
                assert out[r].shape == (0, H)
                continue
            _, ids, w, _ = oracle.route(x, H, Wr, bias, TOPK)
            ref = oracle.moe_experts(x, H, ids, w, stack[0], stack[1], stack[2], I, GROUP, SYM)
            # the layer's sum in another order (slot order of fp32 rows): fp32 rounding of each expert output
            np.testing.assert_allclose(out[r], ref, rtol=0, atol=1e-6 * np.abs(ref).max())
