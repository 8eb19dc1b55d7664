"""GPU parity of the MoE layer's steps as separate calls -- routing with the permutation and dispatch
buffer (moe_q4_route), the expert FFN on rows routed from elsewhere (moe_q4_forward_rows) and the combine
(moe_q4_combine) -- and of expert parallelism in its all-to-all form built from them, with the ranks
emulated on one GPU (the exchange is done by slicing; the multi-rank wiring itself is tested on gloo
ranks).  Routing outputs bit-exact; layer outputs within 1e-2 * rms of the fp64 oracle."""
import numpy as np
import pytest
import torch

import oracle
from moe_linear_layers_b200 import synth
from tests._util import assert_close, cpu_u16, cuda_u16_as, upload_weight

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def q4():
    from moe_linear_layers_b200 import q4 as mod
    return mod


def _stack(tag, E, H, I, group, sym):
    return [oracle.quantize(synth.weights(("ep-gpu", tag, nm), n, k), group, sym)
            for nm, n, k in (("g", E * I, H), ("u", E * I, H), ("d", E * H, I))]


def _local(q4, qs, e0, e1, H, I, group, sym):
    out = []
    for (pk, sc, zr), rows, k in zip(qs, (I, I, H), (H, H, I)):
        sl = slice(e0 * rows, e1 * rows)
        out.append(upload_weight(q4, pk[sl], sc[sl], None if zr is None else zr[sl], (e1 - e0) * rows, k, group, sym))
    return tuple(out)


def test_route_outputs_bit_exact(q4):
    T, H, E, topk = 300, 512, 16, 4
    x = synth.activations(("ep-gpu", "route-x"), T, H)
    Wr, bias = synth.router(("ep-gpu", "route"), E, H)
    _, ids, w, _ = oracle.route(x, H, Wr, bias, topk)
    offsets, perm = oracle.permute(ids, E)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    r = q4.moe_q4_route(cuda_u16_as(x, torch.bfloat16), torch.from_numpy(Wr).cuda(), torch.from_numpy(bias).cuda(),
                        topk, dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    assert np.array_equal(r["topk_ids"].cpu().numpy(), ids)
    np.testing.assert_allclose(r["topk_w"].cpu().numpy(), w, rtol=1e-5, atol=1e-7)
    assert np.array_equal(r["offsets"].cpu().numpy(), offsets)
    pos = np.empty_like(perm)
    pos[perm] = np.arange(perm.size)
    assert np.array_equal(r["pair_pos"].cpu().numpy(), pos)
    assert np.array_equal(r["row_expert"].cpu().numpy(), ids.ravel()[perm])
    assert np.array_equal(cpu_u16(r["x_perm"]), x[perm // topk])


@pytest.mark.parametrize("world", [1, 2, 3])
def test_expert_parallel_all_to_all_emulated_ranks(q4, world):
    """Each emulated rank routes its own tokens, sends each block of its dispatch buffer to the rank owning
    those experts, runs its experts on what it receives, and combines what comes back."""
    T, H, I, E, topk, group, sym = 200, 512, 256, 10, 3, 128, False
    sizes = [80, 120, 0][:world] if world > 1 else [T]
    sizes[-1] += T - sum(sizes)
    x = synth.activations(("ep-gpu", "x"), T, H)
    Wr, bias = synth.router(("ep-gpu", "layer"), E, H)
    qs = _stack("layer", E, H, I, group, sym)
    _, ids, w, _ = oracle.route(x, H, Wr, bias, topk)
    ref = oracle.moe_experts(x, H, ids, w, qs[0], qs[1], qs[2], I, group, sym)
    Wrd, bd = torch.from_numpy(Wr).cuda(), torch.from_numpy(bias).cuda()
    bounds = [q4.expert_range(d, world, E) for d in range(world)]
    local = [_local(q4, qs, e0, e1, H, I, group, sym) for (e0, e1) in bounds]
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    starts = np.concatenate([[0], np.cumsum(sizes)])
    routed = [q4.moe_q4_route(cuda_u16_as(x[starts[r]:starts[r + 1]], torch.bfloat16), Wrd, bd, topk, dev_status=st)
              if sizes[r] else None for r in range(world)]
    offs = [rt["offsets"].cpu().numpy() if rt else np.zeros(E + 1, np.int64) for rt in routed]
    # dispatch: rank d receives from every rank r the block of rows routed to d's experts
    blocks = {}
    o_dest = []
    for d, (e0, e1) in enumerate(bounds):
        xs, es = [], []
        for r in range(world):
            a, b = int(offs[r][e0]), int(offs[r][e1])
            blocks[(r, d)] = (sum(t.shape[0] for t in xs), b - a)
            if b > a:
                xs.append(routed[r]["x_perm"][a:b])
                es.append(routed[r]["row_expert"][a:b])
        x_in = torch.cat(xs) if xs else torch.empty((0, H), dtype=torch.bfloat16, device="cuda")
        e_in = torch.cat(es) if es else torch.empty((0,), dtype=torch.int32, device="cuda")
        o_dest.append(q4.moe_q4_forward_rows(x_in.contiguous(), e_in.contiguous(), e0, local[d], I, dev_status=st))
    # return: rank r gets back, in the order it sent, the results of its blocks; then the combine
    for r in range(world):
        if not sizes[r]:
            continue
        back = [o_dest[d][blocks[(r, d)][0]:blocks[(r, d)][0] + blocks[(r, d)][1]] for d in range(world)]
        o_back = torch.cat(back).contiguous()
        y = q4.moe_q4_combine(o_back, routed[r]["pair_pos"], routed[r]["topk_w"], dev_status=st)
        torch.cuda.synchronize()
        assert int(st.item()) == 0
        assert_close(y.cpu().numpy(), ref[starts[r]:starts[r + 1]], what=f"rank {r} of {world}")


def test_forward_rows_bad_expert_id_and_bf16_combine(q4):
    """A row whose expert id is outside the rank's range is reported (Q4_ERR_SHAPE) and contributes zero;
    the combine's bf16 output is the rounded fp32 combine."""
    R, H, I, E, group, sym = 40, 256, 128, 4, 64, True
    qs = _stack("rows", E, H, I, group, sym)
    ex = _local(q4, qs, 0, E, H, I, group, sym)
    x = synth.activations(("ep-gpu", "rows-x"), R, H)
    ids = (np.arange(R) % E).astype(np.int32) + 5
    ids[7] = 3   # outside [5, 9)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    y = q4.moe_q4_forward_rows(cuda_u16_as(x, torch.bfloat16), torch.from_numpy(ids).cuda(), 5, ex, I, dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == q4.Q4_ERR_SHAPE
    yn = y.cpu().numpy()
    assert np.all(yn[7] == 0)
    ok = np.arange(R) != 7
    ref = oracle.moe_experts(x, H, (ids - 5).clip(0)[:, None], np.where(ok, 1.0, 0.0)[:, None], qs[0], qs[1], qs[2], I,
                             group, sym)
    assert_close(yn, ref, what="rows")
    # combine: token t = rows 2t and 2t + 1 with weights 0.25 / 0.75
    T = R // 2
    pp = torch.arange(R, dtype=torch.int32, device="cuda")
    wt = torch.tensor([[0.25, 0.75]] * T, dtype=torch.float32, device="cuda")
    y32 = q4.moe_q4_combine(y, pp, wt)
    y16 = q4.moe_q4_combine(y, pp, wt, out_dtype=torch.bfloat16)
    torch.cuda.synchronize()
    np.testing.assert_allclose(y32.cpu().numpy(), 0.25 * yn[0::2] + 0.75 * yn[1::2], rtol=1e-6, atol=1e-7)
    assert torch.equal(y16, y32.to(torch.bfloat16))
