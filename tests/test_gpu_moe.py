"""GPU parity of the MoE layer (route -> permute -> grouped gate/up SwiGLU -> grouped down + combine)
against the oracle, through the C ABI.

Expert ids, permutation, offsets and counts are bit-exact (the router logits follow a pinned fp32
reduction order on both sides).  Routing weights: fp32 expf against the fp64 oracle, rtol 1e-5.
Outputs: max|y - y_ref| <= 1e-2 * rms(y_ref) (fp32 output; the down projection's combine uses float
atomics, so the last bits vary with the summation order)."""
import numpy as np
import pytest
import torch

import oracle
from moe_linear_layers_b200 import synth
from tests._util import REL_TOL, assert_close, cpu_u16, cuda_u16_as, rel_err, upload_weight

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def q4():
    from moe_linear_layers_b200 import q4 as mod
    return mod


def _experts(tag, E, H, I, group, sym):
    """Stacked expert weights: gate/up [E*I][H], down [E*H][I], quantized by the oracle."""
    Wg = synth.weights(("moe", tag, "gate"), E * I, H)
    Wu = synth.weights(("moe", tag, "up"), E * I, H)
    Wd = synth.weights(("moe", tag, "down"), E * H, I)
    return [oracle.quantize(W, group, sym) for W in (Wg, Wu, Wd)]


def _run(q4, T, H, I, E, topk, group, sym, tag, skew=1.1, tokens=None, out=torch.float32):
    x = synth.activations(("moe", tag, "x"), T, H)
    Wr, bias = synth.router(("moe", tag), E, H, skew=skew)
    qs = _experts(tag, E, H, I, group, sym)
    logits, ids, w, counts = oracle.route(x, H, Wr, bias, topk)
    offsets, perm = oracle.permute(ids, E)
    ref = oracle.moe_experts(x, H, ids, w, qs[0], qs[1], qs[2], I, group, sym, tokens=tokens)
    ex = (upload_weight(q4, *qs[0], E * I, H, group, sym), upload_weight(q4, *qs[1], E * I, H, group, sym),
          upload_weight(q4, *qs[2], E * H, I, group, sym))
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    y, ids_d, w_d, perm_d, off_d, cnt_d = q4.moe_q4_forward(
        cuda_u16_as(x, torch.bfloat16), torch.from_numpy(Wr).cuda(), torch.from_numpy(bias).cuda(), topk, ex, I,
        out_dtype=out, want_routing=True, dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    assert np.array_equal(ids_d.cpu().numpy(), ids), "expert ids differ"
    np.testing.assert_allclose(w_d.cpu().numpy(), w, rtol=1e-5, atol=1e-7)
    assert np.array_equal(off_d.cpu().numpy(), offsets)
    assert np.array_equal(perm_d.cpu().numpy(), perm)
    assert np.array_equal(cnt_d.cpu().numpy(), counts)
    yn = y.float().cpu().numpy()
    if tokens is not None:
        yn = yn[tokens]
    return yn, ref, counts


@pytest.mark.parametrize("T,H,I,E,topk,group,sym", [
    (64, 256, 128, 8, 2, 128, False),     # small, every expert busy
    (37, 256, 256, 5, 3, 64, True),       # ragged token count, group 64, symmetric
    (16, 128, 128, 1, 1, 128, False),     # a single expert: a dense SwiGLU FFN
    (200, 512, 256, 64, 8, 128, False),   # the workload's expert count / top-8, skewed: some experts empty
    (150, 256, 256, 6, 2, 32, False),     # group 32, asymmetric
    (90, 512, 128, 4, 2, 32, True),       # group 32, symmetric
    (150, 512, 256, 6, 2, 256, False),    # group 256 (a group spans two 128-K stages), asymmetric
    (64, 1024, 512, 8, 2, 256, True),     # group 256, symmetric, several groups per row
])
def test_moe_small(q4, T, H, I, E, topk, group, sym):
    yn, ref, counts = _run(q4, T, H, I, E, topk, group, sym, f"s{T}-{E}")
    assert_close(yn, ref, what="moe")


def test_moe_bf16_output(q4):
    yn, ref, _ = _run(q4, 48, 256, 128, 8, 2, 128, False, "bf16", out=torch.bfloat16)
    # bf16 rounding of the output adds at most 2^-8 |y| on top of the stated bar
    err = np.abs(yn.astype(np.float64) - ref)
    rms = np.sqrt(np.mean(ref * ref))
    assert np.all(err <= REL_TOL * rms + 2.0 ** -8 * np.abs(ref))


def test_moe_workload_full_size(q4):
    """4096 tokens, hidden 2048, 64 experts of intermediate 1024, top-8, asymmetric group 128, router
    logits Zipf-skewed (bias -1.1 ln(e+1)): routing checked for every token, outputs on a sample."""
    tokens = np.arange(0, 4096, 97)
    yn, ref, counts = _run(q4, 4096, 2048, 1024, 64, 8, 128, False, "full", tokens=tokens)
    assert_close(yn, ref, what="moe full")
    assert counts[0] > counts[-1]    # the skew is visible


def test_moe_workspace_too_small(q4):
    from moe_linear_layers_b200.q4 import Q4Error, Q4_ERR_WORKSPACE
    T, H, I, E, topk = 32, 128, 128, 4, 2
    qs = _experts("ws", E, H, I, 128, True)
    ex = tuple(upload_weight(q4, *qq, n, k, 128, True) for qq, n, k in zip(qs, (E * I, E * I, E * H), (H, H, I)))
    x = torch.zeros((T, H), dtype=torch.bfloat16, device="cuda")
    Wr = torch.zeros((E, H), dtype=torch.float32, device="cuda")
    ws = torch.empty(q4.moe_q4_workspace_size(T, H, I, E, topk) - 256, dtype=torch.uint8, device="cuda")
    with pytest.raises(Q4Error) as ei:
        q4.moe_q4_forward(x, Wr, None, topk, ex, I, workspace=ws)
    assert ei.value.status == Q4_ERR_WORKSPACE


@pytest.mark.parametrize("T,H,I,E,topk,I_s,group,sym", [
    (64, 256, 128, 8, 2, 256, 128, False),       # shared expert wider than the routed ones
    (37, 256, 256, 5, 3, 128, 64, True),         # ragged token count, group 64, symmetric
    (300, 512, 256, 16, 4, 512, 128, False),     # several token tiles for the shared expert
])
def test_moe_with_shared_expert(q4, T, H, I, E, topk, I_s, group, sym):
    tag = f"sh{T}-{E}"
    x = synth.activations(("moe", tag, "x"), T, H)
    Wr, bias = synth.router(("moe", tag), E, H, skew=1.1)
    qs = _experts(tag, E, H, I, group, sym)
    qsh = [oracle.quantize(synth.weights(("moe", tag, "shared", nm), n, k), group, sym)
           for nm, n, k in (("gate", I_s, H), ("up", I_s, H), ("down", H, I_s))]
    logits, ids, w, counts = oracle.route(x, H, Wr, bias, topk)
    ref = oracle.moe_experts(x, H, ids, w, qs[0], qs[1], qs[2], I, group, sym)
    ref = ref + oracle.shared_expert(x, H, qsh[0], qsh[1], qsh[2], I_s, group, sym)
    ex = (upload_weight(q4, *qs[0], E * I, H, group, sym), upload_weight(q4, *qs[1], E * I, H, group, sym),
          upload_weight(q4, *qs[2], E * H, I, group, sym))
    sh = (upload_weight(q4, *qsh[0], I_s, H, group, sym), upload_weight(q4, *qsh[1], I_s, H, group, sym),
          upload_weight(q4, *qsh[2], H, I_s, group, sym))
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    y = q4.moe_q4_forward(cuda_u16_as(x, torch.bfloat16), torch.from_numpy(Wr).cuda(), torch.from_numpy(bias).cuda(),
                          topk, ex, I, dev_status=st, shared=sh)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    assert_close(y.cpu().numpy(), np.asarray(ref).reshape(T, H), what="moe + shared expert")


# ---------------------------------------------------------------------------------------------- #
# the expert projections on INT8 activation codes (W4A8): a8_mask bit 0 = gate/up, bit 1 = down
# ---------------------------------------------------------------------------------------------- #

def _run_a8(q4, T, H, I, E, topk, group, sym, mask, tag, tokens=None):
    x = synth.activations(("moe", tag, "x"), T, H)
    Wr, bias = synth.router(("moe", tag), E, H, skew=1.1)
    qs = _experts(tag, E, H, I, group, sym)
    logits, ids, w, counts = oracle.route(x, H, Wr, bias, topk)
    offsets, perm = oracle.permute(ids, E)
    ref = oracle.moe_experts_a8(x, H, ids, w, qs[0], qs[1], qs[2], I, group, sym, mask, tokens=tokens)
    ex = (upload_weight(q4, *qs[0], E * I, H, group, sym), upload_weight(q4, *qs[1], E * I, H, group, sym),
          upload_weight(q4, *qs[2], E * H, I, group, sym))
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    y, ids_d, w_d, perm_d, off_d, cnt_d = q4.moe_q4_forward(
        cuda_u16_as(x, torch.bfloat16), torch.from_numpy(Wr).cuda(), torch.from_numpy(bias).cuda(), topk, ex, I,
        want_routing=True, dev_status=st, a8_mask=mask)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    assert np.array_equal(ids_d.cpu().numpy(), ids), "expert ids differ"
    assert np.array_equal(perm_d.cpu().numpy(), perm)
    assert np.array_equal(off_d.cpu().numpy(), offsets)
    yn = y.cpu().numpy()
    return (yn if tokens is None else yn[tokens]), ref


@pytest.mark.parametrize("mask", [1, 2, 3])
@pytest.mark.parametrize("T,H,I,E,topk,group,sym", [
    (64, 256, 128, 8, 2, 128, False),     # every expert busy
    (37, 256, 256, 5, 3, 64, True),       # ragged token count, group 64, symmetric
    (200, 512, 256, 64, 8, 128, False),   # 64 experts / top-8, skewed: some experts empty
    (300, 512, 384, 4, 2, 64, False),     # several 128-row tiles per expert, group 64 asymmetric
])
def test_moe_a8(q4, T, H, I, E, topk, group, sym, mask):
    yn, ref = _run_a8(q4, T, H, I, E, topk, group, sym, mask, f"a8-{T}-{E}")
    assert_close(yn, ref, what=f"moe a8 mask {mask}")


def test_moe_a8_workload_full_size(q4):
    """The full layer (4096 tokens, 64 experts of 1024, top-8, asymmetric group 128) with every expert
    projection on INT8 activations: routing for every token, outputs on a sample of tokens."""
    tokens = np.arange(0, 4096, 131)
    yn, ref = _run_a8(q4, 4096, 2048, 1024, 64, 8, 128, False, 3, "full", tokens=tokens)
    assert_close(yn, ref, what="moe a8 full")


def test_moe_a8_rejects_shared_expert_and_bad_mask(q4):
    from moe_linear_layers_b200.q4 import Q4Error, Q4_ERR_UNSUPPORTED
    with pytest.raises(ValueError):
        q4.moe_q4_workspace_size(16, 128, 128, 4, 2, I_shared=128, a8_mask=1)
    assert q4._lib.moe_q4_workspace_size_a8(16, 128, 128, 4, 2, 4) == 0
    T, H, I, E, topk = 16, 128, 128, 4, 2
    qs = _experts("a8bad", E, H, I, 128, True)
    ex = tuple(upload_weight(q4, *qq, n, k, 128, True) for qq, n, k in zip(qs, (E * I, E * I, E * H), (H, H, I)))
    x = torch.zeros((T, H), dtype=torch.bfloat16, device="cuda")
    Wr = torch.zeros((E, H), dtype=torch.float32, device="cuda")
    ws = torch.empty(q4.moe_q4_workspace_size(T, H, I, E, topk, a8_mask=3), dtype=torch.uint8, device="cuda")
    with pytest.raises(Q4Error) as ei:
        q4.moe_q4_forward(x, Wr, None, topk, ex, I, workspace=ws, a8_mask=5)
    assert ei.value.status == Q4_ERR_UNSUPPORTED


# ---------------------------------------------------------------------------------------------- #
# expert classes with their own group size and symmetry (moe_q4_forward_classes)
# ---------------------------------------------------------------------------------------------- #

def _run_classes(q4, T, H, I, E, topk, begin, params, tag, tokens=None):
    x = synth.activations(("moe", tag, "x"), T, H)
    Wr, bias = synth.router(("moe", tag), E, H, skew=1.1)
    logits, ids, w, counts = oracle.route(x, H, Wr, bias, topk)
    offsets, perm = oracle.permute(ids, E)
    classes, dev_classes = [], []
    for c, (group, sym) in enumerate(params):
        Ec = begin[c + 1] - begin[c]
        qs = [oracle.quantize(synth.weights(("moe", tag, c, nm), n, k), group, sym)
              for nm, n, k in (("gate", Ec * I, H), ("up", Ec * I, H), ("down", Ec * H, I))]
        classes.append((qs[0], qs[1], qs[2], group, sym))
        dev_classes.append(tuple(upload_weight(q4, *q, n, k, group, sym)
                                 for q, n, k in zip(qs, (Ec * I, Ec * I, Ec * H), (H, H, I))))
    ref = oracle.moe_experts_classes(x, H, ids, w, begin, classes, I, tokens=tokens)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    y, ids_d, w_d, perm_d, off_d, cnt_d = q4.moe_q4_forward_classes(
        cuda_u16_as(x, torch.bfloat16), torch.from_numpy(Wr).cuda(), torch.from_numpy(bias).cuda(), topk, begin,
        dev_classes, I, want_routing=True, dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    assert np.array_equal(ids_d.cpu().numpy(), ids)
    assert np.array_equal(perm_d.cpu().numpy(), perm)
    assert np.array_equal(off_d.cpu().numpy(), offsets)
    yn = y.cpu().numpy()
    return (yn if tokens is None else yn[tokens]), ref


@pytest.mark.parametrize("T,H,I,E,topk,begin,params", [
    (200, 512, 256, 16, 4, [0, 2, 8, 16], [(64, True), (128, False), (64, False)]),
    (37, 256, 128, 5, 3, [0, 1, 5], [(64, False), (128, True)]),
    (300, 256, 128, 8, 2, [0, 8], [(128, False)]),          # one class = the plain layer
    (256, 512, 256, 16, 4, [0, 1, 6, 16], [(32, False), (64, False), (128, False)]),   # the pages' three tiers
    (256, 512, 512, 16, 4, [0, 1, 6, 16], [(32, False), (64, False), (256, False)]),   # the coldest tier at 256
])
def test_moe_classes(q4, T, H, I, E, topk, begin, params):
    yn, ref = _run_classes(q4, T, H, I, E, topk, begin, params, f"cls{T}-{E}")
    assert_close(yn, ref, what="moe classes")


def test_moe_classes_workload_full_size(q4):
    """The 4096-token layer in the pages' three tiers: the 3 most chosen experts (5 % of 64; expert 0 is the
    hottest under the Zipf-skewed logits) at group 32, experts 3-31 at group 64, the rest at group 128."""
    tokens = np.arange(0, 4096, 173)
    yn, ref = _run_classes(q4, 4096, 2048, 1024, 64, 8, [0, 3, 32, 64], [(32, False), (64, False), (128, False)],
                           "clsfull", tokens=tokens)
    assert_close(yn, ref, what="moe classes full")


# ---------------------------------------------------------------------------------------------- #
# expert ranges (moe_q4_forward_range): the unit of expert parallelism
# ---------------------------------------------------------------------------------------------- #

def test_moe_expert_ranges_sum_to_the_layer(q4):
    T, H, I, E, topk, group, sym = 300, 512, 256, 16, 4, 128, False
    tag = "ranges"
    x = synth.activations(("moe", tag, "x"), T, H)
    Wr, bias = synth.router(("moe", tag), E, H, skew=1.1)
    qs = _experts(tag, E, H, I, group, sym)
    _, ids, w, _ = oracle.route(x, H, Wr, bias, topk)
    xd = cuda_u16_as(x, torch.bfloat16)
    Wrd, bd = torch.from_numpy(Wr).cuda(), torch.from_numpy(bias).cuda()
    full = q4.moe_q4_forward(xd, Wrd, bd, topk, tuple(upload_weight(q4, *q, n, k, group, sym) for q, n, k in
                                                     zip(qs, (E * I, E * I, E * H), (H, H, I))), I)

    def sliced(e0, e1):
        out = []
        for (pk, sc, zr), rows, k in zip(qs, (I, I, H), (H, H, I)):
            sl = slice(e0 * rows, e1 * rows)
            out.append(upload_weight(q4, pk[sl], sc[sl], None if zr is None else zr[sl], (e1 - e0) * rows, k, group, sym))
        return tuple(out)

    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    for world in (2, 4, 5):
        parts = []
        for r in range(world):
            e0, e1 = q4.expert_range(r, world, E)
            parts.append(q4.moe_q4_forward_range(xd, Wrd, bd, topk, e0, e1, sliced(e0, e1), I, dev_status=st))
            if r == 1:   # one range against the oracle over the slots routed into it
                mine = (ids >= e0) & (ids < e1)
                ref = oracle.moe_experts(x, H, np.where(mine, ids - e0, 0).astype(np.int32), np.where(mine, w, 0.0),
                                         *[(pk[e0 * rows:e1 * rows], sc[e0 * rows:e1 * rows],
                                            None if zr is None else zr[e0 * rows:e1 * rows])
                                           for (pk, sc, zr), rows in zip(qs, (I, I, H))], I, group, sym)
                torch.cuda.synchronize()
                assert_close(parts[-1].cpu().numpy(), ref, what=f"range {e0}-{e1}")
        total = sum(parts)
        torch.cuda.synchronize()
        assert int(st.item()) == 0
        d = (total - full).abs().max().item() / full.pow(2).mean().sqrt().item()
        assert d <= 1e-5, f"ranges of {world} ranks differ from the layer by {d:.2e} of rms"
