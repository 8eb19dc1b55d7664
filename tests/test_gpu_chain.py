"""GPU parity of the GEMV chain (q4_linear_w4a16_chain: dependent m = 1 stages in one launch) against the
oracle, through the C ABI.  Every output within max|err| <= 1e-2 * rms of the fp64 oracle; the stage order
is checked through a real dependency (a down projection gated from the previous stage's outputs, which
start as NaN); two calls in a row and a CUDA-graph replay reuse the stage counters; a raised abort word is
reported as Q4_ERR_TIMEOUT without a hang."""
import numpy as np
import pytest
import torch

import oracle
from moe_linear_layers_b200 import synth
from tests._util import assert_close, cuda_u16_as, upload_weight

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def q4():
    from moe_linear_layers_b200 import q4 as mod
    assert torch.cuda.is_available()
    return mod


def _linear(q4, tag, n, k, group, sym):
    W = synth.weights(("chain", tag, n, k), n, k)
    pk, sc, zr = oracle.quantize(W, group, sym)
    return (pk, sc, zr), upload_weight(q4, pk, sc, zr, n, k, group, sym)


def _x(tag, k):
    return synth.activations(("chain-x", tag, k), 1, k)


@pytest.mark.parametrize("group,sym", [(128, False), (64, True)])
def test_chain_independent_stages(q4, group, sym):
    """Stages of grouped problems with k 2048 / 8192 / 512 / 64 (split-k, ragged row counts, a single
    group) against the oracle."""
    shapes = [[(2048, 2048), (512, 2048), (77, 2048)], [(1000, 8192)], [(3, 512), (129, 512)], [(64, 64)]]
    stages, refs, outs = [], [], []
    for si, st in enumerate(shapes):
        probs = []
        for pi, (n, k) in enumerate(st):
            if k < group:
                continue
            q, w = _linear(q4, f"{si}.{pi}.{group}.{sym}", n, k, group, sym)
            x = _x(f"{si}.{pi}", k)
            refs.append(oracle.linear_w4a16(x, *q, n, k, group, sym)[0])
            y = torch.full((n,), float("nan"), dtype=torch.float32, device="cuda")
            outs.append(y)
            probs.append((cuda_u16_as(x, torch.bfloat16).view(-1), w, y))
        if probs:
            stages.append(probs)
    chain = q4.GemvChain(stages)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    for call in range(2):   # the second call finds the counters the first one left zero
        for y in outs:
            y.fill_(float("nan"))
        chain(dev_status=st)
        torch.cuda.synchronize()
        assert int(st.item()) == 0
        assert int(chain.sync.abs().sum().item()) == 0, "stage counters not left zero"
        for i, (y, ref) in enumerate(zip(outs, refs)):
            assert_close(y.cpu().numpy(), ref, what=f"call {call} problem {i}")


def test_chain_dependent_swiglu_stage(q4):
    """[gate, up] then down on silu(gate) * up of those outputs (read inside the same launch), then a stage
    whose x is unrelated: the down output matches the oracle's FFN only if the down stage waited."""
    H, I, group = 512, 2048, 128
    qg, wg = _linear(q4, "gate", I, H, group, False)
    qu, wu = _linear(q4, "up", I, H, group, False)
    qd, wd = _linear(q4, "down", H, I, group, False)
    qo, wo = _linear(q4, "other", 256, H, group, False)
    x = _x("ffn", H)
    xo = _x("other", H)
    g = torch.full((I,), float("nan"), dtype=torch.float32, device="cuda")
    u = torch.full((I,), float("nan"), dtype=torch.float32, device="cuda")
    yd = torch.full((H,), float("nan"), dtype=torch.float32, device="cuda")
    yo = torch.full((256,), float("nan"), dtype=torch.float32, device="cuda")
    xd = cuda_u16_as(x, torch.bfloat16).view(-1)
    chain = q4.GemvChain([[(xd, wg, g), (xd, wu, u)], [((g, u), wd, yd)], [(cuda_u16_as(xo, torch.bfloat16).view(-1), wo, yo)]])
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    chain(dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    g_ref = oracle.linear_w4a16(x, *qg, I, H, group, False)
    u_ref = oracle.linear_w4a16(x, *qu, I, H, group, False)
    assert_close(g.cpu().numpy(), g_ref[0], what="gate")
    assert_close(u.cpu().numpy(), u_ref[0], what="up")
    ref = oracle.linear_w4a16_swiglu(g_ref.astype(np.float32), u_ref.astype(np.float32), *qd, H, I, group, False)
    assert_close(yd.cpu().numpy(), ref[0], what="down on silu(gate) * up")
    assert_close(yo.cpu().numpy(), oracle.linear_w4a16(xo, *qo, 256, H, group, False)[0], what="other")


def test_chain_decode_step_full_size_in_a_graph(q4):
    """The LLaMA-3.2-1B-shaped decode step (16 layers x [q,k,v], o, [gate,up], down: 64 stages, 112 GEMVs,
    asymmetric group 128) captured in a CUDA graph and replayed twice; sampled rows of every linear against
    the oracle."""
    stages, checks = [], []
    for layer in range(synth.LLAMA_1B_LAYERS):
        lin = {}
        for nm, n, k in synth.LLAMA_1B_LINEARS:
            W = synth.weights(("chain-step", layer, nm), n, k)
            wd = q4.q4_quantize_pack(torch.from_numpy(W).cuda(), 128, False)
            x = _x(f"step.{layer}.{nm}", k)
            y = torch.empty((n,), dtype=torch.float32, device="cuda")
            lin[nm] = (cuda_u16_as(x, torch.bfloat16).view(-1), wd, y)
            if layer % 5 == 0:
                checks.append((W, x, y, n, k))
        stages += [[lin["q"], lin["k"], lin["v"]], [lin["o"]], [lin["gate"], lin["up"]], [lin["down"]]]
    torch.cuda.synchronize()
    chain = q4.GemvChain(stages)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    chain(dev_status=st)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        chain(dev_status=st)
    for _, _, y, _, _ in checks:
        y.fill_(float("nan"))
    g.replay()
    g.replay()
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    assert int(chain.sync.abs().sum().item()) == 0
    for W, x, y, n, k in checks:
        pk, sc, zr = oracle.quantize(W, 128, False)
        rows = np.arange(0, n, 61)
        ref = oracle.linear_w4a16(x, pk, sc, zr, n, k, 128, False, rows_n=rows)[0]
        full = y.cpu().numpy()
        assert np.all(np.isfinite(full))
        assert_close(full[rows], ref, what=f"{n}x{k}")


def test_chain_raised_abort_word_is_reported(q4):
    """A sync buffer whose abort word is raised (an earlier call gave up) is reported as Q4_ERR_TIMEOUT
    with no work done and no hang; zeroed again, the chain runs correctly."""
    q, w = _linear(q4, "abort", 256, 512, 128, False)
    x = _x("abort", 512)
    y = torch.full((256,), float("nan"), dtype=torch.float32, device="cuda")
    chain = q4.GemvChain([[(cuda_u16_as(x, torch.bfloat16).view(-1), w, y)], [(cuda_u16_as(x, torch.bfloat16).view(-1), w, y)]])
    chain.sync[0] = 1
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    chain(dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == q4.Q4_ERR_TIMEOUT
    chain.reset()
    st.zero_()
    chain(dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    assert_close(y.cpu().numpy(), oracle.linear_w4a16(x, *q, 256, 512, 128, False)[0], what="after reset")
