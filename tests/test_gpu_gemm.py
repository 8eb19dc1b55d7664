"""GPU parity of the tcgen05 tensor-core GEMMs (W4A16 bf16 MMA, W4A8 int8 MMA) against the oracle.

Floating outputs: max|err| <= 1e-2 * rms(fp64 oracle).  bf16 outputs equal the round-to-nearest-even of
the fp32 outputs bit for bit.  W4A8's per-group INT32 partials (debug output) are bit-exact."""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from moe_linear_layers_b200 import synth
from tests._util import assert_close, bf16_rne, cpu_u16, cuda_u16_as, upload_weight

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def q4():
    from moe_linear_layers_b200 import q4 as mod
    return mod


def _w4a16(q4, m, n, k, group, sym, kind="normal", tag="", rows_m=None):
    W = synth.weights(("test", "gemm", tag, n, k, group, sym), n, k)
    pk, sc, zr = oracle.quantize(W, group, sym)
    x = synth.activations(("test", "gemm-x", tag, m, k), m, k, kind)
    ref = oracle.linear_w4a16(x, pk, sc, zr, n, k, group, sym, rows_m=rows_m)
    w = upload_weight(q4, pk, sc, zr, n, k, group, sym)
    xd = cuda_u16_as(x, torch.bfloat16)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    y = q4.q4_linear_w4a16(xd, w, dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    yn = y.cpu().numpy()
    if rows_m is not None:
        yn = yn[rows_m]
    return yn, ref, w, xd, y


def test_w4a16_single_tile(q4):
    yn, ref, *_ = _w4a16(q4, 128, 128, 128, 128, False, tag="tile")
    assert_close(yn, ref, what="one tile")


@pytest.mark.parametrize("m,n,k,group,sym", [
    (5, 128, 128, 128, True),          # smallest m on the tensor-core path, one tile
    (64, 2048, 2048, 128, False),      # prefill m=64
    (200, 333, 256, 64, False),        # ragged m and n, group 64
    (130, 1000, 2048, 128, True),      # ragged, symmetric
    (512, 512, 8192, 128, False),      # long K (64 groups)
    (256, 8192, 2048, 128, False),     # many n tiles
    (1024, 256, 1024, 64, True),
])
def test_w4a16_gemm(q4, m, n, k, group, sym):
    yn, ref, *_ = _w4a16(q4, m, n, k, group, sym, tag="g")
    assert_close(yn, ref, what=f"w4a16 {m}x{n}x{k}")


@pytest.mark.parametrize("m,n,k", [(512, 2048, 2048), (2048, 2048, 8192)])
def test_w4a16_prefill_outlier_channels(q4, m, n, k):
    """Prefill shapes with 1% of activation channels x10; sampled rows of the oracle at full size."""
    rows = np.arange(0, m, max(1, m // 48))
    yn, ref, w, xd, y = _w4a16(q4, m, n, k, 128, False, kind="outlier_channels", tag="pre", rows_m=rows)
    assert_close(yn, ref, what=f"prefill {m}x{n}x{k}")
    y16 = q4.q4_linear_w4a16(xd, w, out_dtype=torch.bfloat16)
    assert np.array_equal(cpu_u16(y16), bf16_rne(y.cpu().numpy()))


def _w4a8(q4, m, n, k, group, tag, want_acc=False, sym=True):
    W = synth.weights(("test", "w4a8", tag, n, k, group), n, k)
    pk, sc, zr = oracle.quantize(W, group, sym)
    x = synth.activations(("test", "w4a8-x", tag, m, k), m, k, "student_t3")
    xq_ref, sa_ref = oracle.act_quant(x, k)
    w = upload_weight(q4, pk, sc, None if sym else zr, n, k, group, sym)
    xq, sa = q4.act_quant_per_token(cuda_u16_as(x, torch.bfloat16))
    acc = torch.zeros((m, n, k // group), dtype=torch.int32, device="cuda") if want_acc else None
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    y = q4.q4_linear_w4a8(xq, sa, w, acc_dbg=acc, dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    assert np.array_equal(xq.cpu().numpy(), xq_ref)
    return y, acc, (xq_ref, sa_ref, pk, sc, zr), w, xq, sa


@pytest.mark.parametrize("m,n,k,group", [(16, 128, 128, 128), (130, 333, 512, 128), (64, 256, 256, 64)])
def test_w4a8_int32_partials_bitexact(q4, m, n, k, group):
    y, acc, (xq, sa, pk, sc, _), *_ = _w4a8(q4, m, n, k, group, "acc", want_acc=True)
    ref, acc_ref = oracle.linear_w4a8(xq, sa, pk, sc, n, k, group, want_acc=True)
    assert np.array_equal(acc.cpu().numpy(), acc_ref)
    assert_close(y.cpu().numpy(), ref, what="w4a8")


@pytest.mark.parametrize("m,n,k", [(16, 2048, 2048), (256, 8192, 2048), (4096, 2048, 8192), (4096, 512, 2048)])
def test_w4a8_workload_shapes(q4, m, n, k):
    y, _, (xq, sa, pk, sc, _), w, xqd, sad = _w4a8(q4, m, n, k, 128, "shape")
    rows = np.arange(0, m, max(1, m // 32))
    ref = oracle.linear_w4a8(xq, sa, pk, sc, n, k, 128, rows_m=rows)
    assert_close(y.cpu().numpy()[rows], ref, what=f"w4a8 {m}x{n}x{k}")
    y16 = q4.q4_linear_w4a8(xqd, sad, w, out_dtype=torch.bfloat16)
    assert np.array_equal(cpu_u16(y16), bf16_rne(y.cpu().numpy()))


@pytest.mark.parametrize("m,n,k,group", [(16, 128, 128, 128), (130, 333, 512, 128), (64, 256, 256, 64),
                                         (200, 1000, 2048, 64)])
def test_w4a8_asym_int32_partials_bitexact(q4, m, n, k, group):
    """Asymmetric weights: the widened INT8 weight is code - zero; partials bit-exact."""
    y, acc, (xq, sa, pk, sc, zr), *_ = _w4a8(q4, m, n, k, group, "asym", want_acc=True, sym=False)
    ref, acc_ref = oracle.linear_w4a8(xq, sa, pk, sc, n, k, group, want_acc=True, zeros=zr, symmetric=False)
    assert np.array_equal(acc.cpu().numpy(), acc_ref)
    assert_close(y.cpu().numpy(), ref, what="w4a8 asym")


@pytest.mark.parametrize("m,n,k", [(4096, 2048, 2048), (256, 8192, 2048)])
def test_w4a8_asym_workload_shapes(q4, m, n, k):
    y, _, (xq, sa, pk, sc, zr), w, xqd, sad = _w4a8(q4, m, n, k, 128, "asym-shape", sym=False)
    rows = np.arange(0, m, max(1, m // 32))
    ref = oracle.linear_w4a8(xq, sa, pk, sc, n, k, 128, rows_m=rows, zeros=zr, symmetric=False)
    assert_close(y.cpu().numpy()[rows], ref, what=f"w4a8 asym {m}x{n}x{k}")


@pytest.mark.parametrize("m,n,k,group,sym", [
    (64, 2048, 1408, 128, False),   # 11 K blocks in splits of 3: a ragged last split
    (64, 2048, 1408, 64, True),     # two groups per K block
    (96, 640, 4096, 128, True),     # 5 output tiles, many splits
])
def test_w4a16_split_k(q4, m, n, k, group, sym):
    """A GEMM of few output tiles split along K (q4_linear_w4a16_ws): against the oracle, and against the
    unsplit form of the same call (the same per-group products, summed in another order)."""
    W = synth.weights(("test", "splitk", n, k, group, sym), n, k)
    pk, sc, zr = oracle.quantize(W, group, sym)
    x = synth.activations(("test", "splitk-x", m, k), m, k)
    ref = oracle.linear_w4a16(x, pk, sc, zr, n, k, group, sym)
    w = upload_weight(q4, pk, sc, zr, n, k, group, sym)
    assert q4._lib.q4_linear_workspace_size(m, ctypes.byref(w.desc)) > 0, "the shape should be split"
    xd = cuda_u16_as(x, torch.bfloat16)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    ys = q4.q4_linear_w4a16(xd, w, dev_status=st)
    yu = q4.q4_linear_w4a16(xd, w, dev_status=st, workspace=None)
    y16 = q4.q4_linear_w4a16(xd, w, out_dtype=torch.bfloat16, dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    assert_close(ys.cpu().numpy(), ref, what="split")
    assert_close(yu.cpu().numpy(), ref, what="unsplit")
    d = np.abs(ys.cpu().numpy() - yu.cpu().numpy()).max() / np.sqrt(np.mean(ref * ref))
    assert d < 1e-5, f"split and unsplit differ by {d} of rms"
    assert np.array_equal(cpu_u16(y16), bf16_rne(ys.cpu().numpy()))


@pytest.mark.parametrize("m,n,k,group,sym", [(16, 1024, 1408, 128, True), (32, 640, 2048, 64, False)])
def test_w4a8_split_k_partials_bitexact(q4, m, n, k, group, sym):
    """W4A8 split along K: every group's INT32 partial bit-exact (each group lies in one K range), y within
    tolerance of the oracle."""
    y, acc, (xq, sa, pk, sc, zr), w, *_ = _w4a8(q4, m, n, k, group, "split", want_acc=True, sym=sym)
    assert q4._lib.q4_linear_workspace_size(m, ctypes.byref(w.desc)) > 0, "the shape should be split"
    kw = {} if sym else dict(zeros=zr, symmetric=False)
    ref, acc_ref = oracle.linear_w4a8(xq, sa, pk, sc, n, k, group, want_acc=True, **kw)
    assert np.array_equal(acc.cpu().numpy(), acc_ref)
    assert_close(y.cpu().numpy(), ref, what="w4a8 split")


def test_stacked_weights_equal_their_parts(q4):
    """Q4Weight.stack: one GEMM over a layer's stacked projections (here q, k, v shaped, asymmetric g128)
    gives each part's output in its column range: equal to the part's own GEMM up to the fp32 order of
    its K sums, and to the oracle."""
    m, k = 64, 1024
    parts = []
    for tag, n in (("q", 512), ("k", 128), ("v", 128)):
        W = synth.weights(("test", "stack", tag, n, k), n, k)
        pk, sc, zr = oracle.quantize(W, 128, False)
        parts.append(((pk, sc, zr), upload_weight(q4, pk, sc, zr, n, k, 128, False), n))
    st = q4.Q4Weight.stack([w for _, w, _ in parts])
    assert st.n == 768 and st.k == k
    x = synth.activations(("test", "stack-x", m, k), m, k)
    xd = cuda_u16_as(x, torch.bfloat16)
    ys = q4.q4_linear_w4a16(xd, st)
    c0 = 0
    for (pk, sc, zr), w, n in parts:
        yp = q4.q4_linear_w4a16(xd, w)
        torch.cuda.synchronize()
        ref = oracle.linear_w4a16(x, pk, sc, zr, n, k, 128, False)
        part = ys[:, c0:c0 + n].cpu().numpy()
        assert_close(part, ref, what=f"stacked part at column {c0}")
        d = np.abs(part - yp.cpu().numpy()).max() / np.sqrt(np.mean(ref * ref))
        assert d < 1e-5, f"stacked and separate differ by {d} of rms"
        c0 += n
    with pytest.raises(ValueError):
        q4.Q4Weight.stack([parts[0][1], q4.q4_quantize_pack(torch.zeros((64, 512), device="cuda"), 128, False)])


@pytest.mark.parametrize("ws", ["auto", None])
def test_dependent_launches_keep_their_order(q4, ws):
    """The dense GEMM, its split-K reduction and the INT8 quantizer start early (programmatic dependent
    launch) and wait only before reading what the previous kernel wrote.  Read after write: y2 = GEMM(y1)
    right after y1 = GEMM(x) (bf16 y1).  Write after read: the quantizer overwrites the INT8 codes the
    previous W4A8 GEMM reads; each result must still be the oracle's for its own input."""
    m, k = 64, 1024
    W1 = synth.weights(("test", "pdl", 1), k, k)
    W2 = synth.weights(("test", "pdl", 2), k, k)
    q1, q2 = oracle.quantize(W1, 128, False), oracle.quantize(W2, 128, False)
    w1, w2 = upload_weight(q4, *q1, k, k, 128, False), upload_weight(q4, *q2, k, k, 128, False)
    x = synth.activations(("test", "pdl-x", m, k), m, k)
    y1 = q4.q4_linear_w4a16(cuda_u16_as(x, torch.bfloat16), w1, out_dtype=torch.bfloat16, workspace=ws)
    y2 = q4.q4_linear_w4a16(y1, w2, workspace=ws)
    torch.cuda.synchronize()
    y1u = cpu_u16(y1).reshape(m, k)
    # the bf16 y1 is held to the file's bf16 rule (rne of the fp32 output): bf16 rounding alone of the
    # exact product is 2.0e-2 of rms at this input, so the 1e-2 bar applies to the fp32 output
    y1f = q4.q4_linear_w4a16(cuda_u16_as(x, torch.bfloat16), w1, workspace=ws)
    torch.cuda.synchronize()
    assert_close(y1f.cpu().numpy(), oracle.linear_w4a16(x, *q1, k, k, 128, False), what="first GEMM")
    assert np.array_equal(y1u.reshape(-1), bf16_rne(y1f.cpu().numpy()).reshape(-1))
    assert_close(y2.cpu().numpy(), oracle.linear_w4a16(y1u, *q2, k, k, 128, False), what="GEMM on its output")
    # write after read through the quantizer and W4A8 (symmetric weights), one INT8 buffer for both inputs
    qs = oracle.quantize(W1, 128, True)
    ws8 = upload_weight(q4, qs[0], qs[1], None, k, k, 128, True)
    xa = synth.activations(("test", "pdl-xa", m, k), m, k, "student_t3")
    xb = synth.activations(("test", "pdl-xb", m, k), m, k, "student_t3")
    xq = torch.empty((m, k), dtype=torch.int8, device="cuda")
    sa = torch.empty((m,), dtype=torch.float32, device="cuda")
    q4.act_quant_per_token(cuda_u16_as(xa, torch.bfloat16), xq=xq, scale_a=sa)
    ya = q4.q4_linear_w4a8(xq, sa, ws8, workspace=ws)
    q4.act_quant_per_token(cuda_u16_as(xb, torch.bfloat16), xq=xq, scale_a=sa)
    yb = q4.q4_linear_w4a8(xq, sa, ws8, workspace=ws)
    torch.cuda.synchronize()
    for xin, y, tag in ((xa, ya, "first"), (xb, yb, "second")):
        xq_ref, sa_ref = oracle.act_quant(xin, k)
        assert_close(y.cpu().numpy(), oracle.linear_w4a8(xq_ref, sa_ref, qs[0], qs[1], k, k, 128), what=f"{tag} W4A8")
