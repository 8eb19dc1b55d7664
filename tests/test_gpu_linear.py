"""GPU parity: quantize/pack, W4A16 GEMV and per-token act-quant against the oracle, through the C ABI.

Integer outputs (codes, packed bytes, scales, zeros, INT8 activations and their scales) must be
bit-exact; floating outputs within max|err| <= 1e-2 * rms(reference) of the fp64 oracle."""
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
    assert torch.cuda.is_available()
    return mod


# ---------------------------------------------------------------------------------------------- #
# quantize + pack (bit-exact)
# ---------------------------------------------------------------------------------------------- #

@pytest.mark.parametrize("n,k,group,sym", [
    (128, 256, 64, True),      # the tiny single-linear workload
    (512, 2048, 128, False),   # k/v projection shape
    (77, 384, 128, False),     # ragged row count, 3 groups
    (3, 8192, 128, True),      # down projection width
    (1, 64, 64, False),        # a single group
    (8192, 2048, 128, False),  # a full gate projection
    (300, 1024, 32, False),    # group 32 (the hottest MoE experts' tier), asymmetric
    (64, 2048, 32, True),      # group 32, symmetric
    (300, 1024, 256, False),   # group 256 (the coldest MoE experts' tier), asymmetric
    (64, 2048, 256, True),     # group 256, symmetric
])
def test_quantize_bitexact(q4, n, k, group, sym):
    W = synth.weights(("test", "quant", n, k, group, sym), n, k)
    pk, sc, zr = oracle.quantize(W, group, sym)
    qw = q4.q4_quantize_pack(torch.from_numpy(W).cuda(), group, sym)
    torch.cuda.synchronize()
    assert np.array_equal(qw.packed.cpu().numpy(), pk)
    assert np.array_equal(cpu_u16(qw.scales), sc)
    if not sym:
        assert np.array_equal(cpu_u16(qw.zeros), zr)


def test_quantize_golden_and_edge_groups(q4):
    """Zero groups, all-positive groups and exact ties run through the kernel too."""
    W = np.zeros((4, 128), np.float32)
    W[1, :64] = np.linspace(0.1, 3.0, 64, dtype=np.float32)
    W[2] = np.repeat(np.array([1.75, -0.875, 0.5, 0.0], np.float32), 32)
    W[3, 64:] = -0.25
    for sym in (True, False):
        pk, sc, zr = oracle.quantize(W, 64, sym)
        qw = q4.q4_quantize_pack(torch.from_numpy(W).cuda(), 64, sym)
        assert np.array_equal(qw.packed.cpu().numpy(), pk)
        assert np.array_equal(cpu_u16(qw.scales), sc)
        if not sym:
            assert np.array_equal(cpu_u16(qw.zeros), zr)


def test_quantize_nonfinite_sets_status(q4):
    W = np.zeros((2, 128), np.float32)
    W[1, 3] = np.inf
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    q4.q4_quantize_pack(torch.from_numpy(W).cuda(), 64, True, dev_status=st)
    assert int(st.item()) == q4.Q4_ERR_NONFINITE


# ---------------------------------------------------------------------------------------------- #
# W4A16 GEMV (m <= 4)
# ---------------------------------------------------------------------------------------------- #

def _gemv_case(q4, n, k, group, sym, m, tag, out=torch.float32):
    W = synth.weights(("test", "gemv", tag, n, k), n, k)
    pk, sc, zr = oracle.quantize(W, group, sym)
    x = synth.activations(("test", "gemv-x", tag, m, k), m, k)
    ref = oracle.linear_w4a16(x, pk, sc, zr, n, k, group, sym)
    w = upload_weight(q4, pk, sc, zr, n, k, group, sym)
    y = q4.q4_linear_w4a16(cuda_u16_as(x, torch.bfloat16), w, out_dtype=out)
    torch.cuda.synchronize()
    return y, ref, w, x


def test_gemv_tiny_workload(q4):
    """W fp32 128x256 N(0, 0.02) with 0.1% outliers x20, symmetric g64; x bf16 1x256; seed 0."""
    W = synth.weights((0, "tiny-linear", "W"), 128, 256)
    x = synth.activations((0, "tiny-linear", "x"), 1, 256)
    pk, sc, zr = oracle.quantize(W, 64, True)
    ref = oracle.linear_w4a16(x, pk, sc, zr, 128, 256, 64, True)
    qw = q4.q4_quantize_pack(torch.from_numpy(W).cuda(), 64, True)   # the product path end to end
    y = q4.q4_linear_w4a16(cuda_u16_as(x, torch.bfloat16), qw)
    assert_close(y.cpu().numpy(), ref, what="tiny")


@pytest.mark.parametrize("n,k,group,sym", [
    (2048, 2048, 128, False), (512, 2048, 128, False), (8192, 2048, 128, False), (2048, 8192, 128, False),
    (2048, 2048, 128, True), (77, 256, 64, False), (300, 16384, 128, True), (1000, 4096, 64, False),
    (5, 1024, 128, True), (1, 32 * 64, 64, False), (3000, 1024 + 64, 64, True),
])
def test_gemv_m1(q4, n, k, group, sym):
    y, ref, *_ = _gemv_case(q4, n, k, group, sym, 1, "m1")
    assert_close(y.cpu().numpy(), ref, what=f"gemv {n}x{k}")


@pytest.mark.parametrize("m", [2, 3, 4])
@pytest.mark.parametrize("n,k,group,sym", [(2048, 2048, 128, False), (333, 8192, 128, True), (64, 256, 64, False)])
def test_gemv_small_m(q4, m, n, k, group, sym):
    y, ref, *_ = _gemv_case(q4, n, k, group, sym, m, "sm")
    assert_close(y.cpu().numpy(), ref, what=f"gemv m={m} {n}x{k}")


@pytest.mark.parametrize("m", [1, 3])
def test_gemv_grouped_matches_oracle(q4, m):
    """q, k, v of one layer (same k, different n) in one launch, each with its own x."""
    shapes = [(2048, 2048), (512, 2048), (512, 2048)]
    xs, ws, ys, refs = [], [], [], []
    for i, (n, k) in enumerate(shapes):
        W = synth.weights(("test", "grp", i), n, k)
        pk, sc, zr = oracle.quantize(W, 128, False)
        x = synth.activations(("test", "grp-x", i, m), m, k)
        refs.append(oracle.linear_w4a16(x, pk, sc, zr, n, k, 128, False))
        ws.append(upload_weight(q4, pk, sc, zr, n, k, 128, False))
        xs.append(cuda_u16_as(x, torch.bfloat16))
        ys.append(torch.empty((m, n), dtype=torch.float32, device="cuda"))
    q4.q4_linear_w4a16_grouped(xs, ws, ys)
    torch.cuda.synchronize()
    for i in range(len(shapes)):
        assert_close(ys[i].cpu().numpy(), refs[i], what=f"grouped problem {i}")
        # the grouped result is the single-call result, bit for bit
        y1 = q4.q4_linear_w4a16(xs[i], ws[i])
        assert torch.equal(y1, ys[i])


def test_gemv_bf16_out_is_rounded_fp32(q4):
    y32, ref, w, x = _gemv_case(q4, 1024, 2048, 128, False, 1, "bf16")
    y16 = q4.q4_linear_w4a16(cuda_u16_as(x, torch.bfloat16), w, out_dtype=torch.bfloat16)
    assert np.array_equal(cpu_u16(y16), bf16_rne(y32.cpu().numpy()))


def test_gemv_nonfinite_x_sets_status(q4):
    W = synth.weights(("test", "nan"), 64, 256)
    pk, sc, zr = oracle.quantize(W, 64, True)
    w = upload_weight(q4, pk, sc, zr, 64, 256, 64, True)
    x = torch.zeros((1, 256), dtype=torch.bfloat16, device="cuda")
    x[0, 17] = float("nan")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    q4.q4_linear_w4a16(x, w, dev_status=st)
    assert int(st.item()) == q4.Q4_ERR_NONFINITE


# ---------------------------------------------------------------------------------------------- #
# per-token INT8 activation quantization (bit-exact)
# ---------------------------------------------------------------------------------------------- #

@pytest.mark.parametrize("m,k", [(16, 2048), (256, 8192), (7, 24), (4096, 2048), (1, 8)])
def test_act_quant_bitexact(q4, m, k):
    x = synth.activations(("test", "aq", m, k), m, k, "student_t3")
    if m > 2:
        x[1] = 0           # an all-zero token
        x[2, : k // 2] = 0
    q_ref, s_ref = oracle.act_quant(x, k)
    xq, s = q4.act_quant_per_token(cuda_u16_as(x, torch.bfloat16))
    torch.cuda.synchronize()
    assert np.array_equal(s.cpu().numpy().view(np.uint32), s_ref.view(np.uint32))
    assert np.array_equal(xq.cpu().numpy(), q_ref)


@pytest.mark.parametrize("m,k", [(33, 1024), (256, 2048), (5, 8192), (3, 20000), (1, 8)])
def test_act_quant_f16_bitexact(q4, m, k):
    """fp16 rows (the MoE's intermediate activations): codes and scales bit-exact against the oracle.
    Rows span fp16's range: subnormal-only rows, ordinary rows, rows near the fp16 maximum."""
    rng = np.random.default_rng(m * 7919 + k)
    mags = [2.0 ** -20, 2.0 ** -14, 1e-3, 0.5, 3.0, 100.0, 8e3]
    h = np.stack([np.clip(rng.standard_normal(k) * mags[i % len(mags)], -65000.0, 65000.0)
                  for i in range(m)]).astype(np.float16)
    if m > 2:
        h[1] = 0
    bits = h.view(np.uint16)
    q_ref, s_ref = oracle.act_quant_f16(bits, k)
    xq, sc = q4.act_quant_per_token(cuda_u16_as(bits, torch.float16))
    torch.cuda.synchronize()
    assert np.array_equal(sc.cpu().numpy().view(np.uint32), s_ref.view(np.uint32))
    assert np.array_equal(xq.cpu().numpy(), q_ref)


def test_act_quant_f16_nonfinite_status(q4):
    h = np.ones((4, 64), np.float16)
    h[2, 5] = np.inf
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    q4.act_quant_per_token(cuda_u16_as(h.view(np.uint16), torch.float16), dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == q4.Q4_ERR_NONFINITE


def test_act_quant_rounding_stress(q4):
    """Quotients at and next to half-integers, scales with full mantissas, and extreme magnitudes (tiny
    rows take the kernel's division path, the rest the reciprocal-and-FMA path): codes and scales
    bit-exact against the oracle's IEEE division."""
    rng = np.random.default_rng(7)
    k = 2048
    rows = []
    # the quotient grid itself: amax 127 gives s = 1, values on and between half-integers
    g = np.arange(-127.0, 127.5, 0.5, dtype=np.float32)
    rows.append(np.resize(g, k))
    # random magnitudes spanning the bf16 exponent range, with the amax chosen to give awkward scales
    for e in (-130, -110, -100, -99, -96, -95, -60, -20, -3, 0, 5, 30, 90, 120):
        r = rng.standard_normal(k).astype(np.float32) * np.float32(2.0 ** e)
        r[rng.integers(k)] = np.float32(1.37 * 2.0 ** (e + 2))
        rows.append(r)
    # values placed right at q + 0.5 of a non-power-of-two scale, and one bf16 ulp to either side
    s = np.float32(100.0) / np.float32(127.0)
    base = (np.arange(k) % 255 - 127).astype(np.float32)
    for d in (0.5, 0.49, 0.51):
        r = ((base + np.float32(d)) * s).astype(np.float32)
        r[0] = np.float32(100.0)
        rows.append(r)
    x = synth.to_bf16_bits(np.stack(rows).astype(np.float32))
    q_ref, s_ref = oracle.act_quant(x, k)
    xq, sc = q4.act_quant_per_token(cuda_u16_as(x, torch.bfloat16))
    torch.cuda.synchronize()
    assert np.array_equal(sc.cpu().numpy().view(np.uint32), s_ref.view(np.uint32))
    assert np.array_equal(xq.cpu().numpy(), q_ref)


def test_act_quant_golden_rows(q4):
    x = synth.to_bf16_bits(np.array([[127, -63.5, 0.5, 2, 0, 0, 0, 0], [-127, 2.5, -2.5, 1.5, 0, 0, 0, 0]], np.float32))
    xq, s = q4.act_quant_per_token(cuda_u16_as(x, torch.bfloat16))
    assert s.cpu().tolist() == [1.0, 1.0]
    assert xq.cpu().numpy()[:, :4].tolist() == [[127, -64, 0, 2], [-127, 2, -2, 2]]


def test_act_quant_nonfinite_sets_status(q4):
    x = torch.ones((3, 64), dtype=torch.bfloat16, device="cuda")
    x[2, 5] = float("inf")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    q4.act_quant_per_token(x, dev_status=st)
    assert int(st.item()) == q4.Q4_ERR_NONFINITE


# ---------------------------------------------------------------------------------------------- #
# dense SwiGLU FFN down projection with the gating fused into the GEMV's input
# ---------------------------------------------------------------------------------------------- #

@pytest.mark.parametrize("m,n,k,group,sym", [(1, 2048, 8192, 128, False), (2, 333, 1024, 64, True),
                                             (4, 512, 2048, 128, False), (1, 130, 64, 64, False)])
def test_w4a16_swiglu_fused_input(q4, m, n, k, group, sym):
    W = synth.weights(("test", "swiglu", n, k, group, sym), n, k)
    pk, sc, zr = oracle.quantize(W, group, sym)
    gate = (synth.normal(synth.stream_key("test", "swiglu-g", m, k), m * k) * 2.0).astype(np.float32).reshape(m, k)
    up = synth.normal(synth.stream_key("test", "swiglu-u", m, k), m * k).astype(np.float32).reshape(m, k)
    ref = oracle.linear_w4a16_swiglu(gate, up, pk, sc, zr, n, k, group, sym)
    w = upload_weight(q4, pk, sc, None if sym else zr, n, k, group, sym)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    y = q4.q4_linear_w4a16_swiglu(torch.from_numpy(gate).cuda(), torch.from_numpy(up).cuda(), w, dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    assert_close(y.cpu().numpy(), ref, what=f"swiglu gemv {m}x{n}x{k}")


def test_w4a16_swiglu_nonfinite_status(q4):
    n, k = 128, 256
    W = synth.weights(("test", "swiglu-nf"), n, k)
    pk, sc, zr = oracle.quantize(W, 128, True)
    w = upload_weight(q4, pk, sc, None, n, k, 128, True)
    gate = torch.ones((1, k), dtype=torch.float32, device="cuda")
    up = torch.ones((1, k), dtype=torch.float32, device="cuda")
    up[0, 77] = float("inf")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    q4.q4_linear_w4a16_swiglu(gate, up, w, dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == q4.Q4_ERR_NONFINITE


# ---------------------------------------------------------------------------------------------- #
# failure detection: a wait that nothing satisfies gives up, records Q4_ERR_TIMEOUT, and the context
# stays usable (no fault, no hang)
# ---------------------------------------------------------------------------------------------- #

@pytest.mark.parametrize("which", [0, 1])
def test_bounded_wait_times_out_cleanly(q4, which):
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    q4.q4_selftest_bounded_wait(which, 2000, st)
    torch.cuda.synchronize()
    assert int(st.item()) == q4.Q4_ERR_TIMEOUT
    # the context still works: a small linear afterwards is correct
    n, k = 64, 256
    W = synth.weights(("test", "after-timeout"), n, k)
    pk, sc, zr = oracle.quantize(W, 128, True)
    w = upload_weight(q4, pk, sc, None, n, k, 128, True)
    x = synth.activations(("test", "after-timeout-x"), 1, k)
    y = q4.q4_linear_w4a16(cuda_u16_as(x, torch.bfloat16), w)
    torch.cuda.synchronize()
    assert_close(y.cpu().numpy(), oracle.linear_w4a16(x, pk, sc, None, n, k, 128, True), what="after timeout")
