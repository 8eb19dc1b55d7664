"""Pins for the oracle: each check ties it to something other than itself -- hand-worked values
(tests/golden/), closed forms (exact-grid round trips), invariants of the method, library routines
computing the same mathematics (numpy fp64 matmul, stable argsort, numpy's fp16 conversion) and
special cases that reduce to a dense layer.  No GPU involved."""
import os

import numpy as np
import pytest

import oracle
from moe_linear_layers_b200 import synth

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _rows(name):
    with open(os.path.join(GOLD, name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                yield [c.strip() for c in line.split("|")]


def _unpack_numpy(packed, k, symmetric):
    """Independent unpacking with numpy bit operations (even k in the low nibble)."""
    lo = (packed & 0x0F).astype(np.int16)
    hi = (packed >> 4).astype(np.int16)
    codes = np.empty((packed.shape[0], k), np.int16)
    codes[:, 0::2] = lo
    codes[:, 1::2] = hi
    if symmetric:
        codes = np.where(codes >= 8, codes - 16, codes)
    return codes


def _f16(bits):
    return np.asarray(bits, dtype=np.uint16).view(np.float16).astype(np.float64)


def _f16_bits(values):
    return np.asarray(values, dtype=np.float16).view(np.uint16)


# ---------------------------------------------------------------------------------------------- #
# number formats
# ---------------------------------------------------------------------------------------------- #

def test_f16_conversion_matches_numpy():
    rng = np.random.default_rng(0)
    vals = np.concatenate([
        rng.standard_normal(20000).astype(np.float32) * np.float32(3.0),
        (rng.standard_normal(5000) * 1e-5).astype(np.float32),      # fp16 subnormal range
        (rng.standard_normal(2000) * 1e-8).astype(np.float32),      # underflow to zero
        (rng.standard_normal(2000) * 6e4).astype(np.float32),       # overflow edge
        np.array([65504, 65519.99, 65520, -65520, 2 ** -24, 2 ** -25, 3 * 2 ** -26, 2 ** -14, 0.0, -0.0,
                  np.inf, -np.inf], np.float32),
    ])
    # exact ties at fp16 resolution: odd multiples of half an ulp
    k = np.arange(1, 4000, 2, dtype=np.float32)
    vals = np.concatenate([vals, (np.float32(1.0) + k * np.float32(2 ** -11)) % np.float32(2.0) + 1.0])
    with np.errstate(over="ignore"):   # values past 65519.99 overflow to infinity on purpose
        ref = vals.astype(np.float16).view(np.uint16)
    got = np.array([oracle.f32_to_f16_bits(float(v)) for v in vals], np.uint16)
    assert np.array_equal(got, ref)
    assert oracle.f32_to_f16_bits(float("nan")) & 0x7C00 == 0x7C00


def test_f16_to_f32_all_patterns():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ref = bits.view(np.float16).astype(np.float32)
    got = np.array([oracle.f16_bits_to_f32(int(b)) for b in bits], np.float32)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan].view(np.uint32), ref[~nan].view(np.uint32))


# ---------------------------------------------------------------------------------------------- #
# quantizer: hand-worked groups
# ---------------------------------------------------------------------------------------------- #

@pytest.mark.parametrize("row", list(_rows("quant_groups.txt")))
def test_golden_groups(row):
    kind, group, values, scale, zero, codes, packed = row
    sym = kind == "sym"
    g = int(group)
    w = np.array([float(v) for v in values.split()], np.float32).reshape(1, -1)
    pk, sc, zr = oracle.quantize(w, g, sym)
    assert int(sc[0, 0]) == int(scale, 16)
    if not sym:
        assert int(zr[0, 0]) == int(zero, 16)
    assert list(pk[0]) == [int(b, 16) for b in packed.split()]
    assert list(oracle.unpack_codes(pk, w.shape[1], sym)[0]) == [int(c) for c in codes.split()]


@pytest.mark.parametrize("row", list(_rows("act_quant.txt")))
def test_golden_act_quant(row):
    values, scale, codes = row
    x = synth.to_bf16_bits(np.array([float(v) for v in values.split()], np.float32)).reshape(1, -1)
    assert np.array_equal(synth.bf16_bits_to_f32(x)[0], np.array([float(v) for v in values.split()], np.float32))
    q, s = oracle.act_quant(x, x.shape[1])
    assert float(s[0]) == float(scale)
    assert list(q[0]) == [int(c) for c in codes.split()]


# ---------------------------------------------------------------------------------------------- #
# quantizer: exact-grid round trip (closed form)
# ---------------------------------------------------------------------------------------------- #

def _exact_grid(n, k, group, symmetric, seed):
    """Weights W = (q - z) * S exactly, with every group's extremes at the code limits, so the
    quantizer must return exactly (q, S, z)."""
    rng = np.random.default_rng(seed)
    ng = k // group
    # fp16 scales: normal fp16 values in [2^-10, 2^-3]
    sbits = rng.integers(0x1400, 0x3000, size=(n, ng)).astype(np.uint16)
    S = _f16(sbits).astype(np.float32)
    if symmetric:
        q = rng.integers(-7, 8, size=(n, k))
        z = np.zeros((n, ng), np.int64)
        for g in range(ng):  # force |q| = 7 somewhere in each group
            q[:, g * group] = np.where(rng.random(n) < 0.5, 7, -7)
    else:
        q = rng.integers(0, 16, size=(n, k))
        z = rng.integers(0, 16, size=(n, ng))
        for g in range(ng):  # both extremes 0 and 15 present
            q[:, g * group] = 0
            q[:, g * group + 1] = 15
    zf = np.repeat(z, group, axis=1)
    Sf = np.repeat(S, group, axis=1)
    W = ((q - zf).astype(np.float32) * Sf).astype(np.float32)
    return W, q, sbits, z


@pytest.mark.parametrize("symmetric", [True, False])
@pytest.mark.parametrize("group", [32, 64, 128, 256])
def test_exact_grid_roundtrip(symmetric, group):
    n, k = 37, 512
    W, q, sbits, z = _exact_grid(n, k, group, symmetric, seed=group + symmetric)
    pk, sc, zr = oracle.quantize(W, group, symmetric)
    assert np.array_equal(sc, sbits)
    if not symmetric:
        assert np.array_equal(_f16(zr), z.astype(np.float64))
    stored = _unpack_numpy(pk, k, symmetric)
    expect = q if symmetric else q
    assert np.array_equal(stored, expect)
    # the dequantized matrix reproduces W exactly
    assert np.array_equal(oracle.dequant(pk, sc, zr, k, group, symmetric), W)


# ---------------------------------------------------------------------------------------------- #
# quantizer: invariants on the workloads' weight distribution
# ---------------------------------------------------------------------------------------------- #

@pytest.mark.parametrize("symmetric", [True, False])
@pytest.mark.parametrize("group", [32, 64, 128, 256])
def test_quant_invariants(symmetric, group):
    n, k = 64, 1024
    W = synth.weights(("pins", "inv", group, symmetric), n, k)
    pk, sc, zr = oracle.quantize(W, group, symmetric)
    codes = _unpack_numpy(pk, k, symmetric)
    if symmetric:
        assert codes.min() >= -7 and codes.max() <= 7          # -8 never produced
    else:
        assert codes.min() >= 0 and codes.max() <= 15
    S = np.repeat(_f16(sc), group, axis=1)
    zf = 0.0 if symmetric else np.repeat(_f16(zr), group, axis=1)
    deq = (codes - zf) * S
    assert np.array_equal(deq.astype(np.float32), oracle.dequant(pk, sc, zr, k, group, symmetric))
    err = np.abs(W.astype(np.float64) - deq)
    lo, hi = (-7, 7) if symmetric else (0, 15)
    interior = (codes > lo) & (codes < hi)
    assert np.all(err[interior] <= S[interior] / 2 * (1 + 1e-6))
    # at the clamped ends fp16 rounding of the scale adds at most 15*|s32 - S| <= S/2 * 2^-6
    assert np.all(err <= S / 2 * (1 + 2.0 ** -6) * (1 + 1e-6))
    # idempotence: quantizing the dequantized weights reproduces the codes, scales and zeros
    pk2, sc2, zr2 = oracle.quantize(deq.astype(np.float32), group, symmetric)
    if symmetric:
        assert np.array_equal(pk2, pk) and np.array_equal(sc2, sc)
    else:
        # holds for every group whose extremes code to 0 and 15 (or whose extreme is the added 0)
        cg = codes.reshape(n, k // group, group)
        ok = ((cg.min(axis=2) == 0) & (cg.max(axis=2) == 15))
        c2 = _unpack_numpy(pk2, k, False).reshape(n, k // group, group)
        assert np.array_equal(c2[ok], cg[ok])
        assert np.array_equal(sc2[ok], sc[ok]) and np.array_equal(zr2[ok], zr[ok])
        assert ok.mean() > 0.5


def test_row_concatenation_invariance():
    W1 = synth.weights(("pins", "cat", 1), 20, 256)
    W2 = synth.weights(("pins", "cat", 2), 12, 256)
    for sym in (True, False):
        a = oracle.quantize(np.concatenate([W1, W2]), 128, sym)
        b1 = oracle.quantize(W1, 128, sym)
        b2 = oracle.quantize(W2, 128, sym)
        for i in range(2):
            assert np.array_equal(a[i], np.concatenate([b1[i], b2[i]]))


def test_nonfinite_is_an_error():
    W = np.zeros((2, 128), np.float32)
    W[1, 5] = np.nan
    with pytest.raises(oracle.OracleError):
        oracle.quantize(W, 64, True)
    W[1, 5] = 1e30   # scale overflows fp16
    with pytest.raises(oracle.OracleError):
        oracle.quantize(W, 64, False)


# ---------------------------------------------------------------------------------------------- #
# W4A16 linear vs a library fp64 matmul on exact-grid weights
# ---------------------------------------------------------------------------------------------- #

@pytest.mark.parametrize("symmetric", [True, False])
def test_linear_matches_numpy_matmul(symmetric):
    n, k, group, m = 45, 384, 128, 5
    W, q, sbits, z = _exact_grid(n, k, group, symmetric, seed=7)
    pk, sc, zr = oracle.quantize(W, group, symmetric)
    x = synth.activations(("pins", "lin"), m, k)
    y = oracle.linear_w4a16(x, pk, sc, zr, n, k, group, symmetric)
    ref = synth.bf16_bits_to_f32(x).astype(np.float64) @ W.astype(np.float64).T
    np.testing.assert_allclose(y, ref, rtol=1e-12, atol=1e-12)
    # sampled outputs are the same numbers
    rm, rn = np.array([4, 0]), np.array([44, 3, 17])
    ys = oracle.linear_w4a16(x, pk, sc, zr, n, k, group, symmetric, rows_m=rm, rows_n=rn)
    assert np.array_equal(ys, y[np.ix_(rm, rn)])


def test_linear_brute_force_tiny():
    """K = G = 4, every combination of a small grid of codes and activations."""
    vals = [-2.0, -0.5, 0.0, 1.0, 3.0]
    xs = np.array(np.meshgrid(*[vals] * 4)).reshape(4, -1).T.astype(np.float32)   # 625 rows
    xb = synth.to_bf16_bits(xs)
    for sym in (True, False):
        rng = np.random.default_rng(3)
        W, q, sbits, z = _exact_grid(16, 4, 4, sym, seed=11 + sym)
        pk, sc, zr = oracle.quantize(W, 4, sym)
        y = oracle.linear_w4a16(xb, pk, sc, zr, 16, 4, 4, sym)
        for i in range(0, xs.shape[0], 37):
            for r in range(16):
                expect = sum(float(xs[i, c]) * float(W[r, c]) for c in range(4))
                assert abs(y[i, r] - expect) <= 1e-12 * (1 + abs(expect))


# ---------------------------------------------------------------------------------------------- #
# activation quantization properties
# ---------------------------------------------------------------------------------------------- #

def test_act_quant_properties():
    x = synth.activations(("pins", "act"), 64, 2048, "student_t3")
    x[3] = 0  # an all-zero token
    q, s = oracle.act_quant(x, 2048)
    xf = synth.bf16_bits_to_f32(x).astype(np.float64)
    amax = np.abs(xf).max(axis=1)
    assert np.array_equal(s, (amax.astype(np.float32) / np.float32(127.0)))
    assert q.min() >= -127 and q.max() <= 127                    # -128 never produced
    nz = s > 0
    err = np.abs(xf[nz] - q[nz] * s[nz, None].astype(np.float64))
    assert np.all(err <= s[nz, None] * (0.5 + 1e-6))
    # the amax element maps to +-127
    i = np.abs(xf).argmax(axis=1)
    assert np.all(np.abs(q[nz, i[nz]]) == 127)
    assert np.all(q[3] == 0) and s[3] == 0


# ---------------------------------------------------------------------------------------------- #
# W4A8: unit scales reduce it to an integer matmul
# ---------------------------------------------------------------------------------------------- #

def test_w4a8_unit_scales_is_integer_matmul():
    n, k, group, m = 33, 512, 128, 7
    rng = np.random.default_rng(5)
    codes = rng.integers(-8, 8, size=(n, k))
    packed = ((codes[:, 0::2] & 0xF) | ((codes[:, 1::2] & 0xF) << 4)).astype(np.uint8)
    scales = np.full((n, k // group), 0x3C00, np.uint16)     # fp16 1.0
    xq = rng.integers(-128, 128, size=(m, k)).astype(np.int8)
    s_a = np.ones(m, np.float32)
    y, acc = oracle.linear_w4a8(xq, s_a, packed, scales, n, k, group, want_acc=True)
    full = xq.astype(np.int64) @ codes.T.astype(np.int64)
    assert np.array_equal(y, full.astype(np.float64))
    for g in range(k // group):
        sl = slice(g * group, (g + 1) * group)
        assert np.array_equal(acc[:, :, g], xq[:, sl].astype(np.int64) @ codes[:, sl].T.astype(np.int64))


def test_w4a8_scaling():
    n, k, group, m = 9, 256, 128, 3
    W, q, sbits, z = _exact_grid(n, k, group, True, seed=21)
    pk, sc, _ = oracle.quantize(W, group, True)
    x = synth.activations(("pins", "w4a8"), m, k, "student_t3")
    xq, s_a = oracle.act_quant(x, k)
    y = oracle.linear_w4a8(xq, s_a, pk, sc, n, k, group)
    ref = (xq.astype(np.float64) * s_a[:, None].astype(np.float64)) @ W.astype(np.float64).T
    np.testing.assert_allclose(y, ref, rtol=1e-12, atol=1e-12)


def test_w4a8_asym_unit_scales_is_integer_matmul_with_zero_points():
    """Asymmetric weights: the widened INT8 weight is q - z (q in 0..15, z the group's zero point)."""
    n, k, group, m = 21, 256, 64, 5
    rng = np.random.default_rng(6)
    codes = rng.integers(0, 16, size=(n, k))
    z = rng.integers(0, 16, size=(n, k // group))
    packed = (codes[:, 0::2] | (codes[:, 1::2] << 4)).astype(np.uint8)
    scales = np.full((n, k // group), 0x3C00, np.uint16)     # fp16 1.0
    zeros = _f16_bits(z.astype(np.float32))
    xq = rng.integers(-128, 128, size=(m, k)).astype(np.int8)
    s_a = np.ones(m, np.float32)
    y, acc = oracle.linear_w4a8(xq, s_a, packed, scales, n, k, group, want_acc=True, zeros=zeros, symmetric=False)
    w_int = codes - np.repeat(z, group, axis=1)
    assert np.array_equal(y, (xq.astype(np.int64) @ w_int.T.astype(np.int64)).astype(np.float64))
    for g in range(k // group):
        sl = slice(g * group, (g + 1) * group)
        assert np.array_equal(acc[:, :, g], xq[:, sl].astype(np.int64) @ w_int[:, sl].T.astype(np.int64))


def test_w4a8_asym_zero_eight_equals_symmetric():
    """Codes c in -8..7 stored symmetric, or as c + 8 with zero point 8, give the same partials."""
    n, k, group, m = 13, 256, 128, 4
    rng = np.random.default_rng(7)
    c = rng.integers(-8, 8, size=(n, k))
    sym_packed = ((c[:, 0::2] & 0xF) | ((c[:, 1::2] & 0xF) << 4)).astype(np.uint8)
    u = c + 8
    asym_packed = (u[:, 0::2] | (u[:, 1::2] << 4)).astype(np.uint8)
    sbits = rng.integers(0x1400, 0x3000, size=(n, k // group)).astype(np.uint16)
    zeros = np.full((n, k // group), 0x4800, np.uint16)      # fp16 8.0
    x = synth.activations(("pins", "w4a8-z8"), m, k, "student_t3")
    xq, s_a = oracle.act_quant(x, k)
    y1, a1 = oracle.linear_w4a8(xq, s_a, sym_packed, sbits, n, k, group, want_acc=True)
    y2, a2 = oracle.linear_w4a8(xq, s_a, asym_packed, sbits, n, k, group, want_acc=True, zeros=zeros,
                                symmetric=False)
    assert np.array_equal(a1, a2) and np.array_equal(y1, y2)


def test_w4a8_asym_scaling():
    """Asymmetric W4A8 equals the fp64 product of the dequantized activations and weights."""
    n, k, group, m = 9, 256, 128, 3
    W, q, sbits, z = _exact_grid(n, k, group, False, seed=22)
    pk, sc, zr = oracle.quantize(W, group, False)
    x = synth.activations(("pins", "w4a8-asym"), m, k, "student_t3")
    xq, s_a = oracle.act_quant(x, k)
    y = oracle.linear_w4a8(xq, s_a, pk, sc, n, k, group, zeros=zr, symmetric=False)
    ref = (xq.astype(np.float64) * s_a[:, None].astype(np.float64)) @ W.astype(np.float64).T
    np.testing.assert_allclose(y, ref, rtol=1e-12, atol=1e-12)


# ---------------------------------------------------------------------------------------------- #
# SwiGLU-gated input of the dense FFN's down projection
# ---------------------------------------------------------------------------------------------- #

def test_silu_mul_identities():
    """silu(g) - silu(-g) = g (sigmoid(-g) = 1 - sigmoid(g)); silu(0) = 0; u scales linearly."""
    g = np.linspace(-30, 30, 2001, dtype=np.float32)
    one = np.ones_like(g)
    d = oracle.silu_mul(g, one) - oracle.silu_mul(-g, one)
    np.testing.assert_allclose(d, g.astype(np.float64), rtol=1e-14, atol=1e-14)
    assert oracle.silu_mul(np.float32(0), np.float32(5)) == 0.0
    u = np.float32(3.0)
    np.testing.assert_allclose(oracle.silu_mul(g, u * one), 3.0 * oracle.silu_mul(g, one), rtol=1e-15)


def test_swiglu_linear_reduces_to_plain_linear_for_saturated_gate():
    """With gate = 32 (sigmoid(32) = 1 - 1.3e-14) and up = x / 32 (exact), h = x to 1e-13: the fused
    product equals the plain W4A16 product on x."""
    n, k, group, m = 24, 512, 128, 2
    W = synth.weights(("pins", "swiglu"), n, k)
    pk, sc, zr = oracle.quantize(W, group, False)
    x = synth.activations(("pins", "swiglu-x"), m, k)
    xf = (x.astype(np.uint32) << 16).view(np.float32)
    gate = np.full((m, k), 32.0, np.float32)
    up = (xf / np.float32(32.0)).astype(np.float32)
    y = oracle.linear_w4a16_swiglu(gate, up, pk, sc, zr, n, k, group, False)
    ref = oracle.linear_w4a16(x, pk, sc, zr, n, k, group, False)
    np.testing.assert_allclose(y, ref, rtol=1e-12, atol=1e-12 * np.abs(ref).max())


def test_shared_expert_is_the_dense_swiglu_ffn():
    """The shared expert (one SwiGLU FFN every token passes through, weight 1) equals the dense FFN computed
    another way: the two W4A16 products from linear_w4a16, silu(g) * u, and the down product of the
    dequantized matrix."""
    T, H, I_s, group = 5, 256, 128, 128
    x = synth.activations(("pins", "shared-x"), T, H)
    qs = [oracle.quantize(synth.weights(("pins", "shared", nm), n, k), group, False)
          for nm, n, k in (("g", I_s, H), ("u", I_s, H), ("d", H, I_s))]
    y = oracle.shared_expert(x, H, qs[0], qs[1], qs[2], I_s, group, False)
    g = oracle.linear_w4a16(x, *qs[0], I_s, H, group, False)
    u = oracle.linear_w4a16(x, *qs[1], I_s, H, group, False)
    h = g / (1.0 + np.exp(-g)) * u
    wd = oracle.dequant(*qs[2], I_s, group, False).astype(np.float64)
    np.testing.assert_allclose(y, h @ wd.T, rtol=1e-11, atol=1e-12 * np.abs(y).max())


# ---------------------------------------------------------------------------------------------- #
# router and permutation
# ---------------------------------------------------------------------------------------------- #

def test_route_selection_and_weights():
    T, H, E, topk = 96, 256, 16, 4
    x = synth.activations(("pins", "route"), T, H)
    Wr, bias = synth.router(("pins", "route"), E, H)
    logits, ids, w, counts = oracle.route(x, H, Wr, bias, topk)
    xf = synth.bf16_bits_to_f32(x).astype(np.float64)
    exact = xf @ Wr.astype(np.float64).T + bias.astype(np.float64)
    bound = (np.abs(xf) @ np.abs(Wr.astype(np.float64)).T) * H * 2.0 ** -23 + np.abs(bias) * 2.0 ** -23
    assert np.all(np.abs(logits - exact) <= bound)
    order = np.lexsort((np.broadcast_to(np.arange(E), logits.shape), -logits.astype(np.float64)), axis=1)
    assert np.array_equal(ids, order[:, :topk])
    p = np.exp(logits.astype(np.float64) - logits.max(axis=1, keepdims=True))
    p /= p.sum(axis=1, keepdims=True)                      # softmax over all experts
    sel = np.take_along_axis(p, ids, axis=1)
    np.testing.assert_allclose(w, sel / sel.sum(axis=1, keepdims=True), rtol=1e-12)
    assert np.array_equal(counts, np.bincount(ids.ravel(), minlength=E))


def _fp32_round(q):
    """The fp32 nearest to the rational q, ties to even (an exact rounding: fp64 conversion can round twice)."""
    from fractions import Fraction
    if q == 0:
        return np.float32(0.0)
    f = np.float32(float(q))
    best = None
    for c in (f, np.nextafter(f, np.float32(np.inf)), np.nextafter(f, np.float32(-np.inf))):
        d = abs(Fraction(float(c)) - q)
        key = (d, int(np.array(c, np.float32).view(np.uint32)) & 1)   # on a tie the even significand wins
        if best is None or key < best[0]:
            best = (key, c)
    return np.float32(best[1])


def _fma32(a, b, c):
    """fp32 fused multiply-add with one rounding: a * b + c formed exactly as a rational, then rounded."""
    from fractions import Fraction
    return _fp32_round(Fraction(float(a)) * Fraction(float(b)) + Fraction(float(c)))


def test_router_logit_pinned_order_bit_exact():
    """The pinned fp32 order of the router logits, restated independently: 32 lane partials, each a chain
    of correctly rounded fp32 fmas over k = l, l + 32, ... from +0, then the xor butterfly p_l + p_(l^s) for
    s = 16, 8, 4, 2, 1 in fp32, logit = lane 0 (+ bias in fp32).  Bit-exact against the oracle; a plain
    sequential fp32 sum of the same products differs for some logits, so the check sees the order."""
    T, H, E = 3, 256, 4
    x = synth.activations(("pins", "router-order"), T, H)
    Wr, bias = synth.router(("pins", "router-order"), E, H)
    xf = synth.bf16_bits_to_f32(x).astype(np.float32)
    logits, _, _, _ = oracle.route(x, H, Wr, bias, 1)
    differs = 0
    for t in range(T):
        for e in range(E):
            p = np.zeros(32, np.float32)
            for lane in range(32):
                for kk in range(lane, H, 32):
                    p[lane] = _fma32(xf[t, kk], Wr[e, kk], p[lane])
            for sft in (16, 8, 4, 2, 1):
                p = np.array([p[lane] + p[lane ^ sft] for lane in range(32)], np.float32)
            want = np.float32(p[0] + bias[e])
            got = np.float32(oracle.router_logit(x[t], Wr[e]) + bias[e])
            assert np.array_equal(np.array(want).view(np.uint32), np.array(got).view(np.uint32)), (t, e)
            assert np.array_equal(np.array(want).view(np.uint32), np.array(logits[t, e]).view(np.uint32)), (t, e)
            seq = np.float32(0.0)
            for kk in range(H):
                seq = np.float32(seq + np.float32(xf[t, kk] * Wr[e, kk]))
            differs += int(seq != p[0])
    assert differs > 0


def test_route_ties_and_degenerate():
    T, H, E, topk = 5, 64, 8, 3
    x = synth.activations(("pins", "tie"), T, H)
    logits, ids, w, counts = oracle.route(x, H, np.zeros((E, H), np.float32), None, topk)
    assert np.all(ids == np.arange(topk)) and np.allclose(w, 1.0 / topk)
    logits, ids, w, counts = oracle.route(x, H, np.zeros((1, H), np.float32), None, 1)
    assert np.all(ids == 0) and np.all(w == 1.0)


def test_permute_is_stable_sort():
    rng = np.random.default_rng(9)
    T, topk, E = 300, 8, 64
    ids = np.stack([rng.permutation(E)[:topk] for _ in range(T)]).astype(np.int32)
    offsets, perm = oracle.permute(ids, E)
    assert np.array_equal(perm, np.argsort(ids.ravel(), kind="stable"))
    assert np.array_equal(offsets, np.concatenate([[0], np.cumsum(np.bincount(ids.ravel(), minlength=E))]))


# ---------------------------------------------------------------------------------------------- #
# MoE special cases: one expert = dense SwiGLU; k = E with equal logits = uniform average
# ---------------------------------------------------------------------------------------------- #

def _dense_swiglu(xf, Wg, Wu, Wd):
    """A SwiGLU FFN in fp64 numpy: (silu(x Wg^T) * (x Wu^T)) Wd^T, the intermediate kept in fp64."""
    g = xf @ Wg.T
    u = xf @ Wu.T
    return (g / (1.0 + np.exp(-g)) * u) @ Wd.T


def _act_quant_f32_numpy(hf):
    """Per-token INT8 codes of one fp32 row restated in numpy (the W4A8 page §3.1): amax, scale = amax/127
    and the quotient as IEEE fp32 operations, round half to even, clamp to [-128, 127]; scale 0 gives
    all-zero codes."""
    hf = np.asarray(hf, np.float32)
    s = np.float32(np.abs(hf).max()) / np.float32(127.0)
    if s == 0:
        return np.zeros(hf.shape, np.int8), np.float32(0.0)
    q = np.clip(np.rint(hf / s), -128, 127).astype(np.int8)
    return q, s


def _stacked_experts(E, H, I, group, sym, seed):
    Wg, Wu, Wd = [], [], []
    for e in range(E):
        Wg.append(_exact_grid(I, H, group, sym, seed + 3 * e)[0])
        Wu.append(_exact_grid(I, H, group, sym, seed + 3 * e + 1)[0])
        Wd.append(_exact_grid(H, I, group, sym, seed + 3 * e + 2)[0])
    return Wg, Wu, Wd


@pytest.mark.parametrize("sym", [True, False])
def test_moe_single_expert_is_dense_swiglu(sym):
    T, H, I, group = 6, 128, 64, 64
    Wg, Wu, Wd = _stacked_experts(1, H, I, group, sym, 100)
    x = synth.activations(("pins", "moe1"), T, H)
    _, ids, w, _ = oracle.route(x, H, np.zeros((1, H), np.float32), None, 1)
    qs = [oracle.quantize(M[0], group, sym) for M in (Wg, Wu, Wd)]
    y = oracle.moe_experts(x, H, ids, w, qs[0], qs[1], qs[2], I, group, sym)
    xf = synth.bf16_bits_to_f32(x).astype(np.float64)
    ref = _dense_swiglu(xf, Wg[0].astype(np.float64), Wu[0].astype(np.float64), Wd[0].astype(np.float64))
    np.testing.assert_allclose(y, ref, rtol=1e-10, atol=1e-12)


def test_moe_all_experts_equal_logits_is_average():
    T, H, I, group, E = 4, 128, 64, 64, 4
    Wg, Wu, Wd = _stacked_experts(E, H, I, group, False, 200)
    x = synth.activations(("pins", "moeE"), T, H)
    _, ids, w, _ = oracle.route(x, H, np.zeros((E, H), np.float32), None, E)
    stack = [oracle.quantize(np.concatenate(M), group, False) for M in (Wg, Wu, Wd)]
    y = oracle.moe_experts(x, H, ids, w, stack[0], stack[1], stack[2], I, group, False)
    xf = synth.bf16_bits_to_f32(x).astype(np.float64)
    ref = sum(_dense_swiglu(xf, Wg[e].astype(np.float64), Wu[e].astype(np.float64), Wd[e].astype(np.float64))
              for e in range(E)) / E
    np.testing.assert_allclose(y, ref, rtol=1e-10, atol=1e-12)
    sub = oracle.moe_experts(x, H, ids, w, stack[0], stack[1], stack[2], I, group, False, tokens=np.array([2]))
    assert np.array_equal(sub[0], y[2])


# ---------------------------------------------------------------------------------------------- #
# the expert FFN with INT8 activations (W4A8 page §3.1 per-token codes, §2.3 INT32 partials and the
# scale_w * scale_a rescale, §5.1 the down projection as the first W4A8 candidate)
# ---------------------------------------------------------------------------------------------- #

def test_act_quant_f16_hand_worked():
    """Per-token quantization of fp16 rows, worked by hand from amax/127 and round-half-even:
    [127, -63.5, 0.5, 2] -> s = 1, codes [127, -64 (tie), 0 (tie), 2];
    [254, 1 + 2^-10, -3, 0] -> s = 2, codes [127, 1 (0.50049 rounds up), -2 (tie -1.5), 0] -- 1 + 2^-10
    exists in fp16 but not in bf16, so a wrong widening of the input fails here."""
    q, s = oracle.act_quant_f16(_f16_bits([[127.0, -63.5, 0.5, 2.0], [254.0, 1.0 + 2.0 ** -10, -3.0, 0.0]]), 4)
    assert list(s) == [1.0, 2.0]
    assert q.tolist() == [[127, -64, 0, 2], [127, 1, -2, 0]]
    z, sz = oracle.act_quant_f16(np.zeros((1, 8), np.uint16), 8)
    assert sz[0] == 0.0 and not z.any()


def test_act_quant_f16_properties():
    rng = np.random.default_rng(7)
    h = (rng.standard_normal((32, 1024)) * 3.0).astype(np.float16)
    q, s = oracle.act_quant_f16(h.view(np.uint16), 1024)
    hf = h.astype(np.float64)
    assert np.array_equal(s, (np.abs(hf).max(axis=1).astype(np.float32) / np.float32(127.0)))
    assert np.all(np.abs(hf - q * s[:, None].astype(np.float64)) <= s[:, None] * (0.5 + 1e-6))
    assert np.all(np.abs(q).max(axis=1) == 127)


def _moe_a8_by_composition(x, H, ids, w, stack, I, group, sym, mask):
    """The same layer assembled from the separately pinned pieces: act_quant, linear_w4a8 on each
    expert's row block, linear_w4a16, and the codes of h (as an fp16 activation) restated in numpy."""
    T, topk = ids.shape
    xq, sa = oracle.act_quant(x, H)
    y = np.zeros((T, H))

    def block(q, e, rows):
        pk, sc, zr = q
        sl = slice(e * rows, (e + 1) * rows)
        return pk[sl], sc[sl], (None if zr is None else zr[sl])

    for t in range(T):
        for j in range(topk):
            e = ids[t, j]
            gq, uq, dq = block(stack[0], e, I), block(stack[1], e, I), block(stack[2], e, H)
            if mask & 1:
                g = oracle.linear_w4a8(xq[t:t + 1], sa[t:t + 1], gq[0], gq[1], I, H, group, zeros=gq[2], symmetric=sym)[0]
                u = oracle.linear_w4a8(xq[t:t + 1], sa[t:t + 1], uq[0], uq[1], I, H, group, zeros=uq[2], symmetric=sym)[0]
            else:
                g = oracle.linear_w4a16(x[t:t + 1], *gq, I, H, group, sym)[0]
                u = oracle.linear_w4a16(x[t:t + 1], *uq, I, H, group, sym)[0]
            h = g / (1.0 + np.exp(-g)) * u
            if mask & 2:   # the codes of h as an fp16 activation (numpy's IEEE conversions)
                h16 = h.astype(np.float32).astype(np.float16)
                hq, sh = _act_quant_f32_numpy(h16.astype(np.float32))
                o = oracle.linear_w4a8(hq[None, :], np.array([sh], np.float32), dq[0], dq[1], H, I, group,
                                       zeros=dq[2], symmetric=sym)[0]
            else:
                o = h @ oracle.dequant(*dq, I, group, sym).astype(np.float64).T
            y[t] += w[t, j] * o
    return y


@pytest.mark.parametrize("mask", [1, 2, 3])
@pytest.mark.parametrize("sym,group", [(False, 64), (True, 128)])
def test_moe_a8_equals_composition(mask, sym, group):
    T, H, I, E, topk = 5, 256, 128, 3, 2
    x = synth.activations(("pins", "moe-a8", mask), T, H)
    Wr, bias = synth.router(("pins", "moe-a8"), E, H)
    _, ids, w, _ = oracle.route(x, H, Wr, bias, topk)
    stack = [oracle.quantize(synth.weights(("pins", "moe-a8", nm), n, k), group, sym)
             for nm, n, k in (("g", E * I, H), ("u", E * I, H), ("d", E * H, I))]
    y = oracle.moe_experts_a8(x, H, ids, w, stack[0], stack[1], stack[2], I, group, sym, mask)
    ref = _moe_a8_by_composition(x, H, ids, w, stack, I, group, sym, mask)
    np.testing.assert_allclose(y, ref, rtol=1e-10, atol=1e-12 * np.abs(ref).max())
    sub = oracle.moe_experts_a8(x, H, ids, w, stack[0], stack[1], stack[2], I, group, sym, mask,
                                tokens=np.array([3, 1]))
    assert np.array_equal(sub, y[[3, 1]])


def test_moe_a8_mask0_is_the_w4a16_layer_and_a8_stays_close():
    """Mask 0 is the W4A16 expert FFN exactly; with INT8 activations the layer moves by the activation
    quantization error only (per-token steps of amax/127: a few per mille of the output's rms)."""
    T, H, I, E, topk, group = 6, 256, 128, 4, 2, 128
    x = synth.activations(("pins", "moe-a8-close"), T, H)
    Wr, bias = synth.router(("pins", "moe-a8"), E, H)
    _, ids, w, _ = oracle.route(x, H, Wr, bias, topk)
    stack = [oracle.quantize(synth.weights(("pins", "moe-a8c", nm), n, k), group, False)
             for nm, n, k in (("g", E * I, H), ("u", E * I, H), ("d", E * H, I))]
    y16 = oracle.moe_experts(x, H, ids, w, stack[0], stack[1], stack[2], I, group, False)
    y0 = oracle.moe_experts_a8(x, H, ids, w, stack[0], stack[1], stack[2], I, group, False, 0)
    assert np.array_equal(y0, y16)
    rms = np.sqrt(np.mean(y16 ** 2))
    for mask in (1, 2, 3):
        y8 = oracle.moe_experts_a8(x, H, ids, w, stack[0], stack[1], stack[2], I, group, False, mask)
        assert 0 < np.sqrt(np.mean((y8 - y16) ** 2)) / rms < 0.03


# ---------------------------------------------------------------------------------------------- #
# expert classes with their own group size (W4A8 page §5.3)
# ---------------------------------------------------------------------------------------------- #

def test_moe_classes_one_class_and_equal_classes_are_the_layer():
    T, H, I, E, topk, group = 6, 256, 128, 6, 2, 64
    x = synth.activations(("pins", "cls-x"), T, H)
    Wr, bias = synth.router(("pins", "cls"), E, H)
    _, ids, w, _ = oracle.route(x, H, Wr, bias, topk)
    stack = [oracle.quantize(synth.weights(("pins", "cls", nm), n, k), group, False)
             for nm, n, k in (("g", E * I, H), ("u", E * I, H), ("d", E * H, I))]
    ref = oracle.moe_experts(x, H, ids, w, stack[0], stack[1], stack[2], I, group, False)
    one = oracle.moe_experts_classes(x, H, ids, w, [0, E], [(stack[0], stack[1], stack[2], group, False)], I)
    assert np.array_equal(one, ref)
    # the same quantized stack cut into classes {0,1}, {2..5}: row blocks of the stacked matrices
    def cut(q, rows_per, e0, e1):
        pk, sc, zr = q
        sl = slice(e0 * rows_per, e1 * rows_per)
        return pk[sl], sc[sl], (None if zr is None else zr[sl])
    classes = [tuple(cut(q, r, a, b) for q, r in zip(stack, (I, I, H))) + (group, False) for a, b in ((0, 2), (2, E))]
    two = oracle.moe_experts_classes(x, H, ids, w, [0, 2, E], classes, I)
    np.testing.assert_allclose(two, ref, rtol=1e-12, atol=1e-14 * np.abs(ref).max())


def test_moe_classes_each_expert_uses_its_class_quantization():
    """Classes with different group sizes and symmetry: every token's output equals the dense SwiGLU FFNs
    of its chosen experts built from each class's own dequantized matrices (numpy), weighted."""
    T, H, I, E, topk = 5, 256, 128, 5, 2
    x = synth.activations(("pins", "cls2-x"), T, H)
    Wr, bias = synth.router(("pins", "cls2"), E, H)
    _, ids, w, _ = oracle.route(x, H, Wr, bias, topk)
    begin = [0, 1, 3, E]
    params = [(64, True), (128, False), (64, False)]
    classes, dense = [], {}
    for c, (group, sym) in enumerate(params):
        Ec = begin[c + 1] - begin[c]
        qs = [oracle.quantize(synth.weights(("pins", "cls2", c, nm), n, k), group, sym)
              for nm, n, k in (("g", Ec * I, H), ("u", Ec * I, H), ("d", Ec * H, I))]
        classes.append((qs[0], qs[1], qs[2], group, sym))
        deq = [oracle.dequant(*q, k, group, sym).astype(np.float64) for q, k in zip(qs, (H, H, I))]
        for le in range(Ec):
            dense[begin[c] + le] = (deq[0][le * I:(le + 1) * I], deq[1][le * I:(le + 1) * I], deq[2][le * H:(le + 1) * H])
    y = oracle.moe_experts_classes(x, H, ids, w, begin, classes, I)
    xf = synth.bf16_bits_to_f32(x).astype(np.float64)
    ref = np.zeros((T, H))
    for t in range(T):
        for j in range(topk):
            Wg, Wu, Wd = dense[ids[t, j]]
            ref[t] += w[t, j] * _dense_swiglu(xf[t:t + 1], Wg, Wu, Wd)[0]
    np.testing.assert_allclose(y, ref, rtol=1e-10, atol=1e-12 * np.abs(ref).max())


# ---------------------------------------------------------------------------------------------- #
# the generator itself: SplitMix64's published output for state 0
# ---------------------------------------------------------------------------------------------- #

def test_splitmix64_reference_values():
    assert [int(v) for v in synth.raw_u64(0, 3)] == [0xE220A8397B1DCDAF, 0x6E789E6AA1B965F4, 0x06C45D188009454F]
