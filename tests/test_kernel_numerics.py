"""Arithmetic facts the kernels rely on, checked on the CPU.

The 16-bit expert path carries the SwiGLU intermediate h as two bf16 values, hi = bf16(h) and
lo = bf16(h - hi), both rounded to nearest even.  bf16 keeps 8 significant bits, so hi is within half a
bf16 ulp (at most 2^-8 relative) of h, the difference h - hi is exact in fp32, and lo is within 2^-8 of
it: hi + lo is within 2^-16 |h| of h (about 2^-17 at worst in practice, as both worst cases rarely meet),
far inside the output tolerance, and over bf16's range (the largest finite bf16 is 3.39e38; fp32
values within half a bf16 ulp of fp32's maximum round to infinity) rather than fp16's 65504.  Checked
here on the CPU over values chosen to stress the rounding (ties, binade edges, the ends of the range)."""
import numpy as np
import torch

BF16_MAX = float(torch.finfo(torch.bfloat16).max)


def _pair(h32):
    t = torch.from_numpy(h32)
    hi = t.to(torch.bfloat16).float()
    lo = (t - hi).to(torch.bfloat16).float()
    return hi.numpy().astype(np.float64), lo.numpy().astype(np.float64)


def test_hi_lo_pair_holds_h_to_2_pow_minus_16():
    rng = np.random.default_rng(7)
    parts = [
        rng.standard_normal(200_000).astype(np.float32) * np.float32(10.0) ** rng.integers(-30, 30, 200_000).astype(np.float32),
        # every fp32 significand pattern near ties of the bf16 rounding: low 16 bits 0x7FFF, 0x8000, 0x8001
        (np.arange(1 << 16, dtype=np.uint32)[:, None] << 16 | np.array([0x7FFF, 0x8000, 0x8001], np.uint32)).ravel()
        .view(np.float32),
        np.array([BF16_MAX, -BF16_MAX, np.finfo(np.float32).tiny * 2**20, 1.0, -1.0, 2.0 - 2**-23, 3.0e38,
                  65504.0 * 16], np.float32),
    ]
    h = np.concatenate(parts)
    # the normal range of both halves, up to the largest finite bf16
    h = h[np.isfinite(h) & (np.abs(h) >= np.finfo(np.float32).tiny * 2**20) & (np.abs(h) <= BF16_MAX)]
    hi, lo = _pair(h)
    err = np.abs(hi + lo - h.astype(np.float64))
    assert np.all(np.isfinite(hi)) and np.all(np.isfinite(lo))
    rel = err / np.abs(h.astype(np.float64))
    assert np.all(rel <= 2.0 ** -16)
    assert np.max(rel) < 1.05 * 2.0 ** -17       # the figure quoted for the pair
    # a single bf16 is off by up to 2^-8 |h|: the second half is what meets the bar
    assert np.max(np.abs(hi - h) / np.abs(h)) > 2.0 ** -9


def test_w4a8_accumulator_preload_is_exact_for_every_group_sum():
    """The W4A8 epilogue preloads each int32 accumulator with the bits of 1.5 * 2^23; after the integer
    MMAs add acc, the bits read as the float 1.5 * 2^23 + acc exactly while 1.5 * 2^23 + acc stays in
    [2^23, 2^24), i.e. |acc| < 2^22, and one subtraction recovers acc.  The largest group sum W4A8 forms
    (group 128, |activation code| <= 128, |16 * weight code| <= 128 on the symmetric path, |code - zero|
    <= 15 on the asymmetric one) is 128 * 128 * 128 = 2^21."""
    bias_bits, bias = 0x4B400000, 1.5 * 2.0 ** 23
    acc = np.concatenate([np.arange(-(1 << 21), (1 << 21) + 1, 997), [-(1 << 21), (1 << 21), -1, 0, 1]]).astype(np.int64)
    bits = (bias_bits + acc).astype(np.uint32)
    got = bits.view(np.float32).astype(np.float64) - bias
    assert np.array_equal(got, acc.astype(np.float64))
    assert 128 * 128 * 128 == 1 << 21 and 128 * (16 * 8) * 128 == 1 << 21 and 128 * 15 * 128 < 1 << 21
    # past 2^22 the sum leaves the binade and the identity fails: the bound is the real limit
    over = np.array([bias_bits + (1 << 22) + 1], np.int64).astype(np.uint32).view(np.float32).astype(np.float64)
    assert over[0] - bias != (1 << 22) + 1
