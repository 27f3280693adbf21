"""Pins of the oracle's W4A8 path with progressive group quantization (CPU only).

[L13] §QServe: 4-bit per-group weights, 8-bit per-token activations, INT8
tensor cores, and a dequantization that multiplies by the group scale before
subtracting the zero point so that packed byte arithmetic cannot overflow.
The readings (level-1 range 119, integer level-2 step, scaled zero) are in the
oracle's header.  The checks here:

* every possible level-2 group range inside [-119, 119], with every integer in
  it: the step is at most 16, every dequantized value fits int8, every value is
  within half a step, and u * s2 fits an unsigned byte;
* the packed-byte arithmetic itself: four codes in a 32-bit word scaled by one
  integer multiply and corrected by a bytewise subtraction give the four
  values; subtracting the zero point first does not;
* the fp32 activation quotient decides the same int8 code as the exact one,
  over every finite fp16 value;
* the GEMM's integer accumulation and its fp16 output against exact
  rational arithmetic.
"""
from fractions import Fraction

import numpy as np
import pytest

import oracle

F16, F64 = np.float16, np.float64


def _all_ranges():
    mn, mx = np.meshgrid(np.arange(-119, 120), np.arange(-119, 120), indexing="ij")
    keep = mn <= mx
    return mn[keep], mx[keep]


def test_level2_every_range_fits_int8():
    """Rows of integer weights with max |W| = 119 quantize at level 1 with s1 = 1 (w8 = W);
    each row's two groups hold one range [mn, mx] and, between them, every integer in it."""
    mn, mx = _all_ranges()
    R = mn.size
    W = np.zeros((R, 384), dtype=np.int64)
    vals = np.minimum(mn[:, None] + np.arange(252)[None, :], mx[:, None])  # mn, mn+1, ..., mx, mx, ...
    for g in range(2):                                             # both groups span [mn, mx]
        W[:, 128 * g], W[:, 128 * g + 1] = mn, mx
        W[:, 128 * g + 2:128 * (g + 1)] = vals[:, 126 * g:126 * (g + 1)]
    W[:, 256], W[:, 257] = 119, -119                               # fixes s1 = 1
    q, s1, s2, zs = oracle.w4a8_quantize_weight(W.astype(F16))
    assert np.all(s1 == F16(1.0))
    w8_hat = oracle.w4a8_dequant_int8(q, s2, zs)
    u = oracle.unpack_v1(q).astype(np.int64)
    s2f = np.repeat(s2.astype(np.int64), 128, axis=1)
    assert s2.max() <= 16
    assert np.all(u * s2f <= 240) and zs.max() <= 240
    assert np.abs(w8_hat).max() <= 127
    assert np.all(2 * np.abs(W - w8_hat) <= s2f)                   # within half a step, no clamping
    # the widest range needs the largest step: [-119, 119] -> 16
    widest = np.nonzero((mn == -119) & (mx == 119))[0][0]
    assert s2[widest, 0] == 16


def test_level1_range_is_the_largest_that_fits():
    """119 is forced: a range of [-120, 120] would dequantize to 128 for some value."""
    def worst(R):
        s2 = -(-2 * R // 15)
        return R + s2 / 2
    assert worst(oracle.W4A8_L1) <= 127 < worst(oracle.W4A8_L1 + 1)


def _pack_bytes(v):
    return sum((int(b) & 0xFF) << (8 * i) for i, b in enumerate(v))


def _bytes_as_int8(word):
    return [((word >> (8 * i)) & 0xFF) - 256 * (((word >> (8 * i)) & 0xFF) > 127) for i in range(4)]


def test_progressive_order_in_packed_bytes():
    """[L13] §QServe: scale first, then subtract the zero point.  Four codes in a word times
    s2 (one 32-bit multiply: no byte carries, as u * s2 <= 240), minus zs in every byte
    (modulo 256 per byte), gives the four int8 values wherever they lie in int8."""
    rng = np.random.default_rng(1)
    broke = 0
    for s2 in range(1, 17):
        for z in range(16):
            zs = z * s2
            for _ in range(40):
                u = rng.integers(0, 16, 4)
                want = [(int(c) - z) * s2 for c in u]
                if max(abs(v) for v in want) > 127:
                    continue
                prod = (_pack_bytes(u) * s2) & 0xFFFFFFFF
                got = _pack_bytes([((prod >> (8 * i)) & 0xFF) - zs for i in range(4)])
                assert _bytes_as_int8(got) == want
                # the other order: signed differences packed, then one multiply
                other = (_pack_bytes([int(c) - z for c in u]) * s2) & 0xFFFFFFFF
                broke += _bytes_as_int8(other) != want
    assert broke > 0, "subtracting first must corrupt neighbouring bytes somewhere"


def test_activation_quotient_fp32_decides_like_exact():
    """Reading 16: for fp16 a, b the fp32 quotient rounds to the same integer as a / b."""
    a = np.arange(65536, dtype=np.uint16).view(F16)
    a = a[np.isfinite(a)].astype(F64)
    rng = np.random.default_rng(2)
    for b in np.unique(rng.uniform(1e-3, 10.0, 300).astype(F16)):
        bb = F64(b)
        sel = np.abs(a / bb) <= 127.5
        q32 = np.rint((a[sel].astype(np.float32) / np.float32(bb)).astype(F64))
        q64 = np.rint(a[sel] / bb)
        assert np.array_equal(q32, q64), b


def test_activation_quantization():
    rng = np.random.default_rng(3)
    x = rng.standard_normal((6, 256)).astype(F16)
    x[2] = 0
    x[3, 17] = F16(40.0)
    x8, sx = oracle.w4a8_quantize_act(x)
    assert sx[2] == F16(1.0 / 127) and not x8[2].any()
    x64, s = x.astype(F64), sx.astype(F64)[:, None]
    assert np.all(np.abs(x8.astype(np.int64)) <= 127)
    assert np.all(np.abs(x64 - x8 * s) <= s / 2 * (1 + 1e-9) + 1e-12)
    for t in (0, 1, 3, 4, 5):
        assert np.abs(x8[t]).max() == 127


def test_gemm_exact():
    rng = np.random.default_rng(4)
    W = (rng.standard_normal((5, 256)) * 0.02).astype(F16)
    x = rng.standard_normal((3, 256)).astype(F16)
    q, s1, s2, zs = oracle.w4a8_quantize_weight(W)
    x8, sx = oracle.w4a8_quantize_act(x)
    y, acc = oracle.w4a8_gemm(x8, sx, q, s1, s2, zs)
    u = oracle.unpack_v1(q)
    for t in range(3):
        for n in range(5):
            a = 0
            for k in range(256):
                g = k // 128
                a += int(x8[t, k]) * (int(u[n, k]) * int(s2[n, g]) - int(zs[n, g]))
            assert acc[t, n] == a
            exact = Fraction(a) * Fraction(float(sx[t])) * Fraction(float(s1[n]))
            assert y[t, n] == F16(float(exact))


def test_level1_per_channel():
    """Level 1 (reading 14): per row, |W - w8 s1| <= s1 / 2, |w8| <= 119, the largest |w8|
    is 119 (or 118 where the fp16 step rounds up); a zero row has s1 = fp16(1/119), codes z."""
    rng = np.random.default_rng(5)
    W = (rng.standard_normal((40, 256)) * rng.uniform(1e-3, 1.0, (40, 1))).astype(F16)
    W[7] = 0
    q, s1, s2, zs = oracle.w4a8_quantize_weight(W)
    assert s1[7] == F16(1.0 / 119)
    W64, s = W.astype(F64), s1.astype(F64)[:, None]
    w8 = np.rint(W64 / s)
    assert np.abs(w8).max() <= 119
    assert np.all(np.abs(W64 - w8 * s) <= s / 2 * (1 + 1e-12))
    rows = [r for r in range(40) if r != 7]
    assert set(np.abs(w8[rows]).max(axis=1)) <= {118.0, 119.0}
    assert np.all(oracle.w4a8_dequant_int8(q, s2, zs)[7] == 0)
