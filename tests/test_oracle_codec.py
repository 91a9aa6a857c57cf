"""Pins of the oracle's group quantiser (FlashLoop, Appendix E "Quantization Setting";
§4.3 "Cross-Loop KV Residual Quantization").

The directed roundings are checked against exact rational arithmetic; the whole
quantiser against hand-derived worked cases (tests/golden/codec_worked.txt) and
against properties fixed by its definition: codes in range, the offset below every
value, the scale covering the range, the reconstruction error bound, monotone codes,
exact constants."""
import math
import os
from fractions import Fraction

import numpy as np
import pytest

from oracle import codec

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "codec_worked.txt")


# ---------------------------------------------------------------- exact reference
def exact_round(fr, prec, emin, emax, mode):
    """Round a Fraction to a binary format with ``prec`` significand bits,
    minimum normal exponent ``emin`` and maximum exponent ``emax``.
    mode: 'RU', 'RD', 'RN' (ties to even). Returns a Fraction or +-inf (float)."""
    if fr == 0:
        return Fraction(0)
    sign = 1 if fr > 0 else -1
    a = abs(fr)
    e = a.numerator.bit_length() - a.denominator.bit_length()
    if Fraction(2) ** e > a:
        e -= 1
    while Fraction(2) ** (e + 1) <= a:
        e += 1
    e = max(e, emin)
    ulp = Fraction(2) ** (e - prec + 1)
    n = a / ulp
    lo = math.floor(n)
    if n == lo:
        m = lo
    elif mode == "RN":
        frac = n - lo
        if frac > Fraction(1, 2) or (frac == Fraction(1, 2) and lo % 2 == 1):
            m = lo + 1
        else:
            m = lo
    elif (mode == "RU") == (sign > 0):
        m = lo + 1
    else:
        m = lo
    val = m * ulp
    maxv = (2 - Fraction(2) ** (1 - prec)) * Fraction(2) ** emax
    if val > maxv:
        if mode == "RN" or (mode == "RU") == (sign > 0):
            return sign * math.inf
        return sign * maxv
    return sign * val


def f32x(fr, mode):
    return exact_round(fr, 24, -126, 127, mode)


def f16x(fr, mode):
    return exact_round(fr, 11, -14, 15, mode)


def _frac(v):
    return Fraction(float(v))


def _samples(g, n):
    mags = np.exp(g.uniform(np.log(1e-6), np.log(1e4), size=n))
    sgn = np.where(g.random(n) < 0.5, -1.0, 1.0)
    x = (mags * sgn).astype(np.float32)
    edge = np.array([0.0, 1.0, -1.0, 0.1, 3.0, 1e-7, 65504.0, 65520.0, -65520.0,
                     6.1e-5, 5.96e-8, 2.0 ** -24, 1.5, 2.5], np.float32)
    return np.concatenate([x, edge])


# ---------------------------------------------------------------- rounding pins
def test_add_directed_exact():
    g = np.random.Generator(np.random.PCG64(11))
    a = _samples(g, 400)
    b = np.roll(_samples(g, 400), 7)
    ru = codec.add_ru(a, b)
    rd = codec.add_rd(a, b)
    for i in range(len(a)):
        ex = _frac(a[i]) + _frac(b[i])
        assert _frac(ru[i]) == f32x(ex, "RU"), (a[i], b[i])
        assert _frac(rd[i]) == f32x(ex, "RD"), (a[i], b[i])


def test_div_directed_exact():
    g = np.random.Generator(np.random.PCG64(12))
    a = _samples(g, 400)
    b = np.abs(np.roll(_samples(g, 400), 3))
    b[b == 0] = 3.0
    b = np.concatenate([b[:-3], np.array([3.0, 15.0, 255.0], np.float32)])
    ru = codec.div_ru(a, b)
    rd = codec.div_rd(a, b)
    for i in range(len(a)):
        ex = _frac(a[i]) / _frac(b[i])
        assert _frac(ru[i]) == f32x(ex, "RU"), (a[i], b[i])
        assert _frac(rd[i]) == f32x(ex, "RD"), (a[i], b[i])


def test_f16_directed_exact():
    g = np.random.Generator(np.random.PCG64(13))
    x = _samples(g, 600)
    up = codec.f16_ru(x)
    dn = codec.f16_rd(x)
    for i in range(len(x)):
        ex = _frac(x[i])
        for got, mode in ((up[i], "RU"), (dn[i], "RD")):
            want = f16x(ex, mode)
            if isinstance(want, float):
                assert np.isinf(got) and np.sign(got) == np.sign(want), (x[i], mode)
            else:
                assert _frac(got) == want, (x[i], mode, got)


def test_fma_exact():
    g = np.random.Generator(np.random.PCG64(14))
    codes = g.integers(0, 256, size=300)
    s = codec.f16_ru(np.abs(_samples(g, 300 - 14)).astype(np.float32)[:300])
    s = np.concatenate([s, np.full(300 - len(s), 1.0, np.float16)])[:300]
    s[~np.isfinite(s)] = np.float16(2.0)
    z = codec.f16_rd(_samples(g, 300 - 14)[:300])
    z = np.concatenate([z, np.full(300 - len(z), -1.0, np.float16)])[:300]
    z[~np.isfinite(z)] = np.float16(-3.0)
    got = codec.fma_f32(codes, s, z)
    for i in range(300):
        ex = codes[i] * _frac(s[i]) + _frac(z[i])
        assert _frac(got[i]) == f32x(ex, "RN")


# ---------------------------------------------------------------- worked cases
def _golden_cases():
    out = []
    with open(GOLDEN) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            parts = [p.split() for p in line.split("|")]
            bits = int(parts[0][0])
            x = np.array([float(v) for v in parts[1]], np.float32)
            out.append((bits, x, Fraction(parts[2][0]), Fraction(parts[3][0]),
                        [int(v) for v in parts[4]], [Fraction(v) for v in parts[5]]))
    return out


@pytest.mark.parametrize("case", range(6))
def test_worked_cases(case):
    bits, x, s, z, codes, deq = _golden_cases()[case]
    c, s_got, z_got, d_got, err = codec.quantize_groups(x[None, :], bits)
    assert not err.any()
    assert _frac(s_got[0]) == s
    assert _frac(z_got[0]) == z
    assert list(c[0]) == codes
    assert [_frac(v) for v in d_got[0]] == deq


# ---------------------------------------------------------------- properties
@pytest.mark.parametrize("bits", [2, 4, 8])
@pytest.mark.parametrize("g", [32, 64])
def test_quantiser_properties(bits, g):
    rs = np.random.Generator(np.random.PCG64(100 + bits + g))
    n = 2000
    scale = np.exp(rs.uniform(np.log(1e-3), np.log(1e2), size=(n, 1)))
    offset = rs.normal(size=(n, 1)) * scale * rs.choice([0.0, 1.0, 30.0], size=(n, 1))
    x = (rs.normal(size=(n, g)) * scale + offset).astype(np.float32)
    c, s, z, deq, err = codec.quantize_groups(x, bits)
    assert not err.any()
    qmax = (1 << bits) - 1
    assert c.max() <= qmax
    sf = s.astype(np.float64)
    zf = z.astype(np.float64)
    x64 = x.astype(np.float64)
    # offset at or below every value; scale covers the range
    assert np.all(zf <= x64.min(axis=1))
    assert np.all(sf * qmax >= x64.max(axis=1) - zf)
    # reconstruction error: half a step plus the binary32 rounding of the steps
    bound = sf[:, None] / 2 + 2.0 ** -22 * (np.abs(x64 - zf[:, None]) + np.abs(x64))
    assert np.all(np.abs(x64 - deq.astype(np.float64)) <= bound)
    # codes are monotone in x within a group
    order = np.argsort(x, axis=1, kind="stable")
    cs = np.take_along_axis(c.astype(np.int64), order, axis=1)
    assert np.all(np.diff(cs, axis=1) >= 0)


def test_constant_groups_exact():
    vals = np.array([0.75, -2.0, 1024.0, 0.0, -0.5, 6.103515625e-05], np.float32)
    x = np.repeat(vals[:, None], 32, axis=1)
    c, s, z, deq, err = codec.quantize_groups(x, 4)
    assert not err.any()
    assert np.all(c == 0) and np.all(s == 0)
    assert np.array_equal(deq, x)


def test_range_error_flag():
    x = np.array([[-70000.0, 0.0, 1.0, 2.0]], np.float32)
    *_, err = codec.quantize_groups(x, 4)
    assert err.all()
    x = np.array([[-60000.0, 60000.0, 0.0, 1.0]], np.float32)  # scale 8000 fits
    *_, err = codec.quantize_groups(x, 4)
    assert not err.any()


def test_pack_layout():
    assert codec.pack_codes(np.array([1, 2, 3, 0], np.uint8), 2)[0] == 1 | (2 << 2) | (3 << 4)
    assert codec.pack_codes(np.array([0xA, 0x5], np.uint8), 4)[0] == 0x5A
    g = np.random.Generator(np.random.PCG64(5))
    for bits in (2, 4, 8):
        c = g.integers(0, 1 << bits, size=(7, 3, 128)).astype(np.uint8)
        p = codec.pack_codes(c, bits)
        assert p.shape == (7, 3, 128 * bits // 8)
        assert np.array_equal(codec.unpack_codes(p, bits, 128), c)


def test_dequantize_matches_quantize():
    g = np.random.Generator(np.random.PCG64(6))
    x = g.normal(size=(5, 2, 128)).astype(np.float32)
    for bits in (2, 4, 8):
        c, s, z, deq, _ = codec.quantize_groups(x.reshape(5, 2, 4, 32), bits)
        packed = codec.pack_codes(c.reshape(5, 2, 128), bits)
        sz = np.stack([s, z], axis=-1)
        back = codec.dequantize(packed, sz, bits, 32, 128)
        assert np.array_equal(back, deq.reshape(5, 2, 128))
