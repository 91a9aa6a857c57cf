"""Exact group quantiser of the cross-loop KV store (oracle; test infrastructure only).

What the pages fix (FlashLoop, §4.3 "Cross-Loop KV Residual Quantization" and
Appendix E "Quantization Setting"): asymmetric group-wise quantisation whose scale
and offset come from the minimum and maximum of each group; the same scheme for the
base state and for the cross-loop residuals.

What they leave open, and the reading taken here (every step in binary32 or
binary16, so that a GPU kernel using the same IEEE operations reproduces the codes
bit for bit):
  mn, mx = min, max of the g values of the group            (exact)
  z      = fp16 rounded toward -inf of mn                    (offset <= every value)
  s      = fp16_RU( f32_RU( f32_RU(mx - z) / (2^b - 1) ) )   (scale covers the range)
  code   = 0                                    if s == 0
         = clamp(rint(f32(f32(x - z) / s)), 0, 2^b - 1)      otherwise (ties to even)
  deq    = fmaf(code, s, z)                                  (one rounding to binary32)
An fp16 overflow of z or s is a range error. ``bits == 0`` means "no quantisation":
the value is stored as binary32 and ``deq == x``.

The directed roundings are computed exactly from round-to-nearest numpy float32
arithmetic: the rounding error of a sum is recovered with Knuth's TwoSum and the
remainder of a quotient with an exact fp64 product, and the sign of that error says
whether the round-to-nearest result has to step one ulp up or down.
Inputs must be finite with magnitude below 2**100 (no overflow in the steps).
"""
import numpy as np

F32 = np.float32
F16 = np.float16
_INF32 = F32(np.inf)
_INF16 = F16(np.inf)


def _f32(a):
    return np.asarray(a, dtype=F32)


def two_sum(a, b):
    """fl32(a+b) and its exact rounding error t (a + b == s + t exactly)."""
    a = _f32(a)
    b = _f32(b)
    with np.errstate(over="ignore", invalid="ignore"):
        s = a + b
        bp = s - a
        ap = s - bp
        t = (a - ap) + (b - bp)
    return s, t


def add_ru(a, b):
    """a + b rounded toward +inf in binary32."""
    s, t = two_sum(a, b)
    return np.where(t > 0, np.nextafter(s, _INF32), s).astype(F32)


def add_rd(a, b):
    """a + b rounded toward -inf in binary32."""
    s, t = two_sum(a, b)
    return np.where(t < 0, np.nextafter(s, -_INF32), s).astype(F32)


def sub_ru(a, b):
    return add_ru(a, -_f32(b))


def _div_remainder_sign(a, b, q):
    """sign of (a/b - q) for binary32 a, b and q = fl32(a/b).

    a - q*b is computed in fp64: q*b has at most 48 significant bits so it is exact,
    and the remainder of a round-to-nearest quotient is representable, so the fp64
    subtraction is exact too."""
    r = a.astype(np.float64) - q.astype(np.float64) * b.astype(np.float64)
    return np.sign(r) * np.sign(b.astype(np.float64))


def div_ru(a, b):
    """a / b rounded toward +inf in binary32 (b != 0)."""
    a = _f32(a)
    b = _f32(b)
    q = (a / b).astype(F32)
    sg = _div_remainder_sign(a, b, q)
    return np.where(sg > 0, np.nextafter(q, _INF32), q).astype(F32)


def div_rd(a, b):
    a = _f32(a)
    b = _f32(b)
    q = (a / b).astype(F32)
    sg = _div_remainder_sign(a, b, q)
    return np.where(sg < 0, np.nextafter(q, -_INF32), q).astype(F32)


def f16_ru(x):
    """binary32 -> binary16 rounded toward +inf (overflow gives +inf)."""
    x = _f32(x)
    with np.errstate(over="ignore", invalid="ignore"):
        h = x.astype(F16)
        back = h.astype(F32)
        return np.where(back < x, np.nextafter(h, _INF16), h).astype(F16)


def f16_rd(x):
    """binary32 -> binary16 rounded toward -inf (overflow gives -inf)."""
    x = _f32(x)
    with np.errstate(over="ignore", invalid="ignore"):
        h = x.astype(F16)
        back = h.astype(F32)
        return np.where(back > x, np.nextafter(h, -_INF16), h).astype(F16)


def fma_f32(a, b, c):
    """fmaf(a, b, c) for a = small integer code, b, c binary16 values.

    code*s has at most 19 significant bits and all binary16 values are multiples of
    2**-24 below 2**16, so code*s + z is exact in fp64 and one conversion gives the
    correctly rounded binary32 result, i.e. fmaf's."""
    r = np.asarray(a, np.float64) * np.asarray(b, np.float64) + np.asarray(c, np.float64)
    return r.astype(F32)


def quantize_groups(x, bits):
    """Quantise binary32 values grouped along the last axis.

    x: float32 [..., g]. bits in {2, 4, 8}.
    Returns codes uint8 [..., g] (unpacked), s float16 [...], z float16 [...],
    deq float32 [..., g] and a boolean range-error flag [...].
    """
    x = _f32(x)
    assert bits in (2, 4, 8)
    qmax = F32((1 << bits) - 1)
    mn = x.min(axis=-1)
    mx = x.max(axis=-1)
    z = f16_rd(mn)
    zf = z.astype(F32)
    t1 = sub_ru(mx, zf)
    t2 = div_ru(t1, np.broadcast_to(qmax, t1.shape))
    s = f16_ru(t2)
    rng_err = ~np.isfinite(z) | ~np.isfinite(s)
    sf = s.astype(F32)
    with np.errstate(invalid="ignore", divide="ignore", over="ignore"):
        diff = (x - zf[..., None]).astype(F32)
        sdiv = np.where(sf == 0, F32(1), sf)[..., None]
        w = (diff / sdiv).astype(F32)
        c = np.clip(np.rint(w), 0, qmax)
        c = np.where((sf == 0)[..., None], 0, c)
        c = np.where(rng_err[..., None], 0, c)
    codes = c.astype(np.uint8)
    deq = fma_f32(codes, s[..., None], z[..., None])
    return codes, s, z, deq, rng_err


def pack_codes(codes, bits):
    """Pack unpacked codes [..., n] (n*bits divisible by 8) little-endian, low bits first."""
    codes = np.asarray(codes, np.uint8)
    if bits == 8:
        return codes.copy()
    per = 8 // bits
    sh = codes.shape
    c = codes.reshape(sh[:-1] + (sh[-1] // per, per)).astype(np.uint16)
    out = np.zeros(c.shape[:-1], np.uint16)
    for i in range(per):
        out |= c[..., i] << (i * bits)
    return out.astype(np.uint8)


def unpack_codes(packed, bits, n):
    """Inverse of pack_codes: [..., n*bits/8] bytes -> [..., n] codes."""
    packed = np.asarray(packed, np.uint8)
    if bits == 8:
        return packed.copy()
    per = 8 // bits
    mask = (1 << bits) - 1
    parts = [(packed >> (i * bits)) & mask for i in range(per)]
    out = np.stack(parts, axis=-1).reshape(packed.shape[:-1] + (packed.shape[-1] * per,))
    assert out.shape[-1] == n
    return out.astype(np.uint8)


def dequantize(packed, sz, bits, group, n):
    """Rebuild binary32 values from packed codes and (s, z) pairs.

    packed: [..., n*bits/8] uint8; sz: float16 [..., n/group, 2] as (s, z)."""
    codes = unpack_codes(packed, bits, n)
    s = sz[..., 0]
    z = sz[..., 1]
    sh = codes.shape[:-1] + (n // group, group)
    c = codes.reshape(sh)
    deq = fma_f32(c, s[..., None], z[..., None])
    return deq.reshape(codes.shape)
