"""Residual-vs-full quantisation of per-loop KV (oracle; test infrastructure only).

Pages: FlashLoop paper §3.3 "Quantization-Friendly KV Residual" (the KV of one loop
differs little from the previous loop's, so quantising that difference loses less than
quantising every loop's KV in full at the same bit width; Figure 2c plots the two
reconstruction errors), §5.3.1 Table 2 (per-loop KIVI-style quantisation as the
ablation), Appendix E (the same asymmetric group-wise scheme for base and residuals).

Two quantisation schemes:
  * "hd" (the store's codec): groups of ``group`` consecutive head_dim elements of one
    token, an 8-bit base at loop 1;
  * "pages" (App. E "Quantization Setting"): INT4 for the base and the residuals alike,
    asymmetric, scale and offset from the group's minimum and maximum, groups of 64; keys
    per channel (a group = 64 consecutive tokens of one (head, channel)), values per token
    (64 consecutive channels of one (token, head)); the most recent 64 tokens kept in
    bfloat16. Readings: a trailing group shorter than 64 (the tokens before the window
    are not a multiple of 64) takes its own minimum and maximum; the window holds the last
    64 tokens of the sequence in every loop, their residual stored in bfloat16 too (the
    "same scheme" for residuals); the scale/offset arithmetic is the codec's.

Readings:
  * full quantisation of loop r: K~_r = Q_b(K_r), every loop on its own, b bits, the
    codec of ``codec.quantize_groups`` (groups along head_dim), or the pages' scheme;
  * residual quantisation: K^_1 = Q_base(K_1) (8 bits), then
    K^_r = fl32(K^_{r-1} + Q_b(fl32(K_r - K^_{r-1}))) - the store's closed-loop chain
    (``kvstore``), every token written in every loop;
  * reconstruction error of loop r: ||K^_r - K_r||_F / ||K_r||_F (relative Frobenius),
    in fp64 over the binary32 values.
"""
import numpy as np

from . import codec


def _quant(x, bits, group):
    """x float32 [n, H, hd] -> the dequantised binary32 values of the codec."""
    n, H, hd = x.shape
    _, _, _, deq, err = codec.quantize_groups(x.reshape(n, H, hd // group, group), bits)
    assert not err.any(), "scale or offset outside binary16"
    return deq.reshape(n, H, hd)


def bf16_f32(x):
    """Round binary32 values to the nearest bfloat16 (ties to even), as binary32: keep the
    upper 16 bits of the binary32 pattern after adding half an ulp of bfloat16 (plus the
    kept lowest bit, for ties to even). Finite inputs."""
    u = np.ascontiguousarray(x, np.float32).view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) & 0xFFFF0000
    return u.astype(np.uint32).view(np.float32)


def pages_quant(x, kind, bits=4, group=64, window=64):
    """The pages' per-loop scheme (see the module header) applied to x float32 [n, H, hd]
    of keys (kind "k": per channel along tokens) or values (kind "v": per token along
    channels); returns the binary32 reconstruction."""
    x = np.asarray(x, np.float32)
    n, H, hd = x.shape
    nq = max(n - window, 0)
    out = np.empty_like(x)
    out[nq:] = bf16_f32(x[nq:])
    if nq == 0:
        return out
    q = x[:nq]
    if kind == "k":
        t = np.ascontiguousarray(q.transpose(1, 2, 0))          # [H, hd, nq]
        rec = np.empty_like(t)
        full = (nq // group) * group
        if full:
            _, _, _, deq, err = codec.quantize_groups(t[..., :full].reshape(H, hd, full // group, group), bits)
            assert not err.any(), "scale or offset outside binary16"
            rec[..., :full] = deq.reshape(H, hd, full)
        if nq > full:
            _, _, _, deq, err = codec.quantize_groups(t[..., full:], bits)
            assert not err.any(), "scale or offset outside binary16"
            rec[..., full:] = deq
        out[:nq] = rec.transpose(2, 0, 1)
    else:
        assert hd % group == 0
        _, _, _, deq, err = codec.quantize_groups(q.reshape(nq, H, hd // group, group), bits)
        assert not err.any(), "scale or offset outside binary16"
        out[:nq] = deq.reshape(nq, H, hd)
    return out


def rel_error(approx, exact):
    a = np.asarray(approx, np.float64)
    e = np.asarray(exact, np.float64)
    return float(np.linalg.norm(a - e) / np.linalg.norm(e))


def residual_vs_full(K, bits, group, base_bits=8, scheme="hd", kind="k"):
    """K: list of float32 [n, H, hd] arrays, one per loop (loop 1 first).

    Returns a dict with, per loop r = 1..R, the relative reconstruction error of the
    residual chain ("residual") and of full b-bit quantisation ("full"), and the
    reconstructions themselves ("hat_residual", "hat_full"). scheme "hd": the store's
    codec (groups along head_dim, a ``base_bits`` base); scheme "pages": the pages'
    scheme for keys or values (``kind``), the base quantised like the residuals."""
    R = len(K)
    if scheme == "pages":
        qb = qr = lambda a: pages_quant(a, kind, bits, group)
    else:
        qb = lambda a: _quant(a, base_bits, group)
        qr = lambda a: _quant(a, bits, group)
    out = {"residual": {}, "full": {}, "hat_residual": {}, "hat_full": {}}
    prev = None
    for r in range(1, R + 1):
        x = np.asarray(K[r - 1], np.float32)
        if r == 1:
            hat = qb(x)
        else:
            resid = (x - prev).astype(np.float32)
            hat = (prev + qr(resid)).astype(np.float32)
        full = qr(x)
        out["hat_residual"][r] = hat
        out["hat_full"][r] = full
        out["residual"][r] = rel_error(hat, x)
        out["full"][r] = rel_error(full, x)
        prev = hat
    return out
