"""Residual-vs-full quantisation of per-loop KV (oracle; test infrastructure only).

Pages: FlashLoop paper §3.3 "Quantization-Friendly KV Residual" (the KV of one loop
differs little from the previous loop's, so quantising that difference loses less than
quantising every loop's KV in full at the same bit width; Figure 2c plots the two
reconstruction errors), §5.3.1 Table 2 (per-loop KIVI-style quantisation as the
ablation), Appendix E (the same asymmetric group-wise scheme for base and residuals).

Readings:
  * full quantisation of loop r: K~_r = Q_b(K_r), every loop on its own, b bits, the
    codec of ``codec.quantize_groups`` (groups along head_dim);
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


def rel_error(approx, exact):
    a = np.asarray(approx, np.float64)
    e = np.asarray(exact, np.float64)
    return float(np.linalg.norm(a - e) / np.linalg.norm(e))


def residual_vs_full(K, bits, group, base_bits=8):
    """K: list of float32 [n, H, hd] arrays, one per loop (loop 1 first).

    Returns a dict with, per loop r = 1..R, the relative reconstruction error of the
    residual chain ("residual") and of full b-bit quantisation ("full"), and the
    reconstructions themselves ("hat_residual", "hat_full")."""
    R = len(K)
    out = {"residual": {}, "full": {}, "hat_residual": {}, "hat_full": {}}
    prev = None
    for r in range(1, R + 1):
        x = np.asarray(K[r - 1], np.float32)
        if r == 1:
            hat = _quant(x, base_bits, group)
        else:
            resid = (x - prev).astype(np.float32)
            hat = (prev + _quant(resid, bits, group)).astype(np.float32)
        full = _quant(x, bits, group)
        out["hat_residual"][r] = hat
        out["hat_full"][r] = full
        out["residual"][r] = rel_error(hat, x)
        out["full"][r] = rel_error(full, x)
        prev = hat
    return out
