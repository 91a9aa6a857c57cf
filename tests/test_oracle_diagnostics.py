"""Pins of the residual-vs-full quantisation diagnostic (oracle/diagnostics.py).

The reconstruction errors are checked against closed forms that do not use the oracle:
a b-bit uniform quantiser over a group of g values spans the group's range R in 2^b - 1
steps, so its error is uniform with RMS (R / (2^b - 1)) / sqrt(12); for N(0, sigma^2)
values the expected range of a group is 2 E[max of g normals] sigma, with E[max]
integrated here numerically. Constant groups are reproduced exactly, and a chain whose
loops do not change keeps shrinking its error (each loop re-quantises what is left)."""
import math

import numpy as np
from scipy import integrate, stats

from cross_loop_sparse_step_b200 import synth
from oracle import diagnostics as odiag


def _expected_max(g):
    f = lambda x: x * g * stats.norm.pdf(x) * stats.norm.cdf(x) ** (g - 1)
    return integrate.quad(f, -10, 10)[0]


def _rms_error(bits, g, sigma=1.0):
    return 2 * _expected_max(g) * sigma / ((2 ** bits - 1) * math.sqrt(12))


def test_full_and_residual_errors_match_closed_forms():
    n, H, hd, g, R, delta = 4096, 2, 128, 32, 4, 0.25
    K = synth.kv_loop_sequence(synth.rng(11), n, H, hd, R, delta=delta)
    res = odiag.residual_vs_full(K, bits=4, group=g)
    # full 4-bit quantisation of N(0, var_r) values: relative error = RMS / 1
    for r in range(1, R + 1):
        assert abs(res["full"][r] - _rms_error(4, g)) < 0.03 * _rms_error(4, g), (r, res["full"][r])
    # the 8-bit base
    assert abs(res["residual"][1] - _rms_error(8, g)) < 0.03 * _rms_error(8, g)
    # loop 2: the residual is the change (the base error is 50x smaller), std delta, and
    # ||K_2|| = sqrt(1 + delta^2) per element
    want2 = _rms_error(4, g, delta) / math.sqrt(1 + delta ** 2)
    assert abs(res["residual"][2] - want2) < 0.05 * want2, (res["residual"][2], want2)
    # residual quantisation beats full quantisation by about the size of the change
    for r in range(2, R + 1):
        assert res["residual"][r] < 0.5 * res["full"][r]


def test_constant_groups_are_exact_and_unchanged_chains_shrink():
    n, H, hd, g = 64, 1, 64, 32
    K1 = np.repeat(np.float32([0.5, -1.25]), 32)[None, None, :].repeat(n, 0)
    K = [K1, K1.copy(), K1.copy()]
    res = odiag.residual_vs_full(K, bits=2, group=g)
    assert all(v == 0.0 for v in res["full"].values())
    assert all(v == 0.0 for v in res["residual"].values())
    K = [synth.kv_values(synth.rng(3), n, H, hd)] * 4
    res = odiag.residual_vs_full(K, bits=4, group=g)
    errs = [res["residual"][r] for r in range(1, 5)]
    assert all(b <= a for a, b in zip(errs, errs[1:])) and errs[-1] < errs[0]


# ---- the pages' scheme (App. E "Quantization Setting"): INT4, groups of 64, keys per
# channel along tokens, values per token, the most recent 64 tokens in bfloat16

def test_pages_scheme_closed_form_and_window():
    n, H, hd = 64 * 20 + 64, 2, 128
    x = synth.kv_values(synth.rng(21), n, H, hd)
    for kind in ("k", "v"):
        y = odiag.pages_quant(x, kind)
        # the window: the last 64 tokens are their bfloat16 roundings, exactly
        win = x[-64:]
        u = win.view(np.uint32).astype(np.uint64)
        want = ((u + 0x7FFF + ((u >> 16) & 1)) & 0xFFFF0000).astype(np.uint32).view(np.float32)
        assert np.array_equal(y[-64:], want)
        # the quantised tokens: 4-bit groups of 64 N(0, 1) values (along tokens for keys,
        # along channels for values) - the uniform-error closed form
        e = odiag.rel_error(y[:-64], x[:-64])
        assert abs(e - _rms_error(4, 64)) < 0.03 * _rms_error(4, 64), (kind, e)


def test_pages_scheme_keys_are_grouped_along_tokens():
    # channels of very different scale (the reason keys are quantised per channel):
    # grouping along tokens keeps each channel's own range, grouping along channels
    # (per token) lets the large channels set every group's step
    n, H, hd = 64 * 8 + 64, 1, 128
    g = synth.rng(5)
    scale = np.exp(np.linspace(np.log(0.05), np.log(20.0), hd)).astype(np.float32)
    x = (synth.kv_values(g, n, H, hd) * scale[None, None, :]).astype(np.float32)
    small = slice(0, 32)   # the smallest-scale channels
    yk, yv = odiag.pages_quant(x, "k"), odiag.pages_quant(x, "v")
    k_err = odiag.rel_error(yk[:-64, :, small], x[:-64, :, small])
    v_err = odiag.rel_error(yv[:-64, :, small], x[:-64, :, small])
    assert k_err < 0.3 * v_err, (k_err, v_err)
    assert abs(k_err - _rms_error(4, 64)) < 0.05 * _rms_error(4, 64), k_err
    # a key channel constant along the tokens of a group is reproduced exactly (range 0),
    # also in a trailing group shorter than 64
    n2 = 64 + 36 + 64
    c = np.float32([0.5, -1.25, 3.0, 0.0] * 32)
    x2 = np.repeat(c[None, None, :], n2, 0).astype(np.float32)
    assert np.array_equal(odiag.pages_quant(x2, "k"), x2)


def test_pages_scheme_residuals_beat_full_quantisation():
    n, H, hd, R = 64 * 16 + 64, 2, 128, 4
    K = synth.kv_loop_sequence(synth.rng(17), n, H, hd, R, delta=0.25)
    for kind in ("k", "v"):
        res = odiag.residual_vs_full(K, bits=4, group=64, scheme="pages", kind=kind)
        # the base is quantised like every loop in full: the same error at loop 1
        assert res["residual"][1] == res["full"][1]
        for r in range(2, R + 1):
            assert res["residual"][r] < 0.5 * res["full"][r], (kind, r, res["residual"][r], res["full"][r])
