"""Pins of the pages' quantisation scheme as a cross-loop store (oracle/kvstore_pages.py).

Checked against what does not come from the store itself: the diagnostic's independent
formulation of the same per-loop scheme (a transpose and reshape instead of a loop over
groups), the closed-form error of a 4-bit uniform quantiser over groups of 64 normal
values, exact cases (constant channels, bfloat16 window values), and the byte count
written out from the scheme's definition."""
import math

import numpy as np
from scipy import integrate, stats

from cross_loop_sparse_step_b200 import synth
from oracle import diagnostics as odiag
from oracle import kvstore_pages as okp


def _rms_error(bits, g, sigma=1.0):
    f = lambda x: x * g * stats.norm.pdf(x) * stats.norm.cdf(x) ** (g - 1)
    emax = integrate.quad(f, -10, 10)[0]
    return 2 * emax * sigma / ((2 ** bits - 1) * math.sqrt(12))


def _bf16(x):
    u = np.ascontiguousarray(x, np.float32).view(np.uint32).astype(np.uint64)
    return ((u + 0x7FFF + ((u >> 16) & 1)) & 0xFFFF0000).astype(np.uint32).view(np.float32)


def _store(n=64 * 12 + 64, H=2, hd=128, R=3, seed=0):
    g = synth.rng(seed)
    K = synth.kv_loop_sequence(g, n, H, hd, R)
    V = synth.kv_loop_sequence(g, n, H, hd, R)
    st = okp.LayerKVPages(n, H, hd, R)
    st.write_base(K[0], V[0])
    acts = {}
    for r in range(2, R + 1):
        act = np.sort(g.choice(n, size=n // 3, replace=False))
        act = np.unique(np.concatenate([act, [n - 1, n - 30]]))   # window tokens active
        acts[r] = act
        st.write_residual(r, act, K[r - 1][act], V[r - 1][act])
    return st, K, V, acts


def test_base_equals_the_diagnostic_formulation():
    st, K, V, _ = _store()
    assert np.array_equal(st.hat[1][0], odiag.pages_quant(K[0], "k"))
    assert np.array_equal(st.hat[1][1], odiag.pages_quant(V[0], "v"))


def test_reconstruction_from_the_stored_codes():
    st, _, _, _ = _store()
    for r in (1, 2, 3):
        assert np.array_equal(st.reconstruct(r), st.hat[r])


def test_window_tokens_hold_bfloat16_values():
    st, K, V, acts = _store()
    n = st.n_tok
    win = np.arange(n - 64, n)
    assert np.array_equal(st.hat[1][0][win], _bf16(K[0][win]))
    for r, act in acts.items():
        on = act[act >= n - 64]
        off = np.setdiff1d(win, act)
        assert np.array_equal(st.hat[r][0][on], _bf16(K[r - 1][on]))
        assert np.array_equal(st.hat[r][1][on], _bf16(V[r - 1][on]))
        assert np.array_equal(st.hat[r][0][off], st.hat[r - 1][0][off])   # kept


def test_base_error_matches_the_closed_form():
    n, H, hd = 64 * 40 + 64, 2, 128
    K = synth.kv_values(synth.rng(4), n, H, hd)
    st = okp.LayerKVPages(n, H, hd, 1)
    st.write_base(K, K)
    e = odiag.rel_error(st.hat[1][0][:-64], K[:-64])
    assert abs(e - _rms_error(4, 64)) < 0.03 * _rms_error(4, 64), e


def test_key_groups_run_over_the_loops_active_rows():
    # a residual that is constant along the active rows of every channel has range 0 in
    # every key group: the new keys are the previous ones plus it, exactly
    n, H, hd = 64 * 6 + 64, 1, 128
    g = synth.rng(8)
    K1 = synth.kv_values(g, n, H, hd)
    st = okp.LayerKVPages(n, H, hd, 2)
    st.write_base(K1, K1)
    act = np.sort(g.choice(n - 64, size=150, replace=False))      # none in the window
    c = np.float32([0.25, -0.5, 1.5, 0.0] * 32)[None, None, :]
    k2 = (st.hat[1][0][act] + c).astype(np.float32)
    st.write_residual(2, act, k2, k2)
    assert np.array_equal(st.hat[2][0][act], k2)
    # values are grouped per token: a channel-constant residual is not constant within a
    # value group, so the values are not exact
    assert not np.array_equal(st.hat[2][1][act], (st.hat[1][1][act] + c).astype(np.float32))


def test_bytes_follow_the_scheme():
    n, H, hd = 64 * 10 + 37 + 64, 3, 128
    st, _, _, acts = _store(n=n, H=H, hd=hd, R=2)
    nq = n - 64
    want1 = 2 * nq * H * hd // 2                     # 4-bit codes of K and V
    want1 += math.ceil(nq / 64) * H * hd * 4         # key (scale, offset) per channel and group
    want1 += nq * H * (hd // 64) * 4                 # value pairs per token and group
    want1 += 2 * 64 * H * hd * 2                     # the bfloat16 window
    assert st.nbytes(1) == want1
    act = acts[2]
    a_q, a_w = int((act < n - 64).sum()), int((act >= n - 64).sum())
    want2 = 2 * a_q * H * hd // 2 + math.ceil(a_q / 64) * H * hd * 4 + a_q * H * (hd // 64) * 4
    want2 += 2 * a_w * H * hd * 2
    assert st.nbytes(2) == want2
