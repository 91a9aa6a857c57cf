"""Pins of the oracle's attention (FlashLoop §4.2 "Loop-Aware Sparse Attention").

* brute force: causal softmax attention at 50 significant digits (mpmath) on N <= 16;
* closed form: equal logits give the running mean of V;
* library: torch's fp64 scaled_dot_product_attention with an additive bias mask;
* cached mass (§4.2): the selected mass plus the unselected probability is 1, the
  rescaled probabilities sum to the cached mass, and with unchanged logits the sparse
  output equals the dense one;
* selections: sort-based brute force, the sink, sizes, ascending order, pruning is a
  subset and keeps the output's bookkeeping (u' + sum_S' p~ V = u + sum_S p~ V)."""
import mpmath
import numpy as np
import pytest
import torch

from oracle import attention

mpmath.mp.dps = 50


def _case(seed, n, H, hd, bias=True):
    g = np.random.Generator(np.random.PCG64(seed))
    q = g.normal(size=(n, H, hd))
    K = g.normal(size=(n, H, hd)).astype(np.float32)
    V = g.normal(size=(n, H, hd)).astype(np.float32)
    b = (g.normal(size=n) * 2).astype(np.float32) if bias else None
    return q, K, V, b


def _mp_attention(q, K, V, b, i, h):
    hd = q.shape[-1]
    sc = mpmath.mpf(1) / mpmath.sqrt(hd)
    s = []
    for j in range(i + 1):
        acc = mpmath.mpf(0)
        for e in range(hd):
            acc += mpmath.mpf(float(q[i, h, e])) * mpmath.mpf(float(K[j, h, e]))
        v = acc * sc
        if b is not None:
            v += mpmath.mpf(float(b[j]))
        s.append(v)
    mx = max(s)
    ex = [mpmath.exp(v - mx) for v in s]
    z = sum(ex)
    return [float(sum(ex[j] / z * mpmath.mpf(float(V[j, h, e])) for j in range(i + 1)))
            for e in range(hd)]


def test_dense_brute_force_mpmath():
    q, K, V, b = _case(1, 12, 2, 8)
    o = attention.dense_attention(q, np.arange(12), K, V, b)
    for i in range(12):
        for h in range(2):
            want = np.array(_mp_attention(q, K, V, b, i, h))
            assert np.max(np.abs(o[i, h] - want)) <= 1e-13 * max(1.0, np.abs(want).max())


def test_uniform_logits_closed_form():
    _, K, V, _ = _case(2, 16, 3, 8)
    q = np.zeros((16, 3, 8))
    o = attention.dense_attention(q, np.arange(16), K, V, None)
    for i in range(16):
        want = V[: i + 1].astype(np.float64).mean(axis=0)
        assert np.allclose(o[i], want, rtol=0, atol=1e-14)


def test_dense_matches_torch_sdpa():
    n, H, hd = 40, 3, 16
    q, K, V, b = _case(3, n, H, hd)
    o = attention.dense_attention(q, np.arange(n), K, V, b)
    qt = torch.tensor(q).permute(1, 0, 2)[None]
    kt = torch.tensor(K.astype(np.float64)).permute(1, 0, 2)[None]
    vt = torch.tensor(V.astype(np.float64)).permute(1, 0, 2)[None]
    mask = torch.full((n, n), float("-inf"), dtype=torch.float64).triu(1)
    mask = mask + torch.tensor(b.astype(np.float64))[None, :]
    ot = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, attn_mask=mask)
    ot = ot[0].permute(1, 0, 2).numpy()
    assert np.max(np.abs(o - ot)) < 1e-12


@pytest.mark.parametrize("stat", ["pv", "p"])
def test_dense_stats_brute_force(stat):
    n, H, hd, k = 30, 2, 8, 5
    q, K, V, b = _case(4, n, H, hd)
    o, S, m, u = attention.dense_attention(q, np.arange(n), K, V, b, k_sel=k, stat=stat)
    for i in range(n):
        s = np.einsum("jhd,hd->hj", K[: i + 1].astype(np.float64), q[i]) / np.sqrt(hd) + b[: i + 1]
        p = np.exp(s - s.max(1, keepdims=True))
        p /= p.sum(1, keepdims=True)
        for h in range(H):
            sel = S[h, i][S[h, i] != attention.SENTINEL].astype(int)
            assert sel[0] == 0 and len(sel) == min(k, i) + 1
            assert list(sel) == sorted(sel)
            if i > k:
                vn = [float(np.linalg.norm(V[j, h].astype(np.float64))) for j in range(i + 1)]
                c = [p[h, j] * (vn[j] if stat == "pv" else 1.0) for j in range(i + 1)]
                brute = sorted(range(1, i + 1), key=lambda j: (-c[j], j))[:k]
                assert list(sel) == [0] + sorted(brute)
            assert abs(m[h, i] - p[h, sel].sum()) < 1e-14
            rest = np.setdiff1d(np.arange(i + 1), sel)
            assert np.allclose(u[h, i], p[h, rest] @ V[rest, h].astype(np.float64), atol=1e-14)
            # cached mass + unselected probability = full mass
            assert abs(m[h, i] + p[h, rest].sum() - 1.0) < 1e-12
            # o = u + sum_S p V
            assert np.allclose(o[i, h], u[h, i] + p[h, sel] @ V[sel, h].astype(np.float64), atol=1e-13)


def test_ties_go_to_smaller_column():
    # identical K rows and V rows: every column has the same statistic
    n, H, hd, k = 12, 1, 4, 3
    K = np.ones((n, H, hd), np.float32)
    V = np.ones((n, H, hd), np.float32)
    q = np.ones((n, H, hd))
    _, S, _, _ = attention.dense_attention(q, np.arange(n), K, V, None, k_sel=k)
    assert list(S[0, n - 1]) == [0, 1, 2, 3]


def test_sparse_equals_dense_when_logits_unchanged():
    """Selected + cached mass = full mass: with the previous loop's own q and K^/V^
    the sparse output reproduces the dense output exactly (u carries the rest)."""
    n, H, hd, k = 48, 3, 16, 6
    q, K, V, b = _case(5, n, H, hd)
    o, S, m, u = attention.dense_attention(q, np.arange(n), K, V, b, k_sel=k)
    act = np.array([3, 7, 20, 33, 47])
    o2, S2, m2, u2 = attention.sparse_attention(q[act], act, act, K, V, S, m, u, b, k_next=k)
    assert np.max(np.abs(o2 - o[act])) < 1e-12
    # rescaled probabilities sum to the cached mass; unchanged budget leaves stats as is
    assert np.array_equal(S2, S[:, act])
    assert np.array_equal(m2, m[:, act]) and np.array_equal(u2, u[:, act])


def test_sparse_all_columns_is_dense():
    n, H, hd = 24, 2, 8
    q, K, V, b = _case(6, n, H, hd)
    S = np.full((H, n, n + 1), attention.SENTINEL, np.uint16)
    for i in range(n):
        S[:, i, : i + 1] = np.arange(i + 1)
    m = np.ones((H, n))
    u = np.zeros((H, n, hd))
    g = np.random.Generator(np.random.PCG64(7))
    q2 = g.normal(size=q.shape)  # new loop, new queries
    o_sp = attention.sparse_attention(q2, np.arange(n), np.arange(n), K, V, S, m, u, b)
    o_dn = attention.dense_attention(q2, np.arange(n), K, V, b)
    assert np.max(np.abs(o_sp - o_dn)) < 1e-13


def test_pruning_subset_and_bookkeeping():
    n, H, hd, k, k2 = 64, 2, 8, 10, 4
    q, K, V, b = _case(8, n, H, hd)
    _, S, m, u = attention.dense_attention(q, np.arange(n), K, V, b, k_sel=k)
    g = np.random.Generator(np.random.PCG64(9))
    q2 = q + 0.3 * g.normal(size=q.shape)
    act = np.arange(0, n, 3)
    o, S2, m2, u2 = attention.sparse_attention(q2[act], act, act, K, V, S, m, u, b, k_next=k2)
    scale = 1 / np.sqrt(hd)
    for ii, t in enumerate(act):
        for h in range(H):
            old = S[h, t][S[h, t] != attention.SENTINEL].astype(int)
            new = S2[h, ii][S2[h, ii] != attention.SENTINEL].astype(int)
            assert set(new) <= set(old) and new[0] == 0
            assert len(new) == min(k2, t) + 1
            s = K[old, h].astype(np.float64) @ q2[t, h] * scale + b[old]
            pt = m[h, t] * np.exp(s - s.max()) / np.exp(s - s.max()).sum()
            keep = np.isin(old, new)
            assert abs(m2[h, ii] - pt[keep].sum()) < 1e-14
            lhs = u2[h, ii] + pt[keep] @ V[new, h].astype(np.float64)
            assert np.allclose(lhs, o[ii, h], atol=1e-13)
            if len(old) - 1 > k2:
                vn = np.linalg.norm(V[old, h].astype(np.float64), axis=1)
                c = pt * vn
                brute = sorted(range(1, len(old)), key=lambda j: (-c[j], old[j]))[:k2]
                assert list(new) == [0] + sorted(old[brute].tolist())


def test_planted_mistake_dropped_u_is_caught(monkeypatch):
    """A plausible slip (forgetting the unselected contribution) must fail the
    unchanged-logits pin."""
    n, H, hd, k = 32, 2, 8, 4
    q, K, V, b = _case(10, n, H, hd)
    o, S, m, u = attention.dense_attention(q, np.arange(n), K, V, b, k_sel=k)
    act = np.arange(10, 32)
    o2 = attention.sparse_attention(q[act], act, act, K, V, S, m, np.zeros_like(u), b)
    assert np.max(np.abs(o2 - o[act])) > 1e-3
