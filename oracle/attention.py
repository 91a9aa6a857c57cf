"""Dense causal attention with column statistics, and loop-aware sparse attention
(oracle; fp64 arithmetic on binary32 K^/V^; test infrastructure only).

Pages: FlashLoop §4.2 "Loop-Aware Sparse Attention". Each sparse loop ranks the
attention columns by statistics of the previous loop and keeps the top-K under a
loop budget; it gathers only those keys/values; a softmax over the selected logits
alone would overstate them, so the selected columns' total probability under the
previous loop's full distribution (the cached mass) rescales the new softmax; the
rescaled contributions update the output ("Eq. 3", absent from the pages); smaller
later budgets prune the set with the statistics of the preceding sparse loop, and
indices and mass are carried from loop to loop.

Readings (the pages are silent or the equation is missing):
  * score s_ij = q_i . K^[j] / sqrt(hd) + b_j, causal (j <= i), b_j a per-column
    logit bias (0 unless a workload sets it);
  * column set per (query, head); column 0 (sink) always kept and not counted in k;
    a query at position i <= k keeps all of [0, i];
  * contribution statistic c_ij = P_ij * ||V^[j]||_2 over the head slice
    (``stat="p"`` uses P_ij alone);
  * dense statistics: S_i = {0} U top-k of c over [1, i] (ties to the smaller j),
    m_i = sum_{S_i} p_ij, u_i = sum_{j not in S_i} p_ij V^[j];
  * sparse output ("Eq. 3"): p~_ij = m_i softmax_{S_i}(s)_j, o_i = u_i + sum_S p~ V^;
    it equals the dense output when S_i holds every causal column (m = 1, u = 0);
  * pruning to k' < k: S'_i = {0} U top-k' of p~ ||V^|| within S_i \\ {0},
    m'_i = sum_{S'} p~, u'_i = u_i + sum_{S \\ S'} p~ V^; with k' >= k nothing changes.
S is stored ascending, padded with 0xFFFF to k + 1 entries.
"""
import numpy as np

SENTINEL = 0xFFFF


def topk_ties_low(c, idx, k):
    """The k entries of idx with the largest c; among equal c the smaller idx wins."""
    order = np.lexsort((idx, -np.asarray(c, np.float64)))
    return np.sort(idx[order[:k]])


def _vnorm(Vhat_cols_h):
    return np.sqrt(np.sum(np.asarray(Vhat_cols_h, np.float64) ** 2, axis=-1))


def _stat(p, vn, stat):
    return p * vn if stat == "pv" else p


def dense_attention(q, q_tok, Khat, Vhat, bias=None, k_sel=None, stat="pv"):
    """Causal softmax attention of queries ``q`` [nq, H, hd] at positions ``q_tok``
    over every column j <= position, reading K^, V^ [n_tok, H, hd].

    Returns o [nq, H, hd] and, when ``k_sel`` is given, the statistics
    S uint16 [H, nq, k_sel + 1], m float64 [H, nq], u float64 [H, nq, hd]."""
    q = np.asarray(q, np.float64)
    nq, H, hd = q.shape
    o = np.zeros((nq, H, hd))
    want = k_sel is not None
    if want:
        S = np.full((H, nq, k_sel + 1), SENTINEL, np.uint16)
        m = np.zeros((H, nq))
        u = np.zeros((H, nq, hd))
    scale = 1.0 / np.sqrt(hd)
    for i in range(nq):
        t = int(q_tok[i])
        cols = np.arange(t + 1)
        K = np.asarray(Khat[: t + 1], np.float64)      # [j, H, hd]
        V = np.asarray(Vhat[: t + 1], np.float64)
        s = np.einsum("jhd,hd->hj", K, q[i]) * scale
        if bias is not None:
            s = s + np.asarray(bias[: t + 1], np.float64)[None, :]
        s = s - s.max(axis=1, keepdims=True)
        e = np.exp(s)
        p = e / e.sum(axis=1, keepdims=True)            # [H, j]
        o[i] = np.einsum("hj,jhd->hd", p, V)
        if not want:
            continue
        for h in range(H):
            if t <= k_sel:
                sel = cols
            else:
                c = _stat(p[h, 1:], _vnorm(V[1:, h]), stat)
                sel = np.concatenate([[0], topk_ties_low(c, cols[1:], k_sel)])
            S[h, i, : len(sel)] = sel
            m[h, i] = p[h, sel].sum()
            mask = np.ones(t + 1, bool)
            mask[sel] = False
            u[h, i] = p[h, mask] @ V[mask, h]
    if want:
        return o, S, m, u
    return o


def sparse_attention(q, q_tok, q_row, Khat, Vhat, S, m, u, bias=None, k_next=None,
                     stat="pv"):
    """Loop-aware sparse attention of queries ``q`` [nq, H, hd].

    ``q_row[i]`` is the row of query i in the carried statistics S [H, rows, k+1],
    m [H, rows], u [H, rows, hd]. Returns o [nq, H, hd] and, when ``k_next`` is given,
    the pruned statistics for these queries: S' [H, nq, k_next+1], m' [H, nq],
    u' [H, nq, hd] (unchanged copies where the budget does not shrink)."""
    q = np.asarray(q, np.float64)
    nq, H, hd = q.shape
    o = np.zeros((nq, H, hd))
    want = k_next is not None
    if want:
        S2 = np.full((H, nq, k_next + 1), SENTINEL, np.uint16)
        m2 = np.zeros((H, nq))
        u2 = np.zeros((H, nq, hd))
    scale = 1.0 / np.sqrt(hd)
    for i in range(nq):
        row = int(q_row[i])
        t = int(q_tok[i])
        for h in range(H):
            sel = S[h, row]
            cols = sel[sel != SENTINEL].astype(np.int64)
            assert cols.size >= 1 and cols[0] == 0 and cols[-1] <= t
            K = np.asarray(Khat[cols, h], np.float64)
            V = np.asarray(Vhat[cols, h], np.float64)
            s = K @ q[i, h] * scale
            if bias is not None:
                s = s + np.asarray(bias, np.float64)[cols]
            e = np.exp(s - s.max())
            pt = float(m[h, row]) * e / e.sum()
            uu = np.asarray(u[h, row], np.float64)
            o[i, h] = uu + pt @ V
            if not want:
                continue
            if cols.size - 1 <= k_next:
                S2[h, i, : cols.size] = cols
                m2[h, i] = m[h, row]
                u2[h, i] = uu
                continue
            c = _stat(pt[1:], _vnorm(V[1:]), stat)
            keep_cols = np.concatenate([[0], topk_ties_low(c, cols[1:], k_next)])
            keep = np.isin(cols, keep_cols)
            S2[h, i, : keep_cols.size] = keep_cols
            m2[h, i] = pt[keep].sum()
            u2[h, i] = uu + pt[~keep] @ V[~keep]
    if want:
        return o, S2, m2, u2
    return o
