"""The R-loop driver: dense loop 1, then loops with the three lazy updates
(oracle; test infrastructure only).

Pages: FlashLoop §1 (R loops of a shared block, a distinct KV per loop), §4 (three
coupled lazy updates: token-sparse updates §4.1, loop-aware sparse attention §4.2,
cross-loop KV residual quantisation §4.3), §3.1 (converged tokens reuse their
state and KV).

Loop r, as this oracle runs it (readings marked in the modules it calls):
  r = 1             every token, dense attention, base KV for every token;
  2 <= r < r_s      every token (dense early loops), residual KV for every token;
  r >= r_s          A_r = top-k_r of the normalized change over A_{r-1};
  every r >= 2      X = h_{r-1}[A_r]; per layer: q, k, v for X at positions A_r;
                    residual KV for A_r; attention of the A_r queries (sparse with
                    the carried statistics when the loop's column budget is set,
                    dense otherwise); output projection and FFN on X;
                    h_r = h_{r-1} with rows A_r replaced by X.
A loop whose successor uses sparse attention also emits the statistics (column set,
mass, unselected contribution) for its queries, with the successor's budget.
Statistics are kept per token: row t holds the state of query t.

``sched`` keys: n_loops, first_sparse (r_s), tok_frac {r: f}, col_k {r: k or None},
base_bits, res_bits {r: b}, group, stat ("pv" or "p").
"""
import numpy as np

from . import attention, block, kvstore, select


def run(layers, h0, sched, n_heads, head_dim, bias=None, eps=1e-6, theta=10000.0,
        select_prev=None, bf16_ops=False):
    """Run loops 1..R. ``layers`` is a list of weight dicts (see ``block``).

    ``select_prev`` optionally maps a loop r to the array used in place of
    h_{r-2}[A_{r-1}] when that loop ranks tokens (a synthetic previous state), or to
    a function of the current rows h_{r-1}[A_{r-1}] returning it. ``bf16_ops``: the
    GEMM operands are bfloat16 tensors (bf16 workloads).
    Returns a dict with per-loop hidden states, active sets, deltas, the per-layer
    KV stores and the statistics after every loop."""
    h0 = np.asarray(h0, np.float64)
    N, d = h0.shape
    R = sched["n_loops"]
    r_s = sched["first_sparse"]
    col_k = sched.get("col_k", {})
    L = len(layers)
    stores = [kvstore.LayerKV(N, n_heads, head_dim, sched["group"], sched["base_bits"],
                              sched["res_bits"], R) for _ in range(L)]
    stat = sched.get("stat", "pv")
    out = {"h": {0: h0.copy()}, "act": {}, "delta": {}, "stats": {}, "stores": stores,
           "k": {}}
    stats = [None] * L

    def next_k(r):
        return col_k.get(r + 1) if r + 1 <= R else None

    for r in range(1, R + 1):
        h_prev = out["h"][r - 1]
        if r == 1:
            act = np.arange(N, dtype=np.int32)
        elif r < r_s:
            act = np.arange(N, dtype=np.int32)
        else:
            cand = out["act"][r - 1]
            hp = out["h"][r - 2][cand]
            if select_prev is not None and r in select_prev:
                sp = select_prev[r]
                hp = np.asarray(sp(h_prev[cand]) if callable(sp) else sp, np.float64)
            kr = select.active_count(sched["tok_frac"][r], N, len(cand))
            act, _, delta = select.select_active(h_prev[cand], hp, cand, kr)
            out["delta"][r] = delta
        out["act"][r] = act
        X = h_prev[act].copy()
        kn = next_k(r)
        new_stats = [None] * L
        for li, layer in enumerate(layers):
            q, k, v = block.qkv(X, act, layer, n_heads, head_dim, eps, theta, bf16_ops)
            if r == 1:
                stores[li].write_base(k.astype(np.float32), v.astype(np.float32))
            else:
                stores[li].write_residual(r, act, k.astype(np.float32), v.astype(np.float32))
            Kh = stores[li].hat[r][0]
            Vh = stores[li].hat[r][1]
            if r >= 2 and col_k.get(r) is not None:
                S, m, u = stats[li]
                res = attention.sparse_attention(q, act, act, Kh, Vh, S, m, u, bias,
                                                 k_next=kn, stat=stat)
            else:
                res = attention.dense_attention(q, act, Kh, Vh, bias, k_sel=kn, stat=stat)
            if kn is not None:
                o, S2, m2, u2 = res
                # token-indexed statistics: row t holds query t
                H = n_heads
                S_full = np.full((H, N, kn + 1), attention.SENTINEL, np.uint16)
                m_full = np.zeros((H, N))
                u_full = np.zeros((H, N, head_dim))
                S_full[:, act] = S2
                m_full[:, act] = m2
                u_full[:, act] = u2
                new_stats[li] = (S_full, m_full, u_full)
            else:
                o = res
            X = block.out_ffn(X, o.reshape(len(act), d), layer, eps, bf16_ops)
        stats = new_stats
        out["stats"][r] = stats
        h = h_prev.copy()
        h[act] = X
        out["h"][r] = h
        out["k"][r] = len(act)
    return out


def kv_bytes_per_token(n_tok, d, n_act, base_bits, res_bits, group):
    """Closed form of the stored KV bytes per token per layer over loops 1..R.

    K and V each hold d values per token: base b/8 bytes each plus 4 bytes of
    (scale, offset) per group; a loop r >= 2 adds the same for its active tokens."""
    def row(bits):
        if bits == 0:
            return 2 * d * 4
        return 2 * (d * bits // 8 + (d // group) * 4)
    total = n_tok * row(base_bits)
    for r, k in n_act.items():
        if r >= 2:
            total += k * row(res_bits[r])
    return total / n_tok
