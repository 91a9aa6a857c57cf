"""Full-size parity for the long-context and loop-depth workloads, on sampled outputs.

* 32K-token Ouro-2.6B shape (16 x 128 heads, int8 base + 2-bit residuals, group 32,
  4916 active tokens, 2048 carried columns): token ranking over all 32768 rows, base and
  residual quantisation of every row, the dense producer with 2048-column statistics on
  sampled queries, and the sparse step of all 4916 active queries (sampled outputs).
* 8K-token loop-depth sweep (group 64, 512 carried columns, residual chains up to 15
  loops deep, 2 and 4 bits): the sparse step at loop 16 after a geometric active-token
  schedule, and a budget shrink.
Carried statistics are synthetic inputs here (sink, biased columns, random others), so
the oracle only has to evaluate the sampled queries."""
import numpy as np
import pytest
import torch

from cross_loop_sparse_step_b200 import configs, synth
from oracle import attention as oatt
from oracle import kvstore as okv
from oracle import select as osel
from tests.gpu_helpers import (assert_close, check_selection, dev, host, sel_to_dev,
                               sel_to_host, upload_store)

pytestmark = pytest.mark.gpu


def _fl():
    from cross_loop_sparse_step_b200 import fl
    return fl


def _stats(rs, n, H, hd, k, q_tok, bias_cols, random_rows):
    """Synthetic carried statistics for the rows of q_tok, min(k, t) + 1 ascending
    columns each with the sink first. Rows in ``random_rows`` (the ones the oracle checks)
    get the biased columns before the query plus random others, per head; the other
    rows get evenly spaced columns. Mass in (0.3, 1); unselected contribution N(0, 0.1^2)."""
    S = np.full((H, n, k + 1), oatt.SENTINEL, np.uint16)
    rand = set(int(x) for x in random_rows)
    for t in q_tok:
        t = int(t)
        if t <= k:
            S[:, t, : t + 1] = np.arange(t + 1)
        elif t not in rand:
            S[:, t, :] = np.concatenate([[0], np.floor(np.linspace(1, t, k)).astype(np.int64)])
        else:
            bc = bias_cols[(bias_cols >= 1) & (bias_cols <= t)][:k]
            for h in range(H):
                pool = np.setdiff1d(np.arange(1, t + 1), bc)
                extra = rs.choice(pool, size=k - len(bc), replace=False)
                S[h, t] = np.sort(np.concatenate([[0], bc, extra]))
    m = rs.uniform(0.3, 1.0, size=(H, n)).astype(np.float32)
    u = (rs.normal(size=(H, n, hd)) * 0.1).astype(np.float32)
    return S, m, u


def _store(rs, n, H, hd, g, res_bits, act_sets, R):
    ost = okv.LayerKV(n, H, hd, g, 8, res_bits, R)
    ost.write_base(synth.kv_values(rs, n, H, hd), synth.kv_values(rs, n, H, hd))
    for r in range(2, R + 1):
        act = act_sets[r]
        kr = (ost.hat[r - 1][0][act] + 0.5 ** (r - 1) * rs.normal(size=(len(act), H, hd))).astype(np.float32)
        vr = (ost.hat[r - 1][1][act] + 0.5 ** (r - 1) * rs.normal(size=(len(act), H, hd))).astype(np.float32)
        ost.write_residual(r, act, kr, vr)
    return ost


def _nested_sets(rs, n, counts, R):
    sets = {1: np.arange(n, dtype=np.int32)}
    for r in range(2, R + 1):
        sets[r] = np.sort(rs.choice(sets[r - 1], size=counts[r], replace=False)).astype(np.int32)
    return sets


def test_32k_select_bit_exact():
    fl = _fl()
    cfg = configs.PREFILL_32K
    N, d = cfg["n_tok"], cfg["d_model"]
    k = configs.active_counts(cfg)[2]
    g = synth.rng(31)
    cur, prev, _ = synth.pareto_delta_pair(g, N, d, 2)
    want_tok, want_pos, delta = osel.select_active(cur, prev, None, k)
    srt = np.sort(delta)[::-1]
    assert (srt[k - 1] - srt[k]) / srt[k - 1] > 1e-5
    out = torch.zeros(k, dtype=torch.int32, device="cuda")
    pos = torch.zeros(k, dtype=torch.int32, device="cuda")
    fl.select_active(dev(cur), dev(prev), k, None, out, pos)
    assert fl.check_device_status() == 0
    assert np.array_equal(host(out), want_tok) and np.array_equal(host(pos), want_pos)


def test_32k_quant_bit_exact():
    fl = _fl()
    cfg = configs.PREFILL_32K
    N, H, hd, g = cfg["n_tok"], cfg["n_heads"], cfg["head_dim"], cfg["group"]
    k2 = configs.active_counts(cfg)[2]
    rs = synth.rng(32)
    ost = okv.LayerKV(N, H, hd, g, 8, {2: 2}, 2)
    store = fl.KVStore(N, H, hd, g, 8, {2: 2}, 2, {2: k2})
    k1, v1 = synth.kv_values(rs, N, H, hd), synth.kv_values(rs, N, H, hd)
    ost.write_base(k1, v1)
    fl.kv_residual_quant(store, 1, dev(k1), dev(v1))
    act = synth.sorted_subset(rs, N, k2)
    k2v = (k1[act] + 0.5 * rs.normal(size=(k2, H, hd))).astype(np.float32)
    v2v = (v1[act] + 0.5 * rs.normal(size=(k2, H, hd))).astype(np.float32)
    ost.write_residual(2, act, k2v, v2v)
    fl.kv_residual_quant(store, 2, dev(k2v), dev(v2v), dev(act))
    assert fl.check_device_status() == 0
    for r, rows in ((1, N), (2, k2)):
        for kv in range(2):
            assert np.array_equal(host(store.codes[(r, kv)])[:rows], ost.codes[(r, kv)])
            assert np.array_equal(host(store.sz[(r, kv)])[:rows].view(np.uint16),
                                  ost.sz[(r, kv)].view(np.uint16))


def test_32k_dense_producer_sampled():
    """The loop-1 producer with 2048-column statistics at the 32K shape, on 24 sampled
    queries (the kernel's grid is one CTA per query and head, so a subset is the same
    launch configuration per query)."""
    fl = _fl()
    cfg = configs.PREFILL_32K
    N, H, hd, g, k = cfg["n_tok"], cfg["n_heads"], cfg["head_dim"], cfg["group"], 2048
    rs = synth.rng(33)
    ost = okv.LayerKV(N, H, hd, g, 8, {}, 1)
    ost.write_base(synth.kv_values(rs, N, H, hd), synth.kv_values(rs, N, H, hd))
    store = fl.KVStore(N, H, hd, g, 8, {}, 1, {})
    upload_store(ost, store, 1)
    bias = synth.col_bias(rs, N, 0.02, 4.0)
    q_tok = np.sort(np.concatenate([[0, 5, 2047, 2048, 2049], rs.choice(np.arange(2050, N), 19, replace=False)])).astype(np.int32)
    q = synth.query_values(rs, len(q_tok), H, hd)
    out = torch.zeros(len(q_tok), H, hd, device="cuda")
    S = torch.full((H, N, k + 1), -1, dtype=torch.int16, device="cuda")
    m = torch.zeros(H, N, device="cuda")
    u = torch.zeros(H, N, hd, device="cuda")
    fl.sparse_loop_attn(dev(q), dev(q_tok), store, 1, out, col_bias=dev(bias), k_next=k,
                        sel_out=S, mass_out=m, unsel_out=u)
    assert fl.check_device_status() == 0
    Kh, Vh = ost.hat[1]
    o, So, mo, uo = oatt.dense_attention(q.astype(np.float64), q_tok, Kh, Vh, bias, k_sel=k)
    assert_close(host(out), o, what="o")

    def cfn(h, i):
        t = q_tok[i]
        cols = np.arange(t + 1)
        s = Kh[cols, h].astype(np.float64) @ q[i, h].astype(np.float64) / np.sqrt(hd) + bias[cols]
        e = np.exp(s - s.max())
        p = e / e.sum()
        return dict(zip(cols.tolist(), (p * np.linalg.norm(Vh[cols, h].astype(np.float64), axis=1)).tolist()))
    Sg = sel_to_host(S)[:, q_tok]
    ties = check_selection(Sg, So, cfn)
    keep = np.ones((H, len(q_tok)), bool)
    for h, i in ties:
        keep[h, i] = False
    assert len(ties) <= 4, ties
    assert_close(host(m)[:, q_tok][keep], mo[keep], what="mass")
    assert_close(host(u)[:, q_tok][keep], uo[keep], what="unsel")


@pytest.mark.parametrize("name,R,loop,bits,k,kn,sample", [
    ("32k", 2, 2, 2, 2048, 2048, 32),
    ("8k-R16", 16, 16, 2, 512, 512, 32),
    ("8k-R16-b4-shrink", 16, 16, 4, 512, 256, 32),
    ("8k-R8-b4", 8, 8, 4, 512, 512, 32),
])
def test_sparse_step_full_size_sampled(name, R, loop, bits, k, kn, sample):
    fl = _fl()
    if name.startswith("32k"):
        cfg = configs.PREFILL_32K
        counts = configs.active_counts(cfg)
        g = cfg["group"]
    else:
        cfg = configs.c4(R, bits)
        counts = configs.active_counts(cfg)
        g = cfg["group"]
    N, H, hd = cfg["n_tok"], cfg["n_heads"], cfg["head_dim"]
    rs = synth.rng(40 + R + bits + kn)
    res = {r: bits for r in range(2, R + 1)}
    sets = _nested_sets(rs, N, counts, R)
    ost = _store(rs, N, H, hd, g, res, sets, R)
    store = fl.KVStore(N, H, hd, g, 8, res, R, {r: counts[r] for r in range(2, R + 1)})
    upload_store(ost, store, loop)
    bias_cols = synth.biased_columns(rs, N, 0.02)
    bias = np.zeros(N, np.float32)
    bias[bias_cols] = 4.0
    bias[0] = 4.0
    act = sets[loop]
    pick = np.sort(rs.choice(len(act), size=min(sample, len(act)), replace=False))
    # statistics for every active query (the kernel's input), synthetic
    S, m, u = _stats(rs, N, H, hd, k, act, bias_cols, act[pick])
    q = synth.query_values(rs, len(act), H, hd)
    out = torch.zeros(len(act), H, hd, dtype=torch.bfloat16, device="cuda")
    Sd, md, ud = sel_to_dev(S), dev(m), dev(u)
    So_d = torch.full((H, N, kn + 1), -1, dtype=torch.int16, device="cuda")
    mo_d = torch.zeros(H, N, device="cuda")
    uo_d = torch.zeros(H, N, hd, device="cuda")
    fl.sparse_loop_attn(dev(q), dev(act), store, loop, out, col_bias=dev(bias), sel=Sd, mass=md,
                        unsel=ud, k_next=kn, sel_out=So_d, mass_out=mo_d, unsel_out=uo_d)
    assert fl.check_device_status() == 0
    Kh, Vh = ost.hat[loop]
    qa = act[pick]
    o, So, mo, uo = oatt.sparse_attention(q[pick].astype(np.float64), qa, qa, Kh, Vh, S,
                                          m.astype(np.float64), u.astype(np.float64), bias,
                                          k_next=kn)
    # the attention output is bf16 here: compare with the oracle's output rounded alike
    from oracle import block as oblk
    assert_close(host(out.float())[pick], oblk.bf16(o), what="o")
    Sg = sel_to_host(So_d)[:, qa]

    def cfn(h, i):
        row = S[h, qa[i]]
        cols = row[row != oatt.SENTINEL].astype(np.int64)
        s = Kh[cols, h].astype(np.float64) @ q[pick][i, h].astype(np.float64) / np.sqrt(hd) + bias[cols]
        e = np.exp(s - s.max())
        pt = m[h, qa[i]] * e / e.sum()
        return dict(zip(cols.tolist(), (pt * np.linalg.norm(Vh[cols, h].astype(np.float64), axis=1)).tolist()))
    ties = check_selection(Sg, So, cfn)
    keep = np.ones((H, len(pick)), bool)
    for h, i in ties:
        keep[h, i] = False
    assert len(ties) <= 4, ties
    assert_close(host(mo_d)[:, qa][keep], mo[keep], what="mass")
    assert_close(host(uo_d)[:, qa][keep], uo[keep], what="unsel")
