"""GPU parity of each C-ABI call against the oracle on identical inputs.

Indices and quantisation codes must be bit-exact; floats within max-abs 2e-2 and
relative L1 5e-3 (gpu_helpers.assert_close). Column selections that the oracle places
within a 1e-5 relative band of the k-th statistic may differ (a near-tie that binary32
and fp64 can break differently); such rows are counted and reported, never silently
skipped. Sizes run from ragged small cases to the full workload shapes (4096 tokens,
16 x 128 heads, 820 active rows)."""
import numpy as np
import pytest
import torch

from cross_loop_sparse_step_b200 import synth
from oracle import attention as oatt
from oracle import block as oblk
from oracle import kvstore as okv
from oracle import select as osel
from tests.gpu_helpers import (assert_close, check_selection, dev, host, sel_to_dev,
                               sel_to_host, upload_store)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from cross_loop_sparse_step_b200 import fl
    assert torch.cuda.is_available()
    yield fl


def _status_ok(fl):
    st = fl.check_device_status()
    assert st == 0, fl.status_str(st)


# ---------------------------------------------------------------- selection
SEL_CASES = [
    # n_rows, d, dtype, k, with row_tok
    (4096, 2048, "bf16", 820, False),   # loop 2 of the 4K workload, full rows
    (4916, 2048, "f32", 4916, True),    # k == n
    (4916, 2048, "f32", 2000, True),    # compact rows of a previous loop
    (1000, 264, "f32", 333, True),      # ragged
    (257, 64, "bf16", 64, False),
    (1, 8, "f32", 1, False),
    (50, 8, "f32", 0, False),
]


@pytest.mark.parametrize("n,d,dt,k,use_tok", SEL_CASES)
def test_select_active_bit_exact(_lib, n, d, dt, k, use_tok):
    fl = _lib
    g = synth.rng(1000 + n + k)
    cur, prev, _ = synth.pareto_delta_pair(g, n, d, 2)
    if dt == "bf16":
        cur, prev = synth.round_bf16(cur), synth.round_bf16(prev)
    row_tok = np.sort(g.choice(max(n * 3, 8), size=n, replace=False)).astype(np.int32) if use_tok else None
    want_tok, want_pos, want_delta = osel.select_active(cur, prev, row_tok, k)
    tdt = torch.bfloat16 if dt == "bf16" else torch.float32
    hc, hp = dev(cur, tdt), dev(prev, tdt)
    rt = dev(row_tok) if use_tok else None
    out_tok = torch.full((max(k, 1),), -7, dtype=torch.int32, device="cuda")
    out_pos = torch.full((max(k, 1),), -7, dtype=torch.int32, device="cuda")
    out_delta = torch.zeros(n, dtype=torch.float32, device="cuda")
    fl.select_active(hc, hp, k, rt, out_tok, out_pos, out_delta)
    _status_ok(fl)
    assert_close(host(out_delta), want_delta, max_abs=1e-4, rel_l1=1e-6, what="delta")
    # the decision margin at the k-th row is far above binary32 rounding
    if 0 < k < n:
        srt = np.sort(want_delta)[::-1]
        assert (srt[k - 1] - srt[k]) / srt[k - 1] > 1e-5
    assert np.array_equal(host(out_tok)[:k], want_tok)
    assert np.array_equal(host(out_pos)[:k], want_pos)


def test_select_ties_smaller_row_wins(_lib):
    fl = _lib
    n, d = 300, 16
    cur = np.ones((n, d), np.float32)
    prev = np.full((n, d), 0.5, np.float32)
    prev[7] = 0.0   # one clearly larger change
    tok = fl.select_active(dev(cur), dev(prev), 5)
    _status_ok(fl)
    assert list(host(tok)) == [0, 1, 2, 3, 7]


# ---------------------------------------------------------------- gather / scatter
@pytest.mark.parametrize("dt", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("n_full,row,n_idx", [(4096, 2048, 820), (37, 3, 11), (5, 6, 5)])
def test_gather_scatter_bit_exact(_lib, dt, n_full, row, n_idx):
    fl = _lib
    g = synth.rng(7)
    src = torch.from_numpy(g.normal(size=(n_full, row)).astype(np.float32)).to(dt).cuda()
    idx = torch.from_numpy(synth.sorted_subset(g, n_full, n_idx)).cuda()
    out = torch.zeros(n_idx, row, dtype=dt, device="cuda")
    fl.gather_scatter(fl.GATHER, src, out, idx, n_full)
    assert torch.equal(out, src[idx.long()])
    dst = torch.zeros(n_full, row, dtype=dt, device="cuda")
    fl.gather_scatter(fl.SCATTER, out, dst, idx, n_full)
    want = torch.zeros_like(dst)
    want[idx.long()] = out
    assert torch.equal(dst, want)
    _status_ok(fl)


def test_gather_out_of_range_is_reported(_lib):
    fl = _lib
    src = torch.ones(4, 8, device="cuda")
    out = torch.zeros(2, 8, device="cuda")
    idx = torch.tensor([1, 9], dtype=torch.int32, device="cuda")
    fl.gather_scatter(fl.GATHER, src, out, idx, 4)
    assert fl.check_device_status() == 6
    assert fl.check_device_status() == 0
    assert torch.equal(out[0], src[1]) and torch.all(out[1] == 0)


# ---------------------------------------------------------------- KV quantisation
QUANT_CASES = [
    # n_tok, H, hd, g, base_bits, res_bits per loop, act sizes, input dtype
    (4096, 16, 128, 32, 8, {2: 4, 3: 2}, {2: 820, 3: 410}, "f32"),
    (4096, 16, 128, 64, 8, {2: 2, 3: 4}, {2: 2048, 3: 205}, "bf16"),
    (256, 4, 64, 32, 8, {2: 4, 3: 4}, {2: 64, 3: 64}, "f32"),
    (97, 3, 64, 64, 8, {2: 8, 3: 2}, {2: 31, 3: 1}, "f32"),
    (64, 2, 128, 32, 0, {2: 0, 3: 4}, {2: 20, 3: 7}, "f32"),
    (64, 2, 64, 32, 8, {2: 0, 3: 2}, {2: 20, 3: 7}, "bf16"),
]


@pytest.mark.parametrize("n,H,hd,g,bb,rb,na,dt", QUANT_CASES)
def test_kv_residual_quant_bit_exact(_lib, n, H, hd, g, bb, rb, na, dt):
    fl = _lib
    rs = synth.rng(n + H + hd + g)
    R = 3
    ost = okv.LayerKV(n, H, hd, g, bb, rb, R)
    store = fl.KVStore(n, H, hd, g, bb, rb, R, {2: na[2], 3: na[3]})
    tdt = torch.bfloat16 if dt == "bf16" else torch.float32
    rnd = synth.round_bf16 if dt == "bf16" else (lambda a: a)
    k1 = rnd(synth.kv_values(rs, n, H, hd, 1.0))
    v1 = rnd(synth.kv_values(rs, n, H, hd, 1.0))
    ost.write_base(k1, v1)
    fl.kv_residual_quant(store, 1, dev(k1, tdt), dev(v1, tdt))
    acts = {1: np.arange(n)}
    ks, vs = {1: k1}, {1: v1}
    for r in (2, 3):
        act = np.sort(rs.choice(acts[r - 1], size=na[r], replace=False)).astype(np.int32)
        acts[r] = act
        kr = rnd((ks[r - 1][act] + 0.5 ** r * rs.normal(size=(na[r], H, hd))).astype(np.float32))
        vr = rnd((vs[r - 1][act] + 0.5 ** r * rs.normal(size=(na[r], H, hd))).astype(np.float32))
        kfull, vfull = ks[r - 1].copy(), vs[r - 1].copy()
        kfull[act], vfull[act] = kr, vr
        ks[r], vs[r] = kfull, vfull
        ost.write_residual(r, act, kr, vr)
        fl.kv_residual_quant(store, r, dev(kr, tdt), dev(vr, tdt), dev(act))
    _status_ok(fl)
    for r in (1, 2, 3):
        rows = n if r == 1 else na[r]
        for kv in range(2):
            want = np.ascontiguousarray(ost.codes[(r, kv)]).view(np.uint8).reshape(rows, H, -1)
            got = host(store.codes[(r, kv)])[:rows]
            assert np.array_equal(got, want), (r, kv, "codes")
            if ost.sz[(r, kv)] is not None:
                assert np.array_equal(host(store.sz[(r, kv)])[:rows].view(np.uint16),
                                      ost.sz[(r, kv)].view(np.uint16)), (r, kv, "scale/offset")
    assert np.array_equal(host(store.slot)[2:], ost.slot[2:])
    vn = np.sqrt((ost.hat[3][1].astype(np.float64) ** 2).sum(-1))
    assert_close(host(store.vnorm), vn, max_abs=1e-4, rel_l1=1e-6, what="vnorm")


def test_quant_range_error_reported(_lib):
    fl = _lib
    n, H, hd = 4, 1, 64
    store = fl.KVStore(n, H, hd, 32, 8, {2: 4}, 2, {2: 1})
    k = torch.zeros(n, H, hd, device="cuda")
    k[0, 0, 0] = -1e6      # offset below the binary16 range
    fl.kv_residual_quant(store, 1, k, torch.zeros_like(k))
    assert fl.check_device_status() == 6


# ---------------------------------------------------------------- attention
def _oracle_store(rs, n, H, hd, g, loops, na, res_bits, scale_r=0.3):
    ost = okv.LayerKV(n, H, hd, g, 8, res_bits, loops)
    k = synth.kv_values(rs, n, H, hd)
    v = synth.kv_values(rs, n, H, hd)
    ost.write_base(k, v)
    act = np.arange(n, dtype=np.int32)
    for r in range(2, loops + 1):
        act = np.sort(rs.choice(act, size=na[r], replace=False)).astype(np.int32)
        kr = (ost.hat[r - 1][0][act] + scale_r ** (r - 1) * rs.normal(size=(len(act), H, hd))).astype(np.float32)
        vr = (ost.hat[r - 1][1][act] + scale_r ** (r - 1) * rs.normal(size=(len(act), H, hd))).astype(np.float32)
        ost.write_residual(r, act, kr, vr)
    return ost, act


def _c_fn(q, t, Kh, Vh, bias, cols_of, pmul=1.0):
    """Oracle statistics c_j = P_j ||V^_j|| of one (query, head) for tie-band checks."""
    def f(h, i):
        cols = cols_of(h, i)
        s = Kh[cols, h].astype(np.float64) @ q[i, h] / np.sqrt(q.shape[-1])
        if bias is not None:
            s = s + bias[cols]
        e = np.exp(s - s.max())
        p = pmul(h, i) * e / e.sum() if callable(pmul) else e / e.sum()
        vn = np.linalg.norm(Vh[cols, h].astype(np.float64), axis=1)
        return dict(zip(cols.tolist(), (p * vn).tolist()))
    return f


ATT_CASES = [
    # n_tok, H, hd, g, k, n_q (None: every token), bias fraction, sample
    (256, 4, 64, 32, 32, None, 0.0, None),
    (300, 2, 128, 64, 16, 77, 0.05, None),
    (4096, 16, 128, 32, 82, 820, 0.02, 48),
]


@pytest.mark.parametrize("n,H,hd,g,k,nq,bf,sample", ATT_CASES)
def test_dense_attention_with_stats(_lib, n, H, hd, g, k, nq, bf, sample):
    fl = _lib
    rs = synth.rng(n + k)
    ost, _ = _oracle_store(rs, n, H, hd, g, 1, {}, {})
    store = fl.KVStore(n, H, hd, g, 8, {}, 1, {})
    upload_store(ost, store, 1)
    bias = synth.col_bias(rs, n, bf, 4.0) if bf else None
    q_tok = np.arange(n, dtype=np.int32) if nq is None else synth.sorted_subset(rs, n, nq)
    q = synth.query_values(rs, len(q_tok), H, hd)
    out = torch.zeros(len(q_tok), H, hd, device="cuda")
    S = torch.full((H, n, k + 1), -1, dtype=torch.int16, device="cuda")
    m = torch.zeros(H, n, device="cuda")
    u = torch.zeros(H, n, hd, device="cuda")
    fl.sparse_loop_attn(dev(q), dev(q_tok), store, 1, out, col_bias=dev(bias) if bias is not None else None,
                        k_next=k, sel_out=S, mass_out=m, unsel_out=u)
    _status_ok(fl)
    pick = np.arange(len(q_tok)) if sample is None else np.sort(rs.choice(len(q_tok), sample, replace=False))
    Kh, Vh = ost.hat[1]
    o, So, mo, uo = oatt.dense_attention(q[pick].astype(np.float64), q_tok[pick], Kh, Vh, bias, k_sel=k)
    assert_close(host(out)[pick], o, what="o")
    Sg = sel_to_host(S)[:, q_tok[pick]]
    ties = check_selection(Sg, So, _c_fn(q[pick].astype(np.float64), None, Kh, Vh, bias,
                                         lambda h, i: np.arange(q_tok[pick][i] + 1)))
    keep = np.ones((H, len(pick)), bool)
    for h, i in ties:
        keep[h, i] = False
    assert len(ties) <= max(2, keep.size // 200), ties
    assert_close(host(m)[:, q_tok[pick]][keep], mo[keep], what="mass")
    assert_close(host(u)[:, q_tok[pick]][keep], uo[keep], what="unsel")


SPARSE_CASES = [
    # n_tok, H, hd, g, loops, k, k_next, act sizes, bias fraction, sample
    (256, 4, 64, 32, 2, 32, 32, {2: 64}, 0.0, None),
    (256, 4, 64, 32, 3, 32, 16, {2: 128, 3: 64}, 0.0, None),
    (512, 2, 128, 32, 4, 40, 8, {2: 200, 3: 100, 4: 37}, 0.05, None),
    (4096, 16, 128, 32, 2, 82, 82, {2: 820}, 0.02, 40),
    (4096, 16, 128, 32, 3, 82, 41, {2: 820, 3: 820}, 0.02, 40),
]


@pytest.mark.parametrize("n,H,hd,g,loops,k,kn,na,bf,sample", SPARSE_CASES)
def test_sparse_loop_attention(_lib, n, H, hd, g, loops, k, kn, na, bf, sample):
    fl = _lib
    rs = synth.rng(n + loops + k + kn)
    rb = {r: 4 for r in range(2, loops + 1)}
    ost, act = _oracle_store(rs, n, H, hd, g, loops, na, rb)
    store = fl.KVStore(n, H, hd, g, 8, rb, loops, na)
    upload_store(ost, store, loops)
    bias = synth.col_bias(rs, n, bf, 4.0) if bf else None
    # statistics carried from a dense previous loop, for every token
    q_prev = synth.query_values(rs, n, H, hd)
    Kp, Vp = ost.hat[loops - 1]
    _, S, m, u = oatt.dense_attention(q_prev.astype(np.float64), np.arange(n), Kp, Vp, bias, k_sel=k)
    q = synth.query_values(rs, len(act), H, hd)
    out = torch.zeros(len(act), H, hd, device="cuda")
    Sd = sel_to_dev(S)
    md = dev(m.astype(np.float32))
    ud = dev(u.astype(np.float32))
    So_d = torch.full((H, n, kn + 1), -1, dtype=torch.int16, device="cuda")
    mo_d = torch.zeros(H, n, device="cuda")
    uo_d = torch.zeros(H, n, hd, device="cuda")
    fl.sparse_loop_attn(dev(q), dev(act), store, loops, out,
                        col_bias=dev(bias) if bias is not None else None,
                        sel=Sd, mass=md, unsel=ud, k_next=kn, sel_out=So_d, mass_out=mo_d,
                        unsel_out=uo_d)
    _status_ok(fl)
    pick = np.arange(len(act)) if sample is None else np.sort(rs.choice(len(act), sample, replace=False))
    Kh, Vh = ost.hat[loops]
    m32 = m.astype(np.float32).astype(np.float64)
    u32 = u.astype(np.float32).astype(np.float64)
    o, So, mo, uo = oatt.sparse_attention(q[pick].astype(np.float64), act[pick], act[pick], Kh, Vh,
                                          S, m32, u32, bias, k_next=kn)
    assert_close(host(out)[pick], o, what="o")
    Sg = sel_to_host(So_d)[:, act[pick]]

    def cols_of(h, i):
        row = S[h, act[pick][i]]
        return row[row != oatt.SENTINEL].astype(np.int64)
    ties = check_selection(Sg, So, _c_fn(q[pick].astype(np.float64), None, Kh, Vh, bias, cols_of,
                                         pmul=lambda h, i: m32[h, act[pick][i]]))
    keep = np.ones((H, len(pick)), bool)
    for h, i in ties:
        keep[h, i] = False
    assert len(ties) <= max(2, keep.size // 200), ties
    assert_close(host(mo_d)[:, act[pick]][keep], mo[keep], what="mass")
    assert_close(host(uo_d)[:, act[pick]][keep], uo[keep], what="unsel")
    if kn >= k:   # unchanged budget: statistics carried bit for bit
        assert np.array_equal(Sg, S[:, act[pick]])
        assert np.array_equal(host(mo_d)[:, act[pick]], m.astype(np.float32)[:, act[pick]])


def test_sparse_attention_in_place_statistics(_lib):
    fl = _lib
    n, H, hd, g, k, kn = 128, 2, 64, 32, 16, 4
    rs = synth.rng(99)
    ost, act = _oracle_store(rs, n, H, hd, g, 2, {2: 40}, {2: 4})
    store = fl.KVStore(n, H, hd, g, 8, {2: 4}, 2, {2: 40})
    upload_store(ost, store, 2)
    q_prev = synth.query_values(rs, n, H, hd)
    _, S, m, u = oatt.dense_attention(q_prev.astype(np.float64), np.arange(n), *ost.hat[1], None, k_sel=k)
    q = synth.query_values(rs, len(act), H, hd)
    Sd, md, ud = sel_to_dev(S), dev(m.astype(np.float32)), dev(u.astype(np.float32))
    out = torch.zeros(len(act), H, hd, device="cuda")
    fl.sparse_loop_attn(dev(q), dev(act), store, 2, out, sel=Sd, mass=md, unsel=ud, k_next=kn,
                        sel_out=Sd, mass_out=md, unsel_out=ud)
    _status_ok(fl)
    o, So, mo, uo = oatt.sparse_attention(q.astype(np.float64), act, act, *ost.hat[2],
                                          S, m.astype(np.float32), u.astype(np.float32), None, k_next=kn)
    assert_close(host(out), o, what="o")
    Sg = sel_to_host(Sd)[:, act, : kn + 1]
    assert np.array_equal(Sg, So)
    assert np.all(sel_to_host(Sd)[:, act, kn + 1:] == oatt.SENTINEL)
    assert_close(host(md)[:, act], mo, what="mass")
    assert_close(host(ud)[:, act], uo, what="unsel")


# ---------------------------------------------------------------- block
BLOCK_CASES = [
    # n_rows, d, H, hd, F, dtype
    (64, 256, 4, 64, 1024, "f32"),
    (77, 256, 2, 128, 512, "f32"),
    (820, 2048, 16, 128, 5632, "bf16"),
    (131, 2048, 16, 128, 5632, "bf16"),
    (1, 256, 2, 128, 512, "bf16"),       # a single row: one ragged 128-row tile
    (128, 256, 2, 128, 512, "bf16"),     # exactly one tile
    (129, 256, 2, 128, 512, "bf16"),     # one row into the next tile
    (4096, 2048, 16, 128, 5632, "bf16"), # every token (loop 1)
    (820, 2048, 16, 128, 5632, "bf16"),  # active rows: tiles cut between CTAs (stream-K)
    (300, 1024, 8, 128, 1536, "bf16"),   # ragged rows, three tile rows cut across CTAs
]


def _weights(rs, d, F, bf16):
    w = synth.layer_weights(rs, d, F, bf16=bf16)
    tdt = torch.bfloat16 if bf16 else torch.float32
    wt = {k: (dev(v, tdt) if k.startswith("w_") else dev(v)) for k, v in w.items()}
    return w, wt


@pytest.mark.parametrize("n,d,H,hd,F,dt", BLOCK_CASES)
def test_block_qkv_and_out_ffn(_lib, n, d, H, hd, F, dt):
    fl = _lib
    rs = synth.rng(n + d)
    bf16 = dt == "bf16"
    w, wt = _weights(rs, d, F, bf16)
    n_tok = 4096
    model = fl.LoopModel([wt], n_tok, H, hd)
    X = synth.embeddings(rs, n, d)
    pos = synth.sorted_subset(rs, n_tok, n)
    q = torch.zeros(n, H, hd, device="cuda")
    k = torch.zeros_like(q)
    v = torch.zeros_like(q)
    ws = torch.empty(model.block_ws_bytes(n), dtype=torch.uint8, device="cuda")
    fl.block_qkv(model, 0, dev(X), dev(pos), q, k, v, ws)
    qo, ko, vo = oblk.qkv(X, pos, w, H, hd)
    assert_close(host(q), qo, what="q")
    assert_close(host(k), ko, what="k")
    assert_close(host(v), vo, what="v")
    attn = synth.query_values(rs, n, H, hd).reshape(n, d)
    if bf16:
        attn = synth.round_bf16(attn)
    x = dev(X)
    fl.block_out_ffn(model, 0, x, dev(attn, torch.bfloat16 if bf16 else torch.float32), ws)
    _status_ok(fl)
    want = oblk.out_ffn(X, attn, w)
    assert_close(host(x), want, what="x")


# ------------------------------------------- KV update fused into the projection
FUSED_CASES = [
    # n_tok, d, H, hd, F, residual bits, active rows per loop
    (4096, 2048, 16, 128, 5632, {2: 4, 3: 4}, {2: 820, 3: 656}),   # the 4K workload's layer
    (1000, 256, 4, 64, 512, {2: 2, 3: 8}, {2: 333, 3: 1}),          # ragged, one-row tail
    (129, 512, 4, 128, 512, {2: 8, 3: 2}, {2: 129, 3: 64}),          # every token active
]


@pytest.mark.parametrize("n_tok,d,H,hd,F,rb,na", FUSED_CASES)
def test_block_qkv_fused_kv_update_bit_exact(_lib, n_tok, d, H, hd, F, rb, na):
    """Codes, scale/offset pairs and slots written by the projection epilogue equal the
    oracle store's for the k and v the same call returns; q, k, v match the oracle."""
    fl = _lib
    rs = synth.rng(n_tok + d + hd)
    w, wt = _weights(rs, d, F, True)
    model = fl.LoopModel([wt], n_tok, H, hd)
    R = 3
    ost = okv.LayerKV(n_tok, H, hd, 32, 8, rb, R)
    store = fl.KVStore(n_tok, H, hd, 32, 8, rb, R, na)
    ws = torch.empty(model.block_ws_bytes(n_tok), dtype=torch.uint8, device="cuda")
    act = np.arange(n_tok, dtype=np.int32)
    for r in range(1, R + 1):
        if r >= 2:
            act = np.sort(rs.choice(act, size=na[r], replace=False)).astype(np.int32)
        X = synth.embeddings(rs, len(act), d)
        q = torch.zeros(len(act), H, hd, device="cuda")
        k, v = torch.zeros_like(q), torch.zeros_like(q)
        fl.block_qkv_kv(model, 0, store, r, dev(X), dev(act), q, ws, k=k, v=v)
        _status_ok(fl)
        qo, ko, vo = oblk.qkv(X, act, w, H, hd)
        assert_close(host(q), qo, what=f"q loop {r}")
        assert_close(host(k), ko, what=f"k loop {r}")
        assert_close(host(v), vo, what=f"v loop {r}")
        kh, vh = host(k), host(v)
        if r == 1:
            ost.write_base(kh, vh)
        else:
            ost.write_residual(r, act, kh, vh)
        rows = len(act)
        for kv in range(2):
            want = np.ascontiguousarray(ost.codes[(r, kv)]).view(np.uint8).reshape(rows, H, -1)
            assert np.array_equal(host(store.codes[(r, kv)])[:rows], want), (r, kv, "codes")
            assert np.array_equal(host(store.sz[(r, kv)])[:rows].view(np.uint16),
                                  ost.sz[(r, kv)].view(np.uint16)), (r, kv, "scale/offset")
        assert np.array_equal(host(store.slot)[1:r + 1], ost.slot[1:r + 1]), (r, "slots")
        vn = np.sqrt((ost.hat[r][1].astype(np.float64) ** 2).sum(-1))
        assert_close(host(store.vnorm), vn, max_abs=1e-4, rel_l1=1e-6, what=f"vnorm loop {r}")
    assert not ost.range_error


def test_block_qkv_fused_rejects_unsupported_store(_lib):
    """A store the epilogue cannot write (group 64) is refused, not silently split."""
    fl = _lib
    rs = synth.rng(7)
    w, wt = _weights(rs, 256, 512, True)
    model = fl.LoopModel([wt], 64, 2, 128)
    store = fl.KVStore(64, 2, 128, 64, 8, {2: 4}, 2, {2: 8})
    ws = torch.empty(model.block_ws_bytes(64), dtype=torch.uint8, device="cuda")
    q = torch.zeros(64, 2, 128, device="cuda")
    with pytest.raises(fl.FLError, match="unsupported"):
        fl.block_qkv_kv(model, 0, store, 1, dev(synth.embeddings(rs, 64, 256)),
                        dev(np.arange(64, dtype=np.int32)), q, ws)
