"""GPU parity of the tensor-core dense producer (query tiles; statistics by candidates
and an exact selection) against the oracle's dense attention with statistics.

fl_sparse_loop_attn takes this form for dense calls (sel == NULL) at head_dim 128 over
a quantised store. Cases: the loop-1 shape of the 4K workload (every token queries;
sampled rows checked), ragged tiles, the probability-only statistic, bf16 queries and
outputs, a dense call at a later loop (residual chains in K^ and V^), and rows whose
statistics are exact ties (zero queries: every column equally likely), which overflow
the candidate buffers and are finished by the exact per-query kernel. The output o,
m' and u' must hold max-abs 2e-2 / relative L1 5e-3; the column sets must match up to
near-ties inside a 1e-5 relative band of the k-th statistic (counted)."""
import numpy as np
import pytest
import torch

from cross_loop_sparse_step_b200 import synth
from oracle import attention as oatt
from oracle import kvstore as okv
from tests.gpu_helpers import assert_close, check_selection, dev, host, sel_to_host, upload_store

pytestmark = pytest.mark.gpu


def _store(rs, n, H, hd, g, R=1, counts=None, bits=None):
    ost = okv.LayerKV(n, H, hd, g, 8, bits or {}, R)
    ost.write_base(synth.kv_values(rs, n, H, hd), synth.kv_values(rs, n, H, hd))
    act = np.arange(n, dtype=np.int32)
    for r in range(2, R + 1):
        act = np.sort(rs.choice(act, size=counts[r], replace=False)).astype(np.int32)
        kr = (ost.hat[r - 1][0][act] + 0.3 * rs.normal(size=(len(act), H, hd))).astype(np.float32)
        vr = (ost.hat[r - 1][1][act] + 0.3 * rs.normal(size=(len(act), H, hd))).astype(np.float32)
        ost.write_residual(r, act, kr, vr)
    return ost


def _c_fn(q, q_tok, Kh, Vh, bias, stat):
    def f(h, i):
        t = int(q_tok[i])
        cols = np.arange(t + 1)
        s = Kh[cols, h].astype(np.float64) @ q[i, h] / np.sqrt(q.shape[-1])
        if bias is not None:
            s = s + bias[cols]
        e = np.exp(s - s.max())
        p = e / e.sum()
        if stat == "pv":
            p = p * np.linalg.norm(Vh[cols, h].astype(np.float64), axis=1)
        return dict(zip(cols.tolist(), p.tolist()))
    return f


CASES = [
    # name, n_tok, H, g, loop, k, n_q (None: every token), bias, sample, stat, bf16, zero_q
    ("4k-loop1", 4096, 16, 32, 1, 82, None, True, 64, "pv", True, False),
    ("ragged-1000-g64-statp", 1000, 2, 64, 1, 40, None, False, 120, "p", False, False),
    ("subset-820", 4096, 4, 32, 1, 82, 820, True, 48, "pv", False, False),
    ("loop3-chains", 2048, 4, 32, 3, 64, None, True, 64, "pv", True, False),
    ("uniform-ties-overflow", 2048, 2, 32, 1, 16, None, False, 40, "p", False, True),
]


@pytest.mark.parametrize("name,n,H,g,loop,k,nq,use_bias,sample,stat,bf16,zero_q", CASES,
                         ids=[c[0] for c in CASES])
def test_dense_tile_matches_oracle(name, n, H, g, loop, k, nq, use_bias, sample, stat, bf16,
                                   zero_q):
    from cross_loop_sparse_step_b200 import fl
    hd = 128
    rs = synth.rng(8000 + n + k + loop)
    counts = {r: max(64, n // (2 * r)) for r in range(2, loop + 1)}
    bits = {r: 4 for r in range(2, loop + 1)}
    ost = _store(rs, n, H, hd, g, loop, counts, bits)
    store = fl.KVStore(n, H, hd, g, 8, bits, loop, counts)
    upload_store(ost, store, loop)
    bias = synth.col_bias(rs, n, 0.02, 4.0) if use_bias else None
    q_tok = np.arange(n, dtype=np.int32) if nq is None else synth.sorted_subset(rs, n, nq)
    q = synth.query_values(rs, len(q_tok), H, hd)
    if zero_q:
        q[:] = 0.0
    tdt = torch.bfloat16 if bf16 else torch.float32
    if bf16:
        q = synth.round_bf16(q)
    out = torch.full((len(q_tok), H, hd), float("nan"), dtype=tdt, device="cuda")
    S = torch.full((H, n, k + 1), -1, dtype=torch.int16, device="cuda")
    m = torch.zeros(H, n, device="cuda")
    u = torch.zeros(H, n, hd, device="cuda")
    kind = fl.STAT_PV if stat == "pv" else fl.STAT_P
    fl.sparse_loop_attn(dev(q, tdt), dev(q_tok), store, loop, out,
                        col_bias=dev(bias) if bias is not None else None, k_next=k, sel_out=S,
                        mass_out=m, unsel_out=u, stat_kind=kind)
    st = fl.check_device_status()
    assert st == 0, (fl.status_str(st), fl.last_error_detail())
    pick = np.sort(rs.choice(len(q_tok), size=min(sample, len(q_tok)), replace=False))
    pick = np.unique(np.concatenate([pick, [0, len(q_tok) - 1]]))
    qt = q_tok[pick]
    Kh, Vh = ost.hat[loop]
    qp = q[pick].astype(np.float64)
    o, So, mo, uo = oatt.dense_attention(qp, qt, Kh, Vh, bias, k_sel=k, stat=stat)
    assert_close(host(out.float())[pick], o, what=f"{name}: o")
    Sg = sel_to_host(S)[:, qt]
    ties = check_selection(Sg, So, _c_fn(qp, qt, Kh, Vh, bias, stat))
    keep = np.ones((H, len(pick)), bool)
    for h, i in ties:
        keep[h, i] = False
    assert len(ties) <= max(2, keep.size // 100), ties[:8]
    assert_close(host(m)[:, qt][keep], mo[keep], what=f"{name}: mass")
    assert_close(host(u)[:, qt][keep], uo[keep], what=f"{name}: unselected part")
    if zero_q:   # exact ties: the smallest columns, bit for bit, and no near-tie slack
        assert not ties
        for i, t in enumerate(qt):
            want = np.arange(min(int(t), k) + 1)
            assert np.array_equal(Sg[0, i][: len(want)], want)


def test_dense_tile_without_statistics():
    """Output only (no statistics requested): the flash pass alone."""
    from cross_loop_sparse_step_b200 import fl
    n, H, hd, g = 3000, 4, 128, 32
    rs = synth.rng(8100)
    ost = _store(rs, n, H, hd, g)
    store = fl.KVStore(n, H, hd, g, 8, {}, 1, {})
    upload_store(ost, store, 1)
    bias = synth.col_bias(rs, n, 0.02, 4.0)
    q_tok = np.arange(n, dtype=np.int32)
    q = synth.query_values(rs, n, H, hd)
    out = torch.zeros(n, H, hd, device="cuda")
    fl.sparse_loop_attn(dev(q), dev(q_tok), store, 1, out, col_bias=dev(bias))
    assert fl.check_device_status() == 0
    pick = np.unique(np.concatenate([rs.choice(n, 60, replace=False), [0, 1, 127, 128, n - 1]]))
    o = oatt.dense_attention(q[pick].astype(np.float64), q_tok[pick], *ost.hat[1], bias)
    assert_close(host(out)[pick], o, what="o")
