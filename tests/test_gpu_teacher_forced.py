"""Stage-by-stage ("teacher-forced") parity of fl_loop_step on the benchmarked workload.

The loop step runs as the benchmark runs it (all layers, loops 1..R, the fused
projection epilogues, the carried statistics updated in place); inspection taps copy,
for a sample of tokens, every layer's input row, q, k, v, attention output and output
row. Each stage is then compared with the oracle on identical inputs - the GPU's own
rows, active set, carried statistics and KV store - so that the comparison holds at
every depth at the standard tolerance (max-abs 2e-2 and relative L1 5e-3) without
letting differences compound along the chain of layers:

  selection    A_r from the GPU's (h, previous state) rows          bit-exact
  projection   q, k, v of the GPU's layer input rows                 tolerance
  KV codes     the oracle quantiser on the GPU's k, v against the
               GPU store's reconstruction of loop r - 1              bit-exact
  attention    dense (loop 1, statistics for loop 2) or sparse with
               the GPU's carried (S, m, u) over the GPU store        tolerance
  statistics   S' (bit-exact up to counted near-ties), m', u'        tolerance
  layer        output projection + FFN of the GPU's input row and
               attention output                                      tolerance

The oracle runs twice for the float stages: with the bf16 workload's operand
rounding (RMSNorm outputs, attention output and SwiGLU product held as bfloat16, the
workload's dtype) and without any rounding (plain fp64); both must hold the tolerance.
"""
import numpy as np
import pytest
import torch

from cross_loop_sparse_step_b200 import configs, synth
from oracle import attention as oatt
from oracle import block as oblk
from oracle import codec as ocodec
from oracle import select as osel
from tests.gpu_helpers import assert_close, check_selection, dev, host, sel_to_host

pytestmark = pytest.mark.gpu


class HostStore:
    """Host copy of one layer's GPU KV store, decoded with the oracle's codec."""

    def __init__(self, st):
        self.st = st
        self.H, self.hd, self.g = st.H, st.hd, st.g
        self.slot = host(st.slot)
        self.codes = {k: host(v) for k, v in st.codes.items()}
        self.sz = {k: (host(v) if v is not None else None) for k, v in st.sz.items()}

    def bits(self, r):
        return self.st.base_bits if r == 1 else self.st.res_bits[r]

    def decode(self, r, kv, rows):
        b = self.bits(r)
        c = self.codes[(r, kv)][rows]
        if b == 0:
            return c.view(np.float32).reshape(len(rows), self.H, self.hd).copy()
        return ocodec.dequantize(c, self.sz[(r, kv)][rows], b, self.g, self.hd)

    def hat(self, r, tokens):
        """K^_r, V^_r (float32 [n, H, hd]) of ``tokens``: base, then loops 2..r."""
        tokens = np.asarray(tokens, np.int64)
        out = []
        for kv in range(2):
            cur = self.decode(1, kv, tokens)
            for rr in range(2, r + 1):
                sl = self.slot[rr][tokens]
                on = sl >= 0
                if not on.any():
                    continue
                d = self.decode(rr, kv, sl[on])
                if self.bits(rr) == 0:
                    cur[on] = d
                else:
                    cur[on] = (cur[on] + d).astype(np.float32)
            out.append(cur)
        return out


def _quantise(x, bits, g, H, hd):
    """Oracle codes (packed) and (s, z) of x float32 [n, H, hd]."""
    n = x.shape[0]
    c, s, z, _, err = ocodec.quantize_groups(x.reshape(n, H, hd // g, g), bits)
    assert not err.any()
    return ocodec.pack_codes(c.reshape(n, H, hd), bits), np.stack([s, z], axis=-1)


def _f64_layer(w):
    return {k: np.asarray(v, np.float64) for k, v in w.items()}


def _check_float(got, want_bf, want_f64, what):
    assert_close(got, want_bf, what=what + " (bf16 operands)")
    assert_close(got, want_f64, what=what + " (fp64)")


def run_teacher_forced(cfg, R, n_tap=256, n_dense_check=32, seed=0):
    from cross_loop_sparse_step_b200 import fl
    N, d, H, hd, F, L = (cfg[k] for k in ("n_tok", "d_model", "n_heads", "head_dim", "d_ffn",
                                          "n_layers"))
    g = synth.rng(seed)
    layers = synth.model_weights(g, L, d, F, bf16=True)
    h0 = synth.embeddings(g, N, d)
    bias = synth.col_bias(g, N, cfg["bias_frac"], cfg["bias_value"])
    cur, prev, _ = synth.pareto_delta_pair(g, N, d, 2)
    change = (cur - prev).astype(np.float32)
    n_active = configs.active_counts(dict(cfg, n_loops=R))
    wt = [{k: (dev(v, torch.bfloat16) if k.startswith("w_") else dev(v)) for k, v in w.items()}
          for w in layers]
    model = fl.LoopModel(wt, N, H, hd, col_bias=dev(bias))
    res = {r: cfg["res_bits"][r] for r in range(2, R + 1)}
    col_k = {r: cfg["col_k"][r] for r in range(2, R + 1)}
    stores = [fl.KVStore(N, H, hd, cfg["group"], cfg["base_bits"], res, R, n_active)
              for _ in range(L)]
    sched = fl.make_schedule(R, cfg["first_sparse"], n_active, col_k)
    run = fl.LoopRunner(model, sched, n_active, stores, max(col_k.values()) + 1)
    run.h.copy_(dev(h0))
    rs = synth.rng(seed + 99)
    tap_tok = np.sort(rs.choice(N, size=n_tap, replace=False)).astype(np.int32)
    tap_tok[0] = 0                      # the sink's row and an early query
    tap_tok = np.unique(np.concatenate([tap_tok, [1, N - 1]])).astype(np.int32)
    run.set_taps(dev(tap_tok))
    stat_rows = torch.from_numpy(tap_tok.astype(np.int64)).cuda()
    report = {"ties": 0, "checked": {}}

    def stats_of(li):
        return (sel_to_host(run.sel[li][:, stat_rows]), host(run.mass[li][:, stat_rows]),
                host(run.unsel[li][:, stat_rows]))

    prev_act = np.arange(N, dtype=np.int32)
    for r in range(1, R + 1):
        # ---- inputs of the loop as the GPU holds them
        if r == 2:
            run.x_prev.copy_(run.h - dev(change))
        if r >= 2:
            k_prev = n_active[r - 1]
            if r == 2:
                rows_cur, rows_prev = host(run.h), host(run.x_prev)
            else:
                rows_cur = host(run.x_cur[:k_prev])
                rows_prev = host(run.x_prev[:k_prev])
        stats_in = [stats_of(li) for li in range(L)] if r >= 2 else None
        for t in run.taps.values():
            if t.is_floating_point():
                t.fill_(float("nan"))
        run.step(r)
        st = fl.check_device_status()
        assert st == 0, fl.status_str(st)
        taps = {k: host(v.float()) for k, v in run.taps.items() if k != "tok"}
        stats_out = [stats_of(li) for li in range(L)] if r < R else None
        # ---- selection
        if r >= 2:
            act = host(run.act[r])[: n_active[r]]
            want_act, _, _ = osel.select_active(rows_cur, rows_prev,
                                                None if r == 2 else prev_act, n_active[r])
            assert np.array_equal(act, want_act), f"loop {r}: active set"
        else:
            act = np.arange(N, dtype=np.int32)
        prev_act = act
        on = np.isin(tap_tok, act)
        idx = np.flatnonzero(on)
        if r == 1:   # the dense loop: attention and statistics on a sub-sample
            att_idx = np.sort(rs.choice(idx, size=min(n_dense_check, len(idx)), replace=False))
            att_idx = np.unique(np.concatenate([att_idx, idx[:2], idx[-1:]]))
        else:
            att_idx = idx
        toks = tap_tok[idx]
        report["checked"][r] = len(idx)
        assert len(idx) > 0
        kn = col_k.get(r + 1) if r < R else None
        for li in range(L):
            w = _f64_layer(layers[li])
            x_in = taps["x_in"][li][idx].astype(np.float64)
            assert np.all(np.isfinite(x_in)), f"loop {r} layer {li}: untapped rows"
            # projection
            qb, kb, vb = oblk.qkv(x_in, toks, w, H, hd, bf16_ops=True)
            qf, kf, vf = oblk.qkv(x_in, toks, w, H, hd, bf16_ops=False)
            for name, wb, wf in (("q", qb, qf), ("k", kb, kf), ("v", vb, vf)):
                _check_float(taps[name][li][idx], wb.reshape(len(idx), d), wf.reshape(len(idx), d),
                             f"loop {r} layer {li} {name}")
            # KV codes of the GPU's own k and v
            hs = HostStore(stores[li])
            k_g = taps["k"][li][idx].reshape(-1, H, hd).astype(np.float32)
            v_g = taps["v"][li][idx].reshape(-1, H, hd).astype(np.float32)
            bits = hs.bits(r)
            if r == 1:
                rows = toks
                ref = [np.zeros_like(k_g), np.zeros_like(v_g)]
            else:
                rows = hs.slot[r][toks]
                assert np.all(rows >= 0), f"loop {r}: slot of active tokens"
                ref = hs.hat(r - 1, toks)
            for kv, x in enumerate((k_g, v_g)):
                resid = x if r == 1 else (x - ref[kv]).astype(np.float32)
                codes, sz = _quantise(resid, bits, hs.g, H, hd)
                assert np.array_equal(hs.codes[(r, kv)][rows], codes), f"loop {r} layer {li} codes"
                assert np.array_equal(hs.sz[(r, kv)][rows].view(np.uint16), sz.view(np.uint16)), \
                    f"loop {r} layer {li} scale/offset"
            # attention on the GPU's q and store
            a_i = np.searchsorted(idx, att_idx)
            q_g = taps["q"][li][att_idx].reshape(-1, H, hd).astype(np.float64)
            qt = tap_tok[att_idx]
            if r == 1:
                cols = np.arange(int(qt.max()) + 1)
            else:
                S_in = stats_in[li][0][:, att_idx]
                cols = np.unique(S_in[S_in != oatt.SENTINEL]).astype(np.int64)
            Kc, Vc = hs.hat(r, cols)
            Kh = np.zeros((N, H, hd), np.float32)
            Vh = np.zeros((N, H, hd), np.float32)
            Kh[cols], Vh[cols] = Kc, Vc
            if r == 1:
                res_o = oatt.dense_attention(q_g, qt, Kh[: len(cols)], Vh[: len(cols)], bias,
                                             k_sel=kn)
            else:
                S_f = np.full((H, N, stats_in[li][0].shape[2]), oatt.SENTINEL, np.uint16)
                m_f = np.zeros((H, N))
                u_f = np.zeros((H, N, hd))
                S_f[:, qt], m_f[:, qt], u_f[:, qt] = (stats_in[li][0][:, att_idx],
                                                      stats_in[li][1][:, att_idx],
                                                      stats_in[li][2][:, att_idx])
                res_o = oatt.sparse_attention(q_g, qt, qt, Kh, Vh, S_f, m_f, u_f, bias, k_next=kn)
            o = res_o[0] if kn is not None else res_o
            o = o.reshape(len(att_idx), d)
            got_o = taps["attn"][li][att_idx]
            _check_float(got_o, oblk.bf16(o), o, f"loop {r} layer {li} attention")
            if kn is not None:
                _, So, mo, uo = res_o
                Sg = stats_out[li][0][:, att_idx, : kn + 1]

                def cfn(h, i, q_g=q_g, qt=qt, Kh=Kh, Vh=Vh, r=r, li=li):
                    t = int(qt[i])
                    if r == 1:
                        cc = np.arange(t + 1)
                        m_in = 1.0
                    else:
                        row = stats_in[li][0][h, att_idx[i]]
                        cc = row[row != oatt.SENTINEL].astype(np.int64)
                        m_in = float(stats_in[li][1][h, att_idx[i]])
                    s = Kh[cc, h].astype(np.float64) @ q_g[i, h] / np.sqrt(hd) + bias[cc]
                    e = np.exp(s - s.max())
                    p = m_in * e / e.sum()
                    vn = np.linalg.norm(Vh[cc, h].astype(np.float64), axis=1)
                    return dict(zip(cc.tolist(), (p * vn).tolist()))
                ties = check_selection(Sg, So, cfn)
                report["ties"] += len(ties)
                assert len(ties) <= max(2, Sg.shape[0] * Sg.shape[1] // 100), ties[:8]
                keep = np.ones(Sg.shape[:2], bool)
                for h, i in ties:
                    keep[h, i] = False
                assert_close(stats_out[li][1][:, att_idx][keep], mo[keep],
                             what=f"loop {r} layer {li} mass")
                assert_close(stats_out[li][2][:, att_idx][keep], uo[keep],
                             what=f"loop {r} layer {li} unselected part")
            # output projection and FFN of the GPU's input row and attention output
            attn_rows = taps["attn"][li][idx].astype(np.float64)
            yb = oblk.out_ffn(x_in, attn_rows, w, bf16_ops=True)
            yf = oblk.out_ffn(x_in, attn_rows, w, bf16_ops=False)
            _check_float(taps["x_out"][li][idx], yb, yf, f"loop {r} layer {li} output")
            if li + 1 < L:
                assert np.array_equal(taps["x_out"][li][idx], taps["x_in"][li + 1][idx])
        # the scattered state: tapped active rows hold the last layer's output
        h_now = host(run.h)
        assert np.array_equal(h_now[toks], taps["x_out"][L - 1][idx])
    return report


def test_4k_workload_all_layers_all_loops():
    """The benchmarked 4K workload: 24 layers, loops 1..4, every stage of every layer."""
    rep = run_teacher_forced(dict(configs.PREFILL_4K), configs.PREFILL_4K["n_loops"])
    print("teacher-forced 4K:", rep)
    assert all(v > 0 for v in rep["checked"].values())


def test_32k_workload_all_layers_loops_1_2():
    """The 32K Ouro-2.6B-shape workload the benchmark times: all 48 layers, the dense loop 1
    (statistics for loop 2, k = 2048 of up to 32K columns) and the sparse loop 2 over the
    column-range tiles, on a sample of tokens."""
    rep = run_teacher_forced(dict(configs.PREFILL_32K), 2, n_tap=64, n_dense_check=10)
    print("teacher-forced 32K:", rep)
    assert all(v > 0 for v in rep["checked"].values())
