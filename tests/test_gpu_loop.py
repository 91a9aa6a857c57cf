"""End-to-end parity of fl_loop_step against the oracle's loop driver.

* the tiny fp32 looped block over R = 4 loops (and its shrinking-budget variant):
  active sets bit-exact, hidden states, carried statistics and the dequantised KV
  store within tolerance after every loop;
* the 4K-token Ouro-1.4B shape (d 2048, 16 x 128 heads, FFN 5632) in binary32 with
  two layers over two loops, free-running: loop-2 selection bit-exact, sampled rows of
  h_2 within tolerance;
* the full 24-layer 4K workload in the configuration the benchmark times: the
  invariants of the method (nested sets of the scheduled size, inactive rows and
  their KV untouched, carried column sets valid, KV bytes equal to the closed form)."""
import numpy as np
import pytest
import torch

from cross_loop_sparse_step_b200 import configs, synth
from oracle import attention as oatt
from oracle import codec as ocodec
from oracle import loop as oloop
from tests.gpu_helpers import assert_close, dev, host, sel_to_host

pytestmark = pytest.mark.gpu


def _sched_dict(cfg):
    return {k: cfg[k] for k in ("n_loops", "first_sparse", "tok_frac", "col_k", "base_bits",
                                "res_bits", "group")}


def _gpu_setup(fl, cfg, layers, n_layers=None):
    N, H, hd = cfg["n_tok"], cfg["n_heads"], cfg["head_dim"]
    bf16 = cfg["dtype"] == "bf16"
    tdt = torch.bfloat16 if bf16 else torch.float32
    wt = [{k: (dev(v, tdt) if k.startswith("w_") else dev(v)) for k, v in w.items()}
          for w in layers]
    return wt


def _decode_hat(store, r, H, hd, g, N):
    """Dequantise the GPU store of loop r's chain for every token (oracle codec decode)."""
    slot = host(store.slot)
    out = []
    for kv in range(2):
        bits = store.base_bits
        codes = host(store.codes[(1, kv)])
        if bits == 0:
            cur = codes.view(np.float32).reshape(N, H, hd).copy()
        else:
            cur = ocodec.dequantize(codes, host(store.sz[(1, kv)]), bits, g, hd)
        for rr in range(2, r + 1):
            sl = slot[rr]
            on = sl >= 0
            if not on.any():
                continue
            b = store.res_bits[rr]
            c = host(store.codes[(rr, kv)])[sl[on]]
            if b == 0:
                d = c.view(np.float32).reshape(-1, H, hd)
                cur[on] = d
            else:
                d = ocodec.dequantize(c, host(store.sz[(rr, kv)])[sl[on]], b, g, hd)
                cur[on] = (cur[on] + d).astype(np.float32)
        out.append(cur)
    return out


@pytest.mark.parametrize("cfg", [configs.TINY_FP32, configs.TINY_FP32_SHRINK], ids=["c1", "c1-shrink"])
def test_tiny_block_end_to_end(cfg):
    from cross_loop_sparse_step_b200 import fl
    N, d, H, hd, F, L, R = (cfg[k] for k in ("n_tok", "d_model", "n_heads", "head_dim", "d_ffn",
                                              "n_layers", "n_loops"))
    g = synth.rng(0)
    layers = synth.model_weights(g, L, d, F)
    h0 = synth.embeddings(g, N, d)
    want = oloop.run(layers, h0, _sched_dict(cfg), H, hd)
    n_active = configs.active_counts(cfg)
    wt = _gpu_setup(fl, cfg, layers)
    model = fl.LoopModel(wt, N, H, hd)
    stores = [fl.KVStore(N, H, hd, cfg["group"], cfg["base_bits"], cfg["res_bits"], R, n_active)
              for _ in range(L)]
    sched = fl.make_schedule(R, cfg["first_sparse"], n_active, cfg["col_k"])
    kmax = max(cfg["col_k"].values())
    run = fl.LoopRunner(model, sched, n_active, stores, kmax + 1)
    run.h.copy_(dev(h0))
    for r in range(1, R + 1):
        run.step(r)
        st = fl.check_device_status()
        assert st == 0, fl.status_str(st)
        if r >= 2:
            got_act = host(run.act[r])[: n_active[r]]
            assert np.array_equal(got_act, want["act"][r]), f"loop {r} active set"
        assert_close(host(run.h), want["h"][r], what=f"h_{r}")
        for li in range(L):
            Kg, Vg = _decode_hat(stores[li], r, H, hd, cfg["group"], N)
            Ko, Vo = want["stores"][li].hat[r]
            assert_close(Kg, Ko, what=f"K^_{r}")
            assert_close(Vg, Vo, what=f"V^_{r}")
            if r < R:
                S, m, u = want["stats"][r][li]
                act = want["act"][r] if r >= 2 else np.arange(N)
                kn = cfg["col_k"][r + 1]
                Sg = sel_to_host(run.sel[li])[:, act, : kn + 1]
                So = S[:, act]
                diff = np.argwhere(np.any(Sg != So, axis=-1))
                assert len(diff) <= max(2, Sg.shape[0] * Sg.shape[1] // 100), diff[:10]
                same = np.all(Sg == So, axis=-1)
                assert_close(host(run.mass[li])[:, act][same], m[:, act][same], what="mass")
                assert_close(host(run.unsel[li])[:, act][same], u[:, act][same], what="unsel")


def _c2_like(n_layers):
    cfg = dict(configs.PREFILL_4K)
    cfg["n_layers"] = n_layers
    return cfg


def test_4k_shape_two_layers_two_loops_fp32():
    """Full 4K shape in binary32, two layers, loops 1 and 2, free-running against the
    oracle's own chain: loop-2 selection bit-exact, h_1 and sampled rows of h_2 within
    the standard tolerance. (The bf16 workload is checked stage by stage on identical
    inputs in test_gpu_teacher_forced.)"""
    dtype = "f32"
    from cross_loop_sparse_step_b200 import fl
    cfg = _c2_like(2)
    cfg["n_loops"] = 2
    cfg["dtype"] = dtype
    bf16 = False
    N, d, H, hd, F, L = (cfg[k] for k in ("n_tok", "d_model", "n_heads", "head_dim", "d_ffn",
                                          "n_layers"))
    g = synth.rng(0)
    layers = synth.model_weights(g, L, d, F, bf16=bf16)
    h0 = synth.embeddings(g, N, d)
    bias = synth.col_bias(g, N, cfg["bias_frac"], cfg["bias_value"])
    cur, prev, _ = synth.pareto_delta_pair(g, N, d, 2)
    n_active = configs.active_counts(cfg)
    wt = _gpu_setup(fl, cfg, layers)
    model = fl.LoopModel(wt, N, H, hd, col_bias=dev(bias))
    res = {2: cfg["res_bits"][2]}
    stores = [fl.KVStore(N, H, hd, cfg["group"], 8, res, 2, n_active) for _ in range(L)]
    sched = fl.make_schedule(2, 2, n_active, {2: cfg["col_k"][2]})
    run = fl.LoopRunner(model, sched, n_active, stores, cfg["col_k"][2] + 1)
    run.h.copy_(dev(h0))
    run.step(1)
    assert fl.check_device_status() == 0
    h1_gpu = host(run.h).copy()
    # synthetic previous state for the ranking: h_1 minus a heavy-tailed change; the
    # oracle receives the same change array (drawn on the host, not by the GPU)
    delta = (cur - prev).astype(np.float32)
    run.x_prev.copy_(run.h - dev(delta))
    run.step(2)
    assert fl.check_device_status() == 0
    sched_o = dict(n_loops=2, first_sparse=2, tok_frac={2: cfg["tok_frac"][2]},
                   col_k={2: cfg["col_k"][2]}, base_bits=8, res_bits=res, group=cfg["group"])
    # the oracle's own loop 1, then its loop 2 ranking with the same synthetic change
    want = oloop.run(layers, h0, sched_o, H, hd, bias,
                     select_prev={2: lambda rows: rows - delta.astype(np.float64)},
                     bf16_ops=bf16)
    assert_close(h1_gpu, want["h"][1], what="h_1")
    assert np.array_equal(host(run.act[2]), want["act"][2])
    h2 = host(run.h)
    rs = synth.rng(5)
    rows = np.concatenate([rs.choice(want["act"][2], 64, replace=False),
                           rs.choice(np.setdiff1d(np.arange(N), want["act"][2]), 16, replace=False)])
    assert_close(h2[rows], want["h"][2][rows], what="h_2 sampled rows")


def test_4k_workload_24_layers_invariants():
    """The benchmark's launch configuration: 24 layers, loops 1..3 with the lazy updates."""
    from cross_loop_sparse_step_b200 import fl
    cfg = dict(configs.PREFILL_4K)
    R = 3
    N, d, H, hd, F, L = (cfg[k] for k in ("n_tok", "d_model", "n_heads", "head_dim", "d_ffn",
                                          "n_layers"))
    torch.manual_seed(0)
    wt = [{"w_qkv": (torch.randn(3 * d, d, device="cuda") * 0.02).bfloat16(),
           "w_o": (torch.randn(d, d, device="cuda") * 0.02).bfloat16(),
           "w_gate_up": (torch.randn(2 * F, d, device="cuda") * 0.02).bfloat16(),
           "w_down": (torch.randn(d, F, device="cuda") * 0.02).bfloat16(),
           "g_attn": torch.ones(d, device="cuda"), "g_ffn": torch.ones(d, device="cuda")}
          for _ in range(L)]
    g = synth.rng(0)
    bias = synth.col_bias(g, N, cfg["bias_frac"], cfg["bias_value"])
    n_active = configs.active_counts(cfg)
    model = fl.LoopModel(wt, N, H, hd, col_bias=dev(bias))
    res = {r: cfg["res_bits"][r] for r in range(2, R + 1)}
    stores = [fl.KVStore(N, H, hd, cfg["group"], 8, res, R, n_active) for _ in range(L)]
    colk = {r: cfg["col_k"][r] for r in range(2, R + 1)}
    sched = fl.make_schedule(R, 2, n_active, colk)
    k = colk[2]
    run = fl.LoopRunner(model, sched, n_active, stores, fl.stat_stride(k))
    run.h.copy_(dev(synth.embeddings(g, N, d)))
    p0 = fl.attn_path_counts()
    run.step(1)
    p1 = fl.attn_path_counts()
    # loop 1: every layer's dense attention on the tensor-core producer
    assert p1["dense-tile"] - p0["dense-tile"] == L, (p0, p1)
    cur, prev, _ = synth.pareto_delta_pair(g, N, d, 2)
    run.x_prev.copy_(run.h - dev((cur - prev).astype(np.float32)))
    for r in range(2, R + 1):
        h_before = host(run.h).copy()
        kv_before = [host(s.codes[(1, 0)]).copy() for s in stores[:2]]
        p0 = fl.attn_path_counts()
        run.step(r)
        p1 = fl.attn_path_counts()
        assert fl.check_device_status() == 0
        # a sparse loop: every layer on the query-tile kernel over staged rows
        tiles = sum(p1[x] - p0[x] for x in ("tile-column-ranges", "tile-union"))
        assert tiles == L and sum(p1.values()) - sum(p0.values()) == L, (r, p0, p1)
        act = host(run.act[r])
        assert len(act) == n_active[r] == 820
        assert np.all(np.diff(act) > 0) and act.min() >= 0 and act.max() < N
        if r > 2:
            assert set(act) <= set(host(run.act[r - 1]).tolist())
        h_after = host(run.h)
        assert np.all(np.isfinite(h_after))
        inactive = np.setdiff1d(np.arange(N), act)
        assert np.array_equal(h_after[inactive], h_before[inactive])
        assert not np.array_equal(h_after[act], h_before[act])
        for li, s in enumerate(stores[:2]):
            assert np.array_equal(host(s.codes[(1, 0)]), kv_before[li])   # base untouched
            slot = host(s.slot)[r]
            assert np.array_equal(np.flatnonzero(slot >= 0), act)
            assert np.array_equal(slot[act], np.arange(len(act)))
            S = sel_to_host(run.sel[li])[:, act]
            assert np.all(S[:, :, 0] == 0)
            valid = S != oatt.SENTINEL
            assert np.all(valid.sum(-1) == np.minimum(k, act)[None, :] + 1)
            for h in (0, 7):
                for i in (0, len(act) // 2, len(act) - 1):
                    row = S[h, i][valid[h, i]].astype(np.int64)
                    assert np.all(np.diff(row) > 0) and row[-1] <= act[i]
            m = host(run.mass[li])[:, act]
            assert np.all((m > 0) & (m <= 1.0 + 1e-5))
    kv_bytes = sum(s.nbytes(r) for s in stores for r in range(1, R + 1)) / (N * L)
    want = oloop.kv_bytes_per_token(N, d, {r: n_active[r] for r in range(2, R + 1)}, 8, res, cfg["group"])
    assert kv_bytes == want
