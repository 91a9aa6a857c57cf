"""Pins of the oracle's loop driver (FlashLoop §1, §4).

* reduction (§4.1: a loop that recomputes every token is the dense loop; §4.2: the
  cached mass keeps the full-softmax scale): with every token active, every column
  selected and quantisation off, the lazy loops equal the dense looped block, which
  is itself checked against an R-fold torch fp64 composition;
* §4.1 / §3.1 invariants: nested active sets of the scheduled sizes, inactive rows
  carried unchanged, inactive tokens reusing the previous loop's K/V;
* §4.3: the KV store rebuilt from its codes equals the running reconstruction, and
  its bytes equal the closed form; the dense-cache arithmetic reproduces the pages'
  48 GiB for the Ouro-2.6B shape (tests/golden/kv_bytes_pages.txt)."""
import os

import numpy as np
import pytest

from cross_loop_sparse_step_b200 import configs, synth
from oracle import loop
from tests.test_oracle_block import _torch_layer

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "kv_bytes_pages.txt")


def _small(seed=0, n=48, d=64, H=4, hd=16, Fd=128, L=2, std=0.1):
    g = synth.rng(seed)
    layers = synth.model_weights(g, L, d, Fd, std=std)
    h0 = synth.embeddings(g, n, d)
    bias = synth.col_bias(g, n, 0.1, 2.0)
    return layers, h0, bias, dict(n=n, d=d, H=H, hd=hd)


def test_full_active_all_columns_no_quant_is_dense_block():
    layers, h0, bias, s = _small()
    n, R = s["n"], 3
    lazy = dict(n_loops=R, first_sparse=2, tok_frac={2: 1.0, 3: 1.0},
                col_k={2: n, 3: n}, base_bits=0, res_bits={2: 0, 3: 0}, group=16)
    dense = dict(lazy, col_k={})
    a = loop.run(layers, h0, lazy, s["H"], s["hd"], bias)
    b = loop.run(layers, h0, dense, s["H"], s["hd"], bias)
    for r in range(1, R + 1):
        assert np.max(np.abs(a["h"][r] - b["h"][r])) < 1e-12
    # the dense looped block against the torch library, applied R times
    x = h0.astype(np.float64)
    for r in range(1, R + 1):
        for layer in layers:
            x = _torch_layer(x, layer, s["H"], s["hd"], bias, kv_f32=True)
        assert np.max(np.abs(b["h"][r] - x)) < 1e-10


def test_lazy_invariants_and_store():
    layers, h0, bias, s = _small(seed=1, n=64)
    n = s["n"]
    sched = dict(n_loops=4, first_sparse=2, tok_frac={2: 0.5, 3: 0.25, 4: 0.2},
                 col_k={2: 8, 3: 6, 4: 4}, base_bits=8, res_bits={2: 4, 3: 2, 4: 4},
                 group=16)
    out = loop.run(layers, h0, sched, s["H"], s["hd"], bias)
    assert list(out["act"][1]) == list(range(n))
    sizes = {2: 32, 3: 16, 4: 13}
    for r in range(2, 5):
        act = out["act"][r]
        assert len(act) == sizes[r]
        assert list(act) == sorted(act)
        assert set(act) <= set(out["act"][r - 1])
        inactive = np.setdiff1d(np.arange(n), act)
        assert np.array_equal(out["h"][r][inactive], out["h"][r - 1][inactive])
        for st in out["stores"]:
            # inactive tokens reuse the previous loop's K/V
            assert np.array_equal(st.hat[r][:, inactive], st.hat[r - 1][:, inactive])
            K, V = st.reconstruct(r, np.arange(n))
            assert np.array_equal(K, st.hat[r][0]) and np.array_equal(V, st.hat[r][1])
        # statistics rows of active queries: sink, sizes, budget of the next loop
        if r < 4:
            S, m, u = out["stats"][r][0]
            k = sched["col_k"][r + 1]
            for t in act:
                sel = S[0, t][S[0, t] != 0xFFFF]
                assert sel[0] == 0 and len(sel) == min(k, t) + 1
                assert 0 < m[0, t] <= 1 + 1e-12
    # stored bytes match the closed form
    d = s["d"]
    per_tok = loop.kv_bytes_per_token(n, d, out["k"], 8, sched["res_bits"], 16)
    held = sum(out["stores"][0].kv_bytes(r) for r in range(1, 5)) / n
    assert per_tok == held


def test_dense_kv_bytes_match_pages():
    with open(GOLDEN) as f:
        for line in f:
            if not line.strip() or line.startswith("#"):
                continue
            lhs, rhs = line.split("|")
            L, R, N, d, elt = (int(v) for v in lhs.split())
            dense = L * R * N * 2 * d * elt
            assert dense == int(rhs) * 2 ** 30


@pytest.mark.parametrize("cfg,want", [(configs.PREFILL_4K, 6144.0), (configs.PREFILL_32K, 4608 + 0.45 * 1536)])
def test_kv_bytes_closed_form_configs(cfg, want):
    n_act = configs.active_counts(cfg)
    got = loop.kv_bytes_per_token(cfg["n_tok"], cfg["d_model"], n_act, cfg["base_bits"],
                                  cfg["res_bits"], cfg["group"])
    assert abs(got - want) < 1e-3 * want   # ceil(f N) rows vs the f N of the estimate
    dense = cfg["n_loops"] * 2 * cfg["d_model"] * 2
    assert dense / got >= 4.0


def test_c1_runs_and_is_reproducible():
    cfg = configs.TINY_FP32
    g = synth.rng(0)
    layers = synth.model_weights(g, cfg["n_layers"], cfg["d_model"], cfg["d_ffn"])
    h0 = synth.embeddings(g, cfg["n_tok"], cfg["d_model"])
    sched = {k: cfg[k] for k in ("n_loops", "first_sparse", "tok_frac", "col_k",
                                 "base_bits", "res_bits", "group")}
    a = loop.run(layers, h0, sched, cfg["n_heads"], cfg["head_dim"])
    assert len(a["act"][2]) == 64
    b = loop.run(layers, h0, sched, cfg["n_heads"], cfg["head_dim"])
    assert np.array_equal(a["h"][4], b["h"][4])


def test_append_equals_full_write():
    """Decode append (§4.3 applied to a generated token): appending a token to loop r
    gives it the same codes and reconstruction as writing loop r with the token among the
    active set, and leaves every other token untouched."""
    from oracle import kvstore
    g = synth.rng(77)
    n, H, hd = 40, 2, 64
    base_k, base_v = synth.kv_values(g, n, H, hd), synth.kv_values(g, n, H, hd)
    act = np.array([3, 9, 17], np.int32)
    new = 39
    rk = (base_k[act] + 0.1 * g.normal(size=(3, H, hd))).astype(np.float32)
    rv = (base_v[act] + 0.1 * g.normal(size=(3, H, hd))).astype(np.float32)
    tk = (base_k[[new]] + 0.1 * g.normal(size=(1, H, hd))).astype(np.float32)
    tv = (base_v[[new]] + 0.1 * g.normal(size=(1, H, hd))).astype(np.float32)
    a = kvstore.LayerKV(n, H, hd, 32, 8, {2: 4}, 2)
    a.write_base(base_k, base_v)
    a.write_residual(2, act, rk, rv)
    a.append(2, [new], tk, tv)
    b = kvstore.LayerKV(n, H, hd, 32, 8, {2: 4}, 2)
    b.write_base(base_k, base_v)
    b.write_residual(2, np.append(act, new), np.concatenate([rk, tk]), np.concatenate([rv, tv]))
    for kv in range(2):
        assert np.array_equal(a.codes[(2, kv)], b.codes[(2, kv)])
        assert np.array_equal(a.hat[2][kv], b.hat[2][kv])
    assert np.array_equal(a.slot, b.slot)
    K, V = a.reconstruct(2, np.arange(n))
    assert np.array_equal(K, a.hat[2][0]) and np.array_equal(V, a.hat[2][1])
