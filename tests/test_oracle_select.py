"""Pins of the oracle's token selection (FlashLoop §4.1 "Cross-Loop Token-Sparse
Updates"): the normalized change against closed forms, the top-k against a
sort-based brute force with the tie rule, the active counts against an independent
decimal computation, and nesting of the sets."""
import numpy as np

from cross_loop_sparse_step_b200 import configs, synth
from oracle import select


def test_normalized_change_closed_form():
    g = np.random.Generator(np.random.PCG64(31))
    h = g.normal(size=(5, 16))
    # previous = 2 * current: ||h - 2h|| / ||2h|| = 1/2
    assert np.allclose(select.normalized_change(h, 2 * h), 0.5, atol=1e-15)
    # unchanged rows have zero change; a zero previous row divides by the floor
    assert np.all(select.normalized_change(h, h) == 0)
    d = select.normalized_change(np.ones((1, 4)), np.zeros((1, 4)))
    assert d[0] == 2.0 / 1e-30


def test_topk_brute_force_and_ties():
    g = np.random.Generator(np.random.PCG64(32))
    for trial in range(20):
        n = int(g.integers(5, 60))
        k = int(g.integers(0, n + 1))
        cur = g.normal(size=(n, 8))
        prev = cur + g.normal(size=(n, 8)) * g.choice([0.0, 0.1, 1.0], size=(n, 1))
        row_tok = np.sort(g.choice(1000, size=n, replace=False))
        tok, pos, delta = select.select_active(cur, prev, row_tok, k)
        brute = sorted(range(n), key=lambda i: (-delta[i], i))[:k]
        assert list(pos) == sorted(brute)
        assert list(tok) == [int(row_tok[i]) for i in sorted(brute)]
        assert set(tok) <= set(row_tok.tolist())
    # exact ties: identical rows, the smaller index wins
    cur = np.ones((6, 4))
    prev = np.zeros((6, 4)) + 0.5
    tok, pos, _ = select.select_active(cur, prev, None, 3)
    assert list(tok) == [0, 1, 2]


def test_active_counts_agree():
    for cfg in configs.CONFIGS.values():
        if cfg.get("decode"):   # one generated token per sequence: no prompt schedule
            continue
        want = configs.active_counts(cfg)
        prev = cfg["n_tok"]
        for r in range(2, cfg["n_loops"] + 1):
            k = select.active_count(cfg["tok_frac"][r], cfg["n_tok"], prev)
            assert k == want[r], (cfg["name"], r)
            prev = k
    assert configs.active_counts(configs.PREFILL_4K)[2] == 820
    assert configs.active_counts(configs.PREFILL_32K)[2] == 4916
    assert configs.active_counts(configs.TINY_FP32)[2] == 64


def test_pareto_pair_concentrates_change():
    g = synth.rng(0)
    cur, prev, rho = synth.pareto_delta_pair(g, 4096, 256, 2)
    d = select.normalized_change(cur, prev)
    top = np.sort(d)[::-1]
    share = top[: 820].sum() / top.sum()
    assert 0.45 < share < 0.8   # alpha = 1.5 Pareto tail: a heavy top 20%
