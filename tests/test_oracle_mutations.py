"""Planted mistakes in the oracle (on the CPU) must be caught by its pins.

Each test swaps one oracle step for a plausible slip and re-runs the check that
should notice it: a rounding direction, a transposed weight, a wrong RoPE sign, a
dropped term of the sparse output, a reversed tie rule."""
import numpy as np

from cross_loop_sparse_step_b200 import synth
from oracle import attention, block, codec, select
from tests.test_oracle_block import _torch_layer


def test_offset_rounded_to_nearest_is_caught(monkeypatch):
    monkeypatch.setattr(codec, "f16_rd", lambda x: np.asarray(x, np.float32).astype(np.float16))
    g = np.random.Generator(np.random.PCG64(1))
    x = (g.normal(size=(500, 32)) * 0.3 + 0.1).astype(np.float32)
    _, _, z, _, _ = codec.quantize_groups(x, 4)
    # the property "offset at or below every value" fails for some group
    assert np.any(z.astype(np.float64) > x.min(axis=1))


def test_transposed_projection_is_caught(monkeypatch):
    g = synth.rng(2)
    n, d, H, hd, Fd = 10, 32, 2, 16, 32
    layer = synth.layer_weights(g, d, Fd, std=0.3)
    X = synth.embeddings(g, n, d).astype(np.float64)
    pos = np.arange(n)
    want = _torch_layer(X, layer, H, hd, None)
    bad = dict(layer, w_o=layer["w_o"].T.copy())
    q, k, v = block.qkv(X, pos, bad, H, hd)
    o = attention.dense_attention(q, pos, k, v, None)
    got = block.out_ffn(X, o.reshape(n, d), bad)
    assert np.max(np.abs(got - want)) > 1e-3


def test_rope_sign_slip_is_caught(monkeypatch):
    orig = block.rope

    def bad(x, pos, theta=10000.0):
        return orig(x, -np.asarray(pos), theta)
    from tests.test_oracle_block import _rope_complex
    import torch
    g = np.random.Generator(np.random.PCG64(3))
    x = g.normal(size=(4, 1, 16))
    pos = np.array([1, 5, 9, 200])
    want = _rope_complex(torch.tensor(x), pos).numpy()
    assert np.max(np.abs(bad(x, pos) - want)) > 1e-3


def test_tie_rule_reversed_is_caught():
    cur = np.ones((6, 4))
    prev = np.zeros((6, 4)) + 0.5
    delta = select.normalized_change(cur, prev)
    pos = np.arange(6)
    wrong = np.sort(np.lexsort((-pos, -delta))[:3])   # larger index wins on ties
    right, _, _ = select.select_active(cur, prev, None, 3)
    assert list(wrong) != list(right)
