"""Pins of the oracle's shared block (RMSNorm, RoPE, projections, SwiGLU FFN).

The block is checked against torch's fp64 library routines (rms_norm, linear,
scaled_dot_product_attention, silu) with RoPE written as complex multiplication,
a different formulation from the oracle's rotate-half; and against closed forms:
RoPE at position 0 is the identity and preserves norms, the q.k product under RoPE
depends only on the position difference, RMSNorm of a constant row."""
import numpy as np
import torch
import torch.nn.functional as F

from cross_loop_sparse_step_b200 import synth
from oracle import attention, block


def _rope_complex(x, pos, theta=10000.0):
    """RoPE as complex rotation: pair (i, i + hd/2) is the complex number
    x_i + 1j * x_{i+hd/2}, multiplied by exp(1j * pos * theta^(-2i/hd))."""
    n, H, hd = x.shape
    half = hd // 2
    z = torch.complex(x[..., :half], x[..., half:])
    freq = theta ** (-torch.arange(half, dtype=torch.float64) * 2 / hd)
    rot = torch.polar(torch.ones(n, half, dtype=torch.float64),
                      torch.tensor(pos, dtype=torch.float64)[:, None] * freq[None])
    z = z * rot[:, None, :]
    return torch.cat([z.real, z.imag], dim=-1)


def _torch_layer(X, layer, H, hd, bias, kv_f32=False):
    """One dense layer from torch fp64 routines; ``kv_f32`` rounds k and v to
    binary32 where the KV store would hold them."""
    X = torch.tensor(X, dtype=torch.float64)
    n, d = X.shape
    W = {k: torch.tensor(v, dtype=torch.float64) for k, v in layer.items()}
    a = F.rms_norm(X, (d,), W["g_attn"], eps=1e-6)
    qkv = F.linear(a, W["w_qkv"])
    q, k, v = qkv.split(d, dim=1)
    pos = np.arange(n)
    q = _rope_complex(q.reshape(n, H, hd), pos)
    k = _rope_complex(k.reshape(n, H, hd), pos)
    v = v.reshape(n, H, hd)
    if kv_f32:
        k = k.to(torch.float32).to(torch.float64)
        v = v.to(torch.float32).to(torch.float64)
    mask = torch.full((n, n), float("-inf"), dtype=torch.float64).triu(1)
    if bias is not None:
        mask = mask + torch.tensor(bias, dtype=torch.float64)[None, :]
    o = F.scaled_dot_product_attention(q.permute(1, 0, 2)[None], k.permute(1, 0, 2)[None],
                                       v.permute(1, 0, 2)[None], attn_mask=mask)
    o = o[0].permute(1, 0, 2).reshape(n, d)
    y = X + F.linear(o, W["w_o"])
    a2 = F.rms_norm(y, (d,), W["g_ffn"], eps=1e-6)
    gate, up = F.linear(a2, W["w_gate_up"]).chunk(2, dim=1)
    return (y + F.linear(F.silu(gate) * up, W["w_down"])).numpy()


def test_layer_matches_torch_library():
    g = synth.rng(21)
    n, d, H, hd, Fd = 20, 64, 4, 16, 96
    layer = synth.layer_weights(g, d, Fd, std=0.2)
    layer["g_attn"] = (1 + 0.1 * g.normal(size=d)).astype(np.float32)
    layer["g_ffn"] = (1 + 0.1 * g.normal(size=d)).astype(np.float32)
    X = synth.embeddings(g, n, d).astype(np.float64)
    bias = (g.normal(size=n)).astype(np.float32)
    pos = np.arange(n)
    q, k, v = block.qkv(X, pos, layer, H, hd)
    o = attention.dense_attention(q, pos, k.astype(np.float64), v.astype(np.float64), bias)
    got = block.out_ffn(X, o.reshape(n, d), layer)
    want = _torch_layer(X, layer, H, hd, bias)
    assert np.max(np.abs(got - want)) < 1e-11


def test_rope_properties():
    g = np.random.Generator(np.random.PCG64(22))
    x = g.normal(size=(6, 3, 32))
    assert np.array_equal(block.rope(x, np.zeros(6)), x)
    y = block.rope(x, np.arange(6) * 37)
    assert np.allclose(np.linalg.norm(y, axis=-1), np.linalg.norm(x, axis=-1), atol=1e-12)
    # relative position: <R(m) q, R(n) k> depends only on m - n
    q = g.normal(size=(1, 1, 32))
    k = g.normal(size=(1, 1, 32))
    a = np.sum(block.rope(q, [10]) * block.rope(k, [3]))
    b = np.sum(block.rope(q, [107]) * block.rope(k, [100]))
    assert abs(a - b) < 1e-11


def test_rope_matches_complex_form():
    g = np.random.Generator(np.random.PCG64(23))
    x = g.normal(size=(9, 2, 64))
    pos = g.integers(0, 40000, size=9)
    want = _rope_complex(torch.tensor(x), pos).numpy()
    assert np.max(np.abs(block.rope(x, pos) - want)) < 1e-10


def test_rmsnorm_constant_row():
    x = np.full((3, 8), -2.5)
    gam = np.arange(1, 9, dtype=np.float64)
    y = block.rmsnorm(x, gam)
    assert np.allclose(y, -2.5 / np.sqrt(6.25 + 1e-6) * gam, rtol=0, atol=1e-15)


def test_silu_closed_form():
    assert block.silu(np.array(0.0)) == 0.0
    assert abs(block.silu(np.array(1.0)) - 1 / (1 + np.exp(-1))) < 1e-16


def test_bf16_operand_rounding():
    """bf16 operand rounding: representable values unchanged, ties to even, and the
    same as torch's float32 -> bfloat16 conversion (a library routine)."""
    x = np.array([1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, 1.0 + 2 ** -9, -3.5, 0.0])
    y = block.bf16(x)
    assert y[0] == 1.0 and y[4] == -3.5 and y[5] == 0.0
    assert y[1] == 1.0            # exact tie 1 + 2^-8 rounds to even (1.0)
    assert y[2] == 1.0 + 2 ** -6  # tie 1 + 3*2^-8 rounds to even (1 + 2^-6)
    assert y[3] == 1.0            # below half an ulp
    g = np.random.Generator(np.random.PCG64(24))
    z = g.normal(size=1000) * 10
    want = torch.tensor(z, dtype=torch.float32).to(torch.bfloat16).to(torch.float64).numpy()
    assert np.array_equal(block.bf16(z.astype(np.float32).astype(np.float64)), want)


def test_bf16_operands_change_only_by_rounding():
    g = synth.rng(25)
    n, d, H, hd, Fd = 12, 64, 4, 16, 96
    layer = synth.layer_weights(g, d, Fd, std=0.2, bf16=True)
    X = synth.embeddings(g, n, d).astype(np.float64)
    a = block.qkv(X, np.arange(n), layer, H, hd)
    b = block.qkv(X, np.arange(n), layer, H, hd, bf16_ops=True)
    for u, v in zip(a, b):
        assert 0 < np.max(np.abs(u - v)) < 2e-2
