"""The shared Transformer block, in fp64 (oracle; test infrastructure only).

Pages: FlashLoop §1 (a looped Transformer applies one shared N-layer block R times,
R x N block executions, a distinct KV per iteration). The pages do not describe the
block itself; the reading taken is a standard pre-norm decoder layer:
  x <- x + Attn(RMSNorm(x)) . W_o
  x <- x + (silu(RMSNorm(x) W_gate) * (RMSNorm(x) W_up)) W_down
  RMSNorm(x) = x / sqrt(mean(x^2) + eps) * gamma,  eps = 1e-6
  RoPE: theta = 10000, rotate-half pairs (i, i + hd/2), position = token index.
No biases, no final norm, no LM head.

Weights are stored like linear-layer weights, [out_features, in_features]:
  w_qkv [3d, d] (rows: q, then k, then v), w_o [d, d],
  w_gate_up [2F, d] (rows: gate, then up), w_down [d, F].
"""
import numpy as np


def rmsnorm(x, gamma, eps=1e-6):
    x = np.asarray(x, np.float64)
    ms = np.mean(x * x, axis=-1, keepdims=True)
    return x / np.sqrt(ms + eps) * np.asarray(gamma, np.float64)


def rope(x, pos, theta=10000.0):
    """x [n, H, hd], pos [n] -> rotated copy (rotate-half pairing)."""
    x = np.asarray(x, np.float64)
    n, H, hd = x.shape
    half = hd // 2
    i = np.arange(half, dtype=np.float64)
    inv_freq = theta ** (-2.0 * i / hd)
    ang = np.asarray(pos, np.float64)[:, None] * inv_freq[None, :]   # [n, half]
    c = np.cos(ang)[:, None, :]
    s = np.sin(ang)[:, None, :]
    a = x[..., :half]
    b = x[..., half:]
    return np.concatenate([a * c - b * s, a * s + b * c], axis=-1)


def silu(x):
    return x / (1.0 + np.exp(-x))


def qkv(X, pos, layer, n_heads, head_dim, eps=1e-6, theta=10000.0):
    """RMSNorm, the fused q/k/v projection and RoPE on q and k.

    X [n, d] rows of the residual stream, pos [n] their token positions.
    Returns q, k, v as fp64 [n, H, hd]."""
    d = n_heads * head_dim
    a = rmsnorm(X, layer["g_attn"], eps)
    y = a @ np.asarray(layer["w_qkv"], np.float64).T
    n = y.shape[0]
    q = y[:, :d].reshape(n, n_heads, head_dim)
    k = y[:, d:2 * d].reshape(n, n_heads, head_dim)
    v = y[:, 2 * d:].reshape(n, n_heads, head_dim)
    return rope(q, pos, theta), rope(k, pos, theta), v


def out_ffn(X, o, layer, eps=1e-6):
    """Output projection with residual, then the SwiGLU FFN with residual.

    X [n, d], o [n, d] (attention output, heads concatenated)."""
    X = np.asarray(X, np.float64)
    y = X + np.asarray(o, np.float64) @ np.asarray(layer["w_o"], np.float64).T
    a = rmsnorm(y, layer["g_ffn"], eps)
    gu = a @ np.asarray(layer["w_gate_up"], np.float64).T
    F = gu.shape[1] // 2
    hmid = silu(gu[:, :F]) * gu[:, F:]
    return y + hmid @ np.asarray(layer["w_down"], np.float64).T
