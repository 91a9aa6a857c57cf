"""The shared Transformer block, in fp64 (oracle; test infrastructure only).

Pages: FlashLoop §1 (a looped Transformer applies one shared N-layer block R times,
R x N block executions, a distinct KV per iteration). The pages do not describe the
block itself; the reading taken is a standard pre-norm decoder layer:
  x <- x + Attn(RMSNorm(x)) . W_o
  x <- x + (silu(RMSNorm(x) W_gate) * (RMSNorm(x) W_up)) W_down
  RMSNorm(x) = x / sqrt(mean(x^2) + eps) * gamma,  eps = 1e-6
  RoPE: theta = 10000, rotate-half pairs (i, i + hd/2), position = token index.
No biases, no final norm, no LM head.
A bf16 workload keeps the residual stream in fp32 and its GEMM operands in bfloat16
(``bf16_ops``); the products are exact sums here (fp64).

Weights are stored like linear-layer weights, [out_features, in_features]:
  w_qkv [3d, d] (rows: q, then k, then v), w_o [d, d],
  w_gate_up [2F, d] (rows: gate, then up), w_down [d, F].
"""
import numpy as np
import torch


def bf16(x):
    """Round to the nearest bfloat16 (ties to even), returned as fp64. A bf16 workload
    holds its GEMM operands as bfloat16 tensors: the RMSNorm outputs, the attention
    output entering W_o and the SwiGLU product entering W_down."""
    t = torch.from_numpy(np.ascontiguousarray(x, np.float64))
    return t.to(torch.float32).to(torch.bfloat16).to(torch.float64).numpy()


def _operand(x, bf16_ops):
    return bf16(x) if bf16_ops else x


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


def qkv(X, pos, layer, n_heads, head_dim, eps=1e-6, theta=10000.0, bf16_ops=False):
    """RMSNorm, the fused q/k/v projection and RoPE on q and k.

    X [n, d] rows of the residual stream, pos [n] their token positions.
    ``bf16_ops``: the GEMM operand (RMSNorm output) is a bfloat16 tensor.
    Returns q, k, v as fp64 [n, H, hd]."""
    d = n_heads * head_dim
    a = _operand(rmsnorm(X, layer["g_attn"], eps), bf16_ops)
    y = a @ np.asarray(layer["w_qkv"], np.float64).T
    n = y.shape[0]
    q = y[:, :d].reshape(n, n_heads, head_dim)
    k = y[:, d:2 * d].reshape(n, n_heads, head_dim)
    v = y[:, 2 * d:].reshape(n, n_heads, head_dim)
    return rope(q, pos, theta), rope(k, pos, theta), v


def out_ffn(X, o, layer, eps=1e-6, bf16_ops=False):
    """Output projection with residual, then the SwiGLU FFN with residual.

    X [n, d], o [n, d] (attention output, heads concatenated). ``bf16_ops``: the
    three GEMM operands (o, the RMSNorm output, the SwiGLU product) are bfloat16."""
    X = np.asarray(X, np.float64)
    o = _operand(np.asarray(o, np.float64), bf16_ops)
    y = X + o @ np.asarray(layer["w_o"], np.float64).T
    a = _operand(rmsnorm(y, layer["g_ffn"], eps), bf16_ops)
    gu = a @ np.asarray(layer["w_gate_up"], np.float64).T
    F = gu.shape[1] // 2
    hmid = _operand(silu(gu[:, :F]) * gu[:, F:], bf16_ops)
    return y + hmid @ np.asarray(layer["w_down"], np.float64).T
