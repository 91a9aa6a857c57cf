"""Seeded synthetic inputs for the loop step.

This module draws random numbers and shapes them into the workloads' inputs; it holds
none of the loop step's arithmetic, so both the GPU path and the CPU oracle may be fed
from it. Every generator takes a numpy ``Generator`` (PCG64) so that a seed fixes the
bytes.

Workload shapes follow the FlashLoop pages: weights N(0, 0.02) with unit RMSNorm
gains, embeddings N(0, 1); hidden-state changes concentrated on few tokens (§3.1:
a small fraction of rows carries most of the change, spread over the context) with
magnitudes shrinking loop over loop; a small, stable set of attention columns that
dominates (§3.2, §4.2), modelled as a positive logit bias on 2% of the columns and
on the sink column 0.
"""
import math

import numpy as np


def rng(seed=0):
    return np.random.Generator(np.random.PCG64(seed))


def round_bf16(x):
    """Round float32 values to the nearest bfloat16 (ties to even); returns float32."""
    x = np.ascontiguousarray(x, np.float32)
    u = x.view(np.uint32).astype(np.uint64)
    lsb = (u >> 16) & 1
    u = ((u + 0x7FFF + lsb) & 0xFFFF0000).astype(np.uint32)
    out = u.view(np.float32)
    return np.where(np.isnan(x), x, out).astype(np.float32)


def layer_weights(g, d, ffn, std=0.02, bf16=False):
    """One layer's weights, linear-layer layout [out, in], float32 arrays."""
    def w(*shape):
        a = (g.standard_normal(shape, dtype=np.float64) * std).astype(np.float32)
        return round_bf16(a) if bf16 else a
    return {
        "w_qkv": w(3 * d, d),
        "w_o": w(d, d),
        "w_gate_up": w(2 * ffn, d),
        "w_down": w(d, ffn),
        "g_attn": np.ones(d, np.float32),
        "g_ffn": np.ones(d, np.float32),
    }


def model_weights(g, n_layers, d, ffn, std=0.02, bf16=False):
    return [layer_weights(g, d, ffn, std, bf16) for _ in range(n_layers)]


def embeddings(g, n_tok, d):
    return g.standard_normal((n_tok, d), dtype=np.float64).astype(np.float32)


def biased_columns(g, n_tok, frac=0.02):
    """ceil(frac * N) distinct columns drawn uniformly from [1, N), ascending."""
    n = int(math.ceil(frac * n_tok))
    n = min(n, n_tok - 1)
    return np.sort(g.choice(np.arange(1, n_tok), size=n, replace=False)).astype(np.int64)


def col_bias(g, n_tok, frac=0.02, value=4.0):
    """Per-column logit bias: ``value`` on the sink 0 and on 2% of the columns."""
    b = np.zeros(n_tok, np.float32)
    if frac > 0:
        b[biased_columns(g, n_tok, frac)] = value
        b[0] = value
    return b


def pareto_delta_pair(g, n_rows, d, loop, alpha=1.5, scale=0.05, decay=0.5):
    """A (current, previous) hidden-state pair whose row changes are heavy-tailed.

    current rows ~ N(0, 1); change_t = rho_t * decay^(loop-2) * scale * sqrt(d) * u_t
    with rho ~ Pareto(alpha, x_m = 1) and u_t a uniformly random unit direction;
    previous = current - change. Returns float32 (h_cur, h_prev, rho)."""
    h_cur = g.standard_normal((n_rows, d), dtype=np.float64)
    rho = g.pareto(alpha, size=n_rows) + 1.0
    u = g.standard_normal((n_rows, d), dtype=np.float64)
    u /= np.linalg.norm(u, axis=1, keepdims=True)
    mag = rho * (decay ** (loop - 2)) * scale * math.sqrt(d)
    h_prev = h_cur - mag[:, None] * u
    return h_cur.astype(np.float32), h_prev.astype(np.float32), rho


def kv_values(g, n_tok, n_heads, head_dim, scale=1.0):
    """Post-RoPE-like K or V values, N(0, scale^2), float32 [n, H, hd]."""
    return (g.standard_normal((n_tok, n_heads, head_dim)) * scale).astype(np.float32)


def query_values(g, n_q, n_heads, head_dim, scale=1.0):
    return (g.standard_normal((n_q, n_heads, head_dim)) * scale).astype(np.float32)


def sorted_subset(g, n, k):
    """k distinct integers from [0, n), ascending."""
    return np.sort(g.choice(n, size=k, replace=False)).astype(np.int32)


def kv_loop_sequence(g, n, H, hd, R, scale=1.0, decay=0.5, delta=0.25):
    """Per-loop K (or V) of n tokens over R loops: K_1 ~ N(0, scale^2) and
    K_r = K_{r-1} + D_r with D_r ~ N(0, (scale * delta * decay^(r-2))^2) - a change that
    shrinks loop after loop (§3.3: cross-loop KV updates are small). float32 arrays."""
    K = [(g.standard_normal((n, H, hd)) * scale).astype(np.float32)]
    for r in range(2, R + 1):
        d = g.standard_normal((n, H, hd)) * scale * delta * decay ** (r - 2)
        K.append((K[-1] + d).astype(np.float32))
    return K
