"""The workloads the loop step is built and measured for.

Shapes follow the looped models the FlashLoop pages evaluate (§5.1: the Ouro family;
§1: Ouro-2.6B with four loops at a 32K prompt; §5.4 Figure 7: loop scaling at 8K).
The per-loop schedules are the workloads' own choices: the pages' loop-wise table
(Appendix E, Table 5) has no values. ``tok_frac[r]`` is the fraction of all prompt
rows recomputed in loop r, ``col_k[r]`` the number of attention columns a query keeps
in loop r besides the sink (None: dense attention), ``res_bits[r]`` the residual
width of loop r (0: stored unquantised).
"""
import math

TINY_FP32 = dict(
    name="tiny-looped-block-fp32",
    n_tok=256, d_model=256, n_heads=4, head_dim=64, d_ffn=1024, n_layers=1, n_loops=4,
    dtype="f32", first_sparse=2,
    tok_frac={2: 0.25, 3: 0.25, 4: 0.25},
    col_k={2: 32, 3: 32, 4: 32},
    base_bits=8, res_bits={2: 4, 3: 4, 4: 4}, group=32,
    bias_frac=0.0, bias_value=0.0, synthetic_delta=False,
)

# the same block with shrinking budgets, to exercise pruning of carried columns
TINY_FP32_SHRINK = dict(TINY_FP32, name="tiny-looped-block-fp32-shrink",
                        tok_frac={2: 0.5, 3: 0.25, 4: 0.125},
                        col_k={2: 32, 3: 16, 4: 8})

PREFILL_4K = dict(
    name="ouro-1.4b-shape-prefill-4k",
    n_tok=4096, d_model=2048, n_heads=16, head_dim=128, d_ffn=5632, n_layers=24,
    n_loops=4, dtype="bf16", first_sparse=2,
    tok_frac={2: 0.2, 3: 0.2, 4: 0.2},
    col_k={2: 82, 3: 82, 4: 82},
    base_bits=8, res_bits={2: 4, 3: 4, 4: 4}, group=32,
    bias_frac=0.02, bias_value=4.0, synthetic_delta=True,
)

PREFILL_32K = dict(
    name="ouro-2.6b-shape-prefill-32k",
    n_tok=32768, d_model=2048, n_heads=16, head_dim=128, d_ffn=5632, n_layers=48,
    n_loops=4, dtype="bf16", first_sparse=2,
    tok_frac={2: 0.15, 3: 0.15, 4: 0.15},
    col_k={2: 2048, 3: 2048, 4: 2048},
    base_bits=8, res_bits={2: 2, 3: 2, 4: 2}, group=32,
    bias_frac=0.02, bias_value=4.0, synthetic_delta=True,
)


def c4(n_loops, res_bits):
    """Loop-depth sweep: active fraction 0.5 * 0.1^((r-2)/(R-2)), r = 2..R."""
    R = n_loops
    frac = {r: 0.5 * 0.1 ** ((r - 2) / (R - 2)) for r in range(2, R + 1)}
    return dict(
        name=f"ouro-2.6b-shape-prefill-8k-R{R}-b{res_bits}",
        n_tok=8192, d_model=2048, n_heads=16, head_dim=128, d_ffn=5632, n_layers=48,
        n_loops=R, dtype="bf16", first_sparse=2,
        tok_frac=frac, col_k={r: 512 for r in range(2, R + 1)},
        base_bits=8, res_bits={r: res_bits for r in range(2, R + 1)}, group=64,
        bias_frac=0.02, bias_value=4.0, synthetic_delta=True,
    )


# Batched decode (§5.3.3, Figure 5: decode with sparse attention and 2/4-bit residuals):
# 64 sequences with 16K..32K cached tokens each; the generated token's loop r >= 2 step
# per layer (its KV appended, sparse attention over 1024 carried columns plus the sink,
# the block on the 64 new rows).
DECODE_B64 = dict(
    name="ouro-2.6b-shape-decode-b64",
    batch=64, ctx_min=16384, ctx_max=32768, d_model=2048, n_heads=16, head_dim=128,
    d_ffn=5632, n_layers=48, n_loops=4, dtype="bf16", col_k=1024, base_bits=8,
    res_bits=2, group=32, active_frac=0.15, bias_frac=0.02, bias_value=4.0, decode=True,
)

CONFIGS = {c["name"]: c for c in (TINY_FP32, TINY_FP32_SHRINK, PREFILL_4K, PREFILL_32K, c4(8, 2),
                                   c4(8, 4), c4(16, 2), c4(16, 4), DECODE_B64)}


def active_counts(cfg):
    """Number of active tokens per loop: all N in loops before the first sparse loop,
    then min(ceil(f_r * N), previous count). The fraction is read as its decimal
    string so that 0.2 * 4096 gives 820, not 819.2000000000001 rounded up to 820 by
    luck."""
    from decimal import Decimal
    N = cfg["n_tok"]
    out = {1: N}
    prev = N
    for r in range(2, cfg["n_loops"] + 1):
        if r < cfg["first_sparse"]:
            k = N
        else:
            k = min(int(math.ceil(Decimal(repr(cfg["tok_frac"][r])) * N)), prev)
        out[r] = k
        prev = k
    return out
