"""One library entry point at a workload's shape, on synthetic inputs - for profiling
a single kernel (ncu) or timing it alone with CUDA events.

Cases (the layer of one sparse loop, or the dense loop-1 attention):
  sparse-attn   fl_sparse_loop_attn with carried statistics: the query-tile kernel
  dense-attn    fl_sparse_loop_attn with sel == NULL and statistics for the next loop
  kv-quant      fl_kv_residual_quant of the loop's active rows
  block         fl_block_qkv + fl_block_out_ffn of the loop's active rows (the GEMMs)
Shapes: 4k (Ouro-1.4B, 820 active rows, 82 carried columns, 4-bit residuals) and 32k
(Ouro-2.6B, 4916 active rows, 2048 carried columns, 2-bit residuals); the store holds
one layer's base codes for every token and the residual rows of loop 2. Statistics
rows are the active rows only, so a 32k case holds about 1 GB on the device.

Usage: python -m cross_loop_sparse_step_b200.kernel_case --case sparse-attn --shape 32k
       [--reps 3] [--warmup 1]
Prints one JSON line: the case, the shape and the average time per call (CUDA events).
"""
import argparse
import json
import math
import sys

import numpy as np
import torch

from cross_loop_sparse_step_b200 import configs, fl, synth

SHAPES = {"4k": configs.PREFILL_4K, "32k": configs.PREFILL_32K}


def make_store(cfg, act, g):
    N, H, hd = cfg["n_tok"], cfg["n_heads"], cfg["head_dim"]
    bits = cfg["res_bits"][2]
    st = fl.KVStore(N, H, hd, cfg["group"], 8, {2: bits}, 2, {2: len(act)})
    k1 = torch.from_numpy(synth.kv_values(g, N, H, hd)).cuda()
    v1 = torch.from_numpy(synth.kv_values(g, N, H, hd)).cuda()
    fl.kv_residual_quant(st, 1, k1, v1)
    a = torch.from_numpy(act).cuda()
    n = len(act)
    k2 = k1[a.long()] + 0.5 * torch.randn(n, H, hd, device="cuda")
    v2 = v1[a.long()] + 0.5 * torch.randn(n, H, hd, device="cuda")
    fl.kv_residual_quant(st, 2, k2, v2, a)
    return st, k2, v2


def carried_sets(cfg, act, g):
    """[H][n_act][k+1] ascending column sets: the sink, the biased columns before the
    query, random others before it (the shape of loop 1's statistics)."""
    N, H, k = cfg["n_tok"], cfg["n_heads"], cfg["col_k"][2]
    bias_cols = synth.biased_columns(g, N, cfg["bias_frac"])
    S = np.full((H, len(act), fl.stat_stride(k)), 0xFFFF, np.uint16)
    for i, t in enumerate(act):
        t = int(t)
        if t <= k:
            S[:, i, : t + 1] = np.arange(t + 1)
            continue
        bc = bias_cols[(bias_cols >= 1) & (bias_cols <= t)][:k]
        need = k - len(bc)
        for h in range(H):
            extra = np.setdiff1d(g.integers(1, t + 1, size=need + need // 2 + 8), bc)
            if len(extra) >= need:
                extra = g.permutation(extra)[:need]
            else:
                pool = np.setdiff1d(np.arange(1, t + 1), bc)
                extra = g.choice(pool, need, replace=False)
            S[h, i, : k + 1] = np.sort(np.concatenate([[0], bc, extra]))
    return S


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--case", required=True, choices=["sparse-attn", "dense-attn", "kv-quant", "block"])
    ap.add_argument("--shape", default="32k", choices=sorted(SHAPES))
    ap.add_argument("--reps", type=int, default=3)
    ap.add_argument("--warmup", type=int, default=1)
    a = ap.parse_args()
    cfg = SHAPES[a.shape]
    N, d, H, hd, F = (cfg[x] for x in ("n_tok", "d_model", "n_heads", "head_dim", "d_ffn"))
    n_act = configs.active_counts(cfg)[2]
    g = synth.rng(0)
    act = synth.sorted_subset(g, N, n_act)
    a_dev = torch.from_numpy(act).cuda()
    bias = torch.from_numpy(synth.col_bias(g, N, cfg["bias_frac"], cfg["bias_value"])).cuda()
    k = cfg["col_k"][2]
    calls = []
    info = {}
    if a.case in ("sparse-attn", "kv-quant"):
        st, k2, v2 = make_store(cfg, act, g)
    if a.case == "sparse-attn":
        S = torch.from_numpy(carried_sets(cfg, act, g).view(np.int16)).cuda()
        m = torch.rand(H, n_act, device="cuda") * 0.5 + 0.5
        u = torch.randn(H, n_act, hd, device="cuda") * 0.1
        q = torch.randn(n_act, H, hd, device="cuda")
        out = torch.empty(n_act, H, hd, dtype=torch.bfloat16, device="cuda")
        rows = torch.arange(n_act, dtype=torch.int32, device="cuda")
        calls.append(lambda: fl.sparse_loop_attn(q, a_dev, st, 2, out, col_bias=bias, sel=S, mass=m,
                                                 unsel=u, q_row=rows, stat_rows=n_act))
        info["carried_columns"] = k + 1
    elif a.case == "dense-attn":
        st = fl.KVStore(N, H, hd, cfg["group"], 8, {}, 1, {})
        k1 = torch.from_numpy(synth.kv_values(g, N, H, hd)).cuda()
        fl.kv_residual_quant(st, 1, k1, k1.clone())
        q = torch.randn(N, H, hd, device="cuda")
        tok = torch.arange(N, dtype=torch.int32, device="cuda")
        out = torch.empty(N, H, hd, dtype=torch.bfloat16, device="cuda")
        S = torch.empty(H, N, fl.stat_stride(k), dtype=torch.int16, device="cuda")
        m = torch.empty(H, N, device="cuda")
        u = torch.empty(H, N, hd, device="cuda")
        calls.append(lambda: fl.sparse_loop_attn(q, tok, st, 1, out, col_bias=bias, k_next=k,
                                                 sel_out=S, mass_out=m, unsel_out=u))
    elif a.case == "kv-quant":
        calls.append(lambda: fl.kv_residual_quant(st, 2, k2, v2, a_dev))
    else:
        w = lambda *s: (torch.randn(*s, device="cuda") * 0.02).to(torch.bfloat16)
        layer = {"w_qkv": w(3 * d, d), "w_o": w(d, d), "w_gate_up": w(2 * F, d),
                 "w_down": w(d, F), "g_attn": torch.ones(d, device="cuda"),
                 "g_ffn": torch.ones(d, device="cuda")}
        model = fl.LoopModel([layer], N, H, hd)
        x = torch.randn(n_act, d, device="cuda")
        qb, kb, vb = (torch.empty(n_act, d, device="cuda") for _ in range(3))
        att = torch.randn(n_act, d, device="cuda").to(torch.bfloat16)
        ws = torch.empty(model.block_ws_bytes(n_act), dtype=torch.uint8, device="cuda")
        calls.append(lambda: fl.block_qkv(model, 0, x, a_dev, qb, kb, vb, ws))
        calls.append(lambda: fl.block_out_ffn(model, 0, x, att, ws))
        info["gflop_per_call"] = 2 * n_act * (4 * d * d + 3 * d * F) / 1e9
    for _ in range(a.warmup):
        for c in calls:
            c()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(a.reps):
        for c in calls:
            c()
    e1.record()
    torch.cuda.synchronize()
    status = fl.check_device_status()
    print(json.dumps({"case": a.case, "shape": a.shape, "n_active": n_act, "reps": a.reps,
                      "avg_ms": e0.elapsed_time(e1) / a.reps, "status": status, **info}))
    return 0 if status == 0 else 1


if __name__ == "__main__":
    sys.exit(main())
