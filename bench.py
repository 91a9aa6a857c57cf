#!/usr/bin/env python
"""Loop-step throughput of the FlashLoop lazy loop step on B200.

Workload (default): the Ouro-2.6B-shaped 32K prefill - 32768 tokens, d_model 2048,
16 x 128 heads, SwiGLU FFN 5632, 48 shared layers, R = 4 loops, bf16 GEMM operands,
15% active tokens per sparse loop (4916), 2048 carried columns per query plus the
sink, int8 base + 2-bit residual KV (group 32), a +4 logit bias on 2% of the columns
and the sink, heavy-tailed (Pareto 1.5) hidden-state changes. Loop 1 (dense, every
token, the producer of the carried statistics) runs before the timed region and is
timed on its own; one timed step is loops 2..R through fl_loop_step: selection,
gather, 48 layers of the block on the active rows (QKV + RoPE, residual KV
quantisation, sparse attention, O projection, FFN), scatter.
value = N * (R - 1) / step time: loop-step tokens/s. The line also reports the
end-to-end prefill rate N / (t_1 + t_2 + ... + t_R) with the dense loop 1 included.
Other workloads: --config (the 4K Ouro-1.4B shape, the 8K loop-depth sweep).

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
Multi-GPU: one process per GPU (torchrun); every rank runs an independent replica of
the workload (the method's prefill loop step has no cross-GPU exchange), time is the
max over ranks, value the sum of tokens over the max time ("weak" scaling).
"""
import argparse
import ctypes
import json
import math
import os
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

METRIC = "loop-step tokens/s at R loops + % of HBM/tensor roofline; KV bytes/token"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# DRAM bytes of one attention call (ncu dram__bytes_read.sum + dram__bytes_write.sum of
# the call's kernels, one capture each) at a workload's sparse-loop shape; None where not
# captured for the current kernels. Summaries and commands: profiles/.
ATTN_TRAFFIC = {
    "ouro-2.6b-shape-prefill-32k": {
        "bytes": (158.77 + 211.36 + 315.78 + 127.90 + 520.55 + 17.00) * 1e6,
        "per_kernel_mb": {"k_kv_stage": 370.13, "k_sel_bitmap": 443.68, "k_attn_tile<2>": 537.55},
        "source": "kernel case sparse-attn 32k (4916 queries x 16 heads, 2048 + 1 carried "
                  "columns, 2-bit residuals: the loop-2 call of this workload)",
        # the softmax of k_attn_tile changed after the capture (non-members masked at -inf
        # before the exponential instead of after it: arithmetic only): reported as null
        "current": False},
}


# Component toggles and loop schedules (paper §5.3 Figure 4: the contribution of each
# lazy update; §4.1: dense early loops; §4.2: progressive pruning with smaller budgets).
VARIANTS = {
    "flashloop": "all three lazy updates as configured",
    "dense": "no lazy update: every token, dense attention, unquantised KV in every loop",
    "token-sparse": "token-sparse updates only: dense attention, unquantised KV",
    "token+attn": "token-sparse updates and sparse attention, unquantised KV",
    "dense-early": "loop 2 dense (every token, dense attention), the lazy updates from loop 3",
    "shrink": "carried column budget halved loop after loop (k, k/2, k/4, ...)",
}


def apply_variant(cfg, variant):
    """The workload with one of VARIANTS applied (a copy)."""
    c = dict(cfg)
    R = c["n_loops"]
    loops = range(2, R + 1)
    if variant in ("dense", "token-sparse", "token+attn"):
        c["base_bits"] = 0
        c["res_bits"] = {r: 0 for r in loops}
    if variant in ("dense", "token-sparse"):
        c["col_k"] = {r: 0 for r in loops}
    if variant == "dense":
        c["first_sparse"] = R + 1
        c["tok_frac"] = {r: 1.0 for r in loops}
    if variant == "dense-early":
        c["first_sparse"] = 3
        c["col_k"] = {**c["col_k"], 2: 0}
        c["tok_frac"] = {**c["tok_frac"], 2: 1.0}
    if variant == "shrink":
        k0 = c["col_k"][2]
        c["col_k"] = {r: max(1, k0 >> (r - 2)) for r in loops}
    c["variant"] = variant
    return c


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--config", default="ouro-2.6b-shape-prefill-32k")
    ap.add_argument("--layers", type=int, default=None, help="override layer count (profiling)")
    ap.add_argument("--variant", default="flashloop", choices=sorted(VARIANTS),
                    help="component toggle or loop schedule (see VARIANTS)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-graph", dest="graph", action="store_false",
                    help="launch each step's kernels eagerly instead of replaying a CUDA graph")
    return ap.parse_args()


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# ---------------------------------------------------------------- clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_uuid):
        self.uuid = gpu_uuid
        self.proc = None
        self.path = os.path.join("/tmp", f"fl_clocks_{os.getpid()}.csv")

    def start(self):
        try:
            cmd = ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                   "-lms", "200"]
            if self.uuid:
                cmd += ["-i", self.uuid]
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(cmd, stdout=self.f, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.f.close()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        try:
            os.remove(self.path)
        except OSError:
            pass
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = set()
        for r in rows:
            for n, v in zip(names, r[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        power = [float(r[3]) for r in rows if r[3].replace(".", "").isdigit()]
        return {"sm_mhz": float(np.median(sm)) if sm else None,
                "sm_max_mhz": max(mx) if mx else None,
                "reasons": sorted(reasons), "samples": len(rows),
                "power_w_max": max(power) if power else None}


# ---------------------------------------------------------------- multi-rank aggregation
def aggregate(t_rank, units_rank, dist=None, device="cpu"):
    """Whole-job throughput over replicas: every rank's units divided by the slowest
    rank's time (max over ranks). Returns (value, t_max, units_total)."""
    import torch
    if dist is None or not dist.is_initialized() or dist.get_world_size() == 1:
        return units_rank / t_rank, t_rank, units_rank
    t = torch.tensor([t_rank], dtype=torch.float64, device=device)
    u = torch.tensor([units_rank], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    dist.all_reduce(u, op=dist.ReduceOp.SUM)
    return float(u.item()) / float(t.item()), float(t.item()), float(u.item())


# ---------------------------------------------------------------- workload
def build_workload(cfg, fl, torch, synth, configs, seed, n_layers=None):
    N, d, H, hd, F = (cfg[k] for k in ("n_tok", "d_model", "n_heads", "head_dim", "d_ffn"))
    L = n_layers or cfg["n_layers"]
    R = cfg["n_loops"]
    dev = "cuda"
    gen = torch.Generator(device=dev)
    gen.manual_seed(seed)

    def w(*shape):
        return (torch.randn(*shape, generator=gen, device=dev) * 0.02).to(torch.bfloat16)
    layers = [{"w_qkv": w(3 * d, d), "w_o": w(d, d), "w_gate_up": w(2 * F, d), "w_down": w(d, F),
               "g_attn": torch.ones(d, device=dev), "g_ffn": torch.ones(d, device=dev)}
              for _ in range(L)]
    g = synth.rng(seed)
    bias = torch.from_numpy(synth.col_bias(g, N, cfg["bias_frac"], cfg["bias_value"])).to(dev)
    n_active = configs.active_counts(cfg)
    model = fl.LoopModel(layers, N, H, hd, col_bias=bias)
    res = {r: cfg["res_bits"][r] for r in range(2, R + 1)}
    stores = [fl.KVStore(N, H, hd, cfg["group"], cfg["base_bits"], res, R, n_active)
              for _ in range(L)]
    col_k = {r: cfg["col_k"][r] for r in range(2, R + 1)}
    sched = fl.make_schedule(R, cfg["first_sparse"], n_active, col_k)
    kmax = max(col_k.values())
    run = fl.LoopRunner(model, sched, n_active, stores, fl.stat_stride(kmax) if kmax > 0 else 0)
    h0 = torch.from_numpy(synth.embeddings(g, N, d)).to(dev)
    # the dense loop 1 (the producer of loop 2's statistics): once cold, then timed warm
    # from the same embeddings (it rewrites the same base KV and statistics)
    loop1 = []
    for _ in range(2):
        run.h.copy_(h0)
        torch.cuda.synchronize()
        t1 = (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
        t1[0].record()
        run.step(1)
        t1[1].record()
        torch.cuda.synchronize()
        loop1.append(t1[0].elapsed_time(t1[1]))
    loop1_ms = loop1[-1]
    cur, prev, _ = synth.pareto_delta_pair(g, N, d, 2)
    run.x_prev.copy_(run.h - torch.from_numpy((cur - prev).astype(np.float32)).to(dev))
    st = fl.check_device_status()
    if st != 0:
        raise RuntimeError(f"loop 1 reported {fl.status_str(st)}")
    snap = (run.h.clone(), run.x_prev.clone())
    return dict(run=run, stores=stores, model=model, layers=layers, n_active=n_active, snap=snap,
                L=L, R=R, N=N, d=d, H=H, hd=hd, F=F, col_k=col_k, res=res, loop1_ms=loop1_ms,
                loop1_cold_ms=loop1[0])


def step_loops(W):
    for r in range(2, W["R"] + 1):
        W["run"].step(r)


def restore(W):
    W["run"].h.copy_(W["snap"][0])
    W["run"].x_prev.copy_(W["snap"][1])


def gemm_flops_per_step(W):
    d, F, L = W["d"], W["F"], W["L"]
    per_row = 2 * (3 * d * d + d * d + 2 * F * d + F * d)
    return sum(W["n_active"][r] * per_row * L for r in range(2, W["R"] + 1))


def attention_bytes_per_launch(W, torch):
    """Algorithmic work of one attention launch (one layer of one loop) per loop r:
    (bytes, algorithmic FLOP, executed tensor FLOP, sparse?).

    Sparse loops, from the carried column sets: q (fp32), S, m, u read; o (bf16) written;
    the compressed KV of the distinct columns each head reads (base K and V plus the
    residual rows of every loop up to r in which the column was active); FLOP 4 hd |S|;
    the query-tile form executes QK^T and PV on 128-column chunks of each tile's union.
    Dense loops: every active query over its causal prefix, FLOP 4 hd (t + 1), the whole
    store read once per head."""
    H, hd, N = W["H"], W["hd"], W["N"]
    g = W["stores"][0].g
    st0 = W["stores"][0]
    slot = st0.slot.cpu().numpy()
    out = {}
    for r in range(2, W["R"] + 1):
        act = W["run"].act[r][: W["n_active"][r]].long()
        nq = act.numel()
        base_row = 2 * (hd + hd // g * 4) if st0.base_bits else 2 * hd * 4
        if W["col_k"][r] > 0:
            k1 = W["run"].sel[0].shape[2]
            sel = W["run"].sel[0][:, act].cpu().numpy().view(np.uint16)
            kv = 0
            for h in range(H):
                cols = np.unique(sel[h][sel[h] != 0xFFFF]).astype(np.int64)
                kv += len(cols) * base_row
                for rr in range(2, r + 1):
                    b = W["res"][rr]
                    nrow = int((slot[rr][cols] >= 0).sum())
                    kv += nrow * (2 * (hd * b // 8 + hd // g * 4) if b else 2 * hd * 4)
            fixed = nq * H * hd * 4 + H * nq * k1 * 2 + H * nq * 4 + H * nq * hd * 4 + nq * H * hd * 2
            flops = 4 * hd * int((sel != 0xFFFF).sum())
            chunks = 0
            for h in range(H):
                for t0 in range(0, nq, 128):
                    blk = sel[h, t0:t0 + 128]
                    u = np.unique(blk[blk != 0xFFFF]).size
                    chunks += -(-u // 128)
            out[r] = (fixed + kv, flops, chunks * 4 * 128 * 128 * hd, True)
        else:
            pos = act.cpu().numpy().astype(np.int64)
            kv = N * H * base_row
            for rr in range(2, r + 1):
                b = W["res"][rr]
                nrow = int((slot[rr] >= 0).sum())
                kv += nrow * H * (2 * (hd * b // 8 + hd // g * 4) if b else 2 * hd * 4)
            flops = 4 * hd * H * int((pos + 1).sum())
            out[r] = (kv + nq * H * hd * 6, flops, flops, False)
    return out


def kv_bytes(W):
    tot = sum(s.nbytes(r) for s in W["stores"] for r in range(1, W["R"] + 1))
    per_tok_layer = tot / (W["N"] * W["L"])
    dense = W["R"] * 2 * W["d"] * 2
    return per_tok_layer, dense


# ---------------------------------------------------------------- CPU baseline (oracle)
class OracleSample:
    """The oracle on a bounded sample of one sparse loop step of the workload.

    Set-up (untimed): ``n_layers`` layers of random bf16 weights, their KV stores with
    every token's base codes, the carried statistics of ``rows`` sampled active queries
    (sink, biased columns, random others). ``run()`` (timed): the token ranking over all
    N rows (h, previous state), then per layer the block, the residual quantisation and
    the sparse attention of the sampled rows. Returns the seconds extrapolated to one
    sparse loop step of the workload (k_r rows x L layers), the measured seconds and the
    sample's description."""

    def __init__(self, cfg, n_layers=1, rows=256, seed=1):
        from cross_loop_sparse_step_b200 import configs, synth
        from oracle import attention as oatt
        from oracle import kvstore as okv
        from oracle import select as osel
        self.cfg = cfg
        N, d, H, hd, F = (cfg[k] for k in ("n_tok", "d_model", "n_heads", "head_dim", "d_ffn"))
        self.k_act = configs.active_counts(cfg)[2]
        kcol = cfg["col_k"][2]
        g = synth.rng(seed)
        self.cur, self.prev, _ = synth.pareto_delta_pair(g, N, d, 2)
        self.layers = synth.model_weights(g, n_layers, d, F, bf16=True)
        self.bias = synth.col_bias(g, N, cfg["bias_frac"], cfg["bias_value"])
        self.stores = []
        for _ in range(n_layers):
            st = okv.LayerKV(N, H, hd, cfg["group"], cfg["base_bits"], cfg["res_bits"],
                             cfg["n_loops"])
            st.write_base(synth.kv_values(g, N, H, hd), synth.kv_values(g, N, H, hd))
            self.stores.append(st)
        act, _, _ = osel.select_active(self.cur, self.prev, None, self.k_act)
        rs = synth.rng(seed + 1)
        self.q_rows = np.sort(rs.choice(act, size=min(rows, len(act)), replace=False)).astype(np.int32)
        self.X = synth.embeddings(g, len(self.q_rows), d).astype(np.float64)
        self.S = np.full((H, N, kcol + 1), oatt.SENTINEL, np.uint16)
        for t in self.q_rows:
            for h in range(H):
                n = min(kcol, int(t)) + 1
                c = np.sort(np.concatenate([[0], rs.choice(np.arange(1, t + 1), n - 1, replace=False)])) \
                    if t > 0 else np.array([0])
                self.S[h, t, :n] = c
        self.m = np.full((H, N), 0.9)
        self.u = np.zeros((H, N, hd))
        self.n_layers = n_layers
        self.desc = (f"loop-2 step sample: token ranking over all {N} rows, then {n_layers} "
                     f"layer(s) x {len(self.q_rows)} active rows (of {self.k_act}) x {H} heads "
                     f"with {kcol} carried columns; extrapolated x{cfg['n_layers']} layers, "
                     f"x{self.k_act}/{len(self.q_rows)} rows")

    def run(self):
        from oracle import attention as oatt
        from oracle import block as oblk
        from oracle import select as osel
        H, hd = self.cfg["n_heads"], self.cfg["head_dim"]
        d = H * hd
        t0 = time.perf_counter()
        osel.select_active(self.cur, self.prev, None, self.k_act)
        t_select = time.perf_counter() - t0
        X = self.X
        t0 = time.perf_counter()
        for li in range(self.n_layers):
            q, k, v = oblk.qkv(X, self.q_rows, self.layers[li], H, hd, bf16_ops=True)
            self.stores[li].write_residual(2, self.q_rows, k.astype(np.float32), v.astype(np.float32))
            Kh, Vh = self.stores[li].hat[2]
            o = oatt.sparse_attention(q, self.q_rows, self.q_rows, Kh, Vh, self.S, self.m, self.u,
                                      self.bias)
            X = oblk.out_ffn(X, o.reshape(len(self.q_rows), d), self.layers[li], bf16_ops=True)
        t_layers = time.perf_counter() - t0
        per_loop = t_select + t_layers / self.n_layers * self.cfg["n_layers"] * (
            self.k_act / len(self.q_rows))
        return per_loop, t_select + t_layers, self.desc


# bounded samples of the oracle per workload size: (layers, rows)
def oracle_sample_size(cfg):
    return (1, 128) if cfg["n_tok"] >= 16384 else (2, 256)


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return os.cpu_count() or 1


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    from cross_loop_sparse_step_b200 import configs
    cfg = configs.CONFIGS[args.config]
    R = cfg["n_loops"]
    n_layers, rows = oracle_sample_size(cfg)
    sample = OracleSample(cfg, n_layers=n_layers, rows=rows, seed=1)
    times, measured = [], []
    desc = sample.desc
    for i in range(args.warmup + args.steps):
        per_loop, meas, desc = sample.run()
        if i >= args.warmup:
            times.append(per_loop)
            measured.append(meas)
    per_loop = float(np.mean(times))
    value = cfg["n_tok"] / per_loop
    cores = blas_threads()
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": per_loop * (R - 1) * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "extrapolated": True,
        "measured_s_per_step": round(float(np.mean(measured)), 3),
        "config": {"workload": cfg["name"], "n_tok": cfg["n_tok"], "layers": cfg["n_layers"],
                   "loops": R},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                         "sample": desc},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------- batched decode
def run_decode(args, cfg):
    """One layer of the decode step of a generated token, loops 2..R, for B sequences:
    the block's q/k/v of the B new rows, each sequence's residual KV row appended,
    sparse attention of every sequence over its own store in one launch, the output
    projection and FFN. Timed per layer (CUDA events, graph replay excluded: the appends
    are per-sequence launches); tokens/s extrapolates to L layers x (R - 1) loops and is
    labelled as such (the dense loop 1 of a decode step is not part of this number)."""
    import torch
    from cross_loop_sparse_step_b200 import fl, synth
    B, d, H, hd, F = (cfg[k] for k in ("batch", "d_model", "n_heads", "head_dim", "d_ffn"))
    R, K, g, bits = cfg["n_loops"], cfg["col_k"], cfg["group"], cfg["res_bits"]
    rs = synth.rng(0)
    ctx = rs.integers(cfg["ctx_min"], cfg["ctx_max"] + 1, size=B)
    n_max = int(ctx.max()) + 1
    stores, bias, stats, rows0, args_keep = [], [], [], {}, []
    res = {r: bits for r in range(2, R + 1)}
    for b in range(B):
        n_ctx = int(ctx[b])
        n_tok = n_ctx + 1
        k_act = int(math.ceil(cfg["active_frac"] * n_ctx))
        act = torch.from_numpy(np.sort(rs.choice(n_ctx, size=k_act, replace=False)).astype(np.int32)).cuda()
        st = fl.KVStore(n_tok, H, hd, g, cfg["base_bits"], res, R, {r: k_act + 1 for r in range(2, R + 1)})
        fl.kv_residual_quant(st, 1, torch.randn(n_tok, H, hd, device="cuda"),
                             torch.randn(n_tok, H, hd, device="cuda"))
        for r in range(2, R + 1):
            kr = torch.randn(k_act, H, hd, device="cuda") * 0.5 ** (r - 1)
            fl.kv_residual_quant(st, r, kr, kr.clone(), act)
        tok = torch.tensor([n_ctx], dtype=torch.int32, device="cuda")
        fl.kv_append(st, 1, torch.randn(1, H, hd, device="cuda"), torch.randn(1, H, hd, device="cuda"), tok)
        stores.append(st)
        rows0[b] = k_act
        bcols = synth.biased_columns(rs, n_ctx, cfg["bias_frac"])
        bb = np.zeros(n_tok, np.float32)
        bb[bcols] = cfg["bias_value"]
        bb[0] = cfg["bias_value"]
        bias.append(torch.from_numpy(bb).cuda())
        S = np.full((H, 1, K + 1), 0xFFFF, np.uint16)
        bc = bcols[bcols <= n_ctx][:K]
        for h in range(H):
            extra = np.setdiff1d(rs.integers(1, n_ctx + 1, size=2 * K), bc)
            extra = rs.permutation(extra)[: K - len(bc)]
            S[h, 0] = np.sort(np.concatenate([[0], bc, extra]))
        stats.append((torch.from_numpy(S.view(np.int16)).cuda(),
                      torch.rand(H, 1, device="cuda") * 0.5 + 0.5,
                      torch.randn(H, 1, hd, device="cuda") * 0.1, tok))
    torch.cuda.synchronize()
    w = lambda *sh: (torch.randn(*sh, device="cuda") * 0.02).to(torch.bfloat16)
    layer = {"w_qkv": w(3 * d, d), "w_o": w(d, d), "w_gate_up": w(2 * F, d), "w_down": w(d, F),
             "g_attn": torch.ones(d, device="cuda"), "g_ffn": torch.ones(d, device="cuda")}
    model = fl.LoopModel([layer], n_max, H, hd)
    x = torch.randn(B, d, device="cuda")
    pos = torch.from_numpy(ctx.astype(np.int32)).cuda()
    q, k, v = (torch.empty(B, H, hd, device="cuda") for _ in range(3))
    attn = torch.empty(B, H, hd, dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(model.block_ws_bytes(B), dtype=torch.uint8, device="cuda")
    q_row = torch.zeros(1, dtype=torch.int32, device="cuda")
    calls = {}
    for r in range(2, R + 1):
        calls[r] = [fl.make_attn_args(q[b:b + 1], stats[b][3], stores[b], r, attn[b:b + 1],
                                      col_bias=bias[b], sel=stats[b][0], mass=stats[b][1],
                                      unsel=stats[b][2], q_row=q_row, stat_rows=1)
                    for b in range(B)]
    arr = {r: (fl.AttnArgs * B)(*calls[r]) for r in calls}
    nb = fl._attn_b_ws(B)
    aws = torch.empty(nb, dtype=torch.uint8, device="cuda")
    stream = fl.stream_handle()

    def layer_step():
        for r in range(2, R + 1):
            fl.block_qkv(model, 0, x, pos, q, k, v, ws)
            for b in range(B):
                fl.kv_append(stores[b], r, k[b:b + 1], v[b:b + 1], stats[b][3], row0=rows0[b])
            rc = fl._attn_b(arr[r], B, fl.ptr(aws), nb, stream)
            if rc != 0:
                raise fl.FLError(rc, "fl_sparse_loop_attn_batched")
            fl.block_out_ffn(model, 0, x, attn, ws)

    for _ in range(args.warmup):
        layer_step()
    torch.cuda.synchronize()
    st = fl.check_device_status()
    if st != 0:
        raise RuntimeError(f"decode warm-up reported {fl.status_str(st)}")
    # attention alone, for its roofline
    ea, eb = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ea.record()
    for _ in range(args.steps):
        fl._attn_b(arr[R], B, fl.ptr(aws), nb, stream)
    eb.record()
    torch.cuda.synchronize()
    attn_us = ea.elapsed_time(eb) / args.steps * 1e3
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(args.steps):
        layer_step()
    e1.record()
    torch.cuda.synchronize()
    st = fl.check_device_status()
    if st != 0:
        raise RuntimeError(f"decode steps reported {fl.status_str(st)}")
    per_layer_ms = e0.elapsed_time(e1) / args.steps      # loops 2..R of one layer
    L = cfg["n_layers"]
    step_ms = per_layer_ms * L
    # algorithmic bytes of one attention launch: per (sequence, head) the carried
    # columns' base codes and scales for K and V, the residual rows of the columns that
    # have them, q, S, m, u read and o written
    kv_b = 0
    for b in range(B):
        slot = stores[b].slot.cpu().numpy()
        S = stats[b][0].cpu().numpy().view(np.uint16)
        for h in range(H):
            cols = S[h, 0][S[h, 0] != 0xFFFF].astype(np.int64)
            kv_b += len(cols) * 2 * (hd + hd // g * 4)
            for rr in range(2, R + 1):
                kv_b += int((slot[rr][cols] >= 0).sum()) * 2 * (hd * bits // 8 + hd // g * 4)
    fixed = B * H * (hd * 4 + (K + 1) * 2 + 4 + hd * 4 + hd * 2)
    attn_bytes = kv_b + fixed
    pk, pk_kind = peaks()
    peak_h = pk.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"])
    weights = 2 * (4 * d * d + 3 * d * F)
    layer_bytes = (R - 1) * (attn_bytes + weights)
    line = {
        "metric": "decode tokens/s (loops 2..R of a generated token, extrapolated to all layers)",
        "value": B / (step_ms / 1e3), "unit": "tokens/s", "n_gpus": 1, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": step_ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "extrapolated": f"measured one layer (x{L} layers); the dense loop 1 of the step excluded",
        "config": {"workload": cfg["name"], "batch": B, "context": [cfg["ctx_min"], cfg["ctx_max"]],
                   "heads": f"{H}x{hd}", "col_k": K, "res_bits": bits, "loops": R},
        "per_layer_us": per_layer_ms * 1e3,
        "roofline": {"bound": "hbm", "kernel": "decode layer step (batched tile attention, "
                     "KV append, projection GEMMs of the B rows)",
                     "achieved": layer_bytes / (per_layer_ms / 1e3) / 1e9, "peak": peak_h,
                     "unit": "GB/s", "frac": layer_bytes / (per_layer_ms / 1e3) / 1e9 / peak_h,
                     "traffic": None, "bytes_per_layer": layer_bytes},
        "attention_roofline": {"bound": "hbm", "kernel": "k_attn_tile_batched",
                               "achieved": attn_bytes / (attn_us / 1e6) / 1e9, "peak": peak_h,
                               "unit": "GB/s", "frac": attn_bytes / (attn_us / 1e6) / 1e9 / peak_h,
                               "avg_launch_us": attn_us, "bytes_per_launch": attn_bytes},
    }
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------- main
def main():
    args = parse()
    if args.impl == "reference":
        return run_reference(args)
    import torch
    import torch.distributed as dist
    from cross_loop_sparse_step_b200 import configs, fl, synth

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local))
    if configs.CONFIGS[args.config].get("decode"):
        return run_decode(args, configs.CONFIGS[args.config])
    cfg = apply_variant(configs.CONFIGS[args.config], args.variant)
    W = build_workload(cfg, fl, torch, synth, configs, seed=rank, n_layers=args.layers)
    R, N = W["R"], W["N"]
    stream = torch.cuda.current_stream()

    for _ in range(args.warmup):
        restore(W)
        step_loops(W)
    torch.cuda.synchronize()
    st = fl.check_device_status()
    if st != 0:
        raise RuntimeError(f"warm-up reported {fl.status_str(st)}")

    # per-kernel events for the roofline: the library records them around every GEMM
    # (kind 0) and attention (kind 1) launch of a step
    lib = fl.lib_handle()
    lib.fl_set_timing_events.argtypes = [ctypes.c_int32, ctypes.c_void_p, ctypes.c_void_p,
                                         ctypes.c_int32]
    lib.fl_timing_recorded.restype = ctypes.c_int32
    lib.fl_launch_count.restype = ctypes.c_int64
    per_step = {0: 4 * W["L"] * (R - 1), 1: W["L"] * (R - 1)}
    reps = 1 if args.graph else args.steps
    ev = {}
    for kind in (0, 1):
        n = per_step[kind] * reps
        b = [torch.cuda.Event(enable_timing=True) for _ in range(n)]
        e = [torch.cuda.Event(enable_timing=True) for _ in range(n)]
        for x in b + e:
            x.record(stream)   # materialise the handles
        ev[kind] = (b, e, (ctypes.c_void_p * n)(*[x.cuda_event for x in b]),
                    (ctypes.c_void_p * n)(*[x.cuda_event for x in e]))
    torch.cuda.synchronize()

    def arm_hooks():
        for kind in (0, 1):
            lib.fl_set_timing_events(kind, ev[kind][2], ev[kind][3], len(ev[kind][0]))

    def disarm_hooks():
        for kind in (0, 1):
            lib.fl_set_timing_events(kind, None, None, 0)

    simt_captured = 0
    attn_paths_step = None   # attention calls of one step by kernel path
    graph = None        # the timed step
    graph_h = None      # the same step with kernel events (per-kernel times, replayed apart:
    kernels_per_step = None   # event nodes between kernels would hold back their overlap)
    if args.graph:
        restore(W)
        torch.cuda.synchronize()
        c0 = lib.fl_launch_count()
        lib.fl_gemm_bf16_cuda_core_count.restype = ctypes.c_int64
        s0 = lib.fl_gemm_bf16_cuda_core_count()
        p0 = fl.attn_path_counts()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            step_loops(W)
        kernels_per_step = lib.fl_launch_count() - c0
        simt_captured = lib.fl_gemm_bf16_cuda_core_count() - s0
        attn_paths_step = {k: v - p0[k] for k, v in fl.attn_path_counts().items() if v - p0[k]}
        restore(W)
        torch.cuda.synchronize()
        arm_hooks()
        graph_h = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph_h):
            step_loops(W)
        disarm_hooks()
        for g in (graph, graph_h):
            for _ in range(2):
                restore(W)
                g.replay()
        torch.cuda.synchronize()
        st = fl.check_device_status()
        if st != 0:
            raise RuntimeError(f"graph warm-up reported {fl.status_str(st)}")

    gpu = torch.cuda.get_device_properties(local)
    uuid = getattr(gpu, "uuid", None)
    clocks = ClockSampler(f"GPU-{uuid}" if uuid else None)
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    kern_ms = {0: [], 1: []}
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    clocks.start()
    time.sleep(0.3)
    launches0 = lib.fl_launch_count()
    lib.fl_gemm_bf16_cuda_core_count.restype = ctypes.c_int64
    simt0 = lib.fl_gemm_bf16_cuda_core_count()
    if not args.graph:
        arm_hooks()
    for i in range(args.steps):
        restore(W)
        torch.cuda.nvtx.range_push("timed_step")   # lets a profiler select the timed work
        starts[i].record(stream)
        if graph is not None:
            graph.replay()
        else:
            step_loops(W)
        ends[i].record(stream)
        torch.cuda.nvtx.range_pop()
    torch.cuda.synchronize()
    if not args.graph:
        disarm_hooks()
        for kind in (0, 1):
            kern_ms[kind] = [x.elapsed_time(y) for x, y in zip(ev[kind][0], ev[kind][1])]
    launches = (lib.fl_launch_count() - launches0) if graph is None else kernels_per_step * args.steps
    simt_launches = lib.fl_gemm_bf16_cuda_core_count() - simt0   # eager steps; a graph
    if graph is not None:                                         # replays captured ones
        simt_launches = simt_captured * args.steps
    clk = clocks.stop()
    if graph_h is not None:   # per-kernel times: the instrumented step, replayed as often
        for i in range(args.steps):
            restore(W)
            graph_h.replay()
            torch.cuda.synchronize()
            for kind in (0, 1):
                kern_ms[kind] += [x.elapsed_time(y) for x, y in zip(ev[kind][0], ev[kind][1])]
    if world > 1:
        dist.barrier()
    st = fl.check_device_status()
    if st != 0:
        raise RuntimeError(f"timed steps reported {fl.status_str(st)}")
    step_ms = [s.elapsed_time(e) for s, e in zip(starts, ends)]
    t_rank = sum(step_ms) / 1e3
    value, t_max, tokens = aggregate(t_rank, N * (R - 1) * args.steps,
                                     dist if world > 1 else None, device="cuda")

    # rooflines of the projection GEMMs and of the sparse attention; the one with the
    # larger share of the step is the line's "roofline"
    pk, pk_kind = peaks()
    gemm_s = sum(kern_ms[0]) / 1e3
    gemm_tflops = gemm_flops_per_step(W) * args.steps / gemm_s / 1e12
    peak_t = pk.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"])
    peak_tb = pk.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
    # the four projections of a layer are recorded in order: QKV, O, gate/up, down
    d_, F_ = W["d"], W["F"]
    proj = {"qkv": 3 * d_ * d_, "o": d_ * d_, "gate_up": 2 * F_ * d_, "down": F_ * d_}
    rows_per_launch = [W["n_active"][r] for r in range(2, R + 1) for _ in range(W["L"])]
    per_gemm = {}
    for j, (name, macs_per_row) in enumerate(proj.items()):
        ms = kern_ms[0][j::4]
        rows = (rows_per_launch * args.steps)[:len(ms)]
        per_gemm[name] = {"avg_us": round(sum(ms) / len(ms) * 1e3, 2),
                          "tflops": round(sum(2 * macs_per_row * n for n in rows)
                                          / (sum(ms) / 1e3) / 1e12, 1)}
    attn_ms = kern_ms[1]
    abytes = attention_bytes_per_launch(W, torch)
    per_loop_launch = W["L"] * args.steps
    attn_bytes_total = sum(abytes[r][0] for r in abytes) * per_loop_launch
    attn_exec_total = sum(abytes[r][2] for r in abytes) * per_loop_launch
    attn_alg_flops = sum(abytes[r][1] for r in abytes) * per_loop_launch
    attn_s = sum(attn_ms) / 1e3
    attn_gbs = attn_bytes_total / attn_s / 1e9
    peak_h = pk.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"])
    step_total_ms = sum(step_ms)
    kvb, dense = kv_bytes(W)
    timing_note = ("per-kernel times from CUDA events around each launch in a separate, "
                   "instrumented replay of the step: upper bounds (the event records hold back "
                   "the overlap of consecutive kernels)")
    gemm_line = {"bound": "tensor", "kernel": "k_gemm_tc (projection GEMMs, tcgen05)",
                 "achieved": gemm_tflops, "peak": peak_t, "unit": "TFLOP/s",
                 "frac": gemm_tflops / peak_t, "frac_of_burst": gemm_tflops / peak_tb,
                 "traffic": None, "peak_source": f"{pk_kind} bf16 sustained",
                 "share_of_step": gemm_s * 1e3 / step_total_ms, "per_gemm": per_gemm,
                 "timing": timing_note}
    all_sparse = all(abytes[r][3] for r in abytes)
    if all_sparse:
        tr = ATTN_TRAFFIC.get(cfg["name"]) if cfg.get("variant", "flashloop") == "flashloop" else None
        attn_line = {"bound": "hbm", "kernel": "sparse attention call: k_kv_stage + k_sel_bitmap + "
                     "k_attn_tile (tcgen05, carried mass)",
                     "achieved": attn_gbs, "peak": peak_h, "unit": "GB/s",
                     "frac": attn_gbs / peak_h,
                     "traffic": tr["bytes"] if tr and tr.get("current", True) else None,
                     "traffic_detail": tr, "peak_source": f"{pk_kind} HBM copy"}
    else:   # dense attention in some timed loop: tensor-bound on its algorithmic FLOP
        attn_line = {"bound": "tensor", "kernel": "k_attn_tile / k_attn_dense_tile (tcgen05)",
                     "achieved": attn_alg_flops / attn_s / 1e12, "peak": peak_t,
                     "unit": "TFLOP/s", "frac": attn_alg_flops / attn_s / 1e12 / peak_t,
                     "traffic": None, "peak_source": f"{pk_kind} bf16 sustained (fp16 same rate)",
                     "hbm_gbs": attn_gbs}
    attn_line.update({
        "bytes_per_launch": {str(r): abytes[r][0] for r in abytes},
        "avg_launch_us": attn_s / len(attn_ms) * 1e6,
        "share_of_step": attn_s * 1e3 / step_total_ms,
        "algorithmic_tflops": attn_alg_flops / attn_s / 1e12,
        "executed_tflops": attn_exec_total / attn_s / 1e12,
        "executed_over_algorithmic_flops": attn_exec_total / max(attn_alg_flops, 1),
        "timing": timing_note})
    attn_dominant = attn_s > gemm_s
    loop_ms = step_total_ms / args.steps
    prefill = {"tokens_per_s": N / ((W["loop1_ms"] + loop_ms) / 1e3),
               "loop1_ms": round(W["loop1_ms"], 3), "loop1_cold_ms": round(W["loop1_cold_ms"], 3),
               "sparse_loops_ms": round(loop_ms, 3),
               "definition": "N / (t_1 + t_2 + ... + t_R), the dense loop 1 timed warm"}
    knobs = {k: os.environ.get(k) for k in ("FL_PDL", "FL_GEMM_SK", "FL_GEMM_BN", "FL_ATTN_TILE")}
    weights_gb = W["L"] * 2 * (4 * W["d"] ** 2 + 3 * W["d"] * W["F"]) / 1e9

    e2e = None
    if not args.no_e2e:
        h_host = W["snap"][0].cpu().pin_memory()
        x_host = W["snap"][1].cpu().pin_memory()
        out_host = torch.empty_like(h_host).pin_memory()
        torch.cuda.synchronize()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.steps):
            W["run"].h.copy_(h_host, non_blocking=True)
            W["run"].x_prev.copy_(x_host, non_blocking=True)
            if graph is not None:
                graph.replay()
            else:
                step_loops(W)
            out_host.copy_(W["run"].h, non_blocking=True)
        e1.record(stream)
        torch.cuda.synchronize()
        te = e0.elapsed_time(e1) / 1e3
        v_e2e, _, _ = aggregate(te, N * (R - 1) * args.steps, dist if world > 1 else None,
                                device="cuda")
        e2e = {"value": v_e2e, "unit": "tokens/s",
               "h2d_bytes_per_step": int(h_host.numel() * 4 + x_host.numel() * 4),
               "d2h_bytes_per_step": int(out_host.numel() * 4)}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        n_layers, rows = oracle_sample_size(cfg)
        sample = OracleSample(cfg, n_layers=n_layers, rows=rows, seed=1)
        per_loop, measured, desc = sample.run()
        cpu = {"value": N / per_loop, "unit": "tokens/s", "cores": blas_threads(),
               "kind": "oracle", "sample": desc, "measured_s": round(measured, 2),
               "extrapolated": True}

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": t_max / args.steps * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": cfg["name"], "n_tok": N, "d_model": W["d"],
                       "heads": f"{W['H']}x{W['hd']}", "d_ffn": W["F"], "layers": W["L"],
                       "loops": R, "timed_loops": list(range(2, R + 1)),
                       "active_tokens": W["n_active"][2], "col_k": cfg["col_k"][2],
                       "res_bits": cfg["res_bits"][2], "group": cfg["group"],
                       "variant": cfg.get("variant", "flashloop"),
                       "parallelism": f"replicas x{world}",
                       "l2": f"inputs larger than L2 ({weights_gb:.2f} GB of bf16 weights "
                             "read per loop step)"},
            "roofline": attn_line if attn_dominant else gemm_line,
            "other_roofline": gemm_line if attn_dominant else attn_line,
            "prefill_e2e": prefill,
            "cpu_baseline": cpu,
            "e2e": e2e,
            "gpu_launches": int(launches),
            "launch_mode": "cuda-graph replay" if graph is not None else "eager",
            "clocks": clk,
            "gemm_bf16_cuda_core_launches": int(simt_launches),
            "attention_paths_per_step": attn_paths_step,
            "knobs": knobs,
            "kv_bytes_per_token_per_layer": kvb,
            "kv_dense_bytes_per_token_per_layer": dense,
            "kv_reduction": dense / kvb,
            "step_ms": [round(x, 3) for x in step_ms],
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
