"""Residual-vs-full quantisation of per-loop KV on the GPU (FlashLoop §3.3, Figure 2c:
quantising the cross-loop change loses less than quantising each loop's KV in full at
the same bit width; §5.3.1 Table 2 uses per-loop full quantisation as the ablation).

For a sequence of per-loop K (or V) of n tokens it writes, through the library's own
quantiser, (a) the residual chain - an 8-bit base at loop 1 and b-bit residuals of every
token against the reconstructed previous loop - and (b) every loop quantised in full with
b bits (a store whose loop-1 base holds zeros in binary32, so the b-bit residual of
loop 2 is the loop's KV itself); it reads both back with fl_kv_reconstruct and reports
the relative reconstruction error ||K^_r - K_r||_F / ||K_r||_F per loop and the stored
bytes per token per loop.

Usage: python -m cross_loop_sparse_step_b200.diagnose [--tokens N] [--loops R] [--bits b]
"""
import argparse
import json
import os
import sys

import torch

from cross_loop_sparse_step_b200 import fl


def _rel(a, b):
    a64, b64 = a.double(), b.double()
    return float(torch.linalg.vector_norm(a64 - b64) / torch.linalg.vector_norm(b64))


def residual_vs_full(K, bits, group, base_bits=8):
    """K: list of device float32 [n, H, hd] tensors (loop 1 first). Returns per-loop
    errors of the residual chain and of full b-bit quantisation, their reconstructions
    and the bytes per token each stores per loop."""
    R = len(K)
    n, H, hd = K[0].shape
    dev = K[0].device
    tok = torch.arange(n, dtype=torch.int32, device=dev)
    rows = {r: n for r in range(2, R + 1)}
    chain = fl.KVStore(n, H, hd, group, base_bits, {r: bits for r in range(2, R + 1)}, R, rows,
                       device=dev)
    out = {"residual": {}, "full": {}, "hat_residual": {}, "hat_full": {},
           "bytes_per_token": {"residual": {}, "full": {}}}
    for r in range(1, R + 1):
        if r == 1:
            fl.kv_residual_quant(chain, 1, K[0], K[0])
        else:
            fl.kv_residual_quant(chain, r, K[r - 1], K[r - 1], tok)
        hk, _ = fl.kv_reconstruct(chain, r, tok)
        out["hat_residual"][r] = hk
        out["residual"][r] = _rel(hk, K[r - 1])
        out["bytes_per_token"]["residual"][r] = chain.nbytes(r) / (2 * n)
        # full quantisation of this loop alone
        full = fl.KVStore(n, H, hd, group, 0, {2: bits}, 2, {2: n}, device=dev, vnorm=False)
        zero = torch.zeros_like(K[r - 1])
        fl.kv_residual_quant(full, 1, zero, zero)
        fl.kv_residual_quant(full, 2, K[r - 1], K[r - 1], tok)
        fk, _ = fl.kv_reconstruct(full, 2, tok)
        out["hat_full"][r] = fk
        out["full"][r] = _rel(fk, K[r - 1])
        out["bytes_per_token"]["full"][r] = full.nbytes(2) / (2 * n)
    st = fl.check_device_status()
    if st != 0:
        raise fl.FLError(st, "residual_vs_full")
    return out


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--tokens", type=int, default=8192)
    ap.add_argument("--heads", type=int, default=16)
    ap.add_argument("--head-dim", type=int, default=128)
    ap.add_argument("--loops", type=int, default=4)
    ap.add_argument("--bits", type=int, default=4)
    ap.add_argument("--group", type=int, default=32)
    ap.add_argument("--delta", type=float, default=0.25)
    ap.add_argument("--seed", type=int, default=0)
    a = ap.parse_args()
    from cross_loop_sparse_step_b200 import synth
    K = synth.kv_loop_sequence(synth.rng(a.seed), a.tokens, a.heads, a.head_dim, a.loops,
                               delta=a.delta)
    Kd = [torch.from_numpy(k).cuda() for k in K]
    res = residual_vs_full(Kd, a.bits, a.group)
    line = {"diagnostic": "residual vs full quantisation of per-loop KV",
            "tokens": a.tokens, "heads": a.heads, "head_dim": a.head_dim, "loops": a.loops,
            "bits": a.bits, "group": a.group, "base_bits": 8,
            "change_std": {r: a.delta * 0.5 ** (r - 2) for r in range(2, a.loops + 1)},
            "rel_error": {"residual": res["residual"], "full": res["full"]},
            "bytes_per_token_per_loop": res["bytes_per_token"]}
    print(json.dumps(line))
    return 0


if __name__ == "__main__":
    sys.exit(main())
