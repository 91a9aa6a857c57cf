"""Cross-loop KV store of one layer in the pages' quantisation scheme (oracle; test
infrastructure only).

Pages: FlashLoop paper Appendix E "Quantization Setting" (INT4 asymmetric group-wise
quantisation with scale and offset from each group's minimum and maximum, groups of 64,
post-RoPE keys per channel and values per token, the most recent 64 tokens kept in
BF16; in sparse loops the active tokens' K/V are packed as cross-loop residuals and
quantised with the same scheme), §3.3 (base state plus residual updates), §4.3
(residuals only for active tokens).

Readings (the pages leave them open):
  * loop 1 quantises every token; loop r >= 2 quantises, for its active tokens, the
    residual x = fl32(k - K^_{r-1}) against the reconstructed previous state and
    K^_r = fl32(K^_{r-1} + deq) - the same closed loop as the store's own codec;
  * a loop's rows are its tokens in ascending order (all tokens at loop 1); a key group
    is 64 consecutive rows of one (head, channel) among the rows outside the window, a
    trailing shorter group taking its own minimum and maximum; a value group is 64
    consecutive channels of one (row, head);
  * the window is the last 64 positions of the sequence; a window token is stored as
    the bfloat16 rounding of its value (loop 1: of k; a loop that recomputes it: of the
    new k, replacing the previous state) and is in no group;
  * scale and offset: the store codec's directed-rounding binary16 pair
    (``codec.quantize_groups``); codes are 4-bit.
"""
import numpy as np

from . import codec
from .diagnostics import bf16_f32

BITS = 4
GROUP = 64
WINDOW = 64


def _quant_k(x):
    """Keys [rows, H, hd] per channel over groups of GROUP consecutive rows ->
    (codes uint8 [rows, H, hd], s, z [n_groups, H, hd] float16, deq float32)."""
    n, H, hd = x.shape
    t = np.ascontiguousarray(x.transpose(1, 2, 0))            # [H, hd, rows]
    ng = (n + GROUP - 1) // GROUP
    codes = np.zeros((H, hd, n), np.uint8)
    deq = np.zeros((H, hd, n), np.float32)
    s = np.zeros((ng, H, hd), np.float16)
    z = np.zeros((ng, H, hd), np.float16)
    for gi in range(ng):
        sl = slice(gi * GROUP, min(n, (gi + 1) * GROUP))
        c, sg, zg, dg, err = codec.quantize_groups(t[..., sl], BITS)
        assert not err.any(), "scale or offset outside binary16"
        codes[..., sl], deq[..., sl], s[gi], z[gi] = c, dg, sg, zg
    return codes.transpose(2, 0, 1).copy(), s, z, deq.transpose(2, 0, 1).copy()


def _quant_v(x):
    """Values [rows, H, hd] per token over groups of GROUP channels."""
    n, H, hd = x.shape
    c, s, z, d, err = codec.quantize_groups(x.reshape(n, H, hd // GROUP, GROUP), BITS)
    assert not err.any(), "scale or offset outside binary16"
    return c.reshape(n, H, hd), s, z, d.reshape(n, H, hd)


class LayerKVPages:
    """K and V (index 0 and 1) of one layer for loops 1..n_loops in the pages' scheme."""

    def __init__(self, n_tok, n_heads, head_dim, n_loops):
        assert head_dim % GROUP == 0
        self.n_tok, self.H, self.hd, self.n_loops = n_tok, n_heads, head_dim, n_loops
        self.win0 = max(n_tok - WINDOW, 0)   # first window position
        self.store = {}   # (loop, kv) -> dict(q_rows, codes, s, z, w_rows, w_vals)
        self.rows = {}    # loop -> token ids ascending
        self.hat = {}     # loop -> float32 [2, n_tok, H, hd]

    def _encode(self, kv, tokens, x):
        """x float32 [len(tokens), H, hd] (tokens ascending) -> the stored entry and the
        reconstruction of those rows."""
        inwin = tokens >= self.win0
        q = ~inwin
        rec = np.empty_like(x)
        entry = {"q_rows": tokens[q].copy(), "w_rows": tokens[inwin].copy(),
                 "w_vals": bf16_f32(x[inwin])}
        rec[inwin] = entry["w_vals"]
        if q.any():
            c, s, z, d = (_quant_k if kv == 0 else _quant_v)(x[q])
            entry.update(codes=c, s=s, z=z)
            rec[q] = d
        return entry, rec

    def write_base(self, k, v):
        tok = np.arange(self.n_tok, dtype=np.int64)
        hat = np.empty((2, self.n_tok, self.H, self.hd), np.float32)
        for kv, x in enumerate((k, v)):
            entry, rec = self._encode(kv, tok, np.asarray(x, np.float32))
            self.store[(1, kv)] = entry
            hat[kv] = rec
        self.rows[1] = tok
        self.hat[1] = hat

    def write_residual(self, r, act_tok, k, v):
        """Loop r >= 2: the active tokens (ascending) with their new k, v [n_act, H, hd]."""
        act = np.asarray(act_tok, np.int64)
        prev = self.hat[r - 1]
        hat = prev.copy()
        for kv, x in enumerate((k, v)):
            x = np.asarray(x, np.float32)
            inwin = act >= self.win0
            resid = (x - prev[kv][act]).astype(np.float32)
            # window tokens store their new value; the others the residual
            entry, rec = self._encode(kv, act, np.where(inwin[:, None, None], x, resid))
            self.store[(r, kv)] = entry
            new = np.where(inwin[:, None, None], rec, (prev[kv][act] + rec).astype(np.float32))
            hat[kv][act] = new
        self.rows[r] = act
        self.hat[r] = hat

    def _decode(self, r, kv):
        """The loop's stored rows decoded: {token: values} as (tokens, values)."""
        e = self.store[(r, kv)]
        toks = [e["w_rows"]]
        vals = [e["w_vals"]]
        if len(e["q_rows"]):
            c = e["codes"].astype(np.float32)
            if kv == 0:
                gi = np.arange(len(e["q_rows"])) // GROUP
                s = e["s"][gi].astype(np.float32)
                z = e["z"][gi].astype(np.float32)
            else:
                n, H, hd = c.shape
                s = np.repeat(e["s"].astype(np.float32), GROUP, axis=-1).reshape(n, H, hd)
                z = np.repeat(e["z"].astype(np.float32), GROUP, axis=-1).reshape(n, H, hd)
            toks.append(e["q_rows"])
            vals.append(codec.fma_f32(c, s, z))
        return np.concatenate(toks), np.concatenate(vals)

    def reconstruct(self, r):
        """K^_r, V^_r of every token rebuilt from the stored codes, scales and window
        values by walking base -> loop 2 -> ... -> loop r (independent of ``hat``)."""
        out = np.empty((2, self.n_tok, self.H, self.hd), np.float32)
        for kv in range(2):
            tok, val = self._decode(1, kv)
            cur = np.empty((self.n_tok, self.H, self.hd), np.float32)
            cur[tok] = val
            for rr in range(2, r + 1):
                tok, val = self._decode(rr, kv)
                win = tok >= self.win0
                cur[tok[win]] = val[win]
                cur[tok[~win]] = (cur[tok[~win]] + val[~win]).astype(np.float32)
            out[kv] = cur
        return out

    def nbytes(self, r):
        """Bytes loop r stores for K and V: 4-bit codes, binary16 (scale, offset) pairs
        per group, bfloat16 window values."""
        tot = 0
        for kv in range(2):
            e = self.store[(r, kv)]
            nq = len(e["q_rows"])
            tot += nq * self.H * self.hd // 2
            if nq:
                tot += e["s"].size * 4          # a binary16 pair per group
            tot += len(e["w_rows"]) * self.H * self.hd * 2
        return tot
