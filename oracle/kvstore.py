"""Cross-loop KV store of one layer: quantised base plus per-loop residuals (oracle).

Pages: FlashLoop §3.3 (the loop-wise KV cache is best kept as a quantised base
state plus quantised cross-loop residual updates), §4.1 (inactive tokens reuse the
previous loop's K/V; only active tokens write new K/V), §4.3 (residuals are
generated and stored only for active tokens), Appendix E (same scheme for base and
residuals).

Readings (the pages leave them open):
  * loop 1 quantises every token's post-RoPE k and v with ``base_bits``;
  * loop r >= 2 quantises, for its active tokens only, the residual
    x = fl32(k - K^_{r-1}) against the RECONSTRUCTED previous state (closed loop),
    and K^_r = fl32(K^_{r-1} + deq); other tokens keep K^_{r-1};
  * groups are ``group`` consecutive elements along head_dim, per token and head,
    for K and for V alike;
  * ``bits == 0`` stores binary32 values: the base holds k itself and a raw
    residual loop holds the new k itself (K^_r = k).

Layout, shared with the C interface because stores built here are uploaded to the
GPU for identical-input tests (the format is the interface, the code is not shared):
  base codes [n_tok][H][hd*b/8] uint8 (b = 0: [n_tok][H][hd] float32)
  base sz    [n_tok][H][hd/g][2] float16, pairs (scale, offset)
  loop r residual: the same per row, rows = the loop's active tokens ascending
  slot[r][t] = row of token t in loop r's arrays, or -1.
"""
import numpy as np

from . import codec


class LayerKV:
    """K and V (index 0 and 1) of one layer for loops 1..n_loops."""

    def __init__(self, n_tok, n_heads, head_dim, group, base_bits, res_bits, n_loops):
        assert head_dim % group == 0
        self.n_tok, self.H, self.hd, self.g = n_tok, n_heads, head_dim, group
        self.base_bits = base_bits
        self.res_bits = dict(res_bits)  # loop r -> bits
        self.n_loops = n_loops
        self.codes = {}   # (loop, kv) -> packed codes or float32 raw values
        self.sz = {}      # (loop, kv) -> float16 [rows, H, hd/g, 2] or None
        self.rows = {}    # loop -> token ids ascending
        self.slot = np.full((n_loops + 1, n_tok), -1, np.int32)  # row 0 unused
        self.hat = {}     # loop -> float32 [2, n_tok, H, hd] reconstructed K^, V^
        self.range_error = False

    # -- writing -----------------------------------------------------------
    def _encode(self, x, bits):
        """x float32 [rows, H, hd] -> (codes, sz, deq)."""
        if bits == 0:
            return x.copy(), None, x.copy()
        n, H, hd = x.shape
        xg = x.reshape(n, H, hd // self.g, self.g)
        c, s, z, deq, err = codec.quantize_groups(xg, bits)
        self.range_error |= bool(err.any())
        packed = codec.pack_codes(c.reshape(n, H, hd), bits)
        sz = np.stack([s, z], axis=-1)
        return packed, sz, deq.reshape(n, H, hd)

    def write_base(self, k, v):
        """Loop 1: every token. k, v float32 [n_tok, H, hd] post-RoPE."""
        hat = np.empty((2, self.n_tok, self.H, self.hd), np.float32)
        for kv, x in enumerate((k, v)):
            x = np.asarray(x, np.float32)
            codes, sz, deq = self._encode(x, self.base_bits)
            self.codes[(1, kv)] = codes
            self.sz[(1, kv)] = sz
            hat[kv] = deq
        self.rows[1] = np.arange(self.n_tok, dtype=np.int32)
        self.slot[1] = np.arange(self.n_tok, dtype=np.int32)
        self.hat[1] = hat

    def write_residual(self, r, act_tok, k, v):
        """Loop r >= 2: active tokens only (ascending). k, v float32 [n_act, H, hd]."""
        assert r >= 2 and (r - 1) in self.hat
        act_tok = np.asarray(act_tok, np.int32)
        bits = self.res_bits[r]
        prev = self.hat[r - 1]
        hat = prev.copy()
        for kv, x in enumerate((k, v)):
            x = np.asarray(x, np.float32)
            if bits == 0:
                codes, sz, newv = x.copy(), None, x.copy()
            else:
                resid = (x - prev[kv][act_tok]).astype(np.float32)
                codes, sz, deq = self._encode(resid, bits)
                newv = (prev[kv][act_tok] + deq).astype(np.float32)
            self.codes[(r, kv)] = codes
            self.sz[(r, kv)] = sz
            hat[kv][act_tok] = newv
        self.rows[r] = act_tok.copy()
        self.slot[r] = -1
        self.slot[r][act_tok] = np.arange(len(act_tok), dtype=np.int32)
        self.hat[r] = hat

    def append(self, r, tokens, k, v):
        """Decode: add ``tokens`` (new positions) to loop r without touching the other
        tokens. Loop 1 writes their base rows (row = token id); loop r >= 2 appends
        residual rows (against each token's loop r-1 reconstruction) after the existing
        rows. k, v float32 [n, H, hd]. The base arrays must already span the tokens."""
        tokens = np.asarray(tokens, np.int64)
        if r == 1:
            bits = self.base_bits
            for kv, x in enumerate((k, v)):
                x = np.asarray(x, np.float32)
                codes, sz, deq = self._encode(x, bits)
                self.codes[(1, kv)][tokens] = codes
                if sz is not None:
                    self.sz[(1, kv)][tokens] = sz
                self.hat[1][kv][tokens] = deq
            return
        bits = self.res_bits[r]
        prev = self.hat[r - 1]
        hat = self.hat[r]
        row0 = len(self.rows[r])
        for kv, x in enumerate((k, v)):
            x = np.asarray(x, np.float32)
            if bits == 0:
                codes, sz, newv = x.copy(), None, x.copy()
            else:
                resid = (x - prev[kv][tokens]).astype(np.float32)
                codes, sz, deq = self._encode(resid, bits)
                newv = (prev[kv][tokens] + deq).astype(np.float32)
            self.codes[(r, kv)] = np.concatenate([self.codes[(r, kv)], codes])
            if sz is not None:
                self.sz[(r, kv)] = np.concatenate([self.sz[(r, kv)], sz])
            hat[kv][tokens] = newv
        self.rows[r] = np.concatenate([self.rows[r], tokens.astype(np.int32)])
        self.slot[r][tokens] = row0 + np.arange(len(tokens), dtype=np.int32)

    def carry(self, r):
        """A loop that writes nothing for this layer keeps the previous state."""
        self.hat[r] = self.hat[r - 1]
        self.rows[r] = np.zeros(0, np.int32)
        self.slot[r] = -1

    # -- reading -----------------------------------------------------------
    def _decode_rows(self, loop, kv, rows):
        bits = self.base_bits if loop == 1 else self.res_bits[loop]
        codes = self.codes[(loop, kv)][rows]
        if bits == 0:
            return codes.astype(np.float32)
        return codec.dequantize(codes, self.sz[(loop, kv)][rows], bits, self.g, self.hd)

    def reconstruct(self, r, tokens):
        """K^_r, V^_r of ``tokens`` rebuilt from the stored codes by walking the
        chain base -> loop 2 -> ... -> loop r (independent of the ``hat`` cache)."""
        tokens = np.asarray(tokens, np.int64)
        out = np.empty((2, len(tokens), self.H, self.hd), np.float32)
        for kv in range(2):
            cur = self._decode_rows(1, kv, tokens)
            for rr in range(2, r + 1):
                if rr not in self.rows:
                    continue
                sl = self.slot[rr][tokens]
                on = sl >= 0
                if not on.any():
                    continue
                d = self._decode_rows(rr, kv, sl[on])
                if self.res_bits[rr] == 0:
                    cur[on] = d
                else:
                    cur[on] = (cur[on] + d).astype(np.float32)
            out[kv] = cur
        return out[0], out[1]

    def kv_bytes(self, r):
        """Bytes held for loop r (codes + scale/offset), K and V together."""
        total = 0
        for kv in range(2):
            total += self.codes[(r, kv)].nbytes
            if self.sz[(r, kv)] is not None:
                total += self.sz[(r, kv)].nbytes
        return total
