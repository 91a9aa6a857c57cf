"""Token selection of the cross-loop token-sparse update (oracle; fp64).

Pages: FlashLoop §4.1 "Cross-Loop Token-Sparse Updates": after the dense early
loops, each loop ranks the tokens updated in the preceding loop by their normalized
hidden-state change and keeps the top-k (k may vary with the loop); skipped tokens
produce no new change, so later selections are restricted to the previous active
set and the sets are nested. §3.1: high-change tokens are few and spread over the
context.

Readings:
  * normalized change d_t = ||h_{r-1,t} - h_{r-2,t}||_2 / max(||h_{r-2,t}||_2, 1e-30);
  * k_r = min(ceil(f_r * N), |A_{r-1}|) with f_r a fraction of all N prompt rows;
  * ties in d go to the smaller token index; the set is returned ascending.
"""
from fractions import Fraction
import math

import numpy as np


def normalized_change(h_cur, h_prev):
    h_cur = np.asarray(h_cur, np.float64)
    h_prev = np.asarray(h_prev, np.float64)
    num = np.sqrt(np.sum((h_cur - h_prev) ** 2, axis=-1))
    den = np.sqrt(np.sum(h_prev ** 2, axis=-1))
    return num / np.maximum(den, 1e-30)


def select_active(h_cur, h_prev, row_tok, k):
    """Rows of (h_cur, h_prev) belong to tokens ``row_tok`` (ascending; None means
    row i is token i). Returns (tokens ascending, their row positions, deltas)."""
    delta = normalized_change(h_cur, h_prev)
    n = delta.shape[0]
    pos = np.arange(n)
    order = np.lexsort((pos, -delta))
    keep = np.sort(order[:k])
    tok = keep if row_tok is None else np.asarray(row_tok)[keep]
    return tok.astype(np.int32), keep.astype(np.int32), delta


def active_count(frac, n_tok, n_prev):
    """k_r = min(ceil(f_r * N), |A_{r-1}|), with f_r read as the exact decimal."""
    k = math.ceil(Fraction(str(frac)) * n_tok)
    return int(min(max(k, 0), n_prev))
