"""Helpers of the GPU parity tests: tolerance checks, uploading oracle-built KV stores
and statistics (oracle -> GPU only), and the tie-band rule for column selections."""
import numpy as np
import torch

from oracle import attention as oatt

# Float tolerance of the GPU path against the fp64 oracle on identical inputs:
# max-abs error <= 2e-2 and relative L1 error sum|g - o| / sum|o| <= 5e-3.
MAX_ABS = 2e-2
REL_L1 = 5e-3


def assert_close(got, want, max_abs=MAX_ABS, rel_l1=REL_L1, what=""):
    got = np.asarray(got, np.float64)
    want = np.asarray(want, np.float64)
    assert got.shape == want.shape, (what, got.shape, want.shape)
    assert np.all(np.isfinite(got)), what
    err = np.abs(got - want)
    ma = float(err.max()) if err.size else 0.0
    den = float(np.abs(want).sum())
    rl = float(err.sum() / den) if den > 0 else float(err.sum())
    assert ma <= max_abs and rl <= rel_l1, f"{what}: max_abs {ma:.3e} rel_l1 {rl:.3e}"
    return ma, rl


def dev(a, dtype=None):
    t = torch.from_numpy(np.ascontiguousarray(a)).cuda()
    return t if dtype is None else t.to(dtype)


def host(t):
    return t.detach().cpu().numpy()


def upload_store(ost, store, upto):
    """Copy the oracle store's loops 1..upto into a GPU KVStore (same layout)."""
    for r in range(1, upto + 1):
        if r not in ost.rows:
            continue
        for kv in range(2):
            codes = ost.codes[(r, kv)]
            dst = store.codes[(r, kv)]
            raw = np.ascontiguousarray(codes).view(np.uint8).reshape(codes.shape[0], codes.shape[1], -1)
            dst[: raw.shape[0]].copy_(torch.from_numpy(raw))
            if ost.sz[(r, kv)] is not None:
                store.sz[(r, kv)][: raw.shape[0]].copy_(torch.from_numpy(ost.sz[(r, kv)]))
    store.slot.copy_(torch.from_numpy(ost.slot))
    if store.vnorm is not None:
        vh = ost.hat[upto][1].astype(np.float64)
        store.vnorm.copy_(torch.from_numpy(np.sqrt((vh ** 2).sum(-1)).astype(np.float32)))


def sel_to_host(t):
    return host(t).view(np.uint16)


def sel_to_dev(S):
    return torch.from_numpy(np.ascontiguousarray(S).view(np.int16)).cuda()


def check_selection(S_gpu, S_or, c_fn, band=1e-5):
    """Compare ascending column sets row by row. A row may differ only where every
    differing column's statistic lies within a relative ``band`` of the row's k-th
    largest statistic (a near-tie that fp32 and fp64 may break differently).
    ``c_fn(h, row)`` returns {column: statistic} from the oracle. Returns the list of
    (h, row) that differ within the band; raises on any other difference."""
    H, n, _ = S_or.shape
    ties = []
    for h in range(H):
        for i in range(n):
            a = S_gpu[h, i]
            b = S_or[h, i]
            if np.array_equal(a, b):
                continue
            ga = set(a[a != oatt.SENTINEL].tolist())
            gb = set(b[b != oatt.SENTINEL].tolist())
            assert len(ga) == len(gb), (h, i, sorted(ga), sorted(gb))
            c = c_fn(h, i)
            kept = sorted((c[j] for j in gb if j != 0), reverse=True)
            thr = kept[-1]
            for j in ga ^ gb:
                assert abs(c[j] - thr) <= band * abs(thr), (h, i, j, c[j], thr)
            ties.append((h, i))
    return ties
