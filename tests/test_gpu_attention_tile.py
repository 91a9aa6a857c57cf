"""GPU parity of the query-tile tensor-core form of the sparse attention.

fl_sparse_loop_attn takes this form for head_dim 128 over a quantised store when the
call writes no statistics (none requested, or updated in place with an unchanged
budget) - the form every sparse loop of fl_loop_step uses on the workloads. Each case
compares the output with the oracle's sparse attention on identical inputs at max-abs
2e-2 and relative L1 5e-3: ragged tiles (fewer queries than a tile, one query past a
tile), groups of 32 and 64, 2/4/8-bit residual chains up to 15 loops deep, fp32 and
bf16 queries and outputs, queries whose set is their whole prefix, and the 4K and 32K
workload shapes on sampled queries. Column sets are synthetic here (sink, biased
columns, random others), so the oracle evaluates only the sampled queries."""
import numpy as np
import pytest
import torch

from cross_loop_sparse_step_b200 import synth
from oracle import attention as oatt
from tests.gpu_helpers import assert_close, dev, host, sel_to_dev, sel_to_host, upload_store
from tests.test_gpu_configs import _nested_sets, _stats, _store

pytestmark = pytest.mark.gpu

CASES = [
    # name, n_tok, H, g, loops, bits per residual loop, active counts, k, bias, sample, q/out bf16
    ("ragged-37", 512, 2, 32, 4, {2: 4, 3: 4, 4: 4}, {2: 200, 3: 100, 4: 37}, 40, True, None, False),
    ("two-tiles-129-g64", 300, 3, 64, 3, {2: 8, 3: 2}, {2: 150, 3: 129}, 16, False, None, False),
    ("bf16-256", 1024, 4, 32, 2, {2: 2}, {2: 256}, 64, True, None, True),
    ("4k-shape", 4096, 16, 32, 4, {2: 4, 3: 4, 4: 4}, {2: 820, 3: 820, 4: 820}, 82, True, 48, True),
    ("8k-R16-chains", 8192, 16, 64, 16, {r: 2 for r in range(2, 17)},
     {r: max(410, int(4096 * 0.8 ** (r - 2))) for r in range(2, 17)}, 512, True, 32, True),
    ("32k-shape", 32768, 16, 32, 2, {2: 2}, {2: 4916}, 2048, True, 24, True),
]
# the same with the statistics stride padded to a multiple of 8 (16-byte rows: the sets
# are read 8 entries per load, the layout the loop step allocates)
PADDED = {"bf16-256", "4k-shape", "32k-shape", "ragged-37"}
CASES = [c + (False,) for c in CASES] + [(c[0] + "-stride8",) + c[1:] + (True,) for c in CASES
                                         if c[0] in PADDED]


@pytest.mark.parametrize("name,n,H,g,R,bits,counts,k,use_bias,sample,bf16,pad", CASES,
                         ids=[c[0] for c in CASES])
def test_tile_attention_matches_oracle(name, n, H, g, R, bits, counts, k, use_bias, sample, bf16,
                                       pad):
    from cross_loop_sparse_step_b200 import fl
    hd = 128
    rs = synth.rng(7000 + n + R + k)
    sets = _nested_sets(rs, n, counts, R)
    ost = _store(rs, n, H, hd, g, bits, sets, R)
    store = fl.KVStore(n, H, hd, g, 8, bits, R, {r: counts[r] for r in range(2, R + 1)})
    upload_store(ost, store, R)
    bias_cols = synth.biased_columns(rs, n, 0.02)
    bias = None
    if use_bias:
        bias = np.zeros(n, np.float32)
        bias[bias_cols] = 4.0
        bias[0] = 4.0
    act = sets[R]
    pick = np.arange(len(act)) if sample is None else \
        np.sort(rs.choice(len(act), size=sample, replace=False))
    # random sets for the checked queries (and for a few early tokens whose set is their
    # whole prefix), evenly spaced sets for the others
    S, m, u = _stats(rs, n, H, hd, k, act, bias_cols, act[pick])
    if pad:
        Sp = np.full(S.shape[:2] + ((k + 1 + 7) // 8 * 8,), 0xFFFF, S.dtype)
        Sp[..., : S.shape[2]] = S
        S = Sp
    q = synth.query_values(rs, len(act), H, hd)
    tdt = torch.bfloat16 if bf16 else torch.float32
    if bf16:
        q = synth.round_bf16(q)
    out = torch.full((len(act), H, hd), float("nan"), dtype=tdt, device="cuda")
    fl.sparse_loop_attn(dev(q, tdt), dev(act), store, R, out,
                        col_bias=dev(bias) if bias is not None else None,
                        sel=sel_to_dev(S), mass=dev(m), unsel=dev(u))
    st = fl.check_device_status()
    assert st == 0, fl.status_str(st)
    qa = act[pick]
    Kh, Vh = ost.hat[R]
    o = oatt.sparse_attention(q[pick].astype(np.float64), qa, qa, Kh, Vh, S,
                              m.astype(np.float64), u.astype(np.float64), bias)
    got = host(out.float())[pick]
    assert_close(got, o, what=f"{name}: o")


def test_tile_attention_in_place_unchanged_statistics():
    """In place with an unchanged budget (the loop step's sparse loops): the output
    matches and the carried statistics are left exactly as they were."""
    from cross_loop_sparse_step_b200 import fl
    n, H, hd, g, R, k = 2048, 8, 128, 32, 3, 96
    rs = synth.rng(7100)
    counts = {2: 600, 3: 410}
    bits = {2: 4, 3: 4}
    sets = _nested_sets(rs, n, counts, R)
    ost = _store(rs, n, H, hd, g, bits, sets, R)
    store = fl.KVStore(n, H, hd, g, 8, bits, R, counts)
    upload_store(ost, store, R)
    act = sets[R]
    bias_cols = synth.biased_columns(rs, n, 0.02)
    S, m, u = _stats(rs, n, H, hd, k, act, bias_cols, act)
    Sd, md, ud = sel_to_dev(S), dev(m), dev(u)
    q = synth.query_values(rs, len(act), H, hd)
    out = torch.zeros(len(act), H, hd, device="cuda")
    fl.sparse_loop_attn(dev(q), dev(act), store, R, out, sel=Sd, mass=md, unsel=ud, k_next=k,
                        sel_out=Sd, mass_out=md, unsel_out=ud)
    assert fl.check_device_status() == 0
    o = oatt.sparse_attention(q.astype(np.float64), act, act, *ost.hat[R], S,
                              m.astype(np.float64), u.astype(np.float64), None)
    assert_close(host(out), o, what="o")
    assert np.array_equal(sel_to_host(Sd), S)
    assert np.array_equal(host(md), m) and np.array_equal(host(ud), u)


def test_tile_attention_reports_columns_past_the_query():
    """A carried column beyond the query's position is an input error: it is skipped and
    recorded as FL_ERR_RANGE, and the call still completes."""
    from cross_loop_sparse_step_b200 import fl
    n, H, hd, g = 256, 2, 128, 32
    rs = synth.rng(7200)
    sets = _nested_sets(rs, n, {2: 64}, 2)
    ost = _store(rs, n, H, hd, g, {2: 4}, sets, 2)
    store = fl.KVStore(n, H, hd, g, 8, {2: 4}, 2, {2: 64})
    upload_store(ost, store, 2)
    act = sets[2]
    S, m, u = _stats(rs, n, H, hd, 8, act, np.array([], np.int64), act)
    t = int(act[-1])
    if t + 1 < n:
        S[0, t, 1] = t + 1   # a column after the query
    q = synth.query_values(rs, len(act), H, hd)
    out = torch.zeros(len(act), H, hd, device="cuda")
    fl.sparse_loop_attn(dev(q), dev(act), store, 2, out, sel=sel_to_dev(S), mass=dev(m),
                        unsel=dev(u))
    st = fl.check_device_status()
    assert st == (6 if t + 1 < n else 0)
    assert torch.all(torch.isfinite(out))
