"""The C-ABI library on the CPU: it loads without a GPU, exports every entry point that
include/fl.h declares, its structs have the layout the C compiler gives them (checked
against gcc), and host validation rejects bad arguments before anything is launched."""
import ctypes
import os
import re
import subprocess
import tempfile

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "fl.h")


def _declared():
    txt = open(HEADER).read()
    txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
    return sorted(set(re.findall(r"\b(fl_[a-z_]+)\s*\(", txt)))


def test_library_exports_every_declared_symbol():
    from cross_loop_sparse_step_b200 import fl
    names = _declared()
    assert len(names) >= 14
    out = subprocess.run(["nm", "-D", "--defined-only", fl.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r" T (fl_\w+)", out))
    missing = [n for n in names if n not in exported]
    assert not missing, missing
    for n in names:
        getattr(fl.lib_handle(), n)


_LAYOUT_C = r"""
#include <stdio.h>
#include <stddef.h>
#include "fl.h"
#define F(T, m) printf(#T "." #m " %zu\n", offsetof(T, m));
int main(void) {
  printf("fl_kv_desc %zu\n", sizeof(fl_kv_desc));
  F(fl_kv_desc, res_bits) F(fl_kv_desc, codes) F(fl_kv_desc, sz) F(fl_kv_desc, slot) F(fl_kv_desc, vnorm)
  printf("fl_attn_args %zu\n", sizeof(fl_attn_args));
  F(fl_attn_args, q_tok) F(fl_attn_args, kv) F(fl_attn_args, sel) F(fl_attn_args, stat_rows)
  F(fl_attn_args, q_row) F(fl_attn_args, k_next) F(fl_attn_args, out_stride) F(fl_attn_args, out)
  F(fl_attn_args, ws_bytes)
  printf("fl_layer_weights %zu\n", sizeof(fl_layer_weights));
  printf("fl_model %zu\n", sizeof(fl_model));
  F(fl_model, rms_eps) F(fl_model, layers) F(fl_model, col_bias)
  printf("fl_schedule %zu\n", sizeof(fl_schedule));
  F(fl_schedule, n_active) F(fl_schedule, col_k) F(fl_schedule, stat_kind)
  printf("fl_loop_state %zu\n", sizeof(fl_loop_state));
  F(fl_loop_state, act) F(fl_loop_state, act_pos) F(fl_loop_state, kv) F(fl_loop_state, sel_stride)
  F(fl_loop_state, ws) F(fl_loop_state, ws_bytes) F(fl_loop_state, taps)
  printf("fl_loop_taps %zu\n", sizeof(fl_loop_taps));
  F(fl_loop_taps, tok) F(fl_loop_taps, x_in) F(fl_loop_taps, attn) F(fl_loop_taps, x_out)
  return 0;
}
"""


def test_struct_layouts_match_c():
    from cross_loop_sparse_step_b200 import fl
    with tempfile.TemporaryDirectory() as d:
        src = os.path.join(d, "layout.c")
        exe = os.path.join(d, "layout")
        open(src, "w").write(_LAYOUT_C)
        subprocess.run(["gcc", "-I", os.path.join(ROOT, "include"), src, "-o", exe], check=True)
        lines = subprocess.run([exe], capture_output=True, text=True, check=True).stdout.split("\n")
    c = dict(l.rsplit(" ", 1) for l in lines if l.strip())
    py = {"fl_kv_desc": fl.KvDesc, "fl_attn_args": fl.AttnArgs, "fl_layer_weights": fl.LayerWeights,
          "fl_model": fl.Model, "fl_schedule": fl.Schedule, "fl_loop_state": fl.LoopState,
          "fl_loop_taps": fl.LoopTaps}
    for key, val in c.items():
        if "." in key:
            s, m = key.split(".")
            assert getattr(py[s], m).offset == int(val), key
        else:
            assert ctypes.sizeof(py[key]) == int(val), key


def test_host_validation_without_gpu():
    from cross_loop_sparse_step_b200 import fl
    lib = fl.lib_handle()
    assert fl.status_str(0) == "ok"
    assert fl.version().count(".") == 2
    # null inputs, bad dtype, k out of range: rejected before any CUDA call
    assert fl._select(None, None, 0, 10, 8, None, 3, None, None, None, None, 0, None) == 1
    p = ctypes.c_void_p(16)
    assert fl._select(p, p, 7, 10, 8, None, 3, p, None, None, None, 0, None) == 3
    assert fl._select(p, p, 0, 10, 8, None, 11, p, None, None, None, 0, None) == 2
    assert fl._select(p, p, 0, 10, 6, None, 3, p, None, None, None, 0, None) == 2  # d % 4
    assert fl._select(p, p, 0, 10, 8, None, 3, p, None, None, None, 0, None) == 7  # no workspace
    assert fl._gs(5, p, p, p, 1, 1, 1, 0, None) == 1
    assert fl._gs(0, p, p, p, 0, 1, 1, 0, None) == 0    # nothing to do
    kv = fl.KvDesc()
    kv.n_tok, kv.n_heads, kv.head_dim, kv.group, kv.base_bits, kv.n_loops = 8, 1, 96, 32, 8, 2
    kv.slot = 16
    assert fl._quant(ctypes.byref(kv), 1, p, p, 0, None, 8, None) == 3   # head_dim 96
    kv.head_dim = 64
    kv.res_bits[2] = 3
    assert fl._quant(ctypes.byref(kv), 1, p, p, 0, None, 8, None) == 3   # 3-bit residual
    kv.res_bits[2] = 4
    assert fl._quant(ctypes.byref(kv), 1, p, p, 0, p, 8, None) == 2      # act_tok at loop 1
    assert fl._quant(ctypes.byref(kv), 3, p, p, 0, p, 8, None) == 2      # loop > n_loops
    assert fl._quant(ctypes.byref(kv), 1, p, p, 0, None, 8, None) == 1   # no code buffers
    # decode append past the residual capacity (one row per token): rejected, no launch
    assert fl._append(ctypes.byref(kv), 2, p, p, 0, p, 4, 5, None) == 2
    assert fl._append(ctypes.byref(kv), 2, p, p, 0, p, 1, 2 ** 31 - 1, None) == 2
    a = fl.AttnArgs()
    assert fl._attn(ctypes.byref(a), None) == 1


def test_attention_workspace_sizes_without_gpu():
    """The attention calls' workspace, sized on the host: a sparse call of many queries
    stages the store as fp16 rows and its column sets as bitmaps; a call of few queries
    streams its columns and needs none; a dense call that hands statistics on stages K^
    twice (hi and lo) and V^. A call given less is rejected before any launch."""
    from cross_loop_sparse_step_b200 import fl
    N, H, hd = 32768, 16, 128
    kv = fl.KvDesc()
    kv.n_tok, kv.n_heads, kv.head_dim, kv.group, kv.base_bits, kv.n_loops = N, H, hd, 32, 8, 2
    kv.res_bits[2] = 2
    kv.slot = 16
    kv.vnorm = 16
    p = 16
    staged = H * N * hd * 2                      # one fp16 [H][N][hd] array
    words = (N + 127) // 128 * 4                 # bitmap words per (query, head)

    a = fl.AttnArgs()
    a.q, a.q_dt, a.q_tok, a.kv, a.loop, a.out, a.out_dt = p, 0, p, ctypes.pointer(kv), 2, p, 0
    a.sel, a.mass, a.unsel, a.stat_rows, a.sel_stride = p, p, p, N, 2049
    a.n_q = 4916
    need = fl._attn_ws(ctypes.byref(a))
    assert need == (2 * staged + 255) // 256 * 256 + H * a.n_q * words * 4
    assert fl._attn(ctypes.byref(a), None) == 7          # no workspace: rejected
    a.ws, a.ws_bytes = p, need - 1
    assert fl._attn(ctypes.byref(a), None) == 7

    a.ws, a.ws_bytes = None, 0
    a.n_q = 32                                           # decode-sized: streamed, no workspace
    assert fl._attn_ws(ctypes.byref(a)) == 0

    d = fl.AttnArgs()
    d.q, d.q_dt, d.q_tok, d.kv, d.loop, d.out, d.out_dt = p, 0, p, ctypes.pointer(kv), 1, p, 0
    d.n_q, d.stat_rows, d.k_next, d.out_stride, d.stat_kind = N, N, 2048, 2049, 0
    d.sel_out, d.mass_out, d.unsel_out = p, p, p
    need_d = fl._attn_ws(ctypes.byref(d))
    assert need_d >= 3 * staged + H * N * words * 4      # K^ hi, K^ lo, V^; bitmaps of S'
    d.sel_out = d.mass_out = d.unsel_out = None          # no statistics: K^ and V^ only
    assert fl._attn_ws(ctypes.byref(d)) == 2 * staged


def test_loop_workspace_covers_the_attention_calls():
    """fl_loop_step's workspace holds, besides the block's buffers, the largest attention
    workspace of its schedule: at the 32K shape the dense loop 1 with statistics for loop
    2 (staged K^ hi, K^ lo, V^ and the bitmaps of S'), more than a sparse loop's staged
    K^, V^ and set bitmaps of its active rows."""
    from cross_loop_sparse_step_b200 import configs, fl
    cfg = configs.PREFILL_32K
    N, d, H, hd, F = (cfg[k] for k in ("n_tok", "d_model", "n_heads", "head_dim", "d_ffn"))
    m = fl.Model()
    m.n_tok, m.d_model, m.n_heads, m.head_dim, m.d_ffn, m.n_layers, m.dt = N, d, H, hd, F, 1, 1
    n_active = configs.active_counts(cfg)
    col_k = {r: cfg["col_k"][r] for r in range(2, cfg["n_loops"] + 1)}
    sched = fl.make_schedule(cfg["n_loops"], cfg["first_sparse"], n_active, col_k)
    total = fl._loop_ws(ctypes.byref(m), ctypes.byref(sched))
    staged = H * N * hd * 2
    words = (N + 127) // 128 * 4
    dense_min = 3 * staged + H * N * words * 4          # loop 1's staging and S' bitmaps
    sparse = 2 * staged + H * n_active[2] * words * 4
    assert total > dense_min > sparse
    # a schedule without statistics: the largest call is a dense one over staged K^, V^
    sched0 = fl.make_schedule(cfg["n_loops"], cfg["n_loops"] + 1, {r: N for r in range(1, 5)},
                              {r: 0 for r in range(2, 5)})
    total0 = fl._loop_ws(ctypes.byref(m), ctypes.byref(sched0))
    assert total0 >= 2 * staged and total0 < total
