"""The allocation-free selection entry point (fl_select_active_noalloc).

It exists for callers that cannot allocate device memory - code running inside a host
runtime that owns all device memory and passes a plugin only its inputs and outputs,
or a deployment with a fixed memory plan. Its scratch lives in a fixed array inside the
library, so the call takes inputs and outputs only. Here it must return exactly what the
workspace-taking fl_select_active returns (indices are bit-exact in every parity test of
this suite), on two calls in a row on different inputs, and reject sizes beyond its
fixed scratch without launching. This file is collected last on purpose."""
import ctypes

import numpy as np
import pytest
import torch

from cross_loop_sparse_step_b200 import synth

pytestmark = pytest.mark.gpu


def _noalloc(fl):
    f = fl.lib_handle().fl_select_active_noalloc
    f.restype = ctypes.c_int32
    f.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int32, ctypes.c_int32,
                  ctypes.c_int32, ctypes.c_void_p, ctypes.c_int32, ctypes.c_void_p,
                  ctypes.c_void_p, ctypes.c_void_p]
    return f


@pytest.mark.parametrize("n,d,dt,k,use_tok", [(4096, 2048, "bf16", 820, False),
                                              (4916, 2048, "f32", 2000, True)])
def test_noalloc_matches_workspace_entry_point(n, d, dt, k, use_tok):
    from cross_loop_sparse_step_b200 import fl
    f = _noalloc(fl)
    tdt = torch.bfloat16 if dt == "bf16" else torch.float32
    for call in range(2):   # two calls in a row share the fixed scratch
        g = synth.rng(500 + 17 * call + n)
        cur, prev, _ = synth.pareto_delta_pair(g, n, d, 2 + call)
        hc = torch.from_numpy(cur).cuda().to(tdt)
        hp = torch.from_numpy(prev).cuda().to(tdt)
        rt = None
        if use_tok:
            rt = torch.from_numpy(np.sort(g.choice(3 * n, size=n, replace=False)).astype(np.int32)).cuda()
        want_tok = torch.full((k,), -1, dtype=torch.int32, device="cuda")
        want_pos = torch.full((k,), -1, dtype=torch.int32, device="cuda")
        fl.select_active(hc, hp, k, rt, want_tok, want_pos)
        got_tok = torch.full((k,), -2, dtype=torch.int32, device="cuda")
        got_pos = torch.full((k,), -2, dtype=torch.int32, device="cuda")
        rc = f(hc.data_ptr(), hp.data_ptr(), fl.dtype_code(hc), n, d,
               None if rt is None else rt.data_ptr(), k, got_tok.data_ptr(), got_pos.data_ptr(),
               fl.stream_handle())
        assert rc == 0, fl.status_str(rc)
        assert fl.check_device_status() == 0
        assert torch.equal(got_tok, want_tok)
        assert torch.equal(got_pos, want_pos)


def test_noalloc_without_positions_and_with_k_zero():
    """out_pos may be NULL (the kept tokens alone), and k = 0 runs only the change pass
    into the shared scratch: both return what the workspace entry point returns."""
    from cross_loop_sparse_step_b200 import fl
    f = _noalloc(fl)
    n, d, k = 3000, 256, 700
    g = synth.rng(901)
    cur, prev, _ = synth.pareto_delta_pair(g, n, d, 2)
    hc, hp = torch.from_numpy(cur).cuda(), torch.from_numpy(prev).cuda()
    want = fl.select_active(hc, hp, k)
    got = torch.full((k,), -3, dtype=torch.int32, device="cuda")
    rc = f(hc.data_ptr(), hp.data_ptr(), fl.F32, n, d, None, k, got.data_ptr(), None,
           fl.stream_handle())
    assert rc == 0, fl.status_str(rc)
    assert fl.check_device_status() == 0
    assert torch.equal(got, want)
    untouched = torch.full((1,), -5, dtype=torch.int32, device="cuda")
    rc = f(hc.data_ptr(), hp.data_ptr(), fl.F32, n, d, None, 0, untouched.data_ptr(), None,
           fl.stream_handle())
    assert rc == 0, fl.status_str(rc)
    assert fl.check_device_status() == 0
    assert int(untouched.item()) == -5


def test_noalloc_rejects_sizes_beyond_its_scratch():
    from cross_loop_sparse_step_b200 import fl
    f = _noalloc(fl)
    x = torch.zeros(8, 8, device="cuda")
    out = torch.zeros(1, dtype=torch.int32, device="cuda")
    rc = f(x.data_ptr(), x.data_ptr(), 0, 65537, 8, None, 1, out.data_ptr(), None,
           fl.stream_handle())
    assert rc == 2   # FL_ERR_SHAPE, nothing launched
