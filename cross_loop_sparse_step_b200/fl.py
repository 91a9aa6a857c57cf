"""ctypes binding of libfl.so (include/fl.h): argument marshalling only.

Every computation runs in the library's CUDA kernels. PyTorch provides the device
memory (tensors) and the stream; this module turns tensors into pointers, fills the
C structs and raises ``FLError`` on a non-zero status. Importing it without the built
library raises at once: there is no fallback path.
"""
import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libfl.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing: build it with `python -m cross_loop_sparse_step_b200.build` "
        "(nvcc, sm_100a). There is no CPU or Python fallback.")
_lib = ctypes.CDLL(LIB_PATH)

MAX_LOOPS = 32
SENTINEL = 0xFFFF
F32, BF16 = 0, 1
GATHER, SCATTER = 0, 1
STAT_PV, STAT_P = 0, 1

c_i32 = ctypes.c_int32
c_sz = ctypes.c_size_t
vp = ctypes.c_void_p


class KvDesc(ctypes.Structure):
    _fields_ = [
        ("n_tok", c_i32), ("n_heads", c_i32), ("head_dim", c_i32), ("group", c_i32),
        ("base_bits", c_i32), ("n_loops", c_i32),
        ("res_bits", c_i32 * (MAX_LOOPS + 1)),
        ("codes", (vp * (MAX_LOOPS + 1)) * 2),
        ("sz", (vp * (MAX_LOOPS + 1)) * 2),
        ("slot", vp), ("vnorm", vp),
    ]


class AttnArgs(ctypes.Structure):
    _fields_ = [
        ("q", vp), ("q_dt", c_i32), ("n_q", c_i32), ("q_tok", vp),
        ("kv", ctypes.POINTER(KvDesc)), ("loop", c_i32), ("col_bias", vp),
        ("sel", vp), ("mass", vp), ("unsel", vp),
        ("stat_rows", c_i32), ("sel_stride", c_i32), ("q_row", vp),
        ("k_next", c_i32), ("sel_out", vp), ("mass_out", vp), ("unsel_out", vp),
        ("out_stride", c_i32), ("stat_kind", c_i32),
        ("out", vp), ("out_dt", c_i32), ("ws", vp), ("ws_bytes", c_sz),
    ]


class LayerWeights(ctypes.Structure):
    _fields_ = [("w_qkv", vp), ("w_o", vp), ("w_gate_up", vp), ("w_down", vp),
                ("g_attn", vp), ("g_ffn", vp)]


class Model(ctypes.Structure):
    _fields_ = [
        ("n_tok", c_i32), ("d_model", c_i32), ("n_heads", c_i32), ("head_dim", c_i32),
        ("d_ffn", c_i32), ("n_layers", c_i32), ("dt", c_i32),
        ("rms_eps", ctypes.c_float), ("rope_theta", ctypes.c_float),
        ("layers", ctypes.POINTER(LayerWeights)), ("col_bias", vp),
    ]


class Schedule(ctypes.Structure):
    _fields_ = [("n_loops", c_i32), ("first_sparse", c_i32),
                ("n_active", c_i32 * (MAX_LOOPS + 1)), ("col_k", c_i32 * (MAX_LOOPS + 1)),
                ("stat_kind", c_i32)]


class LoopTaps(ctypes.Structure):
    _fields_ = [("n", c_i32), ("tok", vp), ("x_in", vp), ("q", vp), ("k", vp), ("v", vp),
                ("attn", vp), ("x_out", vp)]


class LoopState(ctypes.Structure):
    _fields_ = [
        ("h", vp), ("x_cur", vp), ("x_prev", vp),
        ("act", vp * (MAX_LOOPS + 1)), ("act_pos", vp), ("delta", vp),
        ("kv", ctypes.POINTER(KvDesc)),
        ("sel", ctypes.POINTER(vp)), ("mass", ctypes.POINTER(vp)), ("unsel", ctypes.POINTER(vp)),
        ("sel_stride", c_i32), ("ws", vp), ("ws_bytes", c_sz),
        ("taps", ctypes.POINTER(LoopTaps)),
    ]


def _sig(name, res, args):
    f = getattr(_lib, name)
    f.restype = res
    f.argtypes = args
    return f


_status_str = _sig("fl_status_str", ctypes.c_char_p, [c_i32])
_attn_paths = _sig("fl_attn_path_counts", c_i32, [ctypes.POINTER(ctypes.c_int64), c_i32])
_version = _sig("fl_version", ctypes.c_char_p, [])
_check = _sig("fl_check_device_status", c_i32, [vp])
_detail = _sig("fl_last_error_detail", c_i32, [])
_sel_ws = _sig("fl_select_active_workspace_bytes", c_sz, [c_i32])
_select = _sig("fl_select_active", c_i32,
               [vp, vp, c_i32, c_i32, c_i32, vp, c_i32, vp, vp, vp, vp, c_sz, vp])
_gs = _sig("fl_gather_scatter", c_i32, [c_i32, vp, vp, vp, c_i32, c_i32, c_i32, c_i32, vp])
_quant = _sig("fl_kv_residual_quant", c_i32,
              [ctypes.POINTER(KvDesc), c_i32, vp, vp, c_i32, vp, c_i32, vp])
_append = _sig("fl_kv_append", c_i32,
               [ctypes.POINTER(KvDesc), c_i32, vp, vp, c_i32, vp, c_i32, c_i32, vp])
_recon = _sig("fl_kv_reconstruct", c_i32,
               [ctypes.POINTER(KvDesc), c_i32, vp, c_i32, vp, vp, vp])
_attn_b_ws = _sig("fl_sparse_loop_attn_batched_workspace_bytes", c_sz, [c_i32])
_attn_b = _sig("fl_sparse_loop_attn_batched", c_i32, [ctypes.POINTER(AttnArgs), c_i32, vp, c_sz, vp])
_attn_ws = _sig("fl_sparse_loop_attn_workspace_bytes", c_sz, [ctypes.POINTER(AttnArgs)])
_attn = _sig("fl_sparse_loop_attn", c_i32, [ctypes.POINTER(AttnArgs), vp])
_blk_ws = _sig("fl_block_workspace_bytes", c_sz, [ctypes.POINTER(Model), c_i32])
_blk_qkv = _sig("fl_block_qkv", c_i32,
                [ctypes.POINTER(Model), c_i32, vp, c_i32, vp, vp, vp, vp, vp, c_sz, vp])
_blk_qkv_kv = _sig("fl_block_qkv_kv", c_i32,
                   [ctypes.POINTER(Model), c_i32, ctypes.POINTER(KvDesc), c_i32, vp, c_i32, vp,
                    vp, vp, vp, vp, c_sz, vp])
_blk_ffn = _sig("fl_block_out_ffn", c_i32,
                [ctypes.POINTER(Model), c_i32, vp, c_i32, vp, vp, c_sz, vp])
_loop_ws = _sig("fl_loop_step_workspace_bytes", c_sz,
                [ctypes.POINTER(Model), ctypes.POINTER(Schedule)])
_loop = _sig("fl_loop_step", c_i32,
             [ctypes.POINTER(Model), ctypes.POINTER(LoopState), ctypes.POINTER(Schedule), c_i32, vp])


class FLError(RuntimeError):
    def __init__(self, code, what=""):
        self.code = code
        super().__init__(f"{what}: {status_str(code)} ({code})")


def status_str(code):
    return _status_str(code).decode()


def version():
    return _version().decode()


def lib_handle():
    return _lib


def _ok(code, what):
    if code != 0:
        raise FLError(code, what)


def ptr(t):
    return None if t is None else vp(t.data_ptr())


def dtype_code(t):
    if t.dtype == torch.float32:
        return F32
    if t.dtype == torch.bfloat16:
        return BF16
    raise TypeError(f"unsupported dtype {t.dtype}")


def stream_handle(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return vp(s.cuda_stream)


def check_device_status(stream=None):
    """Synchronise and return (and clear) the device status word (0 = ok)."""
    return _check(stream_handle(stream))


def last_error_detail():
    """Detail of the last status returned (for a timed-out wait: the wait's site code)."""
    return _detail()


# ---------------------------------------------------------------- entry points
def select_active_workspace_bytes(n_rows):
    return _sel_ws(n_rows)


def select_active(h_cur, h_prev, k, row_tok=None, out_tok=None, out_pos=None, out_delta=None,
                  ws=None, stream=None):
    n, d = h_cur.shape
    dev = h_cur.device
    out_tok = out_tok if out_tok is not None else torch.empty(k, dtype=torch.int32, device=dev)
    if out_delta is None and ws is None:
        ws = torch.empty(max(1, select_active_workspace_bytes(n)), dtype=torch.uint8, device=dev)
    _ok(_select(ptr(h_cur), ptr(h_prev), dtype_code(h_cur), n, d, ptr(row_tok), k, ptr(out_tok),
                ptr(out_pos), ptr(out_delta), ptr(ws), 0 if ws is None else ws.numel(),
                stream_handle(stream)), "fl_select_active")
    return out_tok


def gather_scatter(op, src, dst, idx, n_full, stream=None):
    row_elems = src.shape[-1] if src.dim() > 1 else 1
    _ok(_gs(op, ptr(src), ptr(dst), ptr(idx), idx.numel(), n_full, row_elems, dtype_code(src),
            stream_handle(stream)), "fl_gather_scatter")


class KVStore:
    """Device buffers of one layer's KV store (fl_kv_desc), allocated with torch.

    ``rows[r]`` is the row capacity of loop r (loop 1: n_tok)."""

    def __init__(self, n_tok, n_heads, head_dim, group, base_bits, res_bits, n_loops, rows,
                 device="cuda", vnorm=True):
        self.n_tok, self.H, self.hd, self.g = n_tok, n_heads, head_dim, group
        self.base_bits, self.res_bits, self.n_loops = base_bits, dict(res_bits), n_loops
        self.codes = {}
        self.sz = {}
        for r in range(1, n_loops + 1):
            bits = base_bits if r == 1 else self.res_bits[r]
            nrow = n_tok if r == 1 else rows[r]
            for kv in range(2):
                if bits == 0:
                    self.codes[(r, kv)] = torch.zeros(nrow, n_heads, head_dim * 4,
                                                      dtype=torch.uint8, device=device)
                    self.sz[(r, kv)] = None
                else:
                    self.codes[(r, kv)] = torch.zeros(nrow, n_heads, head_dim * bits // 8,
                                                      dtype=torch.uint8, device=device)
                    self.sz[(r, kv)] = torch.zeros(nrow, n_heads, head_dim // group, 2,
                                                   dtype=torch.float16, device=device)
        self.slot = torch.full((n_loops + 1, n_tok), -1, dtype=torch.int32, device=device)
        self.vnorm = torch.zeros(n_tok, n_heads, dtype=torch.float32, device=device) if vnorm else None
        self.desc = KvDesc()
        d = self.desc
        d.n_tok, d.n_heads, d.head_dim, d.group = n_tok, n_heads, head_dim, group
        d.base_bits, d.n_loops = base_bits, n_loops
        for r in range(2, n_loops + 1):
            d.res_bits[r] = self.res_bits[r]
        for (r, kv), t in self.codes.items():
            d.codes[kv][r] = t.data_ptr()
        for (r, kv), t in self.sz.items():
            d.sz[kv][r] = t.data_ptr() if t is not None else None
        d.slot = self.slot.data_ptr()
        d.vnorm = self.vnorm.data_ptr() if self.vnorm is not None else None

    def nbytes(self, r):
        n = 0
        for kv in range(2):
            n += self.codes[(r, kv)].numel()
            if self.sz[(r, kv)] is not None:
                n += self.sz[(r, kv)].numel() * 2
        return n


def kv_residual_quant(store, loop, k_new, v_new, act_tok=None, stream=None):
    n_act = k_new.shape[0]
    _ok(_quant(ctypes.byref(store.desc), loop, ptr(k_new), ptr(v_new), dtype_code(k_new),
               ptr(act_tok), n_act, stream_handle(stream)), "fl_kv_residual_quant")


def kv_append(store, loop, k_new, v_new, act_tok, row0=0, stream=None):
    """Decode: add the tokens act_tok to loop `loop` (rows row0.. for loop >= 2)."""
    _ok(_append(ctypes.byref(store.desc), loop, ptr(k_new), ptr(v_new), dtype_code(k_new),
                ptr(act_tok), act_tok.numel(), row0, stream_handle(stream)), "fl_kv_append")


def kv_reconstruct(store, loop, tok, stream=None):
    """K^_loop, V^_loop of the tokens `tok` (int32 device tensor) as float [n, H, hd]."""
    n = tok.numel()
    k = torch.empty(n, store.H, store.hd, dtype=torch.float32, device=tok.device)
    v = torch.empty_like(k)
    _ok(_recon(ctypes.byref(store.desc), loop, ptr(tok), n, ptr(k), ptr(v),
               stream_handle(stream)), "fl_kv_reconstruct")
    return k, v


def make_attn_args(q, q_tok, store, loop, out, col_bias=None, sel=None, mass=None, unsel=None,
                   q_row=None, k_next=0, sel_out=None, mass_out=None, unsel_out=None,
                   stat_kind=STAT_PV, stat_rows=None):
    """fl_attn_args for tensors that the caller keeps alive during the call."""
    a = AttnArgs()
    a.q, a.q_dt, a.n_q, a.q_tok = q.data_ptr(), dtype_code(q), q.shape[0], q_tok.data_ptr()
    a.kv = ctypes.pointer(store.desc)
    a.loop = loop
    a.col_bias = ptr(col_bias)
    a.sel, a.mass, a.unsel = ptr(sel), ptr(mass), ptr(unsel)
    src = sel if sel is not None else sel_out
    a.stat_rows = stat_rows if stat_rows is not None else (src.shape[1] if src is not None else 0)
    a.sel_stride = sel.shape[2] if sel is not None else 0
    a.q_row = ptr(q_row)
    a.k_next = k_next
    a.sel_out, a.mass_out, a.unsel_out = ptr(sel_out), ptr(mass_out), ptr(unsel_out)
    a.out_stride = sel_out.shape[2] if sel_out is not None else 0
    a.stat_kind = stat_kind
    a.out, a.out_dt = out.data_ptr(), dtype_code(out)
    return a


def sparse_loop_attn(q, q_tok, store, loop, out, col_bias=None, sel=None, mass=None, unsel=None,
                     q_row=None, k_next=0, sel_out=None, mass_out=None, unsel_out=None,
                     stat_kind=STAT_PV, stat_rows=None, stream=None):
    a = make_attn_args(q, q_tok, store, loop, out, col_bias, sel, mass, unsel, q_row, k_next,
                       sel_out, mass_out, unsel_out, stat_kind, stat_rows)
    nb = _attn_ws(ctypes.byref(a))
    ws = torch.empty(max(nb, 1), dtype=torch.uint8, device=q.device) if nb else None
    a.ws, a.ws_bytes = ptr(ws), nb
    _ok(_attn(ctypes.byref(a), stream_handle(stream)), "fl_sparse_loop_attn")
    return out


def sparse_loop_attn_batched(args, stream=None):
    """One launch over several calls' fl_attn_args (see make_attn_args)."""
    n = len(args)
    arr = (AttnArgs * n)(*args)
    nb = _attn_b_ws(n)
    dev = torch.cuda.current_device()
    ws = torch.empty(max(nb, 1), dtype=torch.uint8, device=f"cuda:{dev}")
    _ok(_attn_b(arr, n, ptr(ws), nb, stream_handle(stream)), "fl_sparse_loop_attn_batched")
    return ws


class LoopModel:
    """fl_model over torch weight tensors (kept alive by this object)."""

    def __init__(self, layers, n_tok, n_heads, head_dim, col_bias=None, eps=1e-6, theta=10000.0):
        self.layers = layers
        w0 = layers[0]
        d = w0["w_qkv"].shape[1]
        F = w0["w_down"].shape[1]
        self.dt = dtype_code(w0["w_qkv"])
        self.col_bias = col_bias
        self._lw = (LayerWeights * len(layers))()
        for i, w in enumerate(layers):
            self._lw[i] = LayerWeights(w["w_qkv"].data_ptr(), w["w_o"].data_ptr(),
                                       w["w_gate_up"].data_ptr(), w["w_down"].data_ptr(),
                                       w["g_attn"].data_ptr(), w["g_ffn"].data_ptr())
        self.c = Model(n_tok, d, n_heads, head_dim, F, len(layers), self.dt, eps, theta,
                       ctypes.cast(self._lw, ctypes.POINTER(LayerWeights)), ptr(col_bias))

    def block_ws_bytes(self, n_rows):
        return _blk_ws(ctypes.byref(self.c), n_rows)


def block_qkv(model, layer, x, pos, q, k, v, ws, stream=None):
    _ok(_blk_qkv(ctypes.byref(model.c), layer, ptr(x), x.shape[0], ptr(pos), ptr(q), ptr(k),
                 ptr(v), ptr(ws), ws.numel(), stream_handle(stream)), "fl_block_qkv")


def block_qkv_kv(model, layer, store, loop, x, pos, q, ws, k=None, v=None, stream=None):
    """block_qkv with loop `loop`'s KV store update done in the projection epilogue."""
    _ok(_blk_qkv_kv(ctypes.byref(model.c), layer, ctypes.byref(store.desc), loop, ptr(x),
                    x.shape[0], ptr(pos), ptr(q), ptr(k), ptr(v), ptr(ws), ws.numel(),
                    stream_handle(stream)), "fl_block_qkv_kv")


def block_out_ffn(model, layer, x, attn, ws, stream=None):
    _ok(_blk_ffn(ctypes.byref(model.c), layer, ptr(x), x.shape[0], ptr(attn), ptr(ws),
                 ws.numel(), stream_handle(stream)), "fl_block_out_ffn")


def make_schedule(n_loops, first_sparse, n_active, col_k, stat_kind=STAT_PV):
    s = Schedule()
    s.n_loops, s.first_sparse, s.stat_kind = n_loops, first_sparse, stat_kind
    for r, k in n_active.items():
        s.n_active[r] = k
    for r, k in col_k.items():
        s.col_k[r] = k or 0
    return s


ATTN_PATHS = ("tile-column-ranges", "tile-union", "tile-decode", "dense-tile", "sparse-warp",
              "dense-warp", "general", "sparse-stream")


def attn_path_counts():
    """Attention calls of this process by the kernel path that ran (fl_attn_path_counts)."""
    buf = (ctypes.c_int64 * len(ATTN_PATHS))()
    n = _attn_paths(buf, len(ATTN_PATHS))
    assert n == len(ATTN_PATHS), n
    return {name: int(buf[i]) for i, name in enumerate(ATTN_PATHS)}


def stat_stride(k):
    """Statistics row stride for a budget of k columns plus the sink: k + 1. (A sparse
    call whose budget for the next loop is unchanged keeps its statistics in place; the
    attention recognises that case by k_next + 1 >= stride.)"""
    return k + 1


class LoopRunner:
    """Device state of an R-loop run (fl_loop_state) plus the model and schedule."""

    def __init__(self, model, sched, n_active, kv_stores, sel_stride, device="cuda"):
        c = model.c
        N, d, L, H, hd = c.n_tok, c.d_model, c.n_layers, c.n_heads, c.head_dim
        self.model, self.sched, self.kv = model, sched, kv_stores
        self.h = torch.zeros(N, d, dtype=torch.float32, device=device)
        self.x_cur = torch.zeros(N, d, dtype=torch.float32, device=device)
        self.x_prev = torch.zeros(N, d, dtype=torch.float32, device=device)
        self.act = {r: torch.zeros(max(1, n_active[r]), dtype=torch.int32, device=device)
                    for r in range(2, sched.n_loops + 1)}
        self.act_pos = torch.zeros(N, dtype=torch.int32, device=device)
        self.delta = torch.zeros(N, dtype=torch.float32, device=device)
        self.sel = [torch.full((H, N, sel_stride), -1, dtype=torch.int16, device=device)
                    for _ in range(L)] if sel_stride else []
        self.mass = [torch.zeros(H, N, dtype=torch.float32, device=device) for _ in range(L)] if sel_stride else []
        self.unsel = [torch.zeros(H, N, hd, dtype=torch.float32, device=device) for _ in range(L)] if sel_stride else []
        nb = _loop_ws(ctypes.byref(c), ctypes.byref(sched))
        self.ws = torch.empty(nb, dtype=torch.uint8, device=device)
        st = LoopState()
        st.h, st.x_cur, st.x_prev = self.h.data_ptr(), self.x_cur.data_ptr(), self.x_prev.data_ptr()
        for r, t in self.act.items():
            st.act[r] = t.data_ptr()
        st.act_pos, st.delta = self.act_pos.data_ptr(), self.delta.data_ptr()
        self._kvd = (KvDesc * L)(*[s.desc for s in kv_stores])
        st.kv = ctypes.cast(self._kvd, ctypes.POINTER(KvDesc))
        if sel_stride:
            self._sel = (vp * L)(*[t.data_ptr() for t in self.sel])
            self._mass = (vp * L)(*[t.data_ptr() for t in self.mass])
            self._unsel = (vp * L)(*[t.data_ptr() for t in self.unsel])
            st.sel = ctypes.cast(self._sel, ctypes.POINTER(vp))
            st.mass = ctypes.cast(self._mass, ctypes.POINTER(vp))
            st.unsel = ctypes.cast(self._unsel, ctypes.POINTER(vp))
        st.sel_stride = sel_stride
        st.ws, st.ws_bytes = self.ws.data_ptr(), nb
        self.c = st

    def set_taps(self, tok):
        """Inspection taps (fl_loop_taps) for the tokens ``tok`` (int32 device tensor):
        every later step copies each layer's input, q, k, v, attention output and
        output rows of those tokens into ``self.taps`` ([L, n, d] tensors). None turns
        them off."""
        if tok is None:
            self.taps, self._taps = None, None
            self.c.taps = ctypes.POINTER(LoopTaps)()
            return None
        c = self.model.c
        L, n, d = c.n_layers, tok.numel(), c.d_model
        dev = tok.device
        adt = torch.bfloat16 if c.dt == BF16 else torch.float32
        self.taps = {k: torch.full((L, n, d), float("nan"), dtype=torch.float32, device=dev)
                     for k in ("x_in", "q", "k", "v", "x_out")}
        self.taps["attn"] = torch.full((L, n, d), float("nan"), dtype=adt, device=dev)
        self.taps["tok"] = tok
        t = LoopTaps()
        t.n, t.tok = n, tok.data_ptr()
        for k in ("x_in", "q", "k", "v", "attn", "x_out"):
            setattr(t, k, self.taps[k].data_ptr())
        self._taps = t
        self.c.taps = ctypes.pointer(t)
        return self.taps

    def step(self, loop, stream=None):
        _ok(_loop(ctypes.byref(self.model.c), ctypes.byref(self.c), ctypes.byref(self.sched), loop,
                  stream_handle(stream)), f"fl_loop_step(loop={loop})")
