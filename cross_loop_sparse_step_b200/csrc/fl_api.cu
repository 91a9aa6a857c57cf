// The C interface (include/fl.h): host-side validation, workspace carving and the
// launch sequence of each entry point. Nothing here allocates device memory.
#include <atomic>
#include <mutex>
#include <vector>
#include <string.h>

#include "fl_internal.cuh"

__device__ int g_fl_status;  // first error recorded by a kernel on this device

namespace fl {

cudaError_t launch_gemm_simt(fl_dtype dt, const void* A, const void* W, float* C, int M, int N,
                             int K, int ldc, GemmEpi epi, cudaStream_t s);
cudaError_t launch_gemm_tc(const void* A, const void* W, float* C, int M, int N, int K,
                           int ldc, GemmEpi epi, cudaStream_t s, const GemmScratch* scr);
bool gemm_tc_supported(int M, int N, int K);
bool gemm_swiglu_supported(int M, int F, int K);
cudaError_t launch_gemm_swiglu(const void* A, const void* W, void* Y, int M, int F, int K,
                               cudaStream_t s, const GemmScratch* scr);
bool gemm_qkv_supported(int M, int d, int hd);
cudaError_t launch_gemm_qkv(const void* A, const void* W, float* q, float* k, float* v,
                            const int32_t* pos, const float2* rope, int M, int d, int hd,
                            cudaStream_t s, const fl_kv_desc* fuse, int loop,
                            const GemmScratch* scr);

bool pdl_enabled() {
  static int on = -1;
  if (on < 0) {
    const char* e = getenv("FL_PDL");
    on = (e && atoi(e) == 0) ? 0 : 1;
  }
  return on == 1;
}

int* status_word() {
  static int* cache[128] = {nullptr};
  static std::mutex mu;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 128) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  if (!cache[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_fl_status) != cudaSuccess) return nullptr;
    cache[dev] = static_cast<int*>(p);
  }
  return cache[dev];
}

// ---------------------------------------------------------------- launch accounting
static std::atomic<long long> g_launches{0};
void count_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }

struct TimingHook {
  std::vector<cudaEvent_t> begin, end;
  int next = 0;
};
static TimingHook g_hooks[TIMED_KINDS];

// Under stream capture the events become external event-record nodes of the graph, so
// every replay records them again.
static void record_event(cudaEvent_t e, cudaStream_t s) {
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  cudaStreamIsCapturing(s, &cs);
  if (cs == cudaStreamCaptureStatusActive) cudaEventRecordWithFlags(e, s, cudaEventRecordExternal);
  else cudaEventRecord(e, s);
}
void timing_begin(int kind, cudaStream_t s) {
  TimingHook& h = g_hooks[kind];
  if (h.next < (int)h.begin.size()) record_event(h.begin[h.next], s);
}
void timing_end(int kind, cudaStream_t s) {
  TimingHook& h = g_hooks[kind];
  if (h.next < (int)h.end.size()) record_event(h.end[h.next++], s);
}

static std::atomic<long long> g_bf16_simt{0};

cudaError_t launch_gemm(fl_dtype dt, const void* A, const void* W, float* C, int M, int N,
                        int K, int ldc, GemmEpi epi, cudaStream_t s, const GemmScratch* scr) {
  timing_begin(TIMED_GEMM, s);
  cudaError_t e;
  if (dt == FL_BF16 && gemm_tc_supported(M, N, K)) {
    e = launch_gemm_tc(A, W, C, M, N, K, ldc, epi, s, scr);
  } else {
    // binary32 projections always run here; a bf16 one only when its shape cannot be
    // tiled for the tensor cores - counted, so that a caller can see it happened
    if (dt == FL_BF16) g_bf16_simt.fetch_add(1, std::memory_order_relaxed);
    e = launch_gemm_simt(dt, A, W, C, M, N, K, ldc, epi, s);
  }
  timing_end(TIMED_GEMM, s);
  return e;
}

cudaError_t launch_attention_timed(const fl_attn_args& a, int* st, cudaStream_t s) {
  timing_begin(TIMED_ATTN, s);
  cudaError_t e = launch_attention(a, st, s);
  timing_end(TIMED_ATTN, s);
  return e;
}

}  // namespace fl

using namespace fl;

namespace {

inline cudaStream_t S(void* s) { return reinterpret_cast<cudaStream_t>(s); }
inline fl_status cuda_st(cudaError_t e) { return e == cudaSuccess ? FL_OK : FL_ERR_CUDA; }
#define FL_TRY(expr)                              \
  do {                                            \
    cudaError_t _e = (expr);                      \
    if (_e != cudaSuccess) return FL_ERR_CUDA;    \
  } while (0)
#define FL_CHECK(cond, code) \
  do {                       \
    if (!(cond)) return (code); \
  } while (0)

bool valid_dt(fl_dtype dt) { return dt == FL_F32 || dt == FL_BF16; }
bool valid_bits(int b) { return b == 0 || b == 2 || b == 4 || b == 8; }

// Carves aligned sub-buffers out of a caller-provided workspace.
struct Carver {
  uint8_t* base;
  size_t off = 0;
  explicit Carver(void* b) : base(static_cast<uint8_t*>(b)) {}
  void* take(size_t bytes) {
    void* p = base ? base + off : nullptr;
    off += align_up(bytes);
    return p;
  }
};

fl_status check_kv(const fl_kv_desc* kv) {
  FL_CHECK(kv, FL_ERR_INVALID_ARG);
  FL_CHECK(kv->n_tok > 0 && kv->n_tok <= 65535, FL_ERR_SHAPE);
  FL_CHECK(kv->n_heads > 0, FL_ERR_SHAPE);
  FL_CHECK(kv->head_dim == 64 || kv->head_dim == 128, FL_ERR_UNSUPPORTED);
  FL_CHECK(kv->group == 32 || kv->group == 64, FL_ERR_UNSUPPORTED);
  FL_CHECK(kv->head_dim % kv->group == 0, FL_ERR_SHAPE);
  FL_CHECK(kv->base_bits == 0 || kv->base_bits == 8, FL_ERR_UNSUPPORTED);
  FL_CHECK(kv->n_loops >= 1 && kv->n_loops <= FL_MAX_LOOPS, FL_ERR_SHAPE);
  FL_CHECK(kv->slot, FL_ERR_INVALID_ARG);
  for (int r = 2; r <= kv->n_loops; ++r) FL_CHECK(valid_bits(kv->res_bits[r]), FL_ERR_UNSUPPORTED);
  return FL_OK;
}

fl_status check_model(const fl_model* m) {
  FL_CHECK(m && m->layers, FL_ERR_INVALID_ARG);
  FL_CHECK(valid_dt(m->dt), FL_ERR_UNSUPPORTED);
  FL_CHECK(m->n_tok > 0 && m->n_tok <= 65535 && m->n_layers > 0, FL_ERR_SHAPE);
  FL_CHECK(m->head_dim == 64 || m->head_dim == 128, FL_ERR_UNSUPPORTED);
  FL_CHECK(m->n_heads > 0 && m->d_model == m->n_heads * m->head_dim, FL_ERR_SHAPE);
  FL_CHECK(m->d_ffn > 0 && m->d_ffn % 8 == 0 && m->d_model % 8 == 0, FL_ERR_SHAPE);
  for (int l = 0; l < m->n_layers; ++l) {
    const fl_layer_weights& w = m->layers[l];
    FL_CHECK(w.w_qkv && w.w_o && w.w_gate_up && w.w_down && w.g_attn && w.g_ffn,
             FL_ERR_INVALID_ARG);
  }
  return FL_OK;
}

// Block workspace: [RoPE (cos, sin) table of every position][GEMM stream-K scratch]
// [scratch of one half-layer].
size_t rope_tab_bytes(const fl_model* m) {
  return align_up((size_t)m->n_tok * (m->head_dim / 2) * sizeof(float2));
}

size_t block_head_bytes(const fl_model* m) {
  return rope_tab_bytes(m) + align_up(gemm_scratch_bytes());
}

GemmScratch block_scratch(const fl_model* m, void* ws) {
  return gemm_scratch_at(static_cast<uint8_t*>(ws) + rope_tab_bytes(m));
}

size_t block_ws(const fl_model* m, int n) {
  const size_t d = m->d_model, F = m->d_ffn, e = dt_size(m->dt);
  const size_t qkv_path = align_up(n * d * e) + align_up(n * 3 * d * 4);
  const size_t ffn_path = align_up(n * d * e) + align_up(n * 2 * F * 4) + align_up(n * F * e);
  return block_head_bytes(m) + (qkv_path > ffn_path ? qkv_path : ffn_path);
}

bool qkv_fused(const fl_model* m, int n) {
  return m->dt == FL_BF16 && gemm_qkv_supported(n, m->d_model, m->head_dim);
}

// Fills the RoPE table at the head of the block workspace and clears the GEMM hand-over
// flags (once per call or loop step).
fl_status prepare_rope(const fl_model* m, void* ws, cudaStream_t s) {
  FL_TRY(launch_rope_table(static_cast<float2*>(ws), m->n_tok, m->head_dim, m->rope_theta, s));
  FL_TRY(cudaMemsetAsync(static_cast<uint8_t*>(ws) + rope_tab_bytes(m), 0,
                         gemm_scratch_flag_bytes(), s));
  return FL_OK;
}

// The store update of `loop` can ride in the QKV epilogue: bf16 projections, group 32,
// an 8-bit base and 2/4/8-bit residual loops up to `loop`.
bool kv_fusable(const fl_model* m, int n, const fl_kv_desc* kv, int loop) {
  if (!kv || !qkv_fused(m, n) || kv->group != 32 || kv->base_bits != 8) return false;
  if (kv->n_heads != m->n_heads || kv->head_dim != m->head_dim || loop < 1 || loop > kv->n_loops)
    return false;
  for (int r = 2; r <= loop; ++r) {
    const int b = kv->res_bits[r];
    if (b != 2 && b != 4 && b != 8) return false;
  }
  return true;
}

// RMSNorm, QKV projection, RoPE; with `fuse` the KV store update of `loop` happens in the
// projection's epilogue (k, v may then be null).
fl_status run_qkv(const fl_model* m, int layer, const float* x, int n, const int32_t* pos,
                  float* q, float* k, float* v, void* ws, cudaStream_t s,
                  const fl_kv_desc* fuse = nullptr, int loop = 0) {
  const fl_layer_weights& w = m->layers[layer];
  const int d = m->d_model;
  const float2* rope = static_cast<const float2*>(ws);
  const GemmScratch scr = block_scratch(m, ws);
  Carver c(static_cast<uint8_t*>(ws) + block_head_bytes(m));
  void* a = c.take((size_t)n * d * dt_size(m->dt));
  FL_TRY(launch_rmsnorm(x, w.g_attn, m->rms_eps, a, m->dt, n, d, s));
  if (qkv_fused(m, n)) {
    if (fuse && loop >= 2)
      FL_TRY(launch_fill_i32(fuse->slot + (size_t)loop * fuse->n_tok, -1, (size_t)fuse->n_tok, s));
    if (fuse && loop == 1 && fuse->slot) FL_TRY(launch_iota(fuse->slot + fuse->n_tok, fuse->n_tok, s));
    timing_begin(TIMED_GEMM, s);
    cudaError_t e =
        launch_gemm_qkv(a, w.w_qkv, q, k, v, pos, rope, n, d, m->head_dim, s, fuse, loop, &scr);
    timing_end(TIMED_GEMM, s);
    FL_TRY(e);
    return FL_OK;
  }
  float* qkv = (float*)c.take((size_t)n * 3 * d * 4);
  FL_TRY(launch_gemm(m->dt, a, w.w_qkv, qkv, n, 3 * d, d, 3 * d, EPI_STORE, s, &scr));
  FL_TRY(launch_rope_split(qkv, pos, n, m->n_heads, m->head_dim, m->rope_theta, q, k, v, s));
  return FL_OK;
}

fl_status run_out_ffn(const fl_model* m, int layer, float* x, int n, const void* attn, void* ws,
                      cudaStream_t s) {
  const fl_layer_weights& w = m->layers[layer];
  const int d = m->d_model, F = m->d_ffn;
  const GemmScratch scr = block_scratch(m, ws);
  Carver c(static_cast<uint8_t*>(ws) + block_head_bytes(m));
  void* a = c.take((size_t)n * d * dt_size(m->dt));
  float* gu = (float*)c.take((size_t)n * 2 * F * 4);
  void* mid = c.take((size_t)n * F * dt_size(m->dt));
  FL_TRY(launch_gemm(m->dt, attn, w.w_o, x, n, d, d, d, EPI_ADD, s, &scr));
  FL_TRY(launch_rmsnorm(x, w.g_ffn, m->rms_eps, a, m->dt, n, d, s));
  if (m->dt == FL_BF16 && gemm_swiglu_supported(n, F, d)) {
    timing_begin(TIMED_GEMM, s);
    cudaError_t e = launch_gemm_swiglu(a, w.w_gate_up, mid, n, F, d, s, &scr);
    timing_end(TIMED_GEMM, s);
    FL_TRY(e);
  } else {
    FL_TRY(launch_gemm(m->dt, a, w.w_gate_up, gu, n, 2 * F, d, 2 * F, EPI_STORE, s, &scr));
    FL_TRY(launch_swiglu(gu, n, F, mid, m->dt, s));
  }
  FL_TRY(launch_gemm(m->dt, mid, w.w_down, x, n, d, F, d, EPI_ADD, s, &scr));
  return FL_OK;
}

fl_status check_attn(const fl_attn_args* a) {
  FL_CHECK(a && a->q && a->q_tok && a->out, FL_ERR_INVALID_ARG);
  fl_status st = check_kv(a->kv);
  if (st != FL_OK) return st;
  FL_CHECK(valid_dt(a->q_dt) && valid_dt(a->out_dt), FL_ERR_UNSUPPORTED);
  FL_CHECK(a->n_q >= 0, FL_ERR_SHAPE);
  FL_CHECK(a->loop >= 1 && a->loop <= a->kv->n_loops, FL_ERR_SHAPE);
  if (a->sel) {
    FL_CHECK(a->mass && a->unsel, FL_ERR_INVALID_ARG);
    FL_CHECK(a->sel_stride >= 1 && a->stat_rows > 0, FL_ERR_SHAPE);
    FL_CHECK(a->sel_stride <= 8192, FL_ERR_UNSUPPORTED);
  }
  if (a->sel_out) {
    FL_CHECK(a->mass_out && a->unsel_out, FL_ERR_INVALID_ARG);
    FL_CHECK(a->k_next >= 0 && a->out_stride >= a->k_next + 1, FL_ERR_SHAPE);
    FL_CHECK(a->stat_rows > 0, FL_ERR_SHAPE);
    FL_CHECK(a->stat_kind == FL_STAT_PV || a->stat_kind == FL_STAT_P, FL_ERR_INVALID_ARG);
    FL_CHECK(a->stat_kind == FL_STAT_P || a->kv->vnorm, FL_ERR_INVALID_ARG);
    if (a->sel) FL_CHECK(a->out_stride <= a->sel_stride || a->sel_out != a->sel, FL_ERR_SHAPE);
  }
  return FL_OK;
}

}  // namespace

extern "C" {

const char* fl_status_str(fl_status s) {
  switch (s) {
    case FL_OK: return "ok";
    case FL_ERR_INVALID_ARG: return "invalid argument";
    case FL_ERR_SHAPE: return "bad shape";
    case FL_ERR_UNSUPPORTED: return "unsupported dtype, bit width or group size";
    case FL_ERR_CUDA: return "CUDA error";
    case FL_ERR_TIMEOUT: return "device wait timed out";
    case FL_ERR_RANGE: return "index out of range or fp16 overflow";
    case FL_ERR_WORKSPACE: return "workspace too small";
  }
  return "unknown status";
}

const char* fl_version(void) { return "0.1.0"; }

int64_t fl_launch_count(void) { return (int64_t)g_launches.load(); }

int64_t fl_gemm_bf16_cuda_core_count(void) { return (int64_t)g_bf16_simt.load(); }

int32_t fl_attn_path_counts(int64_t* out, int32_t n) {
  for (int i = 0; out && i < n && i < N_ATTN_PATHS; ++i) out[i] = attn_path_count(i);
  return N_ATTN_PATHS;
}

fl_status fl_set_timing_events(int32_t kind, void* const* begin, void* const* end, int32_t n) {
  FL_CHECK(kind >= 0 && kind < TIMED_KINDS && n >= 0, FL_ERR_INVALID_ARG);
  FL_CHECK(n == 0 || (begin && end), FL_ERR_INVALID_ARG);
  TimingHook& h = g_hooks[kind];
  h.begin.clear(); h.end.clear(); h.next = 0;
  for (int i = 0; i < n; ++i) {
    h.begin.push_back(reinterpret_cast<cudaEvent_t>(begin[i]));
    h.end.push_back(reinterpret_cast<cudaEvent_t>(end[i]));
  }
  return FL_OK;
}

int32_t fl_timing_recorded(int32_t kind) {
  if (kind < 0 || kind >= TIMED_KINDS) return -1;
  return g_hooks[kind].next;
}

static std::atomic<int> g_last_detail{0};

fl_status fl_check_device_status(void* stream) {
  if (cudaStreamSynchronize(S(stream)) != cudaSuccess) return FL_ERR_CUDA;
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_fl_status, sizeof(int)) != cudaSuccess) return FL_ERR_CUDA;
  const int zero = 0;
  if (cudaMemcpyToSymbol(g_fl_status, &zero, sizeof(int)) != cudaSuccess) return FL_ERR_CUDA;
  g_last_detail.store(v >> 8);
  return (fl_status)(v & 0xFF);
}

int32_t fl_last_error_detail(void) { return g_last_detail.load(); }

size_t fl_select_active_workspace_bytes(int32_t n_rows) {
  return n_rows > 0 ? align_up((size_t)n_rows * 4) : 0;
}

fl_status fl_select_active(const void* h_cur, const void* h_prev, fl_dtype dt, int32_t n_rows,
                           int32_t d, const int32_t* row_tok, int32_t k, int32_t* out_tok,
                           int32_t* out_pos, float* out_delta, void* ws, size_t ws_bytes,
                           void* stream) {
  FL_CHECK(h_cur && h_prev && out_tok, FL_ERR_INVALID_ARG);
  FL_CHECK(valid_dt(dt), FL_ERR_UNSUPPORTED);
  FL_CHECK(n_rows >= 1 && n_rows <= (1 << 24) && d >= 1, FL_ERR_SHAPE);
  FL_CHECK(d % (dt == FL_BF16 ? 8 : 4) == 0, FL_ERR_SHAPE);
  FL_CHECK(k >= 0 && k <= n_rows, FL_ERR_SHAPE);
  FL_CHECK(((uintptr_t)h_cur % 16 == 0) && ((uintptr_t)h_prev % 16 == 0), FL_ERR_INVALID_ARG);
  float* delta = out_delta;
  if (!delta) {
    FL_CHECK(ws && ws_bytes >= fl_select_active_workspace_bytes(n_rows), FL_ERR_WORKSPACE);
    delta = static_cast<float*>(ws);
  }
  cudaStream_t s = S(stream);
  FL_TRY(launch_row_delta(h_cur, h_prev, dt, n_rows, d, delta, s));
  FL_TRY(launch_topk_rows(delta, n_rows, k, row_tok, out_tok, out_pos, status_word(), s));
  return FL_OK;
}

fl_status fl_gather_scatter(fl_gs_op op, const void* src, void* dst, const int32_t* idx,
                            int32_t n_idx, int32_t n_full, int32_t row_elems, fl_dtype dt,
                            void* stream) {
  FL_CHECK(op == FL_GATHER || op == FL_SCATTER, FL_ERR_INVALID_ARG);
  FL_CHECK(valid_dt(dt), FL_ERR_UNSUPPORTED);
  FL_CHECK(n_idx >= 0 && n_full >= 0 && row_elems >= 1, FL_ERR_SHAPE);
  if (n_idx == 0) return FL_OK;
  FL_CHECK(src && dst && idx, FL_ERR_INVALID_ARG);
  return cuda_st(launch_gather_scatter(op, src, dst, idx, n_idx, n_full,
                                       (size_t)row_elems * dt_size(dt), status_word(), S(stream)));
}

fl_status fl_kv_residual_quant(const fl_kv_desc* kv, int32_t loop, const void* k_new,
                               const void* v_new, fl_dtype dt, const int32_t* act_tok,
                               int32_t n_act, void* stream) {
  fl_status st = check_kv(kv);
  if (st != FL_OK) return st;
  FL_CHECK(k_new && v_new, FL_ERR_INVALID_ARG);
  FL_CHECK(valid_dt(dt), FL_ERR_UNSUPPORTED);
  FL_CHECK(loop >= 1 && loop <= kv->n_loops, FL_ERR_SHAPE);
  if (loop == 1) {
    FL_CHECK(act_tok == nullptr && n_act == kv->n_tok, FL_ERR_SHAPE);
  } else {
    FL_CHECK(n_act >= 0 && n_act <= kv->n_tok, FL_ERR_SHAPE);
    FL_CHECK(n_act == 0 || act_tok, FL_ERR_INVALID_ARG);
  }
  const int bits = loop == 1 ? kv->base_bits : kv->res_bits[loop];
  FL_CHECK(kv->codes[0][loop] && kv->codes[1][loop], FL_ERR_INVALID_ARG);
  if (bits != 0) FL_CHECK(kv->sz[0][loop] && kv->sz[1][loop], FL_ERR_INVALID_ARG);
  for (int r = 2; r < loop; ++r) {
    FL_CHECK(kv->codes[0][r] && kv->codes[1][r], FL_ERR_INVALID_ARG);
    if (kv->res_bits[r] != 0) FL_CHECK(kv->sz[0][r] && kv->sz[1][r], FL_ERR_INVALID_ARG);
  }
  if (loop >= 2) FL_CHECK(kv->codes[0][1] && kv->codes[1][1], FL_ERR_INVALID_ARG);
  return cuda_st(launch_kv_quant(*kv, loop, k_new, v_new, dt, act_tok, n_act, status_word(),
                                 S(stream)));
}

fl_status fl_kv_append(const fl_kv_desc* kv, int32_t loop, const void* k_new, const void* v_new,
                       fl_dtype dt, const int32_t* act_tok, int32_t n_act, int32_t row0,
                       void* stream) {
  fl_status st = check_kv(kv);
  if (st != FL_OK) return st;
  FL_CHECK(k_new && v_new && act_tok, FL_ERR_INVALID_ARG);
  FL_CHECK(valid_dt(dt), FL_ERR_UNSUPPORTED);
  FL_CHECK(loop >= 1 && loop <= kv->n_loops, FL_ERR_SHAPE);
  FL_CHECK(n_act >= 0 && n_act <= kv->n_tok && row0 >= 0, FL_ERR_SHAPE);
  // a residual loop holds at most one row per token: rows row0 .. row0 + n_act - 1 must
  // lie below n_tok (checked in 64 bits, before any launch)
  if (loop >= 2) FL_CHECK((int64_t)row0 + n_act <= (int64_t)kv->n_tok, FL_ERR_SHAPE);
  if (n_act == 0) return FL_OK;
  const int bits = loop == 1 ? kv->base_bits : kv->res_bits[loop];
  FL_CHECK(kv->codes[0][loop] && kv->codes[1][loop], FL_ERR_INVALID_ARG);
  if (bits != 0) FL_CHECK(kv->sz[0][loop] && kv->sz[1][loop], FL_ERR_INVALID_ARG);
  for (int r = 1; r < loop; ++r) {
    FL_CHECK(kv->codes[0][r] && kv->codes[1][r], FL_ERR_INVALID_ARG);
    const int br = r == 1 ? kv->base_bits : kv->res_bits[r];
    if (br != 0) FL_CHECK(kv->sz[0][r] && kv->sz[1][r], FL_ERR_INVALID_ARG);
  }
  return cuda_st(launch_kv_quant(*kv, loop, k_new, v_new, dt, act_tok, n_act, status_word(),
                                 S(stream), loop == 1 ? 0 : row0, true));
}

fl_status fl_kv_reconstruct(const fl_kv_desc* kv, int32_t loop, const int32_t* tok, int32_t n,
                            float* out_k, float* out_v, void* stream) {
  fl_status st = check_kv(kv);
  if (st != FL_OK) return st;
  FL_CHECK(loop >= 1 && loop <= kv->n_loops && n >= 0, FL_ERR_SHAPE);
  if (n == 0) return FL_OK;
  FL_CHECK(tok && out_k && out_v, FL_ERR_INVALID_ARG);
  for (int r = 1; r <= loop; ++r) {
    FL_CHECK(kv->codes[0][r] && kv->codes[1][r], FL_ERR_INVALID_ARG);
    const int b = r == 1 ? kv->base_bits : kv->res_bits[r];
    if (b != 0) FL_CHECK(kv->sz[0][r] && kv->sz[1][r], FL_ERR_INVALID_ARG);
  }
  return cuda_st(launch_kv_reconstruct(*kv, loop, tok, n, out_k, out_v, status_word(), S(stream)));
}

size_t fl_sparse_loop_attn_workspace_bytes(const fl_attn_args* a) {
  return a ? attention_ws_bytes(*a) : 0;
}

fl_status fl_sparse_loop_attn(const fl_attn_args* a, void* stream) {
  fl_status st = check_attn(a);
  if (st != FL_OK) return st;
  if (a->n_q == 0) return FL_OK;
  const size_t need = attention_ws_bytes(*a);
  if (need) FL_CHECK(a->ws && a->ws_bytes >= need, FL_ERR_WORKSPACE);
  return cuda_st(launch_attention_timed(*a, status_word(), S(stream)));
}

size_t fl_sparse_loop_attn_batched_workspace_bytes(int32_t n) {
  return align_up(attention_batched_ws_bytes(n));
}

fl_status fl_sparse_loop_attn_batched(const fl_attn_args* args, int32_t n, void* ws,
                                      size_t ws_bytes, void* stream) {
  FL_CHECK(args && n >= 0, FL_ERR_INVALID_ARG);
  if (n == 0) return FL_OK;
  FL_CHECK(ws && ws_bytes >= fl_sparse_loop_attn_batched_workspace_bytes(n), FL_ERR_WORKSPACE);
  const fl_attn_args& a0 = args[0];
  for (int i = 0; i < n; ++i) {
    const fl_attn_args& a = args[i];
    fl_status st = check_attn(&a);
    if (st != FL_OK) return st;
    FL_CHECK(a.sel != nullptr, FL_ERR_UNSUPPORTED);
    FL_CHECK(a.n_q == a0.n_q && a.kv->n_heads == a0.kv->n_heads &&
             a.kv->head_dim == a0.kv->head_dim && a.sel_stride == a0.sel_stride &&
             a.q_dt == a0.q_dt && a.out_dt == a0.out_dt && a.stat_kind == a0.stat_kind &&
             (a.sel_out != nullptr) == (a0.sel_out != nullptr) && a.k_next == a0.k_next,
             FL_ERR_SHAPE);
    FL_CHECK(sparse_fast_eligible(make_attn_params(a, nullptr)), FL_ERR_UNSUPPORTED);
  }
  if (a0.n_q == 0) return FL_OK;
  timing_begin(TIMED_ATTN, S(stream));
  cudaError_t e = launch_attention_batched(args, n, ws, status_word(), S(stream));
  timing_end(TIMED_ATTN, S(stream));
  return cuda_st(e);
}

size_t fl_block_workspace_bytes(const fl_model* m, int32_t n_rows) {
  if (!m || n_rows <= 0) return 0;
  return block_ws(m, n_rows);
}

fl_status fl_block_qkv(const fl_model* m, int32_t layer, const float* x, int32_t n_rows,
                       const int32_t* pos, float* q, float* k, float* v, void* ws,
                       size_t ws_bytes, void* stream) {
  fl_status st = check_model(m);
  if (st != FL_OK) return st;
  FL_CHECK(layer >= 0 && layer < m->n_layers && n_rows >= 0, FL_ERR_SHAPE);
  if (n_rows == 0) return FL_OK;
  FL_CHECK(x && pos && q && k && v, FL_ERR_INVALID_ARG);
  FL_CHECK(ws && ws_bytes >= block_ws(m, n_rows), FL_ERR_WORKSPACE);
  fl_status rc = prepare_rope(m, ws, S(stream));
  if (rc != FL_OK) return rc;
  return run_qkv(m, layer, x, n_rows, pos, q, k, v, ws, S(stream));
}

fl_status fl_block_qkv_kv(const fl_model* m, int32_t layer, const fl_kv_desc* kv, int32_t loop,
                          const float* x, int32_t n_rows, const int32_t* pos, float* q,
                          float* k_out, float* v_out, void* ws, size_t ws_bytes, void* stream) {
  fl_status st = check_model(m);
  if (st != FL_OK) return st;
  st = check_kv(kv);
  if (st != FL_OK) return st;
  FL_CHECK(layer >= 0 && layer < m->n_layers && n_rows >= 0, FL_ERR_SHAPE);
  FL_CHECK(kv->n_tok == m->n_tok, FL_ERR_SHAPE);
  if (n_rows == 0) return FL_OK;
  FL_CHECK(x && pos && q, FL_ERR_INVALID_ARG);
  FL_CHECK(loop != 1 || n_rows == kv->n_tok, FL_ERR_SHAPE);
  FL_CHECK(kv_fusable(m, n_rows, kv, loop), FL_ERR_UNSUPPORTED);
  for (int r = 1; r <= loop; ++r) {
    FL_CHECK(kv->codes[0][r] && kv->codes[1][r] && kv->sz[0][r] && kv->sz[1][r], FL_ERR_INVALID_ARG);
  }
  FL_CHECK(ws && ws_bytes >= block_ws(m, n_rows), FL_ERR_WORKSPACE);
  fl_status rc = prepare_rope(m, ws, S(stream));
  if (rc != FL_OK) return rc;
  return run_qkv(m, layer, x, n_rows, pos, q, k_out, v_out, ws, S(stream), kv, loop);
}

fl_status fl_block_out_ffn(const fl_model* m, int32_t layer, float* x, int32_t n_rows,
                           const void* attn, void* ws, size_t ws_bytes, void* stream) {
  fl_status st = check_model(m);
  if (st != FL_OK) return st;
  FL_CHECK(layer >= 0 && layer < m->n_layers && n_rows >= 0, FL_ERR_SHAPE);
  if (n_rows == 0) return FL_OK;
  FL_CHECK(x && attn, FL_ERR_INVALID_ARG);
  FL_CHECK(ws && ws_bytes >= block_ws(m, n_rows), FL_ERR_WORKSPACE);
  FL_TRY(cudaMemsetAsync(static_cast<uint8_t*>(ws) + rope_tab_bytes(m), 0,
                         gemm_scratch_flag_bytes(), S(stream)));
  return run_out_ffn(m, layer, x, n_rows, attn, ws, S(stream));
}

// ---------------------------------------------------------------- loop step
// Workspace of the attention calls of a schedule (an upper bound over its loops): the
// store staged as fp16 rows (K^ hi and V^; K^ lo too where a dense call hands statistics
// to a sparse successor) and, for such a call, the dense producer's candidate buffers
// with every token querying at the largest such budget.
static size_t loop_attn_ws(const fl_model* m, const fl_schedule* s) {
  if (!s || m->head_dim != 128) return 0;
  const size_t rows = (size_t)m->n_heads * m->n_tok * m->head_dim * sizeof(uint16_t);
  // the sparse loops' set bitmaps (tiles over plain column ranges): H x active x words
  size_t bm = 0;
  for (int r = 2; r <= s->n_loops && r <= FL_MAX_LOOPS; ++r)
    if (s->col_k[r] > 0) {
      const size_t b = (size_t)m->n_heads * s->n_active[r] * ((m->n_tok + 127) / 128 * 4) * 4;
      bm = b > bm ? b : bm;
    }
  int kmax = 0;
  for (int r = 1; r < s->n_loops && r < FL_MAX_LOOPS; ++r)
    if ((r == 1 || s->col_k[r] == 0) && s->col_k[r + 1] > kmax) kmax = s->col_k[r + 1];
  const size_t sparse = align_up(2 * rows, 256) + bm;
  if (kmax == 0) return sparse;
  AttnParams P{};
  P.H = m->n_heads; P.hd = m->head_dim; P.n_q = m->n_tok; P.k_next = kmax;
  P.kv.n_tok = m->n_tok;
  P.sel_out = reinterpret_cast<uint16_t*>(1);
  const size_t dense = align_up(dense_tile_ws_bytes(P), 256) + 3 * rows;
  return dense > sparse ? dense : sparse;
}

static size_t loop_ws_layout(const fl_model* m, const fl_schedule* sc, Carver* c, int32_t** iota,
                             float** delta, float** q, float** k, float** v, void** attn,
                             void** blk, void** att_ws, size_t* att_bytes) {
  const size_t N = m->n_tok, d = m->d_model;
  *iota = (int32_t*)c->take(N * 4);
  *delta = (float*)c->take(N * 4);
  *q = (float*)c->take(N * d * 4);
  *k = (float*)c->take(N * d * 4);
  *v = (float*)c->take(N * d * 4);
  *attn = c->take(N * d * dt_size(m->dt));
  *blk = c->take(block_ws(m, (int)N));
  *att_bytes = loop_attn_ws(m, sc);
  *att_ws = *att_bytes ? c->take(*att_bytes) : nullptr;
  return c->off;
}

size_t fl_loop_step_workspace_bytes(const fl_model* m, const fl_schedule* s) {
  if (!m || m->n_tok <= 0) return 0;
  Carver c(nullptr);
  int32_t* i; float *dl, *q, *k, *v; void *a, *b, *aw; size_t ab;
  return loop_ws_layout(m, s, &c, &i, &dl, &q, &k, &v, &a, &b, &aw, &ab);
}

fl_status fl_loop_step(const fl_model* m, fl_loop_state* st, const fl_schedule* sc, int32_t loop,
                       void* stream) {
  fl_status rc = check_model(m);
  if (rc != FL_OK) return rc;
  FL_CHECK(st && sc && st->h && st->x_cur && st->x_prev && st->kv, FL_ERR_INVALID_ARG);
  FL_CHECK(sc->n_loops >= 1 && sc->n_loops <= FL_MAX_LOOPS, FL_ERR_SHAPE);
  FL_CHECK(loop >= 1 && loop <= sc->n_loops, FL_ERR_SHAPE);
  FL_CHECK(sc->first_sparse >= 2, FL_ERR_SHAPE);
  const int N = m->n_tok, d = m->d_model, L = m->n_layers;
  const int R = sc->n_loops;
  // schedule consistency
  int prev_k = N;
  for (int r = 2; r <= R; ++r) {
    const int kr = sc->n_active[r];
    FL_CHECK(kr >= 0 && kr <= prev_k, FL_ERR_SHAPE);
    if (r < sc->first_sparse) FL_CHECK(kr == N, FL_ERR_SHAPE);
    prev_k = kr;
    FL_CHECK(sc->col_k[r] >= 0 && sc->col_k[r] + 1 <= (sc->col_k[r] ? st->sel_stride : 1 << 30),
             FL_ERR_SHAPE);
    if (sc->col_k[r] > 0 && r > 2 && sc->col_k[r - 1] > 0)
      FL_CHECK(sc->col_k[r] <= sc->col_k[r - 1], FL_ERR_SHAPE);
  }
  FL_CHECK(st->ws && st->ws_bytes >= fl_loop_step_workspace_bytes(m, sc), FL_ERR_WORKSPACE);
  const bool next_sparse = loop + 1 <= R && sc->col_k[loop + 1] > 0;
  const bool this_sparse = loop >= 2 && sc->col_k[loop] > 0;
  if (next_sparse || this_sparse) {
    FL_CHECK(st->sel && st->mass && st->unsel, FL_ERR_INVALID_ARG);
    for (int l = 0; l < L; ++l) FL_CHECK(st->sel[l] && st->mass[l] && st->unsel[l], FL_ERR_INVALID_ARG);
  }
  for (int l = 0; l < L; ++l) {
    rc = check_kv(&st->kv[l]);
    if (rc != FL_OK) return rc;
    FL_CHECK(st->kv[l].n_tok == N && st->kv[l].n_heads == m->n_heads &&
             st->kv[l].head_dim == m->head_dim && st->kv[l].n_loops >= R, FL_ERR_SHAPE);
  }
  if (loop >= 2) FL_CHECK(st->act[loop] && st->act_pos, FL_ERR_INVALID_ARG);
  if (st->taps) {
    FL_CHECK(st->taps->n >= 0, FL_ERR_SHAPE);
    FL_CHECK(st->taps->n == 0 || st->taps->tok, FL_ERR_INVALID_ARG);
  }

  cudaStream_t s = S(stream);
  int* sw = status_word();
  Carver c(st->ws);
  int32_t* iota; float *delta, *q, *k, *v; void *attn, *blk, *att_ws; size_t att_bytes;
  loop_ws_layout(m, sc, &c, &iota, &delta, &q, &k, &v, &attn, &blk, &att_ws, &att_bytes);
  if (st->delta) delta = st->delta;
  FL_TRY(launch_iota(iota, N, s));

  float* X;
  int M;
  const int32_t* act;
  const size_t row_bytes = (size_t)d * 4;
  if (loop == 1) {
    FL_TRY(cudaMemcpyAsync(st->x_prev, st->h, (size_t)N * row_bytes, cudaMemcpyDeviceToDevice, s));
    X = st->h;
    M = N;
    act = iota;
  } else {
    M = sc->n_active[loop];
    int32_t* a_out = st->act[loop];
    if (loop < sc->first_sparse) {
      FL_TRY(launch_iota(a_out, N, s));
      FL_TRY(launch_iota(st->act_pos, N, s));
    } else {
      const float* cur;
      const float* prv = st->x_prev;
      int rows;
      const int32_t* row_tok;
      if (loop == 2) {
        cur = st->h; rows = N; row_tok = nullptr;
      } else {
        cur = st->x_cur; rows = sc->n_active[loop - 1]; row_tok = st->act[loop - 1];
      }
      FL_TRY(launch_row_delta(cur, prv, FL_F32, rows, d, delta, s));
      FL_TRY(launch_topk_rows(delta, rows, M, row_tok, a_out, st->act_pos, sw, s));
    }
    act = a_out;
    FL_TRY(launch_gather_scatter(FL_GATHER, st->h, st->x_prev, act, M, N, row_bytes, sw, s));
    FL_TRY(cudaMemcpyAsync(st->x_cur, st->x_prev, (size_t)M * row_bytes, cudaMemcpyDeviceToDevice, s));
    X = st->x_cur;
  }
  rc = prepare_rope(m, blk, s);
  if (rc != FL_OK) return rc;
  // inspection taps: rows of the tapped tokens, per layer, into the caller's buffers
  const fl_loop_taps* tp = st->taps;
  const bool tap = tp && tp->n > 0;
  auto tap_rows = [&](const void* src, void* base, size_t row_bytes, int l) -> cudaError_t {
    if (!tap || !base) return cudaSuccess;
    return launch_tap_rows(act, M, tp->tok, tp->n, src,
                           static_cast<uint8_t*>(base) + (size_t)l * tp->n * row_bytes, row_bytes,
                           s);
  };
  for (int l = 0; l < L; ++l) {
    FL_TRY(tap_rows(X, tap ? tp->x_in : nullptr, row_bytes, l));
    // Loop 1 writes the base codes in the projection epilogue. Later loops quantise the
    // residual against K^_{r-1}, whose chain decode is a string of dependent gathers; in
    // the four epilogue warps of the GEMM those stall the tensor pipe (measured: the fused
    // QKV launch took 2.1x the projection plus the separate quantiser), so they keep the
    // separate, wider quantiser launch.
    if (loop == 1 && kv_fusable(m, M, &st->kv[l], loop)) {
      const bool keep_kv = tap && (tp->k || tp->v);   // a tapped step also stores k and v
      rc = run_qkv(m, l, X, M, act, q, keep_kv ? k : nullptr, keep_kv ? v : nullptr, blk, s,
                   &st->kv[l], loop);
      if (rc != FL_OK) return rc;
    } else {
      rc = run_qkv(m, l, X, M, act, q, k, v, blk, s);
      if (rc != FL_OK) return rc;
      FL_TRY(launch_kv_quant(st->kv[l], loop, k, v, FL_F32, loop == 1 ? nullptr : act, M, sw, s));
    }
    fl_attn_args a;
    memset(&a, 0, sizeof(a));
    a.q = q; a.q_dt = FL_F32; a.n_q = M; a.q_tok = act;
    a.kv = &st->kv[l]; a.loop = loop; a.col_bias = m->col_bias;
    a.stat_rows = N; a.sel_stride = st->sel_stride;
    if (this_sparse) {
      a.sel = st->sel[l]; a.mass = st->mass[l]; a.unsel = st->unsel[l];
    }
    if (next_sparse) {
      a.k_next = sc->col_k[loop + 1];
      a.sel_out = st->sel[l]; a.mass_out = st->mass[l]; a.unsel_out = st->unsel[l];
      a.out_stride = st->sel_stride;
      a.stat_kind = sc->stat_kind;
    }
    a.out = attn; a.out_dt = m->dt;
    a.ws = att_ws; a.ws_bytes = att_bytes;
    FL_TRY(tap_rows(q, tap ? tp->q : nullptr, row_bytes, l));
    FL_TRY(tap_rows(k, tap ? tp->k : nullptr, row_bytes, l));
    FL_TRY(tap_rows(v, tap ? tp->v : nullptr, row_bytes, l));
    FL_TRY(launch_attention_timed(a, sw, s));
    FL_TRY(tap_rows(attn, tap ? tp->attn : nullptr, (size_t)d * dt_size(m->dt), l));
    rc = run_out_ffn(m, l, X, M, attn, blk, s);
    if (rc != FL_OK) return rc;
    FL_TRY(tap_rows(X, tap ? tp->x_out : nullptr, row_bytes, l));
  }
  if (loop >= 2)
    FL_TRY(launch_gather_scatter(FL_SCATTER, st->x_cur, st->h, act, M, N, row_bytes, sw, s));
  return FL_OK;
}

}  // extern "C"
