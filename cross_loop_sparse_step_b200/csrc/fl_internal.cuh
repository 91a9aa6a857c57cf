// Internal declarations shared by the library's translation units.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include "../../include/fl.h"

namespace fl {

// ---------------------------------------------------------------- status word
// One int per device (a __device__ variable lives once per device context). Kernels
// receive its address and record the first error with an atomic compare-and-swap.
int* status_word();   // device address for the current device, nullptr on failure

__device__ __forceinline__ void record_error(int* st, int code) {
  if (st) atomicCAS(st, 0, code);
}

// ---------------------------------------------------------------- launch accounting
// Every kernel launch of the library bumps a process-wide counter (read through
// fl_launch_count); GEMM and attention launches can be bracketed by caller events.
void count_launch();

// Programmatic dependent launch: a kernel launched this way may start (its CTAs placed,
// its prologue run) while the previous kernel on the stream drains; it calls
// griddep_wait() before it touches global memory that kernel writes or reads. FL_PDL=0
// turns it off.
bool pdl_enabled();
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t s, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl_enabled() ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kern, static_cast<Args&&>(args)...);
}
__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
enum TimedKind { TIMED_GEMM = 0, TIMED_ATTN = 1, TIMED_KINDS = 2 };
void timing_begin(int kind, cudaStream_t s);
void timing_end(int kind, cudaStream_t s);

// ---------------------------------------------------------------- KV store view
// By-value copy of fl_kv_desc for kernels (loops up to FL_MAX_LOOPS).
struct KvView {
  int n_tok, H, hd, g, base_bits, n_loops;
  int res_bits[FL_MAX_LOOPS + 1];
  const uint8_t* codes[2][FL_MAX_LOOPS + 1];
  const uint16_t* sz[2][FL_MAX_LOOPS + 1];
  const int32_t* slot;
};

inline KvView make_view(const fl_kv_desc& d) {
  KvView v;
  v.n_tok = d.n_tok; v.H = d.n_heads; v.hd = d.head_dim; v.g = d.group;
  v.base_bits = d.base_bits; v.n_loops = d.n_loops;
  for (int r = 0; r <= FL_MAX_LOOPS; ++r) {
    v.res_bits[r] = d.res_bits[r];
    for (int kv = 0; kv < 2; ++kv) { v.codes[kv][r] = d.codes[kv][r]; v.sz[kv][r] = d.sz[kv][r]; }
  }
  v.slot = d.slot;
  return v;
}

__device__ __forceinline__ float half_bits_to_float(uint16_t b) {
  return __half2float(__ushort_as_half(b));
}

// Decode N consecutive elements [e0, e0+N) of one stored row (row `row` of loop
// r's arrays, head h). The N elements lie in one quantisation group. Codes of b
// bits sit little-endian, low bits first. Returns deq = fmaf(code, s, z) or the raw
// binary32 values when bits == 0.
template <int N>
__device__ __forceinline__ void decode_run(const KvView& kv, int which, int r, int bits,
                                           int row, int h, int e0, float* out) {
  const int hd = kv.hd;
  if (bits == 0) {
    const float* p = reinterpret_cast<const float*>(kv.codes[which][r]) +
                     ((size_t)row * kv.H + h) * hd + e0;
#pragma unroll
    for (int i = 0; i < N; ++i) out[i] = p[i];
    return;
  }
  const size_t rowbytes = (size_t)hd * bits / 8;
  const uint8_t* cp = kv.codes[which][r] + ((size_t)row * kv.H + h) * rowbytes;
  const uint32_t szw = reinterpret_cast<const uint32_t*>(kv.sz[which][r])
      [((size_t)row * kv.H + h) * (hd / kv.g) + e0 / kv.g];
  const float s = half_bits_to_float((uint16_t)(szw & 0xFFFFu));
  const float z = half_bits_to_float((uint16_t)(szw >> 16));
  const int mask = (1 << bits) - 1;
#pragma unroll
  for (int i = 0; i < N; ++i) {
    const int bit = (e0 + i) * bits;
    const int code = (cp[bit >> 3] >> (bit & 7)) & mask;
    out[i] = __fmaf_rn((float)code, s, z);
  }
}

// K^ or V^ of token t at loop `upto` for elements [e0, e0+N): base, then every loop
// 2..upto whose slot table lists t, added in order (a raw loop replaces the value).
template <int N>
__device__ __forceinline__ void reconstruct(const KvView& kv, int which, int upto, int t,
                                            int h, int e0, float* acc) {
  decode_run<N>(kv, which, 1, kv.base_bits, t, h, e0, acc);
  for (int r = 2; r <= upto; ++r) {
    const int row = kv.slot[(size_t)r * kv.n_tok + t];
    if (row < 0) continue;
    float d[N];
    const int bits = kv.res_bits[r];
    decode_run<N>(kv, which, r, bits, row, h, e0, d);
    if (bits == 0) {
#pragma unroll
      for (int i = 0; i < N; ++i) acc[i] = d[i];
    } else {
#pragma unroll
      for (int i = 0; i < N; ++i) acc[i] = __fadd_rn(acc[i], d[i]);
    }
  }
}

// Arguments of the attention kernels (a by-value copy of fl_attn_args plus the store view).
// fp16 operand rows of a whole store at one loop, [H][n_tok][hd] each (kv_stage.cu);
// klo (K^ - fp16(K^) as fp16) only where a split-operand pass needs it.
struct KvStage {
  __half* khi;
  __half* klo;
  __half* vhi;
};
size_t kv_stage_bytes(const KvView& kv, bool with_lo);
cudaError_t launch_kv_stage(const KvView& kv, int loop, void* buf, bool with_lo, KvStage* out,
                            cudaStream_t s);

struct AttnParams {
  const void* q; int q_bf16;
  const int32_t* q_tok;
  int n_q, H, hd;
  float scale;
  KvView kv;
  int loop;
  const float* bias;
  const uint16_t* sel; const float* mass; const float* unsel;
  int stat_rows, sel_stride;
  const int32_t* q_row;
  int k_next;
  uint16_t* sel_out; float* mass_out; float* unsel_out;
  int out_stride, stat_kind;
  const float* vnorm;
  void* out; int out_bf16;
  int* st;
  KvStage stage;   // khi == NULL: the kernels decode the store themselves
  // bitmaps of the carried sets, [H][n_q][bm_words] (bit j of word w: column 32 w + j),
  // for query tiles that walk plain column ranges; NULL: tiles walk their sets' union
  const uint32_t* sel_bm;
  int bm_words;
};
// Sparse calls whose tiles walk plain column ranges (their unions are nearly every column
// before the tile: the budget is a sizeable fraction of the prompt), the bitmaps' size,
// and their construction from the call's column sets.
bool sparse_contig(const AttnParams& P);
size_t sel_bitmap_bytes(const AttnParams& P);
cudaError_t launch_sel_bitmap(AttnParams& P, void* buf, cudaStream_t s, bool record = true);

// attention calls by path (fl_attn_path_counts)
enum AttnPath : int { PATH_TILE_CONTIG = 0, PATH_TILE_UNION, PATH_TILE_DECODE, PATH_DENSE_TILE,
                      PATH_SPARSE_WARP, PATH_DENSE_WARP, PATH_GENERAL, PATH_SPARSE_STREAM,
                      N_ATTN_PATHS };
void count_attn_path(int path);
long long attn_path_count(int path);
bool sparse_tile_eligible(const AttnParams& P);
// Sparse calls with few queries (decode): one CTA per (query, head) streaming its carried
// columns from the quantised store (attention_decode.cu).
bool sparse_decode_eligible(const AttnParams& P);
cudaError_t launch_attn_decode(const AttnParams& P, cudaStream_t s);
cudaError_t launch_attn_decode_batched(const AttnParams& P0, const AttnParams* Ps_dev, int n,
                                       cudaStream_t s);
cudaError_t launch_attn_tile(const AttnParams& P, cudaStream_t s);
cudaError_t launch_attn_tile_batched(const AttnParams& P0, const AttnParams* Ps_dev, int n,
                                     cudaStream_t s);
bool sparse_fast_eligible(const AttnParams& P);
cudaError_t launch_attn_sparse_fast(const AttnParams& P, cudaStream_t s);
cudaError_t launch_attn_sparse_batched(const AttnParams& P0, const AttnParams* Ps_dev, int n,
                                       int loop_max, cudaStream_t s);
AttnParams make_attn_params(const fl_attn_args& a, int* st);
size_t attention_batched_ws_bytes(int n);
cudaError_t launch_attention_batched(const fl_attn_args* args, int n, void* ws, int* st,
                                     cudaStream_t s);
bool dense_fast_eligible(const AttnParams& P);
// The tensor-core dense producer (query tiles; statistics by candidates and an exact
// selection), its workspace, and the per-query exact finish of listed rows.
bool dense_tile_eligible(const AttnParams& P);
size_t dense_tile_ws_bytes(const AttnParams& P);
cudaError_t launch_attn_dense_tile(const AttnParams& P, void* ws, cudaStream_t s);
bool dense_rows_supported(const AttnParams& P);
bool dense_list_supported(const AttnParams& P);
cudaError_t launch_attention_list(const AttnParams& P, const int* list, const int* count,
                                  cudaStream_t s);
cudaError_t launch_attn_dense_rows(const AttnParams& P, const int* list, const int* count,
                                   cudaStream_t s);
cudaError_t launch_attn_dense_fast(const AttnParams& P, cudaStream_t s);

template <typename T> __device__ __forceinline__ float to_f32(T x);
template <> __device__ __forceinline__ float to_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 x) {
  return __bfloat162float(x);
}
template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
  return __float2bfloat16_rn(x);
}

inline size_t dt_size(fl_dtype dt) { return dt == FL_BF16 ? 2 : 4; }
inline size_t align_up(size_t x, size_t a = 256) { return (x + a - 1) / a * a; }

// ---------------------------------------------------------------- internal launches
// All return cudaSuccess or the launch error. Arguments are validated by callers.
cudaError_t launch_row_delta(const void* cur, const void* prev, fl_dtype dt, int n_rows,
                             int d, float* delta, cudaStream_t s);
cudaError_t launch_topk_rows(const float* delta, int n, int k, const int32_t* row_tok,
                             int32_t* out_tok, int32_t* out_pos, int* st, cudaStream_t s);
cudaError_t launch_gather_scatter(fl_gs_op op, const void* src, void* dst, const int32_t* idx,
                                  int n_idx, int n_full, size_t row_bytes, int* st,
                                  cudaStream_t s);
// append: keep the slot entries of other tokens and write rows row0.. (decode);
// otherwise rows 0.. and slot[loop] rewritten for exactly the given tokens.
cudaError_t launch_kv_quant(const fl_kv_desc& kv, int loop, const void* k_new,
                            const void* v_new, fl_dtype dt, const int32_t* act_tok, int n_act,
                            int* st, cudaStream_t s, int row0 = 0, bool append = false);
cudaError_t launch_attention(const fl_attn_args& a, int* st, cudaStream_t s);
cudaError_t launch_kv_reconstruct(const fl_kv_desc& kv, int loop, const int32_t* tok, int n,
                                  float* out_k, float* out_v, int* st, cudaStream_t s);
size_t attention_ws_bytes(const fl_attn_args& a);

// Scratch of the tensor-core GEMM's stream-K split: hand-over flags (zero before the first
// launch that uses them; every launch leaves them at zero) and partial accumulator tiles.
struct GemmScratch {
  int* flag; int n_flag;
  float* part; size_t part_bytes;
};
size_t gemm_scratch_bytes();            // for the current device
GemmScratch gemm_scratch_at(void* p);   // the layout of gemm_scratch_bytes() bytes at p
size_t gemm_scratch_flag_bytes();       // the leading flag block (to zero)

// C[M x N] (binary32, leading dim ldc) = or += A[M x K] . W[N x K]^T
enum GemmEpi { EPI_STORE = 0, EPI_ADD = 1 };
cudaError_t launch_gemm(fl_dtype dt, const void* A, const void* W, float* C, int M, int N,
                        int K, int ldc, GemmEpi epi, cudaStream_t s,
                        const GemmScratch* scr = nullptr);
cudaError_t launch_rmsnorm(const float* x, const float* gamma, float eps, void* out,
                           fl_dtype dt, int M, int d, cudaStream_t s);
cudaError_t launch_rope_split(const float* qkv, const int32_t* pos, int M, int H, int hd,
                              float theta, float* q, float* k, float* v, cudaStream_t s);
cudaError_t launch_rope_table(float2* tab, int n_tok, int hd, float theta, cudaStream_t s);
cudaError_t launch_swiglu(const float* gu, int M, int F, void* out, fl_dtype dt,
                          cudaStream_t s);
cudaError_t launch_iota(int32_t* p, int n, cudaStream_t s);
// Copies the rows of the tokens tok[0, n) found in the ascending list act[0, M) from src
// (row p = act position p) to dst row i; tokens not in act are skipped.
cudaError_t launch_tap_rows(const int32_t* act, int M, const int32_t* tok, int n,
                            const void* src, void* dst, size_t row_bytes, cudaStream_t s);
cudaError_t launch_fill_i32(int32_t* p, int32_t v, size_t n, cudaStream_t s);

}  // namespace fl
