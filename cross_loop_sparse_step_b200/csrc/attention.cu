// Loop-aware sparse attention with cached mass, and the dense causal attention that
// produces the column statistics (FlashLoop §4.2 "Loop-Aware Sparse Attention").
//
// One CTA per (query, head). Columns are processed by groups of 8 lanes; lane l of a
// group owns hd/8 consecutive elements, so a 128-element head slice is one 16-byte
// run of base codes per lane. K^ and V^ are dequantised on the load path (base plus
// the residual chain of the loops that rewrote the column), never materialised.
//   1. scores s = q . K^[j] / sqrt(hd) + b_j of every column into shared memory;
//   2. softmax over the columns; sparse: p~ = m * softmax (m = cached mass);
//   3. statistics for the next loop (optional): top-k of c = P * ||V^|| (or P) by a
//      block radix select over the binary32 bits, ties to the smaller column;
//   4. o = u + sum P V^ (u = carried unselected contribution, 0 when dense), and the
//      next loop's m' and u' from the kept / dropped columns.
#include <float.h>
#include <vector>
#include <atomic>

#include "fl_internal.cuh"

namespace fl {
namespace {


template <int NT>
__device__ __forceinline__ float block_reduce(float v, bool is_max, float* red) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const float y = __shfl_xor_sync(0xffffffffu, v, o);
    v = is_max ? fmaxf(v, y) : v + y;
  }
  __syncthreads();
  if (lane == 0) red[w] = v;
  __syncthreads();
  float r = red[0];
  for (int i = 1; i < NT / 32; ++i) r = is_max ? fmaxf(r, red[i]) : r + red[i];
  __syncthreads();
  return r;
}

// Inclusive scan of one int per thread over the CTA; *total gets the CTA sum.
template <int NT>
__device__ __forceinline__ int block_scan(int x, int* ws, int* total) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  __syncthreads();
  if (lane == 31) ws[w] = x;
  __syncthreads();
  int add = 0, tot = 0;
  for (int i = 0; i < NT / 32; ++i) {
    if (i < w) add += ws[i];
    tot += ws[i];
  }
  *total = tot;
  __syncthreads();
  return x + add;
}

__device__ __forceinline__ int col_of(const uint16_t* cols, int idx) {
  return cols ? (int)cols[idx] : idx;
}

// One CTA's work: query qi, head h (every early return is CTA-uniform).
template <int NT, int EPL>
__device__ __forceinline__ void attention_cta(const AttnParams& P, int max_cols, int qi, int h) {
  extern __shared__ __align__(16) uint8_t smem[];
  constexpr int NG = NT / 8;                    // column groups
  float* p = reinterpret_cast<float*>(smem);    // [max_cols] scores, then probabilities
  float* red = p + max_cols;                    // [NG * hd] partial sums
  float* red2 = red + NG * P.hd;                // [NG * hd] partial unselected sums
  int* iws = reinterpret_cast<int*>(red2 + NG * P.hd);   // [256 + 64] scratch
  uint8_t* mark = reinterpret_cast<uint8_t*>(iws + 320);  // [max_cols]
  uint16_t* cols = P.sel ? reinterpret_cast<uint16_t*>(mark + ((max_cols + 15) & ~15)) : nullptr;
  __shared__ float s_red[32];

  const int tid = threadIdx.x;
  const int grp = tid >> 3, li = tid & 7;
  const int hd = P.hd;
  const int t = P.q_tok[qi];
  const bool sparse = P.sel != nullptr;
  const bool want_stats = P.sel_out != nullptr;
  if (t < 0 || t >= P.kv.n_tok) {
    if (tid == 0) record_error(P.st, FL_ERR_RANGE);
    return;
  }
  const int srow = P.q_row ? P.q_row[qi] : t;
  if ((sparse || want_stats) && (srow < 0 || srow >= P.stat_rows)) {
    if (tid == 0) record_error(P.st, FL_ERR_RANGE);
    return;
  }

  // ---- column list
  int n_cols;
  float m_in = 1.f;
  if (sparse) {
    const uint16_t* srow_p = P.sel + ((size_t)h * P.stat_rows + srow) * P.sel_stride;
    int cnt = 0;
    for (int i = tid; i < P.sel_stride; i += NT) {
      const uint16_t c = srow_p[i];
      cols[i] = c;
      cnt += (c != FL_SENTINEL) ? 1 : 0;
    }
    n_cols = (int)block_reduce<NT>((float)cnt, false, s_red);
    m_in = P.mass[(size_t)h * P.stat_rows + srow];
  } else {
    n_cols = t + 1;
  }

  // ---- query slice of this lane
  const int e0 = li * EPL;
  float qv[EPL];
  {
    const size_t off = ((size_t)qi * P.H + h) * hd + e0;
    if (P.q_bf16) {
      const __nv_bfloat16* q = reinterpret_cast<const __nv_bfloat16*>(P.q) + off;
#pragma unroll
      for (int j = 0; j < EPL; ++j) qv[j] = __bfloat162float(q[j]);
    } else {
      const float* q = reinterpret_cast<const float*>(P.q) + off;
#pragma unroll
      for (int j = 0; j < EPL; ++j) qv[j] = q[j];
    }
  }

  // ---- 1. scores
  float lmax = -FLT_MAX;
  for (int base = 0; base < n_cols; base += NG) {
    const int idx = base + grp;
    float dot = 0.f;
    int c = -1;
    if (idx < n_cols) {
      c = col_of(cols, idx);
      if (c <= t) {
        float kk[EPL];
        reconstruct<EPL>(P.kv, 0, P.loop, c, h, e0, kk);
#pragma unroll
        for (int j = 0; j < EPL; ++j) dot = fmaf(qv[j], kk[j], dot);
      }
    }
    dot += __shfl_xor_sync(0xffffffffu, dot, 1);
    dot += __shfl_xor_sync(0xffffffffu, dot, 2);
    dot += __shfl_xor_sync(0xffffffffu, dot, 4);
    if (idx < n_cols && li == 0) {
      float s;
      if (c > t) {  // a carried column beyond the query's position: excluded
        record_error(P.st, FL_ERR_RANGE);
        s = -INFINITY;
      } else {
        s = dot * P.scale + (P.bias ? P.bias[c] : 0.f);
      }
      p[idx] = s;
      lmax = fmaxf(lmax, s);
    }
  }
  const float M = block_reduce<NT>(lmax, true, s_red);
  // ---- 2. softmax
  float lsum = 0.f;
  for (int idx = tid; idx < n_cols; idx += NT) {
    const float e = expf(p[idx] - M);
    p[idx] = e;
    lsum += e;
  }
  const float Z = block_reduce<NT>(lsum, false, s_red);
  const float wmul = (sparse ? m_in : 1.f) / Z;
  for (int idx = tid; idx < n_cols; idx += NT) p[idx] = p[idx] * wmul;
  __syncthreads();

  // ---- 3. selection of the next loop's columns
  int n_keep = n_cols;
  if (want_stats) {
    const int k = P.k_next;
    if (n_cols - 1 <= k) {
      for (int idx = tid; idx < n_cols; idx += NT) mark[idx] = 1;
    } else {
      int* hist = iws;          // 256
      int* sc = iws + 256;      // scan scratch (<= 32) + broadcast
      uint32_t prefix = 0, pmask = 0, need = (uint32_t)k;
      for (int shift = 24; shift >= 0; shift -= 8) {
        for (int i = tid; i < 256; i += NT) hist[i] = 0;
        __syncthreads();
        for (int idx = 1 + tid; idx < n_cols; idx += NT) {
          const int c = col_of(cols, idx);
          float cv = c <= t ? p[idx] : 0.f;
          if (P.stat_kind == FL_STAT_PV && c <= t) cv *= P.vnorm[(size_t)c * P.H + h];
          const uint32_t b = __float_as_uint(cv);
          if ((b & pmask) == prefix) atomicAdd(&hist[(b >> shift) & 255u], 1);
        }
        __syncthreads();
        if (tid == 0) {
          uint32_t above = 0;
          int dg = 255;
          for (; dg > 0; --dg) {
            if (above + (uint32_t)hist[dg] >= need) break;
            above += (uint32_t)hist[dg];
          }
          sc[40] = (int)(prefix | ((uint32_t)dg << shift));
          sc[41] = (int)(need - above);
        }
        __syncthreads();
        prefix = (uint32_t)sc[40];
        need = (uint32_t)sc[41];
        pmask |= 255u << shift;
        __syncthreads();
      }
      if (tid == 0) mark[0] = 1;
      int eq_seen = 0;
      for (int base = 1; base < n_cols; base += NT) {
        const int idx = base + tid;
        uint32_t b = 0;
        const bool valid = idx < n_cols;
        if (valid) {
          const int c = col_of(cols, idx);
          float cv = c <= t ? p[idx] : 0.f;
          if (P.stat_kind == FL_STAT_PV && c <= t) cv *= P.vnorm[(size_t)c * P.H + h];
          b = __float_as_uint(cv);
        }
        const int is_eq = (valid && b == prefix) ? 1 : 0;
        int tot;
        const int incl = block_scan<NT>(is_eq, sc, &tot);
        if (valid) {
          const int rank = eq_seen + incl - is_eq;
          mark[idx] = (b > prefix || (is_eq && (uint32_t)rank < need)) ? 1 : 0;
        }
        eq_seen += tot;
      }
      n_keep = k + 1;
    }
    __syncthreads();
  }

  // ---- 4. value pass
  float oacc[EPL], uacc[EPL];
#pragma unroll
  for (int j = 0; j < EPL; ++j) { oacc[j] = 0.f; uacc[j] = 0.f; }
  for (int base = 0; base < n_cols; base += NG) {
    const int idx = base + grp;
    if (idx < n_cols) {
      const int c = col_of(cols, idx);
      const float w = p[idx];
      if (c <= t && w != 0.f) {
        float vv[EPL];
        reconstruct<EPL>(P.kv, 1, P.loop, c, h, e0, vv);
        const bool drop = want_stats && !mark[idx];
#pragma unroll
        for (int j = 0; j < EPL; ++j) {
          oacc[j] = fmaf(w, vv[j], oacc[j]);
          if (drop) uacc[j] = fmaf(w, vv[j], uacc[j]);
        }
      }
    }
  }
#pragma unroll
  for (int j = 0; j < EPL; ++j) {
    red[grp * hd + e0 + j] = oacc[j];
    red2[grp * hd + e0 + j] = uacc[j];
  }
  __syncthreads();
  const size_t ob = ((size_t)qi * P.H + h) * hd;
  const float* u_in = sparse ? P.unsel + ((size_t)h * P.stat_rows + srow) * hd : nullptr;
  for (int e = tid; e < hd; e += NT) {
    float so = 0.f, su = 0.f;
    for (int gI = 0; gI < NG; ++gI) { so += red[gI * hd + e]; su += red2[gI * hd + e]; }
    const float base_u = sparse ? u_in[e] : 0.f;
    const float o = base_u + so;
    if (P.out_bf16) reinterpret_cast<__nv_bfloat16*>(P.out)[ob + e] = __float2bfloat16_rn(o);
    else reinterpret_cast<float*>(P.out)[ob + e] = o;
    if (want_stats) {
      P.unsel_out[((size_t)h * P.stat_rows + srow) * hd + e] = base_u + su;
    }
  }
  if (!want_stats) return;
  // mass of the kept columns and the kept column list (ascending, padded)
  float lm = 0.f;
  for (int idx = tid; idx < n_cols; idx += NT)
    if (mark[idx]) lm += p[idx];
  float m_out = block_reduce<NT>(lm, false, s_red);
  if (sparse && n_cols - 1 <= P.k_next) m_out = m_in;  // budget not shrinking: m' = m
  uint16_t* so = P.sel_out + ((size_t)h * P.stat_rows + srow) * P.out_stride;
  int written = 0;
  for (int base = 0; base < n_cols; base += NT) {
    const int idx = base + tid;
    const int keep = (idx < n_cols && mark[idx]) ? 1 : 0;
    int tot;
    const int incl = block_scan<NT>(keep, iws + 256, &tot);
    if (keep) {
      const int pos = written + incl - 1;
      if (pos < P.out_stride) so[pos] = (uint16_t)col_of(cols, idx);
    }
    written += tot;
  }
  for (int i = written + tid; i < P.out_stride; i += NT) so[i] = (uint16_t)FL_SENTINEL;
  if (tid == 0) P.mass_out[(size_t)h * P.stat_rows + srow] = m_out;
  (void)n_keep;
}

template <int NT, int EPL>
__global__ void __launch_bounds__(NT) k_attention(AttnParams P, int max_cols) {
  attention_cta<NT, EPL>(P, max_cols, blockIdx.x / P.H, blockIdx.x % P.H);
}

// The (query, head) pairs list[0, *count) (entries h * n_q + query), CTAs striding over
// the list: the exact finish of rows the tensor-core dense producer could not rank.
template <int NT, int EPL>
__global__ void __launch_bounds__(NT) k_attention_list(AttnParams P, int max_cols,
                                                       const int* list, const int* count) {
  const int n = *count;
  for (int x = blockIdx.x; x < n; x += gridDim.x) {
    __syncthreads();   // the previous row's shared-memory reads are done
    const int rh = list[x];
    attention_cta<NT, EPL>(P, max_cols, rh % P.n_q, rh / P.n_q);
  }
}

size_t smem_bytes(int nt, int hd, int max_cols, bool sparse) {
  const int NG = nt / 8;
  size_t b = (size_t)max_cols * 4 + 2 * (size_t)NG * hd * 4 + 320 * 4;
  b += (size_t)((max_cols + 15) & ~15);
  if (sparse) b += (size_t)max_cols * 2;
  return b;
}

template <int NT, int EPL>
cudaError_t launch_t(const AttnParams& P, int max_cols, cudaStream_t s) {
  const size_t sm = smem_bytes(NT, P.hd, max_cols, P.sel != nullptr);
  if (sm > 227 * 1024) return cudaErrorInvalidValue;
  auto kern = k_attention<NT, EPL>;
  static int attr_bytes[128] = {0};   // per device: the largest size allowed so far
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 128) return cudaErrorInvalidDevice;
  if ((int)sm > attr_bytes[dev]) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
    if (e != cudaSuccess) return e;
    attr_bytes[dev] = (int)sm;
  }
  kern<<<P.n_q * P.H, NT, sm, s>>>(P, max_cols);
  count_launch();
  return cudaGetLastError();
}

}  // namespace

// Listed rows of a dense call with statistics, by the general kernel (any store).
bool dense_list_supported(const AttnParams& P) {
  return smem_bytes(256, P.hd, P.kv.n_tok, false) <= 227 * 1024;
}

cudaError_t launch_attention_list(const AttnParams& P, const int* list, const int* count,
                                  cudaStream_t s) {
  const int max_cols = P.kv.n_tok;
  const size_t sm = smem_bytes(256, P.hd, max_cols, false);
  if (sm > 227 * 1024) return cudaErrorInvalidValue;
  auto kern = P.hd == 128 ? k_attention_list<256, 16> : k_attention_list<256, 8>;
  static int attr_bytes[2][128] = {{0}};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 128) return cudaErrorInvalidDevice;
  int& have = attr_bytes[P.hd == 128 ? 1 : 0][dev];
  if ((int)sm > have) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
    if (e != cudaSuccess) return e;
    have = (int)sm;
  }
  int sms = 148;
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  kern<<<sms, 256, sm, s>>>(P, max_cols, list, count);
  count_launch();
  return cudaGetLastError();
}

static bool attn_tile_enabled();

// Sparse calls of at most this many queries stream each query's columns (a query tile
// would be nearly empty and its union would not be shared).
constexpr int kStreamMaxQ = 32;

static std::atomic<long long> g_attn_paths[N_ATTN_PATHS];
void count_attn_path(int path) {
  if (path >= 0 && path < N_ATTN_PATHS) g_attn_paths[path].fetch_add(1, std::memory_order_relaxed);
}
long long attn_path_count(int path) {
  return path >= 0 && path < N_ATTN_PATHS ? g_attn_paths[path].load() : 0;
}


// Staging of the store as fp16 rows (kv_stage.cu) pays off where several query tiles of a
// head would decode the same columns: the dense producer, and sparse calls of more than
// one tile. A single-tile call (decode) gathers its few columns straight from the store.
static bool stage_sparse(const AttnParams& P) { return P.n_q > 128; }

// Workspace of a call: the dense producer's candidate buffers, then the staged rows.
size_t attention_ws_bytes(const fl_attn_args& a) {
  if (!a.kv || !attn_tile_enabled()) return 0;
  const AttnParams P = make_attn_params(a, nullptr);
  if (a.sel) {
    if (!sparse_tile_eligible(P) || !stage_sparse(P)) return 0;
    return align_up(kv_stage_bytes(P.kv, false)) + sel_bitmap_bytes(P);
  }
  if (!dense_tile_eligible(P)) return 0;
  return align_up(dense_tile_ws_bytes(P)) + kv_stage_bytes(P.kv, P.sel_out != nullptr);
}


AttnParams make_attn_params(const fl_attn_args& a, int* st) {
  AttnParams P{};
  P.q = a.q; P.q_bf16 = a.q_dt == FL_BF16;
  P.q_tok = a.q_tok; P.n_q = a.n_q; P.H = a.kv->n_heads; P.hd = a.kv->head_dim;
  P.scale = 1.0f / sqrtf((float)P.hd);
  P.kv = make_view(*a.kv); P.loop = a.loop; P.bias = a.col_bias;
  P.sel = a.sel; P.mass = a.mass; P.unsel = a.unsel;
  P.stat_rows = a.stat_rows; P.sel_stride = a.sel_stride; P.q_row = a.q_row;
  P.k_next = a.k_next; P.sel_out = a.sel_out; P.mass_out = a.mass_out; P.unsel_out = a.unsel_out;
  P.out_stride = a.out_stride; P.stat_kind = a.stat_kind; P.vnorm = a.kv->vnorm;
  P.out = a.out; P.out_bf16 = a.out_dt == FL_BF16; P.st = st;
  return P;
}

size_t attention_batched_ws_bytes(int n) { return (size_t)(n > 0 ? n : 0) * sizeof(AttnParams); }

cudaError_t launch_attention_batched(const fl_attn_args* args, int n, void* ws, int* st,
                                     cudaStream_t s) {
  if (n <= 0) return cudaSuccess;
  std::vector<AttnParams> host(n);
  for (int i = 0; i < n; ++i) host[i] = make_attn_params(args[i], st);
  // pageable source: the copy is staged before this call returns
  cudaError_t e = cudaMemcpyAsync(ws, host.data(), n * sizeof(AttnParams), cudaMemcpyHostToDevice, s);
  if (e != cudaSuccess) return e;
  bool stream = attn_tile_enabled(), tile = stream;
  for (int i = 0; stream && i < n; ++i) stream = sparse_decode_eligible(host[i]) && host[i].n_q <= kStreamMaxQ;
  for (int i = 0; tile && i < n; ++i) tile = sparse_tile_eligible(host[i]);
  if (stream) {
    count_attn_path(PATH_SPARSE_STREAM);
    return launch_attn_decode_batched(host[0], static_cast<const AttnParams*>(ws), n, s);
  }
  count_attn_path(tile ? PATH_TILE_DECODE : PATH_SPARSE_WARP);
  if (tile) return launch_attn_tile_batched(host[0], static_cast<const AttnParams*>(ws), n, s);
  int loop_max = 1;   // shared-memory slices sized for the deepest call
  for (int i = 0; i < n; ++i) loop_max = host[i].loop > loop_max ? host[i].loop : loop_max;
  return launch_attn_sparse_batched(host[0], static_cast<const AttnParams*>(ws), n, loop_max, s);
}

// The query-tile tensor-core form of the sparse attention unless FL_ATTN_TILE=0 (then
// the warp-per-query kernel runs every sparse call).
static bool attn_tile_enabled() {
  static int on = -1;
  if (on < 0) {
    const char* e = getenv("FL_ATTN_TILE");
    on = (e && atoi(e) == 0) ? 0 : 1;
  }
  return on == 1;
}

cudaError_t launch_attention(const fl_attn_args& a, int* st, cudaStream_t s) {
  if (a.n_q <= 0) return cudaSuccess;
  AttnParams P = make_attn_params(a, st);
  const bool sparse = a.sel != nullptr;
  uint8_t* ws = static_cast<uint8_t*>(a.ws);
  if (sparse && attn_tile_enabled() && P.n_q <= kStreamMaxQ && sparse_decode_eligible(P)) {
    count_attn_path(PATH_SPARSE_STREAM);
    return launch_attn_decode(P, s);
  }
  if (sparse && attn_tile_enabled() && sparse_tile_eligible(P)) {
    const size_t sb = align_up(kv_stage_bytes(P.kv, false));
    if (stage_sparse(P) && ws && a.ws_bytes >= sb) {
      cudaError_t e = launch_kv_stage(P.kv, P.loop, ws, false, &P.stage, s);
      if (e != cudaSuccess) return e;
      if (a.ws_bytes >= sb + sel_bitmap_bytes(P)) {
        e = launch_sel_bitmap(P, ws + sb, s);
        if (e != cudaSuccess) return e;
      } else {
        P.stage.khi = nullptr;   // staged rows without set bitmaps: decode in the tiles
      }
    }
    count_attn_path(!P.stage.khi ? PATH_TILE_DECODE : (sparse_contig(P) ? PATH_TILE_CONTIG : PATH_TILE_UNION));
    return launch_attn_tile(P, s);
  }
  if (!sparse && attn_tile_enabled() && dense_tile_eligible(P)) {
    const size_t db = dense_tile_ws_bytes(P);
    if (P.sel_out && a.ws_bytes < db) return cudaErrorInvalidValue;
    const bool lo = P.sel_out != nullptr;
    if (ws && a.ws_bytes >= align_up(db) + kv_stage_bytes(P.kv, lo)) {
      const cudaError_t e = launch_kv_stage(P.kv, P.loop, ws + align_up(db), lo, &P.stage, s);
      if (e != cudaSuccess) return e;
    }
    count_attn_path(PATH_DENSE_TILE);
    return launch_attn_dense_tile(P, a.ws, s);
  }
  if (sparse && sparse_fast_eligible(P)) { count_attn_path(PATH_SPARSE_WARP); return launch_attn_sparse_fast(P, s); }
  if (!sparse && dense_fast_eligible(P)) { count_attn_path(PATH_DENSE_WARP); return launch_attn_dense_fast(P, s); }
  count_attn_path(PATH_GENERAL);
  const int max_cols = sparse ? a.sel_stride : a.kv->n_tok;
  if (sparse) {
    if (P.hd == 128) return launch_t<128, 16>(P, max_cols, s);
    return launch_t<128, 8>(P, max_cols, s);
  }
  if (P.hd == 128) return launch_t<256, 16>(P, max_cols, s);
  return launch_t<256, 8>(P, max_cols, s);
}

}  // namespace fl
