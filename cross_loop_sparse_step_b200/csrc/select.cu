// Active-token selection: normalized hidden-state change per row and an exact
// top-k of rows (FlashLoop §4.1 "Cross-Loop Token-Sparse Updates").
//
// row_delta: one warp per row, 16-byte vector loads of both states, binary32
//   accumulation of sum (cur - prev)^2 and sum prev^2, warp-shuffle reduction.
// topk_rows: one CTA of 1024 threads. A 4-pass radix select over the 32 bits of the
//   (non-negative) binary32 deltas finds the k-th largest value V and how many rows
//   equal to V are still needed; a block scan in row order then keeps every row with
//   delta > V and the first needed rows with delta == V (equal deltas: the smaller
//   row wins), writing them in ascending row order.
#include "fl_internal.cuh"

namespace fl {
namespace {

template <typename T>
struct Vec;  // 16-byte vector of T
template <> struct Vec<float> { static constexpr int N = 4; };
template <> struct Vec<__nv_bfloat16> { static constexpr int N = 8; };

template <typename T>
__device__ __forceinline__ void load16(const T* p, float* out) {
  const uint4 u = *reinterpret_cast<const uint4*>(p);
  if constexpr (sizeof(T) == 4) {
    out[0] = __uint_as_float(u.x); out[1] = __uint_as_float(u.y);
    out[2] = __uint_as_float(u.z); out[3] = __uint_as_float(u.w);
  } else {
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      out[2 * i] = __uint_as_float(w[i] << 16);
      out[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
  }
}

template <typename T>
__global__ void __launch_bounds__(256) k_row_delta(const T* __restrict__ cur,
                                                   const T* __restrict__ prev, int n_rows,
                                                   int d, float* __restrict__ delta) {
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (warp >= n_rows) return;
  constexpr int V = Vec<T>::N;
  const T* c = cur + (size_t)warp * d;
  const T* p = prev + (size_t)warp * d;
  float num = 0.f, den = 0.f;
  for (int e = lane * V; e < d; e += 32 * V) {
    float a[V], b[V];
    load16<T>(c + e, a);
    load16<T>(p + e, b);
#pragma unroll
    for (int i = 0; i < V; ++i) {
      const float df = a[i] - b[i];
      num = fmaf(df, df, num);
      den = fmaf(b[i], b[i], den);
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    num += __shfl_xor_sync(0xffffffffu, num, o);
    den += __shfl_xor_sync(0xffffffffu, den, o);
  }
  if (lane == 0) delta[warp] = sqrtf(num) / fmaxf(sqrtf(den), 1e-30f);
}

constexpr int TK_THREADS = 1024;

// Inclusive block scan of one int per thread (1024 threads); returns the inclusive
// value and writes the block total to *total.
__device__ __forceinline__ int block_scan_incl(int x, int* warp_sums, int* total) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) warp_sums[w] = x;
  __syncthreads();
  if (w == 0) {
    int s = warp_sums[lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, s, o);
      if (lane >= o) s += y;
    }
    warp_sums[lane] = s;  // inclusive over warps
  }
  __syncthreads();
  const int add = w > 0 ? warp_sums[w - 1] : 0;
  *total = warp_sums[31];
  __syncthreads();
  return x + add;
}

__global__ void __launch_bounds__(TK_THREADS) k_topk_rows(const float* __restrict__ delta,
                                                          int n, int k,
                                                          const int32_t* __restrict__ row_tok,
                                                          int32_t* __restrict__ out_tok,
                                                          int32_t* __restrict__ out_pos) {
  __shared__ int hist[256];
  __shared__ uint32_t s_prefix, s_need;
  __shared__ int warp_sums[32];
  const int tid = threadIdx.x;
  const uint32_t* bits = reinterpret_cast<const uint32_t*>(delta);

  uint32_t prefix = 0, pmask = 0;
  uint32_t need = (uint32_t)k;  // rows still to take among those matching the prefix
  if (k < n) {
    for (int shift = 24; shift >= 0; shift -= 8) {
      for (int i = tid; i < 256; i += TK_THREADS) hist[i] = 0;
      __syncthreads();
      for (int i = tid; i < n; i += TK_THREADS) {
        const uint32_t b = bits[i];
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
        s_prefix = prefix | ((uint32_t)dg << shift);
        s_need = need - above;
      }
      __syncthreads();
      prefix = s_prefix;
      need = s_need;
      pmask |= 255u << shift;
      __syncthreads();
    }
  }
  // keep: delta > V, or delta == V among the first `need` such rows (k == n: all)
  int taken = 0, eq_seen = 0;
  for (int base = 0; base < n; base += TK_THREADS) {
    const int i = base + tid;
    uint32_t b = 0;
    bool valid = i < n;
    if (valid) b = bits[i];
    int is_eq = (valid && k < n && b == prefix) ? 1 : 0;
    int tot_eq;
    const int eq_incl = block_scan_incl(is_eq, warp_sums, &tot_eq);
    const int eq_rank = eq_seen + eq_incl - is_eq;
    int keep = 0;
    if (valid) {
      if (k >= n) keep = 1;
      else if (b > prefix) keep = 1;
      else if (is_eq && (uint32_t)eq_rank < need) keep = 1;
    }
    int tot_keep;
    const int kp_incl = block_scan_incl(keep, warp_sums, &tot_keep);
    if (keep) {
      const int o = taken + kp_incl - 1;
      if (o < k) {
        out_tok[o] = row_tok ? row_tok[i] : i;
        if (out_pos) out_pos[o] = i;
      }
    }
    taken += tot_keep;
    eq_seen += tot_eq;
  }
}

}  // namespace

cudaError_t launch_row_delta(const void* cur, const void* prev, fl_dtype dt, int n_rows,
                             int d, float* delta, cudaStream_t s) {
  const int threads = 256;
  const int blocks = (int)(((size_t)n_rows * 32 + threads - 1) / threads);
  if (dt == FL_F32)
    k_row_delta<float><<<blocks, threads, 0, s>>>((const float*)cur, (const float*)prev,
                                                  n_rows, d, delta);
  else
    k_row_delta<__nv_bfloat16><<<blocks, threads, 0, s>>>(
        (const __nv_bfloat16*)cur, (const __nv_bfloat16*)prev, n_rows, d, delta);
  count_launch();
  return cudaGetLastError();
}

cudaError_t launch_topk_rows(const float* delta, int n, int k, const int32_t* row_tok,
                             int32_t* out_tok, int32_t* out_pos, int* st, cudaStream_t s) {
  (void)st;
  if (k <= 0) return cudaSuccess;
  k_topk_rows<<<1, TK_THREADS, 0, s>>>(delta, n, k, row_tok, out_tok, out_pos);
  count_launch();
  return cudaGetLastError();
}

}  // namespace fl
