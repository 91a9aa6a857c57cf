// Row gather / scatter between the full hidden state and compact active-row buffers
// (FlashLoop §4.4: selected tokens are gathered into compact buffers so the
// projections stay regular GEMMs; §4.1: results return to their rows and inactive
// rows keep their state). One CTA per row, 16-byte vector copies when the row size and
// both base addresses allow it, element copies otherwise.
#include "fl_internal.cuh"

namespace fl {
namespace {

template <typename V>
__global__ void __launch_bounds__(256) k_gather_scatter(int op, const uint8_t* __restrict__ src,
                                                        uint8_t* __restrict__ dst,
                                                        const int32_t* __restrict__ idx,
                                                        int n_full, size_t row_bytes, int* st) {
  const int i = blockIdx.x;
  const int j = idx[i];
  if (j < 0 || j >= n_full) {
    if (threadIdx.x == 0) record_error(st, FL_ERR_RANGE);
    return;
  }
  const size_t s_row = (op == FL_GATHER) ? (size_t)j : (size_t)i;
  const size_t d_row = (op == FL_GATHER) ? (size_t)i : (size_t)j;
  const V* s = reinterpret_cast<const V*>(src + s_row * row_bytes);
  V* d = reinterpret_cast<V*>(dst + d_row * row_bytes);
  const size_t n = row_bytes / sizeof(V);
  for (size_t e = threadIdx.x; e < n; e += blockDim.x) d[e] = s[e];
}

__global__ void k_fill_i32(int32_t* p, int32_t v, size_t n) {
  griddep_wait();
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n;
       i += (size_t)gridDim.x * blockDim.x)
    p[i] = v;
}

// Tap copy: block i finds token tok[i] in the ascending row-token list act[0, M) by
// binary search and copies that row of src to row i of dst; absent tokens are skipped.
__global__ void __launch_bounds__(128) k_tap_rows(const int32_t* __restrict__ act, int M,
                                                  const int32_t* __restrict__ tok,
                                                  const uint8_t* __restrict__ src,
                                                  uint8_t* __restrict__ dst, size_t row_bytes) {
  const int t = tok[blockIdx.x];
  int lo = 0, hi = M;   // first position with act[pos] >= t
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    if (act[mid] < t) lo = mid + 1;
    else hi = mid;
  }
  if (lo >= M || act[lo] != t) return;
  const uint4* s = reinterpret_cast<const uint4*>(src + (size_t)lo * row_bytes);
  uint4* d = reinterpret_cast<uint4*>(dst + (size_t)blockIdx.x * row_bytes);
  for (size_t e = threadIdx.x; e < row_bytes / 16; e += blockDim.x) d[e] = s[e];
}

__global__ void k_iota(int32_t* p, int n) {
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x)
    p[i] = i;
}

}  // namespace

cudaError_t launch_gather_scatter(fl_gs_op op, const void* src, void* dst, const int32_t* idx,
                                  int n_idx, int n_full, size_t row_bytes, int* st,
                                  cudaStream_t s) {
  if (n_idx <= 0) return cudaSuccess;
  const bool v16 = row_bytes % 16 == 0 && ((uintptr_t)src % 16 == 0) && ((uintptr_t)dst % 16 == 0);
  const bool v4 = row_bytes % 4 == 0 && ((uintptr_t)src % 4 == 0) && ((uintptr_t)dst % 4 == 0);
  if (v16)
    k_gather_scatter<uint4><<<n_idx, 256, 0, s>>>(op, (const uint8_t*)src, (uint8_t*)dst, idx,
                                                  n_full, row_bytes, st);
  else if (v4)
    k_gather_scatter<uint32_t><<<n_idx, 256, 0, s>>>(op, (const uint8_t*)src, (uint8_t*)dst,
                                                     idx, n_full, row_bytes, st);
  else
    k_gather_scatter<uint16_t><<<n_idx, 256, 0, s>>>(op, (const uint8_t*)src, (uint8_t*)dst,
                                                     idx, n_full, row_bytes, st);
  count_launch();
  return cudaGetLastError();
}

cudaError_t launch_tap_rows(const int32_t* act, int M, const int32_t* tok, int n,
                            const void* src, void* dst, size_t row_bytes, cudaStream_t s) {
  if (n <= 0 || M <= 0 || !dst) return cudaSuccess;
  if (row_bytes % 16 || (uintptr_t)src % 16 || (uintptr_t)dst % 16) return cudaErrorInvalidValue;
  k_tap_rows<<<n, 128, 0, s>>>(act, M, tok, (const uint8_t*)src, (uint8_t*)dst, row_bytes);
  count_launch();
  return cudaGetLastError();
}

cudaError_t launch_fill_i32(int32_t* p, int32_t v, size_t n, cudaStream_t s) {
  if (n == 0) return cudaSuccess;
  const int blocks = (int)((n + 255) / 256 < 4096 ? (n + 255) / 256 : 4096);
  const cudaError_t e = launch_pdl(k_fill_i32, dim3(blocks), dim3(256), 0, s, p, v, n);
  count_launch();
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

cudaError_t launch_iota(int32_t* p, int n, cudaStream_t s) {
  if (n <= 0) return cudaSuccess;
  const int blocks = (n + 255) / 256 < 4096 ? (n + 255) / 256 : 4096;
  k_iota<<<blocks, 256, 0, s>>>(p, n);
  count_launch();
  return cudaGetLastError();
}

}  // namespace fl
