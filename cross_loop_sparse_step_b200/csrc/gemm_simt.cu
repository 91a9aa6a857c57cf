// CUDA-core GEMM for the binary32 model path: C (=|+=) A . W^T with A [M x K] and
// W [N x K] row-major (linear-layer weights), binary32 accumulation. 64 x 64 output
// tiles, K staged through shared memory 16 at a time, a 4 x 4 register tile per
// thread. Used for the fp32 workloads (small shapes); bf16 workloads run on the
// tensor-core GEMM.
#include "fl_internal.cuh"

namespace fl {
namespace {

constexpr int BM = 64, BN = 64, BK = 16;

template <typename T>
__global__ void __launch_bounds__(256) k_gemm_simt(const T* __restrict__ A,
                                                   const T* __restrict__ W,
                                                   float* __restrict__ C, int M, int N, int K,
                                                   int ldc, int epi) {
  __shared__ float As[BK][BM + 4];
  __shared__ float Ws[BK][BN + 4];
  const int tid = threadIdx.x;
  const int tx = tid % 16, ty = tid / 16;
  const int m0 = blockIdx.y * BM, n0 = blockIdx.x * BN;
  float acc[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;

  for (int k0 = 0; k0 < K; k0 += BK) {
    // each thread loads 4 elements of A and 4 of W (64 rows x 16 cols each)
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      const int idx = tid + r * 256;  // 0..1023
      const int row = idx / BK, col = idx % BK;
      const int gm = m0 + row, gn = n0 + row, gk = k0 + col;
      As[col][row] = (gm < M && gk < K) ? to_f32<T>(A[(size_t)gm * K + gk]) : 0.f;
      Ws[col][row] = (gn < N && gk < K) ? to_f32<T>(W[(size_t)gn * K + gk]) : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < BK; ++kk) {
      float a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = As[kk][ty * 4 + i];
#pragma unroll
      for (int j = 0; j < 4; ++j) b[j] = Ws[kk][tx * 4 + j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int gm = m0 + ty * 4 + i;
    if (gm >= M) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int gn = n0 + tx * 4 + j;
      if (gn >= N) continue;
      float* c = C + (size_t)gm * ldc + gn;
      *c = epi == EPI_ADD ? *c + acc[i][j] : acc[i][j];
    }
  }
}

}  // namespace

cudaError_t launch_gemm_simt(fl_dtype dt, const void* A, const void* W, float* C, int M, int N,
                             int K, int ldc, GemmEpi epi, cudaStream_t s) {
  if (M <= 0 || N <= 0) return cudaSuccess;
  dim3 grid((N + BN - 1) / BN, (M + BM - 1) / BM);
  if (dt == FL_F32)
    k_gemm_simt<float><<<grid, 256, 0, s>>>((const float*)A, (const float*)W, C, M, N, K, ldc,
                                            (int)epi);
  else
    k_gemm_simt<__nv_bfloat16><<<grid, 256, 0, s>>>((const __nv_bfloat16*)A,
                                                    (const __nv_bfloat16*)W, C, M, N, K, ldc,
                                                    (int)epi);
  count_launch();
  return cudaGetLastError();
}

}  // namespace fl
