// Row-wise pieces of the shared block (pre-norm layer): RMSNorm into the GEMM operand
// type, RoPE (rotate-half, theta) splitting the fused q/k/v projection, and the SwiGLU
// product. The pages (FlashLoop §1) name the looped block but not its layer; these are
// the standard pre-norm decoder choices.
#include "fl_internal.cuh"

namespace fl {
namespace {

template <typename T>
__global__ void __launch_bounds__(256) k_rmsnorm(const float* __restrict__ x,
                                                 const float* __restrict__ gamma, float eps,
                                                 T* __restrict__ out, int d) {
  const int row = blockIdx.x;
  const float* xr = x + (size_t)row * d;
  float ss = 0.f;
  for (int e = threadIdx.x; e < d; e += blockDim.x) ss = fmaf(xr[e], xr[e], ss);
  __shared__ float red[8];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = ss;
  __syncthreads();
  float tot = 0.f;
  for (int i = 0; i < (int)(blockDim.x >> 5); ++i) tot += red[i];
  const float inv = 1.0f / sqrtf(tot / (float)d + eps);
  T* o = out + (size_t)row * d;
  for (int e = threadIdx.x; e < d; e += blockDim.x) o[e] = from_f32<T>(xr[e] * inv * gamma[e]);
}

// One row per CTA, eight consecutive elements per thread (blockDim = d / 8): the row is
// read once into registers with 16-byte loads, reduced, scaled and written packed.
// Same arithmetic per element as k_rmsnorm: (x * inv) * gamma, rounded once.
template <typename T>
__global__ void __launch_bounds__(1024) k_rmsnorm_v8(const float* __restrict__ x,
                                                    const float* __restrict__ gamma, float eps,
                                                    T* __restrict__ out, int d) {
  griddep_wait();
  const int row = blockIdx.x;
  const int e0 = threadIdx.x * 8;
  const float4* xr = reinterpret_cast<const float4*>(x + (size_t)row * d + e0);
  const float4 a = xr[0], b = xr[1];
  const float v[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
  float ss = 0.f;
#pragma unroll
  for (int j = 0; j < 8; ++j) ss = fmaf(v[j], v[j], ss);
  __shared__ float red[32];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = ss;
  __syncthreads();
  float tot = 0.f;
  for (int i = 0; i < (int)(blockDim.x >> 5); ++i) tot += red[i];
  const float inv = 1.0f / sqrtf(tot / (float)d + eps);
  const float4 ga = reinterpret_cast<const float4*>(gamma + e0)[0];
  const float4 gb = reinterpret_cast<const float4*>(gamma + e0)[1];
  const float g[8] = {ga.x, ga.y, ga.z, ga.w, gb.x, gb.y, gb.z, gb.w};
  float y[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) y[j] = v[j] * inv * g[j];
  T* o = out + (size_t)row * d + e0;
  if constexpr (sizeof(T) == 2) {
    uint32_t w[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const __nv_bfloat162 p2 = __floats2bfloat162_rn(y[2 * j], y[2 * j + 1]);
      w[j] = *reinterpret_cast<const uint32_t*>(&p2);
    }
    *reinterpret_cast<uint4*>(o) = make_uint4(w[0], w[1], w[2], w[3]);
  } else {
    reinterpret_cast<float4*>(o)[0] = make_float4(y[0], y[1], y[2], y[3]);
    reinterpret_cast<float4*>(o)[1] = make_float4(y[4], y[5], y[6], y[7]);
  }
}

// qkv [M][3d] -> q, k (rotated) and v [M][H][hd]; angle = pos * theta^(-2i/hd) in fp64.
__global__ void k_rope_split(const float* __restrict__ qkv, const int32_t* __restrict__ pos,
                             int M, int H, int hd, float theta, float* __restrict__ q,
                             float* __restrict__ k, float* __restrict__ v) {
  const int half = hd / 2;
  const size_t total = (size_t)M * H * half;
  const int d = H * hd;
  for (size_t id = blockIdx.x * (size_t)blockDim.x + threadIdx.x; id < total;
       id += (size_t)gridDim.x * blockDim.x) {
    const int i = (int)(id % half);
    const int h = (int)((id / half) % H);
    const int m = (int)(id / ((size_t)half * H));
    const double inv_freq = pow((double)theta, -2.0 * (double)i / (double)hd);
    double sn, cs;
    sincos((double)pos[m] * inv_freq, &sn, &cs);
    const float c = (float)cs, s = (float)sn;
    const float* row = qkv + (size_t)m * 3 * d;
    const size_t o = (size_t)m * d + (size_t)h * hd;
    const float qa = row[h * hd + i], qb = row[h * hd + i + half];
    const float ka = row[d + h * hd + i], kb = row[d + h * hd + i + half];
    q[o + i] = qa * c - qb * s;
    q[o + i + half] = qa * s + qb * c;
    k[o + i] = ka * c - kb * s;
    k[o + i + half] = ka * s + kb * c;
    v[o + i] = row[2 * d + h * hd + i];
    v[o + i + half] = row[2 * d + h * hd + i + half];
  }
}

// tab[t][i] = (cos, sin)(t * theta^(-2i/hd)), angle and functions in fp64, t < n_tok.
__global__ void k_rope_table(float2* __restrict__ tab, int n_tok, int hd, float theta) {
  const int half = hd / 2;
  const size_t total = (size_t)n_tok * half;
  for (size_t id = blockIdx.x * (size_t)blockDim.x + threadIdx.x; id < total;
       id += (size_t)gridDim.x * blockDim.x) {
    const int i = (int)(id % half);
    const int t = (int)(id / half);
    const double inv_freq = pow((double)theta, -2.0 * (double)i / (double)hd);
    double sn, cs;
    sincos((double)t * inv_freq, &sn, &cs);
    tab[id] = make_float2((float)cs, (float)sn);
  }
}

template <typename T>
__global__ void k_swiglu(const float* __restrict__ gu, int M, int F, T* __restrict__ out) {
  const size_t total = (size_t)M * F;
  for (size_t id = blockIdx.x * (size_t)blockDim.x + threadIdx.x; id < total;
       id += (size_t)gridDim.x * blockDim.x) {
    const size_t m = id / F, f = id % F;
    const float g = gu[m * 2 * F + f], u = gu[m * 2 * F + F + f];
    out[id] = from_f32<T>(g / (1.0f + expf(-g)) * u);
  }
}

int grid_for(size_t n) {
  size_t b = (n + 255) / 256;
  return (int)(b > 148 * 32 ? 148 * 32 : (b == 0 ? 1 : b));
}

}  // namespace

cudaError_t launch_rmsnorm(const float* x, const float* gamma, float eps, void* out,
                           fl_dtype dt, int M, int d, cudaStream_t s) {
  if (M <= 0) return cudaSuccess;
  const bool v8 = d % 256 == 0 && d / 8 <= 1024 && (uintptr_t)x % 16 == 0 &&
                  (uintptr_t)gamma % 16 == 0 && (uintptr_t)out % 16 == 0;
  if (v8) {
    const cudaError_t e =
        dt == FL_F32 ? launch_pdl(k_rmsnorm_v8<float>, dim3(M), dim3(d / 8), 0, s, x, gamma, eps,
                                  (float*)out, d)
                     : launch_pdl(k_rmsnorm_v8<__nv_bfloat16>, dim3(M), dim3(d / 8), 0, s, x, gamma,
                                  eps, (__nv_bfloat16*)out, d);
    if (e != cudaSuccess) return e;
  } else if (dt == FL_F32) {
    k_rmsnorm<float><<<M, 256, 0, s>>>(x, gamma, eps, (float*)out, d);
  } else {
    k_rmsnorm<__nv_bfloat16><<<M, 256, 0, s>>>(x, gamma, eps, (__nv_bfloat16*)out, d);
  }
  count_launch();
  return cudaGetLastError();
}

cudaError_t launch_rope_split(const float* qkv, const int32_t* pos, int M, int H, int hd,
                              float theta, float* q, float* k, float* v, cudaStream_t s) {
  if (M <= 0) return cudaSuccess;
  k_rope_split<<<grid_for((size_t)M * H * hd / 2), 256, 0, s>>>(qkv, pos, M, H, hd, theta, q, k, v);
  count_launch();
  return cudaGetLastError();
}

cudaError_t launch_rope_table(float2* tab, int n_tok, int hd, float theta, cudaStream_t s) {
  if (n_tok <= 0) return cudaSuccess;
  k_rope_table<<<grid_for((size_t)n_tok * hd / 2), 256, 0, s>>>(tab, n_tok, hd, theta);
  count_launch();
  return cudaGetLastError();
}

cudaError_t launch_swiglu(const float* gu, int M, int F, void* out, fl_dtype dt,
                          cudaStream_t s) {
  if (M <= 0) return cudaSuccess;
  if (dt == FL_F32) k_swiglu<float><<<grid_for((size_t)M * F), 256, 0, s>>>(gu, M, F, (float*)out);
  else k_swiglu<__nv_bfloat16><<<grid_for((size_t)M * F), 256, 0, s>>>(gu, M, F, (__nv_bfloat16*)out);
  count_launch();
  return cudaGetLastError();
}

}  // namespace fl
