// Packed binary32 arithmetic of sm_100 (add / fma on float pairs) and pairwise
// decoding of packed KV codes into binary32 pairs.
//
// A code byte c becomes the float 2^23 + c by placing it under the exponent bits of
// 2^23 (one byte permute), and the pair is then rebased with one packed subtraction;
// every step is exact for codes below 2^23.
#pragma once
#include <stdint.h>

namespace fl {
namespace f2 {

__device__ __forceinline__ unsigned long long as_u64(float2 v) {
  return *reinterpret_cast<unsigned long long*>(&v);
}
__device__ __forceinline__ float2 as_f2(unsigned long long v) {
  return *reinterpret_cast<float2*>(&v);
}

// a * b + c, element-wise, round to nearest
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) {
  unsigned long long d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(as_u64(a)), "l"(as_u64(b)), "l"(as_u64(c)));
  return as_f2(d);
}
__device__ __forceinline__ float2 add2(float2 a, float2 b) {
  unsigned long long d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(as_u64(a)), "l"(as_u64(b)));
  return as_f2(d);
}

// float bits 2^23 + byte i of w (exact)
__device__ __forceinline__ float biased(uint32_t w, int i) {
  const uint32_t sel = (uint32_t)i | (4u << 4) | (4u << 8) | (7u << 12);
  return __uint_as_float(__byte_perm(w, 0x4B000000u, sel));
}
__device__ __forceinline__ float2 rebase(float a, float b) {
  return add2(make_float2(a, b), make_float2(-8388608.0f, -8388608.0f));
}

// 4 codes of 8 bits (element order = byte order) -> 2 pairs
__device__ __forceinline__ void dec8(uint32_t w, float2* o) {
  o[0] = rebase(biased(w, 0), biased(w, 1));
  o[1] = rebase(biased(w, 2), biased(w, 3));
}
// 8 codes of 4 bits (element i at bits 4i) -> 4 pairs
__device__ __forceinline__ void dec4(uint32_t w, float2* o) {
  const uint32_t lo = w & 0x0F0F0F0Fu;          // codes 0, 2, 4, 6
  const uint32_t hi = (w >> 4) & 0x0F0F0F0Fu;   // codes 1, 3, 5, 7
#pragma unroll
  for (int k = 0; k < 4; ++k) o[k] = rebase(biased(lo, k), biased(hi, k));
}
// 16 codes of 2 bits (element i at bits 2i) -> 8 pairs
__device__ __forceinline__ void dec2(uint32_t w, float2* o) {
  uint32_t x[4];  // x[j] bytes hold codes j, 4 + j, 8 + j, 12 + j
#pragma unroll
  for (int j = 0; j < 4; ++j) x[j] = (w >> (2 * j)) & 0x03030303u;
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    const int e0 = 2 * k, e1 = 2 * k + 1;
    o[k] = rebase(biased(x[e0 & 3], e0 >> 2), biased(x[e1 & 3], e1 >> 2));
  }
}

// Codes [e0, e0 + EL) of one stored row of `bits` bits as EL/2 binary32 pairs.
template <int EL>
__device__ __forceinline__ void load_pairs(const uint8_t* row, int bits, int e0, float2* c) {
  if (bits == 8) {
    const uint4* p = reinterpret_cast<const uint4*>(row + e0);
#pragma unroll
    for (int k = 0; k < EL / 16; ++k) {
      const uint4 u = p[k];
      dec8(u.x, c + 8 * k);
      dec8(u.y, c + 8 * k + 2);
      dec8(u.z, c + 8 * k + 4);
      dec8(u.w, c + 8 * k + 6);
    }
  } else if (bits == 4) {
    const uint32_t* p = reinterpret_cast<const uint32_t*>(row + e0 / 2);
#pragma unroll
    for (int k = 0; k < EL / 8; ++k) dec4(p[k], c + 4 * k);
  } else {  // 2 bits
    const uint32_t* p = reinterpret_cast<const uint32_t*>(row + e0 / 4);
#pragma unroll
    for (int k = 0; k < EL / 16; ++k) dec2(p[k], c + 8 * k);
  }
}

// sum_j q[j] * c[j] over EL elements held as pairs
template <int EL>
__device__ __forceinline__ float dot_pairs(const float2* q, const float2* c) {
  float2 acc = make_float2(0.f, 0.f);
#pragma unroll
  for (int k = 0; k < EL / 2; ++k) acc = fma2(q[k], c[k], acc);
  return acc.x + acc.y;
}

// o[j] += w * c[j]
template <int EL>
__device__ __forceinline__ void axpy_pairs(float w, const float2* c, float2* o) {
  const float2 ww = make_float2(w, w);
#pragma unroll
  for (int k = 0; k < EL / 2; ++k) o[k] = fma2(ww, c[k], o[k]);
}

}  // namespace f2
}  // namespace fl
