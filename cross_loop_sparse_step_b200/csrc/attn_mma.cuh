// Warp-level tensor-core pieces of the sparse attention: exact small-integer codes as
// fp16 operands, binary32 values as hi + lo fp16 pairs, m16n8k16 MMAs with binary32
// accumulation.
//
// A code c (< 256) enters an MMA as the fp16 subnormal c * 2^-24: the byte c under a zero
// exponent byte (one byte permute, exact), so a dot product comes out scaled by 2^-24,
// a power of two that is taken off exactly. A binary32 value x, scaled by a power of two
// into [2^13, 2^14), splits into hi = fp16(x) and lo = fp16(x - hi) (x - hi is exact),
// so hi + lo keeps 22 bits of x; every product of an MMA is exact and only the binary32
// accumulation rounds.
#pragma once
#include <cuda_fp16.h>
#include <stdint.h>

namespace fl {
namespace mma {

// D (16 x 8, f32) += A (16 x 16, f16, row) . B (16 x 8, f16, col)
__device__ __forceinline__ void m16n8k16(float* d, uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
      "{%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t pack_h2(__half lo, __half hi) {
  return (uint32_t)__half_as_ushort(lo) | ((uint32_t)__half_as_ushort(hi) << 16);
}

// fp16 pair (byte i0 of w, byte i1 of w) * 2^-24 (subnormals, exact)
__device__ __forceinline__ uint32_t code_pair(uint32_t w, int i0, int i1) {
  const uint32_t sel = (uint32_t)i0 | (4u << 4) | ((uint32_t)i1 << 8) | (4u << 12);
  return __byte_perm(w, 0u, sel);
}

constexpr float kCodeUnscale = 16777216.f;   // 2^24

// hi / lo fp16 parts of x (already scaled); returns hi, writes lo
__device__ __forceinline__ __half split_hi(float x, __half* lo) {
  const __half h = __float2half_rn(x);
  *lo = __float2half_rn(x - __half2float(h));
  return h;
}

// 2^e for a scale that brings |x| <= amax into [2^13, 2^14) (1 when amax is 0 or not finite)
__device__ __forceinline__ float pow2_scale_for(float amax, int top) {
  if (!(amax > 0.f) || !isfinite(amax)) return 1.f;
  const int ex = (int)((__float_as_uint(amax) >> 23) & 0xFF) - 127;   // amax in [2^ex, 2^(ex+1))
  int e = top - 1 - ex;
  if (e > 126) e = 126;
  if (e < -126) e = -126;
  return __uint_as_float((uint32_t)(e + 127) << 23);
}

// Codes of `bits` bits (element i at bits [i*bits, (i+1)*bits)) in n_words32 source words,
// spread one code per byte into out (4 codes per word, element order kept).
__device__ __forceinline__ void spread4(uint32_t w, uint32_t* out) {
  const uint32_t lo = w & 0x0F0F0F0Fu, hi = (w >> 4) & 0x0F0F0F0Fu;   // codes 0,2,4,6 / 1,3,5,7
  out[0] = __byte_perm(lo, hi, 0x5140);
  out[1] = __byte_perm(lo, hi, 0x7362);
}
__device__ __forceinline__ void spread2(uint32_t w, uint32_t* out) {
  const uint32_t x0 = w & 0x03030303u, x1 = (w >> 2) & 0x03030303u;   // codes 4j / 4j+1
  const uint32_t x2 = (w >> 4) & 0x03030303u, x3 = (w >> 6) & 0x03030303u;
  const uint32_t a01 = __byte_perm(x0, x1, 0x5140), a23 = __byte_perm(x2, x3, 0x5140);  // j=0,1
  const uint32_t b01 = __byte_perm(x0, x1, 0x7362), b23 = __byte_perm(x2, x3, 0x7362);  // j=2,3
  out[0] = __byte_perm(a01, a23, 0x5410);
  out[1] = __byte_perm(a01, a23, 0x7632);
  out[2] = __byte_perm(b01, b23, 0x5410);
  out[3] = __byte_perm(b01, b23, 0x7632);
}

// The score MMAs' B operand from this lane's quarter qx[HD / 4] of q (lane (g, l) of the
// warp, g = lane / 4, l = lane % 4): q scaled by a power of two into [2^13, 2^14) and split
// into hi + lo fp16; lane (g, l) feeds column n = g of B (hi for even g, lo for odd g)
// with quarter g / 2 and zeros elsewhere, so D column pair (2l, 2l + 1) is quarter l's
// dot. Over k-step ks a lane's logical k {2l, 2l+1, 2l+8, 2l+9} are its elements
// 4 ks .. 4 ks + 3. Returns the factor that turns D back into dot products of codes.
template <int HD>
__device__ __forceinline__ float q_fragments(const float* qx, int lane, uint32_t (*bq)[2]) {
  constexpr int KS = HD / 16;
  float qmax = 0.f;
#pragma unroll
  for (int j = 0; j < HD / 4; ++j) qmax = fmaxf(qmax, fabsf(qx[j]));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) qmax = fmaxf(qmax, __shfl_xor_sync(0xffffffffu, qmax, o));
  const float qscale = pow2_scale_for(qmax, 14);
  const int cg = lane >> 2, l4 = lane & 3;
  const bool feeds = l4 == (cg >> 1);
#pragma unroll
  for (int ks = 0; ks < KS; ++ks) {
    __half part[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      __half lo;
      const __half hi = split_hi(qx[4 * ks + j] * qscale, &lo);
      part[j] = (cg & 1) ? lo : hi;
    }
    bq[ks][0] = feeds ? pack_h2(part[0], part[1]) : 0u;
    bq[ks][1] = feeds ? pack_h2(part[2], part[3]) : 0u;
  }
  return kCodeUnscale / qscale;   // a power of two
}

}  // namespace mma

// This lane's EL codes [e0, e0 + EL) of a stored row, as raw words (EL * bits / 8 bytes,
// at most 32): loaded first, decoded later, so several rows' loads can be in flight.
template <int EL>
struct Raw {
  uint4 w[EL / 16];
};

template <int EL>
__device__ __forceinline__ void load_raw(const uint8_t* row, int bits, int e0, Raw<EL>& r) {
  const uint8_t* src = row + (size_t)e0 * bits / 8;
  if (bits == 8) {
#pragma unroll
    for (int k = 0; k < EL / 16; ++k) r.w[k] = reinterpret_cast<const uint4*>(src)[k];
  } else if (bits == 4) {   // EL / 2 bytes
    if constexpr (EL == 32) {
      r.w[0] = *reinterpret_cast<const uint4*>(src);
    } else {
      const uint2 u = *reinterpret_cast<const uint2*>(src);
      r.w[0] = make_uint4(u.x, u.y, 0u, 0u);
    }
  } else {                  // 2 bits: EL / 4 bytes
    if constexpr (EL == 32) {
      const uint2 u = *reinterpret_cast<const uint2*>(src);
      r.w[0] = make_uint4(u.x, u.y, 0u, 0u);
    } else {
      r.w[0] = make_uint4(*reinterpret_cast<const uint32_t*>(src), 0u, 0u, 0u);
    }
  }
}

template <int EL>
__device__ __forceinline__ uint32_t raw_word(const Raw<EL>& r, int i) {
  const uint4 u = r.w[i >> 2];
  return (i & 3) == 0 ? u.x : (i & 3) == 1 ? u.y : (i & 3) == 2 ? u.z : u.w;
}

// This lane's EL codes as one code per byte (EL / 4 words), from raw words of `bits` bits.
template <int EL>
__device__ __forceinline__ void to_bytes(const Raw<EL>& r, int bits, uint32_t* wb) {
  if (bits == 8) {
#pragma unroll
    for (int i = 0; i < EL / 4; ++i) wb[i] = raw_word(r, i);
  } else if (bits == 4) {
#pragma unroll
    for (int i = 0; i < EL / 8; ++i) mma::spread4(raw_word(r, i), wb + 2 * i);
  } else {
#pragma unroll
    for (int i = 0; i < EL / 16; ++i) mma::spread2(raw_word(r, i), wb + 4 * i);
  }
}

}  // namespace fl
