// Pieces shared by the query-tile tensor-core attention kernels: tile geometry, fp16
// packing, and the reconstruction of K^ / V^ rows from the quantised store (int8 base
// plus the residual rows of the loops that rewrote a token, added in loop order).
#pragma once
#include "fl_internal.cuh"
#include "sm100_ptx.cuh"

namespace fl {
namespace tile {

using namespace sm100;

constexpr int TQ = 128;            // queries per tile = TMEM lanes = MMA M
constexpr int TC = 128;            // columns per chunk
constexpr int HDT = 128;           // head_dim
constexpr uint32_t TILE = TQ * HDT * 2;          // one fp16 128 x 128 operand tile
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRescale = 8.f;    // log2 growth of the maximum that rescales O

// mbar_wait whose outcome agrees across the (converged) warp: false on every lane if it
// failed on any, so warp-collective TMEM accesses that follow stay aligned.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort,
                                          int site = 1) {
  const bool ok = mbar_wait(bar, parity, abort, site);
  return __all_sync(0xffffffffu, ok);
}

__device__ __forceinline__ uint32_t pack_h2(float a, float b) {
  const __half2 h = __floats2half2_rn(a, b);
  return *reinterpret_cast<const uint32_t*>(&h);
}

// Dequantised residual codes of `BITS` bits for elements [e0, e0 + 16) of a stored row,
// added to acc in binary32: acc += fmaf(code, s, z).
template <int BITS>
__device__ __forceinline__ void add_residual16(const uint8_t* row_codes, uint32_t szw, int e0,
                                               float* acc) {
  const float s = half_bits_to_float((uint16_t)(szw & 0xFFFFu));
  const float z = half_bits_to_float((uint16_t)(szw >> 16));
  uint32_t w[BITS / 2];
  if constexpr (BITS == 8) {
    const uint4 v = __ldg(reinterpret_cast<const uint4*>(row_codes + e0));
    w[0] = v.x; w[1] = v.y; w[2] = v.z; w[3] = v.w;
  } else if constexpr (BITS == 4) {
    const uint2 v = __ldg(reinterpret_cast<const uint2*>(row_codes + e0 / 2));
    w[0] = v.x; w[1] = v.y;
  } else {
    w[0] = __ldg(reinterpret_cast<const uint32_t*>(row_codes + e0 / 4));
  }
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const int bit = i * BITS;
    const uint32_t c = (w[bit >> 5] >> (bit & 31)) & ((1u << BITS) - 1u);
    acc[i] = __fadd_rn(acc[i], __fmaf_rn((float)c, s, z));
  }
}

// The base row of K or V (which = 0 / 1) of token `col`, head h: 128 int8 codes and the
// (s, z) pairs of its groups, loaded together so one round of memory latency covers them.
struct BaseRow {
  uint4 raw[8];
  uint32_t sz[4];
};

__device__ __forceinline__ void load_base(const AttnParams& P, int which, int col, int h,
                                          BaseRow& b) {
  const KvView& kv = P.kv;
  if (kv.base_bits == 0) return;   // binary32 rows are read run by run
  const size_t bh = (size_t)col * P.H + h;
  const uint4* cp = reinterpret_cast<const uint4*>(kv.codes[which][1] + bh * HDT);
#pragma unroll
  for (int k = 0; k < 8; ++k) b.raw[k] = __ldg(cp + k);
  const int ng = HDT / kv.g;
  const uint32_t* sp = reinterpret_cast<const uint32_t*>(kv.sz[which][1]) + bh * ng;
#pragma unroll
  for (int k = 0; k < 4; ++k) b.sz[k] = k < ng ? __ldg(sp + k) : 0u;
}

// K^ or V^ elements [e0, e0 + 16) of token `col`: the base (already loaded), then the
// residual rows of the loops in `chain` (bit r set: loop r rewrote the token), added in
// loop order - the store's reconstruction.
__device__ __forceinline__ void reconstruct16(const AttnParams& P, int which, int col, int h,
                                              const BaseRow& b, uint32_t chain, int e0,
                                              float* acc) {
  const KvView& kv = P.kv;
  const int g = kv.g, ng = HDT / g;
  if (kv.base_bits == 0) {   // unquantised store: the binary32 values themselves
    const float4* rp = reinterpret_cast<const float4*>(kv.codes[which][1]) +
                       ((size_t)col * P.H + h) * (HDT / 4) + e0 / 4;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float4 v = __ldg(rp + k);
      acc[4 * k] = v.x; acc[4 * k + 1] = v.y; acc[4 * k + 2] = v.z; acc[4 * k + 3] = v.w;
    }
  } else {
    const uint32_t szw = g == 32 ? b.sz[e0 / 32] : b.sz[e0 / 64];
    const float s = half_bits_to_float((uint16_t)(szw & 0xFFFFu));
    const float z = half_bits_to_float((uint16_t)(szw >> 16));
    const uint32_t w[4] = {b.raw[e0 / 16].x, b.raw[e0 / 16].y, b.raw[e0 / 16].z, b.raw[e0 / 16].w};
#pragma unroll
    for (int i = 0; i < 16; ++i)
      acc[i] = __fmaf_rn((float)((w[i >> 2] >> ((i & 3) * 8)) & 0xFFu), s, z);
  }
  while (chain) {
    const int r = __ffs(chain) - 1;
    chain &= chain - 1;
    const int row = __ldg(kv.slot + (size_t)r * kv.n_tok + col);
    const size_t rh = (size_t)row * P.H + h;
    const int bits = kv.res_bits[r];
    if (bits == 0) {   // an unquantised loop stores the new value itself
      const float4* rp = reinterpret_cast<const float4*>(kv.codes[which][r]) + rh * (HDT / 4) + e0 / 4;
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const float4 v = __ldg(rp + k);
        acc[4 * k] = v.x; acc[4 * k + 1] = v.y; acc[4 * k + 2] = v.z; acc[4 * k + 3] = v.w;
      }
      continue;
    }
    const uint32_t rsz =
        __ldg(reinterpret_cast<const uint32_t*>(kv.sz[which][r]) + rh * ng + e0 / g);
    if (bits == 2) add_residual16<2>(kv.codes[which][r] + rh * (HDT / 4), rsz, e0, acc);
    else if (bits == 4) add_residual16<4>(kv.codes[which][r] + rh * (HDT / 2), rsz, e0, acc);
    else add_residual16<8>(kv.codes[which][r] + rh * HDT, rsz, e0, acc);
  }
}


// Status word value of a bounded wait that ran out: FL_ERR_TIMEOUT in the low byte, the
// wait's site code above it (fl_check_device_status returns the low byte and keeps the
// site for fl_last_error_detail).
__device__ __forceinline__ int timeout_code(int site) {
  return FL_ERR_TIMEOUT | ((site & 0xFFFFFF) << 8);
}

}  // namespace tile
}  // namespace fl
