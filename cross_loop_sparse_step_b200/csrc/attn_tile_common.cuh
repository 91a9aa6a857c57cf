// Pieces shared by the query-tile tensor-core attention kernels: tile geometry, fp16
// packing, and the reconstruction of K^ / V^ rows from the quantised store (int8 base
// plus the residual rows of the loops that rewrote a token, added in loop order).
#pragma once
#include "fl_internal.cuh"
#include "sm100_ptx.cuh"

#include <utility>

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

// 2^x by the PTX ex2.approx.ftz instruction (relative error about 2^-22; subnormal
// inputs and results flushed to zero). Used for softmax weights that are rounded to fp16
// right after, whose smallest subnormal is 2^-24: flushing below 2^-126 changes none.
__device__ __forceinline__ float ex2_ftz(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
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

// The residual rows of one column (K or V) for the loops 2..loop that rewrote the token,
// in loop order: the code row, its bit width and its (s, z) words, fetched once per chunk.
// Three rows are held in named registers (no arrays, so nothing goes to local memory);
// deeper chains walk the remaining loops run by run.
struct ChainRow {
  const uint8_t* codes;
  int bits;
  uint32_t sz0, sz1, sz2, sz3;
};
struct Chain {
  int n;            // rows held (<= 3)
  uint32_t more;    // loops beyond the held rows (bit r: loop r)
  ChainRow r0, r1, r2;
};

template <int I>
__device__ __forceinline__ uint32_t sz_word(const ChainRow& r) {
  if constexpr (I == 0) return r.sz0;
  else if constexpr (I == 1) return r.sz1;
  else if constexpr (I == 2) return r.sz2;
  else return r.sz3;
}

__device__ __forceinline__ ChainRow chain_row(const AttnParams& P, int which, int r, int col,
                                              int h) {
  const KvView& kv = P.kv;
  const int ng = HDT / kv.g;
  const int row = __ldg(kv.slot + (size_t)r * kv.n_tok + col);
  const size_t rh = (size_t)row * P.H + h;
  ChainRow c;
  c.bits = kv.res_bits[r];
  c.codes = kv.codes[which][r] + rh * (c.bits ? HDT * c.bits / 8 : HDT * 4);
  c.sz0 = c.sz1 = c.sz2 = c.sz3 = 0u;
  if (c.bits) {
    const uint32_t* sp = reinterpret_cast<const uint32_t*>(kv.sz[which][r]) + rh * ng;
    c.sz0 = __ldg(sp);
    c.sz1 = __ldg(sp + 1);
    if (ng == 4) { c.sz2 = __ldg(sp + 2); c.sz3 = __ldg(sp + 3); }
  }
  return c;
}

// The rows of the loops in `mask` (bit r set: loop r lists the token) for K or V.
__device__ __forceinline__ void load_chain(const AttnParams& P, int which, int col, int h,
                                           uint32_t mask, Chain& c) {
  c.n = 0;
  c.more = 0;
  c.r0 = c.r1 = c.r2 = ChainRow{nullptr, 0, 0u, 0u, 0u, 0u};
  if (!mask) return;
  int r = __ffs(mask) - 1;
  mask &= mask - 1;
  c.r0 = chain_row(P, which, r, col, h);
  c.n = 1;
  if (!mask) return;
  r = __ffs(mask) - 1;
  mask &= mask - 1;
  c.r1 = chain_row(P, which, r, col, h);
  c.n = 2;
  if (!mask) return;
  r = __ffs(mask) - 1;
  mask &= mask - 1;
  c.r2 = chain_row(P, which, r, col, h);
  c.n = 3;
  c.more = mask;
}

__device__ __forceinline__ void add_chain_run(int b, const uint8_t* cp, uint32_t szw, int e0,
                                              float* acc) {
  if (b == 0) {   // an unquantised loop stores the new value itself
    const float4* rp = reinterpret_cast<const float4*>(cp) + e0 / 4;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float4 v = __ldg(rp + k);
      acc[4 * k] = v.x; acc[4 * k + 1] = v.y; acc[4 * k + 2] = v.z; acc[4 * k + 3] = v.w;
    }
  } else if (b == 2) {
    add_residual16<2>(cp, szw, e0, acc);
  } else if (b == 4) {
    add_residual16<4>(cp, szw, e0, acc);
  } else {
    add_residual16<8>(cp, szw, e0, acc);
  }
}

// Writes the 16 binary32 values x as fp16 into row `row` of a K-major [rows][128]
// operand tile (two 16-byte chunks at elements e0 .. e0 + 15); with `lo` also the
// remainders x - fp16(x) as fp16 into the same place of `lo` (split operands).
__device__ __forceinline__ void store_run(uint8_t* tile, uint8_t* lo, int row, int e0,
                                          const float* x) {
#pragma unroll
  for (int half = 0; half < 2; ++half) {
    const float* y = x + 8 * half;
    const uint32_t off = sw128_offset(row, e0 + 8 * half, TC);
    *reinterpret_cast<uint4*>(tile + off) =
        make_uint4(pack_h2(y[0], y[1]), pack_h2(y[2], y[3]), pack_h2(y[4], y[5]), pack_h2(y[6], y[7]));
    if (lo) {
      float r[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) r[k] = y[k] - __half2float(__float2half_rn(y[k]));
      *reinterpret_cast<uint4*>(lo + off) =
          make_uint4(pack_h2(r[0], r[1]), pack_h2(r[2], r[3]), pack_h2(r[4], r[5]), pack_h2(r[6], r[7]));
    }
  }
}

// One run of 16 elements [16 RUN, 16 RUN + 16) of a column: the base codes of the run
// (8-bit, or binary32 when unquantised), the held residual rows, any deeper loops - the
// store's reconstruction, added in loop order - written as fp16 (and its remainder).
template <int RUN>
__device__ __forceinline__ void decode_run16(const AttnParams& P, int which, int col, int h,
                                             const uint8_t* base_codes, const uint32_t* base_sz,
                                             const Chain& ch, uint8_t* tile, uint8_t* lo,
                                             int row) {
  constexpr int e0 = 16 * RUN;
  const KvView& kv = P.kv;
  const int g = kv.g, ng = HDT / g;
  float acc[16];
  if (kv.base_bits == 0) {
    const float4* rp = reinterpret_cast<const float4*>(base_codes) + e0 / 4;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float4 v = __ldg(rp + k);
      acc[4 * k] = v.x; acc[4 * k + 1] = v.y; acc[4 * k + 2] = v.z; acc[4 * k + 3] = v.w;
    }
  } else {
    const uint4 w4 = __ldg(reinterpret_cast<const uint4*>(base_codes) + RUN);
    const uint32_t szw = __ldg(base_sz + e0 / g);
    const float s = half_bits_to_float((uint16_t)(szw & 0xFFFFu));
    const float z = half_bits_to_float((uint16_t)(szw >> 16));
    const uint32_t w[4] = {w4.x, w4.y, w4.z, w4.w};
#pragma unroll
    for (int i = 0; i < 16; ++i)
      acc[i] = __fmaf_rn((float)((w[i >> 2] >> ((i & 3) * 8)) & 0xFFu), s, z);
  }
  if (ch.n > 0)
    add_chain_run(ch.r0.bits, ch.r0.codes, g == 32 ? sz_word<e0 / 32>(ch.r0) : sz_word<e0 / 64>(ch.r0), e0, acc);
  if (ch.n > 1)
    add_chain_run(ch.r1.bits, ch.r1.codes, g == 32 ? sz_word<e0 / 32>(ch.r1) : sz_word<e0 / 64>(ch.r1), e0, acc);
  if (ch.n > 2)
    add_chain_run(ch.r2.bits, ch.r2.codes, g == 32 ? sz_word<e0 / 32>(ch.r2) : sz_word<e0 / 64>(ch.r2), e0, acc);
  uint32_t more = ch.more;
  while (more) {   // loops beyond the held rows: slot, scales and codes read run by run
    const int r = __ffs(more) - 1;
    more &= more - 1;
    const int rrow = __ldg(kv.slot + (size_t)r * kv.n_tok + col);
    const size_t rh = (size_t)rrow * P.H + h;
    const int bits = kv.res_bits[r];
    const uint32_t rsz =
        bits ? __ldg(reinterpret_cast<const uint32_t*>(kv.sz[which][r]) + rh * ng + e0 / g) : 0u;
    add_chain_run(bits, kv.codes[which][r] + rh * (bits ? HDT * bits / 8 : HDT * 4), rsz, e0, acc);
  }
  store_run(tile, lo, row, e0, acc);
}

template <int... RUNS>
__device__ __forceinline__ void decode_runs(const AttnParams& P, int which, int col, int h,
                                            const uint8_t* bc, const uint32_t* bs, const Chain& ch,
                                            uint8_t* tile, uint8_t* lo, int row,
                                            std::integer_sequence<int, RUNS...>) {
  (decode_run16<RUNS>(P, which, col, h, bc, bs, ch, tile, lo, row), ...);
}

// Decodes K^ or V^ of token `col` (col < 0: zeros) into row `row` of `tile` (and `lo`).
__device__ __forceinline__ void decode_column(const AttnParams& P, int which, int col, int h,
                                              uint32_t chain_mask, uint8_t* tile, uint8_t* lo,
                                              int row) {
  if (col < 0) {
    float z[16];
#pragma unroll
    for (int k = 0; k < 16; ++k) z[k] = 0.f;
#pragma unroll
    for (int e0 = 0; e0 < HDT; e0 += 16) store_run(tile, lo, row, e0, z);
    return;
  }
  const KvView& kv = P.kv;
  const size_t bh = (size_t)col * P.H + h;
  const uint8_t* bc = kv.codes[which][1] + bh * (kv.base_bits ? HDT : HDT * 4);
  const uint32_t* bs = kv.base_bits ? reinterpret_cast<const uint32_t*>(kv.sz[which][1]) + bh * (HDT / kv.g)
                                    : nullptr;
  Chain ch;
  load_chain(P, which, col, h, chain_mask, ch);
  decode_runs(P, which, col, h, bc, bs, ch, tile, lo, row,
              std::make_integer_sequence<int, HDT / 16>{});
}

// Rows wrow0 .. wrow0 + 31 of a K-major operand tile from staged fp16 rows, by one warp:
// lane l names the column of row wrow0 + l (col < 0: zeros); each row (256 bytes) is
// copied by 16 lanes, 16 bytes each, two rows per step, as asynchronous copies into the
// swizzled places. src points at the head's [n_tok][HDT] rows. The caller waits for its
// copies and fences them for the tensor cores before handing the tile over.
__device__ __forceinline__ void copy_rows_warp(const __half* src, uint8_t* tile, int col,
                                               int wrow0, int lane) {
  const int half = lane >> 4, piece = lane & 15;
  const uint32_t t = smem_u32(tile);
#pragma unroll 4
  for (int s = 0; s < 16; ++s) {
    const int rr = 2 * s + half;
    const int c = __shfl_sync(0xffffffffu, col, rr);
    const uint32_t off = sw128_offset(wrow0 + rr, 8 * piece, TC);
    if (c >= 0) cp_async16(t + off, src + (size_t)c * HDT + 8 * piece);
    else *reinterpret_cast<uint4*>(tile + off) = make_uint4(0u, 0u, 0u, 0u);
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
