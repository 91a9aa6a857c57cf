// Quantisation of one group of 32 binary32 values held by one thread, for the fused
// QKV-projection epilogue (FlashLoop §4.4: the cross-loop KV update and quantisation fused
// with the projection; §4.3 / Appendix E: asymmetric min/max group quantisation).
//
// The arithmetic is the store's definition step for step (the same IEEE operations and
// roundings as the standalone quantiser), so the codes are identical:
//   z = fp16_RD(min), s = fp16_RU(f32_RU(f32_RU(max - z) / (2^b - 1))),
//   code = s == 0 ? 0 : clamp(rint(f32(f32(x - z) / s)), 0, 2^b - 1), deq = fmaf(code, s, z);
// loop r >= 2 quantises x - K^_{r-1} with K^ rebuilt from base + chain, K^_r = K^_{r-1} + deq.
#pragma once
#include "fl_internal.cuh"

namespace fl {

// Destination of the fused quantisation (one layer's store, one loop).
struct KvFuse {
  int on;                 // 0: no fused quantisation
  int loop;               // 1: base; >= 2: residual
  uint8_t* codes[2];      // loop's code arrays, K and V
  uint16_t* sz[2];        // loop's (scale, offset) arrays
  int32_t* slot_row;      // slot[loop][*] (loop >= 2), pre-filled with -1
  float* vnorm;           // [n_tok][H] or null
};

// Rebuild K^/V^ of 32 elements [e0, e0+32) of (token t, head h) at loop `upto`:
// base, then each loop 2..upto whose slot lists t, added in binary32.
__device__ __forceinline__ void rebuild32(const KvView& kv, int which, int upto, int t, int h,
                                          int e0, float* acc) {
  decode_run<32>(kv, which, 1, kv.base_bits, t, h, e0, acc);
  for (int r = 2; r <= upto; ++r) {
    const int row = kv.slot[(size_t)r * kv.n_tok + t];
    if (row < 0) continue;
    float d[32];
    decode_run<32>(kv, which, r, kv.res_bits[r], row, h, e0, d);
#pragma unroll
    for (int j = 0; j < 32; ++j) acc[j] = __fadd_rn(acc[j], d[j]);
  }
}

// Quantises x[32] with `bits`; writes codes (packed little-endian, low bits first) at
// `codes_dst` (32 * bits / 8 bytes) and the (s, z) pair at `sz_dst`. Returns the sum of
// squares of the reconstruction (prev + deq, or deq when prev is null) and sets *ok to
// false on an fp16 overflow of s or z (codes are then 0).
__device__ __forceinline__ float quant32(const float* x, int bits, uint8_t* codes_dst,
                                         uint32_t* sz_dst, const float* prev, bool* ok) {
  float mn = x[0], mx = x[0];
#pragma unroll
  for (int j = 1; j < 32; ++j) { mn = fminf(mn, x[j]); mx = fmaxf(mx, x[j]); }
  const __half zh = __float2half_rd(mn);
  const float zf = __half2float(zh);
  const float qmax = (float)((1 << bits) - 1);
  const __half sh = __float2half_ru(__fdiv_ru(__fsub_ru(mx, zf), qmax));
  const float sf = __half2float(sh);
  const bool bad = isinf(zf) || isinf(sf) || isnan(zf) || isnan(sf);
  uint32_t words[8] = {0, 0, 0, 0, 0, 0, 0, 0};
  float ss = 0.f;
#pragma unroll
  for (int j = 0; j < 32; ++j) {
    int code = 0;
    if (!bad && sf != 0.f) code = (int)fminf(fmaxf(rintf(__fdiv_rn(__fsub_rn(x[j], zf), sf)), 0.f), qmax);
    const float deq = __fmaf_rn((float)code, sf, zf);
    const float hat = prev ? __fadd_rn(prev[j], deq) : deq;
    ss = fmaf(hat, hat, ss);
    const int bit = j * bits;
    words[bit >> 5] |= (uint32_t)code << (bit & 31);
  }
  if (bits == 8) {
    uint4* d = reinterpret_cast<uint4*>(codes_dst);
    d[0] = make_uint4(words[0], words[1], words[2], words[3]);
    d[1] = make_uint4(words[4], words[5], words[6], words[7]);
  } else if (bits == 4) {
    *reinterpret_cast<uint4*>(codes_dst) = make_uint4(words[0], words[1], words[2], words[3]);
  } else {
    *reinterpret_cast<uint2*>(codes_dst) = make_uint2(words[0], words[1]);
  }
  *sz_dst = (uint32_t)__half_as_ushort(sh) | ((uint32_t)__half_as_ushort(zh) << 16);
  *ok = !bad;
  return ss;
}

// One quantisation group (32 values of token t, head h, elements [e0, e0+32)) of K
// (which 0) or V (which 1) written to the fused store for loop kf.loop; `i` is the row
// of the token among the call's rows (its residual row). `x` is overwritten. Returns the
// group's share of ||V^||^2 (0 for K).
__device__ __forceinline__ float fuse_group(const KvView& kv, const KvFuse& kf, int which,
                                            float* x, int i, int t, int h, int e0, int* st) {
  const int H = kv.H, hd = kv.hd;
  const int loop = kf.loop;
  const int bits = loop == 1 ? kv.base_bits : kv.res_bits[loop];
  const int dst_row = loop == 1 ? t : i;
  float prev[32];
  if (loop >= 2) {
    rebuild32(kv, which, loop - 1, t, h, e0, prev);
#pragma unroll
    for (int j = 0; j < 32; ++j) x[j] = __fsub_rn(x[j], prev[j]);
  }
  uint8_t* cd = kf.codes[which] + ((size_t)dst_row * H + h) * (size_t)(hd * bits / 8) + e0 * bits / 8;
  uint32_t* sd = reinterpret_cast<uint32_t*>(kf.sz[which]) + ((size_t)dst_row * H + h) * (hd / 32) + e0 / 32;
  bool ok = true;
  const float ss = quant32(x, bits, cd, sd, loop >= 2 ? prev : nullptr, &ok);
  if (!ok) record_error(st, FL_ERR_RANGE);
  if (loop >= 2 && which == 0 && h == 0 && e0 == 0 && kf.slot_row) kf.slot_row[t] = i;
  return which == 1 ? ss : 0.f;
}

}  // namespace fl
