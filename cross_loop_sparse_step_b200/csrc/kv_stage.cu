// The reconstruction K^_loop, V^_loop of every token of one layer's store, written once as
// fp16 operand rows for the query-tile attention kernels (FlashLoop §4.4 "GPU support":
// the quantised KV is dequantised on its way to the attention; §3.3: K^ is the base plus
// the residuals of the loops that rewrote the token).
//
// A query tile touches the union of its queries' columns; tiles of the same head share
// most of them (at a 32K prompt with 2048 carried columns a tile's union is nearly every
// column before it). Decoding inside each tile would redo the same dequantisation once per
// tile, so the store is decoded once per call into a transient buffer and the tiles gather
// fp16 rows from it:
//   hi[h][t][e] = fp16(x),  lo[h][t][e] = fp16(x - fp16(x))  (x = K^ or V^ in binary32)
// lo is written for K only and only when asked (the split operands of the dense kernel's
// candidate pass). One thread per 8 elements of a (token, head): 16 threads read a row's
// codes (128 bytes at 8 bits) and write its 256 fp16 bytes, both contiguous.
#include "fl_internal.cuh"

namespace fl {
namespace {

// 8 codes of `bits` bits from element e0 of a stored row, as unsigned integers.
__device__ __forceinline__ void load_codes8(const uint8_t* row, int bits, int e0, uint32_t* c) {
  if (bits == 8) {
    const uint2 w = __ldg(reinterpret_cast<const uint2*>(row + e0));
#pragma unroll
    for (int i = 0; i < 4; ++i) { c[i] = (w.x >> (8 * i)) & 0xFFu; c[4 + i] = (w.y >> (8 * i)) & 0xFFu; }
  } else if (bits == 4) {
    const uint32_t w = __ldg(reinterpret_cast<const uint32_t*>(row + e0 / 2));
#pragma unroll
    for (int i = 0; i < 8; ++i) c[i] = (w >> (4 * i)) & 0xFu;
  } else {   // 2 bits
    const uint32_t w = __ldg(reinterpret_cast<const uint16_t*>(row + e0 / 4));
#pragma unroll
    for (int i = 0; i < 8; ++i) c[i] = (w >> (2 * i)) & 0x3u;
  }
}

// x[0..8) = the stored row's values at e0: fmaf(code, s, z), or the raw binary32 values.
__device__ __forceinline__ void row_values8(const KvView& kv, int which, int r, int bits, int row,
                                            int h, int e0, float* x) {
  const size_t rh = (size_t)row * kv.H + h;
  if (bits == 0) {
    const float4* p = reinterpret_cast<const float4*>(kv.codes[which][r]) + (rh * kv.hd + e0) / 4;
    const float4 a = __ldg(p), b = __ldg(p + 1);
    x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w; x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
    return;
  }
  uint32_t c[8];
  load_codes8(kv.codes[which][r] + rh * (kv.hd * bits / 8), bits, e0, c);
  const uint32_t szw =
      __ldg(reinterpret_cast<const uint32_t*>(kv.sz[which][r]) + rh * (kv.hd / kv.g) + e0 / kv.g);
  const float s = half_bits_to_float((uint16_t)(szw & 0xFFFFu));
  const float z = half_bits_to_float((uint16_t)(szw >> 16));
#pragma unroll
  for (int i = 0; i < 8; ++i) x[i] = __fmaf_rn((float)c[i], s, z);
}

__device__ __forceinline__ uint32_t pack2(float a, float b) {
  const __half2 v = __floats2half2_rn(a, b);
  return *reinterpret_cast<const uint32_t*>(&v);
}

__global__ void __launch_bounds__(256) k_kv_stage(const KvView kv, int loop, __half* __restrict__ khi,
                                                  __half* __restrict__ klo, __half* __restrict__ vhi) {
  const int per_tok = kv.H * (kv.hd / 8);
  const long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x;
  if (i >= (long long)kv.n_tok * per_tok) return;
  griddep_wait();
  const int t = (int)(i / per_tok), rem = (int)(i % per_tok);
  const int h = rem / (kv.hd / 8), e0 = (rem % (kv.hd / 8)) * 8;
  const size_t o = ((size_t)h * kv.n_tok + t) * kv.hd + e0;
#pragma unroll 1
  for (int which = 0; which < 2; ++which) {
    float acc[8];
    row_values8(kv, which, 1, kv.base_bits, t, h, e0, acc);
    for (int r = 2; r <= loop; ++r) {   // the loops that list the token, in order
      const int row = __ldg(kv.slot + (size_t)r * kv.n_tok + t);
      if (row < 0) continue;
      const int bits = kv.res_bits[r];
      float d[8];
      row_values8(kv, which, r, bits, row, h, e0, d);
#pragma unroll
      for (int k = 0; k < 8; ++k) acc[k] = bits == 0 ? d[k] : __fadd_rn(acc[k], d[k]);
    }
    uint4 hv;
    hv.x = pack2(acc[0], acc[1]); hv.y = pack2(acc[2], acc[3]);
    hv.z = pack2(acc[4], acc[5]); hv.w = pack2(acc[6], acc[7]);
    *reinterpret_cast<uint4*>((which ? vhi : khi) + o) = hv;
    if (which == 0 && klo) {
      float r8[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) r8[k] = acc[k] - __half2float(__float2half_rn(acc[k]));
      uint4 lv;
      lv.x = pack2(r8[0], r8[1]); lv.y = pack2(r8[2], r8[3]);
      lv.z = pack2(r8[4], r8[5]); lv.w = pack2(r8[6], r8[7]);
      *reinterpret_cast<uint4*>(klo + o) = lv;
    }
  }
}

}  // namespace

size_t kv_stage_bytes(const KvView& kv, bool with_lo) {
  return (size_t)(with_lo ? 3 : 2) * kv.H * kv.n_tok * kv.hd * sizeof(__half);
}

cudaError_t launch_kv_stage(const KvView& kv, int loop, void* buf, bool with_lo, KvStage* out,
                            cudaStream_t s) {
  const size_t n = (size_t)kv.H * kv.n_tok * kv.hd;
  __half* base = static_cast<__half*>(buf);
  out->khi = base;
  out->vhi = base + n;
  out->klo = with_lo ? base + 2 * n : nullptr;
  if (kv.n_tok <= 0) return cudaSuccess;
  const long long threads = (long long)kv.n_tok * kv.H * (kv.hd / 8);
  const cudaError_t e = launch_pdl(k_kv_stage, dim3((unsigned)((threads + 255) / 256)), dim3(256), 0, s,
                                   kv, loop, out->khi, out->klo, out->vhi);
  count_launch();
  return e != cudaSuccess ? e : cudaGetLastError();
}

}  // namespace fl
