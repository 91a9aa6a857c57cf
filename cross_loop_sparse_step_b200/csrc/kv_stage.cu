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
// candidate pass). One thread per 16 elements of a (token, head): 8 threads read a row's
// codes (128 bytes at 8 bits) and write its 256 fp16 bytes, both contiguous.
#include "fl_internal.cuh"

namespace fl {
namespace {

// 16 codes of `bits` bits from element e0 (a multiple of 16) of a stored row.
__device__ __forceinline__ void load_codes16(const uint8_t* row, int bits, int e0, uint32_t* w) {
  if (bits == 8) {
    const uint4 v = __ldg(reinterpret_cast<const uint4*>(row + e0));
    w[0] = v.x; w[1] = v.y; w[2] = v.z; w[3] = v.w;
  } else if (bits == 4) {
    const uint2 v = __ldg(reinterpret_cast<const uint2*>(row + e0 / 2));
    w[0] = v.x; w[1] = v.y;
  } else {   // 2 bits
    w[0] = __ldg(reinterpret_cast<const uint32_t*>(row + e0 / 4));
  }
}

// The raw material of 16 elements of one stored row: 64 bytes (codes in the first 16 and
// the (s, z) word, or the binary32 values themselves).
struct Run16 {
  uint4 q[4];
  uint32_t szw;
};

__device__ __forceinline__ void load_run16(const KvView& kv, int which, int r, int bits, int row,
                                           int h, int e0, Run16& x) {
  const size_t rh = (size_t)row * kv.H + h;
  if (bits == 0) {
    const uint4* p = reinterpret_cast<const uint4*>(kv.codes[which][r]) + (rh * kv.hd + e0) / 4;
#pragma unroll
    for (int k = 0; k < 4; ++k) x.q[k] = __ldg(p + k);
    x.szw = 0u;
    return;
  }
  uint32_t w[4] = {0u, 0u, 0u, 0u};
  load_codes16(kv.codes[which][r] + rh * (kv.hd * bits / 8), bits, e0, w);
  x.q[0] = make_uint4(w[0], w[1], w[2], w[3]);
  x.szw = __ldg(reinterpret_cast<const uint32_t*>(kv.sz[which][r]) + rh * (kv.hd / kv.g) + e0 / kv.g);
}

template <int BITS>
__device__ __forceinline__ void add_codes16(const Run16& x, bool first, float* acc) {
  const float s = half_bits_to_float((uint16_t)(x.szw & 0xFFFFu));
  const float z = half_bits_to_float((uint16_t)(x.szw >> 16));
  const uint32_t w[4] = {x.q[0].x, x.q[0].y, x.q[0].z, x.q[0].w};
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    constexpr uint32_t M = (1u << BITS) - 1u;
    const uint32_t c = (w[(i * BITS) >> 5] >> ((i * BITS) & 31)) & M;
    const float d = __fmaf_rn((float)c, s, z);
    acc[i] = first ? d : __fadd_rn(acc[i], d);
  }
}

// acc = the run's values (first = true) or acc + them, in binary32 (a raw loop replaces)
__device__ __forceinline__ void apply_run16(const Run16& x, int bits, bool first, float* acc) {
  if (bits == 0) {
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      acc[4 * k] = __uint_as_float(x.q[k].x); acc[4 * k + 1] = __uint_as_float(x.q[k].y);
      acc[4 * k + 2] = __uint_as_float(x.q[k].z); acc[4 * k + 3] = __uint_as_float(x.q[k].w);
    }
  } else if (bits == 2) {
    add_codes16<2>(x, first, acc);
  } else if (bits == 4) {
    add_codes16<4>(x, first, acc);
  } else {
    add_codes16<8>(x, first, acc);
  }
}

__device__ __forceinline__ uint32_t pack2(float a, float b) {
  const __half2 v = __floats2half2_rn(a, b);
  return *reinterpret_cast<const uint32_t*>(&v);
}

__device__ __forceinline__ void store16(__half* dst, const float* v) {
  uint4* d = reinterpret_cast<uint4*>(dst);
  d[0] = make_uint4(pack2(v[0], v[1]), pack2(v[2], v[3]), pack2(v[4], v[5]), pack2(v[6], v[7]));
  d[1] = make_uint4(pack2(v[8], v[9]), pack2(v[10], v[11]), pack2(v[12], v[13]), pack2(v[14], v[15]));
}

// One thread per 16 elements of a (token, head): the K and V runs' loads are issued
// together (base codes and scales, then per rewriting loop the residual codes), then
// both are reconstructed and written.
__global__ void __launch_bounds__(256) k_kv_stage(const KvView kv, int loop, __half* __restrict__ khi,
                                                  __half* __restrict__ klo, __half* __restrict__ vhi) {
  const int per_tok = kv.H * (kv.hd / 16);
  const long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x;
  if (i >= (long long)kv.n_tok * per_tok) return;
  griddep_wait();
  const int t = (int)(i / per_tok), rem = (int)(i % per_tok);
  const int h = rem / (kv.hd / 16), e0 = (rem % (kv.hd / 16)) * 16;
  const size_t o = ((size_t)h * kv.n_tok + t) * kv.hd + e0;
  float ak[16], av[16];
  {
    Run16 xk, xv;
    load_run16(kv, 0, 1, kv.base_bits, t, h, e0, xk);
    load_run16(kv, 1, 1, kv.base_bits, t, h, e0, xv);
    apply_run16(xk, kv.base_bits, true, ak);
    apply_run16(xv, kv.base_bits, true, av);
  }
  for (int r = 2; r <= loop; ++r) {   // the loops that list the token, in order
    const int row = __ldg(kv.slot + (size_t)r * kv.n_tok + t);
    if (row < 0) continue;
    const int bits = kv.res_bits[r];
    Run16 xk, xv;
    load_run16(kv, 0, r, bits, row, h, e0, xk);
    load_run16(kv, 1, r, bits, row, h, e0, xv);
    apply_run16(xk, bits, bits == 0, ak);
    apply_run16(xv, bits, bits == 0, av);
  }
  store16(khi + o, ak);
  store16(vhi + o, av);
  if (klo) {
    float lo[16];
#pragma unroll
    for (int k = 0; k < 16; ++k) lo[k] = ak[k] - __half2float(__float2half_rn(ak[k]));
    store16(klo + o, lo);
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
  const long long threads = (long long)kv.n_tok * kv.H * (kv.hd / 16);
  const cudaError_t e = launch_pdl(k_kv_stage, dim3((unsigned)((threads + 255) / 256)), dim3(256), 0, s,
                                   kv, loop, out->khi, out->klo, out->vhi);
  count_launch();
  return e != cudaSuccess ? e : cudaGetLastError();
}

}  // namespace fl
