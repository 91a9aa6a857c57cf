// Cross-loop KV residual quantisation (FlashLoop §3.3, §4.3; Appendix E
// "Quantization Setting": asymmetric group-wise min/max quantisation, the same
// scheme for the base state and the residuals).
//
// One warp per (row, head, K|V). Lane l holds the hd/32 consecutive elements
// [l*hd/32, (l+1)*hd/32); a quantisation group of g elements is g/(hd/32) adjacent
// lanes, reduced with xor shuffles. Every step is an IEEE binary32/binary16 operation
// with the stated rounding, so the codes are bit-exact against any implementation of
// the same definition:
//   z = fp16_RD(min), s = fp16_RU(f32_RU(f32_RU(max - z) / (2^b - 1))),
//   code = s == 0 ? 0 : clamp(rint(f32_RN(f32_RN(x - z) / s)), 0, 2^b - 1),
//   deq = fmaf(code, s, z).
// Loop r >= 2 first rebuilds K^_{r-1} of the row (base + chain) and quantises the
// residual x = fl32(k - K^_{r-1}). Codes are OR-combined across the lanes that share a
// 32-bit word and stored little-endian, low bits first.
#include "fl_internal.cuh"

namespace fl {
namespace {

struct QuantOut {
  uint8_t* codes[2];
  uint16_t* sz[2];
  int32_t* slot_row;  // slot[loop][*] (loop >= 2) or nullptr
  float* vnorm;       // [n_tok][H] or nullptr
  int row0;           // first residual row written (loop >= 2)
};

// K^ or V^ of token t at loop `upto` (t is the same for the whole warp, upto <= 31): lanes
// 2..upto look up the slot rows of their loops at once, then the chain's rows are decoded
// and added in loop order (a raw loop replaces the value).
template <int N>
__device__ __forceinline__ void reconstruct_warp(const KvView& kv, int which, int upto, int t,
                                                 int h, int e0, int lane, float* acc) {
  int my_row = -1;
  if (lane >= 2 && lane <= upto) my_row = kv.slot[(size_t)lane * kv.n_tok + t];
  decode_run<N>(kv, which, 1, kv.base_bits, t, h, e0, acc);
  for (int r = 2; r <= upto; ++r) {
    const int row = __shfl_sync(0xffffffffu, my_row, r);
    if (row < 0) continue;
    float d[N];
    const int bits = kv.res_bits[r];
    decode_run<N>(kv, which, r, bits, row, h, e0, d);
    if (bits == 0) {
#pragma unroll
      for (int i = 0; i < N; ++i) acc[i] = d[i];
    } else {
#pragma unroll
      for (int i = 0; i < N; ++i) acc[i] = __fadd_rn(acc[i], d[i]);
    }
  }
}

// Quantises this lane's EPL values x of (row, head h, K|V) (group g = LPG lanes), stores
// codes and (s, z); hat = the reconstruction (prev + deq, or deq at loop 1; raw values
// when bits == 0).
template <int EPL>
__device__ __forceinline__ void quant_store(const KvView& kv, const QuantOut& out, int which,
                                            int loop, int bits, size_t row, int h, int e0,
                                            int lane, const float* xin, const float* x,
                                            const float* prev, float* hat, int* st) {
  const int H = kv.H, hd = kv.hd, g = kv.g;
  if (bits == 0) {
    float* dst = reinterpret_cast<float*>(out.codes[which]) + (row * H + h) * hd + e0;
#pragma unroll
    for (int j = 0; j < EPL; ++j) { dst[j] = xin[j]; hat[j] = xin[j]; }
    return;
  }
  const int LPG = g / EPL;  // lanes per group
  float mn = x[0], mx = x[0];
#pragma unroll
  for (int j = 1; j < EPL; ++j) { mn = fminf(mn, x[j]); mx = fmaxf(mx, x[j]); }
  for (int o = 1; o < LPG; o <<= 1) {
    mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  }
  const __half zh = __float2half_rd(mn);
  const float zf = __half2float(zh);
  const float qmax = (float)((1 << bits) - 1);
  const float t1 = __fsub_ru(mx, zf);
  const float t2 = __fdiv_ru(t1, qmax);
  const __half sh = __float2half_ru(t2);
  const float sf = __half2float(sh);
  const bool bad = isinf(zf) || isinf(sf) || isnan(zf) || isnan(sf);
  if (bad && (lane % LPG) == 0) record_error(st, FL_ERR_RANGE);
  uint32_t word = 0;
#pragma unroll
  for (int j = 0; j < EPL; ++j) {
    int code = 0;
    if (!bad && sf != 0.f) {
      const float w = __fdiv_rn(__fsub_rn(x[j], zf), sf);
      code = (int)fminf(fmaxf(rintf(w), 0.f), qmax);
    }
    const float deq = __fmaf_rn((float)code, sf, zf);
    hat[j] = loop == 1 ? deq : __fadd_rn(prev[j], deq);
    word |= (uint32_t)code << (j * bits);
  }
  // combine the lanes that share one 32-bit output word
  const int wbits = EPL * bits;
  const int LPW = 32 / wbits;
  word <<= (lane % LPW) * wbits;
  for (int o = 1; o < LPW; o <<= 1) word |= __shfl_xor_sync(0xffffffffu, word, o);
  const size_t rowbytes = (size_t)hd * bits / 8;
  if (lane % LPW == 0) {
    uint32_t* cw = reinterpret_cast<uint32_t*>(out.codes[which] + (row * H + h) * rowbytes);
    cw[lane / LPW] = word;
  }
  if (lane % LPG == 0) {
    uint32_t* szw = reinterpret_cast<uint32_t*>(out.sz[which]);
    const uint32_t pair = (uint32_t)__half_as_ushort(sh) | ((uint32_t)__half_as_ushort(zh) << 16);
    szw[(row * H + h) * (hd / g) + e0 / g] = pair;
  }
}

// One warp per (row, head): K and V together, so the loads of both (inputs, the slot rows
// and the chain codes) are in flight at once.
template <int EPL, typename T>
__global__ void __launch_bounds__(256) k_kv_quant(KvView kv, QuantOut out, int loop,
                                                  const T* __restrict__ k_new,
                                                  const T* __restrict__ v_new,
                                                  const int32_t* __restrict__ act_tok,
                                                  int n_act, int* st) {
  griddep_wait();
  const int gw = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  const int H = kv.H, hd = kv.hd;
  if (gw >= n_act * H) return;
  const int h = gw % H;
  const int i = gw / H;
  const int t = act_tok ? act_tok[i] : i;
  if (t < 0 || t >= kv.n_tok) {
    if (lane == 0) record_error(st, FL_ERR_RANGE);
    return;
  }
  const int e0 = lane * EPL;
  const size_t off = ((size_t)i * H + h) * hd + e0;
  float xin[2][EPL];
#pragma unroll
  for (int j = 0; j < EPL; ++j) {
    xin[0][j] = to_f32<T>(k_new[off + j]);
    xin[1][j] = to_f32<T>(v_new[off + j]);
  }
  const int bits = loop == 1 ? kv.base_bits : kv.res_bits[loop];
  float prev[2][EPL], x[2][EPL];
  if (loop >= 2) {
    reconstruct_warp<EPL>(kv, 0, loop - 1, t, h, e0, lane, prev[0]);
    reconstruct_warp<EPL>(kv, 1, loop - 1, t, h, e0, lane, prev[1]);
#pragma unroll
    for (int w = 0; w < 2; ++w)
#pragma unroll
      for (int j = 0; j < EPL; ++j) x[w][j] = bits == 0 ? xin[w][j] : __fsub_rn(xin[w][j], prev[w][j]);
  } else {
#pragma unroll
    for (int w = 0; w < 2; ++w)
#pragma unroll
      for (int j = 0; j < EPL; ++j) { x[w][j] = xin[w][j]; prev[w][j] = 0.f; }
  }
  const size_t row = loop == 1 ? (size_t)t : (size_t)out.row0 + i;
  float hat[EPL];
  quant_store<EPL>(kv, out, 0, loop, bits, row, h, e0, lane, xin[0], x[0], prev[0], hat, st);
  quant_store<EPL>(kv, out, 1, loop, bits, row, h, e0, lane, xin[1], x[1], prev[1], hat, st);
  if (out.vnorm) {   // ||V^|| from the V reconstruction (hat of the second call)
    float ss = 0.f;
#pragma unroll
    for (int j = 0; j < EPL; ++j) ss = fmaf(hat[j], hat[j], ss);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    if (lane == 0) out.vnorm[(size_t)t * H + h] = sqrtf(ss);
  }
  if (loop >= 2 && h == 0 && lane == 0 && out.slot_row) out.slot_row[t] = (int32_t)row;
}

template <int EPL>
cudaError_t launch_epl(const KvView& v, const QuantOut& o, int loop, const void* k,
                       const void* vv, fl_dtype dt, const int32_t* act, int n_act, int* st,
                       cudaStream_t s) {
  const size_t warps = (size_t)n_act * v.H;
  const int blocks = (int)((warps * 32 + 255) / 256);
  const cudaError_t e =
      dt == FL_F32
          ? launch_pdl(k_kv_quant<EPL, float>, dim3(blocks), dim3(256), 0, s, v, o, loop,
                       (const float*)k, (const float*)vv, act, n_act, st)
          : launch_pdl(k_kv_quant<EPL, __nv_bfloat16>, dim3(blocks), dim3(256), 0, s, v, o, loop,
                       (const __nv_bfloat16*)k, (const __nv_bfloat16*)vv, act, n_act, st);
  count_launch();
  return e != cudaSuccess ? e : cudaGetLastError();
}

}  // namespace

cudaError_t launch_kv_quant(const fl_kv_desc& kv, int loop, const void* k_new,
                            const void* v_new, fl_dtype dt, const int32_t* act_tok, int n_act,
                            int* st, cudaStream_t s, int row0, bool append) {
  if (n_act <= 0) return cudaSuccess;
  KvView v = make_view(kv);
  QuantOut o;
  for (int w = 0; w < 2; ++w) { o.codes[w] = kv.codes[w][loop]; o.sz[w] = kv.sz[w][loop]; }
  o.slot_row = nullptr;
  o.vnorm = kv.vnorm;
  o.row0 = row0;
  cudaError_t e;
  if (loop >= 2) {
    o.slot_row = kv.slot + (size_t)loop * kv.n_tok;
    if (!append) {
      e = launch_fill_i32(o.slot_row, -1, (size_t)kv.n_tok, s);
      if (e != cudaSuccess) return e;
    }
  } else if (kv.slot && !append) {
    e = launch_iota(kv.slot + kv.n_tok, kv.n_tok, s);
    if (e != cudaSuccess) return e;
  }
  if (kv.head_dim == 128) return launch_epl<4>(v, o, loop, k_new, v_new, dt, act_tok, n_act, st, s);
  return launch_epl<2>(v, o, loop, k_new, v_new, dt, act_tok, n_act, st, s);
}

// K^_loop and V^_loop of the listed tokens, rebuilt from the store: the base, then the
// residual row of every loop 2..loop that lists the token, added in loop order (the
// store's own reconstruction, bit for bit). One thread per 8 elements of a (token, head).
__global__ void k_kv_reconstruct(const KvView kv, int loop, const int32_t* __restrict__ tok,
                                 int n, float* __restrict__ out_k, float* __restrict__ out_v,
                                 int* st) {
  const int per_row = kv.H * (kv.hd / 8);
  const long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x;
  if (i >= (long long)n * per_row) return;
  const int row = (int)(i / per_row), rem = (int)(i % per_row);
  const int h = rem / (kv.hd / 8), e0 = (rem % (kv.hd / 8)) * 8;
  const int t = tok[row];
  if (t < 0 || t >= kv.n_tok) {
    record_error(st, FL_ERR_RANGE);
    return;
  }
  const size_t o = ((size_t)row * kv.H + h) * kv.hd + e0;
  float acc[8];
  reconstruct<8>(kv, 0, loop, t, h, e0, acc);
#pragma unroll
  for (int k = 0; k < 8; ++k) out_k[o + k] = acc[k];
  reconstruct<8>(kv, 1, loop, t, h, e0, acc);
#pragma unroll
  for (int k = 0; k < 8; ++k) out_v[o + k] = acc[k];
}

cudaError_t launch_kv_reconstruct(const fl_kv_desc& kv, int loop, const int32_t* tok, int n,
                                  float* out_k, float* out_v, int* st, cudaStream_t s) {
  if (n <= 0) return cudaSuccess;
  const long long threads = (long long)n * kv.n_heads * (kv.head_dim / 8);
  const int blocks = (int)((threads + 255) / 256);
  k_kv_reconstruct<<<blocks, 256, 0, s>>>(make_view(kv), loop, tok, n, out_k, out_v, st);
  count_launch();
  return cudaGetLastError();
}

}  // namespace fl
