// Loop-aware sparse attention for calls with few queries - batched decode, where every
// sequence contributes one generated token (FlashLoop §4.2 "Loop-Aware Sparse Attention":
// softmax over the carried columns, rescaled by the cached mass, plus the carried
// unselected contribution; §5.3.3 / Figure 5: decode with sparse attention over a
// quantised KV).
//
// With one query per (sequence, head) a query tile would leave 127 of its 128 rows empty
// and decode every column for a single row. Here one CTA of eight warps streams one
// query's carried columns straight from the quantised store: the warps split the set,
// each lane reconstructs four elements of K^ and V^ per column (the int8 base, then the
// residual row of every loop that rewrote the token, fmaf(code, s, z) added in loop order
// in binary32 - the store's own reconstruction), four columns per step with their loads
// issued together. The logit is a warp sum in binary32, the softmax an online one per
// warp (binary32 throughout), merged across the warps at the end:
//   o = u + m * (sum_w 2^(m_w - M) O_w) / (sum_w 2^(m_w - M) l_w).
#include <float.h>

#include "fl_internal.cuh"

namespace fl {
namespace {

constexpr int DW = 8;        // warps per (query, head)
constexpr int CB = 4;        // columns per warp step
constexpr float kLog2eD = 1.4426950408889634f;

// 4 values of a stored row at elements [e0, e0 + 4) (e0 a multiple of 4), as binary32:
// fmaf(code, s, z), or the raw values when the loop is unquantised.
__device__ __forceinline__ void row4(const KvView& kv, int which, int r, int bits, int row, int h,
                                     int e0, float* x) {
  const size_t rh = (size_t)row * kv.H + h;
  if (bits == 0) {
    const float4 v = __ldg(reinterpret_cast<const float4*>(kv.codes[which][r]) + (rh * kv.hd + e0) / 4);
    x[0] = v.x; x[1] = v.y; x[2] = v.z; x[3] = v.w;
    return;
  }
  const uint8_t* cp = kv.codes[which][r] + rh * (kv.hd * bits / 8);
  uint32_t w;
  if (bits == 8) w = __ldg(reinterpret_cast<const uint32_t*>(cp + e0));
  else if (bits == 4) w = __ldg(reinterpret_cast<const uint16_t*>(cp + e0 / 2));
  else w = __ldg(cp + e0 / 4);
  const uint32_t szw =
      __ldg(reinterpret_cast<const uint32_t*>(kv.sz[which][r]) + rh * (kv.hd / kv.g) + e0 / kv.g);
  const float s = half_bits_to_float((uint16_t)(szw & 0xFFFFu));
  const float z = half_bits_to_float((uint16_t)(szw >> 16));
  const uint32_t m = (1u << bits) - 1u;
#pragma unroll
  for (int i = 0; i < 4; ++i) x[i] = __fmaf_rn((float)((w >> (i * bits)) & m), s, z);
}

// K^ and V^ of the step's columns at elements [e0, e0 + 4): the bases of all columns,
// then loop by loop the slots of all columns and the residual rows of those that the
// loop rewrote (added in loop order; a raw loop replaces) - the loads of the CB columns
// of a phase issued together.
__device__ __forceinline__ void columns4(const AttnParams& P, const int* cols, const bool* ok, int h,
                                         int e0, float (*k)[4], float (*v)[4]) {
  const KvView& kv = P.kv;
#pragma unroll
  for (int j = 0; j < CB; ++j) {
    const int c = ok[j] ? cols[j] : 0;
    row4(kv, 0, 1, kv.base_bits, c, h, e0, k[j]);
    row4(kv, 1, 1, kv.base_bits, c, h, e0, v[j]);
  }
  for (int r = 2; r <= P.loop; ++r) {
    const int bits = kv.res_bits[r];
    int rows[CB];
#pragma unroll
    for (int j = 0; j < CB; ++j) rows[j] = ok[j] ? __ldg(kv.slot + (size_t)r * kv.n_tok + cols[j]) : -1;
#pragma unroll
    for (int j = 0; j < CB; ++j) {
      if (rows[j] < 0) continue;
      float dk[4], dv[4];
      row4(kv, 0, r, bits, rows[j], h, e0, dk);
      row4(kv, 1, r, bits, rows[j], h, e0, dv);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        k[j][i] = bits == 0 ? dk[i] : __fadd_rn(k[j][i], dk[i]);
        v[j][i] = bits == 0 ? dv[i] : __fadd_rn(v[j][i], dv[i]);
      }
    }
  }
}

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

struct DecodeShared {
  float m[DW], l[DW];
  float o[DW][128];
};

__device__ __forceinline__ void decode_cta(const AttnParams& P, int qi, int h) {
  __shared__ DecodeShared sh;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int H = P.H, n_tok = P.kv.n_tok, stride = P.sel_stride;
  const int t = P.q_tok[qi];
  const int srow = P.q_row ? P.q_row[qi] : t;
  if (t < 0 || t >= n_tok || srow < 0 || srow >= P.stat_rows) {   // the whole CTA leaves
    if (threadIdx.x == 0) record_error(P.st, FL_ERR_RANGE);
    return;
  }
  const int e0 = lane * 4;
  const float scale2 = P.scale * kLog2eD;   // logits in log2 units
  float q[4];
  {
    const size_t off = ((size_t)qi * H + h) * 128 + e0;
    if (P.q_bf16) {
      const uint2 w = __ldg(reinterpret_cast<const uint2*>(reinterpret_cast<const __nv_bfloat16*>(P.q) + off));
      const __nv_bfloat162* b2 = reinterpret_cast<const __nv_bfloat162*>(&w);
      q[0] = __low2float(b2[0]); q[1] = __high2float(b2[0]);
      q[2] = __low2float(b2[1]); q[3] = __high2float(b2[1]);
    } else {
      const float4 w = __ldg(reinterpret_cast<const float4*>(reinterpret_cast<const float*>(P.q) + off));
      q[0] = w.x; q[1] = w.y; q[2] = w.z; q[3] = w.w;
    }
  }
  const uint16_t* row = P.sel + ((size_t)h * P.stat_rows + srow) * stride;
  const int per = (stride + DW - 1) / DW;
  const int ebeg = warp * per, eend = min(stride, ebeg + per);
  float m_w = -INFINITY, l_w = 0.f, acc[4] = {0.f, 0.f, 0.f, 0.f};
  for (int e = ebeg; e < eend; e += CB) {
    // the step's columns: lane j < CB reads entry e + j, all lanes take them by shuffle
    int cj = (int)FL_SENTINEL;
    if (lane < CB && e + lane < eend) cj = (int)__ldg(row + e + lane);
    int cols[CB];
#pragma unroll
    for (int j = 0; j < CB; ++j) cols[j] = __shfl_sync(0xffffffffu, cj, j);
    if (cols[0] == (int)FL_SENTINEL) break;   // sets end in sentinels
    float kk[CB][4], vv[CB][4];
    bool ok[CB];
#pragma unroll
    for (int j = 0; j < CB; ++j) {
      const int c = cols[j];
      ok[j] = c != (int)FL_SENTINEL && c <= t;   // uniform across the warp
      if (c != (int)FL_SENTINEL && !ok[j] && lane == 0) record_error(P.st, FL_ERR_RANGE);
    }
    columns4(P, cols, ok, h, e0, kk, vv);
#pragma unroll
    for (int j = 0; j < CB; ++j) {
      const int c = cols[j];
      float d = 0.f;
#pragma unroll
      for (int i = 0; i < 4; ++i) d = fmaf(q[i], kk[j][i], d);
      d = warp_sum(d);
      if (!ok[j]) continue;
      const float x = d * scale2 + (P.bias ? __ldg(P.bias + c) * kLog2eD : 0.f);
      if (x > m_w) {
        const float a = exp2f(m_w - x);   // 0 while m_w = -inf
        l_w *= a;
#pragma unroll
        for (int i = 0; i < 4; ++i) acc[i] *= a;
        m_w = x;
      }
      const float p = exp2f(x - m_w);
      l_w += p;
#pragma unroll
      for (int i = 0; i < 4; ++i) acc[i] = fmaf(p, vv[j][i], acc[i]);
    }
  }
  if (lane == 0) { sh.m[warp] = m_w; sh.l[warp] = l_w; }
#pragma unroll
  for (int i = 0; i < 4; ++i) sh.o[warp][e0 + i] = acc[i];
  __syncthreads();
  if (warp != 0) return;
  float M = -INFINITY;
#pragma unroll
  for (int w = 0; w < DW; ++w) M = fmaxf(M, sh.m[w]);
  float L = 0.f, o[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int w = 0; w < DW; ++w) {
    const float a = sh.m[w] == -INFINITY ? 0.f : exp2f(sh.m[w] - M);
    L = fmaf(sh.l[w], a, L);
#pragma unroll
    for (int i = 0; i < 4; ++i) o[i] = fmaf(sh.o[w][e0 + i], a, o[i]);
  }
  const float mass = P.mass[(size_t)h * P.stat_rows + srow];
  const float f = L > 0.f ? mass / L : 0.f;
  const float4 u = __ldg(reinterpret_cast<const float4*>(P.unsel + ((size_t)h * P.stat_rows + srow) * 128 + e0));
  const float r0 = fmaf(o[0], f, u.x), r1 = fmaf(o[1], f, u.y), r2 = fmaf(o[2], f, u.z), r3 = fmaf(o[3], f, u.w);
  const size_t ob = ((size_t)qi * H + h) * 128 + e0;
  if (P.out_bf16) {
    const __nv_bfloat162 a = __floats2bfloat162_rn(r0, r1), b = __floats2bfloat162_rn(r2, r3);
    *reinterpret_cast<uint2*>(reinterpret_cast<__nv_bfloat16*>(P.out) + ob) =
        make_uint2(*reinterpret_cast<const uint32_t*>(&a), *reinterpret_cast<const uint32_t*>(&b));
  } else {
    *reinterpret_cast<float4*>(reinterpret_cast<float*>(P.out) + ob) = make_float4(r0, r1, r2, r3);
  }
}

// one CTA per (query, head) of one call
__global__ void __launch_bounds__(DW * 32) k_attn_decode(const __grid_constant__ AttnParams P) {
  griddep_wait();
  decode_cta(P, blockIdx.x / P.H, blockIdx.x % P.H);
}

// many calls in one launch: CTA b works on call b / per (per = n_q x heads of a call)
__global__ void __launch_bounds__(DW * 32) k_attn_decode_batched(const AttnParams* __restrict__ Ps, int per) {
  __shared__ AttnParams sP;
  const int call = blockIdx.x / per, b = blockIdx.x % per;
  {
    const uint32_t* src = reinterpret_cast<const uint32_t*>(Ps + call);
    uint32_t* dst = reinterpret_cast<uint32_t*>(&sP);
    for (int i = threadIdx.x; i < (int)(sizeof(AttnParams) / 4); i += blockDim.x) dst[i] = src[i];
  }
  __syncthreads();
  decode_cta(sP, b / sP.H, b % sP.H);
}

}  // namespace

// Sparse calls this kernel serves: head_dim 128, no statistics written (none requested,
// or in place with an unchanged budget) - the tile kernel's conditions, for few queries.
bool sparse_decode_eligible(const AttnParams& P) {
  return sparse_tile_eligible(P);
}

cudaError_t launch_attn_decode(const AttnParams& P, cudaStream_t s) {
  if (P.n_q <= 0) return cudaSuccess;
  const cudaError_t e = launch_pdl(k_attn_decode, dim3((unsigned)(P.n_q * P.H)), dim3(DW * 32), 0, s, P);
  count_launch();
  return e != cudaSuccess ? e : cudaGetLastError();
}

cudaError_t launch_attn_decode_batched(const AttnParams& P0, const AttnParams* Ps_dev, int n,
                                       cudaStream_t s) {
  if (n <= 0 || P0.n_q <= 0) return cudaSuccess;
  const int per = P0.n_q * P0.H;
  k_attn_decode_batched<<<(unsigned)(per * n), DW * 32, 0, s>>>(Ps_dev, per);
  count_launch();
  return cudaGetLastError();
}

}  // namespace fl
