// Dense causal attention of loop 1 and the column statistics it hands to loop 2
// (FlashLoop §4.2: the sparse loops rank columns with statistics of the previous loop;
// the dense loop is where they are produced). One warp per (query, head).
//
// Four lanes per column (a lane owns a quarter of the head slice, one quantisation group
// at head_dim 128), sixteen columns in flight per warp (two per lane group per step):
//   K pass   s_j = (sum over parts of s (q . codes) + z sum(q)) / sqrt(hd) + b_j for
//            j = 0..t, kept in shared memory; the q . codes dot products of 16 columns
//            per step run as warp-level tensor-core MMAs with exact operands (codes as
//            fp16 c * 2^-24, q as scaled hi + lo fp16; attn_mma.cuh);
//   softmax  p_j;
//   select   (when statistics are asked for and t > k) top-k of c_j = p_j ||V^_j||
//            (or p_j) over j = 1..t by a warp radix select on the binary32 bits, equal
//            values to the smaller column; the sink is always kept;
//   V pass   o = sum p V^, and the dropped columns' share u' = sum_{j not kept} p V^;
//            m' = sum_kept p; the kept columns are written ascending.
// Used for loop 1 over an 8-bit base; other cases take the general kernel.
#include <float.h>

#include "attn_mma.cuh"
#include "fl_internal.cuh"
#include "sm100_f32x2.cuh"

namespace fl {
namespace {

__host__ __device__ inline size_t a16(size_t x) { return (x + 15) & ~size_t(15); }

// Per-warp shared memory: p [n_tok] f32 | mark [n_tok] u8 | hist [256] i32.
__host__ __device__ inline size_t dense_warp_smem(int n_tok) {
  return a16((size_t)n_tok * 4) + a16((size_t)n_tok) + 256 * 4;
}

__device__ __forceinline__ void load_sz_pair(const uint16_t* sz, size_t idx, float* s, float* z) {
  const uint32_t pair = reinterpret_cast<const uint32_t*>(sz)[idx];
  *s = half_bits_to_float((uint16_t)(pair & 0xFFFFu));
  *z = half_bits_to_float((uint16_t)(pair >> 16));
}

// 8-bit codes [e0, e0 + EL) of one base row as pairs, and the row's (s, z) for them.
template <int EL>
__device__ __forceinline__ void base_part(const KvView& kv, int which, size_t bh, int e0,
                                          int gidx, int ngrp, float2* c, float* s, float* z) {
  const uint32_t pair = reinterpret_cast<const uint32_t*>(kv.sz[which][1])[bh * ngrp + gidx];
  *s = half_bits_to_float((uint16_t)(pair & 0xFFFFu));
  *z = half_bits_to_float((uint16_t)(pair >> 16));
  f2::load_pairs<EL>(kv.codes[which][1] + bh * (size_t)(EL * 4), 8, e0, c);
}

// One warp's work: query qi, head h; `base` is the warp's shared-memory slice.
template <int HD>
__device__ __forceinline__ void dense_warp(const AttnParams& P, int qi, int h, uint8_t* base) {
  constexpr int EL = HD / 4;
  const int lane = threadIdx.x & 31;
  const int H = P.H, n_tok = P.kv.n_tok, gs = P.kv.g;
  const KvView& kv = P.kv;
  const int l4 = lane & 3, cg = lane >> 2;
  const int e0 = l4 * EL, gidx = e0 / gs, ngrp = HD / gs;

  float* p = reinterpret_cast<float*>(base);
  uint8_t* mark = base + a16((size_t)n_tok * 4);
  int* hist = reinterpret_cast<int*>(mark + a16((size_t)n_tok));

  const int t = P.q_tok[qi];
  const int srow = P.q_row ? P.q_row[qi] : t;
  const bool want_stats = P.sel_out != nullptr;
  if (t < 0 || t >= n_tok || (want_stats && (srow < 0 || srow >= P.stat_rows))) {
    if (lane == 0) record_error(P.st, FL_ERR_RANGE);
    return;
  }
  const int n_cols = t + 1;
  constexpr int KS = HD / 16;
  float qsum = 0.f, dot_unscale;
  uint32_t bq[KS][2];
  {
    float qx[EL];
    const size_t off = ((size_t)qi * H + h) * HD + e0;
#pragma unroll
    for (int k = 0; k < EL / 2; ++k) {
      float a, b;
      if (P.q_bf16) {
        const __nv_bfloat16* qb = reinterpret_cast<const __nv_bfloat16*>(P.q) + off;
        a = __bfloat162float(qb[2 * k]);
        b = __bfloat162float(qb[2 * k + 1]);
      } else {
        const float2 v = reinterpret_cast<const float2*>(reinterpret_cast<const float*>(P.q) + off)[k];
        a = v.x;
        b = v.y;
      }
      qx[2 * k] = a;
      qx[2 * k + 1] = b;
      qsum += a + b;
    }
    dot_unscale = mma::q_fragments<HD>(qx, lane, bq);
  }

  // ---- K pass: 16 columns per step; lane (g, l) loads quarter l of columns i0 + g and
  // i0 + 8 + g (columns past t read column 0 and are masked)
  float lmax = -FLT_MAX;
  for (int i0 = 0; i0 < n_cols; i0 += 16) {
    Raw<EL> raw[2];
    float sb[2], zb[2];
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int col = i0 + 8 * u + cg;
      const uint32_t bh = (uint32_t)(col < n_cols ? col : 0) * H + h;
      load_sz_pair(kv.sz[0][1], (size_t)bh * ngrp + gidx, &sb[u], &zb[u]);
      load_raw<EL>(kv.codes[0][1] + (size_t)bh * HD, 8, e0, raw[u]);
    }
    float d[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int ks = 0; ks < KS; ++ks) {
      const uint32_t w0 = raw_word(raw[0], ks), w1 = raw_word(raw[1], ks);
      mma::m16n8k16(d, mma::code_pair(w0, 0, 1), mma::code_pair(w1, 0, 1),
                    mma::code_pair(w0, 2, 3), mma::code_pair(w1, 2, 3), bq[ks][0], bq[ks][1]);
    }
    float part[2];
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const float dot = (d[2 * u] + d[2 * u + 1]) * dot_unscale;
      part[u] = i0 + 8 * u + cg < n_cols ? fmaf(sb[u], dot, zb[u] * qsum) : 0.f;
    }
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      float v = part[u];
      v += __shfl_xor_sync(0xffffffffu, v, 1);
      v += __shfl_xor_sync(0xffffffffu, v, 2);
      const int c = i0 + 8 * u + cg;
      if (c < n_cols && l4 == 0) {
        const float sc = v * P.scale + (P.bias ? P.bias[c] : 0.f);
        p[c] = sc;
        lmax = fmaxf(lmax, sc);
      }
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) lmax = fmaxf(lmax, __shfl_xor_sync(0xffffffffu, lmax, o));
  __syncwarp();
  float lsum = 0.f;
  for (int c = lane; c < n_cols; c += 32) {
    const float e = expf(p[c] - lmax);
    p[c] = e;
    lsum += e;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) lsum += __shfl_xor_sync(0xffffffffu, lsum, o);
  const float inv = 1.0f / lsum;
  for (int c = lane; c < n_cols; c += 32) p[c] *= inv;
  __syncwarp();

  // ---- statistics: keep the sink and the top-k of c over columns 1..t
  const bool prune = want_stats && (n_cols - 1 > P.k_next);
  if (prune) {
    uint32_t prefix = 0, pmask = 0, need = (uint32_t)P.k_next;
    for (int shift = 24; shift >= 0; shift -= 8) {
      for (int i = lane; i < 256; i += 32) hist[i] = 0;
      __syncwarp();
      for (int c = 1 + lane; c < n_cols; c += 32) {
        float cv = p[c];
        if (P.stat_kind == FL_STAT_PV) cv *= P.vnorm[(size_t)c * H + h];
        const uint32_t b = __float_as_uint(cv);
        if ((b & pmask) == prefix) atomicAdd(&hist[(b >> shift) & 255u], 1);
      }
      __syncwarp();
      uint32_t dg = 0, above = 0;
      if (lane == 0) {
        int d = 255;
        for (; d > 0; --d) {
          if (above + (uint32_t)hist[d] >= need) break;
          above += (uint32_t)hist[d];
        }
        dg = (uint32_t)d;
      }
      dg = __shfl_sync(0xffffffffu, dg, 0);
      above = __shfl_sync(0xffffffffu, above, 0);
      prefix |= dg << shift;
      need -= above;
      pmask |= 255u << shift;
      __syncwarp();
    }
    if (lane == 0) mark[0] = 1;
    int eq_seen = 0;
    for (int b0 = 1; b0 < n_cols; b0 += 32) {
      const int c = b0 + lane;
      const bool valid = c < n_cols;
      uint32_t b = 0;
      if (valid) {
        float cv = p[c];
        if (P.stat_kind == FL_STAT_PV) cv *= P.vnorm[(size_t)c * H + h];
        b = __float_as_uint(cv);
      }
      const bool is_eq = valid && b == prefix;
      const uint32_t bal = __ballot_sync(0xffffffffu, is_eq);
      const int rank = eq_seen + __popc(bal & ((1u << lane) - 1u));
      if (valid) mark[c] = (b > prefix || (is_eq && (uint32_t)rank < need)) ? 1 : 0;
      eq_seen += __popc(bal);
    }
    __syncwarp();
  }

  // ---- V pass
  float2 o[EL / 2], ua[EL / 2];
#pragma unroll
  for (int k = 0; k < EL / 2; ++k) { o[k] = make_float2(0.f, 0.f); ua[k] = make_float2(0.f, 0.f); }
  float oz = 0.f, uz = 0.f;
  for (int i0 = 0; i0 < n_cols; i0 += 16) {
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int c = i0 + 8 * u + cg;
      if (c >= n_cols) continue;
      const float wgt = p[c];
      float2 cf[EL / 2];
      float s, z;
      base_part<EL>(kv, 1, (size_t)c * H + h, e0, gidx, ngrp, cf, &s, &z);
      const float ws = wgt * s;
      f2::axpy_pairs<EL>(ws, cf, o);
      oz = fmaf(wgt, z, oz);
      if (prune && !mark[c]) {
        f2::axpy_pairs<EL>(ws, cf, ua);
        uz = fmaf(wgt, z, uz);
      }
    }
  }
  const float2 oz2 = make_float2(oz, oz), uz2 = make_float2(uz, uz);
#pragma unroll
  for (int k = 0; k < EL / 2; ++k) {
    o[k] = f2::add2(o[k], oz2);
    ua[k] = f2::add2(ua[k], uz2);
#pragma unroll
    for (int off = 4; off < 32; off <<= 1) {
      o[k].x += __shfl_xor_sync(0xffffffffu, o[k].x, off);
      o[k].y += __shfl_xor_sync(0xffffffffu, o[k].y, off);
      ua[k].x += __shfl_xor_sync(0xffffffffu, ua[k].x, off);
      ua[k].y += __shfl_xor_sync(0xffffffffu, ua[k].y, off);
    }
  }
  if (cg == 0) {
    const size_t ob = ((size_t)qi * H + h) * HD + e0;
#pragma unroll
    for (int j = 0; j < EL; ++j) {
      const float ov = (j & 1) ? o[j >> 1].y : o[j >> 1].x;
      if (P.out_bf16) reinterpret_cast<__nv_bfloat16*>(P.out)[ob + j] = __float2bfloat16_rn(ov);
      else reinterpret_cast<float*>(P.out)[ob + j] = ov;
    }
    if (want_stats) {
      float* u_out = P.unsel_out + ((size_t)h * P.stat_rows + srow) * HD + e0;
#pragma unroll
      for (int j = 0; j < EL; ++j) u_out[j] = prune ? ((j & 1) ? ua[j >> 1].y : ua[j >> 1].x) : 0.f;
    }
  }
  if (!want_stats) return;
  __syncwarp();
  uint16_t* so = P.sel_out + ((size_t)h * P.stat_rows + srow) * P.out_stride;
  float lm = 0.f;
  int written = 0;
  for (int b0 = 0; b0 < n_cols; b0 += 32) {
    const int c = b0 + lane;
    const bool keep = c < n_cols && (!prune || mark[c]);
    if (keep) lm += p[c];
    const uint32_t bal = __ballot_sync(0xffffffffu, keep);
    const int pos = written + __popc(bal & ((1u << lane) - 1u));
    if (keep && pos < P.out_stride) so[pos] = (uint16_t)c;
    written += __popc(bal);
  }
  for (int i = written + lane; i < P.out_stride; i += 32) so[i] = (uint16_t)FL_SENTINEL;
#pragma unroll
  for (int o2 = 16; o2 > 0; o2 >>= 1) lm += __shfl_xor_sync(0xffffffffu, lm, o2);
  if (lane == 0) P.mass_out[(size_t)h * P.stat_rows + srow] = lm;
}

template <int HD>
__global__ void __launch_bounds__(128) k_attn_dense(const __grid_constant__ AttnParams P) {
  extern __shared__ __align__(16) uint8_t smem[];
  const int nw = blockDim.x >> 5;
  const int w = threadIdx.x >> 5;
  const int gw = blockIdx.x * nw + w;
  if (gw >= P.n_q * P.H) return;  // whole warp leaves; no CTA-wide barrier below
  dense_warp<HD>(P, gw / P.H, gw % P.H, smem + (size_t)w * dense_warp_smem(P.kv.n_tok));
}

// The (query, head) pairs list[0, *count) (entries h * n_q + query), warps striding over
// the list: the exact finish of rows the tensor-core producer could not rank.
template <int HD>
__global__ void __launch_bounds__(128) k_attn_dense_list(const __grid_constant__ AttnParams P,
                                                         const int* list, const int* count) {
  extern __shared__ __align__(16) uint8_t smem[];
  const int nw = blockDim.x >> 5;
  const int w = threadIdx.x >> 5;
  const int n = *count;
  for (int x = blockIdx.x * nw + w; x < n; x += gridDim.x * nw) {
    const int rh = list[x];
    dense_warp<HD>(P, rh % P.n_q, rh / P.n_q, smem + (size_t)w * dense_warp_smem(P.kv.n_tok));
  }
}

}  // namespace

// The warp-per-query kernel reads the 8-bit base alone: loop 1 of a quantised store.
bool dense_rows_supported(const AttnParams& P) {
  return P.hd == 128 && P.loop == 1 && P.kv.base_bits == 8 &&
         dense_warp_smem(P.kv.n_tok) <= 200 * 1024;
}

cudaError_t launch_attn_dense_rows(const AttnParams& P, const int* list, const int* count,
                                   cudaStream_t s) {
  const size_t per = dense_warp_smem(P.kv.n_tok);
  int nw = (int)((200 * 1024) / per);
  nw = nw < 1 ? 1 : (nw > 4 ? 4 : nw);
  const size_t sm = (size_t)nw * per;
  static int attr_bytes[128] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 128) return cudaErrorInvalidDevice;
  if ((int)sm > attr_bytes[dev]) {
    cudaError_t e = cudaFuncSetAttribute(k_attn_dense_list<128>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
    if (e != cudaSuccess) return e;
    attr_bytes[dev] = (int)sm;
  }
  int sms = 148;
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  k_attn_dense_list<128><<<sms, nw * 32, sm, s>>>(P, list, count);
  count_launch();
  return cudaGetLastError();
}

bool dense_fast_eligible(const AttnParams& P) {
  if (P.sel != nullptr || P.loop != 1) return false;
  if (P.hd != 128 && P.hd != 64) return false;
  if (P.kv.base_bits != 8 || (P.kv.g != 32 && P.kv.g != 64)) return false;
  if (P.sel_out && P.stat_kind == FL_STAT_PV && !P.vnorm) return false;
  return dense_warp_smem(P.kv.n_tok) <= 200 * 1024;
}

cudaError_t launch_attn_dense_fast(const AttnParams& P, cudaStream_t s) {
  const size_t per = dense_warp_smem(P.kv.n_tok);
  int nw = (int)((200 * 1024) / per);
  nw = nw < 1 ? 1 : (nw > 4 ? 4 : nw);
  const size_t sm = (size_t)nw * per;
  const int warps = P.n_q * P.H;
  const int blocks = (warps + nw - 1) / nw;
  auto kern = P.hd == 128 ? k_attn_dense<128> : k_attn_dense<64>;
  static int attr_bytes[2][128] = {{0}};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 128) return cudaErrorInvalidDevice;
  int& have = attr_bytes[P.hd == 128 ? 1 : 0][dev];
  if ((int)sm > have) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
    if (e != cudaSuccess) return e;
    have = (int)sm;
  }
  kern<<<blocks, nw * 32, sm, s>>>(P);
  count_launch();
  return cudaGetLastError();
}

}  // namespace fl
