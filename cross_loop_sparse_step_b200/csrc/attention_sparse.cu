// Loop-aware sparse attention over carried column sets, one warp per (query, head)
// (FlashLoop §4.2 "Loop-Aware Sparse Attention": softmax over the selected logits only,
// rescaled by the cached global mass, plus the carried unselected contribution; the
// K/V of the selected columns are gathered, here straight from the quantised store).
//
// Used when the store is quantised throughout (int8 base, 2/4/8-bit residuals).
//   Four lanes per column, eight columns in flight per warp; each lane owns a quarter
//   of the head slice (one quantisation group at head_dim 128) and keeps its part of q
//   in registers.
//   K pass: every stored row of the column's chain (base, then each loop that rewrote
//     it) contributes s * (q . codes) + z * sum(q) - dequantisation folded into the dot;
//     codes are decoded in pairs and the dots use packed binary32 pair FMAs.
//   softmax over the column set, p~ = m * softmax (m = cached mass).
//   optional budget shrink: warp radix select over the binary32 bits of p~ * ||V^||
//     (ties to the smaller column), ballot-ordered so the kept set stays ascending.
//   V pass: o += (p~ s) codes + p~ z over the chain's rows, and for dropped columns the
//     same into the next loop's u'; the eight column groups are reduced by shuffles.
#include <float.h>

#include "fl_internal.cuh"
#include "sm100_f32x2.cuh"

namespace fl {
namespace {

constexpr int NW = 4;  // warps per CTA

__host__ __device__ inline size_t align16(size_t x) { return (x + 15) & ~size_t(15); }

// Per-warp shared memory: (reserved) [HD + 4] f32 | p [stride] f32 | cols [stride] u16 |
// mark [stride] u8 | hist [256] i32 | list_idx [stride] u16 | list_row [stride] i32.
__host__ __device__ inline size_t warp_smem(int hd, int stride) {
  return align16((size_t)hd * 4 + 16) + align16((size_t)stride * 4) + align16((size_t)stride * 2) +
         align16((size_t)stride) + 256 * 4 + align16((size_t)stride * 2) + align16((size_t)stride * 4);
}

__device__ __forceinline__ void load_sz(const uint16_t* sz, size_t idx, float* s, float* z) {
  const uint32_t pair = reinterpret_cast<const uint32_t*>(sz)[idx];
  *s = half_bits_to_float((uint16_t)(pair & 0xFFFFu));
  *z = half_bits_to_float((uint16_t)(pair >> 16));
}

// Four lanes per column: lane part l4 = lane % 4 owns elements [l4 * EL, (l4 + 1) * EL) of
// the head slice, EL = HD / 4 (32 at HD 128), which lie in one quantisation group.
// SHRINK: the call may shrink the budget (k_next below the carried set size), so the
// dropped columns' contribution is accumulated too.
// One warp's work: (query, head) number gw of the call described by P, with `base` the
// warp's shared-memory slice. No CTA-wide barrier is used.
template <int HD, bool SHRINK>
__device__ __forceinline__ void attn_sparse_warp(const AttnParams& P, int gw, uint8_t* base) {
  constexpr int EL = HD / 4;
  const int lane = threadIdx.x & 31;
  const int qi = gw / P.H, h = gw % P.H;
  const int H = P.H, n_tok = P.kv.n_tok, gs = P.kv.g, stride = P.sel_stride;
  const KvView& kv = P.kv;
  const int l4 = lane & 3, cg = lane >> 2;   // part of the column, column group (0..7)
  const int e0 = l4 * EL;
  const int gidx = e0 / gs;                  // quantisation group of this lane's part
  const int ngrp = HD / gs;

  float* p = reinterpret_cast<float*>(base + align16((size_t)HD * 4 + 16));
  uint16_t* cols = reinterpret_cast<uint16_t*>(reinterpret_cast<uint8_t*>(p) + align16((size_t)stride * 4));
  uint8_t* mark = reinterpret_cast<uint8_t*>(cols) + align16((size_t)stride * 2);
  int* hist = reinterpret_cast<int*>(mark + align16((size_t)stride));

  const int t = P.q_tok[qi];
  const int srow = P.q_row ? P.q_row[qi] : t;
  if (t < 0 || t >= n_tok || srow < 0 || srow >= P.stat_rows) {
    if (lane == 0) record_error(P.st, FL_ERR_RANGE);
    return;
  }
  // statistics for the next loop; nothing to write when they are updated in place and
  // the budget does not shrink (S' = S, m' = m, u' = u)
  const bool want_stats = P.sel_out != nullptr &&
      !(P.sel_out == P.sel && P.mass_out == P.mass && P.unsel_out == P.unsel &&
        P.out_stride == P.sel_stride && P.k_next + 1 >= P.sel_stride);

  // ---- carried column set, cached mass, this lane's part of the query
  const uint16_t* srow_p = P.sel + ((size_t)h * P.stat_rows + srow) * stride;
  int n_cols = 0;
  for (int i0 = 0; i0 < stride; i0 += 32) {
    const int i = i0 + lane;
    const uint16_t c = i < stride ? srow_p[i] : (uint16_t)FL_SENTINEL;
    if (i < stride) cols[i] = c;
    n_cols += __popc(__ballot_sync(0xffffffffu, c != FL_SENTINEL));
  }
  const float m_in = P.mass[(size_t)h * P.stat_rows + srow];
  float2 qv[EL / 2];
  float qsum = 0.f;
  {
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
      qv[k] = make_float2(a, b);
      qsum += a + b;
    }
  }
  __syncwarp();

  // Work is split so every lane stays busy: a base pass over all columns, then one pass
  // per loop r = 2..loop over the compacted list of columns that loop rewrote.
  uint16_t* list_idx = reinterpret_cast<uint16_t*>(reinterpret_cast<uint8_t*>(hist) + 256 * 4);
  int32_t* list_row = reinterpret_cast<int32_t*>(reinterpret_cast<uint8_t*>(list_idx) + align16((size_t)stride * 2));
  // compacts {idx : slot[r][cols[idx]] >= 0} into list_idx / list_row; returns its length
  auto build_list = [&](int r) -> int {
    int n = 0;
    const int32_t* srow_r = kv.slot + (size_t)r * n_tok;
    for (int b0 = 0; b0 < n_cols; b0 += 32) {
      const int idx = b0 + lane;
      int row = -1;
      if (idx < n_cols) {
        const int c = cols[idx];
        if (c <= t && c < n_tok) row = srow_r[c];
      }
      const uint32_t bal = __ballot_sync(0xffffffffu, row >= 0);
      if (row >= 0) {
        const int pos = n + __popc(bal & ((1u << lane) - 1u));
        list_idx[pos] = (uint16_t)idx;
        list_row[pos] = row;
      }
      n += __popc(bal);
    }
    __syncwarp();
    return n;
  };

  // ---- K base pass: 8 columns in flight, score part = s (q . codes) + z sum(q)
  for (int i0 = 0; i0 < n_cols; i0 += 8) {
    const int idx = i0 + cg;
    float part = 0.f;
    int c = -1;
    bool valid = idx < n_cols;
    if (valid) {
      c = cols[idx];
      valid = c <= t && c < n_tok;
    }
    float bias_c = 0.f;
    if (valid) {
      if (P.bias && l4 == 0) bias_c = P.bias[c];
      const size_t bh = (size_t)c * H + h;
      float2 cf[EL / 2];
      float sb, zb;
      load_sz(kv.sz[0][1], bh * ngrp + gidx, &sb, &zb);
      f2::load_pairs<EL>(kv.codes[0][1] + bh * HD, 8, e0, cf);
      const float d = f2::dot_pairs<EL>(qv, cf);
      part = fmaf(sb, d, zb * qsum);
    }
    part += __shfl_xor_sync(0xffffffffu, part, 1);
    part += __shfl_xor_sync(0xffffffffu, part, 2);
    if (idx < n_cols && l4 == 0) {
      if (!valid) {
        record_error(P.st, FL_ERR_RANGE);
        p[idx] = -INFINITY;
      } else {
        p[idx] = part * P.scale + bias_c;
      }
    }
  }
  __syncwarp();
  // ---- K residual passes
  for (int r = 2; r <= P.loop; ++r) {
    const int n_r = build_list(r);
    const int b = kv.res_bits[r];
    const float sc = P.scale;
    for (int i0 = 0; i0 < n_r; i0 += 8) {
      const int li = i0 + cg;
      float part = 0.f;
      if (li < n_r) {
        const size_t rh = (size_t)list_row[li] * H + h;
        float2 cf[EL / 2];
        float sr, zr;
        load_sz(kv.sz[0][r], rh * ngrp + gidx, &sr, &zr);
        f2::load_pairs<EL>(kv.codes[0][r] + rh * (HD * b / 8), b, e0, cf);
        const float d = f2::dot_pairs<EL>(qv, cf);
        part = fmaf(sr, d, zr * qsum);
      }
      part += __shfl_xor_sync(0xffffffffu, part, 1);
      part += __shfl_xor_sync(0xffffffffu, part, 2);
      if (li < n_r && l4 == 0) p[list_idx[li]] += part * sc;
    }
    __syncwarp();
  }
  float lmax = -FLT_MAX;
  for (int idx = lane; idx < n_cols; idx += 32) lmax = fmaxf(lmax, p[idx]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) lmax = fmaxf(lmax, __shfl_xor_sync(0xffffffffu, lmax, o));
  __syncwarp();
  float lsum = 0.f;
  for (int idx = lane; idx < n_cols; idx += 32) {
    const float e = expf(p[idx] - lmax);
    p[idx] = e;
    lsum += e;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) lsum += __shfl_xor_sync(0xffffffffu, lsum, o);
  const float wmul = m_in / lsum;
  for (int idx = lane; idx < n_cols; idx += 32) p[idx] *= wmul;
  __syncwarp();

  // ---- budget shrink: keep the sink and the top-k_next columns by p~ * ||V^||
  const bool prune = SHRINK && want_stats && (n_cols - 1 > P.k_next);
  if (prune) {
    uint32_t prefix = 0, pmask = 0, need = (uint32_t)P.k_next;
    for (int shift = 24; shift >= 0; shift -= 8) {
      for (int i = lane; i < 256; i += 32) hist[i] = 0;
      __syncwarp();
      for (int idx = 1 + lane; idx < n_cols; idx += 32) {
        const int c = cols[idx];
        float cv = c <= t ? p[idx] : 0.f;
        if (P.stat_kind == FL_STAT_PV && c <= t) cv *= P.vnorm[(size_t)c * H + h];
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
      const int idx = b0 + lane;
      const bool valid = idx < n_cols;
      uint32_t b = 0;
      if (valid) {
        const int c = cols[idx];
        float cv = c <= t ? p[idx] : 0.f;
        if (P.stat_kind == FL_STAT_PV && c <= t) cv *= P.vnorm[(size_t)c * H + h];
        b = __float_as_uint(cv);
      }
      const bool is_eq = valid && b == prefix;
      const uint32_t bal = __ballot_sync(0xffffffffu, is_eq);
      const int rank = eq_seen + __popc(bal & ((1u << lane) - 1u));
      if (valid) mark[idx] = (b > prefix || (is_eq && (uint32_t)rank < need)) ? 1 : 0;
      eq_seen += __popc(bal);
    }
    __syncwarp();
  }

  // ---- V passes: o part += (w s) codes + w z for every stored row of the chain
  float2 o[EL / 2], ua[EL / 2];
#pragma unroll
  for (int k = 0; k < EL / 2; ++k) { o[k] = make_float2(0.f, 0.f); ua[k] = make_float2(0.f, 0.f); }
  float oz = 0.f, uz = 0.f;   // the offsets' share, added to every element at the end
  for (int i0 = 0; i0 < n_cols; i0 += 8) {
    const int idx = i0 + cg;
    if (idx >= n_cols) continue;
    const int c = cols[idx];
    if (c > t || c >= n_tok) continue;
    const float wgt = p[idx];
    const size_t bh = (size_t)c * H + h;
    float2 cf[EL / 2];
    float s, z;
    load_sz(kv.sz[1][1], bh * ngrp + gidx, &s, &z);
    f2::load_pairs<EL>(kv.codes[1][1] + bh * HD, 8, e0, cf);
    const float ws = wgt * s;
    f2::axpy_pairs<EL>(ws, cf, o);
    oz = fmaf(wgt, z, oz);
    if (SHRINK && prune && !mark[idx]) {
      f2::axpy_pairs<EL>(ws, cf, ua);
      uz = fmaf(wgt, z, uz);
    }
  }
  for (int r = 2; r <= P.loop; ++r) {
    const int n_r = build_list(r);
    const int b = kv.res_bits[r];
    for (int i0 = 0; i0 < n_r; i0 += 8) {
      const int li = i0 + cg;
      if (li >= n_r) continue;
      const int idx = list_idx[li];
      const float wgt = p[idx];
      const size_t rh = (size_t)list_row[li] * H + h;
      float2 cf[EL / 2];
      float s, z;
      load_sz(kv.sz[1][r], rh * ngrp + gidx, &s, &z);
      f2::load_pairs<EL>(kv.codes[1][r] + rh * (HD * b / 8), b, e0, cf);
      const float ws = wgt * s;
      f2::axpy_pairs<EL>(ws, cf, o);
      oz = fmaf(wgt, z, oz);
      if (SHRINK && prune && !mark[idx]) {
        f2::axpy_pairs<EL>(ws, cf, ua);
        uz = fmaf(wgt, z, uz);
      }
    }
  }
  // reduce the 8 column groups (lanes with the same part differ in bits 2..4)
  const float2 oz2 = make_float2(oz, oz), uz2 = make_float2(uz, uz);
#pragma unroll
  for (int k = 0; k < EL / 2; ++k) {
    o[k] = f2::add2(o[k], oz2);
#pragma unroll
    for (int off = 4; off < 32; off <<= 1) {
      o[k].x += __shfl_xor_sync(0xffffffffu, o[k].x, off);
      o[k].y += __shfl_xor_sync(0xffffffffu, o[k].y, off);
    }
    if (SHRINK) {
      ua[k] = f2::add2(ua[k], uz2);
#pragma unroll
      for (int off = 4; off < 32; off <<= 1) {
        ua[k].x += __shfl_xor_sync(0xffffffffu, ua[k].x, off);
        ua[k].y += __shfl_xor_sync(0xffffffffu, ua[k].y, off);
      }
    }
  }

  // ---- outputs (lanes 0..3 hold the four parts)
  if (cg == 0) {
    const float* u_in = P.unsel + ((size_t)h * P.stat_rows + srow) * HD + e0;
    const size_t ob = ((size_t)qi * H + h) * HD + e0;
    float* u_out = want_stats ? P.unsel_out + ((size_t)h * P.stat_rows + srow) * HD + e0 : nullptr;
#pragma unroll
    for (int j = 0; j < EL; ++j) {
      const float ui = u_in[j];
      const float val = ui + ((j & 1) ? o[j >> 1].y : o[j >> 1].x);
      if (P.out_bf16) reinterpret_cast<__nv_bfloat16*>(P.out)[ob + j] = __float2bfloat16_rn(val);
      else reinterpret_cast<float*>(P.out)[ob + j] = val;
      if (want_stats) u_out[j] = prune ? ui + ((j & 1) ? ua[j >> 1].y : ua[j >> 1].x) : ui;
    }
  }
  if (!want_stats) return;
  __syncwarp();
  uint16_t* so = P.sel_out + ((size_t)h * P.stat_rows + srow) * P.out_stride;
  float lm = 0.f;
  int written = 0;
  for (int b0 = 0; b0 < n_cols; b0 += 32) {
    const int idx = b0 + lane;
    const bool keep = idx < n_cols && (!prune || mark[idx]);
    if (keep && prune) lm += p[idx];
    const uint32_t bal = __ballot_sync(0xffffffffu, keep);
    const int pos = written + __popc(bal & ((1u << lane) - 1u));
    if (keep && pos < P.out_stride) so[pos] = cols[idx];
    written += __popc(bal);
  }
  for (int i = written + lane; i < P.out_stride; i += 32) so[i] = (uint16_t)FL_SENTINEL;
#pragma unroll
  for (int o2 = 16; o2 > 0; o2 >>= 1) lm += __shfl_xor_sync(0xffffffffu, lm, o2);
  if (lane == 0) P.mass_out[(size_t)h * P.stat_rows + srow] = prune ? lm : m_in;
}

template <int HD, bool SHRINK>
__global__ void __launch_bounds__(NW * 32) k_attn_sparse(const __grid_constant__ AttnParams P) {
  extern __shared__ __align__(16) uint8_t smem[];
  const int w = threadIdx.x >> 5;
  const int gw = blockIdx.x * NW + w;
  if (gw >= P.n_q * P.H) return;  // whole warp leaves
  attn_sparse_warp<HD, SHRINK>(P, gw, smem + (size_t)w * warp_smem(HD, P.sel_stride));
}

// Many independent calls in one launch (batched decode: one store per sequence). The
// calls share n_q, heads, head_dim and carried-set stride; `per` = n_q * H warps each.
template <int HD, bool SHRINK>
__global__ void __launch_bounds__(NW * 32)
    k_attn_sparse_batched(const AttnParams* __restrict__ Ps, int n_calls, int per, int stride) {
  extern __shared__ __align__(16) uint8_t smem[];
  const int w = threadIdx.x >> 5;
  const int gw = blockIdx.x * NW + w;
  if (gw >= n_calls * per) return;
  attn_sparse_warp<HD, SHRINK>(Ps[gw / per], gw % per, smem + (size_t)w * warp_smem(HD, stride));
}

}  // namespace

bool sparse_fast_eligible(const AttnParams& P) {
  if (P.hd != 128 && P.hd != 64) return false;
  if (P.kv.base_bits != 8 || (P.kv.g != 32 && P.kv.g != 64)) return false;
  for (int r = 2; r <= P.loop; ++r) {
    const int b = P.kv.res_bits[r];
    if (b != 2 && b != 4 && b != 8) return false;
  }
  if (P.sel_stride < 1 || P.sel_stride > 4096) return false;
  if (P.sel_out && P.stat_kind == FL_STAT_PV && !P.vnorm) return false;
  return (size_t)NW * warp_smem(P.hd, P.sel_stride) <= 200 * 1024;
}

cudaError_t launch_attn_sparse_fast(const AttnParams& P, cudaStream_t s) {
  const size_t sm = (size_t)NW * warp_smem(P.hd, P.sel_stride);
  const int warps = P.n_q * P.H;
  const int blocks = (warps + NW - 1) / NW;
  const bool shrink = P.sel_out != nullptr && P.k_next + 1 < P.sel_stride;
  auto kern = P.hd == 128 ? (shrink ? k_attn_sparse<128, true> : k_attn_sparse<128, false>)
                          : (shrink ? k_attn_sparse<64, true> : k_attn_sparse<64, false>);
  static int attr_bytes[4][128] = {{0}};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 128) return cudaErrorInvalidDevice;
  int& have = attr_bytes[(P.hd == 128 ? 2 : 0) + (shrink ? 1 : 0)][dev];
  if ((int)sm > have) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
    if (e != cudaSuccess) return e;
    have = (int)sm;
  }
  kern<<<blocks, NW * 32, sm, s>>>(P);
  count_launch();
  return cudaGetLastError();
}

// Ps: device array of n AttnParams (already copied by the caller, same shapes).
cudaError_t launch_attn_sparse_batched(const AttnParams& P0, const AttnParams* Ps_dev, int n,
                                       cudaStream_t s) {
  const size_t sm = (size_t)NW * warp_smem(P0.hd, P0.sel_stride);
  const int per = P0.n_q * P0.H;
  const long long warps = (long long)per * n;
  const int blocks = (int)((warps + NW - 1) / NW);
  const bool shrink = P0.sel_out != nullptr && P0.k_next + 1 < P0.sel_stride;
  auto kern = P0.hd == 128 ? (shrink ? k_attn_sparse_batched<128, true> : k_attn_sparse_batched<128, false>)
                           : (shrink ? k_attn_sparse_batched<64, true> : k_attn_sparse_batched<64, false>);
  static int attr_bytes[4][128] = {{0}};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 128) return cudaErrorInvalidDevice;
  int& have = attr_bytes[(P0.hd == 128 ? 2 : 0) + (shrink ? 1 : 0)][dev];
  if ((int)sm > have) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
    if (e != cudaSuccess) return e;
    have = (int)sm;
  }
  kern<<<blocks, NW * 32, sm, s>>>(Ps_dev, n, per, P0.sel_stride);
  count_launch();
  return cudaGetLastError();
}

}  // namespace fl
