// Loop-aware sparse attention over carried column sets, one warp per (query, head)
// (FlashLoop §4.2 "Loop-Aware Sparse Attention": softmax over the selected logits only,
// rescaled by the cached global mass, plus the carried unselected contribution; the
// K/V of the selected columns are gathered, here straight from the quantised store).
//
// Used when the store is quantised throughout (int8 base, 2/4/8-bit residuals).
//   The products run on the tensor cores (warp-level m16n8k16 MMAs, binary32
//   accumulation) with exact operands: codes as the fp16 values c * 2^-24, and q and the
//   softmax weights as hi + lo fp16 pairs after a power-of-two scaling (22 significant
//   bits; see attn_mma.cuh). Dequantisation stays folded: a stored row contributes
//   s * (q . codes) + z * sum(q) to a logit and (p~ s) codes + p~ z to the output.
//   Every pass takes sixteen stored rows per warp iteration, their loads issued before
//   any is used, so each iteration waits for one round of L2 latency.
//   Residual work lists: for the loops that rewrote some carried columns, the (column,
//   loop, row) items are compacted once per loop chunk - slot lookups of several loops
//   issued together - and the K and V passes walk them as one stream, so no lane idles
//   on a column that a loop did not touch.
//   K pass (rows = 16 stored rows, k = head elements, n = hi/lo of each quarter of q):
//     lane (g, l) holds quarter l of rows g and g + 8 and gets back its quarter's dot
//     for both; the scale/offset of the quarter's group are applied and the quarters
//     summed by shuffles. Residual parts are added to the logits loop by loop.
//   softmax over the column set, p~ = m * softmax (m = cached mass).
//   optional budget shrink: warp radix select over the binary32 bits of p~ * ||V^||
//     (ties to the smaller column), ballot-ordered so the kept set stays ascending.
//   V pass (binary32 pairs: the weights vary per stored row, so the sums are axpys):
//     o += (p~ s) codes + p~ z over the chain's rows, and for dropped columns the same
//     into the next loop's u'; lane (g, l) works on quarter l of rows g and g + 8 and the
//     eight row groups are reduced by shuffles.
//   A chunk of residual loops holds loops of one bit width, so each residual pass runs
//   with the width as a compile-time constant and decodes in straight-line code.
#include <float.h>

#include "fl_internal.cuh"
#include "attn_mma.cuh"
#include "sm100_f32x2.cuh"

namespace fl {
namespace {

constexpr int NW = 4;              // warps per CTA
// resident CTAs per SM the register budget is cut for (no spills at either setting)
__host__ __device__ constexpr int min_ctas(bool shrink) { return shrink ? 3 : 6; }
constexpr int ITEM_BYTES = 11;     // u16 column index + u8 loop + i32 row + f32 logit part
constexpr int ITEM_BUDGET = 6144;  // per-warp bytes for residual items beyond one loop's

__host__ __device__ inline size_t align16(size_t x) { return (x + 15) & ~size_t(15); }

// Residual loops whose item lists are held at once (each loop's list needs up to `stride`
// items); at least one.
__host__ __device__ inline int chunk_loops(int loop, int stride) {
  if (loop < 2) return 1;
  int cl = ITEM_BUDGET / (stride * ITEM_BYTES);
  if (cl < 1) cl = 1;
  return cl < loop - 1 ? cl : loop - 1;
}

// Per-warp shared memory: p [stride] f32 | cols [stride] u16 | mark [stride] u8 |
// hist [256] i32 | loff [FL_MAX_LOOPS + 1] i32 | items: it_part [cap] f32 | it_row [cap]
// i32 | it_idx [cap] u16 | it_loop [cap] u8, cap = chunk_loops * stride.
__host__ __device__ inline size_t warp_smem(int stride, int loop) {
  const size_t cap = (size_t)chunk_loops(loop, stride) * stride;
  return align16((size_t)stride * 4) + align16((size_t)stride * 2) + align16((size_t)stride) +
         256 * 4 + align16((FL_MAX_LOOPS + 1) * 4) + 2 * align16(cap * 4) + align16(cap * 2) +
         align16(cap);
}

__device__ __forceinline__ void load_sz(const uint16_t* sz, size_t idx, float* s, float* z) {
  const uint32_t pair = reinterpret_cast<const uint32_t*>(sz)[idx];
  *s = half_bits_to_float((uint16_t)(pair & 0xFFFFu));
  *z = half_bits_to_float((uint16_t)(pair >> 16));
}

// o[j] += w * code[j]
template <int EL>
__device__ __forceinline__ void axpy_raw(float w, const Raw<EL>& r, int bits, float2* o) {
  const float2 ww = make_float2(w, w);
  float2 c[8];
  if (bits == 8) {
#pragma unroll
    for (int i = 0; i < EL / 4; ++i) {
      f2::dec8(raw_word(r, i), c);
      o[2 * i] = f2::fma2(ww, c[0], o[2 * i]);
      o[2 * i + 1] = f2::fma2(ww, c[1], o[2 * i + 1]);
    }
  } else if (bits == 4) {
#pragma unroll
    for (int i = 0; i < EL / 8; ++i) {
      f2::dec4(raw_word(r, i), c);
#pragma unroll
      for (int k = 0; k < 4; ++k) o[4 * i + k] = f2::fma2(ww, c[k], o[4 * i + k]);
    }
  } else {
#pragma unroll
    for (int i = 0; i < EL / 16; ++i) {
      f2::dec2(raw_word(r, i), c);
#pragma unroll
      for (int k = 0; k < 8; ++k) o[8 * i + k] = f2::fma2(ww, c[k], o[8 * i + k]);
    }
  }
}

// A bit width as a type.
template <int B>
struct Width {
  static constexpr int value = B;
};

// One warp's work: (query, head) number gw of the call described by P, with `base` the
// warp's shared-memory slice. No CTA-wide barrier is used.
// Lane part l4 = lane % 4 owns elements [l4 * EL, (l4 + 1) * EL) of the head slice,
// EL = HD / 4, which lie in one quantisation group; lane group cg = lane / 4 (0..7).
// SHRINK: the call may shrink the budget (k_next below the carried set size), so the
// dropped columns' contribution is accumulated too.
template <int HD, bool SHRINK>
__device__ __forceinline__ void attn_sparse_warp(const AttnParams& P, int gw, uint8_t* base) {
  constexpr int EL = HD / 4;
  const int lane = threadIdx.x & 31;
  const int qi = gw / P.H, h = gw % P.H;
  const int H = P.H, n_tok = P.kv.n_tok, gs = P.kv.g, stride = P.sel_stride;
  const KvView& kv = P.kv;
  const int l4 = lane & 3, cg = lane >> 2;
  const int e0 = l4 * EL;
  const int gidx = e0 / gs;                  // quantisation group of this lane's part
  const int ngrp = HD / gs;
  const int loop = P.loop;
  const int CL = chunk_loops(loop, stride);
  const int cap = CL * stride;
  float dot_unscale = 1.f;

  float* p = reinterpret_cast<float*>(base);
  uint16_t* cols = reinterpret_cast<uint16_t*>(base + align16((size_t)stride * 4));
  uint8_t* mark = reinterpret_cast<uint8_t*>(cols) + align16((size_t)stride * 2);
  int* hist = reinterpret_cast<int*>(mark + align16((size_t)stride));
  int* loff = hist + 256;
  float* it_part = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(loff) + align16((FL_MAX_LOOPS + 1) * 4));
  int32_t* it_row = reinterpret_cast<int32_t*>(reinterpret_cast<uint8_t*>(it_part) + align16((size_t)cap * 4));
  uint16_t* it_idx = reinterpret_cast<uint16_t*>(reinterpret_cast<uint8_t*>(it_row) + align16((size_t)cap * 4));
  uint8_t* it_loop = reinterpret_cast<uint8_t*>(it_idx) + align16((size_t)cap * 2);

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
  // this lane's quarter of q, and the score MMAs' B fragments made from it
  constexpr int KS = HD / 16;
  float qsum = 0.f;
  uint32_t bq[KS][2];
  {
    float qx[EL];
    const size_t off = ((size_t)qi * H + h) * HD + e0;
#pragma unroll
    for (int k = 0; k < EL / 2; ++k) {
      float a, b;
      if (P.q_bf16) {
        const __nv_bfloat162 v = reinterpret_cast<const __nv_bfloat162*>(
            reinterpret_cast<const __nv_bfloat16*>(P.q) + off)[k];
        a = __low2float(v);
        b = __high2float(v);
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
  __syncwarp();

  // Residual items of loops [r0, r1): (column index, loop, row) for every carried column
  // that loop rewrote, compacted loop after loop into it_*; loff[k] = first item of loop
  // r0 + k. Each loop's items are first written to a region of `stride` entries (its
  // count held by lane r - r0), the slot lookups of four loops issued together.
  auto build_items = [&](int r0, int r1) -> int {
    int cnt = 0;   // lane k: items of loop r0 + k so far
    for (int b0 = 0; b0 < n_cols; b0 += 32) {
      const int idx = b0 + lane;
      int c = -1;
      if (idx < n_cols) {
        c = cols[idx];
        if (c > t || c >= n_tok) c = -1;
      }
      for (int ra = r0; ra < r1; ra += 4) {
        int row[4];
#pragma unroll
        for (int u = 0; u < 4; ++u)
          row[u] = (c >= 0 && ra + u < r1) ? kv.slot[(size_t)(ra + u) * n_tok + c] : -1;
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int k = ra + u - r0;
          if (ra + u >= r1) break;
          const uint32_t bal = __ballot_sync(0xffffffffu, row[u] >= 0);
          const int have = __shfl_sync(0xffffffffu, cnt, k);
          if (row[u] >= 0) {
            const int pos = k * stride + have + __popc(bal & ((1u << lane) - 1u));
            it_idx[pos] = (uint16_t)idx;
            it_row[pos] = row[u];
          }
          if (lane == k) cnt += __popc(bal);
        }
      }
    }
    // exclusive prefix of the counts over lanes 0..r1-r0-1
    const int nl = r1 - r0;
    int incl = lane < nl ? cnt : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += v;
    }
    const int excl = incl - (lane < nl ? cnt : 0);
    const int total = __shfl_sync(0xffffffffu, incl, 31);
    if (lane <= nl) loff[lane] = lane < nl ? excl : total;
    __syncwarp();
    // move region k down to loff[k] (destinations never pass their sources)
    for (int k = 0; k < nl; ++k) {
      const int n_k = __shfl_sync(0xffffffffu, cnt, k);
      const int dst0 = __shfl_sync(0xffffffffu, excl, k);
      for (int j0 = 0; j0 < n_k; j0 += 32) {
        const int j = j0 + lane;
        uint16_t ix = 0;
        int32_t rw = 0;
        if (j < n_k) { ix = it_idx[k * stride + j]; rw = it_row[k * stride + j]; }
        __syncwarp();
        if (j < n_k) {
          it_idx[dst0 + j] = ix;
          it_row[dst0 + j] = rw;
          it_loop[dst0 + j] = (uint8_t)(r0 + k);
        }
        __syncwarp();
      }
    }
    return total;
  };
  // a chunk: up to CL consecutive residual loops of one bit width
  auto chunk_end = [&](int r0) -> int {
    const int r1 = min(loop + 1, r0 + CL);
    for (int r = r0 + 1; r < r1; ++r)
      if (kv.res_bits[r] != kv.res_bits[r0]) return r;
    return r1;
  };
  const bool one_chunk = loop < 2 || chunk_end(2) == loop + 1;
  int n_items = 0;   // items of the current chunk (all residual loops when one_chunk)

  // ---- K base pass: 16 columns per iteration; lane (g, l) loads quarter l of columns
  // i0 + g and i0 + 8 + g
  for (int i0 = 0; i0 < n_cols; i0 += 16) {
    Raw<EL> raw[2];
    float sb[2], zb[2], bias_c[2];
    int idx[2];
    bool valid[2];
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      // rows past the set or outside [0, t] read column 0 (always stored) and are masked
      idx[u] = i0 + 8 * u + cg;
      const int ci = idx[u] < n_cols ? (int)cols[idx[u]] : 0;
      valid[u] = idx[u] < n_cols && ci <= t && ci < n_tok;
      const int c = valid[u] ? ci : 0;
      bias_c[u] = (P.bias && l4 == 0) ? P.bias[c] : 0.f;
      const uint32_t bh = (uint32_t)c * H + h;
      load_sz(kv.sz[0][1], (size_t)bh * ngrp + gidx, &sb[u], &zb[u]);
      load_raw<EL>(kv.codes[0][1] + (size_t)bh * HD, 8, e0, raw[u]);
    }
    float d[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int ks = 0; ks < KS; ++ks) {
      const uint32_t w0 = raw_word(raw[0], ks), w1 = raw_word(raw[1], ks);
      mma::m16n8k16(d, mma::code_pair(w0, 0, 1), mma::code_pair(w1, 0, 1),
                    mma::code_pair(w0, 2, 3), mma::code_pair(w1, 2, 3), bq[ks][0], bq[ks][1]);
    }
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const float dot = (d[2 * u] + d[2 * u + 1]) * dot_unscale;
      float part = valid[u] ? fmaf(sb[u], dot, zb[u] * qsum) : 0.f;
      part += __shfl_xor_sync(0xffffffffu, part, 1);
      part += __shfl_xor_sync(0xffffffffu, part, 2);
      if (idx[u] < n_cols && l4 == 0) {
        if (!valid[u]) {
          record_error(P.st, FL_ERR_RANGE);
          p[idx[u]] = -INFINITY;
        } else {
          p[idx[u]] = part * P.scale + bias_c[u];
        }
      }
    }
  }
  __syncwarp();

  // ---- K residual passes: items of a chunk as one stream, parts added in loop order
  // (a chunk holds loops of one bit width, a compile-time constant in its pass)
  auto k_res_pass = [&](auto width) {
    constexpr int UB = decltype(width)::value;
    const float sc = P.scale;
    for (int i0 = 0; i0 < n_items; i0 += 16) {
      Raw<EL> raw[2];
      float sr[2], zr[2];
      int bits[2];
      bool on[2];
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        // items past the chunk read item 0 (the chunk has one) and are masked
        const int it0 = i0 + 8 * u + cg;
        on[u] = it0 < n_items;
        const int it = on[u] ? it0 : 0;
        bits[u] = UB;
        const int r = it_loop[it];
        const uint32_t rh = (uint32_t)it_row[it] * H + h;
        load_sz(kv.sz[0][r], (size_t)rh * ngrp + gidx, &sr[u], &zr[u]);
        load_raw<EL>(kv.codes[0][r] + (size_t)rh * (HD * UB / 8), UB, e0, raw[u]);
      }
      uint32_t wb0[EL / 4], wb1[EL / 4];
      to_bytes<EL>(raw[0], bits[0], wb0);
      to_bytes<EL>(raw[1], bits[1], wb1);
      float d[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int ks = 0; ks < KS; ++ks) {
        mma::m16n8k16(d, mma::code_pair(wb0[ks], 0, 1), mma::code_pair(wb1[ks], 0, 1),
                      mma::code_pair(wb0[ks], 2, 3), mma::code_pair(wb1[ks], 2, 3),
                      bq[ks][0], bq[ks][1]);
      }
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const float dot = (d[2 * u] + d[2 * u + 1]) * dot_unscale;
        float part = on[u] ? fmaf(sr[u], dot, zr[u] * qsum) : 0.f;
        part += __shfl_xor_sync(0xffffffffu, part, 1);
        part += __shfl_xor_sync(0xffffffffu, part, 2);
        if (on[u] && l4 == 0) it_part[i0 + 8 * u + cg] = part * sc;
      }
    }
  };
  for (int r0 = 2, r1; r0 <= loop; r0 = r1) {
    r1 = chunk_end(r0);
    n_items = build_items(r0, r1);
    switch (kv.res_bits[r0]) {   // 2, 4 or 8 (checked at launch)
      case 2: k_res_pass(Width<2>{}); break;
      case 4: k_res_pass(Width<4>{}); break;
      default: k_res_pass(Width<8>{}); break;
    }
    __syncwarp();
    for (int k = 0; k < r1 - r0; ++k) {   // loop order; a loop lists a column at most once
      for (int x = loff[k] + lane; x < loff[k + 1]; x += 32) p[it_idx[x]] += it_part[x];
      __syncwarp();
    }
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
  for (int i0 = 0; i0 < n_cols; i0 += 16) {
    Raw<EL> raw[2];
    float s[2], z[2], wgt[2];
    bool valid[2];
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int idx = i0 + 8 * u + cg;
      const int ci = idx < n_cols ? (int)cols[idx] : 0;
      valid[u] = idx < n_cols && ci <= t && ci < n_tok;
      const int c = valid[u] ? ci : 0;   // masked rows read column 0
      wgt[u] = valid[u] ? p[idx] : 0.f;
      const uint32_t bh = (uint32_t)c * H + h;
      load_sz(kv.sz[1][1], (size_t)bh * ngrp + gidx, &s[u], &z[u]);
      load_raw<EL>(kv.codes[1][1] + (size_t)bh * HD, 8, e0, raw[u]);
    }
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      if (!valid[u]) continue;
      const float ws = wgt[u] * s[u];
      axpy_raw<EL>(ws, raw[u], 8, o);
      oz = fmaf(wgt[u], z[u], oz);
      if (SHRINK && prune && !mark[i0 + 8 * u + cg]) {
        axpy_raw<EL>(ws, raw[u], 8, ua);
        uz = fmaf(wgt[u], z[u], uz);
      }
    }
  }
  auto v_res_pass = [&](auto width) {
    constexpr int UB = decltype(width)::value;
    for (int i0 = 0; i0 < n_items; i0 += 16) {
      Raw<EL> raw[2];
      float s[2], z[2], wgt[2];
      int bits[2], idx[2];
      bool on[2];
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const int it0 = i0 + 8 * u + cg;
        on[u] = it0 < n_items;
        const int it = on[u] ? it0 : 0;   // masked items read item 0
        bits[u] = UB;
        const int r = it_loop[it];
        idx[u] = it_idx[it];
        wgt[u] = p[idx[u]];
        const uint32_t rh = (uint32_t)it_row[it] * H + h;
        load_sz(kv.sz[1][r], (size_t)rh * ngrp + gidx, &s[u], &z[u]);
        load_raw<EL>(kv.codes[1][r] + (size_t)rh * (HD * UB / 8), UB, e0, raw[u]);
      }
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        if (!on[u]) continue;
        const float ws = wgt[u] * s[u];
        axpy_raw<EL>(ws, raw[u], bits[u], o);
        oz = fmaf(wgt[u], z[u], oz);
        if (SHRINK && prune && !mark[idx[u]]) {
          axpy_raw<EL>(ws, raw[u], bits[u], ua);
          uz = fmaf(wgt[u], z[u], uz);
        }
      }
    }
  };
  for (int r0 = 2, r1; r0 <= loop; r0 = r1) {
    r1 = chunk_end(r0);
    if (!one_chunk) n_items = build_items(r0, r1);   // else still held from the K pass
    switch (kv.res_bits[r0]) {
      case 2: v_res_pass(Width<2>{}); break;
      case 4: v_res_pass(Width<4>{}); break;
      default: v_res_pass(Width<8>{}); break;
    }
    __syncwarp();
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
__global__ void __launch_bounds__(NW * 32, min_ctas(SHRINK)) k_attn_sparse(const __grid_constant__ AttnParams P) {
  extern __shared__ __align__(16) uint8_t smem[];
  griddep_wait();
  const int w = threadIdx.x >> 5;
  const int gw = blockIdx.x * NW + w;
  if (gw >= P.n_q * P.H) return;  // whole warp leaves
  attn_sparse_warp<HD, SHRINK>(P, gw, smem + (size_t)w * warp_smem(P.sel_stride, P.loop));
}

// Many independent calls in one launch (batched decode: one store per sequence). The
// calls share n_q, heads, head_dim and carried-set stride; `per` = n_q * H warps each;
// `loop` is the deepest call's loop (a warp's slice holds that call's layout).
template <int HD, bool SHRINK>
__global__ void __launch_bounds__(NW * 32, min_ctas(SHRINK))
    k_attn_sparse_batched(const AttnParams* __restrict__ Ps, int n_calls, int per, int stride,
                          int loop) {
  extern __shared__ __align__(16) uint8_t smem[];
  const int w = threadIdx.x >> 5;
  const int gw = blockIdx.x * NW + w;
  if (gw >= n_calls * per) return;
  attn_sparse_warp<HD, SHRINK>(Ps[gw / per], gw % per, smem + (size_t)w * warp_smem(stride, loop));
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
  return (size_t)NW * warp_smem(P.sel_stride, P.loop) <= 200 * 1024;
}

cudaError_t launch_attn_sparse_fast(const AttnParams& P, cudaStream_t s) {
  const size_t sm = (size_t)NW * warp_smem(P.sel_stride, P.loop);
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
  const cudaError_t e = launch_pdl(kern, dim3(blocks), dim3(NW * 32), sm, s, P);
  count_launch();
  return e != cudaSuccess ? e : cudaGetLastError();
}

// Ps: device array of n AttnParams (already copied by the caller, same shapes; loops up
// to loop_max, which sizes every warp's shared-memory slice).
cudaError_t launch_attn_sparse_batched(const AttnParams& P0, const AttnParams* Ps_dev, int n,
                                       int loop_max, cudaStream_t s) {
  const size_t sm = (size_t)NW * warp_smem(P0.sel_stride, loop_max);
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
  kern<<<blocks, NW * 32, sm, s>>>(Ps_dev, n, per, P0.sel_stride, loop_max);
  count_launch();
  return cudaGetLastError();
}

}  // namespace fl
