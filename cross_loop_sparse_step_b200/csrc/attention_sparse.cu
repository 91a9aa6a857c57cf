// Loop-aware sparse attention over carried column sets, one warp per (query, head)
// (FlashLoop §4.2 "Loop-Aware Sparse Attention": softmax over the selected logits only,
// rescaled by the cached global mass, plus the carried unselected contribution; the
// K/V of the selected columns are gathered, here straight from the quantised store).
//
// Used when the store is quantised throughout (int8 base, 2/4/8-bit residuals).
//   K pass, one lane per column: the lane streams the column's 128-byte base code row,
//     its (scale, offset) pairs and the residual rows of every loop that rewrote it,
//     with independent 16-byte loads, and forms q . K^ group by group as
//     s * (q . codes) + z * sum(q) - the dequantisation folded into the dot product.
//   softmax over the column set, p~ = m * softmax (m = cached mass).
//   optional budget shrink: warp radix select over the binary32 bits of p~ * ||V^||
//     (ties to the smaller column), ballot-ordered so the kept set stays ascending.
//   V pass, lanes split head_dim: each column's rows are read coalesced, V^ is rebuilt
//     in the store's order (base, then each residual added in binary32) and
//     accumulated into o and, for dropped columns, into the next loop's u'.
#include <float.h>

#include "fl_internal.cuh"

namespace fl {
namespace {

constexpr int NW = 4;  // warps per CTA

__host__ __device__ inline size_t align16(size_t x) { return (x + 15) & ~size_t(15); }

// Per-warp shared memory: q [HD] | qsum [4] | p [stride] | cols [stride] u16 |
// mark [stride] u8 | hist [256] i32.
__host__ __device__ inline size_t warp_smem(int hd, int stride) {
  return align16((size_t)hd * 4 + 16) + align16((size_t)stride * 4) + align16((size_t)stride * 2) +
         align16((size_t)stride) + 256 * 4;
}

__device__ __forceinline__ float byte_f(uint32_t w, int i) {
  // (float)((w >> 8i) & 0xFF), exact: the byte under the exponent of 2^23, minus 2^23
  const uint32_t sel = (uint32_t)i | (4u << 4) | (4u << 8) | (7u << 12);
  return __uint_as_float(__byte_perm(w, 0x4B000000u, sel)) - 8388608.0f;
}

__device__ __forceinline__ float nib_f(uint32_t w, int i, int bits) {
  const uint32_t c = (w >> (i * bits)) & ((1u << bits) - 1u);
  return __uint_as_float(0x4B000000u | c) - 8388608.0f;
}

// sum_e q[e] * deq[e] over one stored row of HD elements: per group g of `gs` elements,
// s_g * (q_g . codes_g) + z_g * qsum_g. `bits` in {2, 4, 8}.
template <int HD>
__device__ __forceinline__ float row_dot(const uint8_t* codes, const uint32_t* sz, int bits,
                                         int gs, const float* q, const float* qsum) {
  float acc = 0.f;
  const int ngroups = HD / gs;
  const int wpg = gs * bits / 32;  // 32-bit code words per group
  for (int gi = 0; gi < ngroups; ++gi) {
    const uint32_t pair = sz[gi];
    const float s = half_bits_to_float((uint16_t)(pair & 0xFFFFu));
    const float z = half_bits_to_float((uint16_t)(pair >> 16));
    const uint32_t* cw = reinterpret_cast<const uint32_t*>(codes) + gi * wpg;
    const float* qg = q + gi * gs;
    float d = 0.f;
    if (bits == 8) {
      for (int k4 = 0; k4 < wpg; k4 += 4) {
        const uint4 u = *reinterpret_cast<const uint4*>(cw + k4);
        const uint32_t ww[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const float4 qq = *reinterpret_cast<const float4*>(qg + (k4 + j) * 4);
          d = fmaf(qq.x, byte_f(ww[j], 0), d);
          d = fmaf(qq.y, byte_f(ww[j], 1), d);
          d = fmaf(qq.z, byte_f(ww[j], 2), d);
          d = fmaf(qq.w, byte_f(ww[j], 3), d);
        }
      }
    } else {
      const int per = 32 / bits;  // codes per word
      for (int k = 0; k < wpg; ++k) {
        const uint32_t wv = cw[k];
        const float* qw = qg + k * per;
        for (int j = 0; j < per; ++j) d = fmaf(qw[j], nib_f(wv, j, bits), d);
      }
    }
    acc = fmaf(s, d, acc);
    acc = fmaf(z, qsum[gi], acc);
  }
  return acc;
}

template <int HD>
__global__ void __launch_bounds__(NW * 32) k_attn_sparse(const __grid_constant__ AttnParams P) {
  extern __shared__ __align__(16) uint8_t smem[];
  constexpr int EPL = HD / 32;
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int gw = blockIdx.x * NW + w;
  if (gw >= P.n_q * P.H) return;  // whole warp leaves; no CTA-wide barrier below
  const int qi = gw / P.H, h = gw % P.H;
  const int H = P.H, n_tok = P.kv.n_tok, gs = P.kv.g, stride = P.sel_stride;
  const KvView& kv = P.kv;

  uint8_t* base = smem + (size_t)w * warp_smem(HD, stride);
  float* qs = reinterpret_cast<float*>(base);
  float* qsum = qs + HD;
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
  const bool want_stats = P.sel_out != nullptr;

  // ---- carried column set, cached mass, query slice
  const uint16_t* srow_p = P.sel + ((size_t)h * P.stat_rows + srow) * stride;
  int n_cols = 0;
  for (int i0 = 0; i0 < stride; i0 += 32) {
    const int i = i0 + lane;
    const uint16_t c = i < stride ? srow_p[i] : (uint16_t)FL_SENTINEL;
    if (i < stride) cols[i] = c;
    n_cols += __popc(__ballot_sync(0xffffffffu, c != FL_SENTINEL));
  }
  const float m_in = P.mass[(size_t)h * P.stat_rows + srow];
  const int e0 = lane * EPL;
  {
    const size_t off = ((size_t)qi * H + h) * HD + e0;
    float part = 0.f;
#pragma unroll
    for (int j = 0; j < EPL; ++j) {
      const float v = P.q_bf16 ? __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(P.q)[off + j])
                               : reinterpret_cast<const float*>(P.q)[off + j];
      qs[e0 + j] = v;
      part += v;
    }
    const int lpg = gs / EPL;  // lanes per quantisation group
    for (int o = 1; o < lpg; o <<= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
    if (lane % lpg == 0) qsum[e0 / gs] = part;
  }
  __syncwarp();

  // ---- K pass: one lane per column
  float lmax = -FLT_MAX;
  const size_t krow = (size_t)HD;                 // base code bytes per (token, head)
  for (int idx = lane; idx < n_cols; idx += 32) {
    const int c = cols[idx];
    float sc;
    if (c > t || c >= n_tok) {
      record_error(P.st, FL_ERR_RANGE);
      sc = -INFINITY;
    } else {
      const size_t bh = (size_t)c * H + h;
      float acc = row_dot<HD>(kv.codes[0][1] + bh * krow,
                              reinterpret_cast<const uint32_t*>(kv.sz[0][1]) + bh * (HD / gs), 8, gs,
                              qs, qsum);
      for (int r = 2; r <= P.loop; ++r) {
        const int row = kv.slot[(size_t)r * n_tok + c];
        if (row < 0) continue;
        const int b = kv.res_bits[r];
        const size_t rh = (size_t)row * H + h;
        acc += row_dot<HD>(kv.codes[0][r] + rh * (HD * b / 8),
                           reinterpret_cast<const uint32_t*>(kv.sz[0][r]) + rh * (HD / gs), b, gs,
                           qs, qsum);
      }
      sc = acc * P.scale + (P.bias ? P.bias[c] : 0.f);
    }
    p[idx] = sc;
    lmax = fmaxf(lmax, sc);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) lmax = fmaxf(lmax, __shfl_xor_sync(0xffffffffu, lmax, o));
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
  const bool prune = want_stats && (n_cols - 1 > P.k_next);
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

  // ---- V pass: lanes split head_dim
  float o[EPL], ua[EPL];
#pragma unroll
  for (int j = 0; j < EPL; ++j) { o[j] = 0.f; ua[j] = 0.f; }
  const int grp = e0 / gs;
  const uint32_t* vsz1 = reinterpret_cast<const uint32_t*>(kv.sz[1][1]);
  for (int idx = 0; idx < n_cols; ++idx) {
    const int c = cols[idx];
    const float wgt = p[idx];
    if (c > t || c >= n_tok || wgt == 0.f) continue;  // uniform across the warp
    const size_t bh = (size_t)c * H + h;
    float v[EPL];
    {
      const uint32_t pair = vsz1[bh * (HD / gs) + grp];
      const float s = half_bits_to_float((uint16_t)(pair & 0xFFFFu));
      const float z = half_bits_to_float((uint16_t)(pair >> 16));
      const uint8_t* cp = kv.codes[1][1] + bh * HD + e0;
      uint32_t word;
      if (EPL == 4) word = *reinterpret_cast<const uint32_t*>(cp);
      else word = *reinterpret_cast<const uint16_t*>(cp);
#pragma unroll
      for (int j = 0; j < EPL; ++j) v[j] = __fmaf_rn(byte_f(word, j), s, z);
    }
    for (int r = 2; r <= P.loop; ++r) {
      const int row = kv.slot[(size_t)r * n_tok + c];
      if (row < 0) continue;
      const int b = kv.res_bits[r];
      const size_t rh = (size_t)row * H + h;
      const uint32_t pair = reinterpret_cast<const uint32_t*>(kv.sz[1][r])[rh * (HD / gs) + grp];
      const float s = half_bits_to_float((uint16_t)(pair & 0xFFFFu));
      const float z = half_bits_to_float((uint16_t)(pair >> 16));
      const uint8_t* rp = kv.codes[1][r] + rh * (HD * b / 8);
      const int bit0 = e0 * b;
#pragma unroll
      for (int j = 0; j < EPL; ++j) {
        const int bit = bit0 + j * b;
        const int code = (rp[bit >> 3] >> (bit & 7)) & ((1 << b) - 1);
        v[j] = __fadd_rn(v[j], __fmaf_rn((float)code, s, z));
      }
    }
    const bool drop = prune && !mark[idx];
#pragma unroll
    for (int j = 0; j < EPL; ++j) {
      o[j] = fmaf(wgt, v[j], o[j]);
      if (drop) ua[j] = fmaf(wgt, v[j], ua[j]);
    }
  }

  // ---- outputs
  const float* u_in = P.unsel + ((size_t)h * P.stat_rows + srow) * HD;
  const size_t ob = ((size_t)qi * H + h) * HD + e0;
  float* u_out = want_stats ? P.unsel_out + ((size_t)h * P.stat_rows + srow) * HD : nullptr;
#pragma unroll
  for (int j = 0; j < EPL; ++j) {
    const float ui = u_in[e0 + j];
    const float val = ui + o[j];
    if (P.out_bf16) reinterpret_cast<__nv_bfloat16*>(P.out)[ob + j] = __float2bfloat16_rn(val);
    else reinterpret_cast<float*>(P.out)[ob + j] = val;
    if (want_stats) u_out[e0 + j] = prune ? ui + ua[j] : ui;
  }
  if (!want_stats) return;
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
  auto kern = P.hd == 128 ? k_attn_sparse<128> : k_attn_sparse<64>;
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
  kern<<<blocks, NW * 32, sm, s>>>(P);
  count_launch();
  return cudaGetLastError();
}

}  // namespace fl
