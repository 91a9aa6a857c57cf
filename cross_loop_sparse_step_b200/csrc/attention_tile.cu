// Loop-aware sparse attention on the tensor cores, one CTA per (head, tile of 128
// queries) (FlashLoop §4.2 "Loop-Aware Sparse Attention": each query attends to the
// columns its carried set names, softmax over them, rescaled by the cached mass, plus
// the carried unselected contribution; §4.4: the selected K/V are brought into compact
// on-chip buffers and QK^T / PV run on them).
//
// The queries of a tile carry different column sets. The CTA takes the union of the
// tile's sets (a bitmap over the tokens, then ranks by prefix popcounts), walks the
// union in chunks of 128 columns, and runs every chunk as a dense 128 x 128 tile on the
// tensor cores with each query's membership as a mask:
//   producer warps (two groups of four, one per pipeline stage) decode the chunk's K^
//     and V^ rows - int8 base plus the residual chain of every loop that rewrote the
//     column, fmaf(code, s, z) added in loop order, exactly the store's reconstruction -
//     and write them as fp16 operand tiles in the 128-byte-swizzle layout, both as
//     [column][element] rows: K^ is the K-major B operand of Q K^T, V^ the MN-major B
//     operand of P V^;
//   the MMA warp issues S = Q K^T into one of two TMEM score buffers, then, once the
//     softmax has written P, O += P V^ into the TMEM output accumulator
//     (tcgen05.mma kind::f16, M 128, N 128, fp32 accumulation);
//   the softmax warps (thread = query row = TMEM lane) read their row of S, keep the
//     columns their set names (the set is walked in step with the chunks), update an
//     online maximum - the output is rescaled only when the maximum grows by more than
//     2^8, so P stays below 256 in fp16 - and write P = 2^(s - max) as fp16; the row sum
//     is taken over the fp16 values the MMA uses. At the end
//     o = u + m * O / sum, with m the cached mass and u the unselected contribution.
// Operand precision: q, K^, V^ and P enter the MMAs as fp16 (11 significant bits);
// sums are binary32. Every wait is bounded; a wait that runs out records FL_ERR_TIMEOUT,
// the CTA drains its MMAs, frees TMEM and returns.
//
// Taken for head_dim 128 over a quantised store (8-bit base, 2/4/8-bit residuals) when
// the call writes no statistics (none requested, or in place with an unchanged budget).
#include <float.h>

#include "attn_tile_common.cuh"

namespace fl {
namespace {

using namespace sm100;
using namespace tile;

constexpr int NWARPS = 13;         // 0-3, 8-11 producers; 4-7 softmax; 12 MMA
constexpr int NTHR = NWARPS * 32;
constexpr int MAX_WORDS = 2048;                  // bitmap words for n_tok <= 65535

// dynamic shared memory (1024-byte aligned base)
constexpr uint32_t OFF_Q = 0;
constexpr uint32_t OFF_K0 = OFF_Q + TILE;        // stage s: K at OFF_K0 + 2 s TILE, V after it
constexpr uint32_t OFF_P = OFF_K0 + 4 * TILE;
constexpr uint32_t OFF_BITS = OFF_P + TILE;
constexpr uint32_t OFF_PRE = OFF_BITS + MAX_WORDS * 4;
constexpr uint32_t OFF_BIAS = OFF_PRE + MAX_WORDS * 2;   // [2][TC] float (log2 units)
constexpr uint32_t SMEM_BYTES = OFF_BIAS + 2 * TC * 4 + 1024;

struct TileShared {
  uint64_t kv_full[2], kv_empty[2], meta_full[2], s_full[2], p_full[2], pv_done, fin;
  uint32_t tmem;
  int abort_flag;
  int n_union;
  int scan[NWARPS];
};

// rank of token `col` among the union's columns (col must be in the union)
__device__ __forceinline__ int union_rank(const uint32_t* bits, const uint16_t* pre, int col) {
  const int w = col >> 5;
  return (int)pre[w] + __popc(bits[w] & ((1u << (col & 31)) - 1u));
}

// One CTA: head h, the tile of queries starting at q0 of the call described by P.
__device__ __forceinline__ void attn_tile_cta(const AttnParams& P, int h, int q0) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  __shared__ TileShared sh;
  volatile int* abort = &sh.abort_flag;
  uint32_t* bits = reinterpret_cast<uint32_t*>(smem + OFF_BITS);
  uint16_t* pre = reinterpret_cast<uint16_t*>(smem + OFF_PRE);
  float* biasbuf = reinterpret_cast<float*>(smem + OFF_BIAS);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int H = P.H, n_tok = P.kv.n_tok, stride = P.sel_stride;
  const int n_words = (n_tok + 31) >> 5;

  if (threadIdx.x == 0) {
    for (int s = 0; s < 2; ++s) {
      mbar_init(&sh.kv_full[s], 4); mbar_init(&sh.kv_empty[s], 1);
      mbar_init(&sh.meta_full[s], 4); mbar_init(&sh.s_full[s], 1);
    }
    mbar_init(&sh.p_full[0], TQ);
    mbar_init(&sh.p_full[1], TQ);
    mbar_init(&sh.pv_done, 1);
    mbar_init(&sh.fin, 1);
    sh.abort_flag = 0;
    fence_barrier_init();
  }
  for (int w = threadIdx.x; w < n_words; w += NTHR) bits[w] = 0u;
  if (warp == 12) tmem_alloc(&sh.tmem, 512);
  griddep_wait();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sh.tmem;

  // ---- the union of the tile's column sets (entries that are not valid columns of the
  // query - beyond its position or the store - are recorded and skipped here and below)
  for (int i = warp; i < TQ; i += NWARPS) {
    const int qi = q0 + i;
    if (qi >= P.n_q) break;
    const int t = P.q_tok[qi];
    const int srow = P.q_row ? P.q_row[qi] : t;
    if (t < 0 || t >= n_tok || srow < 0 || srow >= P.stat_rows) continue;
    const uint16_t* row = P.sel + ((size_t)h * P.stat_rows + srow) * stride;
    for (int e0 = 0; e0 < stride; e0 += 32) {
      const int e = e0 + lane;
      const int c = e < stride ? (int)row[e] : (int)FL_SENTINEL;
      const bool ok = c != (int)FL_SENTINEL && c < n_tok && c <= t;
      if (ok) atomicOr(&bits[c >> 5], 1u << (c & 31));
      if (__all_sync(0xffffffffu, c == (int)FL_SENTINEL)) break;   // padding reached
    }
  }
  __syncthreads();
  {  // exclusive prefix of the word popcounts (up to 5 words per thread)
    constexpr int PER = (MAX_WORDS + NTHR - 1) / NTHR;
    const int w0 = threadIdx.x * PER;
    int cnt[PER], sum = 0;
#pragma unroll
    for (int k = 0; k < PER; ++k) {
      cnt[k] = (w0 + k < n_words) ? __popc(bits[w0 + k]) : 0;
      sum += cnt[k];
    }
    int incl = sum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    if (lane == 31) sh.scan[warp] = incl;
    __syncthreads();
    int base = incl - sum;
    for (int k = 0; k < warp; ++k) base += sh.scan[k];
    if (threadIdx.x == NTHR - 1) sh.n_union = base + sum;
#pragma unroll
    for (int k = 0; k < PER; ++k) {
      if (w0 + k < n_words) pre[w0 + k] = (uint16_t)base;
      base += cnt[k];
    }
  }
  __syncthreads();
  const int U = sh.n_union;
  const int n_chunks = (U + TC - 1) / TC;

  const float scale2 = P.scale * kLog2e;
  const uint32_t idesc = idesc_f16_f32(TQ, TC);
  const uint32_t idesc_pv = idesc_f16_f32_bmn(TQ, HDT);   // V^ tiles are MN-major

  if (warp >= 4 && warp < 8) {
    // ================================================================ softmax warps
    const int i = (warp - 4) * 32 + lane;      // query row of the tile = TMEM lane
    const int qi = q0 + i;
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
    bool valid = qi < P.n_q;
    int t = 0, srow = 0;
    if (valid) {
      t = P.q_tok[qi];
      srow = P.q_row ? P.q_row[qi] : t;
      if (t < 0 || t >= n_tok || srow < 0 || srow >= P.stat_rows) {
        record_error(P.st, FL_ERR_RANGE);
        valid = false;
      }
    }
    // the query row as fp16 into Q (zeros for rows without a query)
    {
      uint8_t* qt = smem + OFF_Q;
      for (int e0 = 0; e0 < HDT; e0 += 8) {
        float x[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) x[k] = 0.f;
        if (valid) {
          const size_t off = ((size_t)qi * H + h) * HDT + e0;
          if (P.q_bf16) {
            const uint4 v = *reinterpret_cast<const uint4*>(reinterpret_cast<const __nv_bfloat16*>(P.q) + off);
            const __nv_bfloat162* b2 = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
            for (int k = 0; k < 4; ++k) { x[2 * k] = __low2float(b2[k]); x[2 * k + 1] = __high2float(b2[k]); }
          } else {
            const float4 a = *reinterpret_cast<const float4*>(reinterpret_cast<const float*>(P.q) + off);
            const float4 b = *reinterpret_cast<const float4*>(reinterpret_cast<const float*>(P.q) + off + 4);
            x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w; x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
          }
        }
        *reinterpret_cast<uint4*>(qt + sw128_offset(i, e0, TQ)) =
            make_uint4(pack_h2(x[0], x[1]), pack_h2(x[2], x[3]), pack_h2(x[4], x[5]), pack_h2(x[6], x[7]));
      }
      fence_proxy_async_smem();
    }
    // named barrier: Q written by the 4 softmax warps before the MMA warp issues QK
    asm volatile("bar.sync 1, %0;" ::"n"(5 * 32) : "memory");

    const uint16_t* srow_p = valid ? P.sel + ((size_t)h * P.stat_rows + srow) * stride : nullptr;
    // The set is walked 8 entries at a time in step with the chunks: gr[] holds the union
    // ranks of the current group (-1: entry skipped), the next group's loads are issued one
    // group ahead so their latency overlaps a chunk.
    int ent = 0;
    bool ended = !valid;       // a sentinel or the end of the row was reached
    uint32_t nx[8];
    int gr[8], gmax = -1;
    auto load_next = [&]() {
#pragma unroll
      for (int k = 0; k < 8; ++k)
        nx[k] = (!ended && ent + k < stride) ? (uint32_t)srow_p[ent + k] : (uint32_t)FL_SENTINEL;
      ent += 8;
    };
    auto take_next = [&]() {   // ranks of the loaded group; load the one after
      gmax = -1;
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const int c = (int)nx[k];
        gr[k] = -1;
        if (ended || c == (int)FL_SENTINEL) { ended = true; continue; }
        if (c >= n_tok || c > t) { record_error(P.st, FL_ERR_RANGE); continue; }
        gr[k] = union_rank(bits, pre, c);
        gmax = gr[k];
      }
      if (ent >= stride) ended = true;
      load_next();
    };
#pragma unroll
    for (int k = 0; k < 8; ++k) gr[k] = -1;
    load_next();
    if (valid) take_next();
    float m_used = -INFINITY, lsum = 0.f;
    const float m_in = valid ? P.mass[(size_t)h * P.stat_rows + srow] : 0.f;
    uint8_t* pt = smem + OFF_P;
    for (int c = 0; c < n_chunks; ++c) {   // leaves only through warp-uniform waits
      uint32_t mask[4] = {0u, 0u, 0u, 0u};
      const int lo = c * TC, hi = lo + TC;
      while (true) {
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const int pos = gr[k] - lo;
          const uint32_t bit = (pos >= 0 && pos < TC) ? 1u << (pos & 31) : 0u;
          const int w = pos >> 5;   // selects, so the mask stays in registers
          mask[0] |= w == 0 ? bit : 0u;
          mask[1] |= w == 1 ? bit : 0u;
          mask[2] |= w == 2 ? bit : 0u;
          mask[3] |= w == 3 ? bit : 0u;
        }
        if (gmax < hi && !ended) take_next();
        else break;
      }
      __syncwarp();   // reconverge before the warp-collective TMEM accesses
      const int sb = c & 1;
      // waits agree across the warp: the TMEM loads below are warp-collective
      if (!warp_wait(&sh.s_full[sb], (c >> 1) & 1, abort, 101)) break;
      if (!warp_wait(&sh.meta_full[sb], (c >> 1) & 1, abort, 102)) break;
      tc_fence_after();
      const uint32_t s_addr = tmem + lane_base + (uint32_t)(sb * TC);
      const float* bias = biasbuf + sb * TC;
      float cmax = -INFINITY;
#pragma unroll
      for (int g4 = 0; g4 < 4; ++g4) {
        float v[32];
        tmem_ld32(s_addr + g4 * 32, v);
#pragma unroll
        for (int j = 0; j < 32; ++j)
          if (mask[g4] & (1u << j)) cmax = fmaxf(cmax, fmaf(v[j], scale2, bias[g4 * 32 + j]));
      }
      float alpha = 1.f;
      bool rescale = false;
      if (cmax > m_used + kRescale) {
        if (m_used != -INFINITY && lsum > 0.f) { alpha = exp2f(m_used - cmax); rescale = true; }
        m_used = cmax;
      }
      // P of the previous chunk must have been consumed (and O completed) before P is
      // rewritten or O rescaled
      if (c > 0 && !warp_wait(&sh.pv_done, (c - 1) & 1, abort, 103)) break;
      tc_fence_after();
      if (rescale) lsum *= alpha;
      if (__any_sync(0xffffffffu, rescale)) {   // warp-collective; alpha = 1 elsewhere
        const uint32_t o_addr = tmem + lane_base + 2u * TC;
#pragma unroll 1
        for (int g4 = 0; g4 < 4; ++g4) {
          float v[32];
          tmem_ld32(o_addr + g4 * 32, v);
#pragma unroll
          for (int j = 0; j < 32; ++j) v[j] *= alpha;
          tmem_st32(o_addr + g4 * 32, v);
        }
      }
#pragma unroll
      for (int g4 = 0; g4 < 4; ++g4) {
        float v[32];
        tmem_ld32(s_addr + g4 * 32, v);
        uint32_t pk[16];
#pragma unroll
        for (int j = 0; j < 32; j += 2) {
          float a = 0.f, b = 0.f;
          if (mask[g4] & (1u << j)) a = exp2f(fmaf(v[j], scale2, bias[g4 * 32 + j]) - m_used);
          if (mask[g4] & (1u << (j + 1))) b = exp2f(fmaf(v[j + 1], scale2, bias[g4 * 32 + j + 1]) - m_used);
          const __half2 hv = __floats2half2_rn(a, b);
          const float2 back = __half22float2(hv);
          lsum += back.x + back.y;
          pk[j / 2] = *reinterpret_cast<const uint32_t*>(&hv);
        }
#pragma unroll
        for (int q = 0; q < 4; ++q)
          *reinterpret_cast<uint4*>(pt + sw128_offset(i, g4 * 32 + q * 8, TQ)) =
              make_uint4(pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(&sh.p_full[sb]);   // one barrier per score buffer
    }
    // ---- output: o = u + m * O / sum
    bool done_ok = !*abort;
    if (n_chunks > 0 && done_ok) done_ok = mbar_wait(&sh.pv_done, (n_chunks - 1) & 1, abort, 104);
    tc_fence_after();
    if (__all_sync(0xffffffffu, done_ok)) {
      const uint32_t o_addr = tmem + lane_base + 2u * TC;
      const float f = (valid && lsum > 0.f) ? m_in / lsum : 0.f;
      const float* u = valid ? P.unsel + ((size_t)h * P.stat_rows + srow) * HDT : nullptr;
      const size_t ob = ((size_t)qi * H + h) * HDT;
#pragma unroll 1
      for (int g4 = 0; g4 < 4; ++g4) {
        float v[32];
        if (n_chunks > 0) tmem_ld32(o_addr + g4 * 32, v);
        else {
#pragma unroll
          for (int j = 0; j < 32; ++j) v[j] = 0.f;
        }
        if (!valid) continue;
#pragma unroll
        for (int j = 0; j < 32; j += 4) {
          const float4 uu = *reinterpret_cast<const float4*>(u + g4 * 32 + j);
          const float o0 = fmaf(v[j], f, uu.x), o1 = fmaf(v[j + 1], f, uu.y);
          const float o2 = fmaf(v[j + 2], f, uu.z), o3 = fmaf(v[j + 3], f, uu.w);
          if (P.out_bf16) {
            __nv_bfloat16* o = reinterpret_cast<__nv_bfloat16*>(P.out) + ob + g4 * 32 + j;
            const __nv_bfloat162 a = __floats2bfloat162_rn(o0, o1), b = __floats2bfloat162_rn(o2, o3);
            *reinterpret_cast<uint2*>(o) = make_uint2(*reinterpret_cast<const uint32_t*>(&a),
                                                      *reinterpret_cast<const uint32_t*>(&b));
          } else {
            *reinterpret_cast<float4*>(reinterpret_cast<float*>(P.out) + ob + g4 * 32 + j) =
                make_float4(o0, o1, o2, o3);
          }
        }
      }
    }
  } else if (warp == 12) {
    // ================================================================ MMA warp
    asm volatile("bar.sync 1, %0;" ::"n"(5 * 32) : "memory");
    if (lane == 0 && n_chunks > 0) {
      const uint32_t q_base = smem_u32(smem + OFF_Q);
      const uint32_t p_base = smem_u32(smem + OFF_P);
      // Issue whichever MMA is ready: QK^T of the next chunk once its operands are decoded
      // and its score buffer is free (the softmax handed back chunk c - 2), P V^ of the
      // oldest chunk once its P is written. Neither waits on the other, so the two producer
      // groups decode concurrently.
      int qk = 0, pv = 0;
      uint64_t t0 = globaltimer();
      while (pv < n_chunks) {
        bool prog = false;
        if (qk < n_chunks && qk <= pv + 1 && mbar_test_wait(&sh.kv_full[qk & 1], (qk >> 1) & 1)) {
          tc_fence_after();
          const int st = qk & 1;
          const uint32_t k_base = smem_u32(smem + OFF_K0 + 2 * st * TILE);
          const uint32_t d = tmem + (uint32_t)(st * TC);
#pragma unroll
          for (int kk = 0; kk < HDT / 16; ++kk) {
            const uint32_t off = (kk >> 2) * (TQ * 128) + (kk & 3) * 32;
            mma_bf16(d, desc_sw128_kmajor(q_base + off), desc_sw128_kmajor(k_base + off), idesc,
                     kk > 0 ? 1u : 0u);
          }
          mma_commit(&sh.s_full[st]);
          ++qk;
          prog = true;
        }
        if (pv < qk && mbar_test_wait(&sh.p_full[pv & 1], (pv >> 1) & 1)) {
          tc_fence_after();
          const int st = pv & 1;
          const uint32_t v_base = smem_u32(smem + OFF_K0 + (2 * st + 1) * TILE);
          const uint32_t d = tmem + 2u * TC;
#pragma unroll
          for (int kk = 0; kk < TC / 16; ++kk) {
            const uint32_t off = (kk >> 2) * (TQ * 128) + (kk & 3) * 32;
            mma_bf16(d, desc_sw128_kmajor(p_base + off), desc_sw128_mnmajor(v_base + kk * 2048, TC),
                     idesc_pv, (pv > 0 || kk > 0) ? 1u : 0u);
          }
          mma_commit(&sh.pv_done);
          mma_commit(&sh.kv_empty[st]);
          ++pv;
          prog = true;
        }
        if (prog) {
          t0 = globaltimer();
        } else {
          if (*abort) break;
          if (globaltimer() - t0 > kWaitLimitNs) {
            atomicCAS(const_cast<int*>(abort), 0, qk < n_chunks && qk <= pv + 1 ? 106 : 108);
            break;
          }
        }
      }
    }
    if (lane == 0) mma_commit(&sh.fin);   // arrives once every MMA issued above is done
  } else {
    // ================================================================ producer warps
    const int grp = warp < 4 ? 0 : 1;          // stage = chunk parity
    const int jj = (warp & 3) * 32 + lane;     // column of the chunk this lane decodes
    const float* bias_g = P.bias;
    uint8_t* k_tile = smem + OFF_K0 + 2 * grp * TILE;
    uint8_t* v_tile = k_tile + TILE;
    for (int c = grp; c < n_chunks; c += 2) {
      if (__any_sync(0xffffffffu, *abort != 0)) break;   // warp-uniform exit
      if (c >= 2 && !warp_wait(&sh.kv_empty[grp], ((c >> 1) - 1) & 1, abort, 109)) break;
      // column of rank c * TC + jj: the last word whose prefix <= rank, then the bit
      const int R = c * TC + jj;
      int col = -1;
      if (R < U) {
        int lo = 0, hi = n_words - 1;
        while (lo < hi) {
          const int mid = (lo + hi + 1) >> 1;
          if ((int)pre[mid] <= R) lo = mid;
          else hi = mid - 1;
        }
        uint32_t m = bits[lo];
        for (int k = R - (int)pre[lo]; k > 0 && m; --k) m &= m - 1u;
        col = m ? lo * 32 + __ffs(m) - 1 : -1;
        if (col < 0 || col >= n_tok) { record_error(P.st, FL_ERR_RANGE); col = -1; }
      }
      biasbuf[grp * TC + jj] = (col >= 0 && bias_g) ? __ldg(bias_g + col) * kLog2e : 0.f;
      __syncwarp();
      if (lane == 0) mbar_arrive(&sh.meta_full[grp]);
      uint32_t chain = 0;   // loops 2..loop that rewrote the column
      if (col >= 0)
        for (int r = 2; r <= P.loop; ++r)
          if (__ldg(P.kv.slot + (size_t)r * n_tok + col) >= 0) chain |= 1u << r;
      // K^ and V^ rows jj of the chunk (V^ is read as an MN-major operand of P V^)
      decode_column(P, 0, col, h, chain, k_tile, nullptr, jj);
      decode_column(P, 1, col, h, chain, v_tile, nullptr, jj);
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sh.kv_full[grp]);
    }
  }

  // ---- teardown: every MMA done before TMEM is released
  __syncthreads();
  if (warp == 12) {
    if (lane == 0) {
      const uint64_t t0 = globaltimer();
      while (!mbar_try_wait(&sh.fin, 0))
        if (globaltimer() - t0 > kWaitLimitNs) { atomicCAS(&sh.abort_flag, 0, 110); break; }
    }
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
  if (threadIdx.x == 0 && sh.abort_flag) record_error(P.st, timeout_code(sh.abort_flag));
}

__global__ void __launch_bounds__(NTHR, 1) k_attn_tile(const __grid_constant__ AttnParams P) {
  const int n_tiles = (P.n_q + TQ - 1) / TQ;
  attn_tile_cta(P, blockIdx.x / n_tiles, (blockIdx.x % n_tiles) * TQ);
}

// Many calls in one launch (batched decode: one store per sequence): CTA b works on call
// b / per, per = tiles x heads of a call; the call's arguments are copied from global
// memory into shared memory first.
__global__ void __launch_bounds__(NTHR, 1) k_attn_tile_batched(const AttnParams* __restrict__ Ps,
                                                                 int per) {
  __shared__ AttnParams sP;
  const int call = blockIdx.x / per, b = blockIdx.x % per;
  {
    const uint32_t* src = reinterpret_cast<const uint32_t*>(Ps + call);
    uint32_t* dst = reinterpret_cast<uint32_t*>(&sP);
    for (int i = threadIdx.x; i < (int)(sizeof(AttnParams) / 4); i += blockDim.x) dst[i] = src[i];
  }
  __syncthreads();
  const int n_tiles = (sP.n_q + TQ - 1) / TQ;
  attn_tile_cta(sP, b / n_tiles, (b % n_tiles) * TQ);
}

}  // namespace

bool sparse_tile_eligible(const AttnParams& P) {
  if (P.hd != HDT || P.kv.hd != HDT || !P.sel) return false;
  if ((P.kv.base_bits != 8 && P.kv.base_bits != 0) || (P.kv.g != 32 && P.kv.g != 64)) return false;
  if (P.kv.n_tok > 65535 || P.loop > 31) return false;
  for (int r = 2; r <= P.loop; ++r) {
    const int b = P.kv.res_bits[r];
    if (b != 0 && b != 2 && b != 4 && b != 8) return false;
  }
  // statistics: none requested, or updated in place with an unchanged budget
  if (P.sel_out) {
    const bool in_place_unchanged = P.sel_out == P.sel && P.mass_out == P.mass &&
                                    P.unsel_out == P.unsel && P.out_stride == P.sel_stride &&
                                    P.k_next + 1 >= P.sel_stride;
    if (!in_place_unchanged) return false;
  }
  return true;
}

cudaError_t launch_attn_tile(const AttnParams& P, cudaStream_t s) {
  static bool attr_set[128] = {false};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 128) return cudaErrorInvalidDevice;
  if (!attr_set[dev]) {
    const cudaError_t e = cudaFuncSetAttribute(k_attn_tile, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                               (int)SMEM_BYTES);
    if (e != cudaSuccess) return e;
    attr_set[dev] = true;
  }
  const int n_tiles = (P.n_q + TQ - 1) / TQ;
  const cudaError_t e = launch_pdl(k_attn_tile, dim3(n_tiles * P.H), dim3(NTHR), SMEM_BYTES, s, P);
  count_launch();
  return e != cudaSuccess ? e : cudaGetLastError();
}

// Ps: device array of n AttnParams (copied by the caller), every call tile-eligible with
// the same n_q and heads.
cudaError_t launch_attn_tile_batched(const AttnParams& P0, const AttnParams* Ps_dev, int n,
                                     cudaStream_t s) {
  static bool attr_set[128] = {false};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 128) return cudaErrorInvalidDevice;
  if (!attr_set[dev]) {
    const cudaError_t e = cudaFuncSetAttribute(k_attn_tile_batched,
                                               cudaFuncAttributeMaxDynamicSharedMemorySize,
                                               (int)SMEM_BYTES);
    if (e != cudaSuccess) return e;
    attr_set[dev] = true;
  }
  const int per = ((P0.n_q + TQ - 1) / TQ) * P0.H;
  k_attn_tile_batched<<<(unsigned)((long long)per * n), NTHR, SMEM_BYTES, s>>>(Ps_dev, per);
  count_launch();
  return cudaGetLastError();
}

}  // namespace fl
