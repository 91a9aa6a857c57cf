// Loop-aware sparse attention on the tensor cores, one CTA per (head, tile of 128
// queries) (FlashLoop §4.2 "Loop-Aware Sparse Attention": each query attends to the
// columns its carried set names, softmax over them, rescaled by the cached mass, plus
// the carried unselected contribution; §4.4: the selected K/V are brought into compact
// on-chip buffers and QK^T / PV run on them).
//
// The queries of a tile carry different column sets. The CTA walks chunks of 128 columns
// and runs every chunk as a dense 128 x 128 tile on the tensor cores, each query's
// membership applied as a mask. Three modes:
//   CONTIG  chunks of the plain column range [0, t_max] of the tile - taken where the
//           tile's union is nearly every column (a budget that is a sizeable part of the
//           prompt); membership read from the bitmap of each query's set (16 bytes per
//           query and chunk), masked causally;
//   UNION   chunks of the union of the tile's sets (a bitmap over the tokens and prefix
//           popcounts for ranks); the producers turn the union's words and each query's
//           bitmap words over a chunk's span into its 128-bit mask;
//   DECODE  the union, the producers decoding K^ and V^ from the quantised store (int8
//           base plus the residual chain of every loop that rewrote the column, fmaf(code,
//           s, z) added in loop order) - for calls of one tile, where nothing is shared.
// In CONTIG and UNION the store has been staged once per call as fp16 rows (kv_stage.cu)
// and the producers gather a chunk's K^ and V^ rows with cp.async, 16 lanes per 256-byte
// row, into the 128-byte-swizzle K-major layout (K^ as [column][element], V^ the same and
// read as an MN-major operand). Roles:
//   producer warps (two groups of four, one per pipeline stage): the chunk's columns and
//     their rows, the column biases, the masks (UNION);
//   the MMA warp issues S = Q K^T into one of two TMEM score buffers and, once the softmax
//     has written P, O += P V^ into the TMEM output accumulator (tcgen05.mma kind::f16,
//     M 128, N 128, fp32 accumulation), each as soon as its barrier completes;
//   the softmax warps (thread = query row = TMEM lane) take one pass per chunk against a
//     running maximum, rescaling O only when it grows by more than 2^8 (P stays below 256
//     in fp16), and write P = 2^(s - max) as fp16; the row sum is taken over the fp16
//     values the MMA uses. At the end o = u + m * O / sum, with m the cached mass and u
//     the unselected contribution.
// Operand precision: q, K^, V^ and P enter the MMAs as fp16 (11 significant bits); sums
// are binary32. Every wait is bounded; a wait that runs out records FL_ERR_TIMEOUT, the
// CTA drains its MMAs, frees TMEM and returns.
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
constexpr uint32_t OFF_MASK = OFF_BIAS + 2 * TC * 4;     // [2][TQ] uint4: membership of a chunk
constexpr uint32_t SMEM_BYTES = OFF_MASK + 2 * TQ * 16 + 1024;

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

// Column of union rank R (R < n_union): the last bitmap word whose prefix <= R, then the
// bit within it; -1 for R >= U.
__device__ __forceinline__ int rank_column(const uint32_t* bits, const uint16_t* pre, int n_words,
                                           int U, int R) {
  if (R >= U) return -1;
  int lo = 0, hi = n_words - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if ((int)pre[mid] <= R) lo = mid;
    else hi = mid - 1;
  }
  uint32_t m = bits[lo];
  for (int k = R - (int)pre[lo]; k > 0 && m; --k) m &= m - 1u;
  return m ? lo * 32 + __ffs(m) - 1 : -1;
}

// The membership mask of union ranks [r0, r0 + TC) for a query whose set is the bitmap
// qbm: the union's words over the chunk's column span [c0, c1], each AND-ed with the
// query's word; every hit lands at its rank within the chunk (the union bits below it).
// The word loop has the same trip count on every lane.
__device__ __forceinline__ uint4 bitmap_chunk_mask(const uint32_t* bits, const uint32_t* qbm,
                                                   int c0, int c1, int t) {
  uint32_t m0 = 0u, m1 = 0u, m2 = 0u, m3 = 0u;
  const int wa = c0 >> 5, wb = c1 >> 5;
  int base = 0;
#pragma unroll 4
  for (int w = wa; w <= wb; ++w) {
    uint32_t ub = bits[w];
    if (w == wa) ub &= ~((1u << (c0 & 31)) - 1u);
    if (w == wb && (c1 & 31) != 31) ub &= (2u << (c1 & 31)) - 1u;
    // the query's words cover its own columns [0, t] only
    uint32_t qb = 0u;
    if (qbm && w <= (t >> 5)) {
      qb = __ldg(qbm + w);
      if (w == (t >> 5) && (t & 31) != 31) qb &= (2u << (t & 31)) - 1u;
    }
    uint32_t hit = ub & qb;
    while (hit) {
      const int b = __ffs(hit) - 1;
      hit &= hit - 1u;
      const int pos = base + __popc(ub & ((1u << b) - 1u));
      const uint32_t bit = 1u << (pos & 31);
      const int wd = pos >> 5;
      m0 |= wd == 0 ? bit : 0u; m1 |= wd == 1 ? bit : 0u;
      m2 |= wd == 2 ? bit : 0u; m3 |= wd == 3 ? bit : 0u;
    }
    base += __popc(ub);
  }
  return make_uint4(m0, m1, m2, m3);
}

// A query's carried set walked in column order (= union-rank order), 16 entries buffered
// and the next 16 requested ahead. Rows whose stride is a multiple of 8 are 16-byte
// aligned and read 8 entries per load; other strides entry by entry.
struct SetWalk {
  const uint16_t* row;
  int stride, vi, p;
  bool vec, ended;
  uint4 c0, c1, n0, n1;   // current 16 entries (two per word), the next 16
};

// entries 8 i .. 8 i + 7 of the row, sentinels beyond it
__device__ __forceinline__ uint4 set_vec(const SetWalk& w, int i) {
  constexpr uint32_t S2 = 0xFFFFFFFFu;   // two sentinels
  if (8 * i >= w.stride) return make_uint4(S2, S2, S2, S2);
  if (w.vec) return __ldg(reinterpret_cast<const uint4*>(w.row) + i);
  uint32_t e[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    const int j = 8 * i + k;
    e[k] = j < w.stride ? (uint32_t)__ldg(w.row + j) : (uint32_t)FL_SENTINEL;
  }
  return make_uint4(e[0] | e[1] << 16, e[2] | e[3] << 16, e[4] | e[5] << 16, e[6] | e[7] << 16);
}

__device__ __forceinline__ void set_init(SetWalk& w, const uint16_t* row, int stride, bool valid) {
  w.row = row;
  w.stride = valid ? stride : 0;
  w.vec = (stride & 7) == 0 && (reinterpret_cast<uintptr_t>(row) & 15) == 0;
  w.ended = !valid;
  w.c0 = set_vec(w, 0); w.c1 = set_vec(w, 1); w.n0 = set_vec(w, 2); w.n1 = set_vec(w, 3);
  w.vi = 4;
  w.p = 0;
}

__device__ __forceinline__ int set_entry(const SetWalk& w) {
  const uint4 v = w.p < 8 ? w.c0 : w.c1;
  const int q = (w.p >> 1) & 3;
  const uint32_t x = q == 0 ? v.x : (q == 1 ? v.y : (q == 2 ? v.z : v.w));
  return (int)((x >> ((w.p & 1) * 16)) & 0xFFFFu);
}

__device__ __forceinline__ void set_advance(SetWalk& w) {
  if (++w.p == 16) {
    w.c0 = w.n0; w.c1 = w.n1;
    w.n0 = set_vec(w, w.vi); w.n1 = set_vec(w, w.vi + 1);
    w.vi += 2;
    w.p = 0;
  }
}

// The membership mask of the chunk of union ranks [lo, lo + TC) for a query at position
// t: its entries in the chunk, walked on from where the previous call stopped. Entries
// that are not columns of the query (beyond t or the store) are recorded and skipped.
__device__ __forceinline__ uint4 walk_chunk(SetWalk& w, int t, int n_tok, int lo,
                                            const uint32_t* bits, const uint16_t* pre, int* st) {
  uint32_t m0 = 0u, m1 = 0u, m2 = 0u, m3 = 0u;
  while (!w.ended) {
    const int c = set_entry(w);
    if (c == (int)FL_SENTINEL) { w.ended = true; break; }
    if (c >= n_tok || c > t) {
      record_error(st, FL_ERR_RANGE);
      set_advance(w);
      continue;
    }
    const int r = union_rank(bits, pre, c) - lo;
    if (r >= TC) break;   // a later chunk's entry
    if (r >= 0) {
      const uint32_t bit = 1u << (r & 31);
      const int wd = r >> 5;
      m0 |= wd == 0 ? bit : 0u; m1 |= wd == 1 ? bit : 0u;
      m2 |= wd == 2 ? bit : 0u; m3 |= wd == 3 ? bit : 0u;
    }
    set_advance(w);
  }
  return make_uint4(m0, m1, m2, m3);
}

// One CTA: head h, the tile of queries starting at q0 of the call described by P.
// MODE: DECODE - chunks of the tile's union, K^ / V^ decoded from the store by the
// producers; UNION - chunks of the union, rows gathered from the staged fp16 rows;
// CONTIG - chunks of the plain column range [0, t_max] of the tile (for tiles whose union
// is nearly every column anyway: no union, no ranks), staged rows, and each query's
// membership read from the bitmap of its set (P.sel_bm).
enum TileMode : int { DECODE = 0, UNION = 1, CONTIG = 2 };
template <int MODE>
__device__ __forceinline__ void attn_tile_cta(const AttnParams& P, int h, int q0) {
  constexpr bool STAGED = MODE != DECODE;
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
    sh.n_union = -1;
    fence_barrier_init();
  }
  if (MODE != CONTIG)
    for (int w = threadIdx.x; w < n_words; w += NTHR) bits[w] = 0u;
  if (warp == 12) tmem_alloc(&sh.tmem, 512);
  griddep_wait();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sh.tmem;

  if constexpr (MODE == CONTIG) {   // the tile's column range: [0, largest position]
    if (threadIdx.x < TQ && q0 + (int)threadIdx.x < P.n_q) {
      const int t = P.q_tok[q0 + threadIdx.x];
      if (t >= 0 && t < n_tok) atomicMax(&sh.n_union, t);
    }
    __syncthreads();
    if (threadIdx.x == 0) sh.n_union += 1;
    __syncthreads();
  } else {
  const bool vec_rows = (stride & 7) == 0 && (reinterpret_cast<uintptr_t>(P.sel) & 15) == 0;
  // ---- the union of the tile's column sets (entries that are not valid columns of the
  // query - beyond its position or the store - are recorded and skipped here and below)
  for (int i = warp; i < TQ; i += NWARPS) {
    const int qi = q0 + i;
    if (qi >= P.n_q) break;
    const int t = P.q_tok[qi];
    const int srow = P.q_row ? P.q_row[qi] : t;
    if (t < 0 || t >= n_tok || srow < 0 || srow >= P.stat_rows) continue;
    const uint16_t* row = P.sel + ((size_t)h * P.stat_rows + srow) * stride;
    if (vec_rows) {   // 16-byte rows: 4 loads of 8 entries in flight per lane
      const uint4* rv = reinterpret_cast<const uint4*>(row);
      const int nv = stride >> 3;
      for (int v0 = 0; v0 < nv; v0 += 128) {
        uint4 w4[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const int vi = v0 + 32 * k + lane;
          w4[k] = vi < nv ? __ldg(rv + vi) : make_uint4(~0u, ~0u, ~0u, ~0u);
        }
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const uint32_t ws[4] = {w4[k].x, w4[k].y, w4[k].z, w4[k].w};
#pragma unroll
          for (int m = 0; m < 8; ++m) {
            const int c = (int)((ws[m >> 1] >> ((m & 1) * 16)) & 0xFFFFu);
            if (c != (int)FL_SENTINEL && c < n_tok && c <= t) atomicOr(&bits[c >> 5], 1u << (c & 31));
          }
        }
        if (__all_sync(0xffffffffu, (w4[3].w >> 16) == FL_SENTINEL)) break;   // padding reached
      }
      continue;
    }
    for (int e0 = 0; e0 < stride; e0 += 256) {   // 8 loads in flight per lane
      int c8[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const int e = e0 + 32 * k + lane;
        c8[k] = e < stride ? (int)__ldg(row + e) : (int)FL_SENTINEL;
      }
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const int c = c8[k];
        if (c != (int)FL_SENTINEL && c < n_tok && c <= t) atomicOr(&bits[c >> 5], 1u << (c & 31));
      }
      if (__all_sync(0xffffffffu, c8[7] == (int)FL_SENTINEL)) break;   // padding reached
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
  }
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
      // 32 elements per step, their loads issued together (read-only path)
#pragma unroll 1
      for (int e0 = 0; e0 < HDT; e0 += 32) {
        float x[32];
#pragma unroll
        for (int k = 0; k < 32; ++k) x[k] = 0.f;
        if (valid) {
          const size_t off = ((size_t)qi * H + h) * HDT + e0;
          if (P.q_bf16) {
            const uint4* qp = reinterpret_cast<const uint4*>(reinterpret_cast<const __nv_bfloat16*>(P.q) + off);
            uint4 w[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) w[k] = __ldg(qp + k);
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              const __nv_bfloat162* b2 = reinterpret_cast<const __nv_bfloat162*>(&w[k]);
#pragma unroll
              for (int m = 0; m < 4; ++m) { x[8 * k + 2 * m] = __low2float(b2[m]); x[8 * k + 2 * m + 1] = __high2float(b2[m]); }
            }
          } else {
            const float4* qp = reinterpret_cast<const float4*>(reinterpret_cast<const float*>(P.q) + off);
            float4 w[8];
#pragma unroll
            for (int k = 0; k < 8; ++k) w[k] = __ldg(qp + k);
#pragma unroll
            for (int k = 0; k < 8; ++k) { x[4 * k] = w[k].x; x[4 * k + 1] = w[k].y; x[4 * k + 2] = w[k].z; x[4 * k + 3] = w[k].w; }
          }
        }
#pragma unroll
        for (int k = 0; k < 4; ++k)
          *reinterpret_cast<uint4*>(qt + sw128_offset(i, e0 + 8 * k, TQ)) =
              make_uint4(pack_h2(x[8 * k], x[8 * k + 1]), pack_h2(x[8 * k + 2], x[8 * k + 3]),
                         pack_h2(x[8 * k + 4], x[8 * k + 5]), pack_h2(x[8 * k + 6], x[8 * k + 7]));
      }
      fence_proxy_async_smem();
    }
    // named barrier: Q written by the 4 softmax warps before the MMA warp issues QK
    asm volatile("bar.sync 1, %0;" ::"n"(5 * 32) : "memory");

    float m_used = -INFINITY, lsum = 0.f;
    const float m_in = valid ? P.mass[(size_t)h * P.stat_rows + srow] : 0.f;
    uint8_t* pt = smem + OFF_P;
    const uint4* maskbuf = reinterpret_cast<const uint4*>(smem + OFF_MASK);
    // CONTIG: this row's membership words, chunk by chunk, one chunk read ahead
    const uint4* bmrow = MODE == CONTIG && valid
        ? reinterpret_cast<const uint4*>(P.sel_bm + ((size_t)h * P.n_q + qi) * P.bm_words) : nullptr;
    uint4 mk_next = make_uint4(0u, 0u, 0u, 0u);
    if (MODE == CONTIG && bmrow && n_chunks > 0) mk_next = __ldg(bmrow);
    for (int c = 0; c < n_chunks; ++c) {   // leaves only through warp-uniform waits
      const int sb = c & 1;
      // waits agree across the warp: the TMEM loads below are warp-collective
      if (!warp_wait(&sh.s_full[sb], (c >> 1) & 1, abort, 101)) break;
      if (!warp_wait(&sh.meta_full[sb], (c >> 1) & 1, abort, 102)) break;
      tc_fence_after();
      uint4 mk;   // this row's members among the chunk's columns
      if constexpr (MODE == CONTIG) {
        // the bitmap covers the row's own columns: the words of later chunks are not its
        const int nin = valid ? min(max(t - c * TC + 1, 0), TC) : 0;
        mk = mk_next;
        if (bmrow && c + 1 < n_chunks) mk_next = __ldg(bmrow + c + 1);
        if (nin < TC) {
          const uint32_t m4[4] = {nin >= 32 ? ~0u : (nin > 0 ? (1u << nin) - 1u : 0u),
                                  nin >= 64 ? ~0u : (nin > 32 ? (1u << (nin - 32)) - 1u : 0u),
                                  nin >= 96 ? ~0u : (nin > 64 ? (1u << (nin - 64)) - 1u : 0u),
                                  nin > 96 ? (1u << (nin - 96)) - 1u : 0u};
          mk.x &= m4[0]; mk.y &= m4[1]; mk.z &= m4[2]; mk.w &= m4[3];
        }
      } else {
        mk = maskbuf[sb * TQ + i];
      }
      const uint32_t s_addr = tmem + lane_base + (uint32_t)(sb * TC);
      const float* bias = biasbuf + sb * TC;
      // columns in groups of 16 (16 TMEM words per load keeps the row in registers)
      auto mask16 = [&](int g) -> uint32_t {
        const uint32_t w = g < 2 ? mk.x : (g < 4 ? mk.y : (g < 6 ? mk.z : mk.w));
        return (w >> ((g & 1) * 16)) & 0xFFFFu;
      };
      // P of the previous chunk must have been consumed (and O completed) before P is
      // rewritten or O rescaled
      if (c > 0 && !warp_wait(&sh.pv_done, (c - 1) & 1, abort, 103)) break;
      tc_fence_after();
      // P = 2^(s - m_used) as fp16 into the P tile, the row sum over the fp16 values;
      // with `detect`, whether a member column lies more than 2^8 above m_used. The 16-word
      // loads of the next group fly while a group is processed.
      const float lsum0 = lsum;
      auto p_pass = [&](bool detect) -> bool {
        const float2 sc2 = make_float2(scale2, scale2);
        const float2 negm = make_float2(-m_used, -m_used);
        float2 acc = make_float2(0.f, 0.f);          // the row sum, two partial sums
        __half2 hmax = __float2half2_rn(0.f);         // largest P written (overflow check)
        auto group = [&](int g, const uint32_t (&r)[16]) {
          const uint32_t mw = mask16(g);
          uint32_t pk[8] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
          if (__any_sync(0xffffffffu, mw)) {
            const float2* b2 = reinterpret_cast<const float2*>(bias + g * 16);
#pragma unroll
            for (int j = 0; j < 16; j += 2) {
              // x = s * scale2 + bias, P = 2^(x - m_used) for a pair of columns
              const float2 x = __ffma2_rn(make_float2(__uint_as_float(r[j]), __uint_as_float(r[j + 1])),
                                          sc2, b2[j / 2]);
              const float2 d = __fadd2_rn(x, negm);
              // non-members at -inf: 2^-inf = 0
              const float da = (mw >> j) & 1u ? d.x : -INFINITY;
              const float db = (mw >> (j + 1)) & 1u ? d.y : -INFINITY;
              const __half2 ph = __floats2half2_rn(ex2_ftz(da), ex2_ftz(db));
              const uint32_t pv = *reinterpret_cast<const uint32_t*>(&ph);
              if (detect) hmax = __hmax2(hmax, ph);
              acc = __fadd2_rn(acc, __half22float2(ph));
              pk[j / 2] = pv;
            }
          }
#pragma unroll
          for (int q = 0; q < 2; ++q)
            *reinterpret_cast<uint4*>(pt + sw128_offset(i, g * 16 + q * 8, TQ)) =
                make_uint4(pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
        };
        uint32_t ra[16], rb[16];
        tmem_ld16_issue(s_addr, ra);
#pragma unroll 1
        for (int g = 0; g < 8; g += 2) {
          tmem_ld16_wait(ra);
          tmem_ld16_issue(s_addr + (g + 1) * 16, rb);
          group(g, ra);
          tmem_ld16_wait(rb);
          if (g + 2 < 8) tmem_ld16_issue(s_addr + (g + 2) * 16, ra);
          group(g + 1, rb);
        }
        lsum += acc.x + acc.y;
        // a member more than 2^8 above m_used: P above 256 (or infinite, m_used = -inf)
        const float2 hm = __half22float2(hmax);
        return detect && fmaxf(hm.x, hm.y) > 256.f;
      };
      // One pass against the running maximum. A row with a member more than 2^8 above it
      // (a P above 256 after fp16 rounding) takes the maximum of the chunk first (O and the
      // sum rescaled) and writes P again; the common case needs no maximum pass.
      if (__any_sync(0xffffffffu, p_pass(true))) {
        float cmax = -INFINITY;
#pragma unroll 1
        for (int g = 0; g < 8; ++g) {
          const uint32_t mw = mask16(g);
          if (!__any_sync(0xffffffffu, mw)) continue;   // no member in the warp's rows
          float v[16];
          tmem_ld16(s_addr + g * 16, v);
#pragma unroll
          for (int j = 0; j < 16; ++j)
            cmax = fmaxf(cmax, (mw >> j) & 1u ? fmaf(v[j], scale2, bias[g * 16 + j]) : -INFINITY);
        }
        float alpha = 1.f;
        bool rescale = false;
        if (cmax > m_used + kRescale) {
          if (m_used != -INFINITY && lsum0 > 0.f) { alpha = exp2f(m_used - cmax); rescale = true; }
          m_used = cmax;
        }
        lsum = rescale ? lsum0 * alpha : lsum0;
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
        p_pass(false);
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
        } else {   // nothing ready: yield the issue slots to the softmax warp of this SMSP
          if (*abort) break;
          __nanosleep(32);
          if (globaltimer() - t0 > kWaitLimitNs) {
            atomicCAS(const_cast<int*>(abort), 0, qk < n_chunks && qk <= pv + 1 ? 106 : 108);
            break;
          }
        }
      }
    }
    if (lane == 0) mma_commit(&sh.fin);   // arrives once every MMA issued above is done
  } else if constexpr (STAGED) {
    // ========================================== producers (rows from the staged store)
    // two groups of four warps, one per stage (chunk parity): the chunk's columns, their
    // K^ / V^ rows as asynchronous copies (16 lanes per row), the column biases, and in
    // UNION mode the membership masks of the tile's queries (lane jj walks the set of
    // query jj while the copies fly)
    const int grp = warp < 4 ? 0 : 1;
    const int jj = (warp & 3) * 32 + lane;
    uint8_t* k_tile = smem + OFF_K0 + 2 * grp * TILE;
    uint8_t* v_tile = k_tile + TILE;
    uint4* maskbuf = reinterpret_cast<uint4*>(smem + OFF_MASK) + grp * TQ;
    const size_t hoff = (size_t)h * n_tok * HDT;
    // UNION: query jj's bitmap row (invalid queries have none: recorded by the softmax)
    const uint32_t* qbm = nullptr;
    int tq = -1;
    if constexpr (MODE == UNION) {
      const int qi = q0 + jj;
      if (qi < P.n_q) {
        const int t = P.q_tok[qi];
        const int srow = P.q_row ? P.q_row[qi] : t;
        if (t >= 0 && t < n_tok && srow >= 0 && srow < P.stat_rows) {
          qbm = P.sel_bm + ((size_t)h * P.n_q + qi) * P.bm_words;
          tq = t;
        }
      }
    }
    for (int c = grp; c < n_chunks; c += 2) {
      if (__any_sync(0xffffffffu, *abort != 0)) break;   // warp-uniform exit
      if (c >= 2 && !warp_wait(&sh.kv_empty[grp], ((c >> 1) - 1) & 1, abort, 109)) break;
      const int col = MODE == CONTIG ? (c * TC + jj < U ? c * TC + jj : -1)
                                     : rank_column(bits, pre, n_words, U, c * TC + jj);
      copy_rows_warp(P.stage.khi + hoff, k_tile, col, (warp & 3) * 32, lane);
      copy_rows_warp(P.stage.vhi + hoff, v_tile, col, (warp & 3) * 32, lane);
      biasbuf[grp * TC + jj] = (col >= 0 && P.bias) ? __ldg(P.bias + col) * kLog2e : 0.f;
      if constexpr (MODE == UNION) {
        // the chunk's first and last columns (the same on every lane)
        const int c0 = rank_column(bits, pre, n_words, U, c * TC);
        const int c1 = rank_column(bits, pre, n_words, U, min(U, c * TC + TC) - 1);
        maskbuf[jj] = bitmap_chunk_mask(bits, qbm, c0, c1, tq);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&sh.meta_full[grp]);
      cp_async_wait_all();
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sh.kv_full[grp]);
    }
    cp_async_wait_all();   // nothing in flight when the CTA retires
  } else {
    // ================================================================ producer warps
    const int grp = warp < 4 ? 0 : 1;          // stage = chunk parity
    const int jj = (warp & 3) * 32 + lane;     // column of the chunk this lane decodes
    const float* bias_g = P.bias;
    uint8_t* k_tile = smem + OFF_K0 + 2 * grp * TILE;
    uint8_t* v_tile = k_tile + TILE;
    uint4* maskbuf = reinterpret_cast<uint4*>(smem + OFF_MASK) + grp * TQ;
    // this lane also walks the set of query jj of the tile, for the membership masks
    const int qi = q0 + jj;
    int t = -1, srow = 0;
    if (qi < P.n_q) {
      t = P.q_tok[qi];
      srow = P.q_row ? P.q_row[qi] : t;
      if (t < 0 || t >= n_tok || srow < 0 || srow >= P.stat_rows) t = -1;   // recorded by the softmax
    }
    SetWalk walk;
    set_init(walk, t >= 0 ? P.sel + ((size_t)h * P.stat_rows + srow) * stride : P.sel, stride, t >= 0);
    for (int c = grp; c < n_chunks; c += 2) {
      if (__any_sync(0xffffffffu, *abort != 0)) break;   // warp-uniform exit
      if (c >= 2 && !warp_wait(&sh.kv_empty[grp], ((c >> 1) - 1) & 1, abort, 109)) break;
      const int R = c * TC + jj;
      const int col = rank_column(bits, pre, n_words, U, R);
      biasbuf[grp * TC + jj] = (col >= 0 && bias_g) ? __ldg(bias_g + col) * kLog2e : 0.f;
      maskbuf[jj] = walk_chunk(walk, t, n_tok, c * TC, bits, pre, P.st);
      __syncwarp();
      if (lane == 0) mbar_arrive(&sh.meta_full[grp]);
      {   // decoded from the store
        uint32_t chain = 0;   // loops 2..loop that rewrote the column
        if (col >= 0)
          for (int r = 2; r <= P.loop; ++r)
            if (__ldg(P.kv.slot + (size_t)r * n_tok + col) >= 0) chain |= 1u << r;
        decode_column(P, 0, col, h, chain, k_tile, nullptr, jj);
        decode_column(P, 1, col, h, chain, v_tile, nullptr, jj);
      }
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

template <int MODE>
__global__ void __launch_bounds__(NTHR, 1) k_attn_tile(const __grid_constant__ AttnParams P) {
  const int n_tiles = (P.n_q + TQ - 1) / TQ;
  attn_tile_cta<MODE>(P, blockIdx.x / n_tiles, (blockIdx.x % n_tiles) * TQ);
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
  attn_tile_cta<DECODE>(sP, b / n_tiles, (b % n_tiles) * TQ);
}

// The bitmaps of the call's carried sets: one warp per (head, query) builds its row in
// shared memory (the set's entries OR-ed in, 16 per lane in flight), then writes it out.
// Only the words of the query's own columns are written (whole 128-column chunks up to
// its position); readers mask the columns beyond a query's position themselves. Entries
// beyond the query's position or the store are recorded (with `record`) and left out.
constexpr int BM_WARPS = 4;
__global__ void __launch_bounds__(BM_WARPS * 32) k_sel_bitmap(const AttnParams P, uint32_t* __restrict__ bm,
                                                               int record) {
  extern __shared__ uint32_t sbm[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long rh = (long long)blockIdx.x * BM_WARPS + warp;
  if (rh >= (long long)P.H * P.n_q) return;   // whole warp; no block barrier below
  griddep_wait();
  const int i = (int)(rh % P.n_q), h = (int)(rh / P.n_q);
  const int n_tok = P.kv.n_tok, stride = P.sel_stride;
  const int t = P.q_tok[i];
  const int srow = P.q_row ? P.q_row[i] : t;
  if (t < 0 || t >= n_tok || srow < 0 || srow >= P.stat_rows) return;   // recorded by the attention
  const int nw = min((t / TC + 1) * 4, P.bm_words);   // words of the query's chunks
  uint32_t* mine = sbm + (size_t)warp * P.bm_words;
  for (int w = lane; w < nw; w += 32) mine[w] = 0u;
  __syncwarp();
  const uint16_t* row = P.sel + ((size_t)h * P.stat_rows + srow) * stride;
  for (int e0 = 0; e0 < stride; e0 += 512) {
    int c16[16];
#pragma unroll
    for (int k = 0; k < 16; ++k) {
      const int e = e0 + 32 * k + lane;
      c16[k] = e < stride ? (int)__ldg(row + e) : (int)FL_SENTINEL;
    }
#pragma unroll
    for (int k = 0; k < 16; ++k) {
      const int c = c16[k];
      if (c == (int)FL_SENTINEL) continue;
      if (c <= t) atomicOr(&mine[c >> 5], 1u << (c & 31));
      else if (record) record_error(P.st, FL_ERR_RANGE);
    }
    if (__all_sync(0xffffffffu, c16[15] == (int)FL_SENTINEL)) break;   // padding reached
  }
  __syncwarp();
  uint4* dst = reinterpret_cast<uint4*>(bm + (size_t)rh * P.bm_words);
  const uint4* src = reinterpret_cast<const uint4*>(mine);
  for (int w = lane; w < nw / 4; w += 32) dst[w] = src[w];
}

}  // namespace

bool sparse_contig(const AttnParams& P) {
  return (size_t)P.sel_stride * 16 >= (size_t)P.kv.n_tok;
}

static int bm_words_of(const AttnParams& P) { return (P.kv.n_tok + TC - 1) / TC * 4; }

size_t sel_bitmap_bytes(const AttnParams& P) {
  return (size_t)P.H * P.n_q * bm_words_of(P) * sizeof(uint32_t);
}

cudaError_t launch_sel_bitmap(AttnParams& P, void* buf, cudaStream_t s, bool record) {
  P.bm_words = bm_words_of(P);
  P.sel_bm = static_cast<const uint32_t*>(buf);
  const long long rows = (long long)P.H * P.n_q;
  if (rows <= 0) return cudaSuccess;
  const size_t smem = (size_t)BM_WARPS * P.bm_words * sizeof(uint32_t);   // <= 32 KB
  const cudaError_t e = launch_pdl(k_sel_bitmap, dim3((unsigned)((rows + BM_WARPS - 1) / BM_WARPS)),
                                   dim3(BM_WARPS * 32), smem, s, P, static_cast<uint32_t*>(buf),
                                   record ? 1 : 0);
  count_launch();
  return e != cudaSuccess ? e : cudaGetLastError();
}

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
    for (auto k : {k_attn_tile<DECODE>, k_attn_tile<UNION>, k_attn_tile<CONTIG>}) {
      const cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                 (int)SMEM_BYTES);
      if (e != cudaSuccess) return e;
    }
    attr_set[dev] = true;
  }
  const int n_tiles = (P.n_q + TQ - 1) / TQ;
  auto kern = !P.stage.khi || !P.sel_bm ? k_attn_tile<DECODE>
                                        : (sparse_contig(P) ? k_attn_tile<CONTIG> : k_attn_tile<UNION>);
  const cudaError_t e = launch_pdl(kern, dim3(n_tiles * P.H), dim3(NTHR), SMEM_BYTES, s, P);
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
