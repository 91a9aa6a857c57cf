// Dense causal attention and the column statistics it hands to the next loop, on the
// tensor cores, one CTA per (head, tile of 128 queries) (FlashLoop §4.2 "Loop-Aware
// Sparse Attention": the sparse loops rank columns by statistics of the previous loop;
// a dense loop is where they are produced).
//
// Statistics for query i (t = its position, k = the next loop's budget, t > k):
//   S' = {0} U top-k over j in [1, t] of c_j = p_j ||V^_j|| (or p_j), ties to the smaller
//   column; m' = sum over S' of p_j; u' = sum over the other columns of p_j V^_j.
// The ranking of a row depends on s_j + log ||V^_j|| alone, so it is taken in four steps:
//   kernel A, three passes over the tile's column chunks (the same producer / MMA / softmax
//   pipeline as the sparse tile kernel; columns are the contiguous range [0, t_max]):
//     flash  S = Q K^T (fp16 operands), online softmax with a causal mask, O += P V^
//            -> o = O / sum, and the row's final maximum and sum;
//     hist   S again (fp16): a 128-bin histogram per row of kappa_j = s_j + log2 ||V^_j||,
//            1/8 log2 unit per bin below the row's upper bound (final maximum + the
//            largest log2 ||V^|| the row saw) -> the bin holding the k-th largest, and a
//            threshold one margin below it (the margin bounds the fp16 score error);
//     cand   S with split operands (q = hi + lo, K^ = hi + lo, fp16 each; three MMAs,
//            22 significant bits, binary32 sums): every column with kappa at or above the
//            threshold is a candidate - written with its p_j to a per-row buffer;
//   kernel B (one CTA per row and head): exact top-k of c_j = p_j ||V^_j|| among the
//     candidates (radix select on the binary32 bits, equal values to the smaller column),
//     S' written ascending, m' = p_0 + sum of the kept p_j;
//   kernel C, one pass: S (fp16), p_j = 2^(s_j - max) / sum with the row's final maximum
//     and sum, and u' = sum over the columns outside S' of p_j V^_j (P V^ on the tensor
//     cores with the complement of S' as the mask).
// A row whose candidates overflow its buffer (a near-uniform row of more than the buffer's
// spare capacity in one histogram bin) is finished by the exact per-query kernel.
// Every wait is bounded; a wait that runs out records FL_ERR_TIMEOUT, the CTA drains its
// MMAs, frees TMEM and returns. Warp-collective TMEM accesses stay warp-uniform. The
// softmax hands each score buffer back on a barrier of its own: in the passes without
// P V^ nothing else keeps the four softmax warps in step, and with one shared barrier a
// warp running a chunk ahead would complete the previous chunk's phase early.
#include <float.h>

#include "attn_tile_common.cuh"

namespace fl {
namespace {

using namespace sm100;
using namespace tile;

constexpr int NWARPS = 13;         // 0-3, 8-11 producers; 4-7 softmax; 12 MMA
constexpr int NTHR = NWARPS * 32;
constexpr int NBIN = 128;          // histogram bins per row
constexpr float kBinsPerLog2 = 8.f;
constexpr float kMargin = 1.f / 64;   // log2 units; fp16 scores differ by far less

enum : int { PASS_FLASH = 0, PASS_HIST = 1, PASS_CAND = 2, PASS_UNSEL = 3 };

// dynamic shared memory (1024-byte aligned base)
constexpr uint32_t OFF_QHI = 0;
constexpr uint32_t OFF_R1 = OFF_QHI + TILE;      // P | histogram [NBIN][TQ] u16 | Q lo
constexpr uint32_t OFF_ST = OFF_R1 + TILE;       // stage s: tile A at OFF_ST + 2 s TILE, B after
// [2][TC] bias (log2 units), [2][TC] log2 ||V^||, [2][TC] their sum, [2][4] the four
// producer warps' largest log2 ||V^|| of the chunk
constexpr uint32_t OFF_META = OFF_ST + 4 * TILE;
constexpr uint32_t SMEM_BYTES = OFF_META + (6 * TC + 8) * 4 + 1024;
static_assert(NBIN * TQ * 2 <= TILE, "histogram fits its region");

struct DenseArgs {
  AttnParams P;
  int mode;          // 0: flash only, 1: flash + hist + cand, 2: unselected pass
  int k;             // the next loop's budget
  int cap;           // candidates per row
  float2* m1l;       // [H][n_q] (final maximum, log2 units; sum)
  int* dbg;          // [grid][12] a CTA whose wait ran out: site, chunks, t_max, progress
  int* cnt;          // [H][n_q] candidates written (> cap: overflow)
  float* p0;         // [H][n_q] p of the sink column
  uint16_t* ccol;    // [H][n_q][cap]
  float* cp;         // [H][n_q][cap]
};

struct DenseShared {
  uint64_t kv_full[2], kv_empty[2], meta_full[2], s_full[2], p_full[2], pv_done, qlo_ready, hist_done,
      fin;
  uint32_t tmem;
  int abort_flag;
  int t_max;
  int prog[8];   // progress: softmax warps' last chunk step, MMA's, producer groups', hist arrivals
};

// code of a wait for the timeout report: the site, the chunk step and the warp
__device__ __forceinline__ int site_of(int site, int G, int warp) {
  return site | (min(G, 4095) << 8) | ((warp & 15) << 20);
}

__device__ __forceinline__ int pass_of(int mode, int G, int nc) {
  if (mode == 2) return PASS_UNSEL;
  if (mode == 0) return PASS_FLASH;
  const int p = G / nc;
  return p == 0 ? PASS_FLASH : (p == 1 ? PASS_HIST : PASS_CAND);
}
__device__ __forceinline__ bool has_pv(int pass) { return pass == PASS_FLASH || pass == PASS_UNSEL; }

// the query row (fp32 or bf16) as 8 binary32 values from element e0
__device__ __forceinline__ void load_q8(const AttnParams& P, int qi, int h, int e0, float* x) {
  const size_t off = ((size_t)qi * P.H + h) * HDT + e0;
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

// STAGED: operand rows gathered from the staged fp16 rows (P.stage), else decoded from
// the store by the producers.
template <bool STAGED>
__global__ void __launch_bounds__(NTHR, 1) k_attn_dense_tile(const __grid_constant__ DenseArgs A) {
  const AttnParams& P = A.P;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  __shared__ DenseShared sh;
  volatile int* abort = &sh.abort_flag;
  float* meta = reinterpret_cast<float*>(smem + OFF_META);   // bias [2][TC], lvn [2][TC]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int H = P.H, n_tok = P.kv.n_tok;
  const int n_tiles = (P.n_q + TQ - 1) / TQ;
  const int h = blockIdx.x / n_tiles;
  const int q0 = (blockIdx.x % n_tiles) * TQ;
  const int mode = A.mode;
  const bool stats = mode == 1;

  if (threadIdx.x == 0) {
    for (int s = 0; s < 2; ++s) {
      mbar_init(&sh.kv_full[s], 4); mbar_init(&sh.kv_empty[s], 1);
      mbar_init(&sh.meta_full[s], 4); mbar_init(&sh.s_full[s], 1);
    }
    mbar_init(&sh.p_full[0], TQ);
    mbar_init(&sh.p_full[1], TQ);
    mbar_init(&sh.pv_done, 1);
    mbar_init(&sh.qlo_ready, TQ);
    mbar_init(&sh.hist_done, TQ);
    mbar_init(&sh.fin, 1);
    sh.abort_flag = 0;
    sh.t_max = -1;
    for (int k = 0; k < 8; ++k) sh.prog[k] = -1;
    sh.prog[7] = 0;
    fence_barrier_init();
  }
  if (warp == 12) tmem_alloc(&sh.tmem, 512);
  griddep_wait();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sh.tmem;
  if (threadIdx.x < TQ && q0 + (int)threadIdx.x < P.n_q) {
    const int t = P.q_tok[q0 + threadIdx.x];
    if (t >= 0 && t < n_tok) atomicMax(&sh.t_max, t);
  }
  __syncthreads();
  const int t_max = sh.t_max;
  const int nc = (t_max + TC) / TC;                  // chunks covering [0, t_max]
  const int n_pass = stats ? 3 : 1;
  const int total = t_max < 0 ? 0 : nc * n_pass;
  const float scale2 = P.scale * kLog2e;
  const uint32_t idesc = idesc_f16_f32(TQ, TC);
  const uint32_t idesc_pv = idesc_f16_f32_bmn(TQ, HDT);   // V^ tiles are MN-major

  if (warp >= 4 && warp < 8) {
    // ================================================================ softmax warps
    const int i = (warp - 4) * 32 + lane;
    const int qi = q0 + i;
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
    bool valid = qi < P.n_q;
    int t = -1, srow = 0;
    if (valid) {
      t = P.q_tok[qi];
      srow = P.q_row ? P.q_row[qi] : t;
      const bool row_ok = mode == 2 ? (srow >= 0 && srow < P.stat_rows) : true;
      if (t < 0 || t >= n_tok || !row_ok) {
        record_error(P.st, FL_ERR_RANGE);
        valid = false;
        t = -1;
      }
    }
    const size_t rh = (size_t)h * P.n_q + (valid ? qi : 0);
    // Q (hi part: fp16 of q) for every pass
    {
      uint8_t* qt = smem + OFF_QHI;
      for (int e0 = 0; e0 < HDT; e0 += 8) {
        float x[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) x[k] = 0.f;
        if (valid) load_q8(P, qi, h, e0, x);
        *reinterpret_cast<uint4*>(qt + sw128_offset(i, e0, TQ)) =
            make_uint4(pack_h2(x[0], x[1]), pack_h2(x[2], x[3]), pack_h2(x[4], x[5]), pack_h2(x[6], x[7]));
      }
      fence_proxy_async_smem();
    }
    asm volatile("bar.sync 1, %0;" ::"n"(5 * 32) : "memory");

    // unselected pass: the row's final maximum and sum; S' read as a bitmap of columns
    float m_used = -INFINITY, lsum = 0.f;
    const uint4* bmrow = nullptr;
    uint4 sw_next = make_uint4(0u, 0u, 0u, 0u);   // S' words of the next chunk, read ahead
    if (mode == 2 && valid) {
      const float2 ml = A.m1l[rh];
      m_used = ml.x;
      lsum = ml.y;
      bmrow = reinterpret_cast<const uint4*>(P.sel_bm + ((size_t)h * P.n_q + qi) * P.bm_words);
      if (nc > 0) sw_next = __ldg(bmrow);
    }
    const bool sel_row_stats = stats && valid && t > A.k;   // rows that rank columns
    // m_used: the reference of P and the sum (raised only by more than 2^8); m_true: the
    // running maximum (up to the fp16 rounding of P), which anchors the histogram
    float m_true = -INFINITY, lvmax = -INFINITY, ktop = 0.f, thr = -INFINITY, p0 = 0.f;
    int cand = 0;
    uint16_t* hist = reinterpret_cast<uint16_t*>(smem + OFF_R1);
    uint8_t* pt = smem + OFF_R1;
    const bool pv_stat = P.stat_kind == FL_STAT_PV;
    const float2 sc2 = make_float2(scale2, scale2);

    // P = 2^(x - m_used) (x = s * scale2 + bias) as fp16 into the P tile for the columns of
    // the 16-column groups' masks mask16(g); the row sum over the fp16 values when `sum`;
    // the largest P written (in fp16) is returned. TMEM loads of the next group fly while
    // a group is processed.
    auto p_pass = [&](uint32_t s_addr, const float* bias, auto mask16, bool sum) -> float {
      const float2 negm = make_float2(-m_used, -m_used);
      float2 acc = make_float2(0.f, 0.f);
      __half2 hmax = __float2half2_rn(0.f);
      auto group = [&](int g, const uint32_t (&r)[16]) {
        const uint32_t mw = mask16(g);
        uint32_t pk[8] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
        if (__any_sync(0xffffffffu, mw)) {
          const float2* b2 = reinterpret_cast<const float2*>(bias + g * 16);
#pragma unroll
          for (int j = 0; j < 16; j += 2) {
            const float2 x = __ffma2_rn(make_float2(__uint_as_float(r[j]), __uint_as_float(r[j + 1])),
                                        sc2, b2[j / 2]);
            const float2 d = __fadd2_rn(x, negm);
            // non-members at -inf: 2^-inf = 0
            const float da = (mw >> j) & 1u ? d.x : -INFINITY;
            const float db = (mw >> (j + 1)) & 1u ? d.y : -INFINITY;
            const __half2 ph = __floats2half2_rn(ex2_ftz(da), ex2_ftz(db));
            const uint32_t pv = *reinterpret_cast<const uint32_t*>(&ph);
            hmax = __hmax2(hmax, ph);
            if (sum) acc = __fadd2_rn(acc, __half22float2(ph));
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
      if (sum) lsum += acc.x + acc.y;
      const float2 hm = __half22float2(hmax);
      return fmaxf(hm.x, hm.y);
    };
    // causal columns of a 16-column group: [0, nin) of the chunk
    auto causal16 = [](int g, int nin) -> uint32_t {
      const int n = nin - g * 16;
      return n >= 16 ? 0xFFFFu : (n > 0 ? (1u << n) - 1u : 0u);
    };
    // fn(g, r) for the chunk's eight 16-column groups of S, the loads of the next group
    // flying while a group is processed (every lane runs it: the loads are warp-collective)
    auto for_groups = [&](uint32_t s_addr, auto fn) {
      uint32_t ra[16], rb[16];
      tmem_ld16_issue(s_addr, ra);
#pragma unroll 1
      for (int g = 0; g < 8; g += 2) {
        tmem_ld16_wait(ra);
        tmem_ld16_issue(s_addr + (g + 1) * 16, rb);
        fn(g, ra);
        tmem_ld16_wait(rb);
        if (g + 2 < 8) tmem_ld16_issue(s_addr + (g + 2) * 16, ra);
        fn(g + 1, rb);
      }
    };

    for (int G = 0; G < total; ++G) {
      const int pass = pass_of(mode, G, nc);
      const int c = G % nc;
      const int sb = G & 1;
      if (!warp_wait(&sh.s_full[sb], (G >> 1) & 1, abort, site_of(1 + 16 * mode, G, warp))) break;
      if (!warp_wait(&sh.meta_full[sb], (G >> 1) & 1, abort, site_of(2 + 16 * mode, G, warp))) break;
      tc_fence_after();
      const uint32_t s_addr = tmem + lane_base + (uint32_t)(sb * TC);
      const float* bias = meta + sb * TC;
      const float* lvn = meta + 2 * TC + sb * TC;
      const float* blv = meta + 4 * TC + sb * TC;           // bias + log2 ||V^||
      const int nin = t < 0 ? 0 : min(max(t - c * TC + 1, 0), TC);   // causal columns
      if (pass == PASS_FLASH) {
        // the largest log2 ||V^|| the row saw: the chunk's (producers) or, on the diagonal
        // chunk, over the row's own columns
        if (stats) {
          if (nin == TC) {
            const float* lm = meta + 6 * TC + sb * 4;
            lvmax = fmaxf(lvmax, fmaxf(fmaxf(lm[0], lm[1]), fmaxf(lm[2], lm[3])));
          } else {
            for (int jj = 0; jj < nin; ++jj) lvmax = fmaxf(lvmax, lvn[jj]);
          }
        }
        if (c > 0 && !warp_wait(&sh.pv_done, (c - 1) & 1, abort, site_of(3 + 16 * mode, G, warp))) break;
        tc_fence_after();
        // one pass against the running maximum; a row whose P exceeds 2^8 (a column more
        // than 8 above m_used, or the first chunk) takes the chunk's maximum first (O and
        // the sum rescaled) and writes P again
        const float lsum0 = lsum;
        auto mk = [&](int g) { return causal16(g, nin); };
        const float pmax = p_pass(s_addr, bias, mk, true);
        const bool over = pmax > 256.f;
        if (!over && pmax > 0.f) m_true = fmaxf(m_true, m_used + log2f(pmax) + 1.f / 1024);
        if (__any_sync(0xffffffffu, over)) {
          float cmax = -INFINITY;
#pragma unroll 1
          for (int g = 0; g < 8; ++g) {
            const uint32_t mw = causal16(g, nin);
            if (!__any_sync(0xffffffffu, mw)) continue;
            float v[16];
            tmem_ld16(s_addr + g * 16, v);
#pragma unroll
            for (int j = 0; j < 16; ++j)
              cmax = fmaxf(cmax, (mw >> j) & 1u ? fmaf(v[j], scale2, bias[g * 16 + j]) : -INFINITY);
          }
          m_true = fmaxf(m_true, cmax);
          float alpha = 1.f;
          bool rescale = false;
          if (cmax > m_used + kRescale) {
            if (m_used != -INFINITY && lsum0 > 0.f) { alpha = exp2f(m_used - cmax); rescale = true; }
            m_used = cmax;
          }
          lsum = rescale ? lsum0 * alpha : lsum0;
          if (__any_sync(0xffffffffu, rescale)) {
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
          p_pass(s_addr, bias, mk, true);
        }
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(&sh.p_full[sb]);   // one barrier per score buffer (see the header)
        if (lane == 0) sh.prog[warp - 4] = G;
        if (c == nc - 1) {
          // ---- end of the flash pass: o = O / sum; the row's maximum and sum
          if (!warp_wait(&sh.pv_done, (nc - 1) & 1, abort, site_of(4 + 16 * mode, G, warp))) break;
          tc_fence_after();
          const uint32_t o_addr = tmem + lane_base + 2u * TC;
          const float f = (valid && lsum > 0.f) ? 1.f / lsum : 0.f;
          const size_t ob = ((size_t)qi * H + h) * HDT;
#pragma unroll 1
          for (int g4 = 0; g4 < 4; ++g4) {
            float v[32];
            tmem_ld32(o_addr + g4 * 32, v);
            if (!valid) continue;
#pragma unroll
            for (int j = 0; j < 32; j += 4) {
              const float o0 = v[j] * f, o1 = v[j + 1] * f, o2 = v[j + 2] * f, o3 = v[j + 3] * f;
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
          if (stats) {
            if (valid) A.m1l[rh] = make_float2(m_used, lsum);
            ktop = m_true + (pv_stat ? lvmax : 0.f);
            // the histogram takes the P region over (every thread saw the last P V^ finish)
            for (int b = 0; b < NBIN; ++b) hist[b * TQ + i] = 0;
          }
        }
      } else if (pass == PASS_HIST) {
        {
          // kappa = s * scale2 + bias + log2 ||V^|| binned by (ktop - kappa) * 8 below the
          // row's upper bound; each thread counts its own row's bins (16-bit counts in
          // shared memory, no atomics); rows that rank nothing have empty masks
          const float kt8 = ktop * kBinsPerLog2;
          const float2 nb2 = make_float2(-kBinsPerLog2, -kBinsPerLog2);
          uint16_t* hrow = hist + i;
          const float* kb = pv_stat ? blv : bias;
          for_groups(s_addr, [&](int g, const uint32_t (&r)[16]) {
            uint32_t mw = sel_row_stats ? causal16(g, nin) : 0u;
            if (c == 0 && g == 0) mw &= ~1u;   // the sink is kept apart
            if (!__any_sync(0xffffffffu, mw)) return;
            const float2* b2 = reinterpret_cast<const float2*>(kb + g * 16);
#pragma unroll
            for (int j = 0; j < 16; j += 2) {
              const float2 kap = __ffma2_rn(make_float2(__uint_as_float(r[j]), __uint_as_float(r[j + 1])),
                                            sc2, b2[j / 2]);
              const float2 bf = __ffma2_rn(kap, nb2, make_float2(kt8, kt8));
              // NaN-free: kappa finite or -inf
              const int ba = (int)fminf(fmaxf(bf.x, 0.f), (float)(NBIN - 1));
              const int bb = (int)fminf(fmaxf(bf.y, 0.f), (float)(NBIN - 1));
              if ((mw >> j) & 1u) hrow[ba * TQ] += 1;
              if ((mw >> (j + 1)) & 1u) hrow[bb * TQ] += 1;
            }
          });
        }
        tc_fence_before();
        mbar_arrive(&sh.p_full[sb]);   // one barrier per score buffer (see the header)
        if (lane == 0) sh.prog[warp - 4] = G;
        if (c == nc - 1) {
          __syncwarp();
          // ---- the bin of the k-th largest; the candidate threshold one margin below it
          if (sel_row_stats) {
            int acc = 0, b = 0;
            for (; b < NBIN - 1; ++b) {
              acc += hist[b * TQ + i];
              if (acc >= A.k) break;
            }
            thr = b >= NBIN - 1 ? -INFINITY : ktop - (float)(b + 1) / kBinsPerLog2 - kMargin;
          }
          // every row's histogram read: the region becomes Q lo (a bounded wait, not a
          // named barrier, so an aborted warp cannot hold the others)
          mbar_arrive(&sh.hist_done);
          atomicAdd(&sh.prog[7], 1);
          if (!warp_wait(&sh.hist_done, 0, abort, site_of(5 + 16 * mode, G, warp))) break;
          uint8_t* ql = smem + OFF_R1;
          for (int e0 = 0; e0 < HDT; e0 += 8) {
            float x[8];
#pragma unroll
            for (int k = 0; k < 8; ++k) x[k] = 0.f;
            if (valid) load_q8(P, qi, h, e0, x);
#pragma unroll
            for (int k = 0; k < 8; ++k) x[k] = x[k] - __half2float(__float2half_rn(x[k]));
            *reinterpret_cast<uint4*>(ql + sw128_offset(i, e0, TQ)) =
                make_uint4(pack_h2(x[0], x[1]), pack_h2(x[2], x[3]), pack_h2(x[4], x[5]), pack_h2(x[6], x[7]));
          }
          fence_proxy_async_smem();
          mbar_arrive(&sh.qlo_ready);
        }
      } else if (pass == PASS_CAND) {
        // the columns at or above the threshold (kappa from the split-operand scores) are
        // candidates, written in column order with p = 2^(x - max) / sum; the sink apart
        const float inv_l = lsum > 0.f ? 1.f / lsum : 0.f;
        uint16_t* ccol = A.ccol + rh * A.cap;
        float* cpr = A.cp + rh * A.cap;
        for_groups(s_addr, [&](int g, const uint32_t (&r)[16]) {
          const uint32_t mw = sel_row_stats ? causal16(g, nin) : 0u;
          if (!__any_sync(0xffffffffu, mw)) return;
          const float2* b2 = reinterpret_cast<const float2*>(bias + g * 16);
          const float2* l2 = reinterpret_cast<const float2*>(lvn + g * 16);
          float x[16];
          uint32_t hits = 0u;
#pragma unroll
          for (int j = 0; j < 16; j += 2) {
            const float2 xx = __ffma2_rn(make_float2(__uint_as_float(r[j]), __uint_as_float(r[j + 1])),
                                         sc2, b2[j / 2]);
            const float2 kap = pv_stat ? __fadd2_rn(xx, l2[j / 2]) : xx;
            x[j] = xx.x;
            x[j + 1] = xx.y;
            hits |= (kap.x >= thr ? 1u : 0u) << j;
            hits |= (kap.y >= thr ? 1u : 0u) << (j + 1);
          }
          hits &= mw;
          if (c == 0 && g == 0 && (mw & 1u)) {
            p0 = exp2f(x[0] - m_used) * inv_l;
            hits &= ~1u;
          }
          while (hits) {
            const int j = __ffs(hits) - 1;
            hits &= hits - 1u;
            float xj = x[0];
#pragma unroll
            for (int q = 1; q < 16; ++q) xj = j == q ? x[q] : xj;   // select, no local memory
            if (cand < A.cap) {
              ccol[cand] = (uint16_t)(c * TC + g * 16 + j);
              cpr[cand] = exp2f(xj - m_used) * inv_l;
            }
            ++cand;
          }
        });
        tc_fence_before();
        mbar_arrive(&sh.p_full[sb]);   // one barrier per score buffer (see the header)
        if (lane == 0) sh.prog[warp - 4] = G;
        if (c == nc - 1 && sel_row_stats) {
          A.cnt[rh] = cand;
          A.p0[rh] = p0;
        }
      } else {   // PASS_UNSEL: u' over the causal columns outside S'
        const uint4 sw = sw_next;   // S' among the chunk's columns
        if (bmrow && c + 1 < nc) sw_next = __ldg(bmrow + c + 1);
        if (c > 0 && !warp_wait(&sh.pv_done, (c - 1) & 1, abort, site_of(11 + 16 * mode, G, warp))) break;
        tc_fence_after();
        auto mk = [&](int g) -> uint32_t {
          const uint32_t w = g < 2 ? sw.x : (g < 4 ? sw.y : (g < 6 ? sw.z : sw.w));
          return causal16(g, nin) & ~((w >> ((g & 1) * 16)) & 0xFFFFu);
        };
        p_pass(s_addr, bias, mk, false);
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(&sh.p_full[sb]);   // one barrier per score buffer (see the header)
        if (lane == 0) sh.prog[warp - 4] = G;
        if (c == nc - 1) {
          if (!warp_wait(&sh.pv_done, (nc - 1) & 1, abort, site_of(12 + 16 * mode, G, warp))) break;
          tc_fence_after();
          const uint32_t o_addr = tmem + lane_base + 2u * TC;
          const float f = (valid && lsum > 0.f) ? 1.f / lsum : 0.f;
          float* u = valid ? P.unsel_out + ((size_t)h * P.stat_rows + srow) * HDT : nullptr;
#pragma unroll 1
          for (int g4 = 0; g4 < 4; ++g4) {
            float v[32];
            tmem_ld32(o_addr + g4 * 32, v);
            if (!valid) continue;
#pragma unroll
            for (int j = 0; j < 32; j += 4)
              *reinterpret_cast<float4*>(u + g4 * 32 + j) =
                  make_float4(v[j] * f, v[j + 1] * f, v[j + 2] * f, v[j + 3] * f);
          }
        }
      }
    }
  } else if (warp == 12) {
    // ================================================================ MMA warp
    asm volatile("bar.sync 1, %0;" ::"n"(5 * 32) : "memory");
    if (lane == 0 && total > 0) {
      const uint32_t qh = smem_u32(smem + OFF_QHI);
      const uint32_t r1 = smem_u32(smem + OFF_R1);
      bool qlo_seen = false;
      // Issue whichever MMA is ready: QK^T of the next chunk once its operands are decoded
      // and its score buffer is free (the softmax handed back chunk G - 2), the hand-back of
      // the oldest chunk (P V^ where the pass has one, then the stage release) once the
      // softmax is done with it. Neither waits on the other.
      int qk = 0, pv = 0;
      uint64_t t0 = globaltimer();
      while (pv < total) {
        bool prog = false;
        if (qk < total && qk <= pv + 1 && mbar_test_wait(&sh.kv_full[qk & 1], (qk >> 1) & 1)) {
          const int pass = pass_of(mode, qk, nc);
          if (pass == PASS_CAND && !qlo_seen) qlo_seen = mbar_test_wait(&sh.qlo_ready, 0);
          if (pass != PASS_CAND || qlo_seen) {
            tc_fence_after();
            const int st = qk & 1;
            const uint32_t a_t = smem_u32(smem + OFF_ST + 2 * st * TILE);
            const uint32_t b_t = a_t + TILE;
            const uint32_t d = tmem + (uint32_t)(st * TC);
#pragma unroll
            for (int kk = 0; kk < HDT / 16; ++kk) {
              const uint32_t off = (kk >> 2) * (TQ * 128) + (kk & 3) * 32;
              mma_bf16(d, desc_sw128_kmajor(qh + off), desc_sw128_kmajor(a_t + off), idesc,
                       kk > 0 ? 1u : 0u);
              if (pass == PASS_CAND) {   // q_hi K_lo + q_lo K_hi
                mma_bf16(d, desc_sw128_kmajor(qh + off), desc_sw128_kmajor(b_t + off), idesc, 1u);
                mma_bf16(d, desc_sw128_kmajor(r1 + off), desc_sw128_kmajor(a_t + off), idesc, 1u);
              }
            }
            mma_commit(&sh.s_full[st]);
            ++qk;
            prog = true;
          }
        }
        if (pv < qk && mbar_test_wait(&sh.p_full[pv & 1], (pv >> 1) & 1)) {
          tc_fence_after();
          const int pass = pass_of(mode, pv, nc);
          if (has_pv(pass)) {
            const int st = pv & 1, c = pv % nc;
            const uint32_t v_t = smem_u32(smem + OFF_ST + (2 * st + 1) * TILE);
            const uint32_t d = tmem + 2u * TC;
#pragma unroll
            for (int kk = 0; kk < TC / 16; ++kk) {
              const uint32_t off = (kk >> 2) * (TQ * 128) + (kk & 3) * 32;
              mma_bf16(d, desc_sw128_kmajor(r1 + off), desc_sw128_mnmajor(v_t + kk * 2048, TC),
                       idesc_pv, (c > 0 || kk > 0) ? 1u : 0u);
            }
            mma_commit(&sh.pv_done);
          }
          // the stage (operand tiles and its column metadata) is free once the softmax has
          // handed the chunk back - also in passes without P V^, whose metadata it reads
          mma_commit(&sh.kv_empty[pv & 1]);
          sh.prog[4] = pv;
          ++pv;
          prog = true;
        }
        if (prog) {
          t0 = globaltimer();
        } else {   // nothing ready: yield the issue slots to the softmax warp of this SMSP
          if (*abort) break;
          __nanosleep(32);
          if (globaltimer() - t0 > kWaitLimitNs) {
            const bool want_qk = qk < total && qk <= pv + 1;
            atomicCAS(const_cast<int*>(abort), 0,
                      site_of((want_qk ? 6 : 8) + 16 * mode, want_qk ? qk : pv, warp));
            break;
          }
        }
      }
    }
    if (lane == 0) mma_commit(&sh.fin);
  } else {
    // ================================================================ producer warps
    const int grp = warp < 4 ? 0 : 1;
    const int jj = (warp & 3) * 32 + lane;
    uint8_t* a_tile = smem + OFF_ST + 2 * grp * TILE;
    uint8_t* b_tile = a_tile + TILE;
    const bool pv_stat = P.stat_kind == FL_STAT_PV && P.vnorm;
    for (int G = grp; G < total; G += 2) {
      if (__any_sync(0xffffffffu, *abort != 0)) break;
      if (G >= 2 && !warp_wait(&sh.kv_empty[grp], ((G >> 1) - 1) & 1, abort, site_of(9 + 16 * mode, G, warp))) break;
      const int pass = pass_of(mode, G, nc);
      const int c = G % nc;
      const int colv = c * TC + jj;
      const int col = colv <= t_max ? colv : -1;
      const float bv = (col >= 0 && P.bias) ? __ldg(P.bias + col) * kLog2e : 0.f;
      const float lv = (col >= 0 && pv_stat) ? log2f(__ldg(P.vnorm + (size_t)col * H + h)) : 0.f;
      meta[grp * TC + jj] = bv;
      meta[2 * TC + grp * TC + jj] = lv;
      meta[4 * TC + grp * TC + jj] = bv + lv;
      float lm = col >= 0 ? lv : -INFINITY;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) lm = fmaxf(lm, __shfl_xor_sync(0xffffffffu, lm, o));
      if (lane == 0) meta[6 * TC + grp * 4 + (warp & 3)] = lm;
      __syncwarp();
      if (lane == 0) mbar_arrive(&sh.meta_full[grp]);
      // K^ (pass cand: hi part in A, lo part in B) and, with P V^, V^ in B (MN-major)
      if constexpr (STAGED) {   // gathered from the staged fp16 rows
        const size_t hoff = (size_t)h * n_tok * HDT;
        copy_rows_warp(P.stage.khi + hoff, a_tile, col, (warp & 3) * 32, lane);
        if (pass == PASS_CAND) copy_rows_warp(P.stage.klo + hoff, b_tile, col, (warp & 3) * 32, lane);
        if (has_pv(pass)) copy_rows_warp(P.stage.vhi + hoff, b_tile, col, (warp & 3) * 32, lane);
        cp_async_wait_all();
      } else {             // decoded from the store
        uint32_t chain = 0;   // loops 2..loop that rewrote the column
        if (col >= 0)
          for (int r = 2; r <= P.loop; ++r)
            if (__ldg(P.kv.slot + (size_t)r * n_tok + col) >= 0) chain |= 1u << r;
        decode_column(P, 0, col, h, chain, a_tile, pass == PASS_CAND ? b_tile : nullptr, jj);
        if (has_pv(pass)) decode_column(P, 1, col, h, chain, b_tile, nullptr, jj);
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sh.kv_full[grp]);
      if (lane == 0 && (warp & 3) == 0) sh.prog[5 + grp] = G;
    }
  }

  // ---- teardown: every MMA done before TMEM is released
  __syncthreads();
  if (warp == 12) {
    if (lane == 0) {
      const uint64_t t0 = globaltimer();
      while (!mbar_try_wait(&sh.fin, 0))
        if (globaltimer() - t0 > kWaitLimitNs) { atomicCAS(&sh.abort_flag, 0, 10 + 16 * mode); break; }
    }
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
  if (threadIdx.x == 0 && sh.abort_flag) {
    record_error(P.st, timeout_code(sh.abort_flag));
    if (A.dbg) {
      int* d = A.dbg + (size_t)blockIdx.x * 12;
      d[0] = sh.abort_flag; d[1] = nc; d[2] = t_max; d[3] = mode;
      for (int k = 0; k < 8; ++k) d[4 + k] = sh.prog[k];
    }
  }
}

// ---------------------------------------------------------------- kernel B: selection
constexpr int SEL_WARPS = 8;

// Exact top-k of c_j = p_j ||V^_j|| (or p_j) among a row's candidates, equal values to
// the smaller column: S' = {0} U kept (ascending - candidates are stored in column order),
// m' = p_0 + sum of kept p_j. One warp per (row, head): the candidates' keys (binary32
// bits of c, order-preserving for c >= 0) in shared memory, a radix select 8 bits at a
// time with a per-warp histogram, then an ordered compaction by ballots. Rows at
// positions t <= k keep every column [0, t] (m' = 1). A row whose candidates overflowed
// is listed for the exact per-query kernel.
__global__ void __launch_bounds__(SEL_WARPS * 32) k_dense_select(const __grid_constant__ DenseArgs A,
                                                                 int* ovf_n, int* ovf_list) {
  const AttnParams& P = A.P;
  extern __shared__ uint8_t sm[];
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  uint32_t* key = reinterpret_cast<uint32_t*>(sm) + (size_t)w * (A.cap + 256);
  int* hist = reinterpret_cast<int*>(key + A.cap);
  const long long rh = (long long)blockIdx.x * SEL_WARPS + w;
  if (rh >= (long long)P.H * P.n_q) return;   // whole warp leaves; no block barrier below
  const int qi = (int)(rh % P.n_q), h = (int)(rh / P.n_q);
  const int t = P.q_tok[qi];
  const int srow = P.q_row ? P.q_row[qi] : t;
  if (t < 0 || t >= P.kv.n_tok || srow < 0 || srow >= P.stat_rows) return;   // recorded in A
  uint16_t* so = P.sel_out + ((size_t)h * P.stat_rows + srow) * P.out_stride;
  const int k = A.k;
  if (t <= k) {
    for (int j = lane; j < P.out_stride; j += 32) so[j] = j <= t ? (uint16_t)j : (uint16_t)FL_SENTINEL;
    if (lane == 0) P.mass_out[(size_t)h * P.stat_rows + srow] = 1.f;
    return;
  }
  const int n = A.cnt[rh];
  if (n > A.cap || n < k) {   // overflow (or a count that cannot hold k): exact fallback
    if (lane == 0) ovf_list[atomicAdd(ovf_n, 1)] = (int)rh;
    return;
  }
  const bool pv_stat = P.stat_kind == FL_STAT_PV;
  const uint16_t* cc = A.ccol + (size_t)rh * A.cap;
  const float* cp = A.cp + (size_t)rh * A.cap;
  for (int x = lane; x < n; x += 32) {
    const float p = cp[x];
    const float cv = pv_stat ? p * P.vnorm[(size_t)cc[x] * P.H + h] : p;
    key[x] = __float_as_uint(fmaxf(cv, 0.f));
  }
  __syncwarp();
  uint32_t prefix = 0, pmask = 0;
  int need = k;
  for (int shift = 24; shift >= 0; shift -= 8) {
    for (int b = lane; b < 256; b += 32) hist[b] = 0;
    __syncwarp();
    for (int x = lane; x < n; x += 32)
      if ((key[x] & pmask) == prefix) atomicAdd(&hist[(key[x] >> shift) & 255u], 1);
    __syncwarp();
    // the digit holding the need-th largest: suffix sums over the 256 bins, 8 per lane
    int cnt8[8], mine = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) { cnt8[i] = hist[255 - (lane * 8 + i)]; mine += cnt8[i]; }
    int incl = mine;   // inclusive scan from the top digit down
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    const int before = incl - mine;
    int dig = -1, above = 0;
    if (before < need && incl >= need) {
      int acc = before;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        if (dig < 0 && acc + cnt8[i] >= need) { dig = 255 - (lane * 8 + i); above = acc; }
        acc += cnt8[i];
      }
    }
    const uint32_t who = __ballot_sync(0xffffffffu, dig >= 0);
    const int src = who ? __ffs(who) - 1 : 0;
    dig = __shfl_sync(0xffffffffu, dig, src);
    above = __shfl_sync(0xffffffffu, above, src);
    if (!who) { dig = 0; above = 0; }   // cannot happen with n >= k
    prefix |= (uint32_t)dig << shift;
    pmask |= 255u << shift;
    need -= above;
    __syncwarp();
  }
  // keep key > prefix, and the first `need` entries (smallest columns) with key == prefix
  const uint32_t lt = (1u << lane) - 1u;
  int written = 0, eq_seen = 0;
  float mass = 0.f;
  for (int base = 0; base < n; base += 32) {
    const int x = base + lane;
    const bool in = x < n;
    const uint32_t kv = in ? key[x] : 0u;
    const bool eq = in && kv == prefix;
    const uint32_t eb = __ballot_sync(0xffffffffu, eq);
    const bool keep = in && (kv > prefix || (eq && eq_seen + __popc(eb & lt) < need));
    const uint32_t kb = __ballot_sync(0xffffffffu, keep);
    const int pos = written + __popc(kb & lt);
    if (keep && pos < k) {
      so[1 + pos] = cc[x];
      mass += cp[x];
    }
    written += __popc(kb);
    eq_seen += __popc(eb);
  }
  written = min(written, k);
  for (int j = 1 + written + lane; j < P.out_stride; j += 32) so[j] = (uint16_t)FL_SENTINEL;
  if (lane == 0) so[0] = 0;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) mass += __shfl_xor_sync(0xffffffffu, mass, o);
  if (lane == 0) P.mass_out[(size_t)h * P.stat_rows + srow] = A.p0[rh] + mass;
}

}  // namespace

size_t dense_tile_ws_bytes(const AttnParams& P) {
  if (!P.sel_out) return 0;
  const int cap = P.k_next + 1024;
  const size_t rows = (size_t)P.H * P.n_q;
  return align_up(rows * sizeof(float2)) + 2 * align_up(rows * 4) + align_up(rows * cap * 2) +
         align_up(rows * cap * 4) + align_up(4) + align_up(rows * 4) +
         align_up((size_t)((P.n_q + TQ - 1) / TQ) * P.H * 12 * 4) + align_up(sel_bitmap_bytes(P));
}

bool dense_tile_eligible(const AttnParams& P) {
  if (P.sel || P.hd != HDT || P.kv.hd != HDT) return false;
  if ((P.kv.base_bits != 8 && P.kv.base_bits != 0) || (P.kv.g != 32 && P.kv.g != 64)) return false;
  if (P.kv.n_tok > 65535 || P.loop > 31) return false;
  for (int r = 2; r <= P.loop; ++r) {
    const int b = P.kv.res_bits[r];
    if (b != 0 && b != 2 && b != 4 && b != 8) return false;
  }
  if (P.sel_out && P.stat_kind == FL_STAT_PV && !P.vnorm) return false;
  if (P.sel_out && (P.k_next < 1 || P.k_next + 1 > P.out_stride)) return false;
  // rows the candidates cannot rank are finished by a per-query kernel
  if (P.sel_out && !dense_rows_supported(P) && !dense_list_supported(P)) return false;
  return true;
}

cudaError_t launch_attn_dense_tile(const AttnParams& P, void* ws, cudaStream_t s) {
  static bool attr_set[128] = {false};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 128) return cudaErrorInvalidDevice;
  if (!attr_set[dev]) {
    for (auto k : {k_attn_dense_tile<true>, k_attn_dense_tile<false>}) {
      const cudaError_t e =
          cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM_BYTES);
      if (e != cudaSuccess) return e;
    }
    attr_set[dev] = true;
  }
  DenseArgs A{};
  A.P = P;
  A.k = P.k_next;
  A.cap = P.k_next + 1024;
  const size_t rows = (size_t)P.H * P.n_q;
  int* ovf_n = nullptr;
  int* ovf_list = nullptr;
  uint8_t* bm_buf = nullptr;
  if (P.sel_out) {
    uint8_t* p = static_cast<uint8_t*>(ws);
    A.m1l = reinterpret_cast<float2*>(p); p += align_up(rows * sizeof(float2));
    A.cnt = reinterpret_cast<int*>(p); p += align_up(rows * 4);
    A.p0 = reinterpret_cast<float*>(p); p += align_up(rows * 4);
    A.ccol = reinterpret_cast<uint16_t*>(p); p += align_up(rows * A.cap * 2);
    A.cp = reinterpret_cast<float*>(p); p += align_up(rows * A.cap * 4);
    ovf_n = reinterpret_cast<int*>(p); p += align_up(4);
    ovf_list = reinterpret_cast<int*>(p); p += align_up(rows * 4);
    A.dbg = reinterpret_cast<int*>(p); p += align_up((size_t)((P.n_q + TQ - 1) / TQ) * P.H * 12 * 4);
    bm_buf = p;
    cudaError_t e = cudaMemsetAsync(ovf_n, 0, sizeof(int), s);
    if (e != cudaSuccess) return e;
  }
  const int n_tiles = (P.n_q + TQ - 1) / TQ;
  A.mode = P.sel_out ? 1 : 0;
  auto kern = P.stage.khi ? k_attn_dense_tile<true> : k_attn_dense_tile<false>;
  cudaError_t e = launch_pdl(kern, dim3(n_tiles * P.H), dim3(NTHR), SMEM_BYTES, s, A);
  count_launch();
  if (e != cudaSuccess) return e;
  if (!P.sel_out) return cudaGetLastError();
  const size_t sel_smem = (size_t)SEL_WARPS * (A.cap + 256) * 4;
  static int sel_attr[128] = {0};
  if ((int)sel_smem > sel_attr[dev]) {
    e = cudaFuncSetAttribute(k_dense_select, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sel_smem);
    if (e != cudaSuccess) return e;
    sel_attr[dev] = (int)sel_smem;
  }
  k_dense_select<<<(unsigned)((rows + SEL_WARPS - 1) / SEL_WARPS), SEL_WARPS * 32, sel_smem, s>>>(
      A, ovf_n, ovf_list);
  count_launch();
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  // S' as bitmaps for the unselected pass (rows finished by the exact kernels below get
  // theirs from stale sets: their u' is overwritten there)
  {
    AttnParams Q = P;
    Q.sel = P.sel_out;
    Q.sel_stride = P.out_stride;
    e = launch_sel_bitmap(Q, bm_buf, s, false);
    if (e != cudaSuccess) return e;
    A.P.sel_bm = Q.sel_bm;
    A.P.bm_words = Q.bm_words;
  }
  A.mode = 2;
  e = launch_pdl(kern, dim3(n_tiles * P.H), dim3(NTHR), SMEM_BYTES, s, A);
  count_launch();
  if (e != cudaSuccess) return e;
  // rows whose candidates overflowed: the warp-per-query kernel (loop 1, 8-bit base) or
  // the general CTA-per-query kernel (any store)
  if (dense_rows_supported(P)) return launch_attn_dense_rows(P, ovf_list, ovf_n, s);
  return launch_attention_list(P, ovf_list, ovf_n, s);
}

}  // namespace fl
