// Tensor-core GEMM for the bf16 path (FlashLoop §4.4: the gathered active rows keep
// the projections regular GEMMs): C (=|+=) A . W^T, A [M x K] bf16 activations,
// W [N x K] bf16 linear-layer weights, fp32 accumulation in tensor memory.
//
// Persistent CTAs (one per SM) over 128 x BN output tiles, 6 warps:
//   warp 0     TMA producer: A and W tiles (64 K-columns, 128-byte swizzle) into a
//              STAGES-deep shared-memory ring, completion counted on mbarriers;
//   warp 1     allocates TMEM (two accumulators of BN columns) and issues
//              tcgen05.mma (M 128, N BN, K 16) from one thread; tcgen05.commit frees
//              each ring slot and signals the epilogue when a tile is complete;
//   warps 2-5  epilogue: tcgen05.ld of their 32 TMEM lanes (= tile rows), binary32
//              store or accumulate into C (or the SwiGLU product in bf16), then hand
//              the accumulator back to the MMA warp.
// Rows beyond M are zero-filled by TMA and not stored. Every mbarrier wait is bounded
// in time; a wait that runs out records FL_ERR_TIMEOUT and the CTA drains its copies
// in flight, frees TMEM and returns.
#include <mutex>
#include <stdlib.h>
#include <unordered_map>

#include "fl_internal.cuh"
#include "sm100_ptx.cuh"
#include "kv_epilogue.cuh"

namespace fl {
namespace {

using namespace sm100;

constexpr int BM = 128, BK = 64;

// EPI_STORE / EPI_ADD: C[M x N] fp32 (=|+=) A . W^T, tiles of 128 x BN.
// EPI_SWIGLU: W = [gate; up] with `half` rows each; a tile holds BN/2 gate rows and the
// matching BN/2 up rows (two TMA boxes), and the epilogue writes silu(g) * u as bf16 into
// Y [M x half].
constexpr int EPI_SWIGLU = 2;
// EPI_QKV: W = w_qkv [3d x d]; a tile of 128 columns lies in q, k or v; the epilogue writes
// it to q / k / v [M x d] (fp32), rotating q and k by RoPE at position pos[row] with the
// (cos, sin) table rope[pos][i], i < hd/2 (rotate-half pairs (i, i + hd/2)).
constexpr int EPI_QKV = 3;
// EPI_QKV_KV: EPI_QKV plus the KV store update of k and v in the epilogue (qo.kf).
constexpr int EPI_QKV_KV = 4;

struct QkvOut {
  float* q; float* k; float* v;   // k, v may be null when the store update is fused
  const int32_t* pos;
  const float2* rope;
  int d, hd;
  KvFuse kf;                      // fused KV quantisation of k and v (kf.on)
  KvView kv;                      // the store read for the residual's reference
};

// Stream-K split (when the tiles do not fill whole rounds of the grid): the tiles x
// k-blocks units are cut into gridDim.x equal contiguous ranges, one per CTA. A tile cut
// between CTAs is finished by its owner (the CTA holding its k-block 0, which reaches it
// last in its range); each other CTA holding a piece of it (its first segment) stores the
// fp32 partial accumulator to part[cta] and raises flag[cta]. The owner waits for those
// flags, adds the partials in CTA order (a fixed summation order: results do not depend
// on timing) and runs the epilogue; it lowers the flags again for the next launch.
struct SkPlan {
  int on;
  float* part;   // [gridDim.x][BM * BN] float4-interleaved partial tiles
  int* flag;     // [gridDim.x], all zero at launch
};

// Work segment: k-blocks [kb0, kb1) of tile `tile`.
struct Seg {
  int tile, kb0, kb1;
};

__device__ __forceinline__ long long sk_begin(long long units, int cta, int grid) {
  return units * cta / grid;
}

// Walks one CTA's segments: whole tiles blockIdx.x, +gridDim.x, ... without stream-K;
// otherwise its unit range cut at tile boundaries.
struct SegWalk {
  long long cur, end;
  int nk, tiles, sk;
  __device__ SegWalk(bool on, int nk_, int tiles_) : nk(nk_), tiles(tiles_), sk(on) {
    if (sk) {
      const long long units = (long long)tiles * nk;
      cur = sk_begin(units, blockIdx.x, gridDim.x);
      end = sk_begin(units, blockIdx.x + 1, gridDim.x);
    } else {
      cur = blockIdx.x;
      end = tiles;
    }
  }
  __device__ bool next(Seg& g) {
    if (cur >= end) return false;
    if (!sk) {
      g.tile = (int)cur; g.kb0 = 0; g.kb1 = nk;
      cur += gridDim.x;
      return true;
    }
    g.tile = (int)(cur / nk);
    g.kb0 = (int)(cur % nk);
    const long long left = end - cur;
    g.kb1 = left < (long long)(nk - g.kb0) ? g.kb0 + (int)left : nk;
    cur += g.kb1 - g.kb0;
    return true;
  }
};

// Persistent: one CTA per SM walks its segments (M-tile fastest, so the CTAs running
// together share each weight tile through L2).
// Two TMEM accumulators: the epilogue drains segment i while the MMA warp fills i+1.
template <int BN, int STAGES, int EPI, bool SK>
__global__ void __launch_bounds__(192, 1)
    k_gemm_tc(const __grid_constant__ CUtensorMap tma_a, const __grid_constant__ CUtensorMap tma_b,
              float* __restrict__ C, __nv_bfloat16* __restrict__ Y, int M, int N, int K, int ldc,
              int half, const __grid_constant__ QkvOut qo, const SkPlan sk, int* st) {
  constexpr uint32_t A_BYTES = BM * BK * 2;
  constexpr uint32_t B_BYTES = BN * BK * 2;
  constexpr uint32_t STAGE_BYTES = A_BYTES + B_BYTES;
  constexpr uint32_t TMEM_COLS = 2 * BN;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  __shared__ uint64_t full_bar[STAGES], empty_bar[STAGES];
  __shared__ uint64_t accf_bar[2], acce_bar[2], final_bar;
  __shared__ uint32_t tmem_slot;
  __shared__ int abort_flag;
  volatile int* abort = &abort_flag;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nk = K / BK;
  const int m_tiles = (M + BM - 1) / BM;
  const int n_tiles = EPI == EPI_SWIGLU ? half / (BN / 2) : N / BN;
  const int tiles = m_tiles * n_tiles;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) { mbar_init(&full_bar[s], 1); mbar_init(&empty_bar[s], 1); }
    for (int a = 0; a < 2; ++a) { mbar_init(&accf_bar[a], 1); mbar_init(&acce_bar[a], 4); }
    mbar_init(&final_bar, 1);
    abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) { prefetch_tmap(&tma_a); prefetch_tmap(&tma_b); }
  if (warp == 1) tmem_alloc(&tmem_slot, TMEM_COLS);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_slot;
  griddep_wait();   // operands and C may still be in flight from the previous kernel

  if (warp == 0) {
    if (lane == 0) {
      int g = 0;  // k-blocks issued over all segments
      SegWalk walk(SK, nk, tiles);
      Seg sg;
      while (!*abort && walk.next(sg)) {
        const int m0 = (sg.tile % m_tiles) * BM;
        const int nt = sg.tile / m_tiles;
        for (int kb = sg.kb0; kb < sg.kb1; ++kb, ++g) {
          const int s = g % STAGES, i = g / STAGES;
          if (i > 0 && !mbar_wait(&empty_bar[s], (i - 1) & 1, abort)) break;
          uint8_t* a_dst = smem + s * STAGE_BYTES;
          mbar_arrive_expect_tx(&full_bar[s], STAGE_BYTES);
          tma_load_2d(a_dst, &tma_a, &full_bar[s], kb * BK, m0);
          if constexpr (EPI == EPI_SWIGLU) {
            const int f0 = nt * (BN / 2);
            tma_load_2d(a_dst + A_BYTES, &tma_b, &full_bar[s], kb * BK, f0);
            tma_load_2d(a_dst + A_BYTES + B_BYTES / 2, &tma_b, &full_bar[s], kb * BK, half + f0);
          } else {
            tma_load_2d(a_dst + A_BYTES, &tma_b, &full_bar[s], kb * BK, nt * BN);
          }
        }
      }
      if (*abort) {  // drain the copies still in flight before shared memory is released
        const uint64_t t0 = globaltimer();
        for (int x = g > STAGES ? g - STAGES : 0; x < g; ++x) {
          while (!mbar_try_wait(&full_bar[x % STAGES], (x / STAGES) & 1))
            if (globaltimer() - t0 > kWaitLimitNs) break;
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(BM, BN);
      int g = 0, lt = 0;
      SegWalk walk(SK, nk, tiles);
      Seg sg;
      for (; !*abort && walk.next(sg); ++lt) {
        const int a = lt & 1, j = lt >> 1;
        if (lt >= 2 && !mbar_wait(&acce_bar[a], (j - 1) & 1, abort)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem + (uint32_t)(a * BN);
        bool ok = true;
        for (int kb = sg.kb0; kb < sg.kb1; ++kb, ++g) {
          const int s = g % STAGES, i = g / STAGES;
          if (!mbar_wait(&full_bar[s], i & 1, abort)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a_base = smem_u32(smem + s * STAGE_BYTES);
          const uint32_t b_base = a_base + A_BYTES;
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk) {
            mma_bf16(d_tmem, desc_sw128_kmajor(a_base + kk * 32),
                     desc_sw128_kmajor(b_base + kk * 32), idesc,
                     (kb > sg.kb0 || kk > 0) ? 1u : 0u);
          }
          mma_commit(&empty_bar[s]);
        }
        if (!ok) break;
        mma_commit(&accf_bar[a]);
      }
      mma_commit(&final_bar);  // arrives once every MMA issued above has completed
    }
  } else {
    const int ew = warp & 3;  // TMEM lanes [32 ew, 32 ew + 32) belong to this warp
    const int lrow = ew * 32 + lane;
    int lt = 0;
    SegWalk walk(SK, nk, tiles);
    Seg sg;
    for (; walk.next(sg); ++lt) {
      const int a = lt & 1, j = lt >> 1;
      if (!mbar_wait(&accf_bar[a], j & 1, abort)) break;
      tc_fence_after();
      const int tile = sg.tile;
      const int row = (tile % m_tiles) * BM + lrow;
      const int nt = tile / m_tiles;
      const uint32_t t_base = tmem + ((uint32_t)(ew * 32) << 16) + (uint32_t)(a * BN);
      if (SK && sg.kb0 > 0) {
        // a piece of a tile owned by an earlier CTA: park the partial, hand the rows over
        float4* dst = reinterpret_cast<float4*>(sk.part + (size_t)blockIdx.x * (BM * BN));
#pragma unroll 1
        for (int c = 0; c < BN / 32; ++c) {
          float v[32];
          tmem_ld32(t_base + (uint32_t)(c * 32), v);
#pragma unroll
          for (int q = 0; q < 8; ++q)
            dst[(c * 8 + q) * BM + lrow] = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&acce_bar[a]);
          flag_release(&sk.flag[blockIdx.x * 4 + ew]);
        }
        continue;
      }
      // owner of a cut tile: the pieces of CTAs blockIdx.x + 1 .. j_end - 1 are added
      int j_end = blockIdx.x + 1;
      if (SK && sg.kb1 < nk) {
        const long long units = (long long)tiles * nk, tile_end = (long long)(tile + 1) * nk;
        while (j_end < (int)gridDim.x && sk_begin(units, j_end, gridDim.x) < tile_end) ++j_end;
        if (lane == 0) {
          for (int jj = blockIdx.x + 1; jj < j_end; ++jj)
            if (!flag_acquire_reset(&sk.flag[jj * 4 + ew])) { record_error(st, FL_ERR_TIMEOUT); *abort = 1; }
        }
        __syncwarp();
      }
      // accumulator columns [col, col + 32) of this thread's row, pieces included
      auto ld_acc = [&](int col, float* v) {
        tmem_ld32(t_base + (uint32_t)col, v);
        for (int jj = blockIdx.x + 1; SK && jj < j_end; ++jj) {
          const float4* src = reinterpret_cast<const float4*>(sk.part + (size_t)jj * (BM * BN));
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            const float4 pv = __ldcg(src + ((col / 32) * 8 + q) * BM + lrow);
            v[4 * q] += pv.x; v[4 * q + 1] += pv.y; v[4 * q + 2] += pv.z; v[4 * q + 3] += pv.w;
          }
        }
      };
      if constexpr (EPI == EPI_SWIGLU) {
        const int f0 = nt * (BN / 2);
#pragma unroll 1
        for (int c = 0; c < BN / 64; ++c) {
          float gv[32], uv[32];
          ld_acc(c * 32, gv);
          ld_acc(BN / 2 + c * 32, uv);
          if (row < M) {
            uint4* dst = reinterpret_cast<uint4*>(Y + (size_t)row * half + f0 + c * 32);
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4) {
              uint32_t wv[4];
#pragma unroll
              for (int q = 0; q < 4; ++q) {
                const int e = 8 * q4 + 2 * q;
                const float y0 = gv[e] / (1.0f + expf(-gv[e])) * uv[e];
                const float y1 = gv[e + 1] / (1.0f + expf(-gv[e + 1])) * uv[e + 1];
                const __nv_bfloat162 b2 = __floats2bfloat162_rn(y0, y1);
                wv[q] = *reinterpret_cast<const uint32_t*>(&b2);
              }
              dst[q4] = make_uint4(wv[0], wv[1], wv[2], wv[3]);
            }
          }
        }
      } else if constexpr (EPI == EPI_QKV || EPI == EPI_QKV_KV) {
        const int n0 = nt * BN;
        const int which = n0 / qo.d, col0 = n0 % qo.d;
        float* out = which == 0 ? qo.q : (which == 1 ? qo.k : qo.v);
        const bool quant = EPI == EPI_QKV_KV && which >= 1;
        const int hh = qo.hd / 2;
        const int prow = row < M ? qo.pos[row] : 0;
        float vss = 0.f;   // ||V^||^2 of the current head (fused V tiles)
#pragma unroll 1
        for (int c = 0; c < BN / 32; ++c) {
          const int off = (c * 32) % qo.hd;   // offset inside the head
          const int head = (col0 + c * 32) / qo.hd;
          if (which < 2 && off >= hh) continue;  // second halves go with their partners
          float a[32];
          ld_acc(c * 32, a);
          if (which == 2) {
            if (row < M) {
              if (out) {
                float4* dst = reinterpret_cast<float4*>(out + (size_t)row * qo.d + col0 + c * 32);
#pragma unroll
                for (int q = 0; q < 8; ++q)
                  dst[q] = make_float4(a[4 * q], a[4 * q + 1], a[4 * q + 2], a[4 * q + 3]);
              }
              if (quant) {
                vss += fuse_group(qo.kv, qo.kf, 1, a, row, prow, head, off, st);
                if (off + 32 == qo.hd && qo.kf.vnorm)
                  qo.kf.vnorm[(size_t)prow * qo.kv.H + head] = sqrtf(vss);
              }
            }
            if (off + 32 == qo.hd) vss = 0.f;
            continue;
          }
          float b[32];
          ld_acc(c * 32 + hh, b);
          if (row < M) {
            // rotate: (a, b) -> (a cos - b sin, a sin + b cos); (cos, sin) of 4 angles = 2 float4
            const float4* cs = reinterpret_cast<const float4*>(qo.rope + (size_t)prow * hh + off);
#pragma unroll
            for (int q = 0; q < 8; ++q) {
              const float4 r01 = cs[2 * q], r23 = cs[2 * q + 1];
              const float cr[4] = {r01.x, r01.z, r23.x, r23.z}, sr[4] = {r01.y, r01.w, r23.y, r23.w};
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const float x = a[4 * q + e], y = b[4 * q + e];
                a[4 * q + e] = x * cr[e] - y * sr[e];
                b[4 * q + e] = x * sr[e] + y * cr[e];
              }
            }
            if (out) {
              float4* dx = reinterpret_cast<float4*>(out + (size_t)row * qo.d + col0 + c * 32);
              float4* dy = reinterpret_cast<float4*>(out + (size_t)row * qo.d + col0 + c * 32 + hh);
#pragma unroll
              for (int q = 0; q < 8; ++q) {
                dx[q] = make_float4(a[4 * q], a[4 * q + 1], a[4 * q + 2], a[4 * q + 3]);
                dy[q] = make_float4(b[4 * q], b[4 * q + 1], b[4 * q + 2], b[4 * q + 3]);
              }
            }
            if (quant) {
              fuse_group(qo.kv, qo.kf, 0, a, row, prow, head, off, st);
              fuse_group(qo.kv, qo.kf, 0, b, row, prow, head, off + hh, st);
            }
          }
        }
      } else {
        const int n0 = nt * BN;
#pragma unroll 1
        for (int c = 0; c < BN / 32; ++c) {
          float v[32];
          ld_acc(c * 32, v);
          if (row < M) {
            float4* dst = reinterpret_cast<float4*>(C + (size_t)row * ldc + n0 + c * 32);
#pragma unroll
            for (int q = 0; q < 8; ++q) {
              float4 x = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
              if (EPI == EPI_ADD) {
                const float4 y = dst[q];
                x.x += y.x; x.y += y.y; x.z += y.z; x.w += y.w;
              }
              dst[q] = x;
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acce_bar[a]);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    if (lane == 0) {  // every issued MMA must finish before TMEM is released
      const uint64_t t0 = globaltimer();
      while (!mbar_try_wait(&final_bar, 0))
        if (globaltimer() - t0 > kWaitLimitNs) { abort_flag = 1; break; }
    }
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
  if (threadIdx.x == 0 && abort_flag) record_error(st, FL_ERR_TIMEOUT);
}

// ---------------------------------------------------------------- tensor maps
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

struct MapKey {
  const void* p; int rows, cols, box_rows;
  bool operator==(const MapKey& o) const {
    return p == o.p && rows == o.rows && cols == o.cols && box_rows == o.box_rows;
  }
};
struct MapKeyHash {
  size_t operator()(const MapKey& k) const {
    return std::hash<const void*>()(k.p) ^ ((size_t)k.rows << 20) ^ ((size_t)k.cols << 40) ^
           (size_t)k.box_rows;
  }
};

// Row-major bf16 [rows x cols] matrix, boxes of 64 columns x box_rows rows, 128B swizzle.
bool get_map(const void* p, int rows, int cols, int box_rows, CUtensorMap* out) {
  static std::mutex mu;
  static std::unordered_map<MapKey, CUtensorMap, MapKeyHash> cache;
  const MapKey key{p, rows, cols, box_rows};
  {
    std::lock_guard<std::mutex> lock(mu);
    auto it = cache.find(key);
    if (it != cache.end()) { *out = it->second; return true; }
  }
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  CUtensorMap m;
  const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)cols * 2};
  const cuuint32_t box[2] = {(cuuint32_t)BK, (cuuint32_t)box_rows};
  const cuuint32_t estr[2] = {1, 1};
  if (enc(&m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(p), dims, strides, box, estr,
          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return false;
  std::lock_guard<std::mutex> lock(mu);
  if (cache.size() > 4096) cache.clear();
  cache[key] = m;
  *out = m;
  return true;
}

int sm_count() {
  static int sms[128] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 128) return 148;
  if (!sms[dev]) cudaDeviceGetAttribute(&sms[dev], cudaDevAttrMultiProcessorCount, dev);
  return sms[dev] > 0 ? sms[dev] : 148;
}

// Stream-K unless switched off (FL_GEMM_SK=0).
bool sk_enabled() {
  static int on = -1;
  if (on < 0) {
    const char* e = getenv("FL_GEMM_SK");
    on = (e && atoi(e) == 0) ? 0 : 1;
  }
  return on == 1;
}

constexpr int SK_MAX_GRID = 1024;

// Stream-K is taken for 256-wide tiles that do not fill whole rounds of the grid and
// give every CTA at least 64 k-blocks: below that the partial hand-over and the owner's
// longer last epilogue cost more than the balance gains (measured on the projection
// shapes of 820 active rows: a win for the gate/up GEMM at 67 k-blocks per CTA, losses
// for QKV at 36, down at 33 and O at 12).
bool use_sk(int tiles, int nk, int bn) {
  const int sms = sm_count();
  const long long units = (long long)tiles * nk;
  return sk_enabled() && bn == 256 && tiles % sms != 0 && units >= 64LL * sms;
}

template <int BN, int STAGES, int EPI>
cudaError_t launch_bn(const void* A, const void* W, float* C, __nv_bfloat16* Y, int M, int N,
                      int K, int ldc, cudaStream_t s, const GemmScratch* scr,
                      QkvOut qo = QkvOut{}) {
  CUtensorMap ma, mb;
  const int box_b = EPI == EPI_SWIGLU ? BN / 2 : BN;
  if (!get_map(A, M, K, BM, &ma) || !get_map(W, N, K, box_b, &mb)) return cudaErrorInvalidValue;
  const size_t smem = (size_t)STAGES * (BM * BK * 2 + BN * BK * 2) + 1024;
  auto kern_dp = k_gemm_tc<BN, STAGES, EPI, false>;
  auto kern_sk = k_gemm_tc<BN, STAGES, EPI, true>;
  static bool attr_set[128] = {false};   // per device; set on the first (uncaptured) call
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 128) return cudaErrorInvalidDevice;
  if (!attr_set[dev]) {
    cudaError_t e = cudaFuncSetAttribute(kern_dp, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(kern_sk, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    attr_set[dev] = true;
  }
  const int tiles_n = EPI == EPI_SWIGLU ? (N / 2) / (BN / 2) : N / BN;
  const int tiles = tiles_n * ((M + BM - 1) / BM);
  const int sms = sm_count();
  int grid = tiles < sms ? tiles : sms;
  SkPlan plan{0, nullptr, nullptr};
  cudaError_t e;
  if (use_sk(tiles, K / BK, BN) && scr && scr->flag && scr->part && sms * 4 <= scr->n_flag &&
      (size_t)sms * BM * BN * 4 <= scr->part_bytes) {
    grid = sms;
    plan = SkPlan{1, scr->part, scr->flag};
    e = launch_pdl(kern_sk, dim3(grid), dim3(192), smem, s, ma, mb, C, Y, M, N, K, ldc, N / 2, qo,
                   plan, status_word());
  } else {
    e = launch_pdl(kern_dp, dim3(grid), dim3(192), smem, s, ma, mb, C, Y, M, N, K, ldc, N / 2, qo,
                   plan, status_word());
  }
  count_launch();
  return e != cudaSuccess ? e : cudaGetLastError();
}

}  // namespace

// Tile width: 128 or 256 output columns. A 256-wide tile moves 48 KB per k-block for twice
// the MACs of a 128-wide one (32 KB), so it costs between 1.5x (operand-bandwidth bound)
// and 2x (tensor bound) as long; the persistent grid runs ceil(tiles / SMs) rounds.
// The wider tile is taken when its rounds x cost are lower. FL_GEMM_BN=128|256 forces it.
int pick_bn(int M, int n_cols, bool pairs, int K, bool sk) {
  static int forced = -1;
  if (forced < 0) {
    const char* e = getenv("FL_GEMM_BN");
    forced = e ? atoi(e) : 0;
  }
  // pairs (SwiGLU): a tile of width BN produces BN / 2 output columns
  const int out128 = pairs ? 64 : 128, out256 = pairs ? 128 : 256;
  if (n_cols % out256 != 0) return 128;
  if (forced == 128 || forced == 256) return forced;
  const int sms = sm_count();
  const int mt = (M + BM - 1) / BM;
  const long t128 = (long)mt * (n_cols / out128), t256 = (long)mt * (n_cols / out256);
  // stream-K (balanced to a k-block) runs with 256-wide tiles
  if (sk && use_sk((int)t256, K / BK, 256)) return 256;
  const double c128 = (double)((t128 + sms - 1) / sms);
  const double c256 = 1.75 * (double)((t256 + sms - 1) / sms);
  return c256 < c128 ? 256 : 128;
}

// Stream-K scratch: SK_MAX_GRID x 4 flags, then one 128 x 256 fp32 partial tile per SM.
size_t gemm_scratch_flag_bytes() { return (size_t)SK_MAX_GRID * 4 * sizeof(int); }

size_t gemm_scratch_bytes() {
  return gemm_scratch_flag_bytes() + (size_t)sm_count() * BM * 256 * sizeof(float);
}

GemmScratch gemm_scratch_at(void* p) {
  GemmScratch g;
  g.flag = static_cast<int*>(p);
  g.n_flag = SK_MAX_GRID * 4;
  g.part = reinterpret_cast<float*>(static_cast<uint8_t*>(p) + gemm_scratch_flag_bytes());
  g.part_bytes = gemm_scratch_bytes() - gemm_scratch_flag_bytes();
  return g;
}

bool gemm_tc_supported(int M, int N, int K) {
  return M >= 1 && K >= BK && K % BK == 0 && N % 128 == 0 && encode_fn() != nullptr;
}

cudaError_t launch_gemm_tc(const void* A, const void* W, float* C, int M, int N, int K, int ldc,
                           GemmEpi epi, cudaStream_t s, const GemmScratch* scr) {
  if ((uintptr_t)A % 16 || (uintptr_t)W % 16 || (uintptr_t)C % 16 || ldc % 4)
    return cudaErrorInvalidValue;
  const bool wide = pick_bn(M, N, false, K, scr != nullptr) == 256;
  if (epi == EPI_ADD)
    return wide ? launch_bn<256, 4, EPI_ADD>(A, W, C, nullptr, M, N, K, ldc, s, scr)
                : launch_bn<128, 6, EPI_ADD>(A, W, C, nullptr, M, N, K, ldc, s, scr);
  return wide ? launch_bn<256, 4, EPI_STORE>(A, W, C, nullptr, M, N, K, ldc, s, scr)
              : launch_bn<128, 6, EPI_STORE>(A, W, C, nullptr, M, N, K, ldc, s, scr);
}

bool gemm_swiglu_supported(int M, int F, int K) {
  return gemm_tc_supported(M, 2 * F, K) && F % 64 == 0;
}

// Y[M x F] bf16 = silu(A . W_gate^T) * (A . W_up^T), W = [gate; up] of [2F x K].
cudaError_t launch_gemm_swiglu(const void* A, const void* W, void* Y, int M, int F, int K,
                               cudaStream_t s, const GemmScratch* scr) {
  if ((uintptr_t)A % 16 || (uintptr_t)W % 16 || (uintptr_t)Y % 16 || F % 64)
    return cudaErrorInvalidValue;
  if (pick_bn(M, F, true, K, scr != nullptr) == 256)
    return launch_bn<256, 4, EPI_SWIGLU>(A, W, nullptr, reinterpret_cast<__nv_bfloat16*>(Y), M,
                                         2 * F, K, 0, s, scr);
  return launch_bn<128, 6, EPI_SWIGLU>(A, W, nullptr, reinterpret_cast<__nv_bfloat16*>(Y), M,
                                       2 * F, K, 0, s, scr);
}

bool gemm_qkv_supported(int M, int d, int hd) {
  return gemm_tc_supported(M, 3 * d, d) && (hd == 64 || hd == 128) && d % 128 == 0;
}

// q, k, v [M x d] fp32 = split(A . w_qkv^T), q and k rotated by RoPE (table `rope`).
cudaError_t launch_gemm_qkv(const void* A, const void* W, float* q, float* k, float* v,
                            const int32_t* pos, const float2* rope, int M, int d, int hd,
                            cudaStream_t s, const fl_kv_desc* fuse, int loop,
                            const GemmScratch* scr) {
  if ((uintptr_t)A % 16 || (uintptr_t)W % 16 || (uintptr_t)q % 16 || (uintptr_t)k % 16 ||
      (uintptr_t)v % 16)
    return cudaErrorInvalidValue;
  QkvOut qo{};
  qo.q = q; qo.k = k; qo.v = v; qo.pos = pos; qo.rope = rope; qo.d = d; qo.hd = hd;
  qo.kf.on = 0;
  if (fuse) {
    qo.kv = make_view(*fuse);
    qo.kf.on = 1;
    qo.kf.loop = loop;
    for (int w = 0; w < 2; ++w) { qo.kf.codes[w] = fuse->codes[w][loop]; qo.kf.sz[w] = fuse->sz[w][loop]; }
    qo.kf.slot_row = loop >= 2 ? fuse->slot + (size_t)loop * fuse->n_tok : nullptr;
    qo.kf.vnorm = fuse->vnorm;
  }
  if (d % 256 == 0 && pick_bn(M, 3 * d, false, d, scr != nullptr) == 256)
    return fuse ? launch_bn<256, 4, EPI_QKV_KV>(A, W, nullptr, nullptr, M, 3 * d, d, 0, s, scr, qo)
                : launch_bn<256, 4, EPI_QKV>(A, W, nullptr, nullptr, M, 3 * d, d, 0, s, scr, qo);
  return fuse ? launch_bn<128, 6, EPI_QKV_KV>(A, W, nullptr, nullptr, M, 3 * d, d, 0, s, scr, qo)
              : launch_bn<128, 6, EPI_QKV>(A, W, nullptr, nullptr, M, 3 * d, d, 0, s, scr, qo);
}

}  // namespace fl
