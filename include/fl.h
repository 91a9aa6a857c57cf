/*
 * fl.h - C interface of the FlashLoop loop-step library (libfl.so), sm_100a.
 *
 * The library computes the loop-r step of a looped Transformer's shared block with
 * the three lazy updates of "FlashLoop: Fast and Memory-Efficient Looped
 * Transformers via Lazy Updates" (arXiv 2609.29812):
 *   - token-sparse updates            (§4.1 Cross-Loop Token-Sparse Updates)
 *   - loop-aware sparse attention     (§4.2 Loop-Aware Sparse Attention)
 *   - cross-loop KV residual quant.   (§4.3, Appendix E "Quantization Setting")
 * gathered into compact buffers so the projections stay regular GEMMs (§4.4).
 *
 * Conventions (every entry point):
 *   - Returns fl_status. Host-side validation runs first; on error nothing is
 *     launched and no output is touched.
 *   - Pointers named "device" must be device memory of the current CUDA device;
 *     "host" pointers are read before the call returns. The caller allocates and
 *     frees every buffer, including workspaces sized by the *_workspace_bytes
 *     queries. The library never allocates and never synchronises (except
 *     fl_check_device_status).
 *   - `stream` is a cudaStream_t passed as void* (NULL: the legacy default stream).
 *     All work is enqueued asynchronously on it.
 *   - Errors found by a kernel (an index out of range, an fp16 overflow of a scale
 *     or offset, a bounded wait that ran out) are recorded in a per-device status
 *     word; fl_check_device_status reads and clears it. The kernel skips the
 *     offending element and keeps the context usable.
 *   - Row-major layouts throughout. H = n_heads, hd = head_dim, d = H * hd.
 *   - Token indices fit in 16 bits in the statistics (n_tok <= 65535).
 */
#ifndef FL_H
#define FL_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define FL_MAX_LOOPS 32          /* loops are numbered 1..R, R <= FL_MAX_LOOPS */
#define FL_SENTINEL 0xFFFFu      /* pads column sets beyond their size */

typedef enum {
  FL_OK = 0,
  FL_ERR_INVALID_ARG = 1,   /* null pointer, bad enum, negative size */
  FL_ERR_SHAPE = 2,         /* inconsistent or unsupported sizes */
  FL_ERR_UNSUPPORTED = 3,   /* dtype, bit width or group size not built */
  FL_ERR_CUDA = 4,          /* a CUDA runtime call failed */
  FL_ERR_TIMEOUT = 5,       /* a bounded device wait ran out */
  FL_ERR_RANGE = 6,         /* device: index out of range, or fp16 overflow of s/z */
  FL_ERR_WORKSPACE = 7      /* workspace too small */
} fl_status;

typedef enum { FL_F32 = 0, FL_BF16 = 1 } fl_dtype;
typedef enum { FL_GATHER = 0, FL_SCATTER = 1 } fl_gs_op;
typedef enum { FL_STAT_PV = 0, FL_STAT_P = 1 } fl_stat_kind;

const char* fl_status_str(fl_status s);
/* Library version, "major.minor.patch". */
const char* fl_version(void);

/* Number of kernel launches the library has issued in this process. */
int64_t fl_launch_count(void);

/* Number of bf16 projection GEMMs that ran on the CUDA-core kernel instead of the
 * tensor cores because their shape cannot be tiled (K not a multiple of 64 or N not a
 * multiple of 128), in this process. Binary32 projections always use the CUDA cores
 * and are not counted. */
int64_t fl_gemm_bf16_cuda_core_count(void);

/* Attention calls (fl_sparse_loop_attn, fl_sparse_loop_attn_batched and the attention of
 * fl_loop_step) by the kernel path that ran, in this process: out[i] for i < n of
 *   0 sparse query tiles over column ranges (store staged as fp16 rows, set bitmaps)
 *   1 sparse query tiles over the union of the tile's sets (staged rows, set bitmaps)
 *   2 sparse query tiles decoding the store themselves (single-tile and batched calls)
 *   3 dense query tiles (the producer of the next loop's statistics)
 *   4 sparse warp-per-query kernel   5 dense warp-per-query kernel   6 general kernel
 *   7 sparse calls of few queries (decode): one CTA per (query, head) streaming its
 *     carried columns from the quantised store
 * Returns the number of paths (8); n may be smaller. Counted when the host dispatches,
 * so a captured graph's replays are not counted again. */
int32_t fl_attn_path_counts(int64_t* out, int32_t n);

/* Measurement hook. With n > 0 the library records the caller's events begin[i] and
 * end[i] (each a cudaEvent_t passed as void*) on the launch stream around its next n
 * launches of one kind (0: the projection GEMMs, 1: the attention kernel);
 * fl_timing_recorded(kind) says how many pairs were recorded. n = 0 turns it off.
 * During stream capture the records become external event-record nodes of the graph
 * (recorded again at every replay). Not thread-safe: set it from the issuing thread. */
fl_status fl_set_timing_events(int32_t kind, void* const* begin, void* const* end, int32_t n);
int32_t fl_timing_recorded(int32_t kind);

/* Synchronises `stream`, returns the first error a kernel recorded on the current
 * device since the last call (FL_OK if none) and clears it. */
fl_status fl_check_device_status(void* stream);
/* Detail of the error the last fl_check_device_status returned: for FL_ERR_TIMEOUT from
 * a tensor-core attention kernel, the code of the wait that ran out (which kernel, role
 * and barrier; listed beside the kernels' sources); 0 when there is none. */
int32_t fl_last_error_detail(void);

/* ------------------------------------------------------------------------- *
 * Active-token selection (§4.1): rank the rows updated in the previous loop by
 * their normalized hidden-state change
 *     delta_t = ||h_cur[t] - h_prev[t]||_2 / max(||h_prev[t]||_2, 1e-30)
 * and keep the k largest (equal deltas: the smaller row wins), ascending.
 *
 * h_cur, h_prev  device [n_rows][d] of dtype dt (FL_F32 or FL_BF16)
 * row_tok        device [n_rows] token id of each row, ascending; NULL: row i is token i
 * k              0 <= k <= n_rows
 * out_tok        device [k] token ids of the kept rows, ascending
 * out_pos        device [k] their row positions (nullable)
 * out_delta      device [n_rows] the deltas in binary32 (nullable)
 * ws             device workspace of fl_select_active_workspace_bytes(n_rows) bytes
 * Limits: 1 <= n_rows <= 2^24, 1 <= d, d % 8 == 0 for FL_BF16 and d % 4 == 0 for FL_F32.
 * ------------------------------------------------------------------------- */
size_t fl_select_active_workspace_bytes(int32_t n_rows);
fl_status fl_select_active(const void* h_cur, const void* h_prev, fl_dtype dt,
                           int32_t n_rows, int32_t d, const int32_t* row_tok, int32_t k,
                           int32_t* out_tok, int32_t* out_pos, float* out_delta,
                           void* ws, size_t ws_bytes, void* stream);

/* Allocation-free variant of fl_select_active, for callers that cannot allocate
 * device memory at all - for instance code embedded in a host runtime that owns every
 * device byte and hands a plugin only its input and output buffers, or a deployment
 * that plans a fixed memory budget up front and forbids allocations afterwards.
 * (The paper has no counterpart: this is a packaging choice of the library.)
 * Same computation and outputs as fl_select_active (out_delta not offered); the
 * normalized changes go to a fixed scratch array of FL_SELECT_NOALLOC_MAX_ROWS floats
 * (256 KiB) built into the library, which every GPU that loads the library holds until
 * the process exits. n_rows above that maximum returns FL_ERR_SHAPE without launching.
 * The first call on a device looks up the scratch array's device address (with that
 * device current) and caches it: make that first call before any stream capture. The
 * cached address belongs to the device's primary context: after cudaDeviceReset (or
 * anything else that destroys that context) it is stale, so do not call this entry point
 * again in that process. The device status word of every entry point is cached the
 * same way.
 * Every call on a device shares the one scratch array, so calls whose work overlaps on
 * the GPU (other streams or host threads) race; the caller must serialise them. No
 * scratch content has to survive between calls. Calls no allocator of any kind. */
#define FL_SELECT_NOALLOC_MAX_ROWS 65536
fl_status fl_select_active_noalloc(const void* h_cur, const void* h_prev, fl_dtype dt,
                                   int32_t n_rows, int32_t d, const int32_t* row_tok,
                                   int32_t k, int32_t* out_tok, int32_t* out_pos, void* stream);

/* ------------------------------------------------------------------------- *
 * Row gather / scatter into compact buffers (§4.4: selected tokens are gathered
 * into compact, GEMM-friendly buffers; §4.1: results go back to their rows).
 *   FL_GATHER:  dst[i] = src[idx[i]]   for i < n_idx   (src has n_full rows)
 *   FL_SCATTER: dst[idx[i]] = src[i]   for i < n_idx   (dst has n_full rows)
 * Rows hold row_elems elements of dtype dt. idx is a device int32 array; an
 * entry outside [0, n_full) is skipped and recorded as FL_ERR_RANGE.
 * Scatter with repeated indices leaves one of the rows (unspecified which).
 * ------------------------------------------------------------------------- */
fl_status fl_gather_scatter(fl_gs_op op, const void* src, void* dst, const int32_t* idx,
                            int32_t n_idx, int32_t n_full, int32_t row_elems, fl_dtype dt,
                            void* stream);

/* ------------------------------------------------------------------------- *
 * KV store of one layer over loops 1..n_loops (§3.3: a quantised base state plus
 * quantised cross-loop residuals; §4.3: residuals only for active tokens;
 * Appendix E: asymmetric group-wise min/max quantisation, same scheme for base
 * and residuals).
 *
 * Loop 1 (base) holds every token; loop r >= 2 holds compact rows, one per token
 * active in loop r, in ascending token order. For loop r and K (kv=0) / V (kv=1):
 *   codes[kv][r]  device uint8 [rows][H][hd*b/8], b-bit codes packed little-endian,
 *                 low bits first (b = 0: binary32 values, [rows][H][hd] floats)
 *   sz[kv][r]     device binary16 bits [rows][H][hd/group][2] = (scale, offset);
 *                 unused (may be NULL) when b = 0
 * slot            device int32 [n_loops+1][n_tok]: row of token t in loop r's arrays,
 *                 or -1 (row 0 unused; row 1 is the identity once loop 1 is written)
 * vnorm           device float [n_tok][H]: ||V^[t]||_2 of the latest written loop
 *                 (nullable; needed for FL_STAT_PV statistics)
 * Reconstruction of loop r: K^ = base (dequantised); then for r' = 2..r with
 * slot[r'][t] >= 0: K^ = fl32(K^ + deq_r') (or K^ = value_r' when res_bits[r'] = 0).
 * Quantiser of a group of `group` binary32 values x (per token, head, along hd):
 *   z = fp16_RD(min x); s = fp16_RU(f32_RU(f32_RU(max x - z) / (2^b - 1)));
 *   code = s == 0 ? 0 : clamp(rint(f32(f32(x - z) / s)), 0, 2^b - 1);
 *   deq  = fmaf(code, s, z).
 * ------------------------------------------------------------------------- */
typedef struct {
  int32_t n_tok, n_heads, head_dim, group;
  int32_t base_bits;                       /* 0 or 8 */
  int32_t n_loops;                         /* R */
  int32_t res_bits[FL_MAX_LOOPS + 1];      /* loop r >= 2: 0, 2, 4 or 8 */
  uint8_t* codes[2][FL_MAX_LOOPS + 1];
  uint16_t* sz[2][FL_MAX_LOOPS + 1];
  int32_t* slot;
  float* vnorm;
} fl_kv_desc;

/* Write loop `loop` of the store (§4.3; the fusion of the cross-loop KV update
 * and quantisation that §4.4 describes).
 * loop == 1: quantises every token's post-RoPE k and v with base_bits; act_tok must
 *            be NULL and n_act == n_tok.
 * loop >= 2: for the n_act tokens in act_tok (device, ascending, unique), quantises
 *            the residual x = fl32(k - K^_{loop-1}) against the reconstructed
 *            previous state with res_bits[loop]; rewrites slot[loop][*].
 * k_new, v_new  device [n_act][H][hd] of dtype dt, post-RoPE, row i = token act_tok[i]
 * Also refreshes vnorm (if set) for the written tokens. An fp16 overflow of a scale
 * or offset records FL_ERR_RANGE (codes of that group are 0). */
fl_status fl_kv_residual_quant(const fl_kv_desc* kv, int32_t loop, const void* k_new,
                               const void* v_new, fl_dtype dt, const int32_t* act_tok,
                               int32_t n_act, void* stream);

/* Append tokens to loop `loop` of the store without disturbing the other tokens (a
 * decode step's new token, §4.3 applied to generation). loop 1: base rows of the tokens
 * act_tok[i] (the row of a token is its id). loop >= 2: residual rows row0 + i against
 * the tokens' reconstruction at loop - 1 (which must exist), slot[loop][act_tok[i]] =
 * row0 + i; other slot entries are kept. k_new, v_new: device [n_act][H][hd] of dtype dt;
 * act_tok: device int32 [n_act]. Refreshes vnorm for the written tokens. */
fl_status fl_kv_append(const fl_kv_desc* kv, int32_t loop, const void* k_new, const void* v_new,
                       fl_dtype dt, const int32_t* act_tok, int32_t n_act, int32_t row0,
                       void* stream);

/* The reconstruction K^_loop, V^_loop of the n tokens tok[i] (device int32), as the
 * attention reads it: the base, then the residual row of every loop 2..loop whose slot
 * lists the token, added in binary32 in loop order (a raw loop replaces the value).
 * out_k, out_v: device float [n][H][hd]. For inspection and for the residual-vs-full
 * quantisation diagnostic (§3.3); a token outside [0, n_tok) records FL_ERR_RANGE. */
fl_status fl_kv_reconstruct(const fl_kv_desc* kv, int32_t loop, const int32_t* tok, int32_t n,
                            float* out_k, float* out_v, void* stream);

/* ------------------------------------------------------------------------- *
 * Loop-aware sparse attention (§4.2), and the dense causal attention of a loop
 * whose successor is sparse (the producer of the statistics).
 *
 * Score s_ij = q_i . K^_loop[j] / sqrt(hd) + col_bias[j], causal j <= q_tok[i].
 * Sparse (sel != NULL), per query i and head h with S = sel row, m, u of row q_row[i]:
 *     p~_ij = m * softmax over S of s_ij,   o_i = u + sum_{j in S} p~_ij V^[j]
 * (the selected logits are renormalised and rescaled by the cached mass m; u is the
 * unselected columns' contribution carried from the previous loop).
 * Dense (sel == NULL): o_i = sum_{j <= q_tok[i]} softmax(s)_ij V^[j].
 * Statistics for the next loop, when sel_out != NULL (contribution c_ij = P_ij *
 * ||V^[j]||, or P_ij with FL_STAT_P; P = p~ or the dense softmax):
 *   dense:  S' = {0} U top-k_next of c over [1, q_tok] (all of [0, q_tok] if
 *           q_tok <= k_next), m' = sum_{S'} P, u' = sum_{j not in S'} P V^[j]
 *   sparse: k_next >= |S|-1: S' = S, m' = m, u' = u; otherwise S' = {0} U top-k_next
 *           of c within S \ {0}, m' = sum_{S'} p~, u' = u + sum_{S \ S'} p~ V^[j].
 *   Equal statistics: the smaller column wins. Column sets are ascending and padded
 *   with FL_SENTINEL up to the stride.
 * Statistics layout: sel [H][rows][stride] uint16, mass [H][rows] float,
 * unsel [H][rows][hd] float. Output statistics may alias the input ones (in-place
 * update of the rows of this call's queries).
 * ------------------------------------------------------------------------- */
typedef struct {
  const void* q; fl_dtype q_dt;        /* device [n_q][H][hd] post-RoPE */
  int32_t n_q;
  const int32_t* q_tok;                /* device [n_q] token position of each query */
  const fl_kv_desc* kv; int32_t loop;  /* attend to K^_loop, V^_loop */
  const float* col_bias;               /* device [n_tok] or NULL */
  /* carried statistics (sel == NULL: dense attention) */
  const uint16_t* sel; const float* mass; const float* unsel;
  int32_t stat_rows, sel_stride;       /* rows of the statistics arrays; stride >= k+1 */
  const int32_t* q_row;                /* device [n_q] statistics row per query; NULL: q_tok */
  /* statistics for the next loop (sel_out == NULL: none) */
  int32_t k_next;
  uint16_t* sel_out; float* mass_out; float* unsel_out;
  int32_t out_stride;                  /* >= k_next + 1; rows as stat_rows */
  int32_t stat_kind;                   /* fl_stat_kind */
  void* out; fl_dtype out_dt;          /* device [n_q][H][hd] */
  void* ws; size_t ws_bytes;          /* device workspace, see below */
} fl_attn_args;

/* Device workspace of a call (a fl_attn_args whose ws fields are ignored), 0 if none:
 * for a sparse call of more than 128 queries (head_dim 128, no statistics written or in
 * place with an unchanged budget) the store staged once as fp16 rows, K^ and V^
 * [H][n_tok][hd], then the carried sets as column bitmaps [H][n_q][ceil(n_tok/128)*4]
 * uint32; for a dense call the staged K^ and V^ (and K^ - fp16(K^) when it writes
 * statistics) after the statistics producer's buffers. Sparse calls of at most 128
 * queries need none. fl_sparse_loop_attn rejects a call whose ws_bytes is smaller
 * (FL_ERR_WORKSPACE, before any launch). The workspace serves one call at a time. */
size_t fl_sparse_loop_attn_workspace_bytes(const fl_attn_args* a);
fl_status fl_sparse_loop_attn(const fl_attn_args* a, void* stream);

/* n sparse calls (sel != NULL) in one launch - batched decode, where every sequence has
 * its own store and statistics. The calls must agree on n_q, heads, head_dim, sel_stride,
 * dtypes, stat_kind, k_next and whether statistics are written; stores must be quantised
 * throughout (8-bit base, 2/4/8-bit residuals). ws: device workspace of
 * fl_sparse_loop_attn_batched_workspace_bytes(n) bytes, receiving the calls' arguments
 * (copied from host memory during the call, so the call is not meant for stream capture). */
size_t fl_sparse_loop_attn_batched_workspace_bytes(int32_t n);
fl_status fl_sparse_loop_attn_batched(const fl_attn_args* args, int32_t n, void* ws,
                                      size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------------- *
 * The shared block on compact rows (§1: a shared N-layer block applied R times;
 * §4.1: a sparse loop computes only its active rows; §4.4: regular GEMMs on the
 * gathered rows). Pre-norm layer, weights shared across loops:
 *   x <- x + Attn(RMSNorm(x)) W_o^T ;  x <- x + W_down(silu(RMSNorm(x) W_gate^T) *
 *   (RMSNorm(x) W_up^T)),  RMSNorm(x) = x / sqrt(mean(x^2) + eps) * gamma,
 *   RoPE rotate-half with theta on q and k at the tokens' positions.
 * Weights are [out][in] row-major of dtype dt: w_qkv [3d][d] (q, k, v rows),
 * w_o [d][d], w_gate_up [2F][d] (gate rows, then up rows), w_down [d][F]; gains are
 * float [d]. The residual stream x is binary32.
 * ------------------------------------------------------------------------- */
typedef struct {
  const void* w_qkv; const void* w_o; const void* w_gate_up; const void* w_down;
  const float* g_attn; const float* g_ffn;
} fl_layer_weights;

typedef struct {
  int32_t n_tok, d_model, n_heads, head_dim, d_ffn, n_layers;
  fl_dtype dt;                      /* weights and GEMM operands */
  float rms_eps, rope_theta;
  const fl_layer_weights* layers;   /* HOST array [n_layers] of device pointers */
  const float* col_bias;            /* device [n_tok] logit bias per column, nullable */
} fl_model;

/* Device workspace of the block calls: the RoPE table, the projection GEMMs' stream-K
 * scratch (partial tiles and hand-over flags, cleared by every call) and the half-layer
 * intermediates. One workspace serves one call at a time (calls on different streams
 * need their own). Depends on the current device's SM count. */
size_t fl_block_workspace_bytes(const fl_model* m, int32_t n_rows);
/* RMSNorm + fused q/k/v projection + RoPE of n_rows rows x (device float [n][d])
 * at positions pos (device int32 [n]); writes q, k, v (device float [n][H][hd]). */
fl_status fl_block_qkv(const fl_model* m, int32_t layer, const float* x, int32_t n_rows,
                       const int32_t* pos, float* q, float* k, float* v,
                       void* ws, size_t ws_bytes, void* stream);
/* fl_block_qkv with the KV store update of loop `loop` (fl_kv_residual_quant's
 * computation, bit for bit) done in the projection's epilogue - the fusion of the
 * cross-loop KV update and quantisation with the projection that §4.4 describes.
 * The rows' tokens are pos[i] (loop 1: every token, in order; loop >= 2: ascending,
 * residual row i), and slot[loop] is rewritten. k_out / v_out (nullable) also receive
 * the post-RoPE k and v. Needs bf16 weights, group 32, an 8-bit base and 2/4/8-bit
 * residual loops (otherwise FL_ERR_UNSUPPORTED). Workspace: fl_block_workspace_bytes. */
fl_status fl_block_qkv_kv(const fl_model* m, int32_t layer, const fl_kv_desc* kv, int32_t loop,
                          const float* x, int32_t n_rows, const int32_t* pos, float* q,
                          float* k_out, float* v_out, void* ws, size_t ws_bytes, void* stream);
/* x += attn W_o^T, then the SwiGLU FFN with residual, in place on x (device float
 * [n][d]); attn is device [n][d] of dtype m->dt. */
fl_status fl_block_out_ffn(const fl_model* m, int32_t layer, float* x, int32_t n_rows,
                           const void* attn, void* ws, size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------------- *
 * One loop of the looped model with the lazy updates (§4).
 * Loop 1: every token, dense attention, base KV for every token. Loops before
 * first_sparse: every token, residual KV. Loop r >= first_sparse: A_r = the
 * n_active[r] tokens of A_{r-1} with the largest normalized change; gather;
 * per layer: q/k/v, residual KV, attention (sparse when col_k[r] > 0), output
 * projection and FFN; scatter. A loop whose successor has col_k > 0 writes the
 * statistics with that budget.
 * ------------------------------------------------------------------------- */
typedef struct {
  int32_t n_loops;                       /* R */
  int32_t first_sparse;                  /* first loop with token selection, >= 2 */
  int32_t n_active[FL_MAX_LOOPS + 1];    /* tokens recomputed in loop r (r = 1: n_tok) */
  int32_t col_k[FL_MAX_LOOPS + 1];       /* columns kept per query in loop r besides the
                                            sink; 0 = dense attention in loop r */
  int32_t stat_kind;                     /* fl_stat_kind */
} fl_schedule;

/* Inspection taps of fl_loop_step, for stage-by-stage checks of a loop against a
 * reference on identical inputs (NULL in normal use; a tapped step launches extra
 * copy kernels and, at loop 1, also stores the projection's k and v). For each of the
 * n tokens tok[i] (device int32, any order) that the loop recomputes, row i of layer l
 * (at offset (l * n + i) * d elements) receives, for every non-NULL buffer:
 *   x_in   the layer's input row (float)        q, k, v  post-RoPE projections (float)
 *   attn   the attention output (dtype m->dt)   x_out    the layer's output row (float)
 * Rows of tokens the loop does not recompute are not written. */
typedef struct {
  int32_t n;
  const int32_t* tok;
  float* x_in; float* q; float* k; float* v;
  void* attn;
  float* x_out;
} fl_loop_taps;

typedef struct {
  float* h;            /* device [n_tok][d]: h_{r-1} on entry, h_r on return. Before
                          loop 1 the caller writes the embeddings h_0 here. */
  float* x_cur;        /* device [n_tok][d]: rows of the last loop's tokens, new state */
  float* x_prev;       /* device [n_tok][d]: the same rows' previous state. After
                          loop 1 it holds h_0 (every row); loop 2 ranks tokens by
                          (h, x_prev). The caller may rewrite it between loops. */
  int32_t* act[FL_MAX_LOOPS + 1];   /* device [n_active[r]] token ids of loop r (r >= 2) */
  int32_t* act_pos;    /* device [n_tok] positions of A_r within A_{r-1} */
  float* delta;        /* device [n_tok] normalized changes of the last ranking */
  fl_kv_desc* kv;      /* HOST array [n_layers] */
  uint16_t** sel;      /* HOST array [n_layers] of device [H][n_tok][sel_stride] */
  float** mass;        /* HOST array [n_layers] of device [H][n_tok] */
  float** unsel;       /* HOST array [n_layers] of device [H][n_tok][hd] */
  int32_t sel_stride;  /* >= max col_k + 1 */
  void* ws; size_t ws_bytes;
  const fl_loop_taps* taps;  /* HOST pointer, nullable: inspection copies (see above) */
} fl_loop_state;

size_t fl_loop_step_workspace_bytes(const fl_model* m, const fl_schedule* s);
fl_status fl_loop_step(const fl_model* m, fl_loop_state* st, const fl_schedule* s,
                       int32_t loop, void* stream);

#ifdef __cplusplus
}
#endif
#endif /* FL_H */
