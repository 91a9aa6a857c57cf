// Allocation-free variant of the active-token selection, for callers that cannot
// allocate device memory.
//
// Some callers run where no device allocation is possible or allowed: a host runtime
// that hands a plugin only its input and output buffers and owns every byte of device
// memory itself, or a deployment that pre-plans a fixed memory budget and forbids
// allocations after start-up. fl_select_active needs a workspace of n_rows floats for
// the normalized changes; this entry point keeps that scratch in a fixed array inside
// the library instead, so the caller passes inputs and outputs only.
//
// The scratch is a file-scope __device__ array of FL_SELECT_NOALLOC_MAX_ROWS floats
// (256 KiB). Every GPU that loads the library holds it until the process exits. Host
// code cannot use the array's name as a device address (on the host that name is a
// stand-in symbol, not device memory), so the first call on each device looks up the
// array's device address with cudaGetSymbolAddress while that device is current and
// caches it; make that first call before any stream capture. Every call on a device
// shares the one array: calls whose work overlaps on the GPU (other streams, other
// host threads) race and must be serialised by the caller. The kernel writes every
// entry it later reads (one per row), so nothing has to be cleared between calls.
#include <mutex>

#include "fl_internal.cuh"

static __device__ __align__(256) float g_select_scratch[FL_SELECT_NOALLOC_MAX_ROWS];

namespace {

float* scratch_for_current_device(fl_status* rc) {
  static float* cache[128] = {nullptr};
  static std::mutex mu;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 128) {
    *rc = FL_ERR_CUDA;
    return nullptr;
  }
  std::lock_guard<std::mutex> lock(mu);
  if (!cache[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_select_scratch) != cudaSuccess || !p) {
      *rc = FL_ERR_CUDA;
      return nullptr;
    }
    cache[dev] = static_cast<float*>(p);
  }
  *rc = FL_OK;
  return cache[dev];
}

}  // namespace

extern "C" fl_status fl_select_active_noalloc(const void* h_cur, const void* h_prev,
                                              fl_dtype dt, int32_t n_rows, int32_t d,
                                              const int32_t* row_tok, int32_t k,
                                              int32_t* out_tok, int32_t* out_pos,
                                              void* stream) {
  if (!h_cur || !h_prev || !out_tok) return FL_ERR_INVALID_ARG;
  if (dt != FL_F32 && dt != FL_BF16) return FL_ERR_UNSUPPORTED;
  if (n_rows < 1 || d < 1 || k < 0 || k > n_rows) return FL_ERR_SHAPE;
  if (n_rows > FL_SELECT_NOALLOC_MAX_ROWS) return FL_ERR_SHAPE;   // beyond the fixed scratch
  if (d % (dt == FL_BF16 ? 8 : 4) != 0) return FL_ERR_SHAPE;
  if ((uintptr_t)h_cur % 16 || (uintptr_t)h_prev % 16) return FL_ERR_INVALID_ARG;
  fl_status rc;
  float* delta = scratch_for_current_device(&rc);
  if (!delta) return rc;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (fl::launch_row_delta(h_cur, h_prev, dt, n_rows, d, delta, s) != cudaSuccess)
    return FL_ERR_CUDA;
  if (fl::launch_topk_rows(delta, n_rows, k, row_tok, out_tok, out_pos, fl::status_word(), s) !=
      cudaSuccess)
    return FL_ERR_CUDA;
  return FL_OK;
}
