// static_scratch.cu -- csa_index_score_topk_static: the indexer scan + top-k
// for callers that cannot allocate device memory at the call site (see
// cskv.h). Its scratch (the per-query fp32 score rows) is a file-scope
// __device__ array of fixed size instead of a caller-provided workspace.
//
// Host code may not pass the array's name to a kernel: on the host that name
// is a stand-in object, not a device address. The device address is fetched
// once per device with cudaGetSymbolAddress, with that device current, and
// cached; the first call on each device does this set-up.
#include <cuda_runtime.h>
#include <stdint.h>
#include <string.h>

#include <mutex>

#include "cskv.h"
#include "cskv_internal.h"

namespace {

// CSKV_STATIC_INDEX_SCRATCH_FLOATS fp32 score slots (16 MiB), resident on
// every GPU that loads this library until the process exits.
static __device__ __align__(256) float g_index_scratch[CSKV_STATIC_INDEX_SCRATCH_FLOATS];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_ptr[kMaxDevices] = {};

// Device address of g_index_scratch on the current device (set up on first use).
cudaError_t scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_index_scratch);
    if (e != cudaSuccess) return e;
    g_ptr[dev] = p;
  }
  *out = g_ptr[dev];
  return cudaSuccess;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

extern "C" cskv_status csa_index_score_topk_static(const cskv_index_args* a, void* stream) {
  // the same argument rules as csa_index_score_topk
  size_t need = 0;
  cskv_status s = csa_index_ws_bytes(a, &need);
  if (s != CSKV_OK) return s;
  const cskv_layer* L = a->layer;
  if (!L->page_table || !L->idx_pool || !aligned16(L->idx_pool)) return CSKV_ERR_INVALID_ARG;
  if (L->idx_dtype == CSKV_FP4_E2M1 && !L->idx_scale) return CSKV_ERR_INVALID_ARG;
  if (a->n_q == 0) return CSKV_OK;
  if (!a->q_seq || !a->q_pos || !a->q_idx || !a->w || !a->out_idx || !a->out_cnt || !aligned16(a->q_idx))
    return CSKV_ERR_INVALID_ARG;
  if (L->idx_dtype == CSKV_FP4_E2M1 && !a->q_idx_scale) return CSKV_ERR_INVALID_ARG;
  if (need > sizeof(g_index_scratch)) return CSKV_ERR_WORKSPACE;  // beyond the static maximum
  void* ws = nullptr;
  if (scratch_address(&ws) != cudaSuccess) return CSKV_ERR_CUDA;
  // nothing in the scratch needs clearing: the scan writes every score the selection reads
  return csa_index_score_topk(a, ws, sizeof(g_index_scratch), stream);
}
