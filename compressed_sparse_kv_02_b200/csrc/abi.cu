// abi.cu -- the extern "C" entry points of libcskv.so (declared in cskv.h):
// argument checks on the host, workspace sizing, and kernel dispatch. No
// allocation, no synchronisation (except cskv_get_status), no state.
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>
#include <string.h>

#include "cskv.h"
#include "cskv_internal.h"

namespace {

using cskv::AttendParams;
using cskv::FoldParams;
using cskv::IndexParams;

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool pow2(int v) { return v > 0 && (v & (v - 1)) == 0; }

cskv_status from_cuda(cudaError_t e) {
  if (e == cudaSuccess) return CSKV_OK;
  if (e == cudaErrorNotSupported) return CSKV_ERR_UNSUPPORTED;
  return CSKV_ERR_CUDA;
}

int sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) return 148;
  return n;
}

// block overlap of a layer (0 for callers whose struct_size ends before the field)
int32_t layer_overlap(const cskv_layer* L) {
  return L->struct_size >= offsetof(cskv_layer, overlap) + sizeof(int32_t) ? L->overlap : 0;
}

// Shape/dtype rules of a layer (pointers not checked here).
cskv_status check_layer_shape(const cskv_layer* L) {
  if (!L || L->struct_size < offsetof(cskv_layer, overlap)) return CSKV_ERR_INVALID_ARG;
  if (L->kind != CSKV_LAYER_CSA && L->kind != CSKV_LAYER_HCA) return CSKV_ERR_INVALID_ARG;
  if (L->n_win < 1 || !pow2(L->m) || L->m > L->n_win) return CSKV_ERR_INVALID_ARG;
  // the ov tokens an entry borrows from the block before it must still be in the ring
  if (layer_overlap(L) < 0 || layer_overlap(L) > L->n_win - L->m) return CSKV_ERR_INVALID_ARG;
  if (L->d_qk < 16 || L->d_qk > 1024 || L->d_qk % 16) return CSKV_ERR_INVALID_ARG;
  if (L->d_v < 16 || L->d_v > L->d_qk || L->d_v % 16) return CSKV_ERR_INVALID_ARG;
  if (L->page_size < 16 || L->page_size % 16) return CSKV_ERR_INVALID_ARG;
  if (L->kv_dtype != CSKV_BF16 && L->kv_dtype != CSKV_FP8_E4M3) return CSKV_ERR_UNSUPPORTED;
  if (L->gate_cols != 1 && L->gate_cols != L->d_qk) return CSKV_ERR_INVALID_ARG;
  if (L->n_seqs < 1 || L->max_pages_per_seq < 1 || L->n_pages < 1) return CSKV_ERR_INVALID_ARG;
  if (L->kind == CSKV_LAYER_CSA) {
    if (L->idx_dtype != CSKV_BF16 && L->idx_dtype != CSKV_FP4_E2M1) return CSKV_ERR_UNSUPPORTED;
    if (L->d_idx < 32 || L->d_idx > 1024 || L->d_idx % 32) return CSKV_ERR_INVALID_ARG;
    if (L->gate_cols_idx != 1 && L->gate_cols_idx != L->d_idx) return CSKV_ERR_INVALID_ARG;
  }
  return CSKV_OK;
}

cskv_status check_layer_ptrs(const cskv_layer* L) {
  if (!L->page_table || !L->kv_pool || !L->ring_x || !L->ring_z) return CSKV_ERR_INVALID_ARG;
  if (!aligned16(L->kv_pool) || !aligned16(L->ring_x)) return CSKV_ERR_INVALID_ARG;
  if (L->kv_dtype == CSKV_FP8_E4M3 && !L->kv_scale) return CSKV_ERR_INVALID_ARG;
  if (L->kind == CSKV_LAYER_CSA) {
    if (!L->idx_pool || !L->ring_xi || !L->ring_zi || !aligned16(L->idx_pool) || !aligned16(L->ring_xi))
      return CSKV_ERR_INVALID_ARG;
    if (L->idx_dtype == CSKV_FP4_E2M1 && !L->idx_scale) return CSKV_ERR_INVALID_ARG;
  }
  return CSKV_OK;
}

void fill_streams(FoldParams& p, const cskv_layer* L, const void* x, const void* z, const void* xi,
                  const void* zi, bool with_idx) {
  memset(&p.s, 0, sizeof(p.s));
  cskv::FoldStream& a = p.s[0];
  a.x = static_cast<const uint16_t*>(x);
  a.z = static_cast<const uint16_t*>(z);
  a.ring_x = static_cast<const uint16_t*>(L->ring_x);
  a.ring_z = static_cast<const uint16_t*>(L->ring_z);
  a.ring_x_w = static_cast<uint16_t*>(L->ring_x);
  a.ring_z_w = static_cast<uint16_t*>(L->ring_z);
  a.bias = L->pos_bias;
  a.d = L->d_qk;
  a.gc = L->gate_cols;
  a.out_dtype = L->kv_dtype;
  a.pool = L->kv_pool;
  a.scale_f32 = L->kv_scale;
  p.n_streams = 1;
  if (with_idx) {
    cskv::FoldStream& b = p.s[1];
    b.x = static_cast<const uint16_t*>(xi);
    b.z = static_cast<const uint16_t*>(zi);
    b.ring_x = static_cast<const uint16_t*>(L->ring_xi);
    b.ring_z = static_cast<const uint16_t*>(L->ring_zi);
    b.ring_x_w = static_cast<uint16_t*>(L->ring_xi);
    b.ring_z_w = static_cast<uint16_t*>(L->ring_zi);
    b.bias = L->pos_bias_idx;
    b.d = L->d_idx;
    b.gc = L->gate_cols_idx;
    b.out_dtype = L->idx_dtype;
    b.pool = L->idx_pool;
    b.scale_e4m3 = L->idx_scale;
    p.n_streams = 2;
  }
  p.m = L->m;
  p.ov = layer_overlap(L);
  p.n_win = L->n_win;
  p.page_size = L->page_size;
  p.max_pages_per_seq = L->max_pages_per_seq;
  p.n_pages = L->n_pages;
  p.page_table = L->page_table;
  p.n_seqs_layer = L->n_seqs;
}

cskv_status compress_impl(const cskv_compress_args* a, void* stream, int kind) {
  if (!a || a->struct_size < sizeof(cskv_compress_args)) return CSKV_ERR_INVALID_ARG;
  const cskv_layer* L = a->layer;
  cskv_status s = check_layer_shape(L);
  if (s) return s;
  if (L->kind != kind) return CSKV_ERR_INVALID_ARG;
  if ((s = check_layer_ptrs(L))) return s;
  if (a->n_seq < 0 || a->n_tok < 0 || a->tok0 < 0) return CSKV_ERR_INVALID_ARG;
  if (a->n_tok % L->m || a->tok0 % L->m) return CSKV_ERR_INVALID_ARG;
  if (a->n_seq == 0 || a->n_tok == 0) return CSKV_OK;
  const bool csa = kind == CSKV_LAYER_CSA;
  if (!a->seq_ids || !a->x || !a->z || !aligned16(a->x)) return CSKV_ERR_INVALID_ARG;
  if (L->gate_cols != 1 && !aligned16(a->z)) return CSKV_ERR_INVALID_ARG;
  if (csa && (!a->xi || !a->zi || !aligned16(a->xi) || (L->gate_cols_idx != 1 && !aligned16(a->zi))))
    return CSKV_ERR_INVALID_ARG;
  if ((a->tok0 + a->n_tok) / L->m > (int64_t)L->max_pages_per_seq * L->page_size) return CSKV_ERR_INVALID_ARG;
  FoldParams p;
  memset(&p, 0, sizeof(p));
  fill_streams(p, L, a->x, a->z, a->xi, a->zi, csa);
  p.n_seq = a->n_seq;
  p.seq_ids = a->seq_ids;
  p.tok0 = a->tok0;
  p.n_tok = a->n_tok;
  p.status = a->d_status;
  return from_cuda(cskv::launch_fold_bulk(p, static_cast<cudaStream_t>(stream)));
}

// struct_size of the index args before score_bf16 was added (such callers get fp32 selection)
constexpr size_t kIndexArgsV1 = offsetof(cskv_index_args, score_bf16);

int32_t index_score_bf16(const cskv_index_args* a) {
  return a->struct_size >= offsetof(cskv_index_args, score_bf16) + sizeof(int32_t) ? a->score_bf16 : 0;
}

cskv_status check_index(const cskv_index_args* a) {
  if (!a || a->struct_size < kIndexArgsV1) return CSKV_ERR_INVALID_ARG;
  if (index_score_bf16(a) != 0 && index_score_bf16(a) != 1) return CSKV_ERR_INVALID_ARG;
  const cskv_layer* L = a->layer;
  cskv_status s = check_layer_shape(L);
  if (s) return s;
  if (L->kind != CSKV_LAYER_CSA) return CSKV_ERR_INVALID_ARG;
  if (a->n_q < 0 || a->n_heads_idx < 1 || a->n_heads_idx > 16 || a->k < 1 || a->max_pos < 0)
    return CSKV_ERR_INVALID_ARG;
  if (L->d_idx != 64 && L->d_idx != 128) return CSKV_ERR_UNSUPPORTED;
  if (L->idx_dtype == CSKV_FP4_E2M1 && a->n_heads_idx > 8 && L->d_idx != 128) return CSKV_ERR_UNSUPPORTED;
  if (a->n_q > 4096) return CSKV_ERR_UNSUPPORTED;
  if ((a->max_pos + 1) / L->m > (int64_t)1 << 31) return CSKV_ERR_UNSUPPORTED;
  return CSKV_OK;
}

// struct_size of the attend args before the inverse-RoPE fields (such callers get none)
constexpr size_t kAttendArgsV1 = offsetof(cskv_attend_args, rope_dims);

int32_t attend_rope_dims(const cskv_attend_args* a) {
  return a->struct_size >= offsetof(cskv_attend_args, rope_base) + sizeof(float) ? a->rope_dims : 0;
}

cskv_status check_attend(const cskv_attend_args* a, int kind) {
  if (!a || a->struct_size < kAttendArgsV1) return CSKV_ERR_INVALID_ARG;
  {
    const int32_t rd = attend_rope_dims(a);
    if (rd < 0 || rd % 2 || (a->layer && rd > a->layer->d_v) || (rd > 0 && !(a->rope_base > 0.f)))
      return CSKV_ERR_INVALID_ARG;
  }
  const cskv_layer* L = a->layer;
  cskv_status s = check_layer_shape(L);
  if (s) return s;
  if (L->kind != kind) return CSKV_ERR_INVALID_ARG;
  if (a->n_q < 0 || a->n_heads < 1 || a->max_pos < 0) return CSKV_ERR_INVALID_ARG;
  if (kind == CSKV_LAYER_CSA && a->k < 1) return CSKV_ERR_INVALID_ARG;
  if (!(a->sm_scale > 0.f)) return CSKV_ERR_INVALID_ARG;
  if (!cskv::attend_supported(L->d_qk, L->d_v, a->n_heads, L->kv_dtype)) return CSKV_ERR_UNSUPPORTED;
  if (a->n_q > 4096) return CSKV_ERR_UNSUPPORTED;
  return CSKV_OK;
}

void fill_attend(AttendParams& p, const cskv_attend_args* a, int kind) {
  const cskv_layer* L = a->layer;
  memset(&p, 0, sizeof(p));
  p.is_csa = kind == CSKV_LAYER_CSA;
  p.n_q = a->n_q;
  p.n_heads = a->n_heads;
  p.d_qk = L->d_qk;
  p.d_v = L->d_v;
  p.kv_dtype = L->kv_dtype;
  p.m = L->m;
  p.n_win = L->n_win;
  p.page_size = L->page_size;
  p.max_pages_per_seq = L->max_pages_per_seq;
  p.n_seqs_layer = L->n_seqs;
  p.n_pages = L->n_pages;
  p.page_table = L->page_table;
  p.kv_pool = L->kv_pool;
  p.kv_scale = L->kv_scale;
  p.ring_x = static_cast<const uint16_t*>(L->ring_x);
  p.q_seq = a->q_seq;
  p.q_pos = a->q_pos;
  p.max_pos = a->max_pos;
  p.q = static_cast<const uint16_t*>(a->q);
  p.sel_idx = a->sel_idx;
  p.sel_cnt = a->sel_cnt;
  p.k = a->k;
  p.sm_scale = a->sm_scale;
  p.out = static_cast<uint16_t*>(a->out);
  p.lse = a->lse;
  p.x_chunk = static_cast<const uint16_t*>(a->x_chunk);
  p.chunk_pos0 = a->chunk_pos0;
  p.chunk_len = a->chunk_len;
  p.status = a->d_status;
  p.rope_dims = attend_rope_dims(a);
  p.rope_base = p.rope_dims > 0 ? a->rope_base : 0.f;
  p.chunk_desc = a->struct_size >= offsetof(cskv_attend_args, chunk_desc) + sizeof(void*) ? a->chunk_desc : nullptr;
}

cskv_status attend_impl(const cskv_attend_args* a, void* ws, size_t ws_bytes, void* stream, int kind) {
  cskv_status s = check_attend(a, kind);
  if (s) return s;
  if ((s = check_layer_ptrs(a->layer))) return s;
  if (a->n_q == 0) return CSKV_OK;
  if (!a->q_seq || !a->q_pos || !a->q || !a->out || !aligned16(a->q) || !aligned16(a->out))
    return CSKV_ERR_INVALID_ARG;
  if (kind == CSKV_LAYER_CSA && (!a->sel_idx || !a->sel_cnt)) return CSKV_ERR_INVALID_ARG;
  if (a->x_chunk && (!aligned16(a->x_chunk) || a->chunk_len < 0 || a->chunk_pos0 < 0)) return CSKV_ERR_INVALID_ARG;
  const int n_sm = sm_count();
  AttendParams p;
  fill_attend(p, a, kind);
  const size_t need = cskv::attend_ws_bytes(p, n_sm);
  if (!ws || ws_bytes < need || !aligned16(ws)) return CSKV_ERR_WORKSPACE;
  return from_cuda(cskv::launch_attend(p, ws, n_sm, static_cast<cudaStream_t>(stream)));
}

// struct_size of the append args before emit_only was added (such callers get 0)
constexpr size_t kAppendArgsV1 = offsetof(cskv_append_args, d_status) + sizeof(int32_t*);
int32_t append_emit_only(const cskv_append_args* a) {
  return a->struct_size >= offsetof(cskv_append_args, emit_only) + sizeof(int32_t) ? a->emit_only : 0;
}

}  // namespace

extern "C" {

cskv_status cskv_layer_bytes(const cskv_layer* L, size_t* kv_pool, size_t* kv_scale, size_t* idx_pool,
                             size_t* idx_scale, size_t* ring_x, size_t* ring_z, size_t* ring_xi,
                             size_t* ring_zi) {
  cskv_status s = check_layer_shape(L);
  if (s) return s;
  const size_t rows = (size_t)L->n_pages * (size_t)L->page_size;
  const size_t ring_rows = (size_t)L->n_seqs * (size_t)L->n_win;
  const bool csa = L->kind == CSKV_LAYER_CSA;
  const size_t kv_elem = L->kv_dtype == CSKV_BF16 ? 2 : 1;
  if (kv_pool) *kv_pool = rows * L->d_qk * kv_elem;
  if (kv_scale) *kv_scale = L->kv_dtype == CSKV_FP8_E4M3 ? rows * sizeof(float) : 0;
  if (idx_pool) *idx_pool = csa ? (L->idx_dtype == CSKV_BF16 ? rows * L->d_idx * 2 : rows * L->d_idx / 2) : 0;
  if (idx_scale) *idx_scale = csa && L->idx_dtype == CSKV_FP4_E2M1 ? rows * (L->d_idx / 16) : 0;
  if (ring_x) *ring_x = ring_rows * L->d_qk * 2;
  if (ring_z) *ring_z = ring_rows * L->gate_cols * 2;
  if (ring_xi) *ring_xi = csa ? ring_rows * L->d_idx * 2 : 0;
  if (ring_zi) *ring_zi = csa ? ring_rows * L->gate_cols_idx * 2 : 0;
  return CSKV_OK;
}

cskv_status csa_compress_kv(const cskv_compress_args* args, void* stream) {
  return compress_impl(args, stream, CSKV_LAYER_CSA);
}

cskv_status hca_compress_kv(const cskv_compress_args* args, void* stream) {
  return compress_impl(args, stream, CSKV_LAYER_HCA);
}

cskv_status cskv_cache_append(const cskv_append_args* a, void* stream) {
  if (!a || a->struct_size < kAppendArgsV1) return CSKV_ERR_INVALID_ARG;
  const int32_t emit_only = append_emit_only(a);
  if (emit_only && a->ring_only) return CSKV_ERR_INVALID_ARG;
  const cskv_layer* L = a->layer;
  cskv_status s = check_layer_shape(L);
  if (s) return s;
  if ((s = check_layer_ptrs(L))) return s;
  if (a->n_seq < 0 || a->n_new < 0) return CSKV_ERR_INVALID_ARG;
  if (a->n_seq == 0 || a->n_new == 0) return CSKV_OK;
  if (!a->ring_only && a->n_new + L->m - 1 + layer_overlap(L) > L->n_win) return CSKV_ERR_INVALID_ARG;
  if (a->ring_only && a->n_new > L->n_win) return CSKV_ERR_INVALID_ARG;
  const bool csa = L->kind == CSKV_LAYER_CSA;
  if (!a->seq_ids || !a->pos || !a->x || !a->z || !aligned16(a->x)) return CSKV_ERR_INVALID_ARG;
  if (L->gate_cols != 1 && !aligned16(a->z)) return CSKV_ERR_INVALID_ARG;
  if (csa && (!a->xi || !a->zi || !aligned16(a->xi))) return CSKV_ERR_INVALID_ARG;
  FoldParams p;
  memset(&p, 0, sizeof(p));
  fill_streams(p, L, a->x, a->z, a->xi, a->zi, csa);
  p.n_seq = a->n_seq;
  p.seq_ids = a->seq_ids;
  p.pos = a->pos;
  p.n_new = a->n_new;
  p.ring_only = a->ring_only;
  p.emit_only = emit_only;
  p.status = a->d_status;
  return from_cuda(cskv::launch_append(p, static_cast<cudaStream_t>(stream)));
}

cskv_status csa_index_ws_bytes(const cskv_index_args* a, size_t* bytes) {
  cskv_status s = check_index(a);
  if (s) return s;
  if (!bytes) return CSKV_ERR_INVALID_ARG;
  *bytes = cskv::index_ws_bytes(a->n_q, a->max_pos, a->layer->m, a->layer->n_win);
  return CSKV_OK;
}

cskv_status csa_index_score_topk(const cskv_index_args* a, void* ws, size_t ws_bytes, void* stream) {
  cskv_status s = check_index(a);
  if (s) return s;
  const cskv_layer* L = a->layer;
  if (!L->page_table || !L->idx_pool || !aligned16(L->idx_pool)) return CSKV_ERR_INVALID_ARG;
  if (L->idx_dtype == CSKV_FP4_E2M1 && !L->idx_scale) return CSKV_ERR_INVALID_ARG;
  if (a->n_q == 0) return CSKV_OK;
  if (!a->q_seq || !a->q_pos || !a->q_idx || !a->w || !a->out_idx || !a->out_cnt || !aligned16(a->q_idx))
    return CSKV_ERR_INVALID_ARG;
  if (L->idx_dtype == CSKV_FP4_E2M1 && !a->q_idx_scale) return CSKV_ERR_INVALID_ARG;
  const size_t need = cskv::index_ws_bytes(a->n_q, a->max_pos, L->m, L->n_win);
  if (!ws || ws_bytes < need || !aligned16(ws)) return CSKV_ERR_WORKSPACE;
  IndexParams p;
  memset(&p, 0, sizeof(p));
  p.n_q = a->n_q;
  p.n_heads_idx = a->n_heads_idx;
  p.d_idx = L->d_idx;
  p.idx_dtype = L->idx_dtype;
  p.m = L->m;
  p.n_win = L->n_win;
  p.page_size = L->page_size;
  p.max_pages_per_seq = L->max_pages_per_seq;
  p.n_seqs_layer = L->n_seqs;
  p.n_pages = L->n_pages;
  p.page_table = L->page_table;
  p.idx_pool = L->idx_pool;
  p.idx_scale = L->idx_scale;
  p.q_seq = a->q_seq;
  p.q_pos = a->q_pos;
  p.max_pos = a->max_pos;
  p.q_idx = a->q_idx;
  p.q_idx_scale = a->q_idx_scale;
  p.w = a->w;
  p.k = a->k;
  p.out_idx = a->out_idx;
  p.out_cnt = a->out_cnt;
  p.out_scores = a->out_scores;
  p.status = a->d_status;
  p.score_bf16 = index_score_bf16(a);
  return from_cuda(cskv::launch_index(p, ws, sm_count(), static_cast<cudaStream_t>(stream)));
}

cskv_status cskv_attend_ws_bytes(const cskv_attend_args* a, size_t* bytes) {
  if (!a || !bytes) return CSKV_ERR_INVALID_ARG;
  const int kind = a->layer ? a->layer->kind : -1;
  cskv_status s = check_attend(a, kind);
  if (s) return s;
  AttendParams p;
  fill_attend(p, a, kind);
  *bytes = cskv::attend_ws_bytes(p, sm_count());
  return CSKV_OK;
}

cskv_status csa_attend(const cskv_attend_args* a, void* ws, size_t ws_bytes, void* stream) {
  return attend_impl(a, ws, ws_bytes, stream, CSKV_LAYER_CSA);
}

cskv_status hca_attend(const cskv_attend_args* a, void* ws, size_t ws_bytes, void* stream) {
  return attend_impl(a, ws, ws_bytes, stream, CSKV_LAYER_HCA);
}

cskv_status cskv_get_status(int32_t* d_status, void* stream, int32_t* status) {
  if (!d_status || !status) return CSKV_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int32_t h = 0;
  if (cudaMemcpyAsync(&h, d_status, sizeof(int32_t), cudaMemcpyDeviceToHost, st) != cudaSuccess)
    return CSKV_ERR_CUDA;
  if (cudaMemsetAsync(d_status, 0, sizeof(int32_t), st) != cudaSuccess) return CSKV_ERR_CUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return CSKV_ERR_CUDA;
  *status = h;
  return CSKV_OK;
}

cskv_status cskv_selftest_wait(int32_t arrive, uint32_t spin_limit, int32_t* d_status, void* stream) {
  if (!d_status || spin_limit == 0) return CSKV_ERR_INVALID_ARG;
  return from_cuda(cskv::launch_wait_selftest(arrive != 0, spin_limit, d_status, static_cast<cudaStream_t>(stream)));
}

const char* cskv_status_string(cskv_status s) {
  switch (s) {
    case CSKV_OK: return "ok";
    case CSKV_ERR_INVALID_ARG: return "invalid argument";
    case CSKV_ERR_UNSUPPORTED: return "unsupported dtype or shape";
    case CSKV_ERR_WORKSPACE: return "workspace missing or too small";
    case CSKV_ERR_CUDA: return "CUDA launch error";
    case CSKV_ERR_TIMEOUT: return "bounded device wait timed out";
    case CSKV_ERR_OUT_OF_RANGE: return "page id or index out of range on device";
    default: return "unknown status";
  }
}

int32_t cskv_version(void) { return 100; }

}  // extern "C"
