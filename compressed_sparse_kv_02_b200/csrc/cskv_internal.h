// cskv_internal.h -- parameter blocks and launchers shared by the C-ABI layer
// (cskv_abi.cu) and the kernel files. Not part of the public ABI.
#pragma once

#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "cskv.h"

namespace cskv {

// Launch `kern` with programmatic dependent launch allowed: it may be scheduled
// before the kernel ahead of it on the stream has finished, and must call
// grid_dependency_wait() before it reads anything that kernel writes.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, args...);
}

// cuTensorMapEncodeTiled, looked up once through the runtime (null if unavailable)
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder();

// One stream of raw tokens folded into compressed entries (the latent-KV
// stream, or the indexer-key stream of a CSA layer).
struct FoldStream {
  const uint16_t* x;      // new raw rows (bf16 bits)
  const uint16_t* z;      // new gate-logit rows
  const uint16_t* ring_x; // ring rows of the state cache (append path)
  const uint16_t* ring_z;
  uint16_t* ring_x_w;     // ring written by the append path
  uint16_t* ring_z_w;
  const float* bias;      // [m, d] or null
  int d;                  // channels
  int gc;                 // gate columns: 1 or d
  int out_dtype;          // CSKV_BF16 / CSKV_FP8_E4M3 / CSKV_FP4_E2M1
  void* pool;             // entry rows
  float* scale_f32;       // FP8 per-entry scale
  uint8_t* scale_e4m3;    // FP4 per-16 scale bytes
};

struct FoldParams {
  FoldStream s[2];
  int n_streams;
  int m, n_win, page_size, max_pages_per_seq;
  int ov;  // block overlap: an entry also folds the last ov tokens of the block before it
  int64_t n_pages;
  const int32_t* page_table;
  int n_seq;
  const int32_t* seq_ids;
  int n_seqs_layer;
  // bulk: rows [n_seq, n_tok, ...] starting at position tok0
  int64_t tok0, n_tok;
  // append: rows [n_seq, n_new, ...] starting at pos[b]
  const int64_t* pos;
  int n_new;
  int ring_only;  // the rings only
  int emit_only;  // the completed blocks only (the rings already hold the tokens)
  int32_t* status;
};

cudaError_t launch_fold_bulk(const FoldParams& p, cudaStream_t st);
cudaError_t launch_append(const FoldParams& p, cudaStream_t st);

// Lightning indexer scan (scores of every visible entry) + top-k.
struct IndexParams {
  int n_q, n_heads_idx, d_idx, idx_dtype;
  int m, n_win, page_size, max_pages_per_seq, n_seqs_layer;
  int64_t n_pages;
  const int32_t* page_table;
  const void* idx_pool;
  const uint8_t* idx_scale;
  const int32_t* q_seq;
  const int64_t* q_pos;
  int64_t max_pos;
  const void* q_idx;
  const uint8_t* q_idx_scale;
  const float* w;
  int k;
  int32_t* out_idx;
  int32_t* out_cnt;
  float* out_scores;
  int32_t* status;
  int score_bf16;       // scores rounded to bf16 before they are written (and selected)
  // workspace
  float* scores;        // [n_q, vis_stride]
  int64_t vis_stride;
  uint32_t* hist;       // [n_q, 2048] counts of the scores' top 11 key bits (from the scan), or null
  int cluster;          // CTAs per query in the selection kernel
  int slice;            // entries per CTA of the selection kernel
};

size_t index_ws_bytes(int n_q, int64_t max_pos, int m, int n_win);
// tensor-core (tcgen05) scores for calls with many queries: groups of 128 / H_I queries of one
// sequence share every 128-key tile (bf16 keys, H_I = 4 or 8, d_I = 64 or 128)
bool scan_tc_supported(const IndexParams& p);
cudaError_t launch_scan_tc(IndexParams& p, int n_sm, cudaStream_t st);
cudaError_t launch_index(IndexParams& p, void* ws, int n_sm, cudaStream_t st);

// Split-KV attention over window + compressed keys, then the LSE merge.
struct AttendParams {
  int is_csa;
  int n_q, n_heads, d_qk, d_v, kv_dtype;
  int m, n_win, page_size, max_pages_per_seq, n_seqs_layer;
  int64_t n_pages;
  const int32_t* page_table;
  const void* kv_pool;
  const float* kv_scale;
  const uint16_t* ring_x;
  const int32_t* q_seq;
  const int64_t* q_pos;
  int64_t max_pos;
  const uint16_t* q;
  const int32_t* sel_idx;
  const int32_t* sel_cnt;
  int k;
  float sm_scale;
  uint16_t* out;
  float* lse;
  const uint16_t* x_chunk;
  int64_t chunk_pos0, chunk_len;
  int32_t* status;
  int rope_dims;    // inverse RoPE on the last rope_dims output channels (0: none)
  float rope_base;
  const int64_t* chunk_desc;  // [n_seqs_layer, 3] (first row, first position, length) of each sequence's chunk, or null
  // workspace / plan
  float* part_o;   // [n_q * max_splits * n_heads, d_v], or with part_t: [n_q * max_splits, d_v / 4, n_heads, 4]
  int part_t;      // part_o in the head-minor layout (written by attend_tc_kernel)
  float* part_lse; // [n_q * max_splits * n_heads]
  int max_splits;
  int keys_per_split;
};

size_t attend_ws_bytes(const AttendParams& p, int n_sm);

// Row of x_chunk that holds position pos of sequence seq, or -1 (the row is then in the ring).
// One sequence (no chunk_desc): x_chunk holds positions chunk_pos0 .. chunk_pos0 + chunk_len - 1.
// Several (chunk_desc): sequence s's chunk sits at rows desc[s][0] .. + desc[s][2] - 1 of x_chunk
// and holds positions desc[s][1] .. + desc[s][2] - 1; x_chunk has chunk_len rows in all. A
// descriptor that points outside x_chunk is reported and its rows read from the ring.
__device__ __forceinline__ int64_t chunk_row(const AttendParams& p, int seq, int64_t pos) {
  if (!p.x_chunk) return -1;
  int64_t r0 = 0, p0 = p.chunk_pos0, len = p.chunk_len;
  if (p.chunk_desc) {
    r0 = p.chunk_desc[3 * (int64_t)seq];
    p0 = p.chunk_desc[3 * (int64_t)seq + 1];
    len = p.chunk_desc[3 * (int64_t)seq + 2];
    if (r0 < 0 || len < 0 || r0 + len > p.chunk_len) {
      if (p.status) atomicCAS(p.status, 0, CSKV_ERR_OUT_OF_RANGE);
      return -1;
    }
  }
  return (pos >= p0 && pos < p0 + len) ? r0 + pos - p0 : -1;
}
cudaError_t launch_attend(AttendParams& p, void* ws, int n_sm, cudaStream_t st);
bool attend_supported(int d_qk, int d_v, int n_heads, int kv_dtype);
cudaError_t launch_attend_merge(AttendParams& p, cudaStream_t st);
// tensor-core (tcgen05) attention for the 576 / 512 latent with heads in groups of 128
bool attend_tc_supported(int d_qk, int d_v, int n_heads, int kv_dtype, int n_q);
void attend_tc_plan(AttendParams& p, int n_sm);
cudaError_t launch_attend_tc(AttendParams& p, int n_sm, cudaStream_t st);
// tensor-core attention for calls with many queries on the 128-wide latent with 64 heads:
// query pairs, whole key lists, bf16 output written directly
bool attend_pair_supported(const AttendParams& p, int n_sm);
cudaError_t launch_attend_pair(AttendParams& p, int n_sm, cudaStream_t st);

// the bounded-wait check (selftest.cu)
cudaError_t launch_wait_selftest(int arrive, uint32_t spin_limit, int32_t* status, cudaStream_t st);

}  // namespace cskv
