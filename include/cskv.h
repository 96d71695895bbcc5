/*
 * cskv.h -- C ABI of libcskv.so: CSA / HCA hybrid compressed attention on
 * NVIDIA B200 (sm_100a).
 *
 * The method (sources by page title and section):
 *   - DeepSeek-V4 report digest (gitcode.csdn.net/69eb1ea0...), section 3:
 *     CSA compresses every m tokens of KV into one entry, a Lightning Indexer
 *     scores the entries and only the top-k (512 Flash, 1024 Pro) take part
 *     in core attention; HCA compresses every m' = 128 tokens and attends all
 *     entries densely; both add a sliding-window branch over the last
 *     n_win = 128 uncompressed tokens. Section 7: FP4 for the indexer QK
 *     path, and a KV cache of two kinds -- the compressed ("classical") cache
 *     and a state cache holding the window and the tokens of the block not
 *     yet compressed (Figure 6).
 *   - DeepSeek-V4-book ch.1, section 4: m = 4, top-k = 1024 -> 4096
 *     effective tokens; m' = 128 -> n/m' = 8K entries at 1M; the shared MLA
 *     latent KV.
 *   - 10100.com DeepSeek-V4 article, section 2.1 (4:1 compression with
 *     position weighting, low-rank indexer, top-k, 128-token dense window),
 *     section 2.2 (128:1 HCA), section 5 (FP8/FP4 KV, paged KV).
 *
 * Readings taken where the pages are silent:
 *   - compression: per channel c of block j,
 *       C[j,c] = sum_i softmax_i(Z[j*m+i, c] + B[i, c]) * X[j*m+i, c],
 *     Z one logit per token (gate_cols = 1) or per channel (gate_cols = d);
 *     B an optional fp32 position bias [m, d].
 *   - visibility: entry j is visible to the query at position t iff
 *     j*m < t + 1 - n_win; the window is positions max(0, t-n_win+1) .. t.
 *   - indexer score: s(t,j) = sum_h w[t,h] * ReLU(qI[t,h,:] . KI[j,:]) with
 *     one indexer key head shared by the H_I query heads.
 *   - top-k order: (score desc, index asc); output ascending by index,
 *     padded with -1; k_eff = min(k, visible entries).
 *   - attention: one softmax over the window keys and the chosen (CSA) or
 *     all visible (HCA) entries; every query head reads the same latent
 *     vector K_u (d_qk wide) and V_u = its first d_v channels.
 *
 * Conventions shared by every call
 *   - Every function returns a cskv_status; 0 is success. Host-side checks
 *     run before any launch and return CSKV_ERR_INVALID_ARG or
 *     CSKV_ERR_UNSUPPORTED without touching the GPU.
 *   - Errors found on the device (a page id outside the pool, a position
 *     beyond the caller's stated bound) do not trap: the kernel skips the
 *     access and writes the first such code into the caller's status word
 *     (`d_status`, a device int32, may be NULL). cskv_get_status() reads and
 *     clears it.
 *   - Ownership: the caller allocates and frees all device memory (inputs,
 *     outputs, cache pools, page tables, status words, workspaces). The
 *     library never allocates, frees or synchronises, keeps no state between
 *     calls, and only enqueues work on the given stream (a cudaStream_t
 *     passed as void*; NULL is the legacy default stream). Calls are
 *     reentrant; two calls that write the same buffers must be ordered by
 *     the caller.
 *   - All tensors are dense row-major with the shapes given; pointers are
 *     device pointers unless marked "host". bf16 buffers must be 16-byte
 *     aligned and their row lengths multiples of 8 elements.
 *   - Every args struct starts with struct_size = sizeof(the struct), so
 *     the struct can grow without breaking callers.
 */
#ifndef CSKV_H_
#define CSKV_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef int32_t cskv_status;

#define CSKV_OK 0
#define CSKV_ERR_INVALID_ARG (-1)  /* a host-side argument check failed */
#define CSKV_ERR_UNSUPPORTED (-2)  /* dtype / dimension not built into this library */
#define CSKV_ERR_WORKSPACE (-3)    /* workspace missing or smaller than the query said */
#define CSKV_ERR_CUDA (-4)         /* a CUDA launch or attribute call failed */
#define CSKV_ERR_TIMEOUT (-5)      /* a bounded device wait gave up */
#define CSKV_ERR_OUT_OF_RANGE (-6) /* the device met a page id or index outside its buffers */

/* storage dtypes */
#define CSKV_BF16 0
#define CSKV_F32 1
#define CSKV_FP8_E4M3 2 /* OCP E4M3 codes + one fp32 scale per row (entry) */
#define CSKV_FP4_E2M1 3 /* OCP E2M1 codes, two per byte (element 2i in the low nibble),
                           + one E4M3 scale byte per 16 elements */

/* layer kinds */
#define CSKV_LAYER_CSA 0
#define CSKV_LAYER_HCA 1

/*
 * cskv_layer -- one attention layer's KV state (host struct, device buffers).
 *
 * Compressed ("classical") cache: paged. Logical entry j of sequence s lives
 * in page page_table[s * max_pages_per_seq + j / page_size], slot
 * j % page_size. Pool rows are indexed page * page_size + slot.
 *   kv_pool   [n_pages * page_size, d_qk]     bf16, or FP8 codes (uint8)
 *   kv_scale  [n_pages * page_size]           fp32 (FP8 only, else NULL)
 *   idx_pool  [n_pages * page_size, d_idx]    bf16, or [.., d_idx/2] FP4 bytes (CSA)
 *   idx_scale [n_pages * page_size, d_idx/16] E4M3 scale bytes (FP4 only)
 * State cache: a ring of the last n_win raw tokens per sequence; position p
 * sits in slot p % n_win.
 *   ring_x  [n_seqs, n_win, d_qk]       bf16 raw latent KV
 *   ring_z  [n_seqs, n_win, gate_cols]  bf16 gate logits of the KV stream
 *   ring_xi [n_seqs, n_win, d_idx]      bf16 raw indexer keys (CSA)
 *   ring_zi [n_seqs, n_win, gate_cols_idx] bf16 gate logits of the indexer-key stream (CSA)
 * Block overlap (10100.com article, section 2.1: block compression with
 * position weighting and block overlap; the width is a reading): with
 * overlap = ov > 0, entry j folds the tokens at positions max(0, j*m - ov) ..
 * j*m + m - 1 under one softmax (the last ov tokens of the block before it
 * too), and pos_bias / pos_bias_idx have m + ov rows, row r for the token at
 * position j*m - ov + r. The entry is complete when its own block is, so
 * visibility does not change. Requires ov <= n_win - m; a bulk compression
 * that starts at tok0 > 0 reads the ov tokens before tok0 from the ring.
 * overlap = 0 (or a struct_size that ends before the field) is the plain fold.
 * Constraints: m a power of two with m <= n_win; page_size a multiple of 16;
 * d_qk, d_v, d_idx multiples of 16 (d_idx of 32 for FP4); d_v <= d_qk.
 */
typedef struct {
  uint32_t struct_size;
  int32_t kind;      /* CSKV_LAYER_CSA or CSKV_LAYER_HCA */
  int32_t m;         /* tokens per compressed entry: 4 (CSA), 128 (HCA) */
  int32_t n_win;     /* sliding-window length: 128 */
  int32_t d_qk;      /* stored latent width = key width */
  int32_t d_v;       /* value width (the first d_v channels of the latent) */
  int32_t d_idx;     /* indexer key width (CSA); 0 for HCA */
  int32_t page_size; /* compressed entries per page */
  int32_t kv_dtype;  /* CSKV_BF16 or CSKV_FP8_E4M3 */
  int32_t idx_dtype; /* CSKV_BF16 or CSKV_FP4_E2M1 (CSA) */
  int32_t gate_cols;     /* 1 or d_qk */
  int32_t gate_cols_idx; /* 1 or d_idx (CSA) */
  int32_t n_seqs;             /* rows of the page table and of the rings */
  int32_t max_pages_per_seq;  /* row stride of the page table */
  int64_t n_pages;            /* pool capacity in pages (bounds check) */
  const int32_t* page_table;  /* [n_seqs, max_pages_per_seq] */
  void* kv_pool;
  float* kv_scale;
  void* idx_pool;
  uint8_t* idx_scale;
  void* ring_x;
  void* ring_z;
  void* ring_xi;
  void* ring_zi;
  const float* pos_bias;     /* [m + overlap, d_qk] fp32 or NULL (position weighting) */
  const float* pos_bias_idx; /* [m + overlap, d_idx] fp32 or NULL */
  int32_t overlap;           /* block overlap ov (0 = none) */
} cskv_layer;

/*
 * cskv_layer_bytes -- bytes the caller must allocate for each buffer of a
 * layer with the given fields (struct_size, kind, m, n_win, dims, dtypes,
 * gate columns, n_seqs, n_pages, page_size set; pointers ignored). Any output
 * pointer may be NULL. Sizes of buffers a layer does not use are 0.
 */
cskv_status cskv_layer_bytes(const cskv_layer* layer, size_t* kv_pool, size_t* kv_scale,
                             size_t* idx_pool, size_t* idx_scale, size_t* ring_x, size_t* ring_z,
                             size_t* ring_xi, size_t* ring_zi);

/*
 * Bulk compression of a raw token segment straight into a layer's paged
 * cache (cache build, prefill).
 *   seq_ids [n_seq]                       sequence of each input row block
 *   x  [n_seq, n_tok, d_qk] bf16,  z  [n_seq, n_tok, gate_cols] bf16
 *   xi [n_seq, n_tok, d_idx] bf16, zi [n_seq, n_tok, gate_cols_idx] bf16 (CSA)
 *   tok0: position of the first token of every row block (multiple of m);
 *   n_tok: a multiple of m. Entries tok0/m .. (tok0+n_tok)/m - 1 are written.
 * The state-cache rings are not touched (cskv_cache_append does that).
 */
typedef struct {
  uint32_t struct_size;
  const cskv_layer* layer; /* host pointer */
  int32_t n_seq;
  const int32_t* seq_ids;
  int64_t tok0;
  int64_t n_tok;
  const void* x;
  const void* z;
  const void* xi;
  const void* zi;
  int32_t* d_status;
} cskv_compress_args;

/* csa_compress_kv: layer kind CSA; compresses the latent-KV stream (x, z)
 * and the indexer-key stream (xi, zi) with m = layer->m (4). Sources:
 * DeepSeek-V4-book ch.1 section 4; DeepSeek-V4 report digest section 3. */
cskv_status csa_compress_kv(const cskv_compress_args* args, void* stream);
/* hca_compress_kv: layer kind HCA; compresses (x, z) with m = layer->m
 * (128); xi, zi are ignored. Same sources (m' = 128). */
cskv_status hca_compress_kv(const cskv_compress_args* args, void* stream);

/*
 * cskv_cache_append -- the state-cache update of a decode step (report
 * digest section 7, Figure 6: the state cache keeps the window and the
 * not-yet-compressed tokens). For each sequence b, the n_new tokens at
 * positions pos[b] .. pos[b]+n_new-1 are written into the rings; every block
 * that these tokens complete (position p with (p+1) % m == 0) is compressed
 * from the ring and the new rows and written into the paged cache.
 *   seq_ids [n_seq], pos [n_seq] int64
 *   x [n_seq, n_new, d_qk], z [n_seq, n_new, gate_cols],
 *   xi [n_seq, n_new, d_idx], zi [n_seq, n_new, gate_cols_idx] (CSA)
 * Requires n_new + m - 1 + overlap <= n_win (every completed block, and the
 * tokens it overlaps, are still in the ring). ring_only = 1 writes the rings
 * and emits nothing (used after a bulk compression of the same tokens).
 * emit_only = 1 (a field added after d_status; callers whose struct_size ends
 * before it get 0) writes no ring row and only compresses the blocks these
 * tokens complete: for a caller that has already written the same tokens with
 * ring_only = 1, stream-ordered before this call, and that moves the
 * compression off its critical path (an entry completed at position t covers
 * positions inside t's window, so no query up to t reads it). Until this call
 * has completed, the ring rows of the blocks it compresses must not be
 * overwritten (the layer's next append) and the entries it writes not read.
 * ring_only and emit_only together are an invalid argument.
 */
typedef struct {
  uint32_t struct_size;
  const cskv_layer* layer;
  int32_t n_seq;
  int32_t n_new;
  const int32_t* seq_ids;
  const int64_t* pos;
  const void* x;
  const void* z;
  const void* xi;
  const void* zi;
  int32_t ring_only;
  int32_t* d_status;
  int32_t emit_only;
} cskv_append_args;

cskv_status cskv_cache_append(const cskv_append_args* args, void* stream);

/*
 * csa_index_score_topk -- Lightning-indexer scores of every visible entry
 * and the top-k selection (report digest section 3: k = 512 / 1024; section
 * 7: FP4 indexer QK path; DeepSeek-V4-book ch.1 section 4).
 *   q_seq [n_q] int32, q_pos [n_q] int64 (absolute position t of each query)
 *   max_pos (host): an upper bound of every q_pos; sizes the workspace
 *   q_idx  [n_q, n_heads_idx, d_idx] bf16, or FP4 bytes [n_q, n_heads_idx, d_idx/2]
 *   q_idx_scale [n_q, n_heads_idx, d_idx/16] E4M3 bytes (FP4 only)
 *   w      [n_q, n_heads_idx] fp32 (any sign)
 *   out_idx    [n_q, k] int32: ascending entry ids, -1 padded
 *   out_cnt    [n_q] int32: k_eff = min(k, visible entries)
 *   out_scores [n_q, k] fp32 or NULL: the score of each chosen entry (0 for padding)
 *   score_bf16: 0 = select on the fp32 scores; 1 = round every score to bf16
 *     (round to nearest even) before the selection, which then ranks the
 *     rounded scores with the same order (entries whose scores round to the
 *     same value are taken in index order); out_scores then holds the rounded
 *     scores. Report digest section 7: the indexer's scores kept in BF16
 *     rather than FP32 halve the selector's cost at 99.7% recall of the FP32
 *     selection. A caller whose struct_size ends before this field gets 0.
 * The query dtype is layer->idx_dtype. Workspace: csa_index_ws_bytes().
 */
typedef struct {
  uint32_t struct_size;
  const cskv_layer* layer;
  int32_t n_q;
  int32_t n_heads_idx;
  const int32_t* q_seq;
  const int64_t* q_pos;
  int64_t max_pos;
  const void* q_idx;
  const uint8_t* q_idx_scale;
  const float* w;
  int32_t k;
  int32_t* out_idx;
  int32_t* out_cnt;
  float* out_scores;
  int32_t* d_status;
  int32_t score_bf16;
} cskv_index_args;

cskv_status csa_index_ws_bytes(const cskv_index_args* args, size_t* bytes);
cskv_status csa_index_score_topk(const cskv_index_args* args, void* workspace, size_t ws_bytes,
                                 void* stream);

/*
 * csa_index_score_topk_static -- the same scores and selection as
 * csa_index_score_topk, with no workspace argument and no allocation of any
 * kind. The paper has no counterpart to this call; it exists for callers
 * that cannot obtain device memory where they call the indexer: a plugin
 * running inside a host engine that owns all device memory and offers its
 * plugins no workspace, or a latency-critical loop that must not call
 * cudaMalloc (which can synchronise the device and take unbounded time).
 *   - Scratch: a file-scope device array of CSKV_STATIC_INDEX_SCRATCH_FLOATS
 *     fp32 values (16 MiB) inside libcskv.so. Every GPU that loads the
 *     library holds it until the process exits.
 *   - Limit: a call needs csa_index_ws_bytes() bytes of it, i.e. 4 bytes x
 *     (n_q x (the visible entries of max_pos rounded up to 64, plus 2048
 *     histogram counters) + 64); a request above 16 MiB, that is with
 *     n_q x (...) > CSKV_STATIC_INDEX_SCRATCH_FLOATS - 64, returns
 *     CSKV_ERR_WORKSPACE and launches nothing.
 *   - Set-up: the first call on each device looks up the array's device
 *     address (cudaGetSymbolAddress) with that device current and keeps it
 *     for the life of the process; make that first call before any stream
 *     capture. The address belongs to the device's primary context: call
 *     this entry point only with the primary context current (the runtime
 *     API's default), and not after cudaDeviceReset() in the same process.
 *   - Sharing: every call uses the same array and leaves its contents
 *     behind. Nothing in it needs clearing (each call writes every score it
 *     reads and zeroes the counters it uses), but two calls that can run on the GPU at the same time -- on
 *     unordered streams, or from several host threads -- race on it and
 *     corrupt each other's results; order them on one stream or with events.
 *   - Arguments, outputs and errors are otherwise those of
 *     csa_index_score_topk.
 */
#define CSKV_STATIC_INDEX_SCRATCH_FLOATS (4u << 20)
cskv_status csa_index_score_topk_static(const cskv_index_args* args, void* stream);

/*
 * csa_attend / hca_attend -- core attention of one layer (report digest
 * section 3: one softmax over the window of the last n_win raw tokens and
 * the top-k entries (CSA) or all visible entries (HCA); DeepSeek-V4-book
 * ch.1 section 4: the shared latent KV, MQA).
 *   q [n_q, n_heads, d_qk] bf16; out [n_q, n_heads, d_v] bf16;
 *   lse [n_q, n_heads] fp32 or NULL: natural-log sum of exp(sm_scale * q.k)
 *   sel_idx [n_q, k] / sel_cnt [n_q]: csa_index_score_topk's outputs (CSA)
 *   window rows come from the layer's ring; when x_chunk is not NULL, rows of
 *   positions chunk_pos0 .. chunk_pos0 + chunk_len - 1 come from x_chunk
 *   [chunk_len, d_qk] bf16 instead (prefill of one sequence: the ring then
 *   still holds the tokens before the chunk).
 *   rope_dims, rope_base: inverse RoPE on the output ("constraint chain"
 *     essay, innovation 1: with many tokens sharing one compressed entry,
 *     position is restored by an inverse-RoPE correction of the attention
 *     output). When rope_dims > 0 (even, <= d_v), output channels
 *     c0 + 2i, c0 + 2i + 1 (c0 = d_v - rope_dims) are rotated by -t theta_i,
 *     theta_i = rope_base^(-2i / rope_dims), t = the query's position:
 *     (a, b) <- (a cos + b sin, -a sin + b cos). It makes values that carry
 *     RoPE at their key positions relative to the query; it is meaningful
 *     when V includes the RoPE channels (d_v = d_qk). lse is unchanged.
 *     A caller whose struct_size ends before these fields gets none.
 *   chunk_desc [n_seqs, 3] int64 or NULL: prefill of several sequences in one
 *     call (varlen). Sequence s's chunk rows are rows chunk_desc[s][0] ..
 *     chunk_desc[s][0] + chunk_desc[s][2] - 1 of x_chunk and hold its
 *     positions chunk_desc[s][1] .. + chunk_desc[s][2] - 1 (length 0: none);
 *     chunk_len is then the number of rows of x_chunk and chunk_pos0 is not
 *     used. Window rows outside a sequence's chunk come from its ring. A
 *     descriptor outside x_chunk is reported (CSKV_ERR_OUT_OF_RANGE).
 * Workspace: cskv_attend_ws_bytes().
 */
typedef struct {
  uint32_t struct_size;
  const cskv_layer* layer;
  int32_t n_q;
  int32_t n_heads;
  const int32_t* q_seq;
  const int64_t* q_pos;
  int64_t max_pos;
  const void* q;
  const int32_t* sel_idx;
  const int32_t* sel_cnt;
  int32_t k;
  float sm_scale;
  void* out;
  float* lse;
  const void* x_chunk;
  int64_t chunk_pos0;
  int64_t chunk_len;
  int32_t* d_status;
  int32_t rope_dims;
  float rope_base;
  const int64_t* chunk_desc;
} cskv_attend_args;

cskv_status cskv_attend_ws_bytes(const cskv_attend_args* args, size_t* bytes);
cskv_status csa_attend(const cskv_attend_args* args, void* workspace, size_t ws_bytes,
                       void* stream);
cskv_status hca_attend(const cskv_attend_args* args, void* workspace, size_t ws_bytes,
                       void* stream);

/* cskv_get_status -- copies the device status word to *status (host) and
 * clears it; synchronises the stream. */
cskv_status cskv_get_status(int32_t* d_status, void* stream, int32_t* status);

/*
 * cskv_selftest_wait -- checks the bounded device wait behind every
 * mbarrier hand-off of the library's kernels (producer -> consumer stages;
 * no wait may spin forever, so a lost arrival ends the kernel with
 * CSKV_ERR_TIMEOUT in the status word instead of hanging the GPU).
 * Launches one warp that waits on an mbarrier for at most spin_limit polls.
 *   arrive = 1: the barrier's one expected arrival is made first; the wait
 *               succeeds and the status word is left alone.
 *   arrive = 0: nothing arrives and no asynchronous copy is outstanding; the
 *               wait gives up after spin_limit polls and writes
 *               CSKV_ERR_TIMEOUT into *d_status (if it still holds 0).
 * The kernels themselves use a fixed limit of 2^24 polls. Read the result
 * with cskv_get_status(). Errors: CSKV_ERR_INVALID_ARG for a NULL status
 * word or spin_limit = 0; CSKV_ERR_CUDA if the launch fails.
 */
cskv_status cskv_selftest_wait(int32_t arrive, uint32_t spin_limit, int32_t* d_status, void* stream);

/* human-readable name of a status code (static string) */
const char* cskv_status_string(cskv_status s);

/* library version, major * 10000 + minor * 100 + patch */
int32_t cskv_version(void);

#ifdef __cplusplus
}
#endif

#endif /* CSKV_H_ */
