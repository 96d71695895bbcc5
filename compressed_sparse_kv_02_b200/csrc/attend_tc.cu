// attend_tc.cu -- CSA / HCA core attention on the 5th-generation tensor cores
// (tcgen05) for the wide shared latent: d_qk = 576 (512 latent + 64 RoPE
// channels), d_v = 512, query heads in groups of 128 (DeepSeek-V4 report
// digest, section 3: one softmax over the window and the selected / all
// compressed entries; DeepSeek-V4-book ch.1, section 4: the MLA latent shared
// by every head).
//
// With 128 heads on one 576-wide latent every key carries 2 x 128 x 1088
// flops against 1152 bytes: the product sits at the B200's ridge point, so the
// kernel must stream keys at HBM speed and keep the tensor core busy at once.
// Work item = (query, 128-head group, key split), run by a cluster of two CTAs
// that split the key channels:
//   rank 0 holds Q channels 0..319 and loads key channels 0..319;
//   rank 1 holds Q channels 320..575 and loads key channels 256..575;
// each computes a partial S = Q K^T over its channels (heads as M = 128, 32
// keys as N) in tensor memory, sends it to the other CTA through distributed
// shared memory and adds the one it receives, so both hold the full S and run
// the same online softmax (fp32; identical results, since a + b == b + a).
// Each then accumulates O for its half of d_v: O[:, 256 r .. 256 r + 255] +=
// P V, with P (bf16) as the tensor-memory A operand and V read MN-major from
// the first four channel blocks of its key tile (V = the first d_v channels of
// every key). No tensor work is duplicated. Each CTA keeps its last three Q
// blocks in tensor memory (an MMA's A operand may come from there) and the
// rest in shared memory, which leaves room for five key-tile stages and the
// exchange buffers, so the loads run well ahead of the math.
//   - key tiles arrive by TMA when their rows are contiguous (window rows of
//     the ring, HCA entries of one page), by cp.async through a row table
//     otherwise (the CSA selection);
//   - each thread of the softmax warpgroup owns one head row; it sends tile
//     t + 1's partial (asynchronous stores counted on the receiver's
//     mbarrier) before it waits for tile t's, hiding the exchange;
//   - O is rescaled only when a row's running max rises by more than 2^8 (the
//     probabilities stay below 256 in bf16), so most tiles skip it.
// Window keys are taken in ring-slot order (the softmax does not depend on the
// order of its keys), which makes a window tile 32 consecutive ring rows. Each
// item writes its normalised partial output and log-sum-exp;
// attend_merge_kernel combines the splits.
#include <cooperative_groups.h>

#include "cskv_device.cuh"
#include "cskv_internal.h"

namespace cg = cooperative_groups;

namespace cskv {
namespace {

constexpr int kDqk = 576, kDv = 512, kM = 128, kNk = 32;
constexpr int kNb = 5;                         // 64-channel blocks of a key row loaded by each CTA
constexpr int kStageBytes = kNb * kNk * 128;   // 20480 per key-tile stage
// Q blocks of a CTA: the first kQSmem (rank 0: 2, rank 1: 1) in shared memory,
// the last three in tensor memory (the A operand of an MMA may come from either)
constexpr int kQTmem = 3;
constexpr int kQBytes = 2 * kM * 128;          // 32768
constexpr int kNS = 5;                         // key-tile stages
constexpr int kRecvBytes = kM * kNk * 4;       // one partial S tile from the other CTA
constexpr int kThreads = 256;                  // warps 0-3 softmax, warp 4 MMA, warps 5-7 loads
constexpr int kMmaThread = 128;
constexpr int kLoadThread0 = 160;
constexpr int kLoaders = kThreads - kLoadThread0;  // 96
constexpr int kRowCap = 1024;                  // keys per work item (row table in shared memory)
constexpr uint32_t kTmemCols = 512;
// O 256 | S 3 buffers x 32 | P 3 buffers x 16 (bf16 pairs) | Q 3 blocks x 32 (bf16 pairs)
constexpr int kNSP = 3;  // S and P buffers
constexpr uint32_t kColO = 0, kColS = 256, kColP = kColS + kNSP * 32, kColQ = kColP + kNSP * 16;
static_assert(kColQ + kQTmem * 32 <= kTmemCols, "tensor memory budget");
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kRescaleThreshold = 8.0f;      // log2 units
constexpr int kPrefetchTiles = 6;              // L2 prefetch distance of gathered key rows

struct Smem {
  static constexpr int Q = 0;
  static constexpr int K = kQBytes;                     // kNS stages (also the epilogue staging)
  static constexpr int RECV = K + kNS * kStageBytes;    // two slots of the other CTA's partial S
  static constexpr int SEND = RECV + 2 * kRecvBytes;    // two slots of this CTA's partial S on its way out
  static constexpr int BAR = SEND + 2 * kRecvBytes;     // mbarriers
  static constexpr int MASK = BAR + 256;                // valid-key bits, one word per tile
  static constexpr int ROWS = MASK + kRowCap / 8;       // source row of every key of the item
  static constexpr int SCALE = ROWS + kRowCap * 8;      // FP8 entries: the per-entry scale of every key
  static constexpr int TMEM = SCALE + kRowCap * 4;      // allocated tensor-memory address
  static constexpr int FLAGS = TMEM + 16;
  static constexpr int PREF = FLAGS + 16;
  static size_t bytes(int n_q) { return 1024 + PREF + sizeof(int) * (size_t)(n_q + 1); }
};

struct Keys {
  int64_t t, ws;
  int n_w;
  int64_t n;
};

__device__ __forceinline__ Keys keys_of(const AttendParams& p, int b) {
  Keys r;
  r.t = p.q_pos[b];
  r.ws = 0;
  r.n_w = 0;
  r.n = 0;
  if (r.t < 0 || r.t > p.max_pos) return r;
  r.ws = window_start(r.t, p.n_win);
  r.n_w = static_cast<int>(r.t - r.ws + 1);
  int64_t n_c;
  if (p.is_csa) {
    const int64_t c = p.sel_cnt[b];
    n_c = c < 0 ? 0 : (c > p.k ? p.k : c);
  } else {
    n_c = visible_entries(r.t, p.m, p.n_win);
  }
  r.n = r.n_w + n_c;
  return r;
}

// Source row of key u. Window keys come first: in ring-slot order (slot u)
// when every window row is in the ring, in position order when a prefill chunk
// supplies some of them; then the compressed entries (bf16 rows, or FP8 rows
// with their scale in `sc`). Null if invalid.
__device__ __forceinline__ const void* key_src(const AttendParams& p, int b, int seq, const Keys& k, int64_t u,
                                               float& sc) {
  sc = 1.f;
  if (u < k.n_w) {
    if (!p.x_chunk) return p.ring_x + ((int64_t)seq * p.n_win + u) * kDqk;
    const int64_t pos = k.ws + u;
    if (pos >= p.chunk_pos0 && pos < p.chunk_pos0 + p.chunk_len) return p.x_chunk + (pos - p.chunk_pos0) * kDqk;
    return p.ring_x + ((int64_t)seq * p.n_win + pos % p.n_win) * kDqk;
  }
  const int64_t jj = u - k.n_w;
  const int64_t j = p.is_csa ? static_cast<int64_t>(p.sel_idx[(int64_t)b * p.k + jj]) : jj;
  if (j < 0 || j >= visible_entries(k.t, p.m, p.n_win)) return nullptr;
  const int64_t pi = j / p.page_size;
  if (pi >= p.max_pages_per_seq) return nullptr;
  const int32_t page = p.page_table[(int64_t)seq * p.max_pages_per_seq + pi];
  if (page < 0 || page >= p.n_pages) return nullptr;
  const int64_t row = (int64_t)page * p.page_size + j % p.page_size;
  if (p.kv_dtype == CSKV_FP8_E4M3) {
    sc = p.kv_scale[row];
    return static_cast<const uint8_t*>(p.kv_pool) + row * kDqk;
  }
  return static_cast<const uint16_t*>(p.kv_pool) + row * kDqk;
}

// 8 E4M3 codes -> 8 bf16 (exact: every E4M3 value is a bf16 value)
__device__ __forceinline__ uint4 e4m3x8_to_bf16x8(uint2 c) {
  uint32_t o[4];
  const uint32_t w[2] = {c.x, c.y};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const __nv_fp8x2_storage_t v = static_cast<__nv_fp8x2_storage_t>((w[i >> 1] >> (16 * (i & 1))) & 0xffffu);
    const float2 f = __half22float2(__half2(__nv_cvt_fp8x2_to_halfraw2(v, __NV_E4M3)));
    o[i] = pack_bf16(f.x, f.y);
  }
  return make_uint4(o[0], o[1], o[2], o[3]);
}

// byte offset of 16-byte chunk `ch` of row `r` in a swizzled block set whose
// 64-channel (128-byte) blocks are `block_bytes` apart
__device__ __forceinline__ uint32_t swz(int r, int ch, int block_bytes) {
  return (ch >> 3) * block_bytes + r * 128 + (((ch & 7) ^ (r & 7)) << 4);
}

__device__ __forceinline__ void named_sync(int id, int n) {
  asm volatile("bar.sync %0, %1;\n" ::"r"(id), "r"(n) : "memory");
}

// ---------------------------------------------------------------- cluster helpers
__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;\n" : "=r"(r));
  return r;
}
// shared::cluster address of `local` in CTA `rank` of the cluster
__device__ __forceinline__ uint32_t peer_addr(const void* local, uint32_t rank) {
  uint32_t a;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;\n" : "=r"(a) : "r"(smem_u32(local)), "r"(rank));
  return a;
}
__device__ __forceinline__ void st_peer_u32(uint32_t addr, uint32_t v) {
  asm volatile("st.shared::cluster.u32 [%0], %1;\n" ::"r"(addr), "r"(v) : "memory");
}
// arrive on an mbarrier of another CTA (after this thread's reads of the slot
// it frees; the other CTA only writes into that slot again after seeing it)
__device__ __forceinline__ void mbar_arrive_peer(uint32_t addr) {
  asm volatile("mbarrier.arrive.shared::cluster.b64 _, [%0];\n" ::"r"(addr) : "memory");
}
// bulk copy (by the TMA engine) of `bytes` from this CTA's shared memory into
// another CTA's, counted as transaction bytes on that CTA's mbarrier (dst and
// mbar are shared::cluster addresses). The source may be rewritten once that
// mbarrier's phase has completed.
__device__ __forceinline__ void bulk_copy_to_peer(uint32_t dst, const void* src, uint32_t bytes, uint32_t mbar) {
  asm volatile("cp.async.bulk.shared::cluster.shared::cta.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];\n" ::"r"(
                   dst),
               "r"(smem_u32(src)), "r"(bytes), "r"(mbar)
               : "memory");
}
// Partial S of one key tile: NB channel blocks, the first NQS with Q in shared memory, the rest
// with Q in tensor memory; fully unrolled, every descriptor built from its 32-bit address (the
// constant upper half then folds away, which keeps the issue loop short).
template <int NB, int NQS>
__device__ __forceinline__ void issue_s(uint32_t d, uint32_t q_smem, uint32_t q_tmem, uint32_t k_smem,
                                        uint32_t idesc) {
#pragma unroll
  for (int k = 0; k < 4 * NB; ++k) {
    const int j = k >> 2, ks = k & 3;
    const uint64_t db = umma_desc_sw128(k_smem + j * (kNk * 128) + ks * 32, 16, 1024);
    if (j < NQS)
      umma_ss(d, umma_desc_sw128(q_smem + j * (kM * 128) + ks * 32, 16, 1024), db, idesc, k > 0 ? 1u : 0u);
    else
      umma_ts(d, q_tmem + (j - NQS) * 32 + ks * 8, db, idesc, k > 0 ? 1u : 0u);
  }
}

// Pipeline (per CTA; tiles numbered gt across the items of the cluster, the
// same in both CTAs; stage gt % kNS, S / P buffer gt % 3, exchange slot gt & 1):
//   loaders  : wait kempty (P V of tile gt - kNS done) -> TMA, or cp.async +
//              proxy fence, into the stage -> kfull
//   MMA      : wait kfull -> partial S(gt) -> commit sfull; then wait pfull of
//              tile gt - 2 -> O += P V -> commit kempty, obar
//   softmax  : wait sfull(gt + 1) -> send its partial to the other CTA (async
//              stores that count bytes on the receiver's rfull); wait rfull(gt)
//              -> S(gt) = own + received -> free the slot (remote rempty) ->
//              P(gt) (+ rare O rescale after P V of tile gt - 1) -> arrive pfull
// S(gt) needs the softmax only up to tile gt - 3 and the softmax needs S only
// one tile ahead, so neither waits on the other's latest step.
// FP8: the pool holds E4M3 entries with an fp32 scale each (a separate instantiation keeps
// the bf16 kernel's code, and so its instruction-cache footprint, small)
template <bool FP8>
__global__ void __launch_bounds__(kThreads, 1)
    attend_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_ring,
                     const __grid_constant__ CUtensorMap tm_kv, AttendParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = sm + Smem::Q;
  uint8_t* sK = sm + Smem::K;
  uint8_t* sRecv = sm + Smem::RECV;
  uint8_t* sSend = sm + Smem::SEND;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + Smem::BAR);
  uint64_t* kfull = bars;             // [kNS] loaders -> MMA
  uint64_t* kempty = bars + kNS;      // [kNS] MMA -> loaders (commit)
  uint64_t* sfull = bars + 2 * kNS;   // [3] MMA -> softmax (commit)
  uint64_t* pfull = sfull + kNSP;     // [3] softmax -> MMA (128 arrivals)
  uint64_t* obar = pfull + kNSP;      // [3] MMA -> softmax (commit after the P V of that P buffer)
  uint64_t* rfull = obar + kNSP;      // [2] other CTA's partial S landed (one arrival + 16 KB of bytes)
  uint64_t* rempty = rfull + 2;       // [2] other CTA has read what this one sent (4 remote arrivals)
  uint64_t* qbar = rempty + 2;        //     Q landed (TMA)
  uint64_t* dbar = qbar + 1;          //     MMA -> epilogue (commit after the item's last P V)
  uint32_t* sMask = reinterpret_cast<uint32_t*>(sm + Smem::MASK);
  const void** sRow = reinterpret_cast<const void**>(sm + Smem::ROWS);
  float* sScale = reinterpret_cast<float*>(sm + Smem::SCALE);
  constexpr bool fp8 = FP8;
  uint32_t* sTmem = reinterpret_cast<uint32_t*>(sm + Smem::TMEM);
  volatile int* sAbort = reinterpret_cast<int*>(sm + Smem::FLAGS);
  volatile int* sLdOk = reinterpret_cast<int*>(sm + Smem::FLAGS) + 1;  // [2] loader wait results, then [1] send flag
  int* sPref = reinterpret_cast<int*>(sm + Smem::PREF);
  __shared__ int s_wsum[32];

  cg::cluster_group cluster = cg::this_cluster();
  const uint32_t rank = cluster_rank(), peer = rank ^ 1u;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int groups = p.n_heads / kM;
  const int kps = p.keys_per_split;
  const int kb_load0 = rank ? 4 : 0;  // first 64-channel block of the key rows this CTA loads
  const int n_sblk = rank ? 4 : 5;    // blocks of its S partial (Q blocks 0.. of this CTA)
  const int n_qs = n_sblk - kQTmem;   // of which in shared memory
  const int qkb0 = rank ? 5 : 0;      // channel block of its Q block 0
  const int s_blk0 = rank ? 1 : 0;    // first S block inside a stage (blocks 0..3 are V)

  if (tid == 0) {
    for (int i = 0; i < kNS; ++i) {
      mbar_init(&kfull[i], 1);
      mbar_init(&kempty[i], 1);
    }
    for (int i = 0; i < kNSP; ++i) {
      mbar_init(&sfull[i], 1);
      mbar_init(&pfull[i], kM);
      mbar_init(&obar[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&rfull[i], 1);
      mbar_init(&rempty[i], 4);
    }
    mbar_init(qbar, 1 + kM);  // the TMA's arrival and one per softmax thread (tensor-memory blocks)
    mbar_init(dbar, 1);
    fence_barrier_init();
    *sAbort = 0;
  }
  if (tid == kLoadThread0) {
    prefetch_tensormap(&tm_q);
    prefetch_tensormap(&tm_ring);
    prefetch_tensormap(&tm_kv);
  }
  if (warp == 4) {
    tmem_alloc(sTmem, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  cluster.sync();  // barriers of both CTAs initialised before any remote arrival
  tc_fence_after();
  const uint32_t tmem = *sTmem;
  // the set-up above overlaps the tail of the kernel launched before this one; its
  // outputs (the selection, new cache rows) are read only from here on
  grid_dependency_wait();
  grid_dependents_launch();
  {  // items per query: splits x head groups
    int run = 0;
    for (int base = 0; base < p.n_q; base += kThreads) {
      const int b = base + tid;
      int v = 0;
      if (b < p.n_q) {
        const Keys k = keys_of(p, b);
        v = static_cast<int>((k.n + kps - 1) / kps) * groups;
      }
      int tot;
      const int ex = block_exclusive_scan<kThreads>(v, s_wsum, tot);
      if (b < p.n_q) sPref[b] = run + ex;
      run += tot;
    }
    if (tid == 0) sPref[p.n_q] = run;
  }
  __syncthreads();
  if (blockIdx.x == 0)
    for (int b = tid; b < p.n_q; b += kThreads)
      if (p.q_pos[b] < 0 || p.q_pos[b] > p.max_pos) report(p.status, CSKV_ERR_INVALID_ARG);
  const int total = sPref[p.n_q];
  const int n_clusters = gridDim.x / 2;
  uint32_t g = 0;       // tiles processed by this cluster before the current item
  uint32_t n_item = 0;  // items processed before the current one (qbar / dbar phase)

  for (int item = blockIdx.x / 2; item < total; item += n_clusters, ++n_item) {
    int lo = 0, hi = p.n_q - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (sPref[mid] <= item) lo = mid; else hi = mid - 1;
    }
    const int b = lo;
    const int r = item - sPref[b];
    const int grp = r % groups;
    const int split = r / groups;
    const Keys kk = keys_of(p, b);
    const int seq = p.q_seq[b];
    const bool seq_ok = seq >= 0 && seq < p.n_seqs_layer;
    const int64_t u0 = (int64_t)split * kps;
    const int nk = static_cast<int>(kk.n - u0 < kps ? kk.n - u0 : kps);
    const int ntiles = (nk + kNk - 1) / kNk;

    // source rows of this item's keys and one valid-bit word per tile, visible
    // to every role after the barrier; four independent lookups per thread
    for (int i0 = 0; i0 < ntiles * kNk; i0 += 4 * kThreads) {
      const void* src[4];
      float sc[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int i = i0 + q * kThreads + tid;
        sc[q] = 0.f;
        src[q] = (i < nk && seq_ok) ? key_src(p, b, seq, kk, u0 + i, sc[q]) : nullptr;
      }
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int i = i0 + q * kThreads + tid;
        if (i < nk) {
          if (!src[q] && rank == 0) report(p.status, CSKV_ERR_OUT_OF_RANGE);
          sRow[i] = src[q];
        }
        if (i < ntiles * kNk) sScale[i] = src[q] ? sc[q] : 0.f;  // finite for every slot of every tile
        const unsigned bits = __ballot_sync(kFull, src[q] != nullptr);
        if (lane == 0 && i < ntiles * kNk) sMask[i >> 5] = bits;
      }
    }
    __syncthreads();

    if (tid >= kLoadThread0) {
      // ------------------------------------------------------------ loaders
      const int lt = tid - kLoadThread0;
      if (lt == 0) {  // this CTA's shared-memory Q blocks of the head group: 128-row TMA boxes
        mbar_arrive_expect_tx(qbar, n_qs * kM * 128);
        const int qrow = b * p.n_heads + grp * kM;
        for (int j = 0; j < n_qs; ++j) tma_load_2d(sQ + j * (kM * 128), &tm_q, (qkb0 + j) * 64, qrow, qbar);
      }
      // TMA source of tile it: 0 = ring rows, 1 = pool rows, -1 = gathered (cp.async)
      auto tile_src = [&](int it, int& row0) -> int {
        const int64_t a = u0 + (int64_t)it * kNk;
        if (!seq_ok) return -1;
        if (!p.x_chunk && a + kNk <= kk.n_w) {
          row0 = static_cast<int>((int64_t)seq * p.n_win + a);
          return 0;
        }
        if (!p.is_csa && !fp8 && a >= kk.n_w) {
          const int64_t j0 = a - kk.n_w;
          const int64_t pi = j0 / p.page_size;
          // whole tile inside one page and inside the item (rows past the end are not zero)
          if (j0 % p.page_size + kNk > p.page_size || pi >= p.max_pages_per_seq || (it + 1) * kNk > nk) return -1;
          const int32_t page = p.page_table[(int64_t)seq * p.max_pages_per_seq + pi];
          if (page < 0 || page >= p.n_pages) return -1;
          row0 = static_cast<int>((int64_t)page * p.page_size + j0 % p.page_size);
          return 1;
        }
        return -1;
      };
      auto prefetch_tile = [&](int it) {
        if (lt < kNk && it < ntiles) {
          const int i = it * kNk + lt;
          if (i < nk && sRow[i]) {
            const bool row8 = fp8 && u0 + i >= kk.n_w;  // FP8 entry (window rows are bf16)
            prefetch_l2(static_cast<const uint8_t*>(sRow[i]) + kb_load0 * 64 * (row8 ? 1 : 2), kNb * (row8 ? 64 : 128));
          }
        }
      };
      const bool gathered_item = p.is_csa || p.x_chunk || fp8;
      if (gathered_item)
        for (int it = 0; it < kPrefetchTiles; ++it) prefetch_tile(it);
      // Gathered tiles are pipelined by one: tile it's loads are issued before tile it-1 is finished
      // (its FP8 rows widened, its cp.async group waited for) and signalled.
      constexpr int kItems = kNk * kNb * 8;
      constexpr int kPer = (kItems + kLoaders - 1) / kLoaders;
      uint2 pend_codes[kPer];
      int pend_it = -1;  // gathered tile still to be finished
      bool stopped = false;  // uniform over the loaders (decided after a named barrier)
      auto finish = [&](int pit, bool newer_group) {
        const uint32_t pgt = g + pit;
        uint8_t* pdst = sK + (pgt % kNS) * kStageBytes;
        if (fp8) {
#pragma unroll
          for (int q = 0; q < kPer; ++q) {
            const int id = lt + q * kLoaders;
            if (id < kItems) {
              const int kr = id / (kNb * 8), c = id % (kNb * 8);
              const int i = pit * kNk + kr;
              if (i < nk && sRow[i] && u0 + i >= kk.n_w)
                *reinterpret_cast<uint4*>(pdst + swz(kr, c, kNk * 128)) = e4m3x8_to_bf16x8(pend_codes[q]);
            }
          }
        }
        if (newer_group) cp_async_wait<1>(); else cp_async_wait<0>();
        fence_proxy_async_smem();
        named_sync(3, kLoaders);
        if (lt == 0) mbar_arrive(&kfull[pgt % kNS]);
      };
      for (int it = 0; it < ntiles; ++it) {
        const uint32_t gt = g + it;
        const int st = gt % kNS;
        if (gathered_item) prefetch_tile(it + kPrefetchTiles);
        // one thread waits and the loaders agree on its result, so no loader can
        // leave the loop while another waits at a named barrier below
        if (lt == 0)
          sLdOk[it & 1] = !*sAbort && (gt < (uint32_t)kNS || mbar_wait(&kempty[st], ((gt / kNS) - 1) & 1u, p.status));
        named_sync(3, kLoaders);
        if (!sLdOk[it & 1]) {
          *sAbort = 1;
          stopped = true;
          break;
        }
        uint8_t* dst = sK + st * kStageBytes;
        int row0 = 0;
        const int mode = tile_src(it, row0);
        if (mode >= 0) {
          if (lt == 0) {
            mbar_arrive_expect_tx(&kfull[st], kStageBytes);
            const CUtensorMap* map = mode == 0 ? &tm_ring : &tm_kv;
            for (int j = 0; j < kNb; ++j)
              tma_load_2d(dst + j * (kNk * 128), map, (kb_load0 + j) * 64, row0, &kfull[st]);
          }
          if (pend_it >= 0) finish(pend_it, false);
          pend_it = -1;
        } else {
          // consecutive threads take consecutive 16-byte chunks of a row (coalesced); bf16 rows go
          // by cp.async, FP8 entries into registers (widened into the tile when it is finished)
          uint2 codes[kPer];
#pragma unroll
          for (int q = 0; q < kPer; ++q) {
            const int id = lt + q * kLoaders;
            codes[q] = make_uint2(0u, 0u);
            if (id < kItems) {
              const int kr = id / (kNb * 8), c = id % (kNb * 8);
              const int i = it * kNk + kr;
              const void* src = i < nk ? sRow[i] : nullptr;
              if (src && fp8 && u0 + i >= kk.n_w)
                codes[q] = __ldg(reinterpret_cast<const uint2*>(static_cast<const uint8_t*>(src) + kb_load0 * 64 +
                                                                c * 8));
              else
                cp_async16(dst + swz(kr, c, kNk * 128),
                           src ? static_cast<const void*>(static_cast<const uint16_t*>(src) + kb_load0 * 64 + c * 8)
                               : p.q,
                           src ? 16 : 0);
            }
          }
          cp_async_commit();
          if (pend_it >= 0) finish(pend_it, true);
#pragma unroll
          for (int q = 0; q < kPer; ++q) pend_codes[q] = codes[q];
          pend_it = it;
        }
      }
      if (pend_it >= 0 && !stopped) finish(pend_it, false);
    } else if (tid == kMmaThread) {
      // ------------------------------------------------------------ MMA issue
      const uint32_t idesc_s = umma_idesc_bf16(kM, kNk, false);
      const uint32_t idesc_pv = umma_idesc_bf16(kM, 256, true);
      const uint32_t sQa = smem_u32(sQ), sKa = smem_u32(sK);
      bool ok = mbar_wait(qbar, n_item & 1u, p.status);
      for (int it = 0; it <= ntiles + 1 && ok && !*sAbort; ++it) {
        if (it < ntiles) {
          const uint32_t gt = g + it;
          const int st = gt % kNS, buf = gt % kNSP;
          // the tile is shared memory written by TMA or fenced cp.async / stores: the mbarrier
          // orders it; tensor memory reuse is ordered by the fence after the P waits below
          if (!(ok = mbar_wait(&kfull[st], (gt / kNS) & 1u, p.status))) break;
          const uint32_t d = tmem + kColS + buf * kNk;
          const uint32_t kb = sKa + st * kStageBytes + s_blk0 * (kNk * 128);
          // 20 (rank 0) or 16 (rank 1) MMAs into one accumulator
          if (rank == 0)
            issue_s<5, 2>(d, sQa, tmem + kColQ, kb, idesc_s);
          else
            issue_s<4, 1>(d, sQa, tmem + kColQ, kb, idesc_s);
          umma_commit(&sfull[buf]);
        }
        if (it >= 2) {
          const uint32_t gp = g + it - 2;
          const int pb = gp % kNSP, sp = gp % kNS;
          if (!(ok = mbar_wait(&pfull[pb], (gp / kNSP) & 1u, p.status))) break;
          tc_fence_after();
          const uint32_t vb = sKa + sp * kStageBytes;  // blocks 0..3 of the stage: this CTA's V
#pragma unroll
          for (int k2 = 0; k2 < 2; ++k2)
            umma_ts(tmem + kColO, tmem + kColP + pb * 16 + k2 * 8,
                    umma_desc_sw128(vb + k2 * 16 * 128, kNk * 128, 1024), idesc_pv, (it > 2 || k2 > 0) ? 1u : 0u);
          umma_commit(&kempty[sp]);
          umma_commit(&obar[pb]);
        }
      }
      umma_commit(dbar);  // one completion per item, also after an abort
      if (!ok) *sAbort = 1;
    } else if (warp < 4) {
      // ------------------------------------------------------------ softmax (one head row per thread)
      const float sl2 = p.sm_scale * kLog2e;
      const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
      const uint32_t recv_peer = peer_addr(sRecv, peer);
      const uint32_t rfull_peer = peer_addr(rfull, peer);
      const uint32_t rempty_peer = peer_addr(rempty, peer);
      const int rr = tid;  // head row
      float m_used = -INFINITY, l_run = 0.f;
      // Loop control is per warp (the four warps never meet at a barrier inside the loop); a
      // failed wait raises the abort flag, and the other warps stop at their next bounded wait.
      bool ok = true;
      float part[32];
      // own partial of tile gt into part[], and one bulk copy of it into the other CTA's slot gt & 1
      auto produce = [&](uint32_t gt) -> bool {
        const int buf = gt % kNSP, slot = gt & 1;
        if (!__all_sync(kFull, mbar_wait(&sfull[buf], (gt / kNSP) & 1u, p.status))) *sAbort = 1;
        tc_fence_after();
        uint32_t s0[32];
        tmem_ld32(tmem + lane_base + kColS + buf * kNk, s0);
        tmem_ld_wait();
#pragma unroll
        for (int j = 0; j < 32; ++j) part[j] = __uint_as_float(s0[j]);
        // slot gt & 1 of the send buffers here and of the receive slots there held tile gt - 2:
        // both are free once the other CTA has read that tile. Each warp sends its own 32 rows
        // (4 KB) by its own bulk copy, so the warps need not meet.
        bool sent = !*sAbort;
        if (lane == 0 && sent && gt >= 2) sent = mbar_wait(&rempty[slot], ((gt >> 1) - 1) & 1u, p.status);
        sent = __shfl_sync(kFull, sent, 0);
        if (sent) {
          uint8_t* row = sSend + slot * kRecvBytes + rr * 128;
#pragma unroll
          for (int c = 0; c < 8; ++c)
            *reinterpret_cast<uint4*>(row + ((c ^ (rr & 7)) << 4)) =
                make_uint4(__float_as_uint(part[4 * c]), __float_as_uint(part[4 * c + 1]),
                           __float_as_uint(part[4 * c + 2]), __float_as_uint(part[4 * c + 3]));
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0)
            bulk_copy_to_peer(recv_peer + slot * kRecvBytes + warp * 4096, sSend + slot * kRecvBytes + warp * 4096,
                              4096, rfull_peer + slot * 8);
        }
        return sent;
      };
      {  // this thread's head row of the tensor-memory Q blocks (bf16 pairs, low half first)
        const uint16_t* qg = p.q + ((int64_t)b * p.n_heads + grp * kM + rr) * kDqk + (qkb0 + n_qs) * 64;
#pragma unroll 1
        for (int t = 0; t < kQTmem; ++t) {
          uint32_t qv[32];
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            const uint4 v = ldg16(qg + t * 64 + c * 8);
            qv[4 * c] = v.x;
            qv[4 * c + 1] = v.y;
            qv[4 * c + 2] = v.z;
            qv[4 * c + 3] = v.w;
          }
          tmem_st32(tmem + lane_base + kColQ + t * 32, qv);
        }
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(qbar);
      }
      if (ntiles > 0) ok = produce(g);
      for (int it = 0; it < ntiles && ok; ++it) {
        const uint32_t gt = g + it;
        const int buf = gt % kNSP, slot = gt & 1;
        float cur[32];
#pragma unroll
        for (int j = 0; j < 32; ++j) cur[j] = part[j];
        if (it + 1 < ntiles && !(ok = produce(gt + 1))) break;
        // the other CTA's partial of tile gt: one arrival (here) and 16 KB of its bulk copy
        if (tid == 0) mbar_arrive_expect_tx(&rfull[slot], kRecvBytes);
        if (!__all_sync(kFull, mbar_wait(&rfull[slot], (gt >> 1) & 1u, p.status))) *sAbort = 1;
        const uint8_t* src = sRecv + slot * kRecvBytes + rr * 128;
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          const uint4 v = lds16(src + ((c ^ (rr & 7)) << 4));
          cur[4 * c] += __uint_as_float(v.x);
          cur[4 * c + 1] += __uint_as_float(v.y);
          cur[4 * c + 2] += __uint_as_float(v.z);
          cur[4 * c + 3] += __uint_as_float(v.w);
        }
        __syncwarp();
        if (lane == 0) mbar_arrive_peer(rempty_peer + slot * 8);
        const uint32_t valid = sMask[it];
        float v[32];
        float mt = -INFINITY;
        if (fp8) {  // an FP8 entry's logit and value carry its scale
#pragma unroll
          for (int j = 0; j < 32; ++j) cur[j] *= sScale[it * kNk + j];
        }
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          v[j] = ((valid >> j) & 1u) ? cur[j] * sl2 : -INFINITY;  // keys past nk have no row
          mt = fmaxf(mt, v[j]);
        }
        float corr = 1.f;
        bool rescale = false;
        if (mt > m_used + kRescaleThreshold || (m_used == -INFINITY && mt != -INFINITY)) {
          corr = exp2f(m_used - mt);  // 0 when m_used is -inf
          rescale = it > 0;
          l_run *= corr;
          m_used = mt;
        }
        const float msub = m_used == -INFINITY ? 0.f : m_used;
        uint32_t pp[16];
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const float p0 = exp2f(v[2 * j] - msub), p1 = exp2f(v[2 * j + 1] - msub);
          l_run += p0 + p1;
          pp[j] = fp8 ? pack_bf16(p0 * sScale[it * kNk + 2 * j], p1 * sScale[it * kNk + 2 * j + 1]) : pack_bf16(p0, p1);
        }
        // P buffer gt % 3 was read by the P V of tile gt - 3
        if (gt >= (uint32_t)kNSP && !__all_sync(kFull, mbar_wait(&obar[buf], ((gt / kNSP) - 1) & 1u, p.status)))
          *sAbort = 1;
        if (__any_sync(kFull, rescale)) {
          // O takes the rescale once the P V of tile gt - 1 (and so every earlier one) has landed
          const uint32_t gq = gt - 1;
          if (!__all_sync(kFull, mbar_wait(&obar[gq % kNSP], (gq / kNSP) & 1u, p.status))) *sAbort = 1;
          tc_fence_after();
#pragma unroll 1
          for (int c = 0; c < 256; c += 32) {
            uint32_t orow[32];
            tmem_ld32(tmem + lane_base + kColO + c, orow);
            tmem_ld_wait();
#pragma unroll
            for (int j = 0; j < 32; ++j) orow[j] = __float_as_uint(__uint_as_float(orow[j]) * corr);
            tmem_st32(tmem + lane_base + kColO + c, orow);
          }
        }
        tmem_st16(tmem + lane_base + kColP + buf * 16, pp);
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(&pfull[buf]);
      }
      // epilogue: normalised partial output of this split and half, and its log-sum-exp
      ok = __all_sync(kFull, mbar_wait(dbar, n_item & 1u, p.status)) && ok;
      if (!ok) *sAbort = 1;
      tc_fence_after();
      const int head0 = grp * kM;
      const int64_t prow0 = ((int64_t)b * p.max_splits + split) * p.n_heads + head0;
      const float inv = l_run > 0.f ? 1.f / l_run : 0.f;
      // each thread writes its head row straight from tensor memory: part_o is
      // head-minor ([query x split][d_v / 4][heads][4]), so a warp's 16-byte
      // stores cover 32 consecutive heads, 512 contiguous bytes
      float4* po = reinterpret_cast<float4*>(p.part_o) +
                   (((int64_t)b * p.max_splits + split) * (kDv / 4) + rank * 64) * p.n_heads + head0 + rr;
#pragma unroll 1
      for (int c = 0; c < 256; c += 32) {
        uint32_t orow[32];
        if (ok) {
          tmem_ld32(tmem + lane_base + kColO + c, orow);
          tmem_ld_wait();
        }
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const float4 v = ok ? make_float4(__uint_as_float(orow[4 * k]) * inv, __uint_as_float(orow[4 * k + 1]) * inv,
                                            __uint_as_float(orow[4 * k + 2]) * inv, __uint_as_float(orow[4 * k + 3]) * inv)
                              : make_float4(0.f, 0.f, 0.f, 0.f);
          po[(int64_t)(c / 4 + k) * p.n_heads] = v;
        }
      }
      if (rank == 0) p.part_lse[prow0 + tid] = l_run > 0.f ? (m_used + log2f(l_run)) * kLn2 : -INFINITY;
    }
    g += ntiles;
    tc_fence_before();
    __syncthreads();  // shared and tensor memory are reused by the next item
    tc_fence_after();
    if (*sAbort) {
      if (tid == 0) st_peer_u32(peer_addr(const_cast<int*>(sAbort), peer), 1u);  // stop the other CTA too
      break;
    }
  }
  // after an abort, give tensor-core work in flight a bounded chance to land before freeing
  if (*sAbort && tid == kMmaThread) mbar_wait(dbar, n_item & 1u, nullptr);
  cp_async_wait<0>();
  tc_fence_before();
  cluster.sync();  // the other CTA may still write into this one's shared memory until here
  tc_fence_after();
  if (warp == 4) tmem_dealloc(tmem, kTmemCols);
}

bool encode_rows(CUtensorMap* map, const void* base, uint64_t rows, uint32_t box_rows) {
  auto enc = tensor_map_encoder();
  if (!enc) return false;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(kDqk), static_cast<cuuint64_t>(rows)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(kDqk) * 2};
  const cuuint32_t box[2] = {64, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

bool attend_tc_supported(int d_qk, int d_v, int n_heads, int kv_dtype, int n_q) {
  return d_qk == kDqk && d_v == kDv && n_heads % kM == 0 && (kv_dtype == CSKV_BF16 || kv_dtype == CSKV_FP8_E4M3) &&
         Smem::bytes(n_q) <= 232448;  // the per-query prefix table shares shared memory with the tiles
}

// keys per split: queries x head groups x splits ~ one CTA pair per two SMs
void attend_tc_plan(AttendParams& p, int n_sm) {
  const int64_t groups = p.n_heads / kM;
  const int64_t n_max = (int64_t)p.n_win + (p.is_csa ? p.k : visible_entries(p.max_pos, p.m, p.n_win));
  int64_t splits = (n_sm / 2) / ((int64_t)p.n_q * groups);
  if (splits < 1) splits = 1;
  int64_t kps = (n_max + splits - 1) / splits;
  kps = (kps + kNk - 1) / kNk * kNk;
  if (kps < kNk) kps = kNk;
  if (kps > kRowCap) kps = kRowCap;
  p.keys_per_split = static_cast<int>(kps);
  p.max_splits = static_cast<int>((n_max + kps - 1) / kps);
  if (p.max_splits < 1) p.max_splits = 1;
}

cudaError_t launch_attend_tc(AttendParams& p, int n_sm, cudaStream_t st) {
  CUtensorMap tm_q, tm_ring, tm_kv;
  const uint64_t kv_rows = static_cast<uint64_t>(p.n_pages) * p.page_size;
  const uint64_t ring_rows = static_cast<uint64_t>(p.n_seqs_layer) * p.n_win;
  if (kv_rows >= (1ull << 31) || ring_rows >= (1ull << 31)) return cudaErrorNotSupported;
  if (!encode_rows(&tm_q, p.q, static_cast<uint64_t>(p.n_q) * p.n_heads, kM) ||
      !encode_rows(&tm_ring, p.ring_x, ring_rows, kNk) ||
      // an FP8 pool is never read by TMA (its tiles are widened by the loaders)
      !encode_rows(&tm_kv, p.kv_dtype == CSKV_FP8_E4M3 ? static_cast<const void*>(p.ring_x) : p.kv_pool,
                   p.kv_dtype == CSKV_FP8_E4M3 ? ring_rows : kv_rows, kNk))
    return cudaErrorNotSupported;
  const size_t smem = Smem::bytes(p.n_q);
  const bool fp8 = p.kv_dtype == CSKV_FP8_E4M3;
  auto kern = fp8 ? attend_tc_kernel<true> : attend_tc_kernel<false>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  const int64_t upper = (int64_t)p.n_q * p.max_splits * (p.n_heads / kM);
  int64_t clusters = upper < n_sm / 2 ? upper : n_sm / 2;
  if (clusters < 1) clusters = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(2 * clusters), 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  p.part_t = 1;
  e = cudaLaunchKernelEx(&cfg, kern, tm_q, tm_ring, tm_kv, p);
  if (e != cudaSuccess) return e;
  return launch_attend_merge(p, st);
}

}  // namespace cskv
