// attend_tc.cu -- CSA / HCA core attention on the 5th-generation tensor cores
// (tcgen05) for the wide shared latent: d_qk = 576 (512 latent + 64 RoPE
// channels), d_v = 512, query heads in groups of 64 (DeepSeek-V4 report
// digest, section 3: one softmax over the window and the selected / all
// compressed entries; DeepSeek-V4-book ch.1, section 4: the MLA latent shared
// by every head).
//
// With 128 heads on one 576-wide latent every key carries 2 x 128 x 1088
// flops against 1152 bytes, at the B200's ridge point. O for 128 heads x 512
// channels in fp32 would fill a whole SM's tensor memory, so a work item =
// (query, 64-head group, key split): the two head groups of a split run on two
// CTAs that read the same key tiles (the second read is served by L2) and never
// talk to each other. Per CTA, everything is local:
//   - S = Q K^T with the 64 heads as M and a 64-key tile as N, Q (64 x 576) and
//     the key tile (64 x 576) in shared memory; the channel blocks alternate
//     between two accumulators (a tcgen05.mma that accumulates into the tile of
//     the one before it waits for it, ~90 cycles per step, while two chains run
//     at the operand rate), the even blocks at tensor-memory lane offset 0 and
//     the odd ones at lane offset 16 of the same columns (an M = 64 accumulator
//     fills lanes 0-15 of each 32-lane quarter);
//   - O = P V in two halves of 256 channels, O[:, 0:256] at lane offset 0 and
//     O[:, 256:512] at lane offset 16 of columns 0-255, P (bf16) in shared
//     memory as the A operand, V read MN-major from the key tile (V = the first
//     d_v channels of every key);
//   - thread (warp w, lane l) of the softmax warpgroup owns head row 16 w +
//     (l & 15) and keys 32 (l >> 4) .. + 31 of each tile: it reads its lane's
//     accumulator, swaps 32 values with lane l ^ 16 to form the full S of its
//     keys, and the row max is one more swap; the two lanes of a row keep the
//     same running max, and the rare O rescale touches exactly the O rows of
//     every lane (both halves);
//   - one warp issues only S, so the next tile's S runs while this tile's
//     exponentials are taken; softmax thread 0 issues the tile's P V once every
//     row has stored its P (a named barrier that also decides aborts uniformly);
//   - loaders look up each tile's source rows one tile ahead, while the tile
//     before it is copied (its page-table reads included): TMA when a
//     tile's rows are contiguous (window rows of the ring, HCA entries of one
//     page), TMA gather of single rows for a bf16 tile of pool rows (the CSA
//     selection), the codes of an FP8 tile of pool rows staged by cp.async and
//     widened exactly to bf16 in place, cp.async through the looked-up rows
//     otherwise.
// O is rescaled only when a row's running max rises by more than 2^8 (the
// probabilities stay below 256 in bf16), so most tiles skip it. Window keys are
// taken in ring-slot order (the softmax does not depend on the order of its
// keys), which makes a window tile 64 consecutive ring rows. Each item writes
// its normalised partial output and log-sum-exp; attend_merge_t_kernel combines
// the splits.
#include "cskv_device.cuh"
#include "cskv_internal.h"

namespace cskv {
namespace {

constexpr int kDqk = 576, kDv = 512, kH = 64, kNk = 64;
constexpr int kNb = kDqk / 64;                  // 9 channel blocks of a key row
constexpr int kBlkBytes = kNk * 128;            // 8192: one channel block of a 64-row tile
constexpr int kStageBytes = kNb * kBlkBytes;    // 73728: a key tile (also the Q block set)
constexpr int kNS = 2;                          // key-tile stages
constexpr int kPBytes = kH * kNk * 2;           // 8192: P of the tile (bf16)
constexpr int kThreads = 256;                   // warps 0-3 softmax, warp 4 S, warps 5-7 loads
constexpr int kLoadThread0 = 160;
constexpr int kLoaders = kThreads - kLoadThread0;  // 96
constexpr int kChunks = kNk * kNb * 8;          // 16-byte chunks of a bf16 tile (4608)
constexpr int kPer = (kChunks + kLoaders - 1) / kLoaders;  // 48
constexpr uint32_t kTmemCols = 512;
// O[:, 0:256] lanes +0 and O[:, 256:512] lanes +16 of columns 0-255; S buffer k at columns
// 256 + 64 k (even channel blocks at lanes +0, odd ones at lanes +16)
constexpr uint32_t kColO = 0, kColS = 256;
constexpr uint32_t kLane16 = 16u << 16;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kRescaleThreshold = 8.0f;       // log2 units
constexpr int kMaxSplitKeys = 1024;             // keys of one HCA work item at most (16 tiles)

struct Smem {
  static constexpr int Q = 0;                          // 9 blocks of 64 heads x 128 B
  static constexpr int K = Q + kStageBytes;            // kNS key tiles
  static constexpr int P = K + kNS * kStageBytes;      // P of the tile (64 rows x 128 B)
  static constexpr int CODE = P + kPBytes;             // [kNS][kNk] source-row codes of a stage's keys
  static constexpr int SCALE = CODE + kNS * kNk * 4;   // [kNS][kNk] FP8 scale of each key (1 for bf16 rows)
  static constexpr int MASK = SCALE + kNS * kNk * 4;   // [kNS][2] valid-key bits
  static constexpr int BAR = MASK + 32;                // mbarriers
  static constexpr int TMEM = BAR + 16 * 8;            // allocated tensor-memory address
  static constexpr int FLAGS = TMEM + 16;
  static constexpr int PREF = FLAGS + 16;              // [n_q + 1] items per query, exclusive prefix
  static size_t bytes(int n_q) { return 1024 + PREF + sizeof(int) * (size_t)(n_q + 1); }
};

// source-row code: kind in bits [31:30] (0 none, 1 pool entry, 2 ring row, 3 chunk row), row below
constexpr uint32_t kRowBits = 30;
constexpr uint32_t kRowMask = (1u << kRowBits) - 1u;

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

// Code of the source row of key u: window keys first, in ring-slot order (slot
// u) when every window row is in the ring, in position order when a prefill
// chunk supplies some of them; then the compressed entries. 0 if invalid.
__device__ __forceinline__ uint32_t key_code(const AttendParams& p, int b, int seq, const Keys& k, int64_t u) {
  if (u < k.n_w) {
    if (!p.x_chunk) return (2u << kRowBits) | static_cast<uint32_t>((int64_t)seq * p.n_win + u);
    const int64_t pos = k.ws + u;
    const int64_t cr = chunk_row(p, seq, pos);
    if (cr >= 0) return (3u << kRowBits) | static_cast<uint32_t>(cr);
    return (2u << kRowBits) | static_cast<uint32_t>((int64_t)seq * p.n_win + pos % p.n_win);
  }
  const int64_t jj = u - k.n_w;
  const int64_t j = p.is_csa ? static_cast<int64_t>(p.sel_idx[(int64_t)b * p.k + jj]) : jj;
  if (j < 0 || j >= visible_entries(k.t, p.m, p.n_win)) return 0;
  const int64_t pi = j / p.page_size;
  if (pi >= p.max_pages_per_seq) return 0;
  const int32_t page = p.page_table[(int64_t)seq * p.max_pages_per_seq + pi];
  if (page < 0 || page >= p.n_pages) return 0;
  return (1u << kRowBits) | static_cast<uint32_t>((int64_t)page * p.page_size + j % p.page_size);
}

// the bf16 row of a code (an FP8 pool row is read as codes by the loaders)
__device__ __forceinline__ const uint16_t* code_row(const AttendParams& p, uint32_t c) {
  const uint32_t kind = c >> kRowBits, row = c & kRowMask;
  if (kind == 1) return static_cast<const uint16_t*>(p.kv_pool) + (size_t)row * kDqk;
  if (kind == 2) return p.ring_x + (size_t)row * kDqk;
  if (kind == 3) return p.x_chunk + (size_t)row * kDqk;
  return nullptr;
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

__device__ __forceinline__ void named_sync(int id, int n) {
  asm volatile("bar.sync %0, %1;\n" ::"r"(id), "r"(n) : "memory");
}
// named barrier over n threads that also returns the OR of `v` over them (the same in every thread)
__device__ __forceinline__ bool named_sync_or(int id, int n, bool v) {
  uint32_t r;
  asm volatile(
      "{\n .reg .pred q, p;\n setp.ne.u32 q, %1, 0;\n bar.red.or.pred p, %2, %3, q;\n selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(r)
      : "r"(v ? 1u : 0u), "r"(id), "r"(n)
      : "memory");
  return r != 0;
}

// S of one key tile: 9 channel blocks x 4 K-steps (M = 64 heads, N = 64 keys); even blocks
// accumulate at d (lanes +0), odd blocks at d + 16 lanes, the two chains issued alternately
__device__ __forceinline__ void issue_s(uint32_t d, uint32_t q, uint32_t k, uint32_t idesc) {
#pragma unroll
  for (int s = 0; s < 20; ++s) {
    const int ia = 2 * (s >> 2), ks = s & 3;
    umma_ss(d, umma_desc_sw128(q + ia * kBlkBytes + ks * 32, 16, 1024),
            umma_desc_sw128(k + ia * kBlkBytes + ks * 32, 16, 1024), idesc, s > 0 ? 1u : 0u);
    if (s < 16) {
      const int ib = ia + 1;
      umma_ss(d + kLane16, umma_desc_sw128(q + ib * kBlkBytes + ks * 32, 16, 1024),
              umma_desc_sw128(k + ib * kBlkBytes + ks * 32, 16, 1024), idesc, s > 0 ? 1u : 0u);
    }
  }
}

// Pipeline (per CTA; tiles numbered gt across its items; stage and S buffer gt & 1):
//   loaders : look up the tile's source rows -> wait kempty (P V of tile gt - 2 done) ->
//             TMA, or cp.async / widened FP8 stores, into the stage -> kfull
//   S warp  : wait kfull, sfree (softmax has read S(gt - 2)) -> S(gt) -> commit sfull
//   softmax : wait sfull -> read S, swap halves with lane ^ 16, arrive sfree -> P(gt) ->
//             wait obar (P V of gt - 1 done: P buffer free, O settled; rare rescale) ->
//             store P -> named barrier -> thread 0: O += P V(gt) -> commit kempty, obar
// FP8: the pool holds E4M3 entries with an fp32 scale each (a separate
// instantiation keeps the bf16 kernel's code small)
template <bool FP8>
__global__ void __launch_bounds__(kThreads, 1)
    attend_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_ring,
                     const __grid_constant__ CUtensorMap tm_kv, const __grid_constant__ CUtensorMap tm_kvg,
                     AttendParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = sm + Smem::Q;
  uint8_t* sK = sm + Smem::K;
  uint8_t* sP = sm + Smem::P;
  uint32_t* sCode = reinterpret_cast<uint32_t*>(sm + Smem::CODE);
  float* sScale = reinterpret_cast<float*>(sm + Smem::SCALE);
  uint32_t* sMask = reinterpret_cast<uint32_t*>(sm + Smem::MASK);
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + Smem::BAR);
  uint64_t* kfull = bars;             // [2] loaders -> S warp (and the softmax, for the stage's key bits)
  uint64_t* kempty = bars + 2;        // [2] P V of the stage's tile done (commit)
  uint64_t* sfull = bars + 4;         // [2] S of the buffer's tile done (commit)
  uint64_t* sfree = bars + 6;         // [2] softmax has read the buffer (128 arrivals)
  uint64_t* obar = bars + 8;          //     a tile's P V done (commit)
  uint64_t* qbar = bars + 9;          //     Q of the item landed (TMA)
  uint64_t* dbar = bars + 10;         //     the item's last P V done (commit)
  constexpr bool fp8 = FP8;
  uint32_t* sTmem = reinterpret_cast<uint32_t*>(sm + Smem::TMEM);
  volatile int* sAbort = reinterpret_cast<int*>(sm + Smem::FLAGS);
  volatile int* sLdOk = reinterpret_cast<int*>(sm + Smem::FLAGS) + 1;
  volatile int* sPool = reinterpret_cast<int*>(sm + Smem::FLAGS) + 2;  // [2] per code warp: the tile is gatherable
  int* sPref = reinterpret_cast<int*>(sm + Smem::PREF);
  __shared__ int s_wsum[32];

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int groups = p.n_heads / kH;
  const int kps = p.keys_per_split;

  if (tid == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&kfull[i], 1);
      mbar_init(&kempty[i], 1);
      mbar_init(&sfull[i], 1);
      mbar_init(&sfree[i], 128);
    }
    mbar_init(obar, 1);
    mbar_init(qbar, 1);
    mbar_init(dbar, 1);
    fence_barrier_init();
    *sAbort = 0;
  }
  if (tid == kLoadThread0) {
    prefetch_tensormap(&tm_q);
    prefetch_tensormap(&tm_ring);
    prefetch_tensormap(&tm_kv);
    if (!FP8) prefetch_tensormap(&tm_kvg);
  }
  if (warp == 4) {
    tmem_alloc(sTmem, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
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
  uint32_t g = 0;       // tiles processed by this CTA before the current item
  uint32_t n_item = 0;  // items processed before the current one (qbar / dbar phase)

  // consecutive items are the head groups of one split, so the CTAs reading the same keys run together
  for (int item = blockIdx.x; item < total; item += gridDim.x, ++n_item) {
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
    if (tid == 0 && grp == 0 && !seq_ok && kk.n > 0) report(p.status, CSKV_ERR_OUT_OF_RANGE);

    if (tid >= kLoadThread0) {
      // ------------------------------------------------------------ loaders
      const int lt = tid - kLoadThread0, lw = lt >> 5, ll = lt & 31;
      if (lw == 0) {  // Q of the head group: 9 boxes of 64 rows x 64 channels
        if (ll == 0) {
          mbar_arrive_expect_tx(qbar, kStageBytes);
          const int qrow = b * p.n_heads + grp * kH;
          for (int j = 0; j < kNb; ++j) tma_load_2d(sQ + j * kBlkBytes, &tm_q, j * 64, qrow, qbar);
        }
        __syncwarp();
      }
      // TMA source of tile it: 0 = ring rows, 1 = pool rows (row0 set), -1 = looked-up rows
      auto tile_src = [&](int it, int& row0) -> int {
        const int64_t a = u0 + (int64_t)it * kNk;
        if (!seq_ok || (it + 1) * kNk > nk) return -1;  // a partial tile: rows past its end are not zero
        if (!p.x_chunk && a + kNk <= kk.n_w) {
          row0 = static_cast<int>((int64_t)seq * p.n_win + a);
          return 0;
        }
        if (!p.is_csa && !fp8 && a >= kk.n_w) {
          const int64_t j0 = a - kk.n_w;
          const int64_t pi = j0 / p.page_size;
          if (j0 % p.page_size + kNk > p.page_size || pi >= p.max_pages_per_seq) return -1;
          const int32_t page = p.page_table[(int64_t)seq * p.max_pages_per_seq + pi];
          if (page < 0 || page >= p.n_pages) return -1;
          row0 = static_cast<int>((int64_t)page * p.page_size + j0 % p.page_size);
          return 1;
        }
        return -1;
      };
      // the source row of key lt of tile it (threads 0 .. kNk - 1), and its FP8 scale
      auto code_of = [&](int it, float& sc) -> uint32_t {
        sc = 0.f;
        const int i = it * kNk + lt;
        if (lt >= kNk || i >= nk || !seq_ok) return 0u;
        const uint32_t c = key_code(p, b, seq, kk, u0 + i);
        if (!c) {
          if (grp == 0) report(p.status, CSKV_ERR_OUT_OF_RANGE);
          return 0u;
        }
        sc = (fp8 && (c >> kRowBits) == 1u) ? p.kv_scale[c & kRowMask] : 1.f;
        return c;
      };
      auto prefetch = [&](uint32_t c) {  // the row into L2 ahead of its copy
        if (!c) return;
        if (fp8 && (c >> kRowBits) == 1u)
          prefetch_l2(static_cast<const uint8_t*>(p.kv_pool) + (size_t)(c & kRowMask) * kDqk, kDqk);
        else
          prefetch_l2(code_row(p, c), kDqk * 2);
      };
      // the next tile's source (its page-table lookup included) is found before its stage frees
      float nsc = 0.f;
      uint32_t ncode = ntiles > 0 ? code_of(0, nsc) : 0u;
      int nrow0 = 0;
      int nmode = ntiles > 0 ? tile_src(0, nrow0) : -1;
      if (ntiles > 0 && nmode < 0) prefetch(ncode);
      for (int it = 0; it < ntiles; ++it) {
        const uint32_t gt = g + it;
        const int st = gt & 1;
        const uint32_t code = ncode;
        const float scale = nsc;
        // the first loader warp takes the stage wait (all lanes; lane 0 records the result)
        if (lw == 0) {
          bool okw = __shfl_sync(kFull, *sAbort, 0) == 0;
          if (okw && gt >= 2u) okw = __all_sync(kFull, mbar_wait(&kempty[st], ((gt >> 1) - 1) & 1u, p.status));
          if (ll == 0) *sLdOk = okw;
        }
        named_sync(3, kLoaders);
        if (!*sLdOk) {
          *sAbort = 1;
          break;
        }
        if (lt < kNk) {
          sCode[st * kNk + lt] = code;
          sScale[st * kNk + lt] = code ? scale : 0.f;  // finite for every key of the tile
        }
        if (lw < 2) {
          const unsigned bits = __ballot_sync(kFull, code != 0u);
          // a bf16 tile whose rows are all pool rows (or none) is gathered by TMA
          const bool pool = __all_sync(kFull, code == 0u || (code >> kRowBits) == 1u);
          if (ll == 0) {
            sMask[st * 2 + lw] = bits;
            sPool[lw] = pool ? 1 : 0;
          }
        }
        named_sync(3, kLoaders);
        uint8_t* dst = sK + st * kStageBytes;
        const int row0 = nrow0;
        const int mode = nmode;
        if (mode >= 0) {
          if (lt == 0) {
            mbar_arrive_expect_tx(&kfull[st], kStageBytes);
            const CUtensorMap* map = mode == 0 ? &tm_ring : &tm_kv;
            for (int j = 0; j < kNb; ++j) tma_load_2d(dst + j * kBlkBytes, map, j * 64, row0, &kfull[st]);
          }
          if (it + 1 < ntiles) {
            ncode = code_of(it + 1, nsc);
            nmode = tile_src(it + 1, nrow0);
            if (nmode < 0) prefetch(ncode);
          }
        } else if (!fp8 && sPool[0] && sPool[1]) {
          // the tile's rows by TMA gather, four rows of one 64-channel block per copy; a key without
          // a row reads row -1, outside the map: zeros, as the copies below would write
          if (lt == 0) mbar_arrive_expect_tx(&kfull[st], kStageBytes);
          named_sync(3, kLoaders);  // the stage's byte count is set before any of its copies lands
          for (int q = lt; q < kNb * (kNk / 4); q += kLoaders) {
            const int j = q / (kNk / 4), r4 = (q % (kNk / 4)) * 4;
            int y[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const uint32_t cd = sCode[st * kNk + r4 + e];
              y[e] = (cd >> kRowBits) == 1u ? static_cast<int>(cd & kRowMask) : -1;
            }
            tma_gather4(dst + j * kBlkBytes + r4 * 128, &tm_kvg, j * 64, y[0], y[1], y[2], y[3], &kfull[st]);
          }
          if (it + 1 < ntiles) {
            ncode = code_of(it + 1, nsc);
            nmode = tile_src(it + 1, nrow0);
            if (nmode < 0) prefetch(ncode);
          }
        } else if (fp8 && sPool[0] && sPool[1]) {
          // FP8 pool rows: the tile's E4M3 codes (half a bf16 tile) are copied into the stage's upper
          // half by cp.async, block-major (block j's 64 codes of every key at stg + 4096 j), so the
          // next tile's row lookups overlap the copies; then they are widened exactly to bf16 in
          // place, in passes whose writes cover only staged blocks that earlier passes have read:
          // blocks 0-3 (below the staged codes), 4-5, 6, 7, then 8, whose own codes it overwrites
          // (read first, then a barrier). A key without a row gets zeros.
          constexpr int kStg = kStageBytes / 2;            // 36864
          constexpr int kCodeBlk = kNk * 64;               // 4096: one staged block of codes
          static_assert(kStg + kNb * kCodeBlk == kStageBytes && 4 * kBlkBytes <= kStg, "staging");
          uint8_t* stg = dst + kStg;
          const uint8_t* pool = static_cast<const uint8_t*>(p.kv_pool);
          for (int q = lt; q < kNk * kNb * 4; q += kLoaders) {  // (key, block, 16-byte piece)
            const int kr = q / (kNb * 4), j = (q / 4) % kNb, c4 = q % 4;
            const uint32_t cd = sCode[st * kNk + kr];
            if (cd)
              cp_async16(stg + j * kCodeBlk + kr * 64 + c4 * 16,
                         pool + (size_t)(cd & kRowMask) * kDqk + j * 64 + c4 * 16, 16);
          }
          cp_async_commit();
          if (it + 1 < ntiles) {  // the next tile's rows are looked up while the codes fly
            ncode = code_of(it + 1, nsc);
            nmode = tile_src(it + 1, nrow0);
            if (nmode < 0) prefetch(ncode);
          }
          cp_async_wait<0>();
          // the 8 codes of bf16 chunk (key kr, block j, piece pc), and their widened store
          auto codes_at = [&](int kr, int j, int pc) -> uint2 {
            return sCode[st * kNk + kr] ? *reinterpret_cast<const uint2*>(stg + j * kCodeBlk + kr * 64 + pc * 8)
                                        : make_uint2(0u, 0u);
          };
          auto put = [&](int kr, int j, int pc, uint2 c8) {
            *reinterpret_cast<uint4*>(dst + j * kBlkBytes + kr * 128 + ((pc ^ (kr & 7)) << 4)) = e4m3x8_to_bf16x8(c8);
          };
          auto widen = [&](int j0, int j1) {  // blocks j0 .. j1 - 1
            for (int id = lt; id < kNk * (j1 - j0) * 8; id += kLoaders) {
              const int kr = id / ((j1 - j0) * 8), j = j0 + (id / 8) % (j1 - j0), pc = id % 8;
              put(kr, j, pc, codes_at(kr, j, pc));
            }
          };
          named_sync(3, kLoaders);  // every staged code is visible to every loader
          widen(0, 4);
          named_sync(3, kLoaders);
          widen(4, 6);  // overwrites staged blocks 0-2
          named_sync(3, kLoaders);
          widen(6, 7);  // 3-4
          named_sync(3, kLoaders);
          widen(7, 8);  // 5-6
          constexpr int kLastPer = (kNk * 8 + kLoaders - 1) / kLoaders;  // 6
          uint2 last[kLastPer];
#pragma unroll
          for (int k2 = 0; k2 < kLastPer; ++k2) {
            const int id = lt + k2 * kLoaders;
            last[k2] = id < kNk * 8 ? codes_at(id / 8, kNb - 1, id % 8) : make_uint2(0u, 0u);
          }
          named_sync(3, kLoaders);  // block 8 overwrites staged blocks 7-8, read by now
#pragma unroll
          for (int k2 = 0; k2 < kLastPer; ++k2) {
            const int id = lt + k2 * kLoaders;
            if (id < kNk * 8) put(id / 8, kNb - 1, id % 8, last[k2]);
          }
          fence_proxy_async_smem();
          named_sync(3, kLoaders);
          if (lt == 0) mbar_arrive(&kfull[st]);
        } else {
          // consecutive threads take consecutive 16-byte chunks of a row (coalesced): chunk c of key
          // kr is 16-byte piece c & 7 of channel block c >> 3; FP8 entries are read as 8 codes and
          // widened, in passes of kPer / 2 chunks to bound the registers they hold
#pragma unroll
          for (int half = 0; half < 2; ++half) {
            uint2 codes8[kPer / 2];
#pragma unroll
            for (int q = 0; q < kPer / 2; ++q) {
              const int id = lt + (half * (kPer / 2) + q) * kLoaders;
              codes8[q] = make_uint2(0u, 0u);
              if (id < kChunks) {
                const int kr = id / (kNb * 8), c = id % (kNb * 8);
                const uint32_t cd = sCode[st * kNk + kr];
                if (fp8 && (cd >> kRowBits) == 1u) {
                  codes8[q] = __ldg(reinterpret_cast<const uint2*>(static_cast<const uint8_t*>(p.kv_pool) +
                                                                   (size_t)(cd & kRowMask) * kDqk + c * 8));
                } else {
                  const uint16_t* src = code_row(p, cd);
                  cp_async16(dst + (c >> 3) * kBlkBytes + kr * 128 + (((c & 7) ^ (kr & 7)) << 4),
                             src ? static_cast<const void*>(src + c * 8) : static_cast<const void*>(p.q),
                             src ? 16 : 0);
                }
              }
            }
            if (fp8) {
#pragma unroll
              for (int q = 0; q < kPer / 2; ++q) {
                const int id = lt + (half * (kPer / 2) + q) * kLoaders;
                if (id < kChunks) {
                  const int kr = id / (kNb * 8), c = id % (kNb * 8);
                  if ((sCode[st * kNk + kr] >> kRowBits) == 1u)
                    *reinterpret_cast<uint4*>(dst + (c >> 3) * kBlkBytes + kr * 128 + (((c & 7) ^ (kr & 7)) << 4)) =
                        e4m3x8_to_bf16x8(codes8[q]);
                }
              }
            }
          }
          cp_async_commit();
          if (it + 1 < ntiles) {  // the next tile's rows are looked up while this tile's copies fly
            ncode = code_of(it + 1, nsc);
            nmode = tile_src(it + 1, nrow0);
            if (nmode < 0) prefetch(ncode);
          }
          cp_async_wait<0>();
          fence_proxy_async_smem();
          named_sync(3, kLoaders);
          if (lt == 0) mbar_arrive(&kfull[st]);
        }
      }
    } else if (warp == 4) {
      // ------------------------------------------------------------ S issue (lane 0; the warp waits together)
      const bool issuer = lane == 0;
      const uint32_t idesc_s = umma_idesc_bf16(kH, kNk, false);
      const uint32_t sQa = smem_u32(sQ), sKa = smem_u32(sK);
      bool ok = __all_sync(kFull, mbar_wait(qbar, n_item & 1u, p.status));
      tc_fence_after();
      for (int it = 0; it < ntiles && ok; ++it) {
        if (__shfl_sync(kFull, *sAbort, 0)) break;
        const uint32_t gt = g + it;
        const int k = gt & 1;
        // the stage is shared memory written by TMA or fenced cp.async / stores: the mbarrier
        // orders it; S buffer k is free once the softmax has read S(gt - 2)
        if (!(ok = __all_sync(kFull, mbar_wait(&kfull[k], (gt >> 1) & 1u, p.status)))) break;
        if (gt >= 2 && !(ok = __all_sync(kFull, mbar_wait(&sfree[k], ((gt >> 1) - 1) & 1u, p.status)))) break;
        tc_fence_after();
        if (issuer) {
          issue_s(tmem + kColS + k * kNk, sQa, sKa + k * kStageBytes, idesc_s);
          umma_commit(&sfull[k]);
        }
        __syncwarp();
      }
      if (!ok && issuer) *sAbort = 1;
      __syncwarp();
    } else if (warp < 4) {
      // ------------------------------------------------------------ softmax
      // thread (warp, lane): head row hr = 16 warp + (lane & 15), keys 32 kh .. + 31 of each tile
      const float sl2 = p.sm_scale * kLog2e;
      const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
      const int hr = warp * 16 + (lane & 15), kh = lane >> 4;
      const uint32_t idesc_pv = umma_idesc_bf16(kH, 256, true);
      const uint32_t sKa = smem_u32(sK), sPa = smem_u32(sP);
      uint8_t* prow = sP + hr * 128;
      float m_used = -INFINITY, l_run = 0.f;
      bool ok = true;
      // Every softmax warp reaches the named barrier of every tile; a failed bounded wait only
      // marks the tile bad, and the barrier's OR over the 128 threads decides for all of them.
      for (int it = 0; it < ntiles && ok; ++it) {
        const uint32_t gt = g + it;
        const int k = gt & 1;
        bool good = __all_sync(kFull, mbar_wait(&sfull[k], (gt >> 1) & 1u, p.status));
        float s[32];
        if (good) {
          tc_fence_after();
          // this lane's accumulator row (all 64 keys); keep my 32 keys, swap the other 32 with lane ^ 16
          uint32_t a[32], o[32];
          tmem_ld32(tmem + lane_base + kColS + k * kNk, a);
          tmem_ld32(tmem + lane_base + kColS + k * kNk + 32, o);
          tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const float mine = __uint_as_float(kh ? o[j] : a[j]);
            const float give = __uint_as_float(kh ? a[j] : o[j]);
            s[j] = mine + __shfl_xor_sync(kFull, give, 16);
          }
        }
        tc_fence_before();
        mbar_arrive(&sfree[k]);
        // the stage's key bits and scales (written before the loaders' kfull arrival; that phase
        // cannot move on before this tile's P V, which waits for this thread's P)
        if (good) good = __all_sync(kFull, mbar_wait(&kfull[k], (gt >> 1) & 1u, p.status));
        bool rescale = false;
        float corr = 1.f;
        uint32_t pp[16];
        if (good) {
          const uint32_t vm = sMask[k * 2 + kh];
          const float* scl = sScale + k * kNk + 32 * kh;
          if (fp8) {  // an FP8 entry's logit and value carry its scale
#pragma unroll
            for (int j = 0; j < 32; ++j) s[j] *= scl[j];
          }
          float m0 = -INFINITY, m1 = -INFINITY, m2 = -INFINITY, m3 = -INFINITY;
#pragma unroll
          for (int j = 0; j < 32; j += 4) {
            s[j] = ((vm >> j) & 1u) ? s[j] * sl2 : -INFINITY;  // keys past nk have no row
            s[j + 1] = ((vm >> (j + 1)) & 1u) ? s[j + 1] * sl2 : -INFINITY;
            s[j + 2] = ((vm >> (j + 2)) & 1u) ? s[j + 2] * sl2 : -INFINITY;
            s[j + 3] = ((vm >> (j + 3)) & 1u) ? s[j + 3] * sl2 : -INFINITY;
            m0 = fmaxf(m0, s[j]);
            m1 = fmaxf(m1, s[j + 1]);
            m2 = fmaxf(m2, s[j + 2]);
            m3 = fmaxf(m3, s[j + 3]);
          }
          float mt = fmaxf(fmaxf(m0, m1), fmaxf(m2, m3));
          mt = fmaxf(mt, __shfl_xor_sync(kFull, mt, 16));  // the row's max over the tile's 64 keys
          if (mt > m_used + kRescaleThreshold || (m_used == -INFINITY && mt != -INFINITY)) {
            corr = exp2f(m_used - mt);  // 0 when m_used is -inf
            rescale = it > 0;
            l_run *= corr;
            m_used = mt;
          }
          const float msub = m_used == -INFINITY ? 0.f : m_used;
          float l0 = 0.f, l1 = 0.f;
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const float e0 = exp2f(s[2 * j] - msub), e1 = exp2f(s[2 * j + 1] - msub);
            l0 += e0;
            l1 += e1;
            pp[j] = fp8 ? pack_bf16(e0 * scl[2 * j], e1 * scl[2 * j + 1]) : pack_bf16(e0, e1);
          }
          l_run += l0 + l1;
          // the P buffer was read by the P V of tile gt - 1, which also finished O
          if (gt >= 1) good = __all_sync(kFull, mbar_wait(obar, (gt - 1) & 1u, p.status));
        }
        if (good) {
          tc_fence_after();
          if (__any_sync(kFull, rescale)) {
            // lanes +0 hold O[:, 0:256], lanes +16 O[:, 256:512] of the same head rows, and both lanes
            // of a row carry the same corr
#pragma unroll 1
            for (int c = 0; c < 256; c += 32) {
              uint32_t orow[32];
              tmem_ld32(tmem + lane_base + kColO + c, orow);
              tmem_ld_wait();
#pragma unroll
              for (int j = 0; j < 32; ++j) orow[j] = __float_as_uint(__uint_as_float(orow[j]) * corr);
              tmem_st32(tmem + lane_base + kColO + c, orow);
            }
            tmem_st_wait();
          }
          // keys 32 kh + 8 i .. + 7: 16-byte chunk 4 kh + i of the row (one 64-key swizzle atom)
#pragma unroll
          for (int i = 0; i < 4; ++i)
            *reinterpret_cast<uint4*>(prow + (((4 * kh + i) ^ (hr & 7)) << 4)) =
                make_uint4(pp[4 * i], pp[4 * i + 1], pp[4 * i + 2], pp[4 * i + 3]);
          fence_proxy_async_smem();
        }
        tc_fence_before();
        // every row's P is in shared memory, or some warp met a wait that gave up (uniform answer)
        if (named_sync_or(1, 128, !good || *sAbort)) {
          *sAbort = 1;
          ok = false;
          break;
        }
        if (tid == 0) {
          tc_fence_after();
          const uint32_t vb = sKa + k * kStageBytes;  // channel blocks 0..7 of the tile: V
#pragma unroll
          for (int ks = 0; ks < kNk / 16; ++ks) {
            const uint64_t pa = umma_desc_sw128(sPa + ks * 32, 16, 1024);
            const uint32_t acc = (it > 0 || ks > 0) ? 1u : 0u;
            umma_ss(tmem + kColO, pa, umma_desc_sw128(vb + ks * 16 * 128, kBlkBytes, 1024), idesc_pv, acc);
            umma_ss(tmem + kColO + kLane16, pa, umma_desc_sw128(vb + 4 * kBlkBytes + ks * 16 * 128, kBlkBytes, 1024),
                    idesc_pv, acc);
          }
          umma_commit(&kempty[k]);
          umma_commit(obar);
        }
      }
      if (tid == 0) umma_commit(dbar);  // one completion per item, also after an abort
      // epilogue: normalised partial output of this split and head group, and its log-sum-exp
      ok = __all_sync(kFull, mbar_wait(dbar, n_item & 1u, p.status)) && ok;
      if (!ok) *sAbort = 1;
      tc_fence_after();
      const float l_row = l_run + __shfl_xor_sync(kFull, l_run, 16);
      const int head = grp * kH + hr;
      const float inv = l_row > 0.f ? 1.f / l_row : 0.f;
      // part_o is head-minor ([query x split][d_v / 4][heads][4]): the 16 lanes of a half-warp
      // write 16 consecutive heads, 256 contiguous bytes
      float4* po = reinterpret_cast<float4*>(p.part_o) +
                   (((int64_t)b * p.max_splits + split) * (kDv / 4) + kh * 64) * p.n_heads + head;
#pragma unroll 1
      for (int c = 0; c < 256; c += 32) {
        uint32_t orow[32];
        if (ok) {  // warp-uniform
          tmem_ld32(tmem + lane_base + kColO + c, orow);
          tmem_ld_wait();
        }
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          const float4 v = ok ? make_float4(__uint_as_float(orow[4 * q]) * inv, __uint_as_float(orow[4 * q + 1]) * inv,
                                            __uint_as_float(orow[4 * q + 2]) * inv, __uint_as_float(orow[4 * q + 3]) * inv)
                              : make_float4(0.f, 0.f, 0.f, 0.f);
          po[(int64_t)(c / 4 + q) * p.n_heads] = v;
        }
      }
      if (kh == 0)
        p.part_lse[((int64_t)b * p.max_splits + split) * p.n_heads + head] =
            l_row > 0.f ? (m_used + log2f(l_row)) * kLn2 : -INFINITY;
    }
    g += ntiles;
    tc_fence_before();
    __syncthreads();  // shared and tensor memory are reused by the next item
    tc_fence_after();
    if (*sAbort) break;
  }
  // after an abort, give tensor-core work in flight a bounded chance to land before freeing
  if (*sAbort && warp == 0) mbar_wait(dbar, n_item & 1u, nullptr);
  cp_async_wait<0>();
  tc_fence_before();
  __syncthreads();
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
  return d_qk == kDqk && d_v == kDv && n_heads % kH == 0 && (kv_dtype == CSKV_BF16 || kv_dtype == CSKV_FP8_E4M3) &&
         Smem::bytes(n_q) + 128 <= 232448;  // the per-query prefix table shares shared memory with the tiles
}

// keys per split: queries x head groups x splits ~ one CTA per SM
void attend_tc_plan(AttendParams& p, int n_sm) {
  const int64_t groups = p.n_heads / kH;
  const int64_t n_max = (int64_t)p.n_win + (p.is_csa ? p.k : visible_entries(p.max_pos, p.m, p.n_win));
  int64_t splits = n_sm / ((int64_t)p.n_q * groups);
  if (splits < 1) splits = 1;
  int64_t kps = (n_max + splits - 1) / splits;
  kps = (kps + kNk - 1) / kNk * kNk;
  if (kps < kNk) kps = kNk;
  // HCA key counts grow with the context (n / 128 + 128): with many queries of mixed lengths one split
  // per query would leave the longest ones on one CTA, so no HCA item takes more than kMaxSplitKeys
  // keys (a CSA query has at most n_win + k keys, all of similar count)
  if (!p.is_csa && kps > kMaxSplitKeys) kps = kMaxSplitKeys;
  p.keys_per_split = static_cast<int>(kps);
  p.max_splits = static_cast<int>((n_max + kps - 1) / kps);
  if (p.max_splits < 1) p.max_splits = 1;
}

cudaError_t launch_attend_tc(AttendParams& p, int n_sm, cudaStream_t st) {
  CUtensorMap tm_q, tm_ring, tm_kv, tm_kvg;
  const uint64_t kv_rows = static_cast<uint64_t>(p.n_pages) * p.page_size;
  const uint64_t ring_rows = static_cast<uint64_t>(p.n_seqs_layer) * p.n_win;
  if (kv_rows > kRowMask || ring_rows > kRowMask || static_cast<uint64_t>(p.chunk_len) > kRowMask)
    return cudaErrorNotSupported;
  if (!encode_rows(&tm_q, p.q, static_cast<uint64_t>(p.n_q) * p.n_heads, kH) ||
      !encode_rows(&tm_ring, p.ring_x, ring_rows, kNk) ||
      // an FP8 pool is never read by TMA (its tiles are widened by the loaders)
      !encode_rows(&tm_kv, p.kv_dtype == CSKV_FP8_E4M3 ? static_cast<const void*>(p.ring_x) : p.kv_pool,
                   p.kv_dtype == CSKV_FP8_E4M3 ? ring_rows : kv_rows, kNk) ||
      // one-row boxes of the bf16 pool for the gathered tiles (the selection's rows)
      !encode_rows(&tm_kvg, p.kv_dtype == CSKV_FP8_E4M3 ? static_cast<const void*>(p.ring_x) : p.kv_pool,
                   p.kv_dtype == CSKV_FP8_E4M3 ? ring_rows : kv_rows, 1))
    return cudaErrorNotSupported;
  const size_t smem = Smem::bytes(p.n_q);
  const bool fp8 = p.kv_dtype == CSKV_FP8_E4M3;
  auto kern = fp8 ? attend_tc_kernel<true> : attend_tc_kernel<false>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  const int64_t items = (int64_t)p.n_q * p.max_splits * (p.n_heads / kH);
  const int grid = static_cast<int>(items < n_sm ? items : n_sm);
  p.part_t = 1;
  e = launch_pdl(kern, dim3(static_cast<unsigned>(grid < 1 ? 1 : grid)), dim3(kThreads), smem, st, tm_q, tm_ring,
                 tm_kv, tm_kvg, p);
  if (e != cudaSuccess) return e;
  return launch_attend_merge(p, st);
}

}  // namespace cskv
