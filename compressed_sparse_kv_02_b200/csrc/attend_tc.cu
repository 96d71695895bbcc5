// attend_tc.cu -- CSA / HCA core attention on the 5th-generation tensor cores
// (tcgen05) for the wide shared latent: d_qk = 576 (512 latent + 64 RoPE
// channels), d_v = 512, query heads in groups of 128 (DeepSeek-V4 report
// digest, section 3: one softmax over the window and the selected / all
// compressed entries; DeepSeek-V4-book ch.1, section 4: the MLA latent shared
// by every head).
//
// With 128 heads on one 576-wide latent every key carries 2 x 128 x 1088
// flops: the product is a real dense contraction, with the heads as M = 128.
// Work item = (query, 128-head group, key split, half of d_v). Per item:
//   - Q [128 heads x 576] sits in shared memory as nine 128-byte-swizzled
//     K-major blocks of 64 channels (one TMA load per block); 32-key tiles of
//     K stream through two swizzled buffers: by TMA when the tile's rows are
//     contiguous (window rows of the ring, HCA entries of one page), by
//     cp.async through a row table otherwise (the CSA selection);
//   - S = Q K^T (M 128, N 32, K 576) lands in tensor memory as three partial
//     sums over 192 channels each, so consecutive MMAs never wait on one
//     accumulator;
//   - four warps take one head row each from S (tcgen05.ld), run the online
//     softmax in fp32 and write P (bf16) back to tensor memory;
//   - O[:, half] += P V (M 128, N 256, K 32) with P as the tensor-memory A
//     operand and V read MN-major from the same K tile (V = the first d_v
//     channels of each key);
//   - O is rescaled only when a row's running max rises by more than 2^8 (the
//     probabilities stay below 256 in bf16), so most tiles skip it.
// Window keys are taken in ring-slot order (the softmax does not depend on the
// order of its keys), which makes a window tile 32 consecutive ring rows.
// The two d_v halves of a (query, split) run in two CTAs that both compute S
// (the accumulator for all 512 output channels would fill the whole tensor
// memory). Each item writes its normalised partial output and log-sum-exp;
// attend_merge_kernel combines the splits.
#include "cskv_device.cuh"
#include "cskv_internal.h"

namespace cskv {
namespace {

constexpr int kDqk = 576, kDv = 512, kM = 128, kNk = 32;
constexpr int kKb = kDqk / 64;                // 64-channel (128-byte) blocks per row
constexpr int kQBytes = kKb * kM * 128;       // 147456
constexpr int kKBytes = kKb * kNk * 128;      // 36864 per key tile
constexpr int kThreads = 256;                 // warps 0-3 softmax, warp 4 MMA, warps 5-7 loads
constexpr int kMmaThread = 128;
constexpr int kLoadThread0 = 160;
constexpr int kLoaders = kThreads - kLoadThread0;  // 96
constexpr int kRowCap = 1024;                 // keys per work item (row table in shared memory)
constexpr int kSAcc = 3;                      // partial sums of S (K = 3 x 192)
constexpr uint32_t kTmemCols = 512;
// O 256 | S 2 buffers x 3 partials x 32 | P 2 buffers x 16 (bf16 pairs)
constexpr uint32_t kColO = 0, kColS = 256, kColP = 256 + 2 * kSAcc * kNk;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kRescaleThreshold = 8.0f;     // log2 units
constexpr int kPrefetchTiles = 6;             // L2 prefetch distance of gathered key rows
static_assert(kColP + 32 <= kTmemCols, "tensor memory budget");

struct Smem {
  static constexpr int Q = 0;
  static constexpr int K = kQBytes;                  // two tile buffers (also the epilogue staging)
  static constexpr int BAR = K + 2 * kKBytes;        // mbarriers
  static constexpr int MASK = BAR + 128;             // valid-key bits, one word per tile
  static constexpr int ROWS = MASK + kRowCap / 8;    // source row of every key of the item
  static constexpr int TMEM = ROWS + kRowCap * 8;    // allocated tensor-memory address
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
// supplies some of them; then the compressed entries. Null if invalid.
__device__ __forceinline__ const uint16_t* key_src(const AttendParams& p, int b, int seq, const Keys& k,
                                                   int64_t u) {
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
  return static_cast<const uint16_t*>(p.kv_pool) + ((int64_t)page * p.page_size + j % p.page_size) * kDqk;
}

// byte offset of 16-byte chunk `ch` (0..71) of row `r` in a swizzled block set
// whose 64-channel blocks are `block_bytes` apart
__device__ __forceinline__ uint32_t swz(int r, int ch, int block_bytes) {
  return (ch >> 3) * block_bytes + r * 128 + (((ch & 7) ^ (r & 7)) << 4);
}

__device__ __forceinline__ void named_sync(int id, int n) {
  asm volatile("bar.sync %0, %1;\n" ::"r"(id), "r"(n) : "memory");
}

// Pipeline (per CTA, tiles numbered gt across its items; buffer gt & 1):
//   loaders  : wait kempty[buf] (P V of tile gt-2 done) -> TMA, or cp.async +
//              proxy fence, into buf -> kfull[buf]
//   MMA      : wait kfull -> S(gt) = Q K^T into S[buf] -> commit sfull[buf];
//              then wait pfull of tile gt-1 -> O += P V -> commit kempty, obar
//   softmax  : wait sfull[buf] -> S row -> P row into P[buf] (+ rare O rescale
//              after obar of tile gt-1) -> arrive pfull[buf]
// S(gt) is issued before P V (gt-1), so the tensor core overlaps the softmax.
__global__ void __launch_bounds__(kThreads, 1)
    attend_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_ring,
                     const __grid_constant__ CUtensorMap tm_kv, AttendParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = sm + Smem::Q;
  uint8_t* sK = sm + Smem::K;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + Smem::BAR);
  uint64_t* kfull = bars;       // [2] loaders -> MMA
  uint64_t* kempty = bars + 2;  // [2] MMA -> loaders (commit)
  uint64_t* sfull = bars + 4;   // [2] MMA -> softmax (commit)
  uint64_t* pfull = bars + 6;   // [2] softmax -> MMA (128 arrivals)
  uint64_t* obar = bars + 8;    //     MMA -> softmax (commit after each P V)
  uint64_t* qbar = bars + 9;    //     Q landed (TMA)
  uint64_t* dbar = bars + 10;   //     MMA -> epilogue (commit after the item's last P V)
  uint32_t* sMask = reinterpret_cast<uint32_t*>(sm + Smem::MASK);
  const uint16_t** sRow = reinterpret_cast<const uint16_t**>(sm + Smem::ROWS);
  uint32_t* sTmem = reinterpret_cast<uint32_t*>(sm + Smem::TMEM);
  int* sAbort = reinterpret_cast<int*>(sm + Smem::FLAGS);
  volatile int* sLdOk = reinterpret_cast<int*>(sm + Smem::FLAGS) + 1;  // [2], loader wait results
  int* sPref = reinterpret_cast<int*>(sm + Smem::PREF);
  __shared__ int s_wsum[32];

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int groups = p.n_heads / kM;
  const int kps = p.keys_per_split;

  {  // items per query: splits x head groups x 2 halves of d_v
    int run = 0;
    for (int base = 0; base < p.n_q; base += kThreads) {
      const int b = base + tid;
      int v = 0;
      if (b < p.n_q) {
        const Keys k = keys_of(p, b);
        v = static_cast<int>((k.n + kps - 1) / kps) * groups * 2;
      }
      int tot;
      const int ex = block_exclusive_scan<kThreads>(v, s_wsum, tot);
      if (b < p.n_q) sPref[b] = run + ex;
      run += tot;
    }
    if (tid == 0) sPref[p.n_q] = run;
  }
  if (tid == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&kfull[i], 1);
      mbar_init(&kempty[i], 1);
      mbar_init(&sfull[i], 1);
      mbar_init(&pfull[i], kM);
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
  }
  if (warp == 4) {
    tmem_alloc(sTmem, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *sTmem;
  if (blockIdx.x == 0)
    for (int b = tid; b < p.n_q; b += kThreads)
      if (p.q_pos[b] < 0 || p.q_pos[b] > p.max_pos) report(p.status, CSKV_ERR_INVALID_ARG);
  const int total = sPref[p.n_q];
  uint32_t g = 0;       // tiles processed by this CTA before the current item
  uint32_t n_item = 0;  // items processed by this CTA before the current one (qbar phase)

  for (int item = blockIdx.x; item < total; item += gridDim.x, ++n_item) {
    int lo = 0, hi = p.n_q - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (sPref[mid] <= item) lo = mid; else hi = mid - 1;
    }
    const int b = lo;
    const int r = item - sPref[b];
    const int vh = r & 1;
    const int grp = (r >> 1) % groups;
    const int split = (r >> 1) / groups;
    const Keys kk = keys_of(p, b);
    const int seq = p.q_seq[b];
    const bool seq_ok = seq >= 0 && seq < p.n_seqs_layer;
    const int64_t u0 = (int64_t)split * kps;
    const int nk = static_cast<int>(kk.n - u0 < kps ? kk.n - u0 : kps);
    const int ntiles = (nk + kNk - 1) / kNk;

    // source rows of this item's keys and one valid-bit word per tile, visible
    // to every role after the barrier; four independent lookups per thread
    for (int i0 = 0; i0 < ntiles * kNk; i0 += 4 * kThreads) {
      const uint16_t* src[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int i = i0 + q * kThreads + tid;
        src[q] = (i < nk && seq_ok) ? key_src(p, b, seq, kk, u0 + i) : nullptr;
      }
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int i = i0 + q * kThreads + tid;
        if (i < nk) {
          if (!src[q]) report(p.status, CSKV_ERR_OUT_OF_RANGE);
          sRow[i] = src[q];
        }
        const unsigned bits = __ballot_sync(kFull, src[q] != nullptr);
        if (lane == 0 && i < ntiles * kNk) sMask[i >> 5] = bits;
      }
    }
    __syncthreads();

    if (tid >= kLoadThread0) {
      // ------------------------------------------------------------ loaders
      const int lt = tid - kLoadThread0;
      if (lt == 0) {  // Q of this head group: nine 128-row TMA boxes
        mbar_arrive_expect_tx(qbar, kQBytes);
        const int qrow = b * p.n_heads + grp * kM;
        for (int kb = 0; kb < kKb; ++kb) tma_load_2d(sQ + kb * (kM * 128), &tm_q, kb * 64, qrow, qbar);
      }
      // TMA source of tile it: 0 = ring rows, 1 = pool rows, -1 = gathered (cp.async)
      auto tile_src = [&](int it, int& row0) -> int {
        const int64_t a = u0 + (int64_t)it * kNk;
        if (!seq_ok) return -1;
        if (!p.x_chunk && a + kNk <= kk.n_w) {
          row0 = static_cast<int>((int64_t)seq * p.n_win + a);
          return 0;
        }
        if (!p.is_csa && a >= kk.n_w) {
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
          if (i < nk && sRow[i]) prefetch_l2(sRow[i], kDqk * 2);
        }
      };
      for (int it = 0; it < kPrefetchTiles; ++it) prefetch_tile(it);
      for (int it = 0; it < ntiles; ++it) {
        const uint32_t gt = g + it;
        const int buf = gt & 1;
        prefetch_tile(it + kPrefetchTiles);
        // one thread waits and the loaders agree on its result, so no loader can
        // leave the loop while another waits at a named barrier below
        if (lt == 0) sLdOk[it & 1] = gt < 2 || mbar_wait(&kempty[buf], ((gt >> 1) - 1) & 1u, p.status);
        named_sync(3, kLoaders);
        if (!sLdOk[it & 1]) { *sAbort = 1; break; }
        uint8_t* dst = sK + buf * kKBytes;
        int row0 = 0;
        const int mode = tile_src(it, row0);
        if (mode >= 0) {
          if (lt == 0) {
            mbar_arrive_expect_tx(&kfull[buf], kKBytes);
            const CUtensorMap* map = mode == 0 ? &tm_ring : &tm_kv;
            for (int kb = 0; kb < kKb; ++kb) tma_load_2d(dst + kb * (kNk * 128), map, kb * 64, row0, &kfull[buf]);
          }
        } else {
          // consecutive threads take consecutive 16-byte chunks of a row (coalesced)
#pragma unroll 4
          for (int id = lt; id < kNk * 72; id += kLoaders) {
            const int kr = id / 72, c = id % 72;
            const int i = it * kNk + kr;
            const uint16_t* src = i < nk ? sRow[i] : nullptr;
            cp_async16(dst + swz(kr, c, kNk * 128), src ? static_cast<const void*>(src + c * 8) : p.q,
                       src ? 16 : 0);
          }
          cp_async_commit();
          cp_async_wait<0>();
          fence_proxy_async_smem();
          named_sync(3, kLoaders);
          if (lt == 0) mbar_arrive(&kfull[buf]);
        }
      }
    } else if (tid == kMmaThread) {
      // ------------------------------------------------------------ MMA issue
      const uint32_t idesc_s = umma_idesc_bf16(kM, kNk, false);
      const uint32_t idesc_pv = umma_idesc_bf16(kM, 256, true);
      const uint32_t sQa = smem_u32(sQ), sKa = smem_u32(sK);
      bool ok = mbar_wait(qbar, n_item & 1u, p.status);
      for (int it = 0; it <= ntiles && ok; ++it) {
        if (it < ntiles) {
          const uint32_t gt = g + it;
          const int buf = gt & 1;
          if (!(ok = mbar_wait(&kfull[buf], (gt >> 1) & 1u, p.status))) break;
          tc_fence_after();
          const uint32_t kb_base = sKa + buf * kKBytes;
          const uint32_t d = tmem + kColS + buf * (kSAcc * kNk);
          // 36 MMAs (9 blocks x 4 k-steps), round-robin over three accumulators
#pragma unroll 1
          for (int kb3 = 0; kb3 < kKb / kSAcc; ++kb3) {
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) {
#pragma unroll
              for (int a = 0; a < kSAcc; ++a) {
                const int kb = a * (kKb / kSAcc) + kb3;
                const uint64_t da = umma_desc_sw128(sQa + kb * (kM * 128) + ks * 32, 16, 1024);
                const uint64_t db = umma_desc_sw128(kb_base + kb * (kNk * 128) + ks * 32, 16, 1024);
                umma_ss(d + a * kNk, da, db, idesc_s, (kb3 | ks) != 0);
              }
            }
          }
          umma_commit(&sfull[buf]);
        }
        if (it >= 1) {
          const uint32_t gp = g + it - 1;
          const int pb = gp & 1;
          if (!(ok = mbar_wait(&pfull[pb], (gp >> 1) & 1u, p.status))) break;
          tc_fence_after();
          const uint32_t v_base = sKa + pb * kKBytes + vh * 4 * (kNk * 128);
#pragma unroll
          for (int k2 = 0; k2 < 2; ++k2) {
            const uint64_t db = umma_desc_sw128(v_base + k2 * 16 * 128, kNk * 128, 1024);
            umma_ts(tmem + kColO, tmem + kColP + pb * 16 + k2 * 8, db, idesc_pv, (it > 1 || k2 > 0) ? 1u : 0u);
          }
          umma_commit(&kempty[pb]);
          umma_commit(obar);
        }
      }
      umma_commit(dbar);  // one completion per item, also after an abort
      if (!ok) *sAbort = 1;
    } else if (warp < 4) {
      // ------------------------------------------------------------ softmax (one head row per thread)
      const float sl2 = p.sm_scale * kLog2e;
      const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
      float m_used = -INFINITY, l_run = 0.f;
      bool ok = true;
      for (int it = 0; it < ntiles && ok; ++it) {
        const uint32_t gt = g + it;
        const int buf = gt & 1;
        // warp-uniform results keep the warp-wide votes below well defined
        ok = __all_sync(kFull, mbar_wait(&sfull[buf], (gt >> 1) & 1u, p.status));
        if (!ok) break;
        tc_fence_after();
        uint32_t s0[32], s1[32], s2[32];
        const uint32_t sbase = tmem + lane_base + kColS + buf * (kSAcc * kNk);
        tmem_ld32(sbase, s0);
        tmem_ld32(sbase + kNk, s1);
        tmem_ld32(sbase + 2 * kNk, s2);
        tmem_ld_wait();
        const uint32_t valid = sMask[it];
        float v[32];
        float mt = -INFINITY;
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          const float sv = __uint_as_float(s0[j]) + __uint_as_float(s1[j]) + __uint_as_float(s2[j]);
          v[j] = ((valid >> j) & 1u) ? sv * sl2 : -INFINITY;  // keys past nk have no row
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
          pp[j] = pack_bf16(p0, p1);
        }
        if (__any_sync(kFull, rescale)) {
          // O is being accumulated by P V of tile gt-1: rescale after it lands
          // completions of obar so far: gt-1 or gt (P V of tile gt needs this warp's arrival)
          ok = __all_sync(kFull, mbar_wait(obar, (gt - 1) & 1u, p.status));
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
      // staged through the (now idle) key buffers: each thread parks 32 values of its
      // row, then each warp stores 32 whole rows of 128 bytes
      float* stage = reinterpret_cast<float*>(sK);  // [128 rows][33]
#pragma unroll 1
      for (int c = 0; c < 256; c += 32) {
        uint32_t orow[32];
        if (ok) {
          tmem_ld32(tmem + lane_base + kColO + c, orow);
          tmem_ld_wait();
        }
#pragma unroll
        for (int j = 0; j < 32; ++j) stage[tid * 33 + j] = ok ? __uint_as_float(orow[j]) * inv : 0.f;
        named_sync(2, kM);
        for (int rr = 0; rr < 32; ++rr) {
          const int row = warp * 32 + rr;
          p.part_o[(prow0 + row) * kDv + vh * 256 + c + lane] = stage[row * 33 + lane];
        }
        named_sync(2, kM);
      }
      if (vh == 0) p.part_lse[prow0 + tid] = l_run > 0.f ? (m_used + log2f(l_run)) * kLn2 : -INFINITY;
    }
    g += ntiles;
    tc_fence_before();
    __syncthreads();  // shared and tensor memory are reused by the next item
    tc_fence_after();
    if (*sAbort) break;
  }
  // after an abort, give tensor-core work in flight a bounded chance to land before freeing
  if (*sAbort && tid == kMmaThread) mbar_wait(dbar, n_item & 1u, nullptr);
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
  return d_qk == kDqk && d_v == kDv && n_heads % kM == 0 && kv_dtype == CSKV_BF16 &&
         Smem::bytes(n_q) <= 232448;  // the per-query prefix table shares shared memory with the tiles
}

// keys per split: queries x head groups x splits x 2 halves ~ one CTA per SM
void attend_tc_plan(AttendParams& p, int n_sm) {
  const int64_t groups = p.n_heads / kM;
  const int64_t n_max = (int64_t)p.n_win + (p.is_csa ? p.k : visible_entries(p.max_pos, p.m, p.n_win));
  int64_t splits = n_sm / ((int64_t)p.n_q * groups * 2);
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
      !encode_rows(&tm_ring, p.ring_x, ring_rows, kNk) || !encode_rows(&tm_kv, p.kv_pool, kv_rows, kNk))
    return cudaErrorNotSupported;
  const size_t smem = Smem::bytes(p.n_q);
  cudaError_t e = cudaFuncSetAttribute(attend_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  const int64_t upper = (int64_t)p.n_q * p.max_splits * (p.n_heads / kM) * 2;
  int64_t grid = upper < n_sm ? upper : n_sm;
  if (grid < 1) grid = 1;
  attend_tc_kernel<<<static_cast<int>(grid), kThreads, smem, st>>>(tm_q, tm_ring, tm_kv, p);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  return launch_attend_merge(p, st);
}

}  // namespace cskv
