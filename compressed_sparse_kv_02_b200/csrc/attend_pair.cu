// attend_pair.cu -- CSA / HCA core attention on the tensor cores (tcgen05) for
// calls with many queries on the narrow latent: d_qk = d_v = 128, 64 query
// heads (DeepSeek-V4 report digest, section 3: one softmax over the window and
// the selected / all compressed entries; DeepSeek-V4-book ch.1, section 4: every
// head reads the one shared latent row).
//
// A prefill block holds thousands of query positions, so no key split is
// needed: a work item is a PAIR of queries (2i, 2i + 1), each with its own key
// list (window rows, then its selection or every visible entry), run to the end
// by one CTA, which writes the normalised bf16 output itself (no merge pass).
// The 64 heads of one query are an M = 64 tcgen05 tile; the accumulator of such
// a tile fills lanes 0-15 of each 32-lane quarter of tensor memory, and the
// second query's tile sits at lane offset 16, so the two queries' S (and O)
// share the 128 lanes and one softmax warpgroup serves both: thread (warp w,
// lane l) owns head 16 w + (l & 15) of query l >> 4.
//   loaders (warps 5-8): per tile, the source rows of 64 keys of each query,
//     then cp.async of the 2 x 64 rows (16 threads per 256-byte row) into a
//     128-byte-swizzled stage (four stages: the loaders run up to three tiles
//     ahead, so the hand-offs of consecutive tiles overlap); Q of the pair by TMA;
//   MMA (warp 4, lane 0 issues): S(t) = Q K^T (2 x 8 MMAs, M = 64, N = 64, K = 16)
//     into S buffer t & 1; then O += P(t - 1) V (2 x 4 MMAs, N = d_v = 128, V read
//     MN-major from the same stage: V is the first d_v channels of each key);
//   softmax (warps 0-3): max pass over S(t) in tensor memory, lazy O rescale,
//     exp pass writing bf16 P(t) into shared buffer t & 1 (the A operand).
// O is rescaled only when a row's running max rises by more than 2^8, so most
// tiles skip it (the probabilities stay below 256 in bf16).
//
// Shared memory (1024-aligned): Q 32 KB | key stages 4 x 32 KB | P 2 x 16 KB |
// source-row codes | barriers | valid-key bits. Tensor memory: O 128 | S 2 x 64
// columns. A key without a valid source row (an index outside the
// visible entries) is masked out of the softmax and reported.
#include "cskv_device.cuh"
#include "cskv_internal.h"

namespace cskv {
namespace {

constexpr int kD = 128;             // d_qk = d_v
constexpr int kH = 64;              // heads of one query (the M of its tile)
constexpr int kNk = 64;             // keys per tile and query
constexpr int kNS = 4;              // key stages: the loaders run up to three tiles ahead
constexpr int kSlotBytes = kNk * kD * 2;        // 16384: one query's key tile (two 64-channel halves)
constexpr int kHalfBytes = kNk * 128;           // 8192: one 64-channel half of it
constexpr int kStageBytes = 2 * kSlotBytes;     // 32768
constexpr int kQBytes = 2 * kH * kD * 2;        // 32768: Q of both queries
constexpr int kPBytes = 2 * kH * kNk * 2;       // 16384: P of both queries (one buffer)
constexpr int kRows = 2 * kNk;                  // key rows of a tile (both queries)
constexpr int kThreads = 288;       // warps 0-3 softmax, warp 4 MMA, warps 5-8 loads
constexpr int kLoadThread0 = 160;
constexpr int kLoaders = kThreads - kLoadThread0;  // 128
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColO = 0, kColS = 128;       // O | S buffer 0 | S buffer 1 (64 columns each)
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kRescaleThreshold = 8.0f;        // log2 units

struct Smem {
  static constexpr int Q = 0;
  static constexpr int K = Q + kQBytes;
  static constexpr int P = K + kNS * kStageBytes;
  static constexpr int ROWS = P + 2 * kPBytes;    // source-row codes of the tile being issued
  static constexpr int BAR = ROWS + kRows * 4;
  static constexpr int TMEM = BAR + (2 * kNS + 9) * 8;
  static constexpr int FLAGS = TMEM + 4;
  static constexpr int MASK = FLAGS + 8;          // valid-key bits: [stage][query][2 words]
  static constexpr int END = MASK + kNS * 2 * 2 * 4;
  static constexpr size_t bytes() { return 1024 + END; }
};
static_assert(Smem::bytes() <= 232448, "shared memory budget");

// source-row code: kind in bits [31:30] (0 none, 1 pool entry, 2 ring row, 3 chunk row), row below
constexpr uint32_t kRowBits = 30;
constexpr uint32_t kRowMask = (1u << kRowBits) - 1u;

struct Keys {
  int64_t t, ws;
  int n_w;
  int n;  // window + compressed keys (0 for an invalid position)
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
  r.n = static_cast<int>(r.n_w + n_c);
  return r;
}

// Code of the source row of key u (< k.n) of query b: window keys first (ring-slot order when
// every window row is in the ring, position order when a prefill chunk supplies some), then the
// compressed entries. 0 if the row is invalid.
__device__ __forceinline__ uint32_t key_code(const AttendParams& p, int b, int seq, const Keys& k, int u) {
  if (u < k.n_w) {
    if (!p.x_chunk) return (2u << kRowBits) | static_cast<uint32_t>(seq * p.n_win + u);
    const int64_t pos = k.ws + u;
    const int64_t cr = chunk_row(p, seq, pos);
    if (cr >= 0) return (3u << kRowBits) | static_cast<uint32_t>(cr);
    return (2u << kRowBits) | static_cast<uint32_t>(seq * p.n_win + pos % p.n_win);
  }
  const int jj = u - k.n_w;
  const int64_t j = p.is_csa ? static_cast<int64_t>(p.sel_idx[(int64_t)b * p.k + jj]) : jj;
  if (j < 0 || j >= visible_entries(k.t, p.m, p.n_win)) return 0;
  const int64_t pi = j / p.page_size;
  if (pi >= p.max_pages_per_seq) return 0;
  const int32_t page = p.page_table[(int64_t)seq * p.max_pages_per_seq + pi];
  if (page < 0 || page >= p.n_pages) return 0;
  return (1u << kRowBits) | static_cast<uint32_t>((int64_t)page * p.page_size + j % p.page_size);
}

__device__ __forceinline__ const uint16_t* code_row(const AttendParams& p, uint32_t c) {
  const uint32_t kind = c >> kRowBits, row = c & kRowMask;
  if (kind == 1) return static_cast<const uint16_t*>(p.kv_pool) + (size_t)row * kD;
  if (kind == 2) return p.ring_x + (size_t)row * kD;
  if (kind == 3) return p.x_chunk + (size_t)row * kD;
  return nullptr;
}

__device__ __forceinline__ void named_sync(int id, int n) {
  asm volatile("bar.sync %0, %1;\n" ::"r"(id), "r"(n) : "memory");
}

// S of one query: 8 MMAs (K = 16 channels each) over the two 64-channel halves (N = 64 keys)
__device__ __forceinline__ void issue_s(uint32_t d, uint32_t q, uint32_t k, uint32_t idesc) {
#pragma unroll
  for (int ks = 0; ks < 8; ++ks) {
    const uint32_t off = (ks & 3) * 32u;
    umma_ss(d, umma_desc_sw128(q + (ks >> 2) * (kH * 128) + off, 16, 1024),
            umma_desc_sw128(k + (ks >> 2) * kHalfBytes + off, 16, 1024), idesc, ks > 0 ? 1u : 0u);
  }
}
// O += P V of one query: 4 MMAs (K = 16 keys each; P is one 64-key swizzle atom); V MN-major
// (its two 64-channel halves kHalfBytes apart, 8-key groups 1024 bytes apart)
__device__ __forceinline__ void issue_pv(uint32_t d, uint32_t pm, uint32_t v, uint32_t idesc, bool acc) {
#pragma unroll
  for (int ks = 0; ks < 4; ++ks)
    umma_ss(d, umma_desc_sw128(pm + ks * 32, 16, 1024),
            umma_desc_sw128(v + ks * 16 * 128, kHalfBytes, 1024), idesc, (acc || ks > 0) ? 1u : 0u);
}

// Pipeline (tiles numbered gt across the CTA's items; stage gt % 4, S buffer gt & 1,
// P buffer gt & 1):
//   loaders : wait kempty[stage] (P V of tile gt - 4 done) -> cp.async -> kfull[stage]
//   MMA     : wait kfull -> S(gt) -> commit sfull[gt & 1] (and qempty after an item's last S);
//             wait pfull[(gt - 1) & 1] -> P V(gt - 1) -> commit kempty, obar[(gt - 1) & 1]
//   softmax : wait sfull, kfull (valid-key bits) -> row max -> wait obar (P V of tile gt - 2
//             done: P buffer free)
//             -> rescale O if needed (after P V of gt - 1) -> P(gt) -> arrive pfull
__global__ void __launch_bounds__(kThreads, 1)
    attend_pair_kernel(const __grid_constant__ CUtensorMap tm_q, AttendParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = sm + Smem::Q;
  uint8_t* sK = sm + Smem::K;
  uint8_t* sP = sm + Smem::P;
  uint32_t* sRow = reinterpret_cast<uint32_t*>(sm + Smem::ROWS);
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + Smem::BAR);
  uint64_t* kfull = bars;               // [kNS] loaders -> MMA and softmax
  uint64_t* kempty = bars + kNS;        // [kNS] MMA -> loaders (commit after the tile's P V)
  uint64_t* sfull = bars + 2 * kNS;     // [2] MMA -> softmax
  uint64_t* pfull = sfull + 2;          // [2] softmax -> MMA (128 arrivals)
  uint64_t* obar = pfull + 2;           // [2] MMA -> softmax (P V of that P buffer done)
  uint64_t* qfull = obar + 2;           //     Q of the item landed (TMA)
  uint64_t* qempty = qfull + 1;         //     the item's S products are done with Q
  uint64_t* dbar = qempty + 1;          //     the item's last P V is done
  uint32_t* sTmem = reinterpret_cast<uint32_t*>(sm + Smem::TMEM);
  volatile int* sAbort = reinterpret_cast<int*>(sm + Smem::FLAGS);
  volatile int* sLdOk = sAbort + 1;
  uint32_t* sMask = reinterpret_cast<uint32_t*>(sm + Smem::MASK);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) {
    for (int i = 0; i < kNS; ++i) {
      mbar_init(&kfull[i], 1);
      mbar_init(&kempty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&sfull[i], 1);
      mbar_init(&pfull[i], 128);
      mbar_init(&obar[i], 1);
    }
    mbar_init(qfull, 1);
    mbar_init(qempty, 1);
    mbar_init(dbar, 1);
    fence_barrier_init();
    *sAbort = 0;
  }
  if (tid == kLoadThread0) prefetch_tensormap(&tm_q);
  if (warp == 4) {
    tmem_alloc(sTmem, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *sTmem;
  // the set-up above overlaps the tail of the kernel ahead of this one; its outputs
  // (the selection, new cache rows) are read only from here on
  grid_dependency_wait();
  grid_dependents_launch();
  if (blockIdx.x == 0)
    for (int b = tid; b < p.n_q; b += kThreads)
      if (p.q_pos[b] < 0 || p.q_pos[b] > p.max_pos) report(p.status, CSKV_ERR_INVALID_ARG);

  const int n_items = (p.n_q + 1) >> 1;
  uint32_t g = 0;       // tiles of this CTA before the current item
  uint32_t n_item = 0;  // items of this CTA before the current one
  for (int item = blockIdx.x; item < n_items && !*sAbort; item += gridDim.x, ++n_item) {
    const int b0 = 2 * item, b1 = b0 + 1 < p.n_q ? b0 + 1 : -1;
    const Keys k0 = keys_of(p, b0);
    Keys k1;
    k1.n = 0;
    k1.n_w = 0;
    k1.t = 0;
    k1.ws = 0;
    if (b1 >= 0) k1 = keys_of(p, b1);
    const int s0 = p.q_seq[b0], s1 = b1 >= 0 ? p.q_seq[b1] : 0;
    const bool ok0 = s0 >= 0 && s0 < p.n_seqs_layer, ok1 = b1 >= 0 && s1 >= 0 && s1 < p.n_seqs_layer;
    const int n0 = ok0 ? k0.n : 0, n1 = ok1 ? k1.n : 0;
    // a sequence id outside the layer: the query's keys are all masked (zero output), as in the
    // other attention kernels, and the status word says why
    if (tid == 0 && ((!ok0 && k0.n > 0) || (b1 >= 0 && !ok1 && k1.n > 0))) report(p.status, CSKV_ERR_OUT_OF_RANGE);
    // HCA rows of a prefill chunk: consecutive positions t, t + 1 of one sequence see the same
    // entries up to the last one of t + 1 and windows that differ by one row, so the pair shares
    // one key list (window rows ws(t) .. t + 1, then the entries of t + 1) and every tile is loaded
    // once for both; the valid-key bits tell each query which of the keys it sees.
    const bool shared = !p.is_csa && p.x_chunk && ok0 && ok1 && s0 == s1 && k0.n > 0 && k1.n > 0 &&
                        k1.t == k0.t + 1;
    Keys ksh;  // the shared list (window start of t, last position t + 1)
    ksh.t = k1.t;
    ksh.ws = k0.ws;
    ksh.n_w = static_cast<int>(k1.t - k0.ws + 1);
    ksh.n = ksh.n_w + (k1.n - k1.n_w);
    const int nmax = shared ? ksh.n : (n0 > n1 ? n0 : n1);
    const int ntiles = (nmax + kNk - 1) / kNk;

    if (tid >= kLoadThread0) {
      // ---------------------------------------------------------------- loaders
      const int lt = tid - kLoadThread0, lw = lt >> 5, ll = lt & 31;
      // The first loader warp takes the loaders' waits together (no lane of it waits on an
      // mbarrier while the others sit at a barrier); lane 0 issues.
      if (lw == 0) {  // Q of both queries once the last item's S products are done with the buffer
        const bool okq = __all_sync(kFull, n_item == 0 || mbar_wait(qempty, (n_item - 1) & 1u, p.status));
        if (ll == 0) {
          if (okq) {
            mbar_arrive_expect_tx(qfull, kQBytes);
            const int qb1 = b1 >= 0 ? b1 : b0;  // a lone last query: its slot repeats it (never read out)
            for (int h = 0; h < 2; ++h) {
              tma_load_2d(sQ + h * (kH * 128), &tm_q, h * 64, b0 * kH, qfull);
              tma_load_2d(sQ + kQBytes / 2 + h * (kH * 128), &tm_q, h * 64, qb1 * kH, qfull);
            }
          } else {
            *sAbort = 1;
          }
        }
        __syncwarp();
      }
      // this thread's part of every tile: the source row of key (lt & 63) of query lt >> 6, and
      // chunk (lt & 15) of rows (lt >> 4) + 8 q. A tile is signalled as soon as its copy has
      // landed; the next tile's source rows are looked up after that, while the loaders wait
      // for its stage.
      const int chunk = lt & 15, half = chunk >> 3, c8 = chunk & 7;
      const int my_slot = lt >> 6, my_key = lt & (kNk - 1);
      auto code_of = [&](int it) -> uint32_t {
        uint32_t c = 0;
        if (shared) {  // threads 0 .. kNk - 1: key lt of the shared list
          const int u = it * kNk + lt;
          if (lt < kNk && u < ksh.n) {
            c = key_code(p, b1, s1, ksh, u);
            if (!c) report(p.status, CSKV_ERR_OUT_OF_RANGE);
          }
          return c;
        }
        const int u = it * kNk + my_key;
        if (u < (my_slot ? n1 : n0)) {
          c = my_slot ? key_code(p, b1, s1, k1, u) : key_code(p, b0, s0, k0, u);
          if (!c) report(p.status, CSKV_ERR_OUT_OF_RANGE);
        }
        return c;
      };
      uint32_t nc = ntiles > 0 ? code_of(0) : 0u;
      for (int it = 0; it < ntiles; ++it) {
        const uint32_t gt = g + it;
        const int st = gt % kNS;
        const uint32_t c = nc;
        if (lw == 0) {
          bool okw = __shfl_sync(kFull, *sAbort, 0) == 0;
          if (okw && gt >= (uint32_t)kNS)
            okw = __all_sync(kFull, mbar_wait(&kempty[st], ((gt / kNS) - 1) & 1u, p.status));
          if (ll == 0) *sLdOk = okw;
        }
        named_sync(3, kLoaders);  // sLdOk is set (and the last tile's issue has read sRow)
        if (!*sLdOk) {
          *sAbort = 1;
          break;
        }
        sRow[lt] = c;
        if (shared) {  // loader warps 0 and 1 hold keys 32 w .. + 31 of the shared list
          const int u = it * kNk + lt;
          const bool win = u < ksh.n_w;
          // t sees the window rows up to t (all but the last) and its own entries; t + 1 the rows
          // from its window start and every entry of the list
          const bool v0 = c != 0 && (win ? u < ksh.n_w - 1 : u - ksh.n_w < k0.n - k0.n_w);
          const bool v1 = c != 0 && (!win || k0.ws + u >= k1.ws);
          const unsigned m0 = __ballot_sync(kFull, v0), m1 = __ballot_sync(kFull, v1);
          if (ll == 0 && lw < 2) {
            sMask[st * 4 + lw] = m0;
            sMask[st * 4 + 2 + lw] = m1;
          }
        } else {  // valid-key bits of the tile (the softmax reads them after kfull[st]): warp w of
                  // the loaders holds keys 32 (w & 1) .. + 31 of query w >> 1
          const unsigned mw = __ballot_sync(kFull, c != 0);
          if ((lt & 31) == 0) sMask[st * 4 + (lt >> 5)] = mw;
        }
        named_sync(3, kLoaders);
        uint8_t* dst = sK + st * kStageBytes + half * kHalfBytes;
        const int n_q8 = shared ? kNk / 8 : kRows / 8;  // 8-row steps: one list or two
#pragma unroll 4
        for (int q = 0; q < n_q8; ++q) {
          const int row = (lt >> 4) + 8 * q;  // query row / kNk, key row % kNk
          const int key = row & (kNk - 1);
          const uint16_t* src = code_row(p, sRow[row]);
          cp_async16(dst + (row / kNk) * kSlotBytes + key * 128 + ((c8 ^ (key & 7)) << 4),
                     src ? static_cast<const void*>(src + half * 64 + c8 * 8) : static_cast<const void*>(p.q),
                     src ? 16 : 0);
        }
        cp_async_commit();
        cp_async_wait<0>();
        fence_proxy_async_smem();
        named_sync(3, kLoaders);
        if (lt == 0) mbar_arrive(&kfull[st]);
        if (it + 1 < ntiles) nc = code_of(it + 1);
      }
    } else if (warp == 4) {
      // ---------------------------------------------------------------- MMA issue
      // The whole warp takes every wait (it never diverges around a barrier); lane 0 issues the
      // MMAs and their commits.
      const bool issuer = lane == 0;
      const uint32_t idesc_s = umma_idesc_bf16(kH, kNk, false);
      const uint32_t idesc_pv = umma_idesc_bf16(kH, kD, true);
      const uint32_t sQa = smem_u32(sQ), sKa = smem_u32(sK), sPa = smem_u32(sP);
      bool ok = __all_sync(kFull, mbar_wait(qfull, n_item & 1u, p.status));
      tc_fence_after();
      for (int it = 0; it <= ntiles && ok; ++it) {
        if (__shfl_sync(kFull, *sAbort, 0)) break;
        if (it < ntiles) {
          const uint32_t gt = g + it;
          const int st = gt % kNS;
          if (!(ok = __all_sync(kFull, mbar_wait(&kfull[st], (gt / kNS) & 1u, p.status)))) break;
          tc_fence_after();
          if (issuer) {
            const uint32_t d = tmem + kColS + (gt & 1u) * kNk;
            const uint32_t kb = sKa + st * kStageBytes;
            issue_s(d, sQa, kb, idesc_s);
            issue_s(d + (16u << 16), sQa + kQBytes / 2, shared ? kb : kb + kSlotBytes, idesc_s);
            umma_commit(&sfull[gt & 1u]);
            if (it == ntiles - 1) umma_commit(qempty);
          }
          __syncwarp();
        }
        if (it >= 1) {
          const uint32_t gp = g + it - 1;
          const int pb = gp & 1u, sp = gp % kNS;
          if (!(ok = __all_sync(kFull, mbar_wait(&pfull[pb], (gp >> 1) & 1u, p.status)))) break;
          tc_fence_after();
          if (issuer) {
            const uint32_t vb = sKa + sp * kStageBytes, pm = sPa + pb * kPBytes;
            issue_pv(tmem + kColO, pm, vb, idesc_pv, it > 1);
            issue_pv(tmem + kColO + (16u << 16), pm + kPBytes / 2, shared ? vb : vb + kSlotBytes, idesc_pv, it > 1);
            umma_commit(&kempty[sp]);
            umma_commit(&obar[pb]);
          }
          __syncwarp();
        }
      }
      if (issuer) {
        if (ntiles == 0) umma_commit(qempty);
        umma_commit(dbar);  // one completion per item, also after an abort
        if (!ok) *sAbort = 1;
      }
      __syncwarp();
    } else if (warp < 4) {
      // ---------------------------------------------------------------- softmax (one head row per thread)
      const int slot = lane >> 4, h = warp * 16 + (lane & 15);
      const int b_mine = slot ? b1 : b0;
      const float sl2 = p.sm_scale * kLog2e;
      const uint32_t trow = tmem + (static_cast<uint32_t>(warp * 32) << 16);
      uint8_t* prow = sP + slot * (kPBytes / 2) + h * 128;
      const int sw = h & 7;
      float m_used = -INFINITY, l_run = 0.f;
      bool ok = true;
      for (int it = 0; it < ntiles && ok; ++it) {
        const uint32_t gt = g + it;
        const uint32_t sb = trow + kColS + (gt & 1u) * kNk;
        if (!__all_sync(kFull, mbar_wait(&sfull[gt & 1u], (gt >> 1) & 1u, p.status))) {
          *sAbort = 1;
          ok = false;
          break;
        }
        // the stage's valid-key bits (written before the loaders' kfull arrival; that phase
        // cannot move on before this thread's pfull arrival for the tile)
        if (!__all_sync(kFull, mbar_wait(&kfull[gt % kNS], (gt / kNS) & 1u, p.status))) {
          *sAbort = 1;
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t* valid = sMask + (gt % kNS) * 4 + slot * 2;
        // the tile's 64 logits of this row (two loads, one wait); the row max in four chains
        const uint64_t vm = static_cast<uint64_t>(valid[0]) | (static_cast<uint64_t>(valid[1]) << 32);
        float mt;
        {
          uint32_t s[kNk];
          tmem_ld32(sb, *reinterpret_cast<uint32_t(*)[32]>(s));
          tmem_ld32(sb + 32, *reinterpret_cast<uint32_t(*)[32]>(s + 32));
          tmem_ld_wait();
          float m0 = -INFINITY, m1 = -INFINITY, m2 = -INFINITY, m3 = -INFINITY;
#pragma unroll
          for (int j = 0; j < kNk; j += 4) {
            if ((vm >> j) & 1u) m0 = fmaxf(m0, __uint_as_float(s[j]) * sl2);
            if ((vm >> (j + 1)) & 1u) m1 = fmaxf(m1, __uint_as_float(s[j + 1]) * sl2);
            if ((vm >> (j + 2)) & 1u) m2 = fmaxf(m2, __uint_as_float(s[j + 2]) * sl2);
            if ((vm >> (j + 3)) & 1u) m3 = fmaxf(m3, __uint_as_float(s[j + 3]) * sl2);
          }
          mt = fmaxf(fmaxf(m0, m1), fmaxf(m2, m3));
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
        // P buffer gt & 1 was read by the P V of tile gt - 2
        if (gt >= 2 && !__all_sync(kFull, mbar_wait(&obar[gt & 1u], ((gt >> 1) - 1) & 1u, p.status))) {
          *sAbort = 1;
          ok = false;
          break;
        }
        if (__any_sync(kFull, rescale)) {
          // O takes the rescale once the P V of tile gt - 1 (and so every earlier one) has landed
          const uint32_t gq = gt - 1;
          if (!__all_sync(kFull, mbar_wait(&obar[gq & 1u], (gq >> 1) & 1u, p.status))) {
            *sAbort = 1;
            ok = false;
            break;
          }
          tc_fence_after();
#pragma unroll 1
          for (int c = 0; c < kD; c += 32) {
            uint32_t o[32];
            tmem_ld32(trow + kColO + c, o);
            tmem_ld_wait();
#pragma unroll
            for (int j = 0; j < 32; ++j) o[j] = __float_as_uint(__uint_as_float(o[j]) * corr);
            tmem_st32(trow + kColO + c, o);
          }
          tmem_st_wait();
        }
        uint8_t* pbuf = prow + (gt & 1u) * kPBytes;
        {  // the logits again (two loads, one wait), their exponentials, the row sum in two chains
          uint32_t s[kNk];
          tmem_ld32(sb, *reinterpret_cast<uint32_t(*)[32]>(s));
          tmem_ld32(sb + 32, *reinterpret_cast<uint32_t(*)[32]>(s + 32));
          tmem_ld_wait();
          float l0 = 0.f, l1 = 0.f;
          uint32_t pp[kNk / 2];
#pragma unroll
          for (int j = 0; j < kNk / 2; ++j) {
            const float e0 = (vm >> (2 * j)) & 1u ? exp2f(__uint_as_float(s[2 * j]) * sl2 - msub) : 0.f;
            const float e1 = (vm >> (2 * j + 1)) & 1u ? exp2f(__uint_as_float(s[2 * j + 1]) * sl2 - msub) : 0.f;
            l0 += e0;
            l1 += e1;
            pp[j] = pack_bf16(e0, e1);
          }
          l_run += l0 + l1;
          // keys 8 i .. 8 i + 7: 16-byte chunk i of the row (one 64-key atom)
#pragma unroll
          for (int i = 0; i < kNk / 8; ++i)
            *reinterpret_cast<uint4*>(pbuf + ((i ^ sw) << 4)) =
                make_uint4(pp[4 * i], pp[4 * i + 1], pp[4 * i + 2], pp[4 * i + 3]);
        }
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(&pfull[gt & 1u]);
      }
      // epilogue: O / l in bf16, and the log-sum-exp
      ok = __all_sync(kFull, mbar_wait(dbar, n_item & 1u, p.status)) && ok;
      if (!ok) *sAbort = 1;
      tc_fence_after();
      // a row without keys (or after an abort) writes zeros without reading O
      const bool has = ok && l_run > 0.f;
      const float inv = has ? 1.f / l_run : 0.f;
      const bool write = b_mine >= 0;
      uint16_t* orow = write ? p.out + ((int64_t)b_mine * p.n_heads + h) * kD : nullptr;
#pragma unroll 1
      for (int c = 0; c < kD; c += 32) {
        uint32_t o[32];
        if (ok) {  // warp-uniform: every lane takes part in the tensor-memory load
          tmem_ld32(trow + kColO + c, o);
          tmem_ld_wait();
        }
        if (write) {
          const int64_t tq = p.q_pos[b_mine];
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            float f[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) f[e] = has ? __uint_as_float(o[8 * i + e]) * inv : 0.f;
            if (p.rope_dims > 0 && has) {  // inverse RoPE of the output's last rope_dims channels
              float a4[4] = {f[0], f[1], f[2], f[3]}, b4[4] = {f[4], f[5], f[6], f[7]};
              inverse_rope4(a4, c + 8 * i, kD, p.rope_dims, p.rope_base, tq);
              inverse_rope4(b4, c + 8 * i + 4, kD, p.rope_dims, p.rope_base, tq);
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                f[e] = a4[e];
                f[4 + e] = b4[e];
              }
            }
            uint4 v;
            v.x = pack_bf16(f[0], f[1]);
            v.y = pack_bf16(f[2], f[3]);
            v.z = pack_bf16(f[4], f[5]);
            v.w = pack_bf16(f[6], f[7]);
            *reinterpret_cast<uint4*>(orow + c + 8 * i) = v;
          }
        }
      }
      if (write && p.lse) p.lse[(int64_t)b_mine * p.n_heads + h] = has ? (m_used + log2f(l_run)) * kLn2 : -INFINITY;
      // the next item's first P V overwrites O: this thread's reads of it are complete
      tc_fence_before();
    }
    g += ntiles;
  }
  // after an abort, give tensor-core work and copies in flight a bounded chance to land (each
  // warp decides on lane 0's reading of the flag, so it stays converged)
  if (warp == 4 && __shfl_sync(kFull, *sAbort, 0)) {
    if (lane == 0) umma_commit(dbar);
    __syncwarp();
    mbar_wait(dbar, n_item & 1u, nullptr);
  }
  if (warp == kLoadThread0 / 32 && __shfl_sync(kFull, *sAbort, 0)) mbar_wait(qfull, n_item & 1u, nullptr);
  cp_async_wait<0>();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 4) tmem_dealloc(tmem, kTmemCols);
}

bool encode_q(CUtensorMap* map, const void* base, uint64_t rows) {
  auto enc = tensor_map_encoder();
  if (!enc) return false;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(kD), static_cast<cuuint64_t>(rows)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(kD) * 2};
  const cuuint32_t box[2] = {64, static_cast<cuuint32_t>(kH)};
  const cuuint32_t estr[2] = {1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

bool attend_pair_supported(const AttendParams& p, int n_sm) {
  const uint64_t pool_rows = static_cast<uint64_t>(p.n_pages) * p.page_size;
  const uint64_t ring_rows = static_cast<uint64_t>(p.n_seqs_layer) * p.n_win;
  return p.d_qk == kD && p.d_v == kD && p.n_heads == kH && p.kv_dtype == CSKV_BF16 &&
         p.n_q >= 4 * n_sm &&  // enough pairs for every SM without splitting keys
         pool_rows <= kRowMask && ring_rows <= kRowMask && static_cast<uint64_t>(p.chunk_len) <= kRowMask;
}

cudaError_t launch_attend_pair(AttendParams& p, int n_sm, cudaStream_t st) {
  CUtensorMap tm_q;
  if (!encode_q(&tm_q, p.q, static_cast<uint64_t>(p.n_q) * kH)) return cudaErrorNotSupported;
  const size_t smem = Smem::bytes();
  cudaError_t e = cudaFuncSetAttribute(attend_pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  const int items = (p.n_q + 1) / 2;
  const int grid = items < n_sm ? items : n_sm;
  return launch_pdl(attend_pair_kernel, dim3(static_cast<unsigned>(grid)), dim3(kThreads), smem, st, tm_q, p);
}

}  // namespace cskv
