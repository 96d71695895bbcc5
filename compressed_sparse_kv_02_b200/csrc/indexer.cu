// indexer.cu -- Lightning-indexer scores and top-k selection for CSA
// (DeepSeek-V4 report digest, section 3: a light indexer scores the
// compressed entries and only the top-k -- 512 Flash, 1024 Pro -- reach core
// attention; section 7: FP4 indexer QK path; DeepSeek-V4-book ch.1,
// section 4; 10100.com article, section 2.1: low-rank indexer).
//
//   s(t, j) = sum_h w[t,h] * ReLU(qI[t,h,:] . KI[j,:])
//
// index_scan_kernel streams the indexer keys of every visible entry once from
// HBM (the dominant decode cost: n/4 keys per query) and writes fp32 scores.
// Each warp takes 16-key tiles; the dot products run on the tensor cores as
// mma.sync m16n8k16 with keys as M, indexer heads as N (8 per n-tile) and the
// key channels as K. Each thread loads whole 16-byte pieces of its two key
// rows straight into A-fragment registers: the channel order inside a
// k-step is permuted, and the query fragments use the same permutation, so
// the dot product is unchanged while every load is a full 128-bit access.
//
// index_select_kernel picks the top-k per query: a cluster of CTAs holds the
// query's scores in shared memory (one slice per CTA) and runs a radix select
// on order-preserving integer keys in three digits (11, 11 and 10 bits). The
// first digit's histogram is counted by the TMA scan as it writes the scores;
// the later digits are counted over the few keys left in the threshold bin,
// with the per-CTA histograms summed through distributed shared memory. The
// chosen indices are written in ascending order (equal scores prefer the
// lower index).
#include <cooperative_groups.h>
#include <string.h>
#include <cudaTypedefs.h>

#include <mutex>
#include <vector>

#include "cskv_device.cuh"
#include "cskv_internal.h"

namespace cg = cooperative_groups;

namespace cskv {
namespace {

constexpr int kScanThreads = 256;
constexpr int kMaxQueries = 4096;  // queries per call (prefix table in shared memory)
constexpr int kSelThreads = 1024;
constexpr int kSliceCap = 32768;   // scores per CTA of the selection kernel
constexpr int kMaxCluster = 16;   // CTAs per query in the selection kernel (above 8: non-portable)
constexpr int kHistBins = 2048;   // bins of the score-key histogram the TMA scan leaves for the selection
constexpr int kGroupScanMinQueries = 256;  // from this many queries per call the grouped scan is used
constexpr int kStreamSelectMinQueries = 256;  // ... and the one-CTA-per-query streaming select

__device__ __forceinline__ int64_t query_visible(const IndexParams& p, int b) {
  const int64_t t = p.q_pos[b];
  if (t < 0 || t > p.max_pos) return -1;
  return visible_entries(t, p.m, p.n_win);
}

// 8 FP4 values (4 bytes) times one e4m3 block scale -> 8 halves in a uint4.
// Products of an e2m1 value and an e4m3 scale are exact in fp16.
__device__ __forceinline__ uint4 fp4x8_to_half8(uint32_t codes, uint8_t scale) {
  const __half2 s2 = __half2half2(__half(__nv_cvt_fp8_to_halfraw(scale, __NV_E4M3)));
  uint32_t o[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    __half2 v = __half2(__nv_cvt_fp4x2_to_halfraw2(
        static_cast<__nv_fp4x2_storage_t>((codes >> (8 * i)) & 0xffu), __NV_E2M1));
    v = __hmul2(v, s2);
    o[i] = *reinterpret_cast<uint32_t*>(&v);
  }
  return make_uint4(o[0], o[1], o[2], o[3]);
}

// Per-thread registers of one 16-key sub-tile: rows g and g+8.
//   bf16: NCH 16-byte chunks per row (chunk c + 4*jj of the row)
//   FP4:  the thread's d/8 bytes of codes per row (elements [c*d/4, (c+1)*d/4))
//         and its d/64 scale bytes
template <int NCH, bool FP4>
struct SubTile;
template <int NCH>
struct SubTile<NCH, false> {
  uint4 a[NCH], b[NCH];
};
template <int NCH>
struct SubTile<NCH, true> {
  uint32_t a[NCH], b[NCH];
  uint8_t sa[(NCH + 1) / 2], sb[(NCH + 1) / 2];
};

template <int NCH, bool FP4>
__device__ __forceinline__ void load_rows(SubTile<NCH, FP4>& r, const IndexParams& p,
                                          int64_t row0, int g, int c) {
  if constexpr (!FP4) {
    const uint16_t* base = static_cast<const uint16_t*>(p.idx_pool);
    const uint16_t* ra = base + (row0 + g) * p.d_idx;
    const uint16_t* rb = base + (row0 + g + 8) * p.d_idx;
#pragma unroll
    for (int jj = 0; jj < NCH; ++jj) {
      r.a[jj] = ldg16_stream(ra + (c + 4 * jj) * 8);
      r.b[jj] = ldg16_stream(rb + (c + 4 * jj) * 8);
    }
  } else {
    const uint8_t* base = static_cast<const uint8_t*>(p.idx_pool);
    const int rowb = p.d_idx / 2;  // code bytes per row
    const uint8_t* ra = base + (row0 + g) * rowb + c * (NCH * 4);
    const uint8_t* rb = base + (row0 + g + 8) * rowb + c * (NCH * 4);
    if constexpr (NCH == 4) {
      uint4 va = ldg16_stream(ra), vb = ldg16_stream(rb);
      r.a[0] = va.x; r.a[1] = va.y; r.a[2] = va.z; r.a[3] = va.w;
      r.b[0] = vb.x; r.b[1] = vb.y; r.b[2] = vb.z; r.b[3] = vb.w;
    } else {
#pragma unroll
      for (int jj = 0; jj < NCH; ++jj) {
        r.a[jj] = __ldg(reinterpret_cast<const uint32_t*>(ra) + jj);
        r.b[jj] = __ldg(reinterpret_cast<const uint32_t*>(rb) + jj);
      }
    }
    const int sper = p.d_idx / 16;
    const uint8_t* sa = p.idx_scale + (row0 + g) * sper + c * ((NCH + 1) / 2);
    const uint8_t* sb = p.idx_scale + (row0 + g + 8) * sper + c * ((NCH + 1) / 2);
#pragma unroll
    for (int i = 0; i < (NCH + 1) / 2; ++i) {
      r.sa[i] = __ldg(sa + i);
      r.sb[i] = __ldg(sb + i);
    }
  }
}

template <int NCH, bool FP4>
__device__ __forceinline__ uint4 chunk_a(const SubTile<NCH, FP4>& r, int jj) {
  if constexpr (!FP4) return r.a[jj]; else return fp4x8_to_half8(r.a[jj], r.sa[jj / 2]);
}
template <int NCH, bool FP4>
__device__ __forceinline__ uint4 chunk_b(const SubTile<NCH, FP4>& r, int jj) {
  if constexpr (!FP4) return r.b[jj]; else return fp4x8_to_half8(r.b[jj], r.sb[jj / 2]);
}

template <int NCH, int TPW, bool FP4>
struct WarpTile {
  SubTile<NCH, FP4> s[TPW];
  int64_t j0;  // first entry of the tile
  int b;       // query
  unsigned valid;  // bit per sub-tile: loaded from a valid page
};

// NCH: 8-channel chunks per thread (d_idx / 32); NTH: n-tiles of heads
// (ceil(H_I / 8)); TPW: 16-key sub-tiles per warp iteration.
template <int NCH, int NTH, int TPW, bool FP4>
__global__ void __launch_bounds__(kScanThreads, 2) index_scan_kernel(IndexParams p) {
  extern __shared__ int s_pref[];  // [n_q + 1] units per query, exclusive prefix
  __shared__ int s_wsum[32];
  constexpr int KPU = 16 * TPW;  // keys per unit
  const int tid = threadIdx.x;
  {
    int run = 0;
    for (int base = 0; base < p.n_q; base += kScanThreads) {
      const int b = base + tid;
      int u = 0;
      if (b < p.n_q) {
        const int64_t nv = query_visible(p, b);
        u = nv > 0 ? static_cast<int>((nv + KPU - 1) / KPU) : 0;
      }
      int tot;
      const int ex = block_exclusive_scan<kScanThreads>(u, s_wsum, tot);
      if (b < p.n_q) s_pref[b] = run + ex;
      run += tot;
    }
    if (tid == 0) s_pref[p.n_q] = run;
    __syncthreads();
  }
  // invalid positions are reported once, by CTA 0
  if (blockIdx.x == 0) {
    for (int b = tid; b < p.n_q; b += kScanThreads)
      if (query_visible(p, b) < 0) report(p.status, CSKV_ERR_INVALID_ARG);
  }
  const int lane = tid & 31, g = lane >> 2, c = lane & 3;
  const int64_t total = s_pref[p.n_q];
  const int64_t nwarps = (int64_t)gridDim.x * (kScanThreads / 32);
  const int64_t gw = (int64_t)blockIdx.x * (kScanThreads / 32) + (tid >> 5);
  const int64_t u_begin = total * gw / nwarps, u_end = total * (gw + 1) / nwarps;
  if (u_begin >= u_end) return;

  auto locate = [&](int64_t u, WarpTile<NCH, TPW, FP4>& wt) {
    int lo = 0, hi = p.n_q - 1;  // last b with s_pref[b] <= u
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (s_pref[mid] <= u) lo = mid; else hi = mid - 1;
    }
    wt.b = lo;
    wt.j0 = (u - s_pref[lo]) * KPU;
  };
  auto load = [&](int64_t u, WarpTile<NCH, TPW, FP4>& wt) {
    locate(u, wt);
    const int64_t nv = query_visible(p, wt.b);
    const int seq = p.q_seq[wt.b];
    wt.valid = 0;
#pragma unroll
    for (int s = 0; s < TPW; ++s) {
      const int64_t j = wt.j0 + 16 * s;
      int64_t row0 = 0;
      if (j < nv) {
        const int64_t pi = j / p.page_size;
        int32_t page = -1;
        if (seq >= 0 && seq < p.n_seqs_layer && pi < p.max_pages_per_seq)
          page = p.page_table[(int64_t)seq * p.max_pages_per_seq + pi];
        if (page >= 0 && page < p.n_pages) {
          row0 = (int64_t)page * p.page_size + (j % p.page_size);
          wt.valid |= 1u << s;
        } else if (lane == 0) {
          report(p.status, CSKV_ERR_OUT_OF_RANGE);
        }
      }
      if (wt.valid & (1u << s)) load_rows<NCH, FP4>(wt.s[s], p, row0, g, c);
    }
  };

  // query fragments (B operand): head n = 8*nt + g, same channel permutation
  uint4 qf[NTH][NCH];
  float wv[NTH][2];
  int cur_b = -1;
  auto load_query = [&](int b) {
    cur_b = b;
#pragma unroll
    for (int nt = 0; nt < NTH; ++nt) {
      const int n = 8 * nt + g;
#pragma unroll
      for (int jj = 0; jj < NCH; ++jj) {
        if (n < p.n_heads_idx) {
          if constexpr (!FP4) {
            const uint16_t* qr = static_cast<const uint16_t*>(p.q_idx) +
                                 ((int64_t)b * p.n_heads_idx + n) * p.d_idx;
            qf[nt][jj] = ldg16(qr + (c + 4 * jj) * 8);
          } else {
            const uint8_t* qr = static_cast<const uint8_t*>(p.q_idx) +
                                ((int64_t)b * p.n_heads_idx + n) * (p.d_idx / 2) + c * (NCH * 4);
            const uint8_t* qs = p.q_idx_scale + ((int64_t)b * p.n_heads_idx + n) * (p.d_idx / 16) +
                                c * ((NCH + 1) / 2);
            qf[nt][jj] = fp4x8_to_half8(__ldg(reinterpret_cast<const uint32_t*>(qr) + jj), __ldg(qs + jj / 2));
          }
        } else {
          qf[nt][jj] = make_uint4(0u, 0u, 0u, 0u);
        }
      }
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int h = 8 * nt + 2 * c + e;
        wv[nt][e] = h < p.n_heads_idx ? p.w[(int64_t)b * p.n_heads_idx + h] : 0.f;
      }
    }
  };

  auto compute = [&](const WarpTile<NCH, TPW, FP4>& wt) {
    if (wt.b != cur_b) load_query(wt.b);
    const int64_t nv = query_visible(p, wt.b);
    float* out = p.scores + (int64_t)wt.b * p.vis_stride;
#pragma unroll
    for (int s = 0; s < TPW; ++s) {
      const int64_t j = wt.j0 + 16 * s;
      if (j >= nv) break;
      float acc[NTH][4];
#pragma unroll
      for (int nt = 0; nt < NTH; ++nt) acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0.f;
#pragma unroll
      for (int jj = 0; jj < NCH; ++jj) {
        const uint4 ka = chunk_a<NCH, FP4>(wt.s[s], jj);
        const uint4 kb = chunk_b<NCH, FP4>(wt.s[s], jj);
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const uint32_t a[4] = {u4_at(ka, 2 * h), u4_at(kb, 2 * h), u4_at(ka, 2 * h + 1),
                                 u4_at(kb, 2 * h + 1)};
#pragma unroll
          for (int nt = 0; nt < NTH; ++nt) {
            if constexpr (FP4)
              mma_f16(acc[nt], a, u4_at(qf[nt][jj], 2 * h), u4_at(qf[nt][jj], 2 * h + 1));
            else
              mma_bf16(acc[nt], a, u4_at(qf[nt][jj], 2 * h), u4_at(qf[nt][jj], 2 * h + 1));
          }
        }
      }
      float s0 = 0.f, s1 = 0.f;
#pragma unroll
      for (int nt = 0; nt < NTH; ++nt) {
        s0 += wv[nt][0] * fmaxf(acc[nt][0], 0.f) + wv[nt][1] * fmaxf(acc[nt][1], 0.f);
        s1 += wv[nt][0] * fmaxf(acc[nt][2], 0.f) + wv[nt][1] * fmaxf(acc[nt][3], 0.f);
      }
      s0 += __shfl_xor_sync(kFull, s0, 1);
      s0 += __shfl_xor_sync(kFull, s0, 2);
      s1 += __shfl_xor_sync(kFull, s1, 1);
      s1 += __shfl_xor_sync(kFull, s1, 2);
      if (!(wt.valid & (1u << s))) s0 = s1 = -INFINITY;
      if (c == 0) {
        if (j + g < nv) out[j + g] = selected_score(s0, p.score_bf16);
        if (j + g + 8 < nv) out[j + g + 8] = selected_score(s1, p.score_bf16);
      }
    }
  };

  WarpTile<NCH, TPW, FP4> t0, t1;
  load(u_begin, t0);
  for (int64_t u = u_begin; u < u_end; u += 2) {
    if (u + 1 < u_end) load(u + 1, t1);
    compute(t0);
    if (u + 1 >= u_end) break;
    if (u + 2 < u_end) load(u + 2, t0);
    compute(t1);
  }
}

// ---------------------------------------------------------------- TMA-fed scan
// bf16 keys on pages of a multiple of 64 entries. One persistent CTA per SM:
// warp 0 issues 2D TMA loads of 64-key units (rows of d_idx bf16, boxes of 64
// rows x 128 bytes with the 128-byte swizzle) into an NSTAGE-deep ring of
// shared-memory stages; consumer warps 1..16, in four groups of four that take
// every fourth unit, each run one 16-key sub-tile of a unit through mma.sync.
// Under the swizzle, 16-byte chunk ch of row r sits at chunk ch ^ (r % 8) of
// its 128-byte row. A quarter-warp reads the same logical chunks of two rows;
// those rows are chosen 4 apart (fragment row g -> key (g >> 1) + 4 (g & 1))
// so that the two land on disjoint halves of the 128-byte row and every
// 128-bit shared load is conflict-free.
constexpr int kTmaConsumerWarps = 16;  // four groups of four warps
constexpr int kTmaThreads = 32 * (1 + kTmaConsumerWarps);
constexpr int kUnitKeys = 64;
constexpr int kTmaRingBytes = 128 * 1024;

template <int NCH, bool FP4 = false>
struct TmaScanShape {
  // bf16: rows of NCH * 64 bytes (2D TMA, 128-byte swizzle); FP4: the unit's codes (d_I / 2 bytes
  // per row) then its e4m3 scales (d_I / 16 bytes per row), each one contiguous block of the pool
  static constexpr int ROWB = FP4 ? NCH * 16 : NCH * 64;    // code bytes per key row
  static constexpr int SCALEB = FP4 ? NCH * 2 : 0;          // scale bytes per key row
  static constexpr int STAGE_BYTES = kUnitKeys * (ROWB + SCALEB);  // one 64-key unit
  static constexpr int NSTAGE = kTmaRingBytes / STAGE_BYTES;  // a multiple of the consumer groups
  static size_t smem_bytes(int n_q) {
    return 1024 + (size_t)kTmaRingBytes + 2 * NSTAGE * sizeof(uint64_t) + NSTAGE * sizeof(int) +
           sizeof(int) * (size_t)(n_q + 1);
  }
};

template <int NCH, int NTH, bool FP4>
__global__ void __launch_bounds__(kTmaThreads, 1)
    index_scan_tma_kernel(const __grid_constant__ CUtensorMap tmap, IndexParams p) {
  using Sh = TmaScanShape<NCH, FP4>;
  constexpr int NSTAGE = Sh::NSTAGE;
  constexpr int NGROUP = kTmaConsumerWarps / 4;
  static_assert(NSTAGE % NGROUP == 0, "each consumer group owns a fixed set of stages");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* tiles = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(tiles + kTmaRingBytes);
  uint64_t* empty = full + NSTAGE;
  int* s_valid = reinterpret_cast<int*>(empty + NSTAGE);
  int* s_pref = s_valid + NSTAGE;
  __shared__ int s_wsum[32];
  // digit-A histograms (top 11 bits of the score key) of the first and the last
  // query of this CTA's unit range; a query strictly inside the range (short
  // contexts) counts straight into the global histogram
  __shared__ uint32_t s_h[2][kHistBins];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  grid_dependency_wait();     // the keys may have been written by the kernel launched before this one
  grid_dependents_launch();  // the selection kernel may be scheduled as SMs free up
  for (int i = tid; i < 2 * kHistBins; i += kTmaThreads) (&s_h[0][0])[i] = 0u;

  {  // 64-key units per query, exclusive prefix
    int run = 0;
    for (int base = 0; base < p.n_q; base += kTmaThreads) {
      const int b = base + tid;
      int u = 0;
      if (b < p.n_q) {
        const int64_t nv = query_visible(p, b);
        u = nv > 0 ? static_cast<int>((nv + kUnitKeys - 1) / kUnitKeys) : 0;
      }
      int tot;
      const int ex = block_exclusive_scan<kTmaThreads>(u, s_wsum, tot);
      if (b < p.n_q) s_pref[b] = run + ex;
      run += tot;
    }
    if (tid == 0) s_pref[p.n_q] = run;
  }
  if (tid == 0) {
    for (int s = 0; s < NSTAGE; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 4);
    }
    fence_barrier_init();
  }
  __syncthreads();
  if (blockIdx.x == 0)
    for (int b = tid; b < p.n_q; b += kTmaThreads)
      if (query_visible(p, b) < 0) report(p.status, CSKV_ERR_INVALID_ARG);

  const int64_t total = s_pref[p.n_q];
  // the units split over min(grid, total) CTAs, so that every CTA with work has at least one unit
  const int64_t n_work = total < gridDim.x ? total : gridDim.x;
  const int64_t u_begin = blockIdx.x < n_work ? total * blockIdx.x / n_work : total;
  const int64_t n_units = blockIdx.x < n_work ? total * (blockIdx.x + 1) / n_work - u_begin : 0;
  auto locate = [&](int64_t u, int& b, int64_t& j0) {
    int lo = 0, hi = p.n_q - 1;  // last b with s_pref[b] <= u
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (s_pref[mid] <= u) lo = mid; else hi = mid - 1;
    }
    b = lo;
    j0 = (u - s_pref[lo]) * kUnitKeys;
  };
  int b_first = 0, b_last = 0;
  if (n_units > 0) {
    int64_t jx;
    locate(u_begin, b_first, jx);
    locate(u_begin + n_units - 1, b_last, jx);
  }

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    // The warp resolves the pool rows of 32 units at a time (one page-table
    // load per lane, in parallel); lane 0 then issues their loads in order.
    if (lane == 0 && !FP4) prefetch_tensormap(&tmap);
    int64_t issued = 0;
    bool ok = true;
    for (int64_t i0 = 0; i0 < n_units && ok; i0 += 32) {
      int row0 = -1;
      if (i0 + lane < n_units) {
        int b;
        int64_t j0;
        locate(u_begin + i0 + lane, b, j0);
        const int seq = p.q_seq[b];
        const int64_t pi = j0 / p.page_size;
        int32_t page = -1;
        if (seq >= 0 && seq < p.n_seqs_layer && pi < p.max_pages_per_seq)
          page = p.page_table[(int64_t)seq * p.max_pages_per_seq + pi];
        if (page >= 0 && page < p.n_pages) row0 = static_cast<int>((int64_t)page * p.page_size + (j0 % p.page_size));
      }
      const int nb = static_cast<int>(n_units - i0 < 32 ? n_units - i0 : 32);
      for (int k = 0; k < nb; ++k) {
        const int r0 = __shfl_sync(kFull, row0, k);
        if (lane == 0) {
          const int64_t i = i0 + k;
          const int s = static_cast<int>(i % NSTAGE);
          const uint32_t round = static_cast<uint32_t>(i / NSTAGE);
          if (!mbar_wait(&empty[s], (round & 1u) ^ 1u, p.status)) {
            ok = false;
          } else {
            if (r0 >= 0) {
              s_valid[s] = 1;
              mbar_arrive_expect_tx(&full[s], Sh::STAGE_BYTES);
              uint8_t* dst = tiles + (size_t)s * Sh::STAGE_BYTES;
              if constexpr (FP4) {  // 64 consecutive pool rows: their codes, then their scales
                bulk_load(dst, static_cast<const uint8_t*>(p.idx_pool) + (size_t)r0 * Sh::ROWB, kUnitKeys * Sh::ROWB,
                          &full[s]);
                bulk_load(dst + kUnitKeys * Sh::ROWB, p.idx_scale + (size_t)r0 * Sh::SCALEB,
                          kUnitKeys * Sh::SCALEB, &full[s]);
              } else {
#pragma unroll
                for (int box = 0; box < Sh::ROWB / 128; ++box)
                  tma_load_2d(dst + box * (kUnitKeys * 128), &tmap, box * 64, r0, &full[s]);
              }
            } else {
              report(p.status, CSKV_ERR_OUT_OF_RANGE);
              s_valid[s] = 0;
              mbar_arrive(&full[s]);
            }
            issued = i + 1;
          }
        }
        ok = __shfl_sync(kFull, ok, 0);
        if (!ok) break;
      }
    }
    // drain: every load issued must land before the CTA may exit
    if (lane == 0)
      for (int64_t r = issued > NSTAGE ? issued - NSTAGE : 0; r < issued; ++r)
        mbar_wait(&full[r % NSTAGE], static_cast<uint32_t>((r / NSTAGE) & 1), p.status);
    return;
  }

  // -------------------------------------------------------------- consumers
  const int cw = warp - 1, group = cw >> 2, sub = cw & 3;
  const int g = lane >> 2, c = lane & 3;
  const int pg = (g >> 1) + 4 * (g & 1);  // physical row of fragment row g within its 8-row half
  uint4 qf[NTH][NCH];
  float wv[NTH][2];
  int cur_b = -1;
  int64_t cur_nv = 0;
  for (int64_t i = group; i < n_units; i += NGROUP) {
    const int s = static_cast<int>(i % NSTAGE);
    const uint32_t round = static_cast<uint32_t>(i / NSTAGE);
    if (!mbar_wait(&full[s], round & 1u, p.status)) break;
    int b;
    int64_t j0;
    locate(u_begin + i, b, j0);
    if (b != cur_b) {
      cur_b = b;
      cur_nv = query_visible(p, b);
#pragma unroll
      for (int nt = 0; nt < NTH; ++nt) {
        const int n = 8 * nt + g;
        if constexpr (FP4) {  // the thread's channels c*d/4 .. (c+1)*d/4 - 1, as the keys' (fp16, exact)
          const uint8_t* qr = static_cast<const uint8_t*>(p.q_idx) + ((int64_t)b * p.n_heads_idx + n) * (p.d_idx / 2) +
                              c * (NCH * 4);
          const uint8_t* qs = p.q_idx_scale + ((int64_t)b * p.n_heads_idx + n) * (p.d_idx / 16) + c * (NCH / 2);
#pragma unroll
          for (int jj = 0; jj < NCH; ++jj)
            qf[nt][jj] = n < p.n_heads_idx
                             ? fp4x8_to_half8(__ldg(reinterpret_cast<const uint32_t*>(qr) + jj), __ldg(qs + jj / 2))
                             : make_uint4(0u, 0u, 0u, 0u);
        } else {
          const uint16_t* qr = static_cast<const uint16_t*>(p.q_idx) + ((int64_t)b * p.n_heads_idx + n) * p.d_idx;
#pragma unroll
          for (int jj = 0; jj < NCH; ++jj)
            qf[nt][jj] = n < p.n_heads_idx ? ldg16(qr + (c + 4 * jj) * 8) : make_uint4(0u, 0u, 0u, 0u);
        }
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int h = 8 * nt + 2 * c + e;
          wv[nt][e] = h < p.n_heads_idx ? p.w[(int64_t)b * p.n_heads_idx + h] : 0.f;
        }
      }
    }
    const int64_t nv = cur_nv;
    const int64_t j = j0 + 16 * sub;  // this warp's 16 keys
    if (j < nv) {
      float s0 = -INFINITY, s1 = -INFINITY;
      if (s_valid[s]) {
        const uint8_t* tb = tiles + (size_t)s * Sh::STAGE_BYTES;
        const int r0 = 16 * sub + pg;  // rows r0 and r0 + 8 (same swizzle phase)
        // two independent accumulation chains (k-steps h = 0 and h = 1), summed at the end
        float acc[2][NTH][4];
#pragma unroll
        for (int h = 0; h < 2; ++h)
#pragma unroll
          for (int nt = 0; nt < NTH; ++nt) acc[h][nt][0] = acc[h][nt][1] = acc[h][nt][2] = acc[h][nt][3] = 0.f;
        if constexpr (FP4) {
          // rows r0 and r0 + 8: the thread's NCH * 4 code bytes (channels c*d/4 ..) and NCH / 2 scales
          const uint8_t* ca = tb + r0 * Sh::ROWB + c * (NCH * 4);
          const uint8_t* cb = ca + 8 * Sh::ROWB;
          const uint8_t* sa = tb + kUnitKeys * Sh::ROWB + r0 * Sh::SCALEB + c * (NCH / 2);
          const uint8_t* sb = sa + 8 * Sh::SCALEB;
          uint32_t wa[NCH], wb[NCH];
          if constexpr (NCH == 4) {
            const uint4 va = lds16(ca), vb = lds16(cb);
            wa[0] = va.x; wa[1] = va.y; wa[2] = va.z; wa[3] = va.w;
            wb[0] = vb.x; wb[1] = vb.y; wb[2] = vb.z; wb[3] = vb.w;
          } else {
#pragma unroll
            for (int jj = 0; jj < NCH; ++jj) {
              wa[jj] = reinterpret_cast<const uint32_t*>(ca)[jj];
              wb[jj] = reinterpret_cast<const uint32_t*>(cb)[jj];
            }
          }
#pragma unroll
          for (int jj = 0; jj < NCH; ++jj) {
            const uint4 ka = fp4x8_to_half8(wa[jj], sa[jj / 2]);
            const uint4 kb = fp4x8_to_half8(wb[jj], sb[jj / 2]);
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              const uint32_t a[4] = {u4_at(ka, 2 * h), u4_at(kb, 2 * h), u4_at(ka, 2 * h + 1), u4_at(kb, 2 * h + 1)};
#pragma unroll
              for (int nt = 0; nt < NTH; ++nt)
                mma_f16(acc[h][nt], a, u4_at(qf[nt][jj], 2 * h), u4_at(qf[nt][jj], 2 * h + 1));
            }
          }
        } else {
#pragma unroll
          for (int jj = 0; jj < NCH; ++jj) {
            const int q = c + 4 * jj;
            const int off = (q >> 3) * (kUnitKeys * 128) + (((q & 7) ^ pg) << 4);
            const uint4 ka = lds16(tb + off + r0 * 128);
            const uint4 kb = lds16(tb + off + (r0 + 8) * 128);
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              const uint32_t a[4] = {u4_at(ka, 2 * h), u4_at(kb, 2 * h), u4_at(ka, 2 * h + 1), u4_at(kb, 2 * h + 1)};
#pragma unroll
              for (int nt = 0; nt < NTH; ++nt)
                mma_bf16(acc[h][nt], a, u4_at(qf[nt][jj], 2 * h), u4_at(qf[nt][jj], 2 * h + 1));
            }
          }
        }
        s0 = 0.f;
        s1 = 0.f;
#pragma unroll
        for (int nt = 0; nt < NTH; ++nt) {
          const float d0 = acc[0][nt][0] + acc[1][nt][0], d1 = acc[0][nt][1] + acc[1][nt][1];
          const float d2 = acc[0][nt][2] + acc[1][nt][2], d3 = acc[0][nt][3] + acc[1][nt][3];
          s0 += wv[nt][0] * fmaxf(d0, 0.f) + wv[nt][1] * fmaxf(d1, 0.f);
          s1 += wv[nt][0] * fmaxf(d2, 0.f) + wv[nt][1] * fmaxf(d3, 0.f);
        }
        s0 += __shfl_xor_sync(kFull, s0, 1);
        s0 += __shfl_xor_sync(kFull, s0, 2);
        s1 += __shfl_xor_sync(kFull, s1, 1);
        s1 += __shfl_xor_sync(kFull, s1, 2);
        s0 = selected_score(s0, p.score_bf16);
        s1 = selected_score(s1, p.score_bf16);
      }
      if (c == 0) {
        float* out = p.scores + (int64_t)b * p.vis_stride;
        uint32_t* hrow = b == b_first ? s_h[0] : b == b_last ? s_h[1] : nullptr;
        uint32_t* gh = p.hist + (int64_t)b * kHistBins;
        if (j + pg < nv) {
          out[j + pg] = s0;
          const uint32_t d = f2key(s0) >> 21;
          atomicAdd(hrow ? hrow + d : gh + d, 1u);
        }
        if (j + pg + 8 < nv) {
          out[j + pg + 8] = s1;
          const uint32_t d = f2key(s1) >> 21;
          atomicAdd(hrow ? hrow + d : gh + d, 1u);
        }
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[s]);
  }
  // consumers only (the producer warp has returned): flush the shared histograms
  asm volatile("bar.sync 1, %0;\n" ::"r"(kTmaConsumerWarps * 32) : "memory");
  if (n_units > 0) {
    for (int i = tid - 32; i < 2 * kHistBins; i += kTmaConsumerWarps * 32) {
      const int which = i / kHistBins, bin = i % kHistBins;
      const uint32_t v = s_h[which][bin];
      if (v) atomicAdd(p.hist + (int64_t)(which ? b_last : b_first) * kHistBins + bin, v);
    }
  }
}

// ---------------------------------------------------------------- grouped TMA scan
// For calls with many queries (a prefill chunk): consecutive queries of one
// sequence form groups of GQ = 32 / HI (8 queries of 4 indexer heads, or 4 of
// 8), and every 64-key unit is scored against the whole group at once, the
// group's queries x heads filling the mma's N = 32. Keys are read once per
// group instead of once per query. A group starts at every GQ-th query and
// wherever the sequence changes, so it never mixes sequences. The scores are
// the same as the per-query scan's; the digit histogram is left to the select.
template <int NCH, int HI>
__global__ void __launch_bounds__(kTmaThreads, 1)
    index_scan_group_kernel(const __grid_constant__ CUtensorMap tmap, IndexParams p) {
  using Sh = TmaScanShape<NCH>;
  constexpr int NSTAGE = Sh::NSTAGE;
  constexpr int NGROUP = kTmaConsumerWarps / 4;
  constexpr int GQ = 32 / HI;  // queries per group
  constexpr int NTH = 4;       // n-tiles of 8 columns: GQ x HI = 32
  static_assert(HI == 4 || HI == 8, "group shapes");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* tiles = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(tiles + kTmaRingBytes);
  uint64_t* empty = full + NSTAGE;
  int* s_valid = reinterpret_cast<int*>(empty + NSTAGE);
  int* e_start = s_valid + NSTAGE;   // [n_q + 1] first query of each group
  int* e_pref = e_start + p.n_q + 1;  // [n_q + 1] 64-key units before each group
  __shared__ int s_wsum[32];
  __shared__ int s_nent;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  grid_dependency_wait();
  grid_dependents_launch();
  {  // group starts
    int run = 0;
    for (int base = 0; base < p.n_q; base += kTmaThreads) {
      const int b = base + tid;
      int f = 0;
      if (b < p.n_q) f = (b % GQ == 0) || p.q_seq[b] != p.q_seq[b - 1];
      int tot;
      const int ex = block_exclusive_scan<kTmaThreads>(f, s_wsum, tot);
      if (f) e_start[run + ex] = b;
      run += tot;
    }
    if (tid == 0) {
      e_start[run] = p.n_q;
      s_nent = run;
    }
    __syncthreads();
  }
  const int n_ent = s_nent;
  {  // units per group: the most visible entries of its queries
    int run = 0;
    for (int base = 0; base < n_ent; base += kTmaThreads) {
      const int e = base + tid;
      int u = 0;
      if (e < n_ent) {
        int64_t nv = 0;
        for (int b = e_start[e]; b < e_start[e + 1]; ++b) {
          const int64_t v = query_visible(p, b);
          nv = v > nv ? v : nv;
        }
        u = static_cast<int>((nv + kUnitKeys - 1) / kUnitKeys);
      }
      int tot;
      const int ex = block_exclusive_scan<kTmaThreads>(u, s_wsum, tot);
      if (e < n_ent) e_pref[e] = run + ex;
      run += tot;
    }
    if (tid == 0) e_pref[n_ent] = run;
  }
  if (tid == 0) {
    for (int s = 0; s < NSTAGE; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 4);
    }
    fence_barrier_init();
  }
  __syncthreads();
  if (blockIdx.x == 0)
    for (int b = tid; b < p.n_q; b += kTmaThreads)
      if (query_visible(p, b) < 0) report(p.status, CSKV_ERR_INVALID_ARG);

  const int64_t total = e_pref[n_ent];
  const int64_t u_begin = total * blockIdx.x / gridDim.x;
  const int64_t n_units = total * (blockIdx.x + 1) / gridDim.x - u_begin;
  auto locate = [&](int64_t u, int& e, int64_t& j0) {
    int lo = 0, hi = n_ent - 1;  // last e with e_pref[e] <= u
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (e_pref[mid] <= u) lo = mid; else hi = mid - 1;
    }
    e = lo;
    j0 = (u - e_pref[lo]) * kUnitKeys;
  };

  if (warp == 0) {
    // ------------------------------------------------------------ producer (as in the per-query scan)
    if (lane == 0) prefetch_tensormap(&tmap);
    int64_t issued = 0;
    bool ok = true;
    for (int64_t i0 = 0; i0 < n_units && ok; i0 += 32) {
      int row0 = -1;
      if (i0 + lane < n_units) {
        int e;
        int64_t j0;
        locate(u_begin + i0 + lane, e, j0);
        const int seq = p.q_seq[e_start[e]];
        const int64_t pi = j0 / p.page_size;
        int32_t page = -1;
        if (seq >= 0 && seq < p.n_seqs_layer && pi < p.max_pages_per_seq)
          page = p.page_table[(int64_t)seq * p.max_pages_per_seq + pi];
        if (page >= 0 && page < p.n_pages) row0 = static_cast<int>((int64_t)page * p.page_size + (j0 % p.page_size));
      }
      const int nb = static_cast<int>(n_units - i0 < 32 ? n_units - i0 : 32);
      for (int k = 0; k < nb; ++k) {
        const int r0 = __shfl_sync(kFull, row0, k);
        if (lane == 0) {
          const int64_t i = i0 + k;
          const int s = static_cast<int>(i % NSTAGE);
          const uint32_t round = static_cast<uint32_t>(i / NSTAGE);
          if (!mbar_wait(&empty[s], (round & 1u) ^ 1u, p.status)) {
            ok = false;
          } else {
            if (r0 >= 0) {
              s_valid[s] = 1;
              mbar_arrive_expect_tx(&full[s], Sh::STAGE_BYTES);
#pragma unroll
              for (int box = 0; box < Sh::ROWB / 128; ++box)
                tma_load_2d(tiles + (size_t)s * Sh::STAGE_BYTES + box * (kUnitKeys * 128), &tmap, box * 64, r0,
                            &full[s]);
            } else {
              report(p.status, CSKV_ERR_OUT_OF_RANGE);
              s_valid[s] = 0;
              mbar_arrive(&full[s]);
            }
            issued = i + 1;
          }
        }
        ok = __shfl_sync(kFull, ok, 0);
        if (!ok) break;
      }
    }
    if (lane == 0)
      for (int64_t r = issued > NSTAGE ? issued - NSTAGE : 0; r < issued; ++r)
        mbar_wait(&full[r % NSTAGE], static_cast<uint32_t>((r / NSTAGE) & 1), p.status);
    return;
  }

  // -------------------------------------------------------------- consumers
  const int cw = warp - 1, group = cw >> 2, sub = cw & 3;
  const int g = lane >> 2, c = lane & 3;
  const int pg = (g >> 1) + 4 * (g & 1);  // physical row of fragment row g within its 8-row half
  uint4 qf[NTH][NCH];
  float wv[NTH][2];
  // visible entries of the query whose scores this lane writes in n-tile nt (0 past the group's
  // end; < 2^31 by the host checks)
  int nvw[NTH];
  int cur_e = -1, gs = 0;
  for (int64_t i = group; i < n_units; i += NGROUP) {
    const int s = static_cast<int>(i % NSTAGE);
    const uint32_t round = static_cast<uint32_t>(i / NSTAGE);
    if (!mbar_wait(&full[s], round & 1u, p.status)) break;
    int e;
    int64_t j0;
    locate(u_begin + i, e, j0);
    if (e != cur_e) {
      cur_e = e;
      gs = e_start[e];
      const int gn = e_start[e + 1] - gs;
#pragma unroll
      for (int nt = 0; nt < NTH; ++nt) {
        const int m = HI == 8 ? nt : 2 * nt + (c >> 1);
        const int64_t v = m < gn ? query_visible(p, gs + m) : 0;
        nvw[nt] = v > 0 ? static_cast<int>(v) : 0;
      }
#pragma unroll
      for (int nt = 0; nt < NTH; ++nt) {
        const int n = 8 * nt + g;  // this lane's B column
        const int m = n / HI, h = n % HI;
        const uint16_t* qr = static_cast<const uint16_t*>(p.q_idx) + ((int64_t)(gs + m) * p.n_heads_idx + h) * p.d_idx;
#pragma unroll
        for (int jj = 0; jj < NCH; ++jj)
          qf[nt][jj] = m < gn ? ldg16(qr + (c + 4 * jj) * 8) : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
        for (int ee = 0; ee < 2; ++ee) {
          const int n2 = 8 * nt + 2 * c + ee;
          const int m2 = n2 / HI, h2 = n2 % HI;
          wv[nt][ee] = m2 < gn ? p.w[(int64_t)(gs + m2) * p.n_heads_idx + h2] : 0.f;
        }
      }
    }
    const int64_t j = j0 + 16 * sub;  // this warp's 16 keys
    float acc[NTH][4];  // one accumulation chain (the four n-tiles already interleave)
#pragma unroll
    for (int nt = 0; nt < NTH; ++nt) acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0.f;
    const bool valid = s_valid[s] != 0;
    if (valid) {
      const uint8_t* tb = tiles + (size_t)s * Sh::STAGE_BYTES;
      const int r0 = 16 * sub + pg;  // rows r0 and r0 + 8 (same swizzle phase)
#pragma unroll
      for (int jj = 0; jj < NCH; ++jj) {
        const int q = c + 4 * jj;
        const int off = (q >> 3) * (kUnitKeys * 128) + (((q & 7) ^ pg) << 4);
        const uint4 ka = lds16(tb + off + r0 * 128);
        const uint4 kb = lds16(tb + off + (r0 + 8) * 128);
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const uint32_t a[4] = {u4_at(ka, 2 * h), u4_at(kb, 2 * h), u4_at(ka, 2 * h + 1), u4_at(kb, 2 * h + 1)};
#pragma unroll
          for (int nt = 0; nt < NTH; ++nt) mma_bf16(acc[nt], a, u4_at(qf[nt][jj], 2 * h), u4_at(qf[nt][jj], 2 * h + 1));
        }
      }
    }
    // per n-tile: rows (keys) j + pg and j + pg + 8, columns 2c, 2c+1 of the tile
#pragma unroll
    for (int nt = 0; nt < NTH; ++nt) {
      float s0 = -INFINITY, s1 = -INFINITY;
      if (valid) {
        s0 = wv[nt][0] * fmaxf(acc[nt][0], 0.f) + wv[nt][1] * fmaxf(acc[nt][1], 0.f);
        s1 = wv[nt][0] * fmaxf(acc[nt][2], 0.f) + wv[nt][1] * fmaxf(acc[nt][3], 0.f);
        // a query's heads are HI consecutive columns: 2 lanes (HI = 4) or 4 lanes (HI = 8)
        s0 += __shfl_xor_sync(kFull, s0, 1);
        s1 += __shfl_xor_sync(kFull, s1, 1);
        if (HI == 8) {
          s0 += __shfl_xor_sync(kFull, s0, 2);
          s1 += __shfl_xor_sync(kFull, s1, 2);
        }
      }
      const bool writer = HI == 8 ? c == 0 : (c & 1) == 0;
      const int m = HI == 8 ? nt : 2 * nt + (c >> 1);
      if (writer) {
        const int64_t nv = nvw[nt];
        float* out = p.scores + (int64_t)(gs + m) * p.vis_stride;
        if (j + pg < nv) out[j + pg] = selected_score(s0, p.score_bf16);
        if (j + pg + 8 < nv) out[j + pg + 8] = selected_score(s1, p.score_bf16);
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[s]);
  }
}

// ---------------------------------------------------------------- top-k
// Radix select on 32-bit order-preserving keys with three digits:
// A = bits 31..21 (2048 bins), B = bits 20..10 (2048 bins), C = bits 9..0
// (1024 bins). Digit A's histogram comes from the scan (global, per query)
// when the TMA scan ran, else from one pass over the slices. Keys whose digit
// A equals the threshold digit are gathered into a short candidate list, and
// digits B and C are counted over that list only; a threshold bin too large
// for the list falls back to masked passes over the whole slice.
constexpr int kBinsA = 2048, kBinsB = 2048, kBinsC = 1024;
constexpr int kCandCap = 8192;  // candidate keys per CTA held in shared memory

// count digit (key >> shift) & dmask of the keys of src[0, n) with (key & mask) == prefix
__device__ __forceinline__ void hist_pass(const uint32_t* src, int n, uint32_t mask, uint32_t prefix, int shift,
                                          uint32_t dmask, uint32_t* hist) {
  const int lane = threadIdx.x & 31;
  for (int base = 0; base < n; base += kSelThreads) {
    const int i = base + threadIdx.x;
    const uint32_t key = i < n ? src[i] : 0u;
    const bool ok = i < n && (key & mask) == prefix;
    const uint32_t dg = (key >> shift) & dmask;
    const unsigned act = __ballot_sync(kFull, ok);
    if (ok) {
      const unsigned peers = __match_any_sync(act, dg);
      if (lane == __ffs(peers) - 1) atomicAdd(&hist[dg], static_cast<uint32_t>(__popc(peers)));
    }
  }
}

// the same over a short list with keys spread over many bins: one atomic per key
__device__ __forceinline__ void hist_pass_sparse(const uint32_t* src, int n, uint32_t mask, uint32_t prefix,
                                                 int shift, uint32_t dmask, uint32_t* hist) {
  for (int i = threadIdx.x; i < n; i += kSelThreads) {
    const uint32_t key = src[i];
    if ((key & mask) == prefix) atomicAdd(&hist[(key >> shift) & dmask], 1u);
  }
}

// The digit holding the krem-th largest key, given the count of every bin
// (count(bin) for bin in [0, nbins)); bins are walked in descending order.
// Every thread returns the same digit, the rank left inside its bin and the
// bin's count. Uses every thread of the block.
template <typename CountFn>
__device__ __forceinline__ void find_digit(int nbins, int krem, CountFn count, int* s_w, uint32_t* s_res,
                                           uint32_t& digit, int& krem_out, int& bin_cnt) {
  const int per = nbins / kSelThreads;  // 1 or 2 bins per thread
  int c[2] = {0, 0};
  int tot = 0;
  for (int e = 0; e < per; ++e) {
    c[e] = count(nbins - 1 - (threadIdx.x * per + e));
    tot += c[e];
  }
  int all;
  int run = block_exclusive_scan<kSelThreads>(tot, s_w, all);
  for (int e = 0; e < per; ++e) {
    if (run < krem && krem <= run + c[e]) {
      s_res[0] = static_cast<uint32_t>(nbins - 1 - (threadIdx.x * per + e));
      s_res[1] = static_cast<uint32_t>(krem - run);
      s_res[2] = static_cast<uint32_t>(c[e]);
    }
    run += c[e];
  }
  __syncthreads();
  digit = s_res[0];
  krem_out = static_cast<int>(s_res[1]);
  bin_cnt = static_cast<int>(s_res[2]);
  __syncthreads();
}

__device__ __forceinline__ int warp_exclusive_scan(int v, int lane) {
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(kFull, x, o);
    if (lane >= o) x += y;
  }
  return x - v;
}


__global__ void __launch_bounds__(kSelThreads, 1) index_select_kernel(IndexParams p) {
  cg::cluster_group cluster = cg::this_cluster();
  const int CL = p.cluster;
  const int rank = static_cast<int>(cluster.block_rank());
  const int b = blockIdx.x / CL;
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  // [slice] keys | [kCandCap] this CTA's candidates | [kCandCap] the cluster's candidates
  extern __shared__ __align__(16) uint32_t s_keys[];
  uint32_t* s_cand = s_keys + p.slice;
  uint32_t* s_all = s_cand + kCandCap;
  __shared__ uint32_t s_hA[kBinsA], s_hB[kBinsB], s_hC[kBinsC];
  __shared__ int s_w[32];
  __shared__ uint32_t s_res[3];
  __shared__ int s_cnt[3];
  __shared__ int s_ncand;
  __shared__ __align__(8) uint64_t s_bar;
  __shared__ int s_peer[3 * kMaxCluster];
  constexpr int NW = kSelThreads / 32;
  __shared__ int s_wgt[NW], s_weq[NW];
  // per warp: the slice positions of its keys at or above the threshold digit, in index order
  // (built by the conversion pass when digit A is known first); the ordered output walks these
  // short lists instead of the whole slice unless one of them overflowed
  constexpr int kListCapW = 128;
  __shared__ uint16_t s_list[NW][kListCapW];
  __shared__ int s_wlen[NW];
  __shared__ int s_over;

  for (int i = tid; i < kBinsA; i += kSelThreads) s_hA[i] = 0u;
  for (int i = tid; i < kBinsB; i += kSelThreads) s_hB[i] = 0u;
  for (int i = tid; i < kBinsC; i += kSelThreads) s_hC[i] = 0u;
  if (tid == 0) {
    s_ncand = 0;
    s_over = 0;
    s_res[0] = s_res[1] = s_res[2] = 0u;
    mbar_init(&s_bar, 1);
    fence_barrier_init();
  }
  const int k = p.k;
  int64_t nv = query_visible(p, b);
  if (nv < 0) nv = 0;
  const float* sc = p.scores + (int64_t)b * p.vis_stride;
  int32_t* oidx = p.out_idx + (int64_t)b * k;
  float* osc = p.out_scores ? p.out_scores + (int64_t)b * k : nullptr;
  const int64_t lo = (int64_t)rank * p.slice;
  const int64_t hi = lo + p.slice < nv ? lo + p.slice : nv;
  int len = hi > lo ? static_cast<int>(hi - lo) : 0;
  grid_dependency_wait();  // the scores and the digit-A histogram come from the scan
  grid_dependents_launch();
  __syncthreads();
  // the slice's scores (whole 16-byte pieces) land by one bulk copy while digit A is found
  int n4 = nv > k ? len >> 2 : 0;
  if (tid == 0 && n4 > 0) {
    mbar_arrive_expect_tx(&s_bar, static_cast<uint32_t>(n4) * 16u);
    bulk_load(s_keys, sc + lo, static_cast<uint32_t>(n4) * 16u, &s_bar);
  }

  if (nv <= k) {  // everything visible is chosen (uniform across the cluster)
    for (int64_t i = (int64_t)rank * kSelThreads + tid; i < k; i += (int64_t)CL * kSelThreads) {
      oidx[i] = i < nv ? static_cast<int32_t>(i) : -1;
      if (osc) osc[i] = i < nv ? sc[i] : 0.f;
    }
    if (rank == 0 && tid == 0) p.out_cnt[b] = static_cast<int32_t>(nv);
    return;
  }

  bool copy_ok = true;  // this CTA's slice landed
  // digit A from the scan's histogram, when there is one (identical in every CTA)
  uint32_t dA = 0u;
  int krem = k, nA = 0;
  if (p.hist) {
    const uint32_t* gh = p.hist + (int64_t)b * kBinsA;
    find_digit(kBinsA, k, [&](int bin) { return static_cast<int>(gh[bin]); }, s_w, s_res, dA, krem, nA);
  }
  const uint32_t maskA = 0xFFE00000u;
  const unsigned below = (1u << lane) - 1u;
  // appends the keys of digit dA among the flagged ones to this CTA's candidate list
  auto gather = [&](uint32_t key, bool cand) {
    const unsigned m = __ballot_sync(kFull, cand);
    if (m) {
      int at = 0;
      if (lane == __ffs(m) - 1) at = atomicAdd(&s_ncand, __popc(m));
      at = __shfl_sync(kFull, at, __ffs(m) - 1) + __popc(m & below);
      if (cand && at < kCandCap) s_cand[at] = key;  // always true while the histogram matches the scores
    }
  };
  {  // scores -> keys in place; the candidates of digit dA are gathered on the way
    const bool gather_now = p.hist && nA <= kCandCap;
    const uint32_t pre = dA << 21;
    if (n4 > 0 && !mbar_wait(&s_bar, 0u, p.status)) {
      // The copy did not complete within the wait limit (the status word says so): this CTA
      // contributes no keys, the cluster still runs every barrier, and the query's result is
      // withdrawn below (out_cnt = 0).
      copy_ok = false;
      n4 = 0;
      len = 0;
    }
    if (gather_now) {
      // Warp w scans its contiguous part [w*seg, (w+1)*seg) of the slice (seg a multiple of 128,
      // four consecutive scores per lane per step) and keeps the positions of its keys at or above
      // digit dA in order; the slice keeps the raw scores (keys are formed where they are read),
      // the 0..3 scores past the bulk copy are copied in from global memory. The candidates of
      // digit dA are then gathered from the lists.
      const int seg = ((len + NW - 1) / NW + 127) / 128 * 128;
      const int s_lo = wid * seg, s_hi = min(len, s_lo + seg);
      int nl = 0;
      for (int base = s_lo; base < s_hi; base += 128) {
        const int i = base + 4 * lane;
        uint32_t kk[4];
        unsigned valid = 0u;
        if (i + 3 < s_hi && i + 3 < 4 * n4) {
          const uint4 fv = reinterpret_cast<const uint4*>(s_keys)[i >> 2];
          kk[0] = f2key(__uint_as_float(fv.x));
          kk[1] = f2key(__uint_as_float(fv.y));
          kk[2] = f2key(__uint_as_float(fv.z));
          kk[3] = f2key(__uint_as_float(fv.w));
          valid = 15u;
        } else {
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int j = i + e;
            kk[e] = 0u;
            if (j < s_hi) {
              const float f = j < 4 * n4 ? __uint_as_float(s_keys[j]) : sc[lo + j];
              if (j >= 4 * n4) s_keys[j] = __float_as_uint(f);
              kk[e] = f2key(f);
              valid |= 1u << e;
            }
          }
        }
        int nq = 0;
#pragma unroll
        for (int e = 0; e < 4; ++e) nq += ((valid >> e) & 1u) && (kk[e] >> 21) >= dA ? 1 : 0;
        if (__any_sync(kFull, nq > 0)) {
          const int off = warp_exclusive_scan(nq, lane);
          int at = nl + off;
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            if (((valid >> e) & 1u) && (kk[e] >> 21) >= dA) {
              if (at < kListCapW) s_list[wid][at] = static_cast<uint16_t>(i + e);
              ++at;
            }
          }
          nl += __shfl_sync(kFull, off + nq, 31);
        }
      }
      if (lane == 0) {
        s_wlen[wid] = nl;
        if (nl > kListCapW) s_over = 1;
      }
      __syncthreads();
      if (s_over == 0) {
        for (int e0 = 0; e0 < nl; e0 += 32) {
          const int e = e0 + lane;
          const uint32_t key = e < nl ? f2key(__uint_as_float(s_keys[s_list[wid][e]])) : 0u;
          gather(key, e < nl && (key & maskA) == pre);
        }
      }
      __syncthreads();
      // a list overflowed (a threshold bin of heavy ties): the slice is converted in place and
      // gathered whole, and the passes below run over the slice
      if (s_over) {
        for (int j = tid; j < len; j += kSelThreads) {
          const uint32_t key = f2key(__uint_as_float(s_keys[j]));
          s_keys[j] = key;
        }
        for (int base = 0; base < len; base += kSelThreads) {
          const int j = base + tid;
          const uint32_t key = j < len ? s_keys[j] : 0u;
          gather(key, j < len && (key & maskA) == pre);
        }
      }
    } else {
      uint4* k4 = reinterpret_cast<uint4*>(s_keys);
      for (int base = 0; base < n4; base += kSelThreads) {
        const int i = base + tid;
        if (i < n4) {
          const uint4 fv = k4[i];
          k4[i] = make_uint4(f2key(__uint_as_float(fv.x)), f2key(__uint_as_float(fv.y)), f2key(__uint_as_float(fv.z)),
                             f2key(__uint_as_float(fv.w)));
        }
      }
      for (int base = n4 << 2; base < len; base += kSelThreads) {  // the last 0..3 keys
        const int i = base + tid;
        if (i < len) s_keys[i] = f2key(sc[lo + i]);
      }
    }
  }
  __syncthreads();
  if (!p.hist) {  // digit A over the slices, then the candidates
    hist_pass(s_keys, len, 0u, 0u, 21, kBinsA - 1, s_hA);
    cluster.sync();
    find_digit(kBinsA, k, [&](int bin) {
      uint32_t part[kMaxCluster];
#pragma unroll
      for (int r = 0; r < kMaxCluster; ++r) part[r] = r < CL ? *cluster.map_shared_rank(&s_hA[bin], r) : 0u;
      int c = 0;
#pragma unroll
      for (int r = 0; r < kMaxCluster; ++r) c += static_cast<int>(part[r]);
      return c;
    }, s_w, s_res, dA, krem, nA);
    if (nA <= kCandCap)
      for (int base = 0; base < len; base += kSelThreads) {
        const int i = base + tid;
        const uint32_t key = i < len ? s_keys[i] : 0u;
        gather(key, i < len && (key & maskA) == (dA << 21));
      }
  }
  uint32_t prefix = dA << 21, mask = maskA;
  uint32_t dB = 0u, dC = 0u;
  int nB = 0, nC = 0;
  if (nA <= kCandCap) {
    // every CTA copies the cluster's candidates (nA keys in all) and finishes the select alone
    cluster.sync();
    __shared__ int s_pn[kMaxCluster + 1], s_pq[kMaxCluster + 1];  // prefix of keys / 16-byte pieces per peer
    __shared__ int s_nr[kMaxCluster];
    if (tid < CL) s_nr[tid] = min(*cluster.map_shared_rank(&s_ncand, tid), kCandCap);  // the peers' counts at once
    __syncthreads();
    if (tid == 0) {
      int nk = 0, nq = 0;
      for (int r = 0; r < CL; ++r) {
        s_pn[r] = nk;
        s_pq[r] = nq;
        nk += s_nr[r];
        nq += (s_nr[r] + 3) >> 2;
      }
      s_pn[CL] = nk;
      s_pq[CL] = nq;
    }
    __syncthreads();
    const int n_all = min(s_pn[CL], kCandCap);
    for (int t = tid; t < s_pq[CL]; t += kSelThreads) {  // one 16-byte piece of a peer's list per thread
      int r = 0;
      while (r + 1 < CL && s_pq[r + 1] <= t) ++r;
      const int piece = t - s_pq[r];
      const int n_r = s_pn[r + 1] - s_pn[r];
      const uint4 v = reinterpret_cast<const uint4*>(cluster.map_shared_rank(s_cand, r))[piece];
      const uint32_t vv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int j = piece * 4 + e, o = s_pn[r] + j;
        if (j < n_r && o < kCandCap) s_all[o] = vv[e];
      }
    }
    __syncthreads();
    hist_pass_sparse(s_all, n_all, mask, prefix, 10, kBinsB - 1, s_hB);
    __syncthreads();
    find_digit(kBinsB, krem, [&](int bin) { return static_cast<int>(s_hB[bin]); }, s_w, s_res, dB, krem, nB);
    prefix |= dB << 10;
    mask |= 0x001FFC00u;
    hist_pass_sparse(s_all, n_all, mask, prefix, 0, kBinsC - 1, s_hC);
    __syncthreads();
    find_digit(kBinsC, krem, [&](int bin) { return static_cast<int>(s_hC[bin]); }, s_w, s_res, dC, krem, nC);
  } else {
    // a threshold bin too large for the lists: masked passes over the slices, histograms summed over the cluster
    auto remote_count = [&](const uint32_t* h) {
      return [&, h](int bin) {
        uint32_t part[kMaxCluster];
#pragma unroll
        for (int r = 0; r < kMaxCluster; ++r) part[r] = r < CL ? *cluster.map_shared_rank(h + bin, r) : 0u;
        int c = 0;
#pragma unroll
        for (int r = 0; r < kMaxCluster; ++r) c += static_cast<int>(part[r]);
        return c;
      };
    };
    hist_pass(s_keys, len, mask, prefix, 10, kBinsB - 1, s_hB);
    cluster.sync();
    find_digit(kBinsB, krem, remote_count(s_hB), s_w, s_res, dB, krem, nB);
    prefix |= dB << 10;
    mask |= 0x001FFC00u;
    hist_pass(s_keys, len, mask, prefix, 0, kBinsC - 1, s_hC);
    cluster.sync();
    find_digit(kBinsC, krem, remote_count(s_hC), s_w, s_res, dC, krem, nC);
  }
  const uint32_t T = prefix | dC;  // the k-th largest key; take the first krem keys equal to T

  // Ordered output. Warp w owns the contiguous segment [w*seg, (w+1)*seg) of
  // this CTA's slice (seg a multiple of 128: 4 keys per lane per step). Pass
  // 1 counts, per warp, keys above T and equal to T; the counts are scanned
  // over the warps of the CTA and then over the CTAs of the cluster; pass 2
  // writes the chosen ids in index order.
  const int seg = ((len + NW - 1) / NW + 127) / 128 * 128;
  const int s_lo = wid * seg, s_hi = min(len, s_lo + seg);
  auto keys4 = [&](int i, uint32_t (&kk)[4], unsigned& valid) {
    if (i + 3 < s_hi) {
      const uint4 v = *reinterpret_cast<const uint4*>(s_keys + i);
      kk[0] = v.x; kk[1] = v.y; kk[2] = v.z; kk[3] = v.w;
      valid = 15u;
    } else {
      valid = 0u;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        kk[e] = i + e < s_hi ? s_keys[i + e] : 0u;
        valid |= (i + e < s_hi ? 1u : 0u) << e;
      }
    }
  };
  // every key >= T has a digit >= dA, so a complete list holds all of them
  const bool listed = p.hist && nA <= kCandCap && s_over == 0;  // uniform across the CTA
  const int nl = listed ? s_wlen[wid] : 0;
  int gt = 0, eq = 0;
  if (listed) {
    for (int e = lane; e < nl; e += 32) {
      const uint32_t key = f2key(__uint_as_float(s_keys[s_list[wid][e]]));  // raw scores on this path
      gt += key > T;
      eq += key == T;
    }
  } else {
    for (int base = s_lo; base < s_hi; base += 128) {
      uint32_t kk[4];
      unsigned valid;
      keys4(base + 4 * lane, kk, valid);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        gt += ((valid >> e) & 1u) && kk[e] > T;
        eq += ((valid >> e) & 1u) && kk[e] == T;
      }
    }
  }
  gt = __reduce_add_sync(kFull, gt);
  eq = __reduce_add_sync(kFull, eq);
  if (lane == 0) {
    s_wgt[wid] = gt;
    s_weq[wid] = eq;
  }
  __syncthreads();
  if (tid == 0) {
    int tg = 0, te = 0;
    for (int w = 0; w < NW; ++w) {
      tg += s_wgt[w];
      te += s_weq[w];
    }
    s_cnt[0] = tg;
    s_cnt[1] = te;
    s_cnt[2] = copy_ok ? 0 : 1;
  }
  cluster.sync();
  if (tid < 3 * CL) s_peer[tid] = *cluster.map_shared_rank(&s_cnt[tid % 3], tid / 3);  // one remote read each
  __syncthreads();
  bool any_fail = false;
  for (int r = 0; r < CL; ++r) any_fail |= s_peer[3 * r + 2] != 0;
  if (any_fail) {
    // a slice of this query is missing: no selection is reported for it
    if (rank == 0 && tid == 0) p.out_cnt[b] = 0;
    // a copy that gave up may still land: wait for it (bounded) before this CTA's memory is released
    if (!copy_ok && tid == 0) mbar_wait(&s_bar, 0u, nullptr);
    cluster.sync();  // peers may still read this CTA's shared memory
    return;
  }
  // ties are taken in index order: CTA r may take krem minus the ties of CTAs before it
  int eq_before = 0, sel_before = 0, take_eq = 0;
  for (int r = 0; r < CL; ++r) {
    const int g_r = s_peer[3 * r];
    const int e_r = s_peer[3 * r + 1];
    int t_r = krem - eq_before;
    t_r = t_r < 0 ? 0 : (t_r > e_r ? e_r : t_r);
    if (r < rank) {
      sel_before += g_r + t_r;
      eq_before += e_r;
    } else if (r == rank) {
      take_eq = t_r;
      break;
    }
  }
  // the same split inside the CTA, over its warps
  int w_eq_before = 0, w_sel_before = sel_before;
  for (int w = 0; w < wid; ++w) {
    int t_w = take_eq - w_eq_before;
    t_w = t_w < 0 ? 0 : (t_w > s_weq[w] ? s_weq[w] : t_w);
    w_sel_before += s_wgt[w] + t_w;
    w_eq_before += s_weq[w];
  }
  int run_eq = w_eq_before, run_sel = w_sel_before;
  if (listed) {
    for (int e0 = 0; e0 < nl; e0 += 32) {  // one list entry per lane, lanes in index order
      const int e = e0 + lane;
      const int pos = e < nl ? s_list[wid][e] : 0;
      const uint32_t key = e < nl ? f2key(__uint_as_float(s_keys[pos])) : 0u;
      const bool is_eq = e < nl && key == T;
      const unsigned meq = __ballot_sync(kFull, is_eq);
      const bool sel = (e < nl && key > T) || (is_eq && run_eq + __popc(meq & below) < take_eq);
      const unsigned msel = __ballot_sync(kFull, sel);
      const int at = run_sel + __popc(msel & below);
      if (sel && at < k) {
        oidx[at] = static_cast<int32_t>(lo + pos);
        if (osc) osc[at] = key2f(key);
      }
      run_eq += __popc(meq);
      run_sel += __popc(msel);
    }
  }
  for (int base = s_lo; base < s_hi && !listed; base += 128) {
    const int i = base + 4 * lane;
    uint32_t kk[4];
    unsigned valid;
    keys4(i, kk, valid);
    int e_l = 0, g_l = 0;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      e_l += ((valid >> e) & 1u) && kk[e] == T;
      g_l += ((valid >> e) & 1u) && kk[e] > T;
    }
    if (!__any_sync(kFull, (e_l | g_l) != 0)) continue;  // nothing chosen in these 128 keys
    int eq_rank = run_eq + warp_exclusive_scan(e_l, lane);
    bool sel[4];
    int s_l = 0;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const bool v = (valid >> e) & 1u;
      const bool is_eq = v && kk[e] == T;
      sel[e] = (v && kk[e] > T) || (is_eq && eq_rank < take_eq);
      eq_rank += is_eq;
      s_l += sel[e];
    }
    int at = run_sel + warp_exclusive_scan(s_l, lane);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      if (sel[e]) {
        if (at < k) {
          oidx[at] = static_cast<int32_t>(lo + i + e);
          if (osc) osc[at] = key2f(kk[e]);
        }
        ++at;
      }
    }
    run_eq += __reduce_add_sync(kFull, e_l);
    run_sel += __reduce_add_sync(kFull, s_l);
  }
  if (rank == 0 && tid == 0) p.out_cnt[b] = k;
  cluster.sync();  // peers may still read this CTA's shared memory
}

// Clusters of `cl` selection CTAs that can be resident at once on the current
// device, cached per (device, cl, shared memory); 0 if the shape cannot launch.
int max_active_clusters(int cl, size_t smem, const cudaLaunchConfig_t* cfg) {
  struct Entry {
    int dev, cl;
    size_t smem;
    int fit;
  };
  static std::mutex mu;
  static std::vector<Entry> cache;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  {
    std::lock_guard<std::mutex> lock(mu);
    for (const Entry& en : cache)
      if (en.dev == dev && en.cl == cl && en.smem == smem) return en.fit;
  }
  if (!cfg) return 0;
  int fit = 0;
  if (cudaOccupancyMaxActiveClusters(&fit, index_select_kernel, cfg) != cudaSuccess) {
    (void)cudaGetLastError();
    fit = 0;
  }
  std::lock_guard<std::mutex> lock(mu);
  cache.push_back({dev, cl, smem, fit});
  return fit;
}

template <int NCH, int NTH, int TPW, bool FP4>
cudaError_t launch_scan(IndexParams& p, int n_sm, cudaStream_t st) {
  auto kern = index_scan_kernel<NCH, NTH, TPW, FP4>;
  const size_t smem = sizeof(int) * (p.n_q + 1);
  const int64_t units_max = (visible_entries(p.max_pos, p.m, p.n_win) + 16 * TPW - 1) / (16 * TPW);
  const int64_t upper = units_max * p.n_q;
  const int warps = kScanThreads / 32;
  int64_t grid = (upper + warps - 1) / warps;
  if (grid > (int64_t)n_sm * 2) grid = (int64_t)n_sm * 2;
  if (grid < 1) grid = 1;
  kern<<<static_cast<int>(grid), kScanThreads, smem, st>>>(p);
  return cudaGetLastError();
}

template <int NCH, int NTH, bool FP4>
cudaError_t launch_scan_tma(IndexParams& p, int n_sm, cudaStream_t st) {
  CUtensorMap map;
  memset(&map, 0, sizeof(map));
  if (!FP4) {  // FP4 units are two plain bulk copies; bf16 rows go through a swizzled 2D map
    auto enc = tensor_map_encoder();
    if (!enc) return cudaErrorNotSupported;
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(p.d_idx), static_cast<cuuint64_t>(p.n_pages) * p.page_size};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(p.d_idx) * 2};
    const cuuint32_t box[2] = {64, kUnitKeys};
    const cuuint32_t estr[2] = {1, 1};
    if (enc(&map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(p.idx_pool), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  auto kern = index_scan_tma_kernel<NCH, NTH, FP4>;
  const size_t smem = TmaScanShape<NCH, FP4>::smem_bytes(p.n_q);
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  const int64_t units_max = (visible_entries(p.max_pos, p.m, p.n_win) + kUnitKeys - 1) / kUnitKeys;
  int64_t grid = units_max * p.n_q;
  if (grid > n_sm) grid = n_sm;
  if (grid < 1) grid = 1;
  return launch_pdl(kern, dim3(static_cast<unsigned>(grid)), dim3(kTmaThreads), smem, st, map, p);
}

template <int NCH, int HI>
cudaError_t launch_scan_group(IndexParams& p, int n_sm, cudaStream_t st) {
  auto enc = tensor_map_encoder();
  if (!enc) return cudaErrorNotSupported;
  CUtensorMap map;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(p.d_idx), static_cast<cuuint64_t>(p.n_pages) * p.page_size};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(p.d_idx) * 2};
  const cuuint32_t box[2] = {64, kUnitKeys};
  const cuuint32_t estr[2] = {1, 1};
  if (enc(&map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(p.idx_pool), dims, strides, box, estr,
          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  auto kern = index_scan_group_kernel<NCH, HI>;
  const size_t smem = 1024 + (size_t)kTmaRingBytes + 2 * TmaScanShape<NCH>::NSTAGE * sizeof(uint64_t) +
                      TmaScanShape<NCH>::NSTAGE * sizeof(int) + 2 * sizeof(int) * (size_t)(p.n_q + 1);
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  return launch_pdl(kern, dim3(static_cast<unsigned>(n_sm)), dim3(kTmaThreads), smem, st, map, p);
}

// ---------------------------------------------------------------- top-k for many queries
// One CTA of kStrThreads per query and ~25 KB of shared memory, so several queries share an SM
// and their score reads overlap (a prefill block has thousands of queries of ~10^4 scores each).
// The scores are streamed from global memory up to three times: the digit-A histogram (unless the
// scan left one), the gather of the threshold bin, and the ordered output. The digits, the tie rule
// (lower index first among keys equal to the k-th) and the ascending output are those of
// index_select_kernel.
constexpr int kStrThreads = 256;
constexpr int kStrCandCap = 4096;

// digit of the krem-th largest key from a histogram of nbins (nbins a multiple of kStrThreads)
template <typename CountFn>
__device__ __forceinline__ void find_digit_str(int nbins, int krem, CountFn count, int* s_w, uint32_t* s_res,
                                               uint32_t& digit, int& krem_out, int& bin_cnt) {
  const int per = nbins / kStrThreads;  // 4 or 8 bins per thread, from the top
  int tot = 0;
  for (int e = 0; e < per; ++e) tot += count(nbins - 1 - (threadIdx.x * per + e));
  int all;
  int run = block_exclusive_scan<kStrThreads>(tot, s_w, all);
  if (run < krem && krem <= run + tot) {
    for (int e = 0; e < per; ++e) {
      const int bin = nbins - 1 - (threadIdx.x * per + e);
      const int c = count(bin);
      if (run < krem && krem <= run + c) {
        s_res[0] = static_cast<uint32_t>(bin);
        s_res[1] = static_cast<uint32_t>(krem - run);
        s_res[2] = static_cast<uint32_t>(c);
      }
      run += c;
    }
  }
  __syncthreads();
  digit = s_res[0];
  krem_out = static_cast<int>(s_res[1]);
  bin_cnt = static_cast<int>(s_res[2]);
  __syncthreads();
}

// count digit (key >> shift) & dmask of the keys with (key & mask) == prefix; warp-aggregated
__device__ __forceinline__ void str_count(uint32_t key, bool valid, uint32_t mask, uint32_t prefix, int shift,
                                          uint32_t dmask, uint32_t* hist) {
  const bool ok = valid && (key & mask) == prefix;
  const unsigned act = __ballot_sync(kFull, ok);
  if (ok) {
    const uint32_t dg = (key >> shift) & dmask;
    const unsigned peers = __match_any_sync(act, dg);
    if ((threadIdx.x & 31) == __ffs(peers) - 1) atomicAdd(&hist[dg], static_cast<uint32_t>(__popc(peers)));
  }
}

__global__ void __launch_bounds__(kStrThreads) index_select_stream_kernel(IndexParams p) {
  __shared__ uint32_t s_h[kBinsA];          // digit histograms (A, then B, then C)
  __shared__ uint32_t s_cand[kStrCandCap];  // keys of the threshold bin of digit A
  __shared__ int s_w[32];
  __shared__ uint32_t s_res[3];
  __shared__ int s_n;
  const int b = blockIdx.x, tid = threadIdx.x, lane = tid & 31;
  const int k = p.k;
  if (tid == 0) s_res[0] = s_res[1] = s_res[2] = 0u;
  grid_dependency_wait();  // the scores (and the histogram, if any) come from the scan
  grid_dependents_launch();
  int64_t nv64 = query_visible(p, b);
  if (nv64 < 0) nv64 = 0;
  const int nv = static_cast<int>(nv64);
  const float* sc = p.scores + (int64_t)b * p.vis_stride;
  int32_t* oidx = p.out_idx + (int64_t)b * k;
  float* osc = p.out_scores ? p.out_scores + (int64_t)b * k : nullptr;
  if (nv <= k) {  // everything visible is chosen
    for (int i = tid; i < k; i += kStrThreads) {
      oidx[i] = i < nv ? i : -1;
      if (osc) osc[i] = i < nv ? sc[i] : 0.f;
    }
    if (tid == 0) p.out_cnt[b] = nv;
    return;
  }
  // one 4-key group per thread and step; the row is 256-byte aligned, the last 0..3 keys go alone
  const int n4 = nv >> 2;
  auto keys4 = [&](int g, uint32_t (&kk)[4], unsigned& valid) {
    if (g < n4) {
      const float4 v = __ldg(reinterpret_cast<const float4*>(sc) + g);
      kk[0] = f2key(v.x); kk[1] = f2key(v.y); kk[2] = f2key(v.z); kk[3] = f2key(v.w);
      valid = 15u;
    } else {
      valid = 0u;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int i = 4 * g + e;
        kk[e] = i < nv ? f2key(sc[i]) : 0u;
        valid |= (i < nv ? 1u : 0u) << e;
      }
    }
  };
  const int n_groups = (nv + 3) >> 2;
  const int n_steps = (n_groups + kStrThreads - 1) / kStrThreads;

  // digit A (bits 31..21)
  uint32_t dA = 0u;
  int krem = k, nA = 0;
  if (p.hist) {
    const uint32_t* gh = p.hist + (int64_t)b * kBinsA;
    find_digit_str(kBinsA, k, [&](int bin) { return static_cast<int>(gh[bin]); }, s_w, s_res, dA, krem, nA);
  } else {
    for (int i = tid; i < kBinsA; i += kStrThreads) s_h[i] = 0u;
    __syncthreads();
    for (int s = 0; s < n_steps; ++s) {
      const int g = s * kStrThreads + tid;
      uint32_t kk[4];
      unsigned valid = 0u;
      if (g < n_groups) keys4(g, kk, valid);
#pragma unroll
      for (int e = 0; e < 4; ++e) str_count(kk[e], (valid >> e) & 1u, 0u, 0u, 21, kBinsA - 1, s_h);
    }
    __syncthreads();
    find_digit_str(kBinsA, k, [&](int bin) { return static_cast<int>(s_h[bin]); }, s_w, s_res, dA, krem, nA);
  }
  uint32_t prefix = dA << 21, mask = 0xFFE00000u;
  uint32_t dB = 0u, dC = 0u;
  int nB = 0, nC = 0;
  if (nA <= kStrCandCap) {
    // the keys of bin dA into shared memory, then digits B and C over that list
    if (tid == 0) s_n = 0;
    __syncthreads();
    const unsigned below = (1u << lane) - 1u;
    for (int s = 0; s < n_steps; ++s) {
      const int g = s * kStrThreads + tid;
      uint32_t kk[4];
      unsigned valid = 0u;
      if (g < n_groups) keys4(g, kk, valid);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const bool cand = ((valid >> e) & 1u) && (kk[e] & mask) == prefix;
        const unsigned m = __ballot_sync(kFull, cand);
        if (m) {
          int at = 0;
          if (lane == __ffs(m) - 1) at = atomicAdd(&s_n, __popc(m));
          at = __shfl_sync(kFull, at, __ffs(m) - 1) + __popc(m & below);
          if (cand && at < kStrCandCap) s_cand[at] = kk[e];
        }
      }
    }
    for (int i = tid; i < kBinsB; i += kStrThreads) s_h[i] = 0u;
    __syncthreads();
    const int nc = s_n < kStrCandCap ? s_n : kStrCandCap;
    for (int i = tid; i < nc; i += kStrThreads)
      if ((s_cand[i] & mask) == prefix) atomicAdd(&s_h[(s_cand[i] >> 10) & (kBinsB - 1)], 1u);
    __syncthreads();
    find_digit_str(kBinsB, krem, [&](int bin) { return static_cast<int>(s_h[bin]); }, s_w, s_res, dB, krem, nB);
    prefix |= dB << 10;
    mask |= 0x001FFC00u;
    for (int i = tid; i < kBinsC; i += kStrThreads) s_h[i] = 0u;
    __syncthreads();
    for (int i = tid; i < nc; i += kStrThreads)
      if ((s_cand[i] & mask) == prefix) atomicAdd(&s_h[s_cand[i] & (kBinsC - 1)], 1u);
    __syncthreads();
    find_digit_str(kBinsC, krem, [&](int bin) { return static_cast<int>(s_h[bin]); }, s_w, s_res, dC, krem, nC);
  } else {
    // a threshold bin too large for the list: masked histogram passes over the scores
    for (int round = 0; round < 2; ++round) {
      const int shift = round == 0 ? 10 : 0;
      const int nb = round == 0 ? kBinsB : kBinsC;
      for (int i = tid; i < nb; i += kStrThreads) s_h[i] = 0u;
      __syncthreads();
      for (int s = 0; s < n_steps; ++s) {
        const int g = s * kStrThreads + tid;
        uint32_t kk[4];
        unsigned valid = 0u;
        if (g < n_groups) keys4(g, kk, valid);
#pragma unroll
        for (int e = 0; e < 4; ++e) str_count(kk[e], (valid >> e) & 1u, mask, prefix, shift, nb - 1, s_h);
      }
      __syncthreads();
      uint32_t d = 0u;
      int cnt = 0;
      find_digit_str(nb, krem, [&](int bin) { return static_cast<int>(s_h[bin]); }, s_w, s_res, d, krem, cnt);
      if (round == 0) {
        dB = d;
        prefix |= dB << 10;
        mask |= 0x001FFC00u;
      } else {
        dC = d;
      }
    }
  }
  const uint32_t T = prefix | dC;  // the k-th largest key; the first krem keys equal to T are taken

  // ordered output: per step, one scan of (keys above T, keys equal to T) packed in one int
  int written = 0, eq_seen = 0;
  for (int s = 0; s < n_steps; ++s) {
    const int g = s * kStrThreads + tid;
    uint32_t kk[4];
    unsigned valid = 0u;
    if (g < n_groups) keys4(g, kk, valid);
    int ngt = 0, neq = 0;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      ngt += ((valid >> e) & 1u) && kk[e] > T;
      neq += ((valid >> e) & 1u) && kk[e] == T;
    }
    int tot;
    const int ex = block_exclusive_scan<kStrThreads>(ngt | (neq << 16), s_w, tot);
    const int gt_ex = ex & 0xFFFF, eq_ex = ex >> 16;
    const int rem = krem - eq_seen > 0 ? krem - eq_seen : 0;  // equal keys still to take
    int pos = written + gt_ex + (eq_ex < rem ? eq_ex : rem);
    int eq_rank = eq_ex;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      if (!((valid >> e) & 1u)) continue;
      bool take = kk[e] > T;
      if (kk[e] == T) {
        take = eq_rank < rem;
        ++eq_rank;
      }
      if (take && pos < k) {
        oidx[pos] = 4 * g + e;
        if (osc) osc[pos] = key2f(kk[e]);
        ++pos;
      }
    }
    const int tot_gt = tot & 0xFFFF, tot_eq = tot >> 16;
    written += tot_gt + (tot_eq < rem ? tot_eq : rem);
    eq_seen += tot_eq;
  }
  if (tid == 0) p.out_cnt[b] = k;
}

cudaError_t launch_select_stream(IndexParams& p, cudaStream_t st) {
  return launch_pdl(index_select_stream_kernel, dim3(static_cast<unsigned>(p.n_q)), dim3(kStrThreads), 0, st, p);
}

}  // namespace

// cuTensorMapEncodeTiled through the runtime's driver entry point (no libcuda link)
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = []() {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return static_cast<PFN_cuTensorMapEncodeTiled_v12000>(nullptr);
    return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
  }();
  return fn;
}

size_t index_ws_bytes(int n_q, int64_t max_pos, int m, int n_win) {
  const int64_t nv = visible_entries(max_pos, m, n_win);
  const int64_t stride = (nv + 63) / 64 * 64;
  return (sizeof(float) * static_cast<size_t>(stride) + sizeof(uint32_t) * kHistBins) * static_cast<size_t>(n_q) + 256;
}

cudaError_t launch_index(IndexParams& p, void* ws, int n_sm, cudaStream_t st) {
  const int64_t nv_max = visible_entries(p.max_pos, p.m, p.n_win);
  p.vis_stride = (nv_max + 63) / 64 * 64;
  p.scores = static_cast<float*>(ws);
  p.hist = nullptr;
  if (p.n_q > kMaxQueries) return cudaErrorInvalidValue;
  cudaError_t e = cudaSuccess;
  const bool fp4 = p.idx_dtype == CSKV_FP4_E2M1;
  const int nth = (p.n_heads_idx + 7) / 8;
  const bool tma_ok = p.page_size % kUnitKeys == 0 && (p.d_idx == 64 || p.d_idx == 128) && nth <= 2 &&
                      (reinterpret_cast<uintptr_t>(p.idx_pool) & 15u) == 0 &&
                      (!fp4 || (reinterpret_cast<uintptr_t>(p.idx_scale) & 15u) == 0) &&
                      (int64_t)p.n_pages * p.page_size < (int64_t(1) << 31);
  // many queries in one call (a prefill chunk): the grouped scan reads each key once per group
  const bool grouped = tma_ok && !fp4 && p.n_q >= kGroupScanMinQueries && (p.n_heads_idx == 4 || p.n_heads_idx == 8);
  if (nv_max > 0 && grouped) {
    if (scan_tc_supported(p)) e = launch_scan_tc(p, n_sm, st);
    else if (p.d_idx == 64 && p.n_heads_idx == 4) e = launch_scan_group<2, 4>(p, n_sm, st);
    else if (p.d_idx == 64) e = launch_scan_group<2, 8>(p, n_sm, st);
    else if (p.n_heads_idx == 4) e = launch_scan_group<4, 4>(p, n_sm, st);
    else e = launch_scan_group<4, 8>(p, n_sm, st);
    if (e != cudaSuccess) return e;
  } else if (nv_max > 0 && tma_ok) {
    p.hist = reinterpret_cast<uint32_t*>(p.scores + (size_t)p.n_q * p.vis_stride);
    e = cudaMemsetAsync(p.hist, 0, sizeof(uint32_t) * kHistBins * (size_t)p.n_q, st);
    if (e != cudaSuccess) return e;
    if (fp4) {
      if (p.d_idx == 64 && nth == 1) e = launch_scan_tma<2, 1, true>(p, n_sm, st);
      else if (p.d_idx == 64 && nth == 2) e = launch_scan_tma<2, 2, true>(p, n_sm, st);
      else if (p.d_idx == 128 && nth == 1) e = launch_scan_tma<4, 1, true>(p, n_sm, st);
      else e = launch_scan_tma<4, 2, true>(p, n_sm, st);
    } else {
      if (p.d_idx == 64 && nth == 1) e = launch_scan_tma<2, 1, false>(p, n_sm, st);
      else if (p.d_idx == 64 && nth == 2) e = launch_scan_tma<2, 2, false>(p, n_sm, st);
      else if (p.d_idx == 128 && nth == 1) e = launch_scan_tma<4, 1, false>(p, n_sm, st);
      else e = launch_scan_tma<4, 2, false>(p, n_sm, st);
    }
    if (e != cudaSuccess) return e;
  } else if (nv_max > 0) {
    if (!fp4 && p.d_idx == 64 && nth == 1) e = launch_scan<2, 1, 2, false>(p, n_sm, st);
    else if (!fp4 && p.d_idx == 64 && nth == 2) e = launch_scan<2, 2, 2, false>(p, n_sm, st);
    else if (!fp4 && p.d_idx == 128 && nth == 1) e = launch_scan<4, 1, 1, false>(p, n_sm, st);
    else if (!fp4 && p.d_idx == 128 && nth == 2) e = launch_scan<4, 2, 1, false>(p, n_sm, st);
    else if (fp4 && p.d_idx == 64 && nth == 1) e = launch_scan<2, 1, 4, true>(p, n_sm, st);
    else if (fp4 && p.d_idx == 128 && nth == 1) e = launch_scan<4, 1, 4, true>(p, n_sm, st);
    else if (fp4 && p.d_idx == 128 && nth == 2) e = launch_scan<4, 2, 2, true>(p, n_sm, st);
    else return cudaErrorNotSupported;
    if (e != cudaSuccess) return e;
  }
  if (p.n_q == 0) return cudaSuccess;
  // many queries (a prefill block): one small CTA per query, several per SM
  if (p.n_q >= kStreamSelectMinQueries) return launch_select_stream(p, st);
  // selection: a cluster of CL CTAs per query, each holding a slice of scores
  int cl_min = static_cast<int>((nv_max + kSliceCap - 1) / kSliceCap);
  if (cl_min < 1) cl_min = 1;
  if (cl_min > kMaxCluster) return launch_select_stream(p, st);  // slices beyond a 16-CTA cluster
  int cl0 = n_sm / p.n_q;
  if (cl0 > kMaxCluster) cl0 = kMaxCluster;
  if (cl0 < cl_min) cl0 = cl_min;
  // no point in CTAs that would hold fewer than 4096 scores
  while (cl0 > cl_min && (nv_max + cl0 - 1) / cl0 < 4096) --cl0;
  e = cudaFuncSetAttribute(index_select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(sizeof(uint32_t) * (kSliceCap + 2 * kCandCap)));
  if (e != cudaSuccess) return e;
  if (cl0 > 8) {
    e = cudaFuncSetAttribute(index_select_kernel, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    if (e != cudaSuccess) return e;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.blockDim = dim3(kSelThreads, 1, 1);
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  // programmatic dependent launch: CTAs start on SMs the scan has left and wait
  // (griddepcontrol.wait) for its scores before reading them
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  auto shape = [&](int cl) {
    p.cluster = cl;
    p.slice = static_cast<int>(((nv_max + cl - 1) / cl + 3) / 4 * 4);
    if (p.slice < 4) p.slice = 4;
    cfg.gridDim = dim3(static_cast<unsigned>(p.n_q * cl), 1, 1);
    cfg.dynamicSmemBytes = sizeof(uint32_t) * (static_cast<size_t>(p.slice) + 2 * kCandCap);
    attr[0].val.clusterDim.x = static_cast<unsigned>(cl);
  };
  // The largest cluster, down from cl0, whose n_q clusters are all resident at
  // once (a second wave would double the time); clusters above 8 CTAs must fit
  // in one GPC, which not every GPC can host.
  int chosen = -1;
  for (int cl = cl0; cl >= cl_min && chosen < 0; --cl) {
    shape(cl);
    const int fit = max_active_clusters(cl, cfg.dynamicSmemBytes, &cfg);
    if (fit >= p.n_q) chosen = cl;
  }
  // no cluster size fits all queries in one wave (many long queries): the clusters run in waves
  // (one streaming CTA per query would stream the longest queries' scores too slowly)
  if (chosen < 0) {
    chosen = cl0 < 8 ? cl0 : (cl_min > 8 ? cl_min : 8);
    if (chosen > 8) {
      shape(chosen);
      if (max_active_clusters(chosen, cfg.dynamicSmemBytes, &cfg) < 1) return launch_select_stream(p, st);
    }
  }
  shape(chosen);
  return cudaLaunchKernelEx(&cfg, index_select_kernel, p);
}

}  // namespace cskv
