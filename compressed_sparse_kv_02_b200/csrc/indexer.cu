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
// query's scores in shared memory (one slice per CTA), runs a 4-pass 8-bit
// radix select on order-preserving integer keys with the per-CTA histograms
// summed through distributed shared memory, and writes the chosen indices in
// ascending order (equal scores prefer the lower index).
#include <cooperative_groups.h>
#include <cudaTypedefs.h>

#include "cskv_device.cuh"
#include "cskv_internal.h"

namespace cg = cooperative_groups;

namespace cskv {
namespace {

constexpr int kScanThreads = 256;
constexpr int kMaxQueries = 4096;  // queries per call (prefix table in shared memory)
constexpr int kSelThreads = 1024;
constexpr int kSliceCap = 40960;   // scores per CTA of the selection kernel
constexpr int kMaxCluster = 16;   // CTAs per query in the selection kernel (above 8: non-portable)

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
        if (j + g < nv) out[j + g] = s0;
        if (j + g + 8 < nv) out[j + g + 8] = s1;
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

template <int NCH>
struct TmaScanShape {
  static constexpr int ROWB = NCH * 64;                     // bytes per key row
  static constexpr int STAGE_BYTES = kUnitKeys * ROWB;      // one 64-key unit
  static constexpr int NSTAGE = kTmaRingBytes / STAGE_BYTES;  // even
  static size_t smem_bytes(int n_q) {
    return 1024 + (size_t)kTmaRingBytes + 2 * NSTAGE * sizeof(uint64_t) + NSTAGE * sizeof(int) +
           sizeof(int) * (size_t)(n_q + 1);
  }
};

template <int NCH, int NTH>
__global__ void __launch_bounds__(kTmaThreads, 1)
    index_scan_tma_kernel(const __grid_constant__ CUtensorMap tmap, IndexParams p) {
  using Sh = TmaScanShape<NCH>;
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
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

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
  const int64_t u_begin = total * blockIdx.x / gridDim.x;
  const int64_t n_units = total * (blockIdx.x + 1) / gridDim.x - u_begin;
  auto locate = [&](int64_t u, int& b, int64_t& j0) {
    int lo = 0, hi = p.n_q - 1;  // last b with s_pref[b] <= u
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (s_pref[mid] <= u) lo = mid; else hi = mid - 1;
    }
    b = lo;
    j0 = (u - s_pref[lo]) * kUnitKeys;
  };

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    // The warp resolves the pool rows of 32 units at a time (one page-table
    // load per lane, in parallel); lane 0 then issues their loads in order.
    if (lane == 0) prefetch_tensormap(&tmap);
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
        const uint16_t* qr = static_cast<const uint16_t*>(p.q_idx) + ((int64_t)b * p.n_heads_idx + n) * p.d_idx;
#pragma unroll
        for (int jj = 0; jj < NCH; ++jj)
          qf[nt][jj] = n < p.n_heads_idx ? ldg16(qr + (c + 4 * jj) * 8) : make_uint4(0u, 0u, 0u, 0u);
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
      }
      if (c == 0) {
        float* out = p.scores + (int64_t)b * p.vis_stride;
        if (j + pg < nv) out[j + pg] = s0;
        if (j + pg + 8 < nv) out[j + pg + 8] = s1;
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[s]);
  }
}

// ---------------------------------------------------------------- top-k
__device__ __forceinline__ int scan256_inclusive(int v, int* s_w) {
  // threads 0..255 participate; returns the inclusive prefix over them
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    int y = __shfl_up_sync(kFull, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) s_w[wid] = x;
  asm volatile("bar.sync 1, 256;\n" ::);
  int add = 0;
  for (int w = 0; w < wid; ++w) add += s_w[w];
  asm volatile("bar.sync 1, 256;\n" ::);
  return x + add;
}

__global__ void __launch_bounds__(kSelThreads, 1) index_select_kernel(IndexParams p) {
  cg::cluster_group cluster = cg::this_cluster();
  const int CL = p.cluster;
  const int rank = static_cast<int>(cluster.block_rank());
  const int b = blockIdx.x / CL;
  const int tid = threadIdx.x, lane = tid & 31;
  extern __shared__ uint32_t s_keys[];
  __shared__ uint32_t s_hist[4][256];
  __shared__ int s_w[32];
  __shared__ int s_cnt[2];
  __shared__ uint32_t s_digit;
  __shared__ int s_krem;

  const int k = p.k;
  int64_t nv = query_visible(p, b);
  if (nv < 0) nv = 0;
  const float* sc = p.scores + (int64_t)b * p.vis_stride;
  int32_t* oidx = p.out_idx + (int64_t)b * k;
  float* osc = p.out_scores ? p.out_scores + (int64_t)b * k : nullptr;

  if (nv <= k) {  // everything visible is chosen (uniform across the cluster)
    for (int64_t i = (int64_t)rank * kSelThreads + tid; i < k; i += (int64_t)CL * kSelThreads) {
      oidx[i] = i < nv ? static_cast<int32_t>(i) : -1;
      if (osc) osc[i] = i < nv ? sc[i] : 0.f;
    }
    if (rank == 0 && tid == 0) p.out_cnt[b] = static_cast<int32_t>(nv);
    return;
  }

  const int64_t lo = (int64_t)rank * p.slice;
  const int64_t hi = lo + p.slice < nv ? lo + p.slice : nv;
  const int len = hi > lo ? static_cast<int>(hi - lo) : 0;
  for (int i = tid; i < len; i += kSelThreads) s_keys[i] = f2key(sc[lo + i]);
  for (int i = tid; i < 4 * 256; i += kSelThreads) (&s_hist[0][0])[i] = 0u;
  __syncthreads();

  uint32_t prefix = 0u, mask = 0u;
  int krem = k;
  for (int pass = 0; pass < 4; ++pass) {
    const int shift = 24 - 8 * pass;
    for (int base = 0; base < len; base += kSelThreads) {
      const int i = base + tid;
      const uint32_t key = i < len ? s_keys[i] : 0u;
      const bool ok = i < len && (key & mask) == prefix;
      const uint32_t dg = (key >> shift) & 255u;
      const unsigned act = __ballot_sync(kFull, ok);
      if (ok) {
        const unsigned peers = __match_any_sync(act, dg);
        if (lane == __ffs(peers) - 1) atomicAdd(&s_hist[pass][dg], static_cast<uint32_t>(__popc(peers)));
      }
    }
    cluster.sync();
    if (tid < 256) {
      const int bin = 255 - tid;  // descending digit order
      int cnt = 0;
      uint32_t part[kMaxCluster];
#pragma unroll
      for (int r = 0; r < kMaxCluster; ++r)  // all remote loads in flight before the sum
        part[r] = r < CL ? *cluster.map_shared_rank(&s_hist[pass][bin], r) : 0u;
#pragma unroll
      for (int r = 0; r < kMaxCluster; ++r) cnt += static_cast<int>(part[r]);
      const int incl = scan256_inclusive(cnt, s_w);
      const int excl = incl - cnt;
      if (excl < krem && krem <= incl) {
        s_digit = static_cast<uint32_t>(bin);
        s_krem = krem - excl;
      }
    }
    __syncthreads();
    prefix |= s_digit << shift;
    mask |= 255u << shift;
    krem = s_krem;
    __syncthreads();
  }
  const uint32_t T = prefix;  // the k-th largest key; take the first krem keys equal to T

  // Ordered output. Warp w owns the contiguous segment [w*seg, (w+1)*seg) of
  // this CTA's slice. Pass 1 counts, per warp, keys above T and equal to T;
  // the counts are scanned over the warps of the CTA and then over the CTAs
  // of the cluster; pass 2 writes the chosen ids in index order.
  constexpr int NW = kSelThreads / 32;
  const int wid = tid >> 5;
  const int seg = ((len + NW - 1) / NW + 31) / 32 * 32;
  const int s_lo = wid * seg, s_hi = min(len, s_lo + seg);
  int gt = 0, eq = 0;
  for (int base = s_lo; base < s_hi; base += 32) {
    const int i = base + lane;
    const uint32_t key = i < s_hi ? s_keys[i] : 0u;
    gt += __popc(__ballot_sync(kFull, i < s_hi && key > T));
    eq += __popc(__ballot_sync(kFull, i < s_hi && key == T));
  }
  __shared__ int s_wgt[NW], s_weq[NW];
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
  }
  cluster.sync();
  // ties are taken in index order: CTA r may take krem minus the ties of CTAs before it
  int eq_before = 0, sel_before = 0, take_eq = 0;
  for (int r = 0; r < CL; ++r) {
    const int g_r = *cluster.map_shared_rank(&s_cnt[0], r);
    const int e_r = *cluster.map_shared_rank(&s_cnt[1], r);
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
  const unsigned lt = (1u << lane) - 1u;
  for (int base = s_lo; base < s_hi; base += 32) {
    const int i = base + lane;
    const uint32_t key = i < s_hi ? s_keys[i] : 0u;
    const unsigned m_eq = __ballot_sync(kFull, i < s_hi && key == T);
    const int eq_rank = run_eq + __popc(m_eq & lt);
    const bool sel = (i < s_hi && key > T) || ((m_eq >> lane) & 1u && eq_rank < take_eq);
    const unsigned m_sel = __ballot_sync(kFull, sel);
    const int at = run_sel + __popc(m_sel & lt);
    if (sel && at < k) {
      oidx[at] = static_cast<int32_t>(lo + i);
      if (osc) osc[at] = key2f(key);
    }
    run_eq += __popc(m_eq);
    run_sel += __popc(m_sel);
  }
  if (rank == 0 && tid == 0) p.out_cnt[b] = k;
  cluster.sync();  // peers may still read this CTA's shared memory
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

template <int NCH, int NTH>
cudaError_t launch_scan_tma(IndexParams& p, int n_sm, cudaStream_t st) {
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
  auto kern = index_scan_tma_kernel<NCH, NTH>;
  const size_t smem = TmaScanShape<NCH>::smem_bytes(p.n_q);
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  const int64_t units_max = (visible_entries(p.max_pos, p.m, p.n_win) + kUnitKeys - 1) / kUnitKeys;
  int64_t grid = units_max * p.n_q;
  if (grid > n_sm) grid = n_sm;
  if (grid < 1) grid = 1;
  kern<<<static_cast<int>(grid), kTmaThreads, smem, st>>>(map, p);
  return cudaGetLastError();
}

}  // namespace

size_t index_ws_bytes(int n_q, int64_t max_pos, int m, int n_win) {
  const int64_t nv = visible_entries(max_pos, m, n_win);
  const int64_t stride = (nv + 63) / 64 * 64;
  return sizeof(float) * static_cast<size_t>(stride) * static_cast<size_t>(n_q) + 256;
}

cudaError_t launch_index(IndexParams& p, void* ws, int n_sm, cudaStream_t st) {
  const int64_t nv_max = visible_entries(p.max_pos, p.m, p.n_win);
  p.vis_stride = (nv_max + 63) / 64 * 64;
  p.scores = static_cast<float*>(ws);
  if (p.n_q > kMaxQueries) return cudaErrorInvalidValue;
  cudaError_t e = cudaSuccess;
  const bool fp4 = p.idx_dtype == CSKV_FP4_E2M1;
  const int nth = (p.n_heads_idx + 7) / 8;
  const bool tma_ok = !fp4 && p.page_size % kUnitKeys == 0 && (p.d_idx == 64 || p.d_idx == 128) && nth <= 2 &&
                      (reinterpret_cast<uintptr_t>(p.idx_pool) & 15u) == 0 &&
                      (int64_t)p.n_pages * p.page_size < (int64_t(1) << 31);
  if (nv_max > 0 && tma_ok) {
    if (p.d_idx == 64 && nth == 1) e = launch_scan_tma<2, 1>(p, n_sm, st);
    else if (p.d_idx == 64 && nth == 2) e = launch_scan_tma<2, 2>(p, n_sm, st);
    else if (p.d_idx == 128 && nth == 1) e = launch_scan_tma<4, 1>(p, n_sm, st);
    else e = launch_scan_tma<4, 2>(p, n_sm, st);
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
  // selection: a cluster of CL CTAs per query, each holding a slice of scores
  int cl_min = static_cast<int>((nv_max + kSliceCap - 1) / kSliceCap);
  if (cl_min < 1) cl_min = 1;
  if (cl_min > kMaxCluster) return cudaErrorNotSupported;
  int cl_par = n_sm / (p.n_q > 0 ? p.n_q : 1);
  if (cl_par > kMaxCluster) cl_par = kMaxCluster;
  int cl = cl_min > cl_par ? cl_min : cl_par;
  if (cl < 1) cl = 1;
  // no point in CTAs that would hold fewer than 4096 scores
  while (cl > cl_min && (nv_max + cl - 1) / cl < 4096) --cl;
  p.cluster = cl;
  p.slice = static_cast<int>(((nv_max + cl - 1) / cl + 3) / 4 * 4);
  if (p.slice < 4) p.slice = 4;
  const size_t smem = sizeof(uint32_t) * static_cast<size_t>(p.slice);
  e = cudaFuncSetAttribute(index_select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  if (cl > 8) {
    e = cudaFuncSetAttribute(index_select_kernel, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    if (e != cudaSuccess) return e;
  }
  if (p.n_q == 0) return cudaSuccess;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(p.n_q * cl), 1, 1);
  cfg.blockDim = dim3(kSelThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = static_cast<unsigned>(cl);
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cl > 8) {  // a non-portable cluster must fit in one GPC; else fall back to 8
    int n_clusters = 0;
    if (cudaOccupancyMaxActiveClusters(&n_clusters, index_select_kernel, &cfg) != cudaSuccess || n_clusters < 1) {
      (void)cudaGetLastError();
      if (cl_min > 8) return cudaErrorNotSupported;
      cl = 8;
      p.cluster = cl;
      p.slice = static_cast<int>(((nv_max + cl - 1) / cl + 3) / 4 * 4);
      cfg.gridDim = dim3(static_cast<unsigned>(p.n_q * cl), 1, 1);
      cfg.dynamicSmemBytes = sizeof(uint32_t) * static_cast<size_t>(p.slice);
      attr[0].val.clusterDim.x = static_cast<unsigned>(cl);
      e = cudaFuncSetAttribute(index_select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               static_cast<int>(cfg.dynamicSmemBytes));
      if (e != cudaSuccess) return e;
    }
  }
  return cudaLaunchKernelEx(&cfg, index_select_kernel, p);
}

}  // namespace cskv
