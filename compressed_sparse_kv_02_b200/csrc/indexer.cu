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

#include "cskv_device.cuh"
#include "cskv_internal.h"

namespace cg = cooperative_groups;

namespace cskv {
namespace {

constexpr int kScanThreads = 256;
constexpr int kMaxQueries = 4096;  // queries per call (prefix table in shared memory)
constexpr int kSelThreads = 1024;
constexpr int kSliceCap = 40960;   // scores per CTA of the selection kernel

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
      for (int r = 0; r < CL; ++r) cnt += static_cast<int>(*cluster.map_shared_rank(&s_hist[pass][bin], r));
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

  // per-CTA counts, exchanged across the cluster
  int gt = 0, eq = 0;
  for (int i = tid; i < len; i += kSelThreads) {
    gt += s_keys[i] > T;
    eq += s_keys[i] == T;
  }
  int tot;
  block_exclusive_scan<kSelThreads>(gt, s_w, tot);
  if (tid == 0) s_cnt[0] = tot;
  block_exclusive_scan<kSelThreads>(eq, s_w, tot);
  if (tid == 0) s_cnt[1] = tot;
  cluster.sync();
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
  int run_eq = 0, run_sel = 0;
  for (int base = 0; base < len; base += kSelThreads) {
    const int i = base + tid;
    const uint32_t key = i < len ? s_keys[i] : 0u;
    const int is_eq = i < len && key == T;
    int tot_eq;
    const int eq_rank = run_eq + block_exclusive_scan<kSelThreads>(is_eq, s_w, tot_eq);
    const int sel = (i < len && key > T) || (is_eq && eq_rank < take_eq);
    int tot_sel;
    const int at = run_sel + block_exclusive_scan<kSelThreads>(sel, s_w, tot_sel);
    if (sel && sel_before + at < k) {
      oidx[sel_before + at] = static_cast<int32_t>(lo + i);
      if (osc) osc[sel_before + at] = key2f(key);
    }
    run_eq += tot_eq;
    run_sel += tot_sel;
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
  if (nv_max > 0) {
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
  if (cl_min > 8) return cudaErrorNotSupported;
  int cl_par = n_sm / (p.n_q > 0 ? p.n_q : 1);
  if (cl_par > 8) cl_par = 8;
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
  return cudaLaunchKernelEx(&cfg, index_select_kernel, p);
}

}  // namespace cskv
