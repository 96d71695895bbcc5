// attend.cu -- core attention of a CSA or HCA layer for decode-sized query
// batches (DeepSeek-V4 report digest, section 3: one softmax over the last
// n_win = 128 raw tokens and the top-k entries (CSA) or all heavy entries
// (HCA); DeepSeek-V4-book ch.1, section 4: every head reads one shared latent
// KV, MLA/MQA style).
//
// Key list of query (b, t): u < n_w are the window tokens max(0,t-n_win+1)..t
// (from the state-cache ring, or the prefill chunk), then the compressed
// entries (the CSA selection in index order, or every visible HCA entry).
// K_u is the whole stored vector (d_qk), V_u its first d_v channels, so one
// shared-memory tile serves both products.
//
// Work item = (query, head group of 16*MT heads, key split). A CTA stages the
// head group's queries and 32-key tiles in shared memory (cp.async, double
// buffered, gathered through the page table), computes S = Q K^T and O += P V
// with mma.sync m16n8k16 (heads as M), keeps the softmax online in fp32, and
// writes the split's normalised partial output and log-sum-exp; a merge
// kernel combines the splits (log-sum-exp weighting) into bf16 output.
// FP8 entries are staged as bytes, widened to bf16 in shared memory (exact),
// and their per-entry scale is applied to the logits and to P.
#include "cskv_device.cuh"
#include "cskv_internal.h"

namespace cskv {
namespace {

constexpr int KT = 32;  // keys per tile
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr int kMaxQ = 4096;

struct QueryKeys {
  int64_t t, ws;
  int n_w;
  int64_t n_c;
  int64_t n;  // total keys
};

__device__ __forceinline__ QueryKeys query_keys(const AttendParams& p, int b) {
  QueryKeys r;
  r.t = p.q_pos[b];
  if (r.t < 0 || r.t > p.max_pos) {
    r.n_w = 0;
    r.n_c = 0;
    r.n = 0;
    r.ws = 0;
    return r;
  }
  r.ws = window_start(r.t, p.n_win);
  r.n_w = static_cast<int>(r.t - r.ws + 1);
  if (p.is_csa) {
    int64_t c = p.sel_cnt[b];
    r.n_c = c < 0 ? 0 : (c > p.k ? p.k : c);
  } else {
    r.n_c = visible_entries(r.t, p.m, p.n_win);
  }
  r.n = r.n_w + r.n_c;
  return r;
}

// source row of key u of query b; bit 0 of the returned address flags an FP8
// entry (all rows are 16-byte aligned). Returns 0 for an invalid row.
__device__ __forceinline__ uintptr_t key_row(const AttendParams& p, int b, int seq,
                                             const QueryKeys& qk, int64_t u, float& scale) {
  scale = 1.f;
  if (u < qk.n_w) {
    const int64_t pos = qk.ws + u;
    const int64_t cr = chunk_row(p, seq, pos);
    if (cr >= 0) return reinterpret_cast<uintptr_t>(p.x_chunk + cr * p.d_qk);
    return reinterpret_cast<uintptr_t>(p.ring_x + ((int64_t)seq * p.n_win + pos % p.n_win) * p.d_qk);
  }
  const int64_t jj = u - qk.n_w;
  const int64_t j = p.is_csa ? static_cast<int64_t>(p.sel_idx[(int64_t)b * p.k + jj]) : jj;
  const int64_t nvis = visible_entries(qk.t, p.m, p.n_win);
  if (j < 0 || j >= nvis) return 0;
  const int64_t pi = j / p.page_size;
  if (pi >= p.max_pages_per_seq) return 0;
  const int32_t page = p.page_table[(int64_t)seq * p.max_pages_per_seq + pi];
  if (page < 0 || page >= p.n_pages) return 0;
  const int64_t row = (int64_t)page * p.page_size + (j % p.page_size);
  if (p.kv_dtype == CSKV_FP8_E4M3) {
    scale = p.kv_scale[row];
    return reinterpret_cast<uintptr_t>(static_cast<const uint8_t*>(p.kv_pool) + row * p.d_qk) | 1u;
  }
  return reinterpret_cast<uintptr_t>(static_cast<const uint16_t*>(p.kv_pool) + row * p.d_qk);
}

template <int DQK, int MT>
struct AttnSmem {
  static constexpr int SROW = DQK + 8;  // padded row: ldmatrix rows fall in distinct banks
  static constexpr int HG = 16 * MT;
  static size_t bytes(int n_q, int kps, bool fp8) {
    size_t s = sizeof(uint16_t) * (size_t)(HG + 2 * KT) * SROW;
    if (fp8) s += (size_t)2 * KT * DQK;
    s += (sizeof(uintptr_t) + sizeof(float)) * (size_t)kps;
    s += sizeof(int) * (size_t)(n_q + 1);
    return s;
  }
};

template <int DQK, int DV, int MT, int VS, bool FP8>
__global__ void __launch_bounds__(32 * MT * VS) attend_kernel(AttendParams p) {
  constexpr int NW = MT * VS, NTH = 32 * NW;
  constexpr int HG = 16 * MT, DVW = DV / VS;
  constexpr int SROW = AttnSmem<DQK, MT>::SROW;
  constexpr int CPR = DQK / 8;    // 16-byte chunks per bf16 row
  constexpr int CPR8 = DQK / 16;  // 16-byte chunks per FP8 row
  constexpr bool HOIST_Q = DQK <= 256;
  static_assert(DV % (16 * VS) == 0 && DQK % 16 == 0, "shape");

  extern __shared__ __align__(16) uint8_t smem[];
  uint16_t* sQ = reinterpret_cast<uint16_t*>(smem);
  uint16_t* sK = sQ + HG * SROW;  // [2][KT][SROW]
  uint8_t* sK8 = reinterpret_cast<uint8_t*>(sK + 2 * KT * SROW);  // [2][KT][DQK] (FP8)
  uintptr_t* sPtr = reinterpret_cast<uintptr_t*>(sK8 + (FP8 ? 2 * KT * DQK : 0));
  float* sSc = reinterpret_cast<float*>(sPtr + p.keys_per_split);
  int* sPref = reinterpret_cast<int*>(sSc + p.keys_per_split);
  __shared__ int s_wsum[32];

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int mt = warp % MT, vs = warp / MT;
  const int g = lane >> 2, c = lane & 3;
  const int n_groups = p.n_heads / HG;
  const int kps = p.keys_per_split;

  // items per query: splits * head groups; exclusive prefix in shared memory
  {
    int run = 0;
    for (int base = 0; base < p.n_q; base += NTH) {
      const int b = base + tid;
      int v = 0;
      if (b < p.n_q) {
        const QueryKeys qk = query_keys(p, b);
        v = static_cast<int>((qk.n + kps - 1) / kps) * n_groups;
      }
      int tot;
      const int ex = block_exclusive_scan<NTH>(v, s_wsum, tot);
      if (b < p.n_q) sPref[b] = run + ex;
      run += tot;
    }
    if (tid == 0) sPref[p.n_q] = run;
    __syncthreads();
  }
  if (blockIdx.x == 0)
    for (int b = tid; b < p.n_q; b += NTH)
      if (p.q_pos[b] < 0 || p.q_pos[b] > p.max_pos) report(p.status, CSKV_ERR_INVALID_ARG);
  const int total = sPref[p.n_q];

  for (int item = blockIdx.x; item < total; item += gridDim.x) {
    int lo = 0, hi = p.n_q - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (sPref[mid] <= item) lo = mid; else hi = mid - 1;
    }
    const int b = lo;
    const int r = item - sPref[b];
    const int split = r / n_groups, grp = r % n_groups;
    const QueryKeys qk = query_keys(p, b);
    const int seq = p.q_seq[b];
    const int64_t u0 = (int64_t)split * kps;
    const int nk = static_cast<int>((qk.n - u0) < kps ? (qk.n - u0) : kps);
    const bool seq_ok = seq >= 0 && seq < p.n_seqs_layer;

    for (int i = tid; i < nk; i += NTH) {
      float sc = 1.f;
      uintptr_t a = seq_ok ? key_row(p, b, seq, qk, u0 + i, sc) : 0;
      if (a == 0) report(p.status, CSKV_ERR_OUT_OF_RANGE);
      sPtr[i] = a;
      sSc[i] = sc;
    }
    for (int id = tid; id < HG * CPR; id += NTH) {
      const int rr = id / CPR, ch = id % CPR;
      const int h = grp * HG + rr;
      cp_async16(sQ + rr * SROW + ch * 8, p.q + ((int64_t)b * p.n_heads + h) * DQK + ch * 8, 16);
    }
    __syncthreads();  // sPtr ready

    auto issue_tile = [&](int it, int buf) {
      uint16_t* dst = sK + buf * KT * SROW;
      uint8_t* dst8 = sK8 + buf * KT * DQK;
      for (int id = tid; id < KT * CPR; id += NTH) {
        const int rr = id / CPR, ch = id % CPR;
        const int i = it * KT + rr;
        uintptr_t a = i < nk ? sPtr[i] : 0;
        if (FP8 && (a & 1u)) {
          if (ch < CPR8) cp_async16(dst8 + rr * DQK + ch * 16, reinterpret_cast<const void*>((a & ~uintptr_t(1)) + ch * 16), 16);
        } else {
          const bool ok = a != 0;
          const void* src = ok ? reinterpret_cast<const void*>(a + ch * 16) : static_cast<const void*>(p.q);
          cp_async16(dst + rr * SROW + ch * 8, src, ok ? 16 : 0);
        }
      }
      cp_async_commit();
    };

    const int ntiles = (nk + KT - 1) / KT;
    if (ntiles > 0) issue_tile(0, 0);

    float m_run[2] = {-INFINITY, -INFINITY}, l_run[2] = {0.f, 0.f};
    float oacc[DVW / 8][4];
#pragma unroll
    for (int i = 0; i < DVW / 8; ++i) oacc[i][0] = oacc[i][1] = oacc[i][2] = oacc[i][3] = 0.f;
    uint32_t qa[HOIST_Q ? DQK / 16 : 1][4];
    const float sl2 = p.sm_scale * kLog2e;

    for (int it = 0; it < ntiles; ++it) {
      const int buf = it & 1;
      if (it + 1 < ntiles) {
        issue_tile(it + 1, buf ^ 1);
        cp_async_wait<1>();
      } else {
        cp_async_wait<0>();
      }
      __syncthreads();
      const uint16_t* Kb = sK + buf * KT * SROW;
      if constexpr (FP8) {
        // widen FP8 rows of this tile to bf16 (exact) in place of the bf16 tile
        const uint8_t* K8 = sK8 + buf * KT * DQK;
        uint16_t* Kw = sK + buf * KT * SROW;
        for (int id = tid; id < KT * (DQK / 2); id += NTH) {
          const int rr = id / (DQK / 2), e2 = id % (DQK / 2);
          const int i = it * KT + rr;
          if (i < nk && (sPtr[i] & 1u)) {
            const __nv_fp8x2_storage_t v = *reinterpret_cast<const uint16_t*>(K8 + rr * DQK + 2 * e2);
            const __half2 h = __half2(__nv_cvt_fp8x2_to_halfraw2(v, __NV_E4M3));
            const float2 f = __half22float2(h);
            *reinterpret_cast<uint32_t*>(Kw + rr * SROW + 2 * e2) = pack_bf16(f.x, f.y);
          }
        }
        __syncthreads();
      }
      if (HOIST_Q && it == 0) {
#pragma unroll
        for (int ks = 0; ks < (HOIST_Q ? DQK / 16 : 1); ++ks)
          ldmatrix_x4(qa[ks], sQ + (mt * 16 + (lane & 15)) * SROW + ks * 16 + (lane >> 4) * 8);
      }
      // S = Q K^T for this warp's 16 heads and the tile's 32 keys
      float sacc[KT / 8][4];
#pragma unroll
      for (int i = 0; i < KT / 8; ++i) sacc[i][0] = sacc[i][1] = sacc[i][2] = sacc[i][3] = 0.f;
#pragma unroll
      for (int ks = 0; ks < DQK / 16; ++ks) {
        uint32_t a[4];
        if constexpr (HOIST_Q) {
          a[0] = qa[ks][0]; a[1] = qa[ks][1]; a[2] = qa[ks][2]; a[3] = qa[ks][3];
        } else {
          ldmatrix_x4(a, sQ + (mt * 16 + (lane & 15)) * SROW + ks * 16 + (lane >> 4) * 8);
        }
#pragma unroll
        for (int np = 0; np < KT / 16; ++np) {
          uint32_t bb[4];
          ldmatrix_x4(bb, Kb + (np * 16 + (lane >> 4) * 8 + (lane & 7)) * SROW + ks * 16 + ((lane >> 3) & 1) * 8);
          mma_bf16(sacc[2 * np], a, bb[0], bb[1]);
          mma_bf16(sacc[2 * np + 1], a, bb[2], bb[3]);
        }
      }
      // online softmax (rows g and g+8), base-2 domain
      float pr[KT / 8][4];
      float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
      for (int nt = 0; nt < KT / 8; ++nt) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int i = it * KT + nt * 8 + 2 * c + (e & 1);
          float v = -INFINITY;  // keys past the split or without a valid row are masked
          if (i < nk && sPtr[i] != 0) v = sacc[nt][e] * sl2 * (FP8 ? sSc[i] : 1.f);
          pr[nt][e] = v;
          mx[e >> 1] = fmaxf(mx[e >> 1], v);
        }
      }
      float corr[2], msub[2];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        mx[h] = fmaxf(mx[h], __shfl_xor_sync(kFull, mx[h], 1));
        mx[h] = fmaxf(mx[h], __shfl_xor_sync(kFull, mx[h], 2));
        const float mnew = fmaxf(m_run[h], mx[h]);
        msub[h] = mnew == -INFINITY ? 0.f : mnew;
        corr[h] = exp2f(m_run[h] - msub[h]);
        m_run[h] = mnew;
        l_run[h] *= corr[h];
      }
#pragma unroll
      for (int nt = 0; nt < KT / 8; ++nt) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float pv = exp2f(pr[nt][e] - msub[e >> 1]);
          l_run[e >> 1] += pv;
          const int i = it * KT + nt * 8 + 2 * c + (e & 1);
          pr[nt][e] = FP8 ? pv * (i < nk ? sSc[i] : 0.f) : pv;
        }
      }
#pragma unroll
      for (int i = 0; i < DVW / 8; ++i) {
        oacc[i][0] *= corr[0];
        oacc[i][1] *= corr[0];
        oacc[i][2] *= corr[1];
        oacc[i][3] *= corr[1];
      }
      // O += P V (V = the first d_v channels of the same tile)
#pragma unroll
      for (int kk = 0; kk < KT / 16; ++kk) {
        const uint32_t a[4] = {pack_bf16(pr[2 * kk][0], pr[2 * kk][1]), pack_bf16(pr[2 * kk][2], pr[2 * kk][3]),
                               pack_bf16(pr[2 * kk + 1][0], pr[2 * kk + 1][1]),
                               pack_bf16(pr[2 * kk + 1][2], pr[2 * kk + 1][3])};
#pragma unroll
        for (int nd = 0; nd < DVW / 16; ++nd) {
          uint32_t bb[4];
          ldmatrix_x4_trans(bb, Kb + (kk * 16 + (lane & 7) + ((lane >> 3) & 1) * 8) * SROW + vs * DVW + nd * 16 +
                                    (lane >> 4) * 8);
          mma_bf16(oacc[2 * nd], a, bb[0], bb[1]);
          mma_bf16(oacc[2 * nd + 1], a, bb[2], bb[3]);
        }
      }
      __syncthreads();  // the buffer is refilled two tiles later
    }

    // finalise this split: normalised partial output and its log-sum-exp
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      l_run[h] += __shfl_xor_sync(kFull, l_run[h], 1);
      l_run[h] += __shfl_xor_sync(kFull, l_run[h], 2);
    }
    const int head0 = grp * HG + mt * 16 + g;
    const int64_t prow0 = ((int64_t)b * p.max_splits + split) * p.n_heads + head0;
    const int64_t prow1 = prow0 + 8;
    const float inv0 = l_run[0] > 0.f ? 1.f / l_run[0] : 0.f;
    const float inv1 = l_run[1] > 0.f ? 1.f / l_run[1] : 0.f;
#pragma unroll
    for (int nt = 0; nt < DVW / 8; ++nt) {
      const int col = vs * DVW + nt * 8 + 2 * c;
      *reinterpret_cast<float2*>(p.part_o + prow0 * DV + col) = make_float2(oacc[nt][0] * inv0, oacc[nt][1] * inv0);
      *reinterpret_cast<float2*>(p.part_o + prow1 * DV + col) = make_float2(oacc[nt][2] * inv1, oacc[nt][3] * inv1);
    }
    if (vs == 0 && c == 0) {
      p.part_lse[prow0] = l_run[0] > 0.f ? (m_run[0] + log2f(l_run[0])) * kLn2 : -INFINITY;
      p.part_lse[prow1] = l_run[1] > 0.f ? (m_run[1] + log2f(l_run[1])) * kLn2 : -INFINITY;
    }
    __syncthreads();  // shared memory is reused by the next item
  }
}

// out[b,h,:] = sum_s exp(lse_s - L) o_s,  L = log sum_s exp(lse_s)
// d_v / 4 threads per head, four channels each; the split loop issues eight
// independent loads at a time.
__global__ void __launch_bounds__(256) attend_merge_kernel(AttendParams p) {
  const int b = blockIdx.x;
  const QueryKeys qk = query_keys(p, b);
  const int ns = static_cast<int>((qk.n + p.keys_per_split - 1) / p.keys_per_split);
  const int hb = blockDim.x / (p.d_v / 4);  // heads per pass: d_v/4 threads per head
  const int hl = threadIdx.x / (p.d_v / 4);
  const int c4 = (threadIdx.x % (p.d_v / 4)) * 4;
  for (int h = blockIdx.y * hb + hl; h < p.n_heads && hl < hb; h += gridDim.y * hb) {
    const int64_t base = (int64_t)b * p.max_splits * p.n_heads + h;
    float L = -INFINITY;
    for (int s = 0; s < ns; ++s) L = fmaxf(L, p.part_lse[base + (int64_t)s * p.n_heads]);
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    float wsum = 0.f;
    if (L != -INFINITY) {
      for (int s0 = 0; s0 < ns; s0 += 8) {
        float wg[8];
        float4 o[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const int s = s0 + j;
          wg[j] = 0.f;
          o[j] = make_float4(0.f, 0.f, 0.f, 0.f);
          if (s < ns) {
            wg[j] = expf(p.part_lse[base + (int64_t)s * p.n_heads] - L);
            o[j] = *reinterpret_cast<const float4*>(p.part_o + (base + (int64_t)s * p.n_heads) * p.d_v + c4);
          }
        }
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          wsum += wg[j];
          acc[0] += wg[j] * o[j].x;
          acc[1] += wg[j] * o[j].y;
          acc[2] += wg[j] * o[j].z;
          acc[3] += wg[j] * o[j].w;
        }
      }
    }
    const float inv = wsum > 0.f ? 1.f / wsum : 0.f;
    float v[4] = {acc[0] * inv, acc[1] * inv, acc[2] * inv, acc[3] * inv};
    inverse_rope4(v, c4, p.d_v, p.rope_dims, p.rope_base, p.q_pos[b]);
    uint2 packed = make_uint2(pack_bf16(v[0], v[1]), pack_bf16(v[2], v[3]));
    *reinterpret_cast<uint2*>(p.out + ((int64_t)b * p.n_heads + h) * p.d_v + c4) = packed;
    if (p.lse && c4 == 0) p.lse[(int64_t)b * p.n_heads + h] = wsum > 0.f ? L + logf(wsum) : -INFINITY;
  }
}

// The same merge over head-minor partial outputs ([query x split][d_v / 4][heads][4],
// written by attend_tc_kernel): a CTA takes 128 consecutive heads x 2 groups of 4
// channels, so every partial-output load is a warp's 512 contiguous bytes.
constexpr int kMergeRegSplits = 12;  // splits merged from registers in one batch of loads

__global__ void __launch_bounds__(256) attend_merge_t_kernel(AttendParams p) {
  grid_dependency_wait();  // the partial outputs come from the attention kernel ahead of this one
  grid_dependents_launch();
  const int b = blockIdx.x;
  const QueryKeys qk = query_keys(p, b);
  const int ns = static_cast<int>((qk.n + p.keys_per_split - 1) / p.keys_per_split);
  const int h = blockIdx.z * 128 + (threadIdx.x & 127);
  const int g4 = blockIdx.y * 2 + (threadIdx.x >> 7);  // group of 4 output channels
  if (h >= p.n_heads || g4 >= p.d_v / 4) return;
  const int64_t lbase = (int64_t)b * p.max_splits * p.n_heads + h;
  const float4* po = reinterpret_cast<const float4*>(p.part_o);
  float acc[4] = {0.f, 0.f, 0.f, 0.f};
  float wsum = 0.f;
  float L = -INFINITY;
  if (ns <= kMergeRegSplits) {
    // every split's log-sum-exp and partial output are loaded in one batch
    float ls[kMergeRegSplits];
    float4 o[kMergeRegSplits];
#pragma unroll
    for (int s = 0; s < kMergeRegSplits; ++s) {
      ls[s] = -INFINITY;
      o[s] = make_float4(0.f, 0.f, 0.f, 0.f);
      if (s < ns) {
        ls[s] = p.part_lse[lbase + (int64_t)s * p.n_heads];
        o[s] = po[(((int64_t)b * p.max_splits + s) * (p.d_v / 4) + g4) * p.n_heads + h];
      }
    }
#pragma unroll
    for (int s = 0; s < kMergeRegSplits; ++s) L = fmaxf(L, ls[s]);
    if (L != -INFINITY) {
#pragma unroll
      for (int s = 0; s < kMergeRegSplits; ++s) {
        const float wg = s < ns ? expf(ls[s] - L) : 0.f;
        wsum += wg;
        acc[0] += wg * o[s].x;
        acc[1] += wg * o[s].y;
        acc[2] += wg * o[s].z;
        acc[3] += wg * o[s].w;
      }
    }
  } else {
    for (int s = 0; s < ns; ++s) L = fmaxf(L, p.part_lse[lbase + (int64_t)s * p.n_heads]);
    if (L != -INFINITY) {
      for (int s0 = 0; s0 < ns; s0 += 8) {
        float wg[8];
        float4 o[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const int s = s0 + j;
          wg[j] = 0.f;
          o[j] = make_float4(0.f, 0.f, 0.f, 0.f);
          if (s < ns) {
            wg[j] = expf(p.part_lse[lbase + (int64_t)s * p.n_heads] - L);
            o[j] = po[(((int64_t)b * p.max_splits + s) * (p.d_v / 4) + g4) * p.n_heads + h];
          }
        }
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          wsum += wg[j];
          acc[0] += wg[j] * o[j].x;
          acc[1] += wg[j] * o[j].y;
          acc[2] += wg[j] * o[j].z;
          acc[3] += wg[j] * o[j].w;
        }
      }
    }
  }
  const float inv = wsum > 0.f ? 1.f / wsum : 0.f;
  float v[4] = {acc[0] * inv, acc[1] * inv, acc[2] * inv, acc[3] * inv};
  inverse_rope4(v, g4 * 4, p.d_v, p.rope_dims, p.rope_base, p.q_pos[b]);
  const uint2 packed = make_uint2(pack_bf16(v[0], v[1]), pack_bf16(v[2], v[3]));
  *reinterpret_cast<uint2*>(p.out + ((int64_t)b * p.n_heads + h) * p.d_v + g4 * 4) = packed;
  if (p.lse && g4 == 0) p.lse[(int64_t)b * p.n_heads + h] = wsum > 0.f ? L + logf(wsum) : -INFINITY;
}

struct Plan {
  int mt, vs;
};

template <int DQK, int DV, int MT, int VS, bool FP8>
cudaError_t run_attend(AttendParams& p, int n_sm, cudaStream_t st) {
  auto kern = attend_kernel<DQK, DV, MT, VS, FP8>;
  const size_t smem = AttnSmem<DQK, MT>::bytes(p.n_q, p.keys_per_split, FP8);
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  int per_sm = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, 32 * MT * VS, smem);
  if (e != cudaSuccess) return e;
  if (per_sm < 1) return cudaErrorInvalidConfiguration;
  const int64_t groups = p.n_heads / (16 * MT);
  const int64_t upper = (int64_t)p.n_q * p.max_splits * groups;
  int64_t grid = (int64_t)n_sm * per_sm;
  if (grid > upper) grid = upper;
  if (grid < 1) grid = 1;
  kern<<<static_cast<int>(grid), 32 * MT * VS, smem, st>>>(p);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  return launch_attend_merge(p, st);
}

// heads per CTA for each supported shape
Plan plan_for(int d_qk, int d_v, int n_heads) {
  if (d_qk == 128 && d_v == 128) {
    if (n_heads % 32 == 0) return {2, 1};
    if (n_heads % 16 == 0) return {1, 1};
  }
  if (d_qk == 576 && d_v == 512) {
    if (n_heads % 64 == 0) return {4, 2};
    if (n_heads % 32 == 0) return {2, 2};
    if (n_heads % 16 == 0) return {1, 2};
  }
  return {0, 0};
}

}  // namespace

cudaError_t launch_attend_merge(AttendParams& p, cudaStream_t st) {
  if (p.part_t) {
    dim3 mg(static_cast<unsigned>(p.n_q), static_cast<unsigned>((p.d_v / 4 + 1) / 2),
            static_cast<unsigned>((p.n_heads + 127) / 128));
    return launch_pdl(attend_merge_t_kernel, mg, dim3(256), 0, st, p);
  }
  const int hb = 256 / (p.d_v / 4);
  dim3 mg(static_cast<unsigned>(p.n_q), static_cast<unsigned>((p.n_heads + hb - 1) / hb));
  attend_merge_kernel<<<mg, 256, 0, st>>>(p);
  return cudaGetLastError();
}

bool attend_supported(int d_qk, int d_v, int n_heads, int kv_dtype) {
  if (kv_dtype != CSKV_BF16 && kv_dtype != CSKV_FP8_E4M3) return false;
  return plan_for(d_qk, d_v, n_heads).mt > 0;
}

// Choose keys per split so that queries x head groups x splits fills the GPU.
static void choose_split(AttendParams& p, int n_sm) {
  const Plan pl = plan_for(p.d_qk, p.d_v, p.n_heads);
  const int64_t groups = pl.mt ? p.n_heads / (16 * pl.mt) : 1;
  const int64_t n_max = (int64_t)p.n_win + (p.is_csa ? p.k : visible_entries(p.max_pos, p.m, p.n_win));
  const int ctas_per_sm = p.d_qk > 256 ? 1 : 4;
  const int64_t target = (int64_t)n_sm * ctas_per_sm;
  int64_t splits = (target + (int64_t)p.n_q * groups - 1) / ((int64_t)p.n_q * groups);
  if (splits < 1) splits = 1;
  int64_t kps = (n_max + splits - 1) / splits;
  kps = (kps + KT - 1) / KT * KT;
  if (kps < KT) kps = KT;
  if (kps > 1024) kps = 1024;
  p.keys_per_split = static_cast<int>(kps);
  p.max_splits = static_cast<int>((n_max + kps - 1) / kps);
  if (p.max_splits < 1) p.max_splits = 1;
}

size_t attend_ws_bytes(const AttendParams& p0, int n_sm) {
  AttendParams p = p0;
  if (attend_tc_supported(p.d_qk, p.d_v, p.n_heads, p.kv_dtype, p.n_q))
    attend_tc_plan(p, n_sm);
  else
    choose_split(p, n_sm);
  const size_t rows = (size_t)p.n_q * p.max_splits * p.n_heads;
  return rows * p.d_v * sizeof(float) + rows * sizeof(float) + 256;
}

cudaError_t launch_attend(AttendParams& p, void* ws, int n_sm, cudaStream_t st) {
  const bool tc = attend_tc_supported(p.d_qk, p.d_v, p.n_heads, p.kv_dtype, p.n_q);
  if (tc)
    attend_tc_plan(p, n_sm);
  else
    choose_split(p, n_sm);
  if (p.n_q > kMaxQ) return cudaErrorNotSupported;
  const size_t rows = (size_t)p.n_q * p.max_splits * p.n_heads;
  p.part_o = static_cast<float*>(ws);
  p.part_lse = p.part_o + rows * p.d_v;
  if (p.n_q == 0) return cudaSuccess;
  if (attend_pair_supported(p, n_sm)) return launch_attend_pair(p, n_sm, st);
  if (tc) return launch_attend_tc(p, n_sm, st);
  const Plan pl = plan_for(p.d_qk, p.d_v, p.n_heads);
  const bool fp8 = p.kv_dtype == CSKV_FP8_E4M3;
  if (p.d_qk == 128 && p.d_v == 128) {
    if (fp8) {
      if (pl.mt == 2) return run_attend<128, 128, 2, 1, true>(p, n_sm, st);
      if (pl.mt == 1) return run_attend<128, 128, 1, 1, true>(p, n_sm, st);
    } else {
      if (pl.mt == 2) return run_attend<128, 128, 2, 1, false>(p, n_sm, st);
      if (pl.mt == 1) return run_attend<128, 128, 1, 1, false>(p, n_sm, st);
    }
  } else if (p.d_qk == 576 && p.d_v == 512) {
    if (fp8) {
      if (pl.mt == 4) return run_attend<576, 512, 4, 2, true>(p, n_sm, st);
      if (pl.mt == 2) return run_attend<576, 512, 2, 2, true>(p, n_sm, st);
      if (pl.mt == 1) return run_attend<576, 512, 1, 2, true>(p, n_sm, st);
    } else {
      if (pl.mt == 4) return run_attend<576, 512, 4, 2, false>(p, n_sm, st);
      if (pl.mt == 2) return run_attend<576, 512, 2, 2, false>(p, n_sm, st);
      if (pl.mt == 1) return run_attend<576, 512, 1, 2, false>(p, n_sm, st);
    }
  }
  return cudaErrorNotSupported;
}

}  // namespace cskv
