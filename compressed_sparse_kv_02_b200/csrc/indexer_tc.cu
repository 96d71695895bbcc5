// indexer_tc.cu -- Lightning-indexer scores for calls with many queries on the
// 5th-generation tensor cores (DeepSeek-V4 report digest, section 3: the indexer
// scores every visible compressed entry by s = sum_h w_h ReLU(q_h . k), with one
// key per entry shared by the H_I indexer heads).
//
// In a prefill block consecutive queries of one sequence see (almost) the same
// entries, so the scores of a group of G = 128 / H_I queries are one GEMM: the
// 128 keys of a tile as M, the group's G x H_I query heads as N = 128, d_I as K.
// Each key tile is read once per group (the mma.sync grouped scan reads it once
// per 32 / H_I queries).
//   producer (warp 0): a group's query block (TMA, 128 rows) and per-query
//     weights and visible counts into one of two group buffers; 128-key tiles of
//     the paged keys (two 64-row TMA boxes per tile) into a four-stage ring;
//   MMA (warp 1, lane 0 issues): D = K Q^T (M = N = 128, K = d_I) into one of
//     two tensor-memory accumulators;
//   epilogue (warps 2-5, thread = key row = tensor-memory lane): the 128 head
//     dot products of its key, s_m = sum_h w[m, h] max(0, D[m H_I + h]) for every
//     query m of the group, written to the score rows (coalesced across the warp)
//     for the keys the query sees.
// Groups start at every G-th query and wherever the sequence changes. The units
// of work (group, key tile) are split evenly over a persistent grid.
#include "cskv_device.cuh"
#include "cskv_internal.h"

namespace cskv {
namespace {

constexpr int kKT = 128;        // keys per tile (the MMA's M)
constexpr int kNQ = 128;        // query heads per group (the MMA's N)
constexpr int kTcThreads = 192; // warp 0 producer, warp 1 MMA, warps 2-5 epilogue
constexpr uint32_t kTcTmemCols = 256;

template <int KB>  // 64-channel blocks of d_I (1 or 2)
struct TcScan {
  static constexpr int NST = KB == 1 ? 4 : 3;       // key stages
  static constexpr int KSTAGE = kKT * 128 * KB;     // 16 or 32 KB
  static constexpr int QBYTES = kNQ * 128 * KB;     // 16 or 32 KB
  static constexpr int K = 0;
  static constexpr int Q = K + NST * KSTAGE;
  static constexpr int W = Q + 2 * QBYTES;          // [2][kNQ] weights of the group's heads
  static constexpr int NV = W + 2 * kNQ * 4;        // [2][kNQ] visible entries per query (first G used)
  static constexpr int GS = NV + 2 * kNQ * 4;       // [2] group start, [2] group size
  static constexpr int BAR = GS + 16;
  static constexpr int NBAR = 2 * NST + 9;
  static constexpr int TMEM = BAR + NBAR * 8;
  static constexpr int FLAGS = TMEM + 8;
  static constexpr int GRP = FLAGS + 8;             // e_start [n_q + 1], e_pref [n_q + 1]
  static size_t bytes(int n_q) { return 1024 + GRP + 2 * sizeof(int) * (size_t)(n_q + 1); }
};

template <int KB, int HI>
__global__ void __launch_bounds__(kTcThreads, 1)
    index_scan_tc_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_q,
                         IndexParams p) {
  using L = TcScan<KB>;
  constexpr int NST = L::NST;
  constexpr int G = kNQ / HI;  // queries per group
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sK = sm + L::K;
  uint8_t* sQ = sm + L::Q;
  float* sW = reinterpret_cast<float*>(sm + L::W);
  int* sNv = reinterpret_cast<int*>(sm + L::NV);
  int* sGs = reinterpret_cast<int*>(sm + L::GS);  // [0..1] start, [2..3] size
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + L::BAR);
  uint64_t* kfull = bars;             // [NST] producer -> MMA (TMA bytes)
  uint64_t* kempty = bars + NST;      // [NST] MMA -> producer (commit)
  uint64_t* qfull = bars + 2 * NST;   // [2] producer -> MMA, epilogue (TMA bytes + meta)
  uint64_t* qempty = qfull + 2;       // [2] MMA (commit) + epilogue (128) -> producer
  uint64_t* dfull = qempty + 2;       // [2] MMA -> epilogue (commit)
  uint64_t* dempty = dfull + 2;       // [2] epilogue (128) -> MMA
  uint64_t* fin = dempty + 2;         //     every MMA of the CTA has completed (before freeing tensor memory)
  uint32_t* sTmem = reinterpret_cast<uint32_t*>(sm + L::TMEM);
  volatile int* sAbort = reinterpret_cast<int*>(sm + L::FLAGS);
  int* e_start = reinterpret_cast<int*>(sm + L::GRP);
  int* e_pref = e_start + p.n_q + 1;
  __shared__ int s_wsum[32];
  __shared__ int s_nent;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  if (tid == 0) {
    for (int i = 0; i < NST; ++i) {
      mbar_init(&kfull[i], 1);
      mbar_init(&kempty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&qfull[i], 1);
      mbar_init(&qempty[i], 1 + 128);
      mbar_init(&dfull[i], 1);
      mbar_init(&dempty[i], 128);
    }
    mbar_init(fin, 1);
    fence_barrier_init();
    *sAbort = 0;
  }
  if (warp == 1) {
    tmem_alloc(sTmem, kTcTmemCols);
    tmem_relinquish();
  }
  if (tid == 0) {
    prefetch_tensormap(&tm_k);
    prefetch_tensormap(&tm_q);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *sTmem;
  grid_dependency_wait();
  grid_dependents_launch();
  {  // group starts
    int run = 0;
    for (int base = 0; base < p.n_q; base += kTcThreads) {
      const int b = base + tid;
      int f = 0;
      if (b < p.n_q) f = (b % G == 0) || p.q_seq[b] != p.q_seq[b - 1];
      int tot;
      const int ex = block_exclusive_scan<kTcThreads>(f, s_wsum, tot);
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
  {  // key tiles per group: the most visible entries of its queries
    int run = 0;
    for (int base = 0; base < n_ent; base += kTcThreads) {
      const int e = base + tid;
      int u = 0;
      if (e < n_ent) {
        int64_t nv = 0;
        for (int b = e_start[e]; b < e_start[e + 1]; ++b) {
          const int64_t t = p.q_pos[b];
          const int64_t v = (t < 0 || t > p.max_pos) ? 0 : visible_entries(t, p.m, p.n_win);
          nv = v > nv ? v : nv;
        }
        u = static_cast<int>((nv + kKT - 1) / kKT);
      }
      int tot;
      const int ex = block_exclusive_scan<kTcThreads>(u, s_wsum, tot);
      if (e < n_ent) e_pref[e] = run + ex;
      run += tot;
    }
    if (tid == 0) e_pref[n_ent] = run;
  }
  __syncthreads();
  if (blockIdx.x == 0)
    for (int b = tid; b < p.n_q; b += kTcThreads)
      if (p.q_pos[b] < 0 || p.q_pos[b] > p.max_pos) report(p.status, CSKV_ERR_INVALID_ARG);

  const int64_t total = e_pref[n_ent];
  const int64_t u_begin = total * blockIdx.x / gridDim.x;
  const int n_units = static_cast<int>(total * (blockIdx.x + 1) / gridDim.x - u_begin);
  auto locate = [&](int64_t u, int& e, int64_t& j0) {
    int lo = 0, hi = n_ent - 1;  // last e with e_pref[e] <= u
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (e_pref[mid] <= u) lo = mid; else hi = mid - 1;
    }
    e = lo;
    j0 = (u - e_pref[lo]) * kKT;
  };
  const uint32_t idesc = umma_idesc_bf16(kKT, kNQ, false);

  if (warp == 0) {
    // ------------------------------------------------------------------ producer
    int cur_e = -1, n_grp = 0, gs = 0, seq = 0, issued = 0;
    int64_t nvmax = 0;
    bool ok = true;
    for (int i = 0; i < n_units && ok; ++i) {
      int e;
      int64_t j0;
      locate(u_begin + i, e, j0);
      if (e != cur_e) {
        cur_e = e;
        const int qb = n_grp & 1;
        if (n_grp >= 2) ok = __all_sync(kFull, mbar_wait(&qempty[qb], ((n_grp >> 1) - 1) & 1u, p.status));
        if (!ok) break;
        gs = e_start[e];
        const int gn = e_start[e + 1] - gs;
        seq = p.q_seq[gs];
        nvmax = 0;
        for (int c = lane; c < kNQ; c += 32) {
          const int m = c / HI, h = c % HI;
          sW[qb * kNQ + c] = m < gn ? p.w[(int64_t)(gs + m) * p.n_heads_idx + h] : 0.f;
        }
        for (int m = lane; m < G; m += 32) {
          int64_t v = 0;
          if (m < gn) {
            const int64_t t = p.q_pos[gs + m];
            v = (t < 0 || t > p.max_pos) ? 0 : visible_entries(t, p.m, p.n_win);
          }
          sNv[qb * kNQ + m] = static_cast<int>(v);
          nvmax = v > nvmax ? v : nvmax;
        }
        for (int o = 16; o > 0; o >>= 1) {
          const int64_t x = __shfl_xor_sync(kFull, nvmax, o);
          nvmax = x > nvmax ? x : nvmax;
        }
        if (lane == 0) {
          sGs[qb] = gs;
          sGs[2 + qb] = gn;
        }
        __syncwarp();
        if (lane == 0) {  // the group's query block: rows gs H_I .. + 127 (rows past n_q H_I read as zero)
          mbar_arrive_expect_tx(&qfull[qb], L::QBYTES);
          for (int kb = 0; kb < KB; ++kb) tma_load_2d(sQ + qb * L::QBYTES + kb * (kNQ * 128), &tm_q, kb * 64, gs * HI,
                                                      &qfull[qb]);
        }
        ++n_grp;
      }
      const int st = i % NST;
      if (i >= NST) ok = __all_sync(kFull, mbar_wait(&kempty[st], ((i / NST) - 1) & 1u, p.status));
      if (!ok) break;
      // two 64-key halves of the tile, each inside one page (pages hold a multiple of 64 entries)
      int row[2] = {-1, -1};
      for (int hh = 0; hh < 2; ++hh) {
        const int64_t jj = j0 + 64 * hh;
        if (jj >= nvmax) continue;
        const int64_t pi = jj / p.page_size;
        int32_t page = -1;
        if (seq >= 0 && seq < p.n_seqs_layer && pi < p.max_pages_per_seq)
          page = p.page_table[(int64_t)seq * p.max_pages_per_seq + pi];
        if (page >= 0 && page < p.n_pages) row[hh] = static_cast<int>((int64_t)page * p.page_size + jj % p.page_size);
        else if (lane == 0) report(p.status, CSKV_ERR_OUT_OF_RANGE);
      }
      if (lane == 0) {
        const uint32_t bytes = (row[0] >= 0 ? 1u : 0u) * (64 * 128 * KB) + (row[1] >= 0 ? 1u : 0u) * (64 * 128 * KB);
        if (bytes) {
          mbar_arrive_expect_tx(&kfull[st], bytes);
          for (int hh = 0; hh < 2; ++hh)
            if (row[hh] >= 0)
              for (int kb = 0; kb < KB; ++kb)
                tma_load_2d(sK + st * L::KSTAGE + kb * (kKT * 128) + hh * (64 * 128), &tm_k, kb * 64, row[hh],
                            &kfull[st]);
        } else {
          mbar_arrive(&kfull[st]);  // nothing to load (keys past the group's last visible entry)
        }
      }
      issued = i + 1;
      __syncwarp();
    }
    if (!ok && lane == 0) *sAbort = 1;
    if (__shfl_sync(kFull, *sAbort, 0) && lane == 0) {
      // copies that no MMA will wait for: give them a bounded chance to land
      for (int r = issued > NST ? issued - NST : 0; r < issued; ++r)
        mbar_wait(&kfull[r % NST], static_cast<uint32_t>((r / NST) & 1), nullptr);
      if (n_grp > 0) mbar_wait(&qfull[(n_grp - 1) & 1], static_cast<uint32_t>(((n_grp - 1) >> 1) & 1), nullptr);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issue
    int cur_e = -1, n_grp = 0;
    bool ok = true;
    for (int i = 0; i < n_units && ok; ++i) {
      if (__shfl_sync(kFull, *sAbort, 0)) break;
      int e;
      int64_t j0;
      locate(u_begin + i, e, j0);
      if (e != cur_e) {
        if (cur_e >= 0 && lane == 0) umma_commit(&qempty[(n_grp - 1) & 1]);  // the last group's MMAs
        cur_e = e;
        ok = __all_sync(kFull, mbar_wait(&qfull[n_grp & 1], (n_grp >> 1) & 1u, p.status));
        ++n_grp;
        if (!ok) break;
      }
      const int st = i % NST, db = i & 1;
      ok = __all_sync(kFull, mbar_wait(&kfull[st], (i / NST) & 1u, p.status));
      if (ok && i >= 2) ok = __all_sync(kFull, mbar_wait(&dempty[db], ((i >> 1) - 1) & 1u, p.status));
      if (!ok) break;
      tc_fence_after();
      if (lane == 0) {
        const uint32_t a0 = smem_u32(sK + st * L::KSTAGE), b0 = smem_u32(sQ + ((n_grp - 1) & 1) * L::QBYTES);
#pragma unroll
        for (int ks = 0; ks < 4 * KB; ++ks) {
          const uint32_t off = (ks >> 2) * (kKT * 128) + (ks & 3) * 32;
          umma_ss(tmem + db * kNQ, umma_desc_sw128(a0 + off, 16, 1024), umma_desc_sw128(b0 + off, 16, 1024), idesc,
                  ks > 0 ? 1u : 0u);
        }
        umma_commit(&kempty[st]);
        umma_commit(&dfull[db]);
      }
      __syncwarp();
    }
    if (cur_e >= 0 && lane == 0) umma_commit(&qempty[(n_grp - 1) & 1]);
    if (!ok && lane == 0) *sAbort = 1;
    __syncwarp();
  } else {
    // ------------------------------------------------------------------ epilogue
    const int r = 32 * (warp & 3) + lane;  // key row of the tile = tensor-memory lane
    const uint32_t trow = tmem + (static_cast<uint32_t>(32 * (warp & 3)) << 16);
    int cur_e = -1, n_grp = 0, qb = 0, gs = 0, gn = 0;
    bool ok = true;
    for (int i = 0; i < n_units && ok; ++i) {
      int e;
      int64_t j0;
      locate(u_begin + i, e, j0);
      if (e != cur_e) {
        if (cur_e >= 0) mbar_arrive(&qempty[qb]);  // done with the last group's weights and counts
        cur_e = e;
        qb = n_grp & 1;
        ok = __all_sync(kFull, mbar_wait(&qfull[qb], (n_grp >> 1) & 1u, p.status));
        ++n_grp;
        if (!ok) break;
        gs = sGs[qb];
        gn = sGs[2 + qb];
      }
      const int db = i & 1;
      ok = __all_sync(kFull, mbar_wait(&dfull[db], (i >> 1) & 1u, p.status));
      if (!ok) break;
      tc_fence_after();
      uint32_t d[kNQ];
#pragma unroll
      for (int c = 0; c < kNQ / 32; ++c) tmem_ld32(trow + db * kNQ + c * 32, *reinterpret_cast<uint32_t(*)[32]>(d + 32 * c));
      tmem_ld_wait();
      tc_fence_before();
      mbar_arrive(&dempty[db]);
      const int64_t j = j0 + r;
      const float* w = sW + qb * kNQ;
#pragma unroll
      for (int m = 0; m < G; ++m) {
        float s = 0.f;
#pragma unroll
        for (int h = 0; h < HI; ++h) s += w[m * HI + h] * fmaxf(__uint_as_float(d[m * HI + h]), 0.f);
        if (m < gn && j < sNv[qb * kNQ + m]) p.scores[(int64_t)(gs + m) * p.vis_stride + j] = selected_score(s, p.score_bf16);
      }
    }
    if (cur_e >= 0 && ok) mbar_arrive(&qempty[qb]);
    if (!ok && lane == 0) *sAbort = 1;
  }
  // every MMA issued here has completed before the tensor memory is freed (bounded wait)
  if (warp == 1) {
    if (lane == 0) umma_commit(fin);
    __syncwarp();
    mbar_wait(fin, 0u, nullptr);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, kTcTmemCols);
}

bool encode_rows_tc(CUtensorMap* map, const void* base, uint64_t rows, int d, uint32_t box_rows) {
  auto enc = tensor_map_encoder();
  if (!enc) return false;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(rows)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(d) * 2};
  const cuuint32_t box[2] = {64, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int KB, int HI>
cudaError_t run_scan_tc(IndexParams& p, int n_sm, cudaStream_t st) {
  CUtensorMap tm_k, tm_q;
  if (!encode_rows_tc(&tm_k, p.idx_pool, static_cast<uint64_t>(p.n_pages) * p.page_size, p.d_idx, 64) ||
      !encode_rows_tc(&tm_q, p.q_idx, static_cast<uint64_t>(p.n_q) * HI, p.d_idx, kNQ))
    return cudaErrorNotSupported;
  auto kern = index_scan_tc_kernel<KB, HI>;
  const size_t smem = TcScan<KB>::bytes(p.n_q);
  if (smem > 232448) return cudaErrorNotSupported;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  return launch_pdl(kern, dim3(static_cast<unsigned>(n_sm)), dim3(kTcThreads), smem, st, tm_k, tm_q, p);
}

}  // namespace

bool scan_tc_supported(const IndexParams& p) {
  return p.idx_dtype == CSKV_BF16 && (p.d_idx == 64 || p.d_idx == 128) && (p.n_heads_idx == 4 || p.n_heads_idx == 8) &&
         p.page_size % 64 == 0 && static_cast<uint64_t>(p.n_pages) * p.page_size < (1ull << 31) &&
         TcScan<2>::bytes(p.n_q) <= 232448;
}

cudaError_t launch_scan_tc(IndexParams& p, int n_sm, cudaStream_t st) {
  if (p.d_idx == 64 && p.n_heads_idx == 4) return run_scan_tc<1, 4>(p, n_sm, st);
  if (p.d_idx == 64) return run_scan_tc<1, 8>(p, n_sm, st);
  if (p.n_heads_idx == 4) return run_scan_tc<2, 4>(p, n_sm, st);
  return run_scan_tc<2, 8>(p, n_sm, st);
}

}  // namespace cskv
