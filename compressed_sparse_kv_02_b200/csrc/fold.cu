// fold.cu -- KV compression: every m raw tokens fold into one entry by a
// softmax-gated weighted sum (DeepSeek-V4 report digest, section 3: CSA m = 4,
// HCA m' = 128; DeepSeek-V4-book ch.1, section 4; 10100.com article,
// section 2.1: position weighting), and the state-cache append of a decode
// step (report digest, section 7, Figure 6: window + not-yet-compressed
// tokens).
//
// Small blocks (CSA, m = 4) fold one entry per warp: lane l owns the 16-byte
// channel groups l, l+32, l+64, ... (8 channels each), so every load is a
// coalesced 128-bit access across the warp. Large blocks (HCA, m' = 128) and
// the decode append fold one entry per CTA: threads split the entry over
// (channel group, token slice) and merge their partial states in shared
// memory. The gate softmax runs online in fp32 (running max, denominator and
// weighted sum per channel); the entry is rounded to its storage type: bf16
// (RNE), FP8 e4m3 with an fp32 scale per entry (amax / 448), or FP4 e2m1 with
// an e4m3 scale per 16 channels (amax / 6).
#include "cskv_device.cuh"
#include "cskv_internal.h"

namespace cskv {
namespace {

constexpr int kGroupsPerLane = 4;  // d <= 1024 channels
constexpr float kLog2e = 1.4426950408889634f;

__device__ __forceinline__ float bf16_bits_to_f32(uint16_t b) {
  return __uint_as_float(static_cast<uint32_t>(b) << 16);
}

__device__ __forceinline__ void unpack8(const uint4& v, float (&f)[8]) {
  f[0] = __uint_as_float(v.x << 16);
  f[1] = __uint_as_float(v.x & 0xffff0000u);
  f[2] = __uint_as_float(v.y << 16);
  f[3] = __uint_as_float(v.y & 0xffff0000u);
  f[4] = __uint_as_float(v.z << 16);
  f[5] = __uint_as_float(v.z & 0xffff0000u);
  f[6] = __uint_as_float(v.w << 16);
  f[7] = __uint_as_float(v.w & 0xffff0000u);
}

// Online-softmax partial state of channels [c0, c0+8) over tokens i0 .. i1-1
// of one block (token i < 0 is one of the ov tokens of the previous block that
// the entry overlaps): running max (of the logits times log2 e), denominator
// and weighted sum (fp32). rows(i, xr, zr) yields token i's raw row and gate
// row, or false when the token lies before the start of the stream; the
// position bias row of token i is i + ov.
template <class Rows>
__device__ __forceinline__ void fold_partial(const FoldStream& S, int i0, int i1, int c0, Rows rows, int ov,
                                             float (&mx)[8], float (&den)[8], float (&acc)[8]) {
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    mx[e] = -INFINITY;
    den[e] = 0.f;
    acc[e] = 0.f;
  }
#pragma unroll 4
  for (int i = i0; i < i1; ++i) {
    const uint16_t* xr;
    const uint16_t* zr;
    if (!rows(i, xr, zr)) continue;
    float xf[8], zl[8];
    unpack8(ldg16(xr + c0), xf);
    if (S.gc == 1) {
      float zz = bf16_bits_to_f32(zr[0]);
#pragma unroll
      for (int e = 0; e < 8; ++e) zl[e] = zz;
    } else {
      unpack8(ldg16(zr + c0), zl);
    }
    if (S.bias) {
#pragma unroll
      for (int e = 0; e < 8; ++e) zl[e] += S.bias[(int64_t)(i + ov) * S.d + c0 + e];
    }
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const float l2 = zl[e] * kLog2e;  // softmax weights in base 2: 2^(l2 - max) = e^(z - max_z)
      if (l2 > mx[e]) {
        const float corr = exp2f(mx[e] - l2);  // 0 while mx is -inf
        den[e] *= corr;
        acc[e] *= corr;
        mx[e] = l2;
      }
      const float p = exp2f(l2 - mx[e]);
      den[e] += p;
      acc[e] += p * xf[e];
    }
  }
}

// Fold channels [c0, c0+8) over tokens i0 .. i1-1 (a whole block) into out.
template <class Rows>
__device__ __forceinline__ void fold_group(const FoldStream& S, int m, int i0, int i1, int c0, Rows rows, int ov,
                                           float (&out)[8]) {
  float mx[8], den[8], acc[8];
  fold_partial(S, i0, i1, c0, rows, ov, mx, den, acc);
#pragma unroll
  for (int e = 0; e < 8; ++e) out[e] = acc[e] / den[e];
}

// Round one entry to its storage type and store it at pool row `row`. The
// calling threads hold 8 consecutive channels each: a thread holds groups
// first, first + stride, ... (its first `nslots` slots of v); `amax` is the
// entry-wide max |value| (needed for FP8), already reduced by the caller.
// Adjacent threads hold adjacent groups, so an FP4 16-channel block is the
// pair (2q, 2q+1) of threads with the same parity pattern.
__device__ __forceinline__ void store_groups(const FoldStream& S, int64_t row, int first, int stride, int nslots,
                                             const float (&v)[kGroupsPerLane][8], float amax) {
  const int G = S.d / 8;
  if (S.out_dtype == CSKV_BF16) {
    uint16_t* dst = static_cast<uint16_t*>(S.pool) + row * S.d;
#pragma unroll
    for (int gi = 0; gi < kGroupsPerLane; ++gi) {
      const int grp = first + stride * gi;
      if (gi < nslots && grp < G) {
        uint4 o;
        o.x = pack_bf16(v[gi][0], v[gi][1]);
        o.y = pack_bf16(v[gi][2], v[gi][3]);
        o.z = pack_bf16(v[gi][4], v[gi][5]);
        o.w = pack_bf16(v[gi][6], v[gi][7]);
        *reinterpret_cast<uint4*>(dst + grp * 8) = o;
      }
    }
  } else if (S.out_dtype == CSKV_FP8_E4M3) {
    const float s = amax > 0.f ? amax / 448.0f : 1.0f;
    uint8_t* dst = static_cast<uint8_t*>(S.pool) + row * S.d;
#pragma unroll
    for (int gi = 0; gi < kGroupsPerLane; ++gi) {
      const int grp = first + stride * gi;
      if (gi < nslots && grp < G) {
        uint32_t w[2] = {0u, 0u};
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          uint32_t c = __nv_cvt_float_to_fp8(v[gi][e] / s, __NV_SATFINITE, __NV_E4M3);
          w[e >> 2] |= c << (8 * (e & 3));
        }
        *reinterpret_cast<uint2*>(dst + grp * 8) = make_uint2(w[0], w[1]);
        if (grp == 0) S.scale_f32[row] = s;
      }
    }
  } else {  // CSKV_FP4_E2M1: one e4m3 scale per 16 channels = groups (2q, 2q+1)
    uint8_t* dst = static_cast<uint8_t*>(S.pool) + row * (S.d / 2);
#pragma unroll
    for (int gi = 0; gi < kGroupsPerLane; ++gi) {
      const int grp = first + stride * gi;
      const bool mine = gi < nslots && grp < G;
      float a = 0.f;
      if (mine) {
#pragma unroll
        for (int e = 0; e < 8; ++e) a = fmaxf(a, fabsf(v[gi][e]));
      }
      a = fmaxf(a, __shfl_xor_sync(kFull, a, 1));
      if (mine) {
        const __nv_fp8_storage_t sb = __nv_cvt_float_to_fp8(a / 6.0f, __NV_SATFINITE, __NV_E4M3);
        const float sd = __half2float(__half(__nv_cvt_fp8_to_halfraw(sb, __NV_E4M3)));
        uint32_t w = 0u;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          uint32_t c = 0u;
          if (sd > 0.f) c = __nv_cvt_float_to_fp4(v[gi][e] / sd, __NV_E2M1, cudaRoundNearest) & 0xfu;
          w |= c << (4 * e);  // element 2i in the low nibble of byte i
        }
        *reinterpret_cast<uint32_t*>(dst + grp * 4) = w;
        if ((grp & 1) == 0) S.scale_e4m3[row * (S.d / 16) + grp / 2] = sb;
      }
    }
  }
}

// Fold one entry with one warp (small m: every lane runs the m tokens of its
// channel groups) and store it at pool row `row`.
template <class Rows>
__device__ void fold_entry_warp(const FoldStream& S, int m, int ov, int64_t row, Rows rows) {
  const int lane = threadIdx.x & 31;
  const int G = S.d / 8;
  float v[kGroupsPerLane][8];
  float amax = 0.f;
#pragma unroll
  for (int gi = 0; gi < kGroupsPerLane; ++gi) {
    const int grp = lane + 32 * gi;
    if (grp < G) {
      fold_group(S, m, -ov, m, grp * 8, rows, ov, v[gi]);
#pragma unroll
      for (int e = 0; e < 8; ++e) amax = fmaxf(amax, fabsf(v[gi][e]));
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(kFull, amax, o));
  store_groups(S, row, lane, 32, kGroupsPerLane, v, amax);
}

// Fold channels [c_lo, c_hi) of one entry with the whole block: thread t
// takes channel group t % G of the range and token slice t / G; the partial
// online-softmax states (max, denominator, weighted sum) of the slices are
// merged through shared memory. `sm` holds 3 * blockDim.x * 8 floats. For an
// FP8 entry the range must be the whole row (its scale is the row's amax).
template <class Rows>
__device__ void fold_entry_block(const FoldStream& S, int m, int ov, int64_t row, Rows rows, float* sm, int c_lo,
                                 int c_hi) {
  const int G = (c_hi - c_lo) / 8;
  const int t = threadIdx.x;
  const int nt = m + ov;    // tokens of the entry: -ov .. m - 1
  int ns = blockDim.x / G;  // token slices
  if (ns > nt) ns = nt;
  const int per = (nt + ns - 1) / ns;
  const int g = t % G, sl = t / G;
  float* smx = sm;
  float* sden = sm + blockDim.x * 8;
  float* sacc = sm + 2 * blockDim.x * 8;
  if (sl < ns) {
    float mx[8], den[8], acc[8];
    const int i0 = sl * per - ov, i1 = min(m, i0 + per);
    fold_partial(S, i0, i1, c_lo + g * 8, rows, ov, mx, den, acc);
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      smx[(sl * G + g) * 8 + e] = mx[e];
      sden[(sl * G + g) * 8 + e] = den[e];
      sacc[(sl * G + g) * 8 + e] = acc[e];
    }
  }
  __syncthreads();
  // threads 0..G-1 merge the slices of their group
  float v[kGroupsPerLane][8];
  float amax = 0.f;
  if (t < G) {
    float M[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) M[e] = -INFINITY;
    for (int q = 0; q < ns; ++q)
#pragma unroll
      for (int e = 0; e < 8; ++e) M[e] = fmaxf(M[e], smx[(q * G + t) * 8 + e]);
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      float den = 0.f, acc = 0.f;
      for (int q = 0; q < ns; ++q) {
        const float mq = smx[(q * G + t) * 8 + e];
        if (mq == -INFINITY) continue;
        const float f = exp2f(mq - M[e]);
        den += sden[(q * G + t) * 8 + e] * f;
        acc += sacc[(q * G + t) * 8 + e] * f;
      }
      v[0][e] = acc / den;
      amax = fmaxf(amax, fabsf(v[0][e]));
    }
  }
  if (S.out_dtype == CSKV_FP8_E4M3) {  // entry-wide amax: block reduction
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(kFull, amax, o));
    __syncthreads();
    if ((t & 31) == 0) smx[t >> 5] = amax;
    __syncthreads();
    amax = 0.f;
    for (int w = 0; w < (int)(blockDim.x >> 5); ++w) amax = fmaxf(amax, smx[w]);
  }
  if (t < ((G + 31) & ~31)) store_groups(S, row, c_lo / 8 + t, G, t < G ? 1 : 0, v, amax);
  __syncthreads();  // shared memory is reused by the next entry
}

// pool row of entry j of sequence seq, or -1 (and a status code) when the
// page table points outside the pool
__device__ __forceinline__ int64_t entry_row(const FoldParams& p, int seq, int64_t j) {
  if (seq < 0 || seq >= p.n_seqs_layer) {
    report(p.status, CSKV_ERR_OUT_OF_RANGE);
    return -1;
  }
  const int64_t pi = j / p.page_size;
  if (pi >= p.max_pages_per_seq) {
    report(p.status, CSKV_ERR_OUT_OF_RANGE);
    return -1;
  }
  const int32_t page = p.page_table[(int64_t)seq * p.max_pages_per_seq + pi];
  if (page < 0 || page >= p.n_pages) {
    report(p.status, CSKV_ERR_OUT_OF_RANGE);
    return -1;
  }
  return (int64_t)page * p.page_size + (j % p.page_size);
}

constexpr int kWarpFoldMaxM = 16;  // up to this many tokens per entry one warp folds an entry
constexpr int kBlockFoldThreads = 512;

// rows of the bulk input: token i of entry jj of row block b (input row t0 + i,
// stream position pos0 + i); an overlap token before the segment's first
// position comes from the sequence's ring, one before position 0 does not exist
struct BulkRows {
  const FoldStream* S;
  int64_t t0, seg0, pos0;  // input row of token 0, input row of the segment start, position of token 0
  int64_t tok0;            // position of the segment's first token
  int64_t ring_row0;       // seq * n_win
  int n_win;
  __device__ bool operator()(int i, const uint16_t*& xr, const uint16_t*& zr) const {
    const int64_t pos = pos0 + i;
    if (pos < 0) return false;
    if (pos >= tok0) {
      xr = S->x + (t0 + i) * S->d;
      zr = S->z + (t0 + i) * S->gc;
    } else {
      const int64_t r = ring_row0 + pos % n_win;
      xr = S->ring_x + r * S->d;
      zr = S->ring_z + r * S->gc;
    }
    return true;
  }
};

__device__ __forceinline__ void bulk_item(const FoldParams& p, int64_t it, int& si, int64_t& row, BulkRows& r) {
  const int64_t per_seq = p.n_tok / p.m;
  si = static_cast<int>(it / (p.n_seq * per_seq));
  const int64_t rem = it % (p.n_seq * per_seq);
  const int b = static_cast<int>(rem / per_seq);
  const int64_t jj = rem % per_seq;
  row = entry_row(p, p.seq_ids[b], p.tok0 / p.m + jj);
  r.S = &p.s[si];
  r.t0 = (int64_t)b * p.n_tok + jj * p.m;
  r.seg0 = (int64_t)b * p.n_tok;
  r.pos0 = p.tok0 + jj * p.m;
  r.tok0 = p.tok0;
  r.ring_row0 = (int64_t)p.seq_ids[b] * p.n_win;
  r.n_win = p.n_win;
}

// small m (CSA): one warp per entry
__global__ void __launch_bounds__(256) fold_bulk_warp_kernel(FoldParams p) {
  const int warps = blockDim.x / 32;
  const int64_t total = (int64_t)p.n_streams * p.n_seq * (p.n_tok / p.m);
  for (int64_t it = (int64_t)blockIdx.x * warps + (threadIdx.x >> 5); it < total;
       it += (int64_t)gridDim.x * warps) {
    int si;
    int64_t row;
    BulkRows r;
    bulk_item(p, it, si, row, r);
    if (row >= 0) fold_entry_warp(p.s[si], p.m, p.ov, row, r);
  }
}

// large m (HCA): one block per entry, tokens split over thread slices
__global__ void __launch_bounds__(kBlockFoldThreads) fold_bulk_block_kernel(FoldParams p) {
  __shared__ float sm[3 * kBlockFoldThreads * 8];
  const int64_t total = (int64_t)p.n_streams * p.n_seq * (p.n_tok / p.m);
  for (int64_t it = blockIdx.x; it < total; it += gridDim.x) {
    int si;
    int64_t row;
    BulkRows r;
    bulk_item(p, it, si, row, r);
    if (row >= 0) fold_entry_block(p.s[si], p.m, p.ov, row, r, sm, 0, p.s[si].d);  // row is uniform across the block
  }
}

constexpr int kAppendWarps = 16;  // an FP8 entry is folded whole by one CTA: 36 units of 16 channels at d = 576
constexpr int kAppendThreads = 32 * kAppendWarps;
constexpr int kSliceCh = 64;       // channels per CTA of the append kernel (whole row for FP8)
constexpr int kAppendMaxD = 1024;  // channels of the row buffer
constexpr int kFoldPairs = 32;     // channel pairs of one fold pass (64 channels)
constexpr int kFoldGroups = kAppendThreads / kFoldPairs;  // 16 token groups
constexpr int kAppendBatch = 8;  // tokens per thread whose loads are in flight together (m' = 128: all of them)

// Store channels [c_lo, c_hi) of one folded entry from the row buffer `sv`
// (fp32, indexed by channel) into pool row `row` in the stream's storage type:
// bf16 (RNE), FP8 E4M3 with the row scale amax / 448 (the range is the whole
// row), or FP4 E2M1 with one E4M3 scale per 16 channels.
__device__ void store_row(const FoldStream& S, int64_t row, const float* sv, int c_lo, int c_hi, float* s_red) {
  const int t = threadIdx.x;
  if (S.out_dtype == CSKV_BF16) {
    uint16_t* dst = static_cast<uint16_t*>(S.pool) + row * S.d;
    for (int c = c_lo + 8 * t; c < c_hi; c += 8 * kAppendThreads) {
      uint4 o;
      o.x = pack_bf16(sv[c], sv[c + 1]);
      o.y = pack_bf16(sv[c + 2], sv[c + 3]);
      o.z = pack_bf16(sv[c + 4], sv[c + 5]);
      o.w = pack_bf16(sv[c + 6], sv[c + 7]);
      *reinterpret_cast<uint4*>(dst + c) = o;
    }
  } else if (S.out_dtype == CSKV_FP8_E4M3) {
    float a = 0.f;
    for (int c = c_lo + t; c < c_hi; c += kAppendThreads) a = fmaxf(a, fabsf(sv[c]));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(kFull, a, o));
    if ((t & 31) == 0) s_red[t >> 5] = a;
    __syncthreads();
    float amax = 0.f;
    for (int w = 0; w < kAppendWarps; ++w) amax = fmaxf(amax, s_red[w]);
    const float sc = amax > 0.f ? amax / 448.0f : 1.0f;
    uint8_t* dst = static_cast<uint8_t*>(S.pool) + row * S.d;
    for (int c = c_lo + 8 * t; c < c_hi; c += 8 * kAppendThreads) {
      uint32_t w[2] = {0u, 0u};
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const uint32_t code = __nv_cvt_float_to_fp8(sv[c + e] / sc, __NV_SATFINITE, __NV_E4M3);
        w[e >> 2] |= code << (8 * (e & 3));
      }
      *reinterpret_cast<uint2*>(dst + c) = make_uint2(w[0], w[1]);
    }
    if (t == 0) S.scale_f32[row] = sc;
    __syncthreads();  // s_red is reused
  } else {  // FP4: 16-channel blocks, element 2i in the low nibble of byte i
    uint8_t* dst = static_cast<uint8_t*>(S.pool) + row * (S.d / 2);
    for (int c = c_lo + 16 * t; c < c_hi; c += 16 * kAppendThreads) {
      float a = 0.f;
#pragma unroll
      for (int e = 0; e < 16; ++e) a = fmaxf(a, fabsf(sv[c + e]));
      const __nv_fp8_storage_t sb = __nv_cvt_float_to_fp8(a / 6.0f, __NV_SATFINITE, __NV_E4M3);
      const float sd = __half2float(__half(__nv_cvt_fp8_to_halfraw(sb, __NV_E4M3)));
      uint32_t w[2] = {0u, 0u};
#pragma unroll
      for (int e = 0; e < 16; ++e) {
        uint32_t code = 0u;
        if (sd > 0.f) code = __nv_cvt_float_to_fp4(sv[c + e] / sd, __NV_E2M1, cudaRoundNearest) & 0xfu;
        w[e >> 3] |= code << (4 * (e & 7));
      }
      *reinterpret_cast<uint2*>(dst + c / 2) = make_uint2(w[0], w[1]);
      S.scale_e4m3[row * (S.d / 16) + c / 16] = sb;
    }
  }
}

// Grid (sequence, 64-channel slice, stream); an FP8 stream is handled whole by
// slice 0 (its scale is the row's amax). Each CTA copies its channels of the
// new rows into the rings (not with emit_only), then folds its channels of
// every block the new tokens complete (not with ring_only; old rows from the
// ring, new rows from the input; the slots written and the slots read never
// coincide because n_new + m - 1 <= n_win).
// All 512 threads fold: thread (token group g, channel pair) runs the online
// softmax of the gate over tokens g, g + 16, ... of the block for its two
// channels, and one thread per channel merges the 16 groups' states from
// shared memory; the entry is stored from a shared-memory row buffer.
__global__ void __launch_bounds__(kAppendThreads) append_kernel(FoldParams p) {
  __shared__ float sv[kAppendMaxD];
  __shared__ float s_red[kAppendWarps];
  __shared__ float s_mx[kFoldGroups][2 * kFoldPairs], s_den[kFoldGroups][2 * kFoldPairs],
      s_acc[kFoldGroups][2 * kFoldPairs];
  const int b = blockIdx.x, slice = blockIdx.y, si = blockIdx.z;
  const int t = threadIdx.x;
  grid_dependency_wait();  // every input may come from the kernel launched before this one
  grid_dependents_launch();
  const int seq = p.seq_ids[b];
  if (seq < 0 || seq >= p.n_seqs_layer) {
    if (t == 0 && slice == 0 && si == 0) report(p.status, CSKV_ERR_OUT_OF_RANGE);
    return;
  }
  const FoldStream& S = p.s[si];
  const bool whole = S.out_dtype == CSKV_FP8_E4M3;
  const int c_lo = whole ? 0 : slice * kSliceCh;
  const int c_hi = whole ? S.d : min(S.d, c_lo + kSliceCh);
  if (c_lo >= S.d || (whole && slice != 0)) return;
  const int64_t pos = p.pos[b];
  if (!p.emit_only) {  // ring rows of the new tokens (this CTA's channels; gate logits: a per-token logit goes with c_lo == 0)
    const int cx = (c_hi - c_lo) / 8;
    for (int k = t; k < p.n_new * cx; k += kAppendThreads) {
      const int i = k / cx, ch = k % cx;
      const int64_t slot = (pos + i) % p.n_win;
      *reinterpret_cast<uint4*>(S.ring_x_w + ((int64_t)seq * p.n_win + slot) * S.d + c_lo + ch * 8) =
          ldg16(S.x + ((int64_t)b * p.n_new + i) * S.d + c_lo + ch * 8);
    }
    const int z_lo = S.gc == 1 ? (c_lo == 0 ? 0 : 1) : c_lo, z_hi = S.gc == 1 ? 1 : c_hi;
    for (int k = t; k < p.n_new * (z_hi - z_lo); k += kAppendThreads) {
      const int i = k / (z_hi - z_lo), c = z_lo + k % (z_hi - z_lo);
      const int64_t slot = (pos + i) % p.n_win;
      S.ring_z_w[((int64_t)seq * p.n_win + slot) * S.gc + c] = S.z[((int64_t)b * p.n_new + i) * S.gc + c];
    }
  }
  if (p.ring_only) return;
  // blocks completed by positions pos .. pos+n_new-1
  const int64_t j_first = pos / p.m;                 // first block ending at or after pos
  const int64_t j_last = (pos + p.n_new) / p.m - 1;  // last block ending before pos+n_new
  // every thread folds a channel pair over a group of the entry's tokens (tokens tg - ov,
  // tg - ov + 16, ... of the block, the first ov of them the overlap with the block before); the 16
  // groups' partial states (running max in base 2, denominator, weighted sum) then merge per
  // channel through shared memory
  const int cp = t % kFoldPairs, tg = t / kFoldPairs;
  for (int64_t j = j_first; j <= j_last; ++j) {
    const int64_t row = entry_row(p, seq, j);  // uniform across the block
    for (int c0 = c_lo; c0 < c_hi; c0 += 2 * kFoldPairs) {  // 64 channels per pass
      const int c = c0 + 2 * cp;
      const bool active = c < c_hi;
      float mx[2] = {-INFINITY, -INFINITY}, den[2] = {0.f, 0.f}, acc[2] = {0.f, 0.f};
      // kAppendBatch tokens per round: every load of the round is issued before the first
      // weight is computed, so their latencies overlap instead of adding up
      for (int i0 = tg - p.ov; active && i0 < p.m; i0 += kAppendBatch * kFoldGroups) {
        uint32_t xv[kAppendBatch], zv[kAppendBatch];
        float bv[kAppendBatch][2];
        bool ok[kAppendBatch];
#pragma unroll
        for (int u = 0; u < kAppendBatch; ++u) {
          const int i = i0 + u * kFoldGroups;
          const int64_t q = j * p.m + i;
          ok[u] = i < p.m && q >= 0;  // q < 0: before the start of the stream
          xv[u] = zv[u] = 0u;
          bv[u][0] = bv[u][1] = 0.f;
          if (!ok[u]) continue;
          const uint16_t* xr;
          const uint16_t* zr;
          if (q >= pos) {
            xr = S.x + ((int64_t)b * p.n_new + (q - pos)) * S.d;
            zr = S.z + ((int64_t)b * p.n_new + (q - pos)) * S.gc;
          } else {
            const int64_t slot = q % p.n_win;
            xr = S.ring_x + ((int64_t)seq * p.n_win + slot) * S.d;
            zr = S.ring_z + ((int64_t)seq * p.n_win + slot) * S.gc;
          }
          xv[u] = __ldg(reinterpret_cast<const uint32_t*>(xr + c));
          zv[u] = S.gc == 1 ? static_cast<uint32_t>(__ldg(zr)) << 16 : __ldg(reinterpret_cast<const uint32_t*>(zr + c));
          if (S.bias) {
            const float* br = S.bias + (int64_t)(i + p.ov) * S.d + c;
            bv[u][0] = __ldg(br);
            bv[u][1] = __ldg(br + 1);
          }
        }
#pragma unroll
        for (int u = 0; u < kAppendBatch; ++u) {
          if (!ok[u]) continue;
          // a per-token gate (gc == 1) sits in the high half for both channels
          const float zl[2] = {S.gc == 1 ? __uint_as_float(zv[u] & 0xffff0000u) : __uint_as_float(zv[u] << 16),
                               __uint_as_float(zv[u] & 0xffff0000u)};
          const float xf[2] = {__uint_as_float(xv[u] << 16), __uint_as_float(xv[u] & 0xffff0000u)};
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const float l2 = (zl[e] + bv[u][e]) * kLog2e;  // base-2 weights: 2^(l2 - max) = e^(z - max_z)
            const float M = fmaxf(mx[e], l2);
            const float corr = mx[e] == -INFINITY ? 0.f : exp2f(mx[e] - M);
            const float pw = exp2f(l2 - M);
            den[e] = den[e] * corr + pw;
            acc[e] = acc[e] * corr + pw * xf[e];
            mx[e] = M;
          }
        }
      }
      if (active) {
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          s_mx[tg][2 * cp + e] = mx[e];
          s_den[tg][2 * cp + e] = den[e];
          s_acc[tg][2 * cp + e] = acc[e];
        }
      }
      __syncthreads();
      if (t < 2 * kFoldPairs && c0 + t < c_hi) {  // one thread per channel merges the groups that ran tokens
        const int ng = p.m + p.ov < kFoldGroups ? p.m + p.ov : kFoldGroups;
        float M = -INFINITY;
        for (int gi = 0; gi < ng; ++gi) M = fmaxf(M, s_mx[gi][t]);
        float dd = 0.f, aa = 0.f;
        for (int gi = 0; gi < ng; ++gi) {
          const float f = s_mx[gi][t] == -INFINITY ? 0.f : exp2f(s_mx[gi][t] - M);
          dd += s_den[gi][t] * f;
          aa += s_acc[gi][t] * f;
        }
        sv[c0 + t] = aa / dd;
      }
      __syncthreads();
    }
    if (row >= 0) store_row(S, row, sv, c_lo, c_hi, s_red);
    __syncthreads();  // the row buffer is reused by the next block
  }
}

}  // namespace

cudaError_t launch_fold_bulk(const FoldParams& p, cudaStream_t st) {
  const int64_t total = (int64_t)p.n_streams * p.n_seq * (p.n_tok / p.m);
  if (total == 0) return cudaSuccess;
  int dev = 0, n_sm = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev);
  if (p.m <= kWarpFoldMaxM) {
    const int64_t want = (total + 7) / 8;
    const int grid = static_cast<int>(want < (int64_t)n_sm * 8 ? want : (int64_t)n_sm * 8);
    fold_bulk_warp_kernel<<<grid, 256, 0, st>>>(p);
  } else {
    const int grid = static_cast<int>(total < (int64_t)n_sm * 4 ? total : (int64_t)n_sm * 4);
    fold_bulk_block_kernel<<<grid, kBlockFoldThreads, 0, st>>>(p);
  }
  return cudaGetLastError();
}

cudaError_t launch_append(const FoldParams& p, cudaStream_t st) {
  if (p.n_seq == 0 || p.n_new == 0) return cudaSuccess;
  int dmax = 0;
  for (int si = 0; si < p.n_streams; ++si) {
    if (p.s[si].d > kAppendMaxD) return cudaErrorInvalidValue;
    dmax = p.s[si].d > dmax ? p.s[si].d : dmax;
  }
  dim3 grid(static_cast<unsigned>(p.n_seq), static_cast<unsigned>((dmax + kSliceCh - 1) / kSliceCh),
            static_cast<unsigned>(p.n_streams));
  return launch_pdl(append_kernel, grid, dim3(kAppendThreads), 0, st, p);
}

}  // namespace cskv
