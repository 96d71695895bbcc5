// fold.cu -- KV compression: every m raw tokens fold into one entry by a
// softmax-gated weighted sum (DeepSeek-V4 report digest, section 3: CSA m = 4,
// HCA m' = 128; DeepSeek-V4-book ch.1, section 4; 10100.com article,
// section 2.1: position weighting), and the state-cache append of a decode
// step (report digest, section 7, Figure 6: window + not-yet-compressed
// tokens).
//
// One warp folds one entry; lane l owns the 16-byte channel groups l, l+32,
// l+64, ... (8 channels each), so every load is a coalesced 128-bit access
// across the warp. The gate softmax runs online in fp32 (running max,
// denominator and weighted sum per channel); the entry is rounded to its
// storage type: bf16 (RNE), FP8 e4m3 with an fp32 scale per entry
// (amax / 448), or FP4 e2m1 with an e4m3 scale per 16 channels (amax / 6).
#include "cskv_device.cuh"
#include "cskv_internal.h"

namespace cskv {
namespace {

constexpr int kGroupsPerLane = 4;  // d <= 1024 channels

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

// Fold channels [c0, c0+8) of one block. rows(i, xr, zr) yields token i's
// raw row and gate row.
template <class Rows>
__device__ __forceinline__ void fold_group(const FoldStream& S, int m, int c0, Rows rows,
                                           float (&out)[8]) {
  float mx[8], den[8], acc[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    mx[e] = -INFINITY;
    den[e] = 0.f;
    acc[e] = 0.f;
  }
#pragma unroll 4
  for (int i = 0; i < m; ++i) {
    const uint16_t* xr;
    const uint16_t* zr;
    rows(i, xr, zr);
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
      for (int e = 0; e < 8; ++e) zl[e] += S.bias[(int64_t)i * S.d + c0 + e];
    }
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      if (zl[e] > mx[e]) {
        float corr = expf(mx[e] - zl[e]);  // 0 while mx is -inf
        den[e] *= corr;
        acc[e] *= corr;
        mx[e] = zl[e];
      }
      float p = expf(zl[e] - mx[e]);
      den[e] += p;
      acc[e] += p * xf[e];
    }
  }
#pragma unroll
  for (int e = 0; e < 8; ++e) out[e] = acc[e] / den[e];
}

// Fold one entry (whole warp) and store it at pool row `row` (-1: skip).
template <class Rows>
__device__ void fold_entry(const FoldStream& S, int m, int64_t row, Rows rows) {
  const int lane = threadIdx.x & 31;
  const int G = S.d / 8;
  float v[kGroupsPerLane][8];
  float amax = 0.f;
#pragma unroll
  for (int gi = 0; gi < kGroupsPerLane; ++gi) {
    const int grp = lane + 32 * gi;
    if (grp < G) {
      fold_group(S, m, grp * 8, rows, v[gi]);
#pragma unroll
      for (int e = 0; e < 8; ++e) amax = fmaxf(amax, fabsf(v[gi][e]));
    }
  }
  if (row < 0) return;
  if (S.out_dtype == CSKV_BF16) {
    uint16_t* dst = static_cast<uint16_t*>(S.pool) + row * S.d;
#pragma unroll
    for (int gi = 0; gi < kGroupsPerLane; ++gi) {
      const int grp = lane + 32 * gi;
      if (grp < G) {
        uint4 o;
        o.x = pack_bf16(v[gi][0], v[gi][1]);
        o.y = pack_bf16(v[gi][2], v[gi][3]);
        o.z = pack_bf16(v[gi][4], v[gi][5]);
        o.w = pack_bf16(v[gi][6], v[gi][7]);
        *reinterpret_cast<uint4*>(dst + grp * 8) = o;
      }
    }
  } else if (S.out_dtype == CSKV_FP8_E4M3) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(kFull, amax, o));
    const float s = amax > 0.f ? amax / 448.0f : 1.0f;
    uint8_t* dst = static_cast<uint8_t*>(S.pool) + row * S.d;
#pragma unroll
    for (int gi = 0; gi < kGroupsPerLane; ++gi) {
      const int grp = lane + 32 * gi;
      if (grp < G) {
        uint32_t w[2] = {0u, 0u};
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          uint32_t c = __nv_cvt_float_to_fp8(v[gi][e] / s, __NV_SATFINITE, __NV_E4M3);
          w[e >> 2] |= c << (8 * (e & 3));
        }
        *reinterpret_cast<uint2*>(dst + grp * 8) = make_uint2(w[0], w[1]);
      }
    }
    if (lane == 0) S.scale_f32[row] = s;
  } else {  // CSKV_FP4_E2M1: one e4m3 scale per 16 channels = lanes (2q, 2q+1)
    uint8_t* dst = static_cast<uint8_t*>(S.pool) + row * (S.d / 2);
#pragma unroll
    for (int gi = 0; gi < kGroupsPerLane; ++gi) {
      const int grp = lane + 32 * gi;
      float a = 0.f;
      if (grp < G) {
#pragma unroll
        for (int e = 0; e < 8; ++e) a = fmaxf(a, fabsf(v[gi][e]));
      }
      a = fmaxf(a, __shfl_xor_sync(kFull, a, 1));
      if (grp < G) {
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

__global__ void __launch_bounds__(256) fold_bulk_kernel(FoldParams p) {
  const int warps = blockDim.x / 32;
  const int64_t per_seq = p.n_tok / p.m;
  const int64_t total = (int64_t)p.n_streams * p.n_seq * per_seq;
  for (int64_t it = (int64_t)blockIdx.x * warps + (threadIdx.x >> 5); it < total;
       it += (int64_t)gridDim.x * warps) {
    const int si = static_cast<int>(it / (p.n_seq * per_seq));
    const int64_t rem = it % (p.n_seq * per_seq);
    const int b = static_cast<int>(rem / per_seq);
    const int64_t jj = rem % per_seq;
    const FoldStream& S = p.s[si];
    const int64_t row = entry_row(p, p.seq_ids[b], p.tok0 / p.m + jj);
    const int64_t t0 = (int64_t)b * p.n_tok + jj * p.m;
    auto rows = [&](int i, const uint16_t*& xr, const uint16_t*& zr) {
      xr = S.x + (t0 + i) * S.d;
      zr = S.z + (t0 + i) * S.gc;
    };
    if (row >= 0) fold_entry(S, p.m, row, rows);
  }
}

// One CTA per sequence: copy the new rows into the ring, then fold every
// block the new tokens complete (old rows from the ring, new rows from the
// input; the slots written and the slots read never coincide because
// n_new + m - 1 <= n_win).
__global__ void __launch_bounds__(256) append_kernel(FoldParams p) {
  const int b = blockIdx.x;
  const int seq = p.seq_ids[b];
  if (seq < 0 || seq >= p.n_seqs_layer) {
    if (threadIdx.x == 0) report(p.status, CSKV_ERR_OUT_OF_RANGE);
    return;
  }
  const int64_t pos = p.pos[b];
  for (int si = 0; si < p.n_streams; ++si) {
    const FoldStream& S = p.s[si];
    const int cx = S.d / 8;  // 16-byte chunks per x row
    for (int t = threadIdx.x; t < p.n_new * cx; t += blockDim.x) {
      const int i = t / cx, ch = t % cx;
      const int64_t slot = (pos + i) % p.n_win;
      *reinterpret_cast<uint4*>(S.ring_x_w + ((int64_t)seq * p.n_win + slot) * S.d + ch * 8) =
          ldg16(S.x + ((int64_t)b * p.n_new + i) * S.d + ch * 8);
    }
    for (int t = threadIdx.x; t < p.n_new * S.gc; t += blockDim.x) {
      const int i = t / S.gc, c = t % S.gc;
      const int64_t slot = (pos + i) % p.n_win;
      S.ring_z_w[((int64_t)seq * p.n_win + slot) * S.gc + c] = S.z[((int64_t)b * p.n_new + i) * S.gc + c];
    }
  }
  if (p.ring_only) return;
  // blocks completed by positions pos .. pos+n_new-1
  const int64_t j_first = pos / p.m;                 // first block ending at or after pos
  const int64_t j_last = (pos + p.n_new) / p.m - 1;  // last block ending before pos+n_new
  const int64_t nb = j_last >= j_first ? j_last - j_first + 1 : 0;
  const int warps = blockDim.x / 32;
  for (int64_t it = threadIdx.x >> 5; it < nb * p.n_streams; it += warps) {
    const int si = static_cast<int>(it / nb);
    const int64_t j = j_first + it % nb;
    const FoldStream& S = p.s[si];
    const int64_t row = entry_row(p, seq, j);
    auto rows = [&](int i, const uint16_t*& xr, const uint16_t*& zr) {
      const int64_t q = j * p.m + i;
      if (q >= pos) {
        xr = S.x + ((int64_t)b * p.n_new + (q - pos)) * S.d;
        zr = S.z + ((int64_t)b * p.n_new + (q - pos)) * S.gc;
      } else {
        const int64_t slot = q % p.n_win;
        xr = S.ring_x + ((int64_t)seq * p.n_win + slot) * S.d;
        zr = S.ring_z + ((int64_t)seq * p.n_win + slot) * S.gc;
      }
    };
    if (row >= 0) fold_entry(S, p.m, row, rows);
  }
}

}  // namespace

cudaError_t launch_fold_bulk(const FoldParams& p, cudaStream_t st) {
  const int64_t total = (int64_t)p.n_streams * p.n_seq * (p.n_tok / p.m);
  if (total == 0) return cudaSuccess;
  int dev = 0, n_sm = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev);
  const int64_t want = (total + 7) / 8;
  const int grid = static_cast<int>(want < (int64_t)n_sm * 8 ? want : (int64_t)n_sm * 8);
  fold_bulk_kernel<<<grid, 256, 0, st>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_append(const FoldParams& p, cudaStream_t st) {
  if (p.n_seq == 0 || p.n_new == 0) return cudaSuccess;
  append_kernel<<<p.n_seq, 256, 0, st>>>(p);
  return cudaGetLastError();
}

}  // namespace cskv
