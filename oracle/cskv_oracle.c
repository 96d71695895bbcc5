/*
 * cskv_oracle.c -- plain, slow, fp64 CPU oracle for CSA / HCA hybrid
 * compressed attention.
 *
 * TEST INFRASTRUCTURE. Only the tests, the smoke check and the benchmark's
 * CPU-baseline leg load this library. The GPU library shares no code, header,
 * table or helper with it; neither side includes or links the other.
 *
 * Sources (page title, section):
 *   [digest]  "DeepSeek-V4 ..." report digest (gitcode.csdn.net/69eb1ea0...),
 *             section 3 (CSA + HCA hybrid attention) and section 7 (FP4 QAT,
 *             heterogeneous KV cache, Figure 6).
 *   [book]    DeepSeek-V4-book ch.1 "演进地图 -- V1 到 V4 改了什么",
 *             section 4 (change 1: MLA -> CSA x HCA).
 *   [10100]   10100.com DeepSeek-V4 article, sections 2.1 (CSA), 2.2 (HCA),
 *             2.3 (interleaving), 5 (FP8/FP4, paged KV).
 *   [essay]   "constraint chain" essay (gitcode.csdn.net/6a02d7e2...),
 *             "约束1 -> 创新1" (weighted fusion of KV).
 *
 * Readings where the pages are silent (each is listed with its reason in the
 * design notes of the repository):
 *   - gate: per-channel logits Z[n, d] (or one logit per token, Z[n, 1]),
 *     softmax over the m in-block positions, per channel; an optional
 *     additive position bias B[m, d] ([10100] 2.1 "position weighting").
 *   - visibility: compressed entry j is visible to the query at position t
 *     iff its block starts before the window, j*m < t + 1 - n_win; the window
 *     is positions max(0, t - n_win + 1) .. t.
 *   - indexer: s(t, j) = sum_h w[t,h] * max(0, q_I[t,h,:] . K_I[j,:]), with
 *     one shared indexer key head.
 *   - top-k: order (score desc, index asc); output ascending by index,
 *     padded with -1; k_eff = min(k, visible).
 *   - attention: one softmax over window keys U_win and compressed keys;
 *     K_u is the whole stored vector (d_qk), V_u its first d_v channels.
 *   - storage: bf16 by round-to-nearest-even; FP8 e4m3 with one fp32 scale
 *     per entry (scale = amax / 448, an all-zero entry gets scale 1); FP4
 *     e2m1 with one e4m3 scale per 16 elements (scale = e4m3(amax / 6)).
 *     The quantisation decisions are taken in fp32, the precision the GPU
 *     kernels take them in.
 *
 * Every function computes straight from its definition: no blocking, no
 * fusion, no reordering beyond what the definition states. Loops over
 * independent outputs may run on several OpenMP threads; that does not
 * change the arithmetic of any single output.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

#define ORC_OK 0
#define ORC_EINVAL -1

/* storage dtypes of an orc_mat */
#define ORC_F64 0
#define ORC_F32 1
#define ORC_BF16 2
#define ORC_E4M3 3 /* one fp32 scale per row */
#define ORC_E2M1 4 /* one e4m3 scale byte per 16 elements of a row */

typedef struct {
  int32_t dtype;
  int32_t pad_;
  const void* data;  /* rows x cols elements, row-major, densely packed;
                        E2M1: rows x cols/2 bytes, element 2i in the low
                        nibble of byte i, element 2i+1 in the high nibble */
  const void* scale; /* E4M3: float[rows]; E2M1: uint8[rows * cols/16] */
  int64_t rows;
  int64_t cols;
} orc_mat;

/* ------------------------------------------------------------------ */
/* bit-level decoders (bf16: top half of an IEEE binary32; e4m3 / e2m1:  */
/* OCP 8-bit floating point and OCP microscaling format definitions)     */
/* ------------------------------------------------------------------ */

double orc_bf16_to_f64(uint16_t h) {
  uint32_t u = ((uint32_t)h) << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return (double)f;
}

/* E4M3 (OFP8 "E4M3FN"): 1 sign, 4 exponent (bias 7), 3 mantissa bits, no
 * infinities, S.1111.111 is NaN, largest finite 448, subnormals m * 2^-9. */
double orc_e4m3_to_f64(uint8_t b) {
  int s = (b >> 7) & 1;
  int e = (b >> 3) & 15;
  int m = b & 7;
  double v;
  if (e == 15 && m == 7) return NAN;
  if (e == 0)
    v = ldexp((double)m, -9);
  else
    v = ldexp(1.0 + m / 8.0, e - 7);
  return s ? -v : v;
}

/* E2M1 (OCP MX FP4): 1 sign, 2 exponent (bias 1), 1 mantissa bit; values
 * 0, 0.5, 1, 1.5, 2, 3, 4, 6 and their negatives. */
double orc_e2m1_to_f64(uint8_t nib) {
  int s = (nib >> 3) & 1;
  int e = (nib >> 1) & 3;
  int m = nib & 1;
  double v;
  if (e == 0)
    v = 0.5 * m;
  else
    v = ldexp(1.0 + 0.5 * m, e - 1);
  return s ? -v : v;
}

/* element (r, c) of a stored matrix, decoded to fp64 */
double orc_mat_at(const orc_mat* a, int64_t r, int64_t c) {
  int64_t i = r * a->cols + c;
  switch (a->dtype) {
    case ORC_F64:
      return ((const double*)a->data)[i];
    case ORC_F32:
      return (double)((const float*)a->data)[i];
    case ORC_BF16:
      return orc_bf16_to_f64(((const uint16_t*)a->data)[i]);
    case ORC_E4M3: {
      double s = (double)((const float*)a->scale)[r];
      return s * orc_e4m3_to_f64(((const uint8_t*)a->data)[i]);
    }
    case ORC_E2M1: {
      uint8_t byte = ((const uint8_t*)a->data)[i >> 1];
      uint8_t nib = (i & 1) ? (byte >> 4) : (byte & 15);
      uint8_t sc = ((const uint8_t*)a->scale)[r * (a->cols / 16) + c / 16];
      return orc_e4m3_to_f64(sc) * orc_e2m1_to_f64(nib);
    }
    default:
      return NAN;
  }
}

int orc_mat_decode(const orc_mat* a, double* out) {
  if (a->dtype < ORC_F64 || a->dtype > ORC_E2M1) return ORC_EINVAL;
  if (a->dtype == ORC_E2M1 && (a->cols % 16) != 0) return ORC_EINVAL;
  for (int64_t r = 0; r < a->rows; ++r)
    for (int64_t c = 0; c < a->cols; ++c) out[r * a->cols + c] = orc_mat_at(a, r, c);
  return ORC_OK;
}

/* ------------------------------------------------------------------ */
/* round-to-nearest-even encoders                                      */
/* ------------------------------------------------------------------ */

/* nearest representable value of a format with `p` significant bits, smallest
 * normal exponent `emin` (so the subnormal quantum is 2^(emin - p + 1)), ties
 * to even; no overflow handling (callers saturate or check). */
static double round_to_format(double x, int p, int emin) {
  if (x == 0.0 || !isfinite(x)) return x;
  double ax = fabs(x);
  int e;
  frexp(ax, &e);      /* ax in [2^(e-1), 2^e) */
  int ebin = e - 1;   /* ax in [2^ebin, 2^(ebin+1)) */
  if (ebin < emin) ebin = emin;
  double quantum = ldexp(1.0, ebin - (p - 1));
  double q = nearbyint(ax / quantum) * quantum; /* default mode: ties to even */
  return x < 0 ? -q : q;
}

/* fp32 <- fp64, round to nearest even (the C conversion) */
static float to_f32(double x) { return (float)x; }

/* bf16 <- fp32, round to nearest even; returns the bf16 bit pattern */
uint16_t orc_f32_to_bf16_bits(float x) {
  if (isnan(x)) return 0x7FC0;
  double q = round_to_format((double)x, 8, -126);
  float qf = (float)q; /* exact: q has <= 8 significant bits (or is inf) */
  if (fabs(q) > 3.3895313892515355e38) qf = x < 0 ? -INFINITY : INFINITY;
  uint32_t u;
  memcpy(&u, &qf, sizeof u);
  return (uint16_t)(u >> 16);
}

/* e4m3 code of x (fp32 value), round to nearest even, saturate to +-448 */
uint8_t orc_f32_to_e4m3(float x) {
  double v = round_to_format((double)x, 4, -6);
  int s = v < 0 || (v == 0 && signbit(x));
  double a = fabs(v);
  if (a > 448.0) a = 448.0;
  if (a == 0.0) return (uint8_t)(s << 7);
  int e;
  frexp(a, &e);
  int ebin = e - 1;
  uint8_t code;
  if (ebin < -6) { /* subnormal: a = m * 2^-9 */
    int m = (int)(a / ldexp(1.0, -9));
    code = (uint8_t)m;
  } else {
    int m = (int)((a / ldexp(1.0, ebin) - 1.0) * 8.0);
    code = (uint8_t)(((ebin + 7) << 3) | m);
  }
  return (uint8_t)((s << 7) | code);
}

/* e2m1 nibble of x (fp32 value), round to nearest even, saturate to +-6 */
uint8_t orc_f32_to_e2m1(float x) {
  double v = round_to_format((double)x, 2, 0);
  int s = v < 0 || (v == 0 && signbit(x));
  double a = fabs(v);
  if (a > 6.0) a = 6.0;
  uint8_t code;
  if (a < 1.0)
    code = (uint8_t)(a / 0.5); /* 0 or 0.5: exponent field 0 */
  else {
    int e;
    frexp(a, &e);
    int ebin = e - 1; /* 0, 1 or 2 */
    int m = (int)((a / ldexp(1.0, ebin) - 1.0) * 2.0);
    code = (uint8_t)(((ebin + 1) << 1) | m);
  }
  return (uint8_t)((s << 3) | code);
}

/* Store rows of fp64 values in the given storage dtype.
 *   BF16: value -> fp32 (RNE) -> bf16 (RNE).
 *   E4M3: per row, amax over the fp32 values, scale = amax / 448 in fp32
 *         (1 when amax == 0), code = e4m3(value / scale).
 *   E2M1: per 16-element block, amax over the fp32 values, scale byte =
 *         e4m3(amax / 6); value code = e2m1(value / decoded scale) (0 when the
 *         decoded scale is 0).                                               */
int orc_store_rows(const double* in, int64_t rows, int64_t cols, int32_t dtype, void* data,
                   void* scale) {
  if (dtype == ORC_BF16) {
    uint16_t* o = (uint16_t*)data;
    for (int64_t i = 0; i < rows * cols; ++i) o[i] = orc_f32_to_bf16_bits(to_f32(in[i]));
    return ORC_OK;
  }
  if (dtype == ORC_F32) {
    float* o = (float*)data;
    for (int64_t i = 0; i < rows * cols; ++i) o[i] = to_f32(in[i]);
    return ORC_OK;
  }
  if (dtype == ORC_E4M3) {
    uint8_t* o = (uint8_t*)data;
    float* sc = (float*)scale;
    for (int64_t r = 0; r < rows; ++r) {
      float amax = 0.0f;
      for (int64_t c = 0; c < cols; ++c) {
        float a = fabsf(to_f32(in[r * cols + c]));
        if (a > amax) amax = a;
      }
      float s = amax > 0.0f ? amax / 448.0f : 1.0f;
      sc[r] = s;
      for (int64_t c = 0; c < cols; ++c) o[r * cols + c] = orc_f32_to_e4m3(to_f32(in[r * cols + c]) / s);
    }
    return ORC_OK;
  }
  if (dtype == ORC_E2M1) {
    if (cols % 16) return ORC_EINVAL;
    uint8_t* o = (uint8_t*)data;
    uint8_t* sc = (uint8_t*)scale;
    memset(o, 0, (size_t)(rows * cols / 2));
    for (int64_t r = 0; r < rows; ++r) {
      for (int64_t b = 0; b < cols / 16; ++b) {
        float amax = 0.0f;
        for (int64_t c = b * 16; c < b * 16 + 16; ++c) {
          float a = fabsf(to_f32(in[r * cols + c]));
          if (a > amax) amax = a;
        }
        uint8_t sb = orc_f32_to_e4m3(amax / 6.0f);
        sc[r * (cols / 16) + b] = sb;
        float sd = (float)orc_e4m3_to_f64(sb);
        for (int64_t c = b * 16; c < b * 16 + 16; ++c) {
          uint8_t nib = sd > 0.0f ? orc_f32_to_e2m1(to_f32(in[r * cols + c]) / sd) : 0;
          int64_t i = r * cols + c;
          o[i >> 1] |= (uint8_t)((i & 1) ? (nib << 4) : nib);
        }
      }
    }
    return ORC_OK;
  }
  return ORC_EINVAL;
}

/* ------------------------------------------------------------------ */
/* a1 / a2: KV compression ([book] section 4: CSA folds every m = 4     */
/* tokens into one entry, HCA every m' = 128; [digest] section 3;       */
/* [essay]: weighted fusion of several tokens' KV into one; [10100]    */
/* 2.1: position weighting).                                           */
/*                                                                     */
/* For block j and channel c:                                          */
/*   l_i   = Z[j*m + i, c] + B[i, c]           (i = 0 .. m-1)          */
/*   a_i   = exp(l_i - max_i l_i) / sum_i exp(l_i - max_i l_i)         */
/*   C[j,c] = sum_i a_i * X[j*m + i, c]                                */
/* Z has 1 column (one logit per token, shared by all channels) or d.  */
/* ------------------------------------------------------------------ */
int orc_compress(const orc_mat* x, const orc_mat* z, const double* bias, int64_t m,
                 double* out) {
  int64_t n = x->rows, d = x->cols;
  if (m <= 0 || n % m != 0) return ORC_EINVAL;
  if (z->rows != n || (z->cols != 1 && z->cols != d)) return ORC_EINVAL;
  int64_t nb = n / m;
#pragma omp parallel for schedule(static)
  for (int64_t j = 0; j < nb; ++j) {
    double* l = (double*)malloc(sizeof(double) * (size_t)m);
    for (int64_t c = 0; c < d; ++c) {
      double mx = -INFINITY;
      for (int64_t i = 0; i < m; ++i) {
        l[i] = orc_mat_at(z, j * m + i, z->cols == 1 ? 0 : c) + (bias ? bias[i * d + c] : 0.0);
        if (l[i] > mx) mx = l[i];
      }
      double den = 0.0;
      for (int64_t i = 0; i < m; ++i) den += exp(l[i] - mx);
      double acc = 0.0;
      for (int64_t i = 0; i < m; ++i) acc += (exp(l[i] - mx) / den) * orc_mat_at(x, j * m + i, c);
      out[j * d + c] = acc;
    }
    free(l);
  }
  return ORC_OK;
}

/* ------------------------------------------------------------------ */
/* a1 / a2 with block overlap ([10100] 2.1: block compression "combined */
/* with position weighting and block overlap", width unstated).         */
/* Reading: entry j also folds the last `ov` tokens of the block before */
/* it, i.e. the tokens at positions max(0, j*m - ov) .. j*m + m - 1 of  */
/* the stream, under one softmax; the position bias then has m + ov     */
/* rows, row r for the token at position j*m - ov + r. x and z hold the */
/* stream from position 0; ov = 0 is the plain fold above. The entry is */
/* complete when its own block is, so visibility does not change.       */
/*   l_p   = Z[p, c] + B[p - (j*m - ov), c]                             */
/*   a_p   = exp(l_p - max l) / sum_p exp(l_p - max l)                  */
/*   C[j,c] = sum_p a_p X[p, c]     (p over the positions above)        */
/* ------------------------------------------------------------------ */
int orc_compress_overlap(const orc_mat* x, const orc_mat* z, const double* bias, int64_t m, int64_t ov,
                         double* out) {
  int64_t n = x->rows, d = x->cols;
  if (m <= 0 || ov < 0 || n % m != 0) return ORC_EINVAL;
  if (z->rows != n || (z->cols != 1 && z->cols != d)) return ORC_EINVAL;
  int64_t nb = n / m;
#pragma omp parallel for schedule(static)
  for (int64_t j = 0; j < nb; ++j) {
    int64_t first = j * m - ov < 0 ? 0 : j * m - ov;
    int64_t last = j * m + m - 1;
    double* l = (double*)malloc(sizeof(double) * (size_t)(m + ov));
    for (int64_t c = 0; c < d; ++c) {
      double mx = -INFINITY;
      for (int64_t p = first; p <= last; ++p) {
        double v = orc_mat_at(z, p, z->cols == 1 ? 0 : c) + (bias ? bias[(p - (j * m - ov)) * d + c] : 0.0);
        l[p - first] = v;
        if (v > mx) mx = v;
      }
      double den = 0.0;
      for (int64_t p = first; p <= last; ++p) den += exp(l[p - first] - mx);
      double acc = 0.0;
      for (int64_t p = first; p <= last; ++p) acc += (exp(l[p - first] - mx) / den) * orc_mat_at(x, p, c);
      out[j * d + c] = acc;
    }
    free(l);
  }
  return ORC_OK;
}

/* ------------------------------------------------------------------ */
/* BF16 index scores ([digest] section 7: the indexer's scores are kept */
/* in BF16 instead of FP32, which halves the selector's cost at 99.7%   */
/* recall of the FP32 selection). Reading: each score, computed in      */
/* fp32, is rounded to bf16 (round to nearest even) and the top-k of    */
/* the rounded scores is taken with the usual order (score desc, index  */
/* asc), so entries whose scores round together are taken in index      */
/* order. This function does the rounding: fp64 -> fp32 -> bf16.       */
/* ------------------------------------------------------------------ */
int orc_round_scores_bf16(const double* scores, int64_t n, double* out) {
  for (int64_t j = 0; j < n; ++j) out[j] = orc_bf16_to_f64(orc_f32_to_bf16_bits(to_f32(scores[j])));
  return ORC_OK;
}

/* ------------------------------------------------------------------ */
/* Inverse RoPE on the attention output ([essay] "约束1 -> 创新1": with */
/* 128 tokens sharing one compressed entry, position is restored by an */
/* inverse-RoPE correction applied to the attention output). Reading:  */
/* the channels [r0, r0 + d_rope) of each output row form d_rope / 2   */
/* pairs (r0 + 2i, r0 + 2i + 1) carrying RoPE at frequency             */
/*   theta_i = base^(-2i / d_rope);                                    */
/* a value rotated by its key's position p, summed with attention      */
/* weights, becomes relative to the query at position t after a        */
/* rotation by -t theta_i:                                             */
/*   (a, b) <- (a cos(t theta_i) + b sin(t theta_i),                   */
/*              -a sin(t theta_i) + b cos(t theta_i)).                 */
/* o is [rows, cols], rotated in place.                                */
/* ------------------------------------------------------------------ */
int orc_inverse_rope(double* o, int64_t rows, int64_t cols, int64_t r0, int64_t d_rope, int64_t t, double base) {
  if (d_rope <= 0 || d_rope % 2 || r0 < 0 || r0 + d_rope > cols || base <= 0.0) return ORC_EINVAL;
  for (int64_t r = 0; r < rows; ++r) {
    for (int64_t i = 0; i < d_rope / 2; ++i) {
      double theta = pow(base, -2.0 * (double)i / (double)d_rope);
      double ang = (double)t * theta;
      double cs = cos(ang), sn = sin(ang);
      double* a = o + r * cols + r0 + 2 * i;
      double x = a[0], y = a[1];
      a[0] = x * cs + y * sn;
      a[1] = -x * sn + y * cs;
    }
  }
  return ORC_OK;
}

/* ------------------------------------------------------------------ */
/* visibility (reading: an entry is visible iff its block starts before */
/* the window of the last n_win raw tokens; [digest] section 3: both    */
/* branches add the last n_win = 128 uncompressed tokens)               */
/* ------------------------------------------------------------------ */
int64_t orc_visible_entries(int64_t t, int64_t m, int64_t n_win) {
  int64_t lim = t + 1 - n_win; /* entry j visible iff j*m < lim */
  if (lim <= 0) return 0;
  return (lim + m - 1) / m;
}

int64_t orc_window_start(int64_t t, int64_t n_win) {
  int64_t s = t - n_win + 1;
  return s < 0 ? 0 : s;
}

/* ------------------------------------------------------------------ */
/* a4: Lightning-indexer score ([book] section 4; [10100] 2.1 low-rank   */
/* indexer; [digest] section 3): for every visible entry j,             */
/*   s(j) = sum_h w[h] * max(0, sum_c qI[h, c] * KI[j, c])              */
/* ------------------------------------------------------------------ */
int orc_index_scores(const orc_mat* qI, const double* w, const orc_mat* kI, int64_t n_vis,
                     double* scores) {
  int64_t HI = qI->rows, dI = qI->cols;
  if (kI->cols != dI || n_vis > kI->rows) return ORC_EINVAL;
#pragma omp parallel for schedule(static)
  for (int64_t j = 0; j < n_vis; ++j) {
    double s = 0.0;
    for (int64_t h = 0; h < HI; ++h) {
      double dot = 0.0;
      for (int64_t c = 0; c < dI; ++c) dot += orc_mat_at(qI, h, c) * orc_mat_at(kI, j, c);
      s += w[h] * (dot > 0.0 ? dot : 0.0);
    }
    scores[j] = s;
  }
  return ORC_OK;
}

/* ------------------------------------------------------------------ */
/* a5: top-k selection ([digest] section 3: k = 512 Flash, 1024 Pro;    */
/* [10100] 2.1). The k_eff = min(k, n) indices with the largest score;  */
/* equal scores prefer the lower index. Output ascending, -1 padded.    */
/* Returns k_eff. Plain selection: a full sort by (score desc, idx asc).*/
/* ------------------------------------------------------------------ */
static const double* g_sort_scores; /* used only by the comparator below */
static int cmp_score_desc_idx_asc(const void* a, const void* b) {
  int32_t i = *(const int32_t*)a, j = *(const int32_t*)b;
  double si = g_sort_scores[i], sj = g_sort_scores[j];
  if (si > sj) return -1;
  if (si < sj) return 1;
  return (i > j) - (i < j);
}
static int cmp_i32(const void* a, const void* b) {
  int32_t i = *(const int32_t*)a, j = *(const int32_t*)b;
  return (i > j) - (i < j);
}

int64_t orc_topk(const double* scores, int64_t n, int64_t k, int32_t* idx_out) {
  int64_t keff = n < k ? n : k;
  int32_t* order = (int32_t*)malloc(sizeof(int32_t) * (size_t)(n > 0 ? n : 1));
  for (int64_t j = 0; j < n; ++j) order[j] = (int32_t)j;
#pragma omp critical(orc_topk_sort)
  {
    g_sort_scores = scores;
    qsort(order, (size_t)n, sizeof(int32_t), cmp_score_desc_idx_asc);
  }
  qsort(order, (size_t)keff, sizeof(int32_t), cmp_i32);
  for (int64_t i = 0; i < k; ++i) idx_out[i] = i < keff ? order[i] : -1;
  free(order);
  return keff;
}

/* ------------------------------------------------------------------ */
/* a6 / a7: attention over one key set ([digest] section 3: one softmax */
/* over window keys and selected (CSA) or all (HCA) compressed keys;    */
/* shared latent KV, MQA: every head reads the same K_u, and V_u is the */
/* first d_v channels of K_u).                                          */
/*   logit[h,u] = sm_scale * sum_c q[h,c] K_u[c]   (c < d_qk)           */
/*   p[h,u]     = exp(logit - max) / sum_u exp(logit - max)             */
/*   o[h,c]     = sum_u p[h,u] K_u[c]              (c < d_v)            */
/*   lse[h]     = log sum_u exp(logit[h,u])                             */
/* keys[u] is row u of `keys`.                                          */
/* ------------------------------------------------------------------ */
int orc_attend(const orc_mat* q, const orc_mat* keys, int64_t dv, double sm_scale, double* o,
               double* lse) {
  int64_t H = q->rows, dqk = q->cols, N = keys->rows;
  if (keys->cols != dqk || dv > dqk || dv <= 0) return ORC_EINVAL;
#pragma omp parallel for schedule(static)
  for (int64_t h = 0; h < H; ++h) {
    if (N == 0) {
      for (int64_t c = 0; c < dv; ++c) o[h * dv + c] = 0.0;
      if (lse) lse[h] = -INFINITY;
      continue;
    }
    double* lg = (double*)malloc(sizeof(double) * (size_t)N);
    double mx = -INFINITY;
    for (int64_t u = 0; u < N; ++u) {
      double dot = 0.0;
      for (int64_t c = 0; c < dqk; ++c) dot += orc_mat_at(q, h, c) * orc_mat_at(keys, u, c);
      lg[u] = sm_scale * dot;
      if (lg[u] > mx) mx = lg[u];
    }
    double den = 0.0;
    for (int64_t u = 0; u < N; ++u) den += exp(lg[u] - mx);
    for (int64_t c = 0; c < dv; ++c) {
      double acc = 0.0;
      for (int64_t u = 0; u < N; ++u) acc += (exp(lg[u] - mx) / den) * orc_mat_at(keys, u, c);
      o[h * dv + c] = acc;
    }
    if (lse) lse[h] = mx + log(den);
    free(lg);
  }
  return ORC_OK;
}

/* ------------------------------------------------------------------ */
/* One query through a CSA layer and through an HCA layer.              */
/*                                                                      */
/* win:   raw latent-KV rows of positions max(0, t-n_win+1) .. t, in    */
/*        position order (the window branch).                           */
/* kv:    stored compressed entries 0 .. (at least n_vis-1) of the       */
/*        layer, rows of d_qk.                                          */
/* kI:    stored compressed indexer keys (CSA only).                    */
/* The key set is the window rows followed by the chosen entries; the   */
/* order of the key set does not change the softmax.                    */
/* ------------------------------------------------------------------ */
static int attend_union(const orc_mat* q, const orc_mat* win, const orc_mat* kv,
                        const int32_t* sel, int64_t nsel, int64_t dv, double sm_scale, double* o,
                        double* lse) {
  int64_t dqk = q->cols;
  int64_t nw = win->rows;
  int64_t N = nw + nsel;
  double* keys = (double*)malloc(sizeof(double) * (size_t)((N > 0 ? N : 1) * dqk));
  for (int64_t u = 0; u < nw; ++u)
    for (int64_t c = 0; c < dqk; ++c) keys[u * dqk + c] = orc_mat_at(win, u, c);
  for (int64_t i = 0; i < nsel; ++i)
    for (int64_t c = 0; c < dqk; ++c) keys[(nw + i) * dqk + c] = orc_mat_at(kv, sel[i], c);
  orc_mat km = {ORC_F64, 0, keys, NULL, N, dqk};
  int rc = orc_attend(q, &km, dv, sm_scale, o, lse);
  free(keys);
  return rc;
}

int orc_csa_query(int64_t t, int64_t m, int64_t n_win, int64_t k, const orc_mat* q,
                  const orc_mat* qI, const double* w, const orc_mat* win, const orc_mat* kv,
                  const orc_mat* kI, int64_t dv, double sm_scale, int32_t* idx_out,
                  double* scores_out, double* o, double* lse) {
  int64_t n_vis = orc_visible_entries(t, m, n_win);
  if (win->rows != t - orc_window_start(t, n_win) + 1) return ORC_EINVAL;
  if (kv->rows < n_vis || kI->rows < n_vis || win->cols != q->cols || kv->cols != q->cols)
    return ORC_EINVAL;
  double* s = scores_out ? scores_out : (double*)malloc(sizeof(double) * (size_t)(n_vis + 1));
  int rc = orc_index_scores(qI, w, kI, n_vis, s);
  if (rc == ORC_OK) {
    int64_t keff = orc_topk(s, n_vis, k, idx_out);
    rc = attend_union(q, win, kv, idx_out, keff, dv, sm_scale, o, lse);
  }
  if (!scores_out) free(s);
  return rc;
}

int orc_hca_query(int64_t t, int64_t m, int64_t n_win, const orc_mat* q, const orc_mat* win,
                  const orc_mat* kv, int64_t dv, double sm_scale, double* o, double* lse) {
  int64_t n_vis = orc_visible_entries(t, m, n_win);
  if (win->rows != t - orc_window_start(t, n_win) + 1) return ORC_EINVAL;
  if (kv->rows < n_vis || win->cols != q->cols || kv->cols != q->cols) return ORC_EINVAL;
  int32_t* all = (int32_t*)malloc(sizeof(int32_t) * (size_t)(n_vis + 1));
  for (int64_t j = 0; j < n_vis; ++j) all[j] = (int32_t)j;
  int rc = attend_union(q, win, kv, all, n_vis, dv, sm_scale, o, lse);
  free(all);
  return rc;
}

int orc_num_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

void orc_set_num_threads(int n) {
#ifdef _OPENMP
  if (n > 0) omp_set_num_threads(n);
#else
  (void)n;
#endif
}
