/*
 * CPU oracle for absorbed MLA split-KV decode — TEST INFRASTRUCTURE ONLY.
 *
 * This file is the plain, slow, obviously-correct statement of what the GPU
 * path computes.  It is compiled into liboracle.so and called only from the
 * tests, from the smoke check and from the benchmark's CPU-baseline leg.  It
 * shares no code, header or table with the CUDA library and never touches a
 * GPU.  Arithmetic is IEEE fp64 except where the method fixes fp32 (the single
 * fp32 multiply in front of the FP8 rounding).
 *
 * Sources followed (each function cites its own):
 *  - "SGLang & Miles ... Vera Rubin" article (arex-research.com), section
 *    "Kimi K3 的 MLA：更深的流水线、更快的 split-KV 归约":
 *      bullet "更快的 split-KV 归约"  — split one request's KV across CTAs,
 *        a second kernel merges the partial results;
 *      bullet "原生 FP8 转换"          — KV/Q converted to FP8 with a
 *        saturating conversion: overflow clamps to +-448, never NaN.
 *  - "Muse Spark Open" article (theainews.cc), section "内核优化：解码吞吐 3
 *    倍", bullet "RoPE 与 KV 缓存写入融合" — RoPE applied in the kernel that
 *    writes the decode KV cache (the KV-append step before the path).
 *  - The OCP 8-bit floating point specification (E4M3: bias 7, no infinity,
 *    S.1111.111 is NaN, largest finite 448) for the code <-> value map.
 *  - Absorbed MLA as a plain softmax(q k^T * scale) v over one 576-wide latent
 *    row per token (512 latent dims that are also V, plus 64 RoPE dims).  The
 *    pages name MLA but print no formula; this is the standard reading.
 *
 * Every function here is pinned by tests that do not call it back (brute
 * force in NumPy, closed forms, invariants); see tests/test_oracle.py.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>
#include <stdlib.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define D_LATENT 512
#define D_ROPE 64
#define D_ROW 576
#define PAGE 64

/* ------------------------------------------------------------------------ */
/* bf16 and E4M3 values                                                      */
/* ------------------------------------------------------------------------ */

/* bf16 is the top half of an IEEE binary32; its value is exact in fp32. */
static float bf16_to_f32(uint16_t b) {
  uint32_t u = ((uint32_t)b) << 16;
  float f;
  memcpy(&f, &u, 4);
  return f;
}

/* Value of an E4M3 code per the OCP FP8 format: 1 sign bit, 4 exponent bits
 * with bias 7, 3 mantissa bits; exponent 0 is subnormal (m/8 * 2^-6);
 * S.1111.111 is NaN; there is no infinity. */
double oracle_e4m3_value(uint8_t code) {
  int sign = (code >> 7) & 1;
  int e = (code >> 3) & 15;
  int m = code & 7;
  double v;
  if (e == 15 && m == 7) return NAN;
  if (e == 0)
    v = ldexp((double)m / 8.0, -6);
  else
    v = ldexp(1.0 + (double)m / 8.0, e - 7);
  return sign ? -v : v;
}

/* Table of the 256 code values, filled from oracle_e4m3_value (the
 * definition above) before any parallel region uses it. */
static double g_e4m3[256];
static int g_e4m3_ready = 0;
static void init_tables(void) {
  if (g_e4m3_ready) return;
  for (int c = 0; c < 256; ++c) g_e4m3[c] = oracle_e4m3_value((uint8_t)c);
  g_e4m3_ready = 1;
}

/* Round an fp32 value to E4M3, round-to-nearest with ties to the even code,
 * saturating: any finite value of magnitude 448 or more, and +-inf, become
 * +-448 (page 1, bullet "原生 FP8 转换": overflow clamps to +-448 instead of
 * becoming NaN).  NaN maps to the positive NaN code 0x7F.  The non-negative
 * finite codes 0x00..0x7E are increasing in value, so the nearest code is
 * found by bisection for the last code not above |x| and a comparison with
 * its successor; equal distances pick the code with an even mantissa. */
uint8_t oracle_e4m3_encode(float x) {
  init_tables();
  if (isnan(x)) return 0x7F;
  int neg = signbit(x) ? 1 : 0;
  double a = fabs((double)x);
  int best;
  if (a >= 448.0) {
    best = 0x7E;
  } else {
    int lo = 0, hi = 0x7E; /* invariant: value(lo) <= a < value(hi) */
    while (hi - lo > 1) {
      int mid = (lo + hi) / 2;
      if (g_e4m3[mid] <= a) lo = mid; else hi = mid;
    }
    double dlo = a - g_e4m3[lo], dhi = g_e4m3[hi] - a;
    if (dlo < dhi) best = lo;
    else if (dhi < dlo) best = hi;
    else best = (lo & 1) == 0 ? lo : hi;
  }
  return (uint8_t)(best | (neg ? 0x80 : 0x00));
}

/* Step A1 (prep): y = E4M3_satfinite_RN( fl32( fp32(x) * inv_scale ) ).
 * One fp32 multiply rounded to nearest, then one E4M3 rounding — no
 * intermediate 16-bit rounding. */
void oracle_quantize(const uint16_t* x, uint8_t* y, int64_t n, float inv_scale) {
  init_tables();
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < n; ++i) {
    volatile float p = bf16_to_f32(x[i]) * inv_scale; /* one IEEE fp32 RN multiply */
    y[i] = oracle_e4m3_encode(p);
  }
}

/* ------------------------------------------------------------------------ */
/* Attention                                                                 */
/* ------------------------------------------------------------------------ */

/* Dequantised value of element d of token t of request b.
 * kv_dtype 0: E4M3 code times kv_scale; kv_dtype 1: the exact bf16 value. */
static double kv_elem(const void* kv_pages, int kv_dtype, double kv_scale,
                      int64_t page, int slot, int d) {
  int64_t idx = (page * PAGE + slot) * (int64_t)D_ROW + d;
  if (kv_dtype == 0)
    return g_e4m3[((const uint8_t*)kv_pages)[idx]] * kv_scale;
  return (double)bf16_to_f32(((const uint16_t*)kv_pages)[idx]);
}

/* Page that holds token t of request b: block_table[b][t / 64]. */
static int64_t page_of(const int32_t* block_table, int max_pages, int b, int64_t t) {
  return (int64_t)block_table[(int64_t)b * max_pages + t / PAGE];
}

/* One query row over the token range [t0, t1):
 *   s_t = softmax_scale * (sum_i qn_i k_t,i + sum_j qr_j k_t,512+j)
 *   m = max s,  O = sum e^{s_t-m} v_t / sum e^{s_t-m},  LSE = m + ln sum e^{s_t-m}
 * with v_t the first 512 dims of token t's row.  An empty range gives O = 0,
 * LSE = -inf.  Two passes over the tokens: scores and max, then weights. */
static void attend_range(const double* q, const void* kv_pages,
                         int kv_dtype, double kv_scale, const int32_t* block_table,
                         int max_pages, int b, int64_t t0, int64_t t1,
                         double softmax_scale, double* o, double* lse, double* s_buf) {
  for (int d = 0; d < D_LATENT; ++d) o[d] = 0.0;
  if (t1 <= t0) {
    *lse = -INFINITY;
    return;
  }

  double m = -INFINITY;
  for (int64_t t = t0; t < t1; ++t) {
    int64_t page = page_of(block_table, max_pages, b, t);
    int slot = (int)(t % PAGE);
    double acc = 0.0;
    for (int d = 0; d < D_ROW; ++d)
      acc += q[d] * kv_elem(kv_pages, kv_dtype, kv_scale, page, slot, d);
    double s = softmax_scale * acc;
    s_buf[t - t0] = s;
    if (s > m) m = s;
  }
  double l = 0.0;
  for (int64_t t = t0; t < t1; ++t) {
    double w = exp(s_buf[t - t0] - m);
    l += w;
    int64_t page = page_of(block_table, max_pages, b, t);
    int slot = (int)(t % PAGE);
    for (int d = 0; d < D_LATENT; ++d)
      o[d] += w * kv_elem(kv_pages, kv_dtype, kv_scale, page, slot, d);
  }
  for (int d = 0; d < D_LATENT; ++d) o[d] /= l;
  *lse = m + log(l);
}

/* A bf16 query row (q_nope then q_rope) as 576 fp64 values. */
static void q_from_bf16(const uint16_t* qn, const uint16_t* qr, double* q) {
  for (int d = 0; d < D_LATENT; ++d) q[d] = (double)bf16_to_f32(qn[d]);
  for (int d = 0; d < D_ROPE; ++d) q[D_LATENT + d] = (double)bf16_to_f32(qr[d]);
}

/* Causal visible length of query position q of request b (seq_len includes
 * the q_len new tokens): row q sees tokens 0 .. L_b - q_len + q. */
static int64_t visible_len(int64_t L, int q_len, int q) { return L - q_len + q + 1; }

/* Full (unsplit) decode for a list of rows.  rows[i] = (b*q_len + q)*H + h.
 * q_nope: [B][q_len][H][512] bf16, q_rope: [B][q_len][H][64] bf16,
 * kv_pages: [num_pages][64][576] (E4M3 codes or bf16), block_table:
 * [B][max_pages] int32, seq_lens: [B] int32.  Outputs per listed row:
 * out_o[i][512] and out_lse[i] in fp64. */
void oracle_mla_decode_rows(const uint16_t* q_nope, const uint16_t* q_rope,
                            const void* kv_pages, int kv_dtype, float kv_scale,
                            const int32_t* block_table, int max_pages,
                            const int32_t* seq_lens, int B, int q_len, int H,
                            float softmax_scale, const int64_t* rows, int64_t n_rows,
                            double* out_o, double* out_lse) {
  init_tables();
  int64_t max_len = 0;
  for (int b = 0; b < B; ++b)
    if (seq_lens[b] > max_len) max_len = seq_lens[b];
#pragma omp parallel
  {
    double* s_buf = (double*)malloc(sizeof(double) * (size_t)(max_len > 0 ? max_len : 1));
#pragma omp for schedule(dynamic, 1)
    for (int64_t i = 0; i < n_rows; ++i) {
      int64_t r = rows[i];
      int q = (int)((r / H) % q_len);
      int b = (int)(r / ((int64_t)H * q_len));
      int64_t vis = visible_len(seq_lens[b], q_len, q);
      double qv[D_ROW];
      q_from_bf16(q_nope + r * D_LATENT, q_rope + r * D_ROPE, qv);
      attend_range(qv, kv_pages, kv_dtype, (double)kv_scale, block_table, max_pages, b, 0, vis,
                   (double)softmax_scale, out_o + i * D_LATENT, out_lse + i, s_buf);
    }
    free(s_buf);
  }
}

/* Step A2, split planning (page 1, bullet "更快的 split-KV 归约": one request's
 * KV is cut across many CTAs).  The pages do not give the partition; the
 * reading used is equal page-aligned chunks: with n = ceil(L/64) pages and S
 * splits, c = ceil(n/S) and split s owns pages [s*c, min((s+1)*c, n)).
 * Returns the token range [*t0, *t1) of split s, clipped to the causal
 * visible length vis. */
void oracle_split_range(int64_t L, int S, int s, int64_t vis, int64_t* t0, int64_t* t1) {
  int64_t n_pages = (L + PAGE - 1) / PAGE;
  int64_t c = (n_pages + S - 1) / S;
  int64_t p0 = (int64_t)s * c, p1 = (int64_t)(s + 1) * c;
  if (p0 > n_pages) p0 = n_pages;
  if (p1 > n_pages) p1 = n_pages;
  int64_t a = p0 * PAGE, e = p1 * PAGE;
  if (e > vis) e = vis;
  if (a > e) a = e;
  *t0 = a;
  *t1 = e;
}

/* Per-split partial results (steps A3-A8 per split): for each listed row and
 * each split s < num_splits[b], the normalised partial O_s (512 fp64) and its
 * LSE_s (natural log, scaled-score units).  Splits s >= num_splits[b] and
 * empty splits give O_s = 0, LSE_s = -inf.  Output layout per listed row i:
 * out_o[(i*max_splits + s)*512 + d], out_lse[i*max_splits + s]. */
void oracle_mla_partials_rows(const uint16_t* q_nope, const uint16_t* q_rope,
                              const void* kv_pages, int kv_dtype, float kv_scale,
                              const int32_t* block_table, int max_pages,
                              const int32_t* seq_lens, const int32_t* num_splits,
                              int max_splits, int B, int q_len, int H, float softmax_scale,
                              const int64_t* rows, int64_t n_rows, double* out_o,
                              double* out_lse) {
  init_tables();
  int64_t max_len = 0;
  for (int b = 0; b < B; ++b)
    if (seq_lens[b] > max_len) max_len = seq_lens[b];
#pragma omp parallel
  {
    double* s_buf = (double*)malloc(sizeof(double) * (size_t)(max_len > 0 ? max_len : 1));
#pragma omp for schedule(dynamic, 1) collapse(2)
    for (int64_t i = 0; i < n_rows; ++i) {
      for (int s = 0; s < max_splits; ++s) {
        int64_t r = rows[i];
        int q = (int)((r / H) % q_len);
        int b = (int)(r / ((int64_t)H * q_len));
        double* o = out_o + (i * max_splits + s) * D_LATENT;
        double* lse = out_lse + i * max_splits + s;
        int64_t t0 = 0, t1 = 0;
        if (s < num_splits[b])
          oracle_split_range(seq_lens[b], num_splits[b], s,
                             visible_len(seq_lens[b], q_len, q), &t0, &t1);
        double qv[D_ROW];
        q_from_bf16(q_nope + r * D_LATENT, q_rope + r * D_ROPE, qv);
        attend_range(qv, kv_pages, kv_dtype, (double)kv_scale, block_table, max_pages, b, t0,
                     t1, (double)softmax_scale, o, lse, s_buf);
      }
    }
    free(s_buf);
  }
}

/* Per-split partials with an FP8 query (page 1, bullet "原生 FP8 转换": the
 * prep converts Q to FP8 as well as KV).  Query row r is the 576 E4M3 codes
 * q8[r*576 .. r*576+575] (512 latent dims, then 64 RoPE dims), whose values
 * are e4m3(code) * q_scale with one per-tensor scale; splits, causality and
 * the output layout are those of oracle_mla_partials_rows. */
void oracle_mla_partials_rows_q8(const uint8_t* q8, float q_scale, const void* kv_pages,
                                 int kv_dtype, float kv_scale, const int32_t* block_table,
                                 int max_pages, const int32_t* seq_lens,
                                 const int32_t* num_splits, int max_splits, int B, int q_len,
                                 int H, float softmax_scale, const int64_t* rows,
                                 int64_t n_rows, double* out_o, double* out_lse) {
  init_tables();
  int64_t max_len = 0;
  for (int b = 0; b < B; ++b)
    if (seq_lens[b] > max_len) max_len = seq_lens[b];
#pragma omp parallel
  {
    double* s_buf = (double*)malloc(sizeof(double) * (size_t)(max_len > 0 ? max_len : 1));
#pragma omp for schedule(dynamic, 1) collapse(2)
    for (int64_t i = 0; i < n_rows; ++i) {
      for (int s = 0; s < max_splits; ++s) {
        int64_t r = rows[i];
        int q = (int)((r / H) % q_len);
        int b = (int)(r / ((int64_t)H * q_len));
        double* o = out_o + (i * max_splits + s) * D_LATENT;
        double* lse = out_lse + i * max_splits + s;
        int64_t t0 = 0, t1 = 0;
        if (s < num_splits[b])
          oracle_split_range(seq_lens[b], num_splits[b], s,
                             visible_len(seq_lens[b], q_len, q), &t0, &t1);
        double qv[D_ROW];
        for (int d = 0; d < D_ROW; ++d) qv[d] = g_e4m3[q8[r * D_ROW + d]] * (double)q_scale;
        attend_range(qv, kv_pages, kv_dtype, (double)kv_scale, block_table, max_pages, b, t0,
                     t1, (double)softmax_scale, o, lse, s_buf);
      }
    }
    free(s_buf);
  }
}

/* Step A9, the merge done by the second kernel (page 1, bullet
 * "更快的 split-KV 归约"): with M = max_s LSE_s and w_s = e^{LSE_s - M},
 *   O = sum_s w_s O_s / sum_s w_s,   LSE = M + ln sum_s w_s.
 * Inputs are fp32 as the GPU stores them: part_o [R][max_splits][512],
 * part_lse [R][max_splits]; row r uses the first n_splits[r] entries.  If
 * every LSE_s is -inf the result is O = 0, LSE = -inf. */
void oracle_combine(const float* part_o, const float* part_lse, const int32_t* n_splits,
                    int max_splits, int64_t R, double* out_o, double* out_lse) {
#pragma omp parallel for schedule(static)
  for (int64_t r = 0; r < R; ++r) {
    int S = n_splits[r];
    double M = -INFINITY;
    for (int s = 0; s < S; ++s) {
      double v = (double)part_lse[r * max_splits + s];
      if (v > M) M = v;
    }
    double* o = out_o + r * D_LATENT;
    for (int d = 0; d < D_LATENT; ++d) o[d] = 0.0;
    if (M == -INFINITY) {
      out_lse[r] = -INFINITY;
      continue;
    }
    double wsum = 0.0;
    for (int s = 0; s < S; ++s) {
      double w = exp((double)part_lse[r * max_splits + s] - M);
      wsum += w;
      const float* os = part_o + (r * max_splits + s) * D_LATENT;
      for (int d = 0; d < D_LATENT; ++d) o[d] += w * (double)os[d];
    }
    for (int d = 0; d < D_LATENT; ++d) o[d] /= wsum;
    out_lse[r] = M + log(wsum);
  }
}

/* ------------------------------------------------------------------------ */
/* KV append: RoPE on the 64-wide key, saturating E4M3, paged write          */
/* ------------------------------------------------------------------------ */
/*
 * The step before the decode path: each new token's latent (512) and RoPE key
 * (64) are written into the paged FP8 cache.  "Muse Spark Open" article
 * (theainews.cc), section "内核优化：解码吞吐 3 倍", bullet "RoPE 与 KV 缓存写入
 * 融合": the rotary embedding is applied in the same kernel that writes the
 * decode KV cache; "SGLang & Miles ... Vera Rubin" article, bullet "原生 FP8
 * 转换": KV is stored as saturating E4M3.  The pages print no RoPE formula;
 * the reading here is the original rotary position embedding: consecutive
 * dims (2i, 2i+1) of the 64-wide key rotated by the angle pos * theta_i with
 * theta_i = base^(-2i/64).
 */

/* The rotation in fp64, straight from the definition (used by the pins). */
void oracle_rope_f64(const double* x, int64_t pos, double base, double* y) {
  for (int i = 0; i < D_ROPE / 2; ++i) {
    const double theta = pow(base, -2.0 * i / (double)D_ROPE);
    const double a = (double)pos * theta;
    const double c = cos(a), s = sin(a);
    y[2 * i] = x[2 * i] * c - x[2 * i + 1] * s;
    y[2 * i + 1] = x[2 * i] * s + x[2 * i + 1] * c;
  }
}

/* cos_sin[pos][i] = (fl32(cos(pos theta_i)), fl32(sin(pos theta_i))) for
 * pos < max_pos, i < 32: the angle and its cosine and sine in fp64, each
 * rounded once to fp32.  This is the cache of angles a serving engine keeps. */
void oracle_rope_table(int64_t max_pos, double base, float* cos_sin) {
  for (int64_t pos = 0; pos < max_pos; ++pos)
    for (int i = 0; i < D_ROPE / 2; ++i) {
      const double theta = pow(base, -2.0 * i / (double)D_ROPE);
      const double a = (double)pos * theta;
      cos_sin[(pos * (D_ROPE / 2) + i) * 2] = (float)cos(a);
      cos_sin[(pos * (D_ROPE / 2) + i) * 2 + 1] = (float)sin(a);
    }
}

/* Append n_new tokens per request.  Token j of request b has position
 * pos = seq_lens[b] - n_new + j (seq_lens counts the new tokens) and goes to
 * row pos % 64 of page block_table[b][pos / 64]:
 *   latent dim d:   code = E4M3(fl32(x_d * inv_scale))
 *   RoPE pair i:    with (c, s) = cos_sin[pos][i] and x0, x1 the pair's bf16
 *                   values, in fp32 (each operation rounded, no fused
 *                   multiply-add):  y0 = x0 c - x1 s,  y1 = x0 s + x1 c;
 *                   codes E4M3(fl32(y * inv_scale)).
 * Returns the number of tokens skipped because their position, page index or
 * page id was out of range (those tokens are not written). */
int64_t oracle_append_kv(const uint16_t* c_kv, const uint16_t* k_rope, const float* cos_sin,
                         int64_t max_pos, const int32_t* block_table, int max_pages,
                         const int32_t* seq_lens, int B, int n_new, float inv_scale,
                         uint8_t* kv_pages, int64_t num_pages) {
  init_tables();
  int64_t skipped = 0;
  for (int b = 0; b < B; ++b)
    for (int j = 0; j < n_new; ++j) {
      const int64_t pos = (int64_t)seq_lens[b] - n_new + j;
      if (pos < 0 || pos >= max_pos || pos / PAGE >= max_pages) { ++skipped; continue; }
      const int64_t page = block_table[(int64_t)b * max_pages + pos / PAGE];
      if (page < 0 || page >= num_pages) { ++skipped; continue; }
      uint8_t* row = kv_pages + (page * PAGE + pos % PAGE) * D_ROW;
      const uint16_t* xc = c_kv + ((int64_t)b * n_new + j) * D_LATENT;
      const uint16_t* xr = k_rope + ((int64_t)b * n_new + j) * D_ROPE;
      for (int d = 0; d < D_LATENT; ++d) {
        volatile float p = bf16_to_f32(xc[d]) * inv_scale;
        row[d] = oracle_e4m3_encode(p);
      }
      for (int i = 0; i < D_ROPE / 2; ++i) {
        const float c = cos_sin[(pos * (D_ROPE / 2) + i) * 2];
        const float s = cos_sin[(pos * (D_ROPE / 2) + i) * 2 + 1];
        const float x0 = bf16_to_f32(xr[2 * i]), x1 = bf16_to_f32(xr[2 * i + 1]);
        volatile float x0c = x0 * c, x1s = x1 * s, x0s = x0 * s, x1c = x1 * c;
        volatile float y0 = x0c - x1s, y1 = x0s + x1c;
        volatile float p0 = y0 * inv_scale, p1 = y1 * inv_scale;
        row[D_LATENT + 2 * i] = oracle_e4m3_encode(p0);
        row[D_LATENT + 2 * i + 1] = oracle_e4m3_encode(p1);
      }
    }
  return skipped;
}

/* Threads OpenMP will use (reported with CPU timings); the setter lets a
 * timing run the same code on one core. */
void oracle_set_num_threads(int n) {
#ifdef _OPENMP
  if (n > 0) omp_set_num_threads(n);
#else
  (void)n;
#endif
}
int oracle_num_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}
