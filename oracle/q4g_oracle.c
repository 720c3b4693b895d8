/*
 * CPU oracle for the batch-1 q4_0 decode step: TEST INFRASTRUCTURE ONLY.
 * See q4g_oracle.h for the contract and the pages each part follows.
 *
 * Build: gcc -O2 -std=c11 -fopenmp -ffp-contract=off -fPIC -shared (no fast-math).
 * OpenMP is used only across independent outputs (rows of a matrix-vector
 * product, heads of attention, elements of a fill); each output is computed in
 * the natural order written below, so results do not depend on thread count.
 */
#include "q4g_oracle.h"

#include <math.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

#include "../datagen/q4g_datagen.h"

/* ------------------------------------------------------------------------- */
/* IEEE binary16: 1 sign bit, 5 exponent bits (bias 15), 10 fraction bits.    */
/* ------------------------------------------------------------------------- */

uint16_t or_f16_from_double(double x) {
  if (isnan(x)) return 0x7E00;
  uint16_t sign = signbit(x) ? 0x8000 : 0;
  double a = fabs(x);
  /* Largest finite half is 65504; the midpoint to the next step (65536) is 65520,
   * and a tie there goes to the even neighbour, which is infinity. */
  if (a >= 65520.0) return sign | 0x7C00;
  if (a < ldexp(1.0, -14)) {
    /* subnormal: integer count of 2^-24 units, nearest-even (rint in the default mode).
     * 1024 units is 2^-14, whose encoding 0x0400 is the smallest normal: consistent. */
    double units = rint(ldexp(a, 24));
    return sign | (uint16_t)units;
  }
  int e2;
  (void)frexp(a, &e2); /* a in [2^(e2-1), 2^e2) */
  int E = e2 - 1;
  double m = rint(ldexp(a, 10 - E)); /* significand in [1024, 2048] */
  if (m >= 2048.0) {
    m = 1024.0;
    E += 1;
  }
  if (E > 15) return sign | 0x7C00;
  return sign | (uint16_t)((E + 15) << 10) | (uint16_t)(m - 1024.0);
}

double or_f16_to_double(uint16_t h) {
  int s = h >> 15, e = (h >> 10) & 0x1F, f = h & 0x3FF;
  double v;
  if (e == 0)
    v = ldexp((double)f, -24);
  else if (e == 31)
    v = f ? NAN : INFINITY;
  else
    v = ldexp((double)(f + 1024), e - 25);
  return s ? -v : v;
}

/* ------------------------------------------------------------------------- */
/* q4_0 ([zoo] intro: per-block-32 absmax symmetric int4; [e4b] Provenance:    */
/* the ggml q4_0 grid, i.e. codes on [-8, 7]). Reading of the open points:     */
/*   m  = the element of largest |x| in the block (first one on ties), signed  */
/*   d  = fp16(m / -8)            fp32 division, rounded to binary16           */
/*   q  = clamp(round_half_away(x / d), -8, 7)   fp32 division                 */
/*   stored code c = q + 8; an all-zero scale stores every code as 8           */
/*   dequant: (c - 8) * d                                                      */
/* ------------------------------------------------------------------------- */

static int block_is_finite(const float* x) {
  for (int i = 0; i < 32; ++i)
    if (!isfinite(x[i])) return 0;
  return 1;
}

static void pack_block(const float* x, uint8_t* qs16, uint16_t* scale) {
  float amax = 0.0f, m = 0.0f;
  for (int i = 0; i < 32; ++i) {
    float a = fabsf(x[i]);
    if (a > amax) {
      amax = a;
      m = x[i];
    }
  }
  volatile float dm = m / -8.0f;
  uint16_t dh = or_f16_from_double((double)dm);
  float d = (float)or_f16_to_double(dh);
  uint8_t c[32];
  for (int i = 0; i < 32; ++i) {
    if (d == 0.0f) {
      c[i] = 8;
      continue;
    }
    volatile float v = x[i] / d;
    float r = roundf(v); /* C roundf: halfway cases away from zero */
    if (r < -8.0f) r = -8.0f;
    if (r > 7.0f) r = 7.0f;
    c[i] = (uint8_t)((int)r + 8);
  }
  for (int b = 0; b < 16; ++b) qs16[b] = (uint8_t)(c[b] | (c[b + 16] << 4));
  *scale = dh;
}

int or_q4_0_pack(const float* w, int64_t rows, int64_t k, uint8_t* qs, uint16_t* scales) {
  if (rows < 0 || k <= 0 || k % 32 != 0) return -1;
  int64_t nb = k / 32;
  int bad = 0;
#pragma omp parallel for schedule(static) reduction(| : bad)
  for (int64_t r = 0; r < rows; ++r)
    for (int64_t t = 0; t < nb; ++t)
      if (!block_is_finite(w + r * k + 32 * t)) bad |= 1;
  if (bad) return -1;
#pragma omp parallel for schedule(static)
  for (int64_t r = 0; r < rows; ++r)
    for (int64_t t = 0; t < nb; ++t)
      pack_block(w + r * k + 32 * t, qs + r * (k / 2) + 16 * t, scales + r * nb + t);
  return 0;
}

static inline int code_at(const uint8_t* qs_row, int64_t col) {
  uint8_t byte = qs_row[16 * (col / 32) + (col % 16)];
  return (col % 32) < 16 ? (byte & 0x0F) : (byte >> 4);
}

void or_q4_0_unpack(const uint8_t* qs, const uint16_t* scales, int64_t rows, int64_t k, double* w) {
  int64_t nb = k / 32;
#pragma omp parallel for schedule(static)
  for (int64_t r = 0; r < rows; ++r)
    for (int64_t col = 0; col < k; ++col)
      w[r * k + col] = (double)(code_at(qs + r * (k / 2), col) - 8) *
                       or_f16_to_double(scales[r * nb + col / 32]);
}

/* ------------------------------------------------------------------------- */
/* Matrix-vector product on the dequantised weights, natural column order.    */
/* ------------------------------------------------------------------------- */

void or_gemv(const uint8_t* qs, const uint16_t* scales, int64_t n, int64_t k, int nrhs,
             const uint16_t* x16, double* y) {
  int64_t nb = k / 32;
  double* xd = (double*)malloc(sizeof(double) * (size_t)(k * nrhs));
  for (int64_t i = 0; i < k * nrhs; ++i) xd[i] = or_f16_to_double(x16[i]);
#pragma omp parallel for schedule(static)
  for (int64_t r = 0; r < n; ++r) {
    const uint8_t* row = qs + r * (k / 2);
    for (int j = 0; j < nrhs; ++j) {
      const double* x = xd + (int64_t)j * k;
      double acc = 0.0;
      for (int64_t col = 0; col < k; ++col) {
        double wv = (double)(code_at(row, col) - 8) * or_f16_to_double(scales[r * nb + col / 32]);
        acc += wv * x[col];
      }
      y[(int64_t)j * n + r] = acc;
    }
  }
  free(xd);
}

/* y[n] = sum_k W[n][k] * x[k] for fp16 weights W (the fp16 tied head of
 * [12b] "tiered-v3/": the bf16 -> fp16 cast of the table is exact, so the head
 * reads the table's own values); x as fp16 bits; natural k order. */
void or_gemv_f16(const uint16_t* w, int64_t n, int64_t k, int nrhs, const uint16_t* x16, double* y) {
  double* xd = (double*)malloc(sizeof(double) * (size_t)(k * nrhs));
  for (int64_t i = 0; i < k * nrhs; ++i) xd[i] = or_f16_to_double(x16[i]);
#pragma omp parallel for schedule(static)
  for (int64_t r = 0; r < n; ++r) {
    const uint16_t* row = w + r * k;
    for (int j = 0; j < nrhs; ++j) {
      const double* x = xd + (int64_t)j * k;
      double acc = 0.0;
      for (int64_t col = 0; col < k; ++col) acc += or_f16_to_double(row[col]) * x[col];
      y[(int64_t)j * n + r] = acc;
    }
  }
  free(xd);
}

/* ------------------------------------------------------------------------- */
/* Elementwise pieces.                                                        */
/* ------------------------------------------------------------------------- */

/* RMSNorm: y = x / sqrt(mean(x^2) + eps) * w ; w == NULL is the scale-free norm
 * ([zoo] architecture: the value path of full layers uses a scale-free RMSNorm). */
void or_rmsnorm(const double* x, const double* w, int64_t n, double eps, double* y) {
  double ss = 0.0;
  for (int64_t i = 0; i < n; ++i) ss += x[i] * x[i];
  double inv = 1.0 / sqrt(ss / (double)n + eps);
  for (int64_t i = 0; i < n; ++i) y[i] = x[i] * inv * (w ? w[i] : 1.0);
}

/* RoPE, rotate-half pairing (i, i + hd/2). Pair i turns by pos * theta^(-2i/hd)
 * for i < rot_pairs and is left alone otherwise ([zoo] architecture: sliding
 * layers theta 1e4 with every pair rotating; full layers theta 1e6 with the
 * first 64 of 256 pairs rotating and the rest position-free). Angle in double. */
void or_rope(double* x, int64_t hd, int64_t rot_pairs, double theta, int64_t pos) {
  int64_t half = hd / 2;
  for (int64_t i = 0; i < rot_pairs && i < half; ++i) {
    double inv_freq = pow(theta, -2.0 * (double)i / (double)hd);
    double ang = (double)pos * inv_freq;
    double c = cos(ang), s = sin(ang);
    double a = x[i], b = x[i + half];
    x[i] = a * c - b * s;
    x[i + half] = b * c + a * s;
  }
}

double or_gelu_tanh(double g) {
  const double k0 = sqrt(2.0 / 3.14159265358979323846);
  return 0.5 * g * (1.0 + tanh(k0 * (g + 0.044715 * g * g * g)));
}

double or_softcap(double z, double cap) { return cap * tanh(z / cap); }

static inline int64_t pmod(int64_t a, int64_t m) {
  int64_t r = a % m;
  return r < 0 ? r + m : r;
}

/* ------------------------------------------------------------------------- */
/* Attention: scale 1.0, softmax over the live keys ([zoo] flash-decode        */
/* description), keys taken in ascending position.                           */
/* ------------------------------------------------------------------------- */

/* A cache row: fp16 values (h), or int8 codes c with the row's scale s, whose
 * value is c[d] * s ("Gemma-4-12B-CoreAI", per-tier cost section: int8 KV). */
typedef struct {
  const uint16_t* h;
  const int8_t* c;
  float s;
} kvrow;

static inline double kv_at(const kvrow* r, int d) {
  return r->h ? or_f16_to_double(r->h[d]) : (double)r->c[d] * (double)r->s;
}

/* One head: n keys given as rows, in the order they are summed. */
static void attend_one(const double* q, int hd, const kvrow* keys, const kvrow* vals, int64_t n,
                       double* out) {
  double* s = (double*)malloc(sizeof(double) * (size_t)(n > 0 ? n : 1));
  double mx = -INFINITY;
  for (int64_t t = 0; t < n; ++t) {
    double acc = 0.0;
    for (int d = 0; d < hd; ++d) acc += q[d] * kv_at(&keys[t], d);
    s[t] = acc;
    if (acc > mx) mx = acc;
  }
  double l = 0.0;
  for (int64_t t = 0; t < n; ++t) {
    s[t] = exp(s[t] - mx);
    l += s[t];
  }
  for (int d = 0; d < hd; ++d) out[d] = 0.0;
  for (int64_t t = 0; t < n; ++t)
    for (int d = 0; d < hd; ++d) out[d] += s[t] * kv_at(&vals[t], d);
  for (int d = 0; d < hd; ++d) out[d] /= l;
  free(s);
}

/* int8 KV row: s = amax / 127 (fp32 division; amax = largest |x| of the fp16
 * row), code = clamp(rint(x / s), -127, 127) with x / s an fp32 division and
 * rint to nearest even; an all-zero row has s = 0 and codes 0. */
void or_kv_quantize_row(const uint16_t* x16, int hd, int8_t* codes, float* scale) {
  float amax = 0.0f;
  for (int d = 0; d < hd; ++d) {
    const float v = fabsf((float)or_f16_to_double(x16[d]));
    if (v > amax) amax = v;
  }
  const float s = amax / 127.0f;
  *scale = s;
  for (int d = 0; d < hd; ++d) {
    if (s == 0.0f) {
      codes[d] = 0;
      continue;
    }
    float q = rintf((float)or_f16_to_double(x16[d]) / s);
    if (q > 127.0f) q = 127.0f;
    if (q < -127.0f) q = -127.0f;
    codes[d] = (int8_t)q;
  }
}

void or_ring_implied_positions(int64_t R, int64_t W, int64_t q, int64_t* out) {
  for (int64_t j = 0; j < R; ++j) {
    int64_t p = q - pmod(q - j, R); /* [12b] v5 section: implied position */
    out[j] = (p >= 0 && q - p < W) ? p : -1;
  }
}

static void attn_ring_any(const uint16_t* q16, int n_q, int n_kv, int hd, const uint16_t* kc,
                          const uint16_t* vc, const int8_t* k8, const float* ks, const int8_t* v8,
                          const float* vs, int64_t R, int64_t W, int64_t q, double* out) {
  int G = n_q / n_kv;
#pragma omp parallel for schedule(static)
  for (int h = 0; h < n_q; ++h) {
    int g = h / G;
    kvrow* keys = (kvrow*)calloc((size_t)R, sizeof(kvrow));
    kvrow* vals = (kvrow*)calloc((size_t)R, sizeof(kvrow));
    double* qd = (double*)malloc(sizeof(double) * (size_t)hd);
    for (int d = 0; d < hd; ++d) qd[d] = or_f16_to_double(q16[(int64_t)h * hd + d]);
    int64_t n = 0;
    for (int64_t a = R - 1; a >= 0; --a) { /* slots in ascending implied position */
      int64_t j = pmod(q - a, R);
      int64_t p = q - pmod(q - j, R);
      if (p < 0 || q - p >= W) continue;
      const int64_t row = (int64_t)g * R + j;
      if (kc) {
        keys[n].h = kc + row * hd, vals[n].h = vc + row * hd;
      } else {
        keys[n].c = k8 + row * hd, keys[n].s = ks[row];
        vals[n].c = v8 + row * hd, vals[n].s = vs[row];
      }
      ++n;
    }
    attend_one(qd, hd, keys, vals, n, out + (int64_t)h * hd);
    free(keys);
    free(vals);
    free(qd);
  }
}

static void attn_linear_any(const uint16_t* q16, int n_q, int n_kv, int hd, const uint16_t* kc,
                            const uint16_t* vc, const int8_t* k8, const float* ks, const int8_t* v8,
                            const float* vs, int64_t len, double* out) {
  int G = n_q / n_kv;
#pragma omp parallel for schedule(static)
  for (int h = 0; h < n_q; ++h) {
    int g = h / G;
    kvrow* keys = (kvrow*)calloc((size_t)(len > 0 ? len : 1), sizeof(kvrow));
    kvrow* vals = (kvrow*)calloc((size_t)(len > 0 ? len : 1), sizeof(kvrow));
    double* qd = (double*)malloc(sizeof(double) * (size_t)hd);
    for (int d = 0; d < hd; ++d) qd[d] = or_f16_to_double(q16[(int64_t)h * hd + d]);
    for (int64_t p = 0; p < len; ++p) {
      const int64_t row = p * n_kv + g;
      if (kc) {
        keys[p].h = kc + row * hd, vals[p].h = vc + row * hd;
      } else {
        keys[p].c = k8 + row * hd, keys[p].s = ks[row];
        vals[p].c = v8 + row * hd, vals[p].s = vs[row];
      }
    }
    attend_one(qd, hd, keys, vals, len, out + (int64_t)h * hd);
    free(keys);
    free(vals);
    free(qd);
  }
}

void or_attn_ring(const uint16_t* q16, int n_q, int n_kv, int hd, const uint16_t* kc,
                  const uint16_t* vc, int64_t R, int64_t W, int64_t q, double* out) {
  attn_ring_any(q16, n_q, n_kv, hd, kc, vc, NULL, NULL, NULL, NULL, R, W, q, out);
}
void or_attn_ring_i8(const uint16_t* q16, int n_q, int n_kv, int hd, const int8_t* k8, const float* ks,
                     const int8_t* v8, const float* vs, int64_t R, int64_t W, int64_t q, double* out) {
  attn_ring_any(q16, n_q, n_kv, hd, NULL, NULL, k8, ks, v8, vs, R, W, q, out);
}
void or_attn_linear(const uint16_t* q16, int n_q, int n_kv, int hd, const uint16_t* kc,
                    const uint16_t* vc, int64_t len, double* out) {
  attn_linear_any(q16, n_q, n_kv, hd, kc, vc, NULL, NULL, NULL, NULL, len, out);
}
void or_attn_linear_i8(const uint16_t* q16, int n_q, int n_kv, int hd, const int8_t* k8, const float* ks,
                       const int8_t* v8, const float* vs, int64_t len, double* out) {
  attn_linear_any(q16, n_q, n_kv, hd, NULL, NULL, k8, ks, v8, vs, len, out);
}

/* ------------------------------------------------------------------------- */
/* Model.                                                                     */
/* ------------------------------------------------------------------------- */

typedef struct {
  uint8_t* qs;
  uint16_t* sc;
  int64_t rows, cols;
} qmat;

typedef struct {
  int is_full, ordinal;
  qmat wq, wk, wv, wo, wg, wu, wd;
  double *n_in, *n_pa, *n_pf, *n_po, *n_q, *n_k;
  double lscalar;
} layer_t;

struct or_model {
  or_config cfg;
  layer_t* L;
  qmat embed;        /* q4_0 tied table (head_fp16 = 0) */
  uint16_t* embed16; /* fp16 tied table [vocab][h] (head_fp16 = 1) */
  double* n_final;
  int n_sl, n_gl;
};

struct or_cache {
  int64_t capacity, R;
  int n_sl, n_gl, sl_kv, gl_kv, hd_s, hd_g;
  int kv8;                              /* int8 rows with one fp32 scale each */
  uint16_t **ringK, **ringV, **glK, **glV;  /* fp16 rows (kv8 = 0) */
  int8_t **ringK8, **ringV8, **glK8, **glV8;  /* int8 codes (kv8 = 1) */
  float **ringKs, **ringVs, **glKs, **glVs;   /* per-row scales (kv8 = 1) */
};

static int layer_is_full(const or_config* c, int l) {
  return c->full_every > 0 && (l % c->full_every) == c->full_offset;
}

static int make_qmat(qmat* m, uint64_t seed, uint64_t stream, int64_t rows, int64_t cols) {
  m->rows = rows;
  m->cols = cols;
  m->qs = (uint8_t*)malloc((size_t)(rows * cols / 2));
  m->sc = (uint16_t*)malloc(sizeof(uint16_t) * (size_t)(rows * cols / 32));
  if (!m->qs || !m->sc) return -1;
  uint64_t key = dg_key(seed, stream);
  const int64_t chunk = 256;
  float* tmp = (float*)malloc(sizeof(float) * (size_t)(chunk * cols));
  for (int64_t r0 = 0; r0 < rows; r0 += chunk) {
    int64_t nr = rows - r0 < chunk ? rows - r0 : chunk;
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < nr * cols; ++i) tmp[i] = dg_normal(key, (uint64_t)(r0 * cols + i), 0.02f);
    if (or_q4_0_pack(tmp, nr, cols, m->qs + r0 * cols / 2, m->sc + r0 * cols / 32) != 0) {
      free(tmp);
      return -1;
    }
  }
  free(tmp);
  return 0;
}

static double* make_gain(uint64_t seed, uint64_t stream, int64_t n, int variant) {
  double* g = (double*)malloc(sizeof(double) * (size_t)n);
  uint64_t key = dg_key(seed, stream);
  for (int64_t i = 0; i < n; ++i) g[i] = variant == 1 ? (double)dg_gain(key, (uint64_t)i) : 1.0;
  return g;
}

static double* make_qk_gain(uint64_t seed, uint64_t stream, int64_t hd, int variant) {
  double* g = (double*)malloc(sizeof(double) * (size_t)hd);
  uint64_t key = dg_key(seed, stream);
  for (int64_t i = 0; i < hd; ++i) g[i] = (double)dg_qk_gain(key, (uint64_t)i, (int)hd, variant);
  return g;
}

or_model* or_model_create(const or_config* cfg, uint64_t seed, int variant, int nthreads) {
#ifdef _OPENMP
  if (nthreads > 0) omp_set_num_threads(nthreads);
#else
  (void)nthreads;
#endif
  or_model* m = (or_model*)calloc(1, sizeof(or_model));
  m->cfg = *cfg;
  int H = cfg->hidden, Hq = cfg->n_q_heads;
  m->L = (layer_t*)calloc((size_t)cfg->n_layers, sizeof(layer_t));
  for (int l = 0; l < cfg->n_layers; ++l) {
    layer_t* L = &m->L[l];
    L->is_full = layer_is_full(cfg, l);
    L->ordinal = L->is_full ? m->n_gl++ : m->n_sl++;
    int hd = L->is_full ? cfg->gl_head_dim : cfg->sl_head_dim;
    int nkv = L->is_full ? cfg->gl_kv_heads : cfg->sl_kv_heads;
    int rc = 0;
    rc |= make_qmat(&L->wq, seed, DG_STREAM_LAYER(l, DG_T_WQ), (int64_t)Hq * hd, H);
    rc |= make_qmat(&L->wk, seed, DG_STREAM_LAYER(l, DG_T_WK), (int64_t)nkv * hd, H);
    if (!L->is_full) rc |= make_qmat(&L->wv, seed, DG_STREAM_LAYER(l, DG_T_WV), (int64_t)nkv * hd, H);
    rc |= make_qmat(&L->wo, seed, DG_STREAM_LAYER(l, DG_T_WO), H, (int64_t)Hq * hd);
    rc |= make_qmat(&L->wg, seed, DG_STREAM_LAYER(l, DG_T_WGATE), cfg->ffn, H);
    rc |= make_qmat(&L->wu, seed, DG_STREAM_LAYER(l, DG_T_WUP), cfg->ffn, H);
    rc |= make_qmat(&L->wd, seed, DG_STREAM_LAYER(l, DG_T_WDOWN), H, cfg->ffn);
    if (rc) {
      or_model_destroy(m);
      return NULL;
    }
    L->n_in = make_gain(seed, DG_STREAM_LAYER(l, DG_T_NORM_IN), H, variant);
    L->n_pa = make_gain(seed, DG_STREAM_LAYER(l, DG_T_NORM_POST_ATTN), H, variant);
    L->n_pf = make_gain(seed, DG_STREAM_LAYER(l, DG_T_NORM_PRE_FFN), H, variant);
    L->n_po = make_gain(seed, DG_STREAM_LAYER(l, DG_T_NORM_POST_FFN), H, variant);
    L->n_q = make_qk_gain(seed, DG_STREAM_LAYER(l, DG_T_NORM_Q), hd, variant);
    L->n_k = make_qk_gain(seed, DG_STREAM_LAYER(l, DG_T_NORM_K), hd, variant);
    L->lscalar = variant == 1 ? (double)dg_uniform_float(dg_key(seed, DG_STREAM_LAYER(l, DG_T_LAYER_SCALAR)),
                                                    0, 0.5f, 1.5f)
                         : 1.0;
  }
  if (cfg->head_fp16) {
    /* the same N(0, 0.02) draws as the q4_0 table, kept at fp16 */
    m->embed16 = (uint16_t*)malloc(sizeof(uint16_t) * (size_t)cfg->vocab * (size_t)H);
    if (!m->embed16) {
      or_model_destroy(m);
      return NULL;
    }
    uint64_t key = dg_key(seed, DG_STREAM_EMBED);
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < (int64_t)cfg->vocab * H; ++i)
      m->embed16[i] = or_f16_from_double((double)dg_normal(key, (uint64_t)i, 0.02f));
  } else if (make_qmat(&m->embed, seed, DG_STREAM_EMBED, cfg->vocab, H)) {
    or_model_destroy(m);
    return NULL;
  }
  m->n_final = make_gain(seed, DG_STREAM_FINAL_NORM, H, variant);
  return m;
}

static void free_qmat(qmat* q) {
  free(q->qs);
  free(q->sc);
}

void or_model_destroy(or_model* m) {
  if (!m) return;
  for (int l = 0; m->L && l < m->cfg.n_layers; ++l) {
    layer_t* L = &m->L[l];
    free_qmat(&L->wq), free_qmat(&L->wk), free_qmat(&L->wv), free_qmat(&L->wo);
    free_qmat(&L->wg), free_qmat(&L->wu), free_qmat(&L->wd);
    free(L->n_in), free(L->n_pa), free(L->n_pf), free(L->n_po), free(L->n_q), free(L->n_k);
  }
  free(m->L);
  free_qmat(&m->embed);
  free(m->embed16);
  free(m->n_final);
  free(m);
}

int64_t or_model_tensor(const or_model* m, int layer, int tensor, const uint8_t** qs,
                        const uint16_t** scales, int64_t* cols) {
  const qmat* q = NULL;
  if (tensor == 100)
    q = &m->embed;
  else if (layer >= 0 && layer < m->cfg.n_layers) {
    const layer_t* L = &m->L[layer];
    const qmat* all[7] = {&L->wq, &L->wk, &L->wv, &L->wo, &L->wg, &L->wu, &L->wd};
    if (tensor >= 0 && tensor < 7) q = all[tensor];
  }
  if (!q || !q->qs) return 0;
  *qs = q->qs;
  *scales = q->sc;
  *cols = q->cols;
  return q->rows;
}

const uint16_t* or_model_embed_f16(const or_model* m) { return m->embed16; }

/* Allocate every layer's rows, zeroed, or as a copy of src's (copy != 0). */
static void* alloc_copy(size_t bytes, const void* from) {
  void* p = calloc(bytes ? bytes : 1, 1);
  if (from) memcpy(p, from, bytes);
  return p;
}
static void cache_alloc(or_cache* k, int copy, const or_cache* src) {
  const size_t nsl = (size_t)k->n_sl + 1, ngl = (size_t)k->n_gl + 1;
  const size_t rrows = (size_t)k->sl_kv * (size_t)k->R, grows = (size_t)k->gl_kv * (size_t)k->capacity;
  const size_t rvals = rrows * (size_t)k->hd_s, gvals = grows * (size_t)k->hd_g;
  k->ringK = (uint16_t**)calloc(nsl, sizeof(void*)), k->ringV = (uint16_t**)calloc(nsl, sizeof(void*));
  k->glK = (uint16_t**)calloc(ngl, sizeof(void*)), k->glV = (uint16_t**)calloc(ngl, sizeof(void*));
  k->ringK8 = (int8_t**)calloc(nsl, sizeof(void*)), k->ringV8 = (int8_t**)calloc(nsl, sizeof(void*));
  k->glK8 = (int8_t**)calloc(ngl, sizeof(void*)), k->glV8 = (int8_t**)calloc(ngl, sizeof(void*));
  k->ringKs = (float**)calloc(nsl, sizeof(void*)), k->ringVs = (float**)calloc(nsl, sizeof(void*));
  k->glKs = (float**)calloc(ngl, sizeof(void*)), k->glVs = (float**)calloc(ngl, sizeof(void*));
  for (int i = 0; i < k->n_sl; ++i) {
    if (!k->kv8) {
      k->ringK[i] = (uint16_t*)alloc_copy(rvals * 2, copy ? src->ringK[i] : NULL);
      k->ringV[i] = (uint16_t*)alloc_copy(rvals * 2, copy ? src->ringV[i] : NULL);
    } else {
      k->ringK8[i] = (int8_t*)alloc_copy(rvals, copy ? src->ringK8[i] : NULL);
      k->ringV8[i] = (int8_t*)alloc_copy(rvals, copy ? src->ringV8[i] : NULL);
      k->ringKs[i] = (float*)alloc_copy(rrows * sizeof(float), copy ? src->ringKs[i] : NULL);
      k->ringVs[i] = (float*)alloc_copy(rrows * sizeof(float), copy ? src->ringVs[i] : NULL);
    }
  }
  for (int i = 0; i < k->n_gl; ++i) {
    if (!k->kv8) {
      k->glK[i] = (uint16_t*)alloc_copy(gvals * 2, copy ? src->glK[i] : NULL);
      k->glV[i] = (uint16_t*)alloc_copy(gvals * 2, copy ? src->glV[i] : NULL);
    } else {
      k->glK8[i] = (int8_t*)alloc_copy(gvals, copy ? src->glK8[i] : NULL);
      k->glV8[i] = (int8_t*)alloc_copy(gvals, copy ? src->glV8[i] : NULL);
      k->glKs[i] = (float*)alloc_copy(grows * sizeof(float), copy ? src->glKs[i] : NULL);
      k->glVs[i] = (float*)alloc_copy(grows * sizeof(float), copy ? src->glVs[i] : NULL);
    }
  }
}

or_cache* or_cache_create(const or_model* m, int64_t capacity, int64_t ring_slots) {
  const or_config* c = &m->cfg;
  or_cache* k = (or_cache*)calloc(1, sizeof(or_cache));
  k->capacity = capacity;
  k->R = ring_slots > 0 ? ring_slots : c->ring;
  k->n_sl = m->n_sl;
  k->n_gl = m->n_gl;
  k->sl_kv = c->sl_kv_heads;
  k->gl_kv = c->gl_kv_heads;
  k->hd_s = c->sl_head_dim;
  k->hd_g = c->gl_head_dim;
  k->kv8 = c->kv_int8 != 0;
  cache_alloc(k, 0, NULL);
  return k;
}

void or_cache_destroy(or_cache* c) {
  if (!c) return;
  for (int i = 0; i < c->n_sl; ++i) {
    free(c->ringK[i]), free(c->ringV[i]), free(c->ringK8[i]), free(c->ringV8[i]);
    free(c->ringKs[i]), free(c->ringVs[i]);
  }
  for (int i = 0; i < c->n_gl; ++i) {
    free(c->glK[i]), free(c->glV[i]), free(c->glK8[i]), free(c->glV8[i]);
    free(c->glKs[i]), free(c->glVs[i]);
  }
  free(c->ringK), free(c->ringV), free(c->glK), free(c->glV);
  free(c->ringK8), free(c->ringV8), free(c->glK8), free(c->glV8);
  free(c->ringKs), free(c->ringVs), free(c->glKs), free(c->glVs);
  free(c);
}

or_cache* or_cache_clone(const or_cache* c) {
  or_cache* k = (or_cache*)malloc(sizeof(or_cache));
  *k = *c;
  cache_alloc(k, 1, c);
  return k;
}

uint16_t* or_cache_ring(or_cache* c, int sl_index, int kv) {
  if (c->kv8 || sl_index < 0 || sl_index >= c->n_sl) return NULL;
  return kv ? c->ringV[sl_index] : c->ringK[sl_index];
}

uint16_t* or_cache_global(or_cache* c, int gl_index, int kv) {
  if (c->kv8 || gl_index < 0 || gl_index >= c->n_gl) return NULL;
  return kv ? c->glV[gl_index] : c->glK[gl_index];
}

int8_t* or_cache_ring_i8(or_cache* c, int sl_index, int kv, float** scales) {
  if (!c->kv8 || sl_index < 0 || sl_index >= c->n_sl) return NULL;
  *scales = kv ? c->ringVs[sl_index] : c->ringKs[sl_index];
  return kv ? c->ringV8[sl_index] : c->ringK8[sl_index];
}

int8_t* or_cache_global_i8(or_cache* c, int gl_index, int kv, float** scales) {
  if (!c->kv8 || gl_index < 0 || gl_index >= c->n_gl) return NULL;
  *scales = kv ? c->glVs[gl_index] : c->glKs[gl_index];
  return kv ? c->glV8[gl_index] : c->glK8[gl_index];
}

/* ------------------------------------------------------------------------- */
/* One verify block (decode = one row).                                       */
/* ------------------------------------------------------------------------- */

static void to_f16(const double* x, int64_t n, uint16_t* y) {
  for (int64_t i = 0; i < n; ++i) y[i] = or_f16_from_double(x[i]);
}

int or_verify_block(or_model* m, or_cache* c, const int32_t* ids, const float* hidden_in, int K,
                    int64_t pos0, int accepted, int mode, double* logits, int32_t* argmax,
                    double* dump, uint16_t* kv_dump, double* vraw_dump) {
  const or_config* cfg = &m->cfg;
  const int64_t H = cfg->hidden, Hq = cfg->n_q_heads, F = cfg->ffn, V = cfg->vocab;
  const int64_t W = cfg->window, R = c->R;
  if (K < 1 || pos0 < 0 || pos0 + K > c->capacity || accepted < 0 || accepted > K) return -1;
  if (!ids && !hidden_in) return -1;
  for (int i = 0; ids && i < K; ++i)
    if (ids[i] < 0 || ids[i] >= V) return -1;
  const int64_t hdmax = cfg->gl_head_dim > cfg->sl_head_dim ? cfg->gl_head_dim : cfg->sl_head_dim;
  const int64_t kvmax = cfg->gl_kv_heads > cfg->sl_kv_heads ? cfg->gl_kv_heads : cfg->sl_kv_heads;

  double* r = (double*)calloc((size_t)(K * H), sizeof(double));
  double* tmp = (double*)malloc(sizeof(double) * (size_t)(K * (H > F ? H : F)));
  uint16_t* x16 = (uint16_t*)malloc(2 * (size_t)(K * (F > Hq * hdmax ? F : Hq * hdmax)));
  double* qp = (double*)malloc(sizeof(double) * (size_t)(K * Hq * hdmax));
  double* kp = (double*)malloc(sizeof(double) * (size_t)(K * kvmax * hdmax));
  double* vp = (double*)malloc(sizeof(double) * (size_t)(K * kvmax * hdmax));
  uint16_t* q16 = (uint16_t*)malloc(2 * (size_t)(K * Hq * hdmax));
  uint16_t* k16 = (uint16_t*)malloc(2 * (size_t)(K * kvmax * hdmax));
  uint16_t* v16 = (uint16_t*)malloc(2 * (size_t)(K * kvmax * hdmax));
  double* att = (double*)malloc(sizeof(double) * (size_t)(K * Hq * hdmax));
  double* gg = (double*)malloc(sizeof(double) * (size_t)(K * F));
  double* uu = (double*)malloc(sizeof(double) * (size_t)(K * F));
  double* hv = (double*)malloc(sizeof(double) * (size_t)hdmax);
  /* int8 KV: this block's rows as stored (codes and one scale per row) */
  int8_t* k8 = (int8_t*)malloc((size_t)(K * kvmax * hdmax));
  int8_t* v8 = (int8_t*)malloc((size_t)(K * kvmax * hdmax));
  float* k8s = (float*)malloc(sizeof(float) * (size_t)(K * kvmax));
  float* v8s = (float*)malloc(sizeof(float) * (size_t)(K * kvmax));

  /* a1: embedding (tied table, dequantised, times the embedding scale) */
  for (int i = 0; i < K; ++i) {
    if (ids) {
      int64_t tok = ids[i];
      if (cfg->head_fp16) {
        for (int64_t col = 0; col < H; ++col)
          r[i * H + col] = or_f16_to_double(m->embed16[tok * H + col]) * cfg->embed_scale;
      } else {
        const uint8_t* row = m->embed.qs + tok * (H / 2);
        for (int64_t col = 0; col < H; ++col)
          r[i * H + col] = (double)(code_at(row, col) - 8) *
                           or_f16_to_double(m->embed.sc[tok * (H / 32) + col / 32]) * cfg->embed_scale;
      }
    } else {
      for (int64_t col = 0; col < H; ++col) r[i * H + col] = (double)hidden_in[i * H + col];
    }
    if (dump) memcpy(dump + ((int64_t)i * (cfg->n_layers + 1)) * H, r + i * H, sizeof(double) * (size_t)H);
  }

  for (int l = 0; l < cfg->n_layers; ++l) {
    layer_t* L = &m->L[l];
    const int full = L->is_full;
    const int64_t hd = full ? cfg->gl_head_dim : cfg->sl_head_dim;
    const int64_t nkv = full ? cfg->gl_kv_heads : cfg->sl_kv_heads;
    const int64_t G = Hq / nkv;
    const int64_t rot = full ? cfg->rope_pairs_full : hd / 2;
    const double theta = full ? cfg->rope_theta_gl : cfg->rope_theta_sl;
    uint16_t* cK = full ? c->glK[L->ordinal] : c->ringK[L->ordinal];
    uint16_t* cV = full ? c->glV[L->ordinal] : c->ringV[L->ordinal];
    int8_t* cK8 = full ? c->glK8[L->ordinal] : c->ringK8[L->ordinal];
    int8_t* cV8 = full ? c->glV8[L->ordinal] : c->ringV8[L->ordinal];
    float* cKs = full ? c->glKs[L->ordinal] : c->ringKs[L->ordinal];
    float* cVs = full ? c->glVs[L->ordinal] : c->ringVs[L->ordinal];
    const int64_t crows = full ? c->capacity : R; /* rows per KV head in this layer's cache */

    /* a2: pre-attention RMSNorm, stored fp16 */
    for (int i = 0; i < K; ++i) {
      or_rmsnorm(r + i * H, L->n_in, H, cfg->rms_eps, tmp);
      to_f16(tmp, H, x16 + i * H);
    }
    /* a3: projections (full layers have no v_proj) */
    or_gemv(L->wq.qs, L->wq.sc, Hq * hd, H, K, x16, qp);
    or_gemv(L->wk.qs, L->wk.sc, nkv * hd, H, K, x16, kp);
    if (!full) or_gemv(L->wv.qs, L->wv.sc, nkv * hd, H, K, x16, vp);
    /* a4: per-head norms, RoPE, fp16 */
    for (int i = 0; i < K; ++i) {
      int64_t pos = pos0 + i;
      for (int64_t h = 0; h < Hq; ++h) {
        or_rmsnorm(qp + (i * Hq + h) * hd, L->n_q, hd, cfg->rms_eps, hv);
        or_rope(hv, hd, rot, theta, pos);
        to_f16(hv, hd, q16 + (i * Hq + h) * hd);
      }
      for (int64_t g = 0; g < nkv; ++g) {
        const double* kraw = kp + (i * nkv + g) * hd;
        or_rmsnorm(kraw, L->n_k, hd, cfg->rms_eps, hv);
        or_rope(hv, hd, rot, theta, pos);
        to_f16(hv, hd, k16 + (i * nkv + g) * hd);
        /* attention_k_eq_v: on full layers V is the raw k_proj output */
        const double* vsrc = full ? kraw : vp + (i * nkv + g) * hd;
        if (full || cfg->v_norm_sliding)
          or_rmsnorm(vsrc, NULL, hd, cfg->rms_eps, hv);
        else
          memcpy(hv, vsrc, sizeof(double) * (size_t)hd);
        to_f16(hv, hd, v16 + (i * nkv + g) * hd);
        if (g == 0 && vraw_dump)
          memcpy(vraw_dump + ((int64_t)l * K + i) * hdmax, kraw, sizeof(double) * (size_t)hd);
      }
      if (kv_dump) {
        uint16_t* dst = kv_dump + (((int64_t)l * K + i) * 2) * hdmax;
        memcpy(dst, k16 + (i * nkv) * hd, 2 * (size_t)hd);
        memcpy(dst + hdmax, v16 + (i * nkv) * hd, 2 * (size_t)hd);
      }
    }

    /* int8 KV: each fp16 row becomes codes and a scale before it is stored or read */
    if (c->kv8)
      for (int64_t t = 0; t < K * nkv; ++t) {
        or_kv_quantize_row(k16 + t * hd, (int)hd, k8 + t * hd, &k8s[t]);
        or_kv_quantize_row(v16 + t * hd, (int)hd, v8 + t * hd, &v8s[t]);
      }
    /* store row i of this block into its cache row */
#define STORE_ROW(i)                                                                        \
  for (int64_t g = 0; g < nkv; ++g) {                                                       \
    const int64_t pos = pos0 + (i);                                                         \
    const int64_t crow = g * crows + (full ? pos : pmod(pos, R));                           \
    const int64_t t = (i) * nkv + g;                                                        \
    if (c->kv8) {                                                                           \
      memcpy(cK8 + crow * hd, k8 + t * hd, (size_t)hd), cKs[crow] = k8s[t];                 \
      memcpy(cV8 + crow * hd, v8 + t * hd, (size_t)hd), cVs[crow] = v8s[t];                 \
    } else {                                                                                \
      memcpy(cK + crow * hd, k16 + t * hd, 2 * (size_t)hd);                                 \
      memcpy(cV + crow * hd, v16 + t * hd, 2 * (size_t)hd);                                 \
    }                                                                                       \
  }
    /* write rows into the cache: mode 1 writes every row before attention */
    int64_t nwrite_before = mode == 1 ? K : 0;
    for (int64_t i = 0; i < nwrite_before; ++i) {
      STORE_ROW(i)
    }

    /* a5/a6: attention */
#pragma omp parallel for schedule(static) collapse(2)
    for (int i = 0; i < K; ++i)
      for (int64_t h = 0; h < Hq; ++h) {
        int64_t qpos = pos0 + i, g = h / G;
        int64_t nmax = full ? qpos + 1 : (W < R ? R : W);
        kvrow* keys = (kvrow*)calloc((size_t)nmax, sizeof(kvrow));
        kvrow* vals = (kvrow*)calloc((size_t)nmax, sizeof(kvrow));
        double* qd = (double*)malloc(sizeof(double) * (size_t)hd);
        for (int64_t d = 0; d < hd; ++d) qd[d] = or_f16_to_double(q16[(i * Hq + h) * hd + d]);
        /* cache row crow, or row t of this block */
#define CACHE_ROW(n, crow)                                                    \
  if (c->kv8) {                                                               \
    keys[n].c = cK8 + (crow) * hd, keys[n].s = cKs[crow];                     \
    vals[n].c = cV8 + (crow) * hd, vals[n].s = cVs[crow];                     \
  } else {                                                                    \
    keys[n].h = cK + (crow) * hd, vals[n].h = cV + (crow) * hd;               \
  }
        int64_t n = 0;
        if (mode == 1 && !full) {
          /* the ring read literally: every slot, implied position, window test */
          for (int64_t a = R - 1; a >= 0; --a) {
            int64_t j = pmod(qpos - a, R);
            int64_t p = qpos - pmod(qpos - j, R);
            if (p < 0 || qpos - p >= W) continue;
            CACHE_ROW(n, g * R + j)
            ++n;
          }
        } else {
          /* positions of the window (sliding) or the whole prefix (full) */
          int64_t p_lo = full ? 0 : (qpos - W + 1 > 0 ? qpos - W + 1 : 0);
          for (int64_t p = p_lo; p <= qpos; ++p) {
            if (mode == 0 && p >= pos0) { /* this block's own rows */
              const int64_t t = (p - pos0) * nkv + g;
              if (c->kv8) {
                keys[n].c = k8 + t * hd, keys[n].s = k8s[t];
                vals[n].c = v8 + t * hd, vals[n].s = v8s[t];
              } else {
                keys[n].h = k16 + t * hd, vals[n].h = v16 + t * hd;
              }
            } else {
              CACHE_ROW(n, g * crows + (full ? p : pmod(p, R)))
            }
            ++n;
          }
        }
#undef CACHE_ROW
        attend_one(qd, (int)hd, keys, vals, n, att + (i * Hq + h) * hd);
        free(keys), free(vals), free(qd);
      }
    for (int64_t t = 0; t < K * Hq * hd; ++t) x16[t] = or_f16_from_double(att[t]);

    /* mode 0 commits the accepted rows after the block is evaluated */
    if (mode == 0)
      for (int64_t i = 0; i < accepted; ++i) {
        STORE_ROW(i)
      }
#undef STORE_ROW

    /* a7/a8: output projection, post-attention norm, residual */
    or_gemv(L->wo.qs, L->wo.sc, H, Hq * hd, K, x16, tmp);
    for (int i = 0; i < K; ++i) {
      or_rmsnorm(tmp + i * H, L->n_pa, H, cfg->rms_eps, tmp + i * H);
      for (int64_t col = 0; col < H; ++col) r[i * H + col] += tmp[i * H + col];
    }
    /* pre-FFN norm, fp16 */
    for (int i = 0; i < K; ++i) {
      or_rmsnorm(r + i * H, L->n_pf, H, cfg->rms_eps, tmp + i * H);
      to_f16(tmp + i * H, H, x16 + i * H);
    }
    /* a9/a10: gate and up projections, GeGLU (tanh GELU), fp16 */
    or_gemv(L->wg.qs, L->wg.sc, F, H, K, x16, gg);
    or_gemv(L->wu.qs, L->wu.sc, F, H, K, x16, uu);
    for (int64_t t = 0; t < K * F; ++t) x16[t] = or_f16_from_double(or_gelu_tanh(gg[t]) * uu[t]);
    /* a11/a12: down projection, post-FFN norm, residual, layer scalar */
    or_gemv(L->wd.qs, L->wd.sc, H, F, K, x16, tmp);
    for (int i = 0; i < K; ++i) {
      or_rmsnorm(tmp + i * H, L->n_po, H, cfg->rms_eps, tmp + i * H);
      for (int64_t col = 0; col < H; ++col)
        r[i * H + col] = (r[i * H + col] + tmp[i * H + col]) * L->lscalar;
      if (dump)
        memcpy(dump + ((int64_t)i * (cfg->n_layers + 1) + l + 1) * H, r + i * H, sizeof(double) * (size_t)H);
    }
  }

  /* a13: final norm, tied head, softcap, argmax */
  for (int i = 0; i < K; ++i) {
    or_rmsnorm(r + i * H, m->n_final, H, cfg->rms_eps, tmp);
    to_f16(tmp, H, x16 + i * H);
  }
  double* lg = (double*)malloc(sizeof(double) * (size_t)(K * V));
  if (cfg->head_fp16)
    or_gemv_f16(m->embed16, V, H, K, x16, lg);
  else
    or_gemv(m->embed.qs, m->embed.sc, V, H, K, x16, lg);
  for (int i = 0; i < K; ++i) {
    int32_t best = 0;
    float bv = -INFINITY;
    for (int64_t t = 0; t < V; ++t) {
      double z = or_softcap(lg[i * V + t], cfg->softcap);
      lg[i * V + t] = z;
      float zf = (float)z;
      if (zf > bv) {
        bv = zf;
        best = (int32_t)t;
      }
    }
    if (argmax) argmax[i] = best;
  }
  if (logits) memcpy(logits, lg, sizeof(double) * (size_t)(K * V));
  free(lg);
  free(r), free(tmp), free(x16), free(qp), free(kp), free(vp), free(q16), free(k16), free(v16);
  free(att), free(gg), free(uu), free(hv), free(k8), free(v8), free(k8s), free(v8s);
  return 0;
}

/* Array conversions for the Python wrapper. */
void or_f16_from_double_array(const double* x, int64_t n, uint16_t* y) {
  for (int64_t i = 0; i < n; ++i) y[i] = or_f16_from_double(x[i]);
}

void or_f16_to_double_array(const uint16_t* x, int64_t n, double* y) {
  for (int64_t i = 0; i < n; ++i) y[i] = or_f16_to_double(x[i]);
}

int or_num_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

void or_set_num_threads(int n) {
#ifdef _OPENMP
  if (n > 0) omp_set_num_threads(n);
#else
  (void)n;
#endif
}

/* Seeded N(0, sigma) values rounded to fp16 (datagen definition), for loading
 * the same synthetic K/V history as the GPU harness. */
void or_fill_normal_f16(uint16_t* out, int64_t n, uint64_t seed, uint64_t stream, float sigma,
                        int64_t start) {
  uint64_t key = dg_key(seed, stream);
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < n; ++i)
    out[i] = or_f16_from_double((double)dg_normal(key, (uint64_t)(start + i), sigma));
}

void or_fill_code8(int8_t* out, int64_t n, uint64_t seed, uint64_t stream, int64_t start) {
  const uint64_t key = dg_key(seed, stream);
  for (int64_t i = 0; i < n; ++i) out[i] = (int8_t)dg_code8(key, (uint64_t)(start + i));
}
