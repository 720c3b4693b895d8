/*
 * Seeded synthetic-input generators, shared by the CPU oracle and by the GPU
 * test/bench harness. This header holds NONE of the decode method's arithmetic:
 * it only turns (seed, stream, index) into numbers.
 *
 * Every value is a pure function of (seed, stream, index), so a tensor can be
 * filled by any number of threads, on the host or on the device, and come out
 * bit-identical. Only integer operations and exactly-rounded IEEE fp32
 * operations are used, so the CPU and the GPU produce the same bits.
 *
 * Definitions (the Python twin in datagen/__init__.py follows the same ones):
 *   mix64(z)        = SplitMix64 finaliser (Steele, Lea, Flood 2014):
 *                     z ^= z>>30; z *= 0xBF58476D1CE4E5B9; z ^= z>>27;
 *                     z *= 0x94D049BB133111EB; z ^= z>>31
 *   splitmix64(x)   = mix64(x + 0x9E3779B97F4A7C15)
 *   key(seed, s)    = splitmix64(splitmix64(seed) ^ (s * 0xD1B54A32D192ED03))
 *   word(key, i, j) = splitmix64(key + 4*i + j)            (j = 0..3, mod 2^64)
 *   unit normal     = Irwin-Hall sum of twelve 16-bit uniforms taken from
 *                     words j = 0,1,2 (four 16-bit lanes each), centred:
 *                     z = (sum - 393210) / 65536          (exact in fp32)
 *                     mean 0, variance 1 - 2^-32, support (-6, 6)
 *   normal(sigma)   = z * sigma                            (one fp32 multiply)
 *   uniform int     = word(key, i, 3) mod n
 *   uniform float   = lo + (hi - lo) * ((word(key, i, 3) >> 40) * 2^-24)
 */
#ifndef Q4G_DATAGEN_H
#define Q4G_DATAGEN_H

#include <stdint.h>

#ifdef __CUDACC__
#define DG_FN __host__ __device__ static inline
#else
#define DG_FN static inline
#endif

DG_FN uint64_t dg_mix64(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

DG_FN uint64_t dg_splitmix64(uint64_t x) { return dg_mix64(x + 0x9E3779B97F4A7C15ull); }

DG_FN uint64_t dg_key(uint64_t seed, uint64_t stream) {
  return dg_splitmix64(dg_splitmix64(seed) ^ (stream * 0xD1B54A32D192ED03ull));
}

DG_FN uint64_t dg_word(uint64_t key, uint64_t i, unsigned j) {
  return dg_splitmix64(key + 4ull * i + (uint64_t)j);
}

/* Irwin-Hall(12) unit normal; exact in fp32. */
DG_FN float dg_unit_normal(uint64_t key, uint64_t i) {
  int32_t s = 0;
  for (unsigned j = 0; j < 3; ++j) {
    uint64_t w = dg_word(key, i, j);
    s += (int32_t)(w & 0xFFFFu);
    s += (int32_t)((w >> 16) & 0xFFFFu);
    s += (int32_t)((w >> 32) & 0xFFFFu);
    s += (int32_t)((w >> 48) & 0xFFFFu);
  }
  return (float)(s - 393210) * (1.0f / 65536.0f);
}

/* A seeded int8 code: 36 x the same Irwin-Hall(12) normal, rounded to the
 * nearest integer (ties to even) in exact integer arithmetic, clamped to
 * [-127, 127] (synthetic int8 K/V history; 36 codes per standard deviation). */
DG_FN int dg_code8(uint64_t key, uint64_t i) {
  int64_t s = 0;
  for (unsigned j = 0; j < 3; ++j) {
    uint64_t w = dg_word(key, i, j);
    s += (int64_t)(w & 0xFFFFu);
    s += (int64_t)((w >> 16) & 0xFFFFu);
    s += (int64_t)((w >> 32) & 0xFFFFu);
    s += (int64_t)((w >> 48) & 0xFFFFu);
  }
  const int64_t t = 9 * (s - 393210); /* 36 z = t / 2^14 exactly */
  int64_t q = t >> 14;                /* floor */
  const int64_t r = t - q * 16384;    /* 0 <= r < 2^14 */
  if (r > 8192 || (r == 8192 && (q & 1))) q += 1;
  return (int)(q > 127 ? 127 : (q < -127 ? -127 : q));
}

DG_FN float dg_normal(uint64_t key, uint64_t i, float sigma) {
#ifdef __CUDA_ARCH__
  return __fmul_rn(dg_unit_normal(key, i), sigma);
#else
  volatile float z = dg_unit_normal(key, i);
  return z * sigma;
#endif
}

DG_FN uint64_t dg_uniform_int(uint64_t key, uint64_t i, uint64_t n) {
  return dg_word(key, i, 3) % n;
}

DG_FN float dg_uniform_float(uint64_t key, uint64_t i, float lo, float hi) {
  float u = (float)(dg_word(key, i, 3) >> 40) * (1.0f / 16777216.0f);
#ifdef __CUDA_ARCH__
  return __fadd_rn(lo, __fmul_rn(__fsub_rn(hi, lo), u));
#else
  volatile float span = hi - lo;
  volatile float t = span * u;
  return lo + t;
#endif
}

/* Norm gain of the seeded variant: 1 + N(0, 0.1), one fp32 add. */
DG_FN float dg_gain(uint64_t key, uint64_t i) {
#ifdef __CUDA_ARCH__
  return __fadd_rn(1.0f, dg_normal(key, i, 0.1f));
#else
  volatile float z = dg_normal(key, i, 0.1f);
  return 1.0f + z;
#endif
}

/* Base gain of the per-head q_norm / k_norm of the synthetic decoder: hd^(-1/4),
 * so that scale-1.0 attention over two unit-RMS vectors has unit-variance scores
 * (q.k ~ N(0, 1)) instead of standard deviation sqrt(hd). fp32 constants. */
DG_FN float dg_qk_gain_base(int hd) {
  return hd == 256 ? 0.25f : hd == 512 ? 0.21022410381342863f : hd == 64 ? 0.35355339059327373f
       : hd == 32 ? 0.42044820762685725f : 1.0f;
}

/* q_norm / k_norm gain element i: base (variant 0), base * (1 + N(0, 0.1)) in the
 * seeded variant 1 (one fp32 multiply), or 1 in variant 2 (unit gains: the
 * softmax logits q.k are of order head_dim, a sharp softmax). */
DG_FN float dg_qk_gain(uint64_t key, uint64_t i, int hd, int variant) {
  if (variant == 2) return 1.0f;
  float b = dg_qk_gain_base(hd);
  if (variant != 1) return b;
#ifdef __CUDA_ARCH__
  return __fmul_rn(b, dg_gain(key, i));
#else
  volatile float g = dg_gain(key, i);
  return b * g;
#endif
}

/*
 * Stream ids of the synthetic workloads. A weight tensor of shape [rows][cols]
 * draws element (r, c) at index r*cols + c.
 */
#define DG_STREAM_EMBED 0x100ull          /* tied embedding / head [V][h]     */
#define DG_STREAM_FINAL_NORM 0x101ull     /* final RMSNorm gain [h]           */
#define DG_STREAM_LAYER(l, t) (0x1000ull + (uint64_t)(l) * 0x20ull + (uint64_t)(t))
enum {
  DG_T_WQ = 0, DG_T_WK = 1, DG_T_WV = 2, DG_T_WO = 3,
  DG_T_WGATE = 4, DG_T_WUP = 5, DG_T_WDOWN = 6,
  DG_T_NORM_IN = 7, DG_T_NORM_POST_ATTN = 8, DG_T_NORM_PRE_FFN = 9, DG_T_NORM_POST_FFN = 10,
  DG_T_NORM_Q = 11, DG_T_NORM_K = 12, DG_T_LAYER_SCALAR = 13
};
#define DG_STREAM_HIDDEN(pos) (0x200000ull + (uint64_t)(pos)) /* prefill hidden states */
#define DG_STREAM_PREFIX_IDS 0x300000ull  /* random-id prefix, index = position */
#define DG_STREAM_DRAFT_IDS 0x400000ull   /* verify drafts, index = block*K + row */
#define DG_STREAM_ACCEPTED 0x500000ull    /* accepted counts, index = block    */
#define DG_STREAM_BENCH_X(s) (0x600000ull + (uint64_t)(s))   /* GEMV microbench x */
#define DG_STREAM_BENCH_W(s) (0x700000ull + (uint64_t)(s))   /* GEMV microbench W */
#define DG_STREAM_ATTN(s) (0x800000ull + (uint64_t)(s))      /* attention microbench */

#endif /* Q4G_DATAGEN_H */
