/*
 * CPU oracle for the batch-1 q4_0 decode step: TEST INFRASTRUCTURE ONLY.
 *
 * A plain, slow, obviously correct restatement of what the decode step computes,
 * in double precision, rounding to IEEE binary16 only at the storage points the
 * GPU path stores in fp16 (GEMV inputs, q after RoPE, K/V cache rows, attention
 * output, GeGLU output). Only tests/, __graft_entry__.smoke() and bench.py's
 * CPU-baseline leg may load this library. It shares no code with the CUDA path;
 * the only common piece is the seeded input generator (datagen/q4g_datagen.h).
 *
 * Pages followed (titles of the pages the method is described on):
 *   [zoo]   "Gemma 4 12B" model page of coreai-model-zoo: architecture section
 *           (interleaved layers, attention_k_eq_v, dual RoPE, layer_scalar, tied
 *           head, softcap), the q4_0 definition in the intro, the flash-decode
 *           kernel description (scale 1.0, fp32 online softmax).
 *   [12b]   "Gemma-4-12B-CoreAI" (visible-cx): "v5/ - ring extent R = 2W" section
 *           (slot = pos mod R, implied position, window test, single vs two-pass
 *           verify), "The per-tier cost" section (cache shapes).
 *   [e4b]   "gemma-4-E4B-CoreAI" (visible-cx): Provenance table (ggml q4_0 grid),
 *           "stable/" contract (absolute positions, mask derived from positions).
 */
#ifndef Q4G_ORACLE_H
#define Q4G_ORACLE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct {
  int32_t n_layers, hidden, n_q_heads, ffn, vocab;
  int32_t sl_kv_heads, sl_head_dim, window, ring;
  int32_t gl_kv_heads, gl_head_dim, full_every, full_offset, rope_pairs_full;
  double rope_theta_sl, rope_theta_gl, rms_eps, softcap, embed_scale;
  int32_t v_norm_sliding; /* 1: scale-free RMSNorm on sliding-layer V too */
  int32_t head_fp16;      /* 1: the tied embedding / head is fp16 instead of q4_0 */
  int32_t kv_int8;        /* 1: K/V cache rows stored as int8 codes with one fp32 scale per
                             row ("Gemma-4-12B-CoreAI", per-tier cost section) */
} or_config;

/* ---- IEEE binary16 ---- */
uint16_t or_f16_from_double(double x); /* round to nearest even */
double or_f16_to_double(uint16_t h);
void or_f16_from_double_array(const double* x, int64_t n, uint16_t* y);
void or_f16_to_double_array(const uint16_t* x, int64_t n, double* y);
int or_num_threads(void);
void or_set_num_threads(int n);

/* ---- q4_0 (per-block-32 absmax symmetric int4 on the [-8, 7] grid) ----
 * qs[rows][k/2]: byte b of block t holds element 32t+b (low nibble) and
 * 32t+b+16 (high nibble), as code c = q + 8. scales[rows][k/32]: fp16 bits.
 * Returns 0, or -1 for k % 32 != 0 or a non-finite input. */
int or_q4_0_pack(const float* w, int64_t rows, int64_t k, uint8_t* qs, uint16_t* scales);
void or_q4_0_unpack(const uint8_t* qs, const uint16_t* scales, int64_t rows, int64_t k, double* w);

/* y[n] = sum_k dequant(W)[n][k] * x[k]; x as fp16 bits; natural k order. */
void or_gemv(const uint8_t* qs, const uint16_t* scales, int64_t n, int64_t k, int nrhs,
             const uint16_t* x16, double* y);

/* y[n] = sum_k W[n][k] * x[k] for fp16 weights W [n][k]; x as fp16 bits. */
void or_gemv_f16(const uint16_t* w, int64_t n, int64_t k, int nrhs, const uint16_t* x16, double* y);

/* ---- elementwise pieces (double) ---- */
void or_rmsnorm(const double* x, const double* w /* NULL = scale-free */, int64_t n, double eps,
                double* y);
void or_rope(double* x, int64_t head_dim, int64_t rot_pairs, double theta, int64_t pos);
double or_gelu_tanh(double g);
double or_softcap(double z, double cap);

/* ---- standalone attention (one query row), used for kernel-level parity ----
 * Ring: K/V [n_kv][R][hd] fp16, query at absolute position q; a slot j is live
 * iff p = q - ((q - j) mod R) satisfies p >= 0 and q - p < W. Keys are summed
 * in ascending implied position. q16 [n_q][hd]; out [n_q][hd] (double). */
void or_attn_ring(const uint16_t* q16, int n_q, int n_kv, int hd, const uint16_t* kc,
                  const uint16_t* vc, int64_t R, int64_t W, int64_t q, double* out);
/* Linear cache: K/V [L][n_kv][hd]; keys 0..len-1 all live. */
void or_attn_linear(const uint16_t* q16, int n_q, int n_kv, int hd, const uint16_t* kc,
                    const uint16_t* vc, int64_t len, double* out);
/* The same over int8 K/V rows: codes [rows][hd] with one fp32 scale per row
 * (value = code * scale); rows indexed as in the fp16 versions. */
void or_attn_ring_i8(const uint16_t* q16, int n_q, int n_kv, int hd, const int8_t* k8, const float* ks,
                     const int8_t* v8, const float* vs, int64_t R, int64_t W, int64_t q, double* out);
void or_attn_linear_i8(const uint16_t* q16, int n_q, int n_kv, int hd, const int8_t* k8, const float* ks,
                       const int8_t* v8, const float* vs, int64_t len, double* out);
/* int8 KV row from an fp16 row x16[hd]: scale = amax / 127 (fp32 division,
 * amax = largest |x|), code = clamp(rint(x / scale), -127, 127) (fp32
 * division, round to nearest even); an all-zero row: scale 0, codes 0. */
void or_kv_quantize_row(const uint16_t* x16, int hd, int8_t* codes, float* scale);
/* Live-slot mask of the ring for query position q: mask[j] = implied position or -1. */
void or_ring_implied_positions(int64_t R, int64_t W, int64_t q, int64_t* out);

/* Seeded N(0, sigma) rounded to fp16 (datagen definition): synthetic history. */
void or_fill_normal_f16(uint16_t* out, int64_t n, uint64_t seed, uint64_t stream, float sigma,
                        int64_t start);

/* Seeded int8 codes (datagen definition dg_code8): synthetic int8 history. */
void or_fill_code8(int8_t* out, int64_t n, uint64_t seed, uint64_t stream, int64_t start);

/* ---- model ---- */
typedef struct or_model or_model;
typedef struct or_cache or_cache;

/* Weights generated from the seeded recipe: linear weights N(0, 0.02) packed
 * to q4_0; residual-stream norm gains 1 (variants 0 and 2) or 1 + N(0, 0.1)
 * (variant 1); q_norm / k_norm gains hd^(-1/4), times 1 + N(0, 0.1) in
 * variant 1, and 1 in variant 2 (unit gains); layer scalars 1 (variants 0
 * and 2) or U(0.5, 1.5) (variant 1).
 * nthreads <= 0: all. */
or_model* or_model_create(const or_config* cfg, uint64_t seed, int variant, int nthreads);
void or_model_destroy(or_model* m);
/* Packed bytes of one weight tensor, for bit-exact comparison with another packer.
 * tensor: 0 wq, 1 wk, 2 wv, 3 wo, 4 wgate, 5 wup, 6 wdown, 100 embed. Returns rows (0 if absent). */
int64_t or_model_tensor(const or_model* m, int layer, int tensor, const uint8_t** qs,
                        const uint16_t** scales, int64_t* cols);

/* The fp16 tied table [vocab][h] when cfg.head_fp16 (NULL otherwise): fp16 of the
 * same seeded N(0, 0.02) draws the q4_0 table is packed from. */
const uint16_t* or_model_embed_f16(const or_model* m);

or_cache* or_cache_create(const or_model* m, int64_t capacity, int64_t ring_slots /* 0: cfg.ring */);
void or_cache_destroy(or_cache* c);
or_cache* or_cache_clone(const or_cache* c);
/* Direct access to a cache's storage, for loading synthetic history.
 * ring layer index = sliding-layer ordinal; K/V [n_kv][R][hd] fp16.
 * global layer index = full-layer ordinal; K/V [n_kv][capacity][hd] fp16. */
uint16_t* or_cache_ring(or_cache* c, int sl_index, int kv /*0 K, 1 V*/);
uint16_t* or_cache_global(or_cache* c, int gl_index, int kv);
/* The same for a kv_int8 model's cache: codes [n_kv][rows][hd] int8, and
 * *scales [n_kv][rows] fp32 (the fp16 accessors return NULL then, and these
 * return NULL for an fp16 cache). */
int8_t* or_cache_ring_i8(or_cache* c, int sl_index, int kv, float** scales);
int8_t* or_cache_global_i8(or_cache* c, int gl_index, int kv, float** scales);

/* Verify block of K rows at absolute positions pos0..pos0+K-1 (decode = K 1).
 * mode 0 (reference protocol): row i attends the positions
 *   max(0, q_i - W + 1) .. q_i (sliding) / 0 .. q_i (full), taking positions
 *   >= pos0 from this block's own K/V and the rest from the cache; afterwards
 *   rows < accepted are written to the cache. Two-pass verify = a call with
 *   accepted 0, then one with accepted n.
 * mode 1 (single pass over the ring, as the pages describe it): all K rows are
 *   written to the cache first, then each row reads the ring with the
 *   implied-position window test (and the global cache for positions <= q_i).
 * ids: token ids (or NULL with hidden_in [K][h] fp32 replacing the embedding).
 * logits [K][V] (double, softcapped; may be NULL), argmax [K] (decided on the
 * logits rounded to fp32, lowest index on ties; may be NULL).
 * dump (may be NULL): [K][n_layers + 1][h] residual stream after the embedding
 * and after every layer; kv_dump (may be NULL): per layer [K][2][hdmax] the
 * fp16 K and V rows of KV head 0 (hdmax = larger head dim, hd entries used);
 * vraw_dump (may be NULL): per layer [K][hdmax] the raw k_proj output of KV
 * head 0 (double). Returns 0 or -1.
 * Parity unpinned as a whole: the pages print no worked example, expected logits
 * or per-layer values for a decode step, so this composition is pinned only
 * through its parts (q4_0 pack and unpack, GEMV, RMSNorm, RoPE, ring indexing,
 * attention, GeGLU, softcap: each against a closed form, a library routine or
 * brute force) and through a recomposition of those parts from torch primitives. */
int or_verify_block(or_model* m, or_cache* c, const int32_t* ids, const float* hidden_in, int K,
                    int64_t pos0, int accepted, int mode, double* logits, int32_t* argmax,
                    double* dump, uint16_t* kv_dump, double* vraw_dump);

#ifdef __cplusplus
}
#endif
#endif /* Q4G_ORACLE_H */
