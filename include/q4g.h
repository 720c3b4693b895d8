/*
 * libq4g: batch-1 decode step of a dense, interleaved-attention (sliding ring +
 * full layers) Gemma-style decoder with q4_0 weights, for NVIDIA B200 (sm_100a).
 *
 * C ABI: plain pointers and sizes, status codes, no exceptions, no C++ or torch
 * types. Unless a parameter says "host", pointers are DEVICE pointers that the
 * caller allocated (for example through torch) and keeps alive; the library
 * borrows them and never frees them. Handles (q4g_model, q4g_cache) are owned by
 * the library and released by the matching destroy call.
 *
 * Errors: every call validates its arguments on the host first and returns
 * Q4G_EINVAL / Q4G_ERANGE without launching anything. Kernel launches are
 * asynchronous on the given stream; a CUDA failure detected at launch returns
 * Q4G_ECUDA, and a failure that happens later on the device is reported by the
 * next call that synchronises (or by q4g_model_check). q4g_last_error() returns
 * a message for the last failure on the calling thread.
 *
 * Pages the operations are defined on (cited by title and section):
 *   "Gemma 4 12B" (coreai-model-zoo model page): intro (q4_0: per-block-32 absmax
 *     symmetric int4), the architecture paragraph (48 layers, full attention
 *     every 6th layer, attention_k_eq_v, dual RoPE, layer_scalar, tied
 *     embeddings), the flash-decode kernel paragraph (GQA-16:1 decode over the
 *     global cache, scale 1.0, fp32 online softmax, split over 8 groups).
 *   "Gemma-4-12B-CoreAI" (visible-cx): "v5/ - ring extent R = 2W" (slot = pos
 *     mod R, implied position p = q - ((q - j) mod R), window test (q - p) < W,
 *     single-pass verify with accepted_count = K), "The per-tier cost" (global
 *     pair [C][512] fp16 per full layer, ring [n_kv][R][256] per sliding layer),
 *     "Requirements" (engine contract: input_ids, position_ids -> logits),
 *     "tiered-v3/" (verify returning full logits per row).
 *   "gemma-4-E4B-CoreAI" (visible-cx): Provenance table (the ggml q4_0 grid),
 *     "stable/" contract (absolute positions; the mask is derived from them).
 */
#ifndef Q4G_H
#define Q4G_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define Q4G_ABI_VERSION 3

/* A CUDA stream (cudaStream_t / CUstream). NULL selects the legacy default stream. */
typedef struct CUstream_st* q4g_stream_t;

typedef enum {
  Q4G_OK = 0,
  Q4G_EINVAL = 1,   /* bad pointer, shape, alignment or configuration   */
  Q4G_ERANGE = 2,   /* position / row count / accepted_count out of range */
  Q4G_ENOMEM = 3,   /* a library allocation (handles, scratch) failed     */
  Q4G_ECUDA = 4,    /* a CUDA runtime error (launch or sticky device error) */
  Q4G_ETIMEOUT = 5  /* a bounded device-side wait gave up                 */
} q4g_status;

/* Message for the last failure on this thread ("" if none). Never NULL. */
const char* q4g_last_error(void);
const char* q4g_status_string(q4g_status s);
int q4g_abi_version(void);

/* ------------------------------------------------------------------------ */
/* q4_0 weight format ("Gemma 4 12B" intro; "gemma-4-E4B-CoreAI" Provenance). */
/* For a matrix W[rows][k] (k % 32 == 0), each block of 32 consecutive columns  */
/* of a row stores one fp16 scale d = fp16(m / -8), m the block element of     */
/* largest magnitude (the first one on ties, sign kept), and 32 codes          */
/* c = clamp(round_half_away(x / d), -8, 7) + 8 (fp32 division); d == 0 stores  */
/* every code as 8. Dequantised value: (c - 8) * d.                             */
/* Layout (row-major, structure of arrays):                                     */
/*   qs[rows][k/2] uint8: byte b (0..15) of block t holds column 32t+b in its   */
/*                        low nibble and column 32t+b+16 in its high nibble.    */
/*   scales[rows][k/32] uint16 (IEEE binary16 bits).                            */
/* ------------------------------------------------------------------------ */

/* Quantise fp32 rows. on_device = 1: all pointers are device pointers and the
 * call is asynchronous on `stream` except that it synchronises once to report
 * non-finite input. on_device = 0: host pointers; the data is staged through
 * temporary device memory (the packing itself always runs on the GPU) and the
 * call returns when the host outputs are written.
 * Errors: Q4G_EINVAL if k % 32 != 0, rows < 0, a NULL pointer, or any input
 * value is NaN or infinite (outputs are then unspecified). */
q4g_status q4g_q4_0_pack(const float* w, int64_t rows, int64_t k, uint8_t* qs, uint16_t* scales,
                         int on_device, q4g_stream_t stream);

/* Dequantise to fp32 w[rows][k]; same pointer rules as q4g_q4_0_pack. */
q4g_status q4g_q4_0_unpack(const uint8_t* qs, const uint16_t* scales, int64_t rows, int64_t k,
                           float* w, int on_device, q4g_stream_t stream);

/* ------------------------------------------------------------------------ */
/* Standalone kernels (device pointers, asynchronous).                        */
/* ------------------------------------------------------------------------ */

/* q4_0 matrix-vector product, dequantisation fused into the dot product:
 * y[j][r] = sum_c (code(r, c) - 8) * d(r, c/32) * x[j][c] for j < nrhs,
 * fp16 x [nrhs][k], fp32 accumulation, fp32 y [nrhs][n].
 * Requires k % 32 == 0, 1 <= nrhs <= 8, qs 16-byte aligned, scales 2-byte
 * aligned, x 16-byte aligned. No scratch memory. */
q4g_status q4g_gemv(const uint8_t* qs, const uint16_t* scales, int64_t n, int64_t k,
                    const uint16_t* x_f16, int32_t nrhs, float* y, q4g_stream_t stream);

/* fp16 matrix-vector product (the fp16 tied head's GEMV without its epilogue):
 * y[j][r] = sum_c w16[r][c] * x[j][c] for j < nrhs, IEEE binary16 w16 [n][k]
 * and x [nrhs][k], products exact in fp32, fp32 accumulation, fp32 y [nrhs][n].
 * Requires k % 256 == 0, k <= 8192, 1 <= nrhs <= 8, w16 and x 16-byte aligned.
 * No scratch memory. Q4G_EINVAL on a bad size or pointer. */
q4g_status q4g_gemv_f16(const uint16_t* w16, int64_t n, int64_t k, const uint16_t* x_f16, int32_t nrhs,
                        float* y, q4g_stream_t stream);

/* Process-wide choice of the q4_0 GEMV kernel, for tuning and tests (not on
 * the pages). All kernels compute the same operation within the same error
 * bound; the default picks per shape:
 *   Q4G_GEMV_AUTO          the stage kernel where it can take the call, else the
 *                          warp-streamed kernel, else the register kernel,
 *   Q4G_GEMV_WARP_STREAM   per-warp bulk-copy rings (k % 256 == 0),
 *   Q4G_GEMV_REGISTER      plain streaming loads (any k % 32 == 0),
 *   Q4G_GEMV_STAGE         integer dot, every warp of a CTA on each 16-36 KB
 *                          stage of one contiguous bulk-copy stream, one warp
 *                          reducing and refilling (k % 256 == 0, <= 4
 *                          activation rows, 16-byte aligned operands).
 * A kernel that cannot take a call falls back to the automatic choice. Affects launches
 * made (and CUDA graphs captured) after the call. Q4G_EINVAL for other kinds
 * (1 is retired). */
#define Q4G_GEMV_AUTO 0
#define Q4G_GEMV_WARP_STREAM 2
#define Q4G_GEMV_REGISTER 3
#define Q4G_GEMV_STAGE 4
q4g_status q4g_set_gemv_kernel(int32_t kind);

/* Workspace for the split-KV flash-decode entry points below (bytes, >= 256). */
size_t q4g_flash_decode_workspace_bytes(int32_t n_q_heads, int32_t head_dim);

/* Flash-decode over a sliding-window ring ("Gemma-4-12B-CoreAI", v5 section):
 * q [n_q][hd] fp16 (already normed/rotated), K/V ring [n_kv][R][hd] fp16 with
 * slot = position mod R. For the query at absolute position `pos`, slot j is
 * attended iff p = pos - ((pos - j) mod R) satisfies p >= 0 and pos - p < W.
 * Query head h uses KV head h / (n_q / n_kv). Scale 1.0, fp32 online softmax,
 * fp16 output [n_q][hd]. hd must be 256 or 512; W <= R <= 2^30 (Q4G_ERANGE
 * above); pos is any non-negative int64.
 * workspace: device buffer of q4g_flash_decode_workspace_bytes(n_q, hd) bytes,
 * 256-byte aligned, used as scratch by this call (calls that share a workspace
 * must not overlap on the GPU). */
q4g_status q4g_flash_decode_ring(const uint16_t* q, int32_t n_q, int32_t n_kv, int32_t head_dim,
                                 const uint16_t* k_ring, const uint16_t* v_ring, int64_t ring,
                                 int64_t window, int64_t pos, uint16_t* out, void* workspace,
                                 size_t workspace_bytes, q4g_stream_t stream);

/* Flash-decode over a linear cache ("Gemma 4 12B", flash-decode paragraph):
 * K/V [len_capacity][n_kv][hd] fp16, keys 0..len-1 all attended (mask-free,
 * causal by construction), 1 <= len <= 2^30. Otherwise as q4g_flash_decode_ring. */
q4g_status q4g_flash_decode_linear(const uint16_t* q, int32_t n_q, int32_t n_kv, int32_t head_dim,
                                   const uint16_t* k, const uint16_t* v, int64_t len, uint16_t* out,
                                   void* workspace, size_t workspace_bytes, q4g_stream_t stream);

/* The same two over int8 rows (the kv_int8 cache format): codes [.][hd] int8
 * and one fp32 scale per row, scales laid out like the rows without head_dim
 * (ring: [n_kv][ring]; linear: [len_capacity][n_kv]); value = code * scale.
 * Codes 16-byte aligned, scales 4-byte aligned. Otherwise as above. */
q4g_status q4g_flash_decode_ring_i8(const uint16_t* q, int32_t n_q, int32_t n_kv, int32_t head_dim,
                                    const int8_t* k_codes, const float* k_scales, const int8_t* v_codes,
                                    const float* v_scales, int64_t ring, int64_t window, int64_t pos,
                                    uint16_t* out, void* workspace, size_t workspace_bytes,
                                    q4g_stream_t stream);
q4g_status q4g_flash_decode_linear_i8(const uint16_t* q, int32_t n_q, int32_t n_kv, int32_t head_dim,
                                      const int8_t* k_codes, const float* k_scales, const int8_t* v_codes,
                                      const float* v_scales, int64_t len, uint16_t* out, void* workspace,
                                      size_t workspace_bytes, q4g_stream_t stream);

/* Allocation-free variant of q4g_flash_decode_ring (no counterpart on the pages;
 * an integration convenience). It is for callers that cannot allocate device
 * memory at call time -- for example a program whose device memory belongs to a
 * framework's caching allocator that this library cannot reach, or a process
 * that reserves its memory budget at start-up and treats a later cudaMalloc as
 * a failure -- and so cannot provide the workspace the ordinary entry point
 * takes. Same inputs, outputs and results as q4g_flash_decode_ring; the
 * split-KV scratch lives in one fixed device array of
 * Q4G_NOALLOC_SCRATCH_BYTES, which every GPU that loads the library holds until
 * the process exits. It must hold 256 bytes of counters plus, per query head
 * and chunk, 8 bytes of (max, sum) and head_dim * 4 bytes of partial output
 * (chunks = ceil(window / 64) at most); larger requests return Q4G_ERANGE with
 * a message. The call makes no device allocation or free of any kind; it
 * clears the counters (an asynchronous memset on `stream`) and launches one
 * kernel. The first call on a device looks up the array's device address with
 * that device current; make that first call before any stream capture. All
 * calls on a device share the array, and it keeps the last call's contents:
 * calls that overlap on the GPU (other streams, or without ordering between
 * them) race on it and must be serialised by the caller. */
#define Q4G_NOALLOC_SCRATCH_BYTES ((size_t)1 << 20)
q4g_status q4g_flash_decode_ring_noalloc(const uint16_t* q, int32_t n_q, int32_t n_kv,
                                         int32_t head_dim, const uint16_t* k_ring,
                                         const uint16_t* v_ring, int64_t ring, int64_t window,
                                         int64_t pos, uint16_t* out, q4g_stream_t stream);

/* ------------------------------------------------------------------------ */
/* Model and cache.                                                           */
/* ------------------------------------------------------------------------ */

/* Decoder configuration ("Gemma 4 12B" architecture paragraph; values for the
 * 12B-class decoder in brackets). Layer l is a full-attention layer iff
 * full_every > 0 and l % full_every == full_offset [6, 5]; the others are
 * sliding-window layers. */
typedef struct {
  int32_t n_layers;        /* [48] */
  int32_t hidden;          /* h [3840], multiple of 32, at most 8192 */
  int32_t n_q_heads;       /* [16] */
  int32_t ffn;             /* [15360], multiple of 256 */
  int32_t vocab;           /* tied embedding / head rows [262144], multiple of 16 */
  int32_t sl_kv_heads;     /* sliding layers: KV heads [8] */
  int32_t sl_head_dim;     /* sliding head dim [256] (256 only) */
  int32_t window;          /* W [1024] */
  int32_t ring;            /* R [2048]; R >= W + 8 so a verify block never aliases */
  int32_t gl_kv_heads;     /* full layers: KV heads [1] */
  int32_t gl_head_dim;     /* full head dim [512] (512 only) */
  int32_t full_every;      /* [6] */
  int32_t full_offset;     /* [5] */
  int32_t rope_pairs_full; /* rotating frequency pairs on full layers [64] */
  float rope_theta_sl;     /* [1e4] all pairs rotate */
  float rope_theta_gl;     /* [1e6] "proportional": pairs >= rope_pairs_full do not rotate */
  float rms_eps;           /* [1e-6] */
  float softcap;           /* final logit softcap c: c * tanh(z / c) [30] */
  float embed_scale;       /* embedding multiplier [sqrt(h)] */
  int32_t v_norm_sliding;  /* 1: scale-free RMSNorm on sliding-layer V as on full layers */
  int32_t head_fp16;       /* 0: the tied embedding / head is q4_0 (q4g_weights.embed);
                              1: it is fp16 (q4g_weights.embed_f16, [vocab][h] IEEE
                              binary16, the "fp16 vocab path" of "Gemma-4-12B-CoreAI",
                              tiered-v3/ section): the head GEMV reads 2 B per weight
                              and the embedding row is the fp16 row times embed_scale */
  int32_t kv_int8;         /* 0: K/V cache rows fp16; 1: int8 ("Gemma-4-12B-CoreAI",
                              per-tier cost section: int8 KV), each row of head_dim
                              codes with one fp32 scale: scale = amax / 127, code =
                              clamp(rint(x / scale), -127, 127) for the row's fp16
                              values x (both IEEE fp32 divisions), value = code *
                              scale; see q4g_cache_view for the layout */
} q4g_config;

/* One q4_0 tensor in the layout above (device pointers, borrowed). */
typedef struct {
  const uint8_t* qs;      /* 16-byte aligned */
  const uint16_t* scales; /* 4-byte aligned */
} q4g_qtensor;

/* Weights of one layer. Projections are [out][in]:
 *   wq [n_q_heads*hd][h], wk [n_kv*hd][h], wv [n_kv*hd][h] (sliding layers only;
 *   full layers take V from the raw k_proj output: attention_k_eq_v),
 *   wo [h][n_q_heads*hd], wgate/wup [ffn][h], wdown [h][ffn].
 * Norm gains are fp32 device vectors: norm_in/post_attn/pre_ffn/post_ffn [h],
 * norm_q/norm_k [hd]. layer_scalar multiplies the residual at the end of the layer. */
typedef struct {
  q4g_qtensor wq, wk, wv, wo, wgate, wup, wdown;
  const float *norm_in, *norm_post_attn, *norm_pre_ffn, *norm_post_ffn, *norm_q, *norm_k;
  float layer_scalar;
} q4g_layer_weights;

typedef struct {
  const q4g_layer_weights* layers; /* host array [n_layers], copied by q4g_model_create */
  q4g_qtensor embed;               /* tied embedding and LM head [vocab][h] (head_fp16 = 0) */
  const float* norm_final;         /* [h] */
  const uint16_t* embed_f16;       /* tied embedding and LM head [vocab][h] fp16, 16-byte
                                      aligned (head_fp16 = 1; NULL otherwise) */
} q4g_weights;

typedef struct q4g_model q4g_model;
typedef struct q4g_cache q4g_cache;

/* Create a model over borrowed device weights. Validates every shape and
 * alignment, allocates the library's scratch (activations, split-KV partials,
 * counters: a few tens of MB) on the current device. Q4G_EINVAL on a bad
 * configuration or pointer, Q4G_ENOMEM if scratch cannot be allocated. */
q4g_status q4g_model_create(const q4g_config* cfg, const q4g_weights* w, q4g_model** out);
void q4g_model_destroy(q4g_model* m);

/* Reports (and clears) the device-side error word that a bounded wait sets when
 * it gives up (Q4G_ETIMEOUT; every wait inside the kernels is limited in time,
 * 2 s by default) and any sticky CUDA error (Q4G_ECUDA). Synchronises `stream`.
 * Diagnostics: with Q4G_DEBUG_SYNC set in the environment, eager (non-graph)
 * steps synchronise after every launch and name the launch that failed. */
q4g_status q4g_model_check(q4g_model* m, q4g_stream_t stream);

/* Options (defaults in brackets): */
typedef enum {
  Q4G_OPT_CUDA_GRAPH = 1, /* [1] replay a captured CUDA graph per step shape   */
  Q4G_OPT_PDL = 2,        /* [1] programmatic dependent launch between kernels */
  Q4G_OPT_DUMP = 3,       /* [0] value = device float* [K][n_layers+1][h]: residual
                                 stream after the embedding and after each layer */
  Q4G_OPT_PROFILE = 4,    /* [0] 1: launch eagerly and bracket every kernel with CUDA
                                 events on the launching stream (read with
                                 q4g_model_profile_read) */
  Q4G_OPT_TEST_STALL = 5, /* [0] 1: failure-path test. In the next step, one pipeline
                                 stage of the first GEMV expects 16 bytes that never
                                 arrive; its bounded wait (20 ms) gives up, the step
                                 finishes with unspecified results and
                                 q4g_model_check returns Q4G_ETIMEOUT. One-shot. */
  Q4G_OPT_ATTN_CLUSTER = 6, /* [1] sliding layers: the 8 key chunks of a KV head run
                                 as one thread-block cluster and merge their partial
                                 softmax sums through distributed shared memory;
                                 0: split-KV with a merge through global memory */
  Q4G_OPT_TRACE = 8         /* [0] value = device uint64_t* [1536]: %globaltimer stamps
                                 (ns) of CTA 0 of layer 1's launches, 256 entries each:
                                 gate|up at 0, QKV at 256, O at 512, down at 768 (per
                                 GEMV launch: 0 entry, 1 dependency wait done, 2 x
                                 digits built, 3 and 4 (fused norm prologue) first
                                 loads used and second norm reduced, 5 last stage
                                 reduced, 8 + t stage t issued, 72 + t stage t ready,
                                 136 + t stage t reduced, t < 64); the sliding
                                 attention at 1024 when it runs on the cluster kernel
                                 (0 entry, 1 dependency wait, 2 queries ready, 3 scan
                                 done, 4 warps merged, 5 cluster synced, 6 output
                                 written, 7 exit); from 1280, when each CTA of layer
                                 1's gate|up finished its last stage. Unwritten slots
                                 keep their contents. Option values 7, 9, 10 and 11
                                 are retired (Q4G_EINVAL). */
} q4g_option;
q4g_status q4g_model_set_option(q4g_model* m, q4g_option opt, intptr_t value);

/* One kernel launch recorded in profile mode. kind: 0 step init, 1 QKV GEMV,
 * 2 sliding attention, 3 full attention, 4 attention combine, 5 O GEMV,
 * 6 gate|up GEMV, 7 down GEMV, 8 head GEMV. bytes: algorithmic HBM bytes of the
 * launch (q4_0 weights 0.5625 B/weight, fp16 head weights 2 B/weight, plus
 * activations; attention: the live K/V rows, 2 * head_dim * 2 B per key and KV
 * head). */
typedef struct {
  int32_t kind;
  int32_t layer;
  float ms;
  double bytes;
} q4g_launch_record;

/* Synchronises `stream`, copies up to `max` records of the launches made since
 * the last read into `out` (host), clears them and returns how many there were
 * (which may exceed max), or -1 on error (see q4g_last_error). */
int32_t q4g_model_profile_read(q4g_model* m, q4g_launch_record* out, int32_t max,
                               q4g_stream_t stream);

/* KV cache for up to `capacity` positions: per sliding layer a ring K and V of
 * [sl_kv_heads][ring][sl_head_dim] (slot = position mod ring); per full layer K
 * and V of [gl_kv_heads][capacity][gl_head_dim] indexed by absolute position
 * ("Gemma-4-12B-CoreAI": v5 section and "The per-tier cost"); fp16 rows, or int8
 * rows with scales (kv_int8, see q4g_cache_view). The
 * storage is a caller-owned device buffer of q4g_cache_bytes() bytes.
 * 1 <= capacity <= 2^30, else Q4G_ERANGE. */
q4g_status q4g_cache_bytes(const q4g_model* m, int64_t capacity, size_t* bytes);
q4g_status q4g_cache_init(const q4g_model* m, int64_t capacity, void* dev_buf, size_t bytes,
                          q4g_cache** out);
/* Zero the cache contents (asynchronous). */
q4g_status q4g_cache_reset(q4g_cache* c, q4g_stream_t stream);
void q4g_cache_destroy(q4g_cache* c); /* frees the handle, not the caller's buffer */

/* Byte offsets inside the cache buffer, for snapshots and test access. A layer's
 * K (or V) region holds [n_kv][rows][hd] fp16 values, or with kv_int8 [n_kv][rows][hd]
 * int8 codes followed, at scale_offset within the region, by [n_kv][rows] fp32
 * scales (rows = ring for sliding layers, capacity for full layers). */
typedef struct {
  int64_t capacity, ring;
  int32_t n_sliding, n_full, sl_kv_heads, sl_head_dim, gl_kv_heads, gl_head_dim;
  size_t ring_k_offset, ring_v_offset, ring_layer_bytes;       /* layer i at offset + i*bytes */
  size_t global_k_offset, global_v_offset, global_layer_bytes; /* full-layer ordinal i */
  size_t total_bytes;
  int32_t kv_int8;
  size_t ring_scale_offset, global_scale_offset; /* within a layer's K or V region (kv_int8) */
} q4g_cache_view;
q4g_status q4g_cache_layout(const q4g_cache* c, q4g_cache_view* out);

/* ------------------------------------------------------------------------ */
/* Decode and verify ("Gemma-4-12B-CoreAI": Requirements engine contract and    */
/* v5 section; "gemma-4-E4B-CoreAI": stable/ contract).                       */
/* ------------------------------------------------------------------------ */

/* One decode step: token `token` (host value) at absolute position `pos`, which
 * is also the cache row written (ring slot pos mod R on sliding layers, row
 * pos on full layers). Sliding layers attend positions pos-W+1..pos, full layers
 * 0..pos. Writes softcapped fp32 logits [vocab] (if logits != NULL) and the
 * greedy argmax (lowest index on ties) to argmax[0] (if != NULL); device outputs.
 * With logits and argmax both NULL (and no dump buffer set) the step only
 * appends its K/V rows to the cache: the final norm and the head are skipped.
 * Q4G_ERANGE if pos < 0 or pos >= capacity or token outside [0, vocab).
 * The host owns the position counter; the cache holds contents only. */
q4g_status q4g_decode_step(q4g_model* m, q4g_cache* c, int32_t token, int64_t pos, float* logits,
                           int32_t* argmax, q4g_stream_t stream);

/* As q4g_decode_step, but the token id is read from device memory when the step
 * runs (for example the previous step's argmax), so a greedy loop needs no host
 * round trip. An out-of-range id is clamped into [0, vocab) on the device. */
q4g_status q4g_decode_step_device_token(q4g_model* m, q4g_cache* c, const int32_t* token,
                                        int64_t pos, float* logits, int32_t* argmax,
                                        q4g_stream_t stream);

/* As q4g_decode_step with the layer-0 input given directly: hidden [h] fp32
 * (device) replaces the scaled embedding row. */
q4g_status q4g_decode_step_hidden(q4g_model* m, q4g_cache* c, const float* hidden, int64_t pos,
                                  float* logits, int32_t* argmax, q4g_stream_t stream);

/* As q4g_decode_step with HOST buffers: token and position by value, argmax and
 * (optionally, logits_host != NULL) the logits copied back to host memory;
 * returns after `stream` has synchronised. */
q4g_status q4g_decode_step_host(q4g_model* m, q4g_cache* c, int32_t token, int64_t pos,
                                float* logits_host, int32_t* argmax_host, q4g_stream_t stream);

/* Speculative verify of K rows ids[0..K-1] (device) at positions pos0..pos0+K-1
 * in ONE pass ("Gemma-4-12B-CoreAI", v5 section). Row i attends exactly what a
 * decode step at pos0+i after rows 0..i-1 would attend. All K rows are written
 * to the cache; because the ring has R >= W + K slots, a row the caller later
 * rejects sits in a slot whose implied position fails the window test for every
 * later query until it is overwritten, so it is never observed. The caller
 * continues from pos0 + n for its accepted count n. `accepted_count` states how
 * many rows the caller commits (0..K); with R >= W + K every value leads to the
 * same observable state, so it is validated and otherwise has no effect.
 * Outputs: logits [K][vocab] fp32 (if != NULL), argmax [K] (if != NULL).
 * Q4G_ERANGE: K < 1, K > 8, K > R - W, pos0 < 0, pos0 + K > capacity,
 * accepted_count outside [0, K]. */
q4g_status q4g_verify_block(q4g_model* m, q4g_cache* c, const int32_t* ids, int32_t K,
                            int64_t pos0, int32_t accepted_count, float* logits, int32_t* argmax,
                            q4g_stream_t stream);

/* Chunked prefill ("Gemma-4-12B-CoreAI", tiered-v3/ section: a last-row-only
 * prefill entry point at S = 64; "gemma-4-E4B-CoreAI", stable/ contract):
 * tokens ids[0..S-1] (device) at positions pos0..pos0+S-1, 1 <= S <= 64, with
 * exactly the result of S decode steps in order (row i attends what a decode
 * step at pos0+i after rows 0..i-1 attends) up to the rounding of the
 * multi-row GEMVs. Runs as passes of up to 4 rows, every row kept; only the
 * last pass runs the head. Outputs the last row's logits [vocab] (if != NULL)
 * and argmax[0] (if != NULL), device. No alignment precondition on pos0: every
 * row is written to its own slot (pos mod R). Q4G_ERANGE: S outside 1..64,
 * pos0 < 0, pos0 + S > capacity. */
q4g_status q4g_prefill_chunk(q4g_model* m, q4g_cache* c, const int32_t* ids, int32_t S, int64_t pos0,
                             float* logits, int32_t* argmax, q4g_stream_t stream);

#ifdef __cplusplus
}
#endif
#endif /* Q4G_H */
