// Internal host-side interfaces between the translation units of libq4g.
#pragma once

#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace q4g {

// ----------------------------------------------------------------- GEMV ----
struct GemvSeg {
  const uint8_t* qs;
  const uint16_t* sc;
  int32_t rows;
};

enum GemvPro { PRO_X16 = 0, PRO_RESID = 1 };
enum GemvEpi { EPI_STORE = 0, EPI_GEGLU = 1, EPI_HEAD = 2 };

struct GemvParams {
  GemvSeg seg[3];
  const uint16_t* w16;  // fp16 weights [n_rows][k] (launch_gemv_f16 only)
  int32_t nseg;
  int32_t k;        // columns
  int32_t n_rows;   // output rows (STORE / HEAD); the last unit may be partial
  int32_t n_units;  // 16-row units (GEGLU: units of 8 gate + 8 up rows)
  int32_t kr;       // activation rows (<= template KRM)
  int32_t pro, epi;
  // PRO_X16: x [kr][x_stride] fp16
  const __half* x;
  int64_t x_stride;
  // PRO_RESID: r_new = (r_in + rmsnorm(delta) * w_delta) * scale   (delta may be NULL)
  //            x     = fp16(rmsnorm(r_new) * w_x); block 0 stores r_new to r_out
  const float* r_in;
  float* r_out;
  const float* delta;
  const float* w_delta;
  float scale;
  const float* w_x;
  float eps;
  float* dump;  // optional [kr][dump_stride] copy of r_new (block 0)
  int64_t dump_stride;
  // EPI_STORE: y [kr][y_stride]
  float* y;
  int64_t y_stride;
  // EPI_GEGLU: act [kr][act_stride] = fp16(gelu_tanh(gate) * up); seg[0] gate, seg[1] up
  __half* act;
  int64_t act_stride;
  // EPI_HEAD: logits [kr][logits_stride] (optional), softcap, argmax
  float* logits;
  int64_t logits_stride;
  float softcap;
  float* am_val;     // [kMaxRows][grid]
  int32_t* am_idx;   // [kMaxRows][grid]
  int32_t* counter;  // one int, zero between launches
  int32_t* argmax_out;
  // bulk-copy pipeline (set by the launcher)
  int32_t nchunk;       // stage kernel: 32-block column chunks,
  int32_t groups;       //   row groups,
  int32_t stage_rows;   //   rows per stage
  int32_t kc;           // columns per streamed item
  int32_t ns;           // stages per warp
  int32_t stage_bytes;  // codes then scales of one item (2 rows)
  int32_t prefetch_stages;  // stage kernel: stages issued before the dependency wait (0: all)
  int32_t* err;         // error word: bit 0 = a bounded wait gave up
  uint64_t wait_ns;     // limit of one bounded wait
  // optional timeline of CTA 0 (globaltimer ns): [0] entry, [1] after the
  // dependency wait, [2] after the x prologue, [8 + t] stage t issued,
  // [72 + t] stage t ready for its consumers, [136 + t] stage t reduced (t < 64)
  uint64_t* trace;
  uint64_t* trace_ends;  // optional [grid]: when each CTA's reducer finished (stage kernel)
  int32_t stall_test;   // 1: the first stage of the warp that owns unit 0 never completes (tests the timeout path)
};

// GEMV with fp16 weights p.w16 (the fp16 tied head): PRO_RESID or PRO_X16 prologue,
// EPI_HEAD or EPI_STORE epilogue, up to kMaxRows activation rows, k % 256 == 0 and
// k <= 8192, w16 and x 16-byte aligned.
cudaError_t launch_gemv_f16(const GemvParams& p, cudaStream_t st, bool pdl);

// Largest number of activation rows one GEMV launch can stage for k columns.
int gemv_max_rows(int k);
size_t gemv_smem_bytes(int krm, int k);
cudaError_t launch_gemv(const GemvParams& p, cudaStream_t st, bool pdl);
// Q4G_GEMV_* kind; false if out of range
bool set_gemv_kernel_choice(int kind);

constexpr int kGemvTraceSlots = 256;
constexpr int kPrefillChunk = 64;  // rows of one prefill call
constexpr int kPrefillBlock = 4;   // rows per pass inside a prefill call  // one GEMV launch's timeline (GemvParams::trace)
// Device address of the library's error word (bit 0: a bounded wait gave up).
int32_t* device_error_word();

// ------------------------------------------------------------ attention ----
struct AttnParams {
  // queries: either the fused QKV epilogue (qkv != NULL) or ready fp16 q
  const float* qkv;      // [kr][qkv_stride] raw projections (q | k | v)
  int64_t qkv_stride;
  int32_t k_off, v_off;  // column offsets of k and v (v_off < 0: V from raw k, k_eq_v)
  const float* w_q;      // q_norm gains [hd]
  const float* w_k;      // k_norm gains [hd]
  int32_t v_norm;        // scale-free RMSNorm on V
  const float2* rope;    // [kr][rope_pairs] (cos, sin), pairs >= rope_pairs untouched
  int32_t rope_pairs;
  float eps;
  const __half* q16;     // standalone: [kr][n_q][hd] fp16
  // cache
  __half* k_cache;       // ring: [n_kv][R][hd]; linear: [n_kv][cap][hd]
  __half* v_cache;
  // int8 cache (kv8 = 1): codes [n_kv][rows][hd] at k_cache / v_cache (as int8)
  // with one fp32 scale per row, [n_kv][rows] at k_scale / v_scale
  int32_t kv8;
  float* k_scale;
  float* v_scale;
  int64_t cache_rows;    // R (ring) or capacity (linear)
  int32_t ring;          // 1: ring addressing with the implied-position window test
  int64_t window;
  int64_t pos0;
  const int64_t* pos_dev;  // if non-NULL, pos0 is read from here (graph replay)
  int32_t kr;
  int32_t write_kv;      // chunk 0 writes the block rows to the cache
  int32_t n_q, n_kv, hd;
  int32_t n_chunks;
  int32_t m_groups;
  // partials [kr*n_q][n_chunks] of (m, l) and acc [kr*n_q][n_chunks][hd]
  float* part_ml;
  float* part_acc;
  int32_t* counters;     // [n_kv] for the in-kernel combine (ring), zero between launches
  int32_t combine_in_kernel;
  int32_t cluster;       // kAttnCluster: grid y is one cluster, merge through DSMEM (n_chunks == cluster)
  uint64_t* trace;       // optional timeline of the first CTA (ring cluster kernel), %globaltimer ns
  int32_t ring_split;    // ring cluster kernel: 2 = several clusters per KV head, merged through
                         // part_ml / part_acc and counters[n_kv * 4] (zero, left zero)
  __half* out;           // [kr][n_q][hd]
};

constexpr int kAttnCluster = 8;  // CTAs per KV head when the merge runs in a cluster
constexpr int kRingSplitCounters = 64;  // model counters of the two-cluster ring merge (n_kv * kAttnCluster)
size_t attn_smem_bytes(int hd, int m_tiles_per_cta);
size_t attn_partial_floats(int kr, int n_q, int n_chunks, int hd);
cudaError_t launch_attention(const AttnParams& p, cudaStream_t st, bool pdl);
// CUDA-core cluster kernel for ring layers with <= 4 query rows per KV head
// (hd 256): 0 if it does not apply, else the row template it uses
int ring_decode_rows(const AttnParams& p);
cudaError_t launch_attention_ring(const AttnParams& p, cudaStream_t st, bool pdl);
cudaError_t launch_attn_combine(const AttnParams& p, cudaStream_t st, bool pdl);

// Split-KV plan of a standalone flash-decode call (one query row per head) and
// its scratch layout: [256 B of completion counters][(m, l) per query head and
// chunk, rounded up to 256 B][acc per query head, chunk and dim, fp32].
struct FlashPlan {
  int32_t n_chunks, m_groups;
  size_t ml_offset, acc_offset, bytes;
};
constexpr size_t kFlashCounterBytes = 256;
FlashPlan flash_plan(int n_q, int n_kv, int hd, bool ring, int64_t window);
// chunks, row groups and the scratch pointers of p from the plan and the scratch base
void flash_bind(AttnParams& p, const FlashPlan& f, void* scratch);

// --------------------------------------------------------------- misc ----
cudaError_t launch_pack(const float* w, int64_t rows, int64_t k, uint8_t* qs, uint16_t* sc,
                        int32_t* bad_flag, cudaStream_t st);
cudaError_t launch_unpack(const uint8_t* qs, const uint16_t* sc, int64_t rows, int64_t k, float* w,
                          cudaStream_t st);

struct StepParams {
  int32_t kr;
  int64_t pos0;
  const int32_t* ids_dev;   // [kr] token ids on the device (or NULL)
  int32_t ids_host[8];      // used when ids_dev == NULL and hidden == NULL
  const float* hidden;      // [kr][h] replaces the embedding
  const uint8_t* emb_qs;
  const uint16_t* emb_sc;
  const uint16_t* emb_f16;  // fp16 tied table (if non-NULL, instead of the q4_0 one)
  int32_t hidden_size, vocab;
  float embed_scale;
  float* r_out;             // [kr][h]
  float* dump;              // optional [kr][dump_stride]
  int64_t dump_stride;
  // RoPE tables for this step
  const double* inv_freq_sl;  // [pairs_sl]
  const double* inv_freq_gl;  // [pairs_gl]
  int32_t pairs_sl, pairs_gl;
  float2* rope_sl;          // [kr][pairs_sl]
  float2* rope_gl;          // [kr][pairs_gl]
  int64_t* pos_dev;         // written: pos0
  int32_t* counters;        // zeroed
  int32_t n_counters;
};
cudaError_t launch_step_init(const StepParams& p, cudaStream_t st);

int device_sm_count();

// Sets the message q4g_last_error() returns on this thread.
void set_last_error(const char* msg);

}  // namespace q4g
