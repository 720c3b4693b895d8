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

// The weights the next GEMV of the step reads first, for an L2 prefetch issued
// by the current kernel once its own loads are in flight: the next GEMV's
// warp w streams units [w * n_units / tw, (w + 1) * n_units / tw) in order, and
// the first `frac` of every such range is prefetched (tw == 0: nothing).
struct NextGemv {
  GemvSeg seg[3];
  int32_t nseg;
  int32_t k;
  int32_t n_units;    // units of unit_rows rows (GeGLU: unit_rows / 2 gate rows with the same up rows)
  int32_t unit_rows;  // 2 or 8
  int32_t geglu;
  int32_t tw;       // warps of the next GEMV's grid
  float frac;
};

struct GemvParams {
  NextGemv next;
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
  int32_t nchunk;       // column-split kernel: 1024-column chunks,
  int32_t groups;       //   consumer groups,
  int32_t stage_rows;   //   rows per stage
  int32_t kc;           // columns per streamed item
  int32_t ns;           // stages per warp
  int32_t stage_bytes;  // codes then scales of one item (2 rows)
  int32_t prefetch_stages;  // column-split kernel: stages issued before the dependency wait (0: all)
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

// Consecutive GEMVs of a decode step (one activation row) in one persistent,
// cooperative launch; phase i + 1 starts once every CTA has finished phase i.
constexpr int kChainMaxPhases = 4;
struct ChainParams {
  GemvParams ph[kChainMaxPhases];
  int32_t n_ph;
  int32_t* done;      // [n_ph] CTAs that finished each phase; zero before the launch
  int32_t* err;       // bounded-wait error word (NULL: the library's)
  uint64_t wait_ns;   // bounded-wait limit (0: 2 s)
  uint64_t* trace;    // optional [kChainTraceSlots] %globaltimer stamps of CTA 0
};
// trace slots of one chain launch: 0 start, 1 after griddepcontrol.wait, then per
// phase i at 2 + 4 i: inputs ready, digits built, last own stage done, producer
// done issuing; 18 end
constexpr int kChainTraceSlots = 32;
constexpr int kGemvTraceSlots = 256;  // one GEMV launch's timeline (GemvParams::trace)
// Plans every phase in place; false if a phase does not fit the chain kernel.
bool plan_chain(ChainParams& c);
cudaError_t launch_gemv_chain(const ChainParams& c, cudaStream_t st, bool pdl);
// Descriptor of GEMV `p` as the next GEMV of a prefetch (tw = 0 if p does not
// take the streamed path).
NextGemv gemv_next_desc(const GemvParams& p, float frac);
// Device address of the library's error word (bit 0: a bounded wait gave up).
int32_t* device_error_word();

// ------------------------------------------------------------ attention ----
struct AttnParams {
  NextGemv next;
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

// ------------------------------------------------- persistent step kernel ----
// One decode step (one activation row) as one cooperative launch: every layer's
// QKV, attention, attention merge, O, gate|up and down, then the head, run as
// phases separated by grid-wide counters, while one producer warp per CTA
// streams the CTA's weights (and K/V rows) of all phases through one ring of
// shared-memory stages without waiting for activations.
struct StepLayer {
  const uint8_t* q[7];   // codes of wq, wk, wv, wo, wgate, wup, wdown (wv NULL on full layers)
  const uint16_t* s[7];  // scales, same order
  const float* norm_in;
  const float* norm_post_attn;
  const float* norm_pre_ffn;
  const float* norm_post_ffn;
  const float* norm_q;
  const float* norm_k;
  float layer_scalar;
  int32_t full;
  int32_t ordinal;  // sliding or full ordinal (cache layer index)
};

struct StepKernelParams {
  const StepLayer* layers;  // device array [n_layers]
  int32_t n_layers, hidden, n_q, ffn, vocab;
  int32_t sl_nkv, sl_hd, gl_nkv, gl_hd, window, ring;
  int64_t capacity;
  int32_t rope_pairs_sl, rope_pairs_gl, v_norm_sliding;
  float eps, softcap;
  // cache storage (q4g_cache_view offsets)
  char* cache;
  size_t ring_k_off, ring_v_off, ring_layer_bytes, glob_k_off, glob_v_off, glob_layer_bytes;
  // tied embedding / head and the final norm
  const uint8_t* emb_q;
  const uint16_t* emb_s;
  const float* norm_final;
  // Activations passed between CTAs as tagged 64-bit words (low half: the value,
  // fp32 or two fp16; high half: the tag of the step and layer that wrote it). A
  // reader polls its words until their tags match, so a phase waits for exactly the
  // data it reads and there is no grid-wide barrier between the phases of a layer.
  uint64_t* r0;    // [hidden] layer-0 input (step init), then residual ping-pong r0 / r1
  uint64_t* r1;
  uint64_t* qkv;   // [qkv rows] raw projections
  uint64_t* attn;  // [n_q * hd / 2] attention output, fp16 pairs
  uint64_t* o;     // [hidden]
  uint64_t* act;   // [ffn / 2] GeGLU output, fp16 pairs
  uint64_t* d;     // [hidden]
  const uint32_t* epoch;  // this step's number (step init), part of every tag
  float* part_ml;   // attention partials: (m, l) per (query head, chunk)
  float* part_acc;  // and the unnormalised output rows per (query head, chunk)
  const float2* rope_sl;  // this step's (cos, sin) per rotating pair
  const float2* rope_gl;
  const int64_t* pos_dev;
  float* logits;       // [vocab] or NULL
  int32_t* argmax_out;
  float* am_val;       // [grid] head candidates
  int32_t* am_idx;
  int32_t* done;       // [step_kernel_phases(n_layers) + 1] phase counters, zero at launch
  int32_t* tickets;    // [n_layers][sl_nkv] attention merge tickets, zero at launch
  float* dump;         // optional [n_layers + 1][hidden] residual stream
  int32_t* err;        // error word (bit 0: a bounded wait gave up)
  uint64_t wait_ns;
  uint64_t* trace;     // optional [step_kernel_trace_slots(n_layers)] %globaltimer stamps of CTA 0
  int32_t stall_test;  // 1: CTA 0's first stage expects 16 bytes that never arrive
  uint32_t poll_ns;    // back-off between two polls of a counter or of tagged words
  int32_t grid_sync;   // 1: every phase also waits for all CTAs to finish the previous one
};
// phases per step: 6 per layer (QKV, attention, merge, O, gate|up, down) + head
int step_kernel_phases(int n_layers);
int step_kernel_trace_slots(int n_layers);
// counters the kernel needs (zeroed before each launch): the phase counters, then
// the attention merge tickets
int step_kernel_counters(int n_layers, int sl_kv_heads);
// floats of part_acc / part_ml the kernel needs on a grid of `grid` CTAs
size_t step_kernel_partial_floats(const StepKernelParams& p, int grid);
size_t step_kernel_ml_floats(const StepKernelParams& p, int grid);
// false (with a reason) if the shapes do not fit the kernel
bool step_kernel_supported(const StepKernelParams& p, char* why, size_t why_len);
cudaError_t launch_step_kernel(const StepKernelParams& p, cudaStream_t st);

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
  uint64_t* r_tagged;       // optional [h]: the layer-0 input as tagged words (step kernel)
  uint32_t* epoch_dev;      // written: epoch
  uint32_t epoch;           // this step's number
};
cudaError_t launch_step_init(const StepParams& p, cudaStream_t st);

int device_sm_count();

// Sets the message q4g_last_error() returns on this thread.
void set_last_error(const char* msg);

}  // namespace q4g
