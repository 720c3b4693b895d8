// C ABI of libq4g: argument validation, model/cache handles, the per-step
// launch sequence and its CUDA-graph replay. See include/q4g.h for the contract.
#include <math.h>
#include <stdarg.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include <algorithm>
#include <mutex>
#include <string>
#include <vector>

#include "../../include/q4g.h"
#include "q4g_common.cuh"
#include "q4g_internal.h"

using namespace q4g;

// ------------------------------------------------------------------ errors --
namespace {
thread_local std::string g_err;

q4g_status fail(q4g_status s, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof buf, fmt, ap);
  va_end(ap);
  g_err = buf;
  return s;
}

q4g_status cuda_fail(cudaError_t e, const char* where) {
  return fail(Q4G_ECUDA, "%s: %s", where, cudaGetErrorString(e));
}

#define CK(expr)                                         \
  do {                                                   \
    cudaError_t e_ = (expr);                             \
    if (e_ != cudaSuccess) return cuda_fail(e_, #expr);  \
  } while (0)

bool aligned(const void* p, size_t a) { return ((uintptr_t)p % a) == 0; }

// qkv column count of a layer type
struct LayerShape {
  int hd, nkv, nq_cols, k_cols, v_cols, qkv_cols, G, rope_pairs;
};
}  // namespace

extern "C" const char* q4g_last_error(void) { return g_err.c_str(); }

void q4g::set_last_error(const char* msg) { g_err = msg ? msg : ""; }

extern "C" const char* q4g_status_string(q4g_status s) {
  switch (s) {
    case Q4G_OK: return "Q4G_OK";
    case Q4G_EINVAL: return "Q4G_EINVAL";
    case Q4G_ERANGE: return "Q4G_ERANGE";
    case Q4G_ENOMEM: return "Q4G_ENOMEM";
    case Q4G_ECUDA: return "Q4G_ECUDA";
    case Q4G_ETIMEOUT: return "Q4G_ETIMEOUT";
  }
  return "unknown";
}

extern "C" int q4g_abi_version(void) { return Q4G_ABI_VERSION; }

// ------------------------------------------------------------- handles ------
struct GraphEntry {
  int kind;  // rows of the step
  const void* cache;
  const void* logits;
  const void* argmax;
  const void* dump;
  cudaGraphExec_t exec;
};

struct q4g_model {
  q4g_config cfg;
  std::vector<q4g_layer_weights> layers;
  std::vector<int> ordinal;  // sliding or full ordinal of each layer
  std::vector<char> full;
  q4g_qtensor embed;
  const uint16_t* embed_f16;  // the fp16 tied table (head_fp16), else NULL
  const float* norm_final;
  int n_sl = 0, n_gl = 0;
  LayerShape sl{}, gl{};
  int sm_count = 0;
  // scratch
  void* scratch = nullptr;
  size_t scratch_bytes = 0;
  float* r[2];
  float* qkv;
  __half* attn;
  float* o;
  __half* act;
  float* d;
  float* logits_buf;
  int32_t* argmax_buf;
  float* am_val;
  int32_t* am_idx;
  int32_t* counters;
  int n_counters = 0;
  float2* rope_sl;
  float2* rope_gl;
  int64_t* pos_dev;
  double* inv_freq_sl;
  double* inv_freq_gl;
  float* part_ml;
  float* part_acc;
  bool use_graph = true, use_pdl = true, attn_cluster = true;
  uint64_t* trace = nullptr;  // Q4G_OPT_TRACE
  float* dump = nullptr;
  // profile mode: events around every launch
  bool profile = false;
  bool stall_next = false;  // test: the next step's first GEMV waits on a stage that never completes
  std::vector<cudaEvent_t> ev_pool;
  struct Rec {
    int kind, layer;
    double bytes;
    cudaEvent_t a, b;
  };
  std::vector<Rec> recs;
  size_t ev_next = 0;
  // graphs
  cudaStream_t cap_stream = nullptr;
  std::vector<GraphEntry> graphs;
  std::mutex mu;
};

struct q4g_cache {
  const q4g_model* m;
  int64_t capacity;
  char* buf;
  q4g_cache_view view;
};

namespace {

int n_chunks_ring(const q4g_model* m, int m_groups) {
  int n = (m->cfg.window + 63) / 64;
  const int cap = (2 * m->sm_count) / (m->cfg.sl_kv_heads * m_groups);
  if (n > cap) n = cap;
  return n < 1 ? 1 : n;
}

int n_chunks_linear(const q4g_model* m, int m_groups) {
  int n = m->sm_count / (m->cfg.gl_kv_heads * m_groups);
  return n < 1 ? 1 : n;
}

int m_groups_for(int kr, int G) { return (kr * G + 31) / 32; }

q4g_status validate_config(const q4g_config* c) {
  if (!c) return fail(Q4G_EINVAL, "config is NULL");
  if (c->n_layers < 1 || c->hidden < 32 || c->hidden % 32 || c->ffn < 32 || c->ffn % 32 ||
      c->vocab < 1 || c->n_q_heads < 1)
    return fail(Q4G_EINVAL, "hidden and ffn must be positive multiples of 32; layers, heads, vocab >= 1");
  if (c->hidden > 8192)
    return fail(Q4G_EINVAL, "hidden must be <= 8192 (the fused residual prologue keeps it in registers)");
  if (c->sl_head_dim != 256 || c->gl_head_dim != 512)
    return fail(Q4G_EINVAL, "head dims must be 256 (sliding) and 512 (full)");
  if (c->sl_kv_heads < 1 || c->gl_kv_heads < 1 || c->n_q_heads % c->sl_kv_heads ||
      c->n_q_heads % c->gl_kv_heads)
    return fail(Q4G_EINVAL, "n_q_heads must be a multiple of both KV head counts");
  if (c->window < 1 || c->ring < c->window + 1 || c->ring > (1 << 30))
    return fail(Q4G_EINVAL, "need window >= 1, window < ring <= 2^30");
  if (c->rope_pairs_full < 0 || c->rope_pairs_full > c->gl_head_dim / 2)
    return fail(Q4G_EINVAL, "rope_pairs_full out of range");
  if (!(c->rope_theta_sl > 0) || !(c->rope_theta_gl > 0) || !(c->rms_eps >= 0) || !(c->softcap > 0) ||
      !isfinite(c->embed_scale))
    return fail(Q4G_EINVAL, "bad rope theta / eps / softcap / embed_scale");
  if (c->full_every < 0 || (c->full_every > 0 && (c->full_offset < 0 || c->full_offset >= c->full_every)))
    return fail(Q4G_EINVAL, "bad full_every / full_offset");
  if (c->head_fp16 != 0 && c->head_fp16 != 1) return fail(Q4G_EINVAL, "head_fp16 must be 0 or 1");
  if (c->kv_int8 != 0 && c->kv_int8 != 1) return fail(Q4G_EINVAL, "kv_int8 must be 0 or 1");
  return Q4G_OK;
}

q4g_status check_q(const q4g_qtensor& t, const char* name) {
  if (!t.qs || !t.scales) return fail(Q4G_EINVAL, "%s: NULL pointer", name);
  if (!aligned(t.qs, 16) || !aligned(t.scales, 2)) return fail(Q4G_EINVAL, "%s: misaligned", name);
  return Q4G_OK;
}

void free_graphs(q4g_model* m) {
  for (auto& g : m->graphs) cudaGraphExecDestroy(g.exec);
  m->graphs.clear();
}

}  // namespace

extern "C" q4g_status q4g_model_create(const q4g_config* cfg, const q4g_weights* w, q4g_model** out) {
  if (!out) return fail(Q4G_EINVAL, "out is NULL");
  *out = nullptr;
  q4g_status st = validate_config(cfg);
  if (st) return st;
  if (!w || !w->layers || !w->norm_final) return fail(Q4G_EINVAL, "weights are NULL");
  if (cfg->head_fp16) {
    if (!w->embed_f16 || !aligned(w->embed_f16, 16)) return fail(Q4G_EINVAL, "embed_f16: NULL or not 16-byte aligned");
  } else if ((st = check_q(w->embed, "embed"))) {
    return st;
  }
  const q4g_config& c = *cfg;
  q4g_model* m = new (std::nothrow) q4g_model();
  if (!m) return fail(Q4G_ENOMEM, "model handle");
  m->cfg = c;
  m->embed = w->embed;
  m->embed_f16 = c.head_fp16 ? w->embed_f16 : nullptr;
  m->norm_final = w->norm_final;
  for (int l = 0; l < c.n_layers; ++l) {
    const q4g_layer_weights& L = w->layers[l];
    const bool full = c.full_every > 0 && l % c.full_every == c.full_offset;
    char name[64];
    const q4g_qtensor* ts[7] = {&L.wq, &L.wk, &L.wv, &L.wo, &L.wgate, &L.wup, &L.wdown};
    const char* tn[7] = {"wq", "wk", "wv", "wo", "wgate", "wup", "wdown"};
    for (int t = 0; t < 7; ++t) {
      if (t == 2 && full) continue;
      snprintf(name, sizeof name, "layer %d %s", l, tn[t]);
      if ((st = check_q(*ts[t], name))) {
        delete m;
        return st;
      }
    }
    if (!L.norm_in || !L.norm_post_attn || !L.norm_pre_ffn || !L.norm_post_ffn || !L.norm_q || !L.norm_k ||
        !isfinite(L.layer_scalar)) {
      delete m;
      return fail(Q4G_EINVAL, "layer %d: NULL norm gain or bad layer_scalar", l);
    }
    m->layers.push_back(L);
    m->full.push_back(full);
    m->ordinal.push_back(full ? m->n_gl++ : m->n_sl++);
  }
  auto shape = [&](bool full) {
    LayerShape s{};
    s.hd = full ? c.gl_head_dim : c.sl_head_dim;
    s.nkv = full ? c.gl_kv_heads : c.sl_kv_heads;
    s.nq_cols = c.n_q_heads * s.hd;
    s.k_cols = s.nkv * s.hd;
    s.v_cols = full ? 0 : s.nkv * s.hd;
    s.qkv_cols = s.nq_cols + s.k_cols + s.v_cols;
    s.G = c.n_q_heads / s.nkv;
    s.rope_pairs = full ? c.rope_pairs_full : s.hd / 2;
    return s;
  };
  m->sl = shape(false);
  m->gl = shape(true);
  m->sm_count = device_sm_count();

  // ---- scratch layout ----
  const int R = kMaxRows, H = c.hidden;
  const int qkv_max = m->sl.qkv_cols > m->gl.qkv_cols ? m->sl.qkv_cols : m->gl.qkv_cols;
  const int attn_max = c.n_q_heads * c.gl_head_dim;
  size_t part = 0;
  for (int kr = 1; kr <= R; ++kr) {
    const int mgs = m_groups_for(kr, m->sl.G), mgg = m_groups_for(kr, m->gl.G);
    size_t a = attn_partial_floats(kr, c.n_q_heads, n_chunks_ring(m, mgs), c.sl_head_dim);
    size_t b = attn_partial_floats(kr, c.n_q_heads, n_chunks_linear(m, mgg), c.gl_head_dim);
    part = a > part ? a : part;
    part = b > part ? b : part;
  }
  const size_t part_ml = part / 128 + 1024;  // (m, l) per row and chunk: hd >= 256
  // head, attention, then the two-cluster ring attention merge
  m->n_counters = 64 + kRingSplitCounters;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    size_t o = off;
    off += (bytes + 255) & ~(size_t)255;
    return o;
  };
  const size_t o_r0 = take(sizeof(float) * R * H), o_r1 = take(sizeof(float) * R * H);
  const size_t o_qkv = take(sizeof(float) * R * qkv_max);
  const size_t o_attn = take(sizeof(__half) * R * attn_max);
  const size_t o_o = take(sizeof(float) * R * H);
  const size_t o_act = take(sizeof(__half) * R * c.ffn);
  const size_t o_d = take(sizeof(float) * R * H);
  const size_t o_logits = take(sizeof(float) * R * (size_t)c.vocab);
  const size_t o_am = take(sizeof(int32_t) * R);
  const size_t o_amv = take(sizeof(float) * R * 2 * m->sm_count);
  const size_t o_ami = take(sizeof(int32_t) * R * 2 * m->sm_count);
  const size_t o_cnt = take(sizeof(int32_t) * m->n_counters);
  const size_t o_rs = take(sizeof(float2) * R * m->sl.rope_pairs);
  const size_t o_rg = take(sizeof(float2) * R * (m->gl.rope_pairs > 0 ? m->gl.rope_pairs : 1));
  const size_t o_pos = take(sizeof(int64_t));
  const size_t o_ifs = take(sizeof(double) * m->sl.rope_pairs);
  const size_t o_ifg = take(sizeof(double) * (m->gl.rope_pairs > 0 ? m->gl.rope_pairs : 1));
  const size_t o_pml = take(sizeof(float) * 2 * part_ml);
  const size_t o_pacc = take(sizeof(float) * part);
  m->scratch_bytes = off;
  cudaError_t e = cudaMalloc(&m->scratch, off);
  if (e != cudaSuccess) {
    delete m;
    return fail(Q4G_ENOMEM, "scratch (%zu bytes): %s", off, cudaGetErrorString(e));
  }
  char* b = (char*)m->scratch;
  m->r[0] = (float*)(b + o_r0);
  m->r[1] = (float*)(b + o_r1);
  m->qkv = (float*)(b + o_qkv);
  m->attn = (__half*)(b + o_attn);
  m->o = (float*)(b + o_o);
  m->act = (__half*)(b + o_act);
  m->d = (float*)(b + o_d);
  m->logits_buf = (float*)(b + o_logits);
  m->argmax_buf = (int32_t*)(b + o_am);
  m->am_val = (float*)(b + o_amv);
  m->am_idx = (int32_t*)(b + o_ami);
  m->counters = (int32_t*)(b + o_cnt);
  m->rope_sl = (float2*)(b + o_rs);
  m->rope_gl = (float2*)(b + o_rg);
  m->pos_dev = (int64_t*)(b + o_pos);
  m->inv_freq_sl = (double*)(b + o_ifs);
  m->inv_freq_gl = (double*)(b + o_ifg);
  m->part_ml = (float*)(b + o_pml);
  m->part_acc = (float*)(b + o_pacc);
  e = cudaMemset(m->scratch, 0, off);
  // RoPE inverse frequencies theta^(-2i/hd), in fp64 ("Gemma 4 12B" architecture:
  // dual RoPE; the full layers' frequencies are those of head dim 512, first pairs only)
  std::vector<double> fs(m->sl.rope_pairs), fg(m->gl.rope_pairs > 0 ? m->gl.rope_pairs : 1, 0.0);
  for (int i = 0; i < m->sl.rope_pairs; ++i) fs[i] = pow((double)c.rope_theta_sl, -2.0 * i / c.sl_head_dim);
  for (int i = 0; i < m->gl.rope_pairs; ++i) fg[i] = pow((double)c.rope_theta_gl, -2.0 * i / c.gl_head_dim);
  if (e == cudaSuccess) e = cudaMemcpy(m->inv_freq_sl, fs.data(), sizeof(double) * fs.size(), cudaMemcpyHostToDevice);
  if (e == cudaSuccess) e = cudaMemcpy(m->inv_freq_gl, fg.data(), sizeof(double) * fg.size(), cudaMemcpyHostToDevice);
  if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&m->cap_stream, cudaStreamNonBlocking);
  if (e != cudaSuccess) {
    cudaFree(m->scratch);
    delete m;
    return cuda_fail(e, "model_create");
  }
  *out = m;
  return Q4G_OK;
}

extern "C" void q4g_model_destroy(q4g_model* m) {
  if (!m) return;
  free_graphs(m);
  for (cudaEvent_t e : m->ev_pool) cudaEventDestroy(e);
  if (m->cap_stream) cudaStreamDestroy(m->cap_stream);
  cudaFree(m->scratch);
  delete m;
}

extern "C" q4g_status q4g_model_check(q4g_model* m, q4g_stream_t stream) {
  if (!m) return fail(Q4G_EINVAL, "model is NULL");
  CK(cudaStreamSynchronize((cudaStream_t)stream));
  CK(cudaGetLastError());
  int32_t* ew = device_error_word();
  if (!ew) return fail(Q4G_ECUDA, "error word unavailable");
  int32_t word = 0;
  CK(cudaMemcpy(&word, ew, sizeof word, cudaMemcpyDeviceToHost));
  if (word) {
    const int32_t zero = 0;
    CK(cudaMemcpy(ew, &zero, sizeof zero, cudaMemcpyHostToDevice));
    return fail(Q4G_ETIMEOUT, "a bounded device wait gave up (error word 0x%x); results of that step are unspecified",
                word);
  }
  return Q4G_OK;
}

extern "C" q4g_status q4g_model_set_option(q4g_model* m, q4g_option opt, intptr_t value) {
  if (!m) return fail(Q4G_EINVAL, "model is NULL");
  std::lock_guard<std::mutex> lk(m->mu);
  switch (opt) {
    case Q4G_OPT_CUDA_GRAPH: m->use_graph = value != 0; break;
    case Q4G_OPT_PDL: m->use_pdl = value != 0; break;
    case Q4G_OPT_DUMP: m->dump = (float*)value; break;
    case Q4G_OPT_PROFILE: m->profile = value != 0; break;
    case Q4G_OPT_TEST_STALL: m->stall_next = value != 0; break;
    case Q4G_OPT_ATTN_CLUSTER: m->attn_cluster = value != 0; break;
    case Q4G_OPT_TRACE: m->trace = (uint64_t*)value; break;
    default: return fail(Q4G_EINVAL, "unknown option %d", (int)opt);
  }
  free_graphs(m);
  return Q4G_OK;
}

// --------------------------------------------------------------- cache ------
namespace {
size_t up256(size_t x) { return (x + 255) & ~(size_t)255; }
// One layer's K (or V) region: fp16 rows, or int8 codes then the fp32 row scales.
size_t kv_region_bytes(bool kv8, size_t rows, size_t hd, size_t* scale_offset) {
  if (!kv8) {
    if (scale_offset) *scale_offset = 0;
    return up256(rows * hd * 2);
  }
  const size_t so = up256(rows * hd);
  if (scale_offset) *scale_offset = so;
  return up256(so + rows * sizeof(float));
}
}  // namespace

extern "C" q4g_status q4g_cache_bytes(const q4g_model* m, int64_t capacity, size_t* bytes) {
  if (!m || !bytes) return fail(Q4G_EINVAL, "NULL argument");
  if (capacity < 1 || capacity > (int64_t)1 << 30) return fail(Q4G_ERANGE, "capacity must be in [1, 2^30]");
  const q4g_config& c = m->cfg;
  const size_t ring = kv_region_bytes(c.kv_int8, (size_t)c.sl_kv_heads * c.ring, c.sl_head_dim, nullptr);
  const size_t glob = kv_region_bytes(c.kv_int8, (size_t)c.gl_kv_heads * capacity, c.gl_head_dim, nullptr);
  *bytes = 2 * ring * m->n_sl + 2 * glob * m->n_gl;
  return Q4G_OK;
}

extern "C" q4g_status q4g_cache_init(const q4g_model* m, int64_t capacity, void* dev_buf, size_t bytes,
                                     q4g_cache** out) {
  if (!out) return fail(Q4G_EINVAL, "out is NULL");
  *out = nullptr;
  size_t need = 0;
  q4g_status st = q4g_cache_bytes(m, capacity, &need);
  if (st) return st;
  if (!dev_buf || !aligned(dev_buf, 256)) return fail(Q4G_EINVAL, "cache buffer NULL or not 256-byte aligned");
  if (bytes < need) return fail(Q4G_EINVAL, "cache buffer too small: %zu < %zu", bytes, need);
  q4g_cache* c = new (std::nothrow) q4g_cache();
  if (!c) return fail(Q4G_ENOMEM, "cache handle");
  const q4g_config& cf = m->cfg;
  c->m = m;
  c->capacity = capacity;
  c->buf = (char*)dev_buf;
  q4g_cache_view& v = c->view;
  v.capacity = capacity;
  v.ring = cf.ring;
  v.n_sliding = m->n_sl;
  v.n_full = m->n_gl;
  v.sl_kv_heads = cf.sl_kv_heads;
  v.sl_head_dim = cf.sl_head_dim;
  v.gl_kv_heads = cf.gl_kv_heads;
  v.gl_head_dim = cf.gl_head_dim;
  v.kv_int8 = cf.kv_int8;
  v.ring_layer_bytes = kv_region_bytes(cf.kv_int8, (size_t)cf.sl_kv_heads * cf.ring, cf.sl_head_dim,
                                       &v.ring_scale_offset);
  v.global_layer_bytes = kv_region_bytes(cf.kv_int8, (size_t)cf.gl_kv_heads * capacity, cf.gl_head_dim,
                                         &v.global_scale_offset);
  v.ring_k_offset = 0;
  v.ring_v_offset = v.ring_layer_bytes * m->n_sl;
  v.global_k_offset = 2 * v.ring_layer_bytes * m->n_sl;
  v.global_v_offset = v.global_k_offset + v.global_layer_bytes * m->n_gl;
  v.total_bytes = need;
  *out = c;
  return Q4G_OK;
}

extern "C" q4g_status q4g_cache_reset(q4g_cache* c, q4g_stream_t stream) {
  if (!c) return fail(Q4G_EINVAL, "cache is NULL");
  CK(cudaMemsetAsync(c->buf, 0, c->view.total_bytes, (cudaStream_t)stream));
  return Q4G_OK;
}

extern "C" void q4g_cache_destroy(q4g_cache* c) { delete c; }

extern "C" q4g_status q4g_cache_layout(const q4g_cache* c, q4g_cache_view* out) {
  if (!c || !out) return fail(Q4G_EINVAL, "NULL argument");
  *out = c->view;
  return Q4G_OK;
}

// ---------------------------------------------------------- standalone ------
extern "C" q4g_status q4g_q4_0_pack(const float* w, int64_t rows, int64_t k, uint8_t* qs, uint16_t* scales,
                                    int on_device, q4g_stream_t stream) {
  if (rows < 0 || k <= 0 || k % 32) return fail(Q4G_EINVAL, "need rows >= 0 and k a positive multiple of 32");
  if (rows == 0) return Q4G_OK;
  if (!w || !qs || !scales) return fail(Q4G_EINVAL, "NULL pointer");
  cudaStream_t st = (cudaStream_t)stream;
  const size_t nw = (size_t)rows * k, nq = nw / 2, ns = nw / 32;
  const float* dw = w;
  uint8_t* dq = qs;
  uint16_t* ds = scales;
  void* tmp = nullptr;
  int32_t* flag = nullptr;
  // staging for host pointers, plus the device flag for non-finite input
  size_t tbytes = 256 + (on_device ? 0 : ((nw * 4 + 255) & ~255ul) + ((nq + 255) & ~255ul) + ns * 2);
  CK(cudaMallocAsync(&tmp, tbytes, st));
  flag = (int32_t*)tmp;
  if (!on_device) {
    char* t = (char*)tmp + 256;
    dw = (const float*)t;
    dq = (uint8_t*)(t + ((nw * 4 + 255) & ~255ul));
    ds = (uint16_t*)(t + ((nw * 4 + 255) & ~255ul) + ((nq + 255) & ~255ul));
    CK(cudaMemcpyAsync((void*)dw, w, nw * 4, cudaMemcpyHostToDevice, st));
  }
  CK(cudaMemsetAsync(flag, 0, 4, st));
  CK(launch_pack(dw, rows, k, dq, ds, flag, st));
  int32_t bad = 0;
  CK(cudaMemcpyAsync(&bad, flag, 4, cudaMemcpyDeviceToHost, st));
  if (!on_device) {
    CK(cudaMemcpyAsync(qs, dq, nq, cudaMemcpyDeviceToHost, st));
    CK(cudaMemcpyAsync(scales, ds, ns * 2, cudaMemcpyDeviceToHost, st));
  }
  CK(cudaFreeAsync(tmp, st));
  CK(cudaStreamSynchronize(st));
  if (bad) return fail(Q4G_EINVAL, "q4_0 pack: input contains NaN or infinity");
  return Q4G_OK;
}

extern "C" q4g_status q4g_q4_0_unpack(const uint8_t* qs, const uint16_t* scales, int64_t rows, int64_t k,
                                      float* w, int on_device, q4g_stream_t stream) {
  if (rows < 0 || k <= 0 || k % 32) return fail(Q4G_EINVAL, "need rows >= 0 and k a positive multiple of 32");
  if (rows == 0) return Q4G_OK;
  if (!w || !qs || !scales) return fail(Q4G_EINVAL, "NULL pointer");
  cudaStream_t st = (cudaStream_t)stream;
  if (on_device) {
    CK(launch_unpack(qs, scales, rows, k, w, st));
    return Q4G_OK;
  }
  const size_t nw = (size_t)rows * k, nq = nw / 2, ns = nw / 32;
  void* tmp = nullptr;
  const size_t a = (nw * 4 + 255) & ~255ul, bq = (nq + 255) & ~255ul;
  CK(cudaMallocAsync(&tmp, a + bq + ns * 2, st));
  float* dw = (float*)tmp;
  uint8_t* dq = (uint8_t*)tmp + a;
  uint16_t* ds = (uint16_t*)((char*)tmp + a + bq);
  CK(cudaMemcpyAsync(dq, qs, nq, cudaMemcpyHostToDevice, st));
  CK(cudaMemcpyAsync(ds, scales, ns * 2, cudaMemcpyHostToDevice, st));
  CK(launch_unpack(dq, ds, rows, k, dw, st));
  CK(cudaMemcpyAsync(w, dw, nw * 4, cudaMemcpyDeviceToHost, st));
  CK(cudaFreeAsync(tmp, st));
  CK(cudaStreamSynchronize(st));
  return Q4G_OK;
}

extern "C" q4g_status q4g_set_gemv_kernel(int32_t kind) {
  if (!set_gemv_kernel_choice(kind)) return fail(Q4G_EINVAL, "GEMV kernel kind must be 0..4");
  return Q4G_OK;
}

extern "C" q4g_status q4g_gemv(const uint8_t* qs, const uint16_t* scales, int64_t n, int64_t k,
                               const uint16_t* x_f16, int32_t nrhs, float* y, q4g_stream_t stream) {
  if (n < 0 || k <= 0 || k % 32 || n > INT32_MAX || k > (1 << 20))
    return fail(Q4G_EINVAL, "need n >= 0 and k a positive multiple of 32");
  if (nrhs < 1 || nrhs > kMaxRows) return fail(Q4G_EINVAL, "nrhs must be 1..8");
  if (n == 0) return Q4G_OK;
  if (!qs || !scales || !x_f16 || !y) return fail(Q4G_EINVAL, "NULL pointer");
  if (!aligned(qs, 16) || !aligned(scales, 2) || !aligned(x_f16, 16) || !aligned(y, 4))
    return fail(Q4G_EINVAL, "misaligned pointer");
  const int maxr = gemv_max_rows((int)k);
  for (int r0 = 0; r0 < nrhs; r0 += maxr) {
    GemvParams p{};
    p.seg[0] = {qs, scales, (int32_t)n};
    p.nseg = 1;
    p.k = (int)k;
    p.n_rows = (int)n;
    p.n_units = (int)((n + 15) / 16);
    p.kr = nrhs - r0 < maxr ? nrhs - r0 : maxr;
    p.pro = PRO_X16;
    p.epi = EPI_STORE;
    p.x = reinterpret_cast<const __half*>(x_f16) + (size_t)r0 * k;
    p.x_stride = k;
    p.y = y + (size_t)r0 * n;
    p.y_stride = n;
    CK(launch_gemv(p, (cudaStream_t)stream, false));
  }
  return Q4G_OK;
}

extern "C" q4g_status q4g_gemv_f16(const uint16_t* w16, int64_t n, int64_t k, const uint16_t* x_f16, int32_t nrhs,
                                   float* y, q4g_stream_t stream) {
  if (n < 0 || n > INT32_MAX || k <= 0 || k % 256 || k > 8192)
    return fail(Q4G_EINVAL, "need n >= 0 and k a positive multiple of 256, at most 8192");
  if (nrhs < 1 || nrhs > kMaxRows) return fail(Q4G_EINVAL, "nrhs must be 1..8");
  if (n == 0) return Q4G_OK;
  if (!w16 || !x_f16 || !y) return fail(Q4G_EINVAL, "NULL pointer");
  if (!aligned(w16, 16) || !aligned(x_f16, 16) || !aligned(y, 4)) return fail(Q4G_EINVAL, "misaligned pointer");
  GemvParams p{};
  p.w16 = w16;
  p.k = (int)k;
  p.n_rows = (int)n;
  p.kr = nrhs;
  p.pro = PRO_X16;
  p.epi = EPI_STORE;
  p.x = reinterpret_cast<const __half*>(x_f16);
  p.x_stride = k;
  p.y = y;
  p.y_stride = n;
  CK(launch_gemv_f16(p, (cudaStream_t)stream, false));
  return Q4G_OK;
}

extern "C" size_t q4g_flash_decode_workspace_bytes(int32_t n_q_heads, int32_t head_dim) {
  if (n_q_heads < 1 || head_dim < 1) return 256;
  // the largest plan: at most 2 chunks per SM
  const int chunks = 2 * device_sm_count();
  return kFlashCounterBytes + ((sizeof(float) * 2 * (size_t)n_q_heads * chunks + 255) & ~255ul) +
         sizeof(float) * (size_t)n_q_heads * chunks * head_dim;
}

namespace {
q4g_status flash_standalone(const uint16_t* q, int32_t n_q, int32_t n_kv, int32_t hd, const void* kc,
                            const void* vc, const float* ks, const float* vs, int64_t rows, bool ring,
                            int64_t window, int64_t pos, uint16_t* out, void* ws, size_t ws_bytes,
                            cudaStream_t st) {
  if (!q || !kc || !vc || !out || !ws) return fail(Q4G_EINVAL, "NULL pointer");
  const bool kv8 = ks != nullptr || vs != nullptr;
  if (kv8 && (!ks || !vs || !aligned(ks, 4) || !aligned(vs, 4))) return fail(Q4G_EINVAL, "scales NULL or misaligned");
  if (hd != 256 && hd != 512) return fail(Q4G_EINVAL, "head_dim must be 256 or 512");
  if (n_q < 1 || n_kv < 1 || n_q % n_kv) return fail(Q4G_EINVAL, "n_q must be a positive multiple of n_kv");
  if (!aligned(q, 16) || !aligned(kc, 16) || !aligned(vc, 16) || !aligned(out, 16) || !aligned(ws, 256))
    return fail(Q4G_EINVAL, "misaligned pointer");
  if (ws_bytes < q4g_flash_decode_workspace_bytes(n_q, hd)) return fail(Q4G_EINVAL, "workspace too small");
  AttnParams p{};
  p.q16 = reinterpret_cast<const __half*>(q);
  p.k_cache = reinterpret_cast<__half*>(const_cast<void*>(kc));
  p.v_cache = reinterpret_cast<__half*>(const_cast<void*>(vc));
  p.kv8 = kv8;
  p.k_scale = const_cast<float*>(ks);
  p.v_scale = const_cast<float*>(vs);
  p.cache_rows = rows;
  p.ring = ring;
  p.window = window;
  p.pos0 = pos;
  p.kr = 1;
  p.n_q = n_q;
  p.n_kv = n_kv;
  p.hd = hd;
  const FlashPlan plan = flash_plan(n_q, n_kv, hd, ring, window);
  if (plan.bytes > ws_bytes) return fail(Q4G_EINVAL, "workspace too small");
  flash_bind(p, plan, ws);
  p.combine_in_kernel = ring ? 1 : 0;
  p.out = reinterpret_cast<__half*>(out);
  if (ring) {
    AttnParams pc = p;
    pc.cluster = kAttnCluster;
    pc.n_chunks = kAttnCluster;
    if (ring_decode_rows(pc) > 0) {  // few rows per KV head: cluster kernel, no workspace use
      CK(launch_attention(pc, st, false));
      return Q4G_OK;
    }
  }
  if (p.n_kv * p.m_groups > 64) return fail(Q4G_EINVAL, "too many KV heads");
  CK(cudaMemsetAsync(p.counters, 0, 256, st));
  CK(launch_attention(p, st, false));
  if (!ring) CK(launch_attn_combine(p, st, false));
  return Q4G_OK;
}
}  // namespace

extern "C" q4g_status q4g_flash_decode_ring(const uint16_t* q, int32_t n_q, int32_t n_kv, int32_t head_dim,
                                            const uint16_t* k_ring, const uint16_t* v_ring, int64_t ring,
                                            int64_t window, int64_t pos, uint16_t* out, void* workspace,
                                            size_t workspace_bytes, q4g_stream_t stream) {
  if (ring < 1 || window < 1 || window > ring) return fail(Q4G_EINVAL, "need 1 <= window <= ring");
  if (ring > ((int64_t)1 << 30)) return fail(Q4G_ERANGE, "ring > 2^30");
  if (pos < 0) return fail(Q4G_ERANGE, "pos < 0");
  return flash_standalone(q, n_q, n_kv, head_dim, k_ring, v_ring, nullptr, nullptr, ring, true, window, pos, out,
                          workspace, workspace_bytes, (cudaStream_t)stream);
}

extern "C" q4g_status q4g_flash_decode_ring_i8(const uint16_t* q, int32_t n_q, int32_t n_kv, int32_t head_dim,
                                               const int8_t* k_codes, const float* k_scales, const int8_t* v_codes,
                                               const float* v_scales, int64_t ring, int64_t window, int64_t pos,
                                               uint16_t* out, void* workspace, size_t workspace_bytes,
                                               q4g_stream_t stream) {
  if (ring < 1 || window < 1 || window > ring) return fail(Q4G_EINVAL, "need 1 <= window <= ring");
  if (ring > ((int64_t)1 << 30)) return fail(Q4G_ERANGE, "ring > 2^30");
  if (pos < 0) return fail(Q4G_ERANGE, "pos < 0");
  if (!k_scales || !v_scales) return fail(Q4G_EINVAL, "NULL pointer");
  return flash_standalone(q, n_q, n_kv, head_dim, k_codes, v_codes, k_scales, v_scales, ring, true, window, pos,
                          out, workspace, workspace_bytes, (cudaStream_t)stream);
}

extern "C" q4g_status q4g_flash_decode_linear(const uint16_t* q, int32_t n_q, int32_t n_kv, int32_t head_dim,
                                              const uint16_t* k, const uint16_t* v, int64_t len, uint16_t* out,
                                              void* workspace, size_t workspace_bytes, q4g_stream_t stream) {
  if (len < 1 || len > ((int64_t)1 << 30)) return fail(Q4G_ERANGE, "len must be in [1, 2^30]");
  // linear cache [len][n_kv][hd] is addressed as [n_kv][rows][hd] with rows = len only when n_kv == 1
  if (n_kv != 1) return fail(Q4G_EINVAL, "the linear entry point takes one KV head ([len][hd] cache)");
  return flash_standalone(q, n_q, n_kv, head_dim, k, v, nullptr, nullptr, len, false, 0, len - 1, out, workspace,
                          workspace_bytes, (cudaStream_t)stream);
}

extern "C" q4g_status q4g_flash_decode_linear_i8(const uint16_t* q, int32_t n_q, int32_t n_kv, int32_t head_dim,
                                                 const int8_t* k_codes, const float* k_scales,
                                                 const int8_t* v_codes, const float* v_scales, int64_t len,
                                                 uint16_t* out, void* workspace, size_t workspace_bytes,
                                                 q4g_stream_t stream) {
  if (len < 1 || len > ((int64_t)1 << 30)) return fail(Q4G_ERANGE, "len must be in [1, 2^30]");
  if (n_kv != 1) return fail(Q4G_EINVAL, "the linear entry point takes one KV head ([len][hd] cache)");
  if (!k_scales || !v_scales) return fail(Q4G_EINVAL, "NULL pointer");
  return flash_standalone(q, n_q, n_kv, head_dim, k_codes, v_codes, k_scales, v_scales, len, false, 0, len - 1, out,
                          workspace, workspace_bytes, (cudaStream_t)stream);
}

// --------------------------------------------------------------- decode -----
namespace {

char* ring_reg(const q4g_cache* c, int i, int kv) {
  return c->buf + (kv ? c->view.ring_v_offset : c->view.ring_k_offset) + i * c->view.ring_layer_bytes;
}
char* glob_reg(const q4g_cache* c, int i, int kv) {
  return c->buf + (kv ? c->view.global_v_offset : c->view.global_k_offset) + i * c->view.global_layer_bytes;
}
// Cache rows of one layer into p (fp16 values, or int8 codes and their scales).
void bind_cache(AttnParams& p, const q4g_cache* c, bool full, int ord) {
  char* k = full ? glob_reg(c, ord, 0) : ring_reg(c, ord, 0);
  char* v = full ? glob_reg(c, ord, 1) : ring_reg(c, ord, 1);
  p.k_cache = (__half*)k;
  p.v_cache = (__half*)v;
  p.kv8 = c->view.kv_int8;
  if (p.kv8) {
    const size_t so = full ? c->view.global_scale_offset : c->view.ring_scale_offset;
    p.k_scale = (float*)(k + so);
    p.v_scale = (float*)(v + so);
  }
}

// Profile mode: an event before and after each launch on the launching stream.
cudaEvent_t next_event(q4g_model* m) {
  if (m->ev_next == m->ev_pool.size()) {
    cudaEvent_t e;
    if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
    m->ev_pool.push_back(e);
  }
  return m->ev_pool[m->ev_next++];
}

struct Prof {
  q4g_model* m;
  cudaStream_t st;
  cudaEvent_t a = nullptr;
  Prof(q4g_model* m_, cudaStream_t s) : m(m_), st(s) {
    if (m->profile && (a = next_event(m))) cudaEventRecord(a, st);
  }
  cudaError_t done(cudaError_t e, int kind, int layer, double bytes) {
    if (!a || e != cudaSuccess) return e;
    cudaEvent_t b = next_event(m);
    if (!b) return e;
    cudaEventRecord(b, st);
    m->recs.push_back({kind, layer, bytes, a, b});
    return e;
  }
};

double gemv_bytes(int64_t rows, int64_t k, int kr, int out_bytes) {
  return (double)rows * k * 0.5625 + (double)kr * k * 2 + (double)kr * rows * out_bytes;
}

// Q4G_DEBUG_SYNC=1 (eager mode only): synchronise and report after every launch.
cudaError_t debug_sync(cudaError_t e, const char* what, int layer, cudaStream_t st) {
  static const bool on = getenv("Q4G_DEBUG_SYNC") != nullptr;
  if (e != cudaSuccess || !on) return e;
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  cudaStreamIsCapturing(st, &cs);
  if (cs != cudaStreamCaptureStatusNone) return e;
  fprintf(stderr, "[q4g] layer %d %s ...", layer, what);
  e = cudaStreamSynchronize(st);
  fprintf(stderr, " %s\n", cudaGetErrorString(e));
  return e;
}

// All kernels of one step after step_init (the part that is captured in a graph).
cudaError_t enqueue_body(q4g_model* m, const q4g_cache* c, int kr, int64_t pos0, float* logits,
                         int32_t* argmax, cudaStream_t st) {
  const q4g_config& cf = m->cfg;
  const int H = cf.hidden, L = cf.n_layers;
  const bool pdl = m->use_pdl;
  const int64_t dstride = (int64_t)(L + 1) * H;
  cudaError_t e;
  float* rA = m->r[0];
  float* rB = m->r[1];

  // (a2, a3) pre-attention norm (+ previous layer's post-FFN residual) and QKV
  auto qkv_params = [&](int l) {
    const q4g_layer_weights& W = m->layers[l];
    const bool full = m->full[l];
    const LayerShape& S = full ? m->gl : m->sl;
    GemvParams p{};
    p.seg[0] = {W.wq.qs, W.wq.scales, S.nq_cols};
    p.seg[1] = {W.wk.qs, W.wk.scales, S.k_cols};
    p.nseg = 2;
    if (!full) p.seg[2] = {W.wv.qs, W.wv.scales, S.v_cols}, p.nseg = 3;
    p.k = H;
    p.n_rows = S.qkv_cols;
    p.n_units = S.qkv_cols / 16;
    p.kr = kr;
    p.pro = PRO_RESID;
    p.r_in = rA;
    p.r_out = rB;
    if (l > 0) {
      p.delta = m->d;
      p.w_delta = m->layers[l - 1].norm_post_ffn;
      p.scale = m->layers[l - 1].layer_scalar;
    } else {
      p.scale = 1.0f;
    }
    p.w_x = W.norm_in;
    p.eps = cf.rms_eps;
    p.dump = m->dump ? m->dump + (size_t)l * H : nullptr;
    p.dump_stride = dstride;
    p.epi = EPI_STORE;
    p.y = m->qkv;
    p.y_stride = S.qkv_cols;
    return p;
  };
  // (a7) output projection, activation rows [r0, r0 + maxr)
  auto o_params = [&](int l, int r0) {
    const q4g_layer_weights& W = m->layers[l];
    const LayerShape& S = m->full[l] ? m->gl : m->sl;
    const int kin = cf.n_q_heads * S.hd;
    const int maxr = gemv_max_rows(kin);
    GemvParams p{};
    p.seg[0] = {W.wo.qs, W.wo.scales, H};
    p.nseg = 1;
    p.k = kin;
    p.n_rows = H;
    p.n_units = H / 16;
    p.kr = kr - r0 < maxr ? kr - r0 : maxr;
    p.pro = PRO_X16;
    p.x = m->attn + (size_t)r0 * kin;
    p.x_stride = kin;
    p.epi = EPI_STORE;
    p.y = m->o + (size_t)r0 * H;
    p.y_stride = H;
    return p;
  };
  // (a8-a10) post-attention norm + residual, pre-FFN norm, gate|up, GeGLU
  auto gate_up_params = [&](int l) {
    const q4g_layer_weights& W = m->layers[l];
    GemvParams p{};
    p.seg[0] = {W.wgate.qs, W.wgate.scales, cf.ffn};
    p.seg[1] = {W.wup.qs, W.wup.scales, cf.ffn};
    p.nseg = 2;
    p.k = H;
    p.n_rows = 2 * cf.ffn;
    p.n_units = cf.ffn / 8;
    p.kr = kr;
    p.pro = PRO_RESID;
    p.r_in = rB;
    p.r_out = rA;
    p.delta = m->o;
    p.w_delta = W.norm_post_attn;
    p.scale = 1.0f;
    p.w_x = W.norm_pre_ffn;
    p.eps = cf.rms_eps;
    p.epi = EPI_GEGLU;
    p.act = m->act;
    p.act_stride = cf.ffn;
    return p;
  };
  // (a11) down projection, activation rows [r0, r0 + maxr)
  auto down_params = [&](int l, int r0) {
    const q4g_layer_weights& W = m->layers[l];
    const int maxr = gemv_max_rows(cf.ffn);
    GemvParams p{};
    p.seg[0] = {W.wdown.qs, W.wdown.scales, H};
    p.nseg = 1;
    p.k = cf.ffn;
    p.n_rows = H;
    p.n_units = H / 16;
    p.kr = kr - r0 < maxr ? kr - r0 : maxr;
    p.pro = PRO_X16;
    p.x = m->act + (size_t)r0 * cf.ffn;
    p.x_stride = cf.ffn;
    p.epi = EPI_STORE;
    p.y = m->d + (size_t)r0 * H;
    p.y_stride = H;
    return p;
  };
  // (a12, a13) last residual + layer scalar, final norm, tied head, softcap, argmax
  auto head_params = [&]() {
    GemvParams p{};
    p.seg[0] = {m->embed.qs, m->embed.scales, cf.vocab};
    p.nseg = 1;
    p.k = H;
    p.n_rows = cf.vocab;
    p.n_units = (cf.vocab + 15) / 16;
    p.kr = kr;
    p.pro = PRO_RESID;
    p.r_in = rA;
    p.r_out = rB;
    p.delta = m->d;
    p.w_delta = m->layers[L - 1].norm_post_ffn;
    p.scale = m->layers[L - 1].layer_scalar;
    p.w_x = m->norm_final;
    p.eps = cf.rms_eps;
    p.dump = m->dump ? m->dump + (size_t)L * H : nullptr;
    p.dump_stride = dstride;
    p.epi = EPI_HEAD;
    p.logits = logits;
    p.logits_stride = cf.vocab;
    p.softcap = cf.softcap;
    p.am_val = m->am_val;
    p.am_idx = m->am_idx;
    p.counter = m->counters;
    p.argmax_out = argmax ? argmax : m->argmax_buf;
    return p;
  };
  for (int l = 0; l < L; ++l) {
    const q4g_layer_weights& W = m->layers[l];
    const bool full = m->full[l];
    const LayerShape& S = full ? m->gl : m->sl;
    const int ord = m->ordinal[l];
    const GemvParams gate_up = gate_up_params(l);
    // separate launches: the timeline of layer 1's QKV and gate|up (CTA 0)
    uint64_t* const trace_sep = m->trace && l == 1 ? m->trace : nullptr;
    {
      GemvParams p = qkv_params(l);
      p.trace = trace_sep ? trace_sep + kGemvTraceSlots : nullptr;
      if (l == 0 && m->stall_next) {
        p.stall_test = 1;
        p.wait_ns = 20000000ull;  // 20 ms
      }
      Prof pr(m, st);
      e = pr.done(debug_sync(launch_gemv(p, st, pdl), "qkv", l, st), 1, l, gemv_bytes(S.qkv_cols, H, kr, 4));
      if (e != cudaSuccess) return e;
    }
    // (a4-a6) q/k/v epilogue, cache write, split-KV attention, combine
    {
      AttnParams p{};
      p.qkv = m->qkv;
      p.qkv_stride = S.qkv_cols;
      p.k_off = S.nq_cols;
      p.v_off = full ? -1 : S.nq_cols + S.k_cols;
      p.w_q = W.norm_q;
      p.w_k = W.norm_k;
      p.v_norm = full ? 1 : cf.v_norm_sliding;
      p.rope = full ? m->rope_gl : m->rope_sl;
      p.rope_pairs = S.rope_pairs;
      p.eps = cf.rms_eps;
      bind_cache(p, c, full, ord);
      p.cache_rows = full ? c->capacity : cf.ring;
      p.ring = full ? 0 : 1;
      p.window = cf.window;
      p.pos_dev = m->pos_dev;
      p.kr = kr;
      p.write_kv = 1;
      p.n_q = cf.n_q_heads;
      p.n_kv = S.nkv;
      p.hd = S.hd;
      p.m_groups = m_groups_for(kr, S.G);
      p.n_chunks = full ? n_chunks_linear(m, p.m_groups) : n_chunks_ring(m, p.m_groups);
      p.part_ml = m->part_ml;
      p.part_acc = m->part_acc;
      p.counters = m->counters + 8;
      p.combine_in_kernel = full ? 0 : 1;
      if (!full && m->attn_cluster) {
        // sliding layers: the chunks of one KV head form a cluster and merge in DSMEM
        p.trace = trace_sep ? trace_sep + 4 * kGemvTraceSlots : nullptr;
        if (S.nkv * kAttnCluster <= kRingSplitCounters) {
          p.ring_split = 2;
          p.counters = m->counters + 64;
        }
        p.cluster = kAttnCluster;
        p.n_chunks = kAttnCluster;
        p.combine_in_kernel = 0;
      }
      p.out = m->attn;
      const int64_t q_last = pos0 + kr - 1;
      const int64_t keys = full ? q_last + 1 : std::min<int64_t>(q_last + 1, (int64_t)cf.window + kr - 1);
      const double kv_bytes = (double)S.nkv * (keys + kr) * 2.0 * S.hd * 2.0;
      Prof pr(m, st);
      e = pr.done(debug_sync(launch_attention(p, st, pdl), "attention", l, st), full ? 3 : 2, l, kv_bytes);
      if (e != cudaSuccess) return e;
      if (full) {
        Prof pc(m, st);
        e = pc.done(debug_sync(launch_attn_combine(p, st, pdl), "combine", l, st), 4, l,
                    (double)kr * cf.n_q_heads * p.n_chunks * (S.hd + 2) * 4.0);
        if (e != cudaSuccess) return e;
      }
    }
    {
      const int kin = cf.n_q_heads * S.hd;
      const int maxr = gemv_max_rows(kin);
      for (int r0 = 0; r0 < kr; r0 += maxr) {
        GemvParams p = o_params(l, r0);
        p.trace = trace_sep && r0 == 0 ? trace_sep + 2 * kGemvTraceSlots : nullptr;
        Prof pr(m, st);
        e = pr.done(debug_sync(launch_gemv(p, st, pdl), "o_proj", l, st), 5, l, gemv_bytes(H, kin, p.kr, 4));
        if (e != cudaSuccess) return e;
      }
    }
    {
      GemvParams p = gate_up;
      p.trace = trace_sep;
      p.trace_ends = trace_sep ? trace_sep + 5 * kGemvTraceSlots : nullptr;
      Prof pr(m, st);
      e = pr.done(debug_sync(launch_gemv(p, st, pdl), "gate_up", l, st), 6, l, gemv_bytes(2 * cf.ffn, H, kr, 1));
      if (e != cudaSuccess) return e;
    }
    {
      const int maxr = gemv_max_rows(cf.ffn);
      for (int r0 = 0; r0 < kr; r0 += maxr) {
        GemvParams p = down_params(l, r0);
        p.trace = trace_sep && r0 == 0 ? trace_sep + 3 * kGemvTraceSlots : nullptr;
        Prof pr(m, st);
        e = pr.done(debug_sync(launch_gemv(p, st, pdl), "down", l, st), 7, l, gemv_bytes(H, cf.ffn, p.kr, 4));
        if (e != cudaSuccess) return e;
      }
    }
  }
  if (!logits && !argmax && !m->dump) return cudaSuccess;  // no output asked for: the step only fills the cache
  {
    GemvParams p = head_params();
    Prof pr(m, st);
    if (m->embed_f16) {  // (f3) fp16 tied head: 2 bytes per weight
      p.w16 = m->embed_f16;
      e = pr.done(debug_sync(launch_gemv_f16(p, st, pdl), "head_f16", L, st), 8, L,
                  (double)cf.vocab * H * 2 + (logits ? 4.0 * kr * cf.vocab : 0.0));
    } else {
      e = pr.done(debug_sync(launch_gemv(p, st, pdl), "head", L, st), 8, L,
                  gemv_bytes(cf.vocab, H, kr, logits ? 4 : 0));
    }
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

q4g_status run_step(q4g_model* m, q4g_cache* c, int kr, int64_t pos0, const int32_t* ids_dev,
                    const int32_t* ids_host, const float* hidden, float* logits, int32_t* argmax,
                    cudaStream_t st) {
  if (!m || !c) return fail(Q4G_EINVAL, "model or cache is NULL");
  if (c->m != m) return fail(Q4G_EINVAL, "cache belongs to another model");
  const q4g_config& cf = m->cfg;
  if (logits && !aligned(logits, 4)) return fail(Q4G_EINVAL, "logits misaligned");
  std::lock_guard<std::mutex> lk(m->mu);
  StepParams sp{};
  sp.kr = kr;
  sp.pos0 = pos0;
  sp.ids_dev = ids_dev;
  for (int j = 0; ids_host && j < kr; ++j) sp.ids_host[j] = ids_host[j];
  sp.hidden = hidden;
  sp.emb_qs = m->embed.qs;
  sp.emb_sc = m->embed.scales;
  sp.emb_f16 = m->embed_f16;
  sp.hidden_size = cf.hidden;
  sp.vocab = cf.vocab;
  sp.embed_scale = cf.embed_scale;
  sp.r_out = m->r[0];
  sp.dump = m->dump;
  sp.dump_stride = (int64_t)(cf.n_layers + 1) * cf.hidden;
  sp.inv_freq_sl = m->inv_freq_sl;
  sp.inv_freq_gl = m->inv_freq_gl;
  sp.pairs_sl = m->sl.rope_pairs;
  sp.pairs_gl = m->gl.rope_pairs;
  sp.rope_sl = m->rope_sl;
  sp.rope_gl = m->rope_gl;
  sp.pos_dev = m->pos_dev;
  sp.counters = m->counters;
  sp.n_counters = m->n_counters;
  {
    Prof pr(m, st);
    CK(pr.done(launch_step_init(sp, st), 0, -1, (double)kr * cf.hidden * (4 + 0.5625)));
  }
  if (!m->use_graph || m->profile || m->stall_next) {
    cudaError_t e = enqueue_body(m, c, kr, pos0, logits, argmax, st);
    m->stall_next = false;
    CK(e);
    return Q4G_OK;
  }
  cudaGraphExec_t exec = nullptr;
  for (auto& g : m->graphs)
    if (g.kind == kr && g.cache == c && g.logits == logits && g.argmax == argmax && g.dump == m->dump)
      exec = g.exec;
  if (!exec) {
    if (m->graphs.size() >= 16) free_graphs(m);
    cudaGraph_t graph = nullptr;
    CK(cudaStreamBeginCapture(m->cap_stream, cudaStreamCaptureModeThreadLocal));
    cudaError_t e = enqueue_body(m, c, kr, pos0, logits, argmax, m->cap_stream);
    cudaError_t e2 = cudaStreamEndCapture(m->cap_stream, &graph);
    if (e != cudaSuccess) {
      if (graph) cudaGraphDestroy(graph);
      return cuda_fail(e, "capture");
    }
    if (e2 != cudaSuccess) return cuda_fail(e2, "cudaStreamEndCapture");
    e = cudaGraphInstantiate(&exec, graph, 0);
    cudaGraphDestroy(graph);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGraphInstantiate");
    m->graphs.push_back({kr, c, logits, argmax, m->dump, exec});
  }
  CK(cudaGraphLaunch(exec, st));
  return Q4G_OK;
}

}  // namespace

extern "C" q4g_status q4g_decode_step(q4g_model* m, q4g_cache* c, int32_t token, int64_t pos, float* logits,
                                      int32_t* argmax, q4g_stream_t stream) {
  if (!m || !c) return fail(Q4G_EINVAL, "model or cache is NULL");
  if (pos < 0 || pos >= c->capacity) return fail(Q4G_ERANGE, "pos %lld outside [0, %lld)", (long long)pos, (long long)c->capacity);
  if (token < 0 || token >= m->cfg.vocab) return fail(Q4G_ERANGE, "token %d outside [0, %d)", token, m->cfg.vocab);
  return run_step(m, c, 1, pos, nullptr, &token, nullptr, logits, argmax, (cudaStream_t)stream);
}

extern "C" q4g_status q4g_decode_step_device_token(q4g_model* m, q4g_cache* c, const int32_t* token, int64_t pos,
                                                   float* logits, int32_t* argmax, q4g_stream_t stream) {
  if (!m || !c || !token) return fail(Q4G_EINVAL, "NULL argument");
  if (pos < 0 || pos >= c->capacity) return fail(Q4G_ERANGE, "pos outside [0, capacity)");
  return run_step(m, c, 1, pos, token, nullptr, nullptr, logits, argmax, (cudaStream_t)stream);
}

extern "C" q4g_status q4g_decode_step_hidden(q4g_model* m, q4g_cache* c, const float* hidden, int64_t pos,
                                             float* logits, int32_t* argmax, q4g_stream_t stream) {
  if (!m || !c || !hidden) return fail(Q4G_EINVAL, "NULL argument");
  if (pos < 0 || pos >= c->capacity) return fail(Q4G_ERANGE, "pos outside [0, capacity)");
  return run_step(m, c, 1, pos, nullptr, nullptr, hidden, logits, argmax, (cudaStream_t)stream);
}

extern "C" q4g_status q4g_decode_step_host(q4g_model* m, q4g_cache* c, int32_t token, int64_t pos,
                                           float* logits_host, int32_t* argmax_host, q4g_stream_t stream) {
  if (!m || !c || !argmax_host) return fail(Q4G_EINVAL, "NULL argument");
  cudaStream_t st = (cudaStream_t)stream;
  float* dl = logits_host ? m->logits_buf : nullptr;
  q4g_status s = q4g_decode_step(m, c, token, pos, dl, m->argmax_buf, stream);
  if (s) return s;
  CK(cudaMemcpyAsync(argmax_host, m->argmax_buf, sizeof(int32_t), cudaMemcpyDeviceToHost, st));
  if (logits_host)
    CK(cudaMemcpyAsync(logits_host, dl, sizeof(float) * (size_t)m->cfg.vocab, cudaMemcpyDeviceToHost, st));
  CK(cudaStreamSynchronize(st));
  return Q4G_OK;
}

extern "C" q4g_status q4g_verify_block(q4g_model* m, q4g_cache* c, const int32_t* ids, int32_t K, int64_t pos0,
                                       int32_t accepted_count, float* logits, int32_t* argmax,
                                       q4g_stream_t stream) {
  if (!m || !c || !ids) return fail(Q4G_EINVAL, "NULL argument");
  if (K < 1 || K > kMaxRows) return fail(Q4G_ERANGE, "K must be 1..%d", kMaxRows);
  if (K > m->cfg.ring - m->cfg.window) return fail(Q4G_ERANGE, "K > ring - window");
  if (pos0 < 0 || pos0 + K > c->capacity) return fail(Q4G_ERANGE, "block outside [0, capacity)");
  if (accepted_count < 0 || accepted_count > K) return fail(Q4G_ERANGE, "accepted_count outside [0, K]");
  return run_step(m, c, K, pos0, ids, nullptr, nullptr, logits, argmax, (cudaStream_t)stream);
}

extern "C" q4g_status q4g_prefill_chunk(q4g_model* m, q4g_cache* c, const int32_t* ids, int32_t S, int64_t pos0,
                                        float* logits, int32_t* argmax, q4g_stream_t stream) {
  if (!m || !c || !ids) return fail(Q4G_EINVAL, "NULL argument");
  if (S < 1 || S > kPrefillChunk) return fail(Q4G_ERANGE, "S must be 1..%d", kPrefillChunk);
  if (pos0 < 0 || pos0 + S > c->capacity) return fail(Q4G_ERANGE, "chunk outside [0, capacity)");
  if (logits && !aligned(logits, 4)) return fail(Q4G_EINVAL, "logits misaligned");
  // blocks of up to 4 rows (the widest the stage GEMV takes), each one verify pass
  // whose rows are all kept; the head runs for the last block only
  const int kb = std::min(kPrefillBlock, m->cfg.ring - m->cfg.window);
  const cudaStream_t st = (cudaStream_t)stream;
  for (int b0 = 0; b0 < S; b0 += kb) {
    const int n = std::min(kb, S - b0);
    const bool last = b0 + n == S;
    const bool out = last && (logits || argmax);
    q4g_status r = run_step(m, c, n, pos0 + b0, ids + b0, nullptr, nullptr, out ? m->logits_buf : nullptr,
                            out ? m->argmax_buf : nullptr, st);
    if (r != Q4G_OK) return r;
    if (out) {  // the chunk's last row
      if (logits)
        CK(cudaMemcpyAsync(logits, m->logits_buf + (size_t)(n - 1) * m->cfg.vocab, sizeof(float) * m->cfg.vocab,
                           cudaMemcpyDeviceToDevice, st));
      if (argmax)
        CK(cudaMemcpyAsync(argmax, m->argmax_buf + (n - 1), sizeof(int32_t), cudaMemcpyDeviceToDevice, st));
    }
  }
  return Q4G_OK;
}

extern "C" int32_t q4g_model_profile_read(q4g_model* m, q4g_launch_record* out, int32_t max,
                                          q4g_stream_t stream) {
  if (!m || (max > 0 && !out)) {
    fail(Q4G_EINVAL, "NULL argument");
    return -1;
  }
  std::lock_guard<std::mutex> lk(m->mu);
  cudaError_t e = cudaStreamSynchronize((cudaStream_t)stream);
  if (e != cudaSuccess) {
    cuda_fail(e, "q4g_model_profile_read");
    return -1;
  }
  const int32_t n = (int32_t)m->recs.size();
  for (int32_t i = 0; i < n && i < max; ++i) {
    float ms = 0.f;
    cudaEventElapsedTime(&ms, m->recs[i].a, m->recs[i].b);
    out[i] = {m->recs[i].kind, m->recs[i].layer, ms, m->recs[i].bytes};
  }
  m->recs.clear();
  m->ev_next = 0;
  return n;
}
