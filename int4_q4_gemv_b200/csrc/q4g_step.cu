// One decode step of the decoder (one activation row) as one persistent,
// cooperative launch: one CTA per SM runs every layer's
//   QKV GEMV -> attention partials -> attention merge -> O GEMV -> gate|up GEMV
//   (GeGLU) -> down GEMV
// and then the tied head (softcap, argmax) as a sequence of phases. A phase
// starts on a CTA once every CTA has finished the previous one (a grid-wide
// completion counter per phase, bounded wait).
//
// Operations: "Gemma 4 12B" (coreai-model-zoo) architecture paragraph (the
// sandwich RMSNorms, per-head q/k norms, attention_k_eq_v, dual RoPE,
// layer_scalar, tied head and softcap), its intro (q4_0: per-block-32 absmax
// symmetric int4) and its flash-decode paragraph (GQA decode, scale 1.0, fp32
// online softmax, the scan split across cooperating groups with a merge);
// "Gemma-4-12B-CoreAI" (visible-cx), v5 section (ring of R slots, slot =
// position mod R, the live window of W positions).
//
// Why one launch: at batch 1 every GEMV is a weight stream, and a decode step
// is ~290 dependent pieces of work. With one launch per piece, each boundary
// costs a kernel drain, a launch and a cold start of the next weight stream.
// Here the weights never wait for the activations: one producer warp per CTA
// streams the CTA's share of every phase (weights of the GEMVs, K/V rows of the
// attention) in order through one ring of shared-memory stages, so the stages
// of the next phases are already landing while the compute warps wait at a
// phase boundary, compute a norm, or merge attention partials.
//
// Per CTA: 16 compute warps and one feeder warp.
//   * GEMV phase (as the stage kernel): the CTA owns a contiguous range of
//     R-row units; compute warp (c, g) takes the 32-block column chunk c of the
//     4-row group g of every stage with the integer block dot (x as 16-bit
//     block fixed point, dp4a over the raw codes) and writes one partial per
//     row; the feeder adds the chunk partials in chunk order, runs the
//     epilogue (store, GeGLU, softcap + logits + argmax) and refills the slot.
//     The fused prologues (previous residual update, RMSNorm, gains) run on the
//     compute warps after the phase boundary.
//   * attention phase: CTA (KV head, chunk) owns a contiguous range of the
//     live positions (sliding: the last W positions through the ring; full:
//     0..pos); its K/V rows arrive as stages of 32 (hd 256) or 16 (hd 512)
//     keys. The position's own K/V row comes from the QKV output (q/k
//     RMSNorm with gains, RoPE, scale-free V norm, k_eq_v on full layers) and
//     the CTA that owns it writes it to the cache. Lanes hold contiguous dims
//     of the query rows; scores are fp16 x fp16 products accumulated in fp32,
//     online softmax and P.V in fp32; warps merge through shared memory and
//     the CTA writes one (m, l, acc) partial per query row.
//   * merge phase: every CTA merges a slice of the attention output over the
//     chunks in chunk order (deterministic) and writes it as fp16.
// Completion of phase p on a CTA implies that the CTA has finished every read
// and write of phases <= p; that is what makes the reuse of the activation
// buffers across layers safe.
#include "q4g_common.cuh"
#include "q4g_dot.cuh"
#include "q4g_internal.h"

#include <stdio.h>

#include <algorithm>

namespace q4g {

namespace {

constexpr int kSkCompute = 16;                       // compute warps
constexpr int kSkThreads = (kSkCompute + 1) * 32;    // + the feeder warp
constexpr int kSkSlots = 5;                          // ring stages
constexpr int kSkSlotBytes = 36864;                  // 16 rows x 4096 columns, or the K/V rows of 16-32 keys
constexpr int kSkMaxR = 16;                          // rows per GEMV stage
constexpr int kSkMaxNC = 16;                         // 32-block column chunks per stage
constexpr int kSkMaxK = 4096;                        // columns of a fused-norm GEMV (hidden)
constexpr int kSkMergeFloats = 8192;                 // warp partials of the attention merge
constexpr int kSkMaxRopeSl = 128;                    // rotating pairs of a sliding head (hd 256)
constexpr int kSkMaxRopeGl = 256;                    // rotating pairs of a full head (hd 512)

enum : int { PK_QKV = 0, PK_ATT = 1, PK_MRG = 2, PK_O = 3, PK_GU = 4, PK_DN = 5, PK_HEAD = 6 };

struct SkShared {
  uint64_t full[kSkSlots];   // the stage's bytes landed
  uint64_t ready[kSkSlots];  // every compute warp is done with the stage
  uint64_t pub;              // grid-count mode: the feeder stored the last outputs of a GEMV phase
  float red[kSkSlots][kSkMaxNC][kSkMaxR];  // GEMV chunk partials per slot
  float norm[2][kSkCompute];
  alignas(16) unsigned char cursor[512];  // the feeder's producer cursor (lane 0 only), a Cursor
  float2 rope_sl[kSkMaxRopeSl];  // this step's (cos, sin) per rotating pair, copied at entry
  float2 rope_gl[kSkMaxRopeGl];
  int abort_flag;
  int last;  // attention: this CTA is the last of its KV head to write its partial
  int pad_[2];
  union alignas(16) {
    __half xh[kSkMaxK];  // GEMV: the normed fp16 activation row (fused-norm prologue)
    struct {
      float buf[kSkMergeFloats];  // attention: warp partials of one merge round
      float ml[kSkCompute][4][2];
      alignas(16) __half kloc[512];  // the position's own K row (fp16, as stored)
      alignas(16) __half vloc[512];
    } att;
  } u;
};

size_t sk_smem_bytes() { return (size_t)kSkSlots * kSkSlotBytes + sizeof(SkShared); }
static_assert((size_t)kSkSlots * kSkSlotBytes + sizeof(SkShared) <= 232448, "dynamic shared memory of one CTA");

Q4G_DEV void compute_bar() { asm volatile("bar.sync 1, %0;" ::"n"(kSkCompute * 32) : "memory"); }

Q4G_DEV int ld_acquire_gpu(const int32_t* p) {
  int v;
  asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

Q4G_DEV int phase_kind(int p, int L) { return p == 6 * L ? PK_HEAD : p % 6; }

// ------------------------------------------------------------ tagged words --
// An activation element travels as one 64-bit word: value bits low, tag high.
// The tag of what layer l writes in step e is e * 128 + l + 1 (the step's layer-0
// input: e * 128). 64-bit relaxed accesses at gpu scope are single-copy atomic, so
// a reader that sees the tag it expects also sees the value stored with it.
Q4G_DEV uint32_t tag_of(uint32_t epoch, int layer_plus_one) { return epoch * 128u + (uint32_t)layer_plus_one; }
Q4G_DEV uint64_t ld_tagged(const uint64_t* p) {
  uint64_t v;
  asm volatile("ld.relaxed.gpu.global.b64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
  return v;
}
Q4G_DEV void st_tagged(uint64_t* p, uint32_t bits, uint32_t tag) {
  const uint64_t v = ((uint64_t)tag << 32) | bits;
  asm volatile("st.relaxed.gpu.global.b64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}
Q4G_DEV uint32_t half2_bits(__half2 h) { return *reinterpret_cast<const uint32_t*>(&h); }

// Load n tagged words p[i * stride] into v[], re-reading the ones whose tag is not
// yet `tag` (bounded in time; on a timeout the abort flag is set and v keeps
// whatever it holds).
template <int N>
Q4G_DEV void ld_tagged_wait(const uint64_t* p, int stride, int n, uint32_t tag, uint64_t (&v)[N],
                            const StepKernelParams& P, volatile int* abort_flag) {
  unsigned miss = 0;
#pragma unroll
  for (int i = 0; i < N; ++i) {
    if (i < n) {
      v[i] = ld_tagged(p + (size_t)i * stride);
      if ((uint32_t)(v[i] >> 32) != tag) miss |= 1u << i;
    }
  }
  if (!miss) return;
  const uint64_t t0 = global_ns();
  uint32_t sleep = P.poll_ns;  // doubling back-off: every CTA's threads poll, keep the L2 traffic low
  for (int it = 0; it < kSpinLimit && miss; ++it) {
    if (*abort_flag) return;
    __nanosleep(sleep);
    sleep = min(2 * sleep + 32, 2048u);
#pragma unroll
    for (int i = 0; i < N; ++i) {
      if (miss & (1u << i)) {
        v[i] = ld_tagged(p + (size_t)i * stride);
        if ((uint32_t)(v[i] >> 32) == tag) miss &= ~(1u << i);
      }
    }
    if (miss && global_ns() - t0 > P.wait_ns) {
      *abort_flag = 1;
      atomicOr(P.err, 1);
      return;
    }
  }
}

// --------------------------------------------------------------- GEMV phases --
struct GD {
  const uint8_t* q[3];
  const uint16_t* s[3];
  int rows[3];
  int nseg;
  int k, n_rows, n_units, R, NC, G;
  int pro, epi;
  uint32_t tag_in, tag_out;  // tags this phase reads and writes
  const uint64_t* x;  // PRO_X16 input, fp16 pairs (tagged)
  const uint64_t* r_in;
  uint64_t* r_out;
  const uint64_t* delta;
  const float* w_delta;
  float scale;
  const float* w_x;
  float* dump;
  uint64_t* y;    // EPI_STORE, tagged fp32
  uint64_t* act;  // EPI_GEGLU, tagged fp16 pairs
};

Q4G_DEV void gd_geometry(GD& g, int ffn) {
  g.R = g.k <= 4096 ? 16 : g.k <= 8192 ? 8 : 4;
  g.NC = ((g.k >> 5) + 31) >> 5;
  g.G = g.R / 4;
  g.n_units = g.epi == EPI_GEGLU ? ffn / (g.R / 2) : (g.n_rows + g.R - 1) / g.R;
}

Q4G_DEV GD gemv_desc(const StepKernelParams& P, int p, uint32_t epoch) {
  GD g{};
  const int L = P.n_layers, H = P.hidden, kind = phase_kind(p, L), l = p / 6;
  g.tag_in = tag_of(epoch, kind == PK_QKV ? l : kind == PK_HEAD ? L : l + 1);
  g.tag_out = tag_of(epoch, l + 1);
  if (kind == PK_HEAD) {
    const StepLayer& Lp = P.layers[L - 1];
    g.q[0] = P.emb_q, g.s[0] = P.emb_s, g.rows[0] = P.vocab, g.nseg = 1;
    g.k = H, g.n_rows = P.vocab;
    g.pro = PRO_RESID, g.r_in = P.r0, g.r_out = P.r1, g.delta = P.d, g.w_delta = Lp.norm_post_ffn;
    g.scale = Lp.layer_scalar, g.w_x = P.norm_final;
    g.dump = P.dump ? P.dump + (size_t)L * H : nullptr;
    g.epi = EPI_HEAD;
    gd_geometry(g, P.ffn);
    return g;
  }
  const StepLayer& Ly = P.layers[l];
  const int hd = Ly.full ? P.gl_hd : P.sl_hd, nkv = Ly.full ? P.gl_nkv : P.sl_nkv;
  if (kind == PK_QKV) {
    g.q[0] = Ly.q[0], g.s[0] = Ly.s[0], g.rows[0] = P.n_q * hd;
    g.q[1] = Ly.q[1], g.s[1] = Ly.s[1], g.rows[1] = nkv * hd;
    g.nseg = 2;
    if (!Ly.full) g.q[2] = Ly.q[2], g.s[2] = Ly.s[2], g.rows[2] = nkv * hd, g.nseg = 3;
    g.k = H;
    g.n_rows = g.rows[0] + g.rows[1] + (Ly.full ? 0 : g.rows[2]);
    g.pro = PRO_RESID, g.r_in = P.r0, g.r_out = P.r1;
    if (l > 0) {
      g.delta = P.d, g.w_delta = P.layers[l - 1].norm_post_ffn, g.scale = P.layers[l - 1].layer_scalar;
    } else {
      g.scale = 1.0f;
    }
    g.w_x = Ly.norm_in;
    g.dump = P.dump ? P.dump + (size_t)l * H : nullptr;
    g.epi = EPI_STORE, g.y = P.qkv;
  } else if (kind == PK_O) {
    g.q[0] = Ly.q[3], g.s[0] = Ly.s[3], g.rows[0] = H, g.nseg = 1;
    g.k = P.n_q * hd, g.n_rows = H;
    g.pro = PRO_X16, g.x = P.attn;
    g.epi = EPI_STORE, g.y = P.o;
  } else if (kind == PK_GU) {
    g.q[0] = Ly.q[4], g.s[0] = Ly.s[4], g.rows[0] = P.ffn;
    g.q[1] = Ly.q[5], g.s[1] = Ly.s[5], g.rows[1] = P.ffn;
    g.nseg = 2;
    g.k = H, g.n_rows = 2 * P.ffn;
    g.pro = PRO_RESID, g.r_in = P.r1, g.r_out = P.r0, g.delta = P.o, g.w_delta = Ly.norm_post_attn;
    g.scale = 1.0f, g.w_x = Ly.norm_pre_ffn;
    g.epi = EPI_GEGLU, g.act = P.act;
  } else {  // PK_DN
    g.q[0] = Ly.q[6], g.s[0] = Ly.s[6], g.rows[0] = H, g.nseg = 1;
    g.k = P.ffn, g.n_rows = H;
    g.pro = PRO_X16, g.x = P.act;
    g.epi = EPI_STORE, g.y = P.d;
  }
  gd_geometry(g, P.ffn);
  return g;
}

Q4G_DEV void unit_range(int n_units, int& u0, int& n) {
  u0 = (int)((long long)blockIdx.x * n_units / gridDim.x);
  n = (int)((long long)(blockIdx.x + 1) * n_units / gridDim.x) - u0;
}

// Bulk copies of GEMV unit u into stage st: [R rows of codes][R rows of scales]
// (GeGLU: R/2 gate rows then the R/2 up rows of the same index).
Q4G_DEV void issue_gemv(const GD& g, int u, unsigned char* st, uint64_t* bar, uint64_t pol, uint32_t extra) {
  const int kh = g.k >> 1, nb = g.k >> 5, R = g.R;
  if (g.epi == EPI_GEGLU) {
    const int h = R / 2, r0 = h * u;
    const uint32_t qb = (uint32_t)h * kh, sb = (uint32_t)h * nb * 2;
    mbar_arrive_expect_tx(bar, 2 * (qb + sb) + extra);
    bulk_g2s_hint(st, g.q[0] + (size_t)r0 * kh, qb, bar, pol);
    bulk_g2s_hint(st + qb, g.q[1] + (size_t)r0 * kh, qb, bar, pol);
    bulk_g2s_hint(st + (size_t)R * kh, g.s[0] + (size_t)r0 * nb, sb, bar, pol);
    bulk_g2s_hint(st + (size_t)R * kh + sb, g.s[1] + (size_t)r0 * nb, sb, bar, pol);
    return;
  }
  int row = R * u, sgi = 0;
  while (sgi + 1 < g.nseg && row >= g.rows[sgi]) row -= g.rows[sgi], ++sgi;  // units never straddle segments
  const int n = min(R, g.rows[sgi] - row);
  const uint32_t qb = (uint32_t)n * kh, sb = (uint32_t)n * nb * 2;
  mbar_arrive_expect_tx(bar, qb + sb + extra);
  bulk_g2s_hint(st, g.q[sgi] + (size_t)row * kh, qb, bar, pol);
  bulk_g2s_hint(st + (size_t)R * kh, g.s[sgi] + (size_t)row * nb, sb, bar, pol);
}

// ---------------------------------------------------------- attention phases --
struct AD {
  int hd, nkv, G, kv, chunk, nch, active;
  int ring;          // 1: sliding ring
  int R;             // ring slots (ring) or capacity (linear)
  int nscan;         // live positions of this query: pos - nscan + 1 .. pos
  int k0, k1;        // this CTA's scan indices
  int SK;            // keys per stage
  int64_t pos;
  __half* kc;        // this layer's K / V cache (head kv)
  __half* vc;
};

Q4G_DEV AD att_desc(const StepKernelParams& P, int l, int64_t pos) {
  AD a{};
  const StepLayer& Ly = P.layers[l];
  const bool full = Ly.full != 0;
  a.hd = full ? P.gl_hd : P.sl_hd;
  a.nkv = full ? P.gl_nkv : P.sl_nkv;
  a.G = P.n_q / a.nkv;
  a.nch = (int)gridDim.x / a.nkv;
  a.kv = (int)blockIdx.x / a.nch;
  a.chunk = (int)blockIdx.x - a.kv * a.nch;
  a.active = a.kv < a.nkv;
  a.ring = !full;
  a.R = full ? (int)P.capacity : P.ring;
  a.pos = pos;
  a.nscan = full ? (int)(pos + 1) : (int)min(pos + 1, (int64_t)P.window);
  const int cs = (a.nscan + a.nch - 1) / a.nch;
  a.k0 = a.active ? min(a.nscan, a.chunk * cs) : 0;
  a.k1 = a.active ? min(a.nscan, a.k0 + cs) : 0;
  a.SK = 32768 / (a.hd * 4);
  const size_t lb = full ? P.glob_layer_bytes : P.ring_layer_bytes;
  const size_t ko = full ? P.glob_k_off : P.ring_k_off, vo = full ? P.glob_v_off : P.ring_v_off;
  const int kvh = a.active ? a.kv : 0;
  a.kc = reinterpret_cast<__half*>(P.cache + ko + (size_t)Ly.ordinal * lb) + (size_t)kvh * a.R * a.hd;
  a.vc = reinterpret_cast<__half*>(P.cache + vo + (size_t)Ly.ordinal * lb) + (size_t)kvh * a.R * a.hd;
  return a;
}

// cache row of scan index i (position pos - nscan + 1 + i)
Q4G_DEV int att_row(const AD& a, int i) {
  const int64_t p = a.pos - a.nscan + 1 + i;
  return a.ring ? (int)(p % a.R) : (int)p;
}

// Bulk copies of stage i of the CTA's keys: K rows at [0, SK), V rows at
// [SK, 2 SK) of the slot, in scan order; the position's own row (the last scan
// index) is not in the cache yet and is left out.
Q4G_DEV void issue_att(const AD& a, int i, unsigned char* st, uint64_t* bar, uint64_t pol, uint32_t extra) {
  const int ka = a.k0 + i * a.SK, kb = min(a.k1, ka + a.SK);
  const int kc_end = min(kb, a.nscan - 1);  // cached keys [ka, kc_end)
  const int n = max(0, kc_end - ka);
  const uint32_t rb = (uint32_t)a.hd * 2;
  mbar_arrive_expect_tx(bar, 2u * n * rb + extra);
  if (n == 0) return;
  const int r0 = att_row(a, ka);
  const int n1 = a.ring ? min(n, a.R - r0) : n;  // first run up to the ring's end
  unsigned char* kd = st;
  unsigned char* vd = st + (size_t)a.SK * rb;
  bulk_g2s_hint(kd, a.kc + (size_t)r0 * a.hd, (uint32_t)n1 * rb, bar, pol);
  bulk_g2s_hint(vd, a.vc + (size_t)r0 * a.hd, (uint32_t)n1 * rb, bar, pol);
  if (n1 < n) {
    bulk_g2s_hint(kd + (size_t)n1 * rb, a.kc, (uint32_t)(n - n1) * rb, bar, pol);
    bulk_g2s_hint(vd + (size_t)n1 * rb, a.vc, (uint32_t)(n - n1) * rb, bar, pol);
  }
}

// ------------------------------------------------------------- stage counts --
struct StepCtx {
  int L, NP;
  int64_t pos;
  uint32_t epoch;
};

Q4G_DEV int phase_stages(const StepKernelParams& P, const StepCtx& c, int p) {
  const int kind = phase_kind(p, c.L);
  if (kind == PK_MRG) return 0;
  if (kind == PK_ATT) {
    const AD a = att_desc(P, p / 6, c.pos);
    return (a.k1 - a.k0 + a.SK - 1) / a.SK;
  }
  const GD g = gemv_desc(P, p, c.epoch);
  int u0, n;
  unit_range(g.n_units, u0, n);
  return n;
}

// The producer's position in the stage sequence, with the descriptor of its
// phase kept while it issues that phase's stages (recomputed once per phase).
struct Cursor {
  int p, i, n, att;
  GD g;
  int u0;
  AD a;
};

static_assert(sizeof(Cursor) <= 512, "the cursor lives in SkShared::cursor");

Q4G_DEV void cursor_load(const StepKernelParams& P, const StepCtx& c, Cursor& k) {
  k.i = 0;
  k.n = 0;
  for (; k.p < c.NP; ++k.p) {
    const int kind = phase_kind(k.p, c.L);
    if (kind == PK_MRG) continue;
    k.att = kind == PK_ATT;
    if (k.att) {
      k.a = att_desc(P, k.p / 6, c.pos);
      k.n = (k.a.k1 - k.a.k0 + k.a.SK - 1) / k.a.SK;
    } else {
      k.g = gemv_desc(P, k.p, c.epoch);
      unit_range(k.g.n_units, k.u0, k.n);
    }
    if (k.n > 0) return;
  }
}

Q4G_DEV void cursor_issue(const Cursor& k, unsigned char* st, uint64_t* bar, uint64_t pol, uint32_t extra) {
  if (k.att)
    issue_att(k.a, k.i, st, bar, pol, extra);
  else
    issue_gemv(k.g, k.u0 + k.i, st, bar, pol, extra);
}

Q4G_DEV void cursor_next(const StepKernelParams& P, const StepCtx& c, Cursor& k) {
  if (++k.i < k.n) return;
  ++k.p;
  cursor_load(P, c, k);
}

// ----------------------------------------------------------- bounded waits --
Q4G_DEV void sk_abort(const StepKernelParams& P, volatile int* abort_flag) {
  *abort_flag = 1;
  atomicOr(P.err, 1);
}

Q4G_DEV bool sk_wait(uint64_t* bar, uint32_t phase, const StepKernelParams& P, volatile int* abort_flag) {
  if (mbar_try_wait(bar, phase)) return true;
  const uint64_t t0 = global_ns();
  for (int it = 0; it < kSpinLimit; ++it) {
    if (*abort_flag) return false;
    if (mbar_try_wait(bar, phase)) return true;
    if (global_ns() - t0 > P.wait_ns) break;
  }
  sk_abort(P, abort_flag);
  return false;
}

// Whether any lane of the warp has seen the CTA give up. Every lane of the warp must
// call it: it reconverges lanes that waited for different lengths of time, so that
// a guarded block holding warp collectives is entered by all lanes or by none.
Q4G_DEV bool warp_aborted(volatile int* abort_flag) { return __any_sync(0xffffffffu, *abort_flag != 0); }

// Thread 0 of the compute warps: wait until every CTA finished phase p.
Q4G_DEV void wait_phase(const StepKernelParams& P, int p, volatile int* abort_flag) {
  if (*abort_flag) return;
  const int target = (int)gridDim.x;
  if (ld_acquire_gpu(P.done + p) >= target) return;
  const uint64_t t0 = global_ns();
  for (int it = 0; it < kSpinLimit; ++it) {
    __nanosleep(P.poll_ns);  // back off: every CTA polls the same counter that the last CTAs still increment
    if (ld_acquire_gpu(P.done + p) >= target) return;
    if (*abort_flag) return;
    if (global_ns() - t0 > P.wait_ns) break;
  }
  sk_abort(P, abort_flag);
}

// This CTA finished phase p (every thread's writes ordered before by the caller).
Q4G_DEV void signal_phase(const StepKernelParams& P, int p) {
  __threadfence();
  atomicAdd(P.done + p, 1);
}

// ------------------------------------------------ fused-norm prologue (GEMV) --
// r_new = (r_in + rmsnorm(delta) * w_delta) * scale (delta may be NULL),
// x = fp16(rmsnorm(r_new) * w_x) into s.u.xh; CTA 0 stores r_new (and the dump).
// The 512 compute threads only; ends with a compute barrier.
constexpr int kSkR4 = kSkMaxK / (4 * kSkCompute * 32);  // float4 of a hidden row per compute thread

// The gains of the fused-norm prologue (weights: loaded before the phase boundary).
struct ResidGains {
  float4 wd[kSkR4], wx[kSkR4];
};
Q4G_DEV void resid_gains(const GD& g, ResidGains& w) {
  constexpr int NT = kSkCompute * 32;
  const int tid = threadIdx.x, n4 = g.k >> 2;
  const float4 z4 = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
  for (int i = 0; i < kSkR4; ++i) {
    const int c4 = tid + i * NT;
    w.wd[i] = c4 < n4 && g.delta ? __ldg(reinterpret_cast<const float4*>(g.w_delta) + c4) : z4;
    w.wx[i] = c4 < n4 ? __ldg(reinterpret_cast<const float4*>(g.w_x) + c4) : z4;
  }
}

Q4G_DEV float4 tagged4(const uint64_t (&v)[4]) {
  return make_float4(__uint_as_float((uint32_t)v[0]), __uint_as_float((uint32_t)v[1]),
                     __uint_as_float((uint32_t)v[2]), __uint_as_float((uint32_t)v[3]));
}

Q4G_DEV void resid_prologue(const GD& g, const StepKernelParams& P, SkShared& s, const ResidGains& w,
                            volatile int* abort_flag) {
  constexpr int NT = kSkCompute * 32, R4 = kSkR4;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, k = g.k, n4 = k >> 2;
  const bool dl = g.delta != nullptr;
  const float4 z4 = make_float4(0.f, 0.f, 0.f, 0.f);
  float4 rn[R4], dv[R4];
#pragma unroll
  for (int i = 0; i < R4; ++i) {  // the tagged words of the residual and the delta, as they arrive
    const int c4 = tid + i * NT;
    rn[i] = dv[i] = z4;
    if (c4 < n4) {
      uint64_t v[4];
      ld_tagged_wait<4>(g.r_in + 4 * c4, 1, 4, g.tag_in, v, P, abort_flag);
      rn[i] = tagged4(v);
      if (dl) {
        ld_tagged_wait<4>(g.delta + 4 * c4, 1, 4, g.tag_in, v, P, abort_flag);
        dv[i] = tagged4(v);
      }
    }
  }
  const float4(&wdv)[R4] = w.wd;
  const float4(&wxv)[R4] = w.wx;
  if (dl) {
    float ss = 0.f;
#pragma unroll
    for (int i = 0; i < R4; ++i)
      ss = fmaf(dv[i].x, dv[i].x, fmaf(dv[i].y, dv[i].y, fmaf(dv[i].z, dv[i].z, fmaf(dv[i].w, dv[i].w, ss))));
    ss = warp_sum(ss);
    if (lane == 0) s.norm[0][warp] = ss;
    compute_bar();
    float tot = 0.f;
#pragma unroll
    for (int w = 0; w < kSkCompute; ++w) tot += s.norm[0][w];
    const float inv_d = rms_inv(tot, k, P.eps);
#pragma unroll
    for (int i = 0; i < R4; ++i) {
      rn[i].x = __fmul_rn(__fadd_rn(rn[i].x, __fmul_rn(__fmul_rn(dv[i].x, inv_d), wdv[i].x)), g.scale);
      rn[i].y = __fmul_rn(__fadd_rn(rn[i].y, __fmul_rn(__fmul_rn(dv[i].y, inv_d), wdv[i].y)), g.scale);
      rn[i].z = __fmul_rn(__fadd_rn(rn[i].z, __fmul_rn(__fmul_rn(dv[i].z, inv_d), wdv[i].z)), g.scale);
      rn[i].w = __fmul_rn(__fadd_rn(rn[i].w, __fmul_rn(__fmul_rn(dv[i].w, inv_d), wdv[i].w)), g.scale);
    }
  } else if (g.scale != 1.0f) {
#pragma unroll
    for (int i = 0; i < R4; ++i) {
      rn[i].x = __fmul_rn(rn[i].x, g.scale), rn[i].y = __fmul_rn(rn[i].y, g.scale);
      rn[i].z = __fmul_rn(rn[i].z, g.scale), rn[i].w = __fmul_rn(rn[i].w, g.scale);
    }
  }
  float ss2 = 0.f;
#pragma unroll
  for (int i = 0; i < R4; ++i) {
    const int c4 = tid + i * NT;
    ss2 = fmaf(rn[i].x, rn[i].x, fmaf(rn[i].y, rn[i].y, fmaf(rn[i].z, rn[i].z, fmaf(rn[i].w, rn[i].w, ss2))));
    if (blockIdx.x == 0 && c4 < n4) {
      st_tagged(g.r_out + 4 * c4 + 0, __float_as_uint(rn[i].x), g.tag_out);
      st_tagged(g.r_out + 4 * c4 + 1, __float_as_uint(rn[i].y), g.tag_out);
      st_tagged(g.r_out + 4 * c4 + 2, __float_as_uint(rn[i].z), g.tag_out);
      st_tagged(g.r_out + 4 * c4 + 3, __float_as_uint(rn[i].w), g.tag_out);
      if (g.dump) reinterpret_cast<float4*>(g.dump)[c4] = rn[i];
    }
  }
  ss2 = warp_sum(ss2);
  if (lane == 0) s.norm[1][warp] = ss2;
  compute_bar();
  float tot2 = 0.f;
#pragma unroll
  for (int w = 0; w < kSkCompute; ++w) tot2 += s.norm[1][w];
  const float inv_r = rms_inv(tot2, k, P.eps);
#pragma unroll
  for (int i = 0; i < R4; ++i) {
    const int c4 = tid + i * NT;
    if (c4 < n4) {
      __half2* dst = reinterpret_cast<__half2*>(s.u.xh + 4 * c4);
      dst[0] = __floats2half2_rn(__fmul_rn(__fmul_rn(rn[i].x, inv_r), wxv[i].x),
                                 __fmul_rn(__fmul_rn(rn[i].y, inv_r), wxv[i].y));
      dst[1] = __floats2half2_rn(__fmul_rn(__fmul_rn(rn[i].z, inv_r), wxv[i].z),
                                 __fmul_rn(__fmul_rn(rn[i].w, inv_r), wxv[i].w));
    }
  }
  compute_bar();
}

// ----------------------------------------------------- attention (compute) --
// Sum v[0..N) over the 32 lanes and give every lane all N totals (N a power of
// two <= 32): a transposing butterfly, then N broadcasts.
template <int N>
Q4G_DEV void warp_allreduce_n(float (&v)[N], int lane) {
#pragma unroll
  for (int h = N / 2, o = 16; h >= 1; h >>= 1, o >>= 1) {
    const bool upper = lane & o;
#pragma unroll
    for (int i = 0; i < h; ++i) {
      const float send = upper ? v[i] : v[i + h];
      const float keep = upper ? v[i + h] : v[i];
      v[i] = keep + __shfl_xor_sync(0xffffffffu, send, o);
    }
  }
  float t = v[0];
#pragma unroll
  for (int o = 16 / N; o >= 1; o >>= 1) t += __shfl_xor_sync(0xffffffffu, t, o);
#pragma unroll
  for (int idx = 0; idx < N; ++idx) {
    int src = 0;
#pragma unroll
    for (int h = N / 2, o = 16; h >= 1; h >>= 1, o >>= 1) src += (idx & h) ? o : 0;
    v[idx] = __shfl_sync(0xffffffffu, t, src);
  }
}

// acc + a.lo * b.lo + a.hi * b.hi (fp16 products are exact in fp32)
Q4G_DEV float dot2_f16(uint32_t a, uint32_t b, float acc) {
  float r;
  asm("{\n\t.reg .b16 al, ah, bl, bh;\n\t"
      "mov.b32 {al, ah}, %1;\n\t"
      "mov.b32 {bl, bh}, %2;\n\t"
      "fma.rn.f32.f16 %0, al, bl, %3;\n\t"
      "fma.rn.f32.f16 %0, ah, bh, %0;\n\t}"
      : "=f"(r)
      : "r"(a), "r"(b), "f"(acc));
  return r;
}

// NR projection rows of HD values by one warp, lane holding dims
// [lane * HD/32, ...): RMSNorm (gain or scale-free), RoPE on the first `pairs`
// rotate-half pairs (i, i + HD/2), rounded to fp16 (the fp16 words of the lane's
// dims go to out[r][]). Every global load is issued before the first use, so the
// rows cost one round trip; the (cos, sin) table is in shared memory.
template <int HD, int NR>
Q4G_DEV void proj_rows(const uint64_t* const (&src)[NR], uint32_t tag, const float* gain, bool do_norm,
                       const float2* rope, int pairs, float eps, uint32_t (&out)[NR][HD / 64], int lane,
                       const StepKernelParams& P, volatile int* abort_flag) {
  constexpr int DPL = HD / 32;
  float v[NR][DPL], gv[DPL];
#pragma unroll
  for (int e = 0; e < DPL; e += 4) {
    const float4 t = gain ? __ldg(reinterpret_cast<const float4*>(gain + lane * DPL + e)) : make_float4(1.f, 1.f, 1.f, 1.f);
    gv[e] = t.x, gv[e + 1] = t.y, gv[e + 2] = t.z, gv[e + 3] = t.w;
  }
#pragma unroll
  for (int r = 0; r < NR; ++r) {
    uint64_t w[DPL];
    ld_tagged_wait<DPL>(src[r] + lane * DPL, 1, DPL, tag, w, P, abort_flag);
#pragma unroll
    for (int e = 0; e < DPL; ++e) v[r][e] = __uint_as_float((uint32_t)w[e]);
  }
  const bool lo = lane < 16;
#pragma unroll
  for (int r = 0; r < NR; ++r) {
    float ss = 0.f;
#pragma unroll
    for (int e = 0; e < DPL; ++e) ss = fmaf(v[r][e], v[r][e], ss);
    const float inv = do_norm ? rms_inv(warp_sum(ss), HD, eps) : 1.0f;
#pragma unroll
    for (int e = 0; e < DPL; ++e) {
      v[r][e] = __fmul_rn(v[r][e], inv);
      if (gain) v[r][e] = __fmul_rn(v[r][e], gv[e]);
    }
    if (rope) {
#pragma unroll
      for (int e = 0; e < DPL; ++e) {
        const float partner = __shfl_xor_sync(0xffffffffu, v[r][e], 16);
        const int i = (lo ? lane : lane - 16) * DPL + e;  // pair index
        if (i < pairs) {
          const float2 cs = rope[i];
          v[r][e] = lo ? v[r][e] * cs.x - partner * cs.y : v[r][e] * cs.x + partner * cs.y;
        }
      }
    }
#pragma unroll
    for (int e = 0; e < DPL / 2; ++e) {
      const __half2 h = __floats2half2_rn(v[r][2 * e], v[r][2 * e + 1]);
      out[r][e] = *reinterpret_cast<const uint32_t*>(&h);
    }
  }
}

template <int HD, int RPW>
Q4G_DEV void attention_phase(const StepKernelParams& P, const AD& a, int l, SkShared& s, unsigned char* ring,
                             int& T, volatile int* abort_flag, uint64_t* tr, uint32_t epoch) {
  constexpr int DPL = HD / 32, W2 = DPL / 2;  // dims and fp16 words per lane
  constexpr int B = HD == 512 ? 2 : 4;         // keys per group
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int NRG = a.G / RPW, NKG = kSkCompute / NRG;
  const int rg = warp / NKG, kg = warp - rg * NKG;
  const StepLayer& Ly = P.layers[l];
  const bool full = Ly.full != 0;
  const float2* rope = full ? s.rope_gl : s.rope_sl;
  const int pairs = full ? P.rope_pairs_gl : P.rope_pairs_sl;
  const int qkv_k = P.n_q * HD, qkv_v = full ? -1 : qkv_k + a.nkv * HD;
  const bool has_new = a.active && a.k1 == a.nscan && a.k1 > a.k0;
  const int n_st = (a.k1 - a.k0 + a.SK - 1) / a.SK;

  // ---- prologue: the query rows of this warp, the position's own K/V row ----
  uint32_t q[RPW][W2];
  const uint32_t tag = tag_of(epoch, l + 1);  // the QKV outputs of this layer
  if (a.active) {
    const uint64_t* rows[RPW];
#pragma unroll
    for (int t = 0; t < RPW; ++t) rows[t] = P.qkv + (size_t)(a.kv * a.G + rg * RPW + t) * HD;
    proj_rows<HD, RPW>(rows, tag, Ly.norm_q, true, rope, pairs, P.eps, q, lane, P, abort_flag);
  } else {
#pragma unroll
    for (int t = 0; t < RPW; ++t)
#pragma unroll
      for (int e = 0; e < W2; ++e) q[t][e] = 0u;
  }
  if (tr && tid == 0) tr[3] = global_ns();
  if (has_new && warp < 2) {
    uint32_t w[1][W2];
    if (warp == 0) {
      const uint64_t* rows[1] = {P.qkv + qkv_k + (size_t)a.kv * HD};
      proj_rows<HD, 1>(rows, tag, Ly.norm_k, true, rope, pairs, P.eps, w, lane, P, abort_flag);
    } else {
      const uint64_t* rows[1] = {P.qkv + (qkv_v >= 0 ? qkv_v : qkv_k) + (size_t)a.kv * HD};
      proj_rows<HD, 1>(rows, tag, nullptr, full || P.v_norm_sliding != 0, nullptr, 0, P.eps, w, lane, P,
                       abort_flag);
    }
    __half* loc = warp == 0 ? s.u.att.kloc : s.u.att.vloc;
    __half* cache = (warp == 0 ? a.kc : a.vc) + (size_t)att_row(a, a.nscan - 1) * HD;
#pragma unroll
    for (int e = 0; e < W2; e += 2) {
      const uint2 pk = make_uint2(w[0][e], w[0][e + 1]);
      *reinterpret_cast<uint2*>(loc + lane * DPL + 2 * e) = pk;
      *reinterpret_cast<uint2*>(cache + lane * DPL + 2 * e) = pk;
    }
  }
  compute_bar();  // kloc / vloc visible
  if (tr && tid == 0) tr[1] = global_ns();

  // ---- scan: groups of B keys, all RPW rows at once ----
  float m[RPW], lsum[RPW], acc[RPW][DPL];
#pragma unroll
  for (int t = 0; t < RPW; ++t) {
    m[t] = -INFINITY, lsum[t] = 0.f;
#pragma unroll
    for (int e = 0; e < DPL; ++e) acc[t][e] = 0.f;
  }
  const size_t rbytes = (size_t)HD * 2;
  for (int i = 0; i < n_st; ++i, ++T) {
    const int sl = T % kSkSlots;
    if (!warp_aborted(abort_flag)) sk_wait(&s.full[sl], (uint32_t)((T / kSkSlots) & 1), P, abort_flag);
    const int ka = a.k0 + i * a.SK, kb = min(a.k1, ka + a.SK);
    const unsigned char* kbase = ring + (size_t)sl * kSkSlotBytes;
    const unsigned char* vbase = kbase + (size_t)a.SK * rbytes;
    if (!warp_aborted(abort_flag)) {
      for (int j0 = ka + kg; j0 < kb; j0 += NKG * B) {
        float sc[B * RPW];
        bool valid[B];
#pragma unroll
        for (int b = 0; b < B; ++b) {
          const int j = j0 + b * NKG;
          valid[b] = j < kb;
          const __half* kr = j == a.nscan - 1 ? s.u.att.kloc
                                              : reinterpret_cast<const __half*>(kbase + (size_t)(j - ka) * rbytes);
          uint4 kk[DPL / 8];
#pragma unroll
          for (int c = 0; c < DPL / 8; ++c)
            kk[c] = valid[b] ? *reinterpret_cast<const uint4*>(kr + lane * DPL + 8 * c) : make_uint4(0, 0, 0, 0);
#pragma unroll
          for (int t = 0; t < RPW; ++t) {
            float d = 0.f;
#pragma unroll
            for (int c = 0; c < DPL / 8; ++c) {
              d = dot2_f16(kk[c].x, q[t][4 * c + 0], d);
              d = dot2_f16(kk[c].y, q[t][4 * c + 1], d);
              d = dot2_f16(kk[c].z, q[t][4 * c + 2], d);
              d = dot2_f16(kk[c].w, q[t][4 * c + 3], d);
            }
            sc[b * RPW + t] = d;
          }
        }
        warp_allreduce_n<B * RPW>(sc, lane);
#pragma unroll
        for (int t = 0; t < RPW; ++t) {
          float mx = m[t];
#pragma unroll
          for (int b = 0; b < B; ++b) mx = valid[b] ? fmaxf(mx, sc[b * RPW + t]) : mx;
          const float corr = m[t] == -INFINITY ? 0.f : __expf(m[t] - mx);
          m[t] = mx;
          lsum[t] *= corr;
#pragma unroll
          for (int e = 0; e < DPL; ++e) acc[t][e] *= corr;
        }
#pragma unroll
        for (int b = 0; b < B; ++b) {
          if (!valid[b]) continue;
          const int j = j0 + b * NKG;
          const __half* vrow = j == a.nscan - 1 ? s.u.att.vloc
                                                : reinterpret_cast<const __half*>(vbase + (size_t)(j - ka) * rbytes);
          float vf[DPL];
#pragma unroll
          for (int c = 0; c < DPL / 8; ++c) {
            const uint4 vq = *reinterpret_cast<const uint4*>(vrow + lane * DPL + 8 * c);
            const __half2* h2 = reinterpret_cast<const __half2*>(&vq);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const float2 f = __half22float2(h2[e]);
              vf[8 * c + 2 * e] = f.x, vf[8 * c + 2 * e + 1] = f.y;
            }
          }
#pragma unroll
          for (int t = 0; t < RPW; ++t) {
            const float pr = __expf(sc[b * RPW + t] - m[t]);
            lsum[t] += pr;
#pragma unroll
            for (int e = 0; e < DPL; ++e) acc[t][e] = fmaf(pr, vf[e], acc[t][e]);
          }
        }
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&s.ready[sl]);  // this warp is done with the stage
  }

  // ---- merge the NKG warps of each row group through shared memory ----
  if (NRG == 1 && kSkCompute * RPW * HD <= kSkMergeFloats) {
    // every warp holds the same rows: all 16 partials go to shared memory at once,
    // then each compute thread merges output elements over the 16 warps (warp order)
    if (a.active) {
      float* b = s.u.att.buf + (size_t)warp * RPW * HD;
#pragma unroll
      for (int t = 0; t < RPW; ++t) {
#pragma unroll
        for (int e = 0; e < DPL; e += 4)
          *reinterpret_cast<float4*>(b + t * HD + lane * DPL + e) =
              make_float4(acc[t][e], acc[t][e + 1], acc[t][e + 2], acc[t][e + 3]);
        if (lane == 0) s.u.att.ml[warp][t][0] = m[t], s.u.att.ml[warp][t][1] = lsum[t];
      }
    }
    compute_bar();
    if (a.active) {
      for (int el = tid; el < RPW * HD; el += kSkCompute * 32) {
        const int t = el / HD, d = el - t * HD;
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < kSkCompute; ++w) M = fmaxf(M, s.u.att.ml[w][t][0]);
        float L = 0.f, A = 0.f;
#pragma unroll 4
        for (int w = 0; w < kSkCompute; ++w) {
          const float mw = s.u.att.ml[w][t][0];
          if (mw == -INFINITY) continue;
          const float e = __expf(mw - M);
          L = fmaf(s.u.att.ml[w][t][1], e, L);
          A = fmaf(s.u.att.buf[(size_t)w * RPW * HD + t * HD + d], e, A);
        }
        const int h = a.kv * a.G + t;
        const size_t row = (size_t)h * a.nch + a.chunk;
        __stcg(P.part_acc + row * HD + d, A);
        if (d == 0) __stcg(reinterpret_cast<float2*>(P.part_ml + 2 * row), make_float2(M, L));
      }
    }
    return;
  }
  // per round, every row group stores up to S warp partials; kg == 0 merges them
  const int S = min(max(1, kSkMergeFloats / (RPW * HD) / NRG), max(1, NKG - 1));
  const int rounds = (NKG - 1 + S - 1) / S;
  for (int r = 0; r < rounds; ++r) {
    const int lo = 1 + r * S, hi = min(NKG, lo + S);
    if (kg >= lo && kg < hi && a.active) {
      const int slot = rg * S + (kg - lo);
      float* b = s.u.att.buf + (size_t)slot * RPW * HD;
#pragma unroll
      for (int t = 0; t < RPW; ++t) {
#pragma unroll
        for (int e = 0; e < DPL; e += 4)
          *reinterpret_cast<float4*>(b + t * HD + lane * DPL + e) =
              make_float4(acc[t][e], acc[t][e + 1], acc[t][e + 2], acc[t][e + 3]);
        if (lane == 0) s.u.att.ml[slot][t][0] = m[t], s.u.att.ml[slot][t][1] = lsum[t];
      }
    }
    compute_bar();
    if (kg == 0 && a.active) {
      for (int w = lo; w < hi; ++w) {
        const int slot = rg * S + (w - lo);
        const float* b = s.u.att.buf + (size_t)slot * RPW * HD;
#pragma unroll
        for (int t = 0; t < RPW; ++t) {
          const float mw = s.u.att.ml[slot][t][0], lw = s.u.att.ml[slot][t][1];
          if (mw == -INFINITY) continue;
          const float mn = fmaxf(m[t], mw);
          const float c0 = m[t] == -INFINITY ? 0.f : __expf(m[t] - mn), c1 = __expf(mw - mn);
          lsum[t] = lsum[t] * c0 + lw * c1;
#pragma unroll
          for (int e = 0; e < DPL; ++e) acc[t][e] = acc[t][e] * c0 + b[t * HD + lane * DPL + e] * c1;
          m[t] = mn;
        }
      }
    }
    compute_bar();
  }
  // ---- the CTA partial of each query row ----
  if (kg == 0 && a.active) {
#pragma unroll
    for (int t = 0; t < RPW; ++t) {
      const int h = a.kv * a.G + rg * RPW + t;
      const size_t row = (size_t)h * a.nch + a.chunk;
      float* dst = P.part_acc + row * HD + lane * DPL;
#pragma unroll
      for (int e = 0; e < DPL; e += 4)
        __stcg(reinterpret_cast<float4*>(dst + e), make_float4(acc[t][e], acc[t][e + 1], acc[t][e + 2], acc[t][e + 3]));
      if (lane == 0) __stcg(reinterpret_cast<float2*>(P.part_ml + 2 * row), make_float2(m[t], lsum[t]));
    }
  }
}

// The attention output o[h][d] = sum_c acc_c e^(m_c - M) / sum_c l_c e^(m_c - M)
// over the chunks of its KV head, written as tagged fp16 pairs (d, d + 1). Full
// layers: every CTA merges a slice of the pairs, 8 lanes per pair, each over every
// 8th chunk, then a fixed butterfly: deterministic.
Q4G_DEV void merge_phase(const StepKernelParams& P, int l, uint32_t tag) {
  const StepLayer& Ly = P.layers[l];
  const int hd = Ly.full ? P.gl_hd : P.sl_hd, nkv = Ly.full ? P.gl_nkv : P.sl_nkv;
  const int nch = (int)gridDim.x / nkv;
  const int total = P.n_q * hd / 2;  // pairs
  const int o0 = (int)((long long)blockIdx.x * total / gridDim.x);
  const int o1 = (int)((long long)(blockIdx.x + 1) * total / gridDim.x);
  const int tid = threadIdx.x, sub = tid & 7, grp = tid >> 3;  // 64 groups of 8 lanes
  for (int base = o0; base < o1; base += kSkCompute * 4) {
    const int o = base + grp;
    const bool in = o < o1;
    const int h = in ? (2 * o) / hd : 0, d = in ? 2 * o - h * hd : 0;
    const size_t row0 = (size_t)h * nch;
    float M = -INFINITY;
#pragma unroll 4
    for (int c = sub; c < nch && in; c += 8) M = fmaxf(M, __ldcg(P.part_ml + 2 * (row0 + c)));
#pragma unroll
    for (int x = 1; x < 8; x <<= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, x));
    float A0 = 0.f, A1 = 0.f, Ls = 0.f;
#pragma unroll 4
    for (int c = sub; c < nch && in; c += 8) {
      const float2 ml = __ldcg(reinterpret_cast<const float2*>(P.part_ml + 2 * (row0 + c)));
      if (ml.x == -INFINITY) continue;
      const float e = __expf(ml.x - M);
      const float2 a = __ldcg(reinterpret_cast<const float2*>(P.part_acc + (row0 + c) * hd + d));
      Ls = fmaf(ml.y, e, Ls);
      A0 = fmaf(a.x, e, A0);
      A1 = fmaf(a.y, e, A1);
    }
#pragma unroll
    for (int x = 1; x < 8; x <<= 1) {
      A0 += __shfl_xor_sync(0xffffffffu, A0, x);
      A1 += __shfl_xor_sync(0xffffffffu, A1, x);
      Ls += __shfl_xor_sync(0xffffffffu, Ls, x);
    }
    if (in && sub == 0)
      st_tagged(P.attn + ((size_t)h * hd + d) / 2, half2_bits(__floats2half2_rn(A0 / Ls, A1 / Ls)), tag);
  }
}

// The G query rows of KV head kv from its nch chunk partials, as tagged fp16 pairs
// (sliding layers: the last CTA of the head to finish runs this, all compute
// threads, chunk order).
Q4G_DEV void merge_head(const StepKernelParams& P, int hd, int G, int kv, int nch, uint32_t tag) {
  for (int pe = threadIdx.x; pe < G * hd / 2; pe += kSkCompute * 32) {
    const int h = kv * G + (2 * pe) / hd, d = (2 * pe) % hd;
    const size_t row0 = (size_t)h * nch;
    float M = -INFINITY;
#pragma unroll 4
    for (int c = 0; c < nch; ++c) M = fmaxf(M, __ldcg(P.part_ml + 2 * (row0 + c)));
    float A0 = 0.f, A1 = 0.f, Ls = 0.f;
#pragma unroll 4
    for (int c = 0; c < nch; ++c) {
      const float2 ml = __ldcg(reinterpret_cast<const float2*>(P.part_ml + 2 * (row0 + c)));
      if (ml.x == -INFINITY) continue;
      const float e = __expf(ml.x - M);
      const float2 a = __ldcg(reinterpret_cast<const float2*>(P.part_acc + (row0 + c) * hd + d));
      Ls = fmaf(ml.y, e, Ls);
      A0 = fmaf(a.x, e, A0);
      A1 = fmaf(a.y, e, A1);
    }
    st_tagged(P.attn + ((size_t)h * hd + d) / 2, half2_bits(__floats2half2_rn(A0 / Ls, A1 / Ls)), tag);
  }
}

template <int HD>
Q4G_DEV void attention_dispatch(const StepKernelParams& P, const AD& a, int l, SkShared& s, unsigned char* ring,
                                int& T, volatile int* abort_flag, uint64_t* tr, uint32_t epoch) {
  const int G = a.G;
  if (G % 2 == 0) {
    attention_phase<HD, 2>(P, a, l, s, ring, T, abort_flag, tr, epoch);
  } else {
    attention_phase<HD, 1>(P, a, l, s, ring, T, abort_flag, tr, epoch);
  }
}

// ------------------------------------------------------------------ kernel --
__global__ void __launch_bounds__(kSkThreads, 1) step_kernel(const StepKernelParams P) {
  extern __shared__ __align__(128) unsigned char sk_smem[];
  unsigned char* ring = sk_smem;
  SkShared& s = *reinterpret_cast<SkShared*>(sk_smem + (size_t)kSkSlots * kSkSlotBytes);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  StepCtx cx;
  cx.L = P.n_layers;
  cx.NP = 6 * P.n_layers + 1;
  cx.pos = *P.pos_dev;  // written before the launch
  cx.epoch = *P.epoch;
  const uint64_t pol = policy_evict_first();
  uint64_t* const trace = blockIdx.x == 0 ? P.trace : nullptr;
  if (trace && tid == 0) trace[4 * cx.NP] = global_ns();

  if (tid == 0) {
    s.abort_flag = 0;
    for (int i = 0; i < kSkSlots; ++i) mbar_init(&s.full[i], 1), mbar_init(&s.ready[i], kSkCompute);
    mbar_init(&s.pub, 1);
    fence_mbar_init();
  }
  for (int i = tid; i < P.rope_pairs_sl; i += kSkThreads) s.rope_sl[i] = P.rope_sl[i];  // written before the launch
  for (int i = tid; i < P.rope_pairs_gl; i += kSkThreads) s.rope_gl[i] = P.rope_gl[i];
  __syncthreads();
  volatile int* abort_flag = &s.abort_flag;

  if (warp == kSkCompute) {
    // =================== feeder: stage stream, GEMV reductions, epilogues ===================
    // producer cursor: the next stage to issue, kept in shared memory by lane 0
    Cursor& cur = *reinterpret_cast<Cursor*>(s.cursor);
    int issued = 0;
    if (lane == 0) {
      cur.p = 0;
      cursor_load(P, cx, cur);
      for (int k = 0; k < kSkSlots && cur.p < cx.NP; ++k) {
        cursor_issue(cur, ring + (size_t)k * kSkSlotBytes, &s.full[k], pol,
                     P.stall_test && blockIdx.x == 0 && k == 0 ? 16u : 0u);
        ++issued;
        cursor_next(P, cx, cur);
      }
    }
    int T = 0;
    float best_v = -INFINITY;
    int best_i = 0x7fffffff;
    for (int p = 0; p < cx.NP && !warp_aborted(abort_flag); ++p) {
      const int kind = phase_kind(p, cx.L);
      const int n = phase_stages(P, cx, p);
      GD g{};
      int u0 = 0;
      const bool gemv = kind != PK_ATT && kind != PK_MRG;
      if (gemv) {
        g = gemv_desc(P, p, cx.epoch);
        int nn;
        unit_range(g.n_units, u0, nn);
      }
      for (int i = 0; i < n; ++i, ++T) {
        const int sl = T % kSkSlots;
        sk_wait(&s.ready[sl], (uint32_t)((T / kSkSlots) & 1), P, abort_flag);  // a timeout sets the flag
        // compute warps that gave up still hand their slots back without having seen the
        // slot's fill complete: never refill such a slot (its barrier phase may be pending)
        if (warp_aborted(abort_flag)) break;
        float val = 0.f;
        if (gemv && lane < g.R)
          for (int c = 0; c < g.NC; ++c) val += s.red[sl][c][lane];
        __syncwarp();  // every lane read the slot's partials: refill it before the epilogue
        if (lane == 0 && cur.p < cx.NP) {
          cursor_issue(cur, ring + (size_t)sl * kSkSlotBytes, &s.full[sl], pol, 0u);
          ++issued;
          cursor_next(P, cx, cur);
        }
        if (gemv) {
          const int R = g.R, u = u0 + i;
          if (g.epi == EPI_GEGLU) {
            // lane r < R/2: gate row r, up row r + R/2; lanes 2i and 2i + 1 form one fp16 pair
            const int h = R / 2;
            const float up = __shfl_sync(0xffffffffu, val, (lane + h) & 31);
            const float a = gelu_tanh(val) * up;
            const float a_next = __shfl_down_sync(0xffffffffu, a, 1);
            if (lane < h && !(lane & 1))
              st_tagged(g.act + ((size_t)h * u + lane) / 2, half2_bits(__floats2half2_rn(a, a_next)), g.tag_out);
          } else if (lane < R) {
            const int row = R * u + lane;
            if (row < g.n_rows) {
              if (g.epi == EPI_STORE) {
                st_tagged(g.y + row, __float_as_uint(val), g.tag_out);
              } else {
                const float z = P.softcap * tanhf(val / P.softcap);
                if (P.logits) P.logits[row] = z;
                if (z > best_v || (z == best_v && row < best_i)) best_v = z, best_i = row;
              }
            }
          }
        }
      }
      if (warp_aborted(abort_flag)) break;
      if (gemv && n > 0) {
        __syncwarp();
        if (lane == 0) {
          // grid-count mode: the compute warps count this CTA in on the way to the next
          // phase (a fence there, not here: the feeder keeps streaming)
          if (P.grid_sync) mbar_arrive(&s.pub);  // release of this warp's epilogue stores
          if (trace) trace[4 * p + 3] = global_ns();
        }
      }
    }
    // head: per-CTA candidate, the last CTA picks the winner (lowest index on ties)
    if (!warp_aborted(abort_flag)) {
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        const float v2 = __shfl_xor_sync(0xffffffffu, best_v, o);
        const int i2 = __shfl_xor_sync(0xffffffffu, best_i, o);
        if (v2 > best_v || (v2 == best_v && i2 < best_i)) best_v = v2, best_i = i2;
      }
      if (lane == 0) {
        P.am_val[blockIdx.x] = best_v;
        P.am_idx[blockIdx.x] = best_i;
        __threadfence();
        const int ticket = atomicAdd(P.done + cx.NP, 1);
        if (ticket == (int)gridDim.x - 1) {
          __threadfence();
          float v = -INFINITY;
          int ix = 0x7fffffff;
          for (int b = 0; b < (int)gridDim.x; ++b) {
            const float vb = __ldcg(P.am_val + b);
            const int ib = __ldcg(P.am_idx + b);
            if (vb > v || (vb == v && ib < ix)) v = vb, ix = ib;
          }
          P.argmax_out[0] = ix == 0x7fffffff ? 0 : ix;
        }
      }
    }
    // after a timeout, wait (bounded) for the copies still in flight
    if (lane == 0 && *abort_flag) {
      for (int t = issued > kSkSlots ? issued - kSkSlots : 0; t < issued; ++t)
        mbar_wait_bounded(&s.full[t % kSkSlots], (uint32_t)((t / kSkSlots) & 1), P.wait_ns);
    }
    if (trace && lane == 0) trace[4 * cx.NP + 1] = global_ns();
    return;
  }

  // =================== compute warps ===================
  // Tagged mode: a phase starts as soon as this CTA is done with the previous one;
  // its inputs are tagged words polled as they arrive, and the only grid-wide wait
  // is before the merge of a full-attention layer, which reads every CTA's
  // partials. Grid-count mode: every phase starts once every CTA has counted
  // itself done with the previous phase (the tagged reads then succeed at once).
  int T = 0;
  uint32_t pubs = 0;     // completed phases of s.pub
  bool publish = false;  // grid-count mode: the previous phase streamed GEMV stages here
  int prev = -1;         // the previous phase this CTA ran
  for (int p = 0; p < cx.NP; ++p) {
    const int kind = phase_kind(p, cx.L);
    // sliding layers: the last CTA of each KV head merges the head's chunks inside
    // the attention phase, so there is no separate merge phase
    if (kind == PK_MRG && !P.layers[p / 6].full) continue;
    uint64_t* tr = trace ? trace + 4 * p : nullptr;
    if (P.grid_sync && prev >= 0) {
      if (tid == 0) {
        if (publish) {  // the feeder's epilogue of the previous phase is done: count this CTA in
          if (!*abort_flag) sk_wait(&s.pub, pubs & 1, P, abort_flag);
          ++pubs;
          signal_phase(P, prev);
        }
        wait_phase(P, prev, abort_flag);
      }
      compute_bar();  // every compute thread after thread 0's acquire
    }
    publish = false;
    prev = p;
    if (tr && tid == 0) tr[0] = global_ns();
    if (kind == PK_ATT) {
      const int l = p / 6;
      const AD a = att_desc(P, l, cx.pos);
      compute_bar();  // every warp is past the previous phase's use of the shared union
      if (a.hd == 512)
        attention_dispatch<512>(P, a, l, s, ring, T, abort_flag, tr, cx.epoch);
      else
        attention_dispatch<256>(P, a, l, s, ring, T, abort_flag, tr, cx.epoch);
      compute_bar();
      if (a.ring) {  // the last CTA of the KV head merges its chunks
        if (tid == 0) {
          int last = 0;
          if (a.active) {
            __threadfence();  // this CTA's partials before its ticket
            last = atomicAdd(P.tickets + l * P.sl_nkv + a.kv, 1) == a.nch - 1;
            if (last) __threadfence();
          }
          s.last = last;
        }
        compute_bar();
        if (!warp_aborted(abort_flag) && s.last) merge_head(P, a.hd, a.G, a.kv, a.nch, tag_of(cx.epoch, l + 1));
        if (P.grid_sync) {
          compute_bar();
          if (tid == 0) signal_phase(P, p);
        }
      } else if (tid == 0) {
        signal_phase(P, p);  // the full layer's merge reads every CTA's partials
      }
      if (tr && tid == 0) tr[2] = global_ns();
      continue;
    }
    if (kind == PK_MRG) {  // full layers
      if (!P.grid_sync) {
        if (tid == 0) wait_phase(P, p - 1, abort_flag);
        compute_bar();  // every compute thread after thread 0's acquire
      }
      if (!warp_aborted(abort_flag)) merge_phase(P, p / 6, tag_of(cx.epoch, p / 6 + 1));
      if (P.grid_sync) {
        compute_bar();
        if (tid == 0) signal_phase(P, p);
      }
      if (tr && tid == 0) tr[2] = global_ns();
      continue;
    }
    // ---- GEMV phase ----
    const GD g = gemv_desc(P, p, cx.epoch);
    int u0, n;
    unit_range(g.n_units, u0, n);
    // CTA 0 writes the new residual row even when it streams no unit here
    if (g.pro == PRO_RESID && (n > 0 || blockIdx.x == 0)) {
      ResidGains gains;
      resid_gains(g, gains);
      resid_prologue(g, P, s, gains, abort_flag);  // ends with a compute barrier
    }
    if (n == 0) {
      if (P.grid_sync && tid == 0) signal_phase(P, p);
      continue;
    }
    publish = P.grid_sync != 0;
    const int nb = g.k >> 5, kh = g.k >> 1, c = warp % g.NC, grp = warp / g.NC;
    const int blk = 32 * c + lane;
    const bool act = warp < g.NC * g.G;
    const bool has = act && blk < nb;
    uint4 xg[kDigitQuads];
    int4 cv;
    {
      uint4 xv[4];
      const int bb = min(blk, nb - 1);
      if (!has) {
#pragma unroll
        for (int qd = 0; qd < 4; ++qd) xv[qd] = make_uint4(0, 0, 0, 0);
      } else if (g.pro == PRO_RESID) {
#pragma unroll
        for (int qd = 0; qd < 4; ++qd) xv[qd] = *reinterpret_cast<const uint4*>(s.u.xh + 32 * (size_t)bb + 8 * qd);
      } else {  // the block's 16 tagged fp16 pairs
        uint64_t w[16];
        ld_tagged_wait<16>(g.x + 16 * (size_t)bb, 1, 16, g.tag_in, w, P, abort_flag);
#pragma unroll
        for (int qd = 0; qd < 4; ++qd)
          xv[qd] = make_uint4((uint32_t)w[4 * qd], (uint32_t)w[4 * qd + 1], (uint32_t)w[4 * qd + 2],
                              (uint32_t)w[4 * qd + 3]);
      }
      lane_block_digits(xv, xg, cv);
      if (!has) cv = make_int4(0, 0, 0, 0);
    }
    const float xsc = __int_as_float(cv.w);
    if (tr && tid == 0) tr[1] = global_ns();
    const int bq = min(blk, nb - 1);
    for (int i = 0; i < n; ++i, ++T) {
      const int sl = T % kSkSlots;
      if (!warp_aborted(abort_flag)) sk_wait(&s.full[sl], (uint32_t)((T / kSkSlots) & 1), P, abort_flag);
      if (!warp_aborted(abort_flag) && act) {
        const unsigned char* st = ring + (size_t)sl * kSkSlotBytes;
        const unsigned char* sq = st + (size_t)grp * 4 * kh + 16 * bq;
        const unsigned char* ss = st + (size_t)g.R * kh + (size_t)grp * 4 * 2 * nb + 2 * bq;
        float v[4];
#pragma unroll
        for (int r = 0; r < 4; ++r) {
          const uint4 qv = *reinterpret_cast<const uint4*>(sq + (size_t)r * kh);
          const float d = __half2float(*reinterpret_cast<const __half*>(ss + (size_t)r * 2 * nb));
          v[r] = d * xsc * block_dot_int(qv, xg, cv);
        }
        const float tot = cs_reduce_rows<4>(v, lane);
        if ((lane & 7) == 0) s.red[sl][c][grp * 4 + cs_row<4>(lane)] = tot;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&s.ready[sl]);  // release of the partials above
    }
    if (tr && tid == 0) tr[2] = global_ns();
  }
}

}  // namespace

int step_kernel_phases(int n_layers) { return 6 * n_layers + 1; }
int step_kernel_trace_slots(int n_layers) { return 4 * step_kernel_phases(n_layers) + 2; }
int step_kernel_counters(int n_layers, int sl_kv_heads) {
  return step_kernel_phases(n_layers) + 1 + n_layers * sl_kv_heads;
}

size_t step_kernel_partial_floats(const StepKernelParams& p, int grid) {
  const size_t sl = (size_t)p.n_q * (grid / p.sl_nkv) * p.sl_hd;
  const size_t gl = (size_t)p.n_q * (grid / p.gl_nkv) * p.gl_hd;
  return std::max(sl, gl);
}
size_t step_kernel_ml_floats(const StepKernelParams& p, int grid) {
  return 2 * (size_t)p.n_q * (size_t)std::max(grid / p.sl_nkv, grid / p.gl_nkv);
}

bool step_kernel_supported(const StepKernelParams& p, char* why, size_t n) {
  auto no = [&](const char* m) {
    if (why && n) snprintf(why, n, "%s", m);
    return false;
  };
  auto gemv_ok = [&](int k, int rows_unit) {
    if (k % 256 || k > 16384) return false;
    const int R = k <= 4096 ? 16 : k <= 8192 ? 8 : 4;
    const int NC = (k / 32 + 31) / 32;
    if (NC * (R / 4) > kSkCompute) return false;
    if ((size_t)R * (k / 2 + k / 16) > (size_t)kSkSlotBytes) return false;
    return rows_unit % R == 0;
  };
  if (p.hidden > kSkMaxK) return no("hidden > 4096");
  if (p.n_layers > 126) return no("more than 126 layers (the activation tags hold the layer)");
  if (p.rope_pairs_sl > kSkMaxRopeSl || p.rope_pairs_gl > kSkMaxRopeGl) return no("rotating pairs");
  if (p.sl_hd != 256 || p.gl_hd != 512) return no("head dims must be 256 and 512");
  const int G_sl = p.n_q / p.sl_nkv, G_gl = p.n_q / p.gl_nkv;
  for (int i = 0; i < 2; ++i) {
    const int G = i ? G_gl : G_sl, hd = i ? p.gl_hd : p.sl_hd;
    const int rpw = G % 2 == 0 ? 2 : 1;  // query rows per warp
    if (G / rpw > kSkCompute || kSkCompute % (G / rpw)) return no("query heads per KV head");
    if (G * hd > kSkMergeFloats) return no("query heads x head dim of one KV head > 8192");
  }
  if (!gemv_ok(p.hidden, p.n_q * p.sl_hd) || !gemv_ok(p.hidden, p.sl_nkv * p.sl_hd) ||
      !gemv_ok(p.hidden, p.n_q * p.gl_hd) || !gemv_ok(p.hidden, p.gl_nkv * p.gl_hd))
    return no("QKV shapes");
  if (!gemv_ok(p.n_q * p.sl_hd, 16) || !gemv_ok(p.n_q * p.gl_hd, 16) || !gemv_ok(p.ffn, 16))
    return no("O / down shapes");
  {
    const int R = p.hidden <= 4096 ? 16 : p.hidden <= 8192 ? 8 : 4;
    if (p.ffn % (R / 2)) return no("ffn rows per GeGLU stage");
  }
  const int grid = device_sm_count();
  if (grid / p.sl_nkv < 1 || grid / p.gl_nkv < 1) return no("more KV heads than SMs");
  if (sk_smem_bytes() > 232448) return no("shared memory");
  return true;
}

cudaError_t launch_step_kernel(const StepKernelParams& p_in, cudaStream_t st) {
  StepKernelParams p = p_in;
  if (!p.err) p.err = device_error_word();
  if (!p.err) return cudaErrorInvalidValue;
  if (!p.wait_ns) p.wait_ns = 2000000000ull;
  static int configured_dev = -1;
  int dev = 0;
  cudaGetDevice(&dev);
  const size_t smem = sk_smem_bytes();
  if (configured_dev != dev) {
    cudaError_t e = cudaFuncSetAttribute(step_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(step_kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                             cudaSharedmemCarveoutMaxShared);
    if (e != cudaSuccess) return e;
    int bps = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&bps, step_kernel, kSkThreads, smem);
    if (e != cudaSuccess) return e;
    if (bps < 1) return cudaErrorCooperativeLaunchTooLarge;
    configured_dev = dev;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(device_sm_count());
  cfg.blockDim = dim3(kSkThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;  // every CTA resident: the phases wait on each other
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, step_kernel, p);
}

}  // namespace q4g
