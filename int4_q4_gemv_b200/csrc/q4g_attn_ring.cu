// Flash-decode over the sliding ring for a few query rows per KV head, on CUDA
// cores.
//
// Operation ("Gemma 4 12B" page, flash-decode paragraph: GQA decode, scale 1.0,
// fp32 online softmax, the KV scan split across cooperating groups;
// "Gemma-4-12B-CoreAI", v5 section: slot = position mod R, implied position
// p = q - ((q - j) mod R), window test q - p < W).
//
// With 2 query rows per KV head (decode of the sliding layers) a key row is
// used by 2 rows only, so the scan is a latency problem, not a throughput one.
// One SM reads about 50 GB/s, so the keys of one KV head are spread over as
// many SMs as fit: S clusters of CL CTAs (4 x 4 when they all fit at once,
// else one cluster of 16 or 8):
//   * CTA c of cluster h scans keys [g * cs, (g + 1) * cs) by age, g = h * CL + c,
//     warp w a contiguous 1/16 of that;
//   * 16 warps per CTA; each warp copies the K and V rows of all its keys
//     (at most kRingKeysPerWarp) into its own shared-memory buffer with 16-byte
//     asynchronous copies before waiting on the previous kernel (the rows were
//     written by earlier steps), so the scan reads shared memory only;
//   * lane l holds dims 8l .. 8l+7 (hd 256) of the query and of each key; per
//     group of 4 keys the fp32 dot products are reduced over the warp with a
//     transposing butterfly, followed by one online-softmax update and P.V,
//     all in fp32;
//   * warp partials merge in shared memory, CTA partials through distributed
//     shared memory: CTA c of a cluster owns output dims [c * HD/CL, ...);
//   * with S > 1 the CTAs owning the same dims in the S clusters write their
//     partials to global scratch, and the last to finish (a ticket) merges the S
//     partials in cluster order, so the result does not depend on timing.
// The block's own key/value rows (the new positions) come from the prologue;
// global chunk 0 also writes them to the ring.
#include "q4g_common.cuh"
#include "q4g_internal.h"

#include <stdlib.h>

#include <algorithm>
#include <cstddef>

namespace q4g {

namespace {

constexpr int kRingThreads = 512;
constexpr int kRingWarps = kRingThreads / 32;
constexpr int kRingKeysPerWarp = 10;  // 1024-key window, 8 CTAs, 16 warps, up to 4 query rows

template <int HD, int ROWS>
struct RingSmem {
  alignas(16) __half q[ROWS][HD];      // queries after norm and RoPE (fp16, as stored)
  alignas(16) __half kloc[kMaxRows][HD];  // the block's own K rows
  alignas(16) __half vloc[kMaxRows][HD];  // the block's own V rows
  alignas(16) int8_t kloc8[kMaxRows][HD];  // int8 cache: the same rows as stored
  alignas(16) int8_t vloc8[kMaxRows][HD];
  float klocs[kMaxRows], vlocs[kMaxRows];
  float kvs[kRingWarps][kRingKeysPerWarp][2];  // int8 cache: each warp's row scales
  float pm[kRingWarps][ROWS], pl[kRingWarps][ROWS];
  float cacc[ROWS][HD];                // CTA partial, relative to cm
  float cm[ROWS], cl[ROWS];
  union alignas(16) {  // read and written 16 bytes at a time
    __half kv[kRingWarps][kRingKeysPerWarp][2][HD];  // scan: each warp's K and V rows
    int8_t kv8[kRingWarps][kRingKeysPerWarp][2][HD];  // scan, int8 cache
    float part[kRingWarps][ROWS][HD];                // merge: warp partial sums of p * v
  };
};
using RingSmem1 = RingSmem<256, 1>;
using RingSmem2 = RingSmem<256, 2>;
using RingSmem4 = RingSmem<256, 4>;
static_assert(offsetof(RingSmem1, kv) % 16 == 0 && offsetof(RingSmem2, kv) % 16 == 0 &&
                  offsetof(RingSmem4, kv) % 16 == 0 && offsetof(RingSmem1, kloc) % 16 == 0,
              "16-byte accesses need 16-byte aligned buffers");
static_assert(sizeof(RingSmem<256, 4>) <= 227 * 1024, "shared memory of one CTA");

Q4G_DEV void cp_async16(void* dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"((uint32_t)__cvta_generic_to_shared(dst)), "l"(src)
               : "memory");
}
Q4G_DEV void cp_async8(void* dst, const void* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 8;" ::"r"((uint32_t)__cvta_generic_to_shared(dst)), "l"(src)
               : "memory");
}
Q4G_DEV void cp_async4(void* dst, const void* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"((uint32_t)__cvta_generic_to_shared(dst)), "l"(src)
               : "memory");
}
// 8 int8 codes (one 8-byte piece) as floats
Q4G_DEV void unpack8_i8(const uint2 u, float* f) {
  const int8_t* c = reinterpret_cast<const int8_t*>(&u);
#pragma unroll
  for (int i = 0; i < 8; ++i) f[i] = (float)c[i];
}

// Sum v[0..N) over the 32 lanes (N a power of two <= 32) and give every lane
// all N totals: a transposing butterfly (N - 1 + log2(32 / N) shuffles), then
// N broadcasts.
template <int N>
Q4G_DEV void warp_allreduce_vec(float (&v)[N], int lane) {
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
  // lane L holds total number sum_{steps} (L & o ? h : 0)
#pragma unroll
  for (int idx = 0; idx < N; ++idx) {
    int src = 0;
#pragma unroll
    for (int h = N / 2, o = 16; h >= 1; h >>= 1, o >>= 1) src += (idx & h) ? o : 0;
    v[idx] = __shfl_sync(0xffffffffu, t, src);
  }
}

Q4G_DEV void unpack8(const uint4 u, float* f) {
  const __half2* h = reinterpret_cast<const __half2*>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 t = __half22float2(h[i]);
    f[2 * i] = t.x, f[2 * i + 1] = t.y;
  }
}

// One projection vector of the block by one warp: per-head RMSNorm (learned
// gain, or scale-free), RoPE on the first rope_pairs rotate-half pairs, fp16.
// All global loads are issued before the arithmetic that depends on them.
template <int HD>
Q4G_DEV void norm_rope_vec(const AttnParams& p, const float* src, const float* gain, bool do_norm,
                           bool rotate, int j, __half* dst, int lane) {
  constexpr int E = HD / 64;  // elements per lane per half
  float lo[E], hi[E], glo[E], ghi[E];
  float2 cs[E];
#pragma unroll
  for (int e = 0; e < E; ++e) {
    const int i = lane * E + e;
    lo[e] = src[i];
    hi[e] = src[HD / 2 + i];
    glo[e] = gain ? gain[i] : 1.0f;
    ghi[e] = gain ? gain[HD / 2 + i] : 1.0f;
    cs[e] = rotate && i < p.rope_pairs ? p.rope[(size_t)j * p.rope_pairs + i] : make_float2(1.f, 0.f);
  }
  float ss = 0.f;
#pragma unroll
  for (int e = 0; e < E; ++e) ss = fmaf(lo[e], lo[e], fmaf(hi[e], hi[e], ss));
  const float inv = do_norm ? rms_inv(warp_sum(ss), HD, p.eps) : 1.0f;
#pragma unroll
  for (int e = 0; e < E; ++e) {
    const int i = lane * E + e;
    float a = __fmul_rn(lo[e], inv), b = __fmul_rn(hi[e], inv);
    if (gain) a = __fmul_rn(a, glo[e]), b = __fmul_rn(b, ghi[e]);
    if (rotate && i < p.rope_pairs) {
      const float ra = a * cs[e].x - b * cs[e].y;
      const float rb = b * cs[e].x + a * cs[e].y;
      a = ra, b = rb;
    }
    dst[i] = __float2half_rn(a);
    dst[HD / 2 + i] = __float2half_rn(b);
  }
}

// Code size is kept small on purpose: every SM runs one CTA of this kernel per
// layer, so its instructions are fetched cold; the loop over key groups is rolled.
template <int HD, int ROWS, int CL, int S, bool KV8>
__global__ void __launch_bounds__(kRingThreads, 1) attn_ring_kernel(const AttnParams p) {
  static_assert(HD == 256, "one 16-byte piece per lane and row");
  constexpr int B = ROWS <= 2 ? 4 : 2;  // keys per group
  extern __shared__ __align__(16) unsigned char ring_smem[];
  RingSmem<HD, ROWS>& sm = *reinterpret_cast<RingSmem<HD, ROWS>*>(ring_smem);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int kv = blockIdx.x;
  const int chunk = (int)cluster_rank();
  const int half = (int)blockIdx.y / CL;  // cluster index: S clusters per KV head split the keys
  const int gchunk = half * CL + chunk;
  const int G = p.n_q / p.n_kv, nr = p.kr * G;  // nr <= ROWS (host)
  const bool fused = p.qkv != nullptr;
  uint64_t* const tr = kv == 0 && gchunk == 0 && tid == 0 ? p.trace : nullptr;
  auto stamp = [&](int i) {
    if (tr) tr[i] = global_ns();
  };
  stamp(0);

  // The position was written before the first kernel of the step and the cache
  // rows read below by earlier steps: both may be read before griddepcontrol.wait.
  const int64_t pos0 = p.pos_dev ? *p.pos_dev : p.pos0;
  const int64_t q_last = pos0 + p.kr - 1;
  const int R = (int)p.cache_rows, W = (int)p.window;
  const int qlm = (int)(q_last % p.cache_rows);  // slot of the newest key
  const int nscan = (int)min((int64_t)W + p.kr - 1, q_last + 1);
  const int cs = (nscan + CL * S - 1) / (CL * S);
  const int a_begin = min(nscan, gchunk * cs), a_end = min(nscan, a_begin + cs);
  const int kpw = (a_end - a_begin + kRingWarps - 1) / kRingWarps;
  const int wa0 = min(a_end, a_begin + warp * kpw), wa1 = min(a_end, wa0 + kpw);
  const int first_cached = fused ? p.kr : 0;  // ages below are the block's own rows

  // lane l holds dims 8l .. 8l+7 of every row; every cached key of the warp
  // (wa1 - wa0 <= kRingKeysPerWarp, checked on the host) goes to shared memory
  if (!KV8) {
    const __half* kcache = p.k_cache + (size_t)kv * R * HD + lane * 8;
    const __half* vcache = p.v_cache + (size_t)kv * R * HD + lane * 8;
#pragma unroll 1
    for (int a = max(wa0, first_cached); a < wa1; ++a) {
      const size_t off = (size_t)wrap(qlm - a, R) * HD;
      cp_async16(&sm.kv[warp][a - wa0][0][lane * 8], kcache + off);
      cp_async16(&sm.kv[warp][a - wa0][1][lane * 8], vcache + off);
    }
  } else {  // int8 rows: 8 codes per lane, and the rows' scales
    const int8_t* kcache = reinterpret_cast<const int8_t*>(p.k_cache) + (size_t)kv * R * HD + lane * 8;
    const int8_t* vcache = reinterpret_cast<const int8_t*>(p.v_cache) + (size_t)kv * R * HD + lane * 8;
#pragma unroll 1
    for (int a = max(wa0, first_cached); a < wa1; ++a) {
      const size_t row = (size_t)wrap(qlm - a, R);
      cp_async8(&sm.kv8[warp][a - wa0][0][lane * 8], kcache + row * HD);
      cp_async8(&sm.kv8[warp][a - wa0][1][lane * 8], vcache + row * HD);
      if (lane == 0) {
        cp_async4(&sm.kvs[warp][a - wa0][0], p.k_scale + (size_t)kv * R + row);
        cp_async4(&sm.kvs[warp][a - wa0][1], p.v_scale + (size_t)kv * R + row);
      }
    }
  }
  asm volatile("cp.async.commit_group;" ::: "memory");

  pdl_wait();
  stamp(1);
  // ---- prologue: queries and the block's own K/V rows ----
  if (fused) {
    const int nvec = nr + 2 * p.kr;
    for (int vi = warp; vi < nvec; vi += kRingWarps) {
      const int kind = vi < nr ? 0 : vi < nr + p.kr ? 1 : 2;
      const int j = kind == 0 ? vi / G : kind == 1 ? vi - nr : vi - nr - p.kr;
      const size_t col = kind == 0 ? (size_t)(kv * G + vi % G) * HD
                         : kind == 1 || p.v_off < 0 ? p.k_off + (size_t)kv * HD
                                                    : p.v_off + (size_t)kv * HD;
      __half* dst = kind == 0 ? sm.q[vi] : kind == 1 ? sm.kloc[j] : sm.vloc[j];
      norm_rope_vec<HD>(p, p.qkv + (size_t)j * p.qkv_stride + col,
                        kind == 0 ? p.w_q : kind == 1 ? p.w_k : nullptr, kind != 2 || p.v_norm != 0,
                        kind != 2, j, dst, lane);
      if (KV8 && kind != 0) {  // the row as the int8 cache stores it
        __syncwarp();
        kv_quantize_row_warp<HD>(dst, kind == 1 ? sm.kloc8[j] : sm.vloc8[j], kind == 1 ? &sm.klocs[j] : &sm.vlocs[j],
                                 lane);
      }
    }
  } else {
    for (int c = tid; c < nr * HD / 8; c += kRingThreads) {
      const int r = c / (HD / 8), part = c - r * (HD / 8);
      const __half* src = p.q16 + ((size_t)(r / G) * p.n_q + kv * G + r % G) * HD + part * 8;
      *reinterpret_cast<uint4*>(&sm.q[r][part * 8]) = *reinterpret_cast<const uint4*>(src);
    }
  }
  __syncthreads();
  if (fused && p.write_kv && gchunk == 0) {
    if (!KV8) {
      for (int c = tid; c < p.kr * HD / 8; c += kRingThreads) {
        const int j = c / (HD / 8), part = c - j * (HD / 8);
        const size_t row = (size_t)wrap(qlm - (p.kr - 1 - j), R);
        *reinterpret_cast<uint4*>(p.k_cache + ((size_t)kv * R + row) * HD + part * 8) =
            *reinterpret_cast<const uint4*>(&sm.kloc[j][part * 8]);
        *reinterpret_cast<uint4*>(p.v_cache + ((size_t)kv * R + row) * HD + part * 8) =
            *reinterpret_cast<const uint4*>(&sm.vloc[j][part * 8]);
      }
    } else {
      int8_t* k8 = reinterpret_cast<int8_t*>(p.k_cache);
      int8_t* v8 = reinterpret_cast<int8_t*>(p.v_cache);
      for (int c = tid; c < p.kr * HD / 16; c += kRingThreads) {
        const int j = c / (HD / 16), part = c - j * (HD / 16);
        const size_t row = (size_t)wrap(qlm - (p.kr - 1 - j), R);
        *reinterpret_cast<uint4*>(k8 + ((size_t)kv * R + row) * HD + part * 16) =
            *reinterpret_cast<const uint4*>(&sm.kloc8[j][part * 16]);
        *reinterpret_cast<uint4*>(v8 + ((size_t)kv * R + row) * HD + part * 16) =
            *reinterpret_cast<const uint4*>(&sm.vloc8[j][part * 16]);
        if (part == 0) {
          p.k_scale[(size_t)kv * R + row] = sm.klocs[j];
          p.v_scale[(size_t)kv * R + row] = sm.vlocs[j];
        }
      }
    }
  }
  pdl_launch_dependents();
  stamp(2);
  asm volatile("cp.async.wait_group 0;" ::: "memory");
  __syncwarp();  // every lane's copies landed: the warp reads all of them

  // ---- scan: per group of B keys, scores for every row, one online-softmax update ----
  float q[ROWS][8];
#pragma unroll
  for (int r = 0; r < ROWS; ++r) {
    if (r < nr) {
      unpack8(*reinterpret_cast<const uint4*>(&sm.q[r][lane * 8]), q[r]);
    } else {
#pragma unroll
      for (int e = 0; e < 8; ++e) q[r][e] = 0.f;
    }
  }
  // key age a is live for row r (query j) iff d = (a - (kr - 1 - j)) mod R
  // satisfies d < W and d <= q_j
  int shift[ROWS];
  int64_t qpos[ROWS];
#pragma unroll
  for (int r = 0; r < ROWS; ++r) {
    const int j = r < nr ? r / G : 0;
    shift[r] = p.kr - 1 - j;
    qpos[r] = pos0 + j;
  }
  float m[ROWS], l[ROWS], acc[ROWS][8];
#pragma unroll
  for (int r = 0; r < ROWS; ++r) {
    m[r] = -INFINITY, l[r] = 0.f;
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[r][e] = 0.f;
  }
#pragma unroll 1
  for (int a0 = wa0; a0 < wa1; a0 += B) {
    uint4 kb[B], vb[B];  // fp16: 8 values; int8: 8 codes in .x/.y
    float ksc[B], vsc[B];  // int8: the rows' scales
#pragma unroll
    for (int i = 0; i < B; ++i) {
      const int a = a0 + i;
      ksc[i] = vsc[i] = 0.f;
      if (a >= wa1) {
        kb[i] = vb[i] = make_uint4(0, 0, 0, 0);
      } else if (!KV8) {
        if (a < first_cached) {  // the block's own rows, from the prologue
          kb[i] = *reinterpret_cast<const uint4*>(&sm.kloc[p.kr - 1 - a][lane * 8]);
          vb[i] = *reinterpret_cast<const uint4*>(&sm.vloc[p.kr - 1 - a][lane * 8]);
        } else {
          kb[i] = *reinterpret_cast<const uint4*>(&sm.kv[warp][a - wa0][0][lane * 8]);
          vb[i] = *reinterpret_cast<const uint4*>(&sm.kv[warp][a - wa0][1][lane * 8]);
        }
      } else {
        uint2 k2, v2;
        if (a < first_cached) {
          k2 = *reinterpret_cast<const uint2*>(&sm.kloc8[p.kr - 1 - a][lane * 8]);
          v2 = *reinterpret_cast<const uint2*>(&sm.vloc8[p.kr - 1 - a][lane * 8]);
          ksc[i] = sm.klocs[p.kr - 1 - a], vsc[i] = sm.vlocs[p.kr - 1 - a];
        } else {
          k2 = *reinterpret_cast<const uint2*>(&sm.kv8[warp][a - wa0][0][lane * 8]);
          v2 = *reinterpret_cast<const uint2*>(&sm.kv8[warp][a - wa0][1][lane * 8]);
          ksc[i] = sm.kvs[warp][a - wa0][0], vsc[i] = sm.kvs[warp][a - wa0][1];
        }
        kb[i] = make_uint4(k2.x, k2.y, 0, 0);
        vb[i] = make_uint4(v2.x, v2.y, 0, 0);
      }
    }
    float s[B * ROWS];
#pragma unroll
    for (int i = 0; i < B; ++i) {
      float kf[8];
      if (KV8) unpack8_i8(make_uint2(kb[i].x, kb[i].y), kf);
      else unpack8(kb[i], kf);
#pragma unroll
      for (int r = 0; r < ROWS; ++r) {
        float t = 0.f;
#pragma unroll
        for (int e = 0; e < 8; ++e) t = fmaf(q[r][e], kf[e], t);
        s[i * ROWS + r] = t;
      }
    }
    warp_allreduce_vec<B * ROWS>(s, lane);
    if (KV8) {  // q . (code * scale) = scale * (q . code)
#pragma unroll
      for (int i = 0; i < B; ++i)
#pragma unroll
        for (int r = 0; r < ROWS; ++r) s[i * ROWS + r] *= ksc[i];
    }
#pragma unroll
    for (int r = 0; r < ROWS; ++r) {
      if (r >= nr) continue;
      float mx = m[r];
#pragma unroll
      for (int i = 0; i < B; ++i) {
        const int d = wrap(a0 + i - shift[r], R);
        const bool live = a0 + i < wa1 && d < W && (int64_t)d <= qpos[r];
        s[i * ROWS + r] = live ? s[i * ROWS + r] : -INFINITY;
        mx = fmaxf(mx, s[i * ROWS + r]);
      }
      if (mx == -INFINITY) continue;  // nothing live yet for this row
      const float scale = __expf(m[r] - mx);
      l[r] *= scale;
#pragma unroll
      for (int e = 0; e < 8; ++e) acc[r][e] *= scale;
      m[r] = mx;
#pragma unroll
      for (int i = 0; i < B; ++i) {
        const float sv = s[i * ROWS + r];
        const float pv = sv == -INFINITY ? 0.f : __expf(sv - mx);
        float vf[8];
        if (KV8) unpack8_i8(make_uint2(vb[i].x, vb[i].y), vf);
        else unpack8(vb[i], vf);
        l[r] += pv;
        const float pw = KV8 ? pv * vsc[i] : pv;  // p * (code * scale)
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[r][e] = fmaf(pw, vf[e], acc[r][e]);
      }
    }
  }

  // ---- merge: warps in shared memory ----
  stamp(3);
  __syncthreads();  // the partials reuse the key buffers
#pragma unroll
  for (int r = 0; r < ROWS; ++r) {
    if (r >= nr) continue;
    float* dst = &sm.part[warp][r][lane * 8];
    *reinterpret_cast<float4*>(dst) = make_float4(acc[r][0], acc[r][1], acc[r][2], acc[r][3]);
    *reinterpret_cast<float4*>(dst + 4) = make_float4(acc[r][4], acc[r][5], acc[r][6], acc[r][7]);
    if (lane == 0) sm.pm[warp][r] = m[r], sm.pl[warp][r] = l[r];
  }
  __syncthreads();
#pragma unroll 1
  for (int idx = tid; idx < nr * HD; idx += kRingThreads) {
    const int r = idx / HD, d = idx - r * HD;
    float mx = -INFINITY;
    for (int w = 0; w < kRingWarps; ++w) mx = fmaxf(mx, sm.pm[w][r]);
    float o = 0.f, lsum = 0.f;
    if (mx != -INFINITY) {
      for (int w = 0; w < kRingWarps; ++w) {
        const float mw = sm.pm[w][r];
        if (mw == -INFINITY) continue;
        const float e = __expf(mw - mx);
        o = fmaf(sm.part[w][r][d], e, o);
        lsum = fmaf(sm.pl[w][r], e, lsum);
      }
    }
    sm.cacc[r][d] = o;
    if (d == 0) sm.cm[r] = mx, sm.cl[r] = lsum;
  }
  // ---- merge: the CL CTAs of the cluster through distributed shared memory ----
  stamp(4);
  cluster_sync();
  stamp(5);
  constexpr int DPC = HD / CL;
  static_assert(ROWS * DPC <= kRingThreads, "one output element per thread");
  // this thread's output element (r, d): its merged sum, weight and maximum
  float o_t = 0.f, l_t = 0.f, m_t = -INFINITY;
  const bool has_t = tid < nr * DPC;
  const int r_t = tid / DPC, d_t = chunk * DPC + (tid - r_t * DPC);
#pragma unroll 1
  for (int idx = tid; idx < nr * DPC; idx += kRingThreads) {
    const int r = idx / DPC, d = chunk * DPC + (idx - r * DPC);
    float mc[CL], mx = -INFINITY;
#pragma unroll
    for (int c = 0; c < CL; ++c) {
      mc[c] = ld_peer_f32(peer_addr(&sm.cm[r], c));
      mx = fmaxf(mx, mc[c]);
    }
    float o = 0.f, lsum = 0.f;
#pragma unroll
    for (int c = 0; c < CL; ++c) {
      if (mc[c] == -INFINITY) continue;
      const float e = __expf(mc[c] - mx);
      lsum = fmaf(ld_peer_f32(peer_addr(&sm.cl[r], c)), e, lsum);
      o = fmaf(ld_peer_f32(peer_addr(&sm.cacc[r][d], c)), e, o);
    }
    if (S == 1) {
      const int j = r / G;
      p.out[((size_t)j * p.n_q + kv * G + r % G) * HD + d] = __float2half_rn(o / lsum);
    }
    o_t = o, l_t = lsum, m_t = mx;
  }
  stamp(6);
  cluster_sync();  // peers may read this CTA's shared memory until here
  stamp(7);
  if (S == 1) return;
  // ---- merge of the S clusters of this KV head: the last CTA of each
  // (head, output slice) group to finish combines the S partials ----
  __shared__ int s_ticket;
  float* xo = p.part_acc + (size_t)kv * S * ROWS * HD;  // [S][ROWS][HD]
  float* xml = p.part_ml + (size_t)kv * S * ROWS * 2;   // [S][ROWS][2]
  if (has_t) {
    xo[((size_t)half * ROWS + r_t) * HD + d_t] = o_t;
    if (d_t == chunk * DPC) xml[(half * ROWS + r_t) * 2] = m_t, xml[(half * ROWS + r_t) * 2 + 1] = l_t;
  }
  __threadfence();
  __syncthreads();
  if (tid == 0) s_ticket = atomicAdd(&p.counters[kv * CL + chunk], 1);
  __syncthreads();
  if (s_ticket != S - 1) return;
  __threadfence();
  if (has_t) {
    // in cluster order whichever CTA merges, so the result does not depend on timing
    float mh[S], mm = -INFINITY;
#pragma unroll
    for (int h = 0; h < S; ++h) {
      mh[h] = h == half ? m_t : __ldcg(xml + (h * ROWS + r_t) * 2);
      mm = fmaxf(mm, mh[h]);
    }
    float o = 0.f, l = 0.f;
#pragma unroll
    for (int h = 0; h < S; ++h) {
      const float e = mh[h] == -INFINITY ? 0.f : __expf(mh[h] - mm);
      const float oh = h == half ? o_t : __ldcg(xo + ((size_t)h * ROWS + r_t) * HD + d_t);
      const float lh = h == half ? l_t : __ldcg(xml + (h * ROWS + r_t) * 2 + 1);
      o = fmaf(oh, e, o);
      l = fmaf(lh, e, l);
    }
    const int j = r_t / G;
    p.out[((size_t)j * p.n_q + kv * G + r_t % G) * HD + d_t] = __float2half_rn(o / l);
  }
  if (tid == 0) p.counters[kv * CL + chunk] = 0;  // ready for the next layer
}

template <int HD, int ROWS, int CL, int S, bool KV8 = false>
cudaError_t configure_ring() {
  static bool configured = false;
  if (configured) return cudaSuccess;
  auto kern = attn_ring_kernel<HD, ROWS, CL, S, KV8>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)sizeof(RingSmem<HD, ROWS>));
  if (e == cudaSuccess && CL > 8) e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
  if (e == cudaSuccess) configured = true;
  return e;
}

template <int HD, int ROWS, int CL, int S>
cudaLaunchConfig_t ring_config(const AttnParams& p, cudaStream_t st, bool pdl, cudaLaunchAttribute (&attr)[2]) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(p.n_kv, CL * S, 1);
  cfg.blockDim = dim3(kRingThreads);
  cfg.dynamicSmemBytes = sizeof(RingSmem<HD, ROWS>);
  cfg.stream = st;
  int na = 0;
  if (pdl) {
    attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[na].val.programmaticStreamSerializationAllowed = 1;
    ++na;
  }
  attr[na].id = cudaLaunchAttributeClusterDimension;
  attr[na].val.clusterDim.x = 1;
  attr[na].val.clusterDim.y = CL;
  attr[na].val.clusterDim.z = 1;
  ++na;
  cfg.attrs = attr;
  cfg.numAttrs = na;
  return cfg;
}

template <int HD, int ROWS, int CL, int S, bool KV8>
cudaError_t launch_ring_t(const AttnParams& p, cudaStream_t st, bool pdl) {
  cudaError_t e = configure_ring<HD, ROWS, CL, S, KV8>();
  if (e != cudaSuccess) return e;
  cudaLaunchAttribute attr[2];
  const cudaLaunchConfig_t cfg = ring_config<HD, ROWS, CL, S>(p, st, pdl, attr);
  return cudaLaunchKernelEx(&cfg, attn_ring_kernel<HD, ROWS, CL, S, KV8>, p);
}

// CTAs per KV head: 16 (a non-portable cluster, twice the SMs on the scan) when
// eight such clusters fit on the device at once, else 8.
int ring_cluster_size() {
  static int cl = 0;
  if (cl) return cl;
  int pick = 0;
  {
    pick = 8;
    AttnParams p{};
    p.n_kv = 8;
    int n = 0;
    cudaLaunchAttribute attr[2];
    if (configure_ring<256, 2, 16, 1>() == cudaSuccess) {
      const cudaLaunchConfig_t cfg = ring_config<256, 2, 16, 1>(p, 0, false, attr);
      if (cudaOccupancyMaxActiveClusters(&n, attn_ring_kernel<256, 2, 16, 1, false>, &cfg) == cudaSuccess && n >= 8)
        pick = 16;
    }
    cudaGetLastError();  // a refused query leaves no error behind
  }
  cl = pick;
  return cl;
}

}  // namespace

int ring_decode_rows(const AttnParams& p) {
  const int rows = p.kr * (p.n_q / p.n_kv);
  if (!p.ring || p.hd != 256 || rows > 4) return 0;
  // keys per warp: the scan covers window + kr - 1 ages in kAttnCluster CTAs
  const int64_t nscan = p.window + p.kr - 1, per_cta = (nscan + kAttnCluster - 1) / kAttnCluster;
  if ((per_cta + kRingWarps - 1) / kRingWarps > kRingKeysPerWarp) return 0;
  return rows <= 1 ? 1 : rows <= 2 ? 2 : 4;
}

// Four clusters of 4 CTAs per KV head fit at once for this many KV heads
// (cluster placement is per GPC, so the SM count alone does not tell).
bool ring_split_fits(int n_kv) {
  static int max_clusters = -1;
  if (max_clusters < 0) {
    max_clusters = 0;
    AttnParams p{};
    p.n_kv = 8;
    cudaLaunchAttribute attr[2];
    if (configure_ring<256, 2, 4, 4>() == cudaSuccess) {
      const cudaLaunchConfig_t cfg = ring_config<256, 2, 4, 4>(p, 0, false, attr);
      int n = 0;
      if (cudaOccupancyMaxActiveClusters(&n, attn_ring_kernel<256, 2, 4, 4, false>, &cfg) == cudaSuccess) max_clusters = n;
    }
    cudaGetLastError();
  }
  return n_kv * 4 <= max_clusters;
}

namespace {
template <bool KV8>
cudaError_t launch_ring_rows(const AttnParams& p, bool split, bool wide, cudaStream_t st, bool pdl) {
  switch (ring_decode_rows(p)) {
    case 1:
      return split ? launch_ring_t<256, 1, 4, 4, KV8>(p, st, pdl)
             : wide ? launch_ring_t<256, 1, 16, 1, KV8>(p, st, pdl) : launch_ring_t<256, 1, 8, 1, KV8>(p, st, pdl);
    case 2:
      return split ? launch_ring_t<256, 2, 4, 4, KV8>(p, st, pdl)
             : wide ? launch_ring_t<256, 2, 16, 1, KV8>(p, st, pdl) : launch_ring_t<256, 2, 8, 1, KV8>(p, st, pdl);
    case 4:
      return split ? launch_ring_t<256, 4, 4, 4, KV8>(p, st, pdl)
             : wide ? launch_ring_t<256, 4, 16, 1, KV8>(p, st, pdl) : launch_ring_t<256, 4, 8, 1, KV8>(p, st, pdl);
    default: return cudaErrorInvalidValue;
  }
}
}  // namespace

cudaError_t launch_attention_ring(const AttnParams& p, cudaStream_t st, bool pdl) {
  // 16 CTAs per KV head (four clusters of 4, merged through the caller's
  // counters and scratch) when they all fit at once: one SM reads about
  // 50 GB/s, so the scan wants as many SMs as it can get; else one cluster of
  // 16 or 8
  const bool split = p.ring_split == 2 && ring_split_fits(p.n_kv);
  const bool wide = !split && ring_cluster_size() == 16;
  if (p.kv8) return launch_ring_rows<true>(p, split, wide, st, pdl);
  return launch_ring_rows<false>(p, split, wide, st, pdl);
}

}  // namespace q4g
