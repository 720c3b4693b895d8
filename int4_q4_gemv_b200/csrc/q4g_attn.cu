// Split-KV flash-decode attention for the sliding ring and the full layers.
//
// Operation ("Gemma 4 12B" page, flash-decode paragraph: GQA decode over the
// cache, scale 1.0, fp32 online softmax, the KV scan split across cooperating
// groups; "Gemma-4-12B-CoreAI", v5 section: slot = position mod R, implied
// position p = q - ((q - j) mod R), window test q - p < W):
//   o[row] = sum_key softmax_key(q[row] . k[key]) v[key]
// over the live keys of each query row.
//
// Grid (KV head, chunk of keys, group of query rows). The query rows of one KV
// head -- (verify row j, query head h of the group) -- form the M dimension of
// tensor-core tiles (mma.sync m16n8k16, fp16 in, fp32 accumulate): the GQA
// group is folded into the query so every key row is read once for all its
// query heads. Keys stream through shared memory in tiles of 64 with cp.async.
// The probabilities enter the P.V product as fp16 hi + lo parts, so P carries
// ~22 bits. Each CTA writes (m, l, acc) partials; a combine pass (the last CTA
// of a ring head, or a separate kernel for the full layers) merges them in a
// fixed order.
//
// With the fused QKV epilogue (qkv != NULL) the prologue computes, from the raw
// projections: per-head RMSNorm of q (learned gains) and RoPE, RMSNorm of k and
// RoPE, and V = scale-free RMSNorm of the v projection or, on full layers
// (attention_k_eq_v), of the raw k projection. Chunk 0 writes the block's K/V
// rows to the cache; every CTA reads this block's own rows from shared memory.
#include "q4g_common.cuh"
#include "q4g_internal.h"

namespace q4g {

namespace {

constexpr int TK = 64;   // keys per tile
constexpr int MROWS = 32;  // query rows per CTA (two m16 tiles)

Q4G_DEV uint32_t saddr(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }

Q4G_DEV void ldsm_x4(uint32_t (&r)[4], const void* p) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(saddr(p)));
}
Q4G_DEV void ldsm_x2(uint32_t (&r)[2], const void* p) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x2.shared.b16 {%0, %1}, [%2];"
               : "=r"(r[0]), "=r"(r[1])
               : "r"(saddr(p)));
}
Q4G_DEV void ldsm_x2_t(uint32_t (&r)[2], const void* p) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x2.trans.shared.b16 {%0, %1}, [%2];"
               : "=r"(r[0]), "=r"(r[1])
               : "r"(saddr(p)));
}
Q4G_DEV void mma16816(float (&c)[4], const uint32_t (&a)[4], const uint32_t (&b)[2]) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
      "{%8, %9}, {%0, %1, %2, %3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}
Q4G_DEV void cp_async16(void* dst, const void* src, bool valid) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(saddr(dst)), "l"(src),
               "r"(valid ? 16 : 0));
}
Q4G_DEV void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
Q4G_DEV void cp_async4(void* dst, const void* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(saddr(dst)), "l"(src) : "memory");
}

template <int N>
Q4G_DEV void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

template <int HD>
struct Smem {
  static constexpr int LD = HD + 8;  // padded row (halves): conflict-free ldmatrix
  __half q[MROWS][LD];
  __half k[TK][LD];
  __half v[TK][LD];
  __half phi[MROWS][TK + 8];
  __half plo[MROWS][TK + 8];
  __half kloc[kMaxRows][HD];
  __half vloc[kMaxRows][HD];
  alignas(16) int8_t kloc8[kMaxRows][HD];  // int8 cache: the block's rows as stored
  alignas(16) int8_t vloc8[kMaxRows][HD];
  float klocs[kMaxRows], vlocs[kMaxRows];
  float ks[2][TK], vs[2][TK];  // int8 cache: the tile's row scales (0 for no key)
  int32_t kidx[2][TK];  // slot (ring) or position (linear); -1: no key
  float red[8][MROWS];
  float m_run[MROWS], l_run[MROWS], scale[MROWS];
  int ticket;
};

// int8 cache: a tile of TK code rows staged at the end of an fp16 tile's storage
// (byte offset kStage8 of sm.k or sm.v) becomes the fp16 tile (exact: |code| <=
// 127). The fp16 rows of the first TK/2 keys end below the staging area; those of
// the other keys overlap it, so their codes are read into registers before any
// of them is written. Ends with __syncthreads.
template <int HD>
Q4G_DEV void convert_tile8(__half (*dst)[HD + 8], const int8_t* stage, int tid) {
  constexpr int CPR8 = HD / 16;                  // 16-code pieces per row
  constexpr int NHALF = (TK / 2) * CPR8;         // pieces of half a tile
  constexpr int NPER = NHALF / kThreads;
  static_assert(NHALF % kThreads == 0, "whole pieces per thread");
  auto put = [&](int key, int part, uint4 u) {
    const int8_t* c = reinterpret_cast<const int8_t*>(&u);
    __half2 h[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) h[i] = __floats2half2_rn((float)c[2 * i], (float)c[2 * i + 1]);
    uint4* d = reinterpret_cast<uint4*>(&dst[key][part * 16]);
    d[0] = *reinterpret_cast<const uint4*>(&h[0]);
    d[1] = *reinterpret_cast<const uint4*>(&h[4]);
  };
#pragma unroll
  for (int i = 0; i < NPER; ++i) {
    const int c = tid + i * kThreads, key = c / CPR8, part = c - key * CPR8;
    put(key, part, *reinterpret_cast<const uint4*>(stage + (size_t)key * HD + part * 16));
  }
  uint4 u[NPER];
#pragma unroll
  for (int i = 0; i < NPER; ++i) {
    const int c = tid + i * kThreads, key = TK / 2 + c / CPR8, part = c % CPR8;
    u[i] = *reinterpret_cast<const uint4*>(stage + (size_t)key * HD + part * 16);
  }
  __syncthreads();
#pragma unroll
  for (int i = 0; i < NPER; ++i) {
    const int c = tid + i * kThreads, key = TK / 2 + c / CPR8, part = c % CPR8;
    put(key, part, u[i]);
  }
  __syncthreads();
}

// CL > 0: the grid's y dimension is one cluster of CL CTAs (n_chunks == CL);
// the chunk partials are merged through distributed shared memory.
template <int HD, int CL, bool KV8>
__global__ void __launch_bounds__(kThreads, 1) attn_kernel(const AttnParams p) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  Smem<HD>& sm = *reinterpret_cast<Smem<HD>*>(smem_raw);
  constexpr int LD = Smem<HD>::LD;
  constexpr size_t kStage8 = sizeof(sm.k) - (size_t)TK * HD;  // int8 staging inside sm.k / sm.v
  static_assert(kStage8 >= (size_t)(TK / 2) * LD * 2, "staging above the first half tile");
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int kv = blockIdx.x, chunk = blockIdx.y, mg = blockIdx.z;
  const int G = p.n_q / p.n_kv;
  const int M = p.kr * G;                      // query rows of this KV head
  const int row0 = mg * MROWS;                 // first query row of this CTA
  const int nrows = min(MROWS, M - row0);

  pdl_wait();
  const int64_t pos0 = p.pos_dev ? *p.pos_dev : p.pos0;
  const int64_t q_last = pos0 + p.kr - 1;
  const bool fused = p.qkv != nullptr;
  // 32-bit index arithmetic: the host keeps R, the window and linear positions
  // below 2^30; ring positions may be any int64, only q_last mod R enters.
  const int R = (int)p.cache_rows, W = (int)p.window;
  const int qlm = p.ring ? (int)(q_last % p.cache_rows) : 0;  // slot of the newest key

  // ---- key scan of this chunk: ring scans ages, linear scans positions ----
  const int nscan = p.ring ? (int)min((int64_t)W + p.kr - 1, q_last + 1) : (int)(q_last + 1);
  // chunks are whole tiles; trailing chunks may be empty
  const int cs = ((nscan + p.n_chunks - 1) / p.n_chunks + TK - 1) / TK * TK;
  const int a_begin = min(nscan, chunk * cs);
  const int a_end = min(nscan, a_begin + cs);
  const int ntiles = (a_end - a_begin + TK - 1) / TK;

  auto key_row = [&](int a) -> int {  // cache row of scan index a (age for the ring)
    return p.ring ? wrap(qlm - a, R) : a;
  };
  auto key_is_local = [&](int a) -> int {  // block row index or -1
    if (!fused) return -1;
    if (p.ring) return a < p.kr ? p.kr - 1 - a : -1;
    return a >= (int)pos0 ? a - (int)pos0 : -1;
  };

  const float* ksc = KV8 ? p.k_scale + (size_t)kv * p.cache_rows : nullptr;
  const float* vsc = KV8 ? p.v_scale + (size_t)kv * p.cache_rows : nullptr;
  constexpr int CPR = HD / 8;  // 16-byte chunks per row
  constexpr int CPR8 = HD / 16;  // 16-byte chunks per int8 row

  // mode 0: cache rows only (the block's own rows do not exist yet);
  // 1: the block's own rows only, from shared memory; 2: both
  constexpr int kRowBytes = KV8 ? HD : HD * 2;
  constexpr int CPRB = kRowBytes / 16;      // 16-byte pieces per row
  constexpr int KPP = kThreads / CPRB;      // keys per pass of the CTA
  static_assert(kThreads % CPRB == 0 && TK % KPP == 0, "whole rows per pass");
  const int my_part = tid % CPRB, my_key = tid / CPRB;  // a thread's piece in every pass
  auto load_tile = [&](int t, bool kpart, int mode) {
    const int buf = t & 1;
    const int a0 = a_begin + t * TK;
    if (kpart && tid < TK && mode != 1) {
      const int a = a0 + tid;
      sm.kidx[buf][tid] = a < a_end ? key_row(a) : -1;
    }
    if (KV8 && tid < TK) {  // the rows' scales
      const int a = a0 + tid;
      const bool in = a < a_end;
      const int loc = in ? key_is_local(a) : -1;
      float* sd = kpart ? &sm.ks[buf][tid] : &sm.vs[buf][tid];
      if (loc >= 0) {
        if (mode != 0) *sd = kpart ? sm.klocs[loc] : sm.vlocs[loc];
      } else if (mode != 1) {
        if (in) cp_async4(sd, (kpart ? ksc : vsc) + key_row(a));
        else *sd = 0.f;
      }
    }
    unsigned char* dst = reinterpret_cast<unsigned char*>(kpart ? &sm.k[0][0] : &sm.v[0][0]);
    if (KV8) dst += kStage8;
    constexpr size_t kDstRow = KV8 ? HD : (size_t)LD * 2;  // bytes between staged rows
    const unsigned char* src = reinterpret_cast<const unsigned char*>(kpart ? p.k_cache : p.v_cache) +
                               (size_t)kv * p.cache_rows * kRowBytes;
    // CTA-uniform: keys past the chunk's end, or the block's own rows, in this tile?
    const bool tail = a0 + TK > a_end;
    const bool own = fused && (p.ring ? a0 < p.kr : (a0 + TK > (int)pos0 && a0 < (int)pos0 + p.kr));
    if (!tail && !own) {  // every key a cache row: no per-piece tests
      if (mode == 1) return;
      // kept rolled: the unrolled form issues each thread's copies as one burst,
      // which measured 15-25% slower at 2-7 tiles per CTA (and no faster elsewhere)
#pragma unroll 1
      for (int i = 0; i < TK / KPP; ++i) {
        const int key = my_key + i * KPP;
        cp_async16(dst + key * kDstRow + my_part * 16, src + (size_t)key_row(a0 + key) * kRowBytes + my_part * 16,
                   true);
      }
      return;
    }
    for (int i = 0; i < TK / KPP; ++i) {
      const int key = my_key + i * KPP;
      const int a = a0 + key;
      const bool in = a < a_end;
      const int loc = in ? key_is_local(a) : -1;
      unsigned char* d = dst + key * kDstRow + my_part * 16;
      if (loc >= 0) {
        if (mode != 0) {
          const void* l = KV8 ? (const void*)(kpart ? sm.kloc8[loc] : sm.vloc8[loc])
                              : (const void*)(kpart ? sm.kloc[loc] : sm.vloc[loc]);
          *reinterpret_cast<uint4*>(d) = reinterpret_cast<const uint4*>(l)[my_part];
        }
      } else if (mode != 1) {  // a cache row, or zeros for no key
        cp_async16(d, in ? src + (size_t)key_row(a) * kRowBytes + my_part * 16 : src, in);
      }
    }
  };

  // first tile's cache rows go out before the prologue
  if (ntiles > 0) {
    load_tile(0, true, 0);
    cp_async_commit();
    load_tile(0, false, 0);
    cp_async_commit();
  }
  // ---- prologue: queries (and this block's K/V rows) into shared memory ----
  if (fused) {
    const int nvec = nrows + 2 * p.kr;
    constexpr int E = HD / 64;  // elements per lane per half
    for (int vi = warp; vi < nvec; vi += kThreads / 32) {
      int j, kind;  // kind 0: q row, 1: k, 2: v
      const float* src;
      if (vi < nrows) {
        const int r = row0 + vi;
        j = r / G;
        kind = 0;
        src = p.qkv + (size_t)j * p.qkv_stride + (size_t)(kv * G + r % G) * HD;
      } else if (vi < nrows + p.kr) {
        j = vi - nrows;
        kind = 1;
        src = p.qkv + (size_t)j * p.qkv_stride + p.k_off + (size_t)kv * HD;
      } else {
        j = vi - nrows - p.kr;
        kind = 2;
        src = p.qkv + (size_t)j * p.qkv_stride +
              (p.v_off >= 0 ? p.v_off + (size_t)kv * HD : p.k_off + (size_t)kv * HD);
      }
      float lo[E], hi[E];
      float ss = 0.f;
#pragma unroll
      for (int e = 0; e < E; ++e) {
        lo[e] = src[lane * E + e];
        hi[e] = src[HD / 2 + lane * E + e];
        ss = fmaf(lo[e], lo[e], ss);
        ss = fmaf(hi[e], hi[e], ss);
      }
      const bool do_norm = kind != 2 || p.v_norm;
      const float inv = do_norm ? rms_inv(warp_sum(ss), HD, p.eps) : 1.0f;
      const float* gain = kind == 0 ? p.w_q : kind == 1 ? p.w_k : nullptr;
#pragma unroll
      for (int e = 0; e < E; ++e) {
        const int i = lane * E + e;
        float a = __fmul_rn(lo[e], inv), b = __fmul_rn(hi[e], inv);
        if (gain) a = __fmul_rn(a, gain[i]), b = __fmul_rn(b, gain[HD / 2 + i]);
        if (kind != 2 && i < p.rope_pairs) {
          const float2 cs2 = p.rope[(size_t)j * p.rope_pairs + i];
          const float ra = a * cs2.x - b * cs2.y;
          const float rb = b * cs2.x + a * cs2.y;
          a = ra, b = rb;
        }
        __half* dst = kind == 0 ? sm.q[vi] : kind == 1 ? sm.kloc[j] : sm.vloc[j];
        dst[i] = __float2half_rn(a);
        dst[HD / 2 + i] = __float2half_rn(b);
      }
      if (KV8 && kind != 0) {  // the row as the int8 cache stores it
        __syncwarp();
        kv_quantize_row_warp<HD>(kind == 1 ? sm.kloc[j] : sm.vloc[j], kind == 1 ? sm.kloc8[j] : sm.vloc8[j],
                                 kind == 1 ? &sm.klocs[j] : &sm.vlocs[j], lane);
      }
    }
  } else {
    for (int c = tid; c < nrows * CPR; c += kThreads) {
      const int r = c / CPR, part = c - r * CPR;
      const int gr = row0 + r;
      const __half* src = p.q16 + ((size_t)(gr / G) * p.n_q + kv * G + gr % G) * HD + part * 8;
      *reinterpret_cast<uint4*>(&sm.q[r][part * 8]) = *reinterpret_cast<const uint4*>(src);
    }
  }
  // zero the unused query rows of the m16 tiles read below (their results are
  // never written); rows are LD halves, a multiple of 8
  {
    const int zrows = ((nrows + 15) / 16) * 16 - nrows;
    uint4* z = reinterpret_cast<uint4*>(&sm.q[nrows][0]);
    for (int c = tid; c < zrows * LD / 8; c += kThreads) z[c] = make_uint4(0, 0, 0, 0);
  }
  if (tid < MROWS) sm.m_run[tid] = -INFINITY, sm.l_run[tid] = 0.f;
  __syncthreads();

  if (KV8 && fused && p.write_kv && chunk == 0 && mg == 0) {
    int8_t* k8 = reinterpret_cast<int8_t*>(p.k_cache);
    int8_t* v8 = reinterpret_cast<int8_t*>(p.v_cache);
    for (int c = tid; c < p.kr * CPR8; c += kThreads) {
      const int j = c / CPR8, part = c - j * CPR8;
      const int64_t pos = pos0 + j;
      const int64_t row = p.ring ? (int64_t)wrap(qlm - (p.kr - 1 - j), R) : pos;
      *reinterpret_cast<uint4*>(k8 + ((size_t)kv * p.cache_rows + row) * HD + part * 16) =
          *reinterpret_cast<const uint4*>(&sm.kloc8[j][part * 16]);
      *reinterpret_cast<uint4*>(v8 + ((size_t)kv * p.cache_rows + row) * HD + part * 16) =
          *reinterpret_cast<const uint4*>(&sm.vloc8[j][part * 16]);
      if (part == 0) {
        p.k_scale[(size_t)kv * p.cache_rows + row] = sm.klocs[j];
        p.v_scale[(size_t)kv * p.cache_rows + row] = sm.vlocs[j];
      }
    }
  } else if (fused && p.write_kv && chunk == 0 && mg == 0) {
    for (int c = tid; c < p.kr * CPR; c += kThreads) {
      const int j = c / CPR, part = c - j * CPR;
      const int64_t pos = pos0 + j;
      const int64_t row = p.ring ? (int64_t)wrap(qlm - (p.kr - 1 - j), R) : pos;
      *reinterpret_cast<uint4*>(p.k_cache + ((size_t)kv * p.cache_rows + row) * HD + part * 8) =
          *reinterpret_cast<const uint4*>(&sm.kloc[j][part * 8]);
      *reinterpret_cast<uint4*>(p.v_cache + ((size_t)kv * p.cache_rows + row) * HD + part * 8) =
          *reinterpret_cast<const uint4*>(&sm.vloc[j][part * 8]);
    }
  }
  pdl_launch_dependents();

  // ---- tile loop ----
  constexpr int NT_PV = HD / 64;   // 8-dim n-tiles per warp in P.V
  const int mtiles = (nrows + 15) / 16;
  float oacc[2][NT_PV][4];
#pragma unroll
  for (int a = 0; a < 2; ++a)
#pragma unroll
    for (int b = 0; b < NT_PV; ++b)
#pragma unroll
      for (int c = 0; c < 4; ++c) oacc[a][b][c] = 0.f;

  const int g4 = lane >> 2, t4 = lane & 3;
  for (int t = 0; t < ntiles; ++t) {
    const int buf = t & 1;
    if (t == 0 && fused) {  // this block's own rows, now that they exist
      load_tile(0, true, 1);
      load_tile(0, false, 1);
    }
    cp_async_wait<1>();
    __syncthreads();
    if (KV8) convert_tile8<HD>(sm.k, reinterpret_cast<const int8_t*>(&sm.k[0][0]) + kStage8, tid);

    // scores S[row][key] for key n-tile `warp`
    // (even and odd k steps accumulate separately: two independent mma chains)
    float s[2][4];
#pragma unroll
    for (int mt = 0; mt < 2; ++mt) {
      float s1[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int c = 0; c < 4; ++c) s[mt][c] = 0.f;
      if (mt < mtiles) {
#pragma unroll 4
        for (int kk = 0; kk < HD / 16; kk += 2) {
          uint32_t a0[4], b0[2], a1[4], b1[2];
          ldsm_x4(a0, &sm.q[mt * 16 + (lane & 15)][kk * 16 + (lane >> 4) * 8]);
          ldsm_x2(b0, &sm.k[warp * 8 + (lane & 7)][kk * 16 + ((lane >> 3) & 1) * 8]);
          ldsm_x4(a1, &sm.q[mt * 16 + (lane & 15)][(kk + 1) * 16 + (lane >> 4) * 8]);
          ldsm_x2(b1, &sm.k[warp * 8 + (lane & 7)][(kk + 1) * 16 + ((lane >> 3) & 1) * 8]);
          mma16816(s[mt], a0, b0);
          mma16816(s1, a1, b1);
        }
#pragma unroll
        for (int c = 0; c < 4; ++c) s[mt][c] += s1[c];
      }
    }
    __syncthreads();  // K tile consumed
    if (t + 1 < ntiles) {
      load_tile(t + 1, true, 2);
    }
    cp_async_commit();

    // mask and per-tile row maxima (rows of unused m-tiles are never read)
#pragma unroll
    for (int mt = 0; mt < 2; ++mt) {
      if (mt >= mtiles) break;
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        const int lr = mt * 16 + g4 + hh * 8;  // local query row
        const int gr = row0 + lr;
        const int j = gr / G;
        const int64_t qj = pos0 + j;
        // ring: key at slot s has implied position qj - d, d = (qj - s) mod R;
        // it is live when d < W and qj - d >= 0
        const int qjm = p.ring ? wrap(qlm - (p.kr - 1 - j), R) : 0;
        float mx = -INFINITY;
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int key = warp * 8 + t4 * 2 + e;
          const int ks = sm.kidx[buf][key];
          bool live = lr < nrows && ks >= 0;
          if (live) {
            if (p.ring) {
              const int d = wrap(qjm - ks, R);
              live = d < W && (int64_t)d <= qj;
            } else {
              live = (int64_t)ks <= qj;
            }
          }
          float& v = s[mt][hh * 2 + e];
          if (KV8) v *= sm.ks[buf][key];  // q . (code * scale)
          v = live ? v : -INFINITY;
          mx = fmaxf(mx, v);
        }
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
        if (t4 == 0) sm.red[warp][lr] = mx;
      }
    }
    __syncthreads();
    if (tid < MROWS) {
      float mx = sm.red[0][tid];
#pragma unroll
      for (int w = 1; w < 8; ++w) mx = fmaxf(mx, sm.red[w][tid]);
      const float mold = sm.m_run[tid];
      const float mnew = fmaxf(mold, mx);
      sm.scale[tid] = mnew == -INFINITY ? 1.0f : __expf(mold - mnew);
      sm.m_run[tid] = mnew;
    }
    __syncthreads();
    // probabilities (fp16 hi + lo) and per-tile row sums
#pragma unroll
    for (int mt = 0; mt < 2; ++mt) {
      if (mt >= mtiles) break;
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        const int lr = mt * 16 + g4 + hh * 8;
        const float mrow = sm.m_run[lr];
        float sum = 0.f;
        __half2 ph, pl;
        float pv[2];
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const float v = s[mt][hh * 2 + e];
          pv[e] = (v == -INFINITY) ? 0.f : __expf(v - mrow);
          sum += pv[e];
        }
        if (KV8) {  // p * (code * scale): the V scale joins P; the row sum keeps p
          pv[0] *= sm.vs[buf][warp * 8 + t4 * 2];
          pv[1] *= sm.vs[buf][warp * 8 + t4 * 2 + 1];
        }
        ph = __floats2half2_rn(pv[0], pv[1]);
        const float2 phf = __half22float2(ph);
        pl = __floats2half2_rn(pv[0] - phf.x, pv[1] - phf.y);
        *reinterpret_cast<__half2*>(&sm.phi[lr][warp * 8 + t4 * 2]) = ph;
        *reinterpret_cast<__half2*>(&sm.plo[lr][warp * 8 + t4 * 2]) = pl;
        sum += __shfl_xor_sync(0xffffffffu, sum, 1);
        sum += __shfl_xor_sync(0xffffffffu, sum, 2);
        if (t4 == 0) sm.red[warp][lr] = sum;
      }
    }
    cp_async_wait<1>();  // V tile of this step (the next K may still fly)
    __syncthreads();
    if (KV8) convert_tile8<HD>(sm.v, reinterpret_cast<const int8_t*>(&sm.v[0][0]) + kStage8, tid);
    if (tid < MROWS) {
      float sum = 0.f;
#pragma unroll
      for (int w = 0; w < 8; ++w) sum += sm.red[w][tid];
      sm.l_run[tid] = sm.l_run[tid] * sm.scale[tid] + sum;
    }
    // O = O * scale + P . V   (warp owns dims [warp*HD/8, (warp+1)*HD/8))
#pragma unroll
    for (int mt = 0; mt < 2; ++mt) {
      if (mt < mtiles) {
        const float sc0 = sm.scale[mt * 16 + g4], sc1 = sm.scale[mt * 16 + g4 + 8];
#pragma unroll
        for (int nt = 0; nt < NT_PV; ++nt) {
          oacc[mt][nt][0] *= sc0, oacc[mt][nt][1] *= sc0;
          oacc[mt][nt][2] *= sc1, oacc[mt][nt][3] *= sc1;
        }
#pragma unroll
        for (int ks = 0; ks < TK / 16; ++ks) {
          uint32_t ah[4], al[4];
          ldsm_x4(ah, &sm.phi[mt * 16 + (lane & 15)][ks * 16 + (lane >> 4) * 8]);
          ldsm_x4(al, &sm.plo[mt * 16 + (lane & 15)][ks * 16 + (lane >> 4) * 8]);
#pragma unroll
          for (int nt = 0; nt < NT_PV; ++nt) {
            uint32_t b[2];
            ldsm_x2_t(b, &sm.v[ks * 16 + (lane & 15)][warp * (HD / 8) + nt * 8]);
            mma16816(oacc[mt][nt], ah, b);
            mma16816(oacc[mt][nt], al, b);
          }
        }
      }
    }
    __syncthreads();  // V tile and P consumed
    if (t + 1 < ntiles) load_tile(t + 1, false, 2);
    cp_async_commit();
  }
  cp_async_wait<0>();

  if (CL > 0) {
    // ---- merge the CL chunk partials of this KV head through DSMEM ----
    __syncthreads();  // every warp is done with the K tile, reused below
    float* pacc = reinterpret_cast<float*>(&sm.k[0][0]);  // [nrows][HD] unnormalised partial
#pragma unroll
    for (int mt = 0; mt < 2; ++mt) {  // constant bounds: oacc stays in registers
      if (mt >= mtiles) break;
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        const int lr = mt * 16 + g4 + hh * 8;
        if (lr < nrows) {
#pragma unroll
          for (int nt = 0; nt < NT_PV; ++nt) {
            const int d = warp * (HD / 8) + nt * 8 + t4 * 2;
            *reinterpret_cast<float2*>(pacc + (size_t)lr * HD + d) =
                make_float2(oacc[mt][nt][hh * 2], oacc[mt][nt][hh * 2 + 1]);
          }
        }
      }
    }
    cluster_sync();  // all partials and (m, l) of the cluster are visible
    constexpr int DPC = HD / (CL > 0 ? CL : 1);  // output dims merged by this CTA
    const uint32_t rank = cluster_rank();
    for (int w = tid; w < nrows * DPC; w += kThreads) {
      const int lr = w / DPC, d = (int)rank * DPC + (w - lr * DPC);
      float mc[CL > 0 ? CL : 1], mx = -INFINITY;
#pragma unroll
      for (int c = 0; c < CL; ++c) {
        mc[c] = ld_peer_f32(peer_addr(&sm.m_run[lr], c));
        mx = fmaxf(mx, mc[c]);
      }
      float l = 0.f, o = 0.f;
#pragma unroll
      for (int c = 0; c < CL; ++c) {
        if (mc[c] == -INFINITY) continue;
        const float e = __expf(mc[c] - mx);
        l = fmaf(ld_peer_f32(peer_addr(&sm.l_run[lr], c)), e, l);
        o = fmaf(ld_peer_f32(peer_addr(pacc + (size_t)lr * HD + d, c)), e, o);
      }
      const int gr = row0 + lr;
      const int orow = (gr / G) * p.n_q + kv * G + gr % G;
      p.out[(size_t)orow * HD + d] = __float2half_rn(o / l);
    }
    cluster_sync();  // peers may still read this CTA's shared memory until here
    return;
  }

  // ---- partials ----
  const int nq_rows = p.kr * p.n_q;
#pragma unroll
  for (int mt = 0; mt < 2; ++mt) {  // constant bounds: oacc stays in registers
    if (mt >= mtiles) break;
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
      const int lr = mt * 16 + g4 + hh * 8;
      if (lr < nrows) {
        const int gr = row0 + lr;
        const int orow = (gr / G) * p.n_q + kv * G + gr % G;
        float* acc = p.part_acc + ((size_t)orow * p.n_chunks + chunk) * HD;
#pragma unroll
        for (int nt = 0; nt < NT_PV; ++nt) {
          const int d = warp * (HD / 8) + nt * 8 + t4 * 2;
          *reinterpret_cast<float2*>(acc + d) = make_float2(oacc[mt][nt][hh * 2], oacc[mt][nt][hh * 2 + 1]);
        }
      }
    }
  }
  if (tid < nrows) {
    const int gr = row0 + tid;
    const int orow = (gr / G) * p.n_q + kv * G + gr % G;
    p.part_ml[((size_t)orow * p.n_chunks + chunk) * 2] = sm.m_run[tid];
    p.part_ml[((size_t)orow * p.n_chunks + chunk) * 2 + 1] = sm.l_run[tid];
  }
  (void)nq_rows;
  if (!p.combine_in_kernel) return;

  // ---- the last CTA of this (KV head, row group) merges the chunks ----
  __threadfence();
  __syncthreads();
  if (tid == 0) sm.ticket = atomicAdd(&p.counters[kv * p.m_groups + mg], 1);
  __syncthreads();
  if (sm.ticket != p.n_chunks - 1) return;
  __threadfence();
  // chunk weights exp(m_c - m*) / l* per row (one warp per row), in the K/V tiles
  float* wgt = reinterpret_cast<float*>(&sm.k[0][0]);  // [nrows][n_chunks]
  for (int r = warp; r < nrows; r += kThreads / 32) {
    const int gr = row0 + r;
    const int orow = (gr / G) * p.n_q + kv * G + gr % G;
    const float* ml = p.part_ml + (size_t)orow * p.n_chunks * 2;
    float mx = -INFINITY;
    for (int c = lane; c < p.n_chunks; c += 32) mx = fmaxf(mx, __ldcg(ml + 2 * c));
    mx = warp_max(mx);
    float l = 0.f;
    for (int c = lane; c < p.n_chunks; c += 32) {
      const float mc = __ldcg(ml + 2 * c);
      const float e = mc == -INFINITY ? 0.f : __expf(mc - mx);
      wgt[r * p.n_chunks + c] = e;
      l = fmaf(__ldcg(ml + 2 * c + 1), e, l);
    }
    l = warp_sum(l);
    __syncwarp();
    for (int c = lane; c < p.n_chunks; c += 32) wgt[r * p.n_chunks + c] /= l;
  }
  __syncthreads();
  for (int c = tid; c < nrows * HD; c += kThreads) {
    const int r = c / HD, d = c - r * HD;
    const int gr = row0 + r;
    const int orow = (gr / G) * p.n_q + kv * G + gr % G;
    const float* acc = p.part_acc + (size_t)orow * p.n_chunks * HD + d;
    const float* w = wgt + r * p.n_chunks;
    float o = 0.f;
#pragma unroll 8
    for (int ch = 0; ch < p.n_chunks; ++ch)
      if (w[ch] != 0.f) o = fmaf(__ldcg(acc + (size_t)ch * HD), w[ch], o);
    p.out[(size_t)orow * HD + d] = __float2half_rn(o);
  }
  if (tid == 0) p.counters[kv * p.m_groups + mg] = 0;
}

// Separate merge of the chunk partials: block (output row, 128 dims), 8 warps.
// The chunk weights exp(m_c - m*) are computed once per block in shared memory;
// then thread (g, f) sums float4 column f over the chunks g, g + 8, ... (skipping
// empty chunks), and the 8 group sums are added in a fixed order.
constexpr int kCombineThreads = 256;
constexpr int kMaxChunks = 1024;

template <int HD>
__global__ void __launch_bounds__(kCombineThreads) attn_combine_kernel(const AttnParams p) {
  constexpr int F4 = 32;                      // float4 columns per block (128 dims)
  constexpr int NG = kCombineThreads / F4;    // chunk groups
  __shared__ float wgt[kMaxChunks];
  __shared__ float4 part[NG][F4];
  __shared__ float red[2][kCombineThreads / 32];
  pdl_wait();
  pdl_launch_dependents();
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int orow = blockIdx.x;
  const float* ml = p.part_ml + (size_t)orow * p.n_chunks * 2;
  float mx = -INFINITY;
  for (int c = tid; c < p.n_chunks; c += kCombineThreads) mx = fmaxf(mx, ml[2 * c]);
  mx = warp_max(mx);
  if (lane == 0) red[0][warp] = mx;
  __syncthreads();
  mx = red[0][0];
#pragma unroll
  for (int w = 1; w < kCombineThreads / 32; ++w) mx = fmaxf(mx, red[0][w]);
  float l = 0.f;
  for (int c = tid; c < p.n_chunks; c += kCombineThreads) {
    const float mc = ml[2 * c];
    const float e = mc == -INFINITY ? 0.f : __expf(mc - mx);
    wgt[c] = e;
    l = fmaf(ml[2 * c + 1], e, l);
  }
  l = warp_sum(l);
  if (lane == 0) red[1][warp] = l;
  __syncthreads();
  l = 0.f;
#pragma unroll
  for (int w = 0; w < kCombineThreads / 32; ++w) l += red[1][w];
  const int g = tid / F4, f = tid % F4;
  const float4* acc =
      reinterpret_cast<const float4*>(p.part_acc + (size_t)orow * p.n_chunks * HD) + blockIdx.y * F4 + f;
  float4 o = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 4
  for (int c = g; c < p.n_chunks; c += NG) {
    const float w = wgt[c];
    if (w != 0.f) {
      const float4 v = acc[(size_t)c * (HD / 4)];
      o.x = fmaf(v.x, w, o.x), o.y = fmaf(v.y, w, o.y), o.z = fmaf(v.z, w, o.z), o.w = fmaf(v.w, w, o.w);
    }
  }
  part[g][f] = o;
  __syncthreads();
  if (tid < F4) {
    float4 t = part[0][tid];
#pragma unroll
    for (int q = 1; q < NG; ++q) {
      const float4 v = part[q][tid];
      t.x += v.x, t.y += v.y, t.z += v.z, t.w += v.w;
    }
    __half* out = p.out + (size_t)orow * HD + blockIdx.y * 128 + 4 * tid;
    *reinterpret_cast<__half2*>(out) = __floats2half2_rn(t.x / l, t.y / l);
    *reinterpret_cast<__half2*>(out + 2) = __floats2half2_rn(t.z / l, t.w / l);
  }
}

template <int HD, int CL, bool KV8>
cudaError_t launch_attn_kv(const AttnParams& p, cudaStream_t st, bool pdl) {
  static bool configured = false;
  const size_t smem = sizeof(Smem<HD>);
  if (!configured) {
    cudaError_t e = cudaFuncSetAttribute(attn_kernel<HD, CL, KV8>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(attn_kernel<HD, CL, KV8>, cudaFuncAttributePreferredSharedMemoryCarveout,
                             cudaSharedmemCarveoutMaxShared);
    if (e != cudaSuccess) return e;
    configured = true;
  }
  if (CL > 0 && p.n_chunks != CL) return cudaErrorInvalidValue;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(p.n_kv, p.n_chunks, p.m_groups);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  int na = 0;
  if (pdl) {
    attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[na].val.programmaticStreamSerializationAllowed = 1;
    ++na;
  }
  if (CL > 0) {
    attr[na].id = cudaLaunchAttributeClusterDimension;
    attr[na].val.clusterDim.x = 1;
    attr[na].val.clusterDim.y = CL;
    attr[na].val.clusterDim.z = 1;
    ++na;
  }
  cfg.attrs = attr;
  cfg.numAttrs = na;
  return cudaLaunchKernelEx(&cfg, attn_kernel<HD, CL, KV8>, p);
}
template <int HD, int CL>
cudaError_t launch_attn_t(const AttnParams& p, cudaStream_t st, bool pdl) {
  return p.kv8 ? launch_attn_kv<HD, CL, true>(p, st, pdl) : launch_attn_kv<HD, CL, false>(p, st, pdl);
}

template <int HD>
cudaError_t launch_combine_t(const AttnParams& p, cudaStream_t st, bool pdl) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(p.kr * p.n_q, HD / 128);
  cfg.blockDim = dim3(kCombineThreads);
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, attn_combine_kernel<HD>, p);
}

}  // namespace

size_t attn_smem_bytes(int hd, int) {
  return hd == 256 ? sizeof(Smem<256>) : sizeof(Smem<512>);
}

FlashPlan flash_plan(int n_q, int n_kv, int hd, bool ring, int64_t window) {
  FlashPlan f{};
  const int G = n_q / n_kv;
  f.m_groups = (G + 31) / 32;
  const int sms = device_sm_count();
  int nch = ((hd == 256 ? 2 : 1) * sms) / (n_kv * f.m_groups);
  if (ring) {
    const int64_t want = (window + 63) / 64;
    if (want < nch) nch = (int)want;
  }
  if (nch > 2 * sms) nch = 2 * sms;
  f.n_chunks = nch < 1 ? 1 : nch;
  f.ml_offset = kFlashCounterBytes;
  f.acc_offset = f.ml_offset + ((sizeof(float) * 2 * (size_t)n_q * f.n_chunks + 255) & ~(size_t)255);
  f.bytes = f.acc_offset + sizeof(float) * (size_t)n_q * f.n_chunks * hd;
  return f;
}

void flash_bind(AttnParams& p, const FlashPlan& f, void* scratch) {
  char* w = static_cast<char*>(scratch);
  p.m_groups = f.m_groups;
  p.n_chunks = f.n_chunks;
  p.counters = reinterpret_cast<int32_t*>(w);
  p.part_ml = reinterpret_cast<float*>(w + f.ml_offset);
  p.part_acc = reinterpret_cast<float*>(w + f.acc_offset);
}

size_t attn_partial_floats(int kr, int n_q, int n_chunks, int hd) {
  return (size_t)kr * n_q * n_chunks * (size_t)hd;
}

cudaError_t launch_attention(const AttnParams& p, cudaStream_t st, bool pdl) {
  if (p.cluster == kAttnCluster && ring_decode_rows(p) > 0) return launch_attention_ring(p, st, pdl);
  if (p.cluster == kAttnCluster) {
    if (p.hd == 256) return launch_attn_t<256, kAttnCluster>(p, st, pdl);
    if (p.hd == 512) return launch_attn_t<512, kAttnCluster>(p, st, pdl);
    return cudaErrorInvalidValue;
  }
  if (p.cluster != 0) return cudaErrorInvalidValue;
  if (p.hd == 256) return launch_attn_t<256, 0>(p, st, pdl);
  if (p.hd == 512) return launch_attn_t<512, 0>(p, st, pdl);
  return cudaErrorInvalidValue;
}

cudaError_t launch_attn_combine(const AttnParams& p, cudaStream_t st, bool pdl) {
  if (p.hd == 256) return launch_combine_t<256>(p, st, pdl);
  if (p.hd == 512) return launch_combine_t<512>(p, st, pdl);
  return cudaErrorInvalidValue;
}

}  // namespace q4g
