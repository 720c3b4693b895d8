// q4_0 matrix-vector product with the dequantisation fused into the dot product.
//
// Operation ("Gemma 4 12B" page, intro: per-block-32 absmax symmetric int4;
// "gemma-4-E4B-CoreAI", Provenance: the q4_0 grid): y[j][r] = sum_c w(r,c) x[j][c]
// with w(r,c) = (code - 8) * d(r, c/32), x fp16, fp32 accumulation.
//
// Work decomposition (one launch, persistent over 16-row units):
//   * a CTA (8 warps) owns a contiguous, balanced range of 16-row units;
//   * warp w owns columns blocks [w*NB/8, (w+1)*NB/8) of every unit (NB = k/32);
//   * a warp step covers 4 rows x 8 consecutive blocks: lane (r4 = lane/8,
//     b8 = lane%8) loads the 16 code bytes of one block with one 128-bit
//     streaming load; a row's 8 blocks are 128 contiguous bytes, so each load
//     instruction moves four full 128-byte lines;
//   * the four row groups of a unit share the x registers of the step, x is
//     staged once per CTA in shared memory in the order the nibble unpacking
//     produces, and per block the constant 72 * sum(x) removes the +64 offset
//     of the unpacked values and the -8 of the code (see block_dot);
//   * partial row sums are reduced with shuffles across the 8 lanes of a row
//     and in a fixed order across warps through shared memory (deterministic);
//   * the first weight loads are issued before griddepcontrol.wait, so with
//     programmatic dependent launch they overlap the previous kernel's tail.
#include "q4g_common.cuh"
#include "q4g_internal.h"
#include "q4g_prefetch.cuh"

#include <stdlib.h>

namespace q4g {

namespace {

// Slot of column e (0..31) of a block in the x layout (inverse of xperm).
Q4G_DEV int xslot(int e) {
  const int hi = e >> 4, e2 = e & 15, k = e2 >> 2, o = e2 & 3;
  // o: 0 -> 0, 1 -> 4, 2 -> 1, 3 -> 5 ; +2 for the high half of the block
  const int j = ((o & 1) << 2) + (o >> 1) + (hi << 1);
  return 8 * k + j;
}

// Row pointers of the lane's rows in a unit: row group g (0..3) is row
// r4 + 4*(g&1) of half a (g < 2) or half b (g >= 2). Plain and segmented
// matrices: halves are rows 0..7 and 8..15 of the unit; GeGLU pairing: half a
// is 8 gate rows and half b the 8 up rows of the same index.
struct UnitRows {
  const uint8_t* qa;
  const uint8_t* qb;
  const uint16_t* sa;
  const uint16_t* sb;
  int da, db;  // row offset of the second row group of each half (4, or less at a ragged end)
};

Q4G_DEV void seg_row(const GemvParams& p, int row, const GemvSeg*& s, int& r) {
  s = &p.seg[0];
  r = row;
  if (p.nseg > 1 && r >= p.seg[0].rows) {
    r -= p.seg[0].rows;
    s = &p.seg[1];
    if (p.nseg > 2 && r >= p.seg[1].rows) {
      r -= p.seg[1].rows;
      s = &p.seg[2];
    }
  }
}

Q4G_DEV void unit_rows(const GemvParams& p, int u, int r4, int kh, int nb, UnitRows& out) {
  const GemvSeg* sa;
  const GemvSeg* sb;
  int ra, rb;
  if (p.epi == EPI_GEGLU) {
    sa = &p.seg[0], sb = &p.seg[1];
    ra = rb = 8 * u + r4;
  } else {
    seg_row(p, 16 * u, sa, ra);  // a unit never straddles two segments
    sb = sa;
    ra += r4;
    rb = ra + 8;
  }
  // rows past the end of a ragged matrix re-read its last row (results unused)
  const int la = sa->rows - 1, lb = sb->rows - 1;
  out.da = min(ra + 4, la) - min(ra, la);
  out.db = min(rb + 4, lb) - min(rb, lb);
  ra = min(ra, la);
  rb = min(rb, lb);
  out.qa = sa->qs + (size_t)ra * kh;
  out.qb = sb->qs + (size_t)rb * kh;
  out.sa = sa->sc + (size_t)ra * nb;
  out.sb = sb->sc + (size_t)rb * nb;
}

Q4G_DEV void load_step(const UnitRows& r, int blk, int kb1, int kh, int nb, uint4 (&q)[4],
                       uint16_t (&sc)[4]) {
#pragma unroll
  for (int g = 0; g < 4; ++g) {
    const int dr = (g & 1) ? (g < 2 ? r.da : r.db) : 0;
    const uint8_t* qp = (g < 2 ? r.qa : r.qb) + (size_t)dr * kh + (size_t)blk * 16;
    const uint16_t* sp = (g < 2 ? r.sa : r.sb) + (size_t)dr * nb + blk;
    if (blk < kb1) {
      q[g] = ld_stream_u4(qp);
      sc[g] = ld_stream_u16(sp);
    } else {
      q[g] = make_uint4(0, 0, 0, 0);
      sc[g] = 0;
    }
  }
}

// Stage x (fp16) for row j into the permuted shared layout.
Q4G_DEV void put_x(__half* xs_h, int nb, int j, int col, __half v) {
  const int blk = col >> 5, s = xslot(col & 31);
  // layout [j][quarter][blk][8 halves]
  xs_h[((size_t)(j * 4 + (s >> 3)) * nb + blk) * 8 + (s & 7)] = v;
}

// Activations of the step into shared memory, in the order the nibble
// unpacking consumes them, plus the per-block constant 72 * sum(x) that removes
// the +64 of the unpacked codes and the -8 of the code offset.
//   PRO_X16:   x = the fp16 input rows
//   PRO_RESID: r_new = (r_in + rmsnorm(delta) * w_delta) * scale,
//              x = fp16(rmsnorm(r_new) * w_x); block 0 stores r_new (and the dump)
// Ends with __syncthreads().
template <int KRM, int NT = kThreads, bool NAT = false>
Q4G_DEV void stage_x(const GemvParams& p, uint4* xs, float* cblk, float* misc) {
  const int k = p.k, nb = k >> 5, tid = threadIdx.x;
  __half* xs_h = reinterpret_cast<__half*>(xs);
  // NAT: x row j in natural column order at xs_h + j * k, no block constants
  auto put = [&](int j, int col, __half v) {
    if (NAT)
      xs_h[(size_t)j * k + col] = v;
    else
      put_x(xs_h, nb, j, col, v);
  };
  for (int j = 0; j < KRM; ++j) {
    if (j >= p.kr) break;
    if (p.pro == PRO_X16) {
      const __half* xr = p.x + (size_t)j * p.x_stride;
      if ((((uintptr_t)xr) & 15) == 0) {
        for (int c8 = tid; c8 < (k >> 3); c8 += NT) {
          const uint4 v = *reinterpret_cast<const uint4*>(xr + 8 * c8);
          if (NAT) {
            *reinterpret_cast<uint4*>(xs_h + (size_t)j * k + 8 * c8) = v;
          } else {
            const __half* h = reinterpret_cast<const __half*>(&v);
#pragma unroll
            for (int e = 0; e < 8; ++e) put_x(xs_h, nb, j, 8 * c8 + e, h[e]);
          }
        }
      } else {
        for (int c = tid; c < k; c += NT) put(j, c, xr[c]);
      }
    } else {
      // k <= 8192: each thread keeps its float4s of r_new in registers
      constexpr int R4 = (8192 + 4 * NT - 1) / (4 * NT);
      const float4* rin = reinterpret_cast<const float4*>(p.r_in + (size_t)j * k);
      const float4* dl = p.delta ? reinterpret_cast<const float4*>(p.delta + (size_t)j * k) : nullptr;
      const float4* wd = reinterpret_cast<const float4*>(p.w_delta);
      const float4* wx = reinterpret_cast<const float4*>(p.w_x);
      const int n4 = k >> 2;
      float4 rn[R4], dv[R4];
      float ss = 0.f;
#pragma unroll
      for (int i = 0; i < R4; ++i) {
        const int c4 = tid + i * NT;
        if (c4 < n4) {
          rn[i] = rin[c4];
          if (dl) {
            dv[i] = dl[c4];
            ss = fmaf(dv[i].x, dv[i].x, ss);
            ss = fmaf(dv[i].y, dv[i].y, ss);
            ss = fmaf(dv[i].z, dv[i].z, ss);
            ss = fmaf(dv[i].w, dv[i].w, ss);
          }
        }
      }
      if (dl) {
        const float inv_d = rms_inv(block_sum<NT>(ss, misc), k, p.eps);
#pragma unroll
        for (int i = 0; i < R4; ++i) {
          const int c4 = tid + i * NT;
          if (c4 < n4) {
            const float4 w = wd[c4];
            rn[i].x = __fmul_rn(__fadd_rn(rn[i].x, __fmul_rn(__fmul_rn(dv[i].x, inv_d), w.x)), p.scale);
            rn[i].y = __fmul_rn(__fadd_rn(rn[i].y, __fmul_rn(__fmul_rn(dv[i].y, inv_d), w.y)), p.scale);
            rn[i].z = __fmul_rn(__fadd_rn(rn[i].z, __fmul_rn(__fmul_rn(dv[i].z, inv_d), w.z)), p.scale);
            rn[i].w = __fmul_rn(__fadd_rn(rn[i].w, __fmul_rn(__fmul_rn(dv[i].w, inv_d), w.w)), p.scale);
          }
        }
      }
      float ss2 = 0.f;
#pragma unroll
      for (int i = 0; i < R4; ++i) {
        const int c4 = tid + i * NT;
        if (c4 < n4) {
          ss2 = fmaf(rn[i].x, rn[i].x, ss2);
          ss2 = fmaf(rn[i].y, rn[i].y, ss2);
          ss2 = fmaf(rn[i].z, rn[i].z, ss2);
          ss2 = fmaf(rn[i].w, rn[i].w, ss2);
          if (blockIdx.x == 0) {
            reinterpret_cast<float4*>(p.r_out + (size_t)j * k)[c4] = rn[i];
            if (p.dump) reinterpret_cast<float4*>(p.dump + (size_t)j * p.dump_stride)[c4] = rn[i];
          }
        }
      }
      const float inv_r = rms_inv(block_sum<NT>(ss2, misc + 32), k, p.eps);
#pragma unroll
      for (int i = 0; i < R4; ++i) {
        const int c4 = tid + i * NT;
        if (c4 < n4) {
          const float4 w = wx[c4];
          put(j, 4 * c4 + 0, __float2half_rn(__fmul_rn(__fmul_rn(rn[i].x, inv_r), w.x)));
          put(j, 4 * c4 + 1, __float2half_rn(__fmul_rn(__fmul_rn(rn[i].y, inv_r), w.y)));
          put(j, 4 * c4 + 2, __float2half_rn(__fmul_rn(__fmul_rn(rn[i].z, inv_r), w.z)));
          put(j, 4 * c4 + 3, __float2half_rn(__fmul_rn(__fmul_rn(rn[i].w, inv_r), w.w)));
        }
      }
    }
  }
  __syncthreads();
  if (!NAT) {
    for (int t = tid; t < p.kr * nb; t += NT) {
      const int j = t / nb, blk = t - j * nb;
      float sx = 0.f;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const __half* h = xs_h + ((size_t)(j * 4 + q) * nb + blk) * 8;
#pragma unroll
        for (int e = 0; e < 8; ++e) sx += __half2float(h[e]);
      }
      cblk[t] = 72.0f * sx;
    }
    __syncthreads();
  }
}

template <int KRM>
__global__ void __launch_bounds__(kThreads, 2) gemv_q4_kernel(const GemvParams p) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  const int k = p.k, nb = k >> 5, kh = k >> 1;
  uint4* xs = reinterpret_cast<uint4*>(smem_raw);         // [KRM][4][nb]
  float* cblk = reinterpret_cast<float*>(xs + (size_t)KRM * 4 * nb);  // [KRM][nb]
  float* red = cblk + KRM * nb;                           // [8 warps][16 rows][KRM]
  float* misc = red + 8 * 16 * KRM;                       // 64 floats

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int r4 = lane >> 3, b8 = lane & 7;
  const int kb0 = (warp * nb) >> 3, kb1 = ((warp + 1) * nb) >> 3;
  const int span = (nb + 7) >> 3;                 // largest per-warp block range
  const int nsteps = (span + 7) >> 3;             // identical for every warp
  const int u_begin = (int)(((long long)blockIdx.x * p.n_units) / gridDim.x);
  const int u_end = (int)(((long long)(blockIdx.x + 1) * p.n_units) / gridDim.x);
  const int total = (u_end - u_begin) * nsteps;

  // ---- first weight loads (independent of earlier kernels) ----
  uint4 qc[4];
  uint16_t scc[4];
  UnitRows rows;
  int u = u_begin, s = 0;
  if (total > 0) {
    unit_rows(p, u, r4, kh, nb, rows);
    load_step(rows, kb0 + b8, kb1, kh, nb, qc, scc);
  }

  pdl_wait();

  stage_x<KRM>(p, xs, cblk, misc);
  pdl_launch_dependents();

  // ---- main loop over (unit, step) pairs ----
  float yacc[4][KRM];
#pragma unroll
  for (int g = 0; g < 4; ++g)
#pragma unroll
    for (int j = 0; j < KRM; ++j) yacc[g][j] = 0.f;

  float best_v[KRM];
  int best_i[KRM];
#pragma unroll
  for (int j = 0; j < KRM; ++j) best_v[j] = -INFINITY, best_i[j] = 0x7fffffff;

  for (int it = 0; it < total; ++it) {
    // prefetch the next pair
    int un = u, sn = s + 1;
    if (sn == nsteps) sn = 0, ++un;
    uint4 qn[4];
    uint16_t scn[4];
    UnitRows rows_n = rows;
    if (it + 1 < total) {
      if (un != u) unit_rows(p, un, r4, kh, nb, rows_n);
      load_step(rows_n, kb0 + 8 * sn + b8, kb1, kh, nb, qn, scn);
    }
    // compute the current pair
    const int blk = kb0 + 8 * s + b8;
    if (blk < kb1) {
      float d[4];
#pragma unroll
      for (int g = 0; g < 4; ++g) d[g] = __half2float(__ushort_as_half(scc[g]));
#pragma unroll
      for (int j = 0; j < KRM; ++j) {
        if (j < p.kr) {
          uint4 xq[4];
#pragma unroll
          for (int q = 0; q < 4; ++q) xq[q] = lds_u4(xs + (size_t)(j * 4 + q) * nb + blk);
          const float cb = cblk[j * nb + blk];
#pragma unroll
          for (int g = 0; g < 4; ++g) {
            float a0 = -cb, a1 = 0.f;
            block_dot(qc[g], xq, a0, a1);
            yacc[g][j] = fmaf(d[g], a0 + a1, yacc[g][j]);
          }
        }
      }
    }
    if (s == nsteps - 1) {
      // unit complete: reduce the 8 lanes of each row, then across warps
#pragma unroll
      for (int g = 0; g < 4; ++g)
#pragma unroll
        for (int j = 0; j < KRM; ++j) {
          float v = yacc[g][j];
          v += __shfl_xor_sync(0xffffffffu, v, 1);
          v += __shfl_xor_sync(0xffffffffu, v, 2);
          v += __shfl_xor_sync(0xffffffffu, v, 4);
          if (b8 == 0) red[(warp * 16 + 4 * g + r4) * KRM + j] = v;
          yacc[g][j] = 0.f;
        }
      __syncthreads();
      if (tid < 16 * KRM) {
        const int row = tid & 15, j = tid >> 4;
        if (j < p.kr) {
          float acc = 0.f;
#pragma unroll
          for (int w = 0; w < 8; ++w) acc += red[(w * 16 + row) * KRM + j];
          if (p.epi == EPI_STORE) {
            if (16 * u + row < p.n_rows) p.y[(size_t)j * p.y_stride + 16 * u + row] = acc;
          } else if (p.epi == EPI_GEGLU) {
            if (row < 8) {
              float up = 0.f;
#pragma unroll
              for (int w = 0; w < 8; ++w) up += red[(w * 16 + row + 8) * KRM + j];
              p.act[(size_t)j * p.act_stride + 8 * u + row] = __float2half_rn(gelu_tanh(acc) * up);
            }
          } else {
            const float z = p.softcap * tanhf(acc / p.softcap);
            const int idx = 16 * u + row;
            if (idx < p.n_rows) {
              if (p.logits) p.logits[(size_t)j * p.logits_stride + idx] = z;
              if (z > best_v[j] || (z == best_v[j] && idx < best_i[j])) best_v[j] = z, best_i[j] = idx;
            }
          }
        }
      }
      __syncthreads();
    }
#pragma unroll
    for (int g = 0; g < 4; ++g) qc[g] = qn[g], scc[g] = scn[g];
    rows = rows_n;
    u = un;
    s = sn;
  }

  if (p.epi == EPI_HEAD) {
    __shared__ int s_ticket;
    // argmax: within each 16-thread group (whole warps take part in the
    // shuffles; lanes past the last row group carry a neutral value), then
    // across CTAs (the last CTA to finish reduces the per-CTA results)
    if (warp < (16 * KRM + 31) / 32) {
      const int j = tid >> 4;
      const bool valid = j < KRM && j < p.kr;
      float v = -INFINITY;
      int i = 0x7fffffff;
      if (valid) v = best_v[j], i = best_i[j];
#pragma unroll
      for (int o = 8; o > 0; o >>= 1) {
        const float v2 = __shfl_xor_sync(0xffffffffu, v, o);
        const int i2 = __shfl_xor_sync(0xffffffffu, i, o);
        if (v2 > v || (v2 == v && i2 < i)) v = v2, i = i2;
      }
      if ((tid & 15) == 0 && valid) {
        p.am_val[j * gridDim.x + blockIdx.x] = v;
        p.am_idx[j * gridDim.x + blockIdx.x] = i;
      }
    }
    __threadfence();
    __syncthreads();
    if (tid == 0) s_ticket = atomicAdd(p.counter, 1);
    __syncthreads();
    if (s_ticket == (int)gridDim.x - 1) {
      __threadfence();
      for (int j = 0; j < p.kr; ++j) {
        float v = -INFINITY;
        int i = 0x7fffffff;
        for (int b = tid; b < (int)gridDim.x; b += kThreads) {
          const float v2 = __ldcg(p.am_val + j * gridDim.x + b);
          const int i2 = __ldcg(p.am_idx + j * gridDim.x + b);
          if (v2 > v || (v2 == v && i2 < i)) v = v2, i = i2;
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
          const float v2 = __shfl_xor_sync(0xffffffffu, v, o);
          const int i2 = __shfl_xor_sync(0xffffffffu, i, o);
          if (v2 > v || (v2 == v && i2 < i)) v = v2, i = i2;
        }
        __syncthreads();
        if (lane == 0) misc[warp] = v, reinterpret_cast<int*>(misc)[32 + warp] = i;
        __syncthreads();
        if (tid == 0) {
          float bv = misc[0];
          int bi = reinterpret_cast<int*>(misc)[32];
          for (int w = 1; w < kThreads / 32; ++w) {
            const float v2 = misc[w];
            const int i2 = reinterpret_cast<int*>(misc)[32 + w];
            if (v2 > bv || (v2 == bv && i2 < bi)) bv = v2, bi = i2;
          }
          if (p.argmax_out) p.argmax_out[j] = bi == 0x7fffffff ? 0 : bi;
        }
      }
      if (tid == 0) *p.counter = 0;
    }
  }
}


// ---------------------------------------------------------------------------
// Warp-streamed GEMV: every warp is an independent streaming engine.
//
// A unit is 2 rows (a GeGLU unit: gate row u and up row u). The warps of the
// grid own balanced, contiguous ranges of units. A warp walks its units in
// items of (unit, column chunk of kc columns); lane 0 keeps `ns` items of its
// own in flight with 1-D bulk copies into the warp's private ring of shared
// memory stages (one mbarrier per stage). Lane (r2 = lane/16, b16 = lane%16)
// takes row r2 and every 16th block; x is staged once per CTA in shared memory
// and read by all warps. A unit's two sums are reduced with shuffles across the
// 16 lanes of each row; there is no synchronisation between warps after the
// prologue, so warps drift apart and hide each other's latencies.
// ---------------------------------------------------------------------------
constexpr int kWarps = 15;  // 148 SMs x 15 warps balances the row counts of the decoder
constexpr int kWarpThreads = kWarps * 32;
constexpr int kMaxStages = 4;

struct ItemSrc {
  const uint8_t* q[2];
  const uint16_t* s[2];
  int rows;  // 1 or 2 (ragged end)
};

// Source rows of unit u (row pair), column chunk c.
Q4G_DEV ItemSrc item_src(const GemvParams& p, int u, int c) {
  const int kh = p.k >> 1, nb = p.k >> 5;
  const size_t qo = (size_t)c * (p.kc >> 1), so = (size_t)c * (p.kc >> 5);
  ItemSrc it{};
  if (p.epi == EPI_GEGLU) {
    it.q[0] = p.seg[0].qs + (size_t)u * kh + qo;
    it.q[1] = p.seg[1].qs + (size_t)u * kh + qo;
    it.s[0] = p.seg[0].sc + (size_t)u * nb + so;
    it.s[1] = p.seg[1].sc + (size_t)u * nb + so;
    it.rows = 2;
  } else {
    const GemvSeg* sg;
    int r;
    seg_row(p, 2 * u, sg, r);  // segments hold an even number of rows
    it.rows = min(2, sg->rows - r);
    it.q[0] = sg->qs + (size_t)r * kh + qo;
    it.s[0] = sg->sc + (size_t)r * nb + so;
    it.q[1] = it.q[0] + kh;
    it.s[1] = it.s[0] + nb;
  }
  return it;
}

// stage layout: row 0 codes | row 1 codes | row 0 scales | row 1 scales
Q4G_DEV void issue_item(const GemvParams& p, int u, int c, unsigned char* st, uint64_t* bar, bool poison,
                        uint64_t pol) {
  const ItemSrc it = item_src(p, u, c);
  const uint32_t qb = (uint32_t)(p.kc >> 1), sb = (uint32_t)(p.kc >> 4);
  mbar_arrive_expect_tx(bar, (uint32_t)it.rows * (qb + sb) + (poison ? 16u : 0u));
  bulk_g2s_hint(st, it.q[0], qb, bar, pol);
  bulk_g2s_hint(st + 2 * (size_t)qb, it.s[0], sb, bar, pol);
  if (it.rows == 2) {
    bulk_g2s_hint(st + qb, it.q[1], qb, bar, pol);
    bulk_g2s_hint(st + 2 * (size_t)qb + sb, it.s[1], sb, bar, pol);
  }
}

// ---------------------------------------------------------------------------
// Integer form of the block dot product.
//
// x of one block (32 fp16 values) becomes signed 24-bit fixed point relative to
// the block's largest exponent: X_i = round(x_i * 2^(37 - Emax)), exact for
// every value within 2^12 of the block maximum (the rest carry an error below
// 2^-24 of the block maximum), x_i ~= X_i * 2^(Emax - 37). X splits into bytes
// X = d0 + 256 d1 + 65536 d2 (d0, d1 unsigned, d2 signed), so
//   sum_i (c_i - 8) X_i = S0 + 256 S1 + 65536 S2,  S_t = sum_i (c_i - 8) d_t,i,
// and each S_t is a chain of 4-way byte dot products (dp4a) of the raw codes
// with the digits, started at -8 * sum_i d_t,i. Every S_t is exact in int32.
// Layout per x row j: dg[j][2t + h][blk] holds digit t of columns 16h..16h+15
// of block blk (16 bytes), bc[j][blk] = (-8 D0, -8 D1, -8 D2, bits of 2^(Emax-37)).
// ---------------------------------------------------------------------------
template <int NT>
Q4G_DEV void stage_digits(const GemvParams& p, const __half* xn, uint4* dg, int4* bc) {
  const int k = p.k, nb = k >> 5, warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  unsigned char* db = reinterpret_cast<unsigned char*>(dg);
  for (int t = warp; t < p.kr * nb; t += NT / 32) {
    const int j = t / nb, blk = t - j * nb;
    const uint32_t h = __half_as_ushort(xn[(size_t)j * k + blk * 32 + lane]);
    const int E = (h >> 10) & 31, Ee = E ? E : 1;
    const int M = (int)(h & 1023) | (E ? 1024 : 0);
    const int emax = (int)__reduce_max_sync(0xffffffffu, (unsigned)Ee);
    const int sh = 12 + Ee - emax;  // <= 12
    int X = sh >= 0 ? (M << sh) : sh > -12 ? (M + (1 << (-sh - 1))) >> -sh : 0;
    if (h & 0x8000) X = -X;
    const int d0 = X & 255, d1 = (X >> 8) & 255, d2 = X >> 16;
    const int hh = lane >> 4, col = lane & 15;
    db[((size_t)(j * 6 + 0 + hh) * nb + blk) * 16 + col] = (unsigned char)d0;
    db[((size_t)(j * 6 + 2 + hh) * nb + blk) * 16 + col] = (unsigned char)d1;
    db[((size_t)(j * 6 + 4 + hh) * nb + blk) * 16 + col] = (unsigned char)d2;
    const int s0 = __reduce_add_sync(0xffffffffu, d0);
    const int s1 = __reduce_add_sync(0xffffffffu, d1);
    const int s2 = __reduce_add_sync(0xffffffffu, d2);
    if (lane == 0) bc[j * nb + blk] = make_int4(-8 * s0, -8 * s1, -8 * s2, (emax - 37 + 127) << 23);
  }
}

Q4G_DEV float block_dot_int(const uint4 q, const uint4 (&g)[6], const int4 c) {
  const uint32_t w[4] = {q.x, q.y, q.z, q.w};
  int s0 = c.x, s1 = c.y, s2 = c.z;
#pragma unroll
  for (int t = 0; t < 4; ++t) {
    const uint32_t lo = w[t] & 0x0F0F0F0Fu, hi = (w[t] >> 4) & 0x0F0F0F0Fu;
    s0 = dp4a_uu(lo, (&g[0].x)[t], s0);
    s0 = dp4a_uu(hi, (&g[1].x)[t], s0);
    s1 = dp4a_uu(lo, (&g[2].x)[t], s1);
    s1 = dp4a_uu(hi, (&g[3].x)[t], s1);
    s2 = dp4a_us(lo, (&g[4].x)[t], s2);
    s2 = dp4a_us(hi, (&g[5].x)[t], s2);
  }
  return fmaf((float)s2, 65536.0f, (float)(s1 * 256 + s0));
}

// Shared memory of the warp-streamed kernel: the x region (layout per dot
// kind), then 64 floats of reduction scratch, per-warp argmax candidates, the
// mbarriers and the stages.
enum : int { DOT_FMA_HALF = 0, DOT_FMA = 1, DOT_INT = 2 };

__host__ __device__ inline size_t x_region_bytes(int dot, int krm, int k) {
  const size_t nb = (size_t)k / 32;
  return dot == DOT_INT ? (size_t)krm * nb * (96 + 16 + 64) : (size_t)krm * nb * (64 + 4);
}

template <int KRM, int DOT>
__global__ void __launch_bounds__(kWarpThreads, 1) gemv_q4_tma_kernel(const GemvParams p) {
  extern __shared__ __align__(16) unsigned char ws_smem[];
  const int k = p.k, nb = k >> 5, NS = p.ns;
  const int kc = p.kc, nbc = kc >> 5, qb = kc >> 1;
  // x region
  uint4* xs = reinterpret_cast<uint4*>(ws_smem);                        // FMA: [KRM][4][nb]; INT: dg [KRM][6][nb]
  float* cblk = reinterpret_cast<float*>(xs + (size_t)KRM * 4 * nb);     // FMA: [KRM][nb]
  int4* bc = reinterpret_cast<int4*>(xs + (size_t)KRM * 6 * nb);         // INT: [KRM][nb]
  __half* xn = reinterpret_cast<__half*>(bc + (size_t)KRM * nb);         // INT: [KRM][k]
  float* misc = reinterpret_cast<float*>(ws_smem + x_region_bytes(DOT, KRM, k));  // 64 floats
  float* bestv = misc + 64;                                              // [kWarps]
  int* besti = reinterpret_cast<int*>(bestv + kWarps);                   // [kWarps]
  uint64_t* bars = reinterpret_cast<uint64_t*>(((uintptr_t)(besti + kWarps) + 127) & ~(uintptr_t)127);
  unsigned char* stages = reinterpret_cast<unsigned char*>(bars + kWarps * kMaxStages);  // [kWarps][NS][stage]
  __shared__ int s_ticket;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const long long tw = (long long)gridDim.x * kWarps, gw = (long long)blockIdx.x * kWarps + warp;
  const int u_begin = (int)(gw * p.n_units / tw), u_end = (int)((gw + 1) * p.n_units / tw);
  const int nchunk = k / kc;
  const int n_items = (u_end - u_begin) * nchunk;
  uint64_t* wbar = bars + warp * kMaxStages;
  unsigned char* wst = stages + (size_t)warp * NS * p.stage_bytes;
  bool abort_ = false;
  int issued = 0, abort_it = 0;

  const uint64_t pol = policy_evict_first();
  if (lane == 0) {
    for (int s = 0; s < NS; ++s) mbar_init(&wbar[s], 1);
    fence_mbar_init();
    for (; issued < NS && issued < n_items; ++issued)
      issue_item(p, u_begin + issued / nchunk, issued % nchunk, wst + (size_t)issued * p.stage_bytes,
                 &wbar[issued], p.stall_test && u_begin == 0 && issued == 0, pol);  // the warp owning unit 0
    // all own loads issued: start the next GEMV's weights towards L2
    if (issued == n_items) prefetch_next(p.next, gw, tw);
  }
  __syncwarp();

  pdl_wait();
  if (DOT == DOT_INT) {
    stage_x<KRM, kWarpThreads, true>(p, reinterpret_cast<uint4*>(xn), nullptr, misc);
    stage_digits<kWarpThreads>(p, xn, xs, bc);
    __syncthreads();
  } else {
    stage_x<KRM, kWarpThreads>(p, xs, cblk, misc);
  }
  pdl_launch_dependents();

  // acc[r][j]: row r of the unit, activation row j (DOT_FMA_HALF: r = lane / 16 only)
  float acc[2][KRM];
#pragma unroll
  for (int r = 0; r < 2; ++r)
#pragma unroll
    for (int j = 0; j < KRM; ++j) acc[r][j] = 0.f;
  float best_v = -INFINITY;
  int best_i = 0x7fffffff;

  for (int it = 0; it < n_items; ++it) {
    const int s = it % NS, u = u_begin + it / nchunk, c = it % nchunk;
    if (!abort_ && !mbar_wait_bounded(&wbar[s], (uint32_t)((it / NS) & 1), p.wait_ns)) {
      if (lane == 0) atomicOr(p.err, 1);
      abort_ = true;
      abort_it = it;
    }
    const unsigned char* st = wst + (size_t)s * p.stage_bytes;
    const uint16_t* ssc = reinterpret_cast<const uint16_t*>(st + 2 * (size_t)qb);  // [2][nbc]
    if (DOT == DOT_FMA_HALF) {
      const int r2 = lane >> 4, b16 = lane & 15;
      const unsigned char* sq = st + (size_t)r2 * qb;
#pragma unroll 2
      for (int step = 0; step < (nbc + 15) >> 4; ++step) {
        const int bl = 16 * step + b16;
        if (bl < nbc) {
          const uint4 qv = lds_u4(sq + (size_t)bl * 16);
          const float d = __half2float(__ushort_as_half(ssc[r2 * nbc + bl]));
          const int blk = c * nbc + bl;
#pragma unroll
          for (int j = 0; j < KRM; ++j) {
            if (KRM == 1 || j < p.kr) {
              uint4 xq[4];
#pragma unroll
              for (int q = 0; q < 4; ++q) xq[q] = lds_u4(xs + (size_t)(j * 4 + q) * nb + blk);
              float a0 = -cblk[j * nb + blk], a1 = 0.f;
              block_dot(qv, xq, a0, a1);
              acc[0][j] = fmaf(d, a0 + a1, acc[0][j]);
            }
          }
        }
      }
    } else {
      for (int step = 0; step < (nbc + 31) >> 5; ++step) {
        const int bl = 32 * step + lane;
        if (bl < nbc) {
          const uint4 q0 = lds_u4(st + (size_t)bl * 16);
          const uint4 q1 = lds_u4(st + (size_t)qb + (size_t)bl * 16);
          const float d0 = __half2float(__ushort_as_half(ssc[bl]));
          const float d1 = __half2float(__ushort_as_half(ssc[nbc + bl]));
          const int blk = c * nbc + bl;
#pragma unroll
          for (int j = 0; j < KRM; ++j) {
            if (KRM == 1 || j < p.kr) {
              if (DOT == DOT_FMA) {
                uint4 xq[4];
#pragma unroll
                for (int q = 0; q < 4; ++q) xq[q] = lds_u4(xs + (size_t)(j * 4 + q) * nb + blk);
                const float cb = cblk[j * nb + blk];
                float a0 = -cb, a1 = 0.f, b0 = -cb, b1 = 0.f;
                block_dot(q0, xq, a0, a1);
                block_dot(q1, xq, b0, b1);
                acc[0][j] = fmaf(d0, a0 + a1, acc[0][j]);
                acc[1][j] = fmaf(d1, b0 + b1, acc[1][j]);
              } else {
                uint4 g[6];
#pragma unroll
                for (int q = 0; q < 6; ++q) g[q] = lds_u4(xs + (size_t)(j * 6 + q) * nb + blk);
                const int4 cv = bc[j * nb + blk];
                const float xsc = __int_as_float(cv.w);
                acc[0][j] = fmaf(d0 * xsc, block_dot_int(q0, g, cv), acc[0][j]);
                acc[1][j] = fmaf(d1 * xsc, block_dot_int(q1, g, cv), acc[1][j]);
              }
            }
          }
        }
      }
    }
    __syncwarp();
    if (lane == 0 && !abort_ && issued < n_items) {  // refill this stage
      issue_item(p, u_begin + issued / nchunk, issued % nchunk, wst + (size_t)s * p.stage_bytes, &wbar[s],
                 false, pol);
      if (++issued == n_items) prefetch_next(p.next, gw, tw);
    }
    if (c != nchunk - 1) continue;
    // unit complete: the two row sums of every activation row
#pragma unroll
    for (int j = 0; j < KRM; ++j) {
      float v0, v1;
      if (DOT == DOT_FMA_HALF) {
        float v = acc[0][j];
        v += __shfl_xor_sync(0xffffffffu, v, 1);
        v += __shfl_xor_sync(0xffffffffu, v, 2);
        v += __shfl_xor_sync(0xffffffffu, v, 4);
        v += __shfl_xor_sync(0xffffffffu, v, 8);
        const float o = __shfl_xor_sync(0xffffffffu, v, 16);
        v0 = lane < 16 ? v : o;
        v1 = lane < 16 ? o : v;
      } else {
        v0 = warp_sum(acc[0][j]);
        v1 = warp_sum(acc[1][j]);
      }
      acc[0][j] = acc[1][j] = 0.f;
      if (j >= p.kr || lane != 0) continue;
      const int row = 2 * u;
      if (p.epi == EPI_STORE) {
        float* y = p.y + (size_t)j * p.y_stride;
        if (row < p.n_rows) y[row] = v0;
        if (row + 1 < p.n_rows) y[row + 1] = v1;
      } else if (p.epi == EPI_GEGLU) {
        p.act[(size_t)j * p.act_stride + u] = __float2half_rn(gelu_tanh(v0) * v1);
      } else {
#pragma unroll
        for (int r = 0; r < 2; ++r) {
          if (row + r < p.n_rows) {
            const float z = p.softcap * tanhf((r ? v1 : v0) / p.softcap);
            if (p.logits) p.logits[(size_t)j * p.logits_stride + row + r] = z;
            if (KRM == 1 && z > best_v) best_v = z, best_i = row + r;  // rows ascend: first max wins
          }
        }
      }
    }
  }

  if (p.epi == EPI_HEAD) {
    if (lane == 0) bestv[warp] = best_v, besti[warp] = best_i;
    __syncthreads();
    if (tid == 0) {
      float v = -INFINITY;
      int ix = 0x7fffffff;
      for (int w = 0; w < kWarps; ++w)
        if (bestv[w] > v || (bestv[w] == v && besti[w] < ix)) v = bestv[w], ix = besti[w];
      p.am_val[blockIdx.x] = v;
      p.am_idx[blockIdx.x] = ix;
    }
    __threadfence();
    __syncthreads();
    if (tid == 0) s_ticket = atomicAdd(p.counter, 1);
    __syncthreads();
    if (s_ticket == (int)gridDim.x - 1 && tid == 0) {
      __threadfence();
      float v = -INFINITY;
      int ix = 0x7fffffff;
      for (int b = 0; b < (int)gridDim.x; ++b) {
        const float vb = __ldcg(p.am_val + b);
        const int ib = __ldcg(p.am_idx + b);
        if (vb > v || (vb == v && ib < ix)) v = vb, ix = ib;
      }
      if (p.argmax_out) p.argmax_out[0] = ix == 0x7fffffff ? 0 : ix;
      *p.counter = 0;
    }
  }
  // no bulk copy may still be landing in this warp's stages when the CTA exits:
  // after a timeout, wait (bounded) for every item issued from the one that
  // timed out on (at most one per stage)
  if (abort_ && lane == 0)
    for (int i = abort_it; i < issued; ++i) mbar_wait_bounded(&wbar[i % NS], (uint32_t)((i / NS) & 1), p.wait_ns);
}

size_t tma_fixed_bytes(int dot, int krm, int k) {
  return x_region_bytes(dot, krm, k) + 64 * 4 + 2 * kWarps * 4 + 128 + kWarps * kMaxStages * 8;
}

int gemv_dot_kind() {
  static int kind = -1;
  if (kind < 0) {
    const char* e = getenv("Q4G_GEMV_DOT");
    kind = !e ? -1 : e[0] == 'h' ? DOT_FMA_HALF : e[0] == 'f' ? DOT_FMA : DOT_INT;
  }
  return kind;
}

template <int KRM, int DOT>
cudaError_t launch_tma_d(const GemvParams& p, cudaStream_t st, bool pdl) {
  static size_t configured = 0;
  const size_t smem = tma_fixed_bytes(DOT, KRM, p.k) + (size_t)kWarps * p.ns * p.stage_bytes;
  cudaError_t e;
  if (smem > configured) {
    e = cudaFuncSetAttribute(gemv_q4_tma_kernel<KRM, DOT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(gemv_q4_tma_kernel<KRM, DOT>, cudaFuncAttributePreferredSharedMemoryCarveout,
                             cudaSharedmemCarveoutMaxShared);
    if (e != cudaSuccess) return e;
    configured = smem;
  }
  int grid = device_sm_count();
  const int min_units = (p.n_units + kWarps - 1) / kWarps;
  if (grid > min_units) grid = min_units;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kWarpThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, gemv_q4_tma_kernel<KRM, DOT>, p);
}

template <int KRM>
cudaError_t launch_tma_t(const GemvParams& p, int dot, cudaStream_t st, bool pdl) {
  if (dot == DOT_INT) return launch_tma_d<KRM, DOT_INT>(p, st, pdl);
  if (dot == DOT_FMA) return launch_tma_d<KRM, DOT_FMA>(p, st, pdl);
  return launch_tma_d<KRM, DOT_FMA_HALF>(p, st, pdl);
}

__device__ int32_t g_error_word;

bool aligned16(const void* q) { return ((uintptr_t)q & 15) == 0; }

// Column chunk and stage count: the largest chunk (a multiple of 256 columns
// dividing k) whose stages fit beside x with 3 stages per warp, then as many
// stages (<= 4) as fit. The integer dot falls back to the fp16 one when its
// larger x region leaves no room.
bool plan_tma(GemvParams& p, int& dot) {
  const int k = p.k;
  if (k % 256 != 0) return false;
  if (p.epi == EPI_HEAD && p.kr != 1) return false;
  for (int s = 0; s < p.nseg; ++s)
    if (!aligned16(p.seg[s].qs) || !aligned16(p.seg[s].sc) || (s < p.nseg - 1 && p.seg[s].rows % 2))
      return false;
  if (p.pro == PRO_X16 && !aligned16(p.x)) return false;
  const int krm = p.kr <= 1 ? 1 : p.kr <= 2 ? 2 : p.kr <= 4 ? 4 : 8;
  const size_t budget = 220 * 1024;
  // default: the integer dot on the vocabulary head (measured faster there), the
  // fp16 one elsewhere (its smaller x region leaves longer chunks)
  if (dot < 0) dot = p.epi == EPI_HEAD ? DOT_INT : DOT_FMA_HALF;
  for (int pass = 0; pass < 2; ++pass) {
    const int d = pass == 0 ? dot : DOT_FMA;
    if (pass == 1 && dot != DOT_INT) break;
    const size_t fixed = tma_fixed_bytes(d, krm, k);
    if (fixed + 48 * 1024 > budget) continue;
    int best = 0;
    for (int kc = 256; kc <= k && kc <= 4096; kc += 256) {
      if (k % kc) continue;
      const size_t stage = ((size_t)kc / 2 + (size_t)kc / 16) * 2;
      if (fixed + (size_t)kWarps * 3 * stage <= budget) best = kc;
    }
    if (!best) continue;
    const size_t stage = ((size_t)best / 2 + (size_t)best / 16) * 2;
    int ns = 3;
    while (ns < kMaxStages && fixed + (size_t)kWarps * (ns + 1) * stage <= budget) ++ns;
    p.kc = best;
    p.ns = ns;
    p.stage_bytes = (int)stage;
    p.n_units = p.epi == EPI_GEGLU ? p.seg[0].rows : (p.n_rows + 1) / 2;
    dot = d;
    return true;
  }
  return false;
}

template <int KRM>
cudaError_t launch_t(const GemvParams& p, cudaStream_t st, bool pdl) {
  static int configured_smem = 0;
  static int blocks_per_sm = 0;
  const size_t smem = gemv_smem_bytes(KRM, p.k);
  cudaError_t e;
  if ((int)smem > configured_smem) {
    e = cudaFuncSetAttribute(gemv_q4_kernel<KRM>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(gemv_q4_kernel<KRM>, cudaFuncAttributePreferredSharedMemoryCarveout,
                             cudaSharedmemCarveoutMaxShared);
    if (e != cudaSuccess) return e;
    configured_smem = (int)smem;
    blocks_per_sm = 0;
  }
  int bps = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&bps, gemv_q4_kernel<KRM>, kThreads, smem);
  if (e != cudaSuccess) return e;
  (void)blocks_per_sm;
  if (bps < 1) return cudaErrorInvalidConfiguration;
  if (bps > 2) bps = 2;
  int grid = bps * device_sm_count();
  if (grid > p.n_units) grid = p.n_units;
  if (grid < 1) grid = 1;

  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, gemv_q4_kernel<KRM>, p);
}

}  // namespace

size_t gemv_smem_bytes(int krm, int k) {
  const size_t nb = (size_t)k / 32;
  return (size_t)krm * 4 * nb * 16 + (size_t)krm * nb * 4 + 8 * 16 * (size_t)krm * 4 + 64 * 4;
}

int gemv_max_rows(int k) {
  const size_t limit = 200 * 1024;
  int best = 1;
  for (int r : {1, 2, 4, 8})
    if (gemv_smem_bytes(r, k) <= limit) best = r;
  return best;
}

NextGemv gemv_next_desc(const GemvParams& p_in, float frac) {
  NextGemv nx{};
  GemvParams p = p_in;
  int dot = gemv_dot_kind();
  if (getenv("Q4G_GEMV_REGISTER_PATH") || !plan_tma(p, dot)) return nx;
  int grid = device_sm_count();
  const int min_units = (p.n_units + kWarps - 1) / kWarps;
  if (grid > min_units) grid = min_units;
  for (int s = 0; s < 3; ++s) nx.seg[s] = p.seg[s];
  nx.nseg = p.nseg;
  nx.k = p.k;
  nx.n_units = p.n_units;
  nx.geglu = p.epi == EPI_GEGLU;
  nx.tw = grid * kWarps;
  nx.frac = frac;
  return nx;
}

int32_t* device_error_word() {
  static int32_t* ptr[64];
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) return nullptr;
  if (!ptr[dev]) {
    void* a = nullptr;
    if (cudaGetSymbolAddress(&a, g_error_word) != cudaSuccess) return nullptr;
    ptr[dev] = (int32_t*)a;
  }
  return ptr[dev];
}

cudaError_t launch_gemv(const GemvParams& p_in, cudaStream_t st, bool pdl) {
  GemvParams p = p_in;
  int dot = gemv_dot_kind();
  if (!getenv("Q4G_GEMV_REGISTER_PATH") && plan_tma(p, dot)) {
    if (!p.err) p.err = device_error_word();
    if (!p.err) return cudaErrorInvalidValue;
    if (!p.wait_ns) p.wait_ns = 2000000000ull;
    if (p.kr <= 1) return launch_tma_t<1>(p, dot, st, pdl);
    if (p.kr <= 2) return launch_tma_t<2>(p, dot, st, pdl);
    if (p.kr <= 4) return launch_tma_t<4>(p, dot, st, pdl);
    return launch_tma_t<8>(p, dot, st, pdl);
  }
  if (p.kr <= 1) return launch_t<1>(p, st, pdl);
  if (p.kr <= 2) return launch_t<2>(p, st, pdl);
  if (p.kr <= 4) return launch_t<4>(p, st, pdl);
  return launch_t<8>(p, st, pdl);
}

int device_sm_count() {
  static int n = 0;
  if (n == 0) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (n <= 0) n = 1;
  }
  return n;
}

}  // namespace q4g
