// q4_0 matrix-vector product with the dequantisation fused into the dot product.
//
// Operation ("Gemma 4 12B" page, intro: per-block-32 absmax symmetric int4;
// "gemma-4-E4B-CoreAI", Provenance: the q4_0 grid): y[j][r] = sum_c w(r,c) x[j][c]
// with w(r,c) = (code - 8) * d(r, c/32), x fp16, fp32 accumulation.
//
// Kernels (one operation, chosen per call; see launch_gemv):
//   * stage kernel (default, 1-4 activation rows): one CTA per SM streams a
//     contiguous range of 16-36 KB row stages through a bulk-copy ring; every
//     compute warp works on every stage (a column chunk of a row group), with the
//     integer block dot (16-bit block fixed-point x, dp4a over the raw nibble
//     codes); a reducer warp adds the chunk partials in a fixed order, runs the
//     epilogue and refills the slot;
//   * warp-streamed kernel: each warp streams its own row pairs through its own
//     ring, fp16 nibble unpacking with mixed-precision FMAs (the fallback for 5-8
//     activation rows);
//   * register kernel (below): plain streaming loads, any k % 32 == 0;
//   * fp16 GEMV (end of the file): the fp16 tied head.
// The fused prologues (RMSNorm, residual, layer scalar) and epilogues (store,
// GeGLU, softcap + logits + argmax) are shared by all of them. The first weight
// loads of every kernel are issued before griddepcontrol.wait, so with
// programmatic dependent launch they overlap the previous kernel's tail.
//
// Register kernel, work decomposition (one launch, each CTA looping over 16-row units):
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
//     and in a fixed order across warps through shared memory (deterministic).
#include "q4g_common.cuh"
#include "q4g_dot.cuh"
#include "q4g_internal.h"

#include <stdlib.h>

#include <algorithm>
#include <atomic>

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

// The activations of the step, produced in groups of 4 consecutive columns:
//   PRO_X16:   x = the fp16 input rows
//   PRO_RESID: r_new = (r_in + rmsnorm(delta) * w_delta) * scale,
//              x = fp16(rmsnorm(r_new) * w_x); block 0 stores r_new (and the dump)
// emit(j, c4, h, valid) receives columns 4*c4 .. 4*c4+3 of row j. Every thread
// calls emit the same number of times per row (valid = false past the end), so
// emit may use warp shuffles; with NT % 8 == 0 the 8 groups of one 32-column
// block sit in 8 consecutive lanes. Needs k <= 8192 for PRO_RESID.
template <int KRM, int NT, class Emit>
Q4G_DEV void produce_x(const GemvParams& p, float* misc, Emit&& emit) {
  const int k = p.k, tid = threadIdx.x, n4 = k >> 2;
  for (int j = 0; j < KRM; ++j) {
    if (j >= p.kr) break;
    if (p.pro == PRO_X16) {
      const __half* xr = p.x + (size_t)j * p.x_stride;
      const bool vec = (((uintptr_t)xr) & 7) == 0;
      const int iters = (n4 + NT - 1) / NT;
      constexpr int kHoist = (15360 / 4 + NT - 1) / NT;  // rounds whose loads are issued together
      if (vec && iters <= kHoist) {
        // every load first (one round trip), then the rounds; iters is the same
        // for the whole CTA, so a round is skipped by whole warps
        uint2 v[kHoist];
#pragma unroll
        for (int i = 0; i < kHoist; ++i) {
          const int c4 = tid + i * NT;
          v[i] = c4 < n4 ? *reinterpret_cast<const uint2*>(xr + 4 * c4) : make_uint2(0u, 0u);
        }
#pragma unroll
        for (int i = 0; i < kHoist; ++i) {
          if (i < iters) {
            const int c4 = tid + i * NT;
            const __half* hv = reinterpret_cast<const __half*>(&v[i]);
            const __half h[4] = {hv[0], hv[1], hv[2], hv[3]};
            emit(j, c4, h, c4 < n4);
          }
        }
        continue;
      }
      for (int i = 0; i < iters; ++i) {
        const int c4 = tid + i * NT;
        const bool valid = c4 < n4;
        __half h[4];
        if (valid && vec) {
          const uint2 v = *reinterpret_cast<const uint2*>(xr + 4 * c4);
          const __half* hv = reinterpret_cast<const __half*>(&v);
#pragma unroll
          for (int e = 0; e < 4; ++e) h[e] = hv[e];
        } else {
#pragma unroll
          for (int e = 0; e < 4; ++e) h[e] = valid ? xr[4 * c4 + e] : __float2half_rn(0.f);
        }
        emit(j, c4, h, valid);
      }
    } else {
      // k <= 8192: each thread keeps its float4s of r_new in registers
      constexpr int R4 = (8192 + 4 * NT - 1) / (4 * NT);
      const float4* rin = reinterpret_cast<const float4*>(p.r_in + (size_t)j * k);
      const float4* dl = p.delta ? reinterpret_cast<const float4*>(p.delta + (size_t)j * k) : nullptr;
      const float4* wd = reinterpret_cast<const float4*>(p.w_delta);
      const float4* wx = reinterpret_cast<const float4*>(p.w_x);
      // every global load of the prologue in one round (the gains do not
      // depend on the reductions)
      float4 rn[R4], dv[R4], wdv[R4], wxv[R4];
#pragma unroll
      for (int i = 0; i < R4; ++i) {
        const int c4 = tid + i * NT;
        if (c4 < n4) {
          rn[i] = rin[c4];
          wxv[i] = wx[c4];
          if (dl) dv[i] = dl[c4], wdv[i] = wd[c4];
        }
      }
      float ss = 0.f;
#pragma unroll
      for (int i = 0; i < R4; ++i) {
        const int c4 = tid + i * NT;
        if (c4 < n4 && dl) {
          ss = fmaf(dv[i].x, dv[i].x, ss);
          ss = fmaf(dv[i].y, dv[i].y, ss);
          ss = fmaf(dv[i].z, dv[i].z, ss);
          ss = fmaf(dv[i].w, dv[i].w, ss);
        }
      }
      if (p.trace && blockIdx.x == 0 && tid == 0) p.trace[3] = global_ns();
      if (dl) {
        const float inv_d = rms_inv(block_sum<NT>(ss, misc), k, p.eps);
#pragma unroll
        for (int i = 0; i < R4; ++i) {
          const int c4 = tid + i * NT;
          if (c4 < n4) {
            const float4 w = wdv[i];
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
      if (p.trace && blockIdx.x == 0 && tid == 0) p.trace[4] = global_ns();
#pragma unroll
      for (int i = 0; i < R4; ++i) {
        if (i * NT >= n4) break;  // no thread of the CTA has columns left
        const int c4 = tid + i * NT;
        const bool valid = c4 < n4;
        __half h[4];
        if (valid) {
          const float4 w = wxv[i];
          h[0] = __float2half_rn(__fmul_rn(__fmul_rn(rn[i].x, inv_r), w.x));
          h[1] = __float2half_rn(__fmul_rn(__fmul_rn(rn[i].y, inv_r), w.y));
          h[2] = __float2half_rn(__fmul_rn(__fmul_rn(rn[i].z, inv_r), w.z));
          h[3] = __float2half_rn(__fmul_rn(__fmul_rn(rn[i].w, inv_r), w.w));
        } else {
#pragma unroll
          for (int e = 0; e < 4; ++e) h[e] = __float2half_rn(0.f);
        }
        emit(j, c4, h, valid);
      }
    }
  }
}

// Activations into shared memory in the order the fp16 nibble unpacking
// consumes them, plus the per-block constant 72 * sum(x) that removes the +64
// of the unpacked codes and the -8 of the code offset. Ends with __syncthreads().
template <int KRM, int NT = kThreads>
Q4G_DEV void stage_x(const GemvParams& p, uint4* xs, float* cblk, float* misc) {
  const int nb = p.k >> 5, tid = threadIdx.x;
  __half* xs_h = reinterpret_cast<__half*>(xs);
  produce_x<KRM, NT>(p, misc, [&](int j, int c4, const __half (&h)[4], bool valid) {
    if (valid) {
#pragma unroll
      for (int e = 0; e < 4; ++e) put_x(xs_h, nb, j, 4 * c4 + e, h[e]);
    }
  });
  __syncthreads();
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



// Activations as the digits of the integer dot product (block_dot_int):
// thread (block blk, group sub) turns columns 4*sub..4*sub+3 of the block into
// one 32-bit word per digit; the block's largest exponent and digit sums are
// reduced over the block's 8 lanes. Ends with __syncthreads().
template <int KRM, int NT>
Q4G_DEV void stage_digits(const GemvParams& p, uint4* dg, int4* bc, float* misc) {
  const int nb = p.k >> 5;
  uint32_t* dw = reinterpret_cast<uint32_t*>(dg);
  produce_x<KRM, NT>(p, misc, [&](int j, int c4, const __half (&h)[4], bool valid) {
    const int blk = c4 >> 3, sub = c4 & 7;
    int em = max(max(half_exp(h[0]), half_exp(h[1])), max(half_exp(h[2]), half_exp(h[3])));
    em = max(em, __shfl_xor_sync(0xffffffffu, em, 1));
    em = max(em, __shfl_xor_sync(0xffffffffu, em, 2));
    em = max(em, __shfl_xor_sync(0xffffffffu, em, 4));
    uint32_t wdg[2];
    int sd[2] = {0, 0};
    digits4(h, em, wdg, sd);
    int s0 = sd[0], s1 = sd[1];
#pragma unroll
    for (int o = 1; o < 8; o <<= 1) {
      s0 += __shfl_xor_sync(0xffffffffu, s0, o);
      s1 += __shfl_xor_sync(0xffffffffu, s1, o);
    }
    if (valid) {
      const int hh = sub >> 2, wd = sub & 3;
      dw[((size_t)(j * kDigitQuads + 0 + hh) * nb + blk) * 4 + wd] = wdg[0];
      dw[((size_t)(j * kDigitQuads + 2 + hh) * nb + blk) * 4 + wd] = wdg[1];
      if (sub == 0) bc[j * nb + blk] = make_int4(-8 * s0, -8 * s1, 0, (em - 29 + 127) << 23);
    }
  });
  __syncthreads();
}


// The activation rows as fp16 in shared memory ([KRM][k]), from the fused
// residual/RMSNorm prologue. Ends with __syncthreads().
template <int KRM, int NT>
Q4G_DEV void stage_x_half(const GemvParams& p, __half* xh, float* misc) {
  const int k = p.k;
  produce_x<KRM, NT>(p, misc, [&](int j, int c4, const __half (&h)[4], bool valid) {
    if (valid) {
      __half2* d = reinterpret_cast<__half2*>(xh + (size_t)j * k + 4 * c4);
      d[0] = __halves2half2(h[0], h[1]);
      d[1] = __halves2half2(h[2], h[3]);
    }
  });
  __syncthreads();
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


// Shared memory of the warp-streamed kernel: the x region (layout per dot
// kind), then 64 floats of reduction scratch, per-warp argmax candidates, the
// mbarriers and the stages.
enum : int { DOT_FMA_HALF = 0, DOT_FMA = 1, DOT_INT = 2 };

__host__ __device__ inline size_t x_region_bytes(int dot, int krm, int k) {
  const size_t nb = (size_t)k / 32;
  return dot == DOT_INT ? (size_t)krm * nb * (16 * kDigitQuads + 16) : (size_t)krm * nb * (64 + 4);
}

template <int KRM, int DOT>
__global__ void __launch_bounds__(kWarpThreads, 1) gemv_q4_tma_kernel(const GemvParams p) {
  extern __shared__ __align__(16) unsigned char ws_smem[];
  const int k = p.k, nb = k >> 5, NS = p.ns;
  const int kc = p.kc, nbc = kc >> 5, qb = kc >> 1;
  // x region
  uint4* xs = reinterpret_cast<uint4*>(ws_smem);                        // FMA: [KRM][4][nb]; INT: dg [KRM][kDigitQuads][nb]
  float* cblk = reinterpret_cast<float*>(xs + (size_t)KRM * 4 * nb);     // FMA: [KRM][nb]
  int4* bc = reinterpret_cast<int4*>(xs + (size_t)KRM * kDigitQuads * nb);  // INT: [KRM][nb]
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
  }
  __syncwarp();

  pdl_wait();
  if (DOT == DOT_INT) {
    stage_digits<KRM, kWarpThreads>(p, xs, bc, misc);
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
                uint4 g[kDigitQuads];
#pragma unroll
                for (int q = 0; q < kDigitQuads; ++q) g[q] = lds_u4(xs + (size_t)(j * kDigitQuads + q) * nb + blk);
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
      ++issued;
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

// ---------------------------------------------------------------------------
// Helpers of the bulk-copy ring (stage kernel).
// ---------------------------------------------------------------------------

// Wait for `phase` of `bar` until done, until another warp gave up (flag set),
// or until limit_ns pass (then this warp sets the flag and the error word).
Q4G_DEV bool cs_wait(uint64_t* bar, uint32_t phase, const GemvParams& p, volatile int* abort_flag) {
  if (mbar_try_wait(bar, phase)) return true;
  const uint64_t t0 = global_ns();
  for (int it = 0; it < kSpinLimit; ++it) {
    if (*abort_flag) return false;
    if (mbar_try_wait(bar, phase)) return true;
    if (global_ns() - t0 > p.wait_ns) break;
  }
  *abort_flag = 1;
  atomicOr(p.err, 1);
  return false;
}

// Issue the bulk copies of unit u into stage `st` ([R rows of codes][R rows of scales]).
template <int R>
Q4G_DEV void cs_issue(const GemvParams& p, int u, unsigned char* st, uint64_t* bar, bool poison, uint64_t pol) {
  const int kh = p.k >> 1, nb = p.k >> 5;
  if (p.epi == EPI_GEGLU) {
    const int r0 = (R / 2) * u;
    const uint32_t qb = (uint32_t)(R / 2) * kh, sb = (uint32_t)(R / 2) * nb * 2;
    mbar_arrive_expect_tx(bar, 2 * (qb + sb) + (poison ? 16u : 0u));
    bulk_g2s_hint(st, p.seg[0].qs + (size_t)r0 * kh, qb, bar, pol);
    bulk_g2s_hint(st + qb, p.seg[1].qs + (size_t)r0 * kh, qb, bar, pol);
    bulk_g2s_hint(st + 2 * qb, p.seg[0].sc + (size_t)r0 * nb, sb, bar, pol);
    bulk_g2s_hint(st + 2 * qb + sb, p.seg[1].sc + (size_t)r0 * nb, sb, bar, pol);
  } else {
    const GemvSeg* sg;
    int r0;
    seg_row(p, R * u, sg, r0);
    const int n = min(R, sg->rows - r0);
    const uint32_t qb = (uint32_t)n * kh, sb = (uint32_t)n * nb * 2;
    mbar_arrive_expect_tx(bar, qb + sb + (poison ? 16u : 0u));
    bulk_g2s_hint(st, sg->qs + (size_t)r0 * kh, qb, bar, pol);
    bulk_g2s_hint(st + (size_t)R * kh, sg->sc + (size_t)r0 * nb, sb, bar, pol);
  }
}

// ---------------------------------------------------------------------------
// Stage kernel: every compute warp works on every stage.
//
// One CTA per SM streams a contiguous range of R-row stages through a ring of
// NS shared-memory slots ([R rows of codes][R rows of scales] per slot). The R
// rows of a stage form G groups of RG rows and the columns NC chunks of 32
// blocks; compute warp (c, g) takes chunk c of group g, so the NC * G warps go
// through the ring together, in order. A warp sums its RG rows over its lanes,
// writes one partial per row and arrives on ready[s]. The reducer warp waits
// for ready[s], adds the NC partials of each row in chunk order
// (deterministic), runs the epilogue and refills slot s with the stage NS
// ahead: one warp hands every slot back, so there is no empty barrier and no
// per-slot bookkeeping between several consumer groups. Every wait is bounded
// (error word and abort flag); after a timeout the reducer waits, bounded, for
// the copies still in flight.
// ---------------------------------------------------------------------------
constexpr int kStageCompute = 16;
constexpr int kStageThreads = (kStageCompute + 1) * 32;
constexpr int kStageMaxSlots = 16;

__host__ __device__ inline size_t stage_red_bytes(int ns, int nc, int rows, int krm) {
  return ((size_t)ns * nc * rows * krm * 4 + 15) & ~(size_t)15;
}
// x region: the normed fp16 rows (PRO_RESID only; PRO_X16 lanes read x itself)
__host__ __device__ inline size_t stage_x_bytes(int krm, int k, int pro) {
  return pro == PRO_RESID ? (size_t)krm * k * 2 : 0;
}
__host__ __device__ inline size_t stage_fixed_bytes(int krm, int k, int pro, int ns, int nc, int rows) {
  return stage_x_bytes(krm, k, pro) + 64 * 4 + stage_red_bytes(ns, nc, rows, krm) + 128 + 2 * kStageMaxSlots * 8;
}

template <int KRM, int R, int RG>
__global__ void __launch_bounds__(kStageThreads, 1) gemv_q4_stage_kernel(const GemvParams p) {
  extern __shared__ __align__(16) unsigned char sk_smem[];
  constexpr int G = R / RG;
  const int k = p.k, nb = k >> 5, kh = k >> 1, NS = p.ns, NC = p.nchunk;
  __half* xh = reinterpret_cast<__half*>(sk_smem);                        // PRO_RESID: [KRM][k]
  float* misc = reinterpret_cast<float*>(sk_smem + stage_x_bytes(KRM, k, p.pro));  // 64 floats
  float* red = misc + 64;                                                 // [NS][NC][R][KRM]
  uint64_t* bars = reinterpret_cast<uint64_t*>(
      ((uintptr_t)(reinterpret_cast<unsigned char*>(red) + stage_red_bytes(NS, NC, R, KRM)) + 127) &
      ~(uintptr_t)127);
  uint64_t* full = bars;                    // [kStageMaxSlots]: the stage's bytes landed
  uint64_t* ready = bars + kStageMaxSlots;  // [kStageMaxSlots]: every compute warp wrote its partials
  unsigned char* stages = reinterpret_cast<unsigned char*>(bars + 2 * kStageMaxSlots);
  __shared__ int s_abort, s_ticket;
  __shared__ float s_bestv[KRM];
  __shared__ int s_besti[KRM];

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int n_comp = NC * G;
  const bool reducer = warp == kStageCompute;
  const int u0 = (int)((long long)blockIdx.x * p.n_units / gridDim.x);
  const int n_st = (int)((long long)(blockIdx.x + 1) * p.n_units / gridDim.x) - u0;
  const size_t SB = (size_t)p.stage_bytes;
  const uint64_t pol = policy_evict_first();
  int issued = 0;
  uint64_t* const tr = blockIdx.x == 0 ? p.trace : nullptr;
  auto stamp = [&](int i) {
    if (tr) tr[i] = global_ns();
  };

  if (tid == 0) stamp(0), s_abort = 0;
  if (reducer && lane == 0) {
    for (int s = 0; s < NS; ++s) mbar_init(&full[s], 1), mbar_init(&ready[s], n_comp);
    fence_mbar_init();
    const int pre = p.prefetch_stages > 0 ? min(NS, p.prefetch_stages) : NS;
    for (; issued < pre && issued < n_st; ++issued) {
      cs_issue<R>(p, u0 + issued, stages + issued * SB, &full[issued],
                  p.stall_test && u0 == 0 && issued == 0, pol);  // the CTA owning unit 0
      if (issued < 64) stamp(8 + issued);
    }
  }
  __syncthreads();  // barriers initialised before any wait
  pdl_wait();
  if (tid == 0) stamp(1);
  if (p.pro == PRO_RESID) stage_x_half<KRM, kStageThreads>(p, xh, misc);  // ends with __syncthreads
  volatile int* abort_flag = &s_abort;

  // compute warp (c, g): chunk c of row group g. Lane l holds block 32 c + l of
  // every row and builds that block's x digits itself; a lane past the end of
  // the row reads block nb - 1 with zero digits and a zero x scale (no branch).
  const int c = warp % NC, g = warp / NC;
  const int blk = 32 * c + lane;
  const bool has = warp < n_comp && blk < nb;
  uint4 xg[KRM][kDigitQuads];
  int4 cv[KRM];
  float xsc[KRM];
#pragma unroll
  for (int j = 0; j < KRM; ++j) {
    if (has && (KRM == 1 || j < p.kr)) {
      const __half* xb = p.pro == PRO_RESID ? xh + (size_t)j * k + 32 * blk : p.x + (size_t)j * p.x_stride + 32 * blk;
      uint4 xv[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) xv[q] = *reinterpret_cast<const uint4*>(xb + 8 * q);
      lane_block_digits(xv, xg[j], cv[j]);
    } else {
#pragma unroll
      for (int q = 0; q < kDigitQuads; ++q) xg[j][q] = make_uint4(0, 0, 0, 0);
      cv[j] = make_int4(0, 0, 0, 0);
    }
    xsc[j] = __int_as_float(cv[j].w);
  }
  // x read from global: its loads go first, the weight stream resumes after
  if (p.pro != PRO_RESID) __syncthreads();
  if (tid == 0) stamp(2);
  pdl_launch_dependents();

  if (warp < n_comp) {
    const int qoff = 16 * min(blk, nb - 1), soff = 2 * min(blk, nb - 1);
    int s = 0;
    uint32_t ph = 0;
    for (int t = 0; t < n_st; ++t) {
      // warp-uniform decisions: lanes that waited for different lengths of time must
      // all enter the block below (it holds warp collectives) or all leave
      if (!__any_sync(0xffffffffu, *abort_flag != 0)) cs_wait(&full[s], ph, p, abort_flag);
      if (__any_sync(0xffffffffu, *abort_flag != 0)) break;
      if (c == 0 && g == 0 && lane == 0 && t < 64) stamp(72 + t);
      const unsigned char* st = stages + s * SB + (size_t)g * RG * kh + qoff;
      const unsigned char* ss = stages + s * SB + (size_t)R * kh + (size_t)g * RG * 2 * nb + soff;
      float v[KRM][RG];
#pragma unroll
      for (int r = 0; r < RG; ++r) {
        const uint4 qv = *reinterpret_cast<const uint4*>(st + r * kh);
        const float d = __half2float(*reinterpret_cast<const __half*>(ss + r * 2 * nb));
#pragma unroll
        for (int j = 0; j < KRM; ++j)
          v[j][r] = (KRM == 1 || j < p.kr) ? d * xsc[j] * block_dot_int(qv, xg[j], cv[j]) : 0.f;
      }
      float* rs = red + (size_t)s * NC * R * KRM;  // [NC][R][KRM] of this slot
#pragma unroll
      for (int j = 0; j < KRM; ++j) {
        const float tot = cs_reduce_rows<RG>(v[j], lane);
        if ((lane & (32 / RG - 1)) == 0) rs[((size_t)c * R + g * RG + cs_row<RG>(lane)) * KRM + j] = tot;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&ready[s]);  // release of the partials above
      if (++s == NS) s = 0, ph ^= 1u;
    }
  } else if (reducer) {
    // ---------------- reducer: partials -> epilogue, then refill the slot ----------------
    if (lane == 0) {  // the first stages not issued before the dependency wait
      for (; issued < NS && issued < n_st; ++issued) {
        cs_issue<R>(p, u0 + issued, stages + issued * SB, &full[issued], false, pol);
        if (issued < 64) stamp(8 + issued);
      }
    }
    float best_v = -INFINITY;  // of activation row j (head)
    int best_i = 0x7fffffff;
    const int r = lane / KRM, j = lane % KRM;  // lanes l < R * KRM <= 32
    int s = 0;
    uint32_t ph = 0;
    for (int t = 0; t < n_st; ++t) {
      if (!__any_sync(0xffffffffu, *abort_flag != 0)) cs_wait(&ready[s], ph, p, abort_flag);
      if (__any_sync(0xffffffffu, *abort_flag != 0)) break;
      const float* rs = red + (size_t)s * NC * R * KRM;
      float val = 0.f;
      if (lane < R * KRM)
        for (int cc = 0; cc < NC; ++cc) val += rs[((size_t)cc * R + r) * KRM + j];
      const int u = u0 + t;
      if (p.epi == EPI_GEGLU) {
        const float up = __shfl_sync(0xffffffffu, val, (lane + (R / 2) * KRM) & 31);
        if (lane < (R / 2) * KRM && j < p.kr)
          p.act[(size_t)j * p.act_stride + (size_t)(R / 2) * u + r] = __float2half_rn(gelu_tanh(val) * up);
      } else if (lane < R * KRM && j < p.kr) {
        const int row = R * u + r;
        if (row < p.n_rows) {
          if (p.epi == EPI_STORE) {
            p.y[(size_t)j * p.y_stride + row] = val;
          } else {
            const float z = p.softcap * tanhf(val / p.softcap);
            if (p.logits) p.logits[(size_t)j * p.logits_stride + row] = z;
            if (z > best_v || (z == best_v && row < best_i)) best_v = z, best_i = row;
          }
        }
      }
      __syncwarp();  // every lane read slot s's partials before the refill can overwrite them
      if (lane == 0) {
        if (t < 64) stamp(136 + t);
        if (t + NS < n_st) {
          cs_issue<R>(p, u0 + t + NS, stages + s * SB, &full[s], false, pol);
          if (t + NS < 64) stamp(8 + t + NS);
          issued = t + NS + 1;
        }
      }
      if (++s == NS) s = 0, ph ^= 1u;
    }
    if (lane == 0) stamp(5);
    if (lane == 0 && p.trace_ends) p.trace_ends[blockIdx.x] = global_ns();
    if (p.epi == EPI_HEAD) {
      // lanes with the same j (lane % KRM) hold row j's candidates
#pragma unroll
      for (int o = 16; o >= KRM; o >>= 1) {
        const float v2 = __shfl_xor_sync(0xffffffffu, best_v, o);
        const int i2 = __shfl_xor_sync(0xffffffffu, best_i, o);
        if (v2 > best_v || (v2 == best_v && i2 < best_i)) best_v = v2, best_i = i2;
      }
      if (lane < KRM) s_bestv[lane] = best_v, s_besti[lane] = best_i;
    }
  }
  if (p.epi == EPI_HEAD) {
    __syncthreads();
    if (tid == 0) {
      for (int jj = 0; jj < p.kr; ++jj)
        p.am_val[jj * gridDim.x + blockIdx.x] = s_bestv[jj], p.am_idx[jj * gridDim.x + blockIdx.x] = s_besti[jj];
      __threadfence();
      s_ticket = atomicAdd(p.counter, 1);
      if (s_ticket == (int)gridDim.x - 1) {
        __threadfence();
        for (int jj = 0; jj < p.kr; ++jj) {
          float v = -INFINITY;
          int ix = 0x7fffffff;
          for (int b = 0; b < (int)gridDim.x; ++b) {
            const float vb = __ldcg(p.am_val + jj * gridDim.x + b);
            const int ib = __ldcg(p.am_idx + jj * gridDim.x + b);
            if (vb > v || (vb == v && ib < ix)) v = vb, ix = ib;
          }
          if (p.argmax_out) p.argmax_out[jj] = ix == 0x7fffffff ? 0 : ix;
        }
        *p.counter = 0;
      }
    }
  }
  // after a timeout, wait (bounded) for the copies still in flight
  if (reducer && lane == 0 && *abort_flag) {
    for (int t = issued > NS ? issued - NS : 0; t < issued; ++t)
      mbar_wait_bounded(&full[t % NS], (uint32_t)((t / NS) & 1), p.wait_ns);
  }
}

// Plan of the stage kernel: R rows per stage (about 16-36 KB), NC = 32-block
// chunks, G row groups of RG rows, NS slots within the shared-memory budget.
bool plan_stage(GemvParams& p, int& R, int& RG) {
  const int k = p.k, nb = k >> 5;
  if (k % 256 != 0 || p.kr > 4) return false;
  if (p.epi == EPI_GEGLU && (p.nseg != 2 || p.seg[0].rows != p.seg[1].rows || p.seg[0].rows % 8)) return false;
  if (p.pro == PRO_RESID && k > 8192) return false;
  for (int s = 0; s < p.nseg; ++s)
    if (!aligned16(p.seg[s].qs) || !aligned16(p.seg[s].sc) || (s < p.nseg - 1 && p.seg[s].rows % 16))
      return false;
  if (p.pro == PRO_X16 && (!aligned16(p.x) || (p.kr > 1 && p.x_stride % 8))) return false;
  const int NC = (nb + 31) / 32;
  if (NC > kStageCompute) return false;
  const int krm = p.kr <= 1 ? 1 : p.kr <= 2 ? 2 : 4;
  const size_t row_bytes = (size_t)k / 2 + (size_t)k / 16;
  R = 16;
  while (R > 2 && (size_t)R * row_bytes > 36 * 1024) R /= 2;
  if (p.epi == EPI_GEGLU) R = std::max(R, 4);
  while (R * krm > 32) R /= 2;  // one reducer lane per (row, activation row)
  auto units = [&](int r) { return p.epi == EPI_GEGLU ? p.seg[0].rows / (r / 2) : (p.n_rows + r - 1) / r; };
  // keep every SM busy on small matrices
  while (R > 4 && units(R) < 2 * device_sm_count()) R /= 2;
  // four activation rows: two rows per compute warp (the x digits of four rows
  // take most of a lane's registers), so R <= 2 * (compute warps per chunk)
  if (krm == 4) {
    int gmax = kStageCompute / NC;
    while (gmax & (gmax - 1)) --gmax;
    while (R > 2 && R / 2 > gmax) R /= 2;
    if (p.epi == EPI_GEGLU && R < 4) return false;
  }
  int G = std::min(kStageCompute / NC, R == 16 ? 4 : R / 2);
  while (G > 1 && (G & (G - 1))) --G;  // power of two, divides R
  RG = R / G;
  if (R == 16 && RG != 4) return false;
  if (RG != 2 && RG != 4) return false;
  const size_t budget = 220 * 1024, stage = (size_t)R * row_bytes;
  int ns = 0;
  for (int n = kStageMaxSlots; n >= 2; --n)
    if (stage_fixed_bytes(krm, k, p.pro, n, NC, R) + (size_t)n * stage <= budget) {
      ns = n;
      break;
    }
  if (ns < 4) return false;
  // stages issued before the dependency wait: measured best at 2 (more delays
  // the prologue's own loads behind the weight stream)
  p.prefetch_stages = 2;
  p.ns = ns;
  p.nchunk = NC;
  p.groups = G;
  p.stage_rows = R;
  p.stage_bytes = (int)stage;
  p.n_units = units(R);
  return true;
}

template <int KRM, int R, int RG>
cudaError_t launch_stage_r(const GemvParams& p, cudaStream_t st, bool pdl) {
  static size_t configured = 0;
  const size_t smem = stage_fixed_bytes(KRM, p.k, p.pro, p.ns, p.nchunk, R) + (size_t)p.ns * p.stage_bytes;
  cudaError_t e;
  if (smem > configured) {
    e = cudaFuncSetAttribute(gemv_q4_stage_kernel<KRM, R, RG>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(gemv_q4_stage_kernel<KRM, R, RG>, cudaFuncAttributePreferredSharedMemoryCarveout,
                             cudaSharedmemCarveoutMaxShared);
    if (e != cudaSuccess) return e;
    configured = smem;
  }
  int grid = device_sm_count();
  if (grid > p.n_units) grid = p.n_units;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kStageThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, gemv_q4_stage_kernel<KRM, R, RG>, p);
}

template <int KRM>
cudaError_t launch_stage_t(const GemvParams& p, int R, int RG, cudaStream_t st, bool pdl) {
  if constexpr (KRM == 4) {  // two rows per compute warp (plan_stage)
    if (RG != 2 || R > 8) return cudaErrorInvalidValue;
    if (R == 8) return launch_stage_r<4, 8, 2>(p, st, pdl);
    if (R == 4) return launch_stage_r<4, 4, 2>(p, st, pdl);
    return launch_stage_r<4, 2, 2>(p, st, pdl);
  } else {
    if (R == 16) return launch_stage_r<KRM, 16, 4>(p, st, pdl);
    if (R == 8) return RG == 4 ? launch_stage_r<KRM, 8, 4>(p, st, pdl) : launch_stage_r<KRM, 8, 2>(p, st, pdl);
    if (R == 4) return RG == 4 ? launch_stage_r<KRM, 4, 4>(p, st, pdl) : launch_stage_r<KRM, 4, 2>(p, st, pdl);
    return launch_stage_r<KRM, 2, 2>(p, st, pdl);
  }
}

// Kernel choice (q4g_set_gemv_kernel): -1 automatic, 1 warp-streamed,
// 2 register path, 3 stage kernel.
std::atomic<int> g_kernel_choice{-1};

int gemv_kernel_choice() { return g_kernel_choice.load(std::memory_order_relaxed); }

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
  const int choice = gemv_kernel_choice();
  int R = 0, RG = 2;
  if ((choice == 3 || choice == -1) && plan_stage(p, R, RG)) {
    if (!p.err) p.err = device_error_word();
    if (!p.err) return cudaErrorInvalidValue;
    if (!p.wait_ns) p.wait_ns = 2000000000ull;
    if (p.kr > 2) return launch_stage_t<4>(p, R, RG, st, pdl);
    return p.kr > 1 ? launch_stage_t<2>(p, R, RG, st, pdl) : launch_stage_t<1>(p, R, RG, st, pdl);
  }
  p = p_in;
  int dot = -1;
  if (choice != 2 && plan_tma(p, dot)) {
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

// ---------------------------------------------------------------------------
// GEMV with fp16 weights: the tied head in its fp16 variant ("Gemma-4-12B-CoreAI",
// tiered-v3/ section: the vocabulary path kept at fp16). The activation rows (the
// fused residual/final-norm prologue, or given fp16 rows) are staged once per CTA in
// shared memory; every warp of the grid takes rows r = warp, warp + all warps, ...;
// a lane loads its 16-byte pieces of the row (8 weights each) with streaming loads,
// all of them before the first use, and multiplies them with the matching x pieces
// (fp16 products, exact in fp32, accumulated in fp32); the row total comes from a
// warp reduction. Epilogue: softcap, logits and the argmax (per warp, per CTA, then
// the last CTA of the grid; lowest index on ties), or a plain store.
// ---------------------------------------------------------------------------
namespace {

constexpr int kF16Warps = 16;
constexpr int kF16Threads = kF16Warps * 32;
constexpr int kF16Batch = 16;  // 16-byte pieces per lane loaded before use

template <int KRM>
__global__ void __launch_bounds__(kF16Threads, 1) gemv_f16_kernel(const GemvParams p) {
  extern __shared__ __align__(16) unsigned char f16_smem[];
  const int k = p.k, tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  __half* xh = reinterpret_cast<__half*>(f16_smem);                            // [KRM][k]
  float* misc = reinterpret_cast<float*>(f16_smem + (size_t)KRM * k * 2);      // 64 floats
  float* cand_v = misc + 64;                                                   // [kF16Warps][KRM]
  int* cand_i = reinterpret_cast<int*>(cand_v + kF16Warps * KRM);              // [kF16Warps][KRM]
  __shared__ int s_ticket;
  pdl_wait();
  if (p.pro == PRO_RESID) {
    stage_x_half<KRM, kF16Threads>(p, xh, misc);  // ends with __syncthreads
  } else {
    for (int c = tid; c < p.kr * (k / 8); c += kF16Threads) {
      const int j = c / (k / 8), q = c - j * (k / 8);
      *reinterpret_cast<uint4*>(xh + (size_t)j * k + 8 * q) =
          *reinterpret_cast<const uint4*>(p.x + (size_t)j * p.x_stride + 8 * q);
    }
    __syncthreads();
  }
  pdl_launch_dependents();
  const int pieces = k / 8, per_lane = (pieces + 31) / 32;
  float best_v[KRM];
  int best_i[KRM];
#pragma unroll
  for (int j = 0; j < KRM; ++j) best_v[j] = -INFINITY, best_i[j] = 0x7fffffff;
  const int gw = blockIdx.x * kF16Warps + warp, nw = gridDim.x * kF16Warps;
  for (int r = gw; r < p.n_rows; r += nw) {
    const uint4* wrow = reinterpret_cast<const uint4*>(p.w16 + (size_t)r * k);
    float acc[KRM];
#pragma unroll
    for (int j = 0; j < KRM; ++j) acc[j] = 0.f;
    for (int i0 = 0; i0 < per_lane; i0 += kF16Batch) {  // k <= 4096: one batch
      uint4 wv[kF16Batch];
#pragma unroll
      for (int i = 0; i < kF16Batch; ++i) {
        const int c = lane + 32 * (i0 + i);
        if (i0 + i < per_lane && c < pieces) wv[i] = ld_stream_u4(wrow + c);
      }
#pragma unroll
      for (int i = 0; i < kF16Batch; ++i) {
        const int c = lane + 32 * (i0 + i);
        if (i0 + i < per_lane && c < pieces) {
#pragma unroll
          for (int j = 0; j < KRM; ++j) {
            if (KRM == 1 || j < p.kr) {
              const uint4 xv = lds_u4(xh + (size_t)j * k + 8 * c);
              acc[j] = fma2_h_f32(wv[i].x, xv.x, acc[j]);
              acc[j] = fma2_h_f32(wv[i].y, xv.y, acc[j]);
              acc[j] = fma2_h_f32(wv[i].z, xv.z, acc[j]);
              acc[j] = fma2_h_f32(wv[i].w, xv.w, acc[j]);
            }
          }
        }
      }
    }
#pragma unroll
    for (int j = 0; j < KRM; ++j) {
      const float v = warp_sum(acc[j]);
      if (lane == 0 && (KRM == 1 || j < p.kr)) {
        if (p.epi == EPI_STORE) {
          p.y[(size_t)j * p.y_stride + r] = v;
        } else {
          const float z = p.softcap * tanhf(v / p.softcap);
          if (p.logits) p.logits[(size_t)j * p.logits_stride + r] = z;
          if (z > best_v[j] || (z == best_v[j] && r < best_i[j])) best_v[j] = z, best_i[j] = r;
        }
      }
    }
  }
  if (p.epi != EPI_HEAD) return;
  // argmax: lane 0 of each warp holds its candidates; CTA, then grid (last CTA)
  if (lane == 0)
#pragma unroll
    for (int j = 0; j < KRM; ++j) cand_v[warp * KRM + j] = best_v[j], cand_i[warp * KRM + j] = best_i[j];
  __syncthreads();
  if (tid < KRM && tid < p.kr) {
    float v = -INFINITY;
    int i = 0x7fffffff;
    for (int w = 0; w < kF16Warps; ++w) {
      const float v2 = cand_v[w * KRM + tid];
      const int i2 = cand_i[w * KRM + tid];
      if (v2 > v || (v2 == v && i2 < i)) v = v2, i = i2;
    }
    p.am_val[tid * gridDim.x + blockIdx.x] = v;
    p.am_idx[tid * gridDim.x + blockIdx.x] = i;
  }
  __threadfence();
  __syncthreads();
  if (tid == 0) s_ticket = atomicAdd(p.counter, 1);
  __syncthreads();
  if (s_ticket == (int)gridDim.x - 1 && tid < p.kr) {
    __threadfence();
    float v = -INFINITY;
    int i = 0x7fffffff;
    for (int b = 0; b < (int)gridDim.x; ++b) {
      const float v2 = __ldcg(p.am_val + tid * gridDim.x + b);
      const int i2 = __ldcg(p.am_idx + tid * gridDim.x + b);
      if (v2 > v || (v2 == v && i2 < i)) v = v2, i = i2;
    }
    if (p.argmax_out) p.argmax_out[tid] = i == 0x7fffffff ? 0 : i;
  }
  if (s_ticket == (int)gridDim.x - 1 && tid == 0) *p.counter = 0;
}

template <int KRM>
cudaError_t launch_f16_t(const GemvParams& p, cudaStream_t st, bool pdl) {
  const size_t smem = (size_t)KRM * p.k * 2 + 64 * 4 + (size_t)kF16Warps * KRM * 8;
  constexpr int kMaxDev = 64;  // the attribute is per device: raised once on each
  static std::atomic<size_t> configured[kMaxDev];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDev) return cudaErrorInvalidDevice;
  if (smem > configured[dev].load(std::memory_order_relaxed)) {
    cudaError_t e = cudaFuncSetAttribute(gemv_f16_kernel<KRM>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    configured[dev].store(smem, std::memory_order_relaxed);
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(device_sm_count());
  cfg.blockDim = dim3(kF16Threads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, gemv_f16_kernel<KRM>, p);
}

}  // namespace

cudaError_t launch_gemv_f16(const GemvParams& p, cudaStream_t st, bool pdl) {
  if (p.k % 256 || p.k > 8192 || p.kr < 1 || p.kr > kMaxRows) return cudaErrorInvalidValue;
  if (p.kr <= 1) return launch_f16_t<1>(p, st, pdl);
  if (p.kr <= 2) return launch_f16_t<2>(p, st, pdl);
  if (p.kr <= 4) return launch_f16_t<4>(p, st, pdl);
  return launch_f16_t<8>(p, st, pdl);
}

bool set_gemv_kernel_choice(int kind) {
  if (kind < 0 || kind > 4 || kind == 1) return false;
  g_kernel_choice.store(kind - 1);
  return true;
}

int device_sm_count() {
  // per device, looked up once with that device current
  constexpr int kMaxDev = 64;
  static std::atomic<int> counts[kMaxDev];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDev) return 1;
  int n = counts[dev].load(std::memory_order_relaxed);
  if (n == 0) {
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 1;
    counts[dev].store(n, std::memory_order_relaxed);
  }
  return n;
}

}  // namespace q4g
