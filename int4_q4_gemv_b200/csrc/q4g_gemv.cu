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

  // ---- prologue: activations into shared memory ----
  __half* xs_h = reinterpret_cast<__half*>(xs);
  for (int j = 0; j < KRM; ++j) {
    if (j >= p.kr) break;
    if (p.pro == PRO_X16) {
      const __half* xr = p.x + (size_t)j * p.x_stride;
      for (int c = tid; c < k; c += kThreads) put_x(xs_h, nb, j, c, xr[c]);
    } else {
      const float* rin = p.r_in + (size_t)j * k;
      const float* dl = p.delta ? p.delta + (size_t)j * k : nullptr;
      float inv_d = 0.f;
      if (dl) {
        float ss = 0.f;
        for (int c = tid; c < k; c += kThreads) ss = fmaf(dl[c], dl[c], ss);
        inv_d = rms_inv(block_sum(ss, misc), k, p.eps);
      }
      float ss2 = 0.f;
      for (int c = tid; c < k; c += kThreads) {
        float rn = rin[c];
        if (dl) rn = __fmul_rn(__fadd_rn(rn, __fmul_rn(__fmul_rn(dl[c], inv_d), p.w_delta[c])), p.scale);
        ss2 = fmaf(rn, rn, ss2);
        if (blockIdx.x == 0) {
          p.r_out[(size_t)j * k + c] = rn;
          if (p.dump) p.dump[(size_t)j * p.dump_stride + c] = rn;
        }
      }
      const float inv_r = rms_inv(block_sum(ss2, misc + 32), k, p.eps);
      for (int c = tid; c < k; c += kThreads) {
        float rn = rin[c];
        if (dl) rn = __fmul_rn(__fadd_rn(rn, __fmul_rn(__fmul_rn(dl[c], inv_d), p.w_delta[c])), p.scale);
        put_x(xs_h, nb, j, c, __float2half_rn(__fmul_rn(__fmul_rn(rn, inv_r), p.w_x[c])));
      }
    }
  }
  __syncthreads();
  // per-block offset constant 72 * sum(x): removes +64 of the unpacked codes and the -8
  for (int t = tid; t < p.kr * nb; t += kThreads) {
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

cudaError_t launch_gemv(const GemvParams& p, cudaStream_t st, bool pdl) {
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
