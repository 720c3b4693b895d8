// q4_0 packing/unpacking and the per-step initialisation kernel.
#include "q4g_common.cuh"
#include "q4g_internal.h"

namespace q4g {

namespace {

// One warp per 32-column block ("Gemma 4 12B" intro: per-block-32 absmax
// symmetric int4; "gemma-4-E4B-CoreAI" Provenance: codes on the [-8, 7] grid).
//   m = element of largest |x| (lowest column on ties, sign kept; +0 if all are 0)
//   d = fp16_rne(m / -8)          (IEEE fp32 division)
//   c = clamp(roundf(x / d), -8, 7) + 8, or 8 for every column when d == 0
__global__ void pack_kernel(const float* __restrict__ w, int64_t nblocks, int64_t k,
                            uint8_t* __restrict__ qs, uint16_t* __restrict__ sc, int32_t* bad) {
  const int lane = threadIdx.x & 31;
  const int64_t warp_global = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
  const int64_t nb = k >> 5;
  for (int64_t b = warp_global; b < nblocks; b += nwarps) {
    const int64_t row = b / nb, t = b - row * nb;
    const float x = w[row * k + t * 32 + lane];
    if (!isfinite(x)) atomicOr(bad, 1);
    float ax = fabsf(x);
    int idx = lane;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float a2 = __shfl_xor_sync(0xffffffffu, ax, o);
      const int i2 = __shfl_xor_sync(0xffffffffu, idx, o);
      if (a2 > ax || (a2 == ax && i2 < idx)) ax = a2, idx = i2;
    }
    // an all-zero block keeps m = +0 (no element exceeds 0), so d = fp16(-0)
    const float m = ax > 0.0f ? __shfl_sync(0xffffffffu, x, idx) : 0.0f;
    const __half dh = __float2half_rn(__fdiv_rn(m, -8.0f));
    const float d = __half2float(dh);
    int c = 8;
    if (d != 0.0f) {
      float r = roundf(__fdiv_rn(x, d));
      r = fminf(fmaxf(r, -8.0f), 7.0f);
      c = (int)r + 8;
    }
    const int c_hi = __shfl_down_sync(0xffffffffu, c, 16);
    if (lane < 16) qs[row * (k >> 1) + t * 16 + lane] = (uint8_t)(c | (c_hi << 4));
    if (lane == 0) sc[row * nb + t] = __half_as_ushort(dh);
  }
}

__global__ void unpack_kernel(const uint8_t* __restrict__ qs, const uint16_t* __restrict__ sc,
                              int64_t n, int64_t k, float* __restrict__ w) {
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t row = i / k, col = i - row * k;
    const uint8_t byte = qs[row * (k >> 1) + (col >> 5) * 16 + (col & 15)];
    const int c = (col & 31) < 16 ? (byte & 15) : (byte >> 4);
    const float d = __half2float(__ushort_as_half(sc[row * (k >> 5) + (col >> 5)]));
    w[i] = (float)(c - 8) * d;
  }
}

// Per-step state: the layer-0 input rows, RoPE cos/sin for this step's
// positions (angles in fp64: position * theta^(-2i/hd)), the position word
// read by the captured kernels, and zeroed completion counters.
__global__ void step_init_kernel(const StepParams p) {
  const int nb_h = (p.hidden_size + blockDim.x - 1) / blockDim.x;
  const int blk = blockIdx.x;
  if (blk < p.kr * nb_h) {
    const int j = blk / nb_h;
    const int c = (blk - j * nb_h) * blockDim.x + threadIdx.x;
    if (c >= p.hidden_size) return;
    float v;
    if (p.hidden) {
      v = p.hidden[(size_t)j * p.hidden_size + c];
    } else {
      int tok = p.ids_dev ? p.ids_dev[j] : p.ids_host[j];
      tok = tok < 0 ? 0 : (tok >= p.vocab ? p.vocab - 1 : tok);
      const size_t row = (size_t)tok;
      if (p.emb_f16) {  // fp16 tied table
        v = __fmul_rn(__half2float(__ushort_as_half(p.emb_f16[row * p.hidden_size + c])), p.embed_scale);
      } else {
        const uint8_t byte = p.emb_qs[row * (p.hidden_size >> 1) + (c >> 5) * 16 + (c & 15)];
        const int code = (c & 31) < 16 ? (byte & 15) : (byte >> 4);
        const float d = __half2float(__ushort_as_half(p.emb_sc[row * (p.hidden_size >> 5) + (c >> 5)]));
        v = __fmul_rn((float)(code - 8) * d, p.embed_scale);
      }
    }
    p.r_out[(size_t)j * p.hidden_size + c] = v;
    if (p.dump) p.dump[(size_t)j * p.dump_stride + c] = v;
    return;
  }
  // last block: tables and state
  for (int t = threadIdx.x; t < p.kr * (p.pairs_sl + p.pairs_gl); t += blockDim.x) {
    const int j = t / (p.pairs_sl + p.pairs_gl);
    const int i = t - j * (p.pairs_sl + p.pairs_gl);
    const double pos = (double)(p.pos0 + j);
    double s, c;
    if (i < p.pairs_sl) {
      sincos(pos * p.inv_freq_sl[i], &s, &c);
      p.rope_sl[(size_t)j * p.pairs_sl + i] = make_float2((float)c, (float)s);
    } else {
      const int ig = i - p.pairs_sl;
      sincos(pos * p.inv_freq_gl[ig], &s, &c);
      p.rope_gl[(size_t)j * p.pairs_gl + ig] = make_float2((float)c, (float)s);
    }
  }
  for (int t = threadIdx.x; t < p.n_counters; t += blockDim.x) p.counters[t] = 0;
  if (threadIdx.x == 0) *p.pos_dev = p.pos0;
}

}  // namespace

cudaError_t launch_pack(const float* w, int64_t rows, int64_t k, uint8_t* qs, uint16_t* sc,
                        int32_t* bad_flag, cudaStream_t st) {
  const int64_t nblocks = rows * (k >> 5);
  if (nblocks == 0) return cudaSuccess;
  int64_t grid = (nblocks + 7) / 8;
  if (grid > 148 * 64) grid = 148 * 64;
  pack_kernel<<<(unsigned)grid, 256, 0, st>>>(w, nblocks, k, qs, sc, bad_flag);
  return cudaGetLastError();
}

cudaError_t launch_unpack(const uint8_t* qs, const uint16_t* sc, int64_t rows, int64_t k, float* w,
                          cudaStream_t st) {
  const int64_t n = rows * k;
  if (n == 0) return cudaSuccess;
  int64_t grid = (n + 255) / 256;
  if (grid > 148 * 64) grid = 148 * 64;
  unpack_kernel<<<(unsigned)grid, 256, 0, st>>>(qs, sc, n, k, w);
  return cudaGetLastError();
}

cudaError_t launch_step_init(const StepParams& p, cudaStream_t st) {
  const int nb_h = (p.hidden_size + 255) / 256;
  step_init_kernel<<<p.kr * nb_h + 1, 256, 0, st>>>(p);
  return cudaGetLastError();
}

}  // namespace q4g
