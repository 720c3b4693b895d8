// Shared device helpers of libq4g (sm_100a).
#pragma once

#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#define Q4G_DEV __device__ __forceinline__

namespace q4g {

constexpr int kMaxRows = 8;       // verify rows per call
constexpr int kThreads = 256;     // block size of the GEMV and attention kernels
constexpr int kUnitRows = 16;     // GEMV rows per unit of work
constexpr int kSpinLimit = 1 << 22;

// ---------------------------------------------------------------------------
// Programmatic dependent launch. Without the launch attribute both are no-ops.
// ---------------------------------------------------------------------------
Q4G_DEV void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
Q4G_DEV void pdl_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// ---------------------------------------------------------------------------
// Loads. Weights are read once per step: stream them past L1.
// ---------------------------------------------------------------------------
Q4G_DEV uint4 ld_stream_u4(const void* p) {
  uint4 r;
  asm("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
      : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
      : "l"(p));
  return r;
}

Q4G_DEV uint16_t ld_stream_u16(const void* p) {
  uint16_t r;
  asm("ld.global.nc.L1::no_allocate.u16 %0, [%1];" : "=h"(r) : "l"(p));
  return r;
}

Q4G_DEV uint4 lds_u4(const void* p) {
  uint4 r;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "r"((uint32_t)__cvta_generic_to_shared(p)));
  return r;
}

// ---------------------------------------------------------------------------
// q4_0 nibble unpacking. A 32-bit word w of a block's 16 code bytes holds, per
// 16-bit half, the codes of two columns in each nibble. Moving one nibble of
// each half to bits 4..7 and OR-ing the fp16 pattern 0x5400 (64.0, whose
// lowest fraction bit weighs 1/16) yields the exact half2 value (64 + c).
// lop3 immediate 0xEA = (a & b) | c.
// ---------------------------------------------------------------------------
Q4G_DEV uint32_t nib_to_h2(uint32_t v) {
  uint32_t r;
  asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(r) : "r"(v), "n"(0x00F000F0), "n"(0x54005400));
  return r;
}

// acc + w.lo * x.lo + w.hi * x.hi with fp16 products accumulated in fp32
// (mixed-precision fma, products exact).
Q4G_DEV float fma2_h_f32(uint32_t w2, uint32_t x2, float acc) {
  float r;
  asm("{\n\t.reg .b16 wl, wh, xl, xh;\n\t"
      "mov.b32 {wl, wh}, %1;\n\t"
      "mov.b32 {xl, xh}, %2;\n\t"
      "fma.rn.f32.f16 %0, wl, xl, %3;\n\t"
      "fma.rn.f32.f16 %0, wh, xh, %0;\n\t}"
      : "=f"(r)
      : "r"(w2), "r"(x2), "f"(acc));
  return r;
}

// Sum over the 32 columns of one block of (64 + c_i) * x_i, split into two
// accumulators. xq[k] holds the block's x in the order the unpacking of word k
// produces: {x[4k], x[4k+2]}, {x[4k+16], x[4k+18]}, {x[4k+1], x[4k+3]},
// {x[4k+17], x[4k+19]}.
Q4G_DEV void block_dot(const uint4 q, const uint4 (&xq)[4], float& a0, float& a1) {
  const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    a0 = fma2_h_f32(nib_to_h2(w[k] << 4), xq[k].x, a0);
    a1 = fma2_h_f32(nib_to_h2(w[k]), xq[k].y, a1);
    a0 = fma2_h_f32(nib_to_h2(w[k] >> 4), xq[k].z, a0);
    a1 = fma2_h_f32(nib_to_h2(w[k] >> 8), xq[k].w, a1);
  }
}

// 4-way byte dot products with 32-bit accumulation (unsigned x unsigned and
// unsigned x signed).
Q4G_DEV int dp4a_uu(uint32_t a, uint32_t b, int c) {
  int r;
  asm("dp4a.u32.u32 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(c));
  return r;
}
Q4G_DEV int dp4a_us(uint32_t a, uint32_t b, int c) {
  int r;
  asm("dp4a.u32.s32 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(c));
  return r;
}

// Column order of the x layout above: slot s (0..31) of a block holds column
// kXPerm[s]; quarter k = slots 8k..8k+7.
__host__ __device__ constexpr int xperm(int s) {
  // within a quarter: 0:4k 1:4k+2 2:4k+16 3:4k+18 4:4k+1 5:4k+3 6:4k+17 7:4k+19
  return 4 * (s >> 3) + ((s & 7) == 0 ? 0 : (s & 7) == 1 ? 2 : (s & 7) == 2 ? 16 : (s & 7) == 3 ? 18
                       : (s & 7) == 4 ? 1 : (s & 7) == 5 ? 3 : (s & 7) == 6 ? 17 : 19);
}

// ---------------------------------------------------------------------------
// mbarrier and 1-D bulk copies (TMA engine), sm_90+ PTX.
// ---------------------------------------------------------------------------
Q4G_DEV uint32_t smem_u32(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }

Q4G_DEV void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
Q4G_DEV void fence_mbar_init() { asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory"); }
Q4G_DEV void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}
Q4G_DEV void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
// One poll of `phase` of `bar`. With the suspend-time hint the thread sleeps in
// the instruction until the phase completes or ~0.1 ms pass, instead of spinning.
Q4G_DEV bool mbar_try_wait(uint64_t* bar, uint32_t phase) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(phase), "r"(100000u)
      : "memory");
  return ok != 0;
}
// Copy `bytes` (multiple of 16, 16-byte aligned addresses) global -> shared;
// completion is counted on `bar`.
Q4G_DEV void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}
// As bulk_g2s with an L2 eviction-priority policy (createpolicy) for the source.
Q4G_DEV void bulk_g2s_hint(void* dst, const void* src, uint32_t bytes, uint64_t* bar, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], "
      "%4;" ::"r"(smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar)), "l"(policy)
      : "memory");
}
// Weights are read once per step: evict them from L2 first.
Q4G_DEV uint64_t policy_evict_first() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}
Q4G_DEV uint64_t global_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
// Wait for `phase` of `bar` for at most `limit_ns`; false if the limit ran out.
Q4G_DEV bool mbar_wait_bounded(uint64_t* bar, uint32_t phase, uint64_t limit_ns) {
  if (mbar_try_wait(bar, phase)) return true;
  const uint64_t t0 = global_ns();
  for (int it = 0; it < kSpinLimit; ++it) {
    if (mbar_try_wait(bar, phase)) return true;
    if (global_ns() - t0 > limit_ns) break;
  }
  return false;
}

// a mod m in [0, m) for 32-bit a, m > 0; the common case (a >= -m) takes one add
Q4G_DEV int wrap(int a, int m) {
  if (a >= 0) return a < m ? a : a % m;
  a += m;
  return a >= 0 ? a : (a % m + m) % m;
}

// Thread-block clusters: rank, cluster-wide barrier (release/acquire) and loads
// from a peer CTA's shared memory (distributed shared memory).
Q4G_DEV uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
Q4G_DEV void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
Q4G_DEV uint32_t peer_addr(const void* p, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_u32(p)), "r"(rank));
  return r;
}
Q4G_DEV float ld_peer_f32(uint32_t addr) {
  float v;
  asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(addr) : "memory");
  return v;
}
// ---------------------------------------------------------------------------
// Reductions.
// ---------------------------------------------------------------------------
Q4G_DEV float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

Q4G_DEV float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// int8 KV row ("Gemma-4-12B-CoreAI", per-tier cost section: int8 K/V) from an fp16
// row in shared memory, by one warp: scale = amax / 127 and code = clamp(rint(x /
// scale), -127, 127), both IEEE fp32 divisions (round to nearest even); an
// all-zero row has scale 0 and codes 0.
template <int HD>
Q4G_DEV void kv_quantize_row_warp(const __half* x, int8_t* codes, float* scale, int lane) {
  constexpr int E = HD / 32;
  float v[E];
  float amax = 0.f;
#pragma unroll
  for (int e = 0; e < E; ++e) {
    v[e] = __half2float(x[lane * E + e]);
    amax = fmaxf(amax, fabsf(v[e]));
  }
  amax = warp_max(amax);
  const float s = __fdiv_rn(amax, 127.0f);
#pragma unroll
  for (int e = 0; e < E; ++e) {
    int c = 0;
    if (s != 0.f) c = min(max(__float2int_rn(__fdiv_rn(v[e], s)), -127), 127);
    codes[lane * E + e] = (int8_t)c;
  }
  if (lane == 0) *scale = s;
}

// Block-wide sum for blockDim.x == NT; `red` holds >= 32 floats. All threads
// receive the result. Summation order is fixed.
template <int NT = kThreads>
Q4G_DEV float block_sum(float v, float* red) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  v = warp_sum(v);
  __syncthreads();
  if (lane == 0) red[warp] = v;
  __syncthreads();
  float t = 0.f;
#pragma unroll
  for (int i = 0; i < NT / 32; ++i) t += red[i];
  return t;
}

// IEEE division and square root (correctly rounded), so results do not depend
// on compiler flags.
Q4G_DEV float rms_inv(float sumsq, int n, float eps) {
  return __fdiv_rn(1.0f, __fsqrt_rn(__fadd_rn(__fdiv_rn(sumsq, (float)n), eps)));
}

Q4G_DEV float gelu_tanh(float g) {
  const float k0 = 0.7978845608028654f;  // sqrt(2/pi)
  float inner = k0 * (g + 0.044715f * g * g * g);
  return 0.5f * g * (1.0f + tanhf(inner));
}

}  // namespace q4g
