// Flash-decode over the sliding-window ring without any device allocation.
//
// Some callers cannot allocate device memory when they call into the library:
// for example a host program whose device memory is owned by a framework's
// caching allocator that this library cannot reach, or a process that reserves
// its whole memory budget at start-up and treats any later cudaMalloc as a
// failure. For them q4g_flash_decode_ring_noalloc keeps the split-KV scratch
// (completion counters and per-chunk partials) in the fixed-size device array
// below instead of a caller workspace. Every GPU that loads the library holds
// this array until the process exits.
#include <mutex>

#include "../../include/q4g.h"
#include "q4g_common.cuh"
#include "q4g_internal.h"

namespace {

constexpr size_t kScratchBytes = Q4G_NOALLOC_SCRATCH_BYTES;

// Shared by every call on a device; each call clears the counters it needs.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_scratch_ptr[kMaxDevices];

// Device address of the scratch array on the current device. The symbol name is
// only a host-side handle; the address is looked up once per device, with that
// device current, and cached.
cudaError_t scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return cudaSuccess;
}

bool aligned16(const void* p) { return ((uintptr_t)p & 15) == 0; }

q4g_status bad(q4g_status s, const char* msg) {
  q4g::set_last_error(msg);
  return s;
}

}  // namespace

extern "C" q4g_status q4g_flash_decode_ring_noalloc(const uint16_t* q, int32_t n_q, int32_t n_kv,
                                                    int32_t head_dim, const uint16_t* k_ring,
                                                    const uint16_t* v_ring, int64_t ring, int64_t window,
                                                    int64_t pos, uint16_t* out, q4g_stream_t stream) {
  if (!q || !k_ring || !v_ring || !out) return bad(Q4G_EINVAL, "NULL pointer");
  if (head_dim != 256 && head_dim != 512) return bad(Q4G_EINVAL, "head_dim must be 256 or 512");
  if (n_q < 1 || n_kv < 1 || n_q % n_kv) return bad(Q4G_EINVAL, "n_q must be a positive multiple of n_kv");
  if (ring < 1 || window < 1 || window > ring) return bad(Q4G_EINVAL, "need 1 <= window <= ring");
  if (ring > ((int64_t)1 << 30)) return bad(Q4G_ERANGE, "ring > 2^30");
  if (pos < 0) return bad(Q4G_ERANGE, "pos < 0");
  if (!aligned16(q) || !aligned16(k_ring) || !aligned16(v_ring) || !aligned16(out))
    return bad(Q4G_EINVAL, "misaligned pointer");

  q4g::AttnParams p{};
  p.q16 = reinterpret_cast<const __half*>(q);
  p.k_cache = reinterpret_cast<__half*>(const_cast<uint16_t*>(k_ring));
  p.v_cache = reinterpret_cast<__half*>(const_cast<uint16_t*>(v_ring));
  p.cache_rows = ring;
  p.ring = 1;
  p.window = window;
  p.pos0 = pos;
  p.kr = 1;
  p.n_q = n_q;
  p.n_kv = n_kv;
  p.hd = head_dim;
  const q4g::FlashPlan plan = q4g::flash_plan(n_q, n_kv, head_dim, true, window);
  if (n_kv * plan.m_groups * (int)sizeof(int32_t) > (int)q4g::kFlashCounterBytes)
    return bad(Q4G_EINVAL, "too many KV heads for the fixed scratch");
  if (plan.bytes > kScratchBytes)
    return bad(Q4G_ERANGE, "split-KV scratch for these sizes exceeds Q4G_NOALLOC_SCRATCH_BYTES "
                           "(n_q * chunks * head_dim * 4 bytes plus (m, l) and counters)");

  void* base = nullptr;
  cudaError_t e = scratch_address(&base);
  if (e != cudaSuccess) return bad(Q4G_ECUDA, cudaGetErrorString(e));
  q4g::flash_bind(p, plan, base);
  p.combine_in_kernel = 1;
  p.out = reinterpret_cast<__half*>(out);

  cudaStream_t st = (cudaStream_t)stream;
  // the completion counters must start at zero; the partials are overwritten
  if ((e = cudaMemsetAsync(p.counters, 0, q4g::kFlashCounterBytes, st)) != cudaSuccess)
    return bad(Q4G_ECUDA, cudaGetErrorString(e));
  if ((e = q4g::launch_attention(p, st, false)) != cudaSuccess) return bad(Q4G_ECUDA, cudaGetErrorString(e));
  return Q4G_OK;
}
