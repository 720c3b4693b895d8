// Device fills of the seeded synthetic inputs (test and bench harness only).
// Every element is the pure function of (seed, stream, index) that
// datagen/q4g_datagen.h defines, so device fills equal the host/numpy fills.
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "q4g_datagen.h"

namespace {
__global__ void fill_normal_f32(float* out, long long n, unsigned long long key, float sigma, long long start) {
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n; i += (long long)gridDim.x * blockDim.x)
    out[i] = dg_normal(key, (uint64_t)(start + i), sigma);
}
__global__ void fill_normal_f16(__half* out, long long n, unsigned long long key, float sigma, long long start) {
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n; i += (long long)gridDim.x * blockDim.x)
    out[i] = __float2half_rn(dg_normal(key, (uint64_t)(start + i), sigma));
}
__global__ void fill_gain_f32(float* out, long long n, unsigned long long key) {
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n; i += (long long)gridDim.x * blockDim.x)
    out[i] = dg_gain(key, (uint64_t)i);
}
__global__ void fill_uniform_int(int* out, long long n, unsigned long long key, long long hi, long long start) {
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n; i += (long long)gridDim.x * blockDim.x)
    out[i] = (int)dg_uniform_int(key, (uint64_t)(start + i), (uint64_t)hi);
}
__global__ void fill_code8(int8_t* out, long long n, unsigned long long key, long long start) {
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n; i += (long long)gridDim.x * blockDim.x)
    out[i] = (int8_t)dg_code8(key, (uint64_t)(start + i));
}
__global__ void fill_const_f32(float* out, long long n, float v) {
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n; i += (long long)gridDim.x * blockDim.x)
    out[i] = v;
}
unsigned grid_for(long long n) {
  long long g = (n + 255) / 256;
  return (unsigned)(g > 65536 ? 65536 : (g < 1 ? 1 : g));
}
}  // namespace

extern "C" {
int dg_fill_normal_f32(float* out, long long n, unsigned long long seed, unsigned long long stream, float sigma,
                       long long start, cudaStream_t st) {
  fill_normal_f32<<<grid_for(n), 256, 0, st>>>(out, n, dg_key(seed, stream), sigma, start);
  return (int)cudaGetLastError();
}
int dg_fill_normal_f16(void* out, long long n, unsigned long long seed, unsigned long long stream, float sigma,
                       long long start, cudaStream_t st) {
  fill_normal_f16<<<grid_for(n), 256, 0, st>>>((__half*)out, n, dg_key(seed, stream), sigma, start);
  return (int)cudaGetLastError();
}
int dg_fill_gain_f32(float* out, long long n, unsigned long long seed, unsigned long long stream, cudaStream_t st) {
  fill_gain_f32<<<grid_for(n), 256, 0, st>>>(out, n, dg_key(seed, stream));
  return (int)cudaGetLastError();
}
int dg_fill_code8(void* out, long long n, unsigned long long seed, unsigned long long stream, long long start,
                  cudaStream_t st) {
  fill_code8<<<grid_for(n), 256, 0, st>>>((int8_t*)out, n, dg_key(seed, stream), start);
  return (int)cudaGetLastError();
}
int dg_fill_const_f32(float* out, long long n, float v, cudaStream_t st) {
  fill_const_f32<<<grid_for(n), 256, 0, st>>>(out, n, v);
  return (int)cudaGetLastError();
}
int dg_fill_uniform_int(int* out, long long n, unsigned long long seed, unsigned long long stream, long long hi,
                        long long start, cudaStream_t st) {
  fill_uniform_int<<<grid_for(n), 256, 0, st>>>(out, n, dg_key(seed, stream), hi, start);
  return (int)cudaGetLastError();
}
}
