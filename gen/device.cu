// Seeded counter-based generator on the device: the same definition as
// gen/host.py (SplitMix64 counter form, Irwin-Hall(4) normal approximation,
// separate correctly rounded float32 scale and offset, RNE bfloat16).  It
// holds none of the attention method's arithmetic.
#include <cuda_runtime.h>
#include <stdint.h>

namespace {

__device__ __forceinline__ uint64_t mix64(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

__device__ __forceinline__ float normal_at(uint64_t key, uint64_t i, float unit, int has_scale,
                                           float scale, int has_offset, float offset) {
  const uint64_t u = mix64(key + (i + 1ull) * 0x9E3779B97F4A7C15ull);
  const long long s = (long long)(u & 0xFFFFull) + (long long)((u >> 16) & 0xFFFFull) +
                      (long long)((u >> 32) & 0xFFFFull) + (long long)(u >> 48);
  // unit = float32(sqrt(3) / 65536), passed in by the host definition
  float x = __fmul_rn((float)(s - 131070ll), unit);
  if (has_scale) x = __fmul_rn(x, scale);
  if (has_offset) x = __fadd_rn(offset, x);
  return x;
}

__device__ __forceinline__ uint16_t to_bf16(float f) {
  unsigned int b = __float_as_uint(f);
  b += 0x7FFFu + ((b >> 16) & 1u);
  return (uint16_t)(b >> 16);
}

__global__ void fill_bf16(uint16_t* out, uint64_t n, uint64_t key, uint64_t start, float unit, int hs,
                          float sc, int ho, float off) {
  for (uint64_t i = blockIdx.x * (uint64_t)blockDim.x + threadIdx.x; i < n;
       i += (uint64_t)gridDim.x * blockDim.x)
    out[i] = to_bf16(normal_at(key, start + i, unit, hs, sc, ho, off));
}

__global__ void fill_f32(float* out, uint64_t n, uint64_t key, uint64_t start, float unit, int hs,
                         float sc, int ho, float off) {
  for (uint64_t i = blockIdx.x * (uint64_t)blockDim.x + threadIdx.x; i < n;
       i += (uint64_t)gridDim.x * blockDim.x)
    out[i] = normal_at(key, start + i, unit, hs, sc, ho, off);
}

}  // namespace

extern "C" int ds4gen_fill(void* out, int is_bf16, uint64_t n, uint64_t key, uint64_t start,
                           float unit, int has_scale, float scale, int has_offset, float offset,
                           void* stream) {
  if (n == 0) return 0;
  if (!out) return 1;
  const int threads = 256;
  uint64_t blocks = (n + threads - 1) / threads;
  if (blocks > 148ull * 32) blocks = 148ull * 32;
  if (is_bf16)
    fill_bf16<<<(unsigned)blocks, threads, 0, (cudaStream_t)stream>>>(
        (uint16_t*)out, n, key, start, unit, has_scale, scale, has_offset, offset);
  else
    fill_f32<<<(unsigned)blocks, threads, 0, (cudaStream_t)stream>>>(
        (float*)out, n, key, start, unit, has_scale, scale, has_offset, offset);
  return cudaGetLastError() == cudaSuccess ? 0 : 3;
}
