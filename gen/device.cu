// Seeded counter-based generator on the device: the same definition as
// gen/host.py (SplitMix64 counter form; N(0,1) by a table inverse of the
// normal CDF whose (node, slope) pairs the host computes and passes in;
// separate correctly rounded float32 scale and offset; RNE bfloat16).  It
// holds none of the attention method's arithmetic.
#include <cuda_runtime.h>
#include <stdint.h>

namespace {

__device__ __forceinline__ uint64_t mix64(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

// tab: float2 [63 octaves][256 segments] = (node, slope), as gen/host.py
// builds it
__device__ __forceinline__ float normal_at(uint64_t key, uint64_t i, const float2* __restrict__ tab,
                                           int has_scale, float scale, int has_offset, float offset) {
  const uint64_t u = mix64(key + (i + 1ull) * 0x9E3779B97F4A7C15ull);
  uint64_t v = u & 0x7FFFFFFFFFFFFFFFull;
  if (v == 0) v = 1;
  const int e = 62 - (63 - __clzll((long long)v));  // octave: 62 - floor(log2 v)
  const uint64_t w = v << e;                         // leading one at bit 62
  const int seg = (int)((w >> 54) & 0xFFull);
  const float f = __fmul_rn((float)(unsigned int)((w >> 31) & 0x7FFFFFull), 1.1920928955078125e-7f);  // 2^-23
  const float2 td = __ldg(tab + e * 256 + seg);
  float x = __fadd_rn(td.x, __fmul_rn(f, td.y));
  if (u >> 63) x = -x;
  if (has_scale) x = __fmul_rn(x, scale);
  if (has_offset) x = __fadd_rn(offset, x);
  return x;
}

__device__ __forceinline__ uint16_t to_bf16(float f) {
  unsigned int b = __float_as_uint(f);
  b += 0x7FFFu + ((b >> 16) & 1u);
  return (uint16_t)(b >> 16);
}

__global__ void fill_bf16(uint16_t* out, uint64_t n, uint64_t key, uint64_t start, const float2* tab, int hs,
                          float sc, int ho, float off) {
  for (uint64_t i = blockIdx.x * (uint64_t)blockDim.x + threadIdx.x; i < n;
       i += (uint64_t)gridDim.x * blockDim.x)
    out[i] = to_bf16(normal_at(key, start + i, tab, hs, sc, ho, off));
}

__global__ void fill_f32(float* out, uint64_t n, uint64_t key, uint64_t start, const float2* tab, int hs,
                         float sc, int ho, float off) {
  for (uint64_t i = blockIdx.x * (uint64_t)blockDim.x + threadIdx.x; i < n;
       i += (uint64_t)gridDim.x * blockDim.x)
    out[i] = normal_at(key, start + i, tab, hs, sc, ho, off);
}

}  // namespace

// tab: device float [63 * 256 * 2], the host's normal table
extern "C" int ds4gen_fill(void* out, int is_bf16, uint64_t n, uint64_t key, uint64_t start,
                           const void* tab, int has_scale, float scale, int has_offset, float offset,
                           void* stream) {
  if (n == 0) return 0;
  if (!out || !tab) return 1;
  const int threads = 256;
  uint64_t blocks = (n + threads - 1) / threads;
  if (blocks > 148ull * 32) blocks = 148ull * 32;
  const float2* t = static_cast<const float2*>(tab);
  if (is_bf16)
    fill_bf16<<<(unsigned)blocks, threads, 0, (cudaStream_t)stream>>>(
        (uint16_t*)out, n, key, start, t, has_scale, scale, has_offset, offset);
  else
    fill_f32<<<(unsigned)blocks, threads, 0, (cudaStream_t)stream>>>(
        (float*)out, n, key, start, t, has_scale, scale, has_offset, offset);
  return cudaGetLastError() == cudaSuccess ? 0 : 3;
}
