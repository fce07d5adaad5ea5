// Conversion of bf16 cache rows to the block-scaled storage of ds4a_mx.cuh:
// mixed FP8 / BF16 K=V rows and FP4 indexer keys.  One warp per row; lane
// l quantises the 32-value blocks l, l + 32, ... of the row.
#include "ds4a_mx.cuh"

namespace ds4a {
namespace {

// 32 bf16 values at p (64 bytes, 16-byte aligned) -> floats
__device__ __forceinline__ void load32(const uint16_t* p, float (&v)[32]) {
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const uint4 w = reinterpret_cast<const uint4*>(p)[q];
    const unsigned int u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float2 f = bf2x2_to_f2(u[k]);
      v[8 * q + 2 * k] = f.x;
      v[8 * q + 2 * k + 1] = f.y;
    }
  }
}

__global__ void __launch_bounds__(256) quant_kv_fp8_kernel(int n_rows, int D, int R, const uint16_t* __restrict__ in,
                                                           int64_t in_stride, uint8_t* __restrict__ out,
                                                           int64_t out_stride) {
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5, lane = threadIdx.x & 31;
  if (warp >= n_rows) return;
  const uint16_t* src = in + (int64_t)warp * in_stride;
  uint8_t* dst = out + (int64_t)warp * out_stride;
  const int n = D - R, nb = n / kMxBlock;
  for (int b = lane; b < nb; b += 32) {
    float v[32];
    load32(src + b * kMxBlock, v);
    float amax = 0.f;
#pragma unroll
    for (int i = 0; i < 32; ++i) amax = fmaxf(amax, fabsf(v[i]));
    const int code = mx_scale_code<false>(amax);
    const float inv = mx_inv_scale(code);
    uint32_t w[8];
#pragma unroll
    for (int i = 0; i < 8; ++i)
      w[i] = (uint32_t)to_e4m3x2(v[4 * i] * inv, v[4 * i + 1] * inv) |
             ((uint32_t)to_e4m3x2(v[4 * i + 2] * inv, v[4 * i + 3] * inv) << 16);
    reinterpret_cast<uint4*>(dst + b * kMxBlock)[0] = make_uint4(w[0], w[1], w[2], w[3]);
    reinterpret_cast<uint4*>(dst + b * kMxBlock)[1] = make_uint4(w[4], w[5], w[6], w[7]);
    dst[n + 2 * R + b] = (uint8_t)code;
  }
  // the RoPE dims as stored (16-byte pieces), then the zero padding
  for (int q = lane; q < 2 * R / 16; q += 32)
    reinterpret_cast<uint4*>(dst + n)[q] = reinterpret_cast<const uint4*>(src + n)[q];
  for (int k = n + 2 * R + nb + lane; k < kv_fp8_row_bytes(D, R); k += 32) dst[k] = 0;
}

__global__ void __launch_bounds__(256) quant_idx_fp4_kernel(int n_rows, int D, const uint16_t* __restrict__ in,
                                                            int64_t in_stride, uint8_t* __restrict__ codes,
                                                            uint8_t* __restrict__ scales) {
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5, lane = threadIdx.x & 31;
  if (warp >= n_rows) return;
  const uint16_t* src = in + (int64_t)warp * in_stride;
  const int nb = D / kMxBlock;
  for (int b = lane; b < nb; b += 32) {
    float v[32];
    load32(src + b * kMxBlock, v);
    float amax = 0.f;
#pragma unroll
    for (int i = 0; i < 32; ++i) amax = fmaxf(amax, fabsf(v[i]));
    const int code = mx_scale_code<true>(amax);
    const float inv = mx_inv_scale(code);
    uint32_t w[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      uint32_t x = 0;
#pragma unroll
      for (int k = 0; k < 4; ++k) x |= to_e2m1x2(v[8 * i + 2 * k] * inv, v[8 * i + 2 * k + 1] * inv) << (8 * k);
      w[i] = x;
    }
    *reinterpret_cast<uint4*>(codes + (int64_t)warp * (D / 2) + b * 16) = make_uint4(w[0], w[1], w[2], w[3]);
    scales[(int64_t)warp * nb + b] = (uint8_t)code;
  }
}

}  // namespace

cudaError_t launch_quant_kv_fp8(int n_rows, int D, int R, const uint16_t* in, int64_t in_stride, uint8_t* out,
                                int64_t out_stride, cudaStream_t s) {
  if (n_rows <= 0) return cudaSuccess;
  const int blocks = (n_rows + 7) / 8;
  TraceScope tr("quant_kv_fp8", s);
  quant_kv_fp8_kernel<<<blocks, 256, 0, s>>>(n_rows, D, R, in, in_stride, out, out_stride);
  return cudaGetLastError();
}

cudaError_t launch_quant_idx_fp4(int n_rows, int D, const uint16_t* in, int64_t in_stride, uint8_t* codes,
                                 uint8_t* scales, cudaStream_t s) {
  if (n_rows <= 0) return cudaSuccess;
  const int blocks = (n_rows + 7) / 8;
  TraceScope tr("quant_idx_fp4", s);
  quant_idx_fp4_kernel<<<blocks, 256, 0, s>>>(n_rows, D, in, in_stride, codes, scales);
  return cudaGetLastError();
}

}  // namespace ds4a
