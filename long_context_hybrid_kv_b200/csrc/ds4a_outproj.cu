// Grouped low-rank output projection of the attention layer ("DeepSeek-v4
// Beyond Basics" 3.3, after eq. 26: the concatenated head outputs are split
// into g groups, each projected to an intermediate of rank r, and the g
// intermediates together are projected to the hidden size; "DeepSeek V4
// Inside", layer-0 section: grouped W_O, Flash 64 heads in 8 groups;
// "DeepSeek-V4" Transformers documentation: grouped o_a projection followed
// by o_b).
//
//   mid[t][j*r + i] = sum_c W_a[j][i][c] * o[t][j*K1 + c]   (K1 = (H/g) * D)
//   y[t][n]         = sum_c W_b[n][c]    * mid[t][c]        (c < g * r)
//
// Both are "A row-major, B = weight [out][in]" products with K contiguous
// on both sides, so one tensor-core GEMM kernel serves both: tile 128 rows
// x 256 outputs, K in steps of 64 (128-byte rows, 128-byte swizzle), four
// TMA stages, tcgen05.mma M=128 N=256 K=16 into one of two TMEM
// accumulators (2 x 256 columns), so the epilogue of one tile overlaps the
// MMAs of the next.  The first product is "grouped": the A columns of an
// output tile start at its group's slice of o.
//
// Thread block (192 threads, one per SM, persistent over work units):
//   warp 0     lane 0: TMA producer (A and B tiles of every k step)
//   warp 1     TMEM allocation; lane 0 issues the MMAs
//   warps 2-5  epilogue: warp w reads TMEM lane quarter w % 4 (32 rows of
//              the tile), converts to bf16 and stores, or with split K
//              stores its split's float partial sums, which a second kernel
//              adds in split order (deterministic) and rounds.
// Work units: (row tile, output tile, K split), rastered in bands of eight
// row tiles so the A and B tiles that concurrent blocks read stay in L2.
#include <cuda.h>
#include <cudaTypedefs.h>

#include "ds4a_tc.cuh"

namespace ds4a {
namespace {

using namespace tc;

constexpr int kBM = 128, kBN = 256, kBK = 64;
constexpr int kStages = 4;
constexpr int kThreads = 192;
constexpr uint32_t kStageA = kBM * kBK * 2;  // 16 KiB
constexpr uint32_t kStageB = kBN * kBK * 2;  // 32 KiB
constexpr uint32_t kStageBytes = kStageA + kStageB;
constexpr uint32_t kOffBar = kStages * kStageBytes;
constexpr uint32_t kOffMisc = kOffBar + 256;
constexpr uint32_t kSmemBytes = kOffMisc + 64 + 1024;
constexpr int kBand = 8;  // row tiles per raster band

enum Bar { kFull = 0, kEmpty = kFull + kStages, kAccFull0 = kEmpty + kStages, kAccFull1, kAccEmpty0,
           kAccEmpty1, kDrain, kNumBars };

struct GemmParams {
  int M, N, k_steps;      // rows, outputs, K / 64 of one product
  int n_per_group;        // outputs per group (N for an ungrouped product)
  int a_group_k;          // A column offset per group (K of a group's slice; 0 ungrouped)
  int m_tiles, n_tiles, ksplit, steps_per_split, n_units;
  uint16_t* out;          // bf16 [M][ldo] (ksplit == 1)
  int64_t ldo;
  float* acc;             // float [ksplit][M][N] partial sums (ksplit > 1)
  unsigned int* err;
};

struct Unit {
  int m0, n0, k0, k1, a_koff;
};

__device__ __forceinline__ Unit make_unit(const GemmParams& p, int u) {
  Unit w;
  const int ks = u % p.ksplit;
  const int v = u / p.ksplit;
  const int band = v / (kBand * p.n_tiles);
  const int bm = min(kBand, p.m_tiles - band * kBand);
  const int in_band = v - band * kBand * p.n_tiles;
  const int nt = in_band / bm;
  const int mt = band * kBand + in_band % bm;
  w.m0 = mt * kBM;
  w.n0 = nt * kBN;
  w.k0 = ks * p.steps_per_split;
  w.k1 = min(p.k_steps, w.k0 + p.steps_per_split);
  w.a_koff = (w.n0 / p.n_per_group) * p.a_group_k;
  return w;
}

__global__ void __launch_bounds__(kThreads, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap amap, const __grid_constant__ CUtensorMap bmap,
                   const GemmParams p) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar0 = sbase + kOffBar;
  auto bar = [&](int i) { return bar0 + 8u * (uint32_t)i; };
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kOffMisc);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kOffMisc + 8);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  unsigned int* err = p.err;

  if (tid == 0) {
    *abort_flag = 0;
    for (int s = 0; s < kStages; ++s) {
      mbar_init(bar(kFull + s), 1);
      mbar_init(bar(kEmpty + s), 1);
    }
    mbar_init(bar(kAccFull0), 1);
    mbar_init(bar(kAccFull1), 1);
    mbar_init(bar(kAccEmpty0), 128);
    mbar_init(bar(kAccEmpty1), 128);
    mbar_init(bar(kDrain), 1);
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  pdl_trigger();
  // A is a library output (the attention's, or the first product's): every
  // role waits for the preceding kernels before touching global memory
  pdl_wait();

  if (warp == 0) {
    // =================== TMA producer ===================
    if (lane == 0) {
      uint32_t kt = 0;
      for (int u = blockIdx.x; u < p.n_units; u += gridDim.x) {
        const Unit w = make_unit(p, u);
        for (int k = w.k0; k < w.k1; ++k, ++kt) {
          const uint32_t s = kt % kStages;
          if (kt >= (uint32_t)kStages &&
              !mbar_wait(bar(kEmpty + s), ((kt / kStages) - 1) & 1u, abort_flag, err))
            break;
          mbar_expect_tx(bar(kFull + s), kStageBytes);
          const uint32_t dst = sbase + s * kStageBytes;
          tma_load_2d(dst, &amap, w.a_koff + k * kBK, w.m0, bar(kFull + s));
          tma_load_2d(dst + kStageA, &bmap, k * kBK, w.n0, bar(kFull + s));
        }
      }
      // no copy into this block's shared memory is left in flight at exit
      for (uint32_t j = kt > (uint32_t)kStages ? kt - kStages : 0; j < kt; ++j)
        mbar_drain(bar(kFull + j % kStages), (j / kStages) & 1u);
    }
    __syncwarp();
  } else if (warp == 1) {
    // =================== MMA issuer ===================
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16(kBM, kBN, 0, 0);
      const uint64_t a_desc0 = sdesc_sw128(sbase, 16, 1024);
      const uint64_t b_desc0 = sdesc_sw128(sbase + kStageA, 16, 1024);
      uint32_t kt = 0, at = 0;
      for (int u = blockIdx.x; u < p.n_units; u += gridDim.x, ++at) {
        const Unit w = make_unit(p, u);
        const uint32_t ab = at & 1u;
        if (at >= 2) mbar_wait(bar(kAccEmpty0 + ab), ((at >> 1) - 1) & 1u, abort_flag, err);
        tc_fence_after();
        for (int k = w.k0; k < w.k1; ++k, ++kt) {
          const uint32_t s = kt % kStages;
          mbar_wait(bar(kFull + s), (kt / kStages) & 1u, abort_flag, err);
          tc_fence_after();
          const uint64_t soff = (s * kStageBytes) >> 4;
#pragma unroll
          for (int kk = 0; kk < kBK / 16; ++kk)
            mma_bf16(tmem + ab * 256u, a_desc0 + soff + ((kk * 32u) >> 4), b_desc0 + soff + ((kk * 32u) >> 4),
                     idesc, (k > w.k0 || kk > 0) ? 1u : 0u);
          mma_commit(bar(kEmpty + s));
        }
        mma_commit(bar(kAccFull0 + ab));
      }
      mma_commit(bar(kDrain));
      mbar_wait(bar(kDrain), 0, abort_flag, err);
    }
    __syncwarp();
  } else {
    // =================== epilogue ===================
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;  // row of the tile
    const uint32_t t_lane = tmem + ((uint32_t)(quarter * 32) << 16);
    uint32_t at = 0;
    for (int u = blockIdx.x; u < p.n_units; u += gridDim.x, ++at) {
      const Unit w = make_unit(p, u);
      const uint32_t ab = at & 1u;
      mbar_wait(bar(kAccFull0 + ab), (at >> 1) & 1u, abort_flag, err);
      tc_fence_after();
      const int row = w.m0 + r;
      const bool live = row < p.M;
      const bool empty = w.k1 <= w.k0;  // a split with no k steps: its partial is 0
      const int ks = u % p.ksplit;
#pragma unroll 1
      for (int c = 0; c < kBN / 32; ++c) {
        float v[32];
        tmem_ld32(t_lane + ab * 256u + (uint32_t)(c * 32), v);
        tmem_ld_wait();
        if (!live) continue;
        const int col = w.n0 + c * 32;
        if (p.ksplit == 1) {
          uint4* dst = reinterpret_cast<uint4*>(p.out + (int64_t)row * p.ldo + col);
#pragma unroll
          for (int q = 0; q < 4; ++q)
            dst[q] = make_uint4(f2_to_bf2x2(v[8 * q], v[8 * q + 1]), f2_to_bf2x2(v[8 * q + 2], v[8 * q + 3]),
                                f2_to_bf2x2(v[8 * q + 4], v[8 * q + 5]), f2_to_bf2x2(v[8 * q + 6], v[8 * q + 7]));
        } else {
          float4* dst = reinterpret_cast<float4*>(p.acc + ((int64_t)ks * p.M + row) * p.N + col);
#pragma unroll
          for (int q = 0; q < 8; ++q)
            dst[q] = empty ? make_float4(0.f, 0.f, 0.f, 0.f)
                           : make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
        }
      }
      tc_fence_before();
      mbar_arrive(bar(kAccEmpty0 + ab));
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, 512);
}

// split-K partial sums [ksplit][M][N] -> their sum, in split order, as
// bf16; 8 values per thread
__global__ void __launch_bounds__(256) round_bf16_kernel(const float* __restrict__ acc, int M, int N, int ksplit,
                                                         uint16_t* __restrict__ out, int64_t ldo) {
  pdl_trigger();
  pdl_wait();
  const int64_t n8 = (int64_t)M * N / 8, plane = (int64_t)M * N / 4;  // float4 per split
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n8; i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t e = i * 8;
    const int row = (int)(e / N), col = (int)(e % N);
    float4 a = reinterpret_cast<const float4*>(acc)[2 * i];
    float4 b = reinterpret_cast<const float4*>(acc)[2 * i + 1];
    for (int k = 1; k < ksplit; ++k) {
      const float4 c = reinterpret_cast<const float4*>(acc)[k * plane + 2 * i];
      const float4 d = reinterpret_cast<const float4*>(acc)[k * plane + 2 * i + 1];
      a.x += c.x; a.y += c.y; a.z += c.z; a.w += c.w;
      b.x += d.x; b.y += d.y; b.z += d.z; b.w += d.w;
    }
    *reinterpret_cast<uint4*>(out + (int64_t)row * ldo + col) =
        make_uint4(f2_to_bf2x2(a.x, a.y), f2_to_bf2x2(a.z, a.w), f2_to_bf2x2(b.x, b.y), f2_to_bf2x2(b.z, b.w));
  }
}

bool encode_2d(CUtensorMap* map, const void* base, uint64_t cols, uint64_t rows, uint64_t row_stride_elems,
               uint32_t box_rows) {
  PFN_cuTensorMapEncodeTiled_v12000 encode = get_encode();
  if (!encode) return false;
  const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)row_stride_elems * 2};
  const cuuint32_t box[2] = {(cuuint32_t)kBK, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

// Split of K when the row and output tiles alone cannot fill the SMs (few
// tokens: the product streams its weights and is bound by HBM).
int gemm_ksplit(int M, int N, int K) {
  const int tiles = ((M + kBM - 1) / kBM) * (N / kBN);
  const int steps = K / kBK;
  if (tiles >= 74) return 1;
  int ks = 1;
  while (ks * 2 * tiles <= 148 && steps / (ks * 2) >= 4) ks *= 2;
  return ks;
}

size_t gemm_acc_bytes(int M, int N, int K) {
  const int ks = gemm_ksplit(M, N, K);
  return ks > 1 ? (size_t)ks * M * N * sizeof(float) : 0;
}

// One product: out[M][N] (row stride ldo) = A[M][...] x B[N][K]^T, where
// output tile columns n take A's columns from (n / n_per_group) * a_group_k.
// a: bf16 rows of a_cols (row stride a_ld); b: bf16 [N][K].
cudaError_t launch_gemm(const uint16_t* a, int64_t a_cols, int64_t a_ld, const uint16_t* b, int M, int N, int K,
                        int n_per_group, int a_group_k, uint16_t* out, int64_t ldo, float* acc,
                        unsigned int* err, cudaStream_t s) {
  if (M <= 0) return cudaSuccess;
  CUtensorMap amap, bmap;
  if (!encode_2d(&amap, a, (uint64_t)a_cols, (uint64_t)M, (uint64_t)a_ld, kBM)) return cudaErrorInvalidValue;
  if (!encode_2d(&bmap, b, (uint64_t)K, (uint64_t)N, (uint64_t)K, kBN)) return cudaErrorInvalidValue;
  GemmParams p;
  p.M = M; p.N = N; p.k_steps = K / kBK;
  p.n_per_group = n_per_group; p.a_group_k = a_group_k;
  p.m_tiles = (M + kBM - 1) / kBM;
  p.n_tiles = N / kBN;
  p.ksplit = gemm_ksplit(M, N, K);
  p.steps_per_split = (p.k_steps + p.ksplit - 1) / p.ksplit;
  p.n_units = p.m_tiles * p.n_tiles * p.ksplit;
  p.out = out; p.ldo = ldo; p.acc = acc; p.err = err;
  static std::atomic<int> cache[kMaxDevices];
  cudaError_t e = ensure_smem(gemm_tc_kernel, (int)kSmemBytes, cache);
  if (e != cudaSuccess) return e;
  if (p.ksplit > 1 && !acc) return cudaErrorInvalidValue;
  {
    TraceScope tr("out_proj_gemm", s);
    e = launch_pdl(gemm_tc_kernel, dim3(min(p.n_units, 148)), dim3(kThreads), kSmemBytes, s, amap, bmap, p);
  }
  if (e != cudaSuccess || p.ksplit == 1) return e;
  const int64_t n8 = (int64_t)M * N / 8;
  const int64_t blocks = (n8 + 255) / 256;
  const int grid = (int)(blocks < 148 * 8 ? blocks : 148 * 8);
  TraceScope tr("out_proj_round", s);
  return launch_pdl(round_bf16_kernel, dim3(grid), dim3(256), 0, s, (const float*)acc, M, N, p.ksplit, out, ldo);
}

}  // namespace ds4a
