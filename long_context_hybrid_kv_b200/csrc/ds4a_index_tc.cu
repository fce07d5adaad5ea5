// Tensor-core (tcgen05) Lightning-Indexer score for the Flash shape
// (64 indexer heads x 128): "DeepSeek-v4 Beyond Basics" 3.2.2 eq. 16,
//   I[t][s] = sum_h w[t][h] * ReLU(q[t][h] . K[s]).
// Per tile of 128 keys and a group of G queries of one sequence (G = 4 when
// the sequence has several queries, else 1) one product
//   D[key][g*64 + h] = K[key][:] . q[g][h][:]      (M = 128, N = 64 G, K = 128)
// lands in tensor memory; the epilogue thread that owns a key row applies
// the ReLU and the head weights in registers and writes the G scores.
//
// Thread block (320 threads, one per SM):
//   warp 0     lane 0 streams K tiles with TMA (3-D map [B][N_c][128],
//              128-byte swizzle, two 64-dim boxes per tile) into 4 stages,
//              and the group's queries (2-D map over [B*T_q*64][128]);
//   warp 1     TMEM allocation; lane 0 issues the MMAs (8 x K=16 per tile)
//              into two accumulator buffers;
//   warps 2-9  epilogue: two warps per TMEM lane quarter, each with every
//              other query of the group (with G = 1 the second warp of a
//              quarter idles).  The epilogue bounds the prefill indexer (it
//              took ~40 % of its time with one warp per quarter), so two
//              warps per SM sub-partition hide each other's latencies.
// Work: (query group, chunk of key tiles) pairs, taken round-robin by the
// blocks; pairs past a group's visible entries are skipped.
// FP4 keys (E2M1 codes and E8M0 scales per 32 dims): a bulk copy brings a
// tile's packed codes and scales into a raw ring; four more warps (10-13)
// expand them exactly into the same bf16 tile (the hardware unpacks a code
// byte to its two values, times the block's power-of-two scale), and the
// products and the epilogue are unchanged.  Three stages instead of four
// make room for the raw ring.
#include <cuda.h>
#include <cudaTypedefs.h>

#include "ds4a_mx.cuh"
#include "ds4a_tc.cuh"

namespace ds4a {
namespace {

using namespace tc;

constexpr int kHI = 64;
constexpr int kDI = 128;
constexpr int kKT = 128;      // keys per tile
constexpr int kStages = 4;
constexpr int kThreads = 320;
constexpr int kEpiThreads = 256;
// registers are granted for whole groups of four warps: cap the kernel's
// registers as for 384 threads so that its 10 warps fit in one SM's file
constexpr int kRegBoundThreads = 384;
constexpr int kMaxG = 4;

constexpr int kStagesFp4 = 3;
constexpr int kConvThreads = 128;
constexpr uint32_t kRawCodes = kKT * kDI / 2;  // 8 KiB of E2M1 codes per tile
constexpr uint32_t kRawStage = kRawCodes + kKT * (kDI / kMxBlock);  // + 512 B of scales

// shared memory map (offsets from a 1024-aligned base) of either variant
template <bool kFp4>
struct Layout {
  static constexpr int stages = kFp4 ? kStagesFp4 : kStages;
  static constexpr uint32_t k = 0;                                  // stages x 2 blocks x 16 KB
  static constexpr uint32_t raw = stages * 32768;                   // FP4: stages x kRawStage
  static constexpr uint32_t q = (raw + (kFp4 ? stages * kRawStage : 0) + 1023) / 1024 * 1024;
  static constexpr uint32_t w = q + 2 * kMaxG * 8192;               // [G*64] floats
  static constexpr uint32_t bar = w + kMaxG * kHI * 4;
  static constexpr uint32_t misc = bar + 256;
  static constexpr uint32_t bytes = misc + 64 + 1024;
  static constexpr int threads = kFp4 ? kThreads + kConvThreads : kThreads;
};

// barrier slots (FP4 adds the raw ring's full / empty barriers)
constexpr int kKFull = 0, kKEmpty = 4, kQFull = 8, kQEmpty = 9, kAccFull0 = 10, kAccFull1 = 11,
              kAccEmpty0 = 12, kAccEmpty1 = 13, kDrain = 14, kRawFull = 15, kRawEmpty = 19;

struct TcIndexParams {
  IndexArgs a;
  int G;               // queries per group
  int groups_per_b;    // ceil(T_q / G)
  int n_groups;
  int chunk_tiles;     // key tiles per work pair
  int chunks_per_group;
  int n_pairs;
  int keys_once;       // one group per batch: every key tile is read once
};

struct Pair {
  int g, b, t0, nrows, tile0, tile1;  // tiles [tile0, tile1)
  int n_vis[kMaxG];
};

__device__ __forceinline__ Pair make_pair(const TcIndexParams& p, int w) {
  Pair q;
  q.g = w / p.chunks_per_group;
  const int chunk = w % p.chunks_per_group;
  q.b = q.g / p.groups_per_b;
  q.t0 = (q.g % p.groups_per_b) * p.G;
  q.nrows = min(p.G, p.a.T_q - q.t0);
  int vmax = 0;
  for (int i = 0; i < kMaxG; ++i) {
    int nv = 0;
    if (i < q.nrows) {
      const int pos = p.a.q_pos[q.b * p.a.T_q + q.t0 + i];
      nv = pos < 0 ? 0 : min((pos + 1) / p.a.m, p.a.N_c);
    }
    q.n_vis[i] = nv;
    vmax = max(vmax, nv);
  }
  const int tiles = (vmax + kKT - 1) / kKT;
  q.tile0 = min(tiles, chunk * p.chunk_tiles);
  q.tile1 = min(tiles, q.tile0 + p.chunk_tiles);
  return q;
}

template <bool kFp4>
__global__ void __launch_bounds__(kFp4 ? 512 : kRegBoundThreads, 1)
    index_tc_kernel(const __grid_constant__ CUtensorMap kmap, const __grid_constant__ CUtensorMap qmap,
                    const TcIndexParams p) {
  using Lay = Layout<kFp4>;
  constexpr int kS = Lay::stages;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  const uint32_t sbase = smem_u32(smem);
  const uint32_t k_base = sbase + Lay::k, q_base = sbase + Lay::q;
  float* w_s = reinterpret_cast<float*>(smem + Lay::w);
  const uint32_t bar0 = sbase + Lay::bar;
  auto bar = [&](int i) { return bar0 + 8u * (uint32_t)i; };
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Lay::misc);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Lay::misc + 8);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int G = p.G;
  const IndexArgs& a = p.a;
  unsigned int* err = a.err;
  const uint32_t q_bytes = (uint32_t)G * 64u * 256u;
  const uint32_t q_blk = (uint32_t)G * 8192u;  // one 64-dim block of the group's queries

  if (tid == 0) {
    *abort_flag = 0;
    for (int s = 0; s < kS; ++s) {
      mbar_init(bar(kKFull + s), kFp4 ? kConvThreads : 1);
      mbar_init(bar(kKEmpty + s), 1);
      if (kFp4) {
        mbar_init(bar(kRawFull + s), 1);
        mbar_init(bar(kRawEmpty + s), kConvThreads);
      }
    }
    mbar_init(bar(kQFull), 1);
    mbar_init(bar(kQEmpty), 1);
    mbar_init(bar(kAccFull0), 1);
    mbar_init(bar(kAccFull1), 1);
    mbar_init(bar(kAccEmpty0), kEpiThreads);
    mbar_init(bar(kAccEmpty1), kEpiThreads);
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
  // Each role waits for the preceding kernels only before its first read of
  // their output (the keys) or its first write: the queries, weights and
  // positions are inputs that no kernel of the chain writes, so the first
  // pair's queries and weights come in while the preceding kernel finishes.

  if (warp == 0) {
    // =================== TMA producer ===================
    if (lane == 0) {
      uint32_t kt = 0, active = 0;
      const uint64_t pol = l2_evict_first_policy();
      auto load_q = [&](const Pair& q) {
        mbar_expect_tx(bar(kQFull), q_bytes);
        const int qrow = (q.b * a.T_q + q.t0) * kHI;
        tma_load_2d(q_base, &qmap, 0, qrow, bar(kQFull));
        tma_load_2d(q_base + q_blk, &qmap, 64, qrow, bar(kQFull));
      };
      int w_first = -1;
      for (int w = blockIdx.x; w < p.n_pairs; w += gridDim.x) {
        const Pair q = make_pair(p, w);
        if (q.tile1 <= q.tile0) continue;
        load_q(q);
        w_first = w;
        break;
      }
      pdl_wait();
      for (int w = blockIdx.x; w < p.n_pairs; w += gridDim.x) {
        const Pair q = make_pair(p, w);
        if (q.tile1 <= q.tile0) continue;
        if (w != w_first) {
          if (active > 0) mbar_wait(bar(kQEmpty), (active - 1) & 1u, abort_flag, err);
          load_q(q);
        }
        for (int tile = q.tile0; tile < q.tile1; ++tile, ++kt) {
          const uint32_t s = kt % kS;
          if (kFp4) {
            // the tile's packed codes and scales (rows past N_c are not read)
            if (kt >= (uint32_t)kS) mbar_wait(bar(kRawEmpty + s), ((kt / kS) - 1) & 1u, abort_flag, err);
            const int rows = min(kKT, a.N_c - tile * kKT);
            const int64_t key0 = (int64_t)q.b * a.k_bstride + (int64_t)tile * kKT;
            const uint32_t raw = sbase + Lay::raw + s * kRawStage;
            mbar_expect_tx(bar(kRawFull + s), (uint32_t)rows * (kDI / 2 + kDI / kMxBlock));
            if (p.keys_once) {
              bulk_g2s_hint(raw, a.kcodes + key0 * (kDI / 2), (uint32_t)rows * (kDI / 2), bar(kRawFull + s), pol);
              bulk_g2s_hint(raw + kRawCodes, a.kscales + key0 * (kDI / kMxBlock),
                            (uint32_t)rows * (kDI / kMxBlock), bar(kRawFull + s), pol);
            } else {
              bulk_g2s(raw, a.kcodes + key0 * (kDI / 2), (uint32_t)rows * (kDI / 2), bar(kRawFull + s));
              bulk_g2s(raw + kRawCodes, a.kscales + key0 * (kDI / kMxBlock), (uint32_t)rows * (kDI / kMxBlock),
                       bar(kRawFull + s));
            }
            continue;
          }
          if (kt >= (uint32_t)kS)
            mbar_wait(bar(kKEmpty + s), ((kt / kS) - 1) & 1u, abort_flag, err);
          mbar_expect_tx(bar(kKFull + s), 32768u);
          const uint32_t dst = k_base + s * 32768u;
          if (p.keys_once) {
            tma_load_3d_hint(dst, &kmap, 0, tile * kKT, q.b, bar(kKFull + s), pol);
            tma_load_3d_hint(dst + 16384u, &kmap, 64, tile * kKT, q.b, bar(kKFull + s), pol);
          } else {
            tma_load_3d(dst, &kmap, 0, tile * kKT, q.b, bar(kKFull + s));
            tma_load_3d(dst + 16384u, &kmap, 64, tile * kKT, q.b, bar(kKFull + s));
          }
        }
        ++active;
      }
      if (kFp4) {
        // no bulk copy into this block's shared memory is left in flight
        for (uint32_t j = kt > (uint32_t)kS ? kt - kS : 0; j < kt; ++j)
          mbar_drain(bar(kRawFull + j % kS), (j / kS) & 1u);
      }
    }
    if (lane != 0) pdl_wait();
    __syncwarp();
  } else if (warp == 1) {
    // =================== MMA issuer ===================
    pdl_wait();
    if (lane == 0) {
      uint32_t kt = 0, at = 0, active = 0;
      const uint32_t idesc = idesc_bf16(128, 64 * G, 0, 0);
      const uint64_t k_desc0 = sdesc_sw128(k_base, 16, 1024);
      const uint64_t q_desc0 = sdesc_sw128(q_base, 16, 1024);
      for (int w = blockIdx.x; w < p.n_pairs; w += gridDim.x) {
        const Pair q = make_pair(p, w);
        if (q.tile1 <= q.tile0) continue;
        mbar_wait(bar(kQFull), active & 1u, abort_flag, err);
        tc_fence_after();
        for (int tile = q.tile0; tile < q.tile1; ++tile, ++kt, ++at) {
          const uint32_t s = kt % kS;
          const uint32_t ab = at & 1u;
          mbar_wait(bar(kKFull + s), (kt / kS) & 1u, abort_flag, err);
          if (at >= 2) mbar_wait(bar(kAccEmpty0 + ab), ((at >> 1) - 1) & 1u, abort_flag, err);
          tc_fence_after();
          const uint64_t a0 = k_desc0 + ((s * 32768u) >> 4);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint32_t blk = (uint32_t)(kk >> 2);
            const uint32_t koff = (uint32_t)(kk & 3) * 32u;
            mma_bf16(tmem + ab * 256u, a0 + ((blk * 16384u + koff) >> 4), q_desc0 + ((blk * q_blk + koff) >> 4),
                     idesc, kk != 0 ? 1u : 0u);
          }
          mma_commit(bar(kKEmpty + s));
          mma_commit(bar(kAccFull0 + ab));
        }
        mma_commit(bar(kQEmpty));
        ++active;
      }
      mma_commit(bar(kDrain));
      mbar_wait(bar(kDrain), 0, abort_flag, err);
    }
    __syncwarp();
  } else if (kFp4 && warp >= 10) {
    // =================== FP4 -> bf16 converters ===================
    const int r = tid - kThreads;  // key row of the tile
    uint32_t kt = 0;
    for (int w = blockIdx.x; w < p.n_pairs; w += gridDim.x) {
      const Pair q = make_pair(p, w);
      for (int tile = q.tile0; tile < q.tile1; ++tile, ++kt) {
        const uint32_t s = kt % kS;
        mbar_wait(bar(kRawFull + s), (kt / kS) & 1u, abort_flag, err);
        const unsigned char* raw = smem + Lay::raw + s * kRawStage;
        const bool live = tile * kKT + r < a.N_c;
        uint4 cw[4];
        uint32_t sc4 = 0;
        if (live) {
#pragma unroll
          for (int i = 0; i < 4; ++i) cw[i] = reinterpret_cast<const uint4*>(raw + r * (kDI / 2))[i];
          sc4 = *reinterpret_cast<const uint32_t*>(raw + kRawCodes + r * (kDI / kMxBlock));
        }
        mbar_arrive(bar(kRawEmpty + s));  // the raw slot may refill
        if (kt >= (uint32_t)kS) mbar_wait(bar(kKEmpty + s), ((kt / kS) - 1) & 1u, abort_flag, err);
        const uint32_t dst = k_base + s * 32768u;
#pragma unroll
        for (int i = 0; i < 4; ++i) {  // 32 dims = one scale block
          const float sc = mx_scale((int)((sc4 >> (8 * i)) & 255u));
          const uint32_t words[4] = {cw[i].x, cw[i].y, cw[i].z, cw[i].w};
#pragma unroll
          for (int h = 0; h < 2; ++h) {  // 8 code bytes = 16 dims = two 16-byte pieces
            uint32_t o[8];
#pragma unroll
            for (int k = 0; k < 8; ++k) {
              const uint32_t byte = (words[2 * h + (k >> 2)] >> (8 * (k & 3))) & 255u;
              const float2 v = mul_f2(e2m1x2_to_f2(byte), make_float2(sc, sc));
              o[k] = live ? f2_to_bf2x2(v.x, v.y) : 0u;
            }
            // dims 32 i + 16 h .. + 15: block (i >> 1), 16-byte chunks
            const int d0 = 32 * i + 16 * h;
            const uint32_t blk = dst + (uint32_t)(d0 >> 6) * 16384u;
            const uint32_t c0 = (uint32_t)((d0 & 63) >> 3);
            st_shared16(blk + sw128((uint32_t)r, c0), o[0], o[1], o[2], o[3]);
            st_shared16(blk + sw128((uint32_t)r, c0 + 1), o[4], o[5], o[6], o[7]);
          }
        }
        fence_async_smem();
        mbar_arrive(bar(kKFull + s));
      }
    }
  } else {
    // =================== epilogue ===================
    const int et = tid - 64;                 // 0..255
    const int quarter = warp & 3;            // TMEM lane quarter of this warp
    const int r = quarter * 32 + lane;       // key row within the tile
    const int gpar = (warp - 2) >> 2;        // this warp's queries: g = gpar, gpar + 2
    const uint32_t t_lane = tmem + ((uint32_t)(quarter * 32) << 16);
    uint32_t at = 0;
    bool first = true;
    for (int w = blockIdx.x; w < p.n_pairs; w += gridDim.x) {
      const Pair q = make_pair(p, w);
      if (q.tile1 <= q.tile0) continue;
      named_bar(1, kEpiThreads);  // everyone is done with the previous pair's weights
      for (int e = et; e < G * kHI; e += kEpiThreads) {
        const int g = e / kHI;
        w_s[e] = g < q.nrows ? bf2f(a.w[((int64_t)q.b * a.T_q + q.t0 + g) * kHI + (e % kHI)]) : 0.f;
      }
      if (first) pdl_wait();  // before the first score is written
      first = false;
      named_bar(1, kEpiThreads);
      for (int tile = q.tile0; tile < q.tile1; ++tile, ++at) {
        const uint32_t ab = at & 1u;
        mbar_wait(bar(kAccFull0 + ab), (at >> 1) & 1u, abort_flag, err);
        tc_fence_after();
        float sc[kMaxG / 2];
#pragma unroll
        for (int gi = 0; gi < kMaxG / 2; ++gi) {
          const int g = gpar + 2 * gi;
          sc[gi] = 0.f;
          if (g < G) {
            // four independent sums per query (a 64-long FMA chain would
            // stall the warp)
            float s4[4] = {0.f, 0.f, 0.f, 0.f};
            // both 32-column halves in flight, one wait
            float v[2][32];
            tmem_ld32(t_lane + ab * 256u + (uint32_t)(g * 64), v[0]);
            tmem_ld32(t_lane + ab * 256u + (uint32_t)(g * 64 + 32), v[1]);
            tmem_ld_wait();
#pragma unroll
            for (int half = 0; half < 2; ++half) {
              // the weights are the same for every thread: 16-byte broadcast
              // reads, a quarter of the shared-memory instructions
              const float4* w4 = reinterpret_cast<const float4*>(w_s + g * kHI + half * 32);
#pragma unroll
              for (int i = 0; i < 32; i += 4) {
                const float4 ww = w4[i >> 2];
                s4[0] = fmaf(ww.x, fmaxf(v[half][i], 0.f), s4[0]);
                s4[1] = fmaf(ww.y, fmaxf(v[half][i + 1], 0.f), s4[1]);
                s4[2] = fmaf(ww.z, fmaxf(v[half][i + 2], 0.f), s4[2]);
                s4[3] = fmaf(ww.w, fmaxf(v[half][i + 3], 0.f), s4[3]);
              }
            }
            sc[gi] = (s4[0] + s4[1]) + (s4[2] + s4[3]);
          }
        }
        tc_fence_before();
        mbar_arrive(bar(kAccEmpty0 + ab));
        const int s = tile * kKT + r;
#pragma unroll
        for (int gi = 0; gi < kMaxG / 2; ++gi) {
          const int g = gpar + 2 * gi;
          const int nv = gpar ? q.n_vis[2 * gi + 1] : q.n_vis[2 * gi];  // constant indices
          if (g < q.nrows && s < nv)
            a.scores[((int64_t)q.b * a.T_q + q.t0 + g) * a.N_c + s] = sc[gi];
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, 512);
}

}  // namespace

// The driver's tensor-map encoder, looked up once through the runtime (no
// link against the driver library); null when the driver has none.
PFN_cuTensorMapEncodeTiled_v12000 get_encode() {
  // concurrent first calls store the same pointer
  static std::atomic<PFN_cuTensorMapEncodeTiled_v12000> fn{nullptr};
  PFN_cuTensorMapEncodeTiled_v12000 f = fn.load(std::memory_order_acquire);
  if (!f) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess) {
      f = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
      fn.store(f, std::memory_order_release);
    } else {
      (void)cudaGetLastError();
    }
  }
  return f;
}


bool index_scores_tc_supported(const IndexArgs& a) {
  // Flash indexer width; the batch stride of the key pool must be a multiple
  // of 16 bytes for the tensor map
  if (a.kcodes)  // FP4 keys: whole 16-byte runs of scales per 4 keys
    return a.H == kHI && a.D == kDI && (a.k_bstride % 4) == 0 && (a.N_c % 4) == 0;
  return a.H == kHI && a.D == kDI && (a.k_bstride % 8) == 0 && a.N_c >= kKT && get_encode() != nullptr;
}

cudaError_t launch_index_scores_tc(const IndexArgs& a, cudaStream_t s) {
  const int rows = a.B * a.T_q;
  if (rows <= 0 || a.N_c <= 0) return cudaSuccess;
  PFN_cuTensorMapEncodeTiled_v12000 encode = get_encode();
  if (!encode) return cudaErrorNotSupported;
  TcIndexParams p;
  p.a = a;
  p.G = a.T_q >= kMaxG ? kMaxG : 1;
  p.groups_per_b = (a.T_q + p.G - 1) / p.G;
  p.n_groups = a.B * p.groups_per_b;
  const int max_tiles = (a.N_c + kKT - 1) / kKT;
  // about four rounds of pairs over the SMs, whole groups when they are many
  const long long want_pairs = 148ll * 4;
  int chunk = (int)((p.n_groups * (long long)max_tiles + want_pairs - 1) / want_pairs);
  chunk = max(1, min(chunk, max_tiles));
  p.chunk_tiles = chunk;
  p.chunks_per_group = (max_tiles + chunk - 1) / chunk;
  p.n_pairs = p.n_groups * p.chunks_per_group;
  p.keys_once = p.groups_per_b == 1;

  CUtensorMap kmap, qmap;
  memset(&kmap, 0, sizeof(kmap));
  const bool fp4 = a.kcodes != nullptr;
  if (!fp4) {
    const cuuint64_t dims[3] = {(cuuint64_t)kDI, (cuuint64_t)a.N_c, (cuuint64_t)a.B};
    const cuuint64_t strides[2] = {(cuuint64_t)kDI * 2, (cuuint64_t)a.k_bstride * 2};
    const cuuint32_t box[3] = {64, (cuuint32_t)kKT, 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    if (encode(&kmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<uint16_t*>(a.kidx), dims, strides,
               box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  {
    const cuuint64_t dims[2] = {(cuuint64_t)kDI, (cuuint64_t)rows * kHI};
    const cuuint64_t strides[1] = {(cuuint64_t)kDI * 2};
    const cuuint32_t box[2] = {64, (cuuint32_t)(p.G * kHI)};
    const cuuint32_t estr[2] = {1, 1};
    if (encode(&qmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<uint16_t*>(a.q), dims, strides, box,
               estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  static std::atomic<int> cache[kMaxDevices], cache4[kMaxDevices];
  const int grid = min(p.n_pairs, 148);
  if (fp4) {
    cudaError_t e = ensure_smem(index_tc_kernel<true>, (int)Layout<true>::bytes, cache4);
    if (e != cudaSuccess) return e;
    TraceScope tr("index_score_tc_fp4", s);
    return launch_pdl(index_tc_kernel<true>, dim3(grid), dim3(Layout<true>::threads), Layout<true>::bytes, s, kmap,
                      qmap, p);
  }
  cudaError_t e = ensure_smem(index_tc_kernel<false>, (int)Layout<false>::bytes, cache);
  if (e != cudaSuccess) return e;
  TraceScope tr("index_score_tc", s);
  return launch_pdl(index_tc_kernel<false>, dim3(grid), dim3(Layout<false>::threads), Layout<false>::bytes, s, kmap,
                    qmap, p);
}

}  // namespace ds4a
