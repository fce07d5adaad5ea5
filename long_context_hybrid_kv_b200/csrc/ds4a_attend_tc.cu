// Tensor-core (tcgen05) attention for the Flash shape: 64 query heads x 512
// sharing one K=V head ("DeepSeek-v4 Beyond Basics" 3.2.2 eq. 19 and 3.3
// eqs. 24-27; "DeepSeek V4 Inside" sink and window examples).
//
// Every head reads the same K=V rows, so per tile of 128 keys the work is
// two dense products; both run with the 128 keys / 128 dims on the MMA's M
// side and the 64 heads on N ("swap AB"), which keeps M = 128:
//   S^T[key][h]  = KV[key][:] . q^[h][:]          (K = 512, A K-major)
//   O^T[d][h]   += KV[key][d]^T . P^T[key][h]      (K = 128 keys, A MN-major)
// S^T (64 columns) and O^T (4 x 64 columns) live in tensor memory.  The KV
// tile is read once from HBM (gathered rows: pool[idx] then the window) and
// serves both products.
//
// Thread block (one per SM, 288 threads):
//   warps 0-3  softmax + epilogue: thread = key row of S^T (lane), later
//              dim row of O^T; online softmax with a lazy rescale (O^T is
//              rescaled only when a head's running max grows by more than
//              2^8), P^T to shared memory as bf16, final normalisation with
//              the sink, de-rotation of the rope slice by -pos, stores.
//   warp 4     TMEM allocation; lane 0 issues every tcgen05.mma / commit.
//   warps 5-8  producers: q^ = RoPE(RMSNorm(q) * g) into shared memory, then
//              the KV rows by cp.async, one 128-dim chunk (32 KB) at a time,
//              each chunk released by the PV products that read it.
// Work items are (query, key split) pairs taken round-robin by the blocks;
// with one split the block writes the final bf16 output, otherwise the
// float partials (max, sum, accumulator) the combine kernel merges.
#include "ds4a_tc.cuh"

namespace ds4a {
namespace {

using namespace tc;

constexpr int kH = 64;
constexpr int kD = 512;
constexpr int kKT = 128;              // keys per tile
constexpr int kThreads = 288;
constexpr int kSG = 0;                // softmax warps 0-3
constexpr int kMmaWarp = 4;
constexpr int kPG0 = 160;             // first producer thread
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRescaleLog2 = 8.0f;  // lazy-rescale threshold (log2 units)

// shared memory map (offsets from a 1024-aligned base)
constexpr uint32_t kOffKV = 0;              // 8 blocks x [128 keys][128 B]
constexpr uint32_t kOffQ = 131072;          // 8 blocks x [64 heads][128 B]
constexpr uint32_t kOffP = 196608;          // [128 keys][128 B]
constexpr uint32_t kOffBar = 212992;        // mbarriers
constexpr uint32_t kOffMisc = kOffBar + 256;
constexpr uint32_t kOffRowPtr = kOffMisc + 64;      // 128 x 8 B
constexpr uint32_t kOffRed = kOffRowPtr + 1024;     // [4][64] floats
constexpr uint32_t kOffMrun = kOffRed + 1024;       // [64]
constexpr uint32_t kOffAlpha = kOffMrun + 256;      // [64]
constexpr uint32_t kOffInv = kOffAlpha + 256;       // [64]
constexpr uint32_t kSmemBytes = kOffInv + 256 + 1024;  // + alignment slack

enum Bar {
  kQFull = 0, kQEmpty, kKVFull0, kKVFull1, kKVFull2, kKVFull3, kKVEmpty0, kKVEmpty1, kKVEmpty2,
  kKVEmpty3, kSFull, kPFull, kPVDone, kEpiDone, kDrain, kNumBars
};

constexpr uint32_t kIdescQK = idesc_bf16(128, 64, 0, 0);
constexpr uint32_t kIdescPV = idesc_bf16(128, 64, 1, 1);

struct Item {
  int row, split, b, pos;
  int n_sel, win_start, j0, j1, n_tiles;
  const int32_t* idx_row;
};

// Called by all 32 lanes of a warp (the valid-index count is a warp sum).
__device__ __forceinline__ Item make_item(const AttendArgs& a, int w) {
  Item it;
  it.row = w / a.n_splits;
  it.split = w % a.n_splits;
  it.b = it.row / a.T_q;
  it.pos = a.q_pos[it.row];
  it.idx_row = a.sparse ? a.idx + (int64_t)it.row * a.k : nullptr;
  if (it.pos < 0) {
    it.n_sel = 0;
    it.win_start = 0;
    it.j0 = it.j1 = 0;
    it.n_tiles = 0;
    return it;
  }
  int n_sel;
  if (a.sparse) {
    // selected entries come first (ascending, -1 padded): count them with
    // independent loads, 8 per lane in flight
    const int lane = threadIdx.x & 31;
    int cnt = 0;
    for (int base = 0; base < a.k; base += 256) {
      int v[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int j = base + 32 * u + lane;
        v[u] = j < a.k ? it.idx_row[j] : -1;
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) cnt += v[u] >= 0;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) cnt += __shfl_xor_sync(0xffffffffu, cnt, o);
    n_sel = cnt;
  } else {
    n_sel = min((it.pos + 1) / a.m, a.N_c);
  }
  it.n_sel = n_sel;
  it.win_start = max(0, it.pos - a.W + 1);
  const int n_win = a.W > 0 ? it.pos - it.win_start + 1 : 0;
  const int n_keys = n_sel + n_win;
  // splits take whole tiles, as evenly as they divide
  const int tiles = (n_keys + kKT - 1) / kKT;
  const int t0 = (int)((int64_t)it.split * tiles / a.n_splits);
  const int t1 = (int)((int64_t)(it.split + 1) * tiles / a.n_splits);
  it.j0 = t0 * kKT;
  it.j1 = min(n_keys, t1 * kKT);
  it.n_tiles = t1 - t0;
  return it;
}

// row pointer of key j of an item, or nullptr (out of range / bad index)
__device__ __forceinline__ const uint16_t* key_ptr(const AttendArgs& a, const Item& it, int j,
                                                   bool* bad) {
  *bad = false;
  if (j >= it.j1) return nullptr;
  if (j < it.n_sel) {
    const int e = a.sparse ? it.idx_row[j] : j;
    if (e < 0 || e >= a.N_c) {
      *bad = true;
      return nullptr;
    }
    return a.pool + (int64_t)it.b * a.pool_bstride + (int64_t)e * kD;
  }
  const int p = it.win_start + (j - it.n_sel);
  return a.win + (int64_t)it.b * a.win_bstride + (int64_t)(p % a.win_cap) * kD;
}

__global__ void __launch_bounds__(kThreads, 1) attend_tc_kernel(AttendArgs a, int n_items) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  const uint32_t sbase = smem_u32(smem);
  const uint32_t kv_base = sbase + kOffKV, q_base = sbase + kOffQ, p_base = sbase + kOffP;
  const uint32_t bar0 = sbase + kOffBar;
  auto bar = [&](int i) { return bar0 + 8u * (uint32_t)i; };
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kOffMisc);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kOffMisc + 8);
  const uint16_t** rowptr = reinterpret_cast<const uint16_t**>(smem + kOffRowPtr);
  float* red = reinterpret_cast<float*>(smem + kOffRed);
  float* mrun = reinterpret_cast<float*>(smem + kOffMrun);
  float* alpha_s = reinterpret_cast<float*>(smem + kOffAlpha);
  float* inv_s = reinterpret_cast<float*>(smem + kOffInv);
  int* any_rescale = reinterpret_cast<int*>(smem + kOffMisc + 16);

  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;

  if (tid == 0) {
    *abort_flag = 0;
    mbar_init(bar(kQFull), 128);
    mbar_init(bar(kQEmpty), 1);
    for (int c = 0; c < 4; ++c) {
      mbar_init(bar(kKVFull0 + c), 128);
      mbar_init(bar(kKVEmpty0 + c), 1);
    }
    mbar_init(bar(kSFull), 1);
    mbar_init(bar(kPFull), 128);
    mbar_init(bar(kPVDone), 1);
    mbar_init(bar(kEpiDone), 128);
    mbar_init(bar(kDrain), 1);
    fence_barrier_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  unsigned int* err = a.err;

  if (warp < 4) {
    // =================== softmax + epilogue ===================
    const int r = tid;  // key row of S^T / dim row of O^T within a chunk
    const uint32_t t_lane = tmem + ((uint32_t)(32 * warp) << 16);
    const float scale2 = a.scale * kLog2e;
    uint32_t gt = 0, active = 0;
    for (int w = blockIdx.x; w < n_items; w += gridDim.x) {
      const Item it = make_item(a, w);
      const bool final_out = a.n_splits == 1;
      if (it.pos < 0 && r == 0 && it.split == 0) raise_err(err, DS4A_DEV_BAD_POS);
      if (it.n_tiles == 0) {
        // no keys in this item: output 0, or an empty partial
        if (final_out) {
          if (it.pos >= 0)
            for (int e = r; e < kH * kD / 8; e += 128)
              reinterpret_cast<uint4*>(a.out + (int64_t)it.row * kH * kD)[e] = make_uint4(0, 0, 0, 0);
        } else {
          float* part = a.ws + ((int64_t)it.row * a.n_splits + it.split) * (2 * kH + kH * kD);
          if (r < kH) {
            part[r] = -INFINITY;
            part[kH + r] = 0.f;
          }
          for (int e = r; e < kH * kD; e += 128) part[2 * kH + e] = 0.f;
        }
        continue;
      }
      if (r < kH) mrun[r] = -INFINITY;
      float lpart[64];
#pragma unroll
      for (int h = 0; h < 64; ++h) lpart[h] = 0.f;
      named_bar(1, 128);
      for (int tile = 0; tile < it.n_tiles; ++tile, ++gt) {
        const uint32_t sb = gt & 1u;
        mbar_wait(bar(kSFull), gt & 1u, abort_flag, err);
        tc_fence_after();
        float z[64];
        {
          float v[32];
          tmem_ld32(t_lane + sb * 64u, v);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 32; ++i) z[i] = v[i];
          tmem_ld32(t_lane + sb * 64u + 32u, v);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 32; ++i) z[32 + i] = v[i];
        }
        const int j = it.j0 + tile * kKT + r;
        bool bad = false;
        const bool valid = key_ptr(a, it, j, &bad) != nullptr;
#pragma unroll
        for (int h = 0; h < 64; ++h) z[h] = valid ? z[h] * scale2 : -INFINITY;
        float m0, m1;
        warp_reduce64<true>(z, m0, m1);
        red[warp * 64 + 2 * lane] = m0;
        red[warp * 64 + 2 * lane + 1] = m1;
        if (r == 0) *any_rescale = 0;
        named_bar(1, 128);
        if (r < kH) {
          const float mt = fmaxf(fmaxf(red[r], red[64 + r]), fmaxf(red[128 + r], red[192 + r]));
          const float mo = mrun[r];
          float al = 1.f;
          if (mt > mo + kRescaleLog2 || (mo == -INFINITY && mt != -INFINITY)) {
            al = (mo == -INFINITY) ? 0.f : exp2f(mo - mt);
            mrun[r] = mt;
            *any_rescale = 1;
          }
          alpha_s[r] = al;
        }
        named_bar(1, 128);
        uint32_t pk[32];
#pragma unroll
        for (int h = 0; h < 64; h += 2) {
          const float ma = mrun[h], mb = mrun[h + 1];
          const float pa = (z[h] == -INFINITY || ma == -INFINITY) ? 0.f : exp2f(z[h] - ma);
          const float pb = (z[h + 1] == -INFINITY || mb == -INFINITY) ? 0.f : exp2f(z[h + 1] - mb);
          const uint32_t w2 = f2_to_bf2x2(pa, pb);
          pk[h >> 1] = w2;
          const float2 pr = bf2x2_to_f2(w2);
          lpart[h] = lpart[h] * alpha_s[h] + pr.x;
          lpart[h + 1] = lpart[h + 1] * alpha_s[h + 1] + pr.y;
        }
        if (tile > 0) {
          // the previous tile's PV must be done before P^T and O^T change
          mbar_wait(bar(kPVDone), (gt - 1) & 1u, abort_flag, err);
          tc_fence_after();
          if (*any_rescale) {
#pragma unroll 1
            for (int c = 0; c < 4; ++c) {
#pragma unroll 1
              for (int half = 0; half < 2; ++half) {
                float v[32];
                const uint32_t addr = t_lane + 128u + 64u * c + 32u * half;
                tmem_ld32(addr, v);
                tmem_ld_wait();
#pragma unroll
                for (int i = 0; i < 32; ++i) v[i] *= alpha_s[32 * half + i];
                tmem_st32(addr, v);
              }
            }
            tmem_st_wait();
          }
        }
        // P^T row r: 64 heads as bf16 (128 B), 128-byte swizzled
#pragma unroll
        for (int c16 = 0; c16 < 8; ++c16)
          st_shared16(p_base + sw128(r, c16), pk[4 * c16], pk[4 * c16 + 1], pk[4 * c16 + 2],
                      pk[4 * c16 + 3]);
        fence_async_smem();
        tc_fence_before();
        mbar_arrive(bar(kPFull));
      }
      // ---------------- epilogue ----------------
      mbar_wait(bar(kPVDone), (gt - 1) & 1u, abort_flag, err);
      tc_fence_after();
      {
        float s0, s1;
        warp_reduce64<false>(lpart, s0, s1);
        red[warp * 64 + 2 * lane] = s0;
        red[warp * 64 + 2 * lane + 1] = s1;
      }
      named_bar(1, 128);
      if (r < kH) {
        const float l = red[r] + red[64 + r] + red[128 + r] + red[192 + r];
        const float m = mrun[r];
        if (final_out) {
          const float den = (m == -INFINITY) ? 0.f : l + exp2f(a.sink[r] * kLog2e - m);
          inv_s[r] = den > 0.f ? 1.f / den : 0.f;
        } else {
          float* part = a.ws + ((int64_t)it.row * a.n_splits + it.split) * (2 * kH + kH * kD);
          part[r] = (m == -INFINITY) ? -INFINITY : m * 0.6931471805599453f;  // natural-log units
          part[kH + r] = l;
        }
      }
      named_bar(1, 128);
      float cs = 1.f, sn = 0.f;
      const int R = a.R;
#pragma unroll 1
      for (int c = 0; c < 4; ++c) {
        const int d = 128 * c + r;
        const bool rot = final_out && d >= kD - R;
        if (rot) rope_cos_sin(it.pos, (d - (kD - R)) >> 1, R, a.rope_base, &cs, &sn);
#pragma unroll 1
        for (int half = 0; half < 2; ++half) {
          float v[32];
          tmem_ld32(t_lane + 128u + 64u * c + 32u * half, v);
          tmem_ld_wait();
          if (final_out) {
            uint16_t* orow = a.out + (int64_t)it.row * kH * kD;
#pragma unroll
            for (int i = 0; i < 32; ++i) {
              const int h = 32 * half + i;
              float x = v[i] * inv_s[h];
              const float y = __shfl_xor_sync(0xffffffffu, x, 1);
              if (rot) {
                // rotation by -pos: even dim (x, y) -> x cos + y sin; odd
                // dim (y, x) -> -y sin + x cos
                x = (d & 1) ? (x * cs - y * sn) : (x * cs + y * sn);
              }
              orow[h * kD + d] = f2bf(x);
            }
          } else {
            float* part = a.ws + ((int64_t)it.row * a.n_splits + it.split) * (2 * kH + kH * kD);
#pragma unroll
            for (int i = 0; i < 32; ++i) part[2 * kH + (32 * half + i) * kD + d] = v[i];
          }
        }
      }
      tc_fence_before();
      mbar_arrive(bar(kEpiDone));
      ++active;
    }
  } else if (warp == kMmaWarp) {
    // =================== MMA issuer ===================
    uint32_t gt = 0, active = 0;
    for (int w = blockIdx.x; w < n_items; w += gridDim.x) {
      const Item it = make_item(a, w);
      if (it.n_tiles == 0) continue;
      if (lane == 0) {
        mbar_wait(bar(kQFull), active & 1u, abort_flag, err);
        tc_fence_after();
        for (int tile = 0; tile < it.n_tiles; ++tile, ++gt) {
          const uint32_t sb = gt & 1u;
          for (int c = 0; c < 4; ++c) {
            mbar_wait(bar(kKVFull0 + c), gt & 1u, abort_flag, err);
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
              const uint32_t blk = 2u * c + (kk >> 2);
              const uint32_t koff = (uint32_t)(kk & 3) * 32u;
              const uint64_t ad = sdesc_sw128(kv_base + blk * 16384u + koff, 16, 1024);
              const uint64_t bd = sdesc_sw128(q_base + blk * 8192u + koff, 16, 1024);
              mma_bf16(tmem + sb * 64u, ad, bd, kIdescQK, (c | kk) != 0);
            }
          }
          mma_commit(bar(kSFull));
          if (tile == it.n_tiles - 1) mma_commit(bar(kQEmpty));
          mbar_wait(bar(kPFull), gt & 1u, abort_flag, err);
          if (tile == 0 && active > 0) mbar_wait(bar(kEpiDone), (active - 1) & 1u, abort_flag, err);
          tc_fence_after();
          for (int c = 0; c < 4; ++c) {
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
              const uint64_t ad = sdesc_sw128(kv_base + 2u * c * 16384u + kk * 2048u, 16384, 1024);
              const uint64_t bd = sdesc_sw128(p_base + kk * 2048u, 16384, 1024);
              mma_bf16(tmem + 128u + 64u * c, ad, bd, kIdescPV, !(tile == 0 && kk == 0));
            }
            mma_commit(bar(kKVEmpty0 + c));
          }
          mma_commit(bar(kPVDone));
        }
      }
      __syncwarp();
      ++active;
    }
    if (lane == 0) {
      // drain: every MMA issued has finished before the block exits
      mma_commit(bar(kDrain));
      mbar_wait(bar(kDrain), 0, abort_flag, err);
    }
    __syncwarp();
  } else {
    // =================== producers ===================
    const int pt = tid - kPG0;  // 0..127
    const int pw = pt >> 5;     // producer warp 0..3
    uint32_t gt = 0, active = 0;
    // RMSNorm gain of this lane's 16 dims
    float g[16];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      g[i] = a.q_norm_g[8 * lane + i];
      g[8 + i] = a.q_norm_g[256 + 8 * lane + i];
    }
    for (int w = blockIdx.x; w < n_items; w += gridDim.x) {
      const Item it = make_item(a, w);
      if (it.n_tiles == 0) continue;
      // ---- q^ = RoPE_pos(RMSNorm(q) * g) into the K-major swizzled tile ----
      if (active > 0) mbar_wait(bar(kQEmpty), (active - 1) & 1u, abort_flag, err);
      float qc[4], qs[4];  // cos/sin of this lane's rope pairs (dims 256+8l ..)
#pragma unroll
      for (int pr = 0; pr < 4; ++pr) {
        qc[pr] = 1.f;
        qs[pr] = 0.f;
        const int d = 256 + 8 * lane + 2 * pr;
        if (d >= kD - a.R) rope_cos_sin(it.pos, (d - (kD - a.R)) >> 1, a.R, a.rope_base, &qc[pr], &qs[pr]);
      }
      const uint16_t* qrow = a.q + (int64_t)it.row * kH * kD;
#pragma unroll 1
      for (int h8 = 0; h8 < 16; h8 += 8) {
        // issue the 16 loads of 8 heads before using any of them
        uint4 va[8], vb[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const int h = pw * 16 + h8 + u;
          va[u] = *reinterpret_cast<const uint4*>(qrow + h * kD + 8 * lane);
          vb[u] = *reinterpret_cast<const uint4*>(qrow + h * kD + 256 + 8 * lane);
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const int h = pw * 16 + h8 + u;
          float x[16];
          const unsigned int wa[4] = {va[u].x, va[u].y, va[u].z, va[u].w};
          const unsigned int wb[4] = {vb[u].x, vb[u].y, vb[u].z, vb[u].w};
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const float2 fa = bf2x2_to_f2(wa[q]), fb = bf2x2_to_f2(wb[q]);
            x[2 * q] = fa.x;
            x[2 * q + 1] = fa.y;
            x[8 + 2 * q] = fb.x;
            x[8 + 2 * q + 1] = fb.y;
          }
          float ss = 0.f;
#pragma unroll
          for (int i = 0; i < 16; ++i) ss += x[i] * x[i];
          ss = warp_sum(ss);
          const float rstd = rsqrtf(ss / (float)kD + a.eps);
#pragma unroll
          for (int i = 0; i < 16; ++i) x[i] = x[i] * rstd * g[i];
#pragma unroll
          for (int pr = 0; pr < 4; ++pr) {
            const float x0 = x[8 + 2 * pr], x1 = x[8 + 2 * pr + 1];
            x[8 + 2 * pr] = x0 * qc[pr] - x1 * qs[pr];
            x[8 + 2 * pr + 1] = x0 * qs[pr] + x1 * qc[pr];
          }
          // dims 8l..8l+7 -> block l/8, chunk l%8; dims 256+8l.. -> block 4+l/8
          const uint32_t cA = q_base + (uint32_t)(lane >> 3) * 8192u + sw128(h, lane & 7);
          const uint32_t cB = q_base + (uint32_t)(4 + (lane >> 3)) * 8192u + sw128(h, lane & 7);
          st_shared16(cA, f2_to_bf2x2(x[0], x[1]), f2_to_bf2x2(x[2], x[3]), f2_to_bf2x2(x[4], x[5]),
                      f2_to_bf2x2(x[6], x[7]));
          st_shared16(cB, f2_to_bf2x2(x[8], x[9]), f2_to_bf2x2(x[10], x[11]),
                      f2_to_bf2x2(x[12], x[13]), f2_to_bf2x2(x[14], x[15]));
        }
      }
      fence_async_smem();
      mbar_arrive(bar(kQFull));
      // ---- K=V tiles ----
      for (int tile = 0; tile < it.n_tiles; ++tile, ++gt) {
        named_bar(2, 128);  // every producer is done with the previous row pointers
        {
          bool bad = false;
          const uint16_t* p = key_ptr(a, it, it.j0 + tile * kKT + pt, &bad);
          if (bad) raise_err(err, DS4A_DEV_BAD_INDEX);
          rowptr[pt] = p;
        }
        named_bar(2, 128);
        const int piece = pt & 15;  // 16-byte piece of the 256-byte chunk row
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
          if (gt > 0) mbar_wait(bar(kKVEmpty0 + c), (gt - 1) & 1u, abort_flag, err);
          const uint32_t blk = kv_base + (uint32_t)(2 * c + (piece >> 3)) * 16384u;
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const int row = (pt >> 4) + 8 * i;
            const uint16_t* src = rowptr[row];
            const uint32_t dst = blk + sw128(row, piece & 7);
            if (src) cp_async16(dst, src + c * 128 + piece * 8);
            else st_shared_zero16(dst);
          }
          cp_async_commit();
          if (c > 0) {
            cp_async_wait<1>();
            fence_async_smem();
            mbar_arrive(bar(kKVFull0 + c - 1));
          }
        }
        cp_async_wait<0>();
        fence_async_smem();
        mbar_arrive(bar(kKVFull0 + 3));
      }
      ++active;
    }
    cp_async_wait<0>();
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kMmaWarp) tmem_dealloc(tmem, 512);
}

}  // namespace

// Splits of the key range per query for the tensor-core path: enough work
// items to cover the SMs, whole tiles of 128 keys per split.
static int tc_splits(int rows, int keys_max) {
  if (rows >= 148) return 1;
  const int tiles = max(1, (keys_max + kKT - 1) / kKT);
  return max(1, min(tiles, 148 / max(1, rows)));
}

bool attend_tc_supported(const AttendArgs& a) {
  return a.H == kH && a.D == kD && a.R >= 0 && a.R <= 128 && (a.R % 2) == 0;
}

int attend_tc_splits(int B, int T_q, int keys_max) { return tc_splits(B * T_q, keys_max); }

cudaError_t launch_attend_tc(const AttendArgs& a0, cudaStream_t s) {
  AttendArgs a = a0;
  const int rows = a.B * a.T_q;
  if (rows <= 0) return cudaSuccess;
  static int cache[16];
  cudaError_t e = ensure_smem(attend_tc_kernel, (int)kSmemBytes, cache);
  if (e != cudaSuccess) return e;
  const int n_items = rows * a.n_splits;
  const int grid = min(n_items, 148);
  {
    TraceScope tr("attend_tc", s);
    attend_tc_kernel<<<grid, kThreads, kSmemBytes, s>>>(a, n_items);
  }
  e = cudaGetLastError();
  if (e != cudaSuccess || a.n_splits == 1) return e;
  return launch_attend_combine(a, s);
}

}  // namespace ds4a
