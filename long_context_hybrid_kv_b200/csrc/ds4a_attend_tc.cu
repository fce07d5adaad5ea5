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
// Thread block (one per SM, 416 threads):
//   warps 0-7  softmax + epilogue: two warps per TMEM lane quarter, each
//              with 32 of the 64 head columns; thread = key row of S^T,
//              later dim row of O^T; online softmax with a lazy rescale
//              (O^T is rescaled only when a head's running max grows by
//              more than 2^8), P^T to shared memory as bf16, final
//              normalisation with the sink, de-rotation of the rope slice
//              by -pos, stores straight from registers.
//   warp 8     TMEM allocation; lane 0 issues every tcgen05.mma / commit.
//   warps 9-12 producers: the query's 64 heads x 512 by eight TMA tile
//              loads straight into the operand layout (K-major, 128-byte
//              swizzle), normalised and rotated in place (q^ =
//              RoPE_pos(RMSNorm(q) * g)) while the previous item finishes;
//              then the KV rows by cp.async, one 128-dim chunk (32 KB) at a
//              time, each chunk released by the PV products that read it.
// Decode-sized launches (kCompact) prepare q^ in the softmax warps instead,
// before waiting for the preceding kernels.
// Work items are (query, key split) pairs taken round-robin by the blocks;
// with one split the block writes the final bf16 output, otherwise the
// float partials (max, sum, accumulator) the combine kernel merges.
#include "ds4a_mx.cuh"
#include "ds4a_tc.cuh"

namespace ds4a {
namespace {

using namespace tc;

constexpr int kH = 64;
constexpr int kD = 512;
constexpr int kKT = 128;              // keys per tile
constexpr int kThreads = 416;
constexpr int kMmaWarp = 8;
constexpr int kPG0 = 288;             // first producer thread (warps 9-12)
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRescaleLog2 = 8.0f;  // lazy-rescale threshold (log2 units)
// running reference of a head that has seen no key yet: finite, so that
// logit - reference never meets (-inf) - (-inf), and far below any logit
constexpr float kNoRef = -1e30f;

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
constexpr uint32_t kOffSink = kOffInv + 256;        // [64] sink * log2(e)
constexpr uint32_t kOffNext = kOffSink + 256;       // the softmax warps' next work item
constexpr uint32_t kOffValid = kOffNext + 64;       // [2 tiles][128 keys] validity flags
constexpr uint32_t kOffG = kOffValid + 256;        // [512] query RMSNorm gains (prefill form)
constexpr uint32_t kOffRope = kOffG + 2048;         // [<= 64] (cos, sin) of the item's position
// FP8 pools: codes of dims 384..447 staged per row, each row's 16-byte
// scale run
constexpr uint32_t kOffRstd = kOffRope + 512;       // [64] 1 / RMS of each head of the query (prefill form)
constexpr uint32_t kOffStage3 = kOffRstd + 256;     // [128 keys][64 B]
constexpr uint32_t kOffScale = kOffStage3 + 8192;   // [128 keys][16 B]
constexpr uint32_t kSmemBytes = kOffRstd + 256 + 1024;     // bf16 pools (+ alignment slack)
constexpr uint32_t kSmemBytes8 = kOffScale + 2048 + 1024;  // FP8 pools
constexpr int kRow8 = 592;                          // bytes of a mixed FP8 / BF16 row (D 512, R 64)
constexpr int kNope8 = 448;                         // FP8 dims of a row

enum Bar {
  kQFull = 0, kQEmpty, kKVFull0, kKVFull1, kKVFull2, kKVFull3, kKVEmpty0, kKVEmpty1, kKVEmpty2,
  kKVEmpty3, kSFull, kPFull, kPVDone, kEpiDone, kDrain, kQRaw, kNumBars
};

constexpr uint32_t kIdescQK = idesc_bf16(128, 64, 0, 0);
constexpr uint32_t kIdescPV = idesc_bf16(128, 64, 1, 1);

// Key slots of an item: its selected (or, for HCA, visible) entries, then
// the window rows.
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
  it.idx_row = a.sparse ? a.idx + (int64_t)it.row * a.k : nullptr;
  // the index loads go out together with the position load: building an
  // item costs one memory round trip
  int n_sel = 0;
  if (a.sparse) {
    // selected entries come first (ascending, -1 padded): count them with
    // independent loads, 16 per lane in flight
    const int lane = threadIdx.x & 31;
    int cnt = 0;
    for (int base = 0; base < a.k; base += 512) {
      int v[16];
#pragma unroll
      for (int u = 0; u < 16; ++u) {
        const int j = base + 32 * u + lane;
        v[u] = j < a.k ? it.idx_row[j] : -1;
      }
#pragma unroll
      for (int u = 0; u < 16; ++u) cnt += v[u] >= 0;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) cnt += __shfl_xor_sync(0xffffffffu, cnt, o);
    n_sel = cnt;
  }
  it.pos = a.q_pos[it.row];
  if (it.pos < 0) {
    it.n_sel = 0;
    it.win_start = 0;
    it.j0 = it.j1 = 0;
    it.n_tiles = 0;
    return it;
  }
  if (!a.sparse) n_sel = min((it.pos + 1) / a.m, a.N_c);
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
template <bool kFp8>
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
    if (kFp8)  // a mixed FP8 / BF16 row, addressed in bytes
      return reinterpret_cast<const uint16_t*>(a.pool8 + ((int64_t)it.b * a.pool_bstride + e) * kRow8);
    return a.pool + (int64_t)it.b * a.pool_bstride + (int64_t)e * kD;
  }
  const int p = it.win_start + (j - it.n_sel);
  return a.win + (int64_t)it.b * a.win_bstride + (int64_t)(p % a.win_cap) * kD;
}


// kCompact: the issue loops (MMAs, gathers) stay rolled.  A decode block
// runs each of them once with its code fetched cold, and the rolled loop is
// a few cache lines instead of a few hundred instructions; a prefill block
// runs them per tile with the code warm and keeps them unrolled.
// kvmap: the pool as rows of 512 bf16 (box 64 dims x 128 rows, 128-byte
// swizzle) for the dense key ranges of HCA: a tile of 128 consecutive pool
// entries comes in as eight TMA tile loads instead of 2048 gathered
// 16-byte copies (pool_rows_b = rows per sequence; dense = 0: not used).
struct DenseKV {
  int dense;
  int64_t pool_rows_b;
};

template <bool kCompact, bool kFp8>
__global__ void __launch_bounds__(kThreads, 1)
    attend_tc_kernel(const __grid_constant__ CUtensorMap kvmap, DenseKV dkv, AttendArgs a, int n_items,
                     const __grid_constant__ CUtensorMap qmap, const __grid_constant__ CUtensorMap omap) {
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
  float* sink_s = reinterpret_cast<float*>(smem + kOffSink);
  // validity of each key slot of the last two tiles (written by the
  // producers with the row pointers, read by the softmax warps once the
  // tile's rows have landed)
  uint8_t* vflag = smem + kOffValid;

  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;

  if (tid == 0) {
    *abort_flag = 0;
    // decode-sized launches (kCompact): the softmax warps prepare q^ in the
    // kernel and all 256 arrive; otherwise one bulk copy of the prepared
    // image arrives with its bytes
    mbar_init(bar(kQFull), kCompact ? 256 : 128);
    mbar_init(bar(kQEmpty), 1);
    mbar_init(bar(kQRaw), 1);
    for (int c = 0; c < 4; ++c) {
      mbar_init(bar(kKVFull0 + c), 128);
      mbar_init(bar(kKVEmpty0 + c), 1);
    }
    mbar_init(bar(kSFull), 1);
    mbar_init(bar(kPFull), 256);
    mbar_init(bar(kPVDone), 1);
    mbar_init(bar(kEpiDone), 256);
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
  pdl_trigger();
  // the softmax warps of a decode-sized launch wait after preparing q^
  if (!kCompact || warp >= 8) pdl_wait();

  if (warp < 8) {
    // =================== softmax + epilogue (8 warps) ===================
    // warp w reads TMEM lane quarter w % 4 (its 32 key rows of S^T, later
    // 32 dim rows of O^T) and the 32 head columns of half w / 4
    const int q4 = warp & 3, hf = warp >> 2;
    const int r = 32 * q4 + lane;  // key row of S^T / dim row of O^T within a chunk
    const int st = tid;            // 0..255
    const int h0 = 32 * hf;
    const uint32_t t_lane = tmem + ((uint32_t)(32 * q4) << 16);
    const float scale2 = a.scale * kLog2e;
    if (st < kH) sink_s[st] = a.sink[st] * kLog2e;  // read by the epilogues (after a named barrier)
    if (kCompact) {
      // q^ = RoPE_pos(RMSNorm(q) * g) of this block's (only) query, straight
      // into the operand layout before the wait for the preceding kernels:
      // it reads only the query, its position and the weights, none of
      // which a preceding kernel of the chain writes.  Warp w takes heads
      // w, w + 8, ..., four heads' rows in flight per round; lane l holds
      // dims 8l..8l+7 and 256+8l..256+8l+7
      if ((int)blockIdx.x < n_items) {
        const int row = (int)blockIdx.x / a.n_splits;
        const int pos = a.q_pos[row];
        const uint16_t* qrow = a.q + (int64_t)row * kH * kD;
        float rc[4], rs[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          rc[u] = 1.f;
          rs[u] = 0.f;
          const int d = 256 + 8 * lane + 2 * u;
          if (d >= kD - a.R) rope_cos_sin(pos, a.rope.t[(d - (kD - a.R)) >> 1], &rc[u], &rs[u]);
        }
        const float4 g0 = *reinterpret_cast<const float4*>(a.q_norm_g + 8 * lane);
        const float4 g1 = *reinterpret_cast<const float4*>(a.q_norm_g + 8 * lane + 4);
        const float4 g2 = *reinterpret_cast<const float4*>(a.q_norm_g + 256 + 8 * lane);
        const float4 g3 = *reinterpret_cast<const float4*>(a.q_norm_g + 256 + 8 * lane + 4);
        const float g[16] = {g0.x, g0.y, g0.z, g0.w, g1.x, g1.y, g1.z, g1.w,
                             g2.x, g2.y, g2.z, g2.w, g3.x, g3.y, g3.z, g3.w};
        const uint32_t offA = (uint32_t)(lane >> 3) * 8192u, offB = (uint32_t)(4 + (lane >> 3)) * 8192u;
#pragma unroll 1
        for (int h4 = warp; h4 < kH; h4 += 32) {
          uint4 va[4], vb[4];
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const uint16_t* hp = qrow + (h4 + 8 * u) * kD;
            va[u] = *reinterpret_cast<const uint4*>(hp + 8 * lane);
            vb[u] = *reinterpret_cast<const uint4*>(hp + 256 + 8 * lane);
          }
          float ss[4];
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const unsigned int wv[8] = {va[u].x, va[u].y, va[u].z, va[u].w, vb[u].x, vb[u].y, vb[u].z, vb[u].w};
            float acc = 0.f;
#pragma unroll
            for (int q = 0; q < 8; ++q) {
              const float2 f = bf2x2_to_f2(wv[q]);
              acc = fmaf(f.x, f.x, fmaf(f.y, f.y, acc));
            }
            ss[u] = acc;
          }
#pragma unroll
          for (int o = 16; o > 0; o >>= 1)
#pragma unroll
            for (int u = 0; u < 4; ++u) ss[u] += __shfl_xor_sync(0xffffffffu, ss[u], o);
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const int h = h4 + 8 * u;
            const float rstd = rsqrtf(ss[u] / (float)kD + a.eps);
            const unsigned int wv[8] = {va[u].x, va[u].y, va[u].z, va[u].w, vb[u].x, vb[u].y, vb[u].z, vb[u].w};
            uint32_t pq[8];
#pragma unroll
            for (int q = 0; q < 8; ++q) {
              const float2 f = bf2x2_to_f2(wv[q]);
              float x0 = f.x * rstd * g[2 * q], x1 = f.y * rstd * g[2 * q + 1];
              if (q >= 4) {
                const float y0 = x0 * rc[q - 4] - x1 * rs[q - 4], y1 = x0 * rs[q - 4] + x1 * rc[q - 4];
                x0 = y0;
                x1 = y1;
              }
              pq[q] = f2_to_bf2x2(x0, x1);
            }
            const uint32_t sw = sw128((uint32_t)h, (uint32_t)(lane & 7));
            st_shared16(q_base + offA + sw, pq[0], pq[1], pq[2], pq[3]);
            st_shared16(q_base + offB + sw, pq[4], pq[5], pq[6], pq[7]);
          }
        }
        fence_async_smem();
        mbar_arrive(bar(kQFull));
      }
      pdl_wait();
    }
    // Warp 0 builds the next work item during the current item's last tile
    // (its loads overlap the wait for S^T) and leaves it in shared memory;
    // every softmax thread picks it up after the epilogue's last barrier.
    Item* s_next = reinterpret_cast<Item*>(smem + kOffNext);
    uint32_t gt = 0, active = 0;
    Item it;
    if (!kCompact && (int)blockIdx.x < n_items) it = make_item(a, blockIdx.x);
    for (int w = blockIdx.x; w < n_items; w += gridDim.x) {
      const int wn = w + (int)gridDim.x;
      if (kCompact) it = make_item(a, w);  // one item per block
      else if (w != (int)blockIdx.x) it = *s_next;
      const bool final_out = a.n_splits == 1;
      if (it.pos < 0 && st == 0 && it.split == 0) raise_err(err, DS4A_DEV_BAD_POS);
      if (it.n_tiles == 0) {
        // no keys in this item: output 0, or an empty partial
        if (final_out) {
          if (it.pos >= 0)
            for (int e = st; e < kH * kD / 8; e += 256)
              reinterpret_cast<uint4*>(a.out + (int64_t)it.row * kH * kD)[e] = make_uint4(0, 0, 0, 0);
        } else {
          float* part = a.ws + ((int64_t)it.row * a.n_splits + it.split) * (2 * kH + kH * kD);
          if (st < kH) {
            part[st] = -INFINITY;
            part[kH + st] = 0.f;
          }
          for (int e = st; e < kH * kD; e += 256) part[2 * kH + e] = 0.f;
        }
        if (!kCompact && wn < n_items) {
          named_bar(1, 256);  // every softmax thread has read *s_next
          if (warp == 0) {
            const Item nx = make_item(a, wn);
            if (lane == 0) *s_next = nx;
          }
          named_bar(1, 256);
        }
        continue;
      }
      if (st < kH) mrun[st] = kNoRef;
      float lpart[32];
#pragma unroll
      for (int i = 0; i < 32; ++i) lpart[i] = 0.f;
      named_bar(1, 256);
      for (int tile = 0; tile < it.n_tiles; ++tile, ++gt) {
        const uint32_t sb = gt & 1u;
        if (!kCompact && tile == it.n_tiles - 1 && warp == 0 && wn < n_items) {
          const Item nx = make_item(a, wn);
          if (lane == 0) *s_next = nx;
        }
        mbar_wait(bar(kSFull), gt & 1u, abort_flag, err);
        // the last chunk's barrier (complete before S^T is) orders the
        // producers' validity flags of this tile before the read
        mbar_wait(bar(kKVFull0 + 3), gt & 1u, abort_flag, err);
        tc_fence_after();
        // a key slot without a row (zero-filled, so its S^T row is 0) gets
        // -inf through the bias of the scaling FMA
        const float zbias = vflag[(gt & 1u) * kKT + r] != 0 ? 0.f : -INFINITY;
        float z[32];
        tmem_ld32(t_lane + sb * 64u + (uint32_t)h0, z);
        tmem_ld_wait();
        // largest lead of a logit over its head's reference (pairs of
        // columns per instruction)
        float lead = -INFINITY;
        const float4* mrun4 = reinterpret_cast<const float4*>(mrun + h0);  // broadcast, 16 B per read
        const float2 sc2 = make_float2(scale2, scale2), zb2 = make_float2(zbias, zbias);
#pragma unroll
        for (int i4 = 0; i4 < 8; ++i4) {
          const float4 m4 = mrun4[i4];
          const float2 za = fma_f2(make_float2(z[4 * i4], z[4 * i4 + 1]), sc2, zb2);
          const float2 zc = fma_f2(make_float2(z[4 * i4 + 2], z[4 * i4 + 3]), sc2, zb2);
          z[4 * i4] = za.x;
          z[4 * i4 + 1] = za.y;
          z[4 * i4 + 2] = zc.x;
          z[4 * i4 + 3] = zc.y;
          const float2 da = sub_f2(za, make_float2(m4.x, m4.y)), dc = sub_f2(zc, make_float2(m4.z, m4.w));
          lead = fmaxf(lead, fmaxf(fmaxf(da.x, da.y), fmaxf(dc.x, dc.y)));
        }
        const bool over = lead > kRescaleLog2;
        // the running reference moves (and O^T is rescaled) only when some
        // head's logit passes it by more than 2^8: one barrier-reduction
        // decides whether the tile maximum is needed at all
        const bool rescale = bar_or(1, 256, over);
        if (rescale) {
          red[q4 * 64 + h0 + lane] = warp_reduce32<true>(z);
          named_bar(1, 256);
          if (st < kH) {
            const float mt = fmaxf(fmaxf(red[st], red[64 + st]), fmaxf(red[128 + st], red[192 + st]));
            const float mo = mrun[st];
            float al = 1.f;
            if (mt > mo + kRescaleLog2) {  // a -inf tile maximum never moves it
              al = exp2f(mo - mt);               // 0 from the no-key reference
              mrun[st] = mt;
            }
            alpha_s[st] = al;
          }
          named_bar(1, 256);
          const float4* al4 = reinterpret_cast<const float4*>(alpha_s + h0);
#pragma unroll
          for (int i4 = 0; i4 < 8; ++i4) {
            const float4 a4 = al4[i4];
            const float2 la = mul_f2(make_float2(lpart[4 * i4], lpart[4 * i4 + 1]), make_float2(a4.x, a4.y));
            const float2 lc = mul_f2(make_float2(lpart[4 * i4 + 2], lpart[4 * i4 + 3]), make_float2(a4.z, a4.w));
            lpart[4 * i4] = la.x;
            lpart[4 * i4 + 1] = la.y;
            lpart[4 * i4 + 2] = lc.x;
            lpart[4 * i4 + 3] = lc.y;
          }
        }
        uint32_t pk[16];
#pragma unroll
        for (int i = 0; i < 32; i += 2) {
          const float2 m2 = reinterpret_cast<const float2*>(mrun + h0)[i >> 1];
          // a -inf logit gives 2^-inf = 0 (the reference is always finite)
          const float2 d = sub_f2(make_float2(z[i], z[i + 1]), m2);
          const uint32_t w2 = f2_to_bf2x2(ex2_approx(d.x), ex2_approx(d.y));
          pk[i >> 1] = w2;
          const float2 l2 = add_f2(make_float2(lpart[i], lpart[i + 1]), bf2x2_to_f2(w2));
          lpart[i] = l2.x;
          lpart[i + 1] = l2.y;
        }
        if (tile > 0) {
          // the previous tile's PV must be done before P^T and O^T change
          mbar_wait(bar(kPVDone), (gt - 1) & 1u, abort_flag, err);
          tc_fence_after();
        }
        // P^T row r, heads h0 .. h0+31: 64 B = chunks 4 hf .. 4 hf + 3 of the
        // 128-byte swizzled row (written before the O^T rescale, so that the
        // packed probabilities are not live across it)
#pragma unroll
        for (int cc = 0; cc < 4; ++cc)
          st_shared16(p_base + sw128(r, 4 * hf + cc), pk[4 * cc], pk[4 * cc + 1], pk[4 * cc + 2],
                      pk[4 * cc + 3]);
        if (tile > 0 && rescale) {
          const float4* al4 = reinterpret_cast<const float4*>(alpha_s + h0);
#pragma unroll 1
          for (int c = 0; c < 8; ++c) {
            // 16 head columns of one 128-dim chunk at a time
            float v[16];
            const uint32_t addr = t_lane + 128u + 64u * (c >> 1) + (uint32_t)h0 + 16u * (c & 1);
            tmem_ld16(addr, v);
            tmem_ld_wait();
#pragma unroll
            for (int i4 = 0; i4 < 4; ++i4) {
              const float4 a4 = al4[4 * (c & 1) + i4];
              v[4 * i4] *= a4.x;
              v[4 * i4 + 1] *= a4.y;
              v[4 * i4 + 2] *= a4.z;
              v[4 * i4 + 3] *= a4.w;
            }
            tmem_st16(addr, v);
          }
          tmem_st_wait();
        }
        fence_async_smem();
        tc_fence_before();
        mbar_arrive(bar(kPFull));
      }
      // ---------------- epilogue ----------------
      mbar_wait(bar(kPVDone), (gt - 1) & 1u, abort_flag, err);
      tc_fence_after();
      if (warp == 0 && w + (int)gridDim.x < n_items) {
        // the next item's position and indices into L1 while this one's
        // output goes out (its make_item then hits L1)
        const int rn = (w + (int)gridDim.x) / a.n_splits;
        if (lane < 16 && a.sparse && 32 * lane < a.k) prefetch_l1(a.idx + (int64_t)rn * a.k + 32 * lane);
        if (lane == 16) prefetch_l1(a.q_pos + rn);
      }
      red[q4 * 64 + h0 + lane] = warp_reduce32<false>(lpart);
      named_bar(1, 256);
      if (st < kH) {
        const float l = red[st] + red[64 + st] + red[128 + st] + red[192 + st];
        const float m = mrun[st];
        if (final_out) {
          const float den = (m <= kNoRef) ? 0.f : l + exp2f(sink_s[st] - m);
          inv_s[st] = den > 0.f ? 1.f / den : 0.f;
        } else {
          float* part = a.ws + ((int64_t)it.row * a.n_splits + it.split) * (2 * kH + kH * kD);
          part[st] = (m <= kNoRef) ? -INFINITY : m * 0.6931471805599453f;  // natural-log units
          part[kH + st] = l;
        }
      }
      named_bar(1, 256);
      float cs = 1.f, sn = 0.f;
      const int R = a.R;
      // The final output goes out one 128-dim chunk at a time through the
      // P^T buffer (free: the item's PV products are done) as two 64-head x
      // 64-dim boxes (128-byte swizzle) that one thread stores by TMA, so the
      // warps do not wait on the global writes; split partials go straight
      // from registers to global memory as coalesced 128-byte rows.
      const bool odd = r & 1;
#pragma unroll 1
      for (int c = 0; c < 4; ++c) {
        const int d = 128 * c + r;
        const bool rot = final_out && d >= kD - R;
        if (rot) rope_cos_sin(it.pos, a.rope.t[(d - (kD - R)) >> 1], &cs, &sn);
        float v[32];
        tmem_ld32(t_lane + 128u + 64u * c + (uint32_t)h0, v);
        tmem_ld_wait();
        if (final_out) {
          if (c > 0) {
            if (st == 0) bulk_wait_read0();  // the previous chunk's boxes have been read
            named_bar(1, 256);
          }
          // lanes r and r^1 hold dims d and d^1: one exchange per head pair
          // gives the even lane both dims of the even head and the odd lane
          // both dims of the odd head, so each lane rotates its pair (rope
          // slice, by -pos) and writes one 4-byte word of the box
          const uint32_t dd = (uint32_t)(r & 62);  // the pair's first dim within its box
          const uint32_t box = p_base + (uint32_t)(r >> 6) * 8192u;
#pragma unroll
          for (int i = 0; i < 32; i += 2) {
            const float got = __shfl_xor_sync(0xffffffffu, odd ? v[i] : v[i + 1], 1);
            const int h = h0 + i + (odd ? 1 : 0);
            const float s = inv_s[h];
            float2 x = mul_f2(make_float2(odd ? got : v[i], odd ? v[i + 1] : got), make_float2(s, s));
            if (rot)  // (x0 cs + x1 sn, -x0 sn + x1 cs)
              x = fma_f2(make_float2(x.x, x.x), make_float2(cs, -sn), mul_f2(make_float2(x.y, x.y), make_float2(sn, cs)));
            st_shared32(box + (uint32_t)h * 128u + ((((dd >> 3) ^ (uint32_t)(h & 7))) << 4) + (dd & 7u) * 2u,
                        f2_to_bf2x2(x.x, x.y));
          }
          fence_async_smem();
          named_bar(1, 256);
          if (st == 0) {
            tma_store_2d(&omap, 128 * c, it.row * kH, p_base);
            tma_store_2d(&omap, 128 * c + 64, it.row * kH, p_base + 8192u);
            bulk_commit();
          }
        } else {
          float* part = a.ws + ((int64_t)it.row * a.n_splits + it.split) * (2 * kH + kH * kD);
#pragma unroll
          for (int i = 0; i < 32; ++i) part[2 * kH + (h0 + i) * kD + d] = v[i];
        }
      }
      if (final_out) {
        // the boxes have been read before the next item's P^T goes in
        if (st == 0) bulk_wait_read0();
        named_bar(1, 256);
      }
      tc_fence_before();
      mbar_arrive(bar(kEpiDone));
      ++active;
      if (!kCompact && wn < n_items) named_bar(1, 256);  // *s_next is written
    }
  } else if (warp == kMmaWarp) {
    // =================== MMA issuer ===================
    // Descriptors are built once; every product adds a compile-time offset
    // (the start-address field holds addr >> 4 and stays below 2^14), so the
    // issue loop is an add and the MMA per step.
    const uint64_t qk_a0 = sdesc_sw128(kv_base, 16, 1024);
    const uint64_t qk_b0 = sdesc_sw128(q_base, 16, 1024);
    const uint64_t pv_a0 = sdesc_sw128(kv_base, 16384, 1024);
    const uint64_t pv_b0 = sdesc_sw128(p_base, 16384, 1024);
    uint32_t gt = 0, active = 0;
    for (int w = blockIdx.x; w < n_items; w += gridDim.x) {
      const Item it = make_item(a, w);
      if (it.n_tiles == 0) continue;
      if (lane == 0) {
        mbar_wait(bar(kQFull), active & 1u, abort_flag, err);
        tc_fence_after();
        for (int tile = 0; tile < it.n_tiles; ++tile, ++gt) {
          const uint32_t d_s = tmem + (gt & 1u) * 64u;
#pragma unroll(kCompact ? 1 : 4)
          for (int c = 0; c < 4; ++c) {
            mbar_wait(bar(kKVFull0 + c), gt & 1u, abort_flag, err);
            tc_fence_after();
#pragma unroll(kCompact ? 2 : 8)
            for (int kk = 0; kk < 8; ++kk) {
              const uint32_t blk = 2u * c + (kk >> 2);
              const uint32_t koff = (uint32_t)(kk & 3) * 32u;
              mma_bf16(d_s, qk_a0 + ((blk * 16384u + koff) >> 4), qk_b0 + ((blk * 8192u + koff) >> 4),
                       kIdescQK, (c | kk) != 0 ? 1u : 0u);
            }
          }
          mma_commit(bar(kSFull));
          if (tile == it.n_tiles - 1) mma_commit(bar(kQEmpty));
          mbar_wait(bar(kPFull), gt & 1u, abort_flag, err);
          if (tile == 0 && active > 0) mbar_wait(bar(kEpiDone), (active - 1) & 1u, abort_flag, err);
          tc_fence_after();
          const uint32_t acc0 = tile == 0 ? 0u : 1u;
#pragma unroll(kCompact ? 1 : 4)
          for (int c = 0; c < 4; ++c) {
#pragma unroll(kCompact ? 2 : 8)
            for (int kk = 0; kk < 8; ++kk)
              mma_bf16(tmem + 128u + 64u * c, pv_a0 + ((2u * c * 16384u + kk * 2048u) >> 4),
                       pv_b0 + ((kk * 2048u) >> 4), kIdescPV, kk == 0 ? acc0 : 1u);
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
    uint32_t gt = 0, active = 0, q_loads = 0;
    bool tma_used = false;
    if (!kCompact) {
      float* gs = reinterpret_cast<float*>(smem + kOffG);
      for (int d = pt; d < kD; d += 128) gs[d] = a.q_norm_g[d];
      named_bar(2, 128);
    }
    for (int w = blockIdx.x; w < n_items; w += gridDim.x) {
      const Item it = make_item(a, w);
      if (it.n_tiles == 0) continue;
      const int piece = pt & 15;  // 16-byte piece of the 256-byte chunk row
      // row pointers of a tile (every producer is done with the previous ones)
      auto set_rowptr = [&](int tile) {
        named_bar(2, 128);
        bool bad = false;
        const int j = it.j0 + tile * kKT + pt;
        const uint16_t* p = key_ptr<kFp8>(a, it, j, &bad);
        if (bad) raise_err(err, DS4A_DEV_BAD_INDEX);
        rowptr[pt] = p;
        // 0: no row (zero-filled); 1: bf16 row; 2: FP8 pool row
        vflag[(gt & 1u) * kKT + pt] = p == nullptr ? 0 : (kFp8 && j < it.n_sel ? 2 : 1);
        named_bar(2, 128);
      };
      // FP8 pools: chunk c of the tile.  bf16 rows (the window) and missing
      // rows go as in issue_chunk; an FP8 row's codes of dims 128c .. 128c+127
      // land in the row's own 128 bytes of block 2c+1 (chunks 0-2) or in the
      // stage-3 area (chunk 3: dims 384..447), its RoPE dims 448..511 straight
      // into block 7, its 16-byte scale run (chunk 0) in the scale area
      auto issue_chunk8 = [&](int c) {
        if (gt > 0) mbar_wait(bar(kKVEmpty0 + c), (gt - 1) & 1u, abort_flag, err);
        const uint32_t blk = kv_base + (uint32_t)(2 * c + (piece >> 3)) * 16384u;
        for (int i = 0; i < 16; ++i) {
          const int row = (pt >> 4) + 8 * i;
          const uint16_t* src = rowptr[row];
          const uint8_t vf = vflag[(gt & 1u) * kKT + row];
          const uint32_t dst = blk + sw128(row, piece & 7);
          if (vf == 1) {
            cp_async16(dst, src + c * 128 + piece * 8);
          } else if (vf == 0) {
            st_shared_zero16(dst);
          } else {
            const uint8_t* r8 = reinterpret_cast<const uint8_t*>(src);
            if (c < 3) {
              if (piece < 8)
                cp_async16(kv_base + (uint32_t)(2 * c + 1) * 16384u + row * 128u + piece * 16u, r8 + c * 128 + piece * 16);
            } else if (piece < 4) {
              cp_async16(sbase + kOffStage3 + row * 64u + piece * 16u, r8 + 384 + piece * 16);
            } else if (piece >= 8) {
              cp_async16(dst, r8 + kNope8 + (piece - 8) * 16);  // RoPE dims, bf16
            }
            if (c == 0 && piece == 15) cp_async16(sbase + kOffScale + row * 16u, r8 + kNope8 + 128);
          }
        }
        cp_async_commit();
      };
      // every producer's copies of chunk c have landed: thread pt expands its
      // own FP8 row to bf16 (code value times the block's scale, exact)
      auto convert_chunk8 = [&](int c) {
        named_bar(2, 128);
        if (vflag[(gt & 1u) * kKT + pt] != 2) return;
        const unsigned char* stg = c < 3 ? smem + kOffKV + (2 * c + 1) * 16384 + pt * 128 : smem + kOffStage3 + pt * 64;
        const uint32_t sc4 = *reinterpret_cast<const uint32_t*>(smem + kOffScale + pt * 16 + 4 * c);
        // 16 codes = dims 128c + 16q .. + 15 (one scale block per two q) ->
        // the 8-dim pieces 2q, 2q + 1 of the chunk
        auto expand = [&](int q, const uint4 cw) {
          const float sc = mx_scale((int)((sc4 >> (8 * (q >> 1))) & 255u));
          const uint32_t wd[4] = {cw.x, cw.y, cw.z, cw.w};
          uint32_t o[8];
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            const float2 v = mul_f2(e4m3x2_to_f2(wd[k >> 1] >> (16 * (k & 1))), make_float2(sc, sc));
            o[k] = f2_to_bf2x2(v.x, v.y);
          }
          const int p0 = 2 * q;
          const uint32_t b0 = kv_base + (uint32_t)(2 * c + (p0 >> 3)) * 16384u;
          st_shared16(b0 + sw128(pt, p0 & 7), o[0], o[1], o[2], o[3]);
          st_shared16(b0 + sw128(pt, (p0 + 1) & 7), o[4], o[5], o[6], o[7]);
        };
        if (c == 3) {  // dims 384..447 from the stage-3 area into block 6
#pragma unroll 1
          for (int q = 0; q < 4; ++q) expand(q, reinterpret_cast<const uint4*>(stg)[q]);
          return;
        }
        // the row's staged codes sit in its own bytes of block 2c+1: the
        // upper half (q = 4..7, written into block 2c+1) is read first, the
        // lower half is expanded into block 2c, then the upper half
        uint4 hi[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) hi[q] = reinterpret_cast<const uint4*>(stg)[4 + q];
#pragma unroll 1
        for (int q = 0; q < 4; ++q) expand(q, reinterpret_cast<const uint4*>(stg)[q]);
#pragma unroll
        for (int q = 0; q < 4; ++q) expand(4 + q, hi[q]);
      };
      // one 128-dim chunk of the tile: 128 rows x 256 B, 16 cp.async each;
      // rows past the key list or with a bad index are zero-filled
      auto issue_chunk = [&](int c) {
        if (gt > 0) mbar_wait(bar(kKVEmpty0 + c), (gt - 1) & 1u, abort_flag, err);
        const uint32_t blk = kv_base + (uint32_t)(2 * c + (piece >> 3)) * 16384u;
#pragma unroll(kCompact ? 4 : 16)
        for (int i = 0; i < 16; ++i) {
          const int row = (pt >> 4) + 8 * i;
          const uint16_t* src = rowptr[row];
          const uint32_t dst = blk + sw128(row, piece & 7);
          if (src) cp_async16(dst, src + c * 128 + piece * 8);
          else st_shared_zero16(dst);
        }
        cp_async_commit();
      };
      // ---- q^ (prefill form): once the previous item's QK products are
      // done, eight TMA tile loads bring the query's 64 heads x 512 into
      // the operand layout (blocks of 64 dims, 128-byte swizzle); the
      // producers normalise and rotate it in place (prep_qhat) after they
      // have sent out the first two chunks of the item's first tile, so that
      // the transform overlaps those copies ----
      if (!kCompact) {
        named_bar(2, 128);  // every producer is done with the previous item's q^ and angles
        if (pt == 0 && w + (int)gridDim.x < n_items) {
          // the next item's query into L2 now, so that its TMA loads (issued
          // when this item's last QK is done) come from L2
          const int rn = (w + (int)gridDim.x) / a.n_splits;
          prefetch_l2_bulk(a.q + (int64_t)rn * kH * kD, (uint32_t)(kH * kD * 2));
        }
        if (pt == 0) {
          if (active > 0) mbar_wait(bar(kQEmpty), (active - 1) & 1u, abort_flag, err);
          mbar_expect_tx(bar(kQRaw), 65536u);
#pragma unroll 1
          for (int blk = 0; blk < 8; ++blk)
            tma_load_2d(q_base + (uint32_t)blk * 8192u, &qmap, blk * 64, it.row * kH, bar(kQRaw));
          q_loads = active + 1;
        }
        float2* rope_w = reinterpret_cast<float2*>(smem + kOffRope);
        if (pt < a.R / 2) {
          float cs, sn;
          rope_cos_sin(it.pos, a.rope.t[pt], &cs, &sn);
          rope_w[pt] = make_float2(cs, sn);
        }
      }
      float2* rope_s = reinterpret_cast<float2*>(smem + kOffRope);
      float* rstd_s = reinterpret_cast<float*>(smem + kOffRstd);
      auto prep_qhat = [&]() {
        mbar_wait(bar(kQRaw), active & 1u, abort_flag, err);
        named_bar(2, 128);
        // RMS: thread pt takes head pt / 2, dims 256 (pt & 1) .. + 255
        // (blocks 4 (pt & 1) .. + 3), and adds its partner lane's half
        {
          const int h = pt >> 1, half = pt & 1;
          // eight 16-byte reads in flight, four independent sums
          float s4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 1
          for (int q0 = 0; q0 < 32; q0 += 8) {
            uint4 v[8];
#pragma unroll
            for (int u = 0; u < 8; ++u)
              v[u] = *reinterpret_cast<const uint4*>(smem + kOffQ + (4 * half + ((q0 + u) >> 3)) * 8192 +
                                                     sw128((uint32_t)h, (uint32_t)((q0 + u) & 7)));
#pragma unroll
            for (int u = 0; u < 8; ++u) {
              const unsigned int wv[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
#pragma unroll
              for (int k = 0; k < 4; ++k) {
                const float2 f = bf2x2_to_f2(wv[k]);
                s4[k] = fmaf(f.x, f.x, fmaf(f.y, f.y, s4[k]));
              }
            }
          }
          float ss = (s4[0] + s4[1]) + (s4[2] + s4[3]);
          ss += __shfl_xor_sync(0xffffffffu, ss, 1);
          if (half == 0) rstd_s[h] = rsqrtf(ss / (float)kD + a.eps);
        }
        named_bar(2, 128);
        // normalise and rotate in place: thread pt takes the 8-dim piece
        // j = pt % 64 of every other head (pt / 64, + 2, ...), so its gains
        // and angles stay in registers; a warp's 32 pieces of one head are
        // 512 contiguous bytes of the row (no bank conflict)
        {
          const int j = pt & 63, hs = pt >> 6;
          const float* gs = reinterpret_cast<const float*>(smem + kOffG);
          const float4 ga = *reinterpret_cast<const float4*>(gs + 8 * j);
          const float4 gb = *reinterpret_cast<const float4*>(gs + 8 * j + 4);
          const float g8[8] = {ga.x, ga.y, ga.z, ga.w, gb.x, gb.y, gb.z, gb.w};
          const int R = a.R;
          float2 cs4[4];
          bool rot[4];
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const int d = 8 * j + 2 * k;
            rot[k] = d >= kD - R;
            cs4[k] = rot[k] ? rope_s[(d - (kD - R)) >> 1] : make_float2(1.f, 0.f);
          }
          const uint32_t pbase = kOffQ + (uint32_t)(j >> 3) * 8192u;
#pragma unroll 4
          for (int i = 0; i < 32; ++i) {
            const int h = hs + 2 * i;
            unsigned char* p = smem + pbase + sw128((uint32_t)h, (uint32_t)(j & 7));
            const uint4 v = *reinterpret_cast<const uint4*>(p);
            const float rs = rstd_s[h];
            const unsigned int wv[4] = {v.x, v.y, v.z, v.w};
            uint32_t o[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              const float2 f = bf2x2_to_f2(wv[k]);
              float x0 = f.x * rs * g8[2 * k], x1 = f.y * rs * g8[2 * k + 1];
              if (rot[k]) {
                const float y0 = x0 * cs4[k].x - x1 * cs4[k].y, y1 = x0 * cs4[k].y + x1 * cs4[k].x;
                x0 = y0;
                x1 = y1;
              }
              o[k] = f2_to_bf2x2(x0, x1);
            }
            *reinterpret_cast<uint4*>(p) = make_uint4(o[0], o[1], o[2], o[3]);
          }
        }
        fence_async_smem();
        mbar_arrive(bar(kQFull));
      };
      // ---- K=V tiles: each chunk goes out when the PV products of the
      // previous tile have released it ----
      // Two chunks stay in flight: chunk c goes out, then chunk c-1 is
      // retired (a deeper queue over-subscribes L2 across the SMs).
      for (int tile = 0; tile < it.n_tiles; ++tile, ++gt) {
        const int s0 = it.j0 + tile * kKT;
        if (dkv.dense && !a.sparse && s0 + kKT <= it.n_sel) {
          // 128 consecutive pool entries: one thread arms each chunk's
          // barrier with its bytes and starts two TMA tile loads, the
          // others arrive
          const int y = (int)(it.b * dkv.pool_rows_b + s0);
          vflag[(gt & 1u) * kKT + pt] = 1;  // 128 entries inside the visible range
#pragma unroll 1
          for (int c = 0; c < 4; ++c) {
            if (gt > 0) mbar_wait(bar(kKVEmpty0 + c), (gt - 1) & 1u, abort_flag, err);
            if (pt == 0) {
              mbar_expect_tx(bar(kKVFull0 + c), 32768u);
              tma_load_2d(kv_base + (uint32_t)(2 * c) * 16384u, &kvmap, 128 * c, y, bar(kKVFull0 + c));
              tma_load_2d(kv_base + (uint32_t)(2 * c + 1) * 16384u, &kvmap, 128 * c + 64, y, bar(kKVFull0 + c));
              tma_used = true;
            } else {
              mbar_arrive(bar(kKVFull0 + c));
            }
          }
          if (!kCompact && tile == 0) prep_qhat();
          continue;
        }
        set_rowptr(tile);
        if (kFp8) {
#pragma unroll 1
          for (int c = 0; c < 4; ++c) {
            issue_chunk8(c);
            if (!kCompact && tile == 0 && c == 1) prep_qhat();
            if (c > 0) {
              cp_async_wait<1>();
              convert_chunk8(c - 1);
              fence_async_smem();
              mbar_arrive(bar(kKVFull0 + c - 1));
            }
          }
          cp_async_wait<0>();
          convert_chunk8(3);
          fence_async_smem();
          mbar_arrive(bar(kKVFull0 + 3));
          continue;
        }
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
          issue_chunk(c);
          if (!kCompact && tile == 0 && c == 1) prep_qhat();
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
    cp_async_wait<0>();  // nothing of this block is in flight at exit
    if (pt == 0 && tma_used)
      for (int c = 0; c < 4; ++c) mbar_drain(bar(kKVFull0 + c), (gt - 1) & 1u);
    if (pt == 0 && q_loads > 0) mbar_drain(bar(kQRaw), (q_loads - 1) & 1u);
  }

  if (tid == 0) bulk_wait0();  // the output stores have completed
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
  const int n_items = rows * a.n_splits;
  const bool compact = n_items <= 148;  // every block takes at most one item
  static std::atomic<int> cache[kMaxDevices], cache_c[kMaxDevices], cache8[kMaxDevices], cache8c[kMaxDevices];
  const bool fp8 = a.pool8 != nullptr;
  cudaError_t e = fp8 ? (compact ? ensure_smem(attend_tc_kernel<true, true>, (int)kSmemBytes8, cache8c)
                                 : ensure_smem(attend_tc_kernel<false, true>, (int)kSmemBytes8, cache8))
                      : (compact ? ensure_smem(attend_tc_kernel<true, false>, (int)kSmemBytes, cache_c)
                                 : ensure_smem(attend_tc_kernel<false, false>, (int)kSmemBytes, cache));
  if (e != cudaSuccess) return e;
  PFN_cuTensorMapEncodeTiled_v12000 encode = get_encode();
  if (!encode) return cudaErrorNotSupported;
  // the queries as rows of 512 (one per head), for the prefill form's TMA
  // loads into the operand layout
  CUtensorMap qmap;
  {
    const cuuint64_t dims[2] = {(cuuint64_t)kD, (cuuint64_t)rows * kH};
    const cuuint64_t strides[1] = {(cuuint64_t)kD * 2};
    const cuuint32_t box[2] = {64, (cuuint32_t)kH};
    const cuuint32_t estr[2] = {1, 1};
    if (encode(&qmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<uint16_t*>(a.q), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  // the output as rows of 512 (one per head), for the final output's TMA
  // stores (64 heads x 64 dims boxes)
  CUtensorMap omap;
  {
    const cuuint64_t dims[2] = {(cuuint64_t)kD, (cuuint64_t)rows * kH};
    const cuuint64_t strides[1] = {(cuuint64_t)kD * 2};
    const cuuint32_t box[2] = {64, (cuuint32_t)kH};
    const cuuint32_t estr[2] = {1, 1};
    if (encode(&omap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, a.out, dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  // HCA keys are consecutive pool entries: a row view of the pool for TMA
  // tile loads (when the sequences are a whole number of rows apart)
  CUtensorMap kvmap;
  memset(&kvmap, 0, sizeof(kvmap));
  DenseKV dkv;
  dkv.dense = 0;
  dkv.pool_rows_b = a.B > 1 ? a.pool_bstride / kD : 0;
  const int64_t pool_rows = (int64_t)(a.B - 1) * dkv.pool_rows_b + a.N_c;
  if (!a.pool8 && !a.sparse && a.N_c >= kKT && (a.B == 1 || a.pool_bstride % kD == 0) && pool_rows < INT32_MAX) {
    const cuuint64_t dims[2] = {(cuuint64_t)kD, (cuuint64_t)pool_rows};
    const cuuint64_t strides[1] = {(cuuint64_t)kD * 2};
    const cuuint32_t box[2] = {64, (cuuint32_t)kKT};
    const cuuint32_t estr[2] = {1, 1};
    if (encode(&kvmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<uint16_t*>(a.pool), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
    dkv.dense = 1;
  }
  const int grid = min(n_items, 148);
  {
    TraceScope tr("attend_tc", s);
    if (fp8)
      e = compact ? launch_pdl(attend_tc_kernel<true, true>, dim3(grid), dim3(kThreads), kSmemBytes8, s, kvmap, dkv,
                               a, n_items, qmap, omap)
                  : launch_pdl(attend_tc_kernel<false, true>, dim3(grid), dim3(kThreads), kSmemBytes8, s, kvmap, dkv,
                               a, n_items, qmap, omap);
    else
      e = compact ? launch_pdl(attend_tc_kernel<true, false>, dim3(grid), dim3(kThreads), kSmemBytes, s, kvmap, dkv,
                               a, n_items, qmap, omap)
                  : launch_pdl(attend_tc_kernel<false, false>, dim3(grid), dim3(kThreads), kSmemBytes, s, kvmap,
                               dkv, a, n_items, qmap, omap);
  }
  if (e != cudaSuccess || a.n_splits == 1) return e;
  return launch_attend_combine(a, s);
}

}  // namespace ds4a
