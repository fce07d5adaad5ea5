// Shape-generic CUDA kernels of the ds4a path: the KV compressor, the
// indexer score (CUDA-core form), the split attention (CUDA-core form) and
// its combine (the top-k selector is in ds4a_topk.cu).  They serve every
// shape the ABI accepts (the toy widths included); the Flash-0731 shapes
// take the tensor-core kernels of ds4a_index_tc.cu / ds4a_attend_tc.cu
// where those apply.
#include "ds4a_internal.cuh"
#include "ds4a_mx.cuh"

#include <cooperative_groups.h>
#include <float.h>

namespace ds4a {

// ===========================================================================
// KV compressor ("DeepSeek-v4 Beyond Basics" 3.2.2 eqs. 9-12 and 3.3
// eqs. 20-23): per channel, a softmax over the 2m (CSA) or m (HCA) logits
// Z + B weights the matching C values; then RMSNorm * g and RoPE at i*m.
// One thread block per (entry, sequence).  Thread t owns channels
// [V*(t % NC), V*(t % NC) + V) (NC = c/V) and the terms g, g+G, ... of the
// entry (g = t / NC, G = 512 / NC), four terms' loads in flight at a time;
// the G partial softmaxes merge in shared memory.  Loads are 16-byte
// vectors of 8 bf16 when c is a multiple of 8.
// ===========================================================================
constexpr int kCompressThreads = 512;
constexpr float kLog2eC = 1.4426950408889634f;

template <int V>
struct VecLoad;
template <>
struct VecLoad<8> {  // 8 bf16 = 16 bytes
  __device__ static void load(const uint16_t* p, float* out) {
    const uint4 v = *reinterpret_cast<const uint4*>(p);
    const unsigned int w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const float2 f = bf2x2_to_f2(w[u]);
      out[2 * u] = f.x;
      out[2 * u + 1] = f.y;
    }
  }
  __device__ static void load_f(const float* p, float* out) {
    const float4 a = *reinterpret_cast<const float4*>(p);
    const float4 b = *reinterpret_cast<const float4*>(p + 4);
    out[0] = a.x; out[1] = a.y; out[2] = a.z; out[3] = a.w;
    out[4] = b.x; out[5] = b.y; out[6] = b.z; out[7] = b.w;
  }
};
template <>
struct VecLoad<2> {  // 2 bf16 = 4 bytes
  __device__ static void load(const uint16_t* p, float* out) {
    const float2 f = bf2x2_to_f2(*reinterpret_cast<const unsigned int*>(p));
    out[0] = f.x;
    out[1] = f.y;
  }
  __device__ static void load_f(const float* p, float* out) {
    const float2 a = *reinterpret_cast<const float2*>(p);
    out[0] = a.x;
    out[1] = a.y;
  }
};

// Row of one stream (C or Z of half a or b) for token tok of sequence b:
// the caller's streams in range mode; in append mode the new token's input
// row or the ring slot of an earlier token.
__device__ __forceinline__ const uint16_t* term_row(const CompressArgs& a, bool half_a, bool is_z, int b,
                                                    int tok, int newtok) {
  const uint16_t* src = half_a ? (is_z ? a.za : a.ca) : (is_z ? a.zb : a.cb);
  if (a.app_pos == nullptr) return src + ((int64_t)b * a.T_tok + (tok - a.tok_begin)) * a.c;
  if (tok == newtok) return src + (int64_t)b * a.c;
  const bool overlap = a.cb != nullptr;
  const int S = overlap ? 4 : 2;
  const int st = overlap ? (is_z ? 2 : 0) + (half_a ? 0 : 1) : (is_z ? 1 : 0);
  return a.ring + (((int64_t)b * S + st) * a.ring_cap + (tok % a.ring_cap)) * a.c;
}

// Append mode: the entry that sequence b's new token (position p) closes,
// or -1 (no entry closes, a bad position, or an entry past the pool).
__device__ __forceinline__ int closing_entry(const CompressArgs& a, int p, bool report) {
  if (p < 0) {
    if (report) raise_err(a.err, DS4A_DEV_BAD_POS);
    return -1;
  }
  if ((p + 1) % a.m != 0) return -1;
  const int i = (p + 1) / a.m - 1;
  if (i >= a.n_cap) {
    if (report) raise_err(a.err, DS4A_DEV_BAD_INDEX);
    return -1;
  }
  return i;
}

// Append mode: store the new token's rows of every stream (position p >= 0)
// in its ring slot (threads tid0, tid0 + nthr, ... of the block; 16-byte
// pieces when c is a multiple of 8).  The pooling of the entry the token
// closes reads the token's rows from the inputs, not from the ring, so the
// store may come after it.
__device__ __forceinline__ void append_token(const CompressArgs& a, int b, int p, int tid0, int nthr) {
  const bool overlap = a.cb != nullptr;
  const int S = overlap ? 4 : 2;
  const uint16_t* srcs[4] = {a.ca, overlap ? a.cb : a.za, a.za, a.zb};
  const int slot = p % a.ring_cap;
  if (a.c % 8 == 0) {
    const int pieces = a.c / 8;
    for (int k = tid0; k < S * pieces; k += nthr) {
      const int st = k / pieces, q = k % pieces;
      const uint4 v = reinterpret_cast<const uint4*>(srcs[st] + (int64_t)b * a.c)[q];
      reinterpret_cast<uint4*>(a.ring + (((int64_t)b * S + st) * a.ring_cap + slot) * a.c)[q] = v;
    }
  } else {
    for (int k = tid0; k < S * a.c; k += nthr) {
      const int st = k / a.c, q = k % a.c;
      a.ring[(((int64_t)b * S + st) * a.ring_cap + slot) * a.c + q] = srcs[st][(int64_t)b * a.c + q];
    }
  }
}

// Store channels (ch, ch + 1) of entry i of sequence b: as bf16 at dst, or
// (qfmt != 0) rounded to bf16 and then block-quantised (ds4a_mx.cuh).  In
// the block-scaled case every lane of the warp calls it, the warp holding 64
// consecutive channels that start at a multiple of 64 (two 32-channel
// blocks, one per half-warp).
__device__ __forceinline__ void store_entry_pair(const CompressArgs& a, int b, int i, int ch, float x0, float x1,
                                                 uint16_t* dst) {
  const unsigned int packed = f2_to_bf2x2(x0, x1);
  if (a.qfmt == 0) {
    *reinterpret_cast<unsigned int*>(dst) = packed;
    return;
  }
  const float2 v = bf2x2_to_f2(packed);
  float amax = fmaxf(fabsf(v.x), fabsf(v.y));
#pragma unroll
  for (int o = 1; o < 16; o <<= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  const bool lead = (threadIdx.x & 15) == 0;
  if (a.qfmt == 1) {
    uint8_t* row = a.qpool + (int64_t)b * a.q_bstride + (int64_t)i * a.q_row;
    const int R = a.rope_dim, n = a.c - R;
    if (ch >= n) {  // RoPE dims stay bf16
      *reinterpret_cast<unsigned int*>(row + n + 2 * (ch - n)) = packed;
      return;
    }
    const int code = mx_scale_code<false>(amax);
    const float inv = mx_inv_scale(code);
    *reinterpret_cast<uint16_t*>(row + ch) = to_e4m3x2(v.x * inv, v.y * inv);
    if (lead) row[n + 2 * R + ch / kMxBlock] = (uint8_t)code;
    if (ch == 0)
      for (int k = n + 2 * R + n / kMxBlock; k < (int)a.q_row; ++k) row[k] = 0;
  } else {
    uint8_t* row = a.qpool + (int64_t)b * a.q_bstride + (int64_t)i * (a.c / 2);
    const int code = mx_scale_code<true>(amax);
    const float inv = mx_inv_scale(code);
    row[ch / 2] = (uint8_t)to_e2m1x2(v.x * inv, v.y * inv);
    if (lead) a.qscales[(int64_t)b * a.qs_bstride + (int64_t)i * (a.c / kMxBlock) + ch / kMxBlock] = (uint8_t)code;
  }
}

// Short entries (CSA: m = 4, at most 16 terms) of up to 512 channels, a
// multiple of 64 (the K=V entries' 512, the indexer keys' 128), one
// 256-thread block per entry: thread p < c / 2 pools channels 2p, 2p + 1
// over all of the entry's terms with every load in flight at once, so no
// partial softmaxes are merged; the block adds the RMSNorm sum of squares.
// Warp w holds channels 64w .. 64w + 63 (a whole run for the block-scaled
// store).  The softmax takes the exact maximum of the (at most 16) logits
// first.
constexpr int kShortC = 512, kShortTerms = 16, kShortThreads = kShortC / 2;

__device__ __forceinline__ void compress_short(const CompressArgs& a) {
  const int c = a.c;
  const int m = a.m, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, b = blockIdx.y;
  const bool overlap = a.cb != nullptr;
  __shared__ float s_red_short[kShortThreads / 32];
  pdl_trigger();
  int i = a.entry_begin + blockIdx.x, newtok = -1;
  if (a.app_pos != nullptr) {
    pdl_wait();
    newtok = a.app_pos[b];
    i = closing_entry(a, newtok, tid == 0);
    if (i < 0) {
      if (newtok >= 0) append_token(a, b, newtok, tid, kShortThreads);
      return;
    }
  }
  const int n_terms = (overlap && i >= 1) ? 2 * m : m;
  const int ch = 2 * tid;
  float v0 = 0.f, v1 = 0.f, ss = 0.f;
  if (ch < c) {
    float x0[kShortTerms], x1[kShortTerms], c0[kShortTerms], c1[kShortTerms];
    float M0 = -INFINITY, M1 = -INFINITY;
#pragma unroll
    for (int t = 0; t < kShortTerms; ++t) {
      x0[t] = x1[t] = -INFINITY;
      c0[t] = c1[t] = 0.f;
      if (t < n_terms) {
        const bool half_a = t < m;
        const int r = half_a ? t : t - m;
        const int tok = half_a ? i * m + r : (i - 1) * m + r;
        const float2 cf = bf2x2_to_f2(*reinterpret_cast<const unsigned int*>(term_row(a, half_a, false, b, tok, newtok) + ch));
        const float2 zf = bf2x2_to_f2(*reinterpret_cast<const unsigned int*>(term_row(a, half_a, true, b, tok, newtok) + ch));
        const float2 bb = *reinterpret_cast<const float2*>((half_a ? a.bias_a : a.bias_b) + (int64_t)r * c + ch);
        x0[t] = (zf.x + bb.x) * kLog2eC;
        x1[t] = (zf.y + bb.y) * kLog2eC;
        c0[t] = cf.x;
        c1[t] = cf.y;
        M0 = fmaxf(M0, x0[t]);
        M1 = fmaxf(M1, x1[t]);
      }
    }
    float l0 = 0.f, l1 = 0.f, a0 = 0.f, a1 = 0.f;
#pragma unroll
    for (int t = 0; t < kShortTerms; ++t) {
      if (t < n_terms) {
        const float e0 = ex2_approx(x0[t] - M0), e1 = ex2_approx(x1[t] - M1);
        l0 += e0;
        l1 += e1;
        a0 = fmaf(e0, c0[t], a0);
        a1 = fmaf(e1, c1[t], a1);
      }
    }
    v0 = a0 / l0;
    v1 = a1 / l1;
    ss = v0 * v0 + v1 * v1;
  }
  // the token's rows into the ring (after the entry's term loads)
  if (a.app_pos != nullptr) append_token(a, b, newtok, tid, kShortThreads);
  float tot = 0.f;
  if (a.norm_g != nullptr) {
    ss = warp_sum(ss);
    if (lane == 0) s_red_short[warp] = ss;
    __syncthreads();
#pragma unroll
    for (int w = 0; w < kShortThreads / 32; ++w) tot += s_red_short[w];
  }
  if (a.app_pos == nullptr) pdl_wait();  // a preceding kernel may still read the entry this one overwrites
  if (ch >= c) return;
  uint16_t* dst = a.qfmt ? nullptr : a.pool + (int64_t)b * a.pool_bstride + (int64_t)i * c + ch;
  if (a.norm_g == nullptr) {
    store_entry_pair(a, b, i, ch, v0, v1, dst);
    return;
  }
  const float rstd = rsqrtf(tot / (float)c + a.eps);
  const int R = a.rope_dim;
  float x0 = v0 * rstd * a.norm_g[ch];
  float x1 = v1 * rstd * a.norm_g[ch + 1];
  if (ch >= c - R) {
    float cs, sn;
    rope_cos_sin(i * m, a.rope.t[(ch - (c - R)) >> 1], &cs, &sn);
    const float y0 = x0 * cs - x1 * sn;
    const float y1 = x0 * sn + x1 * cs;
    x0 = y0;
    x1 = y1;
  }
  store_entry_pair(a, b, i, ch, x0, x1, dst);
}

__global__ void __launch_bounds__(kShortThreads) compress_short_kernel(const __grid_constant__ CompressArgs a) {
  compress_short(a);
}

template <int V>
__device__ __forceinline__ void compress_body(const CompressArgs& a) {
  extern __shared__ float csm[];
  const int c = a.c, m = a.m;
  const int NC = c / V;
  const int G = kCompressThreads / NC;
  const int tid = threadIdx.x;
  const int cc = tid % NC;
  const int g = tid / NC;
  const int b = blockIdx.y;
  const bool overlap = a.cb != nullptr;
  pdl_trigger();
  // The C/Z rows, gate biases and norm weights are inputs that no kernel of
  // the chain writes: the pooling runs while the preceding kernel finishes,
  // and only the pool write waits for it (a preceding kernel may still read
  // the entry this one overwrites).  In append mode the ring was written by
  // an earlier call, so everything waits.
  int i = a.entry_begin + blockIdx.x, newtok = -1;
  if (a.app_pos != nullptr) {
    pdl_wait();
    newtok = a.app_pos[b];
    i = closing_entry(a, newtok, tid == 0);
    if (i < 0) {
      if (newtok >= 0) append_token(a, b, newtok, tid, kCompressThreads);
      return;
    }
  }
  const int n_terms = (overlap && i >= 1) ? 2 * m : m;

  float mx[V], l[V], acc[V];
#pragma unroll
  for (int u = 0; u < V; ++u) { mx[u] = -INFINITY; l[u] = 0.f; acc[u] = 0.f; }

  if (g < G) {
    for (int t0 = g; t0 < n_terms; t0 += 4 * G) {
      float vals[4][V], zs[4][V], bs[4][V];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int term = t0 + u * G;
        if (term < n_terms) {
          const bool half_a = term < m;
          const int r = half_a ? term : term - m;
          const int tok = half_a ? i * m + r : (i - 1) * m + r;
          VecLoad<V>::load(term_row(a, half_a, false, b, tok, newtok) + cc * V, vals[u]);
          VecLoad<V>::load(term_row(a, half_a, true, b, tok, newtok) + cc * V, zs[u]);
          VecLoad<V>::load_f((half_a ? a.bias_a : a.bias_b) + (int64_t)r * c + cc * V, bs[u]);
        }
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        if (t0 + u * G >= n_terms) break;
#pragma unroll
        for (int q = 0; q < V; ++q) {
          // log2 units; the reference moves only when a logit passes it by
          // more than 2^8 (always for the first term), so the common step
          // is one exp2 and two FMAs
          const float x = (zs[u][q] + bs[u][q]) * kLog2eC;
          if (x > mx[q] + 8.f) {
            const float sc = ex2_approx(mx[q] - x);  // 0 while empty
            l[q] *= sc;
            acc[q] *= sc;
            mx[q] = x;
          }
          const float e = ex2_approx(x - mx[q]);
          l[q] += e;
          acc[q] = fmaf(e, vals[u][q], acc[q]);
        }
      }
    }
  }
  // the token's rows into the ring (their loads overlap the merge below)
  if (a.app_pos != nullptr) append_token(a, b, newtok, tid, kCompressThreads);
  // merge the G partials of every channel
  float* s_m = csm;                 // [G * c]
  float* s_l = s_m + G * c;         // [G * c]
  float* s_a = s_l + G * c;         // [G * c]
  float* s_v = s_a + G * c;         // [c]
  __shared__ float s_red[kCompressThreads / 32];
  if (g < G) {
#pragma unroll
    for (int u = 0; u < V; ++u) {
      s_m[g * c + cc * V + u] = mx[u];
      s_l[g * c + cc * V + u] = l[u];
      s_a[g * c + cc * V + u] = acc[u];
    }
  }
  __syncthreads();
  float ss = 0.f;
  for (int ch = tid; ch < c; ch += kCompressThreads) {
    float M = -INFINITY;
    for (int gg = 0; gg < G; ++gg) M = fmaxf(M, s_m[gg * c + ch]);
    float Ls = 0.f, A = 0.f;
    for (int gg = 0; gg < G; ++gg) {
      const float mm = s_m[gg * c + ch];
      if (mm == -INFINITY) continue;
      const float e = ex2_approx(mm - M);
      Ls += s_l[gg * c + ch] * e;
      A += s_a[gg * c + ch] * e;
    }
    const float v = A / Ls;
    s_v[ch] = v;
    ss += v * v;
  }
  pdl_wait();
  uint16_t* dst = a.qfmt ? nullptr : a.pool + (int64_t)b * a.pool_bstride + (int64_t)i * c;
  if (a.norm_g == nullptr) {
    __syncthreads();
    if (a.qfmt) {
      for (int p2 = tid; p2 < c / 2; p2 += kCompressThreads)
        store_entry_pair(a, b, i, 2 * p2, s_v[2 * p2], s_v[2 * p2 + 1], nullptr);
      return;
    }
    for (int ch = tid; ch < c; ch += kCompressThreads) dst[ch] = f2bf(s_v[ch]);
    return;
  }
  ss = warp_sum(ss);
  if ((tid & 31) == 0) s_red[tid >> 5] = ss;
  __syncthreads();
  float tot = 0.f;
#pragma unroll
  for (int w = 0; w < kCompressThreads / 32; ++w) tot += s_red[w];
  const float rstd = rsqrtf(tot / (float)c + a.eps);
  const int R = a.rope_dim;
  const int pos = i * m;
  for (int p2 = tid; p2 < c / 2; p2 += kCompressThreads) {
    const int ch = 2 * p2;
    float x0 = s_v[ch] * rstd * a.norm_g[ch];
    float x1 = s_v[ch + 1] * rstd * a.norm_g[ch + 1];
    if (ch >= c - R) {
      float cs, sn;
      rope_cos_sin(pos, a.rope.t[(ch - (c - R)) >> 1], &cs, &sn);
      const float y0 = x0 * cs - x1 * sn;
      const float y1 = x0 * sn + x1 * cs;
      x0 = y0;
      x1 = y1;
    }
    store_entry_pair(a, b, i, ch, x0, x1, dst + ch);
  }
}

template <int V>
__global__ void __launch_bounds__(kCompressThreads) compress_kernel(const __grid_constant__ CompressArgs a) {
  compress_body<V>(a);
}

// Two append-mode compressions in one launch (blockIdx.z picks the job):
// one decode step of a CSA layer's K=V and indexer-key compressors, which
// would otherwise each wait for the kernel before them.
struct CompressPair {
  CompressArgs j[2];
};
template <int V>
__global__ void __launch_bounds__(kCompressThreads) compress_pair_kernel(const __grid_constant__ CompressPair p) {
  compress_body<V>(p.j[blockIdx.z]);
}
// whether an entry shape runs in the short-entry kernel: bulk compression
// (a prefill); one entry per sequence (decode) measured faster in the
// 512-thread kernels, whose wider loads put fewer load instructions behind
// the wait for the ring
static bool short_entry(const CompressArgs& a) {
  return a.app_pos == nullptr && a.c <= kShortC && a.c % 64 == 0 && (a.cb != nullptr ? 2 * a.m : a.m) <= kShortTerms;
}

// Long entries (HCA: m' = 128 terms) when there are few of them (decode):
// the Z blocks of a cluster split one entry's terms; each block reduces its
// terms to one partial softmax per channel, then block r merges channels
// [r c/Z, (r+1) c/Z) over the cluster through distributed shared memory, the
// blocks add their RMSNorm sums of squares the same way, and each writes
// its channels.  Same arithmetic as compress_kernel (log2-unit softmax with a
// lazy reference), merged in a different order.
template <int V>
__global__ void __launch_bounds__(kCompressThreads) compress_split_kernel(CompressArgs a, int Z) {
  extern __shared__ float csm[];
  namespace cg = cooperative_groups;
  cg::cluster_group cl = cg::this_cluster();
  const int c = a.c, m = a.m;
  const int NC = c / V;
  const int G = kCompressThreads / NC;
  const int tid = threadIdx.x;
  const int cc = tid % NC;
  const int g = tid / NC;
  const int zr = (int)cl.block_rank();
  const int b = blockIdx.y;
  const bool overlap = a.cb != nullptr;
  pdl_trigger();
  // as in compress_kernel, only the pool write waits for the preceding
  // kernel, except in append mode (the ring comes from an earlier call).
  // Every block of a cluster serves the same sequence, so all of them take
  // the same early exit.
  int i = a.entry_begin + blockIdx.x / Z, newtok = -1;
  if (a.app_pos != nullptr) {
    pdl_wait();
    newtok = a.app_pos[b];
    i = closing_entry(a, newtok, zr == 0 && tid == 0);
    if (i < 0) {
      if (zr == 0 && newtok >= 0) append_token(a, b, newtok, tid, kCompressThreads);
      return;
    }
  }
  const int n_terms = (overlap && i >= 1) ? 2 * m : m;
  const int tz0 = (int)((int64_t)zr * n_terms / Z), tz1 = (int)((int64_t)(zr + 1) * n_terms / Z);

  float mx[V], l[V], acc[V];
#pragma unroll
  for (int u = 0; u < V; ++u) { mx[u] = -INFINITY; l[u] = 0.f; acc[u] = 0.f; }
  if (g < G) {
    for (int t0 = tz0 + g; t0 < tz1; t0 += 4 * G) {
      float vals[4][V], zs[4][V], bs[4][V];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int term = t0 + u * G;
        if (term < tz1) {
          const bool half_a = term < m;
          const int r = half_a ? term : term - m;
          const int tok = half_a ? i * m + r : (i - 1) * m + r;
          VecLoad<V>::load(term_row(a, half_a, false, b, tok, newtok) + cc * V, vals[u]);
          VecLoad<V>::load(term_row(a, half_a, true, b, tok, newtok) + cc * V, zs[u]);
          VecLoad<V>::load_f((half_a ? a.bias_a : a.bias_b) + (int64_t)r * c + cc * V, bs[u]);
        }
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        if (t0 + u * G >= tz1) break;
#pragma unroll
        for (int q = 0; q < V; ++q) {
          const float x = (zs[u][q] + bs[u][q]) * kLog2eC;
          if (x > mx[q] + 8.f) {
            const float sc = ex2_approx(mx[q] - x);
            l[q] *= sc;
            acc[q] *= sc;
            mx[q] = x;
          }
          const float e = ex2_approx(x - mx[q]);
          l[q] += e;
          acc[q] = fmaf(e, vals[u][q], acc[q]);
        }
      }
    }
  }
  // block 0 stores the token's rows into the ring (after its term loads)
  if (a.app_pos != nullptr && zr == 0) append_token(a, b, newtok, tid, kCompressThreads);
  // block partials: [G][c] each, then one (M, L, A) per channel
  float* s_m = csm;
  float* s_l = s_m + G * c;
  float* s_a = s_l + G * c;
  float* p_m = s_a + G * c;  // [c] this block's partial per channel
  float* p_l = p_m + c;
  float* p_a = p_l + c;
  float* s_v = p_a + c;      // [c / Z] pooled values of this block's channels
  __shared__ float s_red[kCompressThreads / 32];
  __shared__ float s_tot;
  if (g < G) {
#pragma unroll
    for (int u = 0; u < V; ++u) {
      s_m[g * c + cc * V + u] = mx[u];
      s_l[g * c + cc * V + u] = l[u];
      s_a[g * c + cc * V + u] = acc[u];
    }
  }
  __syncthreads();
  for (int ch = tid; ch < c; ch += kCompressThreads) {
    float M = -INFINITY;
    for (int gg = 0; gg < G; ++gg) M = fmaxf(M, s_m[gg * c + ch]);
    float Ls = 0.f, A = 0.f;
    if (M != -INFINITY)
      for (int gg = 0; gg < G; ++gg) {
        const float mm = s_m[gg * c + ch];
        if (mm == -INFINITY) continue;
        const float e = ex2_approx(mm - M);
        Ls += s_l[gg * c + ch] * e;
        A += s_a[gg * c + ch] * e;
      }
    p_m[ch] = M;
    p_l[ch] = Ls;
    p_a[ch] = A;
  }
  cl.sync();  // every block's partials are complete
  const int cz = c / Z, ch0 = zr * cz;
  float ss = 0.f;
  for (int k = tid; k < cz; k += kCompressThreads) {
    const int ch = ch0 + k;
    float pm[8], M = -INFINITY;
    for (int r = 0; r < Z; ++r) {
      pm[r] = cl.map_shared_rank(p_m, r)[ch];
      M = fmaxf(M, pm[r]);
    }
    float Ls = 0.f, A = 0.f;
    for (int r = 0; r < Z; ++r) {
      if (pm[r] == -INFINITY) continue;
      const float e = ex2_approx(pm[r] - M);
      Ls += cl.map_shared_rank(p_l, r)[ch] * e;
      A += cl.map_shared_rank(p_a, r)[ch] * e;
    }
    const float v = A / Ls;
    s_v[k] = v;
    ss += v * v;
  }
  pdl_wait();
  uint16_t* dst = a.qfmt ? nullptr : a.pool + (int64_t)b * a.pool_bstride + (int64_t)i * c + ch0;
  if (a.norm_g == nullptr) {
    cl.sync();  // no block leaves while a peer may still read its partials
    if (a.qfmt) {
      for (int p2 = tid; p2 < cz / 2; p2 += kCompressThreads)
        store_entry_pair(a, b, i, ch0 + 2 * p2, s_v[2 * p2], s_v[2 * p2 + 1], nullptr);
      return;
    }
    for (int k = tid; k < cz; k += kCompressThreads) dst[k] = f2bf(s_v[k]);
    return;
  }
  ss = warp_sum(ss);
  if ((tid & 31) == 0) s_red[tid >> 5] = ss;
  __syncthreads();
  if (tid == 0) {
    float t = 0.f;
    for (int w = 0; w < kCompressThreads / 32; ++w) t += s_red[w];
    s_tot = t;
  }
  cl.sync();  // partials read by every peer; every block's sum is in place
  float tot = 0.f;
  for (int r = 0; r < Z; ++r) tot += *cl.map_shared_rank(&s_tot, r);
  cl.sync();  // no block leaves while a peer may still read its sum
  const float rstd = rsqrtf(tot / (float)c + a.eps);
  const int R = a.rope_dim;
  const int pos = i * m;
  for (int p2 = tid; p2 < cz / 2; p2 += kCompressThreads) {
    const int k = 2 * p2, ch = ch0 + k;
    float x0 = s_v[k] * rstd * a.norm_g[ch];
    float x1 = s_v[k + 1] * rstd * a.norm_g[ch + 1];
    if (ch >= c - R) {
      float cs, sn;
      rope_cos_sin(pos, a.rope.t[(ch - (c - R)) >> 1], &cs, &sn);
      const float y0 = x0 * cs - x1 * sn;
      const float y1 = x0 * sn + x1 * cs;
      x0 = y0;
      x1 = y1;
    }
    store_entry_pair(a, b, i, ch, x0, x1, dst + k);
  }
}

// Long entries (HCA decode: m' = 128 terms) when there are few of them, c =
// 512: the 8 blocks of a cluster take 64 channels each over all of the
// entry's terms, so each block's pooled values are final and only the
// RMSNorm sum of squares crosses blocks (one distributed-shared-memory read
// of 8 partial sums).  256 threads, two blocks per SM (so that 32 sequences'
// entries fit the SMs at once); thread (g, cc): terms g, g + 32, ... of the
// channel vector cc (8 channels); the 32 partial softmaxes of a channel
// merge inside the warp (4 term groups) and then over the 8 warps.  Same
// arithmetic as compress_kernel (log2-unit softmax with a lazy reference),
// merged in a different order.
constexpr int kChanZ = 8, kChanC = 512, kChanCz = kChanC / kChanZ, kChanNC = kChanCz / 8, kChanThreads = 256;

// merge the partial (reference, sum, accumulator) (m2, l2, a2) into (m, l, acc)
__device__ __forceinline__ void merge_partial(float& mx, float& l, float& acc, float m2, float l2, float a2) {
  if (m2 == -INFINITY) return;
  if (mx == -INFINITY) {
    mx = m2;
    l = l2;
    acc = a2;
    return;
  }
  const float M = fmaxf(mx, m2);
  const float e1 = ex2_approx(mx - M), e2 = ex2_approx(m2 - M);
  l = l * e1 + l2 * e2;
  acc = acc * e1 + a2 * e2;
  mx = M;
}

__global__ void __cluster_dims__(kChanZ, 1, 1) __launch_bounds__(kChanThreads, 2)
    compress_chan_kernel(const __grid_constant__ CompressArgs a) {
  constexpr int V = 8, NC = kChanNC, G = kChanThreads / NC;
  namespace cg = cooperative_groups;
  cg::cluster_group cl = cg::this_cluster();
  __shared__ float s_m[kChanThreads / 32][kChanCz], s_l[kChanThreads / 32][kChanCz],
      s_a[kChanThreads / 32][kChanCz];
  __shared__ float s_v[kChanCz];
  __shared__ float s_red[kChanThreads / 32];
  __shared__ float s_tot;
  const int m = a.m, c = kChanC;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int cc = tid % NC, g = tid / NC;
  const int zr = (int)cl.block_rank();
  const int ch0 = zr * kChanCz;
  const int b = blockIdx.y;
  const bool overlap = a.cb != nullptr;
  pdl_trigger();
  // every block of a cluster serves the same entry, so all take the same
  // early exit; in append mode everything waits (the ring is a library
  // output), otherwise only the pool write does
  int i = a.entry_begin + blockIdx.x / kChanZ, newtok = -1;
  if (a.app_pos != nullptr) {
    pdl_wait();
    newtok = a.app_pos[b];
    i = closing_entry(a, newtok, zr == 0 && tid == 0);
    if (i < 0) {
      if (zr == 0 && newtok >= 0) append_token(a, b, newtok, tid, kChanThreads);
      return;
    }
  }
  const int n_terms = (overlap && i >= 1) ? 2 * m : m;
  float mx[V], l[V], acc[V];
#pragma unroll
  for (int u = 0; u < V; ++u) { mx[u] = -INFINITY; l[u] = 0.f; acc[u] = 0.f; }
  const int cv = ch0 + cc * V;
  for (int t0 = g; t0 < n_terms; t0 += 4 * G) {
    float vals[4][V], zs[4][V], bs[4][V];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int term = t0 + u * G;
      if (term < n_terms) {
        const bool half_a = term < m;
        const int r = half_a ? term : term - m;
        const int tok = half_a ? i * m + r : (i - 1) * m + r;
        VecLoad<V>::load(term_row(a, half_a, false, b, tok, newtok) + cv, vals[u]);
        VecLoad<V>::load(term_row(a, half_a, true, b, tok, newtok) + cv, zs[u]);
        VecLoad<V>::load_f((half_a ? a.bias_a : a.bias_b) + (int64_t)r * c + cv, bs[u]);
      }
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      if (t0 + u * G >= n_terms) break;
#pragma unroll
      for (int q = 0; q < V; ++q) {
        const float x = (zs[u][q] + bs[u][q]) * kLog2eC;
        if (x > mx[q] + 8.f) {
          const float sc = ex2_approx(mx[q] - x);  // 0 while empty
          l[q] *= sc;
          acc[q] *= sc;
          mx[q] = x;
        }
        const float e = ex2_approx(x - mx[q]);
        l[q] += e;
        acc[q] = fmaf(e, vals[u][q], acc[q]);
      }
    }
  }
  // block 0 stores the token's rows into the ring (after its term loads)
  if (a.app_pos != nullptr && zr == 0) append_token(a, b, newtok, tid, kChanThreads);
  // the warp's 4 term groups of each channel vector (lanes cc, cc + 8, ...)
#pragma unroll
  for (int o = NC; o < 32; o <<= 1)
#pragma unroll
    for (int q = 0; q < V; ++q) {
      const float m2 = __shfl_xor_sync(0xffffffffu, mx[q], o);
      const float l2 = __shfl_xor_sync(0xffffffffu, l[q], o);
      const float a2 = __shfl_xor_sync(0xffffffffu, acc[q], o);
      merge_partial(mx[q], l[q], acc[q], m2, l2, a2);
    }
  if (lane < NC) {
#pragma unroll
    for (int q = 0; q < V; ++q) {
      s_m[warp][cc * V + q] = mx[q];
      s_l[warp][cc * V + q] = l[q];
      s_a[warp][cc * V + q] = acc[q];
    }
  }
  __syncthreads();
  float ss = 0.f;
  if (tid < kChanCz) {
    float M = -INFINITY, Ls = 0.f, A = 0.f;
    for (int w = 0; w < kChanThreads / 32; ++w) merge_partial(M, Ls, A, s_m[w][tid], s_l[w][tid], s_a[w][tid]);
    const float v = A / Ls;
    s_v[tid] = v;
    ss = v * v;
  }
  ss = warp_sum(ss);
  if (lane == 0) s_red[warp] = ss;
  __syncthreads();
  if (tid == 0) {
    float t = 0.f;
    for (int w = 0; w < kChanThreads / 32; ++w) t += s_red[w];
    s_tot = t;
  }
  cl.sync();  // every block's sum of squares is in place
  float tot = 0.f;
#pragma unroll
  for (int r = 0; r < kChanZ; ++r) tot += *cl.map_shared_rank(&s_tot, r);
  cl.sync();  // no block leaves while a peer may still read its sum
  if (a.app_pos == nullptr) pdl_wait();
  if (warp != 0) return;
  // warp 0: the block's 64 channels as 32 pairs (a whole 64-channel run, as
  // the block-scaled store wants)
  uint16_t* dst = a.qfmt ? nullptr : a.pool + (int64_t)b * a.pool_bstride + (int64_t)i * c + ch0;
  if (a.norm_g == nullptr) {
    if (a.qfmt) store_entry_pair(a, b, i, ch0 + 2 * lane, s_v[2 * lane], s_v[2 * lane + 1], nullptr);
    else *reinterpret_cast<unsigned int*>(dst + 2 * lane) = f2_to_bf2x2(s_v[2 * lane], s_v[2 * lane + 1]);
    return;
  }
  const float rstd = rsqrtf(tot / (float)c + a.eps);
  const int R = a.rope_dim;
  const int pos = i * m;
  const int k = 2 * lane, ch = ch0 + k;
  float x0 = s_v[k] * rstd * a.norm_g[ch];
  float x1 = s_v[k + 1] * rstd * a.norm_g[ch + 1];
  if (ch >= c - R) {
    float cs, sn;
    rope_cos_sin(pos, a.rope.t[(ch - (c - R)) >> 1], &cs, &sn);
    const float y0 = x0 * cs - x1 * sn;
    const float y1 = x0 * sn + x1 * cs;
    x0 = y0;
    x1 = y1;
  }
  store_entry_pair(a, b, i, ch, x0, x1, a.qfmt ? nullptr : dst + k);
}

// whether a job runs in the one-block-per-entry kernel with 8-wide loads
static bool plain8(const CompressArgs& a) {
  const int n_terms = a.cb != nullptr ? 2 * a.m : a.m;
  return a.c % 8 == 0 && n_terms < 64;
}

cudaError_t launch_compress_jobs(const CompressArgs* jobs, int n_jobs, cudaStream_t s) {
  if (n_jobs == 2 && jobs[0].app_pos && jobs[1].app_pos && plain8(jobs[0]) && plain8(jobs[1]) &&
      jobs[0].B == jobs[1].B && jobs[0].B > 0) {
    size_t smem = 0;
    for (int j = 0; j < 2; ++j) {
      const int NC = jobs[j].c / 8;
      const int G = NC >= kCompressThreads ? 1 : kCompressThreads / NC;
      const size_t b = (size_t)(3 * G * jobs[j].c + jobs[j].c) * sizeof(float);
      smem = b > smem ? b : smem;
    }
    static std::atomic<int> cache[kMaxDevices];
    cudaError_t e = ensure_smem(compress_pair_kernel<8>, (int)smem, cache);
    if (e != cudaSuccess) return e;
    CompressPair p;
    p.j[0] = jobs[0];
    p.j[1] = jobs[1];
    TraceScope tr("compress", s);
    return launch_pdl(compress_pair_kernel<8>, dim3(1, jobs[0].B, 2), dim3(kCompressThreads), smem, s, p);
  }
  for (int j = 0; j < n_jobs; ++j) {
    const cudaError_t e = launch_compress(jobs[j], s);
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

cudaError_t launch_compress(const CompressArgs& a, cudaStream_t s) {
  // append mode: one (possible) entry per sequence
  const int n = a.app_pos != nullptr ? 1 : a.entry_end - a.entry_begin;
  if (n <= 0 || a.B <= 0) return cudaSuccess;
  const int V = (a.c % 8 == 0) ? 8 : 2;
  const int NC = a.c / V;
  const int G = NC >= kCompressThreads ? 1 : kCompressThreads / NC;
  const int n_terms = a.cb != nullptr ? 2 * a.m : a.m;
  if (short_entry(a)) {
    TraceScope tr("compress", s);
    return launch_pdl(compress_short_kernel, dim3(n, a.B), dim3(kShortThreads), 0, s, a);
  }
  // long entries of 512 channels, few of them (decode): an 8-block cluster
  // per entry, 64 channels per block
  if (V == 8 && a.c == kChanC && n_terms >= 64 && (int64_t)n * a.B <= 32) {
    TraceScope tr("compress", s);
    return launch_pdl(compress_chan_kernel, dim3(n * kChanZ, a.B), dim3(kChanThreads), 0, s, a);
  }
  // other long entries, few of them: split each entry's terms over a cluster
  int Z = 1;
  if (V == 8 && n_terms >= 64)
    while (Z < 8 && (int64_t)n * a.B * Z * 2 <= 148 && n_terms / (2 * Z) >= 16 && a.c % (2 * Z * 2) == 0) Z *= 2;
  if (Z > 1) {
    const size_t smem = (size_t)(3 * G * a.c + 3 * a.c + a.c / Z) * sizeof(float);
    static std::atomic<int> cache_s[kMaxDevices];
    cudaError_t e = ensure_smem(compress_split_kernel<8>, (int)smem, cache_s);
    if (e != cudaSuccess) return e;
    TraceScope tr("compress", s);
    return launch_pdl_cluster(compress_split_kernel<8>, dim3(n * Z, a.B), dim3(kCompressThreads), smem, s, Z, a,
                              Z);
  }
  const size_t smem = (size_t)(3 * G * a.c + a.c) * sizeof(float);
  static std::atomic<int> cache8[kMaxDevices], cache2[kMaxDevices];
  cudaError_t e = V == 8 ? ensure_smem(compress_kernel<8>, (int)smem, cache8)
                         : ensure_smem(compress_kernel<2>, (int)smem, cache2);
  if (e != cudaSuccess) return e;
  TraceScope tr("compress", s);
  return V == 8 ? launch_pdl(compress_kernel<8>, dim3(n, a.B), dim3(kCompressThreads), smem, s, a)
                : launch_pdl(compress_kernel<2>, dim3(n, a.B), dim3(kCompressThreads), smem, s, a);
}

// ===========================================================================
// Indexer score, CUDA-core form (any H_I, D_I <= 128)
// ("DeepSeek-v4 Beyond Basics" 3.2.2 eq. 16):
//   I[s] = sum_h w[h] * ReLU(q[h] . K[s])  for visible s.
// One thread per key; the key tile is staged in shared memory (stride D+1
// keeps the per-thread row reads free of bank conflicts).
// ===========================================================================
constexpr int kIdxKeys = 128;

__global__ void __launch_bounds__(kIdxKeys) index_score_generic_kernel(IndexArgs a) {
  extern __shared__ float ism[];
  const int H = a.H, D = a.D;
  float* qs = ism;              // [H * D]
  float* wsum = qs + H * D;     // [H]
  float* kt = wsum + H;         // [128 * (D + 1)]
  pdl_trigger();
  pdl_wait();
  const int row = blockIdx.x;
  const int b = row / a.T_q;
  const int pos = a.q_pos[row];
  if (pos < 0) {
    if (threadIdx.x == 0 && blockIdx.y == 0) raise_err(a.err, DS4A_DEV_BAD_POS);
    return;
  }
  const int n_vis = min((pos + 1) / a.m, a.N_c);
  const int s0 = blockIdx.y * kIdxKeys;
  if (s0 >= n_vis) return;
  for (int e = threadIdx.x; e < H * D; e += kIdxKeys) qs[e] = bf2f(a.q[(int64_t)row * H * D + e]);
  for (int e = threadIdx.x; e < H; e += kIdxKeys) wsum[e] = bf2f(a.w[(int64_t)row * H + e]);
  const int nk = min(kIdxKeys, n_vis - s0);
  const uint16_t* kb = a.kidx + (int64_t)b * a.k_bstride + (int64_t)s0 * D;
  for (int e = threadIdx.x; e < nk * D; e += kIdxKeys) kt[(e / D) * (D + 1) + (e % D)] = bf2f(kb[e]);
  __syncthreads();
  const int t = threadIdx.x;
  if (t >= nk) return;
  const float* kr = kt + t * (D + 1);
  float score = 0.f;
  for (int h = 0; h < H; ++h) {
    const float* qh = qs + h * D;
    float dot = 0.f;
    for (int d = 0; d < D; ++d) dot = fmaf(qh[d], kr[d], dot);
    score = fmaf(wsum[h], fmaxf(dot, 0.f), score);
  }
  a.scores[(int64_t)row * a.N_c + s0 + t] = score;
}

cudaError_t launch_index_scores_generic(const IndexArgs& a, cudaStream_t s) {
  const int rows = a.B * a.T_q;
  if (rows <= 0 || a.N_c <= 0) return cudaSuccess;
  const size_t smem = (size_t)(a.H * a.D + a.H + kIdxKeys * (a.D + 1)) * sizeof(float);
  static std::atomic<int> cache[kMaxDevices];
  cudaError_t e = ensure_smem(index_score_generic_kernel, (int)smem, cache);
  if (e != cudaSuccess) return e;
  TraceScope tr("index_score_generic", s);
  return launch_pdl(index_score_generic_kernel, dim3(rows, (a.N_c + kIdxKeys - 1) / kIdxKeys), dim3(kIdxKeys),
                    smem, s, a);
}

// ===========================================================================
// Attention, CUDA-core form ("DeepSeek-v4 Beyond Basics" 3.2.2 eq. 19,
// 3.3 eqs. 24-27; "DeepSeek V4 Inside" sink and window examples).
// Thread block = (split, query, sequence).  The query's key list is the
// selected (CSA) or visible (HCA) pool rows followed by the window rows;
// split s takes a contiguous range of it.  q^ = RoPE_p(RMSNorm(q) * g) is
// kept in shared memory as bf16 (the rounding the tensor-core form uses);
// logits, the running max / sum and the output accumulator are float32.
// With one split the block also finishes: divides by the sum plus
// exp(sink), rotates the rope slice back by -p and stores bf16.  With
// several, each writes (max, sum, accumulator) to the workspace and the
// combine kernel finishes.
// ===========================================================================
constexpr int kAttThreads = 256;
constexpr int kAttKT = 8;

struct KeyList {
  int n_sel, n_win, win_start;
};

__device__ __forceinline__ KeyList key_list(const AttendArgs& a, int b, int t, int pos,
                                            const int32_t* idx_row) {
  KeyList kl;
  if (a.sparse) {
    // idx rows are ascending with -1 padding at the end
    int lo = 0, hi = a.k;
    while (lo < hi) {
      const int mid = (lo + hi) >> 1;
      if (idx_row[mid] >= 0) lo = mid + 1; else hi = mid;
    }
    kl.n_sel = lo;
  } else {
    kl.n_sel = min((pos + 1) / a.m, a.N_c);
  }
  kl.win_start = max(0, pos - a.W + 1);
  kl.n_win = a.W > 0 ? pos - kl.win_start + 1 : 0;
  return kl;
}

__device__ __forceinline__ const uint16_t* key_row(const AttendArgs& a, int b, const KeyList& kl,
                                                   const int32_t* idx_row, int j, bool* ok) {
  *ok = true;
  if (j < kl.n_sel) {
    int e = a.sparse ? idx_row[j] : j;
    if (e >= a.N_c || e < 0) {
      *ok = false;
      return nullptr;
    }
    return a.pool + (int64_t)b * a.pool_bstride + (int64_t)e * a.D;
  }
  const int p = kl.win_start + (j - kl.n_sel);
  return a.win + (int64_t)b * a.win_bstride + (int64_t)(p % a.win_cap) * a.D;
}

// cos / sin of the R/2 rope pairs at position pos (float64 phase) into rt
__device__ void rope_table(const AttendArgs& a, int pos, float2* rt) {
  for (int j = threadIdx.x; j < a.R / 2; j += blockDim.x) {
    float cs, sn;
    rope_cos_sin(pos, a.rope.t[j], &cs, &sn);
    rt[j] = make_float2(cs, sn);
  }
}

// q^ = RoPE_pos(RMSNorm(q_h) * g) for all heads into shared memory (bf16)
__device__ void load_qhat(const AttendArgs& a, const uint16_t* qrow, const float2* rt, uint16_t* qh) {
  const int H = a.H, D = a.D, R = a.R;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  for (int h = warp; h < H; h += nw) {
    float ss = 0.f;
    for (int d = lane; d < D; d += 32) {
      const float x = bf2f(qrow[h * D + d]);
      ss += x * x;
    }
    ss = warp_sum(ss);
    const float rstd = rsqrtf(ss / (float)D + a.eps);
    for (int d2 = lane; d2 < D / 2; d2 += 32) {
      const int d = 2 * d2;
      float x0 = bf2f(qrow[h * D + d]) * rstd * a.q_norm_g[d];
      float x1 = bf2f(qrow[h * D + d + 1]) * rstd * a.q_norm_g[d + 1];
      if (d >= D - R) {
        const float2 r = rt[(d - (D - R)) >> 1];
        const float y0 = x0 * r.x - x1 * r.y, y1 = x0 * r.y + x1 * r.x;
        x0 = y0;
        x1 = y1;
      }
      qh[h * D + d] = f2bf(x0);
      qh[h * D + d + 1] = f2bf(x1);
    }
  }
}

// normalise, de-rotate by -pos, store bf16: o[h][d] = acc[h][d] * inv[h]
__device__ void finish_store(const AttendArgs& a, const float* acc, const float* inv,
                             const float2* rt, uint16_t* orow) {
  const int H = a.H, D = a.D, R = a.R;
  for (int e2 = threadIdx.x; e2 < H * D / 2; e2 += blockDim.x) {
    const int h = (2 * e2) / D, d = (2 * e2) % D;
    float x0 = acc[h * D + d] * inv[h];
    float x1 = acc[h * D + d + 1] * inv[h];
    if (d >= D - R) {
      // rotation by -pos: (x cos + y sin, -x sin + y cos)
      const float2 r = rt[(d - (D - R)) >> 1];
      const float y0 = x0 * r.x + x1 * r.y, y1 = -x0 * r.y + x1 * r.x;
      x0 = y0;
      x1 = y1;
    }
    *reinterpret_cast<unsigned int*>(orow + h * D + d) = f2_to_bf2x2(x0, x1);
  }
}

__global__ void __launch_bounds__(kAttThreads) attend_generic_kernel(AttendArgs a) {
  extern __shared__ __align__(16) unsigned char asm_raw[];
  const int H = a.H, D = a.D;
  float* acc = reinterpret_cast<float*>(asm_raw);          // [H*D]
  float* kv = acc + H * D;                                  // [KT*D]
  float* lg = kv + kAttKT * D;                              // [H*KT]
  float* mrow = lg + H * kAttKT;                            // [H]
  float* lrow = mrow + H;                                   // [H]
  float* alpha = lrow + H;                                  // [H]
  // [R/2] pairs; (H*D + KT*D + H*KT) is even, so rounding 3H up keeps 8 B
  float2* rt = reinterpret_cast<float2*>(mrow + ((3 * H + 1) & ~1));
  uint16_t* qh = reinterpret_cast<uint16_t*>(rt + a.R / 2 + 1);  // [H*D]

  const int split = blockIdx.x, t = blockIdx.y, b = blockIdx.z;
  const int row = b * a.T_q + t;
  pdl_trigger();
  pdl_wait();
  const int pos = a.q_pos[row];
  const int tid = threadIdx.x;
  const int lane = tid & 31, warp = tid >> 5, nw = blockDim.x >> 5;
  if (pos < 0) {
    if (tid == 0 && split == 0) raise_err(a.err, DS4A_DEV_BAD_POS);
    return;
  }
  const int32_t* idx_row = a.sparse ? a.idx + (int64_t)row * a.k : nullptr;
  const KeyList kl = key_list(a, b, t, pos, idx_row);
  const int n_keys = kl.n_sel + kl.n_win;
  const int per = (n_keys + a.n_splits - 1) / a.n_splits;
  const int j0 = min(n_keys, split * per), j1 = min(n_keys, j0 + per);

  rope_table(a, pos, rt);
  __syncthreads();
  load_qhat(a, a.q + (int64_t)row * H * D, rt, qh);
  for (int e = tid; e < H * D; e += blockDim.x) acc[e] = 0.f;
  for (int h = tid; h < H; h += blockDim.x) { mrow[h] = -INFINITY; lrow[h] = 0.f; }
  __syncthreads();

  for (int jt = j0; jt < j1; jt += kAttKT) {
    const int nk = min(kAttKT, j1 - jt);
    // stage the K=V rows (rows that failed the bounds check become zeros
    // with a -inf logit)
    __shared__ int s_ok[kAttKT];
    for (int jj = warp; jj < kAttKT; jj += nw) {
      bool ok = false;
      const uint16_t* src = jj < nk ? key_row(a, b, kl, idx_row, jt + jj, &ok) : nullptr;
      if (jj < nk && !ok && lane == 0) raise_err(a.err, DS4A_DEV_BAD_INDEX);
      for (int d = lane; d < D; d += 32) kv[jj * D + d] = (jj < nk && ok) ? bf2f(src[d]) : 0.f;
      if (lane == 0) s_ok[jj] = (jj < nk && ok);
    }
    __syncthreads();
    // logits: one warp per (head, key) pair
    for (int pr = warp; pr < H * kAttKT; pr += nw) {
      const int h = pr / kAttKT, jj = pr % kAttKT;
      float dot = 0.f;
      for (int d = lane; d < D; d += 32) dot = fmaf(bf2f(qh[h * D + d]), kv[jj * D + d], dot);
      dot = warp_sum(dot);
      if (lane == 0) lg[h * kAttKT + jj] = s_ok[jj] ? dot * a.scale : -INFINITY;
    }
    __syncthreads();
    // online softmax
    for (int h = tid; h < H; h += blockDim.x) {
      float mx = mrow[h];
      for (int jj = 0; jj < kAttKT; ++jj) mx = fmaxf(mx, lg[h * kAttKT + jj]);
      const float al = (mrow[h] == -INFINITY) ? 0.f : __expf(mrow[h] - mx);
      float ls = lrow[h] * al;
      for (int jj = 0; jj < kAttKT; ++jj) {
        const float z = lg[h * kAttKT + jj];
        const float p = (z == -INFINITY) ? 0.f : __expf(z - mx);
        lg[h * kAttKT + jj] = p;
        ls += p;
      }
      mrow[h] = mx;
      lrow[h] = ls;
      alpha[h] = al;
    }
    __syncthreads();
    for (int e = tid; e < H * D; e += blockDim.x) {
      const int h = e / D, d = e % D;
      float v = acc[e] * alpha[h];
#pragma unroll
      for (int jj = 0; jj < kAttKT; ++jj) v = fmaf(lg[h * kAttKT + jj], kv[jj * D + d], v);
      acc[e] = v;
    }
    __syncthreads();
  }

  if (a.n_splits == 1) {
    // finish: 1 / (sum + exp(sink - max)), de-rotate, store
    for (int h = tid; h < H; h += blockDim.x) {
      const float mx = mrow[h];
      float den;
      if (mx == -INFINITY) den = 0.f;  // no keys: output 0
      else den = lrow[h] + __expf(a.sink[h] - mx);
      alpha[h] = den > 0.f ? 1.f / den : 0.f;
    }
    __syncthreads();
    finish_store(a, acc, alpha, rt, a.out + (int64_t)row * H * D);
    return;
  }
  float* part = a.ws + ((int64_t)row * a.n_splits + split) * (2 * H + H * D);
  for (int h = tid; h < H; h += blockDim.x) { part[h] = mrow[h]; part[H + h] = lrow[h]; }
  for (int e = tid; e < H * D; e += blockDim.x) part[2 * H + e] = acc[e];
}

// Merge of the key splits of one query: per head, M = max of the split
// maxima, L = sum of l_s exp(m_s - M), o = sum acc_s exp(m_s - M) / (L +
// exp(sink - M)); then the rope slice rotates back by -pos.  Thread block =
// 8 heads of one query.
constexpr int kCombThreads = 256;

// One block per (head, query row), one thread per pair of output dims.
// Every thread merges the splits itself, K at a time with all their loads
// (max, sum, two accumulator values) in flight together (K = 4 when that
// covers every split, keeping registers low for many resident blocks, else
// 8): the split
// maxima and sums are the same addresses for the whole block (broadcast),
// so no shared memory or block barrier is needed and a decode-sized merge
// costs one memory round trip.  The sink enters the denominator as in the
// split-free kernels; the rope slice is de-rotated by -pos at the end.
template <int K>
__global__ void __launch_bounds__(kCombThreads) attend_combine_kernel(AttendArgs a) {
  const int H = a.H, D = a.D, S = a.n_splits, R = a.R;
  const int h = blockIdx.x, t = blockIdx.y, b = blockIdx.z;
  const int row = b * a.T_q + t;
  pdl_trigger();
  const int pos = a.q_pos[row];  // inputs: read before the wait
  const float sink = a.sink[h];
  pdl_wait();
  const int64_t stride = 2 * H + (int64_t)H * D;
  const float* base = a.ws + (int64_t)row * S * stride;
  uint16_t* orow = a.out + ((int64_t)row * H + h) * D;
  for (int d2 = threadIdx.x; d2 < D / 2; d2 += kCombThreads) {
    const int d = 2 * d2;
    float M = -INFINITY, L = 0.f, x0 = 0.f, x1 = 0.f;
    for (int s0 = 0; s0 < S; s0 += K) {
      float ms[K], ls[K];
      float2 v[K];
#pragma unroll
      for (int u = 0; u < K; ++u) {
        ms[u] = -INFINITY;
        ls[u] = 0.f;
        v[u] = make_float2(0.f, 0.f);
        if (s0 + u < S) {
          const float* p = base + (int64_t)(s0 + u) * stride;
          ms[u] = p[h];
          ls[u] = p[H + h];
          v[u] = *reinterpret_cast<const float2*>(p + 2 * H + (int64_t)h * D + d);
        }
      }
      float mc = M;
#pragma unroll
      for (int u = 0; u < K; ++u) mc = fmaxf(mc, ms[u]);
      if (mc == -INFINITY) continue;
      const float sc = __expf(M - mc);  // 0 while nothing was merged
      L *= sc;
      x0 *= sc;
      x1 *= sc;
#pragma unroll
      for (int u = 0; u < K; ++u) {
        // a split with no visible key has max -inf: its accumulator is
        // never read into the sum
        if (ms[u] != -INFINITY) {
          const float e = __expf(ms[u] - mc);
          L = fmaf(ls[u], e, L);
          x0 = fmaf(v[u].x, e, x0);
          x1 = fmaf(v[u].y, e, x1);
        }
      }
      M = mc;
    }
    if (pos < 0) return;
    const float inv = (M == -INFINITY) ? 0.f : 1.f / (L + __expf(sink - M));
    x0 *= inv;
    x1 *= inv;
    if (d >= D - R) {
      float c, sn;
      rope_cos_sin(pos, a.rope.t[(d - (D - R)) >> 1], &c, &sn);
      const float y0 = x0 * c + x1 * sn, y1 = -x0 * sn + x1 * c;
      x0 = y0;
      x1 = y1;
    }
    *reinterpret_cast<unsigned int*>(orow + d) = f2_to_bf2x2(x0, x1);
  }
}

int attend_splits(int B, int T_q, int keys_max, int H, int D, bool tc, size_t ws_bytes,
                  size_t* need) {
  const int rows = B * T_q;
  const size_t per = (size_t)rows * (2 * H + (size_t)H * D) * sizeof(float);
  if (tc) {
    // the tensor-core path needs workspace only for the partials of key
    // splits; with less than they want it splits less (one split: none)
    int want = attend_tc_splits(B, T_q, keys_max);
    if (need) *need = want > 1 ? per * want : 0;
    if (want > 1 && per > 0 && ws_bytes < per * want) {
      want = (int)(ws_bytes / per);
      if (want < 2) want = 1;
    }
    return want;
  }
  int want = 1;
  if (rows > 0 && rows < 2 * 148) {
    want = (2 * 148 + rows - 1) / rows;
    const int by_keys = (keys_max + 63) / 64;
    want = min(want, max(1, by_keys));
    want = min(want, 64);
  }
  if (need) *need = want > 1 ? per * want : 0;
  if (want > 1 && per > 0 && ws_bytes < per * want) {
    want = (int)(ws_bytes / per);
    if (want < 2) want = 1;
  }
  return want;
}

cudaError_t launch_attend_generic(const AttendArgs& a, cudaStream_t s) {
  const int rows = a.B * a.T_q;
  if (rows <= 0) return cudaSuccess;
  const size_t smem = (size_t)(a.H * a.D + kAttKT * a.D + a.H * kAttKT + ((3 * a.H + 1) & ~1)) * sizeof(float) +
                      (size_t)(a.R / 2 + 1) * sizeof(float2) + (size_t)a.H * a.D * sizeof(uint16_t);
  static std::atomic<int> cache[kMaxDevices];
  cudaError_t e0 = ensure_smem(attend_generic_kernel, (int)smem, cache);
  if (e0 != cudaSuccess) return e0;
  {
    TraceScope tr("attend_generic", s);
    cudaError_t e1 = launch_pdl(attend_generic_kernel, dim3(a.n_splits, a.T_q, a.B), dim3(kAttThreads), smem, s, a);
    if (e1 != cudaSuccess) return e1;
  }
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess || a.n_splits == 1) return e;
  return launch_attend_combine(a, s);
}

cudaError_t launch_attend_combine(const AttendArgs& a, cudaStream_t s) {
  TraceScope tr("attend_combine", s);
  return a.n_splits <= 4
             ? launch_pdl(attend_combine_kernel<4>, dim3(a.H, a.T_q, a.B), dim3(kCombThreads), 0, s, a)
             : launch_pdl(attend_combine_kernel<8>, dim3(a.H, a.T_q, a.B), dim3(kCombThreads), 0, s, a);
}

}  // namespace ds4a
