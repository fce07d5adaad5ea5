// Top-k selector of the Lightning indexer ("DeepSeek-v4 Beyond Basics"
// 3.2.2 eq. 17; "Phase 1 Module 1", section on the indexer: the selection
// prunes only when more entries are visible than k): keep the k highest of a row's n_vis
// visible scores, ties to the lower index; write the kept indices
// ascending, padded with -1 when n_vis <= k.
//
// Scores become order-preserving uint32 keys.  A 4-pass 8-bit radix select
// finds the k-th largest key T and how many entries equal to T are needed;
// an ordered compaction then walks the row in index order and keeps every
// key above T and the first `need` keys equal to T, so the output comes out
// ascending without a sort.
//   topk_smem_kernel     one thread block per row, the row's keys staged in
//                        shared memory once (rows up to 12288 entries)
//   topk_cluster_kernel  one 8-block cluster per row (rows up to 262144,
//                        k <= 2048): each block stages a slice; a floor from
//                        the cluster's histogram of per-thread maxima
//                        leaves a short candidate list per block, which
//                        block 0 gathers through distributed shared memory
//                        and selects from (11-bit digits, three passes)
//   topk_cluster_wide_kernel  the same rows for k > 2048: histograms and
//                        compaction offsets summed over the cluster
//   topk_global_kernel   one block per row, every pass reading the scores
//                        from global memory (any length)
#include <cooperative_groups.h>

#include "ds4a_internal.cuh"

namespace cg = cooperative_groups;

namespace ds4a {
namespace {

constexpr int kSmemRowMax = 12288;
constexpr int kCluster = 8;
constexpr int kClusterSlice = 32768;
constexpr int kClusterThreads = 1024;

// inclusive scan of v over the block (thread order); *total = block sum.
// s_warp: >= 33 ints of shared memory.  Every thread must call it.
__device__ __forceinline__ int block_incl_scan(int v, int* s_warp, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int n = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += n;
  }
  if (lane == 31) s_warp[warp] = x;
  __syncthreads();
  if (warp == 0) {
    int w = lane < nw ? s_warp[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int n = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += n;
    }
    if (lane < nw) s_warp[lane] = w;  // inclusive warp prefix
    if (lane == 31) s_warp[32] = w;
  }
  __syncthreads();
  const int r = x + (warp > 0 ? s_warp[warp - 1] : 0);
  *total = s_warp[32];
  __syncthreads();
  return r;
}

// Digit of this pass: the bin holding the remaining-th largest key.
// hist: 256 counts; returns the digit and the count of keys in higher bins.
__device__ __forceinline__ void find_digit(const unsigned int* hist, int remaining, unsigned int* s_digit,
                                           int* s_above) {
  const int lane = threadIdx.x;
  if (lane >= 32) return;
  int cnt[8], sum = 0;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    cnt[j] = (int)hist[255 - 8 * lane - j];
    sum += cnt[j];
  }
  int incl = sum;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int n = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += n;
  }
  const int excl = incl - sum;
  if (excl < remaining && incl >= remaining) {
    int above = excl;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      if (above + cnt[j] >= remaining) {
        *s_digit = 255u - 8u * lane - j;
        *s_above = above;
        break;
      }
      above += cnt[j];
    }
  }
}

// Digit of a pass over 2048 bins (11-bit digits), blocks of 1024 threads:
// the bin holding the remaining-th largest key, counting from the top bin,
// and the count of keys in higher bins.  Every thread must call it.
__device__ __forceinline__ void find_digit2048(const unsigned int* hist, int remaining, int* s_warp,
                                               unsigned int* s_digit, int* s_above) {
  const int t = threadIdx.x;  // bins 2047 - 2t (first) and 2046 - 2t
  const int c0 = (int)hist[2047 - 2 * t], c1 = (int)hist[2046 - 2 * t];
  int tot;
  const int incl = block_incl_scan(c0 + c1, s_warp, &tot);
  const int excl = incl - (c0 + c1);
  if (excl < remaining && incl >= remaining) {
    if (excl + c0 >= remaining) {
      *s_digit = 2047u - 2u * t;
      *s_above = excl;
    } else {
      *s_digit = 2046u - 2u * t;
      *s_above = excl + c0;
    }
  }
  __syncthreads();
}

// Shared-memory slot of key i: XOR-swizzled inside each group of 32 so that
// both the strided passes (thread t reads i = t + j * blockDim) and the
// ordered walks (thread t reads its own run i = t * run + j) are free of
// bank conflicts (a plain layout put a run's 32 threads in one bank).  The
// array is sized to whole groups of 32.
__device__ __forceinline__ int kpos(int i) { return i ^ ((i >> 5) & 31); }

// Stage scores [0, n) of `src` as keys in shared memory (slot kpos(i)),
// every thread's loads in flight together (coalesced, kBatch per thread per
// round), and return the largest key this thread staged.  A 16-byte aligned
// source goes four keys per load: keys 4j .. 4j+3 share one XOR pattern
// (kpos flips bits 0-4 by the group index), so they land permuted inside
// one 16-byte slot and take one 128-bit store.
template <int kBatch>
__device__ __forceinline__ unsigned int stage_keys(const float* __restrict__ src, int n, unsigned int* keys) {
  unsigned int tmax = 0u;
  const int nt = blockDim.x, tid = threadIdx.x;
  int done = 0;
  if ((reinterpret_cast<uintptr_t>(src) & 15u) == 0) {
    const float4* src4 = reinterpret_cast<const float4*>(src);
    const int n4 = n >> 2;
    for (int base = 0; base < n4; base += kBatch * nt) {
      float4 v[kBatch];
#pragma unroll
      for (int u = 0; u < kBatch; ++u) {
        const int j = base + u * nt + tid;
        v[u] = j < n4 ? src4[j] : make_float4(0.f, 0.f, 0.f, 0.f);
      }
#pragma unroll
      for (int u = 0; u < kBatch; ++u) {
        const int j = base + u * nt + tid;
        if (j < n4) {
          const unsigned int k0 = f2key(v[u].x), k1 = f2key(v[u].y), k2 = f2key(v[u].z), k3 = f2key(v[u].w);
          tmax = max(tmax, max(max(k0, k1), max(k2, k3)));
          const int i = 4 * j;
          const unsigned int x = (unsigned int)(i >> 5) & 31u;  // kpos(i + e) = i ^ x ^ e
          const unsigned int m = x & 3u;
          // slot e holds key 4j + (e ^ m): swap pairs when bit 0 of m is
          // set, swap halves when bit 1 is
          const unsigned int a0 = (m & 1u) ? k1 : k0, a1 = (m & 1u) ? k0 : k1;
          const unsigned int a2 = (m & 1u) ? k3 : k2, a3 = (m & 1u) ? k2 : k3;
          uint4 w;
          w.x = (m & 2u) ? a2 : a0;
          w.y = (m & 2u) ? a3 : a1;
          w.z = (m & 2u) ? a0 : a2;
          w.w = (m & 2u) ? a1 : a3;
          *reinterpret_cast<uint4*>(keys + (i ^ (int)(x & ~3u))) = w;
        }
      }
    }
    done = n4 << 2;
  }
  for (int base = done; base < n; base += kBatch * nt) {
    float v[kBatch];
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
      const int i = base + u * nt + tid;
      v[u] = i < n ? src[i] : 0.f;
    }
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
      const int i = base + u * nt + tid;
      if (i < n) {
        const unsigned int key = f2key(v[u]);
        keys[kpos(i)] = key;
        tmax = max(tmax, key);
      }
    }
  }
  return tmax;
}

__device__ __forceinline__ void write_identity(const IndexArgs& a, int n_vis, const float* sc, int32_t* out,
                                               float* so) {
  for (int i = threadIdx.x; i < a.k; i += blockDim.x) {
    out[i] = i < n_vis ? i : -1;
    if (so) so[i] = i < n_vis ? sc[i] : -INFINITY;
  }
}

// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(512) topk_smem_kernel(IndexArgs a) {
  extern __shared__ unsigned int keys[];  // [n_vis]
  __shared__ unsigned int hist[256];
  __shared__ int s_warp[33];
  __shared__ unsigned int s_digit;
  __shared__ int s_above;
  const int row = blockIdx.x, tid = threadIdx.x;
  pdl_trigger();
  pdl_wait();
  const int pos = a.q_pos[row];
  const int n_vis = pos < 0 ? 0 : min((pos + 1) / a.m, a.N_c);
  const float* sc = a.scores + (int64_t)row * a.N_c;
  int32_t* out = a.idx_out + (int64_t)row * a.k;
  float* so = a.score_out ? a.score_out + (int64_t)row * a.k : nullptr;
  if (pos < 0 && tid == 0) raise_err(a.err, DS4A_DEV_BAD_POS);
  if (n_vis <= a.k) {
    write_identity(a, n_vis, sc, out, so);
    return;
  }
  // several blocks share an SM here: two 16-byte loads per thread in flight
  stage_keys<2>(sc, n_vis, keys);
  unsigned int prefix = 0, mask = 0;
  int remaining = a.k;
  for (int pass = 0; pass < 4; ++pass) {
    const int shift = 24 - 8 * pass;
    for (int i = tid; i < 256; i += blockDim.x) hist[i] = 0;
    __syncthreads();
    for (int i = tid; i < n_vis; i += blockDim.x) {
      const unsigned int u = keys[kpos(i)];
      if ((u & mask) == prefix) atomicAdd(&hist[(u >> shift) & 255u], 1u);
    }
    __syncthreads();
    find_digit(hist, remaining, &s_digit, &s_above);
    __syncthreads();
    prefix |= s_digit << shift;
    mask |= 255u << shift;
    remaining -= s_above;
  }
  const unsigned int T = prefix;
  const int need = remaining;
  // ordered compaction: thread t walks keys [t*run, t*run + run)
  const int run = (n_vis + blockDim.x - 1) / blockDim.x;
  const int i0 = min(n_vis, tid * run), i1 = min(n_vis, i0 + run);
  int gt = 0, eq = 0;
#pragma unroll 8
  for (int i = i0; i < i1; ++i) {
    const unsigned int u = keys[kpos(i)];
    gt += u > T;
    eq += u == T;
  }
  int tot;
  const int eq_before = block_incl_scan(eq, s_warp, &tot) - eq;
  const int take_eq = max(0, min(eq, need - eq_before));
  const int sel_before = block_incl_scan(gt + take_eq, s_warp, &tot) - (gt + take_eq);
  int o = sel_before, tr = eq_before;
  for (int i = i0; i < i1; ++i) {
    const unsigned int u = keys[kpos(i)];
    bool keep = u > T;
    if (u == T) keep = tr++ < need;
    if (keep) {
      out[o] = i;
      if (so) so[o] = sc[i];
      ++o;
    }
  }
}

// ---------------------------------------------------------------------------
__global__ void __cluster_dims__(kCluster, 1, 1) __launch_bounds__(kClusterThreads)
    topk_cluster_wide_kernel(IndexArgs a) {
  extern __shared__ unsigned int keys[];  // [kClusterSlice]
  __shared__ unsigned int hist[2048];
  __shared__ unsigned int hist_all[2048];
  __shared__ int s_warp[33];
  __shared__ int s_tot[2];  // this block's tie count, kept count
  __shared__ unsigned int s_digit;
  __shared__ int s_above;
  cg::cluster_group cl = cg::this_cluster();
  const int rank = (int)cl.block_rank();
  const int row = blockIdx.x / kCluster, tid = threadIdx.x;
  pdl_trigger();
  pdl_wait();
  const int pos = a.q_pos[row];
  const int n_vis = pos < 0 ? 0 : min((pos + 1) / a.m, a.N_c);
  const float* sc = a.scores + (int64_t)row * a.N_c;
  int32_t* out = a.idx_out + (int64_t)row * a.k;
  float* so = a.score_out ? a.score_out + (int64_t)row * a.k : nullptr;
  if (n_vis <= a.k) {  // the same branch in every block of the cluster
    if (rank == 0) {
      if (pos < 0 && tid == 0) raise_err(a.err, DS4A_DEV_BAD_POS);
      write_identity(a, n_vis, sc, out, so);
    }
    return;
  }
  const int slice = (n_vis + kCluster - 1) / kCluster;
  const int lo = min(n_vis, rank * slice), hi = min(n_vis, lo + slice);
  const int n = hi - lo;
  for (int i = tid; i < 2048; i += blockDim.x) hist[i] = 0;
  __syncthreads();
  // stage the slice; thread t's keys are t, t + 1024, ...: their maximum
  const unsigned int tmax = stage_keys<8>(sc + lo, n, keys);
  // Histogram (cluster-wide, one 2048-bin pass) of the top 11 bits of the
  // cluster's 8192 per-thread maxima: the lowest key of the bin holding the
  // k-th largest maximum is a floor with at least k keys at or above it
  // (each of those maxima is one), so the select over the keys can skip
  // everything below it and counts about a thousand keys.
  atomicAdd(&hist[tmax >> 21], 1u);
  auto reduce_hist = [&]() {
    cl.sync();  // every block's histogram is complete
    for (int b = tid; b < 2048; b += blockDim.x) {
      unsigned int sum = 0;
#pragma unroll
      for (int r = 0; r < kCluster; ++r) sum += cl.map_shared_rank(hist, r)[b];
      hist_all[b] = sum;
    }
    __syncthreads();
  };
  reduce_hist();
  find_digit2048(hist_all, a.k, s_warp, &s_digit, &s_above);
  const unsigned int floor_key = s_digit << 21;
  // Radix select over the keys >= floor with 11-, 11- and 10-bit digits:
  // the k-th largest key T and how many of the keys equal to T are needed.
  unsigned int prefix = 0, mask = 0;
  int remaining = a.k;
#pragma unroll 1
  for (int pass = 0; pass < 3; ++pass) {
    const int shift = pass == 0 ? 21 : (pass == 1 ? 10 : 0);
    const unsigned int dmask = pass < 2 ? 2047u : 1023u;
    cl.sync();  // peers are done reading this block's previous histogram
    for (int i = tid; i < 2048; i += blockDim.x) hist[i] = 0;
    __syncthreads();
    for (int i = tid; i < n; i += blockDim.x) {
      const unsigned int u = keys[kpos(i)];
      if (u >= floor_key && (u & mask) == prefix) atomicAdd(&hist[(u >> shift) & dmask], 1u);
    }
    reduce_hist();
    find_digit2048(hist_all, remaining, s_warp, &s_digit, &s_above);
    prefix |= s_digit << shift;
    mask |= dmask << shift;
    remaining -= s_above;
  }
  cl.sync();  // no peer still reads this block's histogram
  const unsigned int T = prefix;
  const int need = remaining;
  // ordered compaction across the cluster: block r holds indices
  // [lo, hi), so the ties and kept entries of lower ranks come first
  const int run = (n + blockDim.x - 1) / blockDim.x;
  const int i0 = min(n, tid * run), i1 = min(n, i0 + run);
  int gt = 0, eq = 0;
#pragma unroll 8
  for (int i = i0; i < i1; ++i) {
    const unsigned int u = keys[kpos(i)];
    gt += u > T;
    eq += u == T;
  }
  int eq_tot;
  const int eq_local = block_incl_scan(eq, s_warp, &eq_tot) - eq;
  if (tid == 0) s_tot[0] = eq_tot;
  cl.sync();
  int eq_base = 0;
  for (int r = 0; r < rank; ++r) eq_base += cl.map_shared_rank(s_tot, r)[0];
  const int eq_before = eq_base + eq_local;
  const int take_eq = max(0, min(eq, need - eq_before));
  int sel_tot;
  const int sel_local = block_incl_scan(gt + take_eq, s_warp, &sel_tot) - (gt + take_eq);
  if (tid == 0) s_tot[1] = sel_tot;
  cl.sync();
  int sel_base = 0;
  for (int r = 0; r < rank; ++r) sel_base += cl.map_shared_rank(s_tot, r)[1];
  int o = sel_base + sel_local, tr = eq_before;
  for (int i = i0; i < i1; ++i) {
    const unsigned int u = keys[kpos(i)];
    bool keep = u > T;
    if (u == T) keep = tr++ < need;
    if (keep) {
      out[o] = lo + i;
      if (so) so[o] = sc[lo + i];
      ++o;
    }
  }
  cl.sync();  // no block leaves while a peer may still read its shared memory
}

// ---------------------------------------------------------------------------
// Block-level radix select (1024 threads) over vals[0..n) (slot(i) maps an
// index to its shared-memory slot), counting only values >= floor, 11-, 11-
// and 10-bit digits: the k-th largest value and how many equal to it are
// needed.  hist: 2048 counters of shared memory.
template <typename Slot>
__device__ __forceinline__ void block_select(const unsigned int* vals, int n, Slot slot, unsigned int floor_v, int k,
                                             unsigned int* hist, int* s_warp, unsigned int* s_digit, int* s_above,
                                             unsigned int* T_out, int* need_out) {
  unsigned int prefix = 0, mask = 0;
  int remaining = k;
#pragma unroll 1
  for (int pass = 0; pass < 3; ++pass) {
    const int shift = pass == 0 ? 21 : (pass == 1 ? 10 : 0);
    const unsigned int dmask = pass < 2 ? 2047u : 1023u;
    for (int i = threadIdx.x; i < 2048; i += blockDim.x) hist[i] = 0;
    __syncthreads();
    for (int i = threadIdx.x; i < n; i += blockDim.x) {
      const unsigned int u = vals[slot(i)];
      if (u >= floor_v && (u & mask) == prefix) atomicAdd(&hist[(u >> shift) & dmask], 1u);
    }
    __syncthreads();
    find_digit2048(hist, remaining, s_warp, s_digit, s_above);
    prefix |= *s_digit << shift;
    mask |= dmask << shift;
    remaining -= *s_above;
    __syncthreads();  // every thread has read the digit before the next pass writes it
  }
  *T_out = prefix;
  *need_out = remaining;
}

// Ordered compaction (1024 threads): thread t walks [t*run, t*run + run) of
// vals and keeps every value > T and the first `need` values == T in index
// order; keep(i, o) stores kept i at output position o.  Returns the count.
template <typename Slot, typename Keep>
__device__ __forceinline__ int block_compact(const unsigned int* vals, int n, Slot slot, unsigned int T, int need,
                                             int* s_warp, Keep keep) {
  const int run = (n + blockDim.x - 1) / blockDim.x;
  const int i0 = min(n, (int)threadIdx.x * run), i1 = min(n, i0 + run);
  int gt = 0, eq = 0;
#pragma unroll 8
  for (int i = i0; i < i1; ++i) {
    const unsigned int u = vals[slot(i)];
    gt += u > T;
    eq += u == T;
  }
  int tot;
  const int eq_before = block_incl_scan(eq, s_warp, &tot) - eq;
  const int take_eq = max(0, min(eq, need - eq_before));
  const int sel_before = block_incl_scan(gt + take_eq, s_warp, &tot) - (gt + take_eq);
  int o = sel_before, tr = eq_before;
  for (int i = i0; i < i1; ++i) {
    const unsigned int u = vals[slot(i)];
    bool k_ = u > T;
    if (u == T) k_ = tr++ < need;
    if (k_) keep(i, o++);
  }
  return tot;
}

constexpr int kLocalK = 2048;  // largest k of the local-candidate cluster kernel

// One 8-block cluster per row (rows up to 262144 entries, k <= 2048).
// Every block stages a slice and histograms its threads' maxima (2048 bins
// of the top 11 key bits); after one cluster barrier each block sums the 8
// histograms and takes the floor F = the lowest key of the bin holding the
// k-th largest maximum.  At least k keys of the row lie at or above F (the
// maxima are distinct keys), so the row's k-th largest T >= F and every key
// the selection can keep is >= F.  Each block writes its keys >= F in index
// order; after a second barrier block 0 gathers the lists (rank order, so
// index order) and selects the row's k among them.  When some block has
// more than kLocalK keys >= F (scores crowded into one bin), every block
// instead selects its own k best (a floor from its own maxima, then 11-bit
// digits) and block 0 merges those lists: the row's top k lies in the union
// of the blocks' top k (same tie rule).  Either way the result is exact.
__global__ void __cluster_dims__(kCluster, 1, 1) __launch_bounds__(kClusterThreads)
    topk_cluster_kernel(IndexArgs a) {
  extern __shared__ __align__(16) unsigned int keys[];  // [kClusterSlice]; block 0 reuses it for the gathered lists
  __shared__ __align__(16) unsigned int hist[2048];  // this block's histogram of maxima (read by the peers)
  __shared__ __align__(16) unsigned int hsum[2048];  // the cluster's
  __shared__ unsigned int cand_key[kLocalK];
  __shared__ int cand_idx[kLocalK];
  __shared__ int s_warp[33];
  __shared__ int s_count, s_count2;  // list lengths: first pass, and the per-block top k
  __shared__ int s_cnt[kCluster];
  __shared__ unsigned int s_digit;
  __shared__ int s_above;
  cg::cluster_group cl = cg::this_cluster();
  const int rank = (int)cl.block_rank();
  const int row = blockIdx.x / kCluster, tid = threadIdx.x;
  pdl_trigger();
  pdl_wait();
  const int pos = a.q_pos[row];
  const int n_vis = pos < 0 ? 0 : min((pos + 1) / a.m, a.N_c);
  const float* sc = a.scores + (int64_t)row * a.N_c;
  int32_t* out = a.idx_out + (int64_t)row * a.k;
  float* so = a.score_out ? a.score_out + (int64_t)row * a.k : nullptr;
  if (n_vis <= a.k) {  // the same branch in every block of the cluster
    if (rank == 0) {
      if (pos < 0 && tid == 0) raise_err(a.err, DS4A_DEV_BAD_POS);
      write_identity(a, n_vis, sc, out, so);
    }
    return;
  }
  const int k = a.k;
  // slices start on a multiple of 4 (16-byte aligned loads when the row is)
  const int slice = ((n_vis + kCluster - 1) / kCluster + 3) & ~3;
  const int lo = min(n_vis, rank * slice), hi = min(n_vis, lo + slice);
  const int n = hi - lo;
  for (int i = tid; i < 2048; i += blockDim.x) hist[i] = 0;
  __syncthreads();
  const unsigned int tmax = stage_keys<8>(sc + lo, n, keys);
  // one count per thread (a thread without keys counts in bin 0, below
  // every finite score), 8192 over the cluster
  atomicAdd(&hist[tmax >> 21], 1u);
  auto kslot = [](int i) { return kpos(i); };
  cl.sync();  // every block's histogram of maxima is complete
  for (int i = tid; i < 512; i += blockDim.x) {  // four bins per 16-byte read
    uint4 c[kCluster];
#pragma unroll
    for (int r = 0; r < kCluster; ++r) c[r] = reinterpret_cast<const uint4*>(cl.map_shared_rank(hist, r))[i];
    uint4 t = make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
    for (int r = 0; r < kCluster; ++r) {
      t.x += c[r].x;
      t.y += c[r].y;
      t.z += c[r].z;
      t.w += c[r].w;
    }
    reinterpret_cast<uint4*>(hsum)[i] = t;
  }
  __syncthreads();
  find_digit2048(hsum, k, s_warp, &s_digit, &s_above);
  const unsigned int F = s_digit << 21;
  {
    // this block's keys >= F, in index order (thread t walks its own run)
    const int run = (n + blockDim.x - 1) / blockDim.x;
    const int i0 = min(n, tid * run), i1 = min(n, i0 + run);
    int cnt = 0;
#pragma unroll 8
    for (int i = i0; i < i1; ++i) cnt += keys[kpos(i)] >= F;
    int tot;
    int o = block_incl_scan(cnt, s_warp, &tot) - cnt;
    if (tot <= kLocalK)
      for (int i = i0; i < i1; ++i) {
        const unsigned int u = keys[kpos(i)];
        if (u >= F) {
          cand_key[o] = u;
          cand_idx[o] = lo + i;
          ++o;
        }
      }
    if (tid == 0) s_count = tot;
  }
  cl.sync();  // every block's list (or its count alone, when too long) is in place
  if (tid < kCluster) s_cnt[tid] = *cl.map_shared_rank(&s_count, tid);
  __syncthreads();
  bool overflow = false;
#pragma unroll
  for (int r = 0; r < kCluster; ++r) overflow |= s_cnt[r] > kLocalK;
  if (overflow) {
    // the same decision in every block: each selects its own k best
    if (n <= k) {
      for (int i = tid; i < n; i += blockDim.x) {
        cand_key[i] = keys[kpos(i)];
        cand_idx[i] = lo + i;
      }
      if (tid == 0) s_count2 = n;
    } else {
      // floor: the lowest key of the bin holding the k-th largest of this
      // block's maxima (hist is this block's, no longer read by the peers);
      // no floor when k exceeds the threads
      unsigned int floor_v = 0u;
      if (k <= (int)blockDim.x) {
        find_digit2048(hist, k, s_warp, &s_digit, &s_above);
        floor_v = s_digit << 21;
      }
      unsigned int T;
      int need;
      block_select(keys, n, kslot, floor_v, k, hist, s_warp, &s_digit, &s_above, &T, &need);
      const int cnt = block_compact(keys, n, kslot, T, need, s_warp, [&](int i, int o) {
        cand_key[o] = keys[kpos(i)];
        cand_idx[o] = lo + i;
      });
      if (tid == 0) s_count2 = cnt;
    }
    cl.sync();  // every block's candidate list is complete
    if (tid < kCluster) s_cnt[tid] = *cl.map_shared_rank(&s_count2, tid);
    __syncthreads();
  }
  if (rank == 0) {
    // gather the lists in rank order into keys[0 .. total) and the indices
    // into keys[16384 ..] (total <= 8 kLocalK = 16384)
    int offs[kCluster + 1];
    offs[0] = 0;
#pragma unroll
    for (int r = 0; r < kCluster; ++r) offs[r + 1] = offs[r] + s_cnt[r];
    const int total = offs[kCluster];
    int* gidx = reinterpret_cast<int*>(keys + 16384);
    for (int i = tid; i < total; i += blockDim.x) {
      int r = 0;
#pragma unroll
      for (int q = 1; q < kCluster; ++q) r += i >= offs[q];
      keys[i] = cl.map_shared_rank(cand_key, r)[i - offs[r]];
      gidx[i] = cl.map_shared_rank(cand_idx, r)[i - offs[r]];
    }
    __syncthreads();
    auto plain = [](int i) { return i; };
    unsigned int T;
    int need;
    block_select(keys, total, plain, 0u, k, hist, s_warp, &s_digit, &s_above, &T, &need);
    block_compact(keys, total, plain, T, need, s_warp, [&](int i, int o) {
      const int e = gidx[i];
      out[o] = e;
      if (so) so[o] = sc[e];
    });
  }
  cl.sync();  // no block leaves while block 0 may still read its list
}

// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(1024) topk_global_kernel(IndexArgs a) {
  __shared__ unsigned int hist[256];
  __shared__ int s_warp[33];
  __shared__ unsigned int s_digit;
  __shared__ int s_above;
  const int row = blockIdx.x, tid = threadIdx.x;
  pdl_trigger();
  pdl_wait();
  const int pos = a.q_pos[row];
  const int n_vis = pos < 0 ? 0 : min((pos + 1) / a.m, a.N_c);
  const float* sc = a.scores + (int64_t)row * a.N_c;
  int32_t* out = a.idx_out + (int64_t)row * a.k;
  float* so = a.score_out ? a.score_out + (int64_t)row * a.k : nullptr;
  if (pos < 0 && tid == 0) raise_err(a.err, DS4A_DEV_BAD_POS);
  if (n_vis <= a.k) {
    write_identity(a, n_vis, sc, out, so);
    return;
  }
  unsigned int prefix = 0, mask = 0;
  int remaining = a.k;
  for (int pass = 0; pass < 4; ++pass) {
    const int shift = 24 - 8 * pass;
    for (int i = tid; i < 256; i += blockDim.x) hist[i] = 0;
    __syncthreads();
    for (int i = tid; i < n_vis; i += blockDim.x) {
      const unsigned int u = f2key(sc[i]);
      if ((u & mask) == prefix) atomicAdd(&hist[(u >> shift) & 255u], 1u);
    }
    __syncthreads();
    find_digit(hist, remaining, &s_digit, &s_above);
    __syncthreads();
    prefix |= s_digit << shift;
    mask |= 255u << shift;
    remaining -= s_above;
  }
  const unsigned int T = prefix;
  const int need = remaining;
  // ordered compaction in chunks of blockDim (coalesced reads)
  int out_base = 0, eq_base = 0;
  for (int base = 0; base < n_vis; base += blockDim.x) {
    const int i = base + tid;
    const unsigned int u = i < n_vis ? f2key(sc[i]) : 0u;
    const int eq = (i < n_vis && u == T) ? 1 : 0;
    int eq_tot;
    const int eq_before = eq_base + block_incl_scan(eq, s_warp, &eq_tot) - eq;
    const int keep = (i < n_vis && (u > T || (eq && eq_before < need))) ? 1 : 0;
    int keep_tot;
    const int o = out_base + block_incl_scan(keep, s_warp, &keep_tot) - keep;
    if (keep) {
      out[o] = i;
      if (so) so[o] = sc[i];
    }
    out_base += keep_tot;
    eq_base += eq_tot;
    if (out_base >= a.k) break;
  }
}

}  // namespace

cudaError_t launch_topk(const IndexArgs& a, cudaStream_t s) {
  const int rows = a.B * a.T_q;
  if (rows <= 0) return cudaSuccess;
  if (a.N_c <= kSmemRowMax) {
    const size_t smem = (size_t)((max(1, a.N_c) + 31) & ~31) * sizeof(unsigned int);
    static std::atomic<int> cache[kMaxDevices];
    cudaError_t e = ensure_smem(topk_smem_kernel, (int)smem, cache);
    if (e != cudaSuccess) return e;
    TraceScope tr("topk_smem", s);
    return launch_pdl(topk_smem_kernel, dim3(rows), dim3(512), smem, s, a);
  }
  if (a.N_c <= kCluster * kClusterSlice) {
    const size_t smem = (size_t)kClusterSlice * sizeof(unsigned int);
    if (a.k <= kLocalK) {
      static std::atomic<int> cache[kMaxDevices];
      cudaError_t e = ensure_smem(topk_cluster_kernel, (int)smem, cache);
      if (e != cudaSuccess) return e;
      TraceScope tr("topk_cluster", s);
      return launch_pdl(topk_cluster_kernel, dim3(rows * kCluster), dim3(kClusterThreads), smem, s, a);
    }
    static std::atomic<int> cache_w[kMaxDevices];
    cudaError_t e = ensure_smem(topk_cluster_wide_kernel, (int)smem, cache_w);
    if (e != cudaSuccess) return e;
    TraceScope tr("topk_cluster", s);
    return launch_pdl(topk_cluster_wide_kernel, dim3(rows * kCluster), dim3(kClusterThreads), smem, s, a);
  }
  TraceScope tr("topk_global", s);
  return launch_pdl(topk_global_kernel, dim3(rows), dim3(1024), 0, s, a);
}

}  // namespace ds4a
