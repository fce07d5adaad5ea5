// Internal declarations shared by the ds4a CUDA sources.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include <atomic>
#include <mutex>

#include "ds4a.h"

namespace ds4a {

// ---------------------------------------------------------------------------
// device error word (one per device, per loaded library).  It is a
// __device__ variable of ds4a_api.cu; kernels get its device address in
// their argument struct (err_word() looks it up once per device).
// ---------------------------------------------------------------------------
unsigned int* err_word();

__device__ __forceinline__ void raise_err(unsigned int* w, unsigned int bits) { atomicOr(w, bits); }

// ---------------------------------------------------------------------------
// bf16 helpers
// ---------------------------------------------------------------------------
__device__ __forceinline__ float bf2f(uint16_t u) { return __uint_as_float(((unsigned int)u) << 16); }

// round-to-nearest-even conversions (one cvt instruction each)
__device__ __forceinline__ uint16_t f2bf(float f) {
  uint16_t u;
  asm("cvt.rn.bf16.f32 %0, %1;" : "=h"(u) : "f"(f));
  return u;
}

__device__ __forceinline__ float2 bf2x2_to_f2(unsigned int w) {
  return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u));
}

// a in the low half, b in the high half
__device__ __forceinline__ unsigned int f2_to_bf2x2(float a, float b) {
  unsigned int u;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(u) : "f"(b), "f"(a));
  return u;
}

// packed fp32 pairs: one instruction works on both halves of a float2
__device__ __forceinline__ float2 add_f2(float2 a, float2 b) {
  float2 r;
  asm("{\n .reg .b64 x, y, d;\n mov.b64 x, {%2, %3};\n mov.b64 y, {%4, %5};\n"
      " add.rn.f32x2 d, x, y;\n mov.b64 {%0, %1}, d;\n}"
      : "=f"(r.x), "=f"(r.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return r;
}
__device__ __forceinline__ float2 sub_f2(float2 a, float2 b) {
  float2 r;
  asm("{\n .reg .b64 x, y, d;\n mov.b64 x, {%2, %3};\n mov.b64 y, {%4, %5};\n"
      " sub.rn.f32x2 d, x, y;\n mov.b64 {%0, %1}, d;\n}"
      : "=f"(r.x), "=f"(r.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return r;
}
__device__ __forceinline__ float2 mul_f2(float2 a, float2 b) {
  float2 r;
  asm("{\n .reg .b64 x, y, d;\n mov.b64 x, {%2, %3};\n mov.b64 y, {%4, %5};\n"
      " mul.rn.f32x2 d, x, y;\n mov.b64 {%0, %1}, d;\n}"
      : "=f"(r.x), "=f"(r.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return r;
}
__device__ __forceinline__ float2 fma_f2(float2 a, float2 b, float2 c) {
  float2 r;
  asm("{\n .reg .b64 x, y, z, d;\n mov.b64 x, {%2, %3};\n mov.b64 y, {%4, %5};\n"
      " mov.b64 z, {%6, %7};\n fma.rn.f32x2 d, x, y, z;\n mov.b64 {%0, %1}, d;\n}"
      : "=f"(r.x), "=f"(r.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
  return r;
}

// RoPE frequencies theta_j = base^(-2j/R), j < R/2, divided by pi and
// formed in float64 on the host once per call (float32 would lose ~0.03 rad
// of phase at positions near 2^20).
constexpr int kMaxRopePairs = 256;
struct RopeTheta {
  double t[kMaxRopePairs];
};
void fill_rope_theta(RopeTheta* r, int rope_dim, float base);

// cos / sin of pos * theta_j: one float64 product, an exact reduction of the
// angle (in units of pi) into [-1, 1], then float32 sincospif.
__device__ __forceinline__ void rope_cos_sin(int pos, double theta_over_pi, float* c, float* s) {
  double t = (double)pos * theta_over_pi;
  t -= 2.0 * rint(0.5 * t);
  sincospif((float)t, s, c);
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// 2^x with the hardware approximation (about 2 ulp)
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// order-preserving map float -> uint32 (larger float -> larger key)
__device__ __forceinline__ unsigned int f2key(float f) {
  unsigned int b = __float_as_uint(f);
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

// Per-device caches of the host side hold up to this many devices (a call
// on a device beyond it fails with cudaErrorInvalidDevice).
constexpr int kMaxDevices = 64;

// Serialises the slow path of ensure_smem across host threads.
inline std::mutex& smem_attr_mutex() {
  static std::mutex m;
  return m;
}

// Raise a kernel's dynamic shared-memory limit to `bytes` on the current
// device when it is below that (cache[dev] holds the limit set so far).  The
// limit only grows, under a lock, so a launch that another host thread
// prepared for a smaller size stays valid.  Returns the error of
// cudaFuncSetAttribute, if any.
template <typename F>
inline cudaError_t ensure_smem(F* f, int bytes, std::atomic<int>* cache) {
  if (bytes <= 48 * 1024) return cudaSuccess;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    (void)cudaGetLastError();
    return cudaErrorInvalidDevice;
  }
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  if (cache[dev].load(std::memory_order_acquire) >= bytes) return cudaSuccess;
  std::lock_guard<std::mutex> lock(smem_attr_mutex());
  if (cache[dev].load(std::memory_order_relaxed) >= bytes) return cudaSuccess;
  cudaError_t e = cudaFuncSetAttribute(reinterpret_cast<const void*>(f),
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e != cudaSuccess) {
    (void)cudaGetLastError();  // do not leave it for a later launch check
    return e;
  }
  cache[dev].store(bytes, std::memory_order_release);
  return cudaSuccess;
}

// ---------------------------------------------------------------------------
// programmatic dependent launch: every library kernel is launched with
// programmatic stream serialisation, lets its successor start once all of its
// own blocks are running (pdl_trigger), and waits for its predecessor's
// memory (pdl_wait) before touching global memory.  Every kernel waits, so
// the ordering is transitive along the stream.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                              Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...);
}

// the same with a 1-D thread-block cluster of cx blocks (cx = 1: none)
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl_cluster(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem,
                                      cudaStream_t s, int cx, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = (unsigned)cx;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = cx > 1 ? 2 : 1;
  return cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...);
}

// ---------------------------------------------------------------------------
// launch trace
// ---------------------------------------------------------------------------
struct TraceScope {
  const char* name;
  cudaStream_t stream;
  int slot;
  TraceScope(const char* n, cudaStream_t s);
  ~TraceScope();
};

// ---------------------------------------------------------------------------
// kernels (launchers return cudaError_t of the launch)
// ---------------------------------------------------------------------------
struct CompressArgs {
  int B, T_tok, tok_begin, c, m, rope_dim;
  float rope_base, eps;
  const uint16_t *ca, *cb, *za, *zb;
  const float *bias_a, *bias_b, *norm_g;
  int entry_begin, entry_end;
  uint16_t* pool;
  int64_t pool_bstride;
  unsigned int* err;
  // append mode (app_pos != nullptr): ca..zb are the new token's rows
  // [B, c]; the earlier tokens come from the ring state [B][S][ring_cap][c]
  // (S = 4 streams ca, cb, za, zb for CSA, 2 streams ca, za for HCA; slot =
  // position mod ring_cap); each sequence's entry is the one its token
  // closes, if any, and must be below n_cap
  const int32_t* app_pos;
  uint16_t* ring;
  int ring_cap, n_cap;
  // block-scaled output (qfmt 1: mixed FP8 / BF16 K=V rows of q_row bytes;
  // 2: FP4 codes of c/2 bytes plus c/32 scales per entry) instead of bf16:
  // entry i of sequence b at qpool + b * q_bstride + i * q_row (bytes), its
  // FP4 scales at qscales + b * qs_bstride + i * (c/32)
  int qfmt;
  uint8_t* qpool;
  int64_t q_bstride, q_row;
  uint8_t* qscales;
  int64_t qs_bstride;
  RopeTheta rope;
};
cudaError_t launch_compress(const CompressArgs& a, cudaStream_t s);
// several append-mode jobs of the same batch; two plain jobs share a launch
cudaError_t launch_compress_jobs(const CompressArgs* jobs, int n_jobs, cudaStream_t s);

struct IndexArgs {
  int B, T_q, H, D, m, k, N_c;
  const int32_t* q_pos;
  const uint16_t *q, *w, *kidx;
  // FP4 keys (kcodes != nullptr): E2M1 codes [.., D/2] and E8M0 scales
  // [.., D/32] per key; k_bstride then counts keys
  const uint8_t *kcodes, *kscales;
  int64_t k_bstride;
  float* scores;  // workspace [B*T_q, N_c]
  int32_t* idx_out;
  float* score_out;
  unsigned int* err;
};
cudaError_t launch_index_scores_generic(const IndexArgs& a, cudaStream_t s);
bool index_scores_tc_supported(const IndexArgs& a);
cudaError_t launch_index_scores_tc(const IndexArgs& a, cudaStream_t s);
cudaError_t launch_topk(const IndexArgs& a, cudaStream_t s);

struct AttendArgs {
  int B, T_q, H, D, R, W, m, k, N_c, win_cap, sparse;
  float scale, rope_base, eps;
  const int32_t* q_pos;
  const uint16_t* q;
  const float* q_norm_g;
  const uint16_t* pool;
  // mixed FP8 / BF16 pool rows (DS4A_MX_KV_FP8), instead of pool when set;
  // pool_bstride then counts rows
  const uint8_t* pool8;
  int64_t pool_bstride;
  const int32_t* idx;
  const uint16_t* win;
  int64_t win_bstride;
  const float* sink;
  uint16_t* out;
  float* ws;  // split partials
  int n_splits;
  int keys_max;  // upper bound of keys per query
  unsigned int* err;
  RopeTheta rope;
};
// Key splits per query (and the workspace they need) for the path that
// serves these sizes; fewer when ws_bytes cannot hold the partials.
int attend_splits(int B, int T_q, int keys_max, int H, int D, bool tc, size_t ws_bytes, size_t* need);
int attend_tc_splits(int B, int T_q, int keys_max);
cudaError_t launch_attend_generic(const AttendArgs& a, cudaStream_t s);
bool attend_tc_supported(const AttendArgs& a);
cudaError_t launch_attend_tc(const AttendArgs& a, cudaStream_t s);
cudaError_t launch_attend_combine(const AttendArgs& a, cudaStream_t s);

// bf16 rows -> block-scaled rows (ds4a_mx.cu)
cudaError_t launch_quant_kv_fp8(int n_rows, int D, int R, const uint16_t* in, int64_t in_stride, uint8_t* out,
                                int64_t out_stride, cudaStream_t s);
cudaError_t launch_quant_idx_fp4(int n_rows, int D, const uint16_t* in, int64_t in_stride, uint8_t* codes,
                                 uint8_t* scales, cudaStream_t s);

// Tensor-core GEMM of the grouped output projection (ds4a_outproj.cu):
// out[M][N] (row stride ldo) = A x B^T with B = bf16 [N][K]; output tile
// columns n read A's columns from (n / n_per_group) * a_group_k on.  acc: a
// float [M][N] workspace when gemm_ksplit(M, N, K) > 1.
int gemm_ksplit(int M, int N, int K);
size_t gemm_acc_bytes(int M, int N, int K);
cudaError_t launch_gemm(const uint16_t* a, int64_t a_cols, int64_t a_ld, const uint16_t* b, int M, int N, int K,
                        int n_per_group, int a_group_k, uint16_t* out, int64_t ldo, float* acc,
                        unsigned int* err, cudaStream_t s);

}  // namespace ds4a
