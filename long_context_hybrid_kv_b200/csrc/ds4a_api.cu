// extern "C" entry points of libds4a: argument checks (before any launch),
// dispatch to the kernels, the device error word and the launch trace.
#include "ds4a_internal.cuh"
#include "ds4a_mx.cuh"

#include <math.h>
#include <stdio.h>
#include <vector>

namespace ds4a {

__device__ unsigned int g_err_word = 0;

void fill_rope_theta(RopeTheta* r, int rope_dim, float base) {
  for (int j = 0; j < kMaxRopePairs; ++j)
    r->t[j] = (2 * j < rope_dim) ? pow((double)base, -2.0 * j / (double)rope_dim) / M_PI : 0.0;
}

unsigned int* err_word() {
  // filled once per device; concurrent first calls store the same address
  static std::atomic<unsigned int*> addr[kMaxDevices];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  unsigned int* a = addr[dev].load(std::memory_order_acquire);
  if (!a) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_err_word) != cudaSuccess) return nullptr;
    a = static_cast<unsigned int*>(p);
    addr[dev].store(a, std::memory_order_release);
  }
  return a;
}

// ---------------------------------------------------------------------------
// launch trace
// ---------------------------------------------------------------------------
namespace {
struct TraceRec {
  const char* name;
  cudaEvent_t e0, e1;
};
bool g_trace_on = false;
std::vector<TraceRec> g_trace;
std::vector<cudaEvent_t> g_event_pool;
size_t g_event_used = 0;

cudaEvent_t next_event() {
  if (g_event_used == g_event_pool.size()) {
    cudaEvent_t e;
    if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
    g_event_pool.push_back(e);
  }
  return g_event_pool[g_event_used++];
}
}  // namespace

TraceScope::TraceScope(const char* n, cudaStream_t s) : name(n), stream(s), slot(-1) {
  if (!g_trace_on) return;
  TraceRec r{n, next_event(), next_event()};
  if (!r.e0 || !r.e1) return;
  cudaEventRecord(r.e0, s);
  g_trace.push_back(r);
  slot = (int)g_trace.size() - 1;
}

TraceScope::~TraceScope() {
  if (slot >= 0) cudaEventRecord(g_trace[slot].e1, stream);
}

}  // namespace ds4a

using namespace ds4a;

namespace {

constexpr int kMxBlockApi = kMxBlock;

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int check_cfg(const ds4a_layer_cfg* c) {
  if (!c) return DS4A_EINVAL;
  if (c->n_heads < 1 || c->n_heads > 128) return DS4A_EINVAL;
  if (c->head_dim < 8 || c->head_dim > 512 || (c->head_dim % 8) != 0) return DS4A_EINVAL;
  if (c->rope_dim < 0 || c->rope_dim > c->head_dim || (c->rope_dim & 1)) return DS4A_EINVAL;
  if (c->window < 0 || c->ratio < 1) return DS4A_EINVAL;
  if (!(c->sm_scale > 0.f) || !(c->rope_base > 0.f) || !(c->rms_eps >= 0.f)) return DS4A_EINVAL;
  return DS4A_OK;
}

int check_index_cfg(const ds4a_layer_cfg* c) {
  if (!c) return DS4A_EINVAL;
  if (c->idx_heads < 1 || c->idx_heads > 128) return DS4A_EINVAL;
  if (c->idx_dim < 1 || c->idx_dim > 128) return DS4A_EINVAL;
  if (c->topk < 1 || c->topk > 4096 || c->ratio < 1) return DS4A_EINVAL;
  return DS4A_OK;
}

int cuda_rc(cudaError_t e) { return e == cudaSuccess ? DS4A_OK : DS4A_ECUDA; }

size_t index_ws_bytes(int B, int T_q, int N_c) {
  return (size_t)B * (size_t)T_q * (size_t)(N_c > 0 ? N_c : 0) * sizeof(float);
}

}  // namespace

extern "C" {

int ds4a_version(void) { return 100; }

const char* ds4a_strerror(int code) {
  switch (code) {
    case DS4A_OK: return "ok";
    case DS4A_EINVAL: return "invalid argument (null or misaligned pointer, bad size or config)";
    case DS4A_EUNSUPPORTED: return "unsupported shape";
    case DS4A_ECUDA: return "CUDA error";
    case DS4A_EDEVICE: return "device reported a bad index or position";
    case DS4A_ETIMEOUT: return "a bounded wait inside a kernel ran out";
    case DS4A_ENOSPACE: return "workspace too small";
    default: return "unknown error";
  }
}

int ds4a_compress(const ds4a_layer_cfg* cfg, int B, int T_tok, int tok_begin, int c,
                  const ds4a_bf16* ca, const ds4a_bf16* cb, const ds4a_bf16* za,
                  const ds4a_bf16* zb, const float* bias_a, const float* bias_b,
                  const float* norm_g, int entry_begin, int entry_end, ds4a_bf16* pool,
                  int64_t pool_bstride, ds4a_stream stream) {
  if (!cfg || cfg->ratio < 1) return DS4A_EINVAL;
  if (B < 0 || T_tok < 0 || c < 2 || c > 1024 || (c % 2) != 0) return DS4A_EINVAL;
  if ((c % 8) != 0 && c > 512) return DS4A_EINVAL;  // the 2-wide path covers up to 512
  if (entry_begin < 0 || entry_end < entry_begin) return DS4A_EINVAL;
  if (entry_end == entry_begin || B == 0) return DS4A_OK;
  if (!ca || !za || !bias_a || !pool) return DS4A_EINVAL;
  const bool overlap = cb != nullptr;
  if (overlap && (!zb || !bias_b)) return DS4A_EINVAL;
  if (!overlap && (zb || bias_b)) return DS4A_EINVAL;
  if (!aligned16(ca) || !aligned16(za) || !aligned16(bias_a) || !aligned16(pool)) return DS4A_EINVAL;
  if (overlap && (!aligned16(cb) || !aligned16(zb) || !aligned16(bias_b))) return DS4A_EINVAL;
  if (norm_g) {
    if (check_cfg(cfg) != DS4A_OK) return DS4A_EINVAL;
    if (cfg->rope_dim > c) return DS4A_EINVAL;
  }
  if (pool_bstride < (int64_t)entry_end * c || (pool_bstride % 2) != 0) return DS4A_EINVAL;
  const int m = cfg->ratio;
  // every token the entries read must be in the streams
  const int64_t first_tok = (overlap && entry_begin >= 1) ? (int64_t)(entry_begin - 1) * m
                                                          : (int64_t)entry_begin * m;
  const int64_t last_tok = (int64_t)entry_end * m - 1;
  if (first_tok < tok_begin || last_tok >= (int64_t)tok_begin + T_tok) return DS4A_EINVAL;

  CompressArgs a;
  a.B = B; a.T_tok = T_tok; a.tok_begin = tok_begin; a.c = c; a.m = m;
  a.rope_dim = norm_g ? cfg->rope_dim : 0;
  a.rope_base = cfg->rope_base; a.eps = cfg->rms_eps;
  a.ca = ca; a.cb = cb; a.za = za; a.zb = zb;
  a.bias_a = bias_a; a.bias_b = bias_b; a.norm_g = norm_g;
  a.entry_begin = entry_begin; a.entry_end = entry_end;
  a.pool = pool; a.pool_bstride = pool_bstride;
  a.app_pos = nullptr; a.ring = nullptr; a.ring_cap = 0; a.n_cap = 0;
  a.qfmt = 0; a.qpool = nullptr; a.q_bstride = 0; a.q_row = 0; a.qscales = nullptr; a.qs_bstride = 0;
  fill_rope_theta(&a.rope, a.rope_dim, cfg->rope_base);
  a.err = err_word();
  if (!a.err) return DS4A_ECUDA;
  return cuda_rc(launch_compress(a, (cudaStream_t)stream));
}

size_t ds4a_compress_state_bytes(const ds4a_layer_cfg* cfg, int B, int c, int overlap) {
  if (!cfg || cfg->ratio < 1 || B <= 0 || c <= 0) return 0;
  const size_t S = overlap ? 4 : 2, cap = overlap ? 2 * (size_t)cfg->ratio : (size_t)cfg->ratio;
  return (size_t)B * S * cap * (size_t)c * sizeof(uint16_t);
}

// the arguments of one append job, bf16 (qfmt 0) or block-scaled output
// (qfmt 1, 2), checked; DS4A_OK with *a filled, or an error (nothing to do:
// DS4A_OK with a->B == 0)
static int build_append_args(const ds4a_layer_cfg* cfg, int B, int c, const int32_t* pos,
                             const ds4a_bf16* ca, const ds4a_bf16* cb, const ds4a_bf16* za,
                             const ds4a_bf16* zb, const float* bias_a, const float* bias_b,
                             const float* norm_g, ds4a_bf16* state, int N_cap, ds4a_bf16* pool,
                             int64_t pool_bstride, int qfmt, uint8_t* qpool, uint8_t* qscales,
                             int64_t q_bstride_rows, CompressArgs* out) {
  out->B = 0;
  if (!cfg || cfg->ratio < 1) return DS4A_EINVAL;
  if (B < 0 || N_cap < 0 || c < 2 || c > 1024 || (c % 2) != 0) return DS4A_EINVAL;
  if ((c % 8) != 0 && c > 512) return DS4A_EINVAL;
  if (B == 0) return DS4A_OK;
  if (!pos || !ca || !za || !bias_a || !state) return DS4A_EINVAL;
  if (qfmt == 0 ? !pool : !qpool) return DS4A_EINVAL;
  if (qfmt == 2 && !qscales) return DS4A_EINVAL;
  const bool overlap = cb != nullptr;
  if (overlap && (!zb || !bias_b)) return DS4A_EINVAL;
  if (!overlap && (zb || bias_b)) return DS4A_EINVAL;
  if (!aligned16(pos) || !aligned16(ca) || !aligned16(za) || !aligned16(bias_a) || !aligned16(state) ||
      (pool && !aligned16(pool)) || (qpool && !aligned16(qpool)))
    return DS4A_EINVAL;
  if (overlap && (!aligned16(cb) || !aligned16(zb) || !aligned16(bias_b))) return DS4A_EINVAL;
  if (norm_g) {
    if (check_cfg(cfg) != DS4A_OK) return DS4A_EINVAL;
    if (cfg->rope_dim > c) return DS4A_EINVAL;
  }
  const int R = norm_g ? cfg->rope_dim : 0;
  if (qfmt == 0) {
    if (pool_bstride < (int64_t)N_cap * c || (pool_bstride % 2) != 0) return DS4A_EINVAL;
  } else {
    // 64-channel warps hold whole 32-channel blocks
    if (c % 64 != 0 || (c - R) % kMxBlockApi != 0 || q_bstride_rows < N_cap) return DS4A_EUNSUPPORTED;
  }
  const int m = cfg->ratio;
  if ((int64_t)(overlap ? 2 * m : m) * c > (int64_t)1 << 24) return DS4A_EINVAL;

  CompressArgs a;
  a.B = B; a.T_tok = 1; a.tok_begin = 0; a.c = c; a.m = m;
  a.rope_dim = norm_g ? cfg->rope_dim : 0;
  a.rope_base = cfg->rope_base; a.eps = cfg->rms_eps;
  a.ca = ca; a.cb = cb; a.za = za; a.zb = zb;
  a.bias_a = bias_a; a.bias_b = bias_b; a.norm_g = norm_g;
  a.entry_begin = 0; a.entry_end = 1;
  a.pool = pool; a.pool_bstride = pool_bstride;
  a.app_pos = pos; a.ring = state; a.ring_cap = overlap ? 2 * m : m; a.n_cap = N_cap;
  a.qfmt = qfmt; a.qpool = qpool; a.qscales = qscales;
  a.q_row = qfmt == 1 ? kv_fp8_row_bytes(c, R) : c / 2;
  a.q_bstride = q_bstride_rows * a.q_row;
  a.qs_bstride = q_bstride_rows * (c / kMxBlockApi);
  fill_rope_theta(&a.rope, a.rope_dim, cfg->rope_base);
  a.err = err_word();
  if (!a.err) return DS4A_ECUDA;
  *out = a;
  return DS4A_OK;
}

static int compress_append_common(const ds4a_layer_cfg* cfg, int B, int c, const int32_t* pos,
                                  const ds4a_bf16* ca, const ds4a_bf16* cb, const ds4a_bf16* za,
                                  const ds4a_bf16* zb, const float* bias_a, const float* bias_b,
                                  const float* norm_g, ds4a_bf16* state, int N_cap, ds4a_bf16* pool,
                                  int64_t pool_bstride, int qfmt, uint8_t* qpool, uint8_t* qscales,
                                  int64_t q_bstride_rows, ds4a_stream stream) {
  CompressArgs a;
  const int rc = build_append_args(cfg, B, c, pos, ca, cb, za, zb, bias_a, bias_b, norm_g, state, N_cap, pool,
                                   pool_bstride, qfmt, qpool, qscales, q_bstride_rows, &a);
  if (rc != DS4A_OK || a.B == 0) return rc;
  return cuda_rc(launch_compress(a, (cudaStream_t)stream));
}

int ds4a_compress_append_jobs(const ds4a_layer_cfg* cfg, int B, const int32_t* pos, int N_cap,
                              const ds4a_append_job* jobs, int n_jobs, ds4a_stream stream) {
  if (n_jobs < 0 || n_jobs > 2 || (n_jobs > 0 && !jobs)) return DS4A_EINVAL;
  CompressArgs a[2];
  int n = 0;
  for (int j = 0; j < n_jobs; ++j) {
    const ds4a_append_job& J = jobs[j];
    int qfmt = 0;
    if (J.format == DS4A_MX_KV_FP8) qfmt = 1;
    else if (J.format == DS4A_MX_IDX_FP4) qfmt = 2;
    else if (J.format != 0) return DS4A_EINVAL;
    const int rc = build_append_args(
        cfg, B, J.c, pos, J.ca, J.cb, J.za, J.zb, J.bias_a, J.bias_b, J.norm_g, J.state, N_cap,
        qfmt ? nullptr : static_cast<ds4a_bf16*>(J.pool), J.pool_bstride, qfmt,
        qfmt ? static_cast<uint8_t*>(J.pool) : nullptr, J.scales, J.pool_bstride, &a[n]);
    if (rc != DS4A_OK) return rc;
    if (a[n].B > 0) ++n;
  }
  if (n == 0) return DS4A_OK;
  return cuda_rc(launch_compress_jobs(a, n, (cudaStream_t)stream));
}

int ds4a_compress_append(const ds4a_layer_cfg* cfg, int B, int c, const int32_t* pos,
                         const ds4a_bf16* ca, const ds4a_bf16* cb, const ds4a_bf16* za,
                         const ds4a_bf16* zb, const float* bias_a, const float* bias_b,
                         const float* norm_g, ds4a_bf16* state, int N_cap, ds4a_bf16* pool,
                         int64_t pool_bstride, ds4a_stream stream) {
  return compress_append_common(cfg, B, c, pos, ca, cb, za, zb, bias_a, bias_b, norm_g, state, N_cap, pool,
                                pool_bstride, 0, nullptr, nullptr, 0, stream);
}

int ds4a_compress_append_mx(const ds4a_layer_cfg* cfg, int B, int c, const int32_t* pos,
                            const ds4a_bf16* ca, const ds4a_bf16* cb, const ds4a_bf16* za,
                            const ds4a_bf16* zb, const float* bias_a, const float* bias_b,
                            const float* norm_g, ds4a_bf16* state, int N_cap, int format, uint8_t* pool,
                            uint8_t* scales, int64_t pool_bstride, ds4a_stream stream) {
  if (format != DS4A_MX_KV_FP8 && format != DS4A_MX_IDX_FP4) return DS4A_EINVAL;
  return compress_append_common(cfg, B, c, pos, ca, cb, za, zb, bias_a, bias_b, norm_g, state, N_cap, nullptr, 0,
                                format == DS4A_MX_KV_FP8 ? 1 : 2, pool, scales, pool_bstride, stream);
}

size_t ds4a_kv_fp8_row_bytes(int D, int R) {
  if (D <= 0 || R < 0 || R > D || (D - R) % kMxBlockApi != 0 || (R % 8) != 0) return 0;
  return (size_t)kv_fp8_row_bytes(D, R);
}

int ds4a_quantize_kv_fp8(int n_rows, int D, int R, const ds4a_bf16* in, int64_t in_stride, uint8_t* out,
                         int64_t out_stride, ds4a_stream stream) {
  if (n_rows < 0 || ds4a_kv_fp8_row_bytes(D, R) == 0) return DS4A_EINVAL;
  if (n_rows == 0) return DS4A_OK;
  if (!in || !out || !aligned16(in) || !aligned16(out)) return DS4A_EINVAL;
  if (in_stride < D || in_stride % 8 != 0 || out_stride < kv_fp8_row_bytes(D, R) || out_stride % 16 != 0)
    return DS4A_EINVAL;
  return cuda_rc(launch_quant_kv_fp8(n_rows, D, R, in, in_stride, out, out_stride, (cudaStream_t)stream));
}

int ds4a_quantize_idx_fp4(int n_rows, int D, const ds4a_bf16* in, int64_t in_stride, uint8_t* codes,
                          uint8_t* scales, ds4a_stream stream) {
  if (n_rows < 0 || D <= 0 || D % kMxBlockApi != 0) return DS4A_EINVAL;
  if (n_rows == 0) return DS4A_OK;
  if (!in || !codes || !scales || !aligned16(in) || !aligned16(codes)) return DS4A_EINVAL;
  if (in_stride < D || in_stride % 8 != 0) return DS4A_EINVAL;
  return cuda_rc(launch_quant_idx_fp4(n_rows, D, in, in_stride, codes, scales, (cudaStream_t)stream));
}

size_t ds4a_index_topk_workspace(const ds4a_layer_cfg* cfg, int B, int T_q, int N_c) {
  (void)cfg;
  if (B <= 0 || T_q <= 0 || N_c <= 0) return 0;
  return index_ws_bytes(B, T_q, N_c);
}

int ds4a_index_topk(const ds4a_layer_cfg* cfg, int B, int T_q, const int32_t* q_pos,
                    const ds4a_bf16* q_idx, const ds4a_bf16* w_idx, const ds4a_bf16* k_idx,
                    int64_t k_bstride, int N_c, int32_t* idx_out, float* score_out, void* ws,
                    size_t ws_bytes, ds4a_stream stream) {
  if (check_index_cfg(cfg) != DS4A_OK) return DS4A_EINVAL;
  if (B < 0 || T_q < 0 || N_c < 0) return DS4A_EINVAL;
  if (B == 0 || T_q == 0) return DS4A_OK;
  if (!q_pos || !q_idx || !w_idx || !idx_out) return DS4A_EINVAL;
  if (N_c > 0 && (!k_idx || !ws)) return DS4A_EINVAL;
  if (!aligned16(q_pos) || !aligned16(q_idx) || !aligned16(w_idx) || !aligned16(idx_out))
    return DS4A_EINVAL;
  if ((k_idx && !aligned16(k_idx)) || (score_out && !aligned16(score_out)) || (ws && !aligned16(ws)))
    return DS4A_EINVAL;
  if (N_c > 0 && k_bstride < (int64_t)N_c * cfg->idx_dim) return DS4A_EINVAL;
  if (ws_bytes < index_ws_bytes(B, T_q, N_c)) return DS4A_ENOSPACE;

  IndexArgs a;
  a.B = B; a.T_q = T_q; a.H = cfg->idx_heads; a.D = cfg->idx_dim; a.m = cfg->ratio;
  a.k = cfg->topk; a.N_c = N_c;
  a.q_pos = q_pos; a.q = q_idx; a.w = w_idx; a.kidx = k_idx; a.k_bstride = k_bstride;
  a.kcodes = nullptr; a.kscales = nullptr;
  a.scores = reinterpret_cast<float*>(ws);
  a.idx_out = idx_out; a.score_out = score_out;
  a.err = err_word();
  if (!a.err) return DS4A_ECUDA;
  cudaStream_t s = (cudaStream_t)stream;
  cudaError_t e = cudaSuccess;
  if (N_c > 0) {
    e = index_scores_tc_supported(a) ? launch_index_scores_tc(a, s) : launch_index_scores_generic(a, s);
    if (e != cudaSuccess) return DS4A_ECUDA;
  }
  return cuda_rc(launch_topk(a, s));
}

int ds4a_index_topk_fp4(const ds4a_layer_cfg* cfg, int B, int T_q, const int32_t* q_pos,
                        const ds4a_bf16* q_idx, const ds4a_bf16* w_idx, const uint8_t* k_codes,
                        const uint8_t* k_scales, int64_t k_bstride, int N_c, int32_t* idx_out,
                        float* score_out, void* ws, size_t ws_bytes, ds4a_stream stream) {
  if (check_index_cfg(cfg) != DS4A_OK) return DS4A_EINVAL;
  if (B < 0 || T_q < 0 || N_c < 0) return DS4A_EINVAL;
  if (B == 0 || T_q == 0) return DS4A_OK;
  if (!q_pos || !q_idx || !w_idx || !idx_out) return DS4A_EINVAL;
  if (N_c > 0 && (!k_codes || !k_scales || !ws)) return DS4A_EINVAL;
  if (!aligned16(q_pos) || !aligned16(q_idx) || !aligned16(w_idx) || !aligned16(idx_out)) return DS4A_EINVAL;
  if ((k_codes && !aligned16(k_codes)) || (k_scales && !aligned16(k_scales)) ||
      (score_out && !aligned16(score_out)) || (ws && !aligned16(ws)))
    return DS4A_EINVAL;
  if (N_c > 0 && k_bstride < N_c) return DS4A_EINVAL;
  if (ws_bytes < index_ws_bytes(B, T_q, N_c)) return DS4A_ENOSPACE;
  IndexArgs a;
  a.B = B; a.T_q = T_q; a.H = cfg->idx_heads; a.D = cfg->idx_dim; a.m = cfg->ratio;
  a.k = cfg->topk; a.N_c = N_c;
  a.q_pos = q_pos; a.q = q_idx; a.w = w_idx; a.kidx = nullptr; a.k_bstride = k_bstride;
  a.kcodes = k_codes; a.kscales = k_scales;
  a.scores = reinterpret_cast<float*>(ws);
  a.idx_out = idx_out; a.score_out = score_out;
  // the tensor-core scorer with its FP4 converters is the only FP4 path
  if (N_c > 0 && !index_scores_tc_supported(a)) return DS4A_EUNSUPPORTED;
  a.err = err_word();
  if (!a.err) return DS4A_ECUDA;
  cudaStream_t s = (cudaStream_t)stream;
  if (N_c > 0 && launch_index_scores_tc(a, s) != cudaSuccess) return DS4A_ECUDA;
  return cuda_rc(launch_topk(a, s));
}

size_t ds4a_attend_workspace(const ds4a_layer_cfg* cfg, int B, int T_q, int N_c, int sparse) {
  if (check_cfg(cfg) != DS4A_OK || B <= 0 || T_q <= 0) return 0;
  const int keys_max = (sparse ? cfg->topk : (N_c > 0 ? N_c : 0)) + cfg->window;
  AttendArgs probe{};
  probe.H = cfg->n_heads; probe.D = cfg->head_dim; probe.R = cfg->rope_dim;
  size_t need = 0;
  attend_splits(B, T_q, keys_max, cfg->n_heads, cfg->head_dim, attend_tc_supported(probe), (size_t)-1,
                &need);
  return need;
}

static int attend_common(const ds4a_layer_cfg* cfg, int B, int T_q, const int32_t* q_pos,
                         const ds4a_bf16* q, const float* q_norm_g, const ds4a_bf16* pool,
                         int64_t pool_bstride, int N_c, const int32_t* idx, const ds4a_bf16* win,
                         int win_cap, int64_t win_bstride, const float* sink, ds4a_bf16* out,
                         void* ws, size_t ws_bytes, ds4a_stream stream, int sparse,
                         const uint8_t* pool8 = nullptr) {
  const int64_t bstride8 = pool_bstride;  // rows, for FP8 pools
  if (pool8) {
    // mixed FP8 / BF16 rows: the tensor-core path of the Flash shape only
    if (!cfg || cfg->n_heads != 64 || cfg->head_dim != 512 || cfg->rope_dim != 64) return DS4A_EUNSUPPORTED;
    if (!aligned16(pool8) || (N_c > 0 && pool_bstride < N_c)) return DS4A_EINVAL;
    pool = reinterpret_cast<const ds4a_bf16*>(pool8);  // for the checks below
    pool_bstride = (int64_t)N_c * cfg->head_dim;
  }
  if (check_cfg(cfg) != DS4A_OK) return DS4A_EINVAL;
  if (sparse && (cfg->topk < 1 || cfg->topk > 4096)) return DS4A_EINVAL;
  if (B < 0 || T_q < 0 || N_c < 0) return DS4A_EINVAL;
  if (B == 0 || T_q == 0) return DS4A_OK;
  if (!q_pos || !q || !q_norm_g || !sink || !out) return DS4A_EINVAL;
  if (N_c > 0 && !pool) return DS4A_EINVAL;
  if (sparse && !idx) return DS4A_EINVAL;
  if (cfg->window > 0 && (!win || win_cap < cfg->window)) return DS4A_EINVAL;
  if (!aligned16(q_pos) || !aligned16(q) || !aligned16(q_norm_g) || !aligned16(sink) || !aligned16(out))
    return DS4A_EINVAL;
  if ((pool && !aligned16(pool)) || (idx && !aligned16(idx)) || (win && !aligned16(win)) ||
      (ws && !aligned16(ws)))
    return DS4A_EINVAL;
  const int D = cfg->head_dim;
  if (N_c > 0 && (pool_bstride < (int64_t)N_c * D || (pool_bstride % 8) != 0)) return DS4A_EINVAL;
  if (cfg->window > 0 && (win_bstride < (int64_t)win_cap * D || (win_bstride % 8) != 0))
    return DS4A_EINVAL;
  if (ws_bytes > 0 && !ws) return DS4A_EINVAL;

  const size_t have = ws ? ws_bytes : 0;
  AttendArgs a;
  a.B = B; a.T_q = T_q; a.H = cfg->n_heads; a.D = D; a.R = cfg->rope_dim; a.W = cfg->window;
  a.m = cfg->ratio; a.k = cfg->topk; a.N_c = N_c; a.win_cap = win_cap; a.sparse = sparse;
  a.scale = cfg->sm_scale; a.rope_base = cfg->rope_base; a.eps = cfg->rms_eps;
  a.q_pos = q_pos; a.q = q; a.q_norm_g = q_norm_g; a.pool = pool; a.pool_bstride = pool_bstride;
  a.pool8 = pool8;
  if (pool8) a.pool_bstride = bstride8;
  a.idx = idx; a.win = win; a.win_bstride = win_bstride; a.sink = sink; a.out = out;
  a.ws = reinterpret_cast<float*>(ws);
  a.keys_max = (sparse ? cfg->topk : N_c) + cfg->window;
  // the shape decides the kernel: 64 heads x 512 run on the tensor cores and
  // need the prepared-query workspace (no silent second path); other shapes
  // run the CUDA-core kernel
  const bool tc = attend_tc_supported(a);
  a.n_splits = attend_splits(B, T_q, a.keys_max, a.H, a.D, tc, have, nullptr);
  if (tc && a.n_splits == 0) return DS4A_ENOSPACE;
  fill_rope_theta(&a.rope, a.R, cfg->rope_base);
  a.err = err_word();
  if (!a.err) return DS4A_ECUDA;
  cudaStream_t s = (cudaStream_t)stream;
  return cuda_rc(tc ? launch_attend_tc(a, s) : launch_attend_generic(a, s));
}

int ds4a_sparse_attend(const ds4a_layer_cfg* cfg, int B, int T_q, const int32_t* q_pos,
                       const ds4a_bf16* q, const float* q_norm_g, const ds4a_bf16* pool,
                       int64_t pool_bstride, int N_c, const int32_t* idx, const ds4a_bf16* win,
                       int win_cap, int64_t win_bstride, const float* sink, ds4a_bf16* out,
                       void* ws, size_t ws_bytes, ds4a_stream stream) {
  return attend_common(cfg, B, T_q, q_pos, q, q_norm_g, pool, pool_bstride, N_c, idx, win, win_cap,
                       win_bstride, sink, out, ws, ws_bytes, stream, 1);
}

int ds4a_hca_attend(const ds4a_layer_cfg* cfg, int B, int T_q, const int32_t* q_pos,
                    const ds4a_bf16* q, const float* q_norm_g, const ds4a_bf16* pool,
                    int64_t pool_bstride, int N_c, const ds4a_bf16* win, int win_cap,
                    int64_t win_bstride, const float* sink, ds4a_bf16* out, void* ws,
                    size_t ws_bytes, ds4a_stream stream) {
  return attend_common(cfg, B, T_q, q_pos, q, q_norm_g, pool, pool_bstride, N_c, nullptr, win,
                       win_cap, win_bstride, sink, out, ws, ws_bytes, stream, 0);
}

static int check_oproj(const ds4a_oproj_cfg* c) {
  if (!c) return DS4A_EINVAL;
  if (c->n_heads < 1 || c->head_dim < 1 || c->n_groups < 1 || c->group_rank < 1 || c->hidden < 1)
    return DS4A_EINVAL;
  if (c->n_heads % c->n_groups != 0) return DS4A_EINVAL;
  const int64_t k1 = (int64_t)(c->n_heads / c->n_groups) * c->head_dim;
  if (k1 % 64 != 0 || c->group_rank % 256 != 0 || c->hidden % 256 != 0) return DS4A_EUNSUPPORTED;
  if (k1 > (1 << 20) || (int64_t)c->n_groups * c->group_rank > (1 << 20) || c->hidden > (1 << 20))
    return DS4A_EUNSUPPORTED;
  return DS4A_OK;
}

size_t ds4a_out_proj_workspace(const ds4a_oproj_cfg* cfg, int M) {
  if (check_oproj(cfg) != DS4A_OK || M <= 0) return 0;
  const int k1 = (cfg->n_heads / cfg->n_groups) * cfg->head_dim;
  const int n1 = cfg->n_groups * cfg->group_rank;
  const size_t a = gemm_acc_bytes(M, n1, k1), b = gemm_acc_bytes(M, cfg->hidden, n1);
  return a > b ? a : b;
}

int ds4a_out_proj(const ds4a_oproj_cfg* cfg, int M, const ds4a_bf16* o, const ds4a_bf16* w_a,
                  const ds4a_bf16* w_b, ds4a_bf16* mid, ds4a_bf16* y, void* ws, size_t ws_bytes,
                  ds4a_stream stream) {
  const int rc = check_oproj(cfg);
  if (rc != DS4A_OK) return rc;
  if (M < 0) return DS4A_EINVAL;
  if (M == 0) return DS4A_OK;
  if (!o || !w_a || !w_b || !mid || !y) return DS4A_EINVAL;
  if (!aligned16(o) || !aligned16(w_a) || !aligned16(w_b) || !aligned16(mid) || !aligned16(y) ||
      (ws && !aligned16(ws)))
    return DS4A_EINVAL;
  if (ws_bytes > 0 && !ws) return DS4A_EINVAL;
  if ((ws ? ws_bytes : 0) < ds4a_out_proj_workspace(cfg, M)) return DS4A_ENOSPACE;
  unsigned int* err = err_word();
  if (!err) return DS4A_ECUDA;
  const int H = cfg->n_heads, D = cfg->head_dim, g = cfg->n_groups, r = cfg->group_rank;
  const int k1 = (H / g) * D, n1 = g * r;
  cudaStream_t s = (cudaStream_t)stream;
  float* acc = reinterpret_cast<float*>(ws);
  // mid[t][j r + i] = W_a[j][i] . o[t][j K1 .. (j+1) K1)
  cudaError_t e = launch_gemm(o, (int64_t)H * D, (int64_t)H * D, w_a, M, n1, k1, r, k1, mid, n1, acc, err, s);
  if (e != cudaSuccess) return DS4A_ECUDA;
  // y[t][n] = W_b[n] . mid[t]
  e = launch_gemm(mid, n1, n1, w_b, M, cfg->hidden, n1, cfg->hidden, 0, y, cfg->hidden, acc, err, s);
  return cuda_rc(e);
}

int ds4a_sparse_attend_fp8(const ds4a_layer_cfg* cfg, int B, int T_q, const int32_t* q_pos,
                           const ds4a_bf16* q, const float* q_norm_g, const uint8_t* pool,
                           int64_t pool_bstride, int N_c, const int32_t* idx, const ds4a_bf16* win,
                           int win_cap, int64_t win_bstride, const float* sink, ds4a_bf16* out,
                           void* ws, size_t ws_bytes, ds4a_stream stream) {
  if (N_c > 0 && !pool) return DS4A_EINVAL;
  return attend_common(cfg, B, T_q, q_pos, q, q_norm_g, nullptr, pool_bstride, N_c, idx, win, win_cap,
                       win_bstride, sink, out, ws, ws_bytes, stream, 1, N_c > 0 ? pool : nullptr);
}

int ds4a_hca_attend_fp8(const ds4a_layer_cfg* cfg, int B, int T_q, const int32_t* q_pos,
                        const ds4a_bf16* q, const float* q_norm_g, const uint8_t* pool,
                        int64_t pool_bstride, int N_c, const ds4a_bf16* win, int win_cap,
                        int64_t win_bstride, const float* sink, ds4a_bf16* out, void* ws,
                        size_t ws_bytes, ds4a_stream stream) {
  if (N_c > 0 && !pool) return DS4A_EINVAL;
  return attend_common(cfg, B, T_q, q_pos, q, q_norm_g, nullptr, pool_bstride, N_c, nullptr, win, win_cap,
                       win_bstride, sink, out, ws, ws_bytes, stream, 0, N_c > 0 ? pool : nullptr);
}

int ds4a_check(ds4a_stream stream, uint32_t* bits_out) {
  if (bits_out) *bits_out = 0;
  cudaError_t e = cudaStreamSynchronize((cudaStream_t)stream);
  if (e != cudaSuccess) return DS4A_ECUDA;
  unsigned int bits = 0;
  if (cudaMemcpyFromSymbol(&bits, g_err_word, sizeof(bits)) != cudaSuccess) return DS4A_ECUDA;
  if (bits) {
    const unsigned int zero = 0;
    if (cudaMemcpyToSymbol(g_err_word, &zero, sizeof(zero)) != cudaSuccess) return DS4A_ECUDA;
  }
  if (bits_out) *bits_out = bits;
  if (bits & DS4A_DEV_TIMEOUT) return DS4A_ETIMEOUT;
  if (bits) return DS4A_EDEVICE;
  return cuda_rc(cudaGetLastError());
}

int ds4a_trace_enable(int on) {
  g_trace_on = on != 0;
  g_trace.clear();
  g_event_used = 0;
  return DS4A_OK;
}

int ds4a_trace_read(const char** names, float* ms, int cap) {
  if (cudaDeviceSynchronize() != cudaSuccess) return -DS4A_ECUDA;
  const int n = (int)g_trace.size();
  for (int i = 0; i < n && i < cap; ++i) {
    if (names) names[i] = g_trace[i].name;
    float t = 0.f;
    cudaEventElapsedTime(&t, g_trace[i].e0, g_trace[i].e1);
    if (ms) ms[i] = t;
  }
  return n;
}

}  // extern "C"
