// ds4a_index_topk_noalloc: the indexer top-k for callers that cannot allocate
// device memory.  Some hosts give a library no way to allocate: inference
// engines that reserve all of HBM for their KV caches at start-up and refuse
// later cudaMalloc calls, plugin hosts with a C interface that hand the
// library no allocator, and decode loops that cannot afford the implicit
// device synchronisation cudaMalloc / cudaFree may cause.  This entry point
// needs no workspace from them: the score scratch is a file-scope device
// array of this library, sized for 2^21 scores (8 MiB, B * T_q * N_c <=
// 2097152), which every GPU that loads the library holds until the process
// exits.
#include "ds4a_internal.cuh"

namespace ds4a {
namespace {

constexpr size_t kNoAllocScores = size_t(1) << 21;

// Shared by every call on a device; each call writes every score it later
// reads, so nothing needs clearing between calls.
static __device__ __align__(256) float g_topk_scratch[kNoAllocScores];

// In host code g_topk_scratch names a host-side stand-in, not device
// memory: the kernels get the device address looked up here, once per
// device, with that device current.
float* scratch_for_current_device(int* rc) {
  // filled once per device; concurrent first calls store the same address
  static std::atomic<float*> addr[kMaxDevices];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    *rc = DS4A_ECUDA;
    return nullptr;
  }
  float* a = addr[dev].load(std::memory_order_acquire);
  if (!a) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_topk_scratch);
    if (e != cudaSuccess || p == nullptr) {
      (void)cudaGetLastError();
      *rc = DS4A_ECUDA;
      return nullptr;
    }
    a = static_cast<float*>(p);
    addr[dev].store(a, std::memory_order_release);
  }
  *rc = DS4A_OK;
  return a;
}

}  // namespace
}  // namespace ds4a

extern "C" int ds4a_index_topk_noalloc(const ds4a_layer_cfg* cfg, int B, int T_q,
                                       const int32_t* q_pos, const ds4a_bf16* q_idx,
                                       const ds4a_bf16* w_idx, const ds4a_bf16* k_idx,
                                       int64_t k_bstride, int N_c, int32_t* idx_out,
                                       float* score_out, ds4a_stream stream) {
  if (B < 0 || T_q < 0 || N_c < 0) return DS4A_EINVAL;
  const size_t n_scores = (size_t)B * (size_t)T_q * (size_t)N_c;
  if (n_scores > ds4a::kNoAllocScores) return DS4A_ENOSPACE;
  // no scores to write: the scratch is not needed, so its address is not
  // looked up (such a call may come first and inside a stream capture)
  if (n_scores == 0)
    return ds4a_index_topk(cfg, B, T_q, q_pos, q_idx, w_idx, k_idx, k_bstride, N_c, idx_out, score_out,
                           nullptr, 0, stream);
  int rc = DS4A_OK;
  float* scratch = ds4a::scratch_for_current_device(&rc);
  if (rc != DS4A_OK) return rc;
  return ds4a_index_topk(cfg, B, T_q, q_pos, q_idx, w_idx, k_idx, k_bstride, N_c, idx_out,
                         score_out, scratch, ds4a::kNoAllocScores * sizeof(float), stream);
}
