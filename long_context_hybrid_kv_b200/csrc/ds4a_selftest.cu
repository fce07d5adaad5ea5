// Failure-detection self test: one block waits on an mbarrier that no thread
// arrives at, through the bounded wait of the tensor-core kernels, with a
// short limit.  The wait runs out, the block records DS4A_DEV_TIMEOUT and
// exits; the host reads the error word with ds4a_check.
#include "ds4a_tc.cuh"

namespace ds4a {
namespace {

using namespace tc;

__global__ void wait_timeout_probe_kernel(long long limit, unsigned int* err, int32_t* status) {
  __shared__ __align__(8) unsigned long long bar;
  __shared__ int abort_flag;
  const uint32_t b = smem_u32(&bar);
  if (threadIdx.x == 0) {
    abort_flag = 0;
    mbar_init(b, 1);
    fence_barrier_init();
  }
  __syncthreads();
  // phase 0 never completes: nothing arrives on the barrier
  const bool done = mbar_wait(b, 0, &abort_flag, err, limit);
  __syncthreads();
  if (threadIdx.x == 0) *status = done ? 1 : 2;
}

}  // namespace
}  // namespace ds4a

extern "C" int ds4a_selftest_wait_timeout(int64_t limit_cycles, int32_t* status_out, ds4a_stream stream) {
  if (limit_cycles < 1 || limit_cycles > (int64_t(1) << 32) || !status_out) return DS4A_EINVAL;
  if ((reinterpret_cast<uintptr_t>(status_out) & 3u) != 0) return DS4A_EINVAL;
  unsigned int* err = ds4a::err_word();
  if (!err) return DS4A_ECUDA;
  ds4a::wait_timeout_probe_kernel<<<1, 32, 0, (cudaStream_t)stream>>>((long long)limit_cycles, err, status_out);
  return cudaGetLastError() == cudaSuccess ? DS4A_OK : DS4A_ECUDA;
}
