// Self-test of the failure path of the device-side waits.
//
// One kernel makes the two kinds of bounded wait used by the layer's kernels
// run out on purpose, with a short limit: an mbarrier phase that nothing
// completes (the wait of the GEMM pipelines) and a look-back word that no block
// publishes (the wait of the permutation scan).  Each must give up, record
// MOE_ERR_TIMEOUT in the workspace status word and return; the kernel then
// exits normally and the context stays usable.
#include <cstdint>

#include "moe_internal.h"
#include "sm100.cuh"

namespace moe {

__global__ void __launch_bounds__(64) wait_timeout_selftest_kernel(uint32_t* status, const uint32_t* never_word,
                                                                   uint64_t limit_ns, uint32_t* gave_up) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    if (!mbar_wait(&bar, 0, nullptr, limit_ns)) {  // nothing ever arrives
      record_status(status, kStatusTimeout);
      atomicAdd(gave_up, 1u);
    }
  } else if (threadIdx.x == 32) {
    uint32_t v;
    if (!wait_published(never_word, 0xC0000000u, &v, limit_ns)) {  // nothing publishes
      record_status(status, kStatusTimeout);
      atomicAdd(gave_up, 1u);
    }
  }
}

}  // namespace moe

extern "C" moe_status moe_selftest_wait_timeout(void* ws, size_t ws_bytes, uint32_t limit_us, moe_stream_t stream) {
  using namespace moe;
  if (!ws || (reinterpret_cast<uintptr_t>(ws) % 256) != 0 || ws_bytes < 256) return MOE_ERR_WORKSPACE;
  if (limit_us == 0 || limit_us > 10u * 1000u * 1000u) return MOE_ERR_INVALID_ARG;
  int sms = 0;
  moe_status st = api_check_device(&sms);
  if (st != MOE_OK) return st;
  cudaStream_t s = (cudaStream_t)stream;
  // word 0: status; word 16: the never-published look-back word; word 32: count of waits that gave up
  uint32_t* w = static_cast<uint32_t*>(ws);
  if (cudaMemsetAsync(ws, 0, 256, s) != cudaSuccess) return MOE_ERR_CUDA;
  wait_timeout_selftest_kernel<<<1, 64, 0, s>>>(w, w + 16, (uint64_t)limit_us * 1000ull, w + 32);
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}
