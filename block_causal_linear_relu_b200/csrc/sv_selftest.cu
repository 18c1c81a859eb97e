// sv_selftest_wait_timeout: exercises the failure path of the kernels' bounded waits without any
// GPU fault. One CTA of four warps waits, through the same mbar_wait routine every pipeline role
// uses, on an mbarrier phase that nothing completes. The first waiter to pass kWaitLimitNs raises
// the workspace status word (kDevTimeout | 0x7E00 | warp); the other waiters see the raised word
// and give up at once, as the waiters of a real pipeline do, and the kernel returns normally. The
// CTA holds no TMEM and issues no asynchronous copies, so nothing is left in flight. The host then
// reads SV_ERR_TIMEOUT through sv_device_status and the context stays usable.
#include <cuda_runtime.h>

#include "../../include/svlinattn.h"
#include "sv_internal.h"
#include "sv_ptx.cuh"

namespace {

constexpr uint32_t kSelftestWhere = 0x7E00u;

__global__ void __launch_bounds__(128, 1) selftest_wait_kernel(uint32_t* status) {
  __shared__ __align__(8) uint64_t bar;
  const int warp = threadIdx.x >> 5;
  if (threadIdx.x == 0) {
    sv::mbar_init(&bar, 1);  // one arrival would complete phase 0; none is ever made
    sv::fence_mbar_init();
  }
  __syncthreads();
  if ((threadIdx.x & 31) == 0) sv::mbar_wait(&bar, 0, status, kSelftestWhere | static_cast<uint32_t>(warp));
}

}  // namespace

extern "C" sv_status sv_selftest_wait_timeout(void* ws, size_t ws_bytes, sv_stream_t stream) {
  if (ws == nullptr || ws_bytes < static_cast<size_t>(sv::kHeaderBytes) ||
      (reinterpret_cast<uintptr_t>(ws) & 255u) != 0u)
    return sv::set_last_error(
        SV_ERR_INVALID_ARG, "sv_selftest_wait_timeout: ws must be a 256-byte aligned workspace of at least 256 bytes");
  selftest_wait_kernel<<<1, 128, 0, reinterpret_cast<cudaStream_t>(stream)>>>(static_cast<uint32_t*>(ws));
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return sv::set_last_error(SV_ERR_CUDA, cudaGetErrorString(e));
  return SV_OK;
}
