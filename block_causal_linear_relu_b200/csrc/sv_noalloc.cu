// sv_cache_step_noalloc: the streaming cache step for callers that cannot allocate device memory.
//
// Some callers are not allowed to allocate: an operator running inside a host framework's enqueue
// callback (a plugin interface whose memory is owned by the host), a real-time generation loop that
// must not call cudaMalloc between blocks because it synchronises the device and stalls the stream,
// or code that records its work into a CUDA graph, where allocation calls are not permitted while
// recording. Those callers cannot provide the caller-owned workspace that sv_cache_step asks for.
// This entry point takes its scratch from a fixed array compiled into the library instead; the
// caller still passes q, k, v, o and the cache (S, z).
//
// Costs and rules, stated once here and in include/svlinattn.h:
//  - every device that loads the library holds kNoAllocScratchBytes (16 MiB) of device memory for
//    this array until the process exits, whether or not the entry point is used;
//  - a call whose workspace need (sv_workspace_bytes(SV_OP_CACHE_STEP, ...)) exceeds the array is
//    refused with SV_ERR_INVALID_ARG before anything is launched;
//  - all calls on a device share the one array, which keeps the previous call's contents: calls
//    that may overlap on the GPU (different streams without ordering) race on it;
//  - the first call on each device looks up the array's device address with that device current;
//    make that first call before any stream capture begins.
#include <cuda_runtime.h>

#include <cstdio>
#include <mutex>

#include "../../include/svlinattn.h"
#include "sv_internal.h"

namespace {

constexpr size_t kNoAllocScratchBytes = static_cast<size_t>(16) << 20;  // 16 MiB per device

// The scratch itself. In host code this name is only a stand-in for the symbol; the device address
// comes from cudaGetSymbolAddress below and is what the kernels receive.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_scratch_addr[kMaxDevices] = {};

}  // namespace

extern "C" sv_status sv_cache_step_noalloc(const void* q, const void* k, const void* v, void* o, int B, int H, int N,
                                           int D, sv_dtype dt, float eps, float* S, float* z, int commit,
                                           sv_stream_t stream) {
  const size_t need = sv_workspace_bytes(SV_OP_CACHE_STEP, B, H, N, D, N, dt);
  if (need == 0) return SV_ERR_INVALID_ARG;  // sizes refused; sv_last_error() says why
  if (need > kNoAllocScratchBytes) {
    char msg[256];
    snprintf(msg, sizeof(msg),
             "sv_cache_step_noalloc: this block needs %zu bytes of scratch; the library's static scratch "
             "holds %zu bytes (use sv_cache_step with a caller-owned workspace)",
             need, kNoAllocScratchBytes);
    return sv::set_last_error(SV_ERR_INVALID_ARG, msg);
  }
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices)
    return sv::set_last_error(SV_ERR_CUDA, "sv_cache_step_noalloc: no usable current device");
  void* ws = nullptr;
  {
    std::lock_guard<std::mutex> lock(g_mu);
    if (g_scratch_addr[dev] == nullptr) {
      void* p = nullptr;
      const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
      if (e != cudaSuccess || p == nullptr)
        return sv::set_last_error(SV_ERR_CUDA,
                                  "sv_cache_step_noalloc: cudaGetSymbolAddress of the static scratch failed");
      g_scratch_addr[dev] = p;
    }
    ws = g_scratch_addr[dev];
  }
  // the status word must start at zero; the launch sequence number and the flags behind it keep
  // their values from call to call (the array starts zeroed when the library loads), and the rest is
  // fully rewritten by each call
  if (cudaMemsetAsync(ws, 0, sizeof(uint32_t), reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
    return sv::set_last_error(SV_ERR_CUDA, "sv_cache_step_noalloc: clearing the scratch header failed");
  return sv_cache_step(q, k, v, o, B, H, N, D, dt, eps, S, z, commit, ws, kNoAllocScratchBytes, stream);
}
