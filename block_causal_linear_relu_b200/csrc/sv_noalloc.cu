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
//  - all calls on a device share the one array, which keeps the previous call's contents (the
//    status word, the one-launch kernel's sequence number and flags): calls that may overlap on the
//    GPU (different streams without ordering) race on it;
//  - the first call on each device (or of sv_cache_step_noalloc_status) looks up the array's device
//    address with that device current and keeps it for the life of the process; make that first
//    call before any stream capture begins. After cudaDeviceReset the kept address is stale: the
//    entry point is not supported across a device reset.
//  - a bounded wait that expires raises the array's status word, which stays raised (later calls
//    then give up their waits at once) until sv_cache_step_noalloc_status reads and clears it.
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

// Device address of the scratch on the current device, looked up once per device.
sv_status scratch_address(void** out, const char* who) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    char msg[160];
    snprintf(msg, sizeof(msg), "%s: no usable current device", who);
    return sv::set_last_error(SV_ERR_CUDA, msg);
  }
  std::lock_guard<std::mutex> lock(g_mu);
  if (g_scratch_addr[dev] == nullptr) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || p == nullptr) {
      char msg[200];
      snprintf(msg, sizeof(msg), "%s: cudaGetSymbolAddress of the static scratch failed (%s)", who,
               cudaGetErrorName(e));
      return sv::set_last_error(SV_ERR_CUDA, msg);
    }
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return SV_OK;
}

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
  void* ws = nullptr;
  const sv_status s = scratch_address(&ws, "sv_cache_step_noalloc");
  if (s != SV_OK) return s;
  // Nothing is written here: the array starts zeroed when the library loads, the status word is
  // cleared only by sv_cache_step_noalloc_status, the launch sequence number and the flags behind it
  // keep their values from call to call, and the rest is rewritten by each call. sv_cache_step
  // checks every argument before it launches anything.
  return sv_cache_step(q, k, v, o, B, H, N, D, dt, eps, S, z, commit, ws, kNoAllocScratchBytes, stream);
}

extern "C" sv_status sv_cache_step_noalloc_status(sv_stream_t stream, uint32_t* code) {
  void* ws = nullptr;
  const sv_status s = scratch_address(&ws, "sv_cache_step_noalloc_status");
  if (s != SV_OK) return s;
  return sv_device_status(ws, stream, code);
}
