// Block-causal temporal convolution of SANA-Video's causal Mix-FFN, sm_100a.
//
// The talk ("SANA-Video: Efficient Video Generation with Block Linear Diffusion Transformer", causal
// FFN with temporal conv passage) makes the temporal convolution causal across blocks: a zero token
// is padded between two blocks (block 1 cannot see block 2), and block 2 takes block 1's last token
// as its first token (block 2 sees block 1); both are dropped after the convolution. With a centred
// depthwise kernel of width 3 along time this gives, for frame t of block blk(t):
//
//     y[t] = w0 * x[t-1] + w1 * x[t] + w2 * x[t+1] * [blk(t+1) == blk(t)] + b,   x[-1] = 0 (or the
//            carried frame of the previous block when the call is one block of a stream)
//
// x, y are [B, T, S, C] (T frames of S tokens, C channels; C fastest). The operation is a stencil
// along T with nothing to contract, so it is bound by HBM: each thread owns one 16-byte column
// (8 bf16 or 4 fp32 channels of one token of one batch) and walks the frames with the three-frame
// window in registers, so x is read once and y written once; consecutive threads take consecutive
// channel groups, so every frame's access is a contiguous 512-byte run per warp. Loads run eight
// frames ahead of the stores.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdio>

#include "../../include/svlinattn.h"
#include "sv_internal.h"

namespace {

constexpr int kConvThreads = 256;
constexpr int kAhead = 8;  // frames loaded ahead of the stores

template <typename T>
struct Vec16;
template <>
struct Vec16<__nv_bfloat16> {
  static constexpr int N = 8;
  __device__ static void to_float(const uint4& r, float (&f)[8]) {
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&r);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 p = __bfloat1622float2(h[i]);
      f[2 * i] = p.x;
      f[2 * i + 1] = p.y;
    }
  }
  __device__ static uint4 from_float(const float (&f)[8]) {
    uint4 r;
    __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&r);
#pragma unroll
    for (int i = 0; i < 4; ++i) h[i] = __floats2bfloat162_rn(f[2 * i], f[2 * i + 1]);
    return r;
  }
};
template <>
struct Vec16<float> {
  static constexpr int N = 4;
  __device__ static void to_float(const uint4& r, float (&f)[4]) {
    f[0] = __uint_as_float(r.x);
    f[1] = __uint_as_float(r.y);
    f[2] = __uint_as_float(r.z);
    f[3] = __uint_as_float(r.w);
  }
  __device__ static uint4 from_float(const float (&f)[4]) {
    return make_uint4(__float_as_uint(f[0]), __float_as_uint(f[1]), __float_as_uint(f[2]), __float_as_uint(f[3]));
  }
};

// One thread per (batch, token, 16-byte channel group). `carry` (nullable) holds, per (batch, token),
// the frame before x[0]; with `commit` it then receives x's last frame (the same thread reads it
// first, so the update is in place without a race).
template <typename T>
__global__ void __launch_bounds__(kConvThreads) temporal_conv_kernel(const T* x, T* y, int B, int Tf, int S, int C,
                                                                     int L, const float* __restrict__ w,
                                                                     const float* __restrict__ bias, T* carry,
                                                                     int commit, long long ncols) {
  using V = Vec16<T>;
  constexpr int NV = V::N;
  const long long col = static_cast<long long>(blockIdx.x) * kConvThreads + threadIdx.x;
  if (col >= ncols) return;
  const int per_row = C / NV;
  const long long bs = col / per_row;  // b * S + s
  const int c0 = static_cast<int>(col - bs * per_row) * NV;
  const int b = static_cast<int>(bs / S);
  const int s = static_cast<int>(bs - static_cast<long long>(b) * S);
  // the group's 3 * NV taps are contiguous (16-byte aligned: NV * 12 bytes per group), as are its NV
  // biases: vector loads
  float wt[3 * NV], bb[NV];  // wt[3 i + j]: tap j (t - 1, t, t + 1) of channel c0 + i
#pragma unroll
  for (int i = 0; i < 3 * NV / 4; ++i) {
    const float4 f = __ldg(reinterpret_cast<const float4*>(w + c0 * 3) + i);
    wt[4 * i] = f.x;
    wt[4 * i + 1] = f.y;
    wt[4 * i + 2] = f.z;
    wt[4 * i + 3] = f.w;
  }
#pragma unroll
  for (int i = 0; i < NV / 4; ++i) {
    const float4 f = bias != nullptr ? __ldg(reinterpret_cast<const float4*>(bias + c0) + i) : make_float4(0.f, 0.f, 0.f, 0.f);
    bb[4 * i] = f.x;
    bb[4 * i + 1] = f.y;
    bb[4 * i + 2] = f.z;
    bb[4 * i + 3] = f.w;
  }
  // x (or the carry) may come from the previous kernel in the stream: wait for it here, after the
  // weights, so that the launch overlaps the previous kernel's tail
  asm volatile("griddepcontrol.wait;" ::: "memory");
  if (threadIdx.x == 0) asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const size_t frame = static_cast<size_t>(S) * C;
  const size_t base = (static_cast<size_t>(b) * Tf * S + s) * C + c0;
  const T* xp = x + base;
  T* yp = y + base;
  T* cp = carry != nullptr ? carry + static_cast<size_t>(bs) * C + c0 : nullptr;
  float prev[NV], cur[NV];
  if (cp != nullptr) {
    V::to_float(*reinterpret_cast<const uint4*>(cp), prev);
  } else {
#pragma unroll
    for (int i = 0; i < NV; ++i) prev[i] = 0.f;
  }
  V::to_float(*reinterpret_cast<const uint4*>(xp), cur);
  for (int t0 = 0; t0 < Tf; t0 += kAhead) {
    uint4 raw[kAhead];
#pragma unroll
    for (int u = 0; u < kAhead; ++u) {
      const int t = t0 + 1 + u;
      raw[u] = t < Tf ? *reinterpret_cast<const uint4*>(xp + static_cast<size_t>(t) * frame) : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int u = 0; u < kAhead; ++u) {
      const int t = t0 + u;
      if (t >= Tf) break;
      float nxt[NV], out[NV];
      V::to_float(raw[u], nxt);
      const bool same = t + 1 < Tf && (t + 1) / L == t / L;  // the right neighbour is in t's block
#pragma unroll
      for (int i = 0; i < NV; ++i) {
        float a = fmaf(wt[3 * i], prev[i], bb[i]);
        a = fmaf(wt[3 * i + 1], cur[i], a);
        out[i] = same ? fmaf(wt[3 * i + 2], nxt[i], a) : a;
        prev[i] = cur[i];
        cur[i] = nxt[i];
      }
      *reinterpret_cast<uint4*>(yp + static_cast<size_t>(t) * frame) = V::from_float(out);
    }
  }
  if (commit && cp != nullptr) *reinterpret_cast<uint4*>(cp) = V::from_float(prev);  // x[Tf - 1], exactly
}

sv_status conv_fail(sv_status s, const char* msg) { return sv::set_last_error(s, msg); }

sv_status run_conv(const void* x, void* y, int B, int T, int S, int C, int L, const float* w, const float* bias,
                   void* carry, int commit, sv_dtype dt, cudaStream_t stream) {
  char msg[200];
  if (dt != SV_BF16 && dt != SV_F32) return conv_fail(SV_ERR_UNSUPPORTED, "dtype is not SV_BF16 or SV_F32");
  if (B < 1 || T < 1 || S < 1 || C < 1 || L < 1) {
    snprintf(msg, sizeof(msg), "B=%d T=%d S=%d C=%d frames_per_block=%d must all be >= 1", B, T, S, C, L);
    return conv_fail(SV_ERR_INVALID_ARG, msg);
  }
  const int nv = dt == SV_BF16 ? 8 : 4;
  if (C % nv != 0) {
    snprintf(msg, sizeof(msg), "C=%d must be a multiple of %d (16-byte channel groups)", C, nv);
    return conv_fail(SV_ERR_UNSUPPORTED, msg);
  }
  if (x == nullptr || y == nullptr || w == nullptr) return conv_fail(SV_ERR_INVALID_ARG, "x, y or w is NULL");
  const auto al = [](const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; };
  if (!al(x, 16) || !al(y, 16) || (carry != nullptr && !al(carry, 16)))
    return conv_fail(SV_ERR_INVALID_ARG, "x, y and carry must be 16-byte aligned");
  if (!al(w, 16) || (bias != nullptr && !al(bias, 16)))
    return conv_fail(SV_ERR_INVALID_ARG, "w and bias must be 16-byte aligned");
  const long long ncols = static_cast<long long>(B) * S * (C / nv);
  const long long nblocks = (ncols + kConvThreads - 1) / kConvThreads;
  if (nblocks > 0x7fffffffLL) return conv_fail(SV_ERR_UNSUPPORTED, "too many columns");
  // programmatic dependent launch: the CTAs may start while the previous kernel drains; they wait
  // (griddepcontrol.wait) before touching x, y or the carry
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(nblocks));
  cfg.blockDim = dim3(kConvThreads);
  cfg.stream = stream;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  cudaError_t e;
  if (dt == SV_BF16)
    e = cudaLaunchKernelEx(&cfg, temporal_conv_kernel<__nv_bfloat16>, static_cast<const __nv_bfloat16*>(x),
                           static_cast<__nv_bfloat16*>(y), B, T, S, C, L, w, bias, static_cast<__nv_bfloat16*>(carry),
                           commit, ncols);
  else
    e = cudaLaunchKernelEx(&cfg, temporal_conv_kernel<float>, static_cast<const float*>(x), static_cast<float*>(y), B,
                           T, S, C, L, w, bias, static_cast<float*>(carry), commit, ncols);
  if (e != cudaSuccess) {
    snprintf(msg, sizeof(msg), "temporal conv launch: %s", cudaGetErrorString(e));
    return conv_fail(SV_ERR_CUDA, msg);
  }
  return SV_OK;
}

}  // namespace

extern "C" sv_status sv_temporal_conv(const void* x, void* y, int B, int T, int S, int C, int frames_per_block,
                                      const float* w, const float* bias, sv_dtype dt, sv_stream_t stream) {
  return run_conv(x, y, B, T, S, C, frames_per_block, w, bias, nullptr, 0, dt, reinterpret_cast<cudaStream_t>(stream));
}

extern "C" sv_status sv_temporal_conv_step(const void* x, void* y, int B, int T, int S, int C, const float* w,
                                           const float* bias, void* carry, int commit, sv_dtype dt,
                                           sv_stream_t stream) {
  if (carry == nullptr) return sv::set_last_error(SV_ERR_INVALID_ARG, "carry is NULL");
  return run_conv(x, y, B, T, S, C, T, w, bias, carry, commit, dt, reinterpret_cast<cudaStream_t>(stream));
}
