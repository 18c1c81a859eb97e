// The linear projections around the attention, sm_100a: Q/K/V = X W^T with the ReLU feature map on Q
// and K in the epilogue, written in the [B, H, N, D] layout the attention kernels read; and the
// output projection Y = O_cat W_o^T reading the attention output O [B, H, N, D] directly.
//
// SANA-Video model-family page, 2.0 paragraph: hidden size 2560 (20 heads of 128 features), linear
// attention layers; the feature map is the ReLU of the library's operation. These are dense
// contractions (2560-deep), so they run on the tensor cores: a persistent kernel, one CTA per SM,
// 128 x 256 output tiles, K in 64-deep steps through four TMA stages (A 128 x 64 and B 256 x 64 bf16,
// 128-byte swizzle), tcgen05.mma M=128 N=256 K=16 into one of two fp32 TMEM accumulators, so the
// epilogue of a tile overlaps the MMAs of the next. Warp 0 issues the copies, warp 1 the MMAs, warps
// 2-5 drain TMEM in 64-column chunks: ReLU where the chunk belongs to Q or K, bf16, a swizzled
// staging buffer, and a TMA store of 32 rows x 64 features into the chunk's tensor, head and
// features. Rows are tiled per batch (a tile never holds two batches' tokens); the last row tile of
// a batch is zero-filled on load and clipped on store by the tensor maps. Tiles are numbered column
// tile fastest, so the CTAs working at any moment share a few row tiles of A (read from DRAM once)
// and sweep the whole weight, which stays in L2 (39 MB for the fused Q/K/V weight at hidden 2560);
// numbered the other way, every column tile streamed all of A through L2 again (measured: 3.15 GB of
// DRAM reads for 143 MB of operands).
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdio>
#include <mutex>

#include "../../include/svlinattn.h"
#include "sv_internal.h"
#include "sv_ptx.cuh"

namespace sv {
namespace {

constexpr int kBM = 128, kBN = 256, kBK = 64;
constexpr int kPStages = 4;
constexpr int kPThreads = 192;                      // warp 0 copies, warp 1 MMAs, warps 2-5 epilogue
constexpr int kABytes = kBM * kBK * 2;              // 16 KB
constexpr int kBBytes = kBN * kBK * 2;              // 32 KB
constexpr int kPStageBytes = kABytes + kBBytes;     // 48 KB
constexpr int kStagingOff = kPStages * kPStageBytes;
constexpr int kStagingWarp = 2 * 32 * 128;          // two 4 KB buffers (32 rows x 64 bf16) per epilogue warp
constexpr int kPBarOff = kStagingOff + 4 * kStagingWarp;
constexpr int kPSmem = kPBarOff + 256 + 1024;       // barriers, TMEM slot, alignment slack
static_assert(kPSmem <= 227 * 1024, "projection kernel shared memory");

struct PGeom {
  int B, N;       // batches, tokens per batch
  int K;          // contraction depth (hidden C, or H * D for the output projection)
  int Nout;       // output features (3 * H * D, or C_out)
  int H, D;       // heads and head features (the [B, H, N, D] side)
  int HD;         // H * D: features of one of Q, K, V
  int mtb;        // row tiles per batch
  int mt, nt;     // row and column tiles
  int tiles;      // mt * nt
  int kchunks;    // K / 64
};

__device__ __forceinline__ bool all_lanes(bool ok) { return __all_sync(0xffffffffu, ok); }

__device__ __forceinline__ uint8_t* align1024p(uint8_t* p) {
  uintptr_t a = reinterpret_cast<uintptr_t>(p);
  return reinterpret_cast<uint8_t*>((a + 1023) & ~static_cast<uintptr_t>(1023));
}

// kQKV: A = X [B, N, C] (map dims C, N, 1, B), outputs q, k, v [B, H, N, D] (maps D, N, H, B), ReLU on
// q and k. Otherwise A = O [B, H, N, D] (map dims D, N, H, B; k-step kc reads head kc*64/D), output
// Y [B, N, C_out] (map dims C_out, N, 1, B) in o0.
template <bool kQKV>
__global__ void __launch_bounds__(kPThreads, 1)
    proj_kernel(const __grid_constant__ CUtensorMap a_map, const __grid_constant__ CUtensorMap b_map,
                const __grid_constant__ CUtensorMap o0, const __grid_constant__ CUtensorMap o1,
                const __grid_constant__ CUtensorMap o2, const PGeom g, uint32_t* status) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024p(smem_raw);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kPBarOff);
  uint64_t* full = bars;            // [4] A and B of a step landed
  uint64_t* empty = bars + 4;       // [4] the step's MMAs retired
  uint64_t* accf = bars + 8;        // [2] accumulator holds a finished tile
  uint64_t* acce = bars + 10;       // [2] accumulator drained
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 12);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int i = 0; i < kPStages; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&accf[a], 1);
      mbar_init(&acce[a], 4);
    }
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&a_map);
    prefetch_tmap(&b_map);
    prefetch_tmap(&o0);
    if (kQKV) {
      prefetch_tmap(&o1);
      prefetch_tmap(&o2);
    }
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  griddep_wait();  // the previous kernel may still write X / O or read the outputs
  if (threadIdx.x == 0) griddep_launch_dependents();

  if (warp == 0) {
    if (lane == 0) {  // copies
      const uint64_t pol_a = policy_evict_first();
      const uint64_t pol_b = policy_evict_last();  // W is read by every row tile
      int it = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < g.tiles && ok; tile += gridDim.x) {
        const int n = tile % g.nt, m = tile / g.nt;
        const int b = m / g.mtb, i0 = (m - b * g.mtb) * kBM, n0 = n * kBN;
        for (int kc = 0; kc < g.kchunks; ++kc, ++it) {
          const int s = it % kPStages;
          if (!mbar_wait(&empty[s], ((it / kPStages) & 1) ^ 1, status, 0x5100u | s)) {
            ok = false;
            break;
          }
          uint8_t* sa = smem + s * kPStageBytes;
          mbar_expect_tx(&full[s], kPStageBytes);
          if (kQKV) {
            tma_load_4d(sa, &a_map, &full[s], kc * kBK, i0, 0, b, pol_a);
          } else {
            const int k0 = kc * kBK, h = k0 / g.D;
            tma_load_4d(sa, &a_map, &full[s], k0 - h * g.D, i0, h, b, pol_a);
          }
          tma_load_4d(sa + kABytes, &b_map, &full[s], kc * kBK, n0, 0, 0, pol_b);
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {  // MMAs
      constexpr uint32_t kIdesc = idesc_bf16_f32(kBM, kBN, false, false);
      int it = 0, tl = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < g.tiles && ok; tile += gridDim.x, ++tl) {
        const int a = tl & 1;
        if (!mbar_wait(&acce[a], ((tl >> 1) & 1) ^ 1, status, 0x5300u | a)) break;
        tc_fence_after();
        const uint32_t d = tmem + static_cast<uint32_t>(a * kBN);
        for (int kc = 0; kc < g.kchunks; ++kc, ++it) {
          const int s = it % kPStages;
          if (!mbar_wait(&full[s], (it / kPStages) & 1, status, 0x5310u | s)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = smem_u32(smem + s * kPStageBytes);
          const uint32_t sb = sa + kABytes;
#pragma unroll
          for (int kk = 0; kk < kBK / 16; ++kk)
            mma_bf16(d, sdesc_sw128(sa + kk * 32, 16, 1024), sdesc_sw128(sb + kk * 32, 16, 1024), kIdesc,
                     (kc | kk) != 0 ? 1u : 0u);
          mma_commit(&empty[s]);
        }
        if (ok) mma_commit(&accf[a]);
      }
    }
  } else {  // epilogue: warp w drains TMEM lanes 32 * (w % 4) .. + 31 (rows of the tile)
    const int q = warp & 3;
    const int ew = warp - 2;
    uint8_t* stg = smem + kStagingOff + ew * kStagingWarp;
    int tl = 0, chunk = 0;
    for (int tile = blockIdx.x; tile < g.tiles; tile += gridDim.x, ++tl) {
      const int a = tl & 1;
      if (!all_lanes(mbar_wait(&accf[a], (tl >> 1) & 1, status, 0x5400u | a))) break;
      tc_fence_after();
      const int n = tile % g.nt, m = tile / g.nt;
      const int b = m / g.mtb, i0 = (m - b * g.mtb) * kBM;
      const int row0 = i0 + q * 32;  // first token of this warp's slice
      const uint32_t ta = tmem + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(a * kBN);
#pragma unroll 1
      for (int c = 0; c < kBN / 64; ++c, ++chunk) {
        uint32_t rr[2][32];
        tmem_ld_x32(ta + c * 64, rr[0]);
        tmem_ld_x32(ta + c * 64 + 32, rr[1]);
        tmem_wait_ld();
        if (c == kBN / 64 - 1) {  // the tile's last TMEM read: the accumulator is free
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&acce[a]);
        }
        const int nc = n * kBN + c * 64;  // first output feature of the chunk
        if (nc >= g.Nout) {  // past the last feature: an empty group keeps one group per chunk
          if (lane == 0) bulk_commit();
          continue;
        }
        const bool relu = kQKV && nc < 2 * g.HD;
        uint8_t* ob = stg + (chunk & 1) * (32 * 128);
        if (lane == 0) bulk_wait_read_all_but_one();  // the store that read this buffer two chunks ago
        __syncwarp();
#pragma unroll
        for (int cc = 0; cc < 2; ++cc) {
#pragma unroll
          for (int mm = 0; mm < 4; ++mm) {
            float f[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
              f[u] = __uint_as_float(rr[cc][8 * mm + u]);
              if (relu) f[u] = fmaxf(f[u], 0.f);
            }
            uint4 w;
            w.x = pack_bf16x2(f[0], f[1]);
            w.y = pack_bf16x2(f[2], f[3]);
            w.z = pack_bf16x2(f[4], f[5]);
            w.w = pack_bf16x2(f[6], f[7]);
            const int j = cc * 4 + mm;  // 16-byte chunk of the 128-byte row
            *reinterpret_cast<uint4*>(ob + lane * 128 + ((j ^ (lane & 7)) << 4)) = w;
          }
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          if (row0 < g.N) {
            if (kQKV) {
              const int t = nc / g.HD, f = nc - t * g.HD, h = f / g.D;
              const CUtensorMap* om = t == 0 ? &o0 : (t == 1 ? &o1 : &o2);
              tma_store_4d(om, ob, f - h * g.D, row0, h, b);
            } else {
              tma_store_4d(&o0, ob, nc, row0, 0, b);
            }
          }
          bulk_commit();
        }
      }
    }
    if (lane == 0) bulk_wait_all();
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// The kernels' shared-memory attribute, set once per device (and per kernel), thread-safe.
template <bool kQKV>
cudaError_t ensure_attr() {
  constexpr int kMaxDev = 64;
  static std::mutex mu;
  static bool done[kMaxDev] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDev) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(mu);
  if (!done[dev]) {
    e = cudaFuncSetAttribute(proj_kernel<kQKV>, cudaFuncAttributeMaxDynamicSharedMemorySize, kPSmem);
    if (e != cudaSuccess) return e;
    done[dev] = true;
  }
  return cudaSuccess;
}

template <bool kQKV>
cudaError_t launch_proj(const CUtensorMap& a, const CUtensorMap& bm, const CUtensorMap& o0, const CUtensorMap& o1,
                        const CUtensorMap& o2, const PGeom& g, uint32_t* status, int sm_count, cudaStream_t s) {
  const cudaError_t ea = ensure_attr<kQKV>();
  if (ea != cudaSuccess) return ea;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(g.tiles < sm_count ? g.tiles : sm_count));
  cfg.blockDim = dim3(kPThreads);
  cfg.dynamicSmemBytes = kPSmem;
  cfg.stream = s;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, proj_kernel<kQKV>, a, bm, o0, o1, o2, g, status);
}

sv_status pfail(sv_status st, const char* fmt, int a = 0, int b = 0) {
  char msg[200];
  snprintf(msg, sizeof(msg), fmt, a, b);
  return set_last_error(st, msg);
}

bool al16(const void* p) { return p != nullptr && (reinterpret_cast<uintptr_t>(p) & 15u) == 0u; }

sv_status check_ws_header(void* ws, size_t ws_bytes) {
  if (ws == nullptr || (reinterpret_cast<uintptr_t>(ws) & 255u) != 0u || ws_bytes < static_cast<size_t>(kHeaderBytes))
    return pfail(SV_ERR_INVALID_ARG, "ws must be a 256-byte aligned workspace of at least %d bytes", kHeaderBytes);
  return SV_OK;
}

sv_status sm_count_of_current(int* n) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return pfail(SV_ERR_CUDA, "cannot query the current device");
  int major = 0, minor = 0;
  cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
  cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
  if (major != 10 || minor != 0) return pfail(SV_ERR_UNSUPPORTED, "device is sm_%d%d; built for sm_100a", major, minor);
  return SV_OK;
}

PGeom make_pgeom(int B, int N, int K, int Nout, int H, int D) {
  PGeom g;
  g.B = B;
  g.N = N;
  g.K = K;
  g.Nout = Nout;
  g.H = H;
  g.D = D;
  g.HD = H * D;
  g.mtb = (N + kBM - 1) / kBM;
  g.mt = B * g.mtb;
  g.nt = (Nout + kBN - 1) / kBN;
  g.tiles = g.mt * g.nt;
  g.kchunks = K / kBK;
  return g;
}

// [B, H, N, D] bf16 as (D, N, H, B) with the given box rows.
sv_status bhnd_map(CUtensorMap* m, const void* p, int B, int H, int N, int D, uint32_t box_rows) {
  const uint64_t dims[4] = {static_cast<uint64_t>(D), static_cast<uint64_t>(N), static_cast<uint64_t>(H),
                            static_cast<uint64_t>(B)};
  const uint64_t st[3] = {static_cast<uint64_t>(D) * 2, static_cast<uint64_t>(N) * D * 2,
                          static_cast<uint64_t>(H) * N * D * 2};
  const uint32_t box[4] = {64, box_rows, 1, 1};
  return encode_bf16_4d(m, p, dims, st, box);
}

// [B, N, C] bf16 as (C, N, 1, B).
sv_status bnc_map(CUtensorMap* m, const void* p, int B, int N, int C, uint32_t box_rows) {
  const uint64_t dims[4] = {static_cast<uint64_t>(C), static_cast<uint64_t>(N), 1, static_cast<uint64_t>(B)};
  const uint64_t st[3] = {static_cast<uint64_t>(C) * 2, static_cast<uint64_t>(N) * C * 2,
                          static_cast<uint64_t>(N) * C * 2};
  const uint32_t box[4] = {64, box_rows, 1, 1};
  return encode_bf16_4d(m, p, dims, st, box);
}

// W [Nout, K] bf16 as (K, Nout, 1, 1), 256-row boxes.
sv_status w_map(CUtensorMap* m, const void* p, int Nout, int K) {
  const uint64_t dims[4] = {static_cast<uint64_t>(K), static_cast<uint64_t>(Nout), 1, 1};
  const uint64_t st[3] = {static_cast<uint64_t>(K) * 2, static_cast<uint64_t>(Nout) * K * 2,
                          static_cast<uint64_t>(Nout) * K * 2};
  const uint32_t box[4] = {64, static_cast<uint32_t>(kBN), 1, 1};
  return encode_bf16_4d(m, p, dims, st, box);
}

#define PV_TRY(x)                 \
  do {                            \
    const sv_status _s = (x);     \
    if (_s != SV_OK) return _s;   \
  } while (0)

sv_status check_common(int B, int N, int H, int D) {
  if (B < 1 || N < 1 || H < 1) return pfail(SV_ERR_INVALID_ARG, "B, N and H must be >= 1");
  if (D != 64 && D != 128) return pfail(SV_ERR_UNSUPPORTED, "the projections need D = 64 or 128, got %d", D);
  if (static_cast<long long>(B) * ((N + kBM - 1) / kBM) > (1ll << 24)) return pfail(SV_ERR_UNSUPPORTED, "too many rows");
  return SV_OK;
}

}  // namespace
}  // namespace sv

extern "C" sv_status sv_qkv_projection(const void* x, const void* w_qkv, void* q, void* k, void* v, int B, int N, int C,
                                       int H, int D, void* ws, size_t ws_bytes, sv_stream_t stream) {
  using namespace sv;
  PV_TRY(check_common(B, N, H, D));
  if (C < 64 || C % 64 != 0) return pfail(SV_ERR_UNSUPPORTED, "the hidden size C=%d must be a multiple of 64", C);
  if (!al16(x) || !al16(w_qkv) || !al16(q) || !al16(k) || !al16(v))
    return pfail(SV_ERR_INVALID_ARG, "x, w_qkv, q, k, v must be non-NULL and 16-byte aligned");
  PV_TRY(check_ws_header(ws, ws_bytes));
  int sms = 0;
  PV_TRY(sm_count_of_current(&sms));
  const PGeom g = make_pgeom(B, N, C, 3 * H * D, H, D);
  CUtensorMap am, bm, mq, mk, mv;
  PV_TRY(bnc_map(&am, x, B, N, C, kBM));
  PV_TRY(w_map(&bm, w_qkv, 3 * H * D, C));
  PV_TRY(bhnd_map(&mq, q, B, H, N, D, 32));
  PV_TRY(bhnd_map(&mk, k, B, H, N, D, 32));
  PV_TRY(bhnd_map(&mv, v, B, H, N, D, 32));
  const cudaError_t e = launch_proj<true>(am, bm, mq, mk, mv, g, static_cast<uint32_t*>(ws), sms,
                                          reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return pfail(SV_ERR_CUDA, "projection kernel launch failed (%d)", static_cast<int>(e));
  return SV_OK;
}

extern "C" sv_status sv_out_projection(const void* o, const void* w_o, void* y, int B, int N, int H, int D, int C_out,
                                       void* ws, size_t ws_bytes, sv_stream_t stream) {
  using namespace sv;
  PV_TRY(check_common(B, N, H, D));
  if (C_out < 64 || C_out % 64 != 0) return pfail(SV_ERR_UNSUPPORTED, "C_out=%d must be a multiple of 64", C_out);
  if (!al16(o) || !al16(w_o) || !al16(y)) return pfail(SV_ERR_INVALID_ARG, "o, w_o, y must be non-NULL and 16-byte aligned");
  PV_TRY(check_ws_header(ws, ws_bytes));
  int sms = 0;
  PV_TRY(sm_count_of_current(&sms));
  const PGeom g = make_pgeom(B, N, H * D, C_out, H, D);
  CUtensorMap am, bm, my;
  PV_TRY(bhnd_map(&am, o, B, H, N, D, kBM));
  PV_TRY(w_map(&bm, w_o, C_out, H * D));
  PV_TRY(bnc_map(&my, y, B, N, C_out, 32));
  const cudaError_t e = launch_proj<false>(am, bm, my, my, my, g, static_cast<uint32_t*>(ws), sms,
                                           reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return pfail(SV_ERR_CUDA, "projection kernel launch failed (%d)", static_cast<int>(e));
  return SV_OK;
}
