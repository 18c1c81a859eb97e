// Kernels of ReLU-kernel linear attention (bidirectional and block-causal), sm_100a.
//
// The method (SANA-Video, "Efficient Video Generation with Block Linear Diffusion Transformer",
// talk, block KV cache passage): linear attention keeps a D x D state; a block's state is the sum
// of its tokens' ReLU(k) v^T and is added to the cache of all previous blocks; a block sees itself
// and the cache. Here that becomes three kernels per call:
//
//   1. state_bf16_kernel : per tile of 128 tokens, TMA K/V tiles -> ReLU(K) in shared memory ->
//      tcgen05.mma  [ReLU(K)^T] x [V | 1]  accumulated in TMEM (fp32) over the tiles of a segment
//      (one block of one head); partial states go to workspace slots.
//   2. scan_kernel        : sums the partial slots of each segment and takes the inclusive prefix
//      over blocks (plus the incoming cache); writes the bf16 B operand of the output GEMM and,
//      when asked, the final fp32 cache.
//   3. out_bf16_kernel    : per tile, TMA Q -> ReLU(Q) in shared memory -> tcgen05.mma
//      ReLU(Q) x [P | z]^T into TMEM; the epilogue divides numerator by (denominator + eps),
//      converts to bf16 and TMA-stores the tile.
// The fp32 I/O path runs the same three steps with SIMT fp32 kernels.
#include <cuda_bf16.h>

#include <utility>

#include "sv_internal.h"
#include "sv_ptx.cuh"

namespace sv {

namespace {

constexpr int kThreads = 320;     // warps 0-3 epilogue, 4-7 ReLU, 8 TMA producer, 9 MMA issuer
constexpr int kWarpProducer = 8;
constexpr int kWarpMma = 9;
constexpr int kTmemCols = 512;    // two fp32 accumulators at columns 0 and 256
constexpr int kAtomBytes = kTile * 128;   // 128 rows x 128 B (64 bf16) = one swizzle-128B atom column

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
  uintptr_t a = reinterpret_cast<uintptr_t>(p);
  return reinterpret_cast<uint8_t*>((a + 1023) & ~static_cast<uintptr_t>(1023));
}

__device__ __forceinline__ bool warp_all(bool ok) { return __all_sync(0xffffffffu, ok); }

// ReLU in place over `nchunks` 16-byte chunks of a tile, by the 128 ReLU threads (index r).
__device__ __forceinline__ void relu_tile_inplace(uint8_t* tile, int nchunks, int r) {
  uint4* p = reinterpret_cast<uint4*>(tile);
#pragma unroll 4
  for (int i = r; i < nchunks; i += 128) {
    uint4 x = p[i];
    x.x = relu_bf16x2(x.x);
    x.y = relu_bf16x2(x.y);
    x.z = relu_bf16x2(x.z);
    x.w = relu_bf16x2(x.w);
    p[i] = x;
  }
}

__device__ __forceinline__ bool use_last_map(const TileCoord& c, const Geom& g) {
  return c.blk == g.nblk - 1 && g.Llast != g.L;
}

// ------------------------------------------------------------------------------------------
// 1. block-state reduction (bf16 in, fp32 TMEM accumulation)
// ------------------------------------------------------------------------------------------
namespace st {
constexpr int kStages = 3;
constexpr int kKBytes = 2 * kAtomBytes;          // K tile: 128 tokens x 128 features (two atoms)
constexpr int kStageBytes = 2 * kKBytes;         // K + V
constexpr int kOnesOff = kStages * kStageBytes;  // 16 KB of bf16 ones: B operand of the z column
constexpr int kBarOff = kOnesOff + kAtomBytes;
constexpr int kSmemBytes = kBarOff + 256 + 1024;
}  // namespace st

__global__ void __launch_bounds__(kThreads, 1)
    state_bf16_kernel(const __grid_constant__ CUtensorMap k_main, const __grid_constant__ CUtensorMap k_last,
                      const __grid_constant__ CUtensorMap v_main, const __grid_constant__ CUtensorMap v_last,
                      const Geom geo, float* __restrict__ partials, int2* __restrict__ segcta,
                      uint32_t* status) {
  using namespace st;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kBarOff);
  uint64_t* full = bars;        // TMA landed (K and V)
  uint64_t* relu = bars + 3;    // ReLU(K) written back
  uint64_t* empty = bars + 6;   // MMAs reading the stage retired
  uint64_t* accf = bars + 9;    // accumulator holds a finished segment
  uint64_t* acce = bars + 11;   // accumulator drained by the epilogue
  uint64_t* done = bars + 13;   // every MMA retired (teardown)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 14);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int g = blockIdx.x;
  const long long tb = tile_begin(g, geo);
  const long long te = tile_begin(g + 1, geo);
  const bool two_atoms = geo.D > 64;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&relu[i], 4);
      mbar_init(&empty[i], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&accf[a], 1);
      mbar_init(&acce[a], 4);
    }
    mbar_init(done, 1);
    fence_mbar_init();
  }
  {
    uint4* ones = reinterpret_cast<uint4*>(smem + kOnesOff);
    const uint4 one = make_uint4(0x3F803F80u, 0x3F803F80u, 0x3F803F80u, 0x3F803F80u);
    for (int i = threadIdx.x; i < kAtomBytes / 16; i += kThreads) ones[i] = one;
    if (!two_atoms) {  // features 64..127 never loaded: keep them zero
      for (int s = 0; s < kStages; ++s) {
        uint4* kz = reinterpret_cast<uint4*>(smem + s * kStageBytes + kAtomBytes);
        uint4* vz = reinterpret_cast<uint4*>(smem + s * kStageBytes + kKBytes + kAtomBytes);
        for (int i = threadIdx.x; i < kAtomBytes / 16; i += kThreads) {
          kz[i] = make_uint4(0, 0, 0, 0);
          vz[i] = make_uint4(0, 0, 0, 0);
        }
      }
    }
    fence_proxy_async_smem();
  }
  if (warp == kWarpMma) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  if (warp == kWarpProducer && lane == 0) {
    prefetch_tmap(&k_main);
    prefetch_tmap(&v_main);
    prefetch_tmap(&k_last);
    prefetch_tmap(&v_last);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  if (threadIdx.x == 0) griddep_launch_dependents();

  if (warp == kWarpProducer) {
    if (lane == 0) {
      const uint64_t pol = policy_evict_first();
      const uint32_t tx = two_atoms ? 2u * kKBytes : static_cast<uint32_t>(kKBytes);
      // K, V may come from the previous kernel in the stream, and the partial slots written below
      // may still be read by the previous call's scan: nothing is touched before this wait.
      griddep_wait();
      int k = 0;
      for (long long t = tb; t < te; ++t, ++k) {
        const TileCoord c = tile_coord(t, geo);
        const int s = k % kStages;
        if (!mbar_wait(&empty[s], ((k / kStages) & 1) ^ 1, status, 0x0100u | s)) break;
        const bool lst = use_last_map(c, geo);
        const CUtensorMap* mk = lst ? &k_last : &k_main;
        const CUtensorMap* mv = lst ? &v_last : &v_main;
        const int cb = lst ? 0 : c.blk;
        uint8_t* stg = smem + s * kStageBytes;
        mbar_expect_tx(&full[s], tx);
        tma_load_4d(stg, mk, &full[s], 0, c.tok0, cb, c.bh, pol);
        tma_load_4d(stg + kKBytes, mv, &full[s], 0, c.tok0, cb, c.bh, pol);
        if (two_atoms) {
          tma_load_4d(stg + kAtomBytes, mk, &full[s], 64, c.tok0, cb, c.bh, pol);
          tma_load_4d(stg + kKBytes + kAtomBytes, mv, &full[s], 64, c.tok0, cb, c.bh, pol);
        }
      }
      // the loads issued last into each stage land before the CTA can exit
      for (int j = (k > kStages ? k - kStages : 0); j < k; ++j)
        mbar_wait(&full[j % kStages], (j / kStages) & 1, status, 0x0180u);
    }
  } else if (warp >= 4 && warp < 8) {
    const int r = threadIdx.x - 128;
    const int nchunks = (two_atoms ? kKBytes : kAtomBytes) / 16;
    int k = 0;
    for (long long t = tb; t < te; ++t, ++k) {
      const int s = k % kStages;
      bool ok = mbar_wait(&full[s], (k / kStages) & 1, status, 0x0200u | s);
      if (!warp_all(ok)) break;
      relu_tile_inplace(smem + s * kStageBytes, nchunks, r);
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&relu[s]);
    }
  } else if (warp == kWarpMma) {
    if (lane == 0) {
      constexpr uint32_t kIdescS = idesc_bf16_f32(128, 128, true, true);
      constexpr uint32_t kIdescZ = idesc_bf16_f32(128, 16, true, true);
      const uint32_t ones = smem_u32(smem + kOnesOff);
      int k = 0, j = 0;
      for (long long t = tb; t < te; ++t, ++k) {
        const TileCoord c = tile_coord(t, geo);
        const bool first = (t == tb) || c.tok0 == 0;
        const bool end = c.last || t == te - 1;
        const int a = j & 1;
        const int s = k % kStages;
        const uint32_t ph = (k / kStages) & 1;
        if (first && !mbar_wait(&acce[a], ((j >> 1) & 1) ^ 1, status, 0x0300u | a)) break;
        if (!mbar_wait(&full[s], ph, status, 0x0310u | s)) break;
        if (!mbar_wait(&relu[s], ph, status, 0x0320u | s)) break;
        tc_fence_after();
        const uint32_t kb = smem_u32(smem + s * kStageBytes);
        const uint32_t vb = kb + kKBytes;
        const uint32_t dacc = tmem + static_cast<uint32_t>(a * 256);
#pragma unroll
        for (int kk = 0; kk < kTile / 16; ++kk) {
          // 16 tokens per MMA: two groups of 8 token rows (128 B each) -> +2048 B per step
          const uint64_t ad = sdesc_sw128(kb + kk * 2048, kAtomBytes, 1024);
          const uint64_t bd = sdesc_sw128(vb + kk * 2048, kAtomBytes, 1024);
          const uint64_t od = sdesc_sw128(ones + kk * 2048, kAtomBytes, 1024);
          const uint32_t acc = (first && kk == 0) ? 0u : 1u;
          mma_bf16(dacc, ad, bd, kIdescS, acc);         // S^T columns: ReLU(K)^T V
          mma_bf16(dacc + 128, ad, od, kIdescZ, acc);   // z column: ReLU(K)^T 1
        }
        mma_commit(&empty[s]);
        if (end) {
          mma_commit(&accf[a]);
          ++j;
        }
      }
      mma_commit(done);
      mbar_wait(done, 0, status, 0x03F0u);
    }
  } else {
    // epilogue: warp w drains TMEM lanes 32w..32w+31 (key feature d) into the partial slot
    const int d = warp * 32 + lane;
    int j = 0;
    for (long long t = tb; t < te; ++t) {
      const TileCoord c = tile_coord(t, geo);
      if (!(c.last || t == te - 1)) continue;
      const int a = j & 1;
      bool ok = mbar_wait(&accf[a], (j >> 1) & 1, status, 0x0400u | a);
      if (!warp_all(ok)) break;
      tc_fence_after();
      const uint32_t ta = tmem + (static_cast<uint32_t>(warp * 32) << 16) + static_cast<uint32_t>(a * 256);
      float* dst = partials + static_cast<size_t>(g + c.seg) * (kPartRows * kDPad);
#pragma unroll
      for (int cc = 0; cc < 4; ++cc) {
        uint32_t r[32];
        tmem_ld_x32(ta + cc * 32, r);
        tmem_wait_ld();
#pragma unroll
        for (int jj = 0; jj < 32; ++jj) dst[(cc * 32 + jj) * kDPad + d] = __uint_as_float(r[jj]);
      }
      uint32_t zr;
      tmem_ld_x1(ta + 128, zr);
      tmem_wait_ld();
      dst[kZRow * kDPad + d] = __uint_as_float(zr);
      if (warp == 0 && lane == 0) {  // which CTAs hold the first and the last tile of the segment
        if (t - c.tok0 / kTile >= tb) segcta[c.seg].x = g;
        if (c.last) segcta[c.seg].y = g;
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acce[a]);
      ++j;
    }
  }

  __syncthreads();
  if (warp == kWarpMma) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// ------------------------------------------------------------------------------------------
// 3. output GEMM with the normalising divide in the epilogue (bf16 in/out)
// ------------------------------------------------------------------------------------------
namespace ot {
constexpr int kStages = 3;
constexpr int kQBytes = 2 * kAtomBytes;             // Q tile: 128 tokens x 128 features
constexpr int kBOff = kStages * kQBytes;            // two prefix tiles (double-buffered)
constexpr int kBAtomBytes = kPTileRows * 128;       // 144 rows x 128 B
constexpr int kOOff = kBOff + 2 * kPTileBytes;      // output staging, one 8 KB slice per warp
constexpr int kOWarpBytes = 2 * 32 * 128;
constexpr int kBarOff = kOOff + 4 * kOWarpBytes;
constexpr int kSmemBytes = kBarOff + 256 + 1024;
static_assert(kBOff % 1024 == 0 && kOOff % 1024 == 0 && kBAtomBytes % 1024 == 0, "1024-B atoms");
}  // namespace ot

__global__ void __launch_bounds__(kThreads, 1)
    out_bf16_kernel(const __grid_constant__ CUtensorMap q_main, const __grid_constant__ CUtensorMap q_last,
                    const __grid_constant__ CUtensorMap o_main, const __grid_constant__ CUtensorMap o_last,
                    const Geom geo, const uint8_t* __restrict__ ptiles, const float eps, uint32_t* status) {
  using namespace ot;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kBarOff);
  uint64_t* qfull = bars;
  uint64_t* qrelu = bars + 3;
  uint64_t* qempty = bars + 6;
  uint64_t* bfull = bars + 9;
  uint64_t* bempty = bars + 11;
  uint64_t* accf = bars + 13;
  uint64_t* acce = bars + 15;
  uint64_t* done = bars + 17;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 18);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int g = blockIdx.x;
  const long long tb = tile_begin(g, geo);
  const long long te = tile_begin(g + 1, geo);
  const bool two_atoms = geo.D > 64;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&qfull[i], 1);
      mbar_init(&qrelu[i], 4);
      mbar_init(&qempty[i], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&bfull[a], 1);
      mbar_init(&bempty[a], 1);
      mbar_init(&accf[a], 1);
      mbar_init(&acce[a], 4);
    }
    mbar_init(done, 1);
    fence_mbar_init();
  }
  if (warp == kWarpMma) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  if (warp == kWarpProducer && lane == 0) {
    prefetch_tmap(&q_main);
    prefetch_tmap(&q_last);
    prefetch_tmap(&o_main);
    prefetch_tmap(&o_last);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (threadIdx.x == 0) griddep_launch_dependents();

  if (warp == kWarpProducer) {
    if (lane == 0) {
      const uint64_t pol = policy_evict_first();
      const uint32_t tx = two_atoms ? static_cast<uint32_t>(kQBytes) : static_cast<uint32_t>(kAtomBytes);
      auto load_q = [&](long long t, int s) {
        const TileCoord c = tile_coord(t, geo);
        const bool lst = use_last_map(c, geo);
        const CUtensorMap* mq = lst ? &q_last : &q_main;
        const int cb = lst ? 0 : c.blk;
        uint8_t* stg = smem + s * kQBytes;
        mbar_expect_tx(&qfull[s], tx);
        tma_load_4d(stg, mq, &qfull[s], 0, c.tok0, cb, c.bh, pol);
        if (two_atoms) tma_load_4d(stg + kAtomBytes, mq, &qfull[s], 64, c.tok0, cb, c.bh, pol);
      };
      // Q was final before the state kernel ran, so the first stages fill while the scan runs;
      // the prefix tiles are read only after the scan grid has completed.
      const int pre = static_cast<int>(te - tb < kStages ? te - tb : kStages);
      for (int i = 0; i < pre; ++i) load_q(tb + i, i);
      griddep_wait();
      int k = 0, j = 0, prev = -1;
      for (long long t = tb; t < te; ++t, ++k) {
        const TileCoord c = tile_coord(t, geo);
        if (c.seg != prev) {
          const int bb = j & 1;
          if (!mbar_wait(&bempty[bb], ((j >> 1) & 1) ^ 1, status, 0x1100u | bb)) break;
          mbar_expect_tx(&bfull[bb], kPTileBytes);
          bulk_load(smem + kBOff + bb * kPTileBytes, ptiles + static_cast<size_t>(c.seg) * kPTileBytes,
                    kPTileBytes, &bfull[bb]);
          ++j;
          prev = c.seg;
        }
        if (k >= pre) {
          const int s = k % kStages;
          if (!mbar_wait(&qempty[s], ((k / kStages) & 1) ^ 1, status, 0x1120u | s)) break;
          load_q(t, s);
        }
      }
      for (int i = (k > kStages ? k - kStages : 0); i < (k > pre ? k : pre); ++i)
        mbar_wait(&qfull[i % kStages], (i / kStages) & 1, status, 0x1180u);
      for (int i = (j > 2 ? j - 2 : 0); i < j; ++i) mbar_wait(&bfull[i & 1], (i >> 1) & 1, status, 0x1190u);
    }
  } else if (warp >= 4 && warp < 8) {
    const int r = threadIdx.x - 128;
    const int nchunks = (two_atoms ? kQBytes : kAtomBytes) / 16;
    int k = 0;
    for (long long t = tb; t < te; ++t, ++k) {
      const int s = k % kStages;
      bool ok = mbar_wait(&qfull[s], (k / kStages) & 1, status, 0x1200u | s);
      if (!warp_all(ok)) break;
      relu_tile_inplace(smem + s * kQBytes, nchunks, r);
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&qrelu[s]);
    }
  } else if (warp == kWarpMma) {
    if (lane == 0) {
      constexpr uint32_t kIdescO = idesc_bf16_f32(128, kPTileRows, false, false);
      const int ksteps = two_atoms ? 8 : 4;
      int k = 0, j = 0, prev = -1, bb = 0;
      for (long long t = tb; t < te; ++t, ++k) {
        const TileCoord c = tile_coord(t, geo);
        if (c.seg != prev) {
          bb = j & 1;
          if (!mbar_wait(&bfull[bb], (j >> 1) & 1, status, 0x1300u | bb)) break;
          ++j;
          prev = c.seg;
        }
        const int s = k % kStages;
        const uint32_t ph = (k / kStages) & 1;
        const int a = k & 1;
        if (!mbar_wait(&qfull[s], ph, status, 0x1310u | s)) break;
        if (!mbar_wait(&qrelu[s], ph, status, 0x1320u | s)) break;
        if (!mbar_wait(&acce[a], ((k >> 1) & 1) ^ 1, status, 0x1330u | a)) break;
        tc_fence_after();
        const uint32_t qb = smem_u32(smem + s * kQBytes);
        const uint32_t bbase = smem_u32(smem + kBOff + bb * kPTileBytes);
        const uint32_t dacc = tmem + static_cast<uint32_t>(a * 256);
        for (int kk = 0; kk < ksteps; ++kk) {
          // 16 features per MMA: +32 B inside the 128-B swizzle row, next atom after 4 steps
          const uint64_t ad = sdesc_sw128(qb + (kk >> 2) * kAtomBytes + (kk & 3) * 32, 16, 1024);
          const uint64_t bd = sdesc_sw128(bbase + (kk >> 2) * kBAtomBytes + (kk & 3) * 32, 16, 1024);
          mma_bf16(dacc, ad, bd, kIdescO, kk > 0 ? 1u : 0u);
        }
        mma_commit(&qempty[s]);
        mma_commit(&accf[a]);
        if (c.last || t == te - 1) mma_commit(&bempty[bb]);
      }
      mma_commit(done);
      mbar_wait(done, 0, status, 0x13F0u);
    }
  } else {
    // epilogue: warp w owns tokens 32w..32w+31 of the tile (TMEM lanes)
    uint8_t* ob = smem + kOOff + warp * kOWarpBytes;
    const int ncc = two_atoms ? 4 : 2;
    int k = 0;
    for (long long t = tb; t < te; ++t, ++k) {
      const TileCoord c = tile_coord(t, geo);
      const int a = k & 1;
      bool ok = mbar_wait(&accf[a], (k >> 1) & 1, status, 0x1400u | a);
      if (!warp_all(ok)) break;
      tc_fence_after();
      const uint32_t ta = tmem + (static_cast<uint32_t>(warp * 32) << 16) + static_cast<uint32_t>(a * 256);
      uint32_t dr;
      tmem_ld_x1(ta + kZRow, dr);
      tmem_wait_ld();
      const float inv = __frcp_rn(__uint_as_float(dr) + eps);
      if (lane == 0) bulk_wait_read_all();  // the previous store has finished reading the slice
      __syncwarp();
      for (int cc = 0; cc < ncc; ++cc) {
        uint32_t r[32];
        tmem_ld_x32(ta + cc * 32, r);
        tmem_wait_ld();
#pragma unroll
        for (int m = 0; m < 4; ++m) {
          uint4 w;
          w.x = pack_bf16x2(__uint_as_float(r[8 * m + 0]) * inv, __uint_as_float(r[8 * m + 1]) * inv);
          w.y = pack_bf16x2(__uint_as_float(r[8 * m + 2]) * inv, __uint_as_float(r[8 * m + 3]) * inv);
          w.z = pack_bf16x2(__uint_as_float(r[8 * m + 4]) * inv, __uint_as_float(r[8 * m + 5]) * inv);
          w.w = pack_bf16x2(__uint_as_float(r[8 * m + 6]) * inv, __uint_as_float(r[8 * m + 7]) * inv);
          const int chunk = cc * 4 + m;  // 16-byte chunk of the 256-byte output row
          uint8_t* dst = ob + (chunk >> 3) * 4096 + lane * 128 + (((chunk & 7) ^ (lane & 7)) << 4);
          *reinterpret_cast<uint4*>(dst) = w;
        }
      }
      tc_fence_before();
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&acce[a]);
        const int blen = (c.blk == geo.nblk - 1) ? geo.Llast : geo.L;
        const int row0 = c.tok0 + warp * 32;
        if (row0 < blen) {
          const bool lst = use_last_map(c, geo);
          const CUtensorMap* mo = lst ? &o_last : &o_main;
          const int cb = lst ? 0 : c.blk;
          tma_store_4d(mo, ob, 0, row0, cb, c.bh);
          if (two_atoms) tma_store_4d(mo, ob + 4096, 64, row0, cb, c.bh);
          bulk_commit();
        }
      }
    }
    if (lane == 0) bulk_wait_all();
  }

  __syncthreads();
  if (warp == kWarpMma) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// ------------------------------------------------------------------------------------------
// 2. partial combine + inclusive prefix over blocks (+ incoming cache), both paths
// ------------------------------------------------------------------------------------------
// CTA (bh, row e of the prefix tile): e < 128 are S^T rows (value feature e), e = 128 is z,
// e = 129..143 are the zero rows of the bf16 B operand. Lane q owns key features 4q..4q+3;
// warp j owns blocks [j*nblk/ng, (j+1)*nblk/ng) (at most kScanReg of them when nblk <= 128),
// so every partial load is independent; the running prefix crosses warps through shared memory.
constexpr int kScanReg = 4;
constexpr int kScanMaxWarps = 32;

__device__ __forceinline__ float4 f4add(float4 a, float4 b) {
  return make_float4(a.x + b.x, a.y + b.y, a.z + b.z, a.w + b.w);
}

// Sum of the partial slots g + seg of the CTAs g0..g1 that covered segment `seg` (the state kernel
// records g0/g1 per segment while it flushes).
__device__ __forceinline__ float4 block_sum(const float* __restrict__ partials, const int2* __restrict__ segcta,
                                            int seg, int e, int d0) {
  const int2 r = segcta[seg];
  const int g0 = r.x, g1 = r.y;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int gg = g0; gg <= g1; ++gg)
    acc = f4add(acc, *reinterpret_cast<const float4*>(
                         partials + (static_cast<size_t>(gg + seg) * kPartRows + e) * kDPad + d0));
  return acc;
}

__global__ void __launch_bounds__(1024) scan_kernel(const float* __restrict__ partials,
                                                    const int2* __restrict__ segcta, const Geom geo,
                                                    const float* S_in, const float* z_in, float* S_out,
                                                    float* z_out, uint8_t* __restrict__ ptiles,
                                                    float* __restrict__ p32) {
  griddep_wait();  // partials come from the state kernel; prefix tiles may still be read before it
  griddep_launch_dependents();
  extern __shared__ float4 s_scan[];   // [ng][32] warp totals, then [32] incoming cache
  float4* s_base = s_scan + (blockDim.x >> 5) * 32;
  const int bh = blockIdx.x;
  const int e = blockIdx.y;
  const int q = threadIdx.x & 31;
  const int j = threadIdx.x >> 5;
  const int ng = blockDim.x >> 5;
  const int nblk = geo.nblk;
  const int D = geo.D;
  const int d0 = q * 4;
  const int c0 = static_cast<int>(static_cast<long long>(j) * nblk / ng);
  const int c1 = static_cast<int>(static_cast<long long>(j + 1) * nblk / ng);
  const int cnt = c1 - c0;
  const bool live = e < kPartRows;
  const int seg0 = bh * nblk;

  // pass 1: this warp's block sums (kept in registers) and their total
  float4 sums[kScanReg];
  float4 tot = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
  for (int i = 0; i < kScanReg; ++i) {
    sums[i] = make_float4(0.f, 0.f, 0.f, 0.f);
    if (live && i < cnt) {
      sums[i] = block_sum(partials, segcta, seg0 + c0 + i, e, d0);
      tot = f4add(tot, sums[i]);
    }
  }
  for (int i = kScanReg; i < cnt; ++i)
    if (live) tot = f4add(tot, block_sum(partials, segcta, seg0 + c0 + i, e, d0));

  // incoming cache (S_in row e of S^T, or z_in for the z row)
  float base[4] = {0.f, 0.f, 0.f, 0.f};
  if (j == 0) {
    if (S_in != nullptr && e < D) {
#pragma unroll
      for (int u = 0; u < 4; ++u)
        if (d0 + u < D) base[u] = S_in[(static_cast<size_t>(bh) * D + d0 + u) * D + e];
    }
    if (z_in != nullptr && e == kZRow) {
#pragma unroll
      for (int u = 0; u < 4; ++u)
        if (d0 + u < D) base[u] = z_in[static_cast<size_t>(bh) * D + d0 + u];
    }
  }
  float4 run = make_float4(base[0], base[1], base[2], base[3]);
  if (ng > 1) {
    s_scan[j * 32 + q] = tot;
    if (j == 0) s_base[q] = run;
    __syncthreads();
    run = s_base[q];
    for (int jj = 0; jj < j; ++jj) run = f4add(run, s_scan[jj * 32 + q]);
  }

  // pass 2: running prefix, one prefix tile row chunk per block
  auto emit = [&](int c, const float4& r) {
    const int seg = seg0 + c;
    if (ptiles != nullptr) {
      uint2 w;
      w.x = pack_bf16x2(r.x, r.y);
      w.y = pack_bf16x2(r.z, r.w);
      const size_t off = static_cast<size_t>(seg) * kPTileBytes + (d0 >> 6) * (kPTileRows * 128) + e * 128 +
                         ((((d0 & 63) >> 3) ^ (e & 7)) << 4) + (d0 & 7) * 2;
      *reinterpret_cast<uint2*>(ptiles + off) = w;
    }
    if (p32 != nullptr && live)
      *reinterpret_cast<float4*>(p32 + (static_cast<size_t>(seg) * kPartRows + e) * kDPad + d0) = r;
  };
#pragma unroll
  for (int i = 0; i < kScanReg; ++i) {
    if (i < cnt) {
      run = f4add(run, sums[i]);
      emit(c0 + i, run);
    }
  }
  for (int i = kScanReg; i < cnt; ++i) {
    if (live) run = f4add(run, block_sum(partials, segcta, seg0 + c0 + i, e, d0));
    emit(c0 + i, run);
  }

  // final cache: the warp holding the last block
  if (c1 == nblk && cnt > 0) {
    const float r[4] = {run.x, run.y, run.z, run.w};
    if (S_out != nullptr && e < D) {
#pragma unroll
      for (int u = 0; u < 4; ++u)
        if (d0 + u < D) S_out[(static_cast<size_t>(bh) * D + d0 + u) * D + e] = r[u];
    }
    if (z_out != nullptr && e == kZRow) {
#pragma unroll
      for (int u = 0; u < 4; ++u)
        if (d0 + u < D) z_out[static_cast<size_t>(bh) * D + d0 + u] = r[u];
    }
  }
}

// ------------------------------------------------------------------------------------------
// fp32 I/O path (SIMT fp32; correctness path for fp32 inputs)
// ------------------------------------------------------------------------------------------
__device__ __forceinline__ float relu_f32(float x) { return (x != x) ? x : fmaxf(x, 0.f); }

constexpr int kF32Threads = 256;
constexpr int kStateF32Smem = 2 * kTile * kDPad * 4;                   // K, V tiles
constexpr int kOutF32Smem = kDPad * kPartRows * 4 + kTile * kDPad * 4;  // prefix (transposed), Q tile

__global__ void __launch_bounds__(kF32Threads, 1)
    state_f32_kernel(const float* __restrict__ k, const float* __restrict__ v, const Geom geo,
                     float* __restrict__ partials, int2* __restrict__ segcta) {
  extern __shared__ float fsm[];
  float* Ks = fsm;
  float* Vs = fsm + kTile * kDPad;
  const int D = geo.D;
  const int d = threadIdx.x & 127;
  const int eh = threadIdx.x >> 7;
  const int g = blockIdx.x;
  const long long tb = tile_begin(g, geo);
  const long long te = tile_begin(g + 1, geo);
  float acc[64];
#pragma unroll
  for (int m = 0; m < 64; ++m) acc[m] = 0.f;
  float zacc = 0.f;
  for (long long t = tb; t < te; ++t) {
    const TileCoord c = tile_coord(t, geo);
    const size_t row0 = static_cast<size_t>(c.bh) * geo.N + static_cast<size_t>(c.blk) * geo.L + c.tok0;
    __syncthreads();
    for (int i = threadIdx.x; i < kTile * D; i += kF32Threads) {
      const int rr = i / D, cc = i - rr * D;
      const bool in = rr < c.rows;
      Ks[rr * kDPad + cc] = in ? relu_f32(k[row0 * D + i]) : 0.f;
      Vs[rr * kDPad + cc] = in ? v[row0 * D + i] : 0.f;
    }
    __syncthreads();
    if (d < D) {
      for (int jr = 0; jr < c.rows; ++jr) {
        const float fk = Ks[jr * kDPad + d];
        if (eh == 0) zacc += fk;
#pragma unroll
        for (int m = 0; m < 64; ++m) {
          const int e = eh + 2 * m;
          if (e < D) acc[m] = fmaf(fk, Vs[jr * kDPad + e], acc[m]);
        }
      }
    }
    if (c.last || t == te - 1) {
      float* dst = partials + static_cast<size_t>(g + c.seg) * (kPartRows * kDPad);
#pragma unroll
      for (int m = 0; m < 64; ++m) {
        const int e = eh + 2 * m;
        dst[e * kDPad + d] = (d < D && e < D) ? acc[m] : 0.f;
        acc[m] = 0.f;
      }
      if (eh == 0) dst[kZRow * kDPad + d] = (d < D) ? zacc : 0.f;
      zacc = 0.f;
      if (threadIdx.x == 0) {
        if (t - c.tok0 / kTile >= tb) segcta[c.seg].x = g;
        if (c.last) segcta[c.seg].y = g;
      }
    }
  }
}

__global__ void __launch_bounds__(kF32Threads, 1)
    out_f32_kernel(const float* __restrict__ q, float* __restrict__ o, const Geom geo,
                   const float* __restrict__ p32, const float eps) {
  extern __shared__ float fsm[];
  float* Ps = fsm;                      // [d][e'] with e' = 0..128 (z at 128)
  float* Qs = fsm + kDPad * kPartRows;  // [row][d]
  const int D = geo.D;
  const int g = blockIdx.x;
  const long long tb = tile_begin(g, geo);
  const long long te = tile_begin(g + 1, geo);
  const int e = threadIdx.x & 127;
  const int rh = threadIdx.x >> 7;
  int prev = -1;
  for (long long t = tb; t < te; ++t) {
    const TileCoord c = tile_coord(t, geo);
    const size_t row0 = static_cast<size_t>(c.bh) * geo.N + static_cast<size_t>(c.blk) * geo.L + c.tok0;
    __syncthreads();
    if (c.seg != prev) {
      const float* src = p32 + static_cast<size_t>(c.seg) * kPartRows * kDPad;
      for (int i = threadIdx.x; i < kPartRows * kDPad; i += kF32Threads) {
        const int ee = i / kDPad, dd = i - ee * kDPad;
        Ps[dd * kPartRows + ee] = src[i];
      }
      prev = c.seg;
    }
    for (int i = threadIdx.x; i < kTile * D; i += kF32Threads) {
      const int rr = i / D, cc = i - rr * D;
      Qs[rr * kDPad + cc] = rr < c.rows ? relu_f32(q[row0 * D + i]) : 0.f;
    }
    __syncthreads();
    if (e < D) {
      for (int m = 0; m < 64; ++m) {
        const int rr = rh + 2 * m;
        if (rr >= c.rows) break;
        float num = 0.f, den = 0.f;
        for (int dd = 0; dd < D; ++dd) {
          const float fq = Qs[rr * kDPad + dd];
          num = fmaf(fq, Ps[dd * kPartRows + e], num);
          den = fmaf(fq, Ps[dd * kPartRows + kZRow], den);
        }
        o[(row0 + rr) * D + e] = num / (den + eps);
      }
    }
  }
}

}  // namespace

// ------------------------------------------------------------------------------------------
// launchers
// ------------------------------------------------------------------------------------------
// Every launch allows programmatic dependent launch: a kernel may be scheduled while the previous
// one in the stream drains, and each kernel waits (griddepcontrol.wait) before touching memory
// that the previous kernels write or still read.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                       Args&&... args) {
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
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

size_t state_bf16_smem_bytes() { return st::kSmemBytes; }
size_t out_bf16_smem_bytes() { return ot::kSmemBytes; }
size_t state_f32_smem_bytes() { return kStateF32Smem; }
size_t out_f32_smem_bytes() { return kOutF32Smem; }

cudaError_t set_kernel_attributes() {
  cudaError_t e;
  e = cudaFuncSetAttribute(state_bf16_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, st::kSmemBytes);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(out_bf16_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, ot::kSmemBytes);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(state_f32_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kStateF32Smem);
  if (e != cudaSuccess) return e;
  return cudaFuncSetAttribute(out_f32_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kOutF32Smem);
}

cudaError_t launch_state_bf16(const BlockMaps& k, const BlockMaps& v, const Geom& g, float* partials, int2* segcta,
                              uint32_t* status, cudaStream_t s) {
  return launch_pdl(state_bf16_kernel, dim3(g.G), dim3(kThreads), st::kSmemBytes, s, k.main, k.last, v.main, v.last,
                    g, partials, segcta, status);
}

cudaError_t launch_out_bf16(const BlockMaps& q, const BlockMaps& o, const Geom& g, const void* ptiles, float eps,
                            uint32_t* status, cudaStream_t s) {
  return launch_pdl(out_bf16_kernel, dim3(g.G), dim3(kThreads), ot::kSmemBytes, s, q.main, q.last, o.main, o.last,
                    g, static_cast<const uint8_t*>(ptiles), eps, status);
}

cudaError_t launch_scan(const float* partials, const int2* segcta, const Geom& g, const float* S_in, const float* z_in, float* S_out,
                        float* z_out, void* ptiles_bf16, float* p32, cudaStream_t s) {
  int ng = (g.nblk + kScanReg - 1) / kScanReg;
  if (ng > kScanMaxWarps) ng = kScanMaxWarps;
  if (ng < 1) ng = 1;
  return launch_pdl(scan_kernel, dim3(g.BH, kPTileRows), dim3(32 * ng), (ng + 1) * 32 * sizeof(float4), s,
                    partials, segcta, g, S_in, z_in, S_out,
                    z_out, static_cast<uint8_t*>(ptiles_bf16), p32);
}

cudaError_t launch_state_f32(const float* k, const float* v, const Geom& g, float* partials, int2* segcta,
                             uint32_t*, cudaStream_t s) {
  state_f32_kernel<<<g.G, kF32Threads, kStateF32Smem, s>>>(k, v, g, partials, segcta);
  return cudaGetLastError();
}

cudaError_t launch_out_f32(const float* q, float* o, const Geom& g, const float* p32, float eps, uint32_t*,
                           cudaStream_t s) {
  out_f32_kernel<<<g.G, kF32Threads, kOutF32Smem, s>>>(q, o, g, p32, eps);
  return cudaGetLastError();
}

}  // namespace sv
