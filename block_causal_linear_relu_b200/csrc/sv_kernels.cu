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
// When every head is a single block (bidirectional layer, streaming step), one launch runs the three
// steps: cluster_bf16_kernel when the heads are few (one thread-block cluster per head, the partial
// states exchanged through distributed shared memory), otherwise fused_bf16_kernel (co-resident CTAs:
// the state roles, a per-head combine shared by the CTAs that cover the head, synchronised through
// release/acquire flags, then the output roles).
// The fp32 I/O path runs the same three steps with SIMT fp32 kernels.
// With the 3D rotary embedding (sv_block_causal_attn_rope) the three-kernel path turns the
// feature-mapped K and Q tiles in shared memory after the MMAs that need them unturned (the z
// column of the state, the denominator of the output) have read them, and before the MMAs of the
// numerator: the ReLU warps run one tile behind with the turn.
#include <cuda_bf16.h>

#include <cstdlib>
#include <mutex>
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

// ---- 3D rotary embedding of the feature-mapped features (numerator of the rotated form) ----
// Copies the compact table (RopeDev) into shared memory at `ct`, by `nthreads` threads (index i0).
// The table may come from the previous kernel in the stream: the caller has passed griddepcontrol.wait.
__device__ void stage_rope_table(float2* ct, const RopeDev& rp, int i0, int nthreads) {
  const int ph = rp.pth - rp.pt, pw = rp.half - rp.pth;
  const int e_t = rp.nf * rp.pt, e_h = e_t + rp.h * ph;
  for (int i = i0; i < rp.compact; i += nthreads) {
    int row, j;
    if (i < e_t) {
      row = rp.f0 + i / rp.pt, j = i % rp.pt;
    } else if (i < e_h) {
      row = rp.row_h + (i - e_t) / ph, j = rp.pt + (i - e_t) % ph;
    } else {
      row = rp.row_w + (i - e_h) / pw, j = rp.pth + (i - e_h) % pw;
    }
    ct[i] = __ldg(rp.tab + static_cast<size_t>(row) * rp.half + j);
  }
}
__device__ __forceinline__ float2 ld_shared_f2(uint32_t a) {
  float2 v;
  asm volatile("ld.shared.v2.f32 {%0, %1}, [%2];" : "=f"(v.x), "=f"(v.y) : "r"(a));
  return v;
}
__device__ __forceinline__ uint4 ld_shared_u4(uint32_t a) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(a));
  return v;
}
__device__ __forceinline__ void st_shared_u4(uint32_t a, const uint4& v) {
  asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(a), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
               : "memory");
}
// Shared-memory byte addresses such that pair j of token n's frame / row / column group sits at
// base + 8 j in the compact table at `ct` (each group's entries start at its first pair).
__device__ __forceinline__ void rope_rows_smem(const RopeDev& rp, uint32_t ct, int n, uint32_t& bt, uint32_t& bh,
                                               uint32_t& bw) {
  const int f = n / rp.hw;
  const int rem = n - f * rp.hw;
  const int y = rem / rp.w;
  const int x = rem - y * rp.w;
  const int ph = rp.pth - rp.pt, pw = rp.half - rp.pth;
  const int e_t = rp.nf * rp.pt;
  bt = ct + 8u * static_cast<uint32_t>(f * rp.pt);
  bh = ct + 8u * static_cast<uint32_t>(e_t + y * ph - rp.pt);
  bw = ct + 8u * static_cast<uint32_t>(e_t + rp.h * ph + x * pw - rp.pth);
}
// Table rows of token n's frame, grid row and grid column (the table in global memory).
__device__ __forceinline__ void rope_rows(const RopeDev& rp, int n, const float2*& rt, const float2*& rh,
                                          const float2*& rw) {
  const int f = n / rp.hw;
  const int rem = n - f * rp.hw;
  const int y = rem / rp.w;
  const int x = rem - y * rp.w;
  rt = rp.tab + static_cast<size_t>(rp.f0 + f) * rp.half;
  rh = rp.tab + static_cast<size_t>(rp.row_h + y) * rp.half;
  rw = rp.tab + static_cast<size_t>(rp.row_w + x) * rp.half;
}
// (cos, sin) of pair j: the frame's, the row's or the column's table row by the pair's group.
__device__ __forceinline__ float2 rope_cs(const RopeDev& rp, int j, const float2* rt, const float2* rh,
                                          const float2* rw) {
  return __ldg((j < rp.pt ? rt : (j < rp.pth ? rh : rw)) + j);
}
__device__ __forceinline__ float2 turn_pair(float a, float b, float2 cs) {
  return make_float2(fmaf(a, cs.x, -b * cs.y), fmaf(a, cs.y, b * cs.x));
}

// M consecutive 16-byte chunks c0 .. c0 + M - 1 (one atom) of one tile row at `arow`: every load
// of the group is issued before the first use; straight-line code for the compiler to schedule.
template <bool kSmem, int M>
__device__ __forceinline__ void turn_group(uint32_t arow, int c0, int r7, int pt, int pth, uint32_t bt, uint32_t bh,
                                           uint32_t bw, const float2* rt, const float2* rh, const float2* rw) {
  uint4 x[M];
  float2 cs[M][4];
#pragma unroll
  for (int i = 0; i < M; ++i) x[i] = ld_shared_u4(arow + (static_cast<uint32_t>(((c0 + i) & 7) ^ r7) << 4));
#pragma unroll
  for (int i = 0; i < M; ++i)
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int j = 4 * (c0 + i) + u;
      if constexpr (kSmem)
        cs[i][u] = ld_shared_f2((j < pt ? bt : (j < pth ? bh : bw)) + 8u * j);
      else
        cs[i][u] = __ldg((j < pt ? rt : (j < pth ? rh : rw)) + j);
    }
#pragma unroll
  for (int i = 0; i < M; ++i) {
    uint32_t* w = reinterpret_cast<uint32_t*>(&x[i]);
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const float2 ab = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[u]));
      const float2 t = turn_pair(ab.x, ab.y, cs[i][u]);
      w[u] = pack_bf16x2(t.x, t.y);
    }
    st_shared_u4(arow + (static_cast<uint32_t>(((c0 + i) & 7) ^ r7) << 4), x[i]);
  }
}

// The nca chunks (features < D) of one atom of one tile row at `arow`, logical chunks cbase ..:
// a full atom as one straight-line group, a partial one four chunks at a time.
template <bool kSmem>
__device__ __forceinline__ void turn_atom(uint32_t arow, int cbase, int nca, int r7, int pt, int pth, uint32_t bt,
                                          uint32_t bh, uint32_t bw, const float2* rt, const float2* rh,
                                          const float2* rw) {
  if (nca == 8) {
    turn_group<kSmem, 8>(arow, cbase, r7, pt, pth, bt, bh, bw, rt, rh, rw);
    return;
  }
  for (int c0 = 0; c0 < nca; c0 += 4) {
    switch (nca - c0) {
      case 1: turn_group<kSmem, 1>(arow, cbase + c0, r7, pt, pth, bt, bh, bw, rt, rh, rw); break;
      case 2: turn_group<kSmem, 2>(arow, cbase + c0, r7, pt, pth, bt, bh, bw, rt, rh, rw); break;
      case 3: turn_group<kSmem, 3>(arow, cbase + c0, r7, pt, pth, bt, bh, bw, rt, rh, rw); break;
      default: turn_group<kSmem, 4>(arow, cbase + c0, r7, pt, pth, bt, bh, bw, rt, rh, rw); break;
    }
  }
}

// Turns the feature pairs (2p, 2p + 1) of atom `atom` (features 64 atom .. 64 atom + 63) of row r
// of a 128-row bf16 tile of swizzle-128B atoms in place, if r < rows; row r is token n0 + r. A
// warpgroup (128 threads, thread r owning row r) turns one atom of the whole tile: the row's
// position (frame, grid row, column) is found once and its 16-byte chunks are independent of one
// another. Logical chunk c of a row sits at physical chunk c ^ (r % 8), so at each step the eight
// rows r..r+7 touch eight different chunks and a warp's 16-byte accesses are free of bank
// conflicts. (cos, sin) come from the compact table in shared memory at `ct` when
// rp.compact > 0, else from the table in global memory; the choice is made once, outside the loops.
__device__ __forceinline__ void rope_tile_inplace(uint8_t* tile, int atom, int r, int n0, int rows, const RopeDev& rp,
                                                  uint32_t ct) {
  const int nca = min(8, rp.half / 4 - 8 * atom);  // chunks of this atom holding features < D
  if (r >= rows || nca <= 0) return;
  const int pt = rp.pt, pth = rp.pth;
  const uint32_t arow = smem_u32(tile) + static_cast<uint32_t>(atom * kAtomBytes + r * 128);
  if (rp.compact > 0) {
    uint32_t bt, bh, bw;
    rope_rows_smem(rp, ct, n0 + r, bt, bh, bw);
    turn_atom<true>(arow, 8 * atom, nca, r & 7, pt, pth, bt, bh, bw, nullptr, nullptr, nullptr);
  } else {
    const float2 *rt, *rh, *rw;
    rope_rows(rp, n0 + r, rt, rh, rw);
    turn_atom<false>(arow, 8 * atom, nca, r & 7, pt, pth, 0u, 0u, 0u, rt, rh, rw);
  }
}

__device__ __forceinline__ bool use_last_map(const TileCoord& c, const Geom& g) {
  return c.blk == g.nblk - 1 && g.Llast != g.L;
}

// ------------------------------------------------------------------------------------------
// Pipeline roles. Each persistent kernel runs one CTA per SM with ten warps: warps 0-3 drain the
// TMEM accumulator (epilogue), warps 4-7 apply ReLU in shared memory (and, in the output roles with
// D > 64, drain the second half of the output columns), one thread of warp 8 issues TMA copies, one
// thread of warp 9 issues tcgen05.mma. The roles below are shared by the stand-alone kernels and by
// the single-launch kernels.
// ------------------------------------------------------------------------------------------
struct Maps4 {
  const CUtensorMap* a_main;
  const CUtensorMap* a_last;
  const CUtensorMap* b_main;
  const CUtensorMap* b_last;
};

// generic-proxy writes to global memory (other CTAs) -> visible to this thread's async-proxy copies
__device__ __forceinline__ void fence_proxy_async_global() {
  asm volatile("fence.proxy.async.global;" ::: "memory");
}

// ---- flags between CTAs of the single-launch kernel (release / acquire at GPU scope) ----
__device__ __forceinline__ void st_release_u64(uint64_t* p, uint64_t v) {
  asm volatile("st.release.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}
__device__ __forceinline__ uint32_t atom_add_acq_rel_u32(uint32_t* p, uint32_t v) {
  uint32_t old;
  asm volatile("atom.add.acq_rel.gpu.global.u32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
  return old;
}
__device__ __forceinline__ uint64_t ld_acquire_u64(const uint64_t* p) {
  uint64_t v;
  asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ uint64_t ld_relaxed_u64(const uint64_t* p) {
  uint64_t v;
  asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
  return v;
}
// Waits (bounded) until flags[i] == tag for every i in [i0, i1]; one thread. Up to eight flags are
// read per round trip; the fence after the last one orders everything the flag writers released.
__device__ bool wait_flags(const uint64_t* flags, int i0, int i1, uint64_t tag, uint32_t* status, uint32_t where) {
  const uint64_t t0 = globaltimer_ns();
  int i = i0;
  while (i <= i1) {
    const int n = (i1 - i + 1) < 8 ? (i1 - i + 1) : 8;
    uint64_t v[8];
#pragma unroll
    for (int u = 0; u < 8; ++u)
      if (u < n) v[u] = ld_relaxed_u64(flags + i + u);
    int ready = 0;
#pragma unroll
    for (int u = 0; u < 8; ++u)
      if (u < n && ready == u && v[u] == tag) ++ready;
    i += ready;
    if (ready < n) {
      if (*reinterpret_cast<volatile uint32_t*>(status) != 0u) return false;
      if (globaltimer_ns() - t0 > kWaitLimitNs) {
        raise_status(status, kDevTimeout | where);
        return false;
      }
      __nanosleep(32);
    }
  }
  __threadfence();
  return true;
}

// ---- 1. block-state reduction: ReLU(K)^T [V | 1] accumulated over the tiles of each segment ----
namespace st {
constexpr int kStages = 3;
constexpr int kKBytes = 2 * kAtomBytes;          // K tile: 128 tokens x 128 features (two atoms)
constexpr int kStageBytes = 2 * kKBytes;         // K + V
constexpr int kOnesOff = kStages * kStageBytes;  // 16 token rows of bf16 ones: B operand of the z column
constexpr int kOnesBytes = 2048;
constexpr int kRegionBytes = kOnesOff + kOnesBytes;
constexpr int kNumBars = 14;

struct Bars {
  uint64_t* full;   // [3] TMA landed (K and V)
  uint64_t* relu;   // [3] ReLU(K) written back
  uint64_t* empty;  // [3] MMAs reading the stage retired
  uint64_t* accf;   // [2] accumulator holds a finished segment piece
  uint64_t* acce;   // [2] accumulator drained by the epilogue
  uint64_t* done;   // every MMA retired
};
__device__ __forceinline__ Bars bars_at(uint64_t* p) { return Bars{p, p + 3, p + 6, p + 9, p + 11, p + 13}; }
__device__ __forceinline__ void init_bars(const Bars& b) {
  for (int i = 0; i < kStages; ++i) {
    mbar_init(&b.full[i], 1);
    mbar_init(&b.relu[i], 4);
    mbar_init(&b.empty[i], 1);
  }
  for (int a = 0; a < 2; ++a) {
    mbar_init(&b.accf[a], 1);
    mbar_init(&b.acce[a], 4);
  }
  mbar_init(b.done, 1);
}
// shared memory the MMA reads as constants: ones for the z column; zeros for features >= 64 when D <= 64
__device__ __forceinline__ void init_smem(uint8_t* smem, bool two_atoms, int nthreads) {
  uint4* ones = reinterpret_cast<uint4*>(smem + kOnesOff);
  const uint4 one = make_uint4(0x3F803F80u, 0x3F803F80u, 0x3F803F80u, 0x3F803F80u);
  for (int i = threadIdx.x; i < kOnesBytes / 16; i += nthreads) ones[i] = one;
  if (!two_atoms) {
    for (int s = 0; s < kStages; ++s) {
      uint4* kz = reinterpret_cast<uint4*>(smem + s * kStageBytes + kAtomBytes);
      uint4* vz = reinterpret_cast<uint4*>(smem + s * kStageBytes + kKBytes + kAtomBytes);
      for (int i = threadIdx.x; i < kAtomBytes / 16; i += nthreads) {
        kz[i] = make_uint4(0, 0, 0, 0);
        vz[i] = make_uint4(0, 0, 0, 0);
      }
    }
  }
  fence_proxy_async_smem();
}

// Producer. `wait_first`: K and V (and the partial slots) may belong to the previous kernel in the
// stream, so nothing is touched before griddepcontrol.wait. Returns once every stage it filled has
// been consumed by the MMAs, so the caller may reuse the stage memory.
__device__ void produce(uint8_t* smem, const Bars& b, const Maps4& m, const Geom& geo, long long tb, long long te,
                        bool two_atoms, bool wait_first, uint32_t* status) {
  const uint64_t pol = policy_evict_first();
  const uint32_t tx = two_atoms ? 2u * kKBytes : static_cast<uint32_t>(kKBytes);
  if (wait_first) griddep_wait();
  int k = 0;
  for (long long t = tb; t < te; ++t, ++k) {
    const TileCoord c = tile_coord(t, geo);
    const int s = k % kStages;
    if (!mbar_wait(&b.empty[s], ((k / kStages) & 1) ^ 1, status, 0x0100u | s)) break;
    const bool lst = use_last_map(c, geo);
    const CUtensorMap* mk = lst ? m.a_last : m.a_main;
    const CUtensorMap* mv = lst ? m.b_last : m.b_main;
    const int cb = lst ? 0 : c.blk;
    uint8_t* stg = smem + s * kStageBytes;
    mbar_expect_tx(&b.full[s], tx);
    tma_load_4d(stg, mk, &b.full[s], 0, c.tok0, cb, c.bh, pol);
    tma_load_4d(stg + kKBytes, mv, &b.full[s], 0, c.tok0, cb, c.bh, pol);
    if (two_atoms) {
      tma_load_4d(stg + kAtomBytes, mk, &b.full[s], 64, c.tok0, cb, c.bh, pol);
      tma_load_4d(stg + kKBytes + kAtomBytes, mv, &b.full[s], 64, c.tok0, cb, c.bh, pol);
    }
  }
  for (int j = (k > kStages ? k - kStages : 0); j < k; ++j)
    mbar_wait(&b.empty[j % kStages], (j / kStages) & 1, status, 0x0180u);
}

__device__ void relu_role(uint8_t* smem, const Bars& b, long long tb, long long te, bool two_atoms, int r, int lane,
                          uint32_t* status) {
  const int nchunks = (two_atoms ? kKBytes : kAtomBytes) / 16;
  int k = 0;
  for (long long t = tb; t < te; ++t, ++k) {
    const int s = k % kStages;
    bool ok = mbar_wait(&b.full[s], (k / kStages) & 1, status, 0x0200u | s);
    if (!warp_all(ok)) break;
    relu_tile_inplace(smem + s * kStageBytes, nchunks, r);
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) mbar_arrive(&b.relu[s]);
  }
}

// Rotary form only: per stage, the z products of a tile retired (the turn may overwrite the
// features) and the tile turned (the S products may read it).
struct RopeBars {
  uint64_t* zd;   // [3] count 1 (tcgen05.commit)
  uint64_t* rot;  // [3] one arrival per turning warp: 4 (one atom) or 8 (two atoms)
};
constexpr int kRopeBars = 2 * kStages;
__device__ __forceinline__ RopeBars rope_bars_at(uint64_t* p) { return RopeBars{p, p + kStages}; }
__device__ __forceinline__ void init_rope_bars(const RopeBars& rb, bool two_atoms) {
  for (int i = 0; i < kStages; ++i) {
    mbar_init(&rb.zd[i], 1);
    mbar_init(&rb.rot[i], two_atoms ? 8 : 4);
  }
}

// The rotary form's (cos, sin) table is staged by the turning warps (the ReLU warps and, with two
// atoms, the epilogue warps: nthreads 128 or 256, thread index i0), which then meet on barrier 1.
// The table may be the previous kernel's output, hence griddepcontrol.wait first (K and V are not
// read before it anyway).
__device__ __forceinline__ void stage_and_sync(float2* ct, const RopeDev& rp, int i0, int nthreads) {
  griddep_wait();
  stage_rope_table(ct, rp, i0, nthreads);
  asm volatile("bar.sync 1, %0;" ::"r"(nthreads) : "memory");
}

// Turn of atom `atom` of the k-th tile (global tile t) of this CTA once its z products retired.
__device__ __forceinline__ bool turn_k(uint8_t* smem, const RopeBars& rb, const Geom& geo, int k, long long t,
                                       int atom, int r, int lane, const RopeDev& rp, uint32_t ct, uint32_t* status) {
  const int s = k % kStages;
  const bool ok = mbar_wait(&rb.zd[s], (k / kStages) & 1, status, 0x0240u | s);
  if (!warp_all(ok)) return false;
  const TileCoord c = tile_coord(t, geo);
  rope_tile_inplace(smem + s * kStageBytes, atom, r, c.blk * geo.L + c.tok0, c.rows, rp, ct);
  fence_proxy_async_smem();
  __syncwarp();
  if (lane == 0) mbar_arrive(&rb.rot[s]);
  return true;
}

// relu_role of the rotary form: ReLU of tile k, then (once the MMA warp's z products of the
// unturned tile retired) the turn of its atom 0; the epilogue warps turn atom 1.
// The kernel's Geom and RopeDev are copied into registers here: read through references into the
// parameter space they would be generic loads of long latency on the turn's critical path.
__device__ void relu_rope_role(uint8_t* smem, const Bars& b, const RopeBars& rb, const Geom& geo_p, long long tb,
                               long long te, bool two_atoms, int r, int lane, const RopeDev& rp_p, float2* ct,
                               uint32_t* status) {
  const Geom geo = geo_p;
  const RopeDev rp = rp_p;
  const int nchunks = (two_atoms ? kKBytes : kAtomBytes) / 16;
  stage_and_sync(ct, rp, two_atoms ? 128 + r : r, two_atoms ? 256 : 128);
  const uint32_t cta = smem_u32(ct);
  int k = 0;
  for (long long t = tb; t < te; ++t, ++k) {
    const int s = k % kStages;
    bool ok = mbar_wait(&b.full[s], (k / kStages) & 1, status, 0x0200u | s);
    if (!warp_all(ok)) return;
    relu_tile_inplace(smem + s * kStageBytes, nchunks, r);
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) mbar_arrive(&b.relu[s]);
    if (!turn_k(smem, rb, geo, k, t, 0, r, lane, rp, cta, status)) return;
  }
}

// What the epilogue warps of the rotary form turn (atom 1 of every tile, with two atoms).
struct TurnCtx {
  uint8_t* smem;
  RopeBars rb;
  const RopeDev* rp;
  float2* ct;
};

template <bool kRope>
__device__ void mma_issue(uint8_t* smem, const Bars& b, const Geom& geo, long long tb, long long te, uint32_t tmem,
                          uint32_t* status, const RopeBars* rb) {
  constexpr uint32_t kIdescS = idesc_bf16_f32(128, 128, true, true);
  constexpr uint32_t kIdescZ = idesc_bf16_f32(128, 16, true, true);
  const uint64_t od = sdesc_sw128(smem_u32(smem + kOnesOff), kAtomBytes, 1024);  // same 16 rows of ones each step
  int k = 0, j = 0;
  for (long long t = tb; t < te; ++t, ++k) {
    const TileCoord c = tile_coord(t, geo);
    const bool first = (t == tb) || c.tok0 == 0;
    const bool end = c.last || t == te - 1;
    const int a = j & 1;
    const int s = k % kStages;
    const uint32_t ph = (k / kStages) & 1;
    if (first && !mbar_wait(&b.acce[a], ((j >> 1) & 1) ^ 1, status, 0x0300u | a)) break;
    if (!mbar_wait(&b.full[s], ph, status, 0x0310u | s)) break;
    if (!mbar_wait(&b.relu[s], ph, status, 0x0320u | s)) break;
    tc_fence_after();
    const uint32_t kb = smem_u32(smem + s * kStageBytes);
    const uint32_t vb = kb + kKBytes;
    const uint32_t dacc = tmem + static_cast<uint32_t>(a * 256);
    if constexpr (kRope) {
      // z from the unturned ReLU(K), then S from the turned tile
#pragma unroll
      for (int kk = 0; kk < kTile / 16; ++kk)
        mma_bf16(dacc + 128, sdesc_sw128(kb + kk * 2048, kAtomBytes, 1024), od, kIdescZ,
                 (first && kk == 0) ? 0u : 1u);
      mma_commit(&rb->zd[s]);
      if (!mbar_wait(&rb->rot[s], ph, status, 0x0330u | s)) break;
      tc_fence_after();
#pragma unroll
      for (int kk = 0; kk < kTile / 16; ++kk)
        mma_bf16(dacc, sdesc_sw128(kb + kk * 2048, kAtomBytes, 1024), sdesc_sw128(vb + kk * 2048, kAtomBytes, 1024),
                 kIdescS, (first && kk == 0) ? 0u : 1u);
    } else {
#pragma unroll
      for (int kk = 0; kk < kTile / 16; ++kk) {
        // 16 tokens per MMA: two groups of 8 token rows (128 B each) -> +2048 B per step
        const uint64_t ad = sdesc_sw128(kb + kk * 2048, kAtomBytes, 1024);
        const uint64_t bd = sdesc_sw128(vb + kk * 2048, kAtomBytes, 1024);
        const uint32_t acc = (first && kk == 0) ? 0u : 1u;
        mma_bf16(dacc, ad, bd, kIdescS, acc);         // S^T columns: ReLU(K)^T V
        mma_bf16(dacc + 128, ad, od, kIdescZ, acc);   // z column: ReLU(K)^T 1
      }
    }
    mma_commit(&b.empty[s]);
    if (end) {
      mma_commit(&b.accf[a]);
      ++j;
    }
  }
  mma_commit(b.done);
  mbar_wait(b.done, 0, status, 0x03F0u);
}
__device__ __forceinline__ void mma_role(uint8_t* smem, const Bars& b, const Geom& geo, long long tb, long long te,
                                         uint32_t tmem, uint32_t* status) {
  mma_issue<false>(smem, b, geo, tb, te, tmem, status, nullptr);
}

// Epilogue: warp w drains TMEM lanes 32w..32w+31 (key feature d) into the partial slot g + segment,
// and records which CTAs hold a segment's first and last tile.
// With `slot_ready`, every flushed slot is then published for other CTAs (value `tag`): the four
// warps meet on the CTA barrier `flushed` (count 4) and warp 0 releases the slot's flag.
// With `tc` (rotary form, two atoms) the four warps first turn atom 1 of each tile, in order.
__device__ void epilogue_role(const Bars& b, const Geom& geo, long long tb, long long te, uint32_t tmem, int g,
                              int warp, int lane, float* __restrict__ partials, int2* __restrict__ segcta,
                              uint64_t* slot_ready, uint64_t* flushed, uint64_t tag, uint32_t* status,
                              const TurnCtx* tc = nullptr) {
  const int d = warp * 32 + lane;
  int j = 0;
  RopeDev rp{};
  uint32_t cta = 0;
  if (tc != nullptr) {
    rp = *tc->rp;
    stage_and_sync(tc->ct, rp, d, 256);
    cta = smem_u32(tc->ct);
  }
  for (long long t = tb; t < te; ++t) {
    if (tc != nullptr && !turn_k(tc->smem, tc->rb, geo, static_cast<int>(t - tb), t, 1, d, lane, rp, cta, status))
      break;
    const TileCoord c = tile_coord(t, geo);
    if (!(c.last || t == te - 1)) continue;
    const int a = j & 1;
    bool ok = mbar_wait(&b.accf[a], (j >> 1) & 1, status, 0x0400u | a);
    if (!warp_all(ok)) break;
    tc_fence_after();
    const uint32_t ta = tmem + (static_cast<uint32_t>(warp * 32) << 16) + static_cast<uint32_t>(a * 256);
    float* dst = partials + static_cast<size_t>(g + c.seg) * (kPartRows * kDPad);
    // two halves of 64 columns, each read with one wait (the register budget holds 64 values)
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      uint32_t rr[2][32];
      uint32_t zr = 0;
      tmem_ld_x32(ta + h * 64, rr[0]);
      tmem_ld_x32(ta + h * 64 + 32, rr[1]);
      if (h == 1) tmem_ld_x1(ta + 128, zr);
      tmem_wait_ld();
      if (h == 1) {
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&b.acce[a]);  // the accumulator is free once the values are in registers
      }
#pragma unroll
      for (int cc = 0; cc < 2; ++cc)
#pragma unroll
        for (int jj = 0; jj < 32; ++jj) dst[(h * 64 + cc * 32 + jj) * kDPad + d] = __uint_as_float(rr[cc][jj]);
      if (h == 1) dst[kZRow * kDPad + d] = __uint_as_float(zr);
    }
    if (warp == 0 && lane == 0) {
      if (t - c.tok0 / kTile >= tb) segcta[c.seg].x = g;
      if (c.last) segcta[c.seg].y = g;
    }
    if (slot_ready != nullptr) {
      __syncwarp();
      if (lane == 0) {
        __threadfence();
        mbar_arrive(flushed);
        // every warp sees this flush complete before it can arrive for the next one
        const bool all_written = mbar_wait(flushed, j & 1, status, 0x0480u);
        if (warp == 0 && all_written) st_release_u64(slot_ready + g + c.seg, tag);
      }
    }
    ++j;
  }
}
}  // namespace st

// ---- 3. output GEMM ReLU(Q) [P | z]^T with the normalising divide in the epilogue ----
namespace ot {
constexpr int kStages = 3;
constexpr int kQBytes = 2 * kAtomBytes;             // Q tile: 128 tokens x 128 features
constexpr int kBOff = kStages * kQBytes;            // two prefix tiles (double-buffered)
constexpr int kBAtomBytes = kPTileRows * 128;       // 144 rows x 128 B
constexpr int kOOff = kBOff + 2 * kPTileBytes;      // output staging, one 8 KB slice per warp
constexpr int kOWarpBytes = 2 * 32 * 128;      // two 4 KB atoms: output columns 0..63 and 64..127
constexpr int kAtomBytesO = 32 * 128;
constexpr int kRegionBytes = kOOff + 4 * kOWarpBytes;
constexpr int kNumBars = 18;
static_assert(kBOff % 1024 == 0 && kOOff % 1024 == 0 && kBAtomBytes % 1024 == 0, "1024-B atoms");

struct Bars {
  uint64_t* qfull;   // [3]
  uint64_t* qrelu;   // [3]
  uint64_t* qempty;  // [3]
  uint64_t* bfull;   // [2]
  uint64_t* bempty;  // [2]
  uint64_t* accf;    // [2]
  uint64_t* acce;    // [2]
  uint64_t* done;
};
__device__ __forceinline__ Bars bars_at(uint64_t* p) {
  return Bars{p, p + 3, p + 6, p + 9, p + 11, p + 13, p + 15, p + 17};
}
// The epilogue of a tile runs on 4 warps per 64 output columns: 8 warps for D > 64, else 4.
__device__ __forceinline__ int epi_warps(bool two_atoms) { return two_atoms ? 8 : 4; }

__device__ __forceinline__ void init_bars(const Bars& b, bool two_atoms) {
  for (int i = 0; i < kStages; ++i) {
    mbar_init(&b.qfull[i], 1);
    mbar_init(&b.qrelu[i], 4);
    mbar_init(&b.qempty[i], 1);
  }
  for (int a = 0; a < 2; ++a) {
    mbar_init(&b.bfull[a], 1);
    mbar_init(&b.bempty[a], 1);
    mbar_init(&b.accf[a], 1);
    mbar_init(&b.acce[a], epi_warps(two_atoms));
  }
  mbar_init(b.done, 1);
}

__device__ __forceinline__ void load_q(uint8_t* smem, const Bars& b, const Maps4& m, const Geom& geo,
                                       const TileCoord& c, int s, bool two_atoms, uint64_t pol) {
  const bool lst = use_last_map(c, geo);
  const CUtensorMap* mq = lst ? m.a_last : m.a_main;
  const int cb = lst ? 0 : c.blk;
  uint8_t* stg = smem + s * kQBytes;
  mbar_expect_tx(&b.qfull[s], two_atoms ? static_cast<uint32_t>(kQBytes) : static_cast<uint32_t>(kAtomBytes));
  tma_load_4d(stg, mq, &b.qfull[s], 0, c.tok0, cb, c.bh, pol);
  if (two_atoms) tma_load_4d(stg + kAtomBytes, mq, &b.qfull[s], 64, c.tok0, cb, c.bh, pol);
}

// The output tiles of a CTA: its static range [tb, te), then, when `counter` is set, chunks of
// kDynChunk tiles of [dyn_begin, dyn_end) claimed through an atomic counter by whichever CTA gets
// there first (output tiles are independent, so the result does not depend on who computes what).
// The producer walks the sequence and writes the k-th tile's coordinates into ring[k % kRing]
// (x = segment, y = (batch, head), z = block, w = first token in the block) before the barrier the
// other roles wait on for that tile (qfull); x = -1 ends the sequence. The MMA and epilogue loops
// thus do no index arithmetic of their own: on one thread a tile's coordinates cost a 64-bit
// division chain, which sat on the critical path of short sequences.
// An entry is rewritten (tile k + kRing) only after the MMAs of tile k + kRing - kStages retired,
// by which time every role has read entry k.
constexpr int kRing = 8;
constexpr int kDynChunk = kOutChunk;
constexpr int kRingBytes = kRing * 16;
struct Seq {
  long long tb, te;
  long long dyn_begin, dyn_end;
  uint32_t* counter;
  volatile int4* ring;
};
__device__ __forceinline__ void ring_put(const Seq& sq, int k, const TileCoord& c) {
  volatile int4* e = sq.ring + (k % kRing);
  e->y = c.bh;
  e->z = c.blk;
  e->w = c.tok0;
  e->x = c.seg;
}
__device__ __forceinline__ void ring_end(const Seq& sq, int k) { sq.ring[k % kRing].x = -1; }

// Q was final before the state reduction ran, so the first stages of the static range can fill
// before the prefix exists. Returns how many tiles were issued.
__device__ int prefill(uint8_t* smem, const Bars& b, const Maps4& m, const Geom& geo, const Seq& sq, bool two_atoms) {
  const uint64_t pol = policy_evict_first();
  const int pre = static_cast<int>(sq.te - sq.tb < kStages ? sq.te - sq.tb : kStages);
  for (int i = 0; i < pre; ++i) {
    const TileCoord c = tile_coord(sq.tb + i, geo);
    ring_put(sq, i, c);
    load_q(smem, b, m, geo, c, i, two_atoms, pol);
  }
  return pre;
}

// The rest of the producer: prefix tiles (read only once the prefix is complete) and the Q tiles
// after the prefilled ones.
// With `combined` (single-launch kernel, one block per head), a head's prefix tile is loaded only
// once every CTA sharing the head's combine has published its rows (value `tag`). With ptiles ==
// nullptr the prefix tiles are already in shared memory (buffer j & 1 for the j-th segment) and
// are only signalled to the MMA warp.
__device__ void produce(uint8_t* smem, const Bars& b, const Maps4& m, const Geom& geo, const Seq& sq, int pre,
                        bool two_atoms, const uint8_t* __restrict__ ptiles, const uint64_t* combined, uint64_t tag,
                        uint32_t* status) {
  const uint64_t pol = policy_evict_first();
  int k = 0, j = 0, prev = -1;
  bool ok = true;
  long long t = sq.tb, end = sq.te;
  for (;; ++t, ++k) {
    if (t >= end) {  // static range done: claim the next chunk of the dynamic range, if any
      if (sq.counter == nullptr) break;
      const long long c0 = sq.dyn_begin + static_cast<long long>(atomicAdd(sq.counter, 1u)) * kDynChunk;
      if (c0 >= sq.dyn_end) break;
      t = c0;
      end = c0 + kDynChunk < sq.dyn_end ? c0 + kDynChunk : sq.dyn_end;
    }
    const TileCoord c = tile_coord(t, geo);
    if (c.seg != prev && ptiles == nullptr) {  // the caller already placed the tile in buffer j & 1
      mbar_arrive(&b.bfull[j & 1]);
      ++j;
      prev = c.seg;
    } else if (c.seg != prev) {
      const int bb = j & 1;
      if (combined != nullptr) {
        const CombineRange cr = combine_range(c.seg, geo);
        if (!wait_flags(combined, cr.ga + c.seg, cr.gb + c.seg, tag, status, 0x2200u)) { ok = false; break; }
        fence_proxy_async_global();  // prefix tile written by other CTAs -> bulk copy below
      }
      if (!mbar_wait(&b.bempty[bb], ((j >> 1) & 1) ^ 1, status, 0x1100u | bb)) { ok = false; break; }
      mbar_expect_tx(&b.bfull[bb], kPTileBytes);
      bulk_load(smem + kBOff + bb * kPTileBytes, ptiles + static_cast<size_t>(c.seg) * kPTileBytes, kPTileBytes,
                &b.bfull[bb]);
      ++j;
      prev = c.seg;
    }
    if (k >= pre) {
      const int s = k % kStages;
      if (!mbar_wait(&b.qempty[s], ((k / kStages) & 1) ^ 1, status, 0x1120u | s)) { ok = false; break; }
      ring_put(sq, k, c);
      load_q(smem, b, m, geo, c, s, two_atoms, pol);
    }
  }
  if (ok) {  // end of the sequence: a plain arrival completes the next stage's qfull, its ring entry segment -1
    const int s = k % kStages;
    if (k < pre || mbar_wait(&b.qempty[s], ((k / kStages) & 1) ^ 1, status, 0x1140u | s)) {
      ring_end(sq, k);
      mbar_arrive(&b.qfull[s]);
      ++k;
    }
  }
  for (int i = (k > kStages ? k - kStages : 0); i < k; ++i)
    mbar_wait(&b.qfull[i % kStages], (i / kStages) & 1, status, 0x1180u);
  for (int i = (j > 2 ? j - 2 : 0); i < j; ++i) mbar_wait(&b.bfull[i & 1], (i >> 1) & 1, status, 0x1190u);
}

// Rotary form only: per stage, the denominator products of a Q tile retired, and the tile turned.
struct RopeBars {
  uint64_t* zd;   // [3] count 1 (tcgen05.commit)
  uint64_t* rot;  // [3] one arrival per turning warp: 4 (one atom) or 8 (two atoms)
};
constexpr int kRopeBars = 2 * kStages;
__device__ __forceinline__ RopeBars rope_bars_at(uint64_t* p) { return RopeBars{p, p + kStages}; }
__device__ __forceinline__ void init_rope_bars(const RopeBars& rb, bool two_atoms) {
  for (int i = 0; i < kStages; ++i) {
    mbar_init(&rb.zd[i], 1);
    mbar_init(&rb.rot[i], two_atoms ? 8 : 4);
  }
}

template <bool kRope>
__device__ void mma_issue(uint8_t* smem, const Bars& b, const Geom& geo, const Seq& sq, bool two_atoms, uint32_t tmem,
                          uint32_t* status, const RopeBars* rb) {
  constexpr uint32_t kIdescO = idesc_bf16_f32(128, kPTileRows, false, false);
  constexpr uint32_t kIdescNum = idesc_bf16_f32(128, 128, false, false);
  constexpr uint32_t kIdescDen = idesc_bf16_f32(128, 16, false, false);
  const int ksteps = two_atoms ? 8 : 4;
  int j = 0, prev = -1, bb = 0;
  for (int k = 0;; ++k) {
    const int s = k % kStages;
    const uint32_t ph = (k / kStages) & 1;
    const int a = k & 1;
    if (!mbar_wait(&b.qfull[s], ph, status, 0x1310u | s)) break;
    const int seg = sq.ring[k % kRing].x;
    if (seg < 0) {
      // End of the sequence, announced on this accumulator's barrier under the same flow control
      // as a tile: first the epilogue must have released the accumulator's previous use (tile
      // k - 2), or the barrier could run two phases ahead of a slow epilogue, which would then
      // wait for a parity it already missed. The commit arrives once every MMA issued so far has
      // retired.
      if (!mbar_wait(&b.acce[a], ((k >> 1) & 1) ^ 1, status, 0x1340u | a)) break;
      mma_commit(&b.accf[a]);
      break;
    }
    if (seg != prev) {
      if (j > 0) mma_commit(&b.bempty[(j - 1) & 1]);  // the previous prefix tile is free once its MMAs retire
      bb = j & 1;
      if (!mbar_wait(&b.bfull[bb], (j >> 1) & 1, status, 0x1300u | bb)) break;
      ++j;
      prev = seg;
    }
    if (!mbar_wait(&b.qrelu[s], ph, status, 0x1320u | s)) break;
    if (!mbar_wait(&b.acce[a], ((k >> 1) & 1) ^ 1, status, 0x1330u | a)) break;
    tc_fence_after();
    const uint32_t qb = smem_u32(smem + s * kQBytes);
    const uint32_t bbase = smem_u32(smem + kBOff + bb * kPTileBytes);
    const uint32_t dacc = tmem + static_cast<uint32_t>(a * 256);
    if constexpr (kRope) {
      // denominator from the unturned ReLU(Q) against the z row and its 15 zero rows (B rows
      // 128..143, 16 KB into each atom), then the numerator from the turned tile against P^T
      for (int kk = 0; kk < ksteps; ++kk)
        mma_bf16(dacc + kZRow, sdesc_sw128(qb + (kk >> 2) * kAtomBytes + (kk & 3) * 32, 16, 1024),
                 sdesc_sw128(bbase + (kk >> 2) * kBAtomBytes + kZRow * 128 + (kk & 3) * 32, 16, 1024), kIdescDen,
                 kk > 0 ? 1u : 0u);
      mma_commit(&rb->zd[s]);
      if (!mbar_wait(&rb->rot[s], ph, status, 0x1350u | s)) break;
      tc_fence_after();
      for (int kk = 0; kk < ksteps; ++kk)
        mma_bf16(dacc, sdesc_sw128(qb + (kk >> 2) * kAtomBytes + (kk & 3) * 32, 16, 1024),
                 sdesc_sw128(bbase + (kk >> 2) * kBAtomBytes + (kk & 3) * 32, 16, 1024), kIdescNum, kk > 0 ? 1u : 0u);
    } else {
      for (int kk = 0; kk < ksteps; ++kk) {
        // 16 features per MMA: +32 B inside the 128-B swizzle row, next atom after 4 steps
        const uint64_t ad = sdesc_sw128(qb + (kk >> 2) * kAtomBytes + (kk & 3) * 32, 16, 1024);
        const uint64_t bd = sdesc_sw128(bbase + (kk >> 2) * kBAtomBytes + (kk & 3) * 32, 16, 1024);
        mma_bf16(dacc, ad, bd, kIdescO, kk > 0 ? 1u : 0u);
      }
    }
    mma_commit(&b.qempty[s]);
    mma_commit(&b.accf[a]);
  }
  mma_commit(b.done);
  mbar_wait(b.done, 0, status, 0x13F0u);
}
__device__ __forceinline__ void mma_role(uint8_t* smem, const Bars& b, const Geom& geo, const Seq& sq, bool two_atoms,
                                         uint32_t tmem, uint32_t* status) {
  mma_issue<false>(smem, b, geo, sq, two_atoms, tmem, status, nullptr);
}

// ReLU of the k-th Q tile (stage k % kStages) in place. Returns 1 when done, 0 at the end of the
// sequence, -1 if the grid failed.
__device__ __forceinline__ int relu_q(uint8_t* smem, const Bars& b, const Seq& sq, long long k, bool two_atoms, int r,
                                      int lane, uint32_t* status) {
  const int s = static_cast<int>(k % kStages);
  const bool ok = mbar_wait(&b.qfull[s], static_cast<uint32_t>((k / kStages) & 1), status, 0x1200u | s);
  if (!warp_all(ok)) return -1;
  if (sq.ring[k % kRing].x < 0) return 0;
  relu_tile_inplace(smem + s * kQBytes, (two_atoms ? kQBytes : kAtomBytes) / 16, r);
  fence_proxy_async_smem();
  __syncwarp();
  if (lane == 0) mbar_arrive(&b.qrelu[s]);
  return 1;
}

// Output staging: nbuf (1 or 2) sets of 4 warps x two 4 KB atoms starting at `base`.
struct Staging {
  uint8_t* base;
  int nbuf;
};

// Epilogue of tile k for one warp: TMEM lanes 32q..32q+31 (q = warp % 4, tokens of the tile) and
// output columns 64h..64h+63; numerator times 1 / (denominator + eps), bf16, into this warp's
// swizzled 4 KB staging atom (alternating between buffers when there are two), then a TMA store
// clipped to the block.
// Returns 1 when done, 0 at the end of the sequence, -1 if the grid failed.
__device__ __forceinline__ int epilogue_tile(const Staging& sg, const Bars& b, const Maps4& m, const Geom& geo,
                                             const Seq& sq, long long k, uint32_t tmem, int q, int h, int lane,
                                             float eps, uint32_t* status) {
  const int a = static_cast<int>(k & 1);
  const bool ok = mbar_wait(&b.accf[a], static_cast<uint32_t>((k >> 1) & 1), status, 0x1400u | a);
  if (!warp_all(ok)) return -1;
  const volatile int4* ent = sq.ring + (k % kRing);
  if (ent->x < 0) return 0;
  tc_fence_after();
  const uint32_t ta = tmem + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(a * 256);
  uint32_t dr;
  uint32_t rr[2][32];
  tmem_ld_x1(ta + kZRow, dr);
  tmem_ld_x32(ta + h * 64, rr[0]);
  tmem_ld_x32(ta + h * 64 + 32, rr[1]);
  const int bh = ent->y, blk = ent->z, tok0 = ent->w;  // read while the TMEM loads are in flight
  tmem_wait_ld();
  tc_fence_before();
  __syncwarp();
  if (lane == 0) mbar_arrive(&b.acce[a]);  // the values are in registers: the accumulator is free
  const float inv = __frcp_rn(__uint_as_float(dr) + eps);
  uint8_t* ob = sg.base + ((sg.nbuf > 1 ? static_cast<int>(k & 1) * 4 : 0) + q) * kOWarpBytes + h * kAtomBytesO;
  if (lane == 0) {  // the store that last read this atom (one or two tiles ago) has finished reading it
    if (sg.nbuf > 1)
      bulk_wait_read_all_but_one();
    else
      bulk_wait_read_all();
  }
  __syncwarp();
#pragma unroll
  for (int cc = 0; cc < 2; ++cc) {
#pragma unroll
    for (int mm = 0; mm < 4; ++mm) {
      uint4 w;
      w.x = pack_bf16x2(__uint_as_float(rr[cc][8 * mm + 0]) * inv, __uint_as_float(rr[cc][8 * mm + 1]) * inv);
      w.y = pack_bf16x2(__uint_as_float(rr[cc][8 * mm + 2]) * inv, __uint_as_float(rr[cc][8 * mm + 3]) * inv);
      w.z = pack_bf16x2(__uint_as_float(rr[cc][8 * mm + 4]) * inv, __uint_as_float(rr[cc][8 * mm + 5]) * inv);
      w.w = pack_bf16x2(__uint_as_float(rr[cc][8 * mm + 6]) * inv, __uint_as_float(rr[cc][8 * mm + 7]) * inv);
      const int chunk = cc * 4 + mm;  // 16-byte chunk of the 128-byte row of this atom
      *reinterpret_cast<uint4*>(ob + lane * 128 + ((chunk ^ (lane & 7)) << 4)) = w;
    }
  }
  fence_proxy_async_smem();
  __syncwarp();
  if (lane == 0) {
    const bool in_last = blk == geo.nblk - 1;
    const int blen = in_last ? geo.Llast : geo.L;
    const int row0 = tok0 + q * 32;
    if (row0 < blen) {
      const bool lst = in_last && geo.Llast != geo.L;  // the shorter last block has its own map
      tma_store_4d(lst ? m.b_last : m.b_main, ob, h * 64, row0, lst ? 0 : blk, bh);
    }
    bulk_commit();  // one group per tile (possibly empty), so "all but the latest" means the previous tile
  }
  return 1;
}

// Warps 0-3: epilogue of output columns 0..63 of every tile.
__device__ void epilogue_role(const Staging& sg, const Bars& b, const Maps4& m, const Geom& geo, const Seq& sq,
                              uint32_t tmem, int warp, int lane, float eps, uint32_t* status) {
  for (long long k = 0;; ++k)
    if (epilogue_tile(sg, b, m, geo, sq, k, tmem, warp & 3, 0, lane, eps, status) <= 0) break;
  if (lane == 0) bulk_wait_all();
}

// Warps 4-7: ReLU of the Q tiles, running up to kStages tiles ahead (relu_done <= kStages of them
// already done), and (D > 64) the epilogue of output columns 64..127. Tile k + kStages is ReLU'd
// after the epilogue of tile k: its stage was freed by the MMAs of tile k, which the epilogue has
// waited for, so the order cannot deadlock.
__device__ void relu_epi_role(uint8_t* smem, const Staging& sg, const Bars& b, const Maps4& m, const Geom& geo,
                              const Seq& sq, int relu_done, bool two_atoms, uint32_t tmem, int warp, int lane,
                              float eps, uint32_t* status) {
  const int r = static_cast<int>(threadIdx.x) - 128;
  long long kr = relu_done;  // tiles [0, relu_done) were ReLU'd by the caller
  int rs = 1;                // relu state: 1 more tiles, 0 sequence ended, -1 failed
  for (; kr < kStages && rs > 0; ++kr) rs = relu_q(smem, b, sq, kr, two_atoms, r, lane, status);
  if (rs < 0) return;
  for (long long k = 0;; ++k) {
    if (two_atoms) {
      const int es = epilogue_tile(sg, b, m, geo, sq, k, tmem, warp & 3, 1, lane, eps, status);
      if (es <= 0) break;
    } else if (rs == 0) {
      break;
    }
    if (rs > 0) {
      rs = relu_q(smem, b, sq, kr++, two_atoms, r, lane, status);
      if (rs < 0) break;
    }
  }
  if (two_atoms && lane == 0) bulk_wait_all();
}

// Turn of atom `atom` of the k-th Q tile once its denominator products retired. Returns 1, 0 when
// tile k is the end of the sequence (checked for atom 1, whose turners run ahead of the tiles they
// have seen), -1 if the grid failed.
__device__ __forceinline__ int turn_q(uint8_t* smem, const Bars& b, const RopeBars& rb, const Geom& geo, const Seq& sq,
                                      long long k, int atom, int r, int lane, const RopeDev& rp, uint32_t ct,
                                      uint32_t* status) {
  const int s = static_cast<int>(k % kStages);
  const uint32_t ph = static_cast<uint32_t>((k / kStages) & 1);
  if (atom == 1) {
    const bool ok = mbar_wait(&b.qfull[s], ph, status, 0x1250u | s);
    if (!warp_all(ok)) return -1;
    if (sq.ring[k % kRing].x < 0) return 0;
  }
  const bool ok = mbar_wait(&rb.zd[s], ph, status, 0x1240u | s);
  if (!warp_all(ok)) return -1;
  const volatile int4* ent = sq.ring + (k % kRing);
  const int blk = ent->z, tok0 = ent->w;
  const int blen = blk == geo.nblk - 1 ? geo.Llast : geo.L;
  rope_tile_inplace(smem + s * kQBytes, atom, r, blk * geo.L + tok0, min(kTile, blen - tok0), rp, ct);
  fence_proxy_async_smem();
  __syncwarp();
  if (lane == 0) mbar_arrive(&rb.rot[s]);
  return 1;
}

// relu_epi_role of the rotary form: ReLU of tile k + kStages and the turn of atom 0 of tile
// k + kStages - 1 after the epilogue of tile k (one tile of lag between ReLU and turn, so that the
// denominator products have retired). The turn of tile k + 2 waits for the MMA warp's denominator
// products, which wait for the accumulator that the epilogue of tile k released, so the order
// cannot deadlock; at the end of the sequence every ReLU'd tile is turned. With two atoms the
// epilogue warps turn atom 1 (epi_turn_role).
// `ct`: the compact (cos, sin) table's shared-memory area, staged by the turning warps once the
// scan grid has finished (nothing can be turned before: the first numerator products need its
// prefix anyway).
// Geom and RopeDev are copied into registers, as in the state kernel's relu_rope_role.
__device__ void relu_rot_epi_role(uint8_t* smem, const Staging& sg, const Bars& b, const RopeBars& rb, const Maps4& m,
                                  const Geom& geo_p, const Seq& sq, bool two_atoms, uint32_t tmem, int warp, int lane,
                                  float eps, const RopeDev& rp_p, float2* ct, uint32_t* status) {
  const Geom geo = geo_p;
  const RopeDev rp = rp_p;
  const int r = static_cast<int>(threadIdx.x) - 128;
  st::stage_and_sync(ct, rp, two_atoms ? 128 + r : r, two_atoms ? 256 : 128);
  const uint32_t cta = smem_u32(ct);
  long long kr = 0, kq = 0;  // tiles ReLU'd, tiles turned
  int rs = 1;                // 1 more tiles, 0 sequence ended, -1 failed
  const auto relu_next = [&]() {
    if (rs > 0) {
      rs = relu_q(smem, b, sq, kr, two_atoms, r, lane, status);
      if (rs > 0) ++kr;
    }
  };
  const auto turn_upto = [&](long long upto) -> bool {
    for (; kq < kr && kq < upto; ++kq)
      if (turn_q(smem, b, rb, geo, sq, kq, 0, r, lane, rp, cta, status) < 0) return false;
    return true;
  };
  for (int i = 0; i < kStages; ++i) {
    relu_next();
    if (rs < 0 || !turn_upto(rs == 0 ? kr : i)) return;
  }
  for (long long k = 0;; ++k) {
    if (two_atoms) {
      const int es = epilogue_tile(sg, b, m, geo, sq, k, tmem, warp & 3, 1, lane, eps, status);
      if (es <= 0) break;
    } else if (rs == 0 && kq == kr) {
      break;
    }
    relu_next();
    if (rs < 0 || !turn_upto(rs == 0 ? kr : k + kStages)) break;
  }
  if (two_atoms && lane == 0) bulk_wait_all();
}

// Warps 0-3 of the rotary form with two atoms: the epilogue of output columns 0..63 of tile k, then
// the turn of atom 1 of tile k + 2 (the same place in the order as the ReLU warps' turn of atom 0;
// tiles 0 and 1 are turned first).
__device__ void epi_turn_role(uint8_t* smem, const Staging& sg, const Bars& b, const RopeBars& rb, const Maps4& m,
                              const Geom& geo_p, const Seq& sq, uint32_t tmem, int warp, int lane, float eps,
                              const RopeDev& rp_p, float2* ct, uint32_t* status) {
  const Geom geo = geo_p;
  const RopeDev rp = rp_p;
  const int r = static_cast<int>(threadIdx.x);
  st::stage_and_sync(ct, rp, r, 256);
  const uint32_t cta = smem_u32(ct);
  long long kq = 0;
  int ts = 1;  // 1 more tiles, 0 end of the sequence seen, -1 failed
  const auto turn_upto = [&](long long upto) {
    for (; ts > 0 && kq < upto; ++kq) ts = turn_q(smem, b, rb, geo, sq, kq, 1, r, lane, rp, cta, status);
    return ts >= 0;
  };
  if (turn_upto(2)) {
    for (long long k = 0;; ++k) {
      if (epilogue_tile(sg, b, m, geo, sq, k, tmem, warp & 3, 0, lane, eps, status) <= 0) break;
      if (!turn_upto(k + 3)) break;
    }
  }
  if (lane == 0) bulk_wait_all();
}
}  // namespace ot

// ---- common prologue / epilogue of the persistent kernels ----
__device__ __forceinline__ void prefetch_maps(const Maps4& m) {
  prefetch_tmap(m.a_main);
  prefetch_tmap(m.a_last);
  prefetch_tmap(m.b_main);
  prefetch_tmap(m.b_last);
}
__device__ __forceinline__ uint32_t persistent_setup(uint32_t* tmem_slot, int warp) {
  if (warp == kWarpMma) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  return *tmem_slot;
}
__device__ __forceinline__ void persistent_teardown(uint32_t tmem, int warp) {
  tc_fence_before();
  __syncthreads();
  if (warp == kWarpMma) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// ------------------------------------------------------------------------------------------
// stand-alone kernels
// ------------------------------------------------------------------------------------------
constexpr int kStateSmem = st::kRegionBytes + 1024 + 256 + 1024;   // region, barriers, alignment slack
constexpr int kOutSmem = ot::kRegionBytes + 1024 + 512 + 1024;
// rotary form: the compact (cos, sin) table after the barrier area
constexpr int kRopeTableBytes = kRopeSmemEntries * 8;
constexpr int kStateSmemRope = kStateSmem + kRopeTableBytes;
constexpr int kOutSmemRope = kOutSmem + kRopeTableBytes;
static_assert(kStateSmemRope <= 232448 && kOutSmemRope <= 232448, "227 KB of shared memory per CTA");
// barrier areas (512 B): the barriers, the TMEM slot, then the 16-byte aligned tile ring
static_assert((ot::kNumBars + 2) * 8 + ot::kRingBytes <= 512, "output kernel barrier area");
static_assert((st::kNumBars + ot::kNumBars + 2) * 8 + ot::kRingBytes <= 512, "single-launch barrier area");

static_assert((st::kNumBars + 1 + st::kRopeBars) * 8 <= 256, "state kernel barrier area");
static_assert((ot::kNumBars + 2) * 8 + ot::kRingBytes + ot::kRopeBars * 8 <= 512, "output kernel barrier area (rotary)");

template <bool kRope>
__global__ void __launch_bounds__(kThreads, 1)
    state_bf16_kernel(const __grid_constant__ CUtensorMap k_main, const __grid_constant__ CUtensorMap k_last,
                      const __grid_constant__ CUtensorMap v_main, const __grid_constant__ CUtensorMap v_last,
                      const Geom geo, float* __restrict__ partials, int2* __restrict__ segcta,
                      uint32_t* status, const RopeDev rp) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  uint64_t* barmem = reinterpret_cast<uint64_t*>(smem + st::kRegionBytes);
  const st::Bars b = st::bars_at(barmem);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(barmem + st::kNumBars);
  const st::RopeBars rb = st::rope_bars_at(barmem + st::kNumBars + 1);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int g = blockIdx.x;
  const long long tb = tile_begin(g, geo);
  const long long te = tile_begin(g + 1, geo);
  const bool two_atoms = geo.D > 64;
  const Maps4 m{&k_main, &k_last, &v_main, &v_last};
  if (threadIdx.x == 0) {
    st::init_bars(b);
    if (kRope) st::init_rope_bars(rb, two_atoms);
    fence_mbar_init();
  }
  st::init_smem(smem, two_atoms, kThreads);
  if (warp == kWarpProducer && lane == 0) prefetch_maps(m);
  const uint32_t tmem = persistent_setup(tmem_slot, warp);
  if (threadIdx.x == 0) griddep_launch_dependents();
  if (warp == kWarpProducer) {
    if (lane == 0) st::produce(smem, b, m, geo, tb, te, two_atoms, true, status);
  } else if (warp >= 4 && warp < 8) {
    if constexpr (kRope)
      st::relu_rope_role(smem, b, rb, geo, tb, te, two_atoms, threadIdx.x - 128, lane, rp,
                         reinterpret_cast<float2*>(smem + st::kRegionBytes + 256), status);
    else
      st::relu_role(smem, b, tb, te, two_atoms, threadIdx.x - 128, lane, status);
  } else if (warp == kWarpMma) {
    if (lane == 0) st::mma_issue<kRope>(smem, b, geo, tb, te, tmem, status, &rb);
  } else {
    const st::TurnCtx tc{smem, rb, &rp, reinterpret_cast<float2*>(smem + st::kRegionBytes + 256)};
    st::epilogue_role(b, geo, tb, te, tmem, g, warp, lane, partials, segcta, nullptr, nullptr, 0, status,
                      kRope && two_atoms ? &tc : nullptr);
  }
  persistent_teardown(tmem, warp);
}

template <bool kRope>
__global__ void __launch_bounds__(kThreads, 1)
    out_bf16_kernel(const __grid_constant__ CUtensorMap q_main, const __grid_constant__ CUtensorMap q_last,
                    const __grid_constant__ CUtensorMap o_main, const __grid_constant__ CUtensorMap o_last,
                    const Geom geo, const uint8_t* __restrict__ ptiles, const float eps, uint32_t* status,
                    const RopeDev rp) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  uint64_t* barmem = reinterpret_cast<uint64_t*>(smem + ot::kRegionBytes);
  const ot::Bars b = ot::bars_at(barmem);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(barmem + ot::kNumBars);
  volatile int4* ring = reinterpret_cast<volatile int4*>(barmem + ot::kNumBars + 2);  // 16-byte aligned
  const ot::RopeBars rb = ot::rope_bars_at(barmem + ot::kNumBars + 2 + ot::kRingBytes / 8);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int g = blockIdx.x;
  // static range of this CTA, then chunks of the dynamic tail (counter reset by the scan kernel)
  const ot::Seq sq{out_tile_begin(g, geo), out_tile_begin(g + 1, geo), geo.T - geo.tdyn, geo.T,
                   geo.tdyn > 0 ? status + 6 : nullptr, ring};
  const bool two_atoms = geo.D > 64;
  const Maps4 m{&q_main, &q_last, &o_main, &o_last};
  if (threadIdx.x == 0) {
    ot::init_bars(b, two_atoms);
    if (kRope) ot::init_rope_bars(rb, two_atoms);
    fence_mbar_init();
  }
  if (warp == kWarpProducer && lane == 0) prefetch_maps(m);
  const uint32_t tmem = persistent_setup(tmem_slot, warp);
  if (threadIdx.x == 0) griddep_launch_dependents();
  if (warp == kWarpProducer) {
    if (lane == 0) {
      const int pre = ot::prefill(smem, b, m, geo, sq, two_atoms);
      griddep_wait();  // the prefix tiles and the chunk counter come from the scan grid
      ot::produce(smem, b, m, geo, sq, pre, two_atoms, ptiles, nullptr, 0, status);
    }
  } else if (warp >= 4 && warp < 8) {
    if constexpr (kRope)
      ot::relu_rot_epi_role(smem, ot::Staging{smem + ot::kOOff, 1}, b, rb, m, geo, sq, two_atoms, tmem, warp, lane,
                            eps, rp, reinterpret_cast<float2*>(smem + ot::kRegionBytes + 512), status);
    else
      ot::relu_epi_role(smem, ot::Staging{smem + ot::kOOff, 1}, b, m, geo, sq, 0, two_atoms, tmem, warp, lane, eps,
                        status);
  } else if (warp == kWarpMma) {
    if (lane == 0) ot::mma_issue<kRope>(smem, b, geo, sq, two_atoms, tmem, status, &rb);
  } else if (kRope && two_atoms) {
    ot::epi_turn_role(smem, ot::Staging{smem + ot::kOOff, 1}, b, rb, m, geo, sq, tmem, warp, lane, eps, rp,
                      reinterpret_cast<float2*>(smem + ot::kRegionBytes + 512), status);
  } else {
    ot::epilogue_role(ot::Staging{smem + ot::kOOff, 1}, b, m, geo, sq, tmem, warp, lane, eps, status);
  }
  persistent_teardown(tmem, warp);
}

// ------------------------------------------------------------------------------------------
// 2. partial combine + inclusive prefix over blocks (+ incoming cache), both paths
// ------------------------------------------------------------------------------------------
// CTA (bh, row e of the prefix tile): e < 128 are S^T rows (value feature e), e = 128 is z,
// e = 129..143 are the zero rows of the bf16 B operand. Lane q owns key features 4q..4q+3;
// warp j owns blocks [j*nblk/ng, (j+1)*nblk/ng) (at most kScanReg of them when nblk <= 128),
// so every partial load is independent; the running prefix crosses warps through shared memory.
constexpr int kScanReg = 8;
constexpr int kScanMaxWarps = 16;

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

__global__ void __launch_bounds__(512) scan_kernel(const float* __restrict__ partials,
                                                    const int2* __restrict__ segcta, const Geom geo,
                                                    const float* S_in, const float* z_in, float* S_out,
                                                    float* z_out, uint8_t* __restrict__ ptiles,
                                                    float* __restrict__ p32, const int ng_warps,
                                                    uint32_t* out_chunks) {
  griddep_wait();  // partials come from the state kernel; prefix tiles may still be read before it
  // The output kernel of this call claims its dynamic chunks from this counter only after this
  // grid has completed; the previous call's output kernel completed before the state kernel did.
  if (blockIdx.x == 0 && blockIdx.y == 0 && threadIdx.x == 0) *out_chunks = 0u;
  griddep_launch_dependents();
  // block (bh, rows e = blockIdx.y * R .. + R - 1): warp w handles row r = w / ng, block group j = w % ng
  extern __shared__ float4 s_scan[];   // [R][ng][32] warp totals, then [R][32] incoming cache
  const int ng = ng_warps;
  const int R = (blockDim.x >> 5) / ng;
  const int wr = threadIdx.x >> 5;
  const int r = wr / ng;
  const int bh = blockIdx.x;
  const int e = blockIdx.y * R + r;
  const int q = threadIdx.x & 31;
  const int j = wr - r * ng;
  float4* s_tot = s_scan + r * ng * 32;
  float4* s_base = s_scan + R * ng * 32 + r * 32;
  const int nblk = geo.nblk;
  const int D = geo.D;
  const int d0 = q * 4;
  const int c0 = static_cast<int>(static_cast<long long>(j) * nblk / ng);
  const int c1 = static_cast<int>(static_cast<long long>(j + 1) * nblk / ng);
  const int cnt = c1 - c0;
  const bool live = e < kPartRows;
  const int seg0 = bh * nblk;

  // pass 1: this warp's block sums (kept in registers) and their total. The slot ranges of all
  // kScanReg blocks are fetched together, then the first two slots of every block together (a
  // block of a long sequence is rarely covered by more than two CTAs; further slots follow), so
  // the warp waits for two memory round trips instead of two per block.
  float4 sums[kScanReg];
  float4 tot = make_float4(0.f, 0.f, 0.f, 0.f);
  int2 gr[kScanReg];
#pragma unroll
  for (int i = 0; i < kScanReg; ++i) gr[i] = (live && i < cnt) ? segcta[seg0 + c0 + i] : make_int2(0, -1);
  float4 p0[kScanReg], p1[kScanReg];
#pragma unroll
  for (int i = 0; i < kScanReg; ++i) {
    const size_t row = static_cast<size_t>(seg0 + c0 + i) * kPartRows + e;
    p0[i] = gr[i].y >= gr[i].x ? __ldcg(reinterpret_cast<const float4*>(
                                     partials + (static_cast<size_t>(gr[i].x) * kPartRows + row) * kDPad + d0))
                               : make_float4(0.f, 0.f, 0.f, 0.f);
    p1[i] = gr[i].y >= gr[i].x + 1 ? __ldcg(reinterpret_cast<const float4*>(
                                         partials + (static_cast<size_t>(gr[i].x + 1) * kPartRows + row) * kDPad + d0))
                                   : make_float4(0.f, 0.f, 0.f, 0.f);
  }
#pragma unroll
  for (int i = 0; i < kScanReg; ++i) {
    sums[i] = f4add(p0[i], p1[i]);
    for (int gg = gr[i].x + 2; gg <= gr[i].y; ++gg)
      sums[i] = f4add(sums[i], __ldcg(reinterpret_cast<const float4*>(
                                   partials + (static_cast<size_t>(gg + seg0 + c0 + i) * kPartRows + e) * kDPad + d0)));
    tot = f4add(tot, sums[i]);
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
    s_tot[j * 32 + q] = tot;
    if (j == 0) s_base[q] = run;
    __syncthreads();
    run = s_base[q];
    for (int jj = 0; jj < j; ++jj) run = f4add(run, s_tot[jj * 32 + q]);
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
// 4. one launch for one-block problems (bidirectional forward, streaming cache step)
// ------------------------------------------------------------------------------------------
// State reduction -> combine -> output in one launch (every CTA resident, one per SM).
// Each CTA reduces a contiguous tile range; heads are synchronised one by one instead of with
// grid-wide barriers: a CTA publishes each partial slot it flushes; the CTAs whose range starts
// inside a head split that head's combine once all its slots are published (reading their share of
// the incoming cache while they wait, writing the outgoing cache after publishing), and publish
// their share; a head's output tiles start once its combine is complete. The output tiles are a
// static range per CTA plus chunks of the last ~1/8 of the tiles handed out through a counter, as
// in the output kernel. Flags carry the workspace's launch sequence number (header bytes 8..15,
// advanced by the last CTA to read it), so nothing needs resetting; that CTA also clears the chunk
// counter of the next launch (header bytes 28..35, one per parity of the sequence number). The
// stage memory of the reduction is reused by the output, whose first Q tiles load while the
// combine runs.
namespace fu {
constexpr int kRegion = (st::kRegionBytes > ot::kRegionBytes) ? st::kRegionBytes : ot::kRegionBytes;
constexpr int kSmem = kRegion + 512 + 1024;
// shared memory free during the combine (between the prefilled Q stages and the output staging):
// the cache transpose of up to 128 rows x 129 floats
constexpr int kScratchOff = ot::kBOff;
constexpr int kScratchZOff = kScratchOff + 128 * 129 * 4;  // z row of the share (128 floats)
static_assert(kScratchZOff + 128 * 4 <= ot::kOOff, "combine scratch overlaps the output staging");
}  // namespace fu

// Rows [r0, r1) of head bh's prefix tile (row e < 128: value feature e of S; row 128: z; rows
// 129..143: zero). The cache is [d][e] (key feature major) while a prefix row is one value feature
// e, so S_in and S_out go through the shared-memory transpose sS ([row - r0][d], padded rows) and
// the global side stays coalesced. Row kZRow's z values go through sZ.
__device__ __forceinline__ int cache_rows(const Geom& geo, int r0, int r1) {
  const int e_hi = (r1 < geo.D ? r1 : geo.D);
  return e_hi > r0 ? e_hi - r0 : 0;
}

// Step 1 (independent of the other CTAs): the incoming cache rows of the share into sS / sZ.
// Threads tid = 0..nthr-1 of the caller share the work.
__device__ void combine_load_cache(const Geom& geo, const float* S_in, const float* z_in, int bh, int r0, int r1,
                                   float* sS, float* sZ, int tid, int nthr) {
  const int D = geo.D, ld = D + 1, ns = cache_rows(geo, r0, r1);
  if (S_in != nullptr) {
    // consecutive threads read consecutive e of one key row d; 8 loads per thread in flight
    for (int i0 = tid; i0 < D * ns; i0 += 8 * nthr) {
      float v[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int i = i0 + u * nthr;
        const int d = i / ns, j = i - d * ns;
        v[u] = i < D * ns ? __ldcg(S_in + (static_cast<size_t>(bh) * D + d) * D + r0 + j) : 0.f;
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int i = i0 + u * nthr;
        const int d = i / ns, j = i - d * ns;
        if (i < D * ns) sS[j * ld + d] = v[u];
      }
    }
  }
  if (z_in != nullptr && r0 <= kZRow && kZRow < r1)
    for (int d = tid; d < D; d += nthr) sZ[d] = __ldcg(z_in + static_cast<size_t>(bh) * D + d);
}

// Step 2 (once the head's partial slots exist): each row = cache + the slots of CTAs g0..g1 in
// ascending order, written as the bf16 B operand of the output GEMM; the sums replace the cache
// values in sS / sZ for step 3. Each thread takes two (row, quad) items per pass and keeps up to 8
// slots of each in flight at once; the order of the additions does not depend on the unrolling.
__device__ void combine_sum(const Geom& geo, const float* __restrict__ partials, int g0, int g1, bool has_S,
                            bool has_z, uint8_t* __restrict__ ptiles, int bh, int r0, int r1, float* sS, float* sZ) {
  const int D = geo.D, ld = D + 1;
  for (int base = r0 * 32 + static_cast<int>(threadIdx.x); base < r1 * 32; base += 2 * kThreads) {
    int es[2], ds[2];
    bool vs[2];
    float acc[2][4];
#pragma unroll
    for (int x = 0; x < 2; ++x) {
      const int it = base + x * kThreads;
      es[x] = it >> 5;
      ds[x] = (it & 31) * 4;
      vs[x] = it < r1 * 32 && es[x] < kPartRows;
      acc[x][0] = acc[x][1] = acc[x][2] = acc[x][3] = 0.f;
    }
    for (int gb = g0; gb <= g1; gb += 8) {
      float4 p[2][8];
#pragma unroll
      for (int x = 0; x < 2; ++x)
#pragma unroll
        for (int u = 0; u < 8; ++u)
          p[x][u] = (vs[x] && gb + u <= g1)
                        ? __ldcg(reinterpret_cast<const float4*>(
                              partials + (static_cast<size_t>(gb + u + bh) * kPartRows + es[x]) * kDPad + ds[x]))
                        : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        if (gb + u <= g1) {
#pragma unroll
          for (int x = 0; x < 2; ++x) {
            acc[x][0] += p[x][u].x;
            acc[x][1] += p[x][u].y;
            acc[x][2] += p[x][u].z;
            acc[x][3] += p[x][u].w;
          }
        }
      }
    }
#pragma unroll
    for (int x = 0; x < 2; ++x) {
      const int it = base + x * kThreads;
      if (it >= r1 * 32) break;
      const int e = es[x], d0 = ds[x];
      float* a = acc[x];
      if (e < D) {
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          if (d0 + u < D) {
            float* c = &sS[(e - r0) * ld + d0 + u];
            if (has_S) a[u] += *c;
            *c = a[u];
          }
        }
      } else if (e == kZRow) {
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          if (d0 + u < D) {
            if (has_z) a[u] += sZ[d0 + u];
            sZ[d0 + u] = a[u];
          }
        }
      }
      uint2 w;
      w.x = pack_bf16x2(a[0], a[1]);
      w.y = pack_bf16x2(a[2], a[3]);
      const size_t off = static_cast<size_t>(bh) * kPTileBytes + (d0 >> 6) * (kPTileRows * 128) + e * 128 +
                         ((((d0 & 63) >> 3) ^ (e & 7)) << 4) + (d0 & 7) * 2;
      *reinterpret_cast<uint2*>(ptiles + off) = w;
    }
  }
}

// Step 3 (after the prefix rows are published; nothing in this launch reads the outgoing cache):
// the share's rows of the outgoing cache from sS / sZ.
__device__ void combine_store_cache(const Geom& geo, float* S_out, float* z_out, int bh, int r0, int r1,
                                    const float* sS, const float* sZ, int tid, int nthr) {
  const int D = geo.D, ld = D + 1, ns = cache_rows(geo, r0, r1);
  if (S_out != nullptr) {
    for (int i = tid; i < D * ns; i += nthr) {
      const int d = i / ns, j = i - d * ns;
      S_out[(static_cast<size_t>(bh) * D + d) * D + r0 + j] = sS[j * ld + d];
    }
  }
  if (z_out != nullptr && r0 <= kZRow && kZRow < r1)
    for (int d = tid; d < D; d += nthr) z_out[static_cast<size_t>(bh) * D + d] = sZ[d];
}

__global__ void __launch_bounds__(kThreads, 1)
    fused_bf16_kernel(const __grid_constant__ CUtensorMap k_main, const __grid_constant__ CUtensorMap k_last,
                      const __grid_constant__ CUtensorMap v_main, const __grid_constant__ CUtensorMap v_last,
                      const __grid_constant__ CUtensorMap q_main, const __grid_constant__ CUtensorMap q_last,
                      const __grid_constant__ CUtensorMap o_main, const __grid_constant__ CUtensorMap o_last,
                      const Geom geo, float* __restrict__ partials, int2* __restrict__ segcta,
                      uint64_t* __restrict__ slot_ready, uint64_t* __restrict__ combined,
                      uint8_t* __restrict__ ptiles, const float* S_in, const float* z_in, float* S_out,
                      float* z_out, const float eps, uint32_t* status) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ int s_ok;
  __shared__ uint64_t s_tag;
  uint8_t* smem = align1024(smem_raw);
  uint64_t* barmem = reinterpret_cast<uint64_t*>(smem + fu::kRegion);
  const st::Bars sb = st::bars_at(barmem);
  const ot::Bars ob = ot::bars_at(barmem + st::kNumBars);
  uint64_t* flushed = barmem + st::kNumBars + ot::kNumBars;  // epilogue warps finished a slot (count 4)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(flushed + 1);
  volatile int4* ring = reinterpret_cast<volatile int4*>(flushed + 2);  // 16-byte aligned
  uint64_t* seqp = reinterpret_cast<uint64_t*>(status + 2);  // header bytes 8..15: launch sequence number
  uint32_t* gstart = status + 4;                             // header bytes 16..19: CTAs that read the tag
  uint32_t* chunks = status + 7;  // header bytes 28..35: output-chunk counters, one per launch-tag parity
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int g = blockIdx.x;
  const int G = gridDim.x;
  const long long tb = tile_begin(g, geo);
  const long long te = tile_begin(g + 1, geo);
  const bool two_atoms = geo.D > 64;
  const Maps4 mkv{&k_main, &k_last, &v_main, &v_last};
  const Maps4 mqo{&q_main, &q_last, &o_main, &o_last};
  if (threadIdx.x == 0) {
    st::init_bars(sb);
    ot::init_bars(ob, two_atoms);
    mbar_init(flushed, 4);
    fence_mbar_init();
  }
  st::init_smem(smem, two_atoms, kThreads);
  if (warp == kWarpProducer && lane == 0) {
    prefetch_maps(mkv);
    prefetch_maps(mqo);
  }
  const uint32_t tmem = persistent_setup(tmem_slot, warp);
  // Up to here only this CTA's shared memory and TMEM were touched, so this part overlaps the
  // previous kernel in the stream (programmatic dependent launch). That kernel may still write
  // q, k, v, the cache or this workspace: wait for it to complete before any global access.
  griddep_wait();
  // Thread 0 (epilogue warp 0) is the only user of the launch tag before phase 2: it reads the tag
  // here, off the other roles' path, and shares it through s_tag with phase 2 and 3.
  uint64_t tag = 0;
  if (threadIdx.x == 0) {
    s_ok = 1;
    tag = ld_acquire_u64(seqp) + 1;
    s_tag = tag;
    // The last CTA to read the sequence number advances it for the next launch on this workspace:
    // every CTA has read it by then (acq_rel orders each CTA's read before its increment), and the
    // next launch reads it only after this one has completed.
    if (atom_add_acq_rel_u32(gstart, 1u) == static_cast<uint32_t>(G - 1)) {
      *gstart = 0u;
      // The chunk counter of the other parity was last used by the previous launch, which has
      // completed (this one passed griddepcontrol.wait); the next launch uses it, and it claims
      // chunks only after this launch has completed.
      chunks[(tag + 1) & 1] = 0u;
      st_release_u64(seqp, tag);
    }
    griddep_launch_dependents();  // the next launch may now set up on SMs as they free up
  }

  // phase 1: block states of this CTA's tiles
  int pre = 0;
  if (warp == kWarpProducer) {
    if (lane == 0) st::produce(smem, sb, mkv, geo, tb, te, two_atoms, false, status);
  } else if (warp >= 4 && warp < 8) {
    st::relu_role(smem, sb, tb, te, two_atoms, threadIdx.x - 128, lane, status);
  } else if (warp == kWarpMma) {
    if (lane == 0) st::mma_role(smem, sb, geo, tb, te, tmem, status);
  } else {
    st::epilogue_role(sb, geo, tb, te, tmem, g, warp, lane, partials, segcta, slot_ready, flushed, tag, status);
  }
  tc_fence_before();
  __syncthreads();
  tag = s_tag;

  // phase 2: the Q stages fill (Q does not depend on the state, and the stages are free once the
  // state MMAs retired) while the CTA takes its share of the combine of its head(s): whole prefix
  // rows, so each cache element belongs to exactly one CTA.
  // The output tiles: a static range of the first T - tdyn tiles, then chunks of the last tdyn
  // claimed through this launch's counter, so that the CTAs end together: the next launch's CTAs
  // wait on one another, so every call pays for this launch's slowest CTA.
  const ot::Seq sq{out_tile_begin(g, geo), out_tile_begin(g + 1, geo), geo.T - geo.tdyn, geo.T,
                   geo.tdyn > 0 ? chunks + (tag & 1) : nullptr, ring};
  if (warp == kWarpProducer && lane == 0) pre = ot::prefill(smem, ob, mqo, geo, sq, two_atoms);
  float* sS = reinterpret_cast<float*>(smem + fu::kScratchOff);
  float* sZ = reinterpret_cast<float*>(smem + fu::kScratchZOff);
  const int h0 = tile_coord(tb, geo).seg;
  const int h1 = tile_coord(te - 1, geo).seg;
  for (int h = h0; h <= h1; ++h) {
    const CombineRange cr = combine_range(h, geo);
    if (g < cr.ga || g > cr.gb) continue;
    const int n = cr.gb - cr.ga + 1, idx = g - cr.ga;
    const int r0 = idx * kPTileRows / n, r1 = (idx + 1) * kPTileRows / n;
    combine_load_cache(geo, S_in, z_in, h, r0, r1, sS, sZ, threadIdx.x, kThreads);  // needs no other CTA
    if (threadIdx.x == 0 && s_ok && !wait_flags(slot_ready, cr.g0 + h, cr.g1 + h, tag, status, 0x2000u)) s_ok = 0;
    __syncthreads();
    if (s_ok)
      combine_sum(geo, partials, cr.g0, cr.g1, S_in != nullptr, z_in != nullptr, ptiles, h, r0, r1, sS, sZ);
    __syncthreads();
    if (threadIdx.x == 0 && s_ok) {
      __threadfence();
      st_release_u64(combined + g + h, tag);
    }
    if (s_ok) combine_store_cache(geo, S_out, z_out, h, r0, r1, sS, sZ, threadIdx.x, kThreads);
    __syncthreads();
  }
  fence_proxy_async_smem();  // the combine scratch is next written by TMA copies (async proxy)
  __syncthreads();
  tc_fence_after();

  // phase 3: the output tiles (static range, then claimed chunks), each once its head's combine is
  // complete
  if (s_ok) {
    if (warp == kWarpProducer) {
      if (lane == 0) ot::produce(smem, ob, mqo, geo, sq, pre, two_atoms, ptiles, combined, tag, status);
    } else if (warp >= 4 && warp < 8) {
      ot::relu_epi_role(smem, ot::Staging{smem + ot::kOOff, 1}, ob, mqo, geo, sq, 0, two_atoms, tmem, warp, lane,
                        eps, status);
    } else if (warp == kWarpMma) {
      if (lane == 0) ot::mma_role(smem, ob, geo, sq, two_atoms, tmem, status);
    } else {
      ot::epilogue_role(ot::Staging{smem + ot::kOOff, 1}, ob, mqo, geo, sq, tmem, warp, lane, eps, status);
    }
  } else if (warp == kWarpProducer && lane == 0) {
    for (int i = 0; i < pre; ++i) mbar_wait(&ob.qfull[i], 0, status, 0x2180u);  // prefilled loads land
  }
  persistent_teardown(tmem, warp);
}

// ------------------------------------------------------------------------------------------
// 5. one block per head with one thread-block cluster per head (few heads, e.g. a streaming step)
// ------------------------------------------------------------------------------------------
// Cluster h (C CTAs) owns head h. The head's rows are split between the ranks in units of 16 rows
// (rank r: units [r*U/C, (r+1)*U/C) of the U = ceil(N/16) units), at most 512 rows (4 tiles) per
// rank, so the busiest rank holds ~N/C rows instead of a whole number of 128-row tiles. A range
// that ends inside a tile is loaded with 16-row boxes (a 128-row box would read the next rank's
// rows); the state MMAs of a tile cover only its 16-row steps.
//   phase 1: rank r reduces its rows into TMEM (the state roles, one segment); meanwhile its
//            epilogue warps zero its share of the head's fp32 accumulator [129][128] in the
//            workspace and fetch its share of the incoming cache; after the last state MMA the
//            producer loads every Q tile of the rank (all of them fit: the stages are free), and
//            the ReLU warps apply the feature map to each as it lands.
//   exchange: the epilogue warps drain TMEM into shared memory as [e][d] rows (adding the rank's
//            share of the incoming cache), and one thread adds them to the head's accumulator
//            with TMA bulk reductions (cp.reduce.async.bulk .add.f32, in L2), half by half while
//            the drain goes on. A cluster barrier; then every rank reads the summed state (the
//            inclusive prefix P, fp32) back, writes it as its bf16 B tile and keeps its share of
//            rows for the outgoing cache.
//   phase 3: the output MMAs run back to back over the resident Q tiles; the epilogue stores each
//            tile's output through the tile's own Q slot (its MMA has read it by then).
// Two cluster barriers: B1 (accumulator zeroed; split arrive/wait, so nobody waits for it in
// practice) and B2 (every rank's reduction complete). Both are taken by every thread on every path
// (bounded mbarrier waits only make roles skip work), without .aligned so a warp's lanes may reach
// them at different points. The sums in L2 are in arrival order, so the fp32 state (and hence
// the output) is not bitwise reproducible from call to call on this path; its error stays the
// fp32 summation error.
namespace cl {
constexpr int kMinCluster = 4;
constexpr int kMaxCluster = 8;
constexpr int kUnit = 16;                            // rows per unit of the split between ranks
constexpr int kMaxTiles = 4;                         // resident Q tiles: at most 512 rows per rank
constexpr int kQSlot = 2 * kAtomBytes;               // one Q tile (32 KB), later its output staging
constexpr int kPartOff = kMaxTiles * kQSlot;         // fp32 partial [129][128], later the bf16 B tile
constexpr int kPartBytes = kPartRows * kDPad * 4;
constexpr int kRegion = st::kRegionBytes;
// The partial overlaps the last K/V stage and the ones tile: both are dead once the state MMAs
// retired, which the drain waits for.
static_assert(kPartOff + kPartBytes <= kRegion && kPartOff + kPTileBytes <= kRegion, "partial overflows the region");
static_assert(kPartOff % 1024 == 0, "B tile alignment");
constexpr int kShareRowsMax = (kPTileRows + kMinCluster - 1) / kMinCluster;
constexpr int kScratchOff = kRegion;                 // cache share [row][128] fp32 (S_in, then P)
constexpr int kScratchZOff = kScratchOff + kShareRowsMax * kDPad * 4;
constexpr int kBarOff = (kScratchZOff + kDPad * 4 + 127) / 128 * 128;
constexpr int kNumBars = st::kNumBars + 2 * kMaxTiles + 7;
constexpr int kSmem = kBarOff + 512 + 1024;
static_assert(kNumBars * 8 + 8 <= 512, "barrier area");
static_assert(kSmem <= 227 * 1024, "cluster kernel shared memory");

struct Bars3 {            // phase 3
  uint64_t* qfull;        // [4] Q tile j landed
  uint64_t* qrelu;        // [4] ReLU(Q tile j) written back (4 ReLU warps)
  uint64_t* accf;         // [2] output accumulator holds a tile
  uint64_t* acce;         // [2] output accumulator drained
  uint64_t* done;
  uint64_t* kvi;          // the producer has issued the first K/V stages
  uint64_t* rb;           // the summed state has landed in shared memory (read-back copy)
};
__device__ __forceinline__ Bars3 bars3_at(uint64_t* p) {
  return Bars3{p, p + kMaxTiles, p + 2 * kMaxTiles, p + 2 * kMaxTiles + 2, p + 2 * kMaxTiles + 4,
               p + 2 * kMaxTiles + 5, p + 2 * kMaxTiles + 6};
}

// Tiles of one rank: tile j starts at row tok0(j) of the head and holds rows(j) rows.
struct Range {
  int row0, row1, n, N;
  __device__ __forceinline__ int tok0(int j) const { return row0 + j * kTile; }
  __device__ __forceinline__ int rows(int j) const {
    const int r = row1 - tok0(j);
    return r < kTile ? r : kTile;
  }
  // A tile whose range ends before the head does is loaded with 16-row boxes; one that reaches the
  // head's end uses whole boxes, clipped (and zero-filled) by the tensor map.
  __device__ __forceinline__ bool boxed16(int j) const { return rows(j) < kTile && tok0(j) + kTile < N; }
};

struct Maps {
  const CUtensorMap* k;    // 128-row boxes
  const CUtensorMap* v;
  const CUtensorMap* q;
  const CUtensorMap* o;    // 32-row store boxes
  const CUtensorMap* k16;  // 16-row boxes
  const CUtensorMap* v16;
  const CUtensorMap* q16;
  const CUtensorMap* o16;
  const CUtensorMap* k64;  // 64-row boxes
  const CUtensorMap* v64;
  const CUtensorMap* q64;
};

// non-aligned cluster barrier halves: each thread arrives and waits at its own point
__device__ __forceinline__ void arrive_release() { asm volatile("barrier.cluster.arrive.release;" ::: "memory"); }
__device__ __forceinline__ void arrive_relaxed() { asm volatile("barrier.cluster.arrive.relaxed;" ::: "memory"); }
__device__ __forceinline__ void wait_acquire() { asm volatile("barrier.cluster.wait.acquire;" ::: "memory"); }
__device__ __forceinline__ void named_sync(int id, int nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}
__device__ __forceinline__ void bulk_reduce_add_f32(float* dst, const void* src, uint32_t bytes) {
  asm volatile("cp.reduce.async.bulk.global.shared::cta.bulk_group.add.f32 [%0], [%1], %2;" ::"l"(dst),
               "r"(smem_u32(src)), "r"(bytes)
               : "memory");
}

// Loads rows(j) rows of one [BH, N, D] tensor at (tok0, bh) into `dst` (128-row tile layout, one or
// two 16 KB atoms): one whole box, or for a range ending inside the tile one 64-row box and 16-row
// boxes for the rest (each copy instruction holds the producer for a while, so few and large).
__device__ __forceinline__ void load_rows(uint8_t* dst, const CUtensorMap* m128, const CUtensorMap* m64,
                                          const CUtensorMap* m16, uint64_t* bar, const Range& rg, int j, int bh,
                                          bool two_atoms, uint64_t pol) {
  const int tok0 = rg.tok0(j);
  const int na = two_atoms ? 2 : 1;
  if (!rg.boxed16(j)) {
    for (int a = 0; a < na; ++a) tma_load_4d(dst + a * kAtomBytes, m128, bar, 64 * a, tok0, 0, bh, pol);
    return;
  }
  const int nb = rg.rows(j) / kUnit;
  int u = 0;
  if (nb >= 4) {
    for (int a = 0; a < na; ++a) tma_load_4d(dst + a * kAtomBytes, m64, bar, 64 * a, tok0, 0, bh, pol);
    u = 4;
  }
  for (; u < nb; ++u)
    for (int a = 0; a < na; ++a)
      tma_load_4d(dst + a * kAtomBytes + u * (kUnit * 128), m16, bar, 64 * a, tok0 + u * kUnit, 0, bh, pol);
}

// Producer, phase 1: the rank's K and V tiles through the three stages; then, once every state
// MMA has retired (the stages are free), every Q tile of the rank into its own slot.
__device__ void produce(uint8_t* smem, const st::Bars& b, const Bars3& b3, const Maps& m, const Range& rg, int bh,
                        bool two_atoms, uint32_t* status) {
  const uint64_t pol = policy_evict_first();
  int j = 0;
  for (; j < rg.n; ++j) {
    const int s = j % st::kStages;
    if (j == st::kStages) mbar_arrive(b3.kvi);  // the first stages are in flight
    if (!mbar_wait(&b.empty[s], ((j / st::kStages) & 1) ^ 1, status, 0x3100u | s)) {
      if (j < st::kStages) mbar_arrive(b3.kvi);
      return;
    }
    uint8_t* stg = smem + s * st::kStageBytes;
    // both expect_tx before either copy, so the phase cannot complete early
    const int nb = rg.boxed16(j) ? rg.rows(j) / kUnit : 0;
    const uint32_t per = nb ? static_cast<uint32_t>(nb * kUnit * 128) : static_cast<uint32_t>(kAtomBytes);
    mbar_expect_tx(&b.full[s], (two_atoms ? 4u : 2u) * per);
    load_rows(stg, m.k, m.k64, m.k16, &b.full[s], rg, j, bh, two_atoms, pol);
    load_rows(stg + st::kKBytes, m.v, m.v64, m.v16, &b.full[s], rg, j, bh, two_atoms, pol);
  }
  if (rg.n <= st::kStages) mbar_arrive(b3.kvi);
  for (int i = (rg.n > st::kStages ? rg.n - st::kStages : 0); i < rg.n; ++i)
    if (!mbar_wait(&b.empty[i % st::kStages], (i / st::kStages) & 1, status, 0x3180u)) return;
  for (int i = 0; i < rg.n; ++i) {
    const int nb = rg.boxed16(i) ? rg.rows(i) / kUnit : 0;
    const uint32_t per = nb ? static_cast<uint32_t>(nb * kUnit * 128) : static_cast<uint32_t>(kAtomBytes);
    mbar_expect_tx(&b3.qfull[i], (two_atoms ? 2u : 1u) * per);
    load_rows(smem + i * kQSlot, m.q, m.q64, m.q16, &b3.qfull[i], rg, i, bh, two_atoms, pol);
  }
}

// MMA issuer, phase 1: ReLU(K)^T [V | 1] over the rank's rows into accumulator 0; only the 16-row
// steps that hold rows of the range are issued.
__device__ void mma_state(uint8_t* smem, const st::Bars& b, const Range& rg, uint32_t tmem, uint32_t* status) {
  constexpr uint32_t kIdescS = idesc_bf16_f32(128, 128, true, true);
  constexpr uint32_t kIdescZ = idesc_bf16_f32(128, 16, true, true);
  const uint64_t od = sdesc_sw128(smem_u32(smem + st::kOnesOff), kAtomBytes, 1024);
  for (int j = 0; j < rg.n; ++j) {
    const int s = j % st::kStages;
    const uint32_t ph = (j / st::kStages) & 1;
    if (!mbar_wait(&b.full[s], ph, status, 0x3310u | s)) return;
    if (!mbar_wait(&b.relu[s], ph, status, 0x3320u | s)) return;
    tc_fence_after();
    const uint32_t kb = smem_u32(smem + s * st::kStageBytes);
    const uint32_t vb = kb + st::kKBytes;
    const int steps = (rg.rows(j) + kUnit - 1) / kUnit;
    for (int kk = 0; kk < steps; ++kk) {
      const uint64_t ad = sdesc_sw128(kb + kk * 2048, kAtomBytes, 1024);
      const uint64_t bd = sdesc_sw128(vb + kk * 2048, kAtomBytes, 1024);
      const uint32_t acc = (j == 0 && kk == 0) ? 0u : 1u;
      mma_bf16(tmem, ad, bd, kIdescS, acc);
      mma_bf16(tmem + 128, ad, od, kIdescZ, acc);
    }
    mma_commit(&b.empty[s]);
  }
  mma_commit(&b.accf[0]);
}

__device__ __forceinline__ void st_shared_f32(uint32_t saddr, float v) {
  asm volatile("st.shared.f32 [%0], %1;" ::"r"(saddr), "f"(v) : "memory");
}
__device__ __forceinline__ void st_shared_v4(uint32_t saddr, uint4 v) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(saddr), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
               : "memory");
}

// Rows of the rank's share [r0, r1) that are rows of S (e < D): the incoming and outgoing cache go
// through sS as [row - r0][128] fp32 (features d >= D zero), z through sZ[128].
__device__ __forceinline__ int share_rows(const Geom& geo, int r0, int r1) {
  const int e_hi = r1 < geo.D ? r1 : geo.D;
  return e_hi > r0 ? e_hi - r0 : 0;
}
__device__ __forceinline__ bool share_has_z(int r0, int r1) { return r0 <= kZRow && kZRow < r1; }

// Warps 0-3, phase 1: the share of the incoming cache into sS / sZ (transposed: sS[e - r0][d] =
// S_in[d][e]), loads batched ahead of the stores. The rows reach the accumulator as one more bulk
// reduction, so the drain itself only stores.
__device__ void load_cache_share(const Geom& geo, const float* __restrict__ S_in, const float* __restrict__ z_in,
                                 int bh, int r0, int r1, float* __restrict__ sS, float* __restrict__ sZ, int tid) {
  const int D = geo.D, ns = share_rows(geo, r0, r1);
  if (S_in != nullptr && ns > 0) {
    for (int i = tid; i < ns * kDPad; i += 128) sS[i] = 0.f;  // features d >= D stay zero
    __syncwarp();
    asm volatile("bar.sync 1, 128;" ::: "memory");
    // items (d, e): consecutive threads take consecutive e of one key row d (coalesced reads)
    const float* src = S_in + static_cast<size_t>(bh) * D * D + r0;
    const int items = D * ns;
    for (int i0 = tid; i0 < items; i0 += 8 * 128) {
      float v[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int i = i0 + u * 128;
        const int d = i / ns, j = i - d * ns;
        v[u] = i < items ? __ldcg(src + static_cast<size_t>(d) * D + j) : 0.f;
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int i = i0 + u * 128;
        const int d = i / ns, j = i - d * ns;
        if (i < items) sS[j * kDPad + d] = v[u];
      }
    }
  }
  if (z_in != nullptr && share_has_z(r0, r1))
    sZ[tid] = tid < D ? __ldcg(z_in + static_cast<size_t>(bh) * D + tid) : 0.f;
}

// After the read-back (warp 8, overlapping the output): the share of the outgoing cache from sS /
// sZ. S_out[d][r0 + j] = sS[j][d]: float4 stores along j where the cache is 16-byte aligned (row
// starts then are too: D and r0 are multiples of 4), gathers batched ahead of the stores.
__device__ void store_cache_share(const Geom& geo, float* __restrict__ S_out, float* __restrict__ z_out, int bh,
                                  int r0, int r1, const float* __restrict__ sS, const float* __restrict__ sZ, int tid,
                                  int nthr) {
  const int D = geo.D, ns = share_rows(geo, r0, r1);
  if (S_out != nullptr && ns > 0) {
    float* dst = S_out + static_cast<size_t>(bh) * D * D + r0;
    if ((reinterpret_cast<uintptr_t>(S_out) & 15u) == 0u) {
      const int nq = ns / 4, items = D * nq;  // (d, quad of j)
      for (int i0 = tid; i0 < items; i0 += 4 * nthr) {
        float4 v[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int i = i0 + u * nthr;
          const int d = i / nq, j = (i - d * nq) * 4;
          if (i < items)
            v[u] = make_float4(sS[j * kDPad + d], sS[(j + 1) * kDPad + d], sS[(j + 2) * kDPad + d],
                               sS[(j + 3) * kDPad + d]);
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int i = i0 + u * nthr;
          const int d = i / nq, j = (i - d * nq) * 4;
          if (i < items) *reinterpret_cast<float4*>(dst + static_cast<size_t>(d) * D + j) = v[u];
        }
      }
    } else {
      for (int i = tid; i < D * ns; i += nthr) {
        const int d = i / ns, j = i - d * ns;
        dst[static_cast<size_t>(d) * D + j] = sS[j * kDPad + d];
      }
    }
  }
  if (z_out != nullptr && share_has_z(r0, r1))
    for (int d = tid; d < D; d += nthr) z_out[static_cast<size_t>(bh) * D + d] = sZ[d];
}

// Epilogue warps 0-3: the rank's share of the incoming cache goes to the head's accumulator first
// (bulk reductions of sS / sZ, issued once B1 has published the zeroing); then accumulator 0 (lane =
// key feature d) is drained into the partial [e][d] in shared memory, and thread 0 adds each
// drained half to the accumulator with a bulk reduction. Every thread of the four warps passes both
// named barriers whatever happened before.
__device__ void drain_reduce(const st::Bars& b, const Geom& geo, uint32_t tmem, int warp, int lane, int rank,
                             float* part, float* acc, bool has_S, bool has_z, int r0, int r1, const float* sS,
                             const float* sZ, uint32_t* status) {
  const int d = warp * 32 + lane;
  const bool ok = warp_all(mbar_wait(&b.accf[0], 0, status, 0x3400u));
  wait_acquire();  // B1: every rank has zeroed its share of the accumulator
  if (threadIdx.x == 0) {
    asm volatile("fence.proxy.async.global;" ::: "memory");  // the zeroing B1 acquired -> async proxy
    const int ns = share_rows(geo, r0, r1);
    if (has_S && ns > 0) bulk_reduce_add_f32(acc + r0 * kDPad, sS, static_cast<uint32_t>(ns * kDPad * 4));
    if (has_z && share_has_z(r0, r1)) bulk_reduce_add_f32(acc + kZRow * kDPad, sZ, kDPad * 4);
    bulk_commit();
  }
  if (ok) tc_fence_after();
  const uint32_t ta = tmem + (static_cast<uint32_t>(warp * 32) << 16);
  const uint32_t ps = smem_u32(part) + static_cast<uint32_t>(d * 4);
  // ranks of odd index drain and reduce the second half first, so that the head's ranks do not
  // all add into the same rows of the accumulator at the same time
#pragma unroll
  for (int hh = 0; hh < 2; ++hh) {
    const int h = hh ^ (rank & 1);
    if (ok) {
      uint32_t rr[2][32];
      uint32_t zr = 0;
      tmem_ld_x32(ta + h * 64, rr[0]);
      tmem_ld_x32(ta + h * 64 + 32, rr[1]);
      tmem_ld_x1(ta + 128, zr);
      tmem_wait_ld();
#pragma unroll
      for (int cc = 0; cc < 2; ++cc)
#pragma unroll
        for (int jj = 0; jj < 32; ++jj)
          st_shared_f32(ps + static_cast<uint32_t>((h * 64 + cc * 32 + jj) * kDPad * 4), __uint_as_float(rr[cc][jj]));
      if (h == 1) st_shared_f32(ps + static_cast<uint32_t>(kZRow * kDPad * 4), __uint_as_float(zr));
    }
    fence_proxy_async_smem();  // these generic writes -> the bulk reduction (async proxy)
    named_sync(1, 128);
    if (threadIdx.x == 0) {
      const int e0 = h * 64, e1 = h == 0 ? 64 : kPartRows;
      bulk_reduce_add_f32(acc + e0 * kDPad, part + e0 * kDPad, static_cast<uint32_t>((e1 - e0) * kDPad * 4));
      bulk_commit();
    }
  }
  if (threadIdx.x == 0) {
    bulk_wait_all();  // the reductions are complete in global memory
    asm volatile("fence.proxy.async.global;" ::: "memory");  // ... and ordered before the B2 release
  }
  tc_fence_before();
}

// Read-back, after B2: thread 0 copies the summed state P (fp32 [129][128], in L2) into the partial
// region with one bulk copy; then the 192 threads of warps 0-3, 8 and 9 (index gt) each take twelve
// (row, 8-feature) items into registers, meet, and write them back in place as the bf16 B tile
// (rows 129..143 zero) -- the tile overlaps the fp32 copy, hence the barrier between the two -- and
// the rank's share of rows into sS / sZ for the outgoing cache.
__device__ void read_back(const Geom& geo, const float* acc, const Bars3& b3, uint8_t* region, int r0, int r1,
                          float* __restrict__ sS, float* __restrict__ sZ, int gt, uint32_t* status) {
  constexpr int kGroup = 192, kBatch = 12;
  static_assert(kGroup * kBatch == kPTileRows * 16, "one batch covers the B tile");
  if (threadIdx.x == 0) {
    mbar_expect_tx(b3.rb, kPartRows * kDPad * 4);
    bulk_load(region, acc, kPartRows * kDPad * 4, b3.rb);
  }
  const bool ok = warp_all(mbar_wait(b3.rb, 0, status, 0x3700u));
  const float* src = reinterpret_cast<const float*>(region);
  float4 v[kBatch][2];
#pragma unroll
  for (int i = 0; i < kBatch; ++i) {
    const int it = gt + i * kGroup;
    const int e = it >> 4, d = (it & 15) * 8;
    if (ok && e < kPartRows) {
      v[i][0] = *reinterpret_cast<const float4*>(src + e * kDPad + d);
      v[i][1] = *reinterpret_cast<const float4*>(src + e * kDPad + d + 4);
    } else {
      v[i][0] = v[i][1] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
  }
  named_sync(2, kGroup);  // every fp32 value is in registers before the bf16 tile overwrites them
  const int ns_hi = r0 + share_rows(geo, r0, r1);
  const uint32_t bs = smem_u32(region);
#pragma unroll
  for (int i = 0; i < kBatch; ++i) {
    const int it = gt + i * kGroup;
    const int e = it >> 4, d = (it & 15) * 8;
    uint4 w;
    w.x = pack_bf16x2(v[i][0].x, v[i][0].y);
    w.y = pack_bf16x2(v[i][0].z, v[i][0].w);
    w.z = pack_bf16x2(v[i][1].x, v[i][1].y);
    w.w = pack_bf16x2(v[i][1].z, v[i][1].w);
    st_shared_v4(bs + static_cast<uint32_t>((d >> 6) * (kPTileRows * 128) + e * 128 + ((((d & 63) >> 3) ^ (e & 7)) << 4)),
                 w);
    if (e >= r0 && e < ns_hi) {
      *reinterpret_cast<float4*>(sS + (e - r0) * kDPad + d) = v[i][0];
      *reinterpret_cast<float4*>(sS + (e - r0) * kDPad + d + 4) = v[i][1];
    } else if (e == kZRow && share_has_z(r0, r1)) {
      *reinterpret_cast<float4*>(sZ + d) = v[i][0];
      *reinterpret_cast<float4*>(sZ + d + 4) = v[i][1];
    }
  }
}

// MMA issuer, phase 3: ReLU(Q_j) [P | z]^T for every resident tile, accumulators alternating.
__device__ void mma_out(uint8_t* smem, const Bars3& b3, const Range& rg, bool two_atoms, uint32_t tmem,
                        uint32_t* status) {
  constexpr uint32_t kIdescO = idesc_bf16_f32(128, kPTileRows, false, false);
  const int ksteps = two_atoms ? 8 : 4;
  const uint32_t bbase = smem_u32(smem + kPartOff);
  for (int j = 0; j < rg.n; ++j) {
    const int a = j & 1;
    if (!mbar_wait(&b3.qrelu[j], 0, status, 0x3520u | j)) break;
    if (!mbar_wait(&b3.acce[a], ((j >> 1) & 1) ^ 1, status, 0x3530u | a)) break;
    tc_fence_after();
    const uint32_t qb = smem_u32(smem + j * kQSlot);
    const uint32_t dacc = tmem + static_cast<uint32_t>(a * 256);
    for (int kk = 0; kk < ksteps; ++kk) {
      const uint64_t ad = sdesc_sw128(qb + (kk >> 2) * kAtomBytes + (kk & 3) * 32, 16, 1024);
      const uint64_t bd = sdesc_sw128(bbase + (kk >> 2) * (kPTileRows * 128) + (kk & 3) * 32, 16, 1024);
      mma_bf16(dacc, ad, bd, kIdescO, kk > 0 ? 1u : 0u);
    }
    mma_commit(&b3.accf[a]);
  }
  mma_commit(b3.done);
  mbar_wait(b3.done, 0, status, 0x35F0u);
}

// Epilogue of every tile for one warp: TMEM lanes 32q.. (tokens), output columns 64h..64h+63;
// numerator / (denominator + eps) in bf16 into the tile's own Q slot (rows 32q.. of atom h), then
// a TMA store of those rows (16-row box where the range ends inside the warp's 32 rows).
__device__ void epilogue(uint8_t* smem, const Bars3& b3, const Maps& m, const Range& rg, int bh, uint32_t tmem, int q,
                         int h, int lane, float eps, uint32_t* status) {
  for (int j = 0; j < rg.n; ++j) {
    const int a = j & 1;
    if (!warp_all(mbar_wait(&b3.accf[a], (j >> 1) & 1, status, 0x3600u | a))) break;
    tc_fence_after();
    const uint32_t ta = tmem + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(a * 256);
    uint32_t dr;
    uint32_t rr[2][32];
    tmem_ld_x1(ta + kZRow, dr);
    tmem_ld_x32(ta + h * 64, rr[0]);
    tmem_ld_x32(ta + h * 64 + 32, rr[1]);
    tmem_wait_ld();
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(&b3.acce[a]);
    const float inv = __frcp_rn(__uint_as_float(dr) + eps);
    uint8_t* ob = smem + j * kQSlot + h * kAtomBytes + q * (32 * 128);
#pragma unroll
    for (int cc = 0; cc < 2; ++cc) {
#pragma unroll
      for (int mm = 0; mm < 4; ++mm) {
        uint4 w;
        w.x = pack_bf16x2(__uint_as_float(rr[cc][8 * mm + 0]) * inv, __uint_as_float(rr[cc][8 * mm + 1]) * inv);
        w.y = pack_bf16x2(__uint_as_float(rr[cc][8 * mm + 2]) * inv, __uint_as_float(rr[cc][8 * mm + 3]) * inv);
        w.z = pack_bf16x2(__uint_as_float(rr[cc][8 * mm + 4]) * inv, __uint_as_float(rr[cc][8 * mm + 5]) * inv);
        w.w = pack_bf16x2(__uint_as_float(rr[cc][8 * mm + 6]) * inv, __uint_as_float(rr[cc][8 * mm + 7]) * inv);
        const int chunk = cc * 4 + mm;
        *reinterpret_cast<uint4*>(ob + lane * 128 + ((chunk ^ (lane & 7)) << 4)) = w;
      }
    }
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) {
      const int tok0 = rg.tok0(j), rows = rg.rows(j), valid = rows - q * 32;
      if (valid > 0) {
        if (valid >= 32 || tok0 + rows >= rg.N)  // whole slice, or clipped at the head's end by the map
          tma_store_4d(m.o, ob, h * 64, tok0 + q * 32, 0, bh);
        else                                     // the range ends 16 rows into the slice
          tma_store_4d(m.o16, ob, h * 64, tok0 + q * 32, 0, bh);
      }
      bulk_commit();
    }
  }
  if (lane == 0) bulk_wait_all();
}
}  // namespace cl

__global__ void __launch_bounds__(kThreads, 1)
    cluster_bf16_kernel(const __grid_constant__ CUtensorMap k_map, const __grid_constant__ CUtensorMap v_map,
                        const __grid_constant__ CUtensorMap q_map, const __grid_constant__ CUtensorMap o_map,
                        const __grid_constant__ CUtensorMap k16_map, const __grid_constant__ CUtensorMap v16_map,
                        const __grid_constant__ CUtensorMap q16_map, const __grid_constant__ CUtensorMap o16_map,
                        const __grid_constant__ CUtensorMap k64_map, const __grid_constant__ CUtensorMap v64_map,
                        const __grid_constant__ CUtensorMap q64_map, const Geom geo, float* __restrict__ accum, const float* S_in, const float* z_in,
                        float* S_out, float* z_out, const float eps, uint32_t* status) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  uint64_t* barmem = reinterpret_cast<uint64_t*>(smem + cl::kBarOff);
  const st::Bars sb = st::bars_at(barmem);
  const cl::Bars3 b3 = cl::bars3_at(barmem + st::kNumBars);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(barmem + cl::kNumBars);
  float* part = reinterpret_cast<float*>(smem + cl::kPartOff);
  float* sS = reinterpret_cast<float*>(smem + cl::kScratchOff);
  float* sZ = reinterpret_cast<float*>(smem + cl::kScratchZOff);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int C = static_cast<int>(gridDim.x) / geo.BH;  // cluster size (grid = B*H clusters of C CTAs)
  const int bh = static_cast<int>(cluster_id_x());
  const int r = static_cast<int>(cluster_ctarank());
  const int units = (geo.N + cl::kUnit - 1) / cl::kUnit;
  cl::Range rg;
  rg.row0 = r * units / C * cl::kUnit;
  rg.row1 = (r + 1) * units / C * cl::kUnit;
  if (rg.row1 > geo.N) rg.row1 = geo.N;
  rg.n = (rg.row1 - rg.row0 + kTile - 1) / kTile;
  rg.N = geo.N;
  const int r0 = 4 * (r * (kPTileRows / 4) / C), r1 = 4 * ((r + 1) * (kPTileRows / 4) / C);  // cache share rows
  const bool two_atoms = geo.D > 64;
  const cl::Maps mp{&k_map, &v_map, &q_map, &o_map, &k16_map, &v16_map, &q16_map, &o16_map,
                    &k64_map, &v64_map, &q64_map};
  float* acc = accum + static_cast<size_t>(bh) * kPartRows * kDPad;
  if (threadIdx.x == 0) {
    st::init_bars(sb);
    for (int j = 0; j < cl::kMaxTiles; ++j) {
      mbar_init(&b3.qfull[j], 1);
      mbar_init(&b3.qrelu[j], 4);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&b3.accf[a], 1);
      mbar_init(&b3.acce[a], two_atoms ? 8 : 4);
    }
    mbar_init(b3.done, 1);
    mbar_init(b3.kvi, 1);
    mbar_init(b3.rb, 1);
    fence_mbar_init();
  }
  st::init_smem(smem, two_atoms, kThreads);
  if (warp == kWarpProducer && lane == 0) {
    prefetch_tmap(&k_map);
    prefetch_tmap(&v_map);
    prefetch_tmap(&q_map);
    prefetch_tmap(&o_map);
    prefetch_tmap(&k16_map);
    prefetch_tmap(&v16_map);
    prefetch_tmap(&q16_map);
    prefetch_tmap(&o16_map);
    prefetch_tmap(&k64_map);
    prefetch_tmap(&v64_map);
    prefetch_tmap(&q64_map);
  }
  const uint32_t tmem = persistent_setup(tmem_slot, warp);
  griddep_wait();  // the previous kernel in the stream may still write q, k, v, the cache or the workspace
  if (threadIdx.x == 0) griddep_launch_dependents();

  if (warp < 4) {
    // phase 1 for the epilogue warps: zero this rank's share of the accumulator, fetch its share of
    // the incoming cache, publish the zeroing (B1), then drain and reduce
    // their loads and stores wait until the producer's first K/V copies are issued: issued
    // together, they held back the producer's copy instructions by about a microsecond
    mbar_wait(b3.kvi, 0, status, 0x3050u);
    const int z1 = r1 < kPartRows ? r1 : kPartRows;
    for (int i = threadIdx.x; i < (z1 > r0 ? (z1 - r0) * (kDPad / 4) : 0); i += 128)
      reinterpret_cast<float4*>(acc + r0 * kDPad)[i] = make_float4(0.f, 0.f, 0.f, 0.f);
    cl::load_cache_share(geo, S_in, z_in, bh, r0, r1, sS, sZ, threadIdx.x);
    cl::arrive_release();  // B1
    fence_proxy_async_smem();  // the cache share in sS / sZ -> its bulk reduction (async proxy)
    cl::named_sync(1, 128);
    cl::drain_reduce(sb, geo, tmem, warp, lane, r, part, acc, S_in != nullptr, z_in != nullptr, r0, r1, sS, sZ, status);
    cl::arrive_release();  // B2: this rank's reductions are complete
  } else if (warp < 8) {
    cl::arrive_relaxed();  // B1 (nothing to publish)
    st::relu_role(smem, sb, 0, rg.n, two_atoms, threadIdx.x - 128, lane, status);
    cl::wait_acquire();
    cl::arrive_relaxed();  // B2
    // ReLU of each Q tile as it lands
    for (int j = 0; j < rg.n; ++j) {
      if (!warp_all(mbar_wait(&b3.qfull[j], 0, status, 0x3200u | j))) break;
      relu_tile_inplace(smem + j * cl::kQSlot, (two_atoms ? cl::kQSlot : kAtomBytes) / 16, threadIdx.x - 128);
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&b3.qrelu[j]);
    }
  } else {
    cl::arrive_relaxed();  // B1
    if (lane == 0) {
      if (warp == kWarpProducer)
        cl::produce(smem, sb, b3, mp, rg, bh, two_atoms, status);
      else
        cl::mma_state(smem, sb, rg, tmem, status);
    }
    __syncwarp();
    cl::wait_acquire();
    cl::arrive_relaxed();  // B2
  }
  if (warp < 4 || warp >= 8) {
    cl::wait_acquire();  // B2: the head's summed state is in L2
    const int gt = warp < 4 ? static_cast<int>(threadIdx.x) : 128 + (warp - kWarpProducer) * 32 + lane;
    cl::read_back(geo, acc, b3, smem + cl::kPartOff, r0, r1, sS, sZ, gt, status);
    fence_proxy_async_smem();  // the B tile -> tcgen05.mma (async proxy)
    cl::named_sync(3, 192);
    tc_fence_after();
    // the outgoing cache while the output runs (nothing in this launch reads it): warp 8
    if (warp == kWarpProducer) cl::store_cache_share(geo, S_out, z_out, bh, r0, r1, sS, sZ, lane, 32);
  }
  // phase 3: output MMAs and epilogues
  if (warp < 4) {
    cl::epilogue(smem, b3, mp, rg, bh, tmem, warp, 0, lane, eps, status);
  } else if (warp < 8) {
    cl::wait_acquire();  // B2 (taken here so that the Q ReLU above never waits for it)
    if (two_atoms) cl::epilogue(smem, b3, mp, rg, bh, tmem, warp & 3, 1, lane, eps, status);
  } else if (warp == kWarpMma && lane == 0) {
    cl::mma_out(smem, b3, rg, two_atoms, tmem, status);
  }
  persistent_teardown(tmem, warp);
}

// ------------------------------------------------------------------------------------------
// fp32 I/O path (SIMT fp32; correctness path for fp32 inputs)
// ------------------------------------------------------------------------------------------
__device__ __forceinline__ float relu_f32(float x) { return (x != x) ? x : fmaxf(x, 0.f); }

constexpr int kF32Threads = 256;
constexpr int kStateF32Smem = 2 * kTile * kDPad * 4;                   // K, V tiles
constexpr int kOutF32Smem = kDPad * kPartRows * 4 + kTile * kDPad * 4;  // prefix (transposed), Q tile
constexpr int kF32TurnedBytes = kTile * kDPad * 4;                      // rotary form: the turned tile

// Rotary form: Xt = the feature pairs of the first `rows` rows of X turned (rows beyond: zero).
__device__ void turn_tile_f32(const float* X, float* Xt, int rows, int n0, int D, const RopeDev& rp) {
  const int half = D / 2;
  for (int i = threadIdx.x; i < kTile * half; i += kF32Threads) {
    const int rr = i / half, jj = i - rr * half;
    float2 t = make_float2(0.f, 0.f);
    if (rr < rows) {
      const float2 *rt, *rh, *rw;
      rope_rows(rp, n0 + rr, rt, rh, rw);
      t = turn_pair(X[rr * kDPad + 2 * jj], X[rr * kDPad + 2 * jj + 1], rope_cs(rp, jj, rt, rh, rw));
    }
    Xt[rr * kDPad + 2 * jj] = t.x;
    Xt[rr * kDPad + 2 * jj + 1] = t.y;
  }
}

__global__ void __launch_bounds__(kF32Threads, 1)
    state_f32_kernel(const float* __restrict__ k, const float* __restrict__ v, const Geom geo,
                     float* __restrict__ partials, int2* __restrict__ segcta, const RopeDev rp) {
  extern __shared__ float fsm[];
  float* Ks = fsm;
  float* Vs = fsm + kTile * kDPad;
  float* Kt = fsm + 2 * kTile * kDPad;  // rotary form only
  const bool rope = rp.tab != nullptr;
  const float* KS = rope ? Kt : Ks;     // the S products read the turned features, z the unturned
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
    if (rope) {
      turn_tile_f32(Ks, Kt, c.rows, c.blk * geo.L + c.tok0, D, rp);
      __syncthreads();
    }
    if (d < D) {
      for (int jr = 0; jr < c.rows; ++jr) {
        if (eh == 0) zacc += Ks[jr * kDPad + d];
        const float fk = KS[jr * kDPad + d];
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
                   const float* __restrict__ p32, const float eps, const RopeDev rp) {
  extern __shared__ float fsm[];
  float* Ps = fsm;                      // [d][e'] with e' = 0..128 (z at 128)
  float* Qs = fsm + kDPad * kPartRows;  // [row][d]
  float* Qt = Qs + kTile * kDPad;       // rotary form only: the turned tile
  const bool rope = rp.tab != nullptr;
  const float* QN = rope ? Qt : Qs;     // the numerator reads the turned features, the denominator the unturned
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
    if (rope) {
      turn_tile_f32(Qs, Qt, c.rows, c.blk * geo.L + c.tok0, D, rp);
      __syncthreads();
    }
    if (e < D) {
      for (int m = 0; m < 64; ++m) {
        const int rr = rh + 2 * m;
        if (rr >= c.rows) break;
        float num = 0.f, den = 0.f;
        for (int dd = 0; dd < D; ++dd) {
          num = fmaf(QN[rr * kDPad + dd], Ps[dd * kPartRows + e], num);
          den = fmaf(Qs[rr * kDPad + dd], Ps[dd * kPartRows + kZRow], den);
        }
        o[(row0 + rr) * D + e] = num / (den + eps);
      }
    }
  }
}

// (cos, sin) table of the rotary form: one thread per (row, pair). Row < frames: frame position
// row; then `height` grid rows, then `width` grid columns. Pair j of a group of P pairs starting
// at pair `off` turns by pos * base^(-(j - off) / P) (fp64 angle, rounded to fp32 once); pairs of
// the other groups hold (1, 0).
__global__ void rope_table_kernel(float2* tab, int frames, int height, int width, int half, int pt, int ph, int pw,
                                  double base) {
  const long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= static_cast<long long>(frames + height + width) * half) return;
  const int row = static_cast<int>(i / half);
  const int j = static_cast<int>(i - static_cast<long long>(row) * half);
  int pos, off, P;
  if (row < frames) {
    pos = row, off = 0, P = pt;
  } else if (row < frames + height) {
    pos = row - frames, off = pt, P = ph;
  } else {
    pos = row - frames - height, off = pt + ph, P = pw;
  }
  float2 cs = make_float2(1.f, 0.f);
  if (j >= off && j < off + P) {
    const double ang = static_cast<double>(pos) * pow(base, -static_cast<double>(j - off) / P);
    double sn, cn;
    sincos(ang, &sn, &cn);
    cs = make_float2(static_cast<float>(cn), static_cast<float>(sn));
  }
  tab[i] = cs;
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

size_t state_bf16_smem_bytes() { return kStateSmem; }
size_t out_bf16_smem_bytes() { return kOutSmem; }
size_t state_f32_smem_bytes() { return kStateF32Smem; }
size_t out_f32_smem_bytes() { return kOutF32Smem; }

cudaError_t set_kernel_attributes() {
  cudaError_t e;
  e = cudaFuncSetAttribute(state_bf16_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, kStateSmem);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(state_bf16_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, kStateSmemRope);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(out_bf16_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, kOutSmemRope);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(fused_bf16_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, fu::kSmem);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(cluster_bf16_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, cl::kSmem);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(out_bf16_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, kOutSmem);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(state_f32_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           kStateF32Smem + kF32TurnedBytes);
  if (e != cudaSuccess) return e;
  return cudaFuncSetAttribute(out_f32_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              kOutF32Smem + kF32TurnedBytes);
}

cudaError_t launch_state_bf16(const BlockMaps& k, const BlockMaps& v, const Geom& g, float* partials, int2* segcta,
                              uint32_t* status, cudaStream_t s, const RopeDev* rope) {
  if (rope != nullptr)
    return launch_pdl(state_bf16_kernel<true>, dim3(g.G), dim3(kThreads), kStateSmemRope, s, k.main, k.last, v.main,
                      v.last, g, partials, segcta, status, *rope);
  return launch_pdl(state_bf16_kernel<false>, dim3(g.G), dim3(kThreads), kStateSmem, s, k.main, k.last, v.main,
                    v.last, g, partials, segcta, status, RopeDev{});
}

cudaError_t launch_out_bf16(const BlockMaps& q, const BlockMaps& o, const Geom& g, const void* ptiles, float eps,
                            uint32_t* status, cudaStream_t s, const RopeDev* rope) {
  if (rope != nullptr)
    return launch_pdl(out_bf16_kernel<true>, dim3(g.G), dim3(kThreads), kOutSmemRope, s, q.main, q.last, o.main,
                      o.last,
                      g, static_cast<const uint8_t*>(ptiles), eps, status, *rope);
  return launch_pdl(out_bf16_kernel<false>, dim3(g.G), dim3(kThreads), kOutSmem, s, q.main, q.last, o.main, o.last,
                    g, static_cast<const uint8_t*>(ptiles), eps, status, RopeDev{});
}

cudaError_t launch_rope_table(float2* tab, int frames, int height, int width, int half, int pt, int ph, int pw,
                              double base, cudaStream_t s) {
  const long long n = static_cast<long long>(frames + height + width) * half;
  rope_table_kernel<<<static_cast<unsigned>((n + 255) / 256), 256, 0, s>>>(tab, frames, height, width, half, pt, ph,
                                                                           pw, base);
  return cudaGetLastError();
}

cudaError_t launch_fused_bf16(const BlockMaps& k, const BlockMaps& v, const BlockMaps& q, const BlockMaps& o,
                              const Geom& g, float* partials, int2* segcta, uint64_t* flags, void* ptiles,
                              const float* S_in, const float* z_in, float* S_out, float* z_out, float eps,
                              uint32_t* status, cudaStream_t s) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(g.G);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = fu::kSmem;
  cfg.stream = s;
  // The CTAs wait on one another (flags), so all of them must be resident at once: the grid has at
  // most one CTA per SM and each SM fits exactly one (shared memory, TMEM), so on an otherwise idle
  // device every CTA is placed. The launch uses programmatic stream serialization: each CTA sets up
  // while the previous kernel drains and waits (griddepcontrol.wait) before any global access.
  // A cooperative launch would also guarantee residency when other streams hold SMs, but the
  // runtime then starts the grid only after the previous kernel has fully ended (measured: about
  // 3 us later per launch). With SV_FUSED_COOPERATIVE=1 in the environment the launch is
  // cooperative instead. Either way every wait is bounded: a CTA kept off the device for longer
  // than the wait limit makes the call fail with the timeout status, never hang.
  static const bool cooperative = [] {
    const char* e = std::getenv("SV_FUSED_COOPERATIVE");
    return e != nullptr && e[0] == '1';
  }();
  cudaLaunchAttribute attr[1];
  if (cooperative) {
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
  } else {
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
  }
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, fused_bf16_kernel, k.main, k.last, v.main, v.last, q.main, q.last, o.main, o.last,
                            g, partials, segcta, flags, flags + g.nslots, static_cast<uint8_t*>(ptiles), S_in, z_in,
                            S_out, z_out, eps, status);
}

// Cluster size for the cluster kernel, or 0 when the flag-synchronised kernel should run: the
// largest C in [4, 8] such that every rank gets a tile, B*H clusters of C CTAs can all be resident
// (as the occupancy query reports for this device), and they occupy at least 3/4 of the SMs.
int cluster_size(const Geom& g, int sm_count) {
  static std::mutex mu;
  static int max_active[64][cl::kMaxCluster + 1];
  static bool known[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
  std::lock_guard<std::mutex> lock(mu);
  if (!known[dev]) {
    for (int c = cl::kMinCluster; c <= cl::kMaxCluster; ++c) {
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3(c * 16);
      cfg.blockDim = dim3(kThreads);
      cfg.dynamicSmemBytes = cl::kSmem;
      cudaLaunchAttribute attr[1];
      attr[0].id = cudaLaunchAttributeClusterDimension;
      attr[0].val.clusterDim.x = c;
      attr[0].val.clusterDim.y = 1;
      attr[0].val.clusterDim.z = 1;
      cfg.attrs = attr;
      cfg.numAttrs = 1;
      int n = 0;
      if (cudaOccupancyMaxActiveClusters(&n, cluster_bf16_kernel, &cfg) != cudaSuccess) {
        (void)cudaGetLastError();
        n = 0;
      }
      max_active[dev][c] = n;
    }
    known[dev] = true;
  }
  // every rank gets at least one 16-row unit and at most kMaxTiles tiles of rows
  const int units = cdiv(g.N, cl::kUnit);
  for (int c = cl::kMaxCluster; c >= cl::kMinCluster; --c) {
    if (g.nblk != 1 || units < c || cdiv(units, c) * cl::kUnit > cl::kMaxTiles * kTile) continue;
    if (max_active[dev][c] < g.BH) continue;
    if (static_cast<long long>(g.BH) * c * 4 < static_cast<long long>(sm_count) * 3) continue;
    return c;
  }
  return 0;
}

cudaError_t launch_cluster_bf16(const ClusterMaps& m, const Geom& g, int C, float* accum, const float* S_in,
                                const float* z_in, float* S_out, float* z_out, float eps, uint32_t* status,
                                cudaStream_t s) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(g.BH * C));
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = cl::kSmem;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = static_cast<unsigned>(C);
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, cluster_bf16_kernel, m.k, m.v, m.q, m.o, m.k16, m.v16, m.q16, m.o16, m.k64, m.v64,
                            m.q64, g, accum, S_in, z_in, S_out, z_out, eps, status);
}

cudaError_t launch_scan(const float* partials, const int2* segcta, const Geom& g, const float* S_in, const float* z_in,
                        float* S_out, float* z_out, void* ptiles_bf16, float* p32, uint32_t* out_chunks,
                        cudaStream_t s) {
  // ng warps share the blocks of one row (kScanReg each in registers); R rows per block so that a
  // block has a few warps: at ~124 registers per thread, small blocks pack the SMs best.
  int ng = (g.nblk + kScanReg - 1) / kScanReg;
  if (ng > kScanMaxWarps) ng = kScanMaxWarps;
  if (ng < 1) ng = 1;
  int R = 4;
  while (R > 1 && (R * ng > 4 || kPTileRows % R != 0)) R >>= 1;
  const size_t smem = static_cast<size_t>(R) * (ng + 1) * 32 * sizeof(float4);
  return launch_pdl(scan_kernel, dim3(g.BH, kPTileRows / R), dim3(32 * ng * R), smem, s, partials, segcta, g, S_in,
                    z_in, S_out, z_out, static_cast<uint8_t*>(ptiles_bf16), p32, ng, out_chunks);
}

cudaError_t launch_state_f32(const float* k, const float* v, const Geom& g, float* partials, int2* segcta,
                             uint32_t*, cudaStream_t s, const RopeDev* rope) {
  const int smem = kStateF32Smem + (rope != nullptr ? kF32TurnedBytes : 0);
  state_f32_kernel<<<g.G, kF32Threads, smem, s>>>(k, v, g, partials, segcta, rope != nullptr ? *rope : RopeDev{});
  return cudaGetLastError();
}

cudaError_t launch_out_f32(const float* q, float* o, const Geom& g, const float* p32, float eps, uint32_t*,
                           cudaStream_t s, const RopeDev* rope) {
  const int smem = kOutF32Smem + (rope != nullptr ? kF32TurnedBytes : 0);
  out_f32_kernel<<<g.G, kF32Threads, smem, s>>>(q, o, g, p32, eps, rope != nullptr ? *rope : RopeDev{});
  return cudaGetLastError();
}

}  // namespace sv
