// Internal launch interface between the C-ABI layer (sv_api.cu) and the kernels (sv_kernels.cu).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/svlinattn.h"
#include "sv_geometry.h"

namespace sv {

// Workspace header (the first kHeaderBytes of every workspace, zeroed by sv_workspace_init):
//   bytes  0..3   status word: 0, or kDevTimeout | site of the first bounded wait that expired
//   bytes  8..15  launch sequence number of the one-block kernel (its flags carry it)
//   bytes 16..19  CTAs of the current one-block launch that have read the sequence number
//   bytes 24..27  dynamic output-chunk counter of the output kernel (reset by the scan kernel)
//   bytes 28..35  the one-block kernel's output-chunk counters, one per launch-sequence parity (the
//                 last CTA to read the sequence number clears the one the next launch uses)
//   bytes 40..47  device address of a host-mapped copy of the status word, or 0 (set by
//                 sv_workspace_set_mirror; a kernel that raises the status word also stores it there)

// Tensor maps of one [BH, N, D] bf16 tensor seen as blocks: `main` covers the blocks of length L,
// `last` the shorter last block when N is not a multiple of L (else it repeats `main`).
struct BlockMaps {
  CUtensorMap main;
  CUtensorMap last;
};

// 3D rotary embedding of the feature-mapped q and k, applied to the numerator only
// (sv_block_causal_attn_rope). tab holds (cos, sin) per (row, pair): rows [0, row_h) are frame
// positions, [row_h, row_w) grid rows, [row_w, ...) grid columns; `half` = D / 2 pairs per row.
// Token n of a (batch, head) sequence sits at frame f0 + n / hw, row (n % hw) / w, column n % w.
// Pairs [0, pt) turn with the frame, [pt, pth) with the row, [pth, half) with the column.
// The kernels of the bf16 path first copy the part of the table the call reads into shared
// memory, in a compact form: for each of the nf frames the call's tokens touch (f0 .. f0 + nf - 1)
// the frame group's pt pairs, then for each of the h grid rows the row group's pairs, then for
// each of the w columns the column group's pairs. `compact` is that entry count, or 0 when it
// exceeds kRopeSmemEntries (the kernels then read the table in global memory).
struct RopeDev {
  const float2* tab;
  int half, hw, w, f0, row_h, row_w, pt, pth;
  int nf, h, compact;
};
constexpr int kRopeSmemEntries = 3072;  // 24 KB of (cos, sin) pairs

// bf16 path (rope: nullptr, or the rotation of the numerator's features)
cudaError_t launch_state_bf16(const BlockMaps& k, const BlockMaps& v, const Geom& g, float* partials, int2* segcta,
                              uint32_t* status, cudaStream_t st, const RopeDev* rope = nullptr);
cudaError_t launch_out_bf16(const BlockMaps& q, const BlockMaps& o, const Geom& g, const void* ptiles,
                            float eps, uint32_t* status, cudaStream_t st, const RopeDev* rope = nullptr);
// fills a RopeDev table: rows = frames + height + width, `half` pairs per row
cudaError_t launch_rope_table(float2* tab, int frames, int height, int width, int half, int pt, int ph, int pw,
                              double base, cudaStream_t st);
// bf16, whole sequence in one block: state -> combine -> output in one cooperative launch
cudaError_t launch_fused_bf16(const BlockMaps& k, const BlockMaps& v, const BlockMaps& q, const BlockMaps& o,
                              const Geom& g, float* partials, int2* segcta, uint64_t* flags, void* ptiles,
                              const float* S_in, const float* z_in, float* S_out, float* z_out, float eps,
                              uint32_t* status, cudaStream_t st);
// bf16, whole sequence in one block, few heads: one thread-block cluster of C CTAs per head, whose
// ranks split the head's rows in 16-row units. Maps of the one-block [BH, N, D] tensors: k, v, q
// with 128-row boxes, o with 32-row store boxes, the same four with 16-row boxes and k, v, q with
// 64-row boxes. The head's summed state is reduced in `accum` (fp32 [BH][129][128] in the workspace).
// cluster_size returns the C to use for this geometry (0: use launch_fused_bf16 instead).
struct ClusterMaps {
  CUtensorMap k, v, q, o, k16, v16, q16, o16, k64, v64, q64;
};
int cluster_size(const Geom& g, int sm_count);
cudaError_t launch_cluster_bf16(const ClusterMaps& m, const Geom& g, int C, float* accum, const float* S_in,
                                const float* z_in, float* S_out, float* z_out, float eps, uint32_t* status,
                                cudaStream_t st);
// fp32 path
cudaError_t launch_state_f32(const float* k, const float* v, const Geom& g, float* partials, int2* segcta,
                             uint32_t* status, cudaStream_t st, const RopeDev* rope = nullptr);
cudaError_t launch_out_f32(const float* q, float* o, const Geom& g, const float* p32, float eps,
                           uint32_t* status, cudaStream_t st, const RopeDev* rope = nullptr);
// both paths: combine partials, inclusive prefix over blocks, optional final cache
// out_chunks: the output kernel's dynamic-chunk counter (workspace header bytes 24..27), reset here.
cudaError_t launch_scan(const float* partials, const int2* segcta, const Geom& g, const float* S_in, const float* z_in,
                        float* S_out, float* z_out, void* ptiles_bf16, float* p32, uint32_t* out_chunks,
                        cudaStream_t st);

// A 4-D bf16 tensor map with 128-byte swizzle (dims innermost first, byte strides of dims 1..3).
sv_status encode_bf16_4d(CUtensorMap* m, const void* base, const uint64_t dims[4], const uint64_t strides[3],
                         const uint32_t box[4]);

// Records `msg` as the calling thread's sv_last_error() text and returns `status`.
sv_status set_last_error(sv_status status, const char* msg);

size_t state_bf16_smem_bytes();
size_t out_bf16_smem_bytes();
size_t state_f32_smem_bytes();
size_t out_f32_smem_bytes();
cudaError_t set_kernel_attributes();

}  // namespace sv
