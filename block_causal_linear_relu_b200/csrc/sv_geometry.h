// Problem geometry shared by the host launcher and the kernels.
//
// A (batch, head) pair "bh" holds N tokens split into blocks of L tokens (the last block may be
// shorter). Every block is cut into tiles of kTile = 128 tokens that start at the block's first
// token, so a tile never straddles two blocks. A "segment" is one (bh, block) pair; tiles are
// numbered bh-major, then block, then tile-in-block.
//
// The state kernel and the output kernel are persistent: CTA g of G takes the contiguous tile
// range [g*T/G, (g+1)*T/G). A CTA that ends or changes segment flushes its running partial state
// into slot g + s (s = segment). Because ranges are contiguous and ordered, the pairs (g, s) that
// touch are a monotone staircase and g + s never repeats, so G + nseg - 1 slots suffice and the
// scan sums, for segment s, the slots g + s of g = cta_of(first tile of s) .. cta_of(last tile).
#pragma once

#include <stdint.h>

#ifdef __CUDACC__
#define SV_HD __host__ __device__ __forceinline__
#else
#define SV_HD inline
#endif

namespace sv {

constexpr int kTile = 128;              // tokens per tile (MMA M of the output GEMM, K of the state GEMM)
constexpr int kDPad = 128;              // key/value feature dimension padded to 128
constexpr int kZRow = 128;              // row of the partial/prefix holding z (after the 128 S^T rows)
constexpr int kPartRows = 129;          // S^T rows (value feature e) + the z row
constexpr int kPTileRows = 144;         // B operand rows of the output GEMM: 128 + z row + 15 zero rows
constexpr int kPTileBytes = kPTileRows * kDPad * 2;          // one bf16 prefix tile, 36,864 B
constexpr int kPartBytes = kPartRows * kDPad * 4;            // one fp32 partial, 66,048 B
constexpr int kOutChunk = 4;      // tiles per dynamically handed-out output chunk
constexpr int kHeaderBytes = 256;                            // status word(s) at the workspace start

constexpr uint32_t kDevTimeout = 0x80000000u;                // status bit: a bounded wait expired
constexpr int kMirrorWord = 10;  // header bytes 40..47 (32-bit word 10): device address of a host-mapped status copy
constexpr uint64_t kWaitLimitNs = 2000000000ull;             // 2 s per wait

struct Geom {
  int BH;       // batch * heads
  int N;        // tokens per (batch, head)
  int D;        // key/value feature dimension (<= 128)
  int L;        // block length in tokens, clamped to N
  int nblk;     // number of blocks, ceil(N / L)
  int Llast;    // tokens in the last block
  int tpb;      // tiles per full block
  int tpl;      // tiles in the last block
  int tph;      // tiles per (batch, head)
  int G;        // persistent CTAs
  long long T;  // total tiles
  int nseg;     // BH * nblk
  int nslots;   // G + nseg - 1
  long long tdyn;  // output pass: the last tdyn tiles are handed out dynamically (multiple of kOutChunk)
};

SV_HD int cdiv(long long a, long long b) { return static_cast<int>((a + b - 1) / b); }

SV_HD long long tile_begin(int g, const Geom& q) { return static_cast<long long>(g) * q.T / q.G; }

SV_HD int cta_of_tile(long long t, const Geom& q) {
  return static_cast<int>(((t + 1) * static_cast<long long>(q.G) - 1) / q.T);
}

struct TileCoord {
  int bh;     // (batch, head)
  int blk;    // block index within the head
  int tok0;   // first token of the tile, relative to the block start
  int seg;    // segment = bh * nblk + blk
  int rows;   // valid tokens in this tile (1..128)
  bool last;  // last tile of its segment
};

SV_HD TileCoord tile_coord(long long t, const Geom& q) {
  TileCoord c;
  c.bh = static_cast<int>(t / q.tph);
  int r = static_cast<int>(t - static_cast<long long>(c.bh) * q.tph);
  int b = r / q.tpb;
  if (b > q.nblk - 1) b = q.nblk - 1;
  c.blk = b;
  int i = r - b * q.tpb;
  c.tok0 = i * kTile;
  c.seg = c.bh * q.nblk + b;
  int blen = (b == q.nblk - 1) ? q.Llast : q.L;
  int rem = blen - c.tok0;
  c.rows = rem < kTile ? rem : kTile;
  int ntiles = (b == q.nblk - 1) ? q.tpl : q.tpb;
  c.last = (i == ntiles - 1);
  return c;
}

SV_HD long long seg_first_tile(int seg, const Geom& q) {
  int bh = seg / q.nblk;
  int b = seg - bh * q.nblk;
  return static_cast<long long>(bh) * q.tph + static_cast<long long>(b) * q.tpb;
}

SV_HD int seg_ntiles(int seg, const Geom& q) {
  int b = seg % q.nblk;
  return (b == q.nblk - 1) ? q.tpl : q.tpb;
}

// The combine of head h (one block per head) is shared by the CTAs [ga, gb]: those whose tile
// range starts inside the head, or, when none does, the CTA holding the head's first tile. Each
// CTA then combines one head, apart from heads shorter than a CTA's range.
struct CombineRange {
  int g0, g1;  // CTAs covering the head (their slots g + h hold its partial states)
  int ga, gb;  // CTAs sharing its combine
};
SV_HD CombineRange combine_range(int h, const Geom& geo) {
  const long long f = seg_first_tile(h, geo);
  CombineRange r;
  r.g0 = cta_of_tile(f, geo);
  r.g1 = cta_of_tile(f + seg_ntiles(h, geo) - 1, geo);
  r.ga = tile_begin(r.g0, geo) == f ? r.g0 : r.g0 + 1;
  r.gb = r.g1;
  if (r.ga > r.gb) r.ga = r.gb = r.g0;
  return r;
}

// Host-side construction. Returns false when the sizes are out of range.
inline bool make_geom(Geom& q, int B, int H, int N, int D, int block_len, int sm_count) {
  if (B <= 0 || H <= 0 || N <= 0 || D <= 0 || block_len <= 0 || sm_count <= 0) return false;
  long long bh = static_cast<long long>(B) * H;
  if (bh > (1ll << 30)) return false;
  q.BH = static_cast<int>(bh);
  q.N = N;
  q.D = D;
  q.L = block_len < N ? block_len : N;
  q.nblk = cdiv(N, q.L);
  q.Llast = N - (q.nblk - 1) * q.L;
  q.tpb = cdiv(q.L, kTile);
  q.tpl = cdiv(q.Llast, kTile);
  q.tph = (q.nblk - 1) * q.tpb + q.tpl;
  q.T = static_cast<long long>(q.BH) * q.tph;
  q.G = static_cast<int>(q.T < sm_count ? q.T : sm_count);
  long long nseg = static_cast<long long>(q.BH) * q.nblk;
  if (nseg > (1ll << 30)) return false;
  q.nseg = static_cast<int>(nseg);
  q.nslots = q.G + q.nseg - 1;
  // The output pass splits [0, T - tdyn) statically over the G CTAs and hands out the remaining
  // tdyn tiles in chunks of kOutChunk to whichever CTA finishes first (about 1/8 of the tiles,
  // once every CTA has at least 8 static tiles).
  q.tdyn = q.T >= 9ll * q.G ? (q.T / 8) / kOutChunk * kOutChunk : 0;
  return true;
}

// Static output range of CTA g: [out_tile_begin(g), out_tile_begin(g + 1)) of [0, T - tdyn).
SV_HD long long out_tile_begin(int g, const Geom& q) { return static_cast<long long>(g) * (q.T - q.tdyn) / q.G; }

}  // namespace sv
