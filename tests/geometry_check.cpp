// Host check of the tile/segment/slot geometry shared by the kernels (sv_geometry.h):
// for many shapes it walks every CTA's tile range and verifies that
//  - tiles never straddle blocks and cover every token exactly once,
//  - the partial slot g + seg is unique per (CTA, segment) pair and < nslots,
//  - the CTA interval [cta_of(first), cta_of(last)] of each segment is exactly the set of CTAs
//    that flush a partial for it,
//  - with one block per head, the CTAs sharing a head's combine [ga, gb] form a non-empty
//    sub-interval of the CTAs covering it, so their flags (index g + h) are unique slots,
//  - the output pass's static ranges tile [0, T - tdyn) exactly, every CTA keeps at least 3 static
//    tiles when there is a dynamic tail, and the tail is a whole number of chunks.
#include <cstdio>
#include <cstdlib>
#include <set>
#include <utility>
#include <vector>

#include "../block_causal_linear_relu_b200/csrc/sv_geometry.h"

using namespace sv;

static int check(int B, int H, int N, int L, int sms) {
  Geom g;
  if (!make_geom(g, B, H, N, 128, L, sms)) { printf("make_geom failed\n"); return 1; }
  std::vector<int> covered((size_t)g.BH * g.N, 0);
  std::set<int> slots;
  std::set<std::pair<int, int>> flushes;
  for (int cta = 0; cta < g.G; ++cta) {
    long long tb = tile_begin(cta, g), te = tile_begin(cta + 1, g);
    if (te <= tb) { printf("empty CTA range\n"); return 1; }
    for (long long t = tb; t < te; ++t) {
      if (cta_of_tile(t, g) != cta) { printf("cta_of_tile mismatch\n"); return 1; }
      TileCoord c = tile_coord(t, g);
      int blen = (c.blk == g.nblk - 1) ? g.Llast : g.L;
      if (c.rows < 1 || c.rows > kTile || c.tok0 + c.rows > blen) { printf("tile rows\n"); return 1; }
      if ((c.tok0 + c.rows < blen) == c.last) { printf("last flag\n"); return 1; }
      for (int r = 0; r < c.rows; ++r) covered[(size_t)c.bh * g.N + (size_t)c.blk * g.L + c.tok0 + r]++;
      if (c.last || t == te - 1) {
        int slot = cta + c.seg;
        if (slot >= g.nslots || !slots.insert(slot).second) { printf("slot reuse %d\n", slot); return 1; }
        flushes.insert({c.seg, cta});
      }
    }
  }
  for (size_t i = 0; i < covered.size(); ++i)
    if (covered[i] != 1) { printf("token %zu covered %d times\n", i, covered[i]); return 1; }
  if (g.tdyn < 0 || g.tdyn % kOutChunk != 0 || g.tdyn >= g.T) { printf("tdyn %lld\n", g.tdyn); return 1; }
  if (out_tile_begin(0, g) != 0 || out_tile_begin(g.G, g) != g.T - g.tdyn) { printf("output ranges\n"); return 1; }
  for (int cta = 0; cta < g.G; ++cta) {
    const long long n = out_tile_begin(cta + 1, g) - out_tile_begin(cta, g);
    if (n < 1 || (g.tdyn > 0 && n < 3)) { printf("output static range of cta %d: %lld tiles\n", cta, n); return 1; }
  }
  for (int s = 0; s < g.nseg; ++s) {
    long long f = seg_first_tile(s, g);
    int g0 = cta_of_tile(f, g), g1 = cta_of_tile(f + seg_ntiles(s, g) - 1, g);
    for (int cta = 0; cta < g.G; ++cta) {
      bool in = cta >= g0 && cta <= g1;
      if (in != (flushes.count({s, cta}) > 0)) { printf("scan interval mismatch seg %d cta %d\n", s, cta); return 1; }
    }
    if (g.nblk == 1) {
      CombineRange cr = combine_range(s, g);
      if (cr.g0 != g0 || cr.g1 != g1 || cr.ga < g0 || cr.gb > g1 || cr.ga > cr.gb) {
        printf("combine range seg %d: [%d, %d] of [%d, %d]\n", s, cr.ga, cr.gb, g0, g1);
        return 1;
      }
      // a CTA whose range starts inside the head is always among those sharing its combine
      for (int cta = g0; cta <= g1; ++cta) {
        long long tb = tile_begin(cta, g);
        if (tb >= f && tb < f + seg_ntiles(s, g) && (cta < cr.ga || cta > cr.gb)) {
          printf("combine range seg %d misses cta %d\n", s, cta);
          return 1;
        }
      }
    }
  }
  return 0;
}

int main() {
  const int shapes[][5] = {{1, 20, 55200, 2760, 148}, {2, 20, 8190, 8190, 148}, {1, 2, 256, 64, 148},
                           {1, 3, 700, 300, 148},     {2, 20, 10120, 10120, 148}, {1, 1, 1, 1, 148},
                           {1, 4, 129, 1, 148},       {3, 5, 1000, 999, 7},       {1, 8, 20000, 2760, 148},
                           {1, 20, 2760, 2760, 148},  {2, 2, 5000, 128, 3},       {1, 1, 300, 1000, 148}};
  int bad = 0;
  for (auto& s : shapes) bad |= check(s[0], s[1], s[2], s[3], s[4]);
  srand(1);
  for (int i = 0; i < 300; ++i) {
    int B = 1 + rand() % 3, H = 1 + rand() % 5, N = 1 + rand() % 3000, L = 1 + rand() % (N + 50), sms = 1 + rand() % 200;
    if (check(B, H, N, L, sms)) { printf("failed B=%d H=%d N=%d L=%d sms=%d\n", B, H, N, L, sms); bad = 1; break; }
  }
  printf(bad ? "FAIL\n" : "OK\n");
  return bad;
}
