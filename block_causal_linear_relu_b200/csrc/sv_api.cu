// C-ABI layer: argument validation, workspace layout, TMA tensor maps and the launch sequence
// state -> scan -> output for every entry point of include/svlinattn.h.
#include <cudaTypedefs.h>

#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <string>

#include "../../include/svlinattn.h"
#include "sv_internal.h"

namespace {

using sv::Geom;

thread_local std::string g_last_error;
thread_local cudaEvent_t g_prof_events[4] = {nullptr, nullptr, nullptr, nullptr};

void prof_mark(int i, cudaStream_t s) {
  if (g_prof_events[i] != nullptr) cudaEventRecord(g_prof_events[i], s);
}

sv_status fail(sv_status s, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return s;
}

sv_status cuda_fail(cudaError_t e, const char* what) {
  return fail(SV_ERR_CUDA, "%s: %s (%s)", what, cudaGetErrorName(e), cudaGetErrorString(e));
}

// ---- per-device facts, looked up once ----
struct DevInfo {
  bool ready = false;
  int sm_count = 0;
  int major = 0, minor = 0;
  bool attrs = false;
};
constexpr int kMaxDevices = 64;
std::mutex g_dev_mutex;
DevInfo g_dev[kMaxDevices];

sv_status device_info(DevInfo& out, bool need_attrs) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return fail(SV_ERR_UNSUPPORTED, "device index %d out of range", dev);
  std::lock_guard<std::mutex> lock(g_dev_mutex);
  DevInfo& d = g_dev[dev];
  if (!d.ready) {
    e = cudaDeviceGetAttribute(&d.sm_count, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceGetAttribute(sm count)");
    e = cudaDeviceGetAttribute(&d.major, cudaDevAttrComputeCapabilityMajor, dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceGetAttribute(cc major)");
    e = cudaDeviceGetAttribute(&d.minor, cudaDevAttrComputeCapabilityMinor, dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceGetAttribute(cc minor)");
    d.ready = true;
  }
  if (need_attrs && !d.attrs) {
    if (d.major != 10 || d.minor != 0)
      return fail(SV_ERR_UNSUPPORTED, "device %d is sm_%d%d; this library is built for sm_100a", dev, d.major,
                  d.minor);
    e = sv::set_kernel_attributes();
    if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute");
    d.attrs = true;
  }
  out = d;
  return SV_OK;
}

// ---- tensor-map encoder from the driver, resolved through the runtime (no -lcuda) ----
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// Encoded maps of this thread's recent calls: an encoding depends only on the key below, so a hit
// is exactly the map the driver would encode again (a streaming loop reuses its buffers call after
// call, and each encode costs about a microsecond of host time).
struct MapKey {
  const void* base;
  uint64_t rows, nblk;
  int D, L, N, BH;
  uint32_t box_rows;
  bool operator==(const MapKey& o) const {
    return base == o.base && rows == o.rows && nblk == o.nblk && D == o.D && L == o.L && N == o.N && BH == o.BH &&
           box_rows == o.box_rows;
  }
};
constexpr int kMapCache = 32;
thread_local MapKey g_map_keys[kMapCache];
thread_local CUtensorMap g_maps[kMapCache];
thread_local int g_map_count = 0, g_map_next = 0;

sv_status encode_map_uncached(CUtensorMap* m, const void* base, uint64_t rows, uint64_t nblk, const Geom& g,
                              uint32_t box_rows);

sv_status encode_map(CUtensorMap* m, const void* base, uint64_t rows, uint64_t nblk, const Geom& g,
                     uint32_t box_rows) {
  const MapKey key{base, rows, nblk, g.D, g.L, g.N, g.BH, box_rows};
  for (int i = 0; i < g_map_count; ++i)
    if (g_map_keys[i] == key) {
      *m = g_maps[i];
      return SV_OK;
    }
  const sv_status s = encode_map_uncached(m, base, rows, nblk, g, box_rows);
  if (s != SV_OK) return s;
  const int i = g_map_next;
  g_map_next = (g_map_next + 1) % kMapCache;
  if (g_map_count < kMapCache) ++g_map_count;
  g_map_keys[i] = key;
  g_maps[i] = *m;
  return SV_OK;
}

sv_status encode_map_uncached(CUtensorMap* m, const void* base, uint64_t rows, uint64_t nblk, const Geom& g,
                              uint32_t box_rows) {
  auto fn = encode_fn();
  if (fn == nullptr) return fail(SV_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
  const uint64_t D = static_cast<uint64_t>(g.D);
  cuuint64_t dims[4] = {D, rows, nblk, static_cast<cuuint64_t>(g.BH)};
  cuuint64_t strides[3] = {D * 2, static_cast<uint64_t>(g.L) * D * 2, static_cast<uint64_t>(g.N) * D * 2};
  cuuint32_t box[4] = {64, box_rows, 1, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(SV_ERR_CUDA, "cuTensorMapEncodeTiled failed (CUresult %d)", static_cast<int>(r));
  return SV_OK;
}

}  // namespace

namespace sv {
sv_status encode_bf16_4d(CUtensorMap* m, const void* base, const uint64_t dims[4], const uint64_t strides[3],
                         const uint32_t box[4]) {
  auto fn = encode_fn();
  if (fn == nullptr) return fail(SV_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
  cuuint64_t d[4] = {dims[0], dims[1], dims[2], dims[3]};
  cuuint64_t st[3] = {strides[0], strides[1], strides[2]};
  cuuint32_t bx[4] = {box[0], box[1], box[2], box[3]};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), d, st, bx, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(SV_ERR_CUDA, "cuTensorMapEncodeTiled failed (CUresult %d)", static_cast<int>(r));
  return SV_OK;
}
}  // namespace sv

namespace {

// [BH, N, D] bf16 seen as [BH, nblk, L, D] blocks; the shorter last block gets its own map so that
// TMA bounds-checks every tile against its own block (zero fill on loads, clipping on stores).
sv_status make_block_maps(sv::BlockMaps& bm, const void* x, const Geom& g, uint32_t box_rows) {
  const bool partial = g.Llast != g.L;
  const uint64_t nmain = partial ? g.nblk - 1 : g.nblk;
  sv_status s = encode_map(&bm.main, x, static_cast<uint64_t>(g.L), nmain, g, box_rows);
  if (s != SV_OK) return s;
  if (!partial) {
    bm.last = bm.main;
    return SV_OK;
  }
  const uint8_t* lb = static_cast<const uint8_t*>(x) + static_cast<size_t>(g.nblk - 1) * g.L * g.D * 2;
  return encode_map(&bm.last, lb, static_cast<uint64_t>(g.Llast), 1, g, box_rows);
}

// ---- workspace layout ----
struct WsLayout {
  size_t flags = 0;     // offset of the per-slot ready / combined flags (single-launch path)
  size_t segcta = 0;    // offset of the per-segment (first CTA, last CTA) table
  size_t partials = 0;  // offset of the fp32 partial slots
  size_t ptiles = 0;    // offset of the prefix tiles (bf16 B operands or fp32 prefixes)
  size_t total = 0;
};

size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

WsLayout ws_layout(const Geom& g, sv_dtype dt, bool need_prefix) {
  WsLayout w;
  size_t off = sv::kHeaderBytes;
  w.flags = off;
  off += align256(static_cast<size_t>(g.nslots) * 2 * sizeof(uint64_t));  // ready + combined per slot
  w.segcta = off;
  off += align256(static_cast<size_t>(g.nseg) * sizeof(int2));
  w.partials = off;
  off += align256(static_cast<size_t>(g.nslots) * sv::kPartBytes);
  w.ptiles = off;
  if (need_prefix)
    off += align256(static_cast<size_t>(g.nseg) * (dt == SV_BF16 ? sv::kPTileBytes : sv::kPartBytes));
  w.total = off;
  return w;
}

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

sv_status check_sizes(int B, int H, int N, int D, int block_len, sv_dtype dt) {
  if (dt != SV_BF16 && dt != SV_F32) return fail(SV_ERR_UNSUPPORTED, "dtype %d is not SV_BF16 or SV_F32", (int)dt);
  if (B < 1 || H < 1) return fail(SV_ERR_INVALID_ARG, "B=%d and H=%d must be >= 1", B, H);
  if (N < 1) return fail(SV_ERR_INVALID_ARG, "N=%d must be >= 1", N);
  if (block_len < 1) return fail(SV_ERR_INVALID_ARG, "block_len=%d must be >= 1", block_len);
  if (dt == SV_BF16) {
    // rows of D bf16 values must be a whole number of 16-byte units for the TMA tensor maps; features
    // beyond D inside the 64-wide tile columns are zero-filled on load and clipped on store
    if (D < 8 || D > 128 || D % 8 != 0)
      return fail(SV_ERR_UNSUPPORTED, "bf16 path needs D a multiple of 8 in [8, 128], got D=%d", D);
  } else if (D < 1 || D > 128) {
    return fail(SV_ERR_UNSUPPORTED, "fp32 path needs 1 <= D <= 128, got D=%d", D);
  }
  if (static_cast<long long>(B) * H > (1ll << 24))
    return fail(SV_ERR_UNSUPPORTED, "B*H=%lld exceeds 2^24", static_cast<long long>(B) * H);
  return SV_OK;
}

sv_status geom_for(Geom& g, int B, int H, int N, int D, int block_len, int sm_count) {
  if (!sv::make_geom(g, B, H, N, D, block_len, sm_count)) return fail(SV_ERR_INVALID_ARG, "sizes out of range");
  return SV_OK;
}

sv_status check_io(const char* name, const void* p) {
  if (p == nullptr) return fail(SV_ERR_INVALID_ARG, "%s is NULL", name);
  if (!aligned(p, 16)) return fail(SV_ERR_INVALID_ARG, "%s is not 16-byte aligned", name);
  return SV_OK;
}

sv_status check_cache(const char* name, const void* p, bool required) {
  if (p == nullptr) return required ? fail(SV_ERR_INVALID_ARG, "%s is NULL", name) : SV_OK;
  if (!aligned(p, 4)) return fail(SV_ERR_INVALID_ARG, "%s is not 4-byte aligned", name);
  return SV_OK;
}

sv_status check_ws(void* ws, size_t ws_bytes, size_t need) {
  if (ws == nullptr) return fail(SV_ERR_INVALID_ARG, "workspace is NULL");
  if (!aligned(ws, 256)) return fail(SV_ERR_INVALID_ARG, "workspace is not 256-byte aligned");
  if (ws_bytes < need)
    return fail(SV_ERR_INVALID_ARG, "workspace has %zu bytes, %zu needed", ws_bytes, need);
  return SV_OK;
}

#define SV_TRY(expr)                \
  do {                              \
    sv_status _s = (expr);          \
    if (_s != SV_OK) return _s;     \
  } while (0)

// The whole forward path: state reduction -> partial combine + prefix -> output GEMM.
// With `rope` (the rotary form) the bf16 work always takes the three-kernel path.
sv_status run_forward(const void* q, const void* k, const void* v, void* o, int B, int H, int N, int D, int L,
                      sv_dtype dt, float eps, const float* S_in, const float* z_in, float* S_out, float* z_out,
                      void* ws, size_t ws_bytes, cudaStream_t stream, const sv::RopeDev* rope = nullptr) {
  SV_TRY(check_sizes(B, H, N, D, L, dt));
  SV_TRY(check_io("q", q));
  SV_TRY(check_io("k", k));
  SV_TRY(check_io("v", v));
  SV_TRY(check_io("o", o));
  SV_TRY(check_cache("S_in", S_in, false));
  SV_TRY(check_cache("z_in", z_in, false));
  SV_TRY(check_cache("S_out", S_out, false));
  SV_TRY(check_cache("z_out", z_out, false));
  if (!std::isfinite(eps) || eps < 0.f) return fail(SV_ERR_INVALID_ARG, "eps must be finite and >= 0");
  DevInfo di;
  SV_TRY(device_info(di, true));
  Geom g;
  SV_TRY(geom_for(g, B, H, N, D, L, di.sm_count));
  const WsLayout lay = ws_layout(g, dt, true);
  SV_TRY(check_ws(ws, ws_bytes, lay.total));

  uint8_t* wsb = static_cast<uint8_t*>(ws);
  uint32_t* status = reinterpret_cast<uint32_t*>(wsb);
  float* partials = reinterpret_cast<float*>(wsb + lay.partials);
  int2* segcta = reinterpret_cast<int2*>(wsb + lay.segcta);
  uint64_t* flags = reinterpret_cast<uint64_t*>(wsb + lay.flags);
  void* pre = wsb + lay.ptiles;
  cudaError_t e;
  if (dt == SV_BF16) {
    // one block per head and few heads: one thread-block cluster per head (a single launch)
    const int C = g.nblk == 1 && rope == nullptr ? sv::cluster_size(g, di.sm_count) : 0;
    if (C > 0) {
      sv::ClusterMaps cm;
      SV_TRY(encode_map(&cm.k, k, g.N, 1, g, sv::kTile));
      SV_TRY(encode_map(&cm.v, v, g.N, 1, g, sv::kTile));
      SV_TRY(encode_map(&cm.q, q, g.N, 1, g, sv::kTile));
      SV_TRY(encode_map(&cm.o, o, g.N, 1, g, 32));
      SV_TRY(encode_map(&cm.k16, k, g.N, 1, g, 16));
      SV_TRY(encode_map(&cm.v16, v, g.N, 1, g, 16));
      SV_TRY(encode_map(&cm.q16, q, g.N, 1, g, 16));
      SV_TRY(encode_map(&cm.o16, o, g.N, 1, g, 16));
      SV_TRY(encode_map(&cm.k64, k, g.N, 1, g, 64));
      SV_TRY(encode_map(&cm.v64, v, g.N, 1, g, 64));
      SV_TRY(encode_map(&cm.q64, q, g.N, 1, g, 64));
      prof_mark(0, stream);
      e = sv::launch_cluster_bf16(cm, g, C, partials, S_in, z_in, S_out, z_out, eps, status, stream);
      if (e != cudaSuccess) return cuda_fail(e, "cluster kernel launch");
      prof_mark(1, stream);
      prof_mark(2, stream);
      prof_mark(3, stream);
      return SV_OK;
    }
    sv::BlockMaps mq, mk, mv, mo;
    SV_TRY(make_block_maps(mk, k, g, sv::kTile));
    SV_TRY(make_block_maps(mv, v, g, sv::kTile));
    SV_TRY(make_block_maps(mq, q, g, sv::kTile));
    SV_TRY(make_block_maps(mo, o, g, 32));
    if (g.nblk == 1 && rope == nullptr) {  // one block per head, many heads: a single launch of co-resident CTAs
      prof_mark(0, stream);
      e = sv::launch_fused_bf16(mk, mv, mq, mo, g, partials, segcta, flags, pre, S_in, z_in, S_out, z_out, eps,
                                status, stream);
      if (e != cudaSuccess) return cuda_fail(e, "fused kernel launch");
      prof_mark(1, stream);
      prof_mark(2, stream);
      prof_mark(3, stream);
      return SV_OK;
    }
    prof_mark(0, stream);
    e = sv::launch_state_bf16(mk, mv, g, partials, segcta, status, stream, rope);
    if (e != cudaSuccess) return cuda_fail(e, "state kernel launch");
    prof_mark(1, stream);
    e = sv::launch_scan(partials, segcta, g, S_in, z_in, S_out, z_out, pre, nullptr, status + 6, stream);
    if (e != cudaSuccess) return cuda_fail(e, "scan kernel launch");
    prof_mark(2, stream);
    e = sv::launch_out_bf16(mq, mo, g, pre, eps, status, stream, rope);
    if (e != cudaSuccess) return cuda_fail(e, "output kernel launch");
    prof_mark(3, stream);
  } else {
    float* p32 = static_cast<float*>(pre);
    prof_mark(0, stream);
    e = sv::launch_state_f32(static_cast<const float*>(k), static_cast<const float*>(v), g, partials, segcta,
                             status, stream, rope);
    if (e != cudaSuccess) return cuda_fail(e, "state kernel launch");
    prof_mark(1, stream);
    e = sv::launch_scan(partials, segcta, g, S_in, z_in, S_out, z_out, nullptr, p32, status + 6, stream);
    if (e != cudaSuccess) return cuda_fail(e, "scan kernel launch");
    prof_mark(2, stream);
    e = sv::launch_out_f32(static_cast<const float*>(q), static_cast<float*>(o), g, p32, eps, status, stream, rope);
    if (e != cudaSuccess) return cuda_fail(e, "output kernel launch");
    prof_mark(3, stream);
  }
  return SV_OK;
}

// Table size check shared by sv_rope3d_table_bytes and the attention call: the grid and D.
sv_status check_rope_grid(int frames, int height, int width, int D) {
  if (frames < 1 || height < 1 || width < 1)
    return fail(SV_ERR_INVALID_ARG, "rope grid frames=%d height=%d width=%d must all be >= 1", frames, height, width);
  if (D < 2 || D > 128 || D % 2 != 0) return fail(SV_ERR_INVALID_ARG, "rope D=%d must be even, in [2, 128]", D);
  if (static_cast<long long>(frames) + height + width > (1ll << 24))
    return fail(SV_ERR_INVALID_ARG, "rope table of %lld rows is too large",
                static_cast<long long>(frames) + height + width);
  if (static_cast<long long>(height) * width > 0x7fffffffll)
    return fail(SV_ERR_INVALID_ARG, "rope grid height*width overflows int");
  return SV_OK;
}

sv_status check_rope_pairs(int D, int pt, int ph, int pw) {
  if (pt < 0 || ph < 0 || pw < 0 || 2 * (static_cast<long long>(pt) + ph + pw) != D)
    return fail(SV_ERR_INVALID_ARG, "rope pairs (%d, %d, %d) must be >= 0 and sum to D/2 = %d", pt, ph, pw, D / 2);
  return SV_OK;
}

// Checks a descriptor against the call's N and D and turns it into the kernels' form.
sv_status rope_for(sv::RopeDev& rd, const sv_rope3d* r, int N, int D) {
  if (r == nullptr) return fail(SV_ERR_INVALID_ARG, "rope descriptor is NULL");
  SV_TRY(check_rope_grid(r->frames, r->height, r->width, r->D));
  SV_TRY(check_rope_pairs(r->D, r->pairs_t, r->pairs_h, r->pairs_w));
  if (r->D != D) return fail(SV_ERR_INVALID_ARG, "rope table D=%d differs from the call's D=%d", r->D, D);
  if (r->table == nullptr || !aligned(r->table, 16)) return fail(SV_ERR_INVALID_ARG, "rope table is NULL or not 16-byte aligned");
  const long long hw = static_cast<long long>(r->height) * r->width;
  if (r->frame0 < 0 || r->frame0 + (static_cast<long long>(N) - 1) / hw >= r->frames)
    return fail(SV_ERR_INVALID_ARG, "rope frame0=%d with N=%d tokens of %lld per frame leaves the table's %d frames",
                r->frame0, N, hw, r->frames);
  rd.tab = reinterpret_cast<const float2*>(r->table);
  rd.half = D / 2;
  rd.hw = static_cast<int>(hw);
  rd.w = r->width;
  rd.f0 = r->frame0;
  rd.row_h = r->frames;
  rd.row_w = r->frames + r->height;
  rd.pt = r->pairs_t;
  rd.pth = r->pairs_t + r->pairs_h;
  rd.nf = static_cast<int>((static_cast<long long>(N) - 1) / hw) + 1;
  rd.h = r->height;
  const long long entries = static_cast<long long>(rd.nf) * r->pairs_t + static_cast<long long>(r->height) * r->pairs_h +
                            static_cast<long long>(r->width) * r->pairs_w;
  rd.compact = entries <= sv::kRopeSmemEntries ? static_cast<int>(entries) : 0;
  return SV_OK;
}

}  // namespace

namespace sv {
sv_status set_last_error(sv_status status, const char* msg) {
  g_last_error = msg;
  return status;
}
}  // namespace sv

extern "C" {

size_t sv_workspace_bytes(sv_op op, int B, int H, int N, int D, int block_len, sv_dtype dt) {
  if (op != SV_OP_BLOCK_CAUSAL_ATTN) block_len = N;
  if (op < SV_OP_LINATTN_FWD || op > SV_OP_CACHE_STEP) {
    fail(SV_ERR_INVALID_ARG, "unknown op %d", (int)op);
    return 0;
  }
  if (check_sizes(B, H, N, D, block_len, dt) != SV_OK) return 0;
  DevInfo di;
  if (device_info(di, false) != SV_OK) return 0;
  Geom g;
  if (geom_for(g, B, H, N, D, block_len, di.sm_count) != SV_OK) return 0;
  return ws_layout(g, dt, op != SV_OP_BLOCK_STATE_UPDATE).total;
}

sv_status sv_workspace_init(void* ws, size_t ws_bytes, sv_stream_t stream) {
  if (ws == nullptr || ws_bytes < static_cast<size_t>(sv::kHeaderBytes))
    return fail(SV_ERR_INVALID_ARG, "workspace is NULL or smaller than %d bytes", sv::kHeaderBytes);
  // all of it: the status word, the launch sequence number and the inter-CTA flags start at zero
  cudaError_t e = cudaMemsetAsync(ws, 0, ws_bytes, reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync(workspace)");
  return SV_OK;
}

sv_status sv_workspace_set_mirror(void* ws, size_t ws_bytes, uint32_t* host_word, sv_stream_t stream) {
  if (ws == nullptr || ws_bytes < static_cast<size_t>(sv::kHeaderBytes) || !aligned(ws, 256))
    return fail(SV_ERR_INVALID_ARG, "workspace is NULL, not 256-byte aligned or smaller than %d bytes",
                sv::kHeaderBytes);
  void* dptr = nullptr;
  if (host_word != nullptr) {
    if (!aligned(host_word, 4)) return fail(SV_ERR_INVALID_ARG, "host_word is not 4-byte aligned");
    const cudaError_t e = cudaHostGetDevicePointer(&dptr, host_word, 0);
    if (e != cudaSuccess || dptr == nullptr) {
      (void)cudaGetLastError();
      return fail(SV_ERR_INVALID_ARG, "host_word is not page-locked host memory the device can write (%s)",
                  cudaGetErrorName(e));
    }
  }
  // a pageable source is staged by the runtime before cudaMemcpyAsync returns
  const uint64_t addr = reinterpret_cast<uint64_t>(dptr);
  cudaError_t e = cudaMemcpyAsync(static_cast<uint8_t*>(ws) + 4 * sv::kMirrorWord, &addr, sizeof(addr),
                                  cudaMemcpyHostToDevice, reinterpret_cast<cudaStream_t>(stream));
  if (e == cudaSuccess) e = cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "writing the mirror address into the workspace header");
  return SV_OK;
}

sv_status sv_device_status(void* ws, sv_stream_t stream, uint32_t* code) {
  if (ws == nullptr) return fail(SV_ERR_INVALID_ARG, "workspace is NULL");
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
  uint32_t word = 0;
  e = cudaMemcpyAsync(&word, ws, sizeof(word), cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_fail(e, "reading the status word");
  if (code != nullptr) *code = word;
  if (word == 0) return SV_OK;
  e = cudaMemsetAsync(ws, 0, sizeof(word), s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_fail(e, "clearing the status word");
  return fail(SV_ERR_TIMEOUT, "a kernel's bounded wait expired (status word 0x%08x)", word);
}

sv_status sv_linattn_fwd(const void* q, const void* k, const void* v, void* o, int B, int H, int N, int D,
                         sv_dtype dt, float eps, void* ws, size_t ws_bytes, sv_stream_t stream) {
  return run_forward(q, k, v, o, B, H, N, D, N, dt, eps, nullptr, nullptr, nullptr, nullptr, ws, ws_bytes,
                     reinterpret_cast<cudaStream_t>(stream));
}

sv_status sv_block_causal_attn(const void* q, const void* k, const void* v, void* o, int B, int H, int N, int D,
                               int block_len, sv_dtype dt, float eps, const float* S_in, const float* z_in,
                               float* S_out, float* z_out, void* ws, size_t ws_bytes, sv_stream_t stream) {
  return run_forward(q, k, v, o, B, H, N, D, block_len, dt, eps, S_in, z_in, S_out, z_out, ws, ws_bytes,
                     reinterpret_cast<cudaStream_t>(stream));
}

sv_status sv_cache_step(const void* q, const void* k, const void* v, void* o, int B, int H, int N, int D,
                        sv_dtype dt, float eps, float* S, float* z, int commit, void* ws, size_t ws_bytes,
                        sv_stream_t stream) {
  SV_TRY(check_cache("S", S, true));
  SV_TRY(check_cache("z", z, true));
  return run_forward(q, k, v, o, B, H, N, D, N, dt, eps, S, z, commit ? S : nullptr, commit ? z : nullptr, ws,
                     ws_bytes, reinterpret_cast<cudaStream_t>(stream));
}

size_t sv_rope3d_table_bytes(int frames, int height, int width, int D) {
  if (check_rope_grid(frames, height, width, D) != SV_OK) return 0;
  return (static_cast<size_t>(frames) + height + width) * static_cast<size_t>(D / 2) * 8;
}

sv_status sv_rope3d_table(float* table, size_t table_bytes, int frames, int height, int width, int D, int pairs_t,
                          int pairs_h, int pairs_w, float base, sv_stream_t stream) {
  SV_TRY(check_rope_grid(frames, height, width, D));
  SV_TRY(check_rope_pairs(D, pairs_t, pairs_h, pairs_w));
  if (!std::isfinite(base) || base <= 1.f) return fail(SV_ERR_INVALID_ARG, "rope base must be finite and > 1");
  if (table == nullptr || !aligned(table, 16)) return fail(SV_ERR_INVALID_ARG, "table is NULL or not 16-byte aligned");
  const size_t need = sv_rope3d_table_bytes(frames, height, width, D);
  if (table_bytes < need) return fail(SV_ERR_INVALID_ARG, "table_bytes=%zu < %zu", table_bytes, need);
  DevInfo di;
  SV_TRY(device_info(di, false));
  const cudaError_t e = sv::launch_rope_table(reinterpret_cast<float2*>(table), frames, height, width, D / 2, pairs_t,
                                              pairs_h, pairs_w, static_cast<double>(base),
                                              reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "rope table kernel launch");
  return SV_OK;
}

sv_status sv_block_causal_attn_rope(const void* q, const void* k, const void* v, void* o, int B, int H, int N, int D,
                                    int block_len, sv_dtype dt, float eps, const float* S_in, const float* z_in,
                                    float* S_out, float* z_out, const sv_rope3d* rope, void* ws, size_t ws_bytes,
                                    sv_stream_t stream) {
  SV_TRY(check_sizes(B, H, N, D, block_len, dt));
  sv::RopeDev rd;
  SV_TRY(rope_for(rd, rope, N, D));
  return run_forward(q, k, v, o, B, H, N, D, block_len, dt, eps, S_in, z_in, S_out, z_out, ws, ws_bytes,
                     reinterpret_cast<cudaStream_t>(stream), &rd);
}

sv_status sv_block_state_update(const void* k, const void* v, int B, int H, int N, int D, sv_dtype dt, float* S,
                                float* z, void* ws, size_t ws_bytes, sv_stream_t stream) {
  SV_TRY(check_sizes(B, H, N, D, N, dt));
  SV_TRY(check_io("k", k));
  SV_TRY(check_io("v", v));
  SV_TRY(check_cache("S", S, true));
  SV_TRY(check_cache("z", z, true));
  DevInfo di;
  SV_TRY(device_info(di, true));
  Geom g;
  SV_TRY(geom_for(g, B, H, N, D, N, di.sm_count));
  const WsLayout lay = ws_layout(g, dt, false);
  SV_TRY(check_ws(ws, ws_bytes, lay.total));
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  uint8_t* wsb = static_cast<uint8_t*>(ws);
  uint32_t* status = reinterpret_cast<uint32_t*>(wsb);
  float* partials = reinterpret_cast<float*>(wsb + lay.partials);
  int2* segcta = reinterpret_cast<int2*>(wsb + lay.segcta);
  cudaError_t e;
  if (dt == SV_BF16) {
    sv::BlockMaps mk, mv;
    SV_TRY(make_block_maps(mk, k, g, sv::kTile));
    SV_TRY(make_block_maps(mv, v, g, sv::kTile));
    e = sv::launch_state_bf16(mk, mv, g, partials, segcta, status, s);
  } else {
    e = sv::launch_state_f32(static_cast<const float*>(k), static_cast<const float*>(v), g, partials, segcta,
                             status, s);
  }
  if (e != cudaSuccess) return cuda_fail(e, "state kernel launch");
  e = sv::launch_scan(partials, segcta, g, S, z, S, z, nullptr, nullptr, status + 6, s);
  if (e != cudaSuccess) return cuda_fail(e, "scan kernel launch");
  return SV_OK;
}

sv_status sv_profile_events(void* const* events, int n) {
  if (events == nullptr) {
    for (auto& ev : g_prof_events) ev = nullptr;
    return SV_OK;
  }
  if (n != 4) return fail(SV_ERR_INVALID_ARG, "sv_profile_events needs 4 events, got %d", n);
  for (int i = 0; i < 4; ++i) g_prof_events[i] = static_cast<cudaEvent_t>(events[i]);
  return SV_OK;
}

const char* sv_last_error(void) { return g_last_error.c_str(); }

int sv_version(void) { return 100; }

}  // extern "C"
