// C ABI of the MoE layer library (declared in include/moe.h): argument checks, workspace
// layout, path choice and kernel launches.  Host code only; kernels live in the .cuh files.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <climits>
#include <cmath>
#include <cstdint>
#include <cstdlib>
#include <cstring>
#include <new>
#include <utility>
#include <vector>

#include "moe.h"
#include "common.cuh"
#include "route.cuh"
#include "stream.cuh"
#include "stream_mx.cuh"
#include "gemm.cuh"
#include "gemm_wide.cuh"
#include "expert_gemm.cuh"
#include "expert_gemm_mx.cuh"
#include "ep.cuh"

using namespace moe;

namespace {

constexpr int kMaxE = 256;
constexpr int kMaxHI = 16384;
constexpr int kMaxT = 1 << 20;
// Dispatch defaults until moe_tune measures them.  The weight-streaming family runs only in calls
// so small that expert tiles could not fill the GPU (see default_stream_T); there it takes the
// experts with up to one streaming chunk of rows.  Experts with up to one expert tile of rows take
// the expert-tile kernel, more rows the row-tile grouped GEMM.
constexpr int kDefaultStreamRows = 16;
// Boundary between expert tiles and row tiles, in rows per expert: at a mean load of 128 rows the
// 256-row expert tiles beat the row tiles (20b layer 452 vs 461 us at 1024 tokens, 120b layer
// 1711 vs 1976 us at 4096), at 256 rows the row tiles win (593 vs 632 us; 2565 vs 2707 us).
constexpr int kDefaultTileRows = 192;
// MXFP4: streaming for calls of at most this many tokens (20b layer, rotating token batches:
// streaming 283 vs tiles 308 us at 160 tokens, a tie at 192, tiles 336 vs 390 us at 256)
constexpr int kMxStreamT = 176;
constexpr int kMaxKernelsPerCall = 12;

moe_status static_scratch_address(void** out);  // defined beside the array, at the end

// Profiled kernel kinds (moe_profile_end): one per kernel family and projection.
enum Kind { kKindRouter = 0, kKindRouteFin = 1, kKindGather = 2, kKindGateUp = 3,
            kKindDown = 4, kKindConvert = 5, kKindGateUpTile = 6, kKindDownTile = 7,
            kKindGateUpGemm = 8, kKindDownGemm = 9 };

}  // namespace

// A TMA descriptor for one tensor, re-encoded when the pointer or the row count changes.
struct MapCache {
  const void* ptr = nullptr;
  uint64_t rows = 0;
  CUtensorMap map;
};

// Grouped-GEMM configurations (CTA pairs): <mode, shared-memory stages>.
constexpr int kGemmStages = 6;
#define MOE_GEMM_GATE_UP 0, kGemmStages
#define MOE_GEMM_DOWN 1, kGemmStages
constexpr int kGemmChunkRows = 2 * kGemmBM;  // rows per tile: one 256-row MMA over a CTA pair

struct moe_ctx {
  int E, H, I, k;
  MapCache gate_up_stream, down_stream, gate_up_gemm, down_gemm, x_perm_map, h_map;
  MapCache et_x_map, et_h_map;  // activation rows for the expert-tile kernel (16-row boxes)
  MapCache gu_codes, gu_scales, dn_codes, dn_scales;  // MXFP4 weights (streaming path)
  MapCache gu_codes_t, gu_scales_t, dn_codes_t, dn_scales_t;  // MXFP4 weights (expert tiles)
  int device = 0;
  int num_sms = 148;
  moe_path path = MOE_PATH_AUTO;
  int stream_T = 0;                      // AUTO streams only in calls of at most this many tokens
  int stream_rows = kDefaultStreamRows;  // ... the experts with at most this many rows
  int tile_rows = kDefaultTileRows;      // experts up to this many rows take expert tiles; more:
                                         // row tiles (moved across by the call's counts: snap)
  bool per_expert = false;               // expert tiles and row tiles side by side in a call
  int tile_n = 0;                        // rows per expert tile: 0 by the call's mean load, 128, 256
  bool wide_rows = false;                // row tiles 256 x 512 (two MMAs per K step) or 256 x 256
  uint32_t* d_status = nullptr;
  cudaStream_t aux = nullptr;            // second stream for a call whose families fork
  cudaEvent_t ev_fork = nullptr, ev_join = nullptr;
  void* static_scratch = nullptr;  // device address of the routing scratch array (moe_route_static)
  uint64_t launches = 0;
  // profiling
  int prof_max = 0, prof_calls = 0;
  std::vector<cudaEvent_t> ev;   // pairs
  std::vector<int> ev_kind;
  size_t ev_used = 0;
  bool in_call = false;
};

namespace {

inline size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

struct Carver {
  size_t cur = 0;
  size_t take(size_t bytes) {
    const size_t at = cur;
    cur = align_up(cur + bytes, 256);
    return at;
  }
};

bool shape_ok(int E, int H, int I, int k) {
  return E >= 1 && E <= kMaxE && k >= 1 && k <= E && H >= 64 && H <= kMaxHI && H % 64 == 0 &&
         I >= 64 && I <= kMaxHI && I % 64 == 0;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static bool tried = false;
  if (!tried) {
    tried = true;
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    else
      cudaGetLastError();
  }
  return fn;
}

// 2D bf16 view [rows, cols] (row-major, contiguous) with a [box_rows, box_cols] box.
// promote_256: let L2 fill 256-byte lines for each 128-byte box row (good when the neighbouring
// 128 bytes are read by the same tile soon after; wasteful when they belong to another tile).
bool encode_2d(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols, uint32_t box_rows,
               uint32_t box_cols, CUtensorMapSwizzle swizzle, bool promote_256) {
  auto enc = tensor_map_encoder();
  if (!enc) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * 2};
  cuuint32_t box[2] = {box_cols, box_rows};
  cuuint32_t estr[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle,
             promote_256 ? CU_TENSOR_MAP_L2_PROMOTION_L2_256B : CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 2D map over a byte tensor [rows, cols] (cols bytes per row, a multiple of 16).
bool encode_2d_u8(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols,
                  uint32_t box_rows, uint32_t box_cols, CUtensorMapSwizzle swizzle) {
  auto enc = tensor_map_encoder();
  if (!enc) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols};
  cuuint32_t box[2] = {box_cols, box_rows};
  cuuint32_t estr[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

const CUtensorMap* cached_map_u8(MapCache& mc, const void* ptr, uint64_t rows, uint64_t cols,
                                 uint32_t box_rows, uint32_t box_cols,
                                 CUtensorMapSwizzle swizzle) {
  if (mc.ptr != ptr || mc.rows != rows) {
    mc.ptr = nullptr;
    if (!encode_2d_u8(&mc.map, ptr, rows, cols, box_rows, box_cols, swizzle)) return nullptr;
    mc.ptr = ptr;
    mc.rows = rows;
  }
  return &mc.map;
}

const CUtensorMap* cached_map(MapCache& mc, const void* ptr, uint64_t rows, uint64_t cols,
                              uint32_t box_rows, uint32_t box_cols, bool promote_256 = true) {
  if (mc.ptr != ptr || mc.rows != rows) {
    mc.ptr = nullptr;
    if (!encode_2d(&mc.map, ptr, rows, cols, box_rows, box_cols, CU_TENSOR_MAP_SWIZZLE_128B,
                   promote_256))
      return nullptr;
    mc.ptr = ptr;
    mc.rows = rows;
  }
  return &mc.map;
}

// ---- workspace layouts ---------------------------------------------------------------
struct RouteTmp {
  size_t partial = 0, block_counts = 0, totals = 0;
  int splits = 1, kc_per_split = 0;  // large-T router: hidden-dimension slices per token block
};

constexpr int kTopkMaxSlices = 8;  // partial-logit slices topk_from_partials sums itself

// Large-T router split: enough (token block, hidden slice) blocks for about two per SM, at most
// kTopkMaxSlices slices (so the top-k kernel sums them without a separate pass).
void router_split(const moe_ctx* c, int T, int* splits, int* kc_per_split) {
  const int NB = (T + kRouterTcTokens - 1) / kRouterTcTokens;
  const int nk = c->H / kRouterHSlice;
  int S = std::max(1, std::min(std::min(nk, kTopkMaxSlices), (2 * c->num_sms + NB - 1) / NB));
  const int kcps = (nk + S - 1) / S;
  *kc_per_split = kcps;
  *splits = (nk + kcps - 1) / kcps;
}

// allow_split = false keeps the large-T router unsplit (the fixed-scratch routing entry point).
// fused: the streaming gate/up kernel finishes the routing (StreamRoute).  Its CTAs sum the
// slices cheaply, so each router block takes only as many 64-row chunks as its ring holds (all
// in flight at once: two for more than 64 experts, whose ring has two stages); the finalize
// kernel sums them in one block, so without fusion the blocks take kSmallTChunks chunks.
RouteTmp carve_route_tmp(Carver& cv, const moe_ctx* c, int T, bool allow_split = true,
                         bool fused = false) {
  RouteTmp r;
  if (T <= kSmallT) {
    // partial logits of each group of kc 64-row slices of W_router
    const int nk = c->H / kRouterHSlice;
    const int kc = fused && c->E > 64 ? RouterTcCfg<16>::kStages : kSmallTChunks;
    r.kc_per_split = kc;
    r.splits = (nk + kc - 1) / kc;
    r.partial = cv.take(sizeof(float) * (size_t)r.splits * T * c->E);
  } else {
    const size_t NB = (T + kRouterTcTokens - 1) / kRouterTcTokens;
    r.block_counts = cv.take(sizeof(int32_t) * NB * c->E);
    r.totals = cv.take(sizeof(int32_t) * c->E);
    r.kc_per_split = c->H / kRouterHSlice;
    if (allow_split) {
      router_split(c, T, &r.splits, &r.kc_per_split);
      if (r.splits > 1) r.partial = cv.take(sizeof(float) * (size_t)r.splits * T * c->E);
    }
  }
  return r;
}

// ---- dispatch -------------------------------------------------------------------------
// Three kernel families multiply an expert's rows, chosen on the device from the call's row
// counts (the routing kernels build one work list per family):
//   stream  rows <= stream_rows:      weight streaming on mma.sync, stream-K split (decode)
//   tile    up to tile_rows:          tcgen05 expert tiles, weights as the M operand
//   gemm    more than tile_rows:      2-SM tcgen05 row tiles (prefill, long sequences)
// By default (one_tc) the experts past the streaming bound then all take expert tiles or all
// take row tiles, by their mean count; per_expert keeps each expert's own choice.  The host
// only decides which families may receive rows: an expert holds at most T rows (a token picks
// an expert at most once), so families above T are not launched.
enum Family { kFamStream = 0, kFamTile = 1, kFamGemm = 2, kFamilies = 3 };
constexpr int kFamChunkRows[kFamilies] = {kStreamRB, kEtRows, kGemmChunkRows};
constexpr int kEtWideRows = 256;   // rows per entry of the 256-row expert tiles

struct Plan {
  bool has[kFamilies] = {false, false, false};
  int max_count[kFamilies] = {0, 0, 0};   // family f takes counts in (max_count[f-1], max_count[f]]
  bool snap = false;                      // the call's counts may move experts across a boundary
  bool one_tc = false;                    // expert tiles or row tiles, not both, in one call
  int tile_entry_rows = kEtRows;          // rows per expert-tile entry: 128 or 256 (bf16 only)
  bool fused_route = false;               // the streaming gate/up kernel finishes the routing
  int chunk_rows(int f) const { return f == kFamTile ? tile_entry_rows : kFamChunkRows[f]; }
  int min_count(int f) const {
    int m = 0;
    for (int g = 0; g < f; ++g)
      if (has[g]) m = max_count[g];
    return m;
  }
};

Plan make_plan(const moe_ctx* c, int T, bool mx, moe_path path) {
  Plan p;
  auto only = [&](int f) {
    p.has[f] = true;
    p.max_count[f] = INT_MAX;
  };
  if (mx) {  // MXFP4 experts: weight streaming or expert tiles (no MXFP4 row-tile GEMM)
    if (path == MOE_PATH_STREAM) only(kFamStream);
    else if (path == MOE_PATH_TILE || path == MOE_PATH_GEMM) only(kFamTile);
    else only(T <= kMxStreamT ? kFamStream : kFamTile);
    return p;
  }
  switch (path) {
    case MOE_PATH_STREAM: only(kFamStream); break;
    case MOE_PATH_GEMM: only(kFamGemm); break;
    case MOE_PATH_TILE: only(kFamTile); break;
    default: {
      const bool s_on = T <= c->stream_T && c->stream_rows > 0;
      const int lo = s_on ? c->stream_rows : 0;
      // expert tiles are left out when the mean load is far above their range: an expert
      // that small would be a rare outlier, and row tiles handle it (padded)
      const long long mean = (long long)T * c->k / c->E;
      p.has[kFamStream] = s_on;
      p.has[kFamTile] = T > lo && c->tile_rows > lo && mean < 8LL * c->tile_rows;
      p.has[kFamGemm] = T > std::max(lo, c->tile_rows);
      // one family per call: a mean load of tile_rows over all E experts already puts the call
      // on row tiles (the touched experts' mean is at least that), so no expert-tile launch
      if (!c->per_expert && !s_on && p.has[kFamGemm] &&
          (long long)T * c->k >= (long long)c->tile_rows * c->E)
        p.has[kFamTile] = false;
      p.max_count[kFamStream] = (p.has[kFamTile] || p.has[kFamGemm]) ? c->stream_rows : INT_MAX;
      p.max_count[kFamTile] = p.has[kFamGemm] ? c->tile_rows : INT_MAX;
      p.max_count[kFamGemm] = INT_MAX;
      p.snap = true;
      p.one_tc = !c->per_expert && p.has[kFamTile] && p.has[kFamGemm];
    }
  }
  // bf16 expert tiles of 256 rows when the call's mean load reaches 128 rows per expert
  const bool wide = c->tile_n == 256 ||
                    (c->tile_n == 0 && (long long)T * c->k >= (long long)kEtRows * c->E);
  if (p.has[kFamTile] && wide) p.tile_entry_rows = kEtWideRows;
  // a few tokens on the streaming family alone: its gate/up kernel finishes the routing
  p.fused_route = p.has[kFamStream] && !p.has[kFamTile] && !p.has[kFamGemm] &&
                  T <= kFusedRouteT && (long long)T * c->k <= kFusedRouteRows && T <= kSmallT;
  return p;
}

// Largest T up to which AUTO streams by default: while the expert tiles of the experts T tokens
// are expected to touch (E * (1 - (1 - k/E)^T), uniform routing) fill less than two waves of the
// GPU's SMs, or fill their last wave to less than 85 %.  A tile wave that is mostly empty costs
// as much as a full one, while the stream-K split balances any number of experts.  Measured on the
// 20b and 120b layers (rotating token batches): streaming wins at 4 tokens (2.05 and 2.35 waves of
// tiles) and, on the 20b layer, at 5 (2.43 waves); the 120b tiles win from 5 tokens (2.9 waves).
int default_stream_T(const moe_ctx* c) {
  const double tiles_per_expert = (double)((c->I + kEtM - 1) / kEtM);
  // a layer whose tiles cannot fill two waves even with every expert touched always streams
  if (c->E * tiles_per_expert < 2.0 * c->num_sms) return kMaxT;
  const double miss = 1.0 - (double)c->k / c->E;
  int T = 0;
  double miss_T = 1.0;  // miss^T: probability that a given expert is not touched
  while (T < kMaxT) {
    miss_T *= miss;
    const double waves = c->E * (1.0 - miss_T) * tiles_per_expert / c->num_sms;
    if (!(waves < 2.0 || waves / std::ceil(waves) < 0.85)) break;
    ++T;
    if (miss_T < 1e-6) break;  // the touched count no longer grows
  }
  return T;
}

// Rows an expert of family f can hold in a call: its upper threshold, twice that when the call's
// counts may move neighbours in (snap), unbounded for the last family and for expert tiles that
// may take every non-streamed expert (one_tc).
long long family_row_bound(const Plan& p, int f) {
  if (p.max_count[f] == INT_MAX || (p.one_tc && f == kFamTile)) return LLONG_MAX;
  return (long long)p.max_count[f] * (p.snap ? 2 : 1);
}

// Work-list entries family f can need for T tokens.
int max_chunks(const moe_ctx* c, int T, const Plan& p, int f) {
  const long long R = (long long)T * c->k, rows = p.chunk_rows(f);
  long long n = R / rows + c->E;
  const long long b = family_row_bound(p, f);
  if (b != LLONG_MAX) n = std::min(n, (long long)c->E * ((b + rows - 1) / rows));
  return (int)n;
}

struct Layout {
  size_t topk_idx, topk_w, inv_perm, perm, row_w, offsets;
  size_t sched[kFamilies], chunks[kFamilies];
  size_t done, acc, h, x16, x_perm;
  size_t acc_floats;
  int n_done;
  RouteTmp rt;
  size_t total;
};

Layout make_layout(const moe_ctx* c, int T, const Plan& p, bool mx) {
  Layout L{};
  Carver cv;
  const size_t R = (size_t)T * c->k;
  L.topk_idx = cv.take(4 * R);
  L.topk_w = cv.take(4 * R);
  L.inv_perm = cv.take(4 * R);
  L.perm = cv.take(4 * R);
  L.row_w = cv.take(4 * R);
  L.offsets = cv.take(4 * (size_t)(c->E + 1));
  for (int f = 0; f < kFamilies; ++f)
    if (p.has[f]) {
      L.sched[f] = cv.take(16);
      L.chunks[f] = cv.take(16 * (size_t)max_chunks(c, T, p, f));
    }
  if (p.has[kFamStream]) {
    const int n = max_chunks(c, T, p, kFamStream);
    // one completion counter per (chunk, column tile); the MXFP4 kernels' tiles are narrower
    const int tile_cols = std::min(kStreamCols, kMxTileCols);
    L.n_done = n * ((c->I + tile_cols - 1) / tile_cols);
    L.done = cv.take(4 * (size_t)L.n_done);
    // split-K sums of the streaming family's rows (each entry carries its rows' first index)
    const long long sb = family_row_bound(p, kFamStream);
    const long long srows = sb == LLONG_MAX ? (long long)R : std::min((long long)R, c->E * sb);
    L.acc_floats = (size_t)srows * 2 * c->I;
    L.acc = cv.take(sizeof(float) * L.acc_floats);
  }
  L.h = cv.take(2 * R * c->I);
  if (mx) L.x16 = cv.take(2 * (size_t)T * c->H);  // the layer input in f16
  if (p.has[kFamTile] || p.has[kFamGemm]) L.x_perm = cv.take(2 * R * c->H);
  L.rt = carve_route_tmp(cv, c, T, true, p.fused_route);
  L.total = cv.cur;
  return L;
}

// Workspace of the expert half alone (moe_experts): R received rows in S*E segments.
Layout make_expert_layout(const moe_ctx* c, int R, int S, const Plan& p) {
  Layout L{};
  Carver cv;
  for (int f = 0; f < kFamilies; ++f)
    if (p.has[f]) {
      const long long rows = p.chunk_rows(f), segs = (long long)S * c->E;
      long long n = R / rows + segs;
      const long long b = family_row_bound(p, f);
      if (b != LLONG_MAX)  // every expert's segments together hold <= b rows
        n = std::min(n, (long long)c->E * ((b + rows - 1) / rows + S));
      L.sched[f] = cv.take(16);
      L.chunks[f] = cv.take(16 * (size_t)n);
      if (f == kFamStream) {
        const int tile_cols = std::min(kStreamCols, kMxTileCols);
        L.n_done = (int)(n * ((c->I + tile_cols - 1) / tile_cols));
        L.done = cv.take(4 * (size_t)L.n_done);
        const long long srows = b == LLONG_MAX ? (long long)R : std::min((long long)R, c->E * b);
        L.acc_floats = (size_t)srows * 2 * c->I;
        L.acc = cv.take(sizeof(float) * L.acc_floats);
      }
    }
  L.h = cv.take(2 * (size_t)R * c->I);
  L.perm = cv.take(4 * (size_t)R);  // identity row map of the results
  L.total = cv.cur;
  return L;
}

size_t route_ws_bytes(const moe_ctx* c, int T, bool allow_split = true) {
  Carver cv;
  cv.take(16);  // sched
  carve_route_tmp(cv, c, T, allow_split);
  return cv.cur;
}

// ---- launches ------------------------------------------------------------------------
// Launch with programmatic stream serialisation: the kernel may start (and run the part before
// its pdl_wait()) while the previous kernel on the stream finishes.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t st, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

template <typename F>
moe_status launch(moe_ctx* c, int kind, cudaStream_t st, F&& f) {
  const bool prof = c->prof_max > 0 && c->in_call && c->ev_used + 2 <= c->ev.size();
  if (prof) cudaEventRecord(c->ev[c->ev_used], st);
  cudaError_t err = f();
  if (err == cudaSuccess) err = cudaGetLastError();
  else cudaGetLastError();
  if (prof) {
    cudaEventRecord(c->ev[c->ev_used + 1], st);
    c->ev_kind[c->ev_used / 2] = kind;
    c->ev_used += 2;
  }
  if (err != cudaSuccess) return MOE_ERR_CUDA;
  ++c->launches;
  return MOE_OK;
}

#define MOE_TRY(expr)                    \
  do {                                   \
    const moe_status _s = (expr);        \
    if (_s != MOE_OK) return _s;         \
  } while (0)

template <int NT8>
cudaError_t launch_router_tc(int NB, cudaStream_t st, const uint16_t* x, const uint16_t* Wr,
                             const float* b, int T, int H, int E, int k, const RouteOut& o,
                             int32_t* block_counts, float4* zero4, size_t n_zero4,
                             const RouteTmp& rt, float* partial) {
  return launch_pdl(router_topk_kernel<NT8>, dim3(NB, rt.splits), dim3(128),
                    RouterTcCfg<NT8>::smem(k), st, x, Wr, b, T, H, E, k, o.topk_idx, o.topk_w,
                    block_counts, zero4, n_zero4, rt.kc_per_split, partial);
}

template <int NT8>
cudaError_t launch_router_small(cudaStream_t st, const uint16_t* x, const uint16_t* Wr, int T,
                                int H, int E, float4* zero4, size_t n_zero4, const RouteTmp& rt,
                                float* partial) {
  return launch_pdl(router_partial_small_kernel<NT8>, dim3(1, rt.splits), dim3(128),
                    (size_t)RouterSmallCfg<NT8>::kSmem, st, x, Wr, T, H, E, zero4, n_zero4,
                    rt.kc_per_split, partial);
}

// Routing chain.  zero4/n_zero4: a float scratch region the router kernel zero-fills.
// finalize = false (T <= kSmallT only): stop after the partial logits; the streaming gate/up
// kernel finishes the routing (StreamRoute).
moe_status launch_route(moe_ctx* c, int T, const uint16_t* x, const uint16_t* Wr,
                        const float* b, const RouteOut& o, uint8_t* ws, const RouteTmp& rt,
                        cudaStream_t st, float* zero = nullptr, size_t n_zero_floats = 0,
                        bool finalize = true) {
  float4* zero4 = reinterpret_cast<float4*>(zero);
  const size_t n_zero4 = n_zero_floats / 4;
  const int E = c->E, H = c->H, k = c->k;
  const int nt8 = (E + 7) / 8;
  if (T <= kSmallT) {
    // one token block, the hidden dimension split over rt.splits blocks: partial logits on the
    // tensor cores, then one block finishes the routing
    float* partial = reinterpret_cast<float*>(ws + rt.partial);
    MOE_TRY(launch(c, kKindRouter, st, [&] {
      if (T <= kRouterSmallT) {  // small enough to run beside the previous call's down kernel
        if (nt8 <= 1) return launch_router_small<1>(st, x, Wr, T, H, E, zero4, n_zero4, rt, partial);
        if (nt8 <= 2) return launch_router_small<2>(st, x, Wr, T, H, E, zero4, n_zero4, rt, partial);
        if (nt8 <= 4) return launch_router_small<4>(st, x, Wr, T, H, E, zero4, n_zero4, rt, partial);
        if (nt8 <= 8) return launch_router_small<8>(st, x, Wr, T, H, E, zero4, n_zero4, rt, partial);
        if (nt8 <= 16) return launch_router_small<16>(st, x, Wr, T, H, E, zero4, n_zero4, rt, partial);
        return launch_router_small<32>(st, x, Wr, T, H, E, zero4, n_zero4, rt, partial);
      }
      if (nt8 <= 1) return launch_router_tc<1>(1, st, x, Wr, b, T, H, E, k, o, nullptr, zero4, n_zero4, rt, partial);
      if (nt8 <= 2) return launch_router_tc<2>(1, st, x, Wr, b, T, H, E, k, o, nullptr, zero4, n_zero4, rt, partial);
      if (nt8 <= 4) return launch_router_tc<4>(1, st, x, Wr, b, T, H, E, k, o, nullptr, zero4, n_zero4, rt, partial);
      if (nt8 <= 8) return launch_router_tc<8>(1, st, x, Wr, b, T, H, E, k, o, nullptr, zero4, n_zero4, rt, partial);
      if (nt8 <= 16) return launch_router_tc<16>(1, st, x, Wr, b, T, H, E, k, o, nullptr, zero4, n_zero4, rt, partial);
      return launch_router_tc<32>(1, st, x, Wr, b, T, H, E, k, o, nullptr, zero4, n_zero4, rt, partial);
    }));
    if (!finalize) return MOE_OK;
    const size_t smem_f = (size_t)T * E * 4 + (size_t)T * k * 4 + (size_t)T * 8 * 4 +
                          (256 + 257 + 768) * 4;
    MOE_TRY(launch(c, kKindRouteFin, st, [&] {
      return launch_pdl(route_small_finalize_kernel, dim3(1), dim3(1024), smem_f, st,
                        (const float*)partial, rt.splits, b, T, E, k, o);
    }));
    return MOE_OK;
  }
  const int NB = (T + kRouterTcTokens - 1) / kRouterTcTokens;
  int32_t* block_counts = reinterpret_cast<int32_t*>(ws + rt.block_counts);
  int32_t* totals = reinterpret_cast<int32_t*>(ws + rt.totals);
  float* split_partial = rt.splits > 1 ? reinterpret_cast<float*>(ws + rt.partial) : nullptr;
  MOE_TRY(launch(c, kKindRouter, st, [&] {
    if (nt8 <= 1) return launch_router_tc<1>(NB, st, x, Wr, b, T, H, E, k, o, block_counts, zero4, n_zero4, rt, split_partial);
    if (nt8 <= 2) return launch_router_tc<2>(NB, st, x, Wr, b, T, H, E, k, o, block_counts, zero4, n_zero4, rt, split_partial);
    if (nt8 <= 4) return launch_router_tc<4>(NB, st, x, Wr, b, T, H, E, k, o, block_counts, zero4, n_zero4, rt, split_partial);
    if (nt8 <= 8) return launch_router_tc<8>(NB, st, x, Wr, b, T, H, E, k, o, block_counts, zero4, n_zero4, rt, split_partial);
    if (nt8 <= 16) return launch_router_tc<16>(NB, st, x, Wr, b, T, H, E, k, o, block_counts, zero4, n_zero4, rt, split_partial);
    return launch_router_tc<32>(NB, st, x, Wr, b, T, H, E, k, o, block_counts, zero4, n_zero4, rt, split_partial);
  }));
  if (split_partial) {
    // a few slices are summed by the top-k kernel itself; many first by a wide kernel
    const bool presum = rt.splits > kTopkMaxSlices;
    const int n = T * E;
    if (presum)
      MOE_TRY(launch(c, kKindRouter, st, [&] {
        return launch_pdl(sum_partials_kernel, dim3((n + 255) / 256), dim3(256), 0, st,
                          split_partial, rt.splits, n);
      }));
    const size_t smem_t = (size_t)kRouterTcTokens * (E + 1) * 4 + (size_t)E * 4 +
                          (size_t)kRouterTcTokens * k * 4;
    MOE_TRY(launch(c, kKindRouter, st, [&] {
      return launch_pdl(topk_from_partials_kernel, dim3(NB), dim3(128), smem_t, st,
                        (const float*)split_partial, presum ? 1 : rt.splits, b, T, E, k,
                        o.topk_idx, o.topk_w, block_counts);
    }));
  }
  MOE_TRY(launch(c, kKindRouteFin, st, [&] {
    return launch_pdl(route_scan_kernel, dim3(E), dim3(256), 0, st, block_counts, NB, E, totals);
  }));
  const size_t smem_s = (256 + 257 + 768) * 4 + (size_t)kRouterTcTokens * 8 * 4 +
                        (size_t)kRouterTcTokens * E;
  MOE_TRY(launch(c, kKindRouteFin, st, [&] {
    return launch_pdl(route_scatter_kernel, dim3(NB), dim3(256), smem_s, st,
                      (const int32_t*)o.topk_idx, (const float*)o.topk_w,
                      (const int32_t*)block_counts, (const int32_t*)totals, T, E, k, o);
  }));
  return MOE_OK;
}

bool set_smem_attrs() {
  const int big = 227 * 1024;
  bool ok = true;
  ok &= cudaFuncSetAttribute(route_small_finalize_kernel,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, big) == cudaSuccess;
  ok &= cudaFuncSetAttribute(router_topk_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             big) == cudaSuccess;
  ok &= cudaFuncSetAttribute(router_topk_kernel<2>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             big) == cudaSuccess;
  ok &= cudaFuncSetAttribute(router_topk_kernel<4>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             big) == cudaSuccess;
  ok &= cudaFuncSetAttribute(router_topk_kernel<8>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             big) == cudaSuccess;
  ok &= cudaFuncSetAttribute(router_topk_kernel<16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             big) == cudaSuccess;
  ok &= cudaFuncSetAttribute(router_topk_kernel<32>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             big) == cudaSuccess;
  ok &= cudaFuncSetAttribute(topk_from_partials_kernel,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, big) == cudaSuccess;
  ok &= cudaFuncSetAttribute(stream_gate_up_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             kGateUpSmem) == cudaSuccess;
  ok &= cudaFuncSetAttribute(stream_down_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             kDownSmem) == cudaSuccess;
  ok &= cudaFuncSetAttribute(stream_gate_up_mx_kernel,
                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                             kMxGateUpSmem) == cudaSuccess;
  ok &= cudaFuncSetAttribute(stream_down_mx_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             kMxDownSmem) == cudaSuccess;
  ok &= cudaFuncSetAttribute(grouped_gemm_2sm_kernel<MOE_GEMM_GATE_UP>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                             Gemm2Cfg<kGemmStages>::kSmem) == cudaSuccess;
  ok &= cudaFuncSetAttribute(grouped_gemm_2sm_kernel<MOE_GEMM_DOWN>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                             Gemm2Cfg<kGemmStages>::kSmem) == cudaSuccess;
  ok &= cudaFuncSetAttribute(grouped_gemm_wide_kernel<0>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                             WideCfg<0>::kSmem) == cudaSuccess;
  ok &= cudaFuncSetAttribute(grouped_gemm_wide_kernel<1>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                             WideCfg<1>::kSmem) == cudaSuccess;
  ok &= cudaFuncSetAttribute(expert_tile_kernel<0>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             kEtSmem) == cudaSuccess;
  ok &= cudaFuncSetAttribute(expert_tile_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             kEtSmem) == cudaSuccess;
  ok &= cudaFuncSetAttribute(expert_tile_kernel<0, kEtWideRows>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                             EtCfg<kEtWideRows>::kSmem) == cudaSuccess;
  ok &= cudaFuncSetAttribute(expert_tile_kernel<1, kEtWideRows>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                             EtCfg<kEtWideRows>::kSmem) == cudaSuccess;
  ok &= cudaFuncSetAttribute(expert_tile_mx_kernel<0>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, kEmxSmem) == cudaSuccess;
  ok &= cudaFuncSetAttribute(expert_tile_mx_kernel<1>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, kEmxSmem) == cudaSuccess;
  ok &= cudaFuncSetAttribute(build_segment_lists_kernel,
                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (4 * kMaxSegments + 2 * kMaxE) * 4) == cudaSuccess;
  return ok;
}

moe_status check_common(const moe_ctx* c, int T, const void* x, const void* Wr, const float* b) {
  if (!c) return MOE_ERR_ARG;
  if (T < 0 || T > kMaxT || (long long)T * c->k >= (1ll << 31)) return MOE_ERR_ARG;
  if (T == 0) return MOE_OK;
  if (!x || !Wr || !b) return MOE_ERR_ARG;
  if (!aligned16(x) || !aligned16(Wr) || !aligned16(b)) return MOE_ERR_ARG;
  return MOE_OK;
}

// MXFP4 expert weights: codes and scales of W_gate_up and W_down (null: bf16 weights).
struct MxWeights {
  const void *gu_codes, *gu_scales, *dn_codes, *dn_scales;
};

// The expert half of the layer for one plan: gate/up + SwiGLU, then down + weighted combine,
// by every kernel family in the plan, each on its own work list (found on the device).
struct ExpertIO {
  int R;                              // rows
  const uint16_t* x_tok;              // rows of the streaming family: x_tok[perm[r]]
  const int32_t* perm;                // [R] row -> row of x_tok / of out
  const uint16_t* x_perm;             // [R, H] rows in expert order (tcgen05 families), or null
  const float* row_w;                 // [R] weight of each row's result
  float* out;                         // [*, H] fp32, accumulated through perm
  size_t out_elems;                   // elements of out this phase zero-fills first
  const int4* chunks[kFamilies];
  const int32_t* sched[kFamilies];
  float* acc;                         // streaming family: split-K sums, zero on entry
  int32_t* done;                      // streaming family: completion counters, zero on entry
  uint16_t* h;                        // [R, I] SwiGLU output
  StreamRoute sr{};                   // routing finished by the streaming gate/up kernel, if set
};

moe_status expert_phase(moe_ctx* c, const Plan& p, const ExpertIO& io, const void* W_gate_up_bf16,
                        const void* W_down_bf16, const MxWeights* mx, cudaStream_t st) {
  const size_t R = (size_t)io.R;
  const int pair_grid = c->num_sms & ~1;  // whole CTA pairs
  // With more than one family the row tiles run on the handle's second stream, concurrently
  // with the other families: a family with little or no work is then off the critical path,
  // and families that share a call share the SMs.  `out` is zero-filled before the fork.
  // Expert tiles and row tiles that exclude each other (one_tc) stay on one stream.
  const bool fork = p.has[kFamGemm] && c->aux != nullptr &&
                    (p.has[kFamStream] || (p.has[kFamTile] && !p.one_tc));
  const cudaStream_t gst = fork ? c->aux : st;   // stream of the row-tile family
  // `out` is zero-filled once: before the fork, else by one gate/up kernel (the expert-tile or
  // streaming kernel before its dependency wait, while routing runs; the row-tile GEMM's epilogue
  // warps while its tensor cores run when it is the only family)
  int zero_owner = p.has[kFamTile] ? kFamTile : p.has[kFamStream] ? kFamStream : kFamGemm;
  if (fork) {
    zero_owner = -1;
    const size_t n4 = io.out_elems / 4;
    MOE_TRY(launch(c, kKindGather, st, [&] {
      return launch_pdl(zero_out_kernel, dim3(2 * c->num_sms), dim3(256), 0, st,
                        reinterpret_cast<float4*>(io.out), n4);
    }));
    if (cudaEventRecord(c->ev_fork, st) != cudaSuccess ||
        cudaStreamWaitEvent(c->aux, c->ev_fork, 0) != cudaSuccess)
      return MOE_ERR_CUDA;
  }

  // ---------------------------- gate/up projection + SwiGLU ----------------------------
  if (p.has[kFamStream]) {
    GateUpArgs ga{};
    ga.x = io.x_tok;
    ga.H = c->H;
    ga.I = c->I;
    ga.R = io.R;
    ga.perm = io.perm;
    ga.chunks = io.chunks[kFamStream];
    ga.sched = io.sched[kFamStream];
    ga.acc = io.acc;
    ga.done = io.done;
    ga.h = io.h;
    ga.out = io.out;
    ga.out_elems = zero_owner == kFamStream ? io.out_elems : 0;
    ga.status = c->d_status;
    if (mx) {
      const CUtensorMap* cm = cached_map_u8(c->gu_codes, mx->gu_codes, 2ull * c->I * c->E,
                                            (uint64_t)c->H / 2, kMxBoxRows, kMxKC / 2,
                                            CU_TENSOR_MAP_SWIZZLE_128B);
      const CUtensorMap* sm = cached_map_u8(c->gu_scales, mx->gu_scales,
                                            (uint64_t)c->E * (c->H / 32), 2ull * c->I,
                                            kMxKC / 32, kMxBoxRows, CU_TENSOR_MAP_SWIZZLE_NONE);
      if (!cm || !sm) return MOE_ERR_CUDA;
      MOE_TRY(launch(c, kKindGateUp, st, [&] {
        return launch_pdl(stream_gate_up_mx_kernel, dim3(c->num_sms), dim3(kMxThreads),
                          kMxGateUpSmem, st, ga, *cm, *sm);
      }));
    } else {
      const CUtensorMap* m = cached_map(c->gate_up_stream, W_gate_up_bf16,
                                        (uint64_t)c->E * c->H, 2ull * c->I, kGateUpKC, kBox,
                                        /*promote_256=*/false);
      if (!m) return MOE_ERR_CUDA;
      MOE_TRY(launch(c, kKindGateUp, st, [&] {
        return launch_pdl(stream_gate_up_kernel, dim3(c->num_sms), dim3(kStreamThreads),
                          kGateUpSmem, st, ga, io.sr, *m);
      }));
    }
  }
  const CUtensorMap* wgu = nullptr;
  const CUtensorMap* wdn = nullptr;
  if (!mx && (p.has[kFamTile] || p.has[kFamGemm])) {
    wgu = cached_map(c->gate_up_gemm, W_gate_up_bf16, (uint64_t)c->E * c->H, 2ull * c->I,
                     kGemmBK, 64);
    wdn = cached_map(c->down_gemm, W_down_bf16, (uint64_t)c->E * c->I, (uint64_t)c->H,
                     kGemmBK, 64);
    if (!wgu || !wdn) return MOE_ERR_CUDA;
  }
  if (p.has[kFamTile]) {
    const CUtensorMap* xm = cached_map(c->et_x_map, io.x_perm, R, (uint64_t)c->H, kEtRowBox, 64);
    if (!xm) return MOE_ERR_CUDA;
    const CUtensorMap *cm = nullptr, *sm = nullptr;
    if (mx) {  // codes [E*2I, H/2] in 128 x 32-byte boxes, scales [E*H/32, 2I] in 2 x 128 boxes
      cm = cached_map_u8(c->gu_codes_t, mx->gu_codes, 2ull * c->I * c->E, (uint64_t)c->H / 2,
                         kEtM, kEtBK / 2, CU_TENSOR_MAP_SWIZZLE_NONE);
      sm = cached_map_u8(c->gu_scales_t, mx->gu_scales, (uint64_t)c->E * (c->H / 32),
                         2ull * c->I, kEtBK / 32, kEtM, CU_TENSOR_MAP_SWIZZLE_NONE);
      if (!cm || !sm) return MOE_ERR_CUDA;
    }
    EtArgs e{};
    e.K = c->H;
    e.Ncols = c->I;
    e.w_rows = c->H;
    e.chunks = io.chunks[kFamTile];
    e.sched = io.sched[kFamTile];
    e.h = io.h;
    e.H = c->H;
    e.status = c->d_status;
    if (zero_owner == kFamTile) {
      e.zero4 = reinterpret_cast<float4*>(io.out);
      e.n_zero4 = io.out_elems / 4;
    }
    MOE_TRY(launch(c, kKindGateUpTile, st, [&] {
      if (mx)
        return launch_pdl(expert_tile_mx_kernel<0>, dim3(c->num_sms), dim3(kEmxThreads),
                          kEmxSmem, st, e, *cm, *sm, *xm);
      if (p.tile_entry_rows == kEtWideRows)
        return launch_pdl(expert_tile_kernel<0, kEtWideRows>, dim3(c->num_sms), dim3(kEtThreads),
                          EtCfg<kEtWideRows>::kSmem, st, e, *wgu, *xm);
      return launch_pdl(expert_tile_kernel<0>, dim3(c->num_sms), dim3(kEtThreads), kEtSmem, st,
                        e, *wgu, *xm);
    }));
  }
  if (p.has[kFamGemm]) {
    const CUtensorMap* am = cached_map(c->x_perm_map, io.x_perm, R, (uint64_t)c->H, kGemmBM, 64);
    if (!am) return MOE_ERR_CUDA;
    GemmArgs g{};
    g.K = c->H;
    g.Ncols = c->I;
    g.sub_stride = c->I;
    g.w_rows = c->H;
    g.chunks = io.chunks[kFamGemm];
    g.sched = io.sched[kFamGemm];
    g.h = io.h;
    g.H = c->H;
    g.status = c->d_status;
    // the epilogue warps zero-fill `out`, which the down projections accumulate into
    if (zero_owner == kFamGemm) {
      g.zero4 = reinterpret_cast<float4*>(io.out);
      g.n_zero4 = io.out_elems / 4;
    }
    MOE_TRY(launch(c, kKindGateUpGemm, gst, [&] {
      if (c->wide_rows)
        return launch_pdl(grouped_gemm_wide_kernel<0>, dim3(pair_grid), dim3(kWideThreads),
                          WideCfg<0>::kSmem, gst, g, *am, *wgu);
      return launch_pdl(grouped_gemm_2sm_kernel<MOE_GEMM_GATE_UP>, dim3(pair_grid),
                        dim3(kGemmThreads), Gemm2Cfg<kGemmStages>::kSmem, gst, g, *am, *wgu);
    }));
  }

  // ---------------------------- down projection + weighted combine ----------------------------
  if (p.has[kFamStream]) {
    DownArgs da{};
    da.h = io.h;
    da.H = c->H;
    da.I = c->I;
    da.R = io.R;
    da.perm = io.perm;
    da.row_w = io.row_w;
    da.chunks = io.chunks[kFamStream];
    da.sched = io.sched[kFamStream];
    da.out = io.out;
    da.status = c->d_status;
    if (mx) {
      const CUtensorMap* cm = cached_map_u8(c->dn_codes, mx->dn_codes, (uint64_t)c->H * c->E,
                                            (uint64_t)c->I / 2, kMxBoxRows, kMxKC / 2,
                                            CU_TENSOR_MAP_SWIZZLE_128B);
      const CUtensorMap* sm = cached_map_u8(c->dn_scales, mx->dn_scales,
                                            (uint64_t)c->E * (c->I / 32), (uint64_t)c->H,
                                            kMxKC / 32, kMxBoxRows, CU_TENSOR_MAP_SWIZZLE_NONE);
      if (!cm || !sm) return MOE_ERR_CUDA;
      MOE_TRY(launch(c, kKindDown, st, [&] {
        return launch_pdl(stream_down_mx_kernel, dim3(c->num_sms), dim3(kMxDnThreads),
                          kMxDownSmem, st, da, *cm, *sm);
      }));
    } else {
      const CUtensorMap* m = cached_map(c->down_stream, W_down_bf16, (uint64_t)c->E * c->I,
                                        (uint64_t)c->H, kDownKC, kBox, /*promote_256=*/false);
      if (!m) return MOE_ERR_CUDA;
      MOE_TRY(launch(c, kKindDown, st, [&] {
        return launch_pdl(stream_down_kernel, dim3(c->num_sms), dim3(kStreamThreads),
                          kDownSmem, st, da, *m);
      }));
    }
  }
  if (p.has[kFamTile]) {
    const CUtensorMap* hm = cached_map(c->et_h_map, io.h, R, (uint64_t)c->I, kEtRowBox, 64);
    if (!hm) return MOE_ERR_CUDA;
    const CUtensorMap *cm = nullptr, *sm = nullptr;
    if (mx) {  // codes [E*H, I/2], scales [E*I/32, H]
      cm = cached_map_u8(c->dn_codes_t, mx->dn_codes, (uint64_t)c->H * c->E, (uint64_t)c->I / 2,
                         kEtM, kEtBK / 2, CU_TENSOR_MAP_SWIZZLE_NONE);
      sm = cached_map_u8(c->dn_scales_t, mx->dn_scales, (uint64_t)c->E * (c->I / 32),
                         (uint64_t)c->H, kEtBK / 32, kEtM, CU_TENSOR_MAP_SWIZZLE_NONE);
      if (!cm || !sm) return MOE_ERR_CUDA;
    }
    EtArgs e{};
    e.K = c->I;
    e.Ncols = c->H;
    e.w_rows = c->I;
    e.chunks = io.chunks[kFamTile];
    e.sched = io.sched[kFamTile];
    e.perm = io.perm;
    e.row_w = io.row_w;
    e.out = io.out;
    e.H = c->H;
    e.status = c->d_status;
    MOE_TRY(launch(c, kKindDownTile, st, [&] {
      if (mx)
        return launch_pdl(expert_tile_mx_kernel<1>, dim3(c->num_sms), dim3(kEmxThreads),
                          kEmxSmem, st, e, *cm, *sm, *hm);
      if (p.tile_entry_rows == kEtWideRows)
        return launch_pdl(expert_tile_kernel<1, kEtWideRows>, dim3(c->num_sms), dim3(kEtThreads),
                          EtCfg<kEtWideRows>::kSmem, st, e, *wdn, *hm);
      return launch_pdl(expert_tile_kernel<1>, dim3(c->num_sms), dim3(kEtThreads), kEtSmem, st,
                        e, *wdn, *hm);
    }));
  }
  if (p.has[kFamGemm]) {
    const CUtensorMap* hm = cached_map(c->h_map, io.h, R, (uint64_t)c->I, kGemmBM, 64);
    if (!hm) return MOE_ERR_CUDA;
    GemmArgs d{};
    d.K = c->I;
    d.Ncols = c->H;
    d.sub_stride = 0;
    d.w_rows = c->I;
    d.chunks = io.chunks[kFamGemm];
    d.sched = io.sched[kFamGemm];
    d.perm = io.perm;
    d.row_w = io.row_w;
    d.out = io.out;
    d.H = c->H;
    d.status = c->d_status;
    MOE_TRY(launch(c, kKindDownGemm, gst, [&] {
      if (c->wide_rows)
        return launch_pdl(grouped_gemm_wide_kernel<1>, dim3(pair_grid), dim3(kWideThreads),
                          WideCfg<1>::kSmem, gst, d, *hm, *wdn);
      return launch_pdl(grouped_gemm_2sm_kernel<MOE_GEMM_DOWN>, dim3(pair_grid),
                        dim3(kGemmThreads), Gemm2Cfg<kGemmStages>::kSmem, gst, d, *hm, *wdn);
    }));
  }
  if (fork && (cudaEventRecord(c->ev_join, c->aux) != cudaSuccess ||
               cudaStreamWaitEvent(st, c->ev_join, 0) != cudaSuccess))
    return MOE_ERR_CUDA;
  return MOE_OK;
}

// Work lists of one plan inside a layout, as the routing (or segment) kernels fill them.
void plan_lists(const Plan& p, const Layout& L, uint8_t* ws, RouteOut& o, ExpertIO& io) {
  o.n_lists = 0;
  for (int f = 0; f < kFamilies; ++f) {
    io.chunks[f] = nullptr;
    io.sched[f] = nullptr;
    if (!p.has[f]) continue;
    WorkList& wl = o.wl[o.n_lists++];
    wl.chunks = reinterpret_cast<int4*>(ws + L.chunks[f]);
    wl.sched = reinterpret_cast<int32_t*>(ws + L.sched[f]);
    wl.chunk_rows = p.chunk_rows(f);
    wl.min_count = p.min_count(f);
    wl.max_count = p.max_count[f];
    io.chunks[f] = wl.chunks;
    io.sched[f] = wl.sched;
  }
  o.snap = p.snap ? 1 : 0;
  o.one_of = p.one_tc ? (p.has[kFamStream] ? 1 : 0) : -1;  // the expert-tile list's index
  o.zero_i32 = p.has[kFamStream] ? reinterpret_cast<int32_t*>(ws + L.done) : nullptr;
  o.n_zero = p.has[kFamStream] ? L.n_done : 0;
  io.acc = p.has[kFamStream] ? reinterpret_cast<float*>(ws + L.acc) : nullptr;
  io.done = o.zero_i32;
  io.h = reinterpret_cast<uint16_t*>(ws + L.h);
}

// The whole layer for one plan: routing (with one work list per family that may receive
// rows), the rows in expert order for the tcgen05 families, then the expert half.  All
// kernels go on one stream with programmatic serialisation.
moe_status forward_plan(moe_ctx* c, int T, const void* x_bf16, const void* W_router_bf16,
                        const float* b_router, const void* W_gate_up_bf16,
                        const void* W_down_bf16, float* out, uint8_t* ws, size_t ws_bytes,
                        cudaStream_t st, const MxWeights* mx = nullptr) {
  const Plan p = make_plan(c, T, mx != nullptr, c->path);
  const Layout L = make_layout(c, T, p, mx != nullptr);
  if (ws_bytes < L.total) return MOE_ERR_WORKSPACE;
  const size_t R = (size_t)T * c->k;
  RouteOut o{};
  ExpertIO io{};
  o.topk_idx = reinterpret_cast<int32_t*>(ws + L.topk_idx);
  o.topk_w = reinterpret_cast<float*>(ws + L.topk_w);
  o.offsets = reinterpret_cast<int32_t*>(ws + L.offsets);
  o.perm = reinterpret_cast<int32_t*>(ws + L.perm);
  o.inv_perm = reinterpret_cast<int32_t*>(ws + L.inv_perm);
  o.row_w = reinterpret_cast<float*>(ws + L.row_w);
  plan_lists(p, L, ws, o, io);
  const uint16_t* x = static_cast<const uint16_t*>(x_bf16);
  uint16_t* x16 = mx ? reinterpret_cast<uint16_t*>(ws + L.x16) : nullptr;
  uint16_t* x_perm = L.x_perm ? reinterpret_cast<uint16_t*>(ws + L.x_perm) : nullptr;
  if (mx && p.has[kFamStream]) {  // the MXFP4 streaming kernels take f16 activations
    const size_t n = (size_t)T * c->H;
    const int blocks = (int)std::min<size_t>((n / 8 + 255) / 256, (size_t)c->num_sms * 4);
    MOE_TRY(launch(c, kKindConvert, st, [&] {
      return launch_pdl(to_f16_kernel, dim3(blocks), dim3(256), 0, st, x, x16, n, c->d_status);
    }));
  }
  // With enough 64-token blocks to cover the GPU the scatter also writes the rows in expert
  // order (each token row read once); otherwise a wide gather kernel does it.
  const int NB = (T + kRouterTcTokens - 1) / kRouterTcTokens;
  const bool fused_copy = x_perm && T > kSmallT && NB >= c->num_sms;
  if (fused_copy) {
    o.x = x;
    o.x_perm = x_perm;
    o.H = c->H;
  }
  // A few tokens on the streaming family alone: the gate/up kernel finishes the routing from
  // the partial logits (no finalize kernel in between); the router zero-fills the completion
  // counters and the split-K sums that follow them.
  const bool fuse = p.fused_route;
  if (fuse) {
    io.sr.partial = reinterpret_cast<const float*>(ws + L.rt.partial);
    io.sr.S = L.rt.splits;
    io.sr.b_router = b_router;
    io.sr.T = T;
    io.sr.E = c->E;
    io.sr.k = c->k;
    io.sr.o = o;
    MOE_TRY(launch_route(c, T, x, static_cast<const uint16_t*>(W_router_bf16), b_router, o, ws,
                         L.rt, st, reinterpret_cast<float*>(ws + L.done),
                         (L.acc - L.done) / 4 + L.acc_floats, /*finalize=*/false));
  } else {
    MOE_TRY(launch_route(c, T, x, static_cast<const uint16_t*>(W_router_bf16), b_router, o, ws,
                         L.rt, st, io.acc, L.acc_floats));
  }
  if (x_perm && !fused_copy)
    MOE_TRY(launch(c, kKindGather, st, [&] {
      return launch_pdl(gather_rows_kernel, dim3((unsigned)((R + 7) / 8)), dim3(256), 0, st, x,
                        (const int32_t*)o.perm, (int)R, c->H, x_perm);
    }));
  io.R = (int)R;
  io.x_tok = mx ? x16 : x;
  io.perm = o.perm;
  io.x_perm = x_perm;
  io.row_w = o.row_w;
  io.out = out;
  io.out_elems = (size_t)T * c->H;
  return expert_phase(c, p, io, W_gate_up_bf16, W_down_bf16, mx, st);
}

size_t forward_ws_bytes(const moe_ctx* c, int T, bool mx, moe_path path) {
  return make_layout(c, T, make_plan(c, T, mx, path), mx).total;
}

__global__ void selftest_timeout_kernel(uint32_t* status, uint64_t limit_ns) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_barrier_init();
  }
  __syncthreads();
  // Nothing ever arrives on `bar`: the wait must run out and report it.
  if (threadIdx.x == 0 && !mbar_wait_bounded(&bar, 0, limit_ns)) atomicOr(status, kStatusTimeout);
}

}  // namespace

extern "C" {

moe_status moe_create(int E, int H, int I, int k, moe_t* out) {
  if (!out) return MOE_ERR_ARG;
  *out = nullptr;
  if (!shape_ok(E, H, I, k)) return MOE_ERR_ARG;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return MOE_ERR_DEVICE;
  }
  cudaDeviceProp prop;
  if (cudaGetDeviceProperties(&prop, dev) != cudaSuccess) {
    cudaGetLastError();
    return MOE_ERR_DEVICE;
  }
  if (prop.major != 10) return MOE_ERR_DEVICE;
  if (!set_smem_attrs()) {
    cudaGetLastError();
    return MOE_ERR_CUDA;
  }
  moe_ctx* c = new (std::nothrow) moe_ctx();
  if (!c) return MOE_ERR_ARG;
  c->E = E;
  c->H = H;
  c->I = I;
  c->k = k;
  c->device = dev;
  c->num_sms = prop.multiProcessorCount;
  c->stream_T = default_stream_T(c);
  // row-tile width of the grouped GEMM: MOE_ROW_TILE=512 or 256 (default below)
  if (const char* v = getenv("MOE_ROW_TILE")) c->wide_rows = strcmp(v, "512") == 0;
  // rows per expert tile: MOE_TILE_ROWS=128 or 256 (default: by each call's mean load)
  if (const char* v = getenv("MOE_TILE_ROWS")) c->tile_n = atoi(v) == 256 ? 256 : atoi(v) == 128 ? 128 : 0;
  if (cudaMalloc(&c->d_status, sizeof(uint32_t)) != cudaSuccess ||
      cudaMemset(c->d_status, 0, sizeof(uint32_t)) != cudaSuccess) {
    cudaGetLastError();
    if (c->d_status) cudaFree(c->d_status);
    delete c;
    return MOE_ERR_CUDA;
  }
  // the routing scratch of moe_route_static, looked up with this handle's device current;
  // the second stream and its fork / join events for calls whose kernel families fork
  if (static_scratch_address(&c->static_scratch) != MOE_OK ||
      cudaStreamCreateWithFlags(&c->aux, cudaStreamNonBlocking) != cudaSuccess ||
      cudaEventCreateWithFlags(&c->ev_fork, cudaEventDisableTiming) != cudaSuccess ||
      cudaEventCreateWithFlags(&c->ev_join, cudaEventDisableTiming) != cudaSuccess) {
    cudaGetLastError();
    if (c->ev_fork) cudaEventDestroy(c->ev_fork);
    if (c->aux) cudaStreamDestroy(c->aux);
    cudaFree(c->d_status);
    delete c;
    return MOE_ERR_CUDA;
  }
  *out = c;
  return MOE_OK;
}

moe_status moe_destroy(moe_t c) {
  if (!c) return MOE_OK;
  for (cudaEvent_t e : c->ev) cudaEventDestroy(e);
  if (c->ev_fork) cudaEventDestroy(c->ev_fork);
  if (c->ev_join) cudaEventDestroy(c->ev_join);
  if (c->aux) cudaStreamDestroy(c->aux);
  if (c->d_status) cudaFree(c->d_status);
  delete c;
  return MOE_OK;
}

size_t moe_route_workspace_bytes(moe_t c, int T) {
  if (!c || T < 0 || T > kMaxT) return 0;
  if (T == 0) return 0;
  return route_ws_bytes(c, T);
}

size_t moe_workspace_bytes(moe_t c, int T) {
  if (!c || T < 0 || T > kMaxT) return 0;
  if (T == 0) return 0;
  return forward_ws_bytes(c, T, false, c->path);
}

moe_status moe_route(moe_t c, int T, const void* x_bf16, const void* W_router_bf16,
                     const float* b_router, int32_t* topk_idx, float* topk_w,
                     int32_t* expert_offsets, int32_t* perm, int32_t* inv_perm, void* workspace,
                     size_t ws_bytes, moe_stream_t stream) {
  MOE_TRY(check_common(c, T, x_bf16, W_router_bf16, b_router));
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (!expert_offsets || !aligned16(expert_offsets)) return MOE_ERR_ARG;
  if (T == 0) {
    if (cudaMemsetAsync(expert_offsets, 0, sizeof(int32_t) * (c->E + 1), st) != cudaSuccess)
      return MOE_ERR_CUDA;
    return MOE_OK;
  }
  if (!topk_idx || !topk_w || !perm || !inv_perm) return MOE_ERR_ARG;
  if (!aligned16(topk_idx) || !aligned16(topk_w) || !aligned16(perm) || !aligned16(inv_perm))
    return MOE_ERR_ARG;
  const size_t need = route_ws_bytes(c, T);
  if (!workspace || !aligned16(workspace) || ws_bytes < need) return MOE_ERR_WORKSPACE;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  Carver cv;
  cv.take(16);  // the work-list word of the forward layouts (kept: same scratch size)
  const RouteTmp rt = carve_route_tmp(cv, c, T);
  RouteOut o{};
  o.topk_idx = topk_idx;
  o.topk_w = topk_w;
  o.offsets = expert_offsets;
  o.perm = perm;
  o.inv_perm = inv_perm;
  o.row_w = nullptr;
  o.n_lists = 0;  // routing only: no work lists
  o.zero_i32 = nullptr;
  o.n_zero = 0;
  return launch_route(c, T, static_cast<const uint16_t*>(x_bf16),
                      static_cast<const uint16_t*>(W_router_bf16), b_router, o, ws, rt, st);
}

moe_status moe_forward(moe_t c, int T, const void* x_bf16, const void* W_router_bf16,
                       const float* b_router, const void* W_gate_up_bf16,
                       const void* W_down_bf16, float* out, void* workspace, size_t ws_bytes,
                       moe_stream_t stream) {
  MOE_TRY(check_common(c, T, x_bf16, W_router_bf16, b_router));
  if (T == 0) return MOE_OK;
  if (!W_gate_up_bf16 || !W_down_bf16 || !out) return MOE_ERR_ARG;
  if (!aligned16(W_gate_up_bf16) || !aligned16(W_down_bf16) || !aligned16(out))
    return MOE_ERR_ARG;
  if (!workspace || !aligned16(workspace)) return MOE_ERR_WORKSPACE;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  c->in_call = c->prof_max > 0 && c->prof_calls < c->prof_max;
  const moe_status s = forward_plan(c, T, x_bf16, W_router_bf16, b_router, W_gate_up_bf16,
                                    W_down_bf16, out, ws, ws_bytes, st);
  if (c->in_call) ++c->prof_calls;
  c->in_call = false;
  return s;
}

size_t moe_workspace_bytes_mxfp4(moe_t c, int T) {
  if (!c || T < 0 || T > kMaxT || (long long)T * c->k >= (1ll << 31)) return 0;
  if (T == 0) return 0;
  return forward_ws_bytes(c, T, /*mx=*/true, c->path);
}

moe_status moe_forward_mxfp4(moe_t c, int T, const void* x_bf16, const void* W_router_bf16,
                             const float* b_router, const void* gu_codes, const void* gu_scales,
                             const void* dn_codes, const void* dn_scales, float* out,
                             void* workspace, size_t ws_bytes, moe_stream_t stream) {
  MOE_TRY(check_common(c, T, x_bf16, W_router_bf16, b_router));
  if (T == 0) return MOE_OK;
  if (!gu_codes || !gu_scales || !dn_codes || !dn_scales || !out) return MOE_ERR_ARG;
  if (!aligned16(gu_codes) || !aligned16(gu_scales) || !aligned16(dn_codes) ||
      !aligned16(dn_scales) || !aligned16(out))
    return MOE_ERR_ARG;
  if (!workspace || !aligned16(workspace)) return MOE_ERR_WORKSPACE;
  const MxWeights mx{gu_codes, gu_scales, dn_codes, dn_scales};
  c->in_call = c->prof_max > 0 && c->prof_calls < c->prof_max;
  const moe_status s = forward_plan(c, T, x_bf16, W_router_bf16, b_router, nullptr, nullptr,
                                      out, static_cast<uint8_t*>(workspace), ws_bytes,
                                      reinterpret_cast<cudaStream_t>(stream), &mx);
  if (c->in_call) ++c->prof_calls;
  c->in_call = false;
  return s;
}

moe_status moe_permute(moe_t c, int T, const void* x_bf16, const int32_t* perm,
                       const int32_t* inv_perm, const float* topk_w, void* x_perm_bf16,
                       float* row_w, moe_stream_t stream) {
  if (!c || T < 0 || T > kMaxT || (long long)T * c->k >= (1ll << 31)) return MOE_ERR_ARG;
  if (T == 0) return MOE_OK;
  if (!x_bf16 || !perm || !inv_perm || !topk_w || !x_perm_bf16 || !row_w) return MOE_ERR_ARG;
  if (!aligned16(x_bf16) || !aligned16(x_perm_bf16)) return MOE_ERR_ARG;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const long long R = (long long)T * c->k;
  return launch(c, kKindGather, st, [&] {
    return launch_pdl(permute_rows_kernel, dim3((unsigned)((R + 7) / 8)), dim3(256), 0, st,
                      static_cast<const uint16_t*>(x_bf16), perm, inv_perm, topk_w, T, c->k,
                      c->H, static_cast<uint16_t*>(x_perm_bf16), row_w, c->d_status);
  });
}

moe_status moe_combine(moe_t c, int T, const int32_t* inv_perm, const float* y_rows, float* out,
                       moe_stream_t stream) {
  if (!c || T < 0 || T > kMaxT || (long long)T * c->k >= (1ll << 31)) return MOE_ERR_ARG;
  if (T == 0) return MOE_OK;
  if (!inv_perm || !y_rows || !out || !aligned16(y_rows) || !aligned16(out)) return MOE_ERR_ARG;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  return launch(c, kKindDown, st, [&] {
    return launch_pdl(combine_rows_kernel, dim3((unsigned)((T + 7) / 8)), dim3(256), 0, st,
                      inv_perm, y_rows, T, c->k, c->H, out, c->d_status);
  });
}

size_t moe_experts_workspace_bytes(moe_t c, int R, int S) {
  if (!c || R < 0 || R > kMaxT * 256 || S < 1 || (long long)S * c->E > kMaxSegments) return 0;
  if (R == 0) return 0;
  return make_expert_layout(c, R, S, make_plan(c, R, false, c->path)).total;
}

moe_status moe_experts(moe_t c, int R, int S, const int32_t* seg_counts, const void* x_rows_bf16,
                       const float* row_w, const void* W_gate_up_bf16, const void* W_down_bf16,
                       float* y_rows, void* workspace, size_t ws_bytes, moe_stream_t stream) {
  if (!c || R < 0 || R > kMaxT * 256 || S < 1 || (long long)S * c->E > kMaxSegments)
    return MOE_ERR_ARG;
  if (R == 0) return MOE_OK;
  if (!seg_counts || !x_rows_bf16 || !row_w || !W_gate_up_bf16 || !W_down_bf16 || !y_rows)
    return MOE_ERR_ARG;
  if (!aligned16(x_rows_bf16) || !aligned16(W_gate_up_bf16) || !aligned16(W_down_bf16) ||
      !aligned16(y_rows))
    return MOE_ERR_ARG;
  if (!workspace || !aligned16(workspace)) return MOE_ERR_WORKSPACE;
  const Plan p = make_plan(c, R, false, c->path);
  const Layout L = make_expert_layout(c, R, S, p);
  if (ws_bytes < L.total) return MOE_ERR_WORKSPACE;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  c->in_call = c->prof_max > 0 && c->prof_calls < c->prof_max;
  RouteOut o{};
  ExpertIO io{};
  plan_lists(p, L, ws, o, io);
  int32_t* iota = reinterpret_cast<int32_t*>(ws + L.perm);
  const int grid = (int)std::max<long long>(1, std::min<long long>(c->num_sms, (R + 1023) / 1024));
  const size_t smem = (size_t)(4 * S * c->E + 2 * c->E) * 4;
  moe_status s = launch(c, kKindRouteFin, st, [&] {
    return launch_pdl(build_segment_lists_kernel, dim3(grid), dim3(1024), smem, st, seg_counts,
                      S, c->E, R, o, iota, reinterpret_cast<float4*>(io.acc), L.acc_floats / 4,
                      c->d_status);
  });
  if (s == MOE_OK) {
    io.R = R;
    io.x_tok = static_cast<const uint16_t*>(x_rows_bf16);
    io.perm = iota;
    io.x_perm = static_cast<const uint16_t*>(x_rows_bf16);
    io.row_w = row_w;
    io.out = y_rows;
    io.out_elems = (size_t)R * c->H;
    s = expert_phase(c, p, io, W_gate_up_bf16, W_down_bf16, nullptr, st);
  }
  if (c->in_call) ++c->prof_calls;
  c->in_call = false;
  return s;
}

moe_status moe_last_dispatch(moe_t c, int T, int mxfp4, const void* workspace, size_t ws_bytes,
                             int32_t* entries, moe_stream_t stream) {
  if (!c || !entries || T < 1 || T > kMaxT || !workspace) return MOE_ERR_ARG;
  const Plan p = make_plan(c, T, mxfp4 != 0, c->path);
  const Layout L = make_layout(c, T, p, mxfp4 != 0);
  if (ws_bytes < L.total) return MOE_ERR_WORKSPACE;
  if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
    return MOE_ERR_CUDA;
  for (int f = 0; f < kFamilies; ++f) {
    entries[f] = -1;
    if (!p.has[f]) continue;
    int32_t v = 0;
    if (cudaMemcpy(&v, static_cast<const uint8_t*>(workspace) + L.sched[f], sizeof(v),
                   cudaMemcpyDeviceToHost) != cudaSuccess)
      return MOE_ERR_CUDA;
    entries[f] = v;
  }
  return MOE_OK;
}

moe_status moe_set_path(moe_t c, moe_path path, int crossover_T) {
  if (!c) return MOE_ERR_ARG;
  if (path != MOE_PATH_AUTO && path != MOE_PATH_STREAM && path != MOE_PATH_GEMM &&
      path != MOE_PATH_TILE)
    return MOE_ERR_ARG;
  c->path = path;
  if (crossover_T >= 0) c->stream_T = crossover_T;
  return MOE_OK;
}

moe_status moe_get_path(moe_t c, moe_path* path, int* crossover_T) {
  if (!c) return MOE_ERR_ARG;
  if (path) *path = c->path;
  if (crossover_T) *crossover_T = c->stream_T;
  return MOE_OK;
}

moe_status moe_set_dispatch(moe_t c, int stream_rows, int tile_rows, int per_expert) {
  if (!c) return MOE_ERR_ARG;
  if (stream_rows >= 0) c->stream_rows = stream_rows;
  if (tile_rows >= 0) c->tile_rows = tile_rows;
  if (per_expert >= 0) c->per_expert = per_expert != 0;
  return MOE_OK;
}

moe_status moe_get_dispatch(moe_t c, int* stream_rows, int* tile_rows, int* per_expert) {
  if (!c) return MOE_ERR_ARG;
  if (stream_rows) *stream_rows = c->stream_rows;
  if (tile_rows) *tile_rows = c->tile_rows;
  if (per_expert) *per_expert = c->per_expert ? 1 : 0;
  return MOE_OK;
}

size_t moe_tune_workspace_bytes(moe_t c, int T_max) {
  if (!c || T_max < 1 || T_max > kMaxT) return 0;
  size_t need = 0;
  for (moe_path p : {MOE_PATH_STREAM, MOE_PATH_TILE, MOE_PATH_GEMM, MOE_PATH_AUTO})
    need = std::max(need, forward_ws_bytes(c, T_max, false, p));
  return need;
}

moe_status moe_tune(moe_t c, int T_max, const void* x_bf16, const void* W_router_bf16,
                    const float* b_router, const void* W_gate_up_bf16, const void* W_down_bf16,
                    float* out, void* workspace, size_t ws_bytes, moe_stream_t stream,
                    int* crossover_out) {
  if (!c || T_max < 1 || T_max > kMaxT) return MOE_ERR_ARG;
  MOE_TRY(check_common(c, T_max, x_bf16, W_router_bf16, b_router));
  if (!W_gate_up_bf16 || !W_down_bf16 || !out || !aligned16(out)) return MOE_ERR_ARG;
  if (!workspace || ws_bytes < moe_tune_workspace_bytes(c, T_max)) return MOE_ERR_WORKSPACE;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const moe_path saved_path = c->path;
  const int saved_prof = c->prof_max;
  c->prof_max = 0;  // tuning launches are not profiled
  cudaEvent_t e0 = nullptr, e1 = nullptr;
  if (cudaEventCreate(&e0) != cudaSuccess || cudaEventCreate(&e1) != cudaSuccess) {
    cudaGetLastError();
    if (e0) cudaEventDestroy(e0);
    c->prof_max = saved_prof;
    return MOE_ERR_CUDA;
  }
  // median of 5 timed calls after 2 warm-up calls, for one path at one token count
  auto time_path = [&](moe_path p, int T, float* ms_out) -> moe_status {
    c->path = p;
    float v[5];
    for (int rep = 0; rep < 7; ++rep) {
      if (rep >= 2 && cudaEventRecord(e0, st) != cudaSuccess) return MOE_ERR_CUDA;
      MOE_TRY(moe_forward(c, T, x_bf16, W_router_bf16, b_router, W_gate_up_bf16, W_down_bf16,
                          out, workspace, ws_bytes, stream));
      if (rep >= 2) {
        if (cudaEventRecord(e1, st) != cudaSuccess || cudaEventSynchronize(e1) != cudaSuccess ||
            cudaEventElapsedTime(&v[rep - 2], e0, e1) != cudaSuccess)
          return MOE_ERR_CUDA;
      }
    }
    std::sort(v, v + 5);
    *ms_out = v[2];
    return MOE_OK;
  };
  // Largest T at which family `lo` is not slower than family `hi` over the whole layer (0 if
  // never); stops once `hi` has been faster for a doubling of T.
  static const int kCandidates[] = {1, 2, 4, 8, 12, 16, 24, 32, 48, 64, 96, 128, 192, 256, 384,
                                    512, 768, 1024, 1536, 2048, 3072, 4096};
  auto crossover_T = [&](moe_path lo, moe_path hi, int* T_out) -> moe_status {
    int cross = 0;
    for (int T : kCandidates) {
      if (T > T_max) break;
      float tl = 0.f, th = 0.f;
      MOE_TRY(time_path(lo, T, &tl));
      MOE_TRY(time_path(hi, T, &th));
      if (tl <= th) cross = T;
      else if (T >= 2 * std::max(cross, 1)) break;
    }
    *T_out = cross;
    return MOE_OK;
  };
  // The expert-tile / row-tile boundary measured at T tokens becomes a per-expert row count:
  // the mean rows per expert at that T (uniform routing: T*k/E).
  auto rows_at = [&](int T) {
    return T == 0 ? 0 : std::max(1, (int)(((long long)T * c->k + c->E - 1) / c->E));
  };
  int Ts = 0, Tt = 0;
  moe_status s = crossover_T(MOE_PATH_STREAM, MOE_PATH_TILE, &Ts);
  if (s == MOE_OK) s = crossover_T(MOE_PATH_TILE, MOE_PATH_GEMM, &Tt);
  cudaEventDestroy(e0);
  cudaEventDestroy(e1);
  c->path = saved_path;
  c->prof_max = saved_prof;
  if (s != MOE_OK) return s;
  // streaming runs in calls of at most Ts tokens; the tile family ends where the row-tile GEMM
  // wins (if T_max never let it win, the measured band is kept as the lower bound)
  c->stream_T = Ts;
  c->tile_rows = Tt >= T_max ? std::max(c->tile_rows, rows_at(Tt)) : std::max(1, rows_at(Tt));
  if (crossover_out) *crossover_out = c->stream_T;
  return MOE_OK;
}

moe_status moe_sync_status(moe_t c, moe_stream_t stream) {
  if (!c) return MOE_ERR_ARG;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(st) != cudaSuccess) return MOE_ERR_CUDA;
  uint32_t word = 0;
  if (cudaMemcpy(&word, c->d_status, sizeof(word), cudaMemcpyDeviceToHost) != cudaSuccess)
    return MOE_ERR_CUDA;
  if (word != 0) {
    if (cudaMemset(c->d_status, 0, sizeof(word)) != cudaSuccess) return MOE_ERR_CUDA;
    if (word & kStatusTimeout) return MOE_ERR_TIMEOUT;
    if (word & (kStatusBadIndex | kStatusBadCounts)) return MOE_ERR_ARG;
    if (word & kStatusF16Range) return MOE_ERR_UNSUPPORTED;
  }
  return MOE_OK;
}

const char* moe_status_string(moe_status s) {
  switch (s) {
    case MOE_OK: return "ok";
    case MOE_ERR_ARG: return "invalid argument";
    case MOE_ERR_UNSUPPORTED: return "unsupported on this build or device";
    case MOE_ERR_WORKSPACE: return "workspace missing or too small";
    case MOE_ERR_CUDA: return "CUDA error";
    case MOE_ERR_TIMEOUT: return "device-side wait timed out";
    case MOE_ERR_DEVICE: return "no usable sm_100 device";
  }
  return "unknown status";
}

uint64_t moe_launch_count(moe_t c) { return c ? c->launches : 0; }

moe_status moe_profile_begin(moe_t c, int max_calls) {
  if (!c || max_calls < 1 || max_calls > (1 << 20)) return MOE_ERR_ARG;
  for (cudaEvent_t e : c->ev) cudaEventDestroy(e);
  c->ev.assign((size_t)max_calls * kMaxKernelsPerCall * 2, nullptr);
  c->ev_kind.assign((size_t)max_calls * kMaxKernelsPerCall, -1);
  for (auto& e : c->ev)
    if (cudaEventCreate(&e) != cudaSuccess) {
      cudaGetLastError();
      return MOE_ERR_CUDA;
    }
  c->prof_max = max_calls;
  c->prof_calls = 0;
  c->ev_used = 0;
  return MOE_OK;
}

moe_status moe_profile_end(moe_t c, float* ms, int* launches, int n_kinds) {
  if (!c || n_kinds < 0) return MOE_ERR_ARG;
  for (int i = 0; i < n_kinds; ++i) {
    if (ms) ms[i] = 0.f;
    if (launches) launches[i] = 0;
  }
  moe_status s = MOE_OK;
  for (size_t p = 0; p + 1 < c->ev_used; p += 2) {
    float t = 0.f;
    if (cudaEventSynchronize(c->ev[p + 1]) != cudaSuccess ||
        cudaEventElapsedTime(&t, c->ev[p], c->ev[p + 1]) != cudaSuccess) {
      cudaGetLastError();
      s = MOE_ERR_CUDA;
      continue;
    }
    const int kind = c->ev_kind[p / 2];
    if (kind >= 0 && kind < n_kinds) {
      if (ms) ms[kind] += t;
      if (launches) launches[kind] += 1;
    }
  }
  for (cudaEvent_t e : c->ev) cudaEventDestroy(e);
  c->ev.clear();
  c->ev_kind.clear();
  c->ev_used = 0;
  c->prof_max = 0;
  c->prof_calls = 0;
  return s;
}

const char* moe_profile_kind_name(int kind) {
  static const char* names[MOE_PROFILE_KINDS] = {
      "router",       "route_finalize", "gather",  "gate_up_stream", "down_stream",
      "to_f16",       "gate_up_tile",   "down_tile", "gate_up_gemm", "down_gemm"};
  if (kind < 0 || kind >= MOE_PROFILE_KINDS) return "unknown";
  return names[kind];
}

moe_status moe_selftest_timeout(moe_t c, int limit_us, moe_stream_t stream) {
  if (!c || limit_us < 1 || limit_us > 1000000) return MOE_ERR_ARG;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  selftest_timeout_kernel<<<1, 32, 0, st>>>(c->d_status, (uint64_t)limit_us * 1000ull);
  if (cudaGetLastError() != cudaSuccess) return MOE_ERR_CUDA;
  ++c->launches;
  return MOE_OK;
}

}  // extern "C"

// ------------------------------------------------------------------------------------------
// Routing without caller-provided device memory.
//
// Some callers cannot hand the library a workspace: code that runs where device allocation is
// not allowed or not wanted at call time (a host process whose device memory is owned
// entirely by another allocator or memory pool, a latency-critical serving loop that
// forbids allocation after start-up, a plain C caller with no allocator of its own).  For
// them, moe_route_static uses this fixed array in the library's own device memory instead.
// Its size is fixed at build time; every device that loads the library holds it until the
// process exits.  Calls share it, so two of them that overlap on the GPU race.
// ------------------------------------------------------------------------------------------
namespace {
constexpr size_t kRouteStaticScratchBytes = size_t(2) << 20;  // 2 MiB
}  // namespace

static __device__ __align__(256) uint8_t g_route_static_scratch[kRouteStaticScratchBytes];

namespace {
// Device address of g_route_static_scratch in the current device's context.  In host code the
// array's name only stands for the symbol; its device address comes from the runtime, which
// allocates nothing to answer.  moe_create calls this with the handle's device current and
// keeps the answer in the handle, whose lifetime is bounded by that context's.
moe_status static_scratch_address(void** out) {
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_route_static_scratch) != cudaSuccess || p == nullptr) {
    cudaGetLastError();
    return MOE_ERR_CUDA;
  }
  *out = p;
  return MOE_OK;
}
}  // namespace

extern "C" {

size_t moe_route_static_max_bytes(void) { return kRouteStaticScratchBytes; }

moe_status moe_route_static(moe_t c, int T, const void* x_bf16, const void* W_router_bf16,
                            const float* b_router, int32_t* topk_idx, float* topk_w,
                            int32_t* expert_offsets, int32_t* perm, int32_t* inv_perm,
                            moe_stream_t stream) {
  MOE_TRY(check_common(c, T, x_bf16, W_router_bf16, b_router));
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (!expert_offsets || !aligned16(expert_offsets)) return MOE_ERR_ARG;
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return MOE_ERR_DEVICE;
  }
  if (dev != c->device) return MOE_ERR_ARG;
  if (T == 0) {
    if (cudaMemsetAsync(expert_offsets, 0, sizeof(int32_t) * (c->E + 1), st) != cudaSuccess)
      return MOE_ERR_CUDA;
    return MOE_OK;
  }
  if (!topk_idx || !topk_w || !perm || !inv_perm) return MOE_ERR_ARG;
  if (!aligned16(topk_idx) || !aligned16(topk_w) || !aligned16(perm) || !aligned16(inv_perm))
    return MOE_ERR_ARG;
  if (route_ws_bytes(c, T, /*allow_split=*/false) > kRouteStaticScratchBytes)
    return MOE_ERR_WORKSPACE;
  if (!c->static_scratch) return MOE_ERR_CUDA;
  uint8_t* ws = static_cast<uint8_t*>(c->static_scratch);
  Carver cv;
  cv.take(16);  // the work-list word of the forward layouts (kept: same scratch size)
  const RouteTmp rt = carve_route_tmp(cv, c, T, /*allow_split=*/false);
  RouteOut o{};
  o.topk_idx = topk_idx;
  o.topk_w = topk_w;
  o.offsets = expert_offsets;
  o.perm = perm;
  o.inv_perm = inv_perm;
  o.row_w = nullptr;
  o.n_lists = 0;  // routing only: no work lists
  o.zero_i32 = nullptr;
  o.n_zero = 0;
  // Every scratch word the routing kernels read is written earlier in the same call (the
  // partial logits or the per-block counts and totals), so nothing needs clearing.
  return launch_route(c, T, static_cast<const uint16_t*>(x_bf16),
                      static_cast<const uint16_t*>(W_router_bf16), b_router, o, ws, rt, st);
}

}  // extern "C"
