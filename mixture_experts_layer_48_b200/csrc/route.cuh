// Routing kernels: router logits, top-k with a softmax over the selected logits, expert
// histogram, offsets, the stable token -> row permutation and the per-path work lists.
//
// The layer routes every token to its top-k experts by router score (top-4 of 32 in the
// Persona Kappa forum post's "Architecture Summary"; top-4 of 128 in the hearth-lean-loomed-v1
// card).  Ties go to the lower expert index; inside an expert's row segment tokens ascend.
//
// Two chains:
//   T <= kSmallT : router_partial_kernel (H/64 blocks, one 64-row slice of W_router each)
//                  -> route_small_finalize_kernel (one block: sum, top-k, softmax,
//                     histogram, scan, permutation, work list).
//   T >  kSmallT : router_topk_kernel (32 tokens per block, all experts, full H; top-k and a
//                  block histogram) -> route_scan_kernel (one block per expert: prefix over
//                  blocks) -> route_scatter_kernel (32 tokens per block: permutation).
#pragma once

#include "common.cuh"

namespace moe {

constexpr int kSmallT = 64;        // largest T handled by the single-block finalize
constexpr int kRouteTile = 32;     // tokens per block in the large-T chain
constexpr int kRouterHSlice = 64;  // W_router rows per block in router_partial_kernel

// Outputs of routing, all in device memory.
struct RouteOut {
  int32_t* topk_idx;   // [T, k]
  float* topk_w;       // [T, k]
  int32_t* offsets;    // [E + 1]
  int32_t* perm;       // [T * k]
  int32_t* inv_perm;   // [T, k]
  float* row_w;        // [T * k] routing weight of each row (may be null)
  int4* chunks;        // work list: {expert, first row, rows, 0}; null = none
  int32_t* sched;      // [0] number of chunks, [1] number of experts with rows
  int chunk_rows;      // rows per work-list entry
  int32_t* zero_i32;   // region zeroed by the chain (completion counters), may be null
  int n_zero;
};

// ---------------------------------------------------------------------------------------
// top-k of one token held by a warp.  lg points at the token's E logits in shared memory;
// on return lg[0..k) holds the selected logits (slot order) and sel[0..k) the experts.
// Equal logits go to the lower expert index.
// ---------------------------------------------------------------------------------------
MOE_DEVINL void warp_topk(float* lg, int E, int k, int32_t* sel) {
  const int lane = threadIdx.x & 31;
  constexpr int kMaxPer = 8;  // E <= 256
  float v[kMaxPer];
#pragma unroll
  for (int m = 0; m < kMaxPer; ++m) {
    const int e = lane + 32 * m;
    v[m] = (e < E) ? lg[e] : -INFINITY;
  }
  __syncwarp();
  for (int j = 0; j < k; ++j) {
    // local best: largest value, then lowest expert index (m ascending = index ascending)
    float bv = -INFINITY;
    int be = 0x7fffffff;
#pragma unroll
    for (int m = 0; m < kMaxPer; ++m) {
      const int e = lane + 32 * m;
      if (e < E && (v[m] > bv || (v[m] == bv && e < be))) {
        bv = v[m];
        be = e;
      }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, bv, off);
      const int oe = __shfl_xor_sync(0xffffffffu, be, off);
      if (ov > bv || (ov == bv && oe < be)) {
        bv = ov;
        be = oe;
      }
    }
    // remove the winner from its owner lane (NaN-free inputs: -inf is below every logit)
    if ((be & 31) == lane) {
#pragma unroll
      for (int m = 0; m < kMaxPer; ++m)
        if (lane + 32 * m == be) v[m] = -INFINITY;
    }
    if (lane == 0) {
      sel[j] = be;
      lg[j] = bv;  // the token's logits are all in registers by now
    }
    __syncwarp();
  }
}

// Routing weights of one token (softmax over its k selected logits, lg[0] the largest).
MOE_DEVINL float warp_softmax_denominator(const float* lg, int k) {
  const int lane = threadIdx.x & 31;
  const float l0 = lg[0];
  float s = 0.f;
  for (int j = lane; j < k; j += 32) s += expf(lg[j] - l0);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
  return s;
}

// ---------------------------------------------------------------------------------------
// Small T: partial router logits over one 64-row slice of W_router.
// grid (H/64, ceil(T/32)), block 256.  partial layout [H/64][T][E].
// ---------------------------------------------------------------------------------------
// Grid-stride zero fill of a scratch region by every block of the launching kernel.
MOE_DEVINL void zero_fill_f4(float4* z, size_t n4) {
  const size_t nthreads = (size_t)gridDim.x * gridDim.y * blockDim.x;
  const size_t b = (size_t)blockIdx.y * gridDim.x + blockIdx.x;
  for (size_t i = b * blockDim.x + threadIdx.x; i < n4; i += nthreads)
    z[i] = make_float4(0.f, 0.f, 0.f, 0.f);
}

__global__ void __launch_bounds__(256) router_partial_kernel(const uint16_t* __restrict__ x,
                                                             const uint16_t* __restrict__ Wr,
                                                             int T, int H, int E,
                                                             float* __restrict__ partial,
                                                             float4* zero4, size_t n_zero4) {
  zero_fill_f4(zero4, n_zero4);
  extern __shared__ __align__(128) uint8_t smem_raw[];
  uint16_t* xs = reinterpret_cast<uint16_t*>(smem_raw);  // [32][64]
  uint16_t* ws = xs + kRouteTile * kRouterHSlice;          // [64][E]
  const int s = blockIdx.x, h0 = s * kRouterHSlice, t0 = blockIdx.y * kRouteTile;
  const int nt = min(kRouteTile, T - t0);
  for (int i = threadIdx.x; i < nt * 8; i += blockDim.x) {
    const int r = i >> 3, c = i & 7;
    reinterpret_cast<uint4*>(xs)[r * 8 + c] =
        reinterpret_cast<const uint4*>(x + (size_t)(t0 + r) * H + h0)[c];
  }
  const uint16_t* wsrc = Wr + (size_t)h0 * E;
  for (int i = threadIdx.x; i < kRouterHSlice * E; i += blockDim.x) ws[i] = wsrc[i];
  __syncthreads();
  for (int o = threadIdx.x; o < nt * E; o += blockDim.x) {
    const int t = o / E, e = o - t * E;
    float acc = 0.f;
#pragma unroll 16
    for (int h = 0; h < kRouterHSlice; ++h)
      acc = fmaf(bf16_to_f32(xs[t * kRouterHSlice + h]), bf16_to_f32(ws[h * E + e]), acc);
    partial[((size_t)s * T + t0 + t) * E + e] = acc;
  }
}

// Work list of one routing: expert e's rows split into entries of at most chunk_rows rows.
// Called by all threads of a block with count/off in shared memory (E <= 256 entries).
MOE_DEVINL void build_work_list(const int32_t* cnt, const int32_t* off, int E,
                                const RouteOut& o, int32_t* scratch /* [256 + 1] smem */) {
  const int tid = threadIdx.x;
  if (o.chunks == nullptr) return;
  // chunk counts per expert, exclusive scan by thread 0 (E <= 256)
  for (int e = tid; e < E; e += blockDim.x)
    scratch[e] = (cnt[e] + o.chunk_rows - 1) / o.chunk_rows;
  __syncthreads();
  if (tid == 0) {
    int run = 0, active = 0;
    for (int e = 0; e < E; ++e) {
      const int c = scratch[e];
      scratch[e] = run;
      run += c;
      active += cnt[e] > 0;
    }
    scratch[256] = run;
    o.sched[0] = run;
    o.sched[1] = active;
  }
  __syncthreads();
  for (int e = tid; e < E; e += blockDim.x) {
    int base = scratch[e];
    for (int r0 = 0; r0 < cnt[e]; r0 += o.chunk_rows)
      o.chunks[base++] = make_int4(e, off[e] + r0, min(o.chunk_rows, cnt[e] - r0), 0);
  }
}

// ---------------------------------------------------------------------------------------
// Small T (T <= kSmallT): everything after the partial logits, in one block of 1024.
// ---------------------------------------------------------------------------------------
__global__ void __launch_bounds__(1024)
    route_small_finalize_kernel(const float* __restrict__ partial, int S,
                                const float* __restrict__ b_router, int T, int E, int k,
                                RouteOut o) {
  extern __shared__ __align__(128) uint8_t smem_raw[];
  float* lg = reinterpret_cast<float*>(smem_raw);                    // [T][E]
  int32_t* sel = reinterpret_cast<int32_t*>(lg + T * E);             // [T][k]
  uint32_t* bits = reinterpret_cast<uint32_t*>(sel + T * k);         // [T][8]
  int32_t* cnt = reinterpret_cast<int32_t*>(bits + T * 8);           // [256]
  int32_t* off = cnt + 256;                                          // [257]
  int32_t* scratch = off + 257;                                      // [257]
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nwarps = blockDim.x >> 5;

  for (int i = tid; i < T * E; i += blockDim.x) {
    const int e = i % E;
    float v = 0.f;
    for (int s = 0; s < S; ++s) v += partial[(size_t)s * T * E + i];
    lg[i] = v + b_router[e];
  }
  for (int i = tid; i < T * 8; i += blockDim.x) bits[i] = 0u;
  for (int i = tid; i < 256; i += blockDim.x) cnt[i] = 0;
  __syncthreads();

  for (int t = warp; t < T; t += nwarps) {
    float* row = lg + t * E;
    int32_t* srow = sel + t * k;
    warp_topk(row, E, k, srow);
    const float denom = warp_softmax_denominator(row, k);
    float wv[8];  // k <= 256: at most 8 slots per lane
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const int j = lane + 32 * q;
      wv[q] = (j < k) ? expf(row[j] - row[0]) / denom : 0.f;
    }
    __syncwarp();  // every lane has read row[0] before any weight overwrites it
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const int j = lane + 32 * q;
      if (j < k) {
        o.topk_idx[t * k + j] = srow[j];
        o.topk_w[t * k + j] = wv[q];
        row[j] = wv[q];  // keep the weight for the row map below
        atomicAdd(&cnt[srow[j]], 1);
        atomicOr(&bits[t * 8 + (srow[j] >> 5)], 1u << (srow[j] & 31));
      }
    }
  }
  __syncthreads();
  if (tid == 0) {
    int run = 0;
    for (int e = 0; e < E; ++e) {
      off[e] = run;
      run += cnt[e];
    }
    off[E] = run;
  }
  __syncthreads();
  for (int e = tid; e <= E; e += blockDim.x) o.offsets[e] = off[e];
  // stable permutation: rank of (t, e) = number of earlier tokens that chose e
  for (int i = tid; i < T * k; i += blockDim.x) {
    const int t = i / k, e = sel[i];
    const int word = e >> 5;
    const uint32_t bit = 1u << (e & 31);
    int rank = 0;
    for (int t2 = 0; t2 < t; ++t2) rank += (bits[t2 * 8 + word] & bit) ? 1 : 0;
    const int r = off[e] + rank;
    o.perm[r] = t;
    o.inv_perm[i] = r;
    if (o.row_w) o.row_w[r] = lg[t * E + (i - t * k)];
  }
  __syncthreads();
  build_work_list(cnt, off, E, o, scratch);
  for (int i = tid; i < o.n_zero; i += blockDim.x) o.zero_i32[i] = 0;
}

// ---------------------------------------------------------------------------------------
// Large T, step 1: logits of 32 tokens x all E experts over the full H, then top-k,
// softmax and the block's expert histogram.  grid ceil(T/32), block 256.
// Thread (warp w, lane l) owns token l of the tile and experts [w*EPW, (w+1)*EPW).
// ---------------------------------------------------------------------------------------
template <int EPW>
__global__ void __launch_bounds__(256)
    router_topk_kernel(const uint16_t* __restrict__ x, const uint16_t* __restrict__ Wr,
                       const float* __restrict__ b_router, int T, int H, int E, int k,
                       int32_t* __restrict__ topk_idx, float* __restrict__ topk_w,
                       int32_t* __restrict__ block_counts, float4* zero4, size_t n_zero4) {
  zero_fill_f4(zero4, n_zero4);
  extern __shared__ __align__(128) uint8_t smem_raw[];
  uint16_t* xsT = reinterpret_cast<uint16_t*>(smem_raw);          // [64][32] (h-major)
  uint16_t* ws = xsT + kRouterHSlice * kRouteTile;                  // [64][8*EPW]
  const int EP = 8 * EPW;                                           // padded expert count
  float* lg = reinterpret_cast<float*>(ws + kRouterHSlice * EP);    // [32][EP]
  int32_t* cnt = reinterpret_cast<int32_t*>(lg + kRouteTile * EP);  // [EP]
  int32_t* sel = cnt + EP;                                          // [32][k]
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int t0 = blockIdx.x * kRouteTile, nt = min(kRouteTile, T - t0);

  float acc[EPW];
#pragma unroll
  for (int m = 0; m < EPW; ++m) acc[m] = 0.f;
  for (int i = tid; i < EP; i += blockDim.x) cnt[i] = 0;

  for (int h0 = 0; h0 < H; h0 += kRouterHSlice) {
    {  // x tile, transposed to [h][t]
      const int r = tid >> 3, c = tid & 7;  // 32 tokens x 8 chunks of 8
      uint4 v = make_uint4(0, 0, 0, 0);
      if (r < nt) v = reinterpret_cast<const uint4*>(x + (size_t)(t0 + r) * H + h0)[c];
      const uint16_t* pv = reinterpret_cast<const uint16_t*>(&v);
#pragma unroll
      for (int q = 0; q < 8; ++q) xsT[(c * 8 + q) * kRouteTile + r] = pv[q];
    }
    for (int i = tid; i < kRouterHSlice * EP; i += blockDim.x) {
      const int hh = i / EP, e = i - hh * EP;
      ws[i] = (e < E) ? Wr[(size_t)(h0 + hh) * E + e] : uint16_t(0);
    }
    __syncthreads();
#pragma unroll 4
    for (int hh = 0; hh < kRouterHSlice; ++hh) {
      const float xv = bf16_to_f32(xsT[hh * kRouteTile + lane]);
      const uint16_t* wrow = ws + hh * EP + warp * EPW;
      if constexpr (EPW % 4 == 0) {
#pragma unroll
        for (int m = 0; m < EPW; m += 4) {
          const uint2 wv = *reinterpret_cast<const uint2*>(wrow + m);
          acc[m + 0] = fmaf(xv, bf16lo(wv.x), acc[m + 0]);
          acc[m + 1] = fmaf(xv, bf16hi(wv.x), acc[m + 1]);
          acc[m + 2] = fmaf(xv, bf16lo(wv.y), acc[m + 2]);
          acc[m + 3] = fmaf(xv, bf16hi(wv.y), acc[m + 3]);
        }
      } else {
#pragma unroll
        for (int m = 0; m < EPW; ++m) acc[m] = fmaf(xv, bf16_to_f32(wrow[m]), acc[m]);
      }
    }
    __syncthreads();
  }
#pragma unroll
  for (int m = 0; m < EPW; ++m) {
    const int e = warp * EPW + m;
    if (e < E) lg[lane * EP + e] = acc[m] + b_router[e];
  }
  __syncthreads();
  for (int tt = warp; tt < nt; tt += 8) {
    float* row = lg + tt * EP;
    int32_t* srow = sel + tt * k;
    warp_topk(row, E, k, srow);
    const float denom = warp_softmax_denominator(row, k);
    const size_t t = (size_t)(t0 + tt);
    for (int j = lane; j < k; j += 32) {
      topk_idx[t * k + j] = srow[j];
      topk_w[t * k + j] = expf(row[j] - row[0]) / denom;
      atomicAdd(&cnt[srow[j]], 1);
    }
    __syncwarp();
  }
  __syncthreads();
  for (int e = tid; e < E; e += blockDim.x) block_counts[(size_t)blockIdx.x * E + e] = cnt[e];
}

// ---------------------------------------------------------------------------------------
// Large T, step 2: for expert e (one block each) the exclusive prefix of its per-block
// counts, in place, and its total.  block 256.
// ---------------------------------------------------------------------------------------
__global__ void __launch_bounds__(256) route_scan_kernel(int32_t* __restrict__ block_counts,
                                                         int NB, int E,
                                                         int32_t* __restrict__ totals) {
  __shared__ int32_t part[256];
  const int e = blockIdx.x, tid = threadIdx.x;
  const int per = (NB + blockDim.x - 1) / blockDim.x;
  const int b0 = tid * per, b1 = min(NB, b0 + per);
  int s = 0;
  for (int b = b0; b < b1; ++b) s += block_counts[(size_t)b * E + e];
  part[tid] = s;
  __syncthreads();
  if (tid == 0) {
    int run = 0;
    for (int i = 0; i < (int)blockDim.x; ++i) {
      const int v = part[i];
      part[i] = run;
      run += v;
    }
    totals[e] = run;
  }
  __syncthreads();
  int run = part[tid];
  for (int b = b0; b < b1; ++b) {
    const int v = block_counts[(size_t)b * E + e];
    block_counts[(size_t)b * E + e] = run;
    run += v;
  }
}

// ---------------------------------------------------------------------------------------
// Large T, step 3: stable scatter.  Block b handles tokens [32b, 32b+32); warp w takes
// experts w, w+8, ...; lane = token, so a ballot gives each token its rank among the block's
// earlier tokens that chose the same expert.  block 256.
// ---------------------------------------------------------------------------------------
__global__ void __launch_bounds__(256)
    route_scatter_kernel(const int32_t* __restrict__ topk_idx, const float* __restrict__ topk_w,
                         const int32_t* __restrict__ block_base,
                         const int32_t* __restrict__ totals, int T, int E, int k, RouteOut o) {
  extern __shared__ __align__(128) uint8_t smem_raw[];
  int32_t* cnt = reinterpret_cast<int32_t*>(smem_raw);  // [256]
  int32_t* off = cnt + 256;                             // [257]
  int32_t* scratch = off + 257;                         // [257]
  uint32_t* bits = reinterpret_cast<uint32_t*>(scratch + 257);  // [32][8]
  uint8_t* slot = reinterpret_cast<uint8_t*>(bits + kRouteTile * 8);  // [32][E] (k <= 256)
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int t0 = blockIdx.x * kRouteTile, nt = min(kRouteTile, T - t0);

  for (int e = tid; e < E; e += blockDim.x) cnt[e] = totals[e];
  for (int i = tid; i < kRouteTile * 8; i += blockDim.x) bits[i] = 0u;
  __syncthreads();
  if (tid == 0) {
    int run = 0;
    for (int e = 0; e < E; ++e) {
      off[e] = run;
      run += cnt[e];
    }
    off[E] = run;
  }
  for (int i = tid; i < nt * k; i += blockDim.x) {
    const int tt = i / k, j = i - tt * k;
    const int e = topk_idx[(size_t)t0 * k + i];
    atomicOr(&bits[tt * 8 + (e >> 5)], 1u << (e & 31));
    slot[tt * E + e] = (uint8_t)j;
  }
  __syncthreads();
  if (blockIdx.x == 0)
    for (int e = tid; e <= E; e += blockDim.x) o.offsets[e] = off[e];
  for (int e = warp; e < E; e += 8) {
    const bool chose = lane < nt && (bits[lane * 8 + (e >> 5)] & (1u << (e & 31)));
    const uint32_t mask = __ballot_sync(0xffffffffu, chose);
    if (chose) {
      const int rank = __popc(mask & ((1u << lane) - 1u));
      const int r = off[e] + block_base[(size_t)blockIdx.x * E + e] + rank;
      const int t = t0 + lane;
      const int j = slot[lane * E + e];
      o.perm[r] = t;
      o.inv_perm[(size_t)t * k + j] = r;
      if (o.row_w) o.row_w[r] = topk_w[(size_t)t * k + j];
    }
  }
  if (blockIdx.x == 0) build_work_list(cnt, off, E, o, scratch);
  for (int i = blockIdx.x * blockDim.x + tid; i < o.n_zero; i += gridDim.x * blockDim.x)
    o.zero_i32[i] = 0;
}

// Gather of token rows into expert order for the grouped GEMM: x_perm[r] = x[perm[r]].
// One warp per row, 16-byte copies.  grid ceil(R/8), block 256.
__global__ void __launch_bounds__(256) gather_rows_kernel(const uint16_t* __restrict__ x,
                                                          const int32_t* __restrict__ perm,
                                                          int R, int H,
                                                          uint16_t* __restrict__ x_perm) {
  const int r = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  if (r >= R) return;
  const uint4* src = reinterpret_cast<const uint4*>(x + (size_t)perm[r] * H);
  uint4* dst = reinterpret_cast<uint4*>(x_perm + (size_t)r * H);
  for (int c = lane; c < H / 8; c += 32) dst[c] = src[c];
}

}  // namespace moe
