// Routing kernels: router logits, top-k with a softmax over the selected logits, expert
// histogram, offsets, the stable token -> row permutation and the per-path work lists.
//
// The layer routes every token to its top-k experts by router score (top-4 of 32 in the
// Persona Kappa forum post's "Architecture Summary"; top-4 of 128 in the hearth-lean-loomed-v1
// card).  Ties go to the lower expert index; inside an expert's row segment tokens ascend.
//
// Two chains:
//   T <= kSmallT : router_topk_kernel split over the hidden dimension (one block per
//                  kSmallTChunks 64-row slices of W_router, partial logits on the tensor cores;
//                  router_partial_small_kernel, the same products in less shared memory, for
//                  T <= 16) -> route_small_finalize_kernel (one block: sum of the slices, top-k,
//                  softmax, histogram, scan, permutation, work lists), or the streaming gate/up
//                  kernel itself for a few tokens.
//   T >  kSmallT : router_topk_kernel (64 tokens per block, all experts on the tensor cores;
//                  top-k and a block histogram) -> route_scan_kernel (one block per expert:
//                  prefix over blocks) -> route_scatter_kernel (permutation, 64 tokens per
//                  block, two 32-token ballot passes).
#pragma once

#include <climits>

#include "common.cuh"

namespace moe {

// Sum of the S partial logits base[s * stride], s = 0 .. S-1, added in slice order (every
// routing path sums them this way, so all paths select the same experts).  The loads go out up
// to 32 at a time: one round trip to L2 per 32 slices.
MOE_DEVINL float sum_slices(const float* base, size_t stride, int S) {
  constexpr int kBatch = 32;
  float v = 0.f;
  for (int s0 = 0; s0 < S; s0 += kBatch) {
    float p[kBatch];
#pragma unroll
    for (int q = 0; q < kBatch; ++q)
      p[q] = s0 + q < S ? __ldcg(base + (size_t)(s0 + q) * stride) : 0.f;
#pragma unroll
    for (int q = 0; q < kBatch; ++q)
      if (s0 + q < S) v += p[q];
  }
  return v;
}

constexpr int kSmallT = 64;        // largest T handled by the single-block finalize
constexpr int kRouterHSlice = 64;  // W_router rows per router pipeline stage
constexpr int kSmallTChunks = 4;   // T <= kSmallT: 64-row slices of W_router per router block

// Exclusive prefix sum over n <= 256 values by one warp (lane l holds entries 8l .. 8l+7):
// val(e) gives entry e, put(e, prefix) receives its exclusive prefix.  Returns the total on
// every lane.
template <typename Val, typename Put>
MOE_DEVINL int warp_exclusive_scan(int n, Val val, Put put) {
  const int lane = threadIdx.x & 31;
  int loc[8], sum = 0;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int e = lane * 8 + i;
    loc[i] = e < n ? val(e) : 0;
    sum += loc[i];
  }
  int incl = sum;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += y;
  }
  int run = incl - sum;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int e = lane * 8 + i;
    if (e < n) put(e, run);
    run += loc[i];
  }
  return __shfl_sync(0xffffffffu, incl, 31);
}

// One work list: the row segments of the experts whose row count lies in (min_count,
// max_count], cut into chunks of at most chunk_rows rows.  Each expert kernel family walks
// its own list, so the kernel that multiplies an expert's rows is chosen per expert on the
// device, from the histogram.
struct WorkList {
  int4* chunks;        // {expert, first row, rows, first row among the list's rows}
  int32_t* sched;      // [0] number of chunks
  int chunk_rows;
  int min_count, max_count;
};
constexpr int kMaxWorkLists = 3;

// Outputs of routing, all in device memory.
struct RouteOut {
  int32_t* topk_idx;   // [T, k]
  float* topk_w;       // [T, k]
  int32_t* offsets;    // [E + 1]
  int32_t* perm;       // [T * k]
  int32_t* inv_perm;   // [T, k]
  float* row_w;        // [T * k] routing weight of each row (may be null)
  WorkList wl[kMaxWorkLists];
  int n_lists;         // work lists to build (0: routing only)
  int snap;            // 1: let the call's counts move a barely-populated side of a boundary
  int one_of = -1;     // >= 0: the experts of lists one_of and one_of + 1 all go to one of the
                       // two, the upper one if their mean count reaches the boundary
  int32_t* zero_i32;   // region zeroed by the chain (completion counters), may be null
  int n_zero;
  const uint16_t* x;   // with x_perm non-null: copy token rows into expert order
  uint16_t* x_perm;    // [T * k, H]
  int H;
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

// ---------------------------------------------------------------------------------------
// top-k of one token held by one thread (k <= K <= kThreadTopK): bv/be receive the k largest
// of row[0..E) in descending order.  Experts are scanned in ascending order and a later expert
// ranks above a held one only when strictly larger, so equal logits go to the lower expert
// index, as in the warp version above.  Branch-free insertion, all slots in registers.
// ---------------------------------------------------------------------------------------
constexpr int kThreadTopK = 8;

template <int K>
MOE_DEVINL void thread_topk(const float* row, int E, int k, float (&bv)[K], int (&be)[K]) {
#pragma unroll
  for (int j = 0; j < K; ++j) {
    bv[j] = -INFINITY;
    be[j] = -1;  // empty slot
  }
  for (int e = 0; e < E; ++e) {
    const float v = row[e];
    bool gt[K];  // v ranks above slot j (slots past k never do)
#pragma unroll
    for (int j = 0; j < K; ++j) gt[j] = j < k && (be[j] < 0 || v > bv[j]);
    // gt is monotone (gt[j-1] implies gt[j]): slot j takes slot j-1's entry when v ranks above
    // j-1, else v itself when it ranks above j
#pragma unroll
    for (int j = K - 1; j > 0; --j) {
      bv[j] = gt[j - 1] ? bv[j - 1] : (gt[j] ? v : bv[j]);
      be[j] = gt[j - 1] ? be[j - 1] : (gt[j] ? e : be[j]);
    }
    bv[0] = gt[0] ? v : bv[0];
    be[0] = gt[0] ? e : be[0];
  }
}

// In place: the selected logits bv[0..k) (bv[0] the largest) become their softmax weights,
// the denominator summed in slot order.
template <int K>
MOE_DEVINL void thread_softmax(int k, float (&bv)[K]) {
  const float top = bv[0];
  float denom = 0.f;
#pragma unroll
  for (int j = 0; j < K; ++j) {
    bv[j] = (j < k) ? expf(bv[j] - top) : 0.f;
    denom += bv[j];
  }
#pragma unroll
  for (int j = 0; j < K; ++j) bv[j] = bv[j] / denom;
}

// One token per thread: top-k, weights, the token's outputs and the block histogram.
template <int K>
MOE_DEVINL void thread_route_token(const float* row, int E, int k, size_t t,
                                   int32_t* topk_idx, float* topk_w, int32_t* cnt) {
  float bv[K];
  int be[K];
  thread_topk<K>(row, E, k, bv, be);
  thread_softmax<K>(k, bv);
#pragma unroll
  for (int j = 0; j < K; ++j)
    if (j < k) {
      topk_idx[t * k + j] = be[j];
      topk_w[t * k + j] = bv[j];
      atomicAdd(&cnt[be[j]], 1);
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

// Top-k, softmax and the block's expert histogram for up to 64 tokens whose logits (bias added)
// are in shared memory, row stride `ld` (odd, so one-thread-per-token reads are free of bank
// conflicts); one thread per token for k <= kThreadTopK, else one warp.  Ends with the block's
// counts.
MOE_DEVINL void topk_block_epilogue(float* lg, int ld, int nt, int t0, int E, int k, int32_t* sel,
                                    int32_t* cnt, int32_t* topk_idx, float* topk_w,
                                    int32_t* block_counts) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nwarps = blockDim.x >> 5;
  if (k <= kThreadTopK) {  // one thread per token (blockDim >= 64 >= nt)
    if (tid < nt) {
      if (k <= 4)
        thread_route_token<4>(lg + tid * ld, E, k, (size_t)(t0 + tid), topk_idx, topk_w, cnt);
      else
        thread_route_token<8>(lg + tid * ld, E, k, (size_t)(t0 + tid), topk_idx, topk_w, cnt);
    }
    __syncthreads();
    for (int e = tid; e < E; e += blockDim.x) block_counts[(size_t)blockIdx.x * E + e] = cnt[e];
    return;
  }
  for (int tt = warp; tt < nt; tt += nwarps) {
    float* row = lg + tt * ld;
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

// Grid-stride zero fill of a scratch region by every block of the launching kernel.
MOE_DEVINL void zero_fill_f4(float4* z, size_t n4) {
  const size_t nthreads = (size_t)gridDim.x * gridDim.y * blockDim.x;
  const size_t b = (size_t)blockIdx.y * gridDim.x + blockIdx.x;
  for (size_t i = b * blockDim.x + threadIdx.x; i < n4; i += nthreads)
    z[i] = make_float4(0.f, 0.f, 0.f, 0.f);
}

// Which work list takes each expert (fam[e], -1 for an expert without rows): the list whose
// (min_count, max_count] holds its count.  With o.snap, the call's own counts then move experts
// across a boundary between neighbouring lists l (lower) and l + 1, so that an almost uniform
// routing does not split the experts over two half-filled launches:
//   - if the upper side holds no more experts than the lower one and none of them has more than
//     twice the boundary, they all join the lower list;
//   - else, if the lower side holds fewer experts and none of them has half the boundary or
//     less, they all join the upper list.
// With o.one_of = l, the experts of lists l and l + 1 then all go to one of the two: the upper
// one if their mean count is at least the boundary, else the lower one.
// A skewed routing (counts far on both sides) keeps the per-expert choice.  Called by all
// threads of a block; cnt and fam in shared memory (E <= 256).
MOE_DEVINL void assign_families(const int32_t* cnt, int E, const RouteOut& o, int32_t* fam) {
  const int tid = threadIdx.x;
  for (int e = tid; e < E; e += blockDim.x) {
    int f = -1;
    const int c = cnt[e];
    for (int l = 0; l < o.n_lists && c > 0; ++l)
      if (c > o.wl[l].min_count && c <= o.wl[l].max_count) f = l;
    fam[e] = f;
  }
  __syncthreads();
  if (o.snap && tid < 32) {
    const int lane = tid;
    for (int l = 0; l + 1 < o.n_lists; ++l) {
      const int b = o.wl[l].max_count;  // the boundary: lower list takes counts <= b
      int n_lo = 0, n_hi = 0, max_hi = 0, min_lo = INT_MAX;
      for (int e = lane; e < E; e += 32) {
        if (fam[e] == l) {
          ++n_lo;
          min_lo = min(min_lo, cnt[e]);
        } else if (fam[e] == l + 1) {
          ++n_hi;
          max_hi = max(max_hi, cnt[e]);
        }
      }
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) {
        n_lo += __shfl_xor_sync(0xffffffffu, n_lo, off);
        n_hi += __shfl_xor_sync(0xffffffffu, n_hi, off);
        max_hi = max(max_hi, __shfl_xor_sync(0xffffffffu, max_hi, off));
        min_lo = min(min_lo, __shfl_xor_sync(0xffffffffu, min_lo, off));
      }
      int from = -1, to = -1;
      if (n_lo > 0 && n_hi > 0) {
        if (n_hi <= n_lo && max_hi <= 2 * b) from = l + 1, to = l;
        else if (n_lo < n_hi && min_lo > b / 2) from = l, to = l + 1;
      }
      if (from >= 0)
        for (int e = lane; e < E; e += 32)
          if (fam[e] == from) fam[e] = to;
      __syncwarp();
    }
  }
  if (o.one_of >= 0 && tid < 32) {
    const int lane = tid, l = o.one_of;
    const int b = o.wl[l].max_count;
    long long rows = 0;
    int n = 0;
    for (int e = lane; e < E; e += 32)
      if (fam[e] == l || fam[e] == l + 1) {
        ++n;
        rows += cnt[e];
      }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      n += __shfl_xor_sync(0xffffffffu, n, off);
      rows += __shfl_xor_sync(0xffffffffu, rows, off);
    }
    const int to = rows >= (long long)b * n ? l + 1 : l;
    for (int e = lane; e < E; e += 32)
      if (fam[e] == l || fam[e] == l + 1) fam[e] = to;
  }
  __syncthreads();
}

// Work lists of one routing: each expert with rows goes to its list (assign_families), its rows
// split there into entries of at most chunk_rows rows, in expert order.  Each entry is {expert,
// first row, rows, first row among the list's rows} (the last field lets a kernel keep per-row
// scratch for its own rows only).  Called by all threads of a block with count/off in shared
// memory (E <= 256 entries); scratch holds [768] ints of shared memory.
MOE_DEVINL void build_work_lists(const int32_t* cnt, const int32_t* off, int E,
                                 const RouteOut& o, int32_t* scratch) {
  const int tid = threadIdx.x;
  if (o.n_lists == 0) return;
  int32_t* chunk_base = scratch;        // [256] first entry of each expert in its list
  int32_t* row_base = scratch + 256;    // [256] first row of each expert among its list's rows
  int32_t* fam = scratch + 512;         // [256] list of each expert
  assign_families(cnt, E, o, fam);
  // warp l < n_lists: exclusive scans of list l's entries and rows, in expert order
  const int warp = tid >> 5;
  if (warp < o.n_lists) {
    const WorkList& L = o.wl[warp];
    auto member = [&](int e) { return fam[e] == warp; };
    const int total = warp_exclusive_scan(
        E, [&](int e) { return member(e) ? (cnt[e] + L.chunk_rows - 1) / L.chunk_rows : 0; },
        [&](int e, int pre) {
          if (member(e)) chunk_base[e] = pre;
        });
    warp_exclusive_scan(E, [&](int e) { return member(e) ? cnt[e] : 0; },
                        [&](int e, int pre) {
                          if (member(e)) row_base[e] = pre;
                        });
    if ((tid & 31) == 0) L.sched[0] = total;
  }
  __syncthreads();
  for (int e = tid; e < E; e += blockDim.x) {
    const int c = cnt[e], l = fam[e];
    if (l < 0) continue;
    const WorkList& L = o.wl[l];
    int base = chunk_base[e];
    for (int r0 = 0; r0 < c; r0 += L.chunk_rows)
      L.chunks[base++] = make_int4(e, off[e] + r0, min(L.chunk_rows, c - r0), row_base[e] + r0);
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
  int32_t* scratch = off + 257;                                      // [768]
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nwarps = blockDim.x >> 5;
  pdl_wait();
  pdl_launch_next();

  for (int i = tid; i < T * E; i += blockDim.x)
    lg[i] = sum_slices(partial + i, (size_t)T * E, S) + b_router[i % E];
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
  if (warp == 0) {
    const int total = warp_exclusive_scan(E, [&](int e) { return cnt[e]; },
                                          [&](int e, int pre) { off[e] = pre; });
    if (lane == 0) off[E] = total;
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
  build_work_lists(cnt, off, E, o, scratch);
  for (int i = tid; i < o.n_zero; i += blockDim.x) o.zero_i32[i] = 0;
}

// ---------------------------------------------------------------------------------------
// Large T, step 1: logits of 64 tokens x all experts on the tensor cores, then top-k, softmax
// and the block's expert histogram.  grid ceil(T/64), block 128 (4 warps x 16 tokens).
// x[64 tokens x 64] and W_router[64 x E] chunks stream through a 4-deep cp.async ring; each warp multiplies its 16 tokens with all experts (mma.sync m16n8k16, bf16 in,
// fp32 accumulate).  Reading x once is the cost, so the kernel runs at memory speed.
// NT8 = experts / 8 rounded up to a power of two; padding experts are zero and never chosen.
// ---------------------------------------------------------------------------------------
constexpr int kRouterTcTokens = 64;
constexpr int kRouterTcXPitch = 72;  // elements; 144-byte rows keep ldmatrix conflict-free

template <int NT8>
struct RouterTcCfg {
  // cp.async ring depth (chunks of 64 hidden rows); wide expert sets keep two to fit in smem
  static constexpr int kStages = NT8 >= 16 ? 2 : 4;
  static constexpr int EP = NT8 * 8;
  static constexpr int WP = EP + 8;
  static constexpr int kXBytes = kStages * kRouterTcTokens * kRouterTcXPitch * 2;
  static constexpr int kWBytes = kStages * kRouterHSlice * WP * 2;
  static constexpr int kLgBytes = kRouterTcTokens * (EP + 1) * 4;
  static size_t smem(int k) { return kXBytes + kWBytes + kLgBytes + EP * 4 + (size_t)kRouterTcTokens * k * 4; }
};

MOE_DEVINL void cp_async16(void* smem_dst, const void* gsrc, bool valid) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(smem_dst)),
               "l"(gsrc), "r"(valid ? 16 : 0)
               : "memory");
}
MOE_DEVINL void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
MOE_DEVINL void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

template <int NT8>
__global__ void __launch_bounds__(128)
    router_topk_kernel(const uint16_t* __restrict__ x, const uint16_t* __restrict__ Wr,
                       const float* __restrict__ b_router, int T, int H, int E, int k,
                       int32_t* __restrict__ topk_idx, float* __restrict__ topk_w,
                       int32_t* __restrict__ block_counts, float4* zero4, size_t n_zero4,
                       int kc_per_split, float* __restrict__ partial) {
  using C = RouterTcCfg<NT8>;
  constexpr int EP = C::EP, WP = C::WP, XP = kRouterTcXPitch, TT = kRouterTcTokens;
  extern __shared__ __align__(128) uint8_t smem_raw[];
  uint16_t* xs = reinterpret_cast<uint16_t*>(smem_raw);                // [stages][64][XP]
  uint16_t* wsm = reinterpret_cast<uint16_t*>(smem_raw + C::kXBytes);   // [stages][64][WP]
  float* lg = reinterpret_cast<float*>(smem_raw + C::kXBytes + C::kWBytes);  // [64][EP+1]
  int32_t* cnt = reinterpret_cast<int32_t*>(lg + TT * (EP + 1));            // [EP]
  int32_t* sel = cnt + EP;                                                   // [64][k]
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int t0 = blockIdx.x * TT, nt = min(TT, T - t0);
  // this block's slice of the hidden dimension: chunks [kc0, kc0 + nk) of 64 rows
  const int kc0 = blockIdx.y * kc_per_split;
  const int nk = min(H / kRouterHSlice - kc0, kc_per_split);
  const bool vec_w = (E % 8) == 0;

  // x and W_router are the caller's inputs, which no kernel of this library writes: the loads
  // and the products run before the dependency wait, everything this kernel writes after it
  for (int i = tid; i < EP; i += blockDim.x) cnt[i] = 0;
  for (int i = tid; i < C::kStages * kRouterHSlice * WP; i += blockDim.x)
    wsm[i] = 0;  // padding experts stay zero
  __syncthreads();

  auto load_chunk = [&](int kc, int buf) {
    const int h0 = (kc0 + kc) * kRouterHSlice;
    uint16_t* xb = xs + buf * TT * XP;
    for (int i = tid; i < TT * 8; i += blockDim.x) {  // 64 rows x 8 pieces of 16 B
      const int r = i >> 3, c = i & 7;
      const bool ok = r < nt;
      cp_async16(xb + r * XP + c * 8, x + (size_t)(t0 + (ok ? r : 0)) * H + h0 + c * 8, ok);
    }
    uint16_t* wb = wsm + buf * kRouterHSlice * WP;
    if (vec_w) {
      const int per_row = E / 8;
      for (int i = tid; i < kRouterHSlice * per_row; i += blockDim.x) {
        const int r = i / per_row, c = i - r * per_row;
        cp_async16(wb + r * WP + c * 8, Wr + (size_t)(h0 + r) * E + c * 8, true);
      }
    } else {
      for (int i = tid; i < kRouterHSlice * E; i += blockDim.x) {
        const int r = i / E, c = i - r * E;
        wb[r * WP + c] = Wr[(size_t)(h0 + r) * E + c];
      }
    }
  };

  float acc[NT8][4];
#pragma unroll
  for (int n = 0; n < NT8; ++n) acc[n][0] = acc[n][1] = acc[n][2] = acc[n][3] = 0.f;

  // prologue: stages-1 chunks in flight; every iteration commits one group (maybe empty)
#pragma unroll
  for (int p = 0; p < C::kStages - 1; ++p) {
    if (p < nk) load_chunk(p, p);
    cp_async_commit();
  }
  for (int kc = 0; kc < nk; ++kc) {
    const int buf = kc % C::kStages;
    cp_async_wait<C::kStages - 2>();       // chunk kc has landed
    __syncthreads();                       // ... for every thread; buffer kc-1 is free again
    {
      const int nx = kc + C::kStages - 1;
      if (nx < nk) load_chunk(nx, nx % C::kStages);
      cp_async_commit();
    }
    const uint32_t xb = smem_u32(xs + buf * TT * XP);
    const uint32_t wb = smem_u32(wsm + buf * kRouterHSlice * WP);
#pragma unroll
    for (int k16 = 0; k16 < kRouterHSlice / 16; ++k16) {
      const int i = lane >> 3, j = lane & 7;
      uint32_t a0, a1, a2, a3;
      ldsm_x4(xb + ((16 * warp + (i & 1) * 8 + j) * XP + k16 * 16 + (i >> 1) * 8) * 2, a0, a1, a2,
              a3);
#pragma unroll
      for (int n = 0; n < NT8; n += 2) {
        // matrices 0/1: experts [8n, 8n+8) at k 0-7 / 8-15; 2/3: experts [8n+8, 8n+16)
        const int krow = k16 * 16 + (i & 1) * 8 + j;
        const int ncol = 8 * n + ((i >> 1) & 1) * 8;
        uint32_t b0, b1, b2, b3;
        if constexpr (NT8 == 1) {
          ldsm_x2_trans(wb + (krow * WP + ncol) * 2, b0, b1);
          mma_bf16_16816(acc[n], a0, a1, a2, a3, b0, b1);
        } else {
          ldsm_x4_trans(wb + (krow * WP + ncol) * 2, b0, b1, b2, b3);
          mma_bf16_16816(acc[n], a0, a1, a2, a3, b0, b1);
          mma_bf16_16816(acc[n + 1], a0, a1, a2, a3, b2, b3);
        }
      }
    }
  }
  cp_async_wait<0>();
  pdl_wait();
  pdl_launch_next();
  zero_fill_f4(zero4, n_zero4);
  // C fragment: c0,c1 -> token 16w + lane/4, experts 8n + 2(lane%4) + {0,1}; c2,c3 -> token + 8
  if (partial != nullptr) {  // one slice of the hidden dimension: partial logits, no bias
#pragma unroll
    for (int n = 0; n < NT8; ++n)
#pragma unroll
      for (int v = 0; v < 4; ++v) {
        const int tt = 16 * warp + (lane >> 2) + 8 * (v >> 1);
        const int e = 8 * n + 2 * (lane & 3) + (v & 1);
        if (e < E && tt < nt) partial[((size_t)blockIdx.y * T + t0 + tt) * E + e] = acc[n][v];
      }
    return;
  }
#pragma unroll
  for (int n = 0; n < NT8; ++n)
#pragma unroll
    for (int v = 0; v < 4; ++v) {
      const int tt = 16 * warp + (lane >> 2) + 8 * (v >> 1);
      const int e = 8 * n + 2 * (lane & 3) + (v & 1);
      if (e < E) lg[tt * (EP + 1) + e] = acc[n][v] + b_router[e];
    }
  __syncthreads();
  topk_block_epilogue(lg, EP + 1, nt, t0, E, k, sel, cnt, topk_idx, topk_w, block_counts);
}

// Partial logits of a call of at most 16 tokens (grid (1, slices), one hidden-dimension slice
// per block) in little shared memory: one 16-token tile that all four warps share, the experts
// split over the warps (n-tile n on warp n % 4), and pipeline stages of one 16-deep K step (four
// stages, at most 12 KB, up to 64 experts; two, 10 KB, at 128; 18 KB at 256).  Up to 128
// experts a block fits on an SM beside a CTA of the streaming or expert-tile kernels, so its
// loads and products run while the previous call's down kernel still holds the SMs, instead of
// after it.  Every (token, expert) sum takes the same MMAs, on the same operands and in the same
// K order, as in router_topk_kernel, so the partial logits are the same numbers.
constexpr int kRouterSmallT = 16;
constexpr int kRouterSmallXPitch = 24;  // elements; 48-byte rows keep ldmatrix conflict-free
template <int NT8>
struct RouterSmallCfg {
  static constexpr int kStages = NT8 <= 8 ? 4 : 2;
  static constexpr int EP = NT8 * 8;
  static constexpr int WP = EP + 8;
  static constexpr int kXStage = kRouterSmallT * kRouterSmallXPitch;  // elements
  static constexpr int kWStage = 16 * WP;                              // elements
  static constexpr int kSmem = kStages * (kXStage + kWStage) * 2;
};

template <int NT8>
__global__ void __launch_bounds__(128)
    router_partial_small_kernel(const uint16_t* __restrict__ x, const uint16_t* __restrict__ Wr,
                                int T, int H, int E, float4* zero4, size_t n_zero4,
                                int kc_per_split, float* __restrict__ partial) {
  using C = RouterSmallCfg<NT8>;
  constexpr int WP = C::WP, XP = kRouterSmallXPitch;
  constexpr int NW = (NT8 + 3) / 4;  // n-tiles per warp
  extern __shared__ __align__(128) uint8_t smem_raw[];
  uint16_t* xs = reinterpret_cast<uint16_t*>(smem_raw);  // [stages][16][XP]
  uint16_t* wsm = xs + C::kStages * C::kXStage;           // [stages][16][WP]
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  // this block's slice of the hidden dimension: K steps of 16 rows from h_first
  const int kc0 = blockIdx.y * kc_per_split;
  const int nsteps = min(H / kRouterHSlice - kc0, kc_per_split) * (kRouterHSlice / 16);
  const int h_first = kc0 * kRouterHSlice;
  const bool vec_w = (E % 8) == 0;

  // x and W_router are the caller's inputs, which no kernel of this library writes: the loads
  // and the products run before the dependency wait, everything this kernel writes after it
  for (int i = tid; i < C::kStages * C::kWStage; i += blockDim.x) wsm[i] = 0;  // padding experts
  __syncthreads();

  auto load_step = [&](int s, int buf) {
    const int h0 = h_first + 16 * s;
    uint16_t* xb = xs + buf * C::kXStage;
    if (tid < 2 * kRouterSmallT) {  // 16 rows x 2 pieces of 16 B; rows past T are zero-filled
      const int r = tid >> 1, c = tid & 1;
      const bool ok = r < T;
      cp_async16(xb + r * XP + c * 8, x + (size_t)(ok ? r : 0) * H + h0 + c * 8, ok);
    }
    uint16_t* wb = wsm + buf * C::kWStage;
    if (vec_w) {
      const int per_row = E / 8;
      for (int i = tid; i < 16 * per_row; i += blockDim.x) {
        const int r = i / per_row, c = i - r * per_row;
        cp_async16(wb + r * WP + c * 8, Wr + (size_t)(h0 + r) * E + c * 8, true);
      }
    } else {
      for (int i = tid; i < 16 * E; i += blockDim.x) {
        const int r = i / E, c = i - r * E;
        wb[r * WP + c] = Wr[(size_t)(h0 + r) * E + c];
      }
    }
  };

  float acc[NW][4];
#pragma unroll
  for (int j = 0; j < NW; ++j) acc[j][0] = acc[j][1] = acc[j][2] = acc[j][3] = 0.f;
  // prologue: stages-1 steps in flight; every iteration commits one group (maybe empty)
#pragma unroll
  for (int p = 0; p < C::kStages - 1; ++p) {
    if (p < nsteps) load_step(p, p);
    cp_async_commit();
  }
  for (int s = 0; s < nsteps; ++s) {
    const int buf = s % C::kStages;
    cp_async_wait<C::kStages - 2>();  // step s has landed
    __syncthreads();                   // ... for every thread; buffer s-1 is free again
    {
      const int nx = s + C::kStages - 1;
      if (nx < nsteps) load_step(nx, nx % C::kStages);
      cp_async_commit();
    }
    const uint32_t xb = smem_u32(xs + buf * C::kXStage);
    const uint32_t wb = smem_u32(wsm + buf * C::kWStage);
    const int i = lane >> 3, j8 = lane & 7;
    uint32_t a0, a1, a2, a3;
    ldsm_x4(xb + (((i & 1) * 8 + j8) * XP + (i >> 1) * 8) * 2, a0, a1, a2, a3);
#pragma unroll
    for (int j = 0; j < NW; ++j) {
      const int n = warp + 4 * j;
      if (n < NT8) {  // matrices 0/1: experts [8n, 8n+8) at k 0-7 / 8-15
        uint32_t b0, b1;
        ldsm_x2_trans(wb + (((i & 1) * 8 + j8) * WP + 8 * n) * 2, b0, b1);
        mma_bf16_16816(acc[j], a0, a1, a2, a3, b0, b1);
      }
    }
  }
  cp_async_wait<0>();
  pdl_wait();
  pdl_launch_next();
  zero_fill_f4(zero4, n_zero4);
  // C fragment: c0,c1 -> token lane/4, experts 8n + 2(lane%4) + {0,1}; c2,c3 -> token + 8
#pragma unroll
  for (int j = 0; j < NW; ++j)
#pragma unroll
    for (int v = 0; v < 4; ++v) {
      const int n = warp + 4 * j;
      const int tt = (lane >> 2) + 8 * (v >> 1);
      const int e = 8 * n + 2 * (lane & 3) + (v & 1);
      if (n < NT8 && e < E && tt < T) partial[((size_t)blockIdx.y * T + tt) * E + e] = acc[j][v];
    }
}

// Sum of the S partial-logit slices of every (token, expert), in slice order, written in place
// into slice 0 (each thread owns one element).  grid ceil(n/256), block 256.
__global__ void __launch_bounds__(256) sum_partials_kernel(float* __restrict__ partial, int S,
                                                           int n) {
  pdl_wait();
  pdl_launch_next();
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n) return;
  partial[i] = sum_slices(partial + i, (size_t)n, S);
}

// Large T with too few token blocks to fill the GPU: the router kernel runs split over the hidden
// dimension and writes partial logits [S, T, E] (for many slices first summed into slice 0 by
// sum_partials_kernel); this kernel sums the slices it is given in slice order, adds the bias and
// finishes the 64-token block like the fused kernel.  grid ceil(T/64), block 128.
__global__ void __launch_bounds__(128)
    topk_from_partials_kernel(const float* __restrict__ partial, int S,
                              const float* __restrict__ b_router, int T, int E, int k,
                              int32_t* __restrict__ topk_idx, float* __restrict__ topk_w,
                              int32_t* __restrict__ block_counts) {
  extern __shared__ __align__(128) uint8_t smem_raw[];
  const int P = E | 1;                                       // odd row pitch
  float* lg = reinterpret_cast<float*>(smem_raw);           // [64][P]
  int32_t* cnt = reinterpret_cast<int32_t*>(lg + kRouterTcTokens * P);  // [E]
  int32_t* sel = cnt + E;                                    // [64][k]
  const int tid = threadIdx.x;
  const int t0 = blockIdx.x * kRouterTcTokens, nt = min(kRouterTcTokens, T - t0);
  pdl_wait();
  pdl_launch_next();
  for (int i = tid; i < E; i += blockDim.x) cnt[i] = 0;
  // this block's logits are one contiguous run of nt * E floats in every slice; eight
  // independent loads per thread in flight, slices added in order
  const int n = nt * E;
  const float* src = partial + (size_t)t0 * E;
  const size_t TE = (size_t)T * E;
  for (int base = tid; base < n; base += 8 * blockDim.x) {
    float v[8];
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const int i = base + q * blockDim.x;
      v[q] = i < n ? src[i] : 0.f;
    }
    for (int s = 1; s < S; ++s)
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        const int i = base + q * blockDim.x;
        if (i < n) v[q] += src[s * TE + i];
      }
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const int i = base + q * blockDim.x;
      if (i < n) {
        const int tt = i / E, e = i - tt * E;
        lg[tt * P + e] = v[q] + b_router[e];
      }
    }
  }
  __syncthreads();
  topk_block_epilogue(lg, P, nt, t0, E, k, sel, cnt, topk_idx, topk_w, block_counts);
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
  pdl_wait();
  pdl_launch_next();
  const int per = (NB + blockDim.x - 1) / blockDim.x;
  const int b0 = tid * per, b1 = min(NB, b0 + per);
  int s = 0;
  for (int b = b0; b < b1; ++b) s += block_counts[(size_t)b * E + e];
  part[tid] = s;
  __syncthreads();
  if (tid < 32) {  // blockDim.x == 256: one warp scans the 256 partial sums in place
    const int total = warp_exclusive_scan(256, [&](int i) { return part[i]; },
                                          [&](int i, int pre) { part[i] = pre; });
    if (tid == 0) totals[e] = total;
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
// Large T, step 3: stable scatter.  Block b handles the router's tokens [64b, 64b+64); warp w
// takes experts w, w+8, ...; in two passes lane = token (first and second 32 tokens), and a
// ballot gives each token its rank among the block's earlier tokens that chose the expert.
// block 256.
// ---------------------------------------------------------------------------------------
__global__ void __launch_bounds__(256)
    route_scatter_kernel(const int32_t* __restrict__ topk_idx, const float* __restrict__ topk_w,
                         const int32_t* __restrict__ block_base,
                         const int32_t* __restrict__ totals, int T, int E, int k, RouteOut o) {
  constexpr int TT = kRouterTcTokens;
  extern __shared__ __align__(128) uint8_t smem_raw[];
  int32_t* cnt = reinterpret_cast<int32_t*>(smem_raw);  // [256]
  int32_t* off = cnt + 256;                             // [257]
  int32_t* scratch = off + 257;                         // [768]
  uint32_t* bits = reinterpret_cast<uint32_t*>(scratch + 768);  // [64][8]
  uint8_t* slot = reinterpret_cast<uint8_t*>(bits + TT * 8);    // [64][E] (k <= 256)
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int t0 = blockIdx.x * TT, nt = min(TT, T - t0);
  pdl_wait();
  pdl_launch_next();

  for (int e = tid; e < E; e += blockDim.x) cnt[e] = totals[e];
  for (int i = tid; i < TT * 8; i += blockDim.x) bits[i] = 0u;
  __syncthreads();
  if (warp == 0) {
    const int total = warp_exclusive_scan(E, [&](int e) { return cnt[e]; },
                                          [&](int e, int pre) { off[e] = pre; });
    if (lane == 0) off[E] = total;
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
    const int base = off[e] + block_base[(size_t)blockIdx.x * E + e];
    int before = 0;  // tokens of the first pass that chose e
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      const int tt = half * 32 + lane;
      const bool chose = tt < nt && (bits[tt * 8 + (e >> 5)] & (1u << (e & 31)));
      const uint32_t mask = __ballot_sync(0xffffffffu, chose);
      if (chose) {
        const int r = base + before + __popc(mask & ((1u << lane) - 1u));
        const int t = t0 + tt;
        const int j = slot[tt * E + e];
        o.perm[r] = t;
        o.inv_perm[(size_t)t * k + j] = r;
        if (o.row_w) o.row_w[r] = topk_w[(size_t)t * k + j];
      }
      before += __popc(mask);
    }
  }
  if (blockIdx.x == 0) build_work_lists(cnt, off, E, o, scratch);
  for (int i = blockIdx.x * blockDim.x + tid; i < o.n_zero; i += gridDim.x * blockDim.x)
    o.zero_i32[i] = 0;
  if (o.x_perm) {
    // rows in expert order for the grouped GEMM: each token's row is read once and written to
    // its k rows (inv_perm of this block's tokens was written above by this block)
    __syncthreads();
    const int n16 = o.H / 8;  // 16-byte pieces per row
#pragma unroll 4
    for (int i = tid; i < nt * n16; i += blockDim.x) {
      const int tt = i / n16, c = i - tt * n16;
      const size_t t = (size_t)(t0 + tt);
      const uint4 v = reinterpret_cast<const uint4*>(o.x + t * o.H)[c];
      for (int j = 0; j < k; ++j)
        reinterpret_cast<uint4*>(o.x_perm + (size_t)o.inv_perm[t * k + j] * o.H)[c] = v;
    }
  }
}

// Zero-fill of the layer output before its kernel families fork onto two streams (every down
// kernel adds into it).  grid-stride, float4 stores.
__global__ void __launch_bounds__(256) zero_out_kernel(float4* __restrict__ z, size_t n4) {
  pdl_wait();  // the previous call's down kernels may still add into `out`
  pdl_launch_next();
  zero_fill_f4(z, n4);
}

// Rows in expert order for the grouped GEMM when T is small: x_perm[r] = x[perm[r]].
// One warp per row, 16-byte copies.  grid ceil(R/8), block 256.
__global__ void __launch_bounds__(256) gather_rows_kernel(const uint16_t* __restrict__ x,
                                                          const int32_t* __restrict__ perm,
                                                          int R, int H,
                                                          uint16_t* __restrict__ x_perm) {
  const int r = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  pdl_wait();
  pdl_launch_next();
  if (r >= R) return;
  const uint4* src = reinterpret_cast<const uint4*>(x + (size_t)perm[r] * H);
  uint4* dst = reinterpret_cast<uint4*>(x_perm + (size_t)r * H);
  const int n = H / 8;
  int c = lane;
  for (; c + 96 < n; c += 128) {  // four loads in flight before the stores
    const uint4 v0 = src[c], v1 = src[c + 32], v2 = src[c + 64], v3 = src[c + 96];
    dst[c] = v0;
    dst[c + 32] = v1;
    dst[c + 64] = v2;
    dst[c + 96] = v3;
  }
  for (; c < n; c += 32) dst[c] = src[c];
}

}  // namespace moe
