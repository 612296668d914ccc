// Kernels for running the layer with its experts split across GPUs (expert parallelism).
//
// With E/G experts per GPU, each GPU routes its own tokens, sends every routed row to the GPU
// that owns the row's expert (dispatch), multiplies the rows it receives by its own experts,
// and sends the weighted results back to the rows' home GPU, which adds a token's k results
// (combine).  The pages' runs kept every expert on each GPU (the Persona Kappa forum post's
// training config sets an expert-parallel degree of 1); splitting them cuts the expert weight
// bytes each GPU streams in decode by G.  The exchange itself is two all-to-all steps over
// NVLink driven by the host; these kernels are the device work on either side of it:
//
//   permute_rows_kernel      rows in expert order, x_perm[r] = x[perm[r]], and each row's
//                            routing weight (sent with the row)
//   build_segment_lists_kernel   work lists of the received rows: they arrive as segments
//                            (source GPU, expert), source-major; an expert's kernel family is
//                            chosen from its rows over all sources (assign_families), each
//                            segment makes its own chunks; also the identity row map of the
//                            expert kernels' output
//   combine_rows_kernel      out[t] = sum_j y[inv_perm[t, j]] in slot order j
#pragma once

#include "common.cuh"
#include "route.cuh"

namespace moe {

constexpr uint32_t kStatusBadIndex = 2u;   // a row index outside its buffer (skipped)
constexpr uint32_t kStatusBadCounts = 4u;  // segment counts that do not sum to the row count

// x_perm[r] = x[perm[r]] and row_w[r] = topk_w[perm[r], j] for the slot j with
// inv_perm[perm[r], j] == r.  One warp per row, 16-byte copies.  grid ceil(R/8), block 256.
__global__ void __launch_bounds__(256)
    permute_rows_kernel(const uint16_t* __restrict__ x, const int32_t* __restrict__ perm,
                        const int32_t* __restrict__ inv_perm, const float* __restrict__ topk_w,
                        int T, int k, int H, uint16_t* __restrict__ x_perm,
                        float* __restrict__ row_w, uint32_t* status) {
  const int r = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  pdl_wait();
  pdl_launch_next();
  const int R = T * k;
  if (r >= R) return;
  const int t = perm[r];
  if (t < 0 || t >= T) {
    if (lane == 0) atomicOr(status, kStatusBadIndex);
    return;
  }
  for (int j = lane; j < k; j += 32)
    if (inv_perm[(size_t)t * k + j] == r) row_w[r] = topk_w[(size_t)t * k + j];
  const uint4* src = reinterpret_cast<const uint4*>(x + (size_t)t * H);
  uint4* dst = reinterpret_cast<uint4*>(x_perm + (size_t)r * H);
  for (int c = lane; c < H / 8; c += 32) dst[c] = src[c];
}

// out[t, :] = sum over j < k of y[inv_perm[t, j], :], added in slot order.  One warp per token,
// 16-byte loads.  grid ceil(T/8), block 256.
__global__ void __launch_bounds__(256)
    combine_rows_kernel(const int32_t* __restrict__ inv_perm, const float* __restrict__ y,
                        int T, int k, int H, float* __restrict__ out, uint32_t* status) {
  const int t = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  pdl_wait();
  pdl_launch_next();
  if (t >= T) return;
  const long long R = (long long)T * k;
  float4* dst = reinterpret_cast<float4*>(out + (size_t)t * H);
  for (int c = lane; c < H / 4; c += 32) {
    float4 s = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int j = 0; j < k; ++j) {
      const int r = inv_perm[(size_t)t * k + j];
      if (r < 0 || r >= R) {
        atomicOr(status, kStatusBadIndex);
        continue;
      }
      const float4 v = reinterpret_cast<const float4*>(y + (size_t)r * H)[c];
      s.x += v.x;
      s.y += v.y;
      s.z += v.z;
      s.w += v.w;
    }
    dst[c] = s;
  }
}

constexpr int kMaxSegments = 4096;  // sources x experts of one expert-half call

// Work lists of R received rows that arrive as S*E segments, seg_counts[s][e] rows of expert e
// from source s, in (s, e) order.  Block 0 builds the lists (family of expert e from its total
// over all sources); every block writes part of the identity row map perm[r] = r and zeroes the
// completion counters.  Counts that do not add up to R are reported in the status word; rows
// past R are never listed.  Also zero-fills zero4[0, n_zero4).  block 1024; dynamic smem
// (4*S*E + 2*E) ints.
__global__ void __launch_bounds__(1024)
    build_segment_lists_kernel(const int32_t* __restrict__ seg_counts, int S, int E, int R,
                               RouteOut o, int32_t* __restrict__ perm_iota, float4* zero4,
                               size_t n_zero4, uint32_t* status) {
  extern __shared__ int32_t seg_smem[];
  const int n = S * E;
  int32_t* seg_off = seg_smem;   // [n] first row of each segment
  int32_t* cnt = seg_off + n;    // [n] rows of each segment inside [0, R)
  int32_t* base = cnt + n;       // [n] first work-list entry of each segment
  int32_t* rbase = base + n;     // [n] first row of each segment among its list's rows
  int32_t* total = rbase + n;    // [E] rows of each expert over all sources
  int32_t* fam = total + E;      // [E] work list of each expert
  const int tid = threadIdx.x;
  pdl_wait();
  pdl_launch_next();
  for (int i = blockIdx.x * blockDim.x + tid; i < R; i += gridDim.x * blockDim.x) perm_iota[i] = i;
  for (int i = blockIdx.x * blockDim.x + tid; i < o.n_zero; i += gridDim.x * blockDim.x)
    o.zero_i32[i] = 0;
  zero_fill_f4(zero4, n_zero4);  // the streaming family's split-K sums
  if (blockIdx.x != 0) return;
  if (tid == 0) {
    int run = 0;
    for (int i = 0; i < n; ++i) {
      const int c = max(0, seg_counts[i]);
      seg_off[i] = run;
      cnt[i] = min(c, max(0, R - run));
      run += c;
    }
    if (run != R) atomicOr(status, kStatusBadCounts);
  }
  __syncthreads();
  for (int e = tid; e < E; e += blockDim.x) {
    int s_ = 0;
    for (int s = 0; s < S; ++s) s_ += cnt[s * E + e];
    total[e] = s_;
  }
  __syncthreads();
  assign_families(total, E, o, fam);  // an expert's family from its rows over all sources
  // thread l < n_lists: exclusive scan of list l's entries over the segments in order
  if (tid < o.n_lists) {
    const WorkList& L = o.wl[tid];
    int run = 0, rows = 0;
    for (int i = 0; i < n; ++i) {
      if (fam[i % E] == tid) {
        base[i] = run;
        rbase[i] = rows;
        run += (cnt[i] + L.chunk_rows - 1) / L.chunk_rows;
        rows += cnt[i];
      }
    }
    L.sched[0] = run;
  }
  __syncthreads();
  for (int i = tid; i < n; i += blockDim.x) {
    const int e = i % E, c = cnt[i], l = fam[e];
    if (c == 0 || l < 0) continue;
    const WorkList& L = o.wl[l];
    int b = base[i];
    for (int r0 = 0; r0 < c; r0 += L.chunk_rows)
      L.chunks[b++] = make_int4(e, seg_off[i] + r0, min(L.chunk_rows, c - r0), rbase[i] + r0);
  }
}

}  // namespace moe
