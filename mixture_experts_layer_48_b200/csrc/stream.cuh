// Weight-streaming expert kernels for small token counts.
//
// With a handful of tokens per step each expert sees about one token (the regime the
// hearth-lean-loomed-v1 card describes in "Why 12-16 streams can be slow on Vulkan"), so
// the expert matmuls are matrix-vector products whose cost is reading the touched experts'
// weights once from HBM.  These kernels stream those weights through shared memory at HBM
// bandwidth and apply them to every row routed to the expert.
//
// Layout: a persistent grid (one CTA per SM).  Each CTA has one producer warp and five
// consumer warps around a 4-stage shared-memory ring.  The producer issues TMA tensor loads
// (one destination CTA) of 64-column weight boxes with the 128-byte swizzle, and bulk copies of the
// rows' activations.  Consumer warp w owns box w of a 320-column tile and multiplies it with
// the expert's rows on the tensor cores: the weight block is the 16-row A operand (read with
// ldmatrix.trans, since W is [K, N] with N contiguous), the <= 16 activation rows are the
// 8-wide B operand (mma.sync m16n8k16, bf16 in, fp32 accumulate).  The arithmetic costs a few
// instructions per 16 x 16 x 8 block, so the kernels stay bound by the weight stream.
//
// Work: tiles are (row chunk of one expert, 320-column block); the tiles' K stages form one
// sequence that is cut into equal contiguous ranges, one per CTA (stream-K), so every SM
// streams the same number of bytes whatever the routing.
//
//   gate/up kernel: columns [c0, c0+320) of the gate half AND the same columns of the up half,
//     so a thread holds matching gate and up sums.  A CTA that covers a tile's whole K range
//     applies SwiGLU from registers; otherwise the pieces add their partial sums into an fp32
//     accumulator (zero-filled by the router kernel) with atomics, and the piece that
//     completes the tile's stage count (a release/acquire counter) writes h = silu(g) * u as
//     bf16.  The kernel also zero-fills `out` (before it waits for the routing kernels).
//   down kernel: y = h W_down[e] per row, scaled by the row's routing weight, added into
//     out[token] with fp32 atomics (the combine).
#pragma once

#include "common.cuh"
#include "route.cuh"

namespace moe {

constexpr int kStreamRB = 16;                          // rows per work-list chunk (<= 2 n8 tiles)
constexpr int kStreamWarps = 5;                        // consumer warps
constexpr int kStreamConsumers = 32 * kStreamWarps;
constexpr int kStreamThreads = kStreamConsumers + 32;  // + 1 producer warp
constexpr int kBox = 64;                               // columns per TMA box (128 B)
constexpr int kStreamCols = kBox * kStreamWarps;       // 320 columns per tile
constexpr int kStreamStages = 5;
constexpr int kGateUpKC = 32;                          // W_gate_up rows per stage
constexpr int kDownKC = 64;                            // W_down rows per stage

constexpr int kGUBoxBytes = kGateUpKC * kBox * 2;                  // 4 KB
constexpr int kDNBoxBytes = kDownKC * kBox * 2;                    // 8 KB
constexpr int kGUStageW = 2 * kStreamWarps * kGUBoxBytes;          // gate + up boxes, 40 KB
constexpr int kDNStageW = kStreamWarps * kDNBoxBytes;              // 40 KB
constexpr int kGUXPitch = kGateUpKC * 2 + 16;                      // activation row pitch (bytes)
constexpr int kDNXPitch = kDownKC * 2 + 16;                        // padded: conflict-free ldmatrix
constexpr int kGUStageX = kStreamRB * kGUXPitch;
constexpr int kDNStageX = kStreamRB * kDNXPitch;
constexpr int kFusedRouteT = 8;       // largest call whose routing the gate/up kernel finishes
constexpr int kFusedRouteRows = 64;   // ... with at most this many routed rows
constexpr int kFusedRouteSmem = kFusedRouteRows * (16 + 4) + 16;  // its work list and row map
constexpr int kGateUpSmem = 1024 + kStreamStages * (kGUStageW + kGUStageX) + 2 * kStreamStages * 8 +
                            kFusedRouteSmem;
constexpr int kDownSmem = 1024 + kStreamStages * (kDNStageW + kDNStageX) + 2 * kStreamStages * 8;
static_assert(kGUStageW % 1024 == 0 && kDNStageW % 1024 == 0, "128B-swizzle atoms need 1 KB");
static_assert(kGUXPitch % 16 == 0 && kDNXPitch % 16 == 0, "bulk copy alignment");

// Stream-K work split: the (tile, K stage) pairs of all tiles form one sequence of
// units * nk stages; CTA b takes the contiguous range [b*total/G, (b+1)*total/G).  Every CTA
// streams the same number of weight bytes (to one stage); a tile's K range may be shared by
// two or three CTAs, whose partial sums meet in fp32 atomics.
struct StreamKRange {
  long long g0, g1;
};
MOE_DEVINL StreamKRange stream_k_range(long long units, int nk) {
  const long long total = units * nk;
  return StreamKRange{total * blockIdx.x / gridDim.x, total * (blockIdx.x + 1) / gridDim.x};
}

struct GateUpArgs {
  const uint16_t* x;     // [T, H]
  int H, I, R;
  const int32_t* perm;   // [R]
  const int4* chunks;    // work list {expert, first row, rows, first row among the list's rows}
  const int32_t* sched;  // [0] chunk count
  float* acc;            // [rows of the list, 2I] gate | up sums (row = entry .w + r), zero on entry
  int32_t* done;         // [chunks * tiles] completion counters, zero on entry
  uint16_t* h;           // [R, I] bf16 SwiGLU output
  float* out;            // [T, H] zero-filled here
  size_t out_elems;
  uint32_t* status;
};

// Routing of a call of at most kFusedRouteT tokens (and T*k <= kFusedRouteRows rows), done by
// every CTA of the gate/up kernel from the router's partial logits instead of by a finalize
// kernel between them: the sum of the slices in slice order, top-k, softmax, histogram, scan,
// the stable permutation and the work list, in shared memory, with the same functions and the
// same order of operations as route_small_finalize_kernel (so the results are identical).  Every
// CTA needs the work list before its first copy; CTA 0 also writes the routing results for the
// caller and the down kernel.  Each touched expert holds at most T <= 16 rows: one entry.
struct StreamRoute {
  const float* partial;   // [S][T][E] partial logits; null: the routing kernels built the list
  int S;
  const float* b_router;  // [E]
  int T, E, k;
  RouteOut o;             // topk_idx, topk_w, offsets, perm, inv_perm, row_w, wl[0]
};

struct DownArgs {
  const uint16_t* h;     // [R, I]
  int H, I, R;
  const int32_t* perm;   // [R]
  const float* row_w;    // [R]
  const int4* chunks;
  const int32_t* sched;
  float* out;            // [T, H], zero on entry
  uint32_t* status;
};

MOE_DEVINL void record_timeout(uint32_t* status) { atomicOr(status, kStatusTimeout); }

// Byte offset, inside a [rows][64] bf16 box stored with the 128-byte swizzle, of the 16-byte
// chunk that lane provides to ldmatrix.x4.trans for m-tile mt (16 columns) and k-step ks
// (16 rows).  Matrices: 0 (cols 0-7, rows 0-7), 1 (cols 8-15, rows 0-7), 2 (cols 0-7,
// rows 8-15), 3 (cols 8-15, rows 8-15) -- the order of the A fragment registers.
MOE_DEVINL uint32_t a_frag_offset(int lane, int mt, int ks) {
  const int i = lane >> 3, j = lane & 7;
  const int krow = ks * 16 + (i >> 1) * 8 + j;
  const int chunk = 2 * mt + (i & 1);
  return (uint32_t)(krow * 128 + ((chunk ^ j) << 4));
}

// Byte offset of the 16-byte activation chunk lane provides to ldmatrix (B operand):
// matrices 0/1 = rows 0-7 at k 0-7 / 8-15, matrices 2/3 = rows 8-15 likewise.
MOE_DEVINL uint32_t b_frag_offset(int lane, int ks, int pitch) {
  const int row = (lane & 7) + ((lane >> 4) << 3);
  return (uint32_t)(row * pitch + (ks * 16 + ((lane >> 3) & 1) * 8) * 2);
}

// ------------------------------------------------------------------------------------------
// gate/up projection + SwiGLU
// ------------------------------------------------------------------------------------------
template <int NB>
MOE_DEVINL void gateup_stage_mma(uint32_t wbase, uint32_t xbase, int warp_c, int lane,
                                 float (&accg)[4][2][4], float (&accu)[4][2][4]) {
  const uint32_t gbox = wbase + warp_c * kGUBoxBytes;
  const uint32_t ubox = wbase + (kStreamWarps + warp_c) * kGUBoxBytes;
#pragma unroll
  for (int ks = 0; ks < kGateUpKC / 16; ++ks) {
    uint32_t b[2][2];
    const uint32_t baddr = xbase + b_frag_offset(lane, ks, kGUXPitch);
    if constexpr (NB == 1) {
      ldsm_x2(baddr, b[0][0], b[0][1]);
    } else {
      ldsm_x4(baddr, b[0][0], b[0][1], b[1][0], b[1][1]);
    }
#pragma unroll
    for (int mt = 0; mt < 4; ++mt) {
      const uint32_t off = a_frag_offset(lane, mt, ks);
      uint32_t a0, a1, a2, a3;
      ldsm_x4_trans(gbox + off, a0, a1, a2, a3);
#pragma unroll
      for (int nb = 0; nb < NB; ++nb)
        mma_bf16_16816(accg[mt][nb], a0, a1, a2, a3, b[nb][0], b[nb][1]);
      ldsm_x4_trans(ubox + off, a0, a1, a2, a3);
#pragma unroll
      for (int nb = 0; nb < NB; ++nb)
        mma_bf16_16816(accu[mt][nb], a0, a1, a2, a3, b[nb][0], b[nb][1]);
    }
  }
}

// What the fused routing keeps in shared memory past the prologue (its scratch is the ring).
struct FusedRouteSmem {
  int4 chunks[kFusedRouteRows];     // the streaming work list
  int32_t perm[kFusedRouteRows];    // row -> token
  int32_t n_chunks;
};
static_assert(sizeof(FusedRouteSmem) <= kFusedRouteSmem, "fused routing shared memory");

// The routing finish of StreamRoute, by every thread of the block.  scratch: at least
// (T*E + T*k + 256 + 257 + 256) * 4 bytes of shared memory that nothing else uses until the
// barrier this function ends with.
MOE_DEVINL void fused_route_cta(const StreamRoute& r, uint8_t* scratch, FusedRouteSmem& fs) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nwarps = blockDim.x >> 5;
  const int T = r.T, E = r.E, k = r.k, S = r.S;
  const bool writer = blockIdx.x == 0;
  const RouteOut& o = r.o;
  float* lg = reinterpret_cast<float*>(scratch);           // [T][E]
  int32_t* sel = reinterpret_cast<int32_t*>(lg + T * E);   // [T][k]
  int32_t* cnt = sel + T * k;                              // [256]
  int32_t* off = cnt + 256;                                // [257]
  int32_t* first = off + 257;                              // [256] list entry of each expert
  for (int i = tid; i < T * E; i += blockDim.x)  // slices in order, as the finalize kernel
    lg[i] = sum_slices(r.partial + i, (size_t)T * E, S) + r.b_router[i % E];
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
        if (writer) {
          o.topk_idx[t * k + j] = srow[j];
          o.topk_w[t * k + j] = wv[q];
        }
        row[j] = wv[q];  // the weight, for the row map below
        atomicAdd(&cnt[srow[j]], 1);
      }
    }
  }
  __syncthreads();
  if (warp == 0) {
    const int total = warp_exclusive_scan(E, [&](int e) { return cnt[e]; },
                                          [&](int e, int pre) { off[e] = pre; });
    const int n = warp_exclusive_scan(E, [&](int e) { return cnt[e] > 0 ? 1 : 0; },
                                      [&](int e, int pre) { first[e] = pre; });
    if (lane == 0) {
      off[E] = total;
      fs.n_chunks = n;
    }
  }
  __syncthreads();
  // stable permutation: rank of (t, e) = earlier tokens that chose e (a token's k are distinct)
  for (int i = tid; i < T * k; i += blockDim.x) {
    const int t = i / k, e = sel[i];
    int rank = 0;
    for (int i2 = 0; i2 < t * k; ++i2) rank += sel[i2] == e ? 1 : 0;
    const int rw = off[e] + rank;
    fs.perm[rw] = t;
    if (writer) {
      o.perm[rw] = t;
      o.inv_perm[i] = rw;
      if (o.row_w) o.row_w[rw] = lg[t * E + (i - t * k)];
    }
  }
  for (int e = tid; e < E; e += blockDim.x)
    if (cnt[e] > 0) {  // one entry per touched expert (at most T <= 16 rows)
      const int4 ch = make_int4(e, off[e], cnt[e], off[e]);
      fs.chunks[first[e]] = ch;
      if (writer) o.wl[0].chunks[first[e]] = ch;
    }
  if (writer) {
    for (int e = tid; e <= E; e += blockDim.x) o.offsets[e] = off[e];
    if (tid == 0) o.wl[0].sched[0] = fs.n_chunks;
  }
  fence_proxy_async_smem();  // the ring's copies overwrite the scratch next
  __syncthreads();
}

// The weight tensor map views W_gate_up as [E*H rows, 2I columns], box [32 x 64], 128B swizzle.
__global__ void __launch_bounds__(kStreamThreads, 1)
    stream_gate_up_kernel(const GateUpArgs a, const StreamRoute r,
                          const __grid_constant__ CUtensorMap wmap) {
  extern __shared__ __align__(128) uint8_t smem_raw[];
  __shared__ int s_last;
  uint8_t* wring = align1k(smem_raw);
  uint8_t* xring = wring + kStreamStages * kGUStageW;
  uint64_t* full = reinterpret_cast<uint64_t*>(xring + kStreamStages * kGUStageX);
  uint64_t* empty = full + kStreamStages;
  FusedRouteSmem* fs = reinterpret_cast<FusedRouteSmem*>(empty + kStreamStages);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) {
    for (int s = 0; s < kStreamStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kStreamWarps);
    }
    fence_barrier_init();
  }
  __syncthreads();

  if (tid == 32 * kStreamWarps) tma_prefetch_desc(&wmap);
  // `out` is written only by this call's down kernel, which cannot start before this one
  {
    float4* o4 = reinterpret_cast<float4*>(a.out);
    const size_t n4 = a.out_elems / 4;
    for (size_t i = (size_t)blockIdx.x * blockDim.x + tid; i < n4; i += (size_t)gridDim.x * blockDim.x)
      o4[i] = make_float4(0.f, 0.f, 0.f, 0.f);
  }
  pdl_wait();  // the routing results below come from the previous kernels
  pdl_launch_next();

  const int4* chunks = a.chunks;
  const int32_t* perm = a.perm;
  int n_chunks;
  if (r.partial != nullptr) {  // finish the routing here (every CTA the same way)
    fused_route_cta(r, wring, *fs);
    chunks = fs->chunks;
    perm = fs->perm;
    n_chunks = fs->n_chunks;
  } else {
    n_chunks = a.sched[0];
  }
  const int I2 = 2 * a.I;
  const int NT = (a.I + kStreamCols - 1) / kStreamCols;
  const int nk = a.H / kGateUpKC;
  const StreamKRange rng = stream_k_range((long long)n_chunks * NT, nk);

  if (warp == kStreamWarps) {
    // ---------------- producer ----------------
    bool aborted = false;
    uint32_t it = 0;
    int last_it[kStreamStages];
#pragma unroll
    for (int s = 0; s < kStreamStages; ++s) last_it[s] = -1;
    for (long long g = rng.g0; g < rng.g1;) {
      const int unit = (int)(g / nk), kb = (int)(g % nk);
      const int ke = (int)min((long long)nk, kb + (rng.g1 - g));
      g += ke - kb;
      const int4 ch = chunks[unit / NT];
      const int col0 = (unit % NT) * kStreamCols;
      const int tok = (lane < ch.z) ? perm[ch.y + lane] : 0;
      // lanes 0-4 load gate boxes, lanes 5-9 the matching up boxes
      const int box_col = lane < kStreamWarps ? col0 + kBox * lane
                                              : a.I + col0 + kBox * (lane - kStreamWarps);
      const uint32_t bytes = (uint32_t)kGUStageW + (uint32_t)ch.z * kGateUpKC * 2u;
      for (int kst = kb; kst < ke; ++kst, ++it) {
        const int slot = it % kStreamStages;
        const uint32_t ph = (it / kStreamStages) & 1u;
        if (!aborted && lane == 0 && !mbar_wait_bounded(&empty[slot], ph ^ 1u, kWaitLimitNs)) {
          aborted = true;
          record_timeout(a.status);
        }
        aborted = __shfl_sync(0xffffffffu, aborted, 0);
        if (aborted) continue;
        if (lane == 0) mbar_arrive_expect_tx(&full[slot], bytes);
        __syncwarp();
        const int k0 = kst * kGateUpKC;
        if (lane < 2 * kStreamWarps)
          tma_load_2d(wring + slot * kGUStageW + lane * kGUBoxBytes, &wmap, box_col,
                      ch.x * a.H + k0, &full[slot]);
        if (lane < ch.z)
          bulk_g2s(xring + slot * kGUStageX + lane * kGUXPitch, a.x + (size_t)tok * a.H + k0,
                   kGateUpKC * 2, &full[slot]);
        last_it[slot] = it;
      }
    }
    // never leave the CTA with copies in flight
    if (lane == 0) {
      for (int s = 0; s < kStreamStages; ++s)
        if (last_it[s] >= 0 &&
            !mbar_wait_bounded(&full[s], (last_it[s] / kStreamStages) & 1u, kWaitLimitNs))
          record_timeout(a.status);
    }
    return;
  }

  // ---------------- consumers ----------------
  const int ctid = tid;  // 0..159; warp = box index
  const uint32_t wring_s = smem_u32(wring), xring_s = smem_u32(xring);
  bool aborted = false;
  uint32_t it = 0;
  for (long long g = rng.g0; g < rng.g1;) {
    const int unit = (int)(g / nk), kb = (int)(g % nk);
    const int ke = (int)min((long long)nk, kb + (rng.g1 - g));
    g += ke - kb;
    const int4 ch = chunks[unit / NT];
    const int col0 = (unit % NT) * kStreamCols;
    const int wg = min(kStreamCols, a.I - col0);
    const int nrows = ch.z;
    float accg[4][2][4], accu[4][2][4];
#pragma unroll
    for (int mt = 0; mt < 4; ++mt)
#pragma unroll
      for (int nb = 0; nb < 2; ++nb)
#pragma unroll
        for (int v = 0; v < 4; ++v) accg[mt][nb][v] = accu[mt][nb][v] = 0.f;

    for (int kst = kb; kst < ke; ++kst, ++it) {
      const int slot = it % kStreamStages;
      const uint32_t ph = (it / kStreamStages) & 1u;
      if (!aborted && !mbar_wait_bounded(&full[slot], ph, kWaitLimitNs)) {
        aborted = true;
        record_timeout(a.status);
      }
      if (!aborted) {
        const uint32_t wb = wring_s + slot * kGUStageW, xb = xring_s + slot * kGUStageX;
        if (nrows <= 8)
          gateup_stage_mma<1>(wb, xb, warp, lane, accg, accu);
        else
          gateup_stage_mma<2>(wb, xb, warp, lane, accg, accu);
      }
      __syncwarp();
      if (lane == 0 && !aborted) mbar_arrive(&empty[slot]);
    }
    // every consumer warp walks the same units and takes the barriers below even after giving
    // up on a wait (skipping only the data work), so no warp is left at a barrier

    // ---- epilogue: C fragment (m = weight column, n = row) ----
    // value v of tile (mt, nb): column 64*warp + 16*mt + (lane>>2) + 8*(v>>1),
    //                           row nb*8 + 2*(lane&3) + (v&1)
    if (kb == 0 && ke == nk) {  // this CTA holds the whole K range: SwiGLU from registers
#pragma unroll
      for (int mt = 0; mt < 4; ++mt)
#pragma unroll
        for (int nb = 0; nb < 2; ++nb)
#pragma unroll
          for (int v = 0; v < 4; ++v) {
            const int cl = kBox * warp + 16 * mt + (lane >> 2) + 8 * (v >> 1);
            const int r = nb * 8 + 2 * (lane & 3) + (v & 1);
            if (!aborted && r < nrows && cl < wg) {
              const float hv = silu_f32(accg[mt][nb][v]) * accu[mt][nb][v];
              a.h[(size_t)(ch.y + r) * a.I + col0 + cl] = (uint16_t)f32_to_bf16_bits(hv);
            }
          }
      continue;
    }
#pragma unroll
    for (int mt = 0; mt < 4; ++mt)
#pragma unroll
      for (int nb = 0; nb < 2; ++nb)
#pragma unroll
        for (int v = 0; v < 4; ++v) {
          const int cl = kBox * warp + 16 * mt + (lane >> 2) + 8 * (v >> 1);
          const int r = nb * 8 + 2 * (lane & 3) + (v & 1);
          if (!aborted && r < nrows && cl < wg) {
            float* p = a.acc + ((size_t)ch.w + r) * I2 + col0 + cl;
            atomicAdd(p, accg[mt][nb][v]);
            atomicAdd(p + a.I, accu[mt][nb][v]);
          }
        }
    // Completion count in K stages: the piece that brings it to nk applies SwiGLU.  The
    // barrier orders every thread's atomics before thread 0's release; thread 0's acquire
    // and the second barrier order the last piece's reads after all other pieces' atomics.
    named_bar_sync(1, kStreamConsumers);
    if (ctid == 0)
      s_last = !aborted && atom_add_acq_rel_gpu(&a.done[unit], ke - kb) + (ke - kb) == nk;
    named_bar_sync(1, kStreamConsumers);
    if (s_last) {
      for (int i = ctid; i < nrows * (wg / 2); i += kStreamConsumers) {
        const int r = i / (wg / 2), cl = 2 * (i - r * (wg / 2));
        const float* p = a.acc + ((size_t)ch.w + r) * I2 + col0 + cl;
        const float2 gs = __ldcg(reinterpret_cast<const float2*>(p));
        const float2 us = __ldcg(reinterpret_cast<const float2*>(p + a.I));
        *reinterpret_cast<uint32_t*>(a.h + (size_t)(ch.y + r) * a.I + col0 + cl) =
            pack_bf16x2(silu_f32(gs.x) * us.x, silu_f32(gs.y) * us.y);
      }
    }
  }
}

// ------------------------------------------------------------------------------------------
// down projection + routing weight + combine
// ------------------------------------------------------------------------------------------
template <int NB>
MOE_DEVINL void down_stage_mma(uint32_t wbase, uint32_t xbase, int warp_c, int lane,
                               float (&acc)[4][2][4]) {
  const uint32_t box = wbase + warp_c * kDNBoxBytes;
#pragma unroll
  for (int ks = 0; ks < kDownKC / 16; ++ks) {
    uint32_t b[2][2];
    const uint32_t baddr = xbase + b_frag_offset(lane, ks, kDNXPitch);
    if constexpr (NB == 1) {
      ldsm_x2(baddr, b[0][0], b[0][1]);
    } else {
      ldsm_x4(baddr, b[0][0], b[0][1], b[1][0], b[1][1]);
    }
#pragma unroll
    for (int mt = 0; mt < 4; ++mt) {
      uint32_t a0, a1, a2, a3;
      ldsm_x4_trans(box + a_frag_offset(lane, mt, ks), a0, a1, a2, a3);
#pragma unroll
      for (int nb = 0; nb < NB; ++nb)
        mma_bf16_16816(acc[mt][nb], a0, a1, a2, a3, b[nb][0], b[nb][1]);
    }
  }
}

// The weight tensor map views W_down as [E*I rows, H columns], box [64 x 64], 128B swizzle.
__global__ void __launch_bounds__(kStreamThreads, 1)
    stream_down_kernel(const DownArgs a, const __grid_constant__ CUtensorMap wmap) {
  extern __shared__ __align__(128) uint8_t smem_raw[];
  uint8_t* wring = align1k(smem_raw);
  uint8_t* xring = wring + kStreamStages * kDNStageW;
  uint64_t* full = reinterpret_cast<uint64_t*>(xring + kStreamStages * kDNStageX);
  uint64_t* empty = full + kStreamStages;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) {
    for (int s = 0; s < kStreamStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kStreamWarps);
    }
    fence_barrier_init();
  }
  __syncthreads();

  if (tid == 32 * kStreamWarps) tma_prefetch_desc(&wmap);
  pdl_wait();  // h and the work list come from the previous kernels
  pdl_launch_next();

  const int NT = (a.H + kStreamCols - 1) / kStreamCols;
  const int nk = a.I / kDownKC;
  const StreamKRange rng = stream_k_range((long long)a.sched[0] * NT, nk);

  if (warp == kStreamWarps) {
    bool aborted = false;
    uint32_t it = 0;
    int last_it[kStreamStages];
#pragma unroll
    for (int s = 0; s < kStreamStages; ++s) last_it[s] = -1;
    for (long long g = rng.g0; g < rng.g1;) {
      const int unit = (int)(g / nk), kb = (int)(g % nk);
      const int ke = (int)min((long long)nk, kb + (rng.g1 - g));
      g += ke - kb;
      const int4 ch = a.chunks[unit / NT];
      const int col0 = (unit % NT) * kStreamCols;
      const uint32_t bytes = (uint32_t)kDNStageW + (uint32_t)ch.z * kDownKC * 2u;
      for (int kst = kb; kst < ke; ++kst, ++it) {
        const int slot = it % kStreamStages;
        const uint32_t ph = (it / kStreamStages) & 1u;
        if (!aborted && lane == 0 && !mbar_wait_bounded(&empty[slot], ph ^ 1u, kWaitLimitNs)) {
          aborted = true;
          record_timeout(a.status);
        }
        aborted = __shfl_sync(0xffffffffu, aborted, 0);
        if (aborted) continue;
        if (lane == 0) mbar_arrive_expect_tx(&full[slot], bytes);
        __syncwarp();
        const int k0 = kst * kDownKC;
        if (lane < kStreamWarps)
          tma_load_2d(wring + slot * kDNStageW + lane * kDNBoxBytes, &wmap, col0 + kBox * lane,
                      ch.x * a.I + k0, &full[slot]);
        if (lane < ch.z)
          bulk_g2s(xring + slot * kDNStageX + lane * kDNXPitch,
                   a.h + (size_t)(ch.y + lane) * a.I + k0, kDownKC * 2, &full[slot]);
        last_it[slot] = it;
      }
    }
    if (lane == 0) {
      for (int s = 0; s < kStreamStages; ++s)
        if (last_it[s] >= 0 &&
            !mbar_wait_bounded(&full[s], (last_it[s] / kStreamStages) & 1u, kWaitLimitNs))
          record_timeout(a.status);
    }
    return;
  }

  const uint32_t wring_s = smem_u32(wring), xring_s = smem_u32(xring);
  bool aborted = false;
  uint32_t it = 0;
  for (long long g = rng.g0; g < rng.g1;) {
    const int unit = (int)(g / nk), kb = (int)(g % nk);
    const int ke = (int)min((long long)nk, kb + (rng.g1 - g));
    g += ke - kb;
    const int4 ch = a.chunks[unit / NT];
    const int col0 = (unit % NT) * kStreamCols;
    const int wc = min(kStreamCols, a.H - col0);
    const int nrows = ch.z;
    float acc[4][2][4];
#pragma unroll
    for (int mt = 0; mt < 4; ++mt)
#pragma unroll
      for (int nb = 0; nb < 2; ++nb)
#pragma unroll
        for (int v = 0; v < 4; ++v) acc[mt][nb][v] = 0.f;
    for (int kst = kb; kst < ke; ++kst, ++it) {
      const int slot = it % kStreamStages;
      const uint32_t ph = (it / kStreamStages) & 1u;
      if (!aborted && !mbar_wait_bounded(&full[slot], ph, kWaitLimitNs)) {
        aborted = true;
        record_timeout(a.status);
      }
      if (!aborted) {
        const uint32_t wb = wring_s + slot * kDNStageW, xb = xring_s + slot * kDNStageX;
        if (nrows <= 8)
          down_stage_mma<1>(wb, xb, warp, lane, acc);
        else
          down_stage_mma<2>(wb, xb, warp, lane, acc);
      }
      __syncwarp();
      if (lane == 0 && !aborted) mbar_arrive(&empty[slot]);
    }
    if (aborted) continue;
    // rows this thread holds: nb*8 + 2*(lane&3) + {0,1}
    int tok[2][2];
    float wt[2][2];
#pragma unroll
    for (int nb = 0; nb < 2; ++nb)
#pragma unroll
      for (int q = 0; q < 2; ++q) {
        const int r = nb * 8 + 2 * (lane & 3) + q;
        tok[nb][q] = r < nrows ? a.perm[ch.y + r] : -1;
        wt[nb][q] = r < nrows ? a.row_w[ch.y + r] : 0.f;
      }
#pragma unroll
    for (int mt = 0; mt < 4; ++mt)
#pragma unroll
      for (int nb = 0; nb < 2; ++nb)
#pragma unroll
        for (int v = 0; v < 4; ++v) {
          const int cl = kBox * warp + 16 * mt + (lane >> 2) + 8 * (v >> 1);
          const int t = tok[nb][v & 1];
          if (t >= 0 && cl < wc)
            atomicAdd(a.out + (size_t)t * a.H + col0 + cl, wt[nb][v & 1] * acc[mt][nb][v]);
        }
  }
}

}  // namespace moe
