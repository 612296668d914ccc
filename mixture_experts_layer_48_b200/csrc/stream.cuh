// Weight-streaming expert kernels for small token counts.
//
// With a handful of tokens per step each expert sees about one token (the regime the
// hearth-lean-loomed-v1 card describes in "Why 12-16 streams can be slow on Vulkan"), so
// the expert matmuls are matrix-vector products whose cost is reading the touched experts'
// weights once from HBM.  These kernels stream those weights through shared memory at full
// HBM bandwidth and apply them to every row routed to the expert.
//
// Layout: a persistent grid (one CTA per SM).  Each CTA has one producer warp that issues
// bulk async copies (cp.async.bulk, 16-byte aligned rows, no multicast) of [KC x 320] weight
// tiles into a 4-stage shared-memory ring, and 5 consumer warps (160 threads, 2 columns each)
// that multiply the tile with the expert's rows (<= 16 per work item) in fp32 using packed
// FFMA2.  Work items are (row chunk of one expert, 320-column tile, K split); the number of
// K splits is chosen on the device from the routing so that every SM gets the same share.
//
//   gate/up kernel: columns [c0, c0+320) of the gate half AND the same columns of the up half,
//     so one item holds matching gate and up sums.  Split partial sums go to a scratch
//     buffer; the last CTA of a (chunk, tile) -- found with a fenced counter -- reduces them
//     and writes h = silu(g) * u as bf16.  It also zero-fills `out` for the next kernel.
//   down kernel: y = h W_down[e] per row, scaled by the row's routing weight, added into
//     out[token] with fp32 vector atomics (the combine).
#pragma once

#include "common.cuh"

namespace moe {

constexpr int kStreamRB = 16;            // rows per work-list chunk
constexpr int kStreamConsumers = 160;    // consumer threads (5 warps)
constexpr int kStreamThreads = 192;      // + 1 producer warp
constexpr int kStreamCols = 320;         // columns per tile (2 per consumer thread)
constexpr int kStreamStages = 4;
constexpr int kGateUpKC = 32;            // W_gate_up rows per stage
constexpr int kDownKC = 64;              // W_down rows per stage
constexpr int kStreamSplitMax = 16;

constexpr int kGateUpStageBytes = 2 * kGateUpKC * kStreamCols * 2 + kStreamRB * kGateUpKC * 2;
constexpr int kDownStageBytes = kDownKC * kStreamCols * 2 + kStreamRB * kDownKC * 2;
constexpr int kGateUpSmem = kStreamStages * kGateUpStageBytes + 2 * kStreamStages * 8;
constexpr int kDownSmem = kStreamStages * kDownStageBytes + 2 * kStreamStages * 8;
static_assert(kGateUpStageBytes % 16 == 0 && kDownStageBytes % 16 == 0, "stage alignment");

struct SplitPlan {
  int S;   // number of K splits (every split non-empty)
  int ks;  // K stages per split (the last may have fewer)
};

// Split count minimising the per-CTA makespan ceil(units*S / G) * ks with ks = ceil(nk/S).
MOE_DEVINL SplitPlan choose_splits(int units, int nk, int G, int smax) {
  SplitPlan best{1, nk};
  long long best_cost = -1;
  const int top = min(smax, nk);
  for (int S = 1; S <= top; ++S) {
    const int ks = (nk + S - 1) / S;
    const int Se = (nk + ks - 1) / ks;
    if (Se != S) continue;  // an equivalent smaller S was already costed
    const long long rounds = ((long long)units * S + G - 1) / G;
    const long long cost = rounds * ks;
    if (best_cost < 0 || cost < best_cost) {
      best_cost = cost;
      best = SplitPlan{S, ks};
    }
  }
  return best;
}

struct GateUpArgs {
  const uint16_t* x;     // [T, H]
  const uint16_t* Wgu;   // [E, H, 2I]
  int H, I, R;
  const int32_t* perm;   // [R]
  const int4* chunks;    // work list
  const int32_t* sched;  // [0] chunk count
  int split_cap;         // largest K split count the scratch buffer holds
  float* part;           // [split_cap, R, 2I] split partial sums (split_cap > 1)
  int32_t* done;         // [chunks * tiles] completion counters, zero on entry
  uint16_t* h;           // [R, I] bf16 SwiGLU output
  float* out;            // [T, H] zero-filled here
  size_t out_elems;
  uint32_t* status;
};

struct DownArgs {
  const uint16_t* h;     // [R, I]
  const uint16_t* Wd;    // [E, I, H]
  int H, I, R;
  const int32_t* perm;   // [R]
  const float* row_w;    // [R]
  const int4* chunks;
  const int32_t* sched;
  float* out;            // [T, H], zero on entry
  uint32_t* status;
};

// Ring bookkeeping shared by the producer and the consumers of one CTA.
struct Ring {
  uint64_t* full;
  uint64_t* empty;
};

MOE_DEVINL void record_timeout(uint32_t* status) { atomicOr(status, kStatusTimeout); }

// ------------------------------------------------------------------------------------------
// gate/up projection + SwiGLU
// ------------------------------------------------------------------------------------------
__global__ void __launch_bounds__(kStreamThreads, 1) stream_gate_up_kernel(const GateUpArgs a) {
  extern __shared__ __align__(128) uint8_t smem_raw[];
  __shared__ int s_last;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem_raw + kStreamStages * kGateUpStageBytes);
  Ring ring{bars, bars + kStreamStages};
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) {
    for (int s = 0; s < kStreamStages; ++s) {
      mbar_init(&ring.full[s], 1);
      mbar_init(&ring.empty[s], kStreamConsumers / 32);
    }
    fence_barrier_init();
  }
  __syncthreads();

  const int I2 = 2 * a.I;
  const int NT = (a.I + kStreamCols - 1) / kStreamCols;
  const int units = a.sched[0] * NT;
  const int nk = a.H / kGateUpKC;
  const SplitPlan plan = choose_splits(units, nk, gridDim.x, a.split_cap);
  const int items = units * plan.S;

  if (warp == 0) {
    // ---------------- producer ----------------
    bool aborted = false;
    uint32_t it = 0;
    int last_it[kStreamStages];
#pragma unroll
    for (int s = 0; s < kStreamStages; ++s) last_it[s] = -1;
    for (int id = blockIdx.x; id < items; id += gridDim.x) {
      const int unit = id / plan.S, sp = id - unit * plan.S;
      const int4 ch = a.chunks[unit / NT];
      const int col0 = (unit % NT) * kStreamCols;
      const int wg = min(kStreamCols, a.I - col0);
      const int kb = sp * plan.ks, ke = min(nk, kb + plan.ks);
      const int tok = (lane < ch.z) ? a.perm[ch.y + lane] : 0;
      const uint32_t bytes = 2u * kGateUpKC * wg * 2u + (uint32_t)ch.z * kGateUpKC * 2u;
      for (int kst = kb; kst < ke; ++kst, ++it) {
        const int slot = it % kStreamStages;
        const uint32_t ph = (it / kStreamStages) & 1u;
        if (!aborted && lane == 0 &&
            !mbar_wait_bounded(&ring.empty[slot], ph ^ 1u, kWaitLimitNs)) {
          aborted = true;
          record_timeout(a.status);
        }
        aborted = __shfl_sync(0xffffffffu, aborted, 0);
        if (aborted) continue;
        uint8_t* stage = smem_raw + slot * kGateUpStageBytes;
        uint16_t* Wg_s = reinterpret_cast<uint16_t*>(stage);
        uint16_t* Wu_s = Wg_s + kGateUpKC * kStreamCols;
        uint16_t* X_s = Wu_s + kGateUpKC * kStreamCols;
        if (lane == 0) mbar_arrive_expect_tx(&ring.full[slot], bytes);
        __syncwarp();
        const int k0 = kst * kGateUpKC;
        const uint16_t* src = a.Wgu + ((size_t)ch.x * a.H + k0 + lane) * I2 + col0;
        bulk_g2s(Wg_s + lane * kStreamCols, src, wg * 2, &ring.full[slot]);
        bulk_g2s(Wu_s + lane * kStreamCols, src + a.I, wg * 2, &ring.full[slot]);
        if (lane < ch.z)
          bulk_g2s(X_s + lane * kGateUpKC, a.x + (size_t)tok * a.H + k0, kGateUpKC * 2,
                   &ring.full[slot]);
        last_it[slot] = it;
      }
    }
    // never leave the CTA with copies in flight
    if (lane == 0) {
      for (int s = 0; s < kStreamStages; ++s)
        if (last_it[s] >= 0 &&
            !mbar_wait_bounded(&ring.full[s], (last_it[s] / kStreamStages) & 1u, kWaitLimitNs))
          record_timeout(a.status);
    }
    return;
  }

  // ---------------- consumers ----------------
  const int ctid = tid - 32;
  {
    float4* o4 = reinterpret_cast<float4*>(a.out);
    const size_t n4 = a.out_elems / 4;
    for (size_t i = (size_t)blockIdx.x * kStreamConsumers + ctid; i < n4;
         i += (size_t)gridDim.x * kStreamConsumers)
      o4[i] = make_float4(0.f, 0.f, 0.f, 0.f);
  }
  bool aborted = false;
  uint32_t it = 0;
  const int c = 2 * ctid;
  for (int id = blockIdx.x; id < items; id += gridDim.x) {
    const int unit = id / plan.S, sp = id - unit * plan.S;
    const int4 ch = a.chunks[unit / NT];
    const int col0 = (unit % NT) * kStreamCols;
    const int wg = min(kStreamCols, a.I - col0);
    const int kb = sp * plan.ks, ke = min(nk, kb + plan.ks);
    const int nrows = ch.z;
    float2 accg[kStreamRB], accu[kStreamRB];
#pragma unroll
    for (int r = 0; r < kStreamRB; ++r) accg[r] = accu[r] = make_float2(0.f, 0.f);

    for (int kst = kb; kst < ke; ++kst, ++it) {
      const int slot = it % kStreamStages;
      const uint32_t ph = (it / kStreamStages) & 1u;
      if (!aborted && !mbar_wait_bounded(&ring.full[slot], ph, kWaitLimitNs)) {
        aborted = true;
        record_timeout(a.status);
      }
      if (!aborted) {
        const uint8_t* stage = smem_raw + slot * kGateUpStageBytes;
        const uint32_t* Wg32 = reinterpret_cast<const uint32_t*>(stage);
        const uint32_t* Wu32 = Wg32 + kGateUpKC * kStreamCols / 2;
        const uint32_t* X32 = Wu32 + kGateUpKC * kStreamCols / 2;
#pragma unroll 2
        for (int kk = 0; kk < kGateUpKC; kk += 2) {
          const uint32_t g0 = Wg32[kk * (kStreamCols / 2) + ctid];
          const uint32_t g1 = Wg32[(kk + 1) * (kStreamCols / 2) + ctid];
          const uint32_t u0 = Wu32[kk * (kStreamCols / 2) + ctid];
          const uint32_t u1 = Wu32[(kk + 1) * (kStreamCols / 2) + ctid];
          const float2 G0 = make_float2(bf16lo(g0), bf16hi(g0));
          const float2 G1 = make_float2(bf16lo(g1), bf16hi(g1));
          const float2 U0 = make_float2(bf16lo(u0), bf16hi(u0));
          const float2 U1 = make_float2(bf16lo(u1), bf16hi(u1));
#pragma unroll
          for (int r = 0; r < kStreamRB; ++r) {
            if (r < nrows) {
              const uint32_t xv = X32[r * (kGateUpKC / 2) + (kk >> 1)];
              const float2 x0 = make_float2(bf16lo(xv), bf16lo(xv));
              const float2 x1 = make_float2(bf16hi(xv), bf16hi(xv));
              accg[r] = __ffma2_rn(x0, G0, accg[r]);
              accg[r] = __ffma2_rn(x1, G1, accg[r]);
              accu[r] = __ffma2_rn(x0, U0, accu[r]);
              accu[r] = __ffma2_rn(x1, U1, accu[r]);
            }
          }
        }
      }
      __syncwarp();
      if (lane == 0 && !aborted) mbar_arrive(&ring.empty[slot]);
    }

    // ---- epilogue ----
    const bool mine = c < wg;
    if (plan.S == 1) {
      if (mine && !aborted) {
#pragma unroll
        for (int r = 0; r < kStreamRB; ++r)
          if (r < nrows) {
            const float hx = silu_f32(accg[r].x) * accu[r].x;
            const float hy = silu_f32(accg[r].y) * accu[r].y;
            *reinterpret_cast<uint32_t*>(a.h + (size_t)(ch.y + r) * a.I + col0 + c) =
                pack_bf16x2(hx, hy);
          }
      }
      continue;
    }
    if (mine) {
#pragma unroll
      for (int r = 0; r < kStreamRB; ++r)
        if (r < nrows) {
          float* p = a.part + ((size_t)sp * a.R + ch.y + r) * I2 + col0 + c;
          *reinterpret_cast<float2*>(p) = accg[r];
          *reinterpret_cast<float2*>(p + a.I) = accu[r];
        }
    }
    __threadfence();
    named_bar_sync(1, kStreamConsumers);
    if (ctid == 0) s_last = (atomicAdd(&a.done[unit], 1) == plan.S - 1);
    named_bar_sync(1, kStreamConsumers);
    if (s_last && mine && !aborted) {
      __threadfence();
      for (int r = 0; r < nrows; ++r) {
        float2 g = make_float2(0.f, 0.f), u = make_float2(0.f, 0.f);
        for (int s = 0; s < plan.S; ++s) {
          const float* p = a.part + ((size_t)s * a.R + ch.y + r) * I2 + col0 + c;
          const float2 pg = ld_cg_f2(p), pu = ld_cg_f2(p + a.I);
          g.x += pg.x; g.y += pg.y;
          u.x += pu.x; u.y += pu.y;
        }
        *reinterpret_cast<uint32_t*>(a.h + (size_t)(ch.y + r) * a.I + col0 + c) =
            pack_bf16x2(silu_f32(g.x) * u.x, silu_f32(g.y) * u.y);
      }
    }
  }
}

// ------------------------------------------------------------------------------------------
// down projection + routing weight + combine
// ------------------------------------------------------------------------------------------
__global__ void __launch_bounds__(kStreamThreads, 1) stream_down_kernel(const DownArgs a) {
  extern __shared__ __align__(128) uint8_t smem_raw[];
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem_raw + kStreamStages * kDownStageBytes);
  Ring ring{bars, bars + kStreamStages};
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) {
    for (int s = 0; s < kStreamStages; ++s) {
      mbar_init(&ring.full[s], 1);
      mbar_init(&ring.empty[s], kStreamConsumers / 32);
    }
    fence_barrier_init();
  }
  __syncthreads();

  const int NT = (a.H + kStreamCols - 1) / kStreamCols;
  const int units = a.sched[0] * NT;
  const int nk = a.I / kDownKC;
  const SplitPlan plan = choose_splits(units, nk, gridDim.x, kStreamSplitMax);
  const int items = units * plan.S;

  if (warp == 0) {
    bool aborted = false;
    uint32_t it = 0;
    int last_it[kStreamStages];
#pragma unroll
    for (int s = 0; s < kStreamStages; ++s) last_it[s] = -1;
    for (int id = blockIdx.x; id < items; id += gridDim.x) {
      const int unit = id / plan.S, sp = id - unit * plan.S;
      const int4 ch = a.chunks[unit / NT];
      const int col0 = (unit % NT) * kStreamCols;
      const int wc = min(kStreamCols, a.H - col0);
      const int kb = sp * plan.ks, ke = min(nk, kb + plan.ks);
      const uint32_t bytes = (uint32_t)kDownKC * wc * 2u + (uint32_t)ch.z * kDownKC * 2u;
      for (int kst = kb; kst < ke; ++kst, ++it) {
        const int slot = it % kStreamStages;
        const uint32_t ph = (it / kStreamStages) & 1u;
        if (!aborted && lane == 0 &&
            !mbar_wait_bounded(&ring.empty[slot], ph ^ 1u, kWaitLimitNs)) {
          aborted = true;
          record_timeout(a.status);
        }
        aborted = __shfl_sync(0xffffffffu, aborted, 0);
        if (aborted) continue;
        uint8_t* stage = smem_raw + slot * kDownStageBytes;
        uint16_t* W_s = reinterpret_cast<uint16_t*>(stage);
        uint16_t* H_s = W_s + kDownKC * kStreamCols;
        if (lane == 0) mbar_arrive_expect_tx(&ring.full[slot], bytes);
        __syncwarp();
        const int k0 = kst * kDownKC;
        const uint16_t* src = a.Wd + ((size_t)ch.x * a.I + k0) * a.H + col0;
        bulk_g2s(W_s + lane * kStreamCols, src + (size_t)lane * a.H, wc * 2, &ring.full[slot]);
        bulk_g2s(W_s + (lane + 32) * kStreamCols, src + (size_t)(lane + 32) * a.H, wc * 2,
                 &ring.full[slot]);
        if (lane < ch.z)
          bulk_g2s(H_s + lane * kDownKC, a.h + (size_t)(ch.y + lane) * a.I + k0, kDownKC * 2,
                   &ring.full[slot]);
        last_it[slot] = it;
      }
    }
    if (lane == 0) {
      for (int s = 0; s < kStreamStages; ++s)
        if (last_it[s] >= 0 &&
            !mbar_wait_bounded(&ring.full[s], (last_it[s] / kStreamStages) & 1u, kWaitLimitNs))
          record_timeout(a.status);
    }
    return;
  }

  const int ctid = tid - 32;
  const int c = 2 * ctid;
  bool aborted = false;
  uint32_t it = 0;
  for (int id = blockIdx.x; id < items; id += gridDim.x) {
    const int unit = id / plan.S, sp = id - unit * plan.S;
    const int4 ch = a.chunks[unit / NT];
    const int col0 = (unit % NT) * kStreamCols;
    const int wc = min(kStreamCols, a.H - col0);
    const int kb = sp * plan.ks, ke = min(nk, kb + plan.ks);
    const int nrows = ch.z;
    float2 acc[kStreamRB];
#pragma unroll
    for (int r = 0; r < kStreamRB; ++r) acc[r] = make_float2(0.f, 0.f);
    for (int kst = kb; kst < ke; ++kst, ++it) {
      const int slot = it % kStreamStages;
      const uint32_t ph = (it / kStreamStages) & 1u;
      if (!aborted && !mbar_wait_bounded(&ring.full[slot], ph, kWaitLimitNs)) {
        aborted = true;
        record_timeout(a.status);
      }
      if (!aborted) {
        const uint8_t* stage = smem_raw + slot * kDownStageBytes;
        const uint32_t* W32 = reinterpret_cast<const uint32_t*>(stage);
        const uint32_t* H32 = W32 + kDownKC * kStreamCols / 2;
#pragma unroll 4
        for (int kk = 0; kk < kDownKC; kk += 2) {
          const uint32_t w0 = W32[kk * (kStreamCols / 2) + ctid];
          const uint32_t w1 = W32[(kk + 1) * (kStreamCols / 2) + ctid];
          const float2 W0 = make_float2(bf16lo(w0), bf16hi(w0));
          const float2 W1 = make_float2(bf16lo(w1), bf16hi(w1));
#pragma unroll
          for (int r = 0; r < kStreamRB; ++r) {
            if (r < nrows) {
              const uint32_t hv = H32[r * (kDownKC / 2) + (kk >> 1)];
              acc[r] = __ffma2_rn(make_float2(bf16lo(hv), bf16lo(hv)), W0, acc[r]);
              acc[r] = __ffma2_rn(make_float2(bf16hi(hv), bf16hi(hv)), W1, acc[r]);
            }
          }
        }
      }
      __syncwarp();
      if (lane == 0 && !aborted) mbar_arrive(&ring.empty[slot]);
    }
    if (c < wc && !aborted) {
#pragma unroll
      for (int r = 0; r < kStreamRB; ++r)
        if (r < nrows) {
          const int row = ch.y + r;
          const float w = a.row_w[row];
          red_add_f32x2(a.out + (size_t)a.perm[row] * a.H + col0 + c, w * acc[r].x,
                        w * acc[r].y);
        }
    }
  }
}

}  // namespace moe
