// Grouped GEMM on the 5th-generation tensor cores for the many-token regime.
//
// When each expert sees hundreds of rows (prefill, long packed sequences), the expert matmuls are
// dense [rows x K] x [K x N] products, one per expert, and the layer is bound by tensor-core
// throughput.  Both projections run through one persistent, warp-specialised kernel template:
//
//   warp 0      TMA producer: per K stage, one [128 rows x 64] box of the activations (K-major,
//               128-byte swizzle) and [64 x 64] boxes of the expert's weight columns (the weights
//               are [K, N] with N contiguous, i.e. the MN-major operand), into a smem ring.
//   warp 1      owns the tensor memory (allocates all 512 columns); one lane issues
//               tcgen05.mma (M = 128, N = 128..256, K = 16, bf16 in, fp32 accumulate in TMEM) and
//               tcgen05.commit to release smem stages and to hand finished accumulators over.
//   warps 2-5   epilogue: tcgen05.ld of the accumulator rows (one TMEM lane per row), then
//                 gate/up:  h = silu(g) * u  -> bf16 row of h          (SwiGLU fused)
//                 down:     out[token] += w * y  with fp32 vector atomics (weight + combine)
//               Two accumulator buffers let the epilogue of one tile overlap the next tile's MMAs.
//
// Tiles are (128-row chunk of one expert's rows, column block); the work list of chunks is built
// on the device by the routing kernels, and CTAs walk the tile list round-robin.  Rows of a
// chunk beyond the expert's segment are computed but never stored.  Every wait is bounded: on a
// timeout the CTA records it in the status word, skips the remaining work, drains its own copies
// and MMAs, frees the tensor memory and returns.
#pragma once

#include "common.cuh"

namespace moe {

constexpr int kGemmBM = 128;                 // rows per tile (MMA M)
constexpr int kGemmBK = 64;                  // K per stage (one 128-byte swizzle row)
constexpr int kGemmThreads = 192;
constexpr int kGemmEpiWarp0 = 2;

template <int NSUB, int SUBN, int STAGES>
struct GemmCfg {
  static constexpr int kN = NSUB * SUBN;                     // accumulator columns per tile
  static constexpr int kAccBufs = (2 * kN <= 512) ? 2 : 1;
  static constexpr int kTmemCols = 512;
  static constexpr int kABytes = kGemmBM * kGemmBK * 2;      // 16 KB
  static constexpr int kBAtomBytes = kGemmBK * 64 * 2;       // 8 KB: 64 K-rows x 64 columns
  static constexpr int kBAtomsPerSub = SUBN / 64;
  static constexpr int kBBytes = NSUB * kBAtomsPerSub * kBAtomBytes;
  static constexpr int kStageBytes = kABytes + kBBytes;
  static constexpr int kSmem = 1024 + STAGES * kStageBytes + 256;
  static_assert(SUBN % 64 == 0 && SUBN >= 64 && SUBN <= 256, "MMA N: whole 64-column atoms");
  static_assert(kAccBufs * kN <= kTmemCols, "tensor memory");
  static_assert(kSmem <= 227 * 1024, "shared memory");
};

struct GemmArgs {
  int K;                 // reduction length: H (gate/up) or I (down)
  int Ncols;             // output columns of one matrix: I (gate/up) or H (down)
  int sub_stride;        // column offset between sub-tiles in the weight (I for gate/up)
  int w_rows;            // weight rows per expert (= K)
  const int4* chunks;    // {expert, first row, rows}, rows <= 128
  const int32_t* sched;  // [0] number of chunks
  uint16_t* h;           // gate/up output [R, I] bf16
  const int32_t* perm;   // down: token of each row
  const float* row_w;    // down: routing weight of each row
  float* out;            // down: [T, H] fp32, zero on entry
  int H;
  uint32_t* status;
};

MOE_DEVINL bool wait_or_abort(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                              uint32_t* status) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  while (true) {
    if (*abort_flag) return false;
    if (mbar_try_wait(bar, parity)) return true;
    if (globaltimer_ns() - t0 > kWaitLimitNs) {
      atomicOr(status, kStatusTimeout);
      *abort_flag = 1;
      return false;
    }
  }
}

// MODE 0: gate/up projection with the SwiGLU epilogue (NSUB = 2: gate block, up block).
// MODE 1: down projection with the routing-weight + combine epilogue (NSUB = 1).
template <int MODE, int NSUB, int SUBN, int STAGES>
__global__ void __launch_bounds__(kGemmThreads, 1)
    grouped_gemm_kernel(const GemmArgs a, const __grid_constant__ CUtensorMap amap,
                        const __grid_constant__ CUtensorMap bmap) {
  using C = GemmCfg<NSUB, SUBN, STAGES>;
  extern __shared__ __align__(128) uint8_t smem_raw[];
  __shared__ uint32_t s_tmem;
  __shared__ int s_abort;
  uint8_t* ring = align1k(smem_raw);
  uint64_t* bars = reinterpret_cast<uint64_t*>(ring + STAGES * C::kStageBytes);
  uint64_t* full = bars;
  uint64_t* empty = full + STAGES;
  uint64_t* acc_full = empty + STAGES;
  uint64_t* acc_empty = acc_full + 2;
  uint64_t* drain = acc_empty + 2;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  if (warp == 1) {
    tmem_alloc(&s_tmem, C::kTmemCols);
    tmem_relinquish();
  }
  if (tid == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], 128);
    }
    mbar_init(drain, 1);
    s_abort = 0;
    fence_barrier_init();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = s_tmem;

  const int NT = (a.Ncols + SUBN - 1) / SUBN;
  const int tiles = a.sched[0] * NT;
  const int nk = a.K / kGemmBK;
  volatile int* abort_flag = &s_abort;

  if (warp == 0) {
    // ------------------------------ TMA producer ------------------------------
    if (lane == 0) {
      tma_prefetch_desc(&amap);
      tma_prefetch_desc(&bmap);
      uint32_t it = 0;
      int last_it[STAGES];
#pragma unroll
      for (int s = 0; s < STAGES; ++s) last_it[s] = -1;
      for (int t = blockIdx.x; t < tiles && !*abort_flag; t += gridDim.x) {
        const int4 ch = a.chunks[t / NT];
        const int n0 = (t % NT) * SUBN;
        for (int kst = 0; kst < nk; ++kst, ++it) {
          const int slot = it % STAGES;
          const uint32_t ph = (it / STAGES) & 1u;
          if (!wait_or_abort(&empty[slot], ph ^ 1u, abort_flag, a.status)) break;
          mbar_arrive_expect_tx(&full[slot], C::kStageBytes);
          uint8_t* st = ring + slot * C::kStageBytes;
          const int k0 = kst * kGemmBK;
          tma_load_2d(st, &amap, k0, ch.y, &full[slot]);
#pragma unroll
          for (int sub = 0; sub < NSUB; ++sub)
#pragma unroll
            for (int j = 0; j < C::kBAtomsPerSub; ++j)
              tma_load_2d(st + C::kABytes + (sub * C::kBAtomsPerSub + j) * C::kBAtomBytes, &bmap,
                          sub * a.sub_stride + n0 + 64 * j, ch.x * a.w_rows + k0, &full[slot]);
          last_it[slot] = it;
        }
      }
      // never leave with copies in flight
      for (int s = 0; s < STAGES; ++s)
        if (last_it[s] >= 0 &&
            !mbar_wait_bounded(&full[s], (last_it[s] / STAGES) & 1u, kWaitLimitNs))
          atomicOr(a.status, kStatusTimeout);
    }
  } else if (warp == 1) {
    // ------------------------------ MMA issuer ------------------------------
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(kGemmBM, SUBN, false, true);
      const uint32_t ring_s = smem_u32(ring);
      uint32_t it = 0;
      int tile_i = 0;
      bool issued = false;
      for (int t = blockIdx.x; t < tiles && !*abort_flag; t += gridDim.x, ++tile_i) {
        const int buf = tile_i % C::kAccBufs;
        const uint32_t aph = (tile_i / C::kAccBufs) & 1u;
        if (!wait_or_abort(&acc_empty[buf], aph ^ 1u, abort_flag, a.status)) break;
        tc_fence_after();
        const uint32_t d = tmem_base + buf * C::kN;
        bool ok = true;
        for (int kst = 0; kst < nk; ++kst, ++it) {
          const int slot = it % STAGES;
          const uint32_t ph = (it / STAGES) & 1u;
          if (!wait_or_abort(&full[slot], ph, abort_flag, a.status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_s = ring_s + slot * C::kStageBytes;
          const uint32_t b_s = a_s + C::kABytes;
#pragma unroll
          for (int k16 = 0; k16 < kGemmBK / 16; ++k16) {
            // A: K-major, rows of 128 B, 8-row groups 1 KB apart; +32 B per 16 K
            const uint64_t adesc = smem_desc_sw128(a_s + k16 * 32, 16, 1024);
#pragma unroll
            for (int sub = 0; sub < NSUB; ++sub) {
              // B: MN-major, 64-column atoms 8 KB apart, 8-row K groups 1 KB apart; +2 KB per 16 K
              const uint64_t bdesc = smem_desc_sw128(
                  b_s + sub * C::kBAtomsPerSub * C::kBAtomBytes + k16 * 2048, C::kBAtomBytes, 1024);
              tc_mma_bf16(d + sub * SUBN, adesc, bdesc, idesc, (kst | k16) != 0);
            }
          }
          tc_commit(&empty[slot]);
          issued = true;
        }
        if (!ok) break;
        tc_commit(&acc_full[buf]);
      }
      if (issued) {  // all MMAs complete before the tensor memory is freed
        tc_commit(drain);
        if (!mbar_wait_bounded(drain, 0, kWaitLimitNs)) atomicOr(a.status, kStatusTimeout);
      }
    }
  } else {
    // ------------------------------ epilogue ------------------------------
    const int q = warp & 3;                 // TMEM lane quarter this warp may read
    const int row = 32 * q + lane;          // tile row held by this thread
    int tile_i = 0;
    for (int t = blockIdx.x; t < tiles; t += gridDim.x, ++tile_i) {
      const int buf = tile_i % C::kAccBufs;
      const uint32_t aph = (tile_i / C::kAccBufs) & 1u;
      if (!wait_or_abort(&acc_full[buf], aph, abort_flag, a.status)) break;
      tc_fence_after();
      const int4 ch = a.chunks[t / NT];
      const int n0 = (t % NT) * SUBN;
      const bool valid = row < ch.z;
      const uint32_t taddr = tmem_base + ((uint32_t)(32 * q) << 16) + buf * C::kN;
      if constexpr (MODE == 0) {
        uint16_t* hrow = a.h + (size_t)(ch.y + row) * a.Ncols + n0;
#pragma unroll 1
        for (int c = 0; c < SUBN; c += 32) {
          float g[32], u[32];
          tmem_ld32(taddr + c, g);
          tmem_ld32(taddr + SUBN + c, u);
          if (valid && n0 + c < a.Ncols) {
            uint32_t p[16];
#pragma unroll
            for (int i = 0; i < 16; ++i)
              p[i] = pack_bf16x2(silu_f32(g[2 * i]) * u[2 * i], silu_f32(g[2 * i + 1]) * u[2 * i + 1]);
            uint4* dst = reinterpret_cast<uint4*>(hrow + c);
#pragma unroll
            for (int i = 0; i < 4; ++i) dst[i] = make_uint4(p[4 * i], p[4 * i + 1], p[4 * i + 2], p[4 * i + 3]);
          }
        }
      } else {
        const int tok = valid ? a.perm[ch.y + row] : 0;
        const float w = valid ? a.row_w[ch.y + row] : 0.f;
        float* orow = a.out + (size_t)tok * a.H + n0;
#pragma unroll 1
        for (int c = 0; c < SUBN; c += 32) {
          float y[32];
          tmem_ld32(taddr + c, y);
          if (valid && n0 + c < a.Ncols) {
#pragma unroll
            for (int i = 0; i < 8; ++i)
              red_add_f32x4(orow + c + 4 * i, w * y[4 * i], w * y[4 * i + 1], w * y[4 * i + 2],
                            w * y[4 * i + 3]);
          }
        }
      }
      tc_fence_before();
      mbar_arrive(&acc_empty[buf]);
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem_base, C::kTmemCols);
}

}  // namespace moe
