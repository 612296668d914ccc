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
// The kernel runs on CTA pairs (see grouped_gemm_2sm_kernel).  Tiles are (256-row chunk of one
// expert's rows, column block); the work list of chunks is built on the device by the routing
// kernels, and CTA pairs walk the tile list round-robin.  Rows of a
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

struct GemmArgs {
  int K;                 // reduction length: H (gate/up) or I (down)
  int Ncols;             // output columns of one matrix: I (gate/up) or H (down)
  int sub_stride;        // column offset between sub-tiles in the weight (I for gate/up)
  int w_rows;            // weight rows per expert (= K)
  const int4* chunks;    // {expert, first row, rows}, rows <= 256 (one chunk per CTA pair)
  const int32_t* sched;  // [0] number of chunks
  uint16_t* h;           // gate/up output [R, I] bf16
  const int32_t* perm;   // down: token of each row
  const float* row_w;    // down: routing weight of each row
  float* out;            // down: [T, H] fp32, zero on entry
  int H;
  uint32_t* status;
  float4* zero4;         // gate/up: region its epilogue warps zero-fill (the down output), or null
  size_t n_zero4;
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


// ------------------------------------------------------------------------------------------------
// The kernel runs on CTA pairs (cluster of 2, tcgen05 cta_group::2).  One MMA instruction covers
// 256 rows x N = 256 columns: each CTA of the pair stages its own 128 activation rows and HALF of
// the instruction's weight columns, and the even CTA issues MMAs that read both CTAs' shared
// memory; each CTA's tensor memory receives its 128 rows x all 256 columns.
//   gate/up: the even CTA stages 128 gate columns, the odd CTA the same 128 up columns, so one
//            instruction yields [gate | up] for the 256 rows and every thread holds the matching
//            gate and up sums of its row for the SwiGLU.  Tile = 128 columns of I.
//   down:    the CTAs stage columns [n0, n0+128) and [n0+128, n0+256) of W_down.  Tile = 256
//            columns of H.
// Per SM a stage is 16 KB of rows + 16 KB of weights for 128 x 256 x 64 MACs.
//
// Barriers: both CTAs' TMA loads complete on the even CTA's `full` barrier (the even CTA
// expects the pair's bytes); the MMA thread's commits arrive on `empty` / `acc_full` in both
// CTAs; both CTAs' epilogue threads arrive on the even CTA's `acc_empty`.  The pair starts and
// ends with a cluster barrier so no CTA signals an uninitialised or exited peer.
// ------------------------------------------------------------------------------------------------
constexpr int kGemmN = 256;                                  // MMA N (columns of D per CTA)
constexpr int kGemmHalf = kGemmN / 2;                        // weight columns staged per CTA
constexpr int kEpiPitch = 36;                                // floats per staged row (16B-aligned)
constexpr int kEpiStageBytes = 4 * 32 * kEpiPitch * 4;       // 4 epilogue warps x 32 x 32 fp32

template <int STAGES>
struct Gemm2Cfg {
  static constexpr int kAccBufs = 2;
  static constexpr int kTmemCols = 512;
  static constexpr int kABytes = kGemmBM * kGemmBK * 2;      // this CTA's 128 rows, 16 KB
  static constexpr int kBAtomBytes = kGemmBK * 64 * 2;       // 8 KB: 64 K-rows x 64 columns
  static constexpr int kBAtoms = kGemmHalf / 64;
  static constexpr int kBBytes = kBAtoms * kBAtomBytes;
  static constexpr int kStageBytes = kABytes + kBBytes;
  static constexpr int kSmem = 1024 + STAGES * kStageBytes + 256 + kEpiStageBytes;
  static_assert(kAccBufs * kGemmN <= kTmemCols, "tensor memory");
  static_assert(kSmem <= 227 * 1024, "shared memory");
};

// MODE 0: gate/up projection with the SwiGLU epilogue.  MODE 1: down projection with the
// routing-weight + combine epilogue.
template <int MODE, int STAGES>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kGemmThreads, 1)
    grouped_gemm_2sm_kernel(const GemmArgs a, const __grid_constant__ CUtensorMap amap,
                            const __grid_constant__ CUtensorMap bmap) {
  using C = Gemm2Cfg<STAGES>;
  constexpr int TW = MODE == 0 ? kGemmHalf : kGemmN;         // output columns per tile
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
  float* epi_stage = reinterpret_cast<float*>(ring + STAGES * C::kStageBytes + 256);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;

  if (warp == 1) {
    tmem_alloc_2sm(&s_tmem, C::kTmemCols);
    tmem_relinquish_2sm();
  }
  if (tid == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], 2 * 128);
    }
    mbar_init(drain, 1);
    s_abort = 0;
    fence_barrier_init();
  }
  tc_fence_before();
  cluster_sync_all();
  tc_fence_after();
  const uint32_t tmem_base = s_tmem;
  if (tid == 0) {
    tma_prefetch_desc(&amap);
    tma_prefetch_desc(&bmap);
  }
  pdl_wait();  // activations, work list and (down) h come from the previous kernels
  pdl_launch_next();

  const int NT = (a.Ncols + TW - 1) / TW;
  const int tiles = a.sched[0] * NT;
  const int nk = a.K / kGemmBK;
  const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
  volatile int* abort_flag = &s_abort;

  if (warp == 0) {
    // ------------------------------ TMA producer (both CTAs) ------------------------------
    if (lane == 0) {
      uint32_t it = 0;
      int last_it[STAGES];
#pragma unroll
      for (int s = 0; s < STAGES; ++s) last_it[s] = -1;
      for (int t = pair; t < tiles && !*abort_flag; t += npairs) {
        const int4 ch = a.chunks[t / NT];
        const int n0 = (t % NT) * TW;
        const int row0 = ch.y + (int)rank * kGemmBM;
        // this CTA's weight columns: gate (even) / up (odd) block, or its half of the tile
        const int col0 = MODE == 0 ? (int)rank * a.sub_stride + n0 : n0 + (int)rank * kGemmHalf;
        bool ok = true;
        for (int kst = 0; kst < nk; ++kst, ++it) {
          const int slot = it % STAGES;
          const uint32_t ph = (it / STAGES) & 1u;
          if (!wait_or_abort(&empty[slot], ph ^ 1u, abort_flag, a.status)) {
            ok = false;
            break;
          }
          const uint32_t bar = mapa_shared(smem_u32(&full[slot]), 0);
          if (leader) mbar_arrive_expect_tx(&full[slot], 2 * C::kStageBytes);
          uint8_t* st = ring + slot * C::kStageBytes;
          const int k0 = kst * kGemmBK;
          tma_load_2d_pair(st, &amap, k0, row0, bar);
#pragma unroll
          for (int j = 0; j < C::kBAtoms; ++j)
            tma_load_2d_pair(st + C::kABytes + j * C::kBAtomBytes, &bmap, col0 + 64 * j,
                             ch.x * a.w_rows + k0, bar);
          last_it[slot] = it;
        }
        if (!ok) break;
      }
      // the even CTA's full barriers count both CTAs' copies: drain them before the pair exits
      if (leader)
        for (int s = 0; s < STAGES; ++s)
          if (last_it[s] >= 0 &&
              !mbar_wait_bounded(&full[s], (last_it[s] / STAGES) & 1u, kWaitLimitNs))
            atomicOr(a.status, kStatusTimeout);
    }
  } else if (warp == 1) {
    // ------------------------------ MMA issuer (even CTA) ------------------------------
    if (leader && lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(2 * kGemmBM, kGemmN, false, true);
      const uint32_t ring_s = smem_u32(ring);
      // descriptors of slot 0; a slot / K-step offset only moves the 14-bit start address field
      // (addresses stay below 256 KB, so adding (offset >> 4) never carries out of it)
      const uint64_t adesc0 = smem_desc_sw128(ring_s, 16, 1024);
      const uint64_t bdesc0 = smem_desc_sw128(ring_s + C::kABytes, C::kBAtomBytes, 1024);
      uint32_t it = 0;
      int tile_i = 0;
      bool issued = false;
      for (int t = pair; t < tiles && !*abort_flag; t += npairs, ++tile_i) {
        const int buf = tile_i % C::kAccBufs;
        const uint32_t aph = (tile_i / C::kAccBufs) & 1u;
        if (!wait_or_abort(&acc_empty[buf], aph ^ 1u, abort_flag, a.status)) break;
        tc_fence_after();
        const uint32_t d = tmem_base + buf * kGemmN;
        bool ok = true;
        for (int kst = 0; kst < nk; ++kst, ++it) {
          const int slot = it % STAGES;
          const uint32_t ph = (it / STAGES) & 1u;
          if (!wait_or_abort(&full[slot], ph, abort_flag, a.status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t soff = (uint64_t)((slot * C::kStageBytes) >> 4);
#pragma unroll
          for (int k16 = 0; k16 < kGemmBK / 16; ++k16)
            tc_mma_bf16_2sm(d, adesc0 + soff + (k16 * 32 >> 4), bdesc0 + soff + (k16 * 2048 >> 4),
                            idesc, (kst | k16) != 0);
          const uint32_t e_local = smem_u32(&empty[slot]);
          tc_commit_2sm(e_local);
          tc_commit_2sm(mapa_shared(e_local, 1));
          issued = true;
        }
        if (!ok) break;
        const uint32_t f_local = smem_u32(&acc_full[buf]);
        tc_commit_2sm(f_local);
        tc_commit_2sm(mapa_shared(f_local, 1));
      }
      if (issued) {  // all MMAs complete before the tensor memory is freed
        tc_commit_2sm(smem_u32(drain));
        if (!mbar_wait_bounded(drain, 0, kWaitLimitNs)) atomicOr(a.status, kStatusTimeout);
      }
    }
  } else {
    // ------------------------------ epilogue (both CTAs) ------------------------------
    const int q = warp & 3;
    const int row = 32 * q + lane;
    // gate/up: zero-fill this CTA's share of the down projection's output, one piece after
    // each tile (the tensor cores run meanwhile; the rest of the share after the last tile)
    size_t z_beg = 0, z_end = 0, z_piece = 0;
    if (MODE == 0 && a.zero4 != nullptr) {
      const size_t per = (a.n_zero4 + gridDim.x - 1) / gridDim.x;
      z_beg = min(a.n_zero4, (size_t)blockIdx.x * per);
      z_end = min(a.n_zero4, z_beg + per);
      const int my_tiles = max(1, (tiles - pair + npairs - 1) / npairs);
      z_piece = ((z_end - z_beg + my_tiles - 1) / my_tiles + 127) / 128 * 128;
    }
    const int et = tid - kGemmEpiWarp0 * 32;  // 0..127
    auto zero_piece = [&](size_t stop) {
      for (size_t i = z_beg + et; i < stop; i += 128) a.zero4[i] = make_float4(0.f, 0.f, 0.f, 0.f);
      z_beg = stop;
    };
    int tile_i = 0;
    for (int t = pair; t < tiles; t += npairs, ++tile_i) {
      const int buf = tile_i % C::kAccBufs;
      const uint32_t aph = (tile_i / C::kAccBufs) & 1u;
      if (!wait_or_abort(&acc_full[buf], aph, abort_flag, a.status)) break;
      tc_fence_after();
      const int4 ch = a.chunks[t / NT];
      const int n0 = (t % NT) * TW;
      const int r0 = ch.y + (int)rank * kGemmBM;          // first row of this CTA's half
      const bool valid = row < ch.z - (int)rank * kGemmBM;
      const uint32_t taddr = tmem_base + ((uint32_t)(32 * q) << 16) + buf * kGemmN;
      if constexpr (MODE == 0) {
        uint16_t* hrow = a.h + (size_t)(r0 + row) * a.Ncols + n0;
#pragma unroll 1
        for (int c = 0; c < kGemmHalf; c += 32) {
          float g[32], u[32];
          tmem_ld32(taddr + c, g);
          tmem_ld32(taddr + kGemmHalf + c, u);
          if (valid && n0 + c < a.Ncols) {
            uint32_t p[16];
#pragma unroll
            for (int i = 0; i < 16; ++i)
              p[i] = pack_bf16x2(silu_fast(g[2 * i]) * u[2 * i], silu_fast(g[2 * i + 1]) * u[2 * i + 1]);
            uint4* dst = reinterpret_cast<uint4*>(hrow + c);
#pragma unroll
            for (int i = 0; i < 4; ++i) dst[i] = make_uint4(p[4 * i], p[4 * i + 1], p[4 * i + 2], p[4 * i + 3]);
          }
        }
      } else {
        // Each thread holds 32 columns of its own row; the atomics go out transposed through
        // shared memory so that one instruction covers 4 rows x 128 contiguous bytes instead of
        // 32 scattered rows.
        const int tok = valid ? a.perm[r0 + row] : -1;
        const float w = valid ? a.row_w[r0 + row] : 0.f;
        float* stage = epi_stage + (warp - kGemmEpiWarp0) * 32 * kEpiPitch;
#pragma unroll 1
        for (int c = 0; c < kGemmN; c += 32) {
          float y[32];
          tmem_ld32(taddr + c, y);
          if (n0 + c >= a.Ncols) continue;  // whole chunk past H (warp-uniform)
#pragma unroll
          for (int j = 0; j < 32; ++j) stage[lane * kEpiPitch + j] = w * y[j];
          __syncwarp();
#pragma unroll
          for (int it = 0; it < 8; ++it) {
            const int rr = 4 * it + (lane >> 3), cc = 4 * (lane & 7);
            const int t = __shfl_sync(0xffffffffu, tok, rr);
            const float4 v = *reinterpret_cast<const float4*>(stage + rr * kEpiPitch + cc);
            if (t >= 0) red_add_f32x4(a.out + (size_t)t * a.H + n0 + c + cc, v.x, v.y, v.z, v.w);
          }
          __syncwarp();
        }
      }
      tc_fence_before();
      mbar_arrive_cluster(mapa_shared(smem_u32(&acc_empty[buf]), 0));
      if (MODE == 0 && z_beg < z_end) zero_piece(min(z_end, z_beg + z_piece));
    }
    if (MODE == 0 && z_beg < z_end) zero_piece(z_end);
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync_all();
  tc_fence_after();
  if (warp == 1) tmem_dealloc_2sm(tmem_base, C::kTmemCols);
}

}  // namespace moe
