// Row-tile grouped GEMM on CTA pairs with 256 x 512 tiles (two N = 256 MMAs per K step).
//
// The 256 x 256 row-tile kernel (gemm.cuh) loads 32 KB per SM per K step of 64 for 128 x 256 x 64
// MACs: 64 bytes per SM clock at the full MMA rate, more than the shared-memory fill it gets (about
// 52 B per SM clock measured), so its tensor pipe idles ~18 % of the time.  Here each CTA of the
// pair stages its 128 activation rows once and twice the weight columns, and the pair issues two
// M = 256, N = 256 MMAs per K step that share the activation tile: 48 KB per SM per K step for
// 128 x 512 x 64 MACs, 48 B per SM clock.
//
// The accumulators of one tile fill the whole tensor memory (two 256-column halves, D_a and D_b),
// so tiles cannot be double-buffered.  Instead the eight epilogue warps drain D_a first (and hand
// it back on its own barrier), then D_b, while the MMA thread already runs the next tile's D_a
// MMAs on the stages in flight and catches up on D_b once it is free.
//
//   gate/up (MODE 0): tile = 256 rows x 256 columns of I; D_a = [gate n0..n0+127 | up n0..n0+127]
//            (even CTA stages the gate columns, odd CTA the up columns), D_b the next 128 of each.
//   down    (MODE 1): tile = 256 rows x 512 columns of H; D_a = columns n0..n0+255 (even CTA
//            stages the first 128), D_b = n0+256..n0+511.
//
// Warps: 0 TMA producer (both CTAs), 1 TMEM owner + MMA issuer (even CTA, one lane), 2-9
// epilogue (warp w: TMEM lane quarter w % 4, column half (w - 2) / 4 of each accumulator half).
// Every wait is bounded; on a timeout the pair records it, winds down, drains its copies and MMAs,
// frees the tensor memory and returns.
#pragma once

#include "common.cuh"
#include "gemm.cuh"

namespace moe {

constexpr int kWideThreads = 320;
constexpr int kWideEpiWarp0 = 2;
constexpr int kWideEpiThreads = 256;

template <int MODE>
struct WideCfg {
  static constexpr int kStages = MODE == 0 ? 4 : 3;
  static constexpr int kABytes = kGemmBM * kGemmBK * 2;           // 16 KB: this CTA's 128 rows
  static constexpr int kBAtomBytes = kGemmBK * 64 * 2;            // 8 KB: 64 K x 64 columns
  static constexpr int kBHalfBytes = 2 * kBAtomBytes;             // 128 columns of one MMA
  static constexpr int kStageBytes = kABytes + 2 * kBHalfBytes;   // 48 KB
  static constexpr int kEpiBytes = MODE == 1 ? 8 * 32 * kEpiPitch * 4 : 0;
  static constexpr int kSmem = 1024 + kStages * kStageBytes + 256 + kEpiBytes;
  static_assert(kSmem <= 227 * 1024, "shared memory");
};

// Whether a tile has columns for its second accumulator half.
template <int MODE>
MOE_DEVINL bool wide_has_b(int n0, int Ncols) {
  return MODE == 0 ? n0 + 128 < Ncols : n0 + 256 < Ncols;
}

template <int MODE>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kWideThreads, 1)
    grouped_gemm_wide_kernel(const GemmArgs a, const __grid_constant__ CUtensorMap amap,
                             const __grid_constant__ CUtensorMap bmap) {
  using C = WideCfg<MODE>;
  constexpr int S = C::kStages;
  constexpr int TW = MODE == 0 ? 256 : 512;  // output columns per tile (per matrix for gate/up)
  extern __shared__ __align__(128) uint8_t smem_raw[];
  __shared__ uint32_t s_tmem;
  __shared__ int s_abort;
  uint8_t* ring = align1k(smem_raw);
  uint64_t* bars = reinterpret_cast<uint64_t*>(ring + S * C::kStageBytes);
  uint64_t* full = bars;
  uint64_t* empty = full + S;
  uint64_t* acc_full = empty + S;
  uint64_t* acc_empty_a = acc_full + 1;
  uint64_t* acc_empty_b = acc_empty_a + 1;
  uint64_t* drain = acc_empty_b + 1;
  float* epi_stage = reinterpret_cast<float*>(ring + S * C::kStageBytes + 256);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;

  if (warp == 1) {
    tmem_alloc_2sm(&s_tmem, 512);
    tmem_relinquish_2sm();
  }
  if (tid == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(acc_full, 1);
    mbar_init(acc_empty_a, 2 * kWideEpiThreads);
    mbar_init(acc_empty_b, 2 * kWideEpiThreads);
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
      int last_it[S];
#pragma unroll
      for (int s = 0; s < S; ++s) last_it[s] = -1;
      for (int t = pair; t < tiles && !*abort_flag; t += npairs) {
        const int4 ch = a.chunks[t / NT];
        const int n0 = (t % NT) * TW;
        const bool hb = wide_has_b<MODE>(n0, a.Ncols);
        const int row0 = ch.y + (int)rank * kGemmBM;
        // this CTA's first weight column of each accumulator half
        const int ca = MODE == 0 ? (int)rank * a.sub_stride + n0 : n0 + (int)rank * 128;
        const int cb = ca + (MODE == 0 ? 128 : 256);
        const uint32_t tx = 2u * (uint32_t)(C::kABytes + (hb ? 2 : 1) * C::kBHalfBytes);
        bool ok = true;
        for (int kst = 0; kst < nk; ++kst, ++it) {
          const int slot = it % S;
          const uint32_t ph = (it / S) & 1u;
          if (!wait_or_abort(&empty[slot], ph ^ 1u, abort_flag, a.status)) {
            ok = false;
            break;
          }
          const uint32_t bar = mapa_shared(smem_u32(&full[slot]), 0);
          if (leader) mbar_arrive_expect_tx(&full[slot], tx);
          uint8_t* st = ring + slot * C::kStageBytes;
          const int k0 = kst * kGemmBK;
          const int wrow = ch.x * a.w_rows + k0;
          tma_load_2d_pair(st, &amap, k0, row0, bar);
#pragma unroll
          for (int j = 0; j < 2; ++j)
            tma_load_2d_pair(st + C::kABytes + j * C::kBAtomBytes, &bmap, ca + 64 * j, wrow, bar);
          if (hb)
#pragma unroll
            for (int j = 0; j < 2; ++j)
              tma_load_2d_pair(st + C::kABytes + C::kBHalfBytes + j * C::kBAtomBytes, &bmap,
                               cb + 64 * j, wrow, bar);
          last_it[slot] = it;
        }
        if (!ok) break;
      }
      if (leader)
        for (int s = 0; s < S; ++s)
          if (last_it[s] >= 0 && !mbar_wait_bounded(&full[s], (last_it[s] / S) & 1u, kWaitLimitNs))
            atomicOr(a.status, kStatusTimeout);
    }
  } else if (warp == 1) {
    // ------------------------------ MMA issuer (even CTA) ------------------------------
    if (leader && lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(2 * kGemmBM, 256, false, true);
      const uint32_t ring_s = smem_u32(ring);
      const uint64_t adesc0 = smem_desc_sw128(ring_s, 16, 1024);
      const uint64_t bdesc0 = smem_desc_sw128(ring_s + C::kABytes, C::kBAtomBytes, 1024);
      constexpr uint64_t kBHalfOff = (uint64_t)(C::kBHalfBytes >> 4);
      const uint32_t d_a = tmem_base, d_b = tmem_base + 256;
      const uint32_t e_local = smem_u32(empty), f_local = smem_u32(acc_full);
      uint32_t it = 0;
      int tile_i = 0;
      bool issued = false;
      auto mma_step = [&](uint32_t d, int slot, uint64_t boff, int kst) {
        const uint64_t soff = (uint64_t)((slot * C::kStageBytes) >> 4);
#pragma unroll
        for (int k16 = 0; k16 < kGemmBK / 16; ++k16)
          tc_mma_bf16_2sm(d, adesc0 + soff + (k16 * 32 >> 4),
                          bdesc0 + soff + boff + (k16 * 2048 >> 4), idesc, (kst | k16) != 0);
      };
      for (int t = pair; t < tiles && !*abort_flag; t += npairs, ++tile_i) {
        const int n0 = (t % NT) * TW;
        const bool hb = wide_has_b<MODE>(n0, a.Ncols);
        const uint32_t aph = tile_i & 1u;  // phase of the previous tile's drains
        if (!wait_or_abort(acc_empty_a, aph ^ 1u, abort_flag, a.status)) break;
        tc_fence_after();
        bool b_ready = false, ok = true;
        int kb = 0;                       // next K step whose D_b MMAs are still to issue
        const uint32_t it0 = it;
        for (int kst = 0; kst < nk; ++kst, ++it) {
          const int slot = it % S;
          const uint32_t ph = (it / S) & 1u;
          if (!wait_or_abort(&full[slot], ph, abort_flag, a.status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          mma_step(d_a, slot, 0, kst);
          // D_b is free once the previous tile's epilogue handed it back; wait for it at the
          // latest when every stage holds a K step whose D_b MMAs are pending
          if (!b_ready) {
            if (mbar_try_wait(acc_empty_b, aph ^ 1u)) {
              b_ready = true;
            } else if (kst == nk - 1 || kst - kb == S - 1) {
              if (!wait_or_abort(acc_empty_b, aph ^ 1u, abort_flag, a.status)) {
                ok = false;
                break;
              }
              b_ready = true;
            }
            if (b_ready) tc_fence_after();
          }
          if (b_ready) {
            for (; kb <= kst; ++kb) {
              const int bslot = (it0 + kb) % S;
              if (hb) mma_step(d_b, bslot, kBHalfOff, kb);
              tc_commit_2sm(e_local + bslot * 8);
              tc_commit_2sm(mapa_shared(e_local + bslot * 8, 1));
            }
          }
          issued = true;
        }
        if (!ok) break;
        tc_commit_2sm(f_local);
        tc_commit_2sm(mapa_shared(f_local, 1));
      }
      if (issued) {  // all MMAs complete before the tensor memory is freed
        tc_commit_2sm(smem_u32(drain));
        if (!mbar_wait_bounded(drain, 0, kWaitLimitNs)) atomicOr(a.status, kStatusTimeout);
      }
    }
  } else {
    // ------------------------------ epilogue (both CTAs, warps 2-9) ------------------------------
    const int q = warp & 3;                         // TMEM lanes 32q .. 32q + 31
    const int part = (warp - kWideEpiWarp0) >> 2;   // which column half of each accumulator half
    const int row = 32 * q + lane;
    const int et = tid - kWideEpiWarp0 * 32;        // 0..255
    size_t z_beg = 0, z_end = 0, z_piece = 0;
    if (MODE == 0 && a.zero4 != nullptr) {
      const size_t per = (a.n_zero4 + gridDim.x - 1) / gridDim.x;
      z_beg = min(a.n_zero4, (size_t)blockIdx.x * per);
      z_end = min(a.n_zero4, z_beg + per);
      const int my_tiles = max(1, (tiles - pair + npairs - 1) / npairs);
      z_piece = ((z_end - z_beg + my_tiles - 1) / my_tiles + 255) / 256 * 256;
    }
    auto zero_piece = [&](size_t stop) {
      for (size_t i = z_beg + et; i < stop; i += kWideEpiThreads)
        a.zero4[i] = make_float4(0.f, 0.f, 0.f, 0.f);
      z_beg = stop;
    };
    float* stage = epi_stage + (warp - kWideEpiWarp0) * 32 * kEpiPitch;
    const uint32_t ea = mapa_shared(smem_u32(acc_empty_a), 0);
    const uint32_t eb = mapa_shared(smem_u32(acc_empty_b), 0);
    int tile_i = 0;
    for (int t = pair; t < tiles; t += npairs, ++tile_i) {
      if (!wait_or_abort(acc_full, tile_i & 1u, abort_flag, a.status)) break;
      tc_fence_after();
      const int4 ch = a.chunks[t / NT];
      const int n0 = (t % NT) * TW;
      const int r0 = ch.y + (int)rank * kGemmBM;
      const bool valid = row < ch.z - (int)rank * kGemmBM;
      const uint32_t tl = tmem_base + ((uint32_t)(32 * q) << 16);
#pragma unroll 1
      for (int half = 0; half < 2; ++half) {
        const uint32_t taddr = tl + half * 256;
        if constexpr (MODE == 0) {
          // columns c0 .. c0+63 of gate (accumulator columns part*64 + c) and of up (+128)
          const int c0 = n0 + half * 128 + part * 64;
          uint16_t* hrow = a.h + (size_t)(r0 + row) * a.Ncols + c0;
#pragma unroll 1
          for (int c = 0; c < 64; c += 32) {
            float g[32], u[32];
            tmem_ld32(taddr + part * 64 + c, g);
            tmem_ld32(taddr + 128 + part * 64 + c, u);
            if (valid && c0 + c < a.Ncols) {
              uint32_t p[16];
#pragma unroll
              for (int i = 0; i < 16; ++i)
                p[i] = pack_bf16x2(silu_fast(g[2 * i]) * u[2 * i],
                                   silu_fast(g[2 * i + 1]) * u[2 * i + 1]);
              uint4* dst = reinterpret_cast<uint4*>(hrow + c);
#pragma unroll
              for (int i = 0; i < 4; ++i)
                dst[i] = make_uint4(p[4 * i], p[4 * i + 1], p[4 * i + 2], p[4 * i + 3]);
            }
          }
        } else {
          // 128 columns of this half: c0 .. c0+127, staged so that each vector atomic covers 4
          // rows x 128 contiguous bytes
          const int c0 = n0 + half * 256 + part * 128;
          const int tok = valid ? a.perm[r0 + row] : -1;
          const float w = valid ? a.row_w[r0 + row] : 0.f;
#pragma unroll 1
          for (int c = 0; c < 128; c += 32) {
            float y[32];
            tmem_ld32(taddr + part * 128 + c, y);
            if (c0 + c >= a.Ncols) continue;  // warp-uniform
#pragma unroll
            for (int j = 0; j < 32; ++j) stage[lane * kEpiPitch + j] = w * y[j];
            __syncwarp();
#pragma unroll
            for (int it2 = 0; it2 < 8; ++it2) {
              const int rr = 4 * it2 + (lane >> 3), cc = 4 * (lane & 7);
              const int tk = __shfl_sync(0xffffffffu, tok, rr);
              const float4 v = *reinterpret_cast<const float4*>(stage + rr * kEpiPitch + cc);
              if (tk >= 0) red_add_f32x4(a.out + (size_t)tk * a.H + c0 + c + cc, v.x, v.y, v.z, v.w);
            }
            __syncwarp();
          }
        }
        tc_fence_before();
        mbar_arrive_cluster(half == 0 ? ea : eb);
      }
      if (MODE == 0 && z_beg < z_end) zero_piece(min(z_end, z_beg + z_piece));
    }
    if (MODE == 0 && z_beg < z_end) zero_piece(z_end);
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync_all();
  tc_fence_after();
  if (warp == 1) tmem_dealloc_2sm(tmem_base, 512);
}

}  // namespace moe
