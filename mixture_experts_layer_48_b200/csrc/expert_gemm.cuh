// Expert-tile grouped GEMM on the 5th-generation tensor cores: the expert's weights are the
// M operand and its routed rows the N operand.
//
// Between decode (each expert sees about one token: the weight-streaming kernels) and prefill
// (hundreds of rows per expert: the row-tile grouped GEMM) lies the regime where an expert holds
// tens to a couple of hundred rows.  The hearth-lean-loomed-v1 card ("Why 12-16 streams can be
// slow on Vulkan") describes exactly this band, where the choice between a mat-vec and a mat-mat
// kernel per expert swings the call by 5x.  Here the layer is still bound by reading each
// touched expert's weights once from HBM, but the products are too many for the CUDA-core-fed
// mma.sync streaming kernel and too few rows to fill a 256-row MMA tile.  So the roles swap:
//
//   D[w, n] = sum_k W[k, w] * X[n, k]       w: 128 weight columns (TMEM lanes)
//                                           n: the chunk's rows, rounded up to 16 (MMA N <= 128,
//                                              or <= 256 in the 256-row variant)
//
// and each tile streams a [K x 128]-column block of one expert's weights exactly once for all of
// that expert's rows (up to 128 or 256 per tile).  Work: tiles = (row chunk of one expert,
// column block); per K stage of 64 a tile loads two 128-column weight blocks (gate and up, or two
// neighbouring blocks of W_down: 32 KB) and the chunk's rows (16 rows per box, up to 16 or 32 KB).
//
//   warp 0      TMA producer (weights as 64 x 64 boxes with the 128-byte swizzle: the MN-major
//               A operand; activation rows as 16 x 64 boxes: the K-major B operand)
//   warp 1      TMEM owner (512 columns) and, on one lane, the MMA issuer: per K step of 16 two
//               tcgen05.mma M = 128, N = rows, bf16 in, fp32 accumulate; tcgen05.commit releases
//               the stage and hands over finished accumulators (two buffers of 2 x 128 columns)
//   warps 2-5   epilogue (one TMEM lane = one weight column per thread), through a shared-memory
//               transpose so that global stores run along the rows:
//                 gate/up: h[row, col] = silu(g) * u, bf16        (SwiGLU fused)
//                 down:    out[token, col] += w_row * y  with fp32 vector atomics
//
// Every wait is bounded: on a timeout the CTA records it in the status word, skips the remaining
// work, drains its own copies and MMAs, frees the tensor memory and returns.
#pragma once

#include "common.cuh"
#include "gemm.cuh"

namespace moe {

constexpr int kEtM = 128;                                  // weight columns per MMA
constexpr int kEtRows = 128;                               // rows per tile (max MMA N)
constexpr int kEtBK = 64;                                  // K per stage
constexpr int kEtStages = 4;
constexpr int kEtThreads = 192;
constexpr int kEtRowBox = 16;                              // activation rows per TMA box
constexpr int kEtBoxBytes = kEtBK * 64 * 2;                // 8 KB: 64 K-rows x 64 weight columns
constexpr int kEtABytes = 4 * kEtBoxBytes;                 // two 128-column matrices
constexpr int kEtBBytes = kEtRows * kEtBK * 2;             // 16 KB: 128 rows x 64 K
constexpr int kEtStageBytes = kEtABytes + kEtBBytes;       // 48 KB
constexpr int kEtPitch = 33;                               // floats per staged row (odd: no bank conflicts)
constexpr int kEtEpiBytes = 4 * 32 * kEtPitch * 4;
constexpr int kEtSmem = 1024 + kEtStages * kEtStageBytes + 256 + kEtEpiBytes;
constexpr int kEtTmemCols = 512;
static_assert(kEtSmem <= 227 * 1024, "shared memory");

// Tile shapes by rows per tile (the MMA's largest N): 128 rows keep two accumulator buffers of
// 2 x 128 TMEM columns (the epilogue of one tile overlaps the MMAs of the next) and four stages;
// 256 rows fill the 512 columns with one buffer (gate 256 | up 256) and take three stages of
// 64 KB.  Per K step a 256-row tile reads the weight blocks once for twice the rows: the same
// operand bytes per FLOP as the 2-SM row tiles, with rows padded to 16 instead of 256.
template <int ROWS>
struct EtCfg {
  static_assert(ROWS == 128 || ROWS == 256, "rows per tile");
  static constexpr int kStages = ROWS == 128 ? 4 : 3;
  static constexpr int kBBytes = ROWS * kEtBK * 2;
  static constexpr int kStageBytes = kEtABytes + kBBytes;
  static constexpr int kAccBufs = kEtTmemCols / (2 * ROWS);
  static constexpr int kSmem = 1024 + kStages * kStageBytes + 256 + kEtEpiBytes;
  static_assert(kSmem <= 227 * 1024, "shared memory");
  static_assert(kStageBytes % 1024 == 0, "128-byte swizzle atoms");
};

struct EtArgs {
  int K;                 // reduction length: H (gate/up) or I (down)
  int Ncols;             // gate/up: I (columns of each of gate and up); down: H
  int w_rows;            // weight rows per expert (= K)
  const int4* chunks;    // {expert, first row, rows <= ROWS}
  const int32_t* sched;  // [0] number of chunks
  uint16_t* h;           // gate/up output [R, I] bf16
  const int32_t* perm;   // down: token of each row
  const float* row_w;    // down: routing weight of each row
  float* out;            // down: [T, H] fp32 (zero on entry)
  int H;
  uint32_t* status;
  float4* zero4;         // gate/up: region zero-filled before the dependency wait, or null
  size_t n_zero4;
};

// Columns of output per tile: gate/up 128 (the same 128 columns of gate and of up), down 256.
template <int MODE>
MOE_DEVINL int et_tile_cols() { return MODE == 0 ? kEtM : 2 * kEtM; }

// 64-column boxes of matrix j (0, 1) that hold valid columns, for a tile whose first output
// column is n0 (gate/up: both matrices span the same columns).
template <int MODE>
MOE_DEVINL int et_boxes(int j, int n0, int Ncols) {
  const int vc = min(et_tile_cols<MODE>(), Ncols - n0) / 64;   // Ncols % 64 == 0
  if (MODE == 0) return vc;
  return j == 0 ? min(2, vc) : max(0, vc - 2);
}

// Epilogue of the expert-tile kernels (warps 2-5, one TMEM lane quarter each): waits for each
// tile's accumulators, writes h = silu(g) * u (gate/up) or adds w * y into out (down) through a
// shared-memory transpose, and hands the accumulator buffer back.
template <int MODE, int ROWS>
MOE_DEVINL void et_epilogue(const EtArgs& a, uint32_t tmem_base, uint64_t* acc_full,
                            uint64_t* acc_empty, float* epi, int tiles, int NT,
                            volatile int* abort_flag) {
  using C = EtCfg<ROWS>;
  constexpr int TW = MODE == 0 ? kEtM : 2 * kEtM;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int q = warp & 3;                       // TMEM lanes 32q .. 32q + 31
  float* stage = epi + (warp - 2) * 32 * kEtPitch;
  int tile_i = 0;
  for (int t = blockIdx.x; t < tiles; t += gridDim.x, ++tile_i) {
    const int buf = tile_i % C::kAccBufs;
    const uint32_t aph = (tile_i / C::kAccBufs) & 1u;
    if (!wait_or_abort(&acc_full[buf], aph, abort_flag, a.status)) break;
    tc_fence_after();
    const int4 ch = a.chunks[t / NT];
    const int n0 = (t % NT) * TW;
    const int nrows = ch.z;
    const uint32_t tbase = tmem_base + ((uint32_t)(32 * q) << 16) + buf * 2 * ROWS;
    if constexpr (MODE == 0) {
      // this warp's 32 columns of gate and up: valid when the tile's last box is
      const bool cols_ok = n0 + 32 * q < a.Ncols;  // warp-uniform
      for (int r0 = 0; cols_ok && r0 < nrows; r0 += 32) {
        float g[32], u[32];
        tmem_ld32(tbase + r0, g);
        tmem_ld32(tbase + ROWS + r0, u);
#pragma unroll
        for (int i = 0; i < 32; ++i) stage[i * kEtPitch + lane] = silu_fast(g[i]) * u[i];
        __syncwarp();
        // rows r0 + rr, 8 columns (16 bytes of h) per lane
#pragma unroll
        for (int it2 = 0; it2 < 4; ++it2) {
          const int rr = (lane >> 2) + 8 * it2, cc = 8 * (lane & 3);
          if (r0 + rr < nrows) {
            const float* sp = stage + rr * kEtPitch + cc;
            const uint4 v = make_uint4(pack_bf16x2(sp[0], sp[1]), pack_bf16x2(sp[2], sp[3]),
                                       pack_bf16x2(sp[4], sp[5]), pack_bf16x2(sp[6], sp[7]));
            *reinterpret_cast<uint4*>(a.h + (size_t)(ch.y + r0 + rr) * a.Ncols + n0 + 32 * q + cc) = v;
          }
        }
        __syncwarp();
      }
    } else {
#pragma unroll 1
      for (int j = 0; j < 2; ++j) {
        const int col0 = n0 + j * kEtM + 32 * q;
        if (col0 >= a.Ncols) continue;  // warp-uniform: columns past H
        for (int r0 = 0; r0 < nrows; r0 += 32) {
          float y[32];
          tmem_ld32(tbase + j * ROWS + r0, y);
          const bool rv = r0 + lane < nrows;
          const int tok = rv ? a.perm[ch.y + r0 + lane] : -1;
          const float w = rv ? a.row_w[ch.y + r0 + lane] : 0.f;
#pragma unroll
          for (int i = 0; i < 32; ++i)
            stage[i * kEtPitch + lane] = __shfl_sync(0xffffffffu, w, i) * y[i];
          __syncwarp();
          // rows r0 + rr, 4 columns (one 16-byte vector atomic) per lane
#pragma unroll
          for (int it2 = 0; it2 < 8; ++it2) {
            const int rr = (lane >> 3) + 4 * it2, cc = 4 * (lane & 7);
            const int tk = __shfl_sync(0xffffffffu, tok, rr);
            if (tk >= 0) {
              const float* sp = stage + rr * kEtPitch + cc;
              red_add_f32x4(a.out + (size_t)tk * a.H + col0 + cc, sp[0], sp[1], sp[2], sp[3]);
            }
          }
          __syncwarp();
        }
      }
    }
    tc_fence_before();
    mbar_arrive(&acc_empty[buf]);
  }
}

// MODE 0: gate/up projection with the SwiGLU epilogue.  MODE 1: down projection with the
// routing-weight + combine epilogue.  wmap: the weights as [E*K rows, columns], box 64 x 64,
// 128-byte swizzle.  xmap: the activation rows [R, K], box 16 x 64, 128-byte swizzle.
template <int MODE, int ROWS = kEtRows>
__global__ void __launch_bounds__(kEtThreads, 1)
    expert_tile_kernel(const EtArgs a, const __grid_constant__ CUtensorMap wmap,
                       const __grid_constant__ CUtensorMap xmap) {
  using C = EtCfg<ROWS>;
  constexpr int kStages = C::kStages, kStageBytes = C::kStageBytes, kBufs = C::kAccBufs;
  extern __shared__ __align__(128) uint8_t smem_raw[];
  __shared__ uint32_t s_tmem;
  __shared__ int s_abort;
  uint8_t* ring = align1k(smem_raw);
  uint64_t* bars = reinterpret_cast<uint64_t*>(ring + kStages * kStageBytes);
  uint64_t* full = bars;
  uint64_t* empty = full + kStages;
  uint64_t* acc_full = empty + kStages;
  uint64_t* acc_empty = acc_full + 2;
  uint64_t* drain = acc_empty + 2;
  float* epi = reinterpret_cast<float*>(ring + kStages * kStageBytes + 256);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  if (warp == 1) {
    tmem_alloc(&s_tmem, kEtTmemCols);
    tmem_relinquish();
  }
  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < kBufs; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], 128);
    }
    mbar_init(drain, 1);
    s_abort = 0;
    fence_barrier_init();
    tma_prefetch_desc(&wmap);
    tma_prefetch_desc(&xmap);
  }
  // gate/up: the zero-fill of the down projection's output (only this call's down kernels
  // write it, and they run after this kernel)
  if (MODE == 0 && a.zero4 != nullptr)
    for (size_t i = (size_t)blockIdx.x * blockDim.x + tid; i < a.n_zero4;
         i += (size_t)gridDim.x * blockDim.x)
      a.zero4[i] = make_float4(0.f, 0.f, 0.f, 0.f);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = s_tmem;
  pdl_wait();  // work list, activation rows and (down) h come from the previous kernels
  pdl_launch_next();

  constexpr int TW = MODE == 0 ? kEtM : 2 * kEtM;
  const int NT = (a.Ncols + TW - 1) / TW;
  const int tiles = a.sched[0] * NT;
  const int nk = a.K / kEtBK;
  volatile int* abort_flag = &s_abort;

  if (warp == 0) {
    // ------------------------------ TMA producer ------------------------------
    if (lane == 0) {
      uint32_t it = 0;
      int last_it[kStages];
#pragma unroll
      for (int s = 0; s < kStages; ++s) last_it[s] = -1;
      for (int t = blockIdx.x; t < tiles && !*abort_flag; t += gridDim.x) {
        const int4 ch = a.chunks[t / NT];
        const int n0 = (t % NT) * TW;
        const int nb0 = et_boxes<MODE>(0, n0, a.Ncols), nb1 = et_boxes<MODE>(1, n0, a.Ncols);
        // first weight column of matrix j: gate / up block, or the two halves of the tile
        const int c0 = n0, c1 = MODE == 0 ? a.Ncols + n0 : n0 + kEtM;
        const int nrb = (ch.z + kEtRowBox - 1) / kEtRowBox;
        const uint32_t bytes = (uint32_t)(nb0 + nb1) * kEtBoxBytes + (uint32_t)nrb * kEtRowBox * kEtBK * 2;
        const int wrow0 = ch.x * a.w_rows;
        bool ok = true;
        for (int kst = 0; kst < nk; ++kst, ++it) {
          const int slot = it % kStages;
          const uint32_t ph = (it / kStages) & 1u;
          if (!wait_or_abort(&empty[slot], ph ^ 1u, abort_flag, a.status)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&full[slot], bytes);
          uint8_t* st = ring + slot * kStageBytes;
          const int k0 = kst * kEtBK;
          for (int b = 0; b < nb0; ++b)
            tma_load_2d(st + b * kEtBoxBytes, &wmap, c0 + 64 * b, wrow0 + k0, &full[slot]);
          for (int b = 0; b < nb1; ++b)
            tma_load_2d(st + (2 + b) * kEtBoxBytes, &wmap, c1 + 64 * b, wrow0 + k0, &full[slot]);
          for (int r = 0; r < nrb; ++r)
            tma_load_2d(st + kEtABytes + r * (kEtRowBox * kEtBK * 2), &xmap, k0,
                        ch.y + r * kEtRowBox, &full[slot]);
          last_it[slot] = it;
        }
        if (!ok) break;
      }
      // never leave the CTA with copies in flight
      for (int s = 0; s < kStages; ++s)
        if (last_it[s] >= 0 &&
            !mbar_wait_bounded(&full[s], (last_it[s] / kStages) & 1u, kWaitLimitNs))
          atomicOr(a.status, kStatusTimeout);
    }
  } else if (warp == 1) {
    // ------------------------------ MMA issuer ------------------------------
    if (lane == 0) {
      const uint32_t ring_s = smem_u32(ring);
      // slot 0's descriptors; a slot / K-step offset only moves the 14-bit start address
      // (addresses stay below 256 KB, so adding (offset >> 4) never carries out of the field)
      const uint64_t adesc0 = smem_desc_sw128(ring_s, kEtBoxBytes, 1024);          // MN-major
      const uint64_t bdesc0 = smem_desc_sw128(ring_s + kEtABytes, 16, 1024);       // K-major
      uint32_t it = 0;
      int tile_i = 0;
      bool issued = false;
      for (int t = blockIdx.x; t < tiles && !*abort_flag; t += gridDim.x, ++tile_i) {
        const int4 ch = a.chunks[t / NT];
        const int n0 = (t % NT) * TW;
        const int nb0 = et_boxes<MODE>(0, n0, a.Ncols), nb1 = et_boxes<MODE>(1, n0, a.Ncols);
        const int N = ((ch.z + kEtRowBox - 1) / kEtRowBox) * kEtRowBox;
        const uint32_t idesc = idesc_bf16_f32(kEtM, N, /*a_mn_major=*/true, /*b_mn_major=*/false);
        const int buf = tile_i % kBufs;
        const uint32_t aph = (tile_i / kBufs) & 1u;
        if (!wait_or_abort(&acc_empty[buf], aph ^ 1u, abort_flag, a.status)) break;
        tc_fence_after();
        const uint32_t d0 = tmem_base + buf * 2 * ROWS, d1 = d0 + ROWS;
        bool ok = true;
        for (int kst = 0; kst < nk; ++kst, ++it) {
          const int slot = it % kStages;
          const uint32_t ph = (it / kStages) & 1u;
          if (!wait_or_abort(&full[slot], ph, abort_flag, a.status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t soff = (uint64_t)((slot * kStageBytes) >> 4);
#pragma unroll
          for (int k16 = 0; k16 < kEtBK / 16; ++k16) {
            const uint64_t ak = adesc0 + soff + ((k16 * 16 * 128) >> 4);
            const uint64_t bk = bdesc0 + soff + ((k16 * 32) >> 4);
            const uint32_t acc = (kst | k16) != 0;
            if (nb0) tc_mma_bf16(d0, ak, bk, idesc, acc);
            if (nb1) tc_mma_bf16(d1, ak + ((2 * kEtBoxBytes) >> 4), bk, idesc, acc);
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
    et_epilogue<MODE, ROWS>(a, tmem_base, acc_full, acc_empty, epi, tiles, NT, abort_flag);
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem_base, kEtTmemCols);
}

}  // namespace moe
