// Expert-tile grouped GEMM with MXFP4 expert weights (W4A16) on the 5th-generation tensor cores.
//
// The checkpoints' experts are natively MXFP4 with bf16 activations (Persona Kappa forum post,
// "Quantization-Aware Training").  The block-scaled tcgen05 MMA kinds take both operands in a
// narrow format (the activations would have to be quantized too), so this kernel keeps the
// activations in bf16 and widens the weights on chip: the E2M1 codes and E8M0 scales stream from
// HBM at a quarter of the bf16 weight bytes, converter warps expand each [128 columns x 64 K]
// block into bf16 in shared memory, and the same kind::f16 MMA as the bf16 expert-tile kernel
// multiplies it with the rows.  An E2M1 value times 2^(s - 127) has at most two significant bits,
// so the bf16 weight is exact for scale codes 2 <= s <= 252 (smaller s: bf16 subnormals, exact
// down to 2^-133; larger s with large codes: beyond bf16's range).
//
//   warp 0      TMA producer: per K stage of 64, the codes of two 128-column matrices ([128 rows
//               x 32 bytes] boxes of the [columns, K/2] code layout) and their scales ([2 x 128]
//               boxes of the [K/32, columns] layout) into a deep ring (8 stages of 8.5 KB)
//   warps 6-13  converters: four warps per matrix, thread c widens column c (64 codes) to bf16 in
//               the 128-byte-swizzled K-major layout (the A operand), and one of them issues the
//               TMA loads of the stage's activation rows (the B operand), into a 2-stage ring
//   warp 1      TMEM owner and MMA issuer: two tcgen05.mma M = 128, N = rows per K step of 16
//               (A K-major here), commits release the stage and hand over the accumulators
//   warps 2-5   epilogue, as in the bf16 expert-tile kernel (SwiGLU / weighted fp32 combine)
//
// Tiles, work lists, accumulators and the epilogue are those of expert_tile_kernel.  Every wait
// is bounded: on a timeout the CTA records it, winds down, drains its copies and MMAs, frees the
// tensor memory and returns.
#pragma once

#include "common.cuh"
#include "expert_gemm.cuh"
#include "stream_mx.cuh"

namespace moe {

constexpr int kEmxRawStages = 8;
constexpr int kEmxAbStages = 2;
constexpr int kEmxConvWarp0 = 6;
constexpr int kEmxConvWarps = 8;                              // one per matrix row of 64 codes
constexpr int kEmxThreads = 32 * (kEmxConvWarp0 + kEmxConvWarps);   // 14 warps
constexpr int kEmxCodesBytes = kEtM * (kEtBK / 2);            // 4 KB: 128 columns x 32 bytes
constexpr int kEmxScaleBytes = (kEtBK / 32) * kEtM;           // 256 B: 2 blocks x 128 columns
constexpr int kEmxRawBytes = 2 * kEmxCodesBytes + 2 * kEmxScaleBytes;   // 8.5 KB
constexpr int kEmxABytes = 2 * kEtM * kEtBK * 2;              // 32 KB: two bf16 matrices
constexpr int kEmxAbBytes = kEmxABytes + kEtBBytes;           // 48 KB
constexpr int kEmxSmem = 1024 + kEmxAbStages * kEmxAbBytes + kEmxRawStages * kEmxRawBytes + 256 +
                         kEtEpiBytes;
static_assert(kEmxRawBytes % 128 == 0, "TMA destinations stay 128-byte aligned");
static_assert(kEmxSmem <= 227 * 1024, "shared memory");

// Two fp32 values to a bf16 pair (hardware round to nearest even), first in the low half.
MOE_DEVINL uint32_t cvt_bf16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

// Eight E2M1 codes (one 32-bit word, first element in the low nibble of byte 0) times the block
// scale to eight bf16 values (16 bytes, K order).  Every step is exact: E2M1 -> f16 -> fp32, a
// product with a power of two, and bf16 holds the result (see the file comment).
MOE_DEVINL uint4 e2m1x8_scaled_bf16(uint32_t w, float scale) {
  uint32_t h[4];
  e2m1x8_to_f16x2(w, h);
  uint32_t o[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float lo, hi;
    asm("{\n .reg .f16 a, b;\n mov.b32 {a, b}, %2;\n cvt.f32.f16 %0, a;\n cvt.f32.f16 %1, b;\n}"
        : "=f"(lo), "=f"(hi)
        : "r"(h[i]));
    o[i] = cvt_bf16x2(lo * scale, hi * scale);
  }
  return make_uint4(o[0], o[1], o[2], o[3]);
}

// MODE 0: gate/up projection with the SwiGLU epilogue; MODE 1: down projection with the
// routing-weight + combine epilogue.  cmap: codes [E*N rows, K/2 bytes], box 128 x 32.  smap:
// scales [E*K/32 rows, N bytes], box 2 x 128.  xmap: activation rows [R, K], box 16 x 64, 128-byte
// swizzle.
template <int MODE>
__global__ void __launch_bounds__(kEmxThreads, 1)
    expert_tile_mx_kernel(const EtArgs a, const __grid_constant__ CUtensorMap cmap,
                          const __grid_constant__ CUtensorMap smap,
                          const __grid_constant__ CUtensorMap xmap) {
  extern __shared__ __align__(128) uint8_t smem_raw[];
  __shared__ uint32_t s_tmem;
  __shared__ int s_abort;
  uint8_t* ab = align1k(smem_raw);                               // [2][A 32 KB | B 16 KB]
  uint8_t* raw = ab + kEmxAbStages * kEmxAbBytes;                // [8][codes 8 KB | scales 512]
  uint64_t* bars = reinterpret_cast<uint64_t*>(raw + kEmxRawStages * kEmxRawBytes);
  uint64_t* raw_full = bars;
  uint64_t* raw_empty = raw_full + kEmxRawStages;
  uint64_t* ab_full = raw_empty + kEmxRawStages;
  uint64_t* ab_empty = ab_full + kEmxAbStages;
  uint64_t* acc_full = ab_empty + kEmxAbStages;
  uint64_t* acc_empty = acc_full + 2;
  uint64_t* drain = acc_empty + 2;
  float* epi = reinterpret_cast<float*>(raw + kEmxRawStages * kEmxRawBytes + 256);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  if (warp == 1) {
    tmem_alloc(&s_tmem, kEtTmemCols);
    tmem_relinquish();
  }
  if (tid == 0) {
    for (int s = 0; s < kEmxRawStages; ++s) {
      mbar_init(&raw_full[s], 1);
      mbar_init(&raw_empty[s], kEmxConvWarps);
    }
    for (int s = 0; s < kEmxAbStages; ++s) {
      mbar_init(&ab_full[s], 1 + kEmxConvWarps);  // the row loads' expect_tx + the converters
      mbar_init(&ab_empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], 128);
    }
    mbar_init(drain, 1);
    s_abort = 0;
    fence_barrier_init();
    tma_prefetch_desc(&cmap);
    tma_prefetch_desc(&smap);
    tma_prefetch_desc(&xmap);
  }
  if (MODE == 0 && a.zero4 != nullptr)
    for (size_t i = (size_t)blockIdx.x * blockDim.x + tid; i < a.n_zero4;
         i += (size_t)gridDim.x * blockDim.x)
      a.zero4[i] = make_float4(0.f, 0.f, 0.f, 0.f);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = s_tmem;
  pdl_wait();
  pdl_launch_next();

  constexpr int TW = MODE == 0 ? kEtM : 2 * kEtM;
  const int NT = (a.Ncols + TW - 1) / TW;
  const int tiles = a.sched[0] * NT;
  const int nk = a.K / kEtBK;
  const int kblk = a.K / 32;                                      // scale rows per expert
  volatile int* abort_flag = &s_abort;

  if (warp == 0) {
    // ------------------------------ codes and scales ------------------------------
    if (lane == 0) {
      uint32_t it = 0;
      int last_it[kEmxRawStages];
#pragma unroll
      for (int s = 0; s < kEmxRawStages; ++s) last_it[s] = -1;
      for (int t = blockIdx.x; t < tiles && !*abort_flag; t += gridDim.x) {
        const int4 ch = a.chunks[t / NT];
        const int n0 = (t % NT) * TW;
        const bool m0 = et_boxes<MODE>(0, n0, a.Ncols) > 0, m1 = et_boxes<MODE>(1, n0, a.Ncols) > 0;
        const int c0 = n0, c1 = MODE == 0 ? a.Ncols + n0 : n0 + kEtM;   // first weight column
        const int ncols_all = MODE == 0 ? 2 * a.Ncols : a.Ncols;          // columns per expert
        const uint32_t bytes = (uint32_t)((m0 ? 1 : 0) + (m1 ? 1 : 0)) * (kEmxCodesBytes + kEmxScaleBytes);
        bool ok = true;
        for (int kst = 0; kst < nk; ++kst, ++it) {
          const int slot = it % kEmxRawStages;
          const uint32_t ph = (it / kEmxRawStages) & 1u;
          if (!wait_or_abort(&raw_empty[slot], ph ^ 1u, abort_flag, a.status)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&raw_full[slot], bytes);
          uint8_t* st = raw + slot * kEmxRawBytes;
          const int crow = ch.x * ncols_all;                 // first code row of this expert
          const int srow = ch.x * kblk + kst * (kEtBK / 32); // first scale row of this stage
          if (m0) {
            tma_load_2d(st, &cmap, kst * (kEtBK / 2), crow + c0, &raw_full[slot]);
            tma_load_2d(st + 2 * kEmxCodesBytes, &smap, c0, srow, &raw_full[slot]);
          }
          if (m1) {
            tma_load_2d(st + kEmxCodesBytes, &cmap, kst * (kEtBK / 2), crow + c1, &raw_full[slot]);
            tma_load_2d(st + 2 * kEmxCodesBytes + kEmxScaleBytes, &smap, c1, srow, &raw_full[slot]);
          }
          last_it[slot] = it;
        }
        if (!ok) break;
      }
      for (int s = 0; s < kEmxRawStages; ++s)
        if (last_it[s] >= 0 &&
            !mbar_wait_bounded(&raw_full[s], (last_it[s] / kEmxRawStages) & 1u, kWaitLimitNs))
          atomicOr(a.status, kStatusTimeout);
    }
  } else if (warp >= kEmxConvWarp0) {
    // ------------------------------ converters (+ activation rows) ------------------------------
    const int cti = tid - kEmxConvWarp0 * 32;                       // 0..255
    const int j = cti / kEtM, ct = cti % kEtM;                      // matrix, weight column
    uint32_t it = 0;
    int last_ab[kEmxAbStages] = {-1, -1};
    bool aborted = false;
    for (int t = blockIdx.x; t < tiles && !aborted; t += gridDim.x) {
      const int4 ch = a.chunks[t / NT];
      const int n0 = (t % NT) * TW;
      const bool m0 = et_boxes<MODE>(0, n0, a.Ncols) > 0, m1 = et_boxes<MODE>(1, n0, a.Ncols) > 0;
      const int nrb = (ch.z + kEtRowBox - 1) / kEtRowBox;
      const uint32_t xbytes = (uint32_t)nrb * kEtRowBox * kEtBK * 2;
      for (int kst = 0; kst < nk; ++kst, ++it) {
        const int rs = it % kEmxRawStages, as = it % kEmxAbStages;
        const uint32_t rph = (it / kEmxRawStages) & 1u, aph = (it / kEmxAbStages) & 1u;
        // every lane waits itself: the codes it reads were written by TMA, and the A slot it
        // overwrites was last read by the MMAs
        bool ok = wait_or_abort(&raw_full[rs], rph, abort_flag, a.status) &&
                  wait_or_abort(&ab_empty[as], aph ^ 1u, abort_flag, a.status);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) {
          aborted = true;
          break;
        }
        uint8_t* abs_ = ab + as * kEmxAbBytes;
        if (cti == 0) {  // this stage's activation rows (the B operand)
          mbar_arrive_expect_tx(&ab_full[as], xbytes);
          for (int r = 0; r < nrb; ++r)
            tma_load_2d(abs_ + kEmxABytes + r * (kEtRowBox * kEtBK * 2), &xmap, kst * kEtBK,
                        ch.y + r * kEtRowBox, &ab_full[as]);
          last_ab[as] = (int)it;
        }
        const uint8_t* rst = raw + rs * kEmxRawBytes;
        if (j == 0 ? m0 : m1) {  // warp-uniform: four warps per matrix
          const uint4* codes = reinterpret_cast<const uint4*>(rst + j * kEmxCodesBytes + ct * 32);
          const uint8_t* sc = rst + 2 * kEmxCodesBytes + j * kEmxScaleBytes;
          const float s0 = e8m0_to_f32(sc[ct]), s1 = e8m0_to_f32(sc[kEtM + ct]);
          const uint4 q0 = codes[0], q1 = codes[1];               // 64 codes: K 0-31, 32-63
          const uint32_t w[8] = {q0.x, q0.y, q0.z, q0.w, q1.x, q1.y, q1.z, q1.w};
          uint8_t* arow = abs_ + j * (kEtM * kEtBK * 2) + ct * 128;
#pragma unroll
          for (int c = 0; c < 8; ++c)
            *reinterpret_cast<uint4*>(arow + ((c ^ (ct & 7)) << 4)) =
                e2m1x8_scaled_bf16(w[c], c < 4 ? s0 : s1);
        }
        fence_proxy_async_smem();  // the MMA reads A through the async proxy
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&ab_full[as]);
          mbar_arrive(&raw_empty[rs]);
        }
      }
    }
    // never leave the CTA with row copies in flight
    if (cti == 0)
      for (int s = 0; s < kEmxAbStages; ++s)
        if (last_ab[s] >= 0 &&
            !mbar_wait_bounded(&ab_full[s], (last_ab[s] / kEmxAbStages) & 1u, kWaitLimitNs))
          atomicOr(a.status, kStatusTimeout);
  } else if (warp == 1) {
    // ------------------------------ MMA issuer ------------------------------
    if (lane == 0) {
      const uint32_t ab_s = smem_u32(ab);
      const uint64_t adesc0 = smem_desc_sw128(ab_s, 16, 1024);               // K-major
      const uint64_t bdesc0 = smem_desc_sw128(ab_s + kEmxABytes, 16, 1024);  // K-major
      uint32_t it = 0;
      int tile_i = 0;
      bool issued = false;
      for (int t = blockIdx.x; t < tiles && !*abort_flag; t += gridDim.x, ++tile_i) {
        const int4 ch = a.chunks[t / NT];
        const int n0 = (t % NT) * TW;
        const bool m0 = et_boxes<MODE>(0, n0, a.Ncols) > 0, m1 = et_boxes<MODE>(1, n0, a.Ncols) > 0;
        const int N = ((ch.z + kEtRowBox - 1) / kEtRowBox) * kEtRowBox;
        const uint32_t idesc = idesc_bf16_f32(kEtM, N, /*a_mn_major=*/false, /*b_mn_major=*/false);
        const int buf = tile_i & 1;
        const uint32_t aph = (tile_i >> 1) & 1u;
        if (!wait_or_abort(&acc_empty[buf], aph ^ 1u, abort_flag, a.status)) break;
        tc_fence_after();
        const uint32_t d0 = tmem_base + buf * 2 * kEtM, d1 = d0 + kEtM;
        bool ok = true;
        for (int kst = 0; kst < nk; ++kst, ++it) {
          const int slot = it % kEmxAbStages;
          const uint32_t ph = (it / kEmxAbStages) & 1u;
          if (!wait_or_abort(&ab_full[slot], ph, abort_flag, a.status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t soff = (uint64_t)((slot * kEmxAbBytes) >> 4);
#pragma unroll
          for (int k16 = 0; k16 < kEtBK / 16; ++k16) {
            const uint64_t ak = adesc0 + soff + ((k16 * 32) >> 4);
            const uint64_t bk = bdesc0 + soff + ((k16 * 32) >> 4);
            const uint32_t acc = (kst | k16) != 0;
            if (m0) tc_mma_bf16(d0, ak, bk, idesc, acc);
            if (m1) tc_mma_bf16(d1, ak + ((kEtM * kEtBK * 2) >> 4), bk, idesc, acc);
          }
          tc_commit(&ab_empty[slot]);
          issued = true;
        }
        if (!ok) break;
        tc_commit(&acc_full[buf]);
      }
      if (issued) {
        tc_commit(drain);
        if (!mbar_wait_bounded(drain, 0, kWaitLimitNs)) atomicOr(a.status, kStatusTimeout);
      }
    }
  } else {
    // ------------------------------ epilogue (warps 2-5) ------------------------------
    et_epilogue<MODE, kEtRows>(a, tmem_base, acc_full, acc_empty, epi, tiles, NT, abort_flag);
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem_base, kEtTmemCols);
}

}  // namespace moe
