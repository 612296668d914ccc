// Weight-streaming expert kernels for MXFP4 experts (W4A16: 4-bit weights, bf16 activations).
//
// The experts' native format (Persona Kappa forum post, "Quantization-Aware Training": MXFP4,
// activations kept in bf16), read as OCP Microscaling FP4: E2M1 codes in blocks of 32 along the
// reduction dimension K, each block of a weight column sharing one E8M0 scale 2^(s - 127).
// Storage per expert of a [K, N] matrix: codes [N, K/2] bytes (row n = weight column n; byte j
// holds element 2j in bits 0-3 and 2j + 1 in bits 4-7) and scales [K/32, N] bytes.
//
// Same persistent, stream-K organisation as the bf16 streaming kernels (stream.cuh): one CTA
// per SM, a producer warp and consumer warps around a shared-memory ring, tiles of (row chunk
// of one expert, 160 weight columns for gate/up, 320 for down), the same epilogues.  What
// changes is the weight stream, a quarter of the bytes:
//
//   * per stage, 256 K (the last stage of a row holds what is left: H = 2880 is 11 * 256 + 64):
//     one TMA box of [32 columns x 128 bytes] codes per 32-column group and matrix (128-byte
//     swizzle; whole 128-byte rows, so a stage needs as few copy requests per byte as the bf16
//     kernels), one box of [8 blocks x 32 columns] scales, and the rows' activations (bulk
//     copies);
//   * consumer warps own one 16-column m-tile each: ten for gate/up (gate and up of the same
//     columns, for the SwiGLU), twenty for down (one matrix leaves room for both);
//   * a thread's A fragment of mma.sync m16n8k16 comes from one 32-bit shared load per weight
//     column: the K order inside each 32-element block is permuted so that thread t of a quad
//     holds elements 8t..8t+7 (the same permutation on the activation side, whose 8 values are
//     one 16-byte load);
//   * the hardware converts each code pair to f16 (cvt.rn.f16x2.e2m1x2, exact: E2M1 values
//     are f16 numbers; there is no bf16 form), and the products run as f16 MMAs: one block's
//     two MMAs give an fp32 tile that is added to the accumulator times the block's E8M0 scale
//     (fp32, exact for every scale).  The activations are therefore f16: the layer input is
//     converted once per call (to_f16_kernel) and the gate/up kernel writes h in f16.
//     Converting a bf16 value to f16 is exact for magnitudes 2^-14 .. 65504 (f16 keeps more
//     mantissa bits than bf16); below that range f16 keeps fewer bits, above it the value
//     overflows to infinity.  That range is the one departure from bf16 arithmetic.
#pragma once

#include "stream.cuh"

namespace moe {

constexpr int kMxWarps = 10;                        // consumer warps, one m-tile each
constexpr int kMxConsumers = 32 * kMxWarps;
constexpr int kMxThreads = kMxConsumers + 32;       // + 1 producer warp
constexpr int kMxKC = 256;                          // K per stage (8 scale blocks)
constexpr int kMxBoxRows = 32;                      // weight columns per box (two warps)
constexpr int kMxTileCols = 160;                    // weight columns per tile and matrix
constexpr int kMxBoxes = kMxTileCols / kMxBoxRows;  // boxes per tile and matrix
constexpr int kMxBoxBytes = kMxBoxRows * kMxKC / 2;  // 4 KB of codes, 128-byte rows
constexpr int kMxScaleBytes = (kMxKC / 32) * kMxBoxRows;  // 256 B: [8 blocks][32 columns]
constexpr int kMxXPitch = kMxKC * 2 + 64;           // 576 B per activation row (144 words): the
                                                    // 16-byte fragment loads hit no bank twice
// The down kernel has one matrix, so it affords twice the tile width and twice the warps.
constexpr int kMxDnWarps = 2 * kMxWarps;
constexpr int kMxDnConsumers = 32 * kMxDnWarps;
constexpr int kMxDnThreads = kMxDnConsumers + 32;
constexpr int kMxDnTileCols = 2 * kMxTileCols;             // 320 columns of H
constexpr int kMxDnBoxes = kMxDnTileCols / kMxBoxRows;     // 10
constexpr int kMxGUW = 2 * kMxBoxes * kMxBoxBytes;         // gate + up codes, 40 KB
constexpr int kMxGUS = 2 * kMxBoxes * kMxScaleBytes;       // 2.5 KB
constexpr int kMxDNW = kMxDnBoxes * kMxBoxBytes;           // 40 KB
constexpr int kMxDNS = kMxDnBoxes * kMxScaleBytes;         // 2.5 KB
constexpr int kMxX = kStreamRB * kMxXPitch;                // 9 KB
constexpr int kMxGUStage = (kMxGUW + kMxGUS + kMxX + 1023) / 1024 * 1024;  // 53 KB
constexpr int kMxDNStage = (kMxDNW + kMxDNS + kMxX + 1023) / 1024 * 1024;  // 53 KB
constexpr int kMxGUStages = 4;
constexpr int kMxDNStages = 4;
constexpr int kMxGateUpSmem = 1024 + kMxGUStages * kMxGUStage + 2 * kMxGUStages * 8;
constexpr int kMxDownSmem = 1024 + kMxDNStages * kMxDNStage + 2 * kMxDNStages * 8;
static_assert(kMxGateUpSmem <= 227 * 1024 && kMxDownSmem <= 227 * 1024, "shared memory");

// Byte offset of 16-byte chunk c of row r in a box of 128-byte rows stored with the 128-byte
// swizzle (chunk index XOR row bits 0-2; the box starts on a 1024-byte boundary).
MOE_DEVINL uint32_t sw128_offset(int r, int c) {
  return (uint32_t)(r * 128 + ((c ^ (r & 7)) << 4));
}

// Four code pairs (one 32-bit word, pair i in byte i, first element in the low nibble) to four
// f16x2 values, first element in the low half.
MOE_DEVINL void e2m1x8_to_f16x2(uint32_t w, uint32_t (&h)[4]) {
  asm("{\n .reg .b8 b0, b1, b2, b3;\n mov.b32 {b0, b1, b2, b3}, %4;\n"
      " cvt.rn.f16x2.e2m1x2 %0, b0;\n cvt.rn.f16x2.e2m1x2 %1, b1;\n"
      " cvt.rn.f16x2.e2m1x2 %2, b2;\n cvt.rn.f16x2.e2m1x2 %3, b3;\n}"
      : "=r"(h[0]), "=r"(h[1]), "=r"(h[2]), "=r"(h[3])
      : "r"(w));
}

// Two fp32 values to an f16 pair (round to nearest), first in the low half.
MOE_DEVINL uint32_t pack_f16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

// The layer input in f16 for the MXFP4 streaming kernels: x16[i] = f16(x[i]) for n elements
// (n even).  An input beyond f16's range sets kStatusF16Range in the status word (its f16 value
// is infinite).  grid-stride, 8 elements per thread and step.
__global__ void __launch_bounds__(256) to_f16_kernel(const uint16_t* __restrict__ x,
                                                     uint16_t* __restrict__ x16, size_t n,
                                                     uint32_t* status) {
  pdl_wait();  // x16 may still be read by the previous call's gate/up kernel until it ends
  pdl_launch_next();
  const size_t n8 = n / 8;
  for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n8;
       i += (size_t)gridDim.x * blockDim.x) {
    const uint4 v = reinterpret_cast<const uint4*>(x)[i];
    const uint32_t in[4] = {v.x, v.y, v.z, v.w};
    uint32_t o[4];
    bool big = false;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float lo = __uint_as_float(in[j] << 16), hi = __uint_as_float(in[j] & 0xffff0000u);
      big |= fabsf(lo) > 65504.f || fabsf(hi) > 65504.f;   // beyond f16: would become inf
      o[j] = pack_f16x2(lo, hi);
    }
    if (big) atomicOr(status, kStatusF16Range);
    reinterpret_cast<uint4*>(x16)[i] = make_uint4(o[0], o[1], o[2], o[3]);
  }
}

// d = A B (f16 in, fp32 out, zero accumulator in) and d += A B.
MOE_DEVINL void mma_f16_16816_zero(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                   uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%10,%10,%10,%10};"
      : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1), "f"(0.f));
}
MOE_DEVINL void mma_f16_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                              uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// E8M0 scale code to its value 2^(s - 127): the exponent field s, except s = 0 (the fp32
// subnormal 2^-127, bit pattern 0x00400000, larger than 0 << 23 and below every 1 << 23 and
// up) and s = 255 (NaN).
MOE_DEVINL float e8m0_to_f32(uint32_t s) {
  const uint32_t b = max(s << 23, 0x00400000u);
  return __uint_as_float(s == 255 ? 0x7fc00000u : b);
}

MOE_DEVINL uint32_t lds_u8(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.shared.u8 %0, [%1];" : "=r"(v) : "r"(addr));
  return v;
}

// Activation fragments (f16 rows) of one 32-element block for the permuted K order: rows g
// (n8 tile 0) and 8 + g (tile 1), elements 8t..8t+7, one 16-byte load; [nb][step][reg].
template <int NB>
MOE_DEVINL void mx_b_frags(uint32_t xbase, int kb, int lane, uint32_t (&b)[2][2][2]) {
  const int g = lane >> 2, t = lane & 3;
#pragma unroll
  for (int nb = 0; nb < NB; ++nb) {
    uint4 v;
    asm volatile("ld.shared.v4.b32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "r"(xbase + (uint32_t)((8 * nb + g) * kMxXPitch + (32 * kb + 8 * t) * 2)));
    b[nb][0][0] = v.x;
    b[nb][0][1] = v.y;
    b[nb][1][0] = v.z;
    b[nb][1][1] = v.w;
  }
}

// One matrix's contribution of one 32-element block to the accumulators of m-tile mt:
// box = shared address of this warp's codes box (32 rows), sc = of its scales ([8][32] bytes).
template <int NB>
MOE_DEVINL void mx_block_mma(uint32_t box, uint32_t sc, int mt, int kb, int lane,
                             const uint32_t (&b)[2][2][2], float (&acc)[2][4]) {
  const int g = lane >> 2, t = lane & 3;
  const int ra = 16 * mt + g, rb = ra + 8;
  uint32_t wa, wb;
  asm volatile("ld.shared.b32 %0, [%1];" : "=r"(wa) : "r"(box + sw128_offset(ra, kb) + 4 * t));
  asm volatile("ld.shared.b32 %0, [%1];" : "=r"(wb) : "r"(box + sw128_offset(rb, kb) + 4 * t));
  uint32_t ha[4], hb[4];
  e2m1x8_to_f16x2(wa, ha);
  e2m1x8_to_f16x2(wb, hb);
  const float sa = e8m0_to_f32(lds_u8(sc + kb * kMxBoxRows + ra));
  const float sb = e8m0_to_f32(lds_u8(sc + kb * kMxBoxRows + rb));
#pragma unroll
  for (int nb = 0; nb < NB; ++nb) {
    float tmp[4];
    mma_f16_16816_zero(tmp, ha[0], hb[0], ha[1], hb[1], b[nb][0][0], b[nb][0][1]);
    mma_f16_16816(tmp, ha[2], hb[2], ha[3], hb[3], b[nb][1][0], b[nb][1][1]);
    acc[nb][0] = fmaf(sa, tmp[0], acc[nb][0]);
    acc[nb][1] = fmaf(sa, tmp[1], acc[nb][1]);
    acc[nb][2] = fmaf(sb, tmp[2], acc[nb][2]);
    acc[nb][3] = fmaf(sb, tmp[3], acc[nb][3]);
  }
}


// Blocks of 32 elements in the stage that starts at k0 of a K-long reduction (the last stage
// of a row may be short).
MOE_DEVINL int mx_stage_blocks(int K, int k0) { return min(kMxKC, K - k0) / 32; }

// One stage of one warp: the m-tile's contribution from `nmat` matrices (gate/up: 2, down: 1)
// over the stage's valid blocks.  boxes[m] / scs[m]: shared addresses of the matrices' codes
// box and scales box of this warp's columns; xb: the rows' activations.
template <int NB, int NMAT>
MOE_DEVINL void mx_stage(const uint32_t (&boxes)[NMAT], const uint32_t (&scs)[NMAT], uint32_t xb,
                         int mt, int nkb, int lane, float (&acc)[NMAT][2][4]) {
#pragma unroll
  for (int kb = 0; kb < kMxKC / 32; ++kb) {
    if (kb < nkb) {
      uint32_t b[2][2][2];
      mx_b_frags<NB>(xb, kb, lane, b);
#pragma unroll
      for (int m = 0; m < NMAT; ++m) mx_block_mma<NB>(boxes[m], scs[m], mt, kb, lane, b, acc[m]);
    }
  }
}

// ------------------------------------------------------------------------------------------
// gate/up projection + SwiGLU, MXFP4 weights; a.x is the f16 copy of the input, a.h receives
// f16.  Codes of W_gate_up: [E * 2I rows, H/2 bytes]; scales: [E * H/32 rows, 2I bytes].
// ------------------------------------------------------------------------------------------
__global__ void __launch_bounds__(kMxThreads, 1)
    stream_gate_up_mx_kernel(const GateUpArgs a, const __grid_constant__ CUtensorMap cmap,
                             const __grid_constant__ CUtensorMap smap) {
  extern __shared__ __align__(128) uint8_t smem_raw[];
  __shared__ int s_last;
  uint8_t* ring = align1k(smem_raw);
  uint64_t* full = reinterpret_cast<uint64_t*>(ring + kMxGUStages * kMxGUStage);
  uint64_t* empty = full + kMxGUStages;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) {
    for (int s = 0; s < kMxGUStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kMxWarps);
    }
    fence_barrier_init();
  }
  __syncthreads();

  if (tid == kMxConsumers) {
    tma_prefetch_desc(&cmap);
    tma_prefetch_desc(&smap);
  }
  // `out` is written only by this call's down kernel, which cannot start before this one
  {
    float4* o4 = reinterpret_cast<float4*>(a.out);
    const size_t n4 = a.out_elems / 4;
    for (size_t i = (size_t)blockIdx.x * blockDim.x + tid; i < n4; i += (size_t)gridDim.x * blockDim.x)
      o4[i] = make_float4(0.f, 0.f, 0.f, 0.f);
  }
  pdl_wait();  // the routing results below come from the previous kernels
  pdl_launch_next();

  const int I2 = 2 * a.I;
  const int NT = (a.I + kMxTileCols - 1) / kMxTileCols;
  const int nk = (a.H + kMxKC - 1) / kMxKC;
  const StreamKRange rng = stream_k_range((long long)a.sched[0] * NT, nk);

  if (warp == kMxWarps) {
    // ---------------- producer ----------------
    bool aborted = false;
    uint32_t it = 0;
    int last_it[kMxGUStages];
#pragma unroll
    for (int s = 0; s < kMxGUStages; ++s) last_it[s] = -1;
    for (long long g = rng.g0; g < rng.g1;) {
      const int unit = (int)(g / nk), kb = (int)(g % nk);
      const int ke = (int)min((long long)nk, kb + (rng.g1 - g));
      g += ke - kb;
      const int4 ch = a.chunks[unit / NT];
      const int col0 = (unit % NT) * kMxTileCols;
      const int tok = (lane < ch.z) ? a.perm[ch.y + lane] : 0;
      // lanes 0-4: gate boxes, 5-9: the matching up boxes (codes); lanes 10-19 their scales
      const int j = lane % (2 * kMxBoxes);
      const int box_col = j < kMxBoxes ? col0 + kMxBoxRows * j
                                       : a.I + col0 + kMxBoxRows * (j - kMxBoxes);
      for (int kst = kb; kst < ke; ++kst, ++it) {
        const int slot = it % kMxGUStages;
        const uint32_t ph = (it / kMxGUStages) & 1u;
        if (!aborted && lane == 0 && !mbar_wait_bounded(&empty[slot], ph ^ 1u, kWaitLimitNs)) {
          aborted = true;
          record_timeout(a.status);
        }
        aborted = __shfl_sync(0xffffffffu, aborted, 0);
        if (aborted) continue;
        const int k0 = kst * kMxKC;
        const uint32_t xbytes = (uint32_t)min(kMxKC, a.H - k0) * 2u;
        // the boxes always deliver their full size (a short stage's columns past the row's end
        // are filled with zeros); the rows' copies only the stage's valid part
        if (lane == 0)
          mbar_arrive_expect_tx(&full[slot], (uint32_t)(kMxGUW + kMxGUS) + (uint32_t)ch.z * xbytes);
        __syncwarp();
        uint8_t* st = ring + slot * kMxGUStage;
        if (lane < 2 * kMxBoxes)
          tma_load_2d(st + lane * kMxBoxBytes, &cmap, k0 / 2, ch.x * I2 + box_col, &full[slot]);
        else if (lane < 4 * kMxBoxes)
          tma_load_2d(st + kMxGUW + j * kMxScaleBytes, &smap, box_col,
                      ch.x * (a.H / 32) + k0 / 32, &full[slot]);
        if (lane < ch.z)
          bulk_g2s(st + kMxGUW + kMxGUS + lane * kMxXPitch, a.x + (size_t)tok * a.H + k0, xbytes,
                   &full[slot]);
        last_it[slot] = it;
      }
    }
    // never leave the CTA with copies in flight
    if (lane == 0) {
      for (int s = 0; s < kMxGUStages; ++s)
        if (last_it[s] >= 0 &&
            !mbar_wait_bounded(&full[s], (last_it[s] / kMxGUStages) & 1u, kWaitLimitNs))
          record_timeout(a.status);
    }
    return;
  }

  // ---------------- consumers ----------------
  const int ctid = tid;                       // 0..319
  const int box = warp >> 1, mt = warp & 1;   // this warp: m-tile mt of box `box`
  const uint32_t ring_s = smem_u32(ring);
  bool aborted = false;
  uint32_t it = 0;
  for (long long g = rng.g0; g < rng.g1;) {
    const int unit = (int)(g / nk), kb0 = (int)(g % nk);
    const int ke = (int)min((long long)nk, kb0 + (rng.g1 - g));
    g += ke - kb0;
    const int4 ch = a.chunks[unit / NT];
    const int col0 = (unit % NT) * kMxTileCols;
    const int wg = min(kMxTileCols, a.I - col0);
    const int nrows = ch.z;
    float acc[2][2][4];  // [gate / up][nb][v]
#pragma unroll
    for (int m = 0; m < 2; ++m)
#pragma unroll
      for (int nb = 0; nb < 2; ++nb)
#pragma unroll
        for (int v = 0; v < 4; ++v) acc[m][nb][v] = 0.f;

    for (int kst = kb0; kst < ke; ++kst, ++it) {
      const int slot = it % kMxGUStages;
      const uint32_t ph = (it / kMxGUStages) & 1u;
      if (!aborted && !mbar_wait_bounded(&full[slot], ph, kWaitLimitNs)) {
        aborted = true;
        record_timeout(a.status);
      }
      if (!aborted) {
        const uint32_t st = ring_s + slot * kMxGUStage;
        const uint32_t boxes[2] = {st + box * kMxBoxBytes, st + (kMxBoxes + box) * kMxBoxBytes};
        const uint32_t scs[2] = {st + kMxGUW + box * kMxScaleBytes,
                                 st + kMxGUW + (kMxBoxes + box) * kMxScaleBytes};
        const uint32_t xb = st + kMxGUW + kMxGUS;
        const int nkb = mx_stage_blocks(a.H, kst * kMxKC);
        if (nrows <= 8)
          mx_stage<1, 2>(boxes, scs, xb, mt, nkb, lane, acc);
        else
          mx_stage<2, 2>(boxes, scs, xb, mt, nkb, lane, acc);
      }
      __syncwarp();
      if (lane == 0 && !aborted) mbar_arrive(&empty[slot]);
    }
    // every consumer warp walks the same units and takes the barriers below even after giving
    // up on a wait (skipping only the data work), so no warp is left at a barrier

    // ---- epilogue: as in stream_gate_up_kernel; value v of n-tile nb: column
    //      32*box + 16*mt + (lane>>2) + 8*(v>>1), row nb*8 + 2*(lane&3) + (v&1)
    if (kb0 == 0 && ke == nk) {  // this CTA holds the whole K range: SwiGLU from registers
#pragma unroll
      for (int nb = 0; nb < 2; ++nb)
#pragma unroll
        for (int v = 0; v < 4; ++v) {
          const int cl = kMxBoxRows * box + 16 * mt + (lane >> 2) + 8 * (v >> 1);
          const int r = nb * 8 + 2 * (lane & 3) + (v & 1);
          if (!aborted && r < nrows && cl < wg) {
            const float hv = silu_f32(acc[0][nb][v]) * acc[1][nb][v];
            a.h[(size_t)(ch.y + r) * a.I + col0 + cl] = (uint16_t)pack_f16x2(hv, 0.f);
          }
        }
      continue;
    }
#pragma unroll
    for (int nb = 0; nb < 2; ++nb)
#pragma unroll
      for (int v = 0; v < 4; ++v) {
        const int cl = kMxBoxRows * box + 16 * mt + (lane >> 2) + 8 * (v >> 1);
        const int r = nb * 8 + 2 * (lane & 3) + (v & 1);
        if (!aborted && r < nrows && cl < wg) {
          float* p = a.acc + ((size_t)ch.w + r) * I2 + col0 + cl;
          atomicAdd(p, acc[0][nb][v]);
          atomicAdd(p + a.I, acc[1][nb][v]);
        }
      }
    // Completion count in K stages: the piece that brings it to nk applies SwiGLU.  The
    // barrier orders every thread's atomics before thread 0's release; thread 0's acquire
    // and the second barrier order the last piece's reads after all other pieces' atomics.
    named_bar_sync(1, kMxConsumers);
    if (ctid == 0)
      s_last = !aborted && atom_add_acq_rel_gpu(&a.done[unit], ke - kb0) + (ke - kb0) == nk;
    named_bar_sync(1, kMxConsumers);
    if (s_last) {
      for (int i = ctid; i < nrows * (wg / 2); i += kMxConsumers) {
        const int r = i / (wg / 2), cl = 2 * (i - r * (wg / 2));
        const float* p = a.acc + ((size_t)ch.w + r) * I2 + col0 + cl;
        const float2 gs = __ldcg(reinterpret_cast<const float2*>(p));
        const float2 us = __ldcg(reinterpret_cast<const float2*>(p + a.I));
        *reinterpret_cast<uint32_t*>(a.h + (size_t)(ch.y + r) * a.I + col0 + cl) =
            pack_f16x2(silu_f32(gs.x) * us.x, silu_f32(gs.y) * us.y);
      }
    }
  }
}

// ------------------------------------------------------------------------------------------
// down projection + routing weight + combine, MXFP4 weights (h in f16).  Codes of W_down:
// [E * H rows, I/2 bytes]; scales: [E * I/32 rows, H bytes].
// ------------------------------------------------------------------------------------------
__global__ void __launch_bounds__(kMxDnThreads, 1)
    stream_down_mx_kernel(const DownArgs a, const __grid_constant__ CUtensorMap cmap,
                          const __grid_constant__ CUtensorMap smap) {
  extern __shared__ __align__(128) uint8_t smem_raw[];
  uint8_t* ring = align1k(smem_raw);
  uint64_t* full = reinterpret_cast<uint64_t*>(ring + kMxDNStages * kMxDNStage);
  uint64_t* empty = full + kMxDNStages;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) {
    for (int s = 0; s < kMxDNStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kMxDnWarps);
    }
    fence_barrier_init();
  }
  __syncthreads();

  if (tid == kMxDnConsumers) {
    tma_prefetch_desc(&cmap);
    tma_prefetch_desc(&smap);
  }
  pdl_wait();  // h and the work list come from the previous kernels
  pdl_launch_next();

  const int NT = (a.H + kMxDnTileCols - 1) / kMxDnTileCols;
  const int nk = (a.I + kMxKC - 1) / kMxKC;
  const StreamKRange rng = stream_k_range((long long)a.sched[0] * NT, nk);

  if (warp == kMxDnWarps) {
    bool aborted = false;
    uint32_t it = 0;
    int last_it[kMxDNStages];
#pragma unroll
    for (int s = 0; s < kMxDNStages; ++s) last_it[s] = -1;
    for (long long g = rng.g0; g < rng.g1;) {
      const int unit = (int)(g / nk), kb = (int)(g % nk);
      const int ke = (int)min((long long)nk, kb + (rng.g1 - g));
      g += ke - kb;
      const int4 ch = a.chunks[unit / NT];
      const int col0 = (unit % NT) * kMxDnTileCols;
      const int j = lane % kMxDnBoxes;
      const int box_col = col0 + kMxBoxRows * j;
      for (int kst = kb; kst < ke; ++kst, ++it) {
        const int slot = it % kMxDNStages;
        const uint32_t ph = (it / kMxDNStages) & 1u;
        if (!aborted && lane == 0 && !mbar_wait_bounded(&empty[slot], ph ^ 1u, kWaitLimitNs)) {
          aborted = true;
          record_timeout(a.status);
        }
        aborted = __shfl_sync(0xffffffffu, aborted, 0);
        if (aborted) continue;
        const int k0 = kst * kMxKC;
        const uint32_t xbytes = (uint32_t)min(kMxKC, a.I - k0) * 2u;
        if (lane == 0)
          mbar_arrive_expect_tx(&full[slot], (uint32_t)(kMxDNW + kMxDNS) + (uint32_t)ch.z * xbytes);
        __syncwarp();
        uint8_t* st = ring + slot * kMxDNStage;
        if (lane < kMxDnBoxes)
          tma_load_2d(st + lane * kMxBoxBytes, &cmap, k0 / 2, ch.x * a.H + box_col, &full[slot]);
        else if (lane < 2 * kMxDnBoxes)
          tma_load_2d(st + kMxDNW + j * kMxScaleBytes, &smap, box_col,
                      ch.x * (a.I / 32) + k0 / 32, &full[slot]);
        if (lane < ch.z)
          bulk_g2s(st + kMxDNW + kMxDNS + lane * kMxXPitch, a.h + (size_t)(ch.y + lane) * a.I + k0,
                   xbytes, &full[slot]);
        last_it[slot] = it;
      }
    }
    if (lane == 0) {
      for (int s = 0; s < kMxDNStages; ++s)
        if (last_it[s] >= 0 &&
            !mbar_wait_bounded(&full[s], (last_it[s] / kMxDNStages) & 1u, kWaitLimitNs))
          record_timeout(a.status);
    }
    return;
  }

  const int box = warp >> 1, mt = warp & 1;   // this warp: m-tile mt of box `box`
  const uint32_t ring_s = smem_u32(ring);
  bool aborted = false;
  uint32_t it = 0;
  for (long long g = rng.g0; g < rng.g1;) {
    const int unit = (int)(g / nk), kb0 = (int)(g % nk);
    const int ke = (int)min((long long)nk, kb0 + (rng.g1 - g));
    g += ke - kb0;
    const int4 ch = a.chunks[unit / NT];
    const int col0 = (unit % NT) * kMxDnTileCols;
    const int wc = min(kMxDnTileCols, a.H - col0);
    const int nrows = ch.z;
    float acc[1][2][4];
#pragma unroll
    for (int nb = 0; nb < 2; ++nb)
#pragma unroll
      for (int v = 0; v < 4; ++v) acc[0][nb][v] = 0.f;
    for (int kst = kb0; kst < ke; ++kst, ++it) {
      const int slot = it % kMxDNStages;
      const uint32_t ph = (it / kMxDNStages) & 1u;
      if (!aborted && !mbar_wait_bounded(&full[slot], ph, kWaitLimitNs)) {
        aborted = true;
        record_timeout(a.status);
      }
      if (!aborted) {
        const uint32_t st = ring_s + slot * kMxDNStage;
        const uint32_t boxes[1] = {st + box * kMxBoxBytes};
        const uint32_t scs[1] = {st + kMxDNW + box * kMxScaleBytes};
        const uint32_t xb = st + kMxDNW + kMxDNS;
        const int nkb = mx_stage_blocks(a.I, kst * kMxKC);
        if (nrows <= 8)
          mx_stage<1, 1>(boxes, scs, xb, mt, nkb, lane, acc);
        else
          mx_stage<2, 1>(boxes, scs, xb, mt, nkb, lane, acc);
      }
      __syncwarp();
      if (lane == 0 && !aborted) mbar_arrive(&empty[slot]);
    }
    if (aborted) continue;
    // ---- epilogue: as in stream_down_kernel ----
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
    for (int nb = 0; nb < 2; ++nb)
#pragma unroll
      for (int v = 0; v < 4; ++v) {
        const int cl = kMxBoxRows * box + 16 * mt + (lane >> 2) + 8 * (v >> 1);
        const int t = tok[nb][v & 1];
        if (t >= 0 && cl < wc)
          atomicAdd(a.out + (size_t)t * a.H + col0 + cl, wt[nb][v & 1] * acc[0][nb][v]);
      }
  }
}

}  // namespace moe
