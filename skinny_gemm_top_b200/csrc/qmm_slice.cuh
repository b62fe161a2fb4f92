// Decode MoE layer in one launch, split along the expert intermediate
// dimension (the decode hot path: T <= 8 tokens).
//
// What it computes (onnxruntime PR "Enable SM80+ FP16/BF16 mixed INT2/INT4
// QMoE prefill by default", Description): top-k routing, FC1 with expert bias
// and interleaved SwiGLU, FC2, the top-k weighted finalize with FC2 bias; the
// shared experts of the layer get every token with weight 1.
//
// Work split (B200 design): every active expert's intermediate dimension I is
// cut into granules of kCols columns of h (16 for an INT4 FC2, 32 INT2: the K
// width of one slab of the QMOE_ROWS_KSPLIT FC2 layout; 64 ternary, half of
// one 128-column record).  Each
// CTA gets a contiguous range of granules: with at least two CTAs per active
// expert, every expert (shared ones first, then the selected ones in expert
// order) gets its own group of CTAs, so a CTA's range lies inside one expert;
// otherwise (or when that would leave the busiest CTA with much more than an
// even share) the experts' granule list is split evenly.  For its range a CTA
// streams
//   FC1: the gate/up rows of its granules (8 j per 16-row tile, all H columns),
//        and turns them into w_t * SwiGLU(gate, up) for every token t, as bf16
//        in shared memory (w_t = router weight of token t for that expert, 0
//        when the token did not pick it, 1 for a shared expert);
//   FC2: the matching columns of the down matrix, for all H rows,
// so one pass over each weight byte serves all tokens (the remedy of the QMoE
// note), no CTA waits for another, and FC2's weights stream in while FC1 is
// still computing.  Each CTA adds its [T][H] partial output to an fp32
// accumulator with vector atomics; the last CTA (ticket) rounds it to bf16.
//
// Inside a CTA the range's FC1 tiles form chunks of up to 10 tiles of one
// expert (8 for INT2 or ternary FC2: whole granules).  Each of the 12 warps streams, through
// its own ring of item buffers, the chunk's k-units w, w+12, ... (all the
// chunk's tiles: one contiguous run of codes, one TMA bulk copy) and then,
// after a cross-warp reduction (fixed warp order) has produced the chunk's h,
// the FC2 granules the chunk completed, restricted to its own 16-row tiles of
// the output (cp.async), whose partial sums stay in registers for the whole
// launch.  With a single token, the CTAs of the shared experts know their
// work before the routing and request their first items before
// griddepcontrol.wait: they depend on nothing the previous launch writes.
//
// Codes become bf16 MMA operands with the LOP3 magic-number unpack
// (unpack.cuh) and are multiplied on the tensor cores (mma.sync m16n8k16,
// tokens in N); the per-block scale multiplies the fp32 partial product of
// its block, so c * s is never rounded.
#pragma once
#include <climits>

#include "device_common.cuh"
#include "qmm_small.cuh"
#include "slice.h"
#include "unpack.cuh"

namespace qmoe {

constexpr int kSThreads = kSW * 32;

// FC2 granule of the K-split layout: kCols columns of h; kRowBytes code bytes
// loaded per 16-row tile.  A ternary granule is half of a 128-column record:
// its CTA loads the whole record and uses its own four k-steps (the record's
// other half, read by the neighbouring granule's CTA at about the same time,
// is mostly served by L2), so that twice as many CTAs share a ternary layer.
template <int F> struct KsTr;
template <> struct KsTr<4> { static constexpr int kCols = 16, kRowBytes = 128, kKsteps = 1, kBlocks = 1, kPerRec = 1; };
template <> struct KsTr<2> { static constexpr int kCols = 32, kRowBytes = 128, kKsteps = 2, kBlocks = 1, kPerRec = 1; };
template <> struct KsTr<3> { static constexpr int kCols = 64, kRowBytes = 416, kKsteps = 4, kBlocks = 1, kPerRec = 2; };

// FC1 tiles per chunk at most: whole granules up to 10 tiles; a ternary
// granule (16 tiles) is two chunks of 8.
template <int F2>
struct SChunkGeom {
  static constexpr int TPG = KsTr<F2>::kCols / 8;  // FC1 tiles per granule
  static constexpr int kMT = TPG <= kSChunk ? (kSChunk / TPG) * TPG : 8;
};

constexpr int round128c(int v) { return (v + 127) / 128 * 128; }

// Shared-memory layout (byte offsets; x rows and the rings follow at kFixed).
struct SliceSmemLayout {
  static constexpr int kBars = 0;                                       // [kSW][kSNB] u64
  static constexpr int kXBar = kBars + kSW * kSNB * 8;                  // x bulk-copy barrier
  static constexpr int kDBar = kXBar + 8;                               // barrier nothing arrives at (fault injection)
  static constexpr int kMisc = kXBar + 16;                              // 16 ints
  static constexpr int kVst = kMisc + 64;                               // [kSW][kSNB] int: item virtual offsets
  static constexpr int kPst = kVst + kSW * kSNB * 4;                    // [kSW][kSNB] int: item ring offsets
  static constexpr int kRoute = round128c(kPst + kSW * kSNB * 4);       // DecodeRoute
  static constexpr int kWmat = kRoute + round128c((int)sizeof(DecodeRoute));  // [kDecMaxTK][8] f32
  static constexpr int kChunks = kWmat + kDecMaxTK * 8 * 4;            // [kSMaxChunks] SChunk
  static constexpr int kLut = kChunks + kSMaxChunks * (int)sizeof(SChunk);  // 243 u32 (ternary)
  static constexpr int kCorr = kLut + 1024;                             // [kSMaxH / 64][8] f32
  static constexpr int kSx = kCorr + round128c((kSMaxH / 64) * 8 * 4);  // [kSMaxH / 64][8] f32 (affine codes)
  static constexpr int kH = kSx + round128c((kSMaxH / 64) * 8 * 4);     // [kSHWin][32] uint2
  static constexpr int kRed = kH + kSHWin * 32 * 8;                     // [kSW][kSRed][32] float4
  static constexpr int kFixed = kRed + kSW * kSRed * 32 * 16;           // x rows start here
};

// misc[] slots
constexpr int kMiscChunks = 0, kMiscLast = 1, kMiscAbort = 2, kMiscEarly = 3;

__device__ __forceinline__ void red_add_v4_f32(float* addr, float4 v) {
  asm volatile("red.relaxed.gpu.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(addr), "f"(v.x), "f"(v.y),
               "f"(v.z), "f"(v.w)
               : "memory");
}

__device__ __forceinline__ float4 ld_relaxed_v4(const float* addr) {
  float4 v;
  asm volatile("ld.relaxed.gpu.global.v4.f32 {%0, %1, %2, %3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "l"(addr)
               : "memory");
  return v;
}

// Chunks of granules [ga, gb) of one expert appended to the table.
template <int F2>
__device__ void slice_add_piece(SChunk* tab, int* n, int expert, int wsel, int ga, int gb, unsigned* status) {
  using CG = SChunkGeom<F2>;
  constexpr int TPG = CG::TPG;
  auto push = [&](int etile0, int nt, int g0, int ngc, int hoff) {
    if (*n >= kSMaxChunks) {
      atomicOr(status, kStatusBadSegment);
      return;
    }
    SChunk C;
    C.expert = expert;
    C.wsel = wsel;
    C.etile0 = etile0;
    C.nt = nt;
    C.g0 = g0;
    C.ngc = ngc;
    C.hoff = hoff;
    C.pad = 0;
    tab[(*n)++] = C;
  };
  static_assert(TPG <= kSChunk, "a granule fits in one chunk");
  constexpr int gmax = CG::kMT / TPG;
  const int ng = gb - ga, nch = (ng + gmax - 1) / gmax;
  for (int i = 0; i < nch; ++i) {  // near-equal granule counts
    const int g0 = ga + ng * i / nch, g1 = ga + ng * (i + 1) / nch;
    push(g0 * TPG, (g1 - g0) * TPG, g0, g1 - g0, 0);
  }
}

// Router weight of token n for the chunk's expert (0 past the batch).
__device__ __forceinline__ float slice_weight(const SChunk& C, const float* wmat, int n, int T) {
  if (n >= T) return 0.f;
  return C.wsel < 0 ? 1.f : wmat[C.wsel * 8 + n];
}

// A warp's position in its item sequence: per chunk the k-units warp,
// warp + 12, ... of FC1, then (with output rows) the chunk's completed
// granules in groups of ngm.
struct SIt {
  int c, kind, a;
};

__device__ __forceinline__ bool slice_fix(SIt& it, const SChunk* tab, int nch, int KU1, bool rows, int warp) {
  for (;;) {
    if (it.c >= nch) return false;
    if (it.kind == 0) {
      if (it.a < KU1) return true;
      it.kind = 1;
      it.a = 0;
    }
    if (rows && it.a < tab[it.c].ngc) return true;
    ++it.c;
    it.kind = 0;
    it.a = warp;
  }
}

// FC1 item: the chunk's nt tiles at k-unit ku (codes then scales in the
// buffer), accumulated into acc1.  B fragments come from the x rows in shared
// memory (columns k % 16 >= 8 already divided by the code multiplier); the
// constant-operand correction of each 64-column block is the precomputed
// corr1.  Tiles go four at a time so that their MMA chains overlap.  Affine
// codes (aff): the zero points follow the scales in the buffer, and each
// block adds z * (sum of its activations), sx1.
template <int F1, int MT>
__device__ __forceinline__ void slice_fc1(const uint8_t* st, int nt, int ku, const uint8_t* xrow, const float* corr1,
                                          const float* sx1, bool aff, const uint32_t* lut, int lane,
                                          float (&acc1)[MT][4]) {
  using T1 = FmtTraits<F1>;
  constexpr int BPK = T1::kKUcols / 64;
  const int g = lane >> 2, n0 = 2 * (lane & 3);
  const uint8_t* scales = st + nt * T1::kCodeBytes;  // [BPK][nt][32 B]
  uint32_t bfr[BPK][4][2];
  float cr[BPK][2];
#pragma unroll
  for (int bl = 0; bl < BPK; ++bl) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      uint32_t r[4];
      ldmatrix_x4(r, xrow + (ku * T1::kKUcols + bl * 64 + h * 32 + (lane >> 3) * 8) * 2);
      bfr[bl][2 * h][0] = r[0];
      bfr[bl][2 * h][1] = r[1];
      bfr[bl][2 * h + 1][0] = r[2];
      bfr[bl][2 * h + 1][1] = r[3];
    }
    cr[bl][0] = corr1[(ku * BPK + bl) * 8 + n0];
    cr[bl][1] = corr1[(ku * BPK + bl) * 8 + n0 + 1];
  }
  if constexpr (F1 == 3) {
#pragma unroll
    for (int i = 0; i < MT; ++i) {
      if (i >= nt) break;
      uint32_t am[8][4];
      unpack_tern_record(st + i * T1::kCodeBytes + lane * 13, lut, am);
#pragma unroll
      for (int bl = 0; bl < 2; ++bl) {
        float tmp[4] = {cr[bl][0], cr[bl][1], cr[bl][0], cr[bl][1]};
#pragma unroll
        for (int k2 = 0; k2 < 4; ++k2) mma_bf16_16816(tmp, am[bl * 4 + k2], bfr[bl][k2][0], bfr[bl][k2][1]);
        const uint32_t sc = *reinterpret_cast<const uint32_t*>(scales + (bl * nt + i) * 32 + g * 4);
        const float slo = bf16_lo(sc), shi = bf16_hi(sc);
        acc1[i][0] = fmaf(slo, tmp[0], acc1[i][0]);
        acc1[i][1] = fmaf(slo, tmp[1], acc1[i][1]);
        acc1[i][2] = fmaf(shi, tmp[2], acc1[i][2]);
        acc1[i][3] = fmaf(shi, tmp[3], acc1[i][3]);
      }
    }
  } else {
#pragma unroll
    for (int i0 = 0; i0 < MT; i0 += 4) {
      if (i0 >= nt) break;
      float tmp[4][4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        tmp[i][0] = cr[0][0];
        tmp[i][1] = cr[0][1];
        tmp[i][2] = cr[0][0];
        tmp[i][3] = cr[0][1];
      }
      if constexpr (F1 == 2) {
        uint2 wd[4];
#pragma unroll
        for (int i = 0; i < 4; ++i)
          wd[i] = i0 + i < nt ? *reinterpret_cast<const uint2*>(st + (i0 + i) * 256 + lane * 8) : make_uint2(0u, 0u);
#pragma unroll
        for (int w = 0; w < 2; ++w)
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            if (i0 + i >= MT) break;
            uint32_t a0[4], a1[4];
            unpack_int2_word(w ? wd[i].y : wd[i].x, a0, a1);
            mma_bf16_16816(tmp[i], a0, bfr[0][2 * w][0], bfr[0][2 * w][1]);
            mma_bf16_16816(tmp[i], a1, bfr[0][2 * w + 1][0], bfr[0][2 * w + 1][1]);
          }
      } else {
        uint4 wd[4];
#pragma unroll
        for (int i = 0; i < 4; ++i)
          wd[i] = i0 + i < nt ? *reinterpret_cast<const uint4*>(st + (i0 + i) * 512 + lane * 16)
                              : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
        for (int w = 0; w < 4; ++w)
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            if (i0 + i >= MT) break;
            uint32_t a[4];
            unpack_int4_word(w == 0 ? wd[i].x : w == 1 ? wd[i].y : w == 2 ? wd[i].z : wd[i].w, a);
            mma_bf16_16816(tmp[i], a, bfr[0][w][0], bfr[0][w][1]);
          }
      }
      if (aff) {  // z * (sum of the block's activations), per row and token
        const float sxa = sx1[ku * 8 + n0], sxb = sx1[ku * 8 + n0 + 1];
        const uint8_t* zeros = scales + nt * 32;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          if (i0 + i >= MT || i0 + i >= nt) break;
          const uint32_t zc = *reinterpret_cast<const uint32_t*>(zeros + (i0 + i) * 32 + g * 4);
          const float zlo = bf16_lo(zc), zhi = bf16_hi(zc);
          acc1[i0 + i][0] = fmaf(zlo, sxa, acc1[i0 + i][0]);
          acc1[i0 + i][1] = fmaf(zlo, sxb, acc1[i0 + i][1]);
          acc1[i0 + i][2] = fmaf(zhi, sxa, acc1[i0 + i][2]);
          acc1[i0 + i][3] = fmaf(zhi, sxb, acc1[i0 + i][3]);
        }
      }
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        if (i0 + i >= MT || i0 + i >= nt) break;
        const uint32_t sc = *reinterpret_cast<const uint32_t*>(scales + (i0 + i) * 32 + g * 4);
        const float slo = bf16_lo(sc), shi = bf16_hi(sc);
        acc1[i0 + i][0] = fmaf(slo, tmp[i][0], acc1[i0 + i][0]);
        acc1[i0 + i][1] = fmaf(slo, tmp[i][1], acc1[i0 + i][1]);
        acc1[i0 + i][2] = fmaf(shi, tmp[i][2], acc1[i0 + i][2]);
        acc1[i0 + i][3] = fmaf(shi, tmp[i][3], acc1[i0 + i][3]);
      }
    }
  }
}

// FC2 item: ng granules of this warp's nr row tiles, accumulated into acc2.
// B fragments are the h window's k-steps from window granule wg0 on.
template <int F2>
__device__ __forceinline__ void slice_fc2(const uint8_t* st, int ng, int nr, int wg0, int g_abs, bool aff,
                                          const uint2* hfrag, const uint32_t* lut, int lane,
                                          float (&acc2)[kSRT][4]) {
  using K2 = KsTr<F2>;
  using Tr2 = FmtTraits<F2>;
  const int g = lane >> 2;
  const uint32_t aconst[4] = {aff ? kAffConst : Tr2::kConstLo, aff ? kAffConst : Tr2::kConstLo,
                              aff ? kAffConst : Tr2::kConstHi, aff ? kAffConst : Tr2::kConstHi};
  const uint32_t* sbuf = reinterpret_cast<const uint32_t*>(st + ng * nr * K2::kRowBytes);
  // affine codes: zero points after the scales
  const uint32_t* zbuf = sbuf + ng * K2::kBlocks * nr * 8;
  for (int gi = 0; gi < ng; ++gi) {
    uint2 b[K2::kKsteps];
#pragma unroll
    for (int s = 0; s < K2::kKsteps; ++s) b[s] = hfrag[((wg0 + gi) * K2::kKsteps + s) * 32 + lane];
    float cr[K2::kBlocks][4];
#pragma unroll
    for (int bl = 0; bl < K2::kBlocks; ++bl) {
      cr[bl][0] = cr[bl][1] = cr[bl][2] = cr[bl][3] = 0.f;
#pragma unroll
      for (int s = 0; s < K2::kKsteps / K2::kBlocks; ++s) {
        const uint2 bb = b[bl * (K2::kKsteps / K2::kBlocks) + s];
        mma_bf16_16816(cr[bl], aconst, bb.x, bb.y);
      }
    }
    float sx[4] = {0.f, 0.f, 0.f, 0.f};  // affine: the granule's sum of h per token
    if constexpr (F2 != 3) {
      if (aff) {
        const uint32_t asum[4] = {kBf16One, kBf16One, sum_const_hi<F2>(), sum_const_hi<F2>()};
#pragma unroll
        for (int s = 0; s < K2::kKsteps; ++s) mma_bf16_16816(sx, asum, b[s].x, b[s].y);
      }
    }
    const uint8_t* cbase = st + gi * nr * K2::kRowBytes;
#pragma unroll
    for (int i = 0; i < kSRT; ++i) {
      if (i >= nr) break;
      if constexpr (F2 == 3) {
        // this granule's half of the record (the other half's unpack is dead code)
        uint32_t am[8][4];
        unpack_tern_record(cbase + i * 416 + lane * 13, lut, am);
        float tmp[4] = {cr[0][0], cr[0][1], cr[0][2], cr[0][3]};
        if ((g_abs + gi) & 1) {
#pragma unroll
          for (int s = 0; s < 4; ++s) mma_bf16_16816(tmp, am[4 + s], b[s].x, b[s].y);
        } else {
#pragma unroll
          for (int s = 0; s < 4; ++s) mma_bf16_16816(tmp, am[s], b[s].x, b[s].y);
        }
        const uint32_t sc = sbuf[(gi * nr + i) * 8 + g];
        const float slo = bf16_lo(sc), shi = bf16_hi(sc);
        acc2[i][0] = fmaf(slo, tmp[0], acc2[i][0]);
        acc2[i][1] = fmaf(slo, tmp[1], acc2[i][1]);
        acc2[i][2] = fmaf(shi, tmp[2], acc2[i][2]);
        acc2[i][3] = fmaf(shi, tmp[3], acc2[i][3]);
      } else {
        const uint32_t w = *reinterpret_cast<const uint32_t*>(cbase + i * 128 + lane * 4);
        float tmp[4] = {cr[0][0], cr[0][1], cr[0][2], cr[0][3]};
        if constexpr (F2 == 2) {
          uint32_t a0[4], a1[4];
          unpack_int2_word(w, a0, a1);
          mma_bf16_16816(tmp, a0, b[0].x, b[0].y);
          mma_bf16_16816(tmp, a1, b[1].x, b[1].y);
        } else {
          uint32_t a[4];
          unpack_int4_word(w, a);
          mma_bf16_16816(tmp, a, b[0].x, b[0].y);
        }
        if (aff) {
          const uint32_t zc = zbuf[(gi * nr + i) * 8 + g];
          const float zlo = bf16_lo(zc), zhi = bf16_hi(zc);
          acc2[i][0] = fmaf(zlo, sx[0], acc2[i][0]);
          acc2[i][1] = fmaf(zlo, sx[1], acc2[i][1]);
          acc2[i][2] = fmaf(zhi, sx[2], acc2[i][2]);
          acc2[i][3] = fmaf(zhi, sx[3], acc2[i][3]);
        }
        const uint32_t sc = sbuf[(gi * nr + i) * 8 + g];
        const float slo = bf16_lo(sc), shi = bf16_hi(sc);
        acc2[i][0] = fmaf(slo, tmp[0], acc2[i][0]);
        acc2[i][1] = fmaf(slo, tmp[1], acc2[i][1]);
        acc2[i][2] = fmaf(shi, tmp[2], acc2[i][2]);
        acc2[i][3] = fmaf(shi, tmp[3], acc2[i][3]);
      }
    }
  }
}

// This CTA's chunk table: its range of the experts' granule list.  Experts
// in list order: shared (slot j < n_shared: expert E + j) then the selected
// ones (expert of_sel(r)).  When slice_grouped holds, slot s gets a group of
// CTAs (sizes differing by at most one) and CTA j of a group of n takes
// granules [gpe*j/n, gpe*(j+1)/n); otherwise the list is split evenly.
template <int F2, class OfSel>
__device__ void slice_partition(SChunk* tab, int* n, int c, int G, int nslots, int ns, int E, int gpe, OfSel of_sel,
                                unsigned* status) {
  auto expert_of = [&](int s) { return s < ns ? E + s : of_sel(s - ns); };
  if (slice_grouped(G, nslots, gpe)) {
    const int cps = G / nslots, rem = G % nslots, big = rem * (cps + 1);
    int s, j, m;
    if (c < big) {
      s = c / (cps + 1);
      j = c - s * (cps + 1);
      m = cps + 1;
    } else {
      s = rem + (c - big) / cps;
      j = (c - big) - (s - rem) * cps;
      m = cps;
    }
    slice_add_piece<F2>(tab, n, expert_of(s), s < ns ? -1 : s - ns, gpe * j / m, gpe * (j + 1) / m, status);
    return;
  }
  const long long N = (long long)nslots * gpe;
  const int u0 = (int)(N * c / G), u1 = (int)(N * (c + 1) / G);
  for (int u = u0; u < u1;) {
    const int s = u / gpe, g = u - s * gpe, g1 = min(gpe, g + (u1 - u));
    slice_add_piece<F2>(tab, n, expert_of(s), s < ns ? -1 : s - ns, g, g1, status);
    u += g1 - g;
  }
}

template <int F1, int F2, bool AFF>
__global__ void __launch_bounds__(kSThreads, 1) qmm_slice_kernel(const SliceParams p) {
  using T1 = FmtTraits<F1>;
  using K2 = KsTr<F2>;
  using Tr2 = FmtTraits<F2>;
  using L = SliceSmemLayout;
  constexpr int MT = SChunkGeom<F2>::kMT;
  constexpr int BPK = T1::kKUcols / 64;
  extern __shared__ __align__(128) uint8_t smem[];
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBars);
  uint64_t* xbar = reinterpret_cast<uint64_t*>(smem + L::kXBar);
  uint64_t* dbar = reinterpret_cast<uint64_t*>(smem + L::kDBar);
  int* misc = reinterpret_cast<int*>(smem + L::kMisc);
  DecodeRoute& R = *reinterpret_cast<DecodeRoute*>(smem + L::kRoute);
  float* wmat = reinterpret_cast<float*>(smem + L::kWmat);
  SChunk* tab = reinterpret_cast<SChunk*>(smem + L::kChunks);
  uint32_t* lut = reinterpret_cast<uint32_t*>(smem + L::kLut);
  float* corr1 = reinterpret_cast<float*>(smem + L::kCorr);
  float* sx1 = reinterpret_cast<float*>(smem + L::kSx);
  constexpr bool aff = AFF;  // affine codes (zero points): a separate instantiation
  uint2* hfrag = reinterpret_cast<uint2*>(smem + L::kH);
  uint16_t* hbits = reinterpret_cast<uint16_t*>(smem + L::kH);
  float4* red = reinterpret_cast<float4*>(smem + L::kRed);
  const int xpitch = p.H * 2 + 16;  // padded rows: conflict-free ldmatrix
  uint8_t* xs = smem + L::kFixed;
  uint8_t* rings = xs + ((p.xrows * xpitch + 127) / 128) * 128;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int G = gridDim.x, c = blockIdx.x;
  const int T = p.T, RB = p.ring_bytes;
  uint64_t* wbar = bars + warp * kSNB;
  int* vst = reinterpret_cast<int*>(smem + L::kVst) + warp * kSNB;
  int* pst = reinterpret_cast<int*>(smem + L::kPst) + warp * kSNB;
  uint8_t* ring = rings + (size_t)warp * RB;
  // this warp's FC2 output rows: 16-row tiles [r0, r0 + nr)
  const int r0 = warp * p.NT2 / kSW, nr = (warp + 1) * p.NT2 / kSW - r0;

  if (lane == 0)
    for (int s = 0; s < kSNB; ++s) mbar_init(&wbar[s], 33);  // lane 0's arrival + 32 cp.async arrivals
  if (tid == 0) {
    mbar_init(xbar, 1);
    mbar_init(dbar, 1);
    misc[kMiscAbort] = 0;
    misc[kMiscChunks] = 0;
    misc[kMiscEarly] = 0;
    // One token: k experts are selected, so the CTA groups are known now; a
    // CTA of a shared expert knows its whole chunk table before the routing.
    const int nslots = p.n_shared + p.k;
    if (T == 1 && slice_grouped(G, nslots, p.gpe)) {
      const int cps = G / nslots, rem = G % nslots, big = rem * (cps + 1);
      const int s = c < big ? c / (cps + 1) : rem + (c - big) / cps;
      if (s < p.n_shared) {
        int n = 0;
        slice_partition<F2>(tab, &n, c, G, nslots, p.n_shared, p.E, p.gpe, [](int) { return 0; }, p.status);
        misc[kMiscChunks] = n;
        misc[kMiscEarly] = 1;
      }
    }
  }
  if constexpr (F1 == 3 || F2 == 3)
    for (int i = tid; i < 243; i += kSThreads) lut[i] = tern_lut_entry(i);
  fence_mbar_init();
  __syncthreads();

  // ---- the warp's ring: items in order, any size, one barrier each ----
  int nch = misc[kMiscChunks];
  SIt prod{0, 0, warp};
  bool pv = slice_fix(prod, tab, nch, p.KU1, nr > 0, warp);
  // head / hp: virtual and physical ring offset of the next item; islot / cslot: issued / consumed item % kSNB
  int issued = 0, cons = 0, head = 0, hp = 0, islot = 0, cslot = 0;
  bool ok = true;
  auto refill = [&]() {
    while (ok && pv && issued < cons + kSNB) {
      __syncwarp();
      const SChunk& C = tab[prod.c];
      const int ngi = min(p.ngm, C.ngc - prod.a);
      constexpr int zb = aff ? 1 : 0;  // affine codes: zero points after the scales
      const int bytes = prod.kind == 0 ? C.nt * (T1::kCodeBytes + (1 + zb) * BPK * 32)
                                       : ngi * nr * (K2::kRowBytes + (1 + zb) * K2::kBlocks * 32);
      int v = head, ph = hp;
      if (ph + bytes > RB) {  // items never wrap around the ring's end
        v += RB - ph;
        ph = 0;
      }
      const int tail = issued > cons ? vst[cslot] : v;
      if (v + bytes > tail + RB) break;  // the oldest items still hold the space
      if (lane == 0) {
        vst[islot] = v;
        pst[islot] = ph;
      }
      uint8_t* st = ring + ph;
      uint64_t* bar = &wbar[islot];
      if (prod.kind == 0) {  // FC1: the chunk's tiles at k-unit a (one contiguous run), and their scales
        const int ku = prod.a;
        if (lane == 0) {
          mbar_arrive_expect_tx(bar, (uint32_t)(C.nt * T1::kCodeBytes));
          bulk_copy_g2s(st,
                        p.c1 + (unsigned long long)C.expert * p.c1_stride +
                            ((unsigned long long)ku * p.NT1 + C.etile0) * T1::kCodeBytes,
                        (uint32_t)(C.nt * T1::kCodeBytes), bar);
        }
#pragma unroll
        for (int bl = 0; bl < BPK; ++bl) {
          const int sb = (ku * T1::kKUcols + bl * 64) >> (p.block1 == 128 ? 7 : 6);
          const uint8_t* ss =
              p.s1 + (unsigned long long)C.expert * p.s1_stride + ((unsigned long long)sb * p.NT1 + C.etile0) * 32;
          if (lane < 2 * C.nt) cp_async16(st + C.nt * T1::kCodeBytes + bl * C.nt * 32 + 16 * lane, ss + 16 * lane);
          if (zb && lane < 2 * C.nt)
            cp_async16(st + C.nt * T1::kCodeBytes + (BPK + bl) * C.nt * 32 + 16 * lane,
                       p.z1 + (ss - p.s1) + 16 * lane);
        }
      } else {  // FC2: granules [a, a + ngi) of the chunk, this warp's rows of each slab, and their scales
        if (lane == 0) mbar_arrive(bar);
        const int per = nr * (K2::kRowBytes / 16);
        for (int gi = 0; gi < ngi; ++gi) {
          const int slab = C.g0 + prod.a + gi;  // granule of the expert = K-split slab (ternary: half a record)
          const uint8_t* src = p.c2 + (unsigned long long)C.expert * p.c2_stride +
                               ((unsigned long long)(slab / K2::kPerRec) * p.NT2 + r0) * K2::kRowBytes;
          uint8_t* dst = st + gi * nr * K2::kRowBytes;
          for (int i = lane; i < per; i += 32) cp_async16(dst + 16 * i, src + 16 * i);
#pragma unroll
          for (int bl = 0; bl < K2::kBlocks; ++bl) {
            const int sb = (slab * K2::kCols + bl * 64) >> (p.block2 == 128 ? 7 : 6);
            const uint8_t* ss =
                p.s2 + (unsigned long long)C.expert * p.s2_stride + ((unsigned long long)sb * p.NT2 + r0) * 32;
            if (lane < 2 * nr) cp_async16(st + ngi * nr * K2::kRowBytes + (gi * K2::kBlocks + bl) * nr * 32 + 16 * lane,
                                          ss + 16 * lane);
            if (zb && lane < 2 * nr)
              cp_async16(st + ngi * nr * K2::kRowBytes + ((ngi + gi) * K2::kBlocks + bl) * nr * 32 + 16 * lane,
                         p.z2 + (ss - p.s2) + 16 * lane);
          }
        }
      }
      cp_async_arrive(bar);
      head = v + bytes;
      hp = ph + bytes;
      islot = islot == kSNB - 1 ? 0 : islot + 1;
      ++issued;
      prod.a += prod.kind == 0 ? kSW : p.ngm;
      pv = slice_fix(prod, tab, nch, p.KU1, nr > 0, warp);
    }
    __syncwarp();
  };
  refill();  // a shared expert's CTA with one token: its first items, before the dependency wait

  // ---- after the previous launches: x rows, routing ----
  pdl_wait();
  if (warp == kSW - 1) {  // the first T warps route
    if (lane == 0) mbar_arrive_expect_tx(xbar, (uint32_t)(T * p.H * 2));
    __syncwarp();
    if (lane < T) bulk_copy_g2s(xs + lane * xpitch, p.x + (size_t)lane * p.H, (uint32_t)(p.H * 2), xbar);
  }
  for (int i = tid; i < (p.xrows - T) * xpitch / 4; i += kSThreads)  // zero row for tokens >= T
    reinterpret_cast<uint32_t*>(xs + T * xpitch)[i] = 0u;
  for (int i = tid; i < kDecMaxTK * 8; i += kSThreads) wmat[i] = 0.f;
  decode_route(p.logits, T, p.E, p.k, R);  // ends with a CTA barrier
  pdl_trigger();
  const int nsel = R.nseg;
  for (int i = tid; i < T * p.k; i += kSThreads) {  // weight of (token, selected expert)
    const int e = R.ids[i];
    int r = 0;
    while (r < nsel - 1 && R.segs[r].expert != e) ++r;
    wmat[r * 8 + i / p.k] = R.w[i];
  }
  if (tid == 0 && !misc[kMiscEarly]) {
    int n = 0;
    slice_partition<F2>(tab, &n, c, G, p.n_shared + nsel, p.n_shared, p.E, p.gpe,
                        [&](int r) { return R.segs[r].expert; }, p.status);
    misc[kMiscChunks] = n;
  }
  __syncthreads();
  nch = misc[kMiscChunks];
  pv = slice_fix(prod, tab, nch, p.KU1, nr > 0, warp);
  refill();

  // x landed (bounded wait), then the hi columns divided by the code multiplier
  if (!mbar_wait_sleep_bounded(xbar, 0, p.status, p.wait_ns)) misc[kMiscAbort] = 1;
  if (p.inject == 1 && tid == 0 && !mbar_wait_sleep_bounded(dbar, 0, p.status, p.wait_ns)) misc[kMiscAbort] = 1;
  __syncthreads();
  if constexpr (T1::kBetaHi == 4) {
    for (int i = tid; i < T * p.H / 16; i += kSThreads) {  // one 8-column high half per item
      const int n = i / (p.H / 16), k16 = i - n * (p.H / 16);
      uint4* q = reinterpret_cast<uint4*>(xs + n * xpitch + (k16 * 16 + 8) * 2);
      uint4 v = *q;
      v.x = fma_bf16x2(v.x, kBf16Quarter, kBf16NegZero);
      v.y = fma_bf16x2(v.y, kBf16Quarter, kBf16NegZero);
      v.z = fma_bf16x2(v.z, kBf16Quarter, kBf16NegZero);
      v.w = fma_bf16x2(v.w, kBf16Quarter, kBf16NegZero);
      *q = v;
    }
    __syncthreads();
  }
  // per-lane x row for ldmatrix: token lane & 7, or the zero row past the batch
  const uint8_t* xrow = xs + min(lane & 7, p.xrows - 1) * xpitch;
  // constant-operand correction of FC1 per 64-column block and token (and,
  // for affine codes, the block's sum of the activations)
  {
    const uint32_t aconst[4] = {aff ? kAffConst : T1::kConstLo, aff ? kAffConst : T1::kConstLo,
                                aff ? kAffConst : T1::kConstHi, aff ? kAffConst : T1::kConstHi};
    const uint32_t asum[4] = {kBf16One, kBf16One, sum_const_hi<F1>(), sum_const_hi<F1>()};
    for (int b = warp; b < p.H / 64; b += kSW) {
      float cr[4] = {0.f, 0.f, 0.f, 0.f}, sx[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        uint32_t r[4];
        ldmatrix_x4(r, xrow + (b * 64 + h * 32 + (lane >> 3) * 8) * 2);
        mma_bf16_16816(cr, aconst, r[0], r[1]);
        mma_bf16_16816(cr, aconst, r[2], r[3]);
        if (aff) {
          mma_bf16_16816(sx, asum, r[0], r[1]);
          mma_bf16_16816(sx, asum, r[2], r[3]);
        }
      }
      if (lane < 4) {
        corr1[b * 8 + 2 * lane] = cr[0];
        corr1[b * 8 + 2 * lane + 1] = cr[1];
        if (aff) {
          sx1[b * 8 + 2 * lane] = sx[0];
          sx1[b * 8 + 2 * lane + 1] = sx[1];
        }
      }
    }
  }
  __syncthreads();

  // ---- stream ----
  float acc2[kSRT][4];
#pragma unroll
  for (int i = 0; i < kSRT; ++i) acc2[i][0] = acc2[i][1] = acc2[i][2] = acc2[i][3] = 0.f;
  ok = misc[kMiscAbort] == 0;
  uint32_t cpar = 0;  // phase parity of the consumed slot
  int drain = ok ? INT_MAX : 0;  // first item that may still be in flight after a wait gave up
  auto wait_item = [&]() -> const uint8_t* {
    if (ok && __any_sync(0xffffffffu, !mbar_wait_sleep_bounded(&wbar[cslot], cpar, p.status, p.wait_ns))) {
      ok = false;
      drain = cons;
      misc[kMiscAbort] = 1;
    }
    return ring + pst[cslot];
  };
  auto next_item = [&]() {
    __syncwarp();
    ++cons;
    if (++cslot == kSNB) {
      cslot = 0;
      cpar ^= 1u;
    }
    refill();
  };
  for (int ci = 0; ci < nch; ++ci) {
    const SChunk C = tab[ci];
    float acc1[MT][4];
#pragma unroll
    for (int i = 0; i < MT; ++i) acc1[i][0] = acc1[i][1] = acc1[i][2] = acc1[i][3] = 0.f;
    for (int ku = warp; ku < p.KU1; ku += kSW) {
      const uint8_t* st = wait_item();
      if (ok) slice_fc1<F1, MT>(st, C.nt, ku, xrow, corr1, sx1, aff, lut, lane, acc1);
      next_item();
    }
    // cross-warp reduction (fixed warp order) -> w * SwiGLU -> h window (bf16,
    // B-fragment order), kSRed tiles per round
#pragma unroll
    for (int c0 = 0; c0 < MT; c0 += kSRed) {
      if (c0 < C.nt) {
#pragma unroll
        for (int i = 0; i < kSRed; ++i)
          if (c0 + i < MT && c0 + i < C.nt)
            red[(warp * kSRed + i) * 32 + lane] =
                make_float4(acc1[c0 + i][0], acc1[c0 + i][1], acc1[c0 + i][2], acc1[c0 + i][3]);
        __syncthreads();
        if (tid < kSRed * 32 && c0 + (tid >> 5) < C.nt) {
          const int i = tid >> 5, ln = tid & 31;
          float4 v = red[i * 32 + ln];
          for (int w = 1; w < kSW; ++w) {
            const float4 u = red[(w * kSRed + i) * 32 + ln];
            v.x += u.x; v.y += u.y; v.z += u.z; v.w += u.w;
          }
          const int tc = c0 + i;                          // tile of the chunk
          const int j = (C.etile0 + tc) * 8 + (ln >> 2);  // h column within the expert
          float bg = 0.f, bu = 0.f;
          if (p.b1) {
            bg = bf16_to_f(p.b1[(size_t)C.expert * 2 * p.I + 2 * j]);
            bu = bf16_to_f(p.b1[(size_t)C.expert * 2 * p.I + 2 * j + 1]);
          }
          const int wcol = (C.hoff + tc) * 8 + (ln >> 2);  // column in the h window
          const int ks = wcol >> 4, jj = wcol & 15;
          const float mult = (Tr2::kBetaHi == 4 && jj >= 8) ? 0.25f : 1.f;
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const int n = 2 * (ln & 3) + h;
            const float hv = silu_f((h ? v.y : v.x) + bg) * ((h ? v.w : v.z) + bu);
            const float val = slice_weight(C, wmat, n, T) * hv * mult;
            hbits[((ks * 32 + 4 * n + ((jj & 7) >> 1)) * 2 + (jj >> 3)) * 2 + (jj & 1)] =
                __bfloat16_as_ushort(__float2bfloat16_rn(val));
          }
        }
        __syncthreads();
      }
    }
    if (nr > 0)
      for (int a = 0; a < C.ngc; a += p.ngm) {  // window granule a: the chunk's completed granule a
        const uint8_t* st = wait_item();
        if (ok) slice_fc2<F2>(st, min(p.ngm, C.ngc - a), nr, a, C.g0 + a, aff, hfrag, lut, lane, acc2);
        next_item();
      }
  }
  // Nothing may land in shared memory past this point: after a wait gave up,
  // wait (bounded again) for the items issued from then on, and for x.
  for (int i = drain; i < issued; ++i) mbar_wait_sleep_bounded(&wbar[i % kSNB], (i / kSNB) & 1, p.status, p.wait_ns);
  if (misc[kMiscAbort] && tid == 0) mbar_wait_sleep_bounded(xbar, 0, p.status, p.wait_ns);
  cp_async_wait_all();
  __syncthreads();

  // ---- partial output -> fp32 accumulator (vector atomics); last CTA rounds to bf16 ----
  float* ys = reinterpret_cast<float*>(rings);  // [T][H], on the drained rings
  if (nch > 0) {
    const int g = lane >> 2, n0 = 2 * (lane & 3);
#pragma unroll
    for (int i = 0; i < kSRT; ++i) {
      if (i >= nr) break;
      const int row = (r0 + i) * 16 + g;
      if (n0 < T) {
        ys[n0 * p.H + row] = acc2[i][0];
        ys[n0 * p.H + row + 8] = acc2[i][2];
      }
      if (n0 + 1 < T) {
        ys[(n0 + 1) * p.H + row] = acc2[i][1];
        ys[(n0 + 1) * p.H + row + 8] = acc2[i][3];
      }
    }
    __syncthreads();
    if (p.b2) {  // FC2 bias, by the CTA whose chunk completes the expert's first granule
      for (int s = 0; s < nch; ++s) {
        const SChunk C = tab[s];
        if (C.g0 != 0 || C.ngc == 0) continue;
        for (int idx = tid; idx < T * p.H; idx += kSThreads) {
          const int n = idx / p.H, r = idx - n * p.H;
          ys[idx] += slice_weight(C, wmat, n, T) * bf16_to_f(p.b2[(size_t)C.expert * p.H + r]);
        }
      }
      __syncthreads();
    }
    if (misc[kMiscAbort] == 0)
      for (int i = tid; i < T * p.H / 4; i += kSThreads)
        red_add_v4_f32(p.yacc + 4 * i, reinterpret_cast<const float4*>(ys)[i]);
  }
  __syncthreads();
  if (tid == 0) {
    if (misc[kMiscAbort]) atomicAdd(p.ticket + 1, 1);  // counted before this CTA's ticket
    misc[kMiscLast] = atomic_add_acq_rel_gpu(p.ticket, 1) == G - 1;
    // after a CTA gave up a wait the sum is incomplete: y stays as it was
    if (misc[kMiscLast] && *(volatile int*)(p.ticket + 1) != 0) misc[kMiscLast] = 0;
  }
  __syncthreads();
  if (misc[kMiscLast]) {
    for (int i = tid; i < T * p.H / 4; i += kSThreads) {
      const float4 v = ld_relaxed_v4(p.yacc + 4 * i);
      uint2 o;
      o.x = pack_bf16x2(v.x, v.y);
      o.y = pack_bf16x2(v.z, v.w);
      reinterpret_cast<uint2*>(p.y)[i] = o;
    }
  }
}

// Clears the fp32 accumulator and the tickets of the decode kernel launched
// after it.  It lets that launch start at once (its CTAs wait for this
// kernel's completion before their first access to either), then waits for
// the launch before it, which may still read them.
__global__ void slice_reset_kernel(float* yacc, int n4, int* ticket) {
  pdl_trigger();
  pdl_wait();
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n4; i += gridDim.x * blockDim.x)
    reinterpret_cast<float4*>(yacc)[i] = make_float4(0.f, 0.f, 0.f, 0.f);
  if (blockIdx.x == 0 && threadIdx.x == 0) ticket[0] = ticket[1] = 0;
}

}  // namespace qmoe
