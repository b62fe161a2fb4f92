// Large-M grouped expert matmul on the 5th-generation tensor cores (tcgen05).
//
// For experts that receive many tokens (prefill), the expert is a dense
// contraction: each 128-row weight tile is dequantized once per token tile
// into shared memory and multiplied on the tensor cores with fp32
// accumulators in tensor memory.  This is the "decompress, then dense matmul"
// remedy of the QMoE note, done tile by tile so that the full bf16 expert is
// never materialized (the onnxruntime PR's Description: "Avoid full A16
// expert-weight materialization").
//
// One persistent CTA per SM, 19 warps, all waits bounded:
//   warp 0      weight producer: packed codes + scales (cp.async.bulk) of every
//               64-column k-stage, into a ring of CS stages;
//   warp 18     token producer: the token tile of every k-stage
//               (cp.async.bulk.tensor 2-D, 128-byte swizzle, no multicast),
//               into a ring of kGStages stages;
//   warp 1      TMEM allocator and single-thread MMA issuer
//               (tcgen05.mma.cta_group::1.kind::f16, M=128, N<=256, bf16);
//   warps 2-9   dequantize (one 16-row tile each): codes -> bf16(c*s) in the UMMA K-major
//               128-byte-swizzle layout;
//   warps 10-17 epilogue (two per TMEM lane quarter, alternate 32-column chunks):
//               tcgen05.ld the fp32 accumulators, bias + SwiGLU
//               (FC1), bias (FC2) or nothing (single linear), store.
// Two TMEM accumulators (2 x 256 columns) let the epilogue of one unit overlap
// the main loop of the next.  Template parameters: BT = token rows per unit (256
// for expert tiles, 128 for the single linear), CS = weight-ring depth.  A
// k-stage of packed weights is only 2-4 KB, so with few tokens (the single
// linear) the ring must hold many of them to keep enough bytes in flight.
//
// The weight operand is bf16_rne(c*s): the tensor-core product needs one bf16
// operand per weight, so this path rounds the dequantized weight once (the
// small-M path keeps c*s exact by scaling fp32 partial sums instead).
#pragma once
#include <cuda.h>

#include "device_common.cuh"
#include "qmm_small.cuh"
#include "unpack.cuh"

namespace qmoe {

constexpr int kGRows = 128;        // UMMA M: weight rows per unit
constexpr int kGTok = 256;         // UMMA N upper bound: tokens per unit
constexpr int kGStages = 4;
constexpr int kGDeqWarps = 8;     // one 16-row tile of the 128-row unit each
constexpr int kGDeqTiles = 8 / kGDeqWarps;
constexpr int kGEpiWarps = 8;     // two per TMEM lane quarter
constexpr int kGWarps = 3 + kGDeqWarps + kGEpiWarps;
constexpr int kGTokWarp = 2 + kGDeqWarps + kGEpiWarps;  // the token producer
constexpr int kGThreads = kGWarps * 32;
constexpr int kGABytes = kGRows * 64 * 2;      // 16 KB bf16 weight tile per k-stage
constexpr int kGTmaRows = 64;                  // rows per 2-D TMA box
constexpr int kLinBT = 128;                    // single linear: token rows per unit
constexpr int kGAccCols = 256;

struct GSeg {
  int expert;
  int slot0;  // first expert-sorted slot row of the tile
  int ntok;   // 1..256
  int pad;
};

struct GroupedParams {
  const uint8_t* codes;
  unsigned long long codes_stride;
  const uint8_t* scales;
  unsigned long long scales_stride;
  const uint8_t* zeros;  // affine codes: zero points, laid out like the scales; NULL: symmetric
  int NT;       // 16-row tiles per matrix
  int K;
  int block;
  int rtiles;   // 128-row tiles per matrix
  const int* ngseg;
  const GSeg* gsegs;
  const uint16_t* bias;
  int bias_rows;
  uint16_t* hrows;  // SWIGLU output [slot][I] bf16
  int I;
  float* yslot;     // FC2 output [slot][H]
  int H;
  uint16_t* y;      // single linear output [token][N] bf16 (EPI_LINEAR)
  int N;
  int ntok;         // ngseg == nullptr: segments are chunks of BT of ntok token rows of matrix 0
  unsigned* status;
};

template <int BT>
__device__ __forceinline__ int g_nseg(const GroupedParams& p) {
  return p.ngseg ? *p.ngseg : (p.ntok + BT - 1) / BT;
}

template <int BT>
__device__ __forceinline__ GSeg g_seg(const GroupedParams& p, int i) {
  if (p.gsegs) return p.gsegs[i];
  GSeg sg;
  sg.expert = 0;
  sg.slot0 = i * BT;
  sg.ntok = min(BT, p.ntok - i * BT);
  sg.pad = 0;
  return sg;
}

template <int FMT, int BT, int CS>
struct GGeom {
  static constexpr int kCodeBytes = 8 * FmtTraits<FMT>::kCodeBytes;  // 8 tiles of 16 rows, 64 columns
  static constexpr int kCStage = kCodeBytes + 2 * 8 * 32;  // codes, scales, zero points (affine)
  static constexpr int kBBytes = BT * 64 * 2;                         // token tile per k-stage
  static constexpr int kCRing = ((CS * kCStage + 127) / 128) * 128;
  static constexpr int kBars = (((2 * CS + 4 * kGStages + 5) * 8 + 16 + 127) / 128) * 128;
  static constexpr int kSmem = 1024 /*align slack*/ + kGStages * (kGABytes + kBBytes) + kCRing + kBars;
};

// ---- tcgen05 / TMA helpers ----------------------------------------------------

__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, int x, int y, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], "
      "[%4];" ::"r"(smem_addr(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_addr(bar))
      : "memory");
}

// K-major operand with 128-byte swizzle: 8-row atoms of 1024 bytes.
__device__ __forceinline__ uint64_t umma_desc_sw128(const void* p) {
  const uint64_t a = smem_addr(p);
  return ((a >> 4) & 0x3FFFull) | (1ull << 16) /* LBO 16 B */ | ((uint64_t)(1024 >> 4) << 32) /* SBO */ |
         (1ull << 46) /* sm100 descriptor version */ | (2ull << 61) /* SWIZZLE_128B */;
}

// kind::f16 instruction descriptor: D fp32, A/B bf16, both K-major, M = 128.
__device__ __forceinline__ uint32_t umma_idesc_bf16(int n) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(n >> 3) << 17) | ((uint32_t)(kGRows >> 4) << 24);
}

__device__ __forceinline__ void umma_bf16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                          uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate));
}

__device__ __forceinline__ void umma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   smem_addr(bar))
               : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&v)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,"
      "%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
        "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15]),
        "=r"(v[16]), "=r"(v[17]), "=r"(v[18]), "=r"(v[19]), "=r"(v[20]), "=r"(v[21]), "=r"(v[22]), "=r"(v[23]),
        "=r"(v[24]), "=r"(v[25]), "=r"(v[26]), "=r"(v[27]), "=r"(v[28]), "=r"(v[29]), "=r"(v[30]), "=r"(v[31])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// Bounded wait that also gives up as soon as another role has aborted.
__device__ __forceinline__ bool gwait(uint64_t* bar, uint32_t parity, unsigned* status, volatile int* abort_flag) {
  if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = global_timer_ns();
  for (uint32_t it = 0;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 63) == 0) {
      if (*abort_flag) return false;
      if (global_timer_ns() - t0 > kWaitLimitNs) {
        *abort_flag = 1;
        if (status) atomicOr(status, kStatusTimeout);
        return false;
      }
    }
  }
}

template <int FMT, int EPI, int BT, int CS>
__global__ void __launch_bounds__(kGThreads, 1)
    qmm_grouped_kernel(const __grid_constant__ CUtensorMap tmap, const GroupedParams p) {
  using Tr = FmtTraits<FMT>;
  using GG = GGeom<FMT, BT, CS>;
  constexpr bool kKS = EPI == EPI_FC2;  // FC2 weights are packed QMOE_ROWS_KSPLIT
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024 - (smem_addr(smem_raw) & 1023)) & 1023);
  uint8_t* sA = smem;                                        // [kGStages][16 KB]
  uint8_t* sB = sA + kGStages * kGABytes;                    // [kGStages][BT rows x 128 B]
  uint8_t* sC = sB + kGStages * GG::kBBytes;                 // [CS][codes | scales]
  uint64_t* bars = reinterpret_cast<uint64_t*>(sC + GG::kCRing);
  uint64_t* full_c = bars;                                   // [CS]
  uint64_t* empty_c = bars + CS;                             // [CS]
  uint64_t* full_ab = bars + 2 * CS;                         // [kGStages]
  uint64_t* empty_ab = bars + 2 * CS + kGStages;             // [kGStages]
  uint64_t* tm_full = bars + 2 * CS + 2 * kGStages;
  uint64_t* tm_empty = tm_full + 2;
  uint64_t* mma_done = tm_empty + 2;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(mma_done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int n_units = g_nseg<BT>(p) * p.rtiles;
  if ((int)blockIdx.x >= n_units) return;
  const int KS = p.K / 64;

  if (tid == 0) {
    for (int s = 0; s < CS; ++s) {
      mbar_init(&full_c[s], 1);
      mbar_init(&empty_c[s], kGDeqWarps);
    }
    for (int s = 0; s < kGStages; ++s) {
      mbar_init(&full_ab[s], 1 + kGDeqWarps);
      mbar_init(&empty_ab[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tm_full[a], 1);
      mbar_init(&tm_empty[a], kGEpiWarps);
    }
    mbar_init(mma_done, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_addr(tmem_holder)),
                 "r"(2 * kGAccCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;

  if (warp == 0) {
    // ---------------- weight producer ----------------
    // The two copies of a stage are issued by different lanes in one step: a
    // bulk copy costs ~117 cycles to issue from one lane, while the SM accepts
    // one every ~56.
    uint32_t it = 0;
    bool ok = true;
    for (int u = blockIdx.x; u < n_units && ok && !*abort_flag; u += gridDim.x) {
      const GSeg sg = g_seg<BT>(p, u / p.rtiles);
      const int rt = u % p.rtiles;
      for (int ks = 0; ks < KS; ++ks, ++it) {
        const int s = it % CS;
        const uint32_t ph = (it / CS) & 1u;
        const int w_ok = lane == 0 ? (int)gwait(&empty_c[s], ph ^ 1u, p.status, abort_flag) : 0;
        if (!__shfl_sync(0xffffffffu, w_ok, 0)) { ok = false; break; }
        uint8_t* cdst = sC + s * GG::kCStage;
        if (lane == 0) mbar_arrive_expect_tx(&full_c[s], GG::kCodeBytes + (p.zeros ? 2 : 1) * 8 * 32);
        __syncwarp();
        constexpr int kSlabs = kKS ? (FMT == 2 ? 2 : 4) : 1;  // FC2 (KSPLIT): one 8-tile copy per slab
        if (lane < kSlabs) {
          const unsigned long long off =
              kKS ? (((unsigned long long)ks * kSlabs + lane) * p.NT + rt * 8) * 128
                  : ((unsigned long long)ks * p.NT + rt * 8) * Tr::kCodeBytes;
          bulk_copy_g2s(cdst + lane * (GG::kCodeBytes / kSlabs), p.codes + (unsigned long long)sg.expert * p.codes_stride + off,
                        GG::kCodeBytes / kSlabs, &full_c[s]);
        }
        if (lane == kSlabs) {
          const int sb = ks * 64 / p.block;
          bulk_copy_g2s(cdst + GG::kCodeBytes, p.scales + (unsigned long long)sg.expert * p.scales_stride +
                                                   ((unsigned long long)sb * p.NT + rt * 8) * 32,
                        8 * 32, &full_c[s]);
        }
        if (lane == kSlabs + 1 && p.zeros) {
          const int sb = ks * 64 / p.block;
          bulk_copy_g2s(cdst + GG::kCodeBytes + 8 * 32, p.zeros + (unsigned long long)sg.expert * p.scales_stride +
                                                            ((unsigned long long)sb * p.NT + rt * 8) * 32,
                        8 * 32, &full_c[s]);
        }
      }
    }
  } else if (warp == kGTokWarp) {
    // ---------------- token producer ----------------
    uint32_t it = 0;
    bool ok = true;
    for (int u = blockIdx.x; u < n_units && ok && !*abort_flag; u += gridDim.x) {
      const GSeg sg = g_seg<BT>(p, u / p.rtiles);
      const int nsub = (sg.ntok + kGTmaRows - 1) / kGTmaRows;
      for (int ks = 0; ks < KS; ++ks, ++it) {
        const int s = it % kGStages;
        const uint32_t ph = (it / kGStages) & 1u;
        const int w_ok = lane == 0 ? (int)gwait(&empty_ab[s], ph ^ 1u, p.status, abort_flag) : 0;
        if (!__shfl_sync(0xffffffffu, w_ok, 0)) { ok = false; break; }
        if (lane == 0) mbar_arrive_expect_tx(&full_ab[s], (uint32_t)(nsub * kGTmaRows * 128));
        __syncwarp();
        if (lane < nsub)
          tma_load_2d(sB + s * GG::kBBytes + lane * kGTmaRows * 128, &tmap, ks * 64, sg.slot0 + lane * kGTmaRows,
                      &full_ab[s]);
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      uint32_t it = 0, acc_it = 0;
      for (int u = blockIdx.x; u < n_units && !*abort_flag; u += gridDim.x, ++acc_it) {
        const GSeg sg = g_seg<BT>(p, u / p.rtiles);
        const int n = (sg.ntok + 15) / 16 * 16;
        const uint32_t idesc = umma_idesc_bf16(n);
        const uint32_t a = acc_it & 1u;
        if (!gwait(&tm_empty[a], ((acc_it >> 1) & 1u) ^ 1u, p.status, abort_flag)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + a * kGAccCols;
        bool ok = true;
        for (int ks = 0; ks < KS; ++ks, ++it) {
          const int s = it % kGStages;
          const uint32_t ph = (it / kGStages) & 1u;
          if (!gwait(&full_ab[s], ph, p.status, abort_flag)) { ok = false; break; }
          tc_fence_after();
          const uint64_t ad = umma_desc_sw128(sA + s * kGABytes);
          const uint64_t bd = umma_desc_sw128(sB + s * GG::kBBytes);
#pragma unroll
          for (int j = 0; j < 4; ++j)  // 16 bf16 = 32 bytes per k-step: +2 in the 16-byte address field
            umma_bf16(d_tmem, ad + 2 * j, bd + 2 * j, idesc, (ks > 0 || j > 0) ? 1u : 0u);
          umma_commit(&empty_ab[s]);
        }
        if (!ok) break;
        umma_commit(&tm_full[a]);
      }
      // every MMA this thread issued has completed before TMEM is released
      umma_commit(mma_done);
      gwait(mma_done, 0, p.status, abort_flag);
      if (*abort_flag) mbar_wait_bounded(mma_done, 0, nullptr);
    }
  } else if (warp < 2 + kGDeqWarps) {
    // ---------------- dequantize ----------------
    const int d = warp - 2, g = lane >> 2, q = lane & 3;
    const bool aff = p.zeros != nullptr;
    uint32_t it = 0;
    for (int u = blockIdx.x; u < n_units && !*abort_flag; u += gridDim.x) {
      for (int ks = 0; ks < KS; ++ks, ++it) {
        const int sc = it % CS;
        const uint32_t phc = (it / CS) & 1u;
        const int s = it % kGStages;
        const uint32_t ph = (it / kGStages) & 1u;
        if (!gwait(&full_c[sc], phc, p.status, abort_flag)) break;
        const uint8_t* cs = sC + sc * GG::kCStage;
        uint32_t am[kGDeqTiles][4][4];
        uint32_t sw[kGDeqTiles], zw[kGDeqTiles];
#pragma unroll
        for (int tt = 0; tt < kGDeqTiles; ++tt) {
          const int tile = kGDeqTiles * d + tt;
          // lane word w: [tile][lane][w] (PLAIN, GATE_UP) or [w][tile][lane] (KSPLIT: FC2)
          auto word = [&](int w) -> uint32_t {
            constexpr int W = FMT == 2 ? 2 : 4;
            return kKS ? *reinterpret_cast<const uint32_t*>(cs + w * (8 * 128) + tile * 128 + lane * 4)
                       : *reinterpret_cast<const uint32_t*>(cs + tile * Tr::kCodeBytes + (lane * W + w) * 4);
          };
          if constexpr (FMT == 2) {
            unpack_int2_word(word(0), am[tt][0], am[tt][1]);
            unpack_int2_word(word(1), am[tt][2], am[tt][3]);
          } else {
            unpack_int4_word(word(0), am[tt][0]);
            unpack_int4_word(word(1), am[tt][1]);
            unpack_int4_word(word(2), am[tt][2]);
            unpack_int4_word(word(3), am[tt][3]);
          }
          sw[tt] = *reinterpret_cast<const uint32_t*>(cs + GG::kCodeBytes + tile * 32 + g * 4);
          zw[tt] = aff ? *reinterpret_cast<const uint32_t*>(cs + GG::kCodeBytes + 8 * 32 + tile * 32 + g * 4) : 0u;
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty_c[sc]);
        if (!gwait(&empty_ab[s], ph ^ 1u, p.status, abort_flag)) break;
        uint8_t* as = sA + s * kGABytes;
#pragma unroll
        for (int tt = 0; tt < kGDeqTiles; ++tt) {
          const int tile = kGDeqTiles * d + tt;
#pragma unroll
          for (int f = 0; f < 4; ++f) {
            // signed code c (exact small integer): c = (128 + beta*u) / beta - (128 / beta + bias);
            // affine codes: u = (128 + beta*u) / beta - 128 / beta
            const uint32_t mul = (f >= 2) ? Tr::kCodeMulHi : kBf16One;
            const uint32_t sub = aff ? ((f >= 2) ? aff_sub_hi<FMT>() : kAffConst)
                                     : ((f >= 2) ? Tr::kCodeSubHi : Tr::kConstLo);
            // the row's bf16 scale (and zero point) in both halves, straight from its bits (no fp32 round trip)
            const uint32_t sp = __byte_perm(sw[tt], 0u, (f & 1) ? 0x3232u : 0x1010u);
            const uint32_t zp = aff ? __byte_perm(zw[tt], 0u, (f & 1) ? 0x3232u : 0x1010u) : kBf16NegZero;
            const int pr = tile * 16 + g + 8 * (f & 1);
            uint8_t* rowp = as + (pr >> 3) * 1024 + (pr & 7) * 128;
#pragma unroll
            for (int k2 = 0; k2 < 4; ++k2) {
              const uint32_t c = fma_bf16x2(am[tt][k2][f], mul, sub);
              const uint32_t wv = fma_bf16x2(c, sp, zp);  // bf16_rne(c * s) or bf16_rne(s * u + z): one rounding
              const int chunk = 2 * k2 + (f >> 1);
              *reinterpret_cast<uint32_t*>(rowp + ((chunk ^ (pr & 7)) << 4) + 4 * q) = wv;
            }
          }
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&full_ab[s]);
      }
    }
  } else if (warp < 2 + kGDeqWarps + kGEpiWarps) {
    // ---------------- epilogue ----------------
    const int quarter = warp & 3;
    const int half = (warp - 2 - kGDeqWarps) >> 2;  // which alternate 32-column chunks
    const int r = quarter * 32 + lane;  // accumulator lane = tile row
    uint32_t acc_it = 0;
    for (int u = blockIdx.x; u < n_units && !*abort_flag; u += gridDim.x, ++acc_it) {
      const GSeg sg = g_seg<BT>(p, u / p.rtiles);
      const int rt = u % p.rtiles;
      const uint32_t a = acc_it & 1u;
      if (!gwait(&tm_full[a], (acc_it >> 1) & 1u, p.status, abort_flag)) break;
      tc_fence_after();
      const uint32_t tbase = tmem_base + ((uint32_t)(quarter * 32) << 16) + a * kGAccCols;
      const int prow = rt * kGRows + r;  // physical row of the matrix
      float bias_v = 0.f, bias_u = 0.f;
      int j = 0;
      bool gate = false;
      if (EPI == EPI_SWIGLU) {
        const int t16 = prow >> 4, rr = prow & 15;
        gate = rr < 8;
        j = t16 * 8 + (rr & 7);
        if (p.bias) {
          const uint16_t* bp = p.bias + (size_t)sg.expert * p.bias_rows;
          bias_v = bf16_to_f(bp[2 * j]);
          bias_u = bf16_to_f(bp[2 * j + 1]);
        }
      } else if (p.bias) {
        bias_v = bf16_to_f(p.bias[(size_t)sg.expert * p.bias_rows + prow]);
      }
      for (int c0 = 32 * half; c0 < sg.ntok; c0 += 64) {
        uint32_t v[32];
        tmem_ld32(tbase + c0, v);
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const int n = c0 + i;
          float x = __uint_as_float(v[i]);
          if (EPI == EPI_SWIGLU) {
            const float up = __shfl_down_sync(0xffffffffu, x, 8);
            if (gate && n < sg.ntok) {
              const float h = silu_f(x + bias_v) * (up + bias_u);
              p.hrows[(size_t)(sg.slot0 + n) * p.I + j] = __bfloat16_as_ushort(__float2bfloat16_rn(h));
            }
          } else if (EPI == EPI_LINEAR) {
            if (n < sg.ntok) p.y[(size_t)(sg.slot0 + n) * p.N + prow] = __bfloat16_as_ushort(__float2bfloat16_rn(x));
          } else {
            if (n < sg.ntok) p.yslot[(size_t)(sg.slot0 + n) * p.H + prow] = x + bias_v;
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tm_empty[a]);
    }
  }

  __syncthreads();
  if (*abort_flag && tid == 0) {
    // give copies still in flight time to land before the CTA exits (bounded)
    const unsigned long long t0 = global_timer_ns();
    while (global_timer_ns() - t0 < 5000000ull) {
    }
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(2 * kGAccCols)
                 : "memory");
  }
}

}  // namespace qmoe
