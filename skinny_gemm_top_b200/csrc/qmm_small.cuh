// Small-M quantized expert matmul (the decode hot loop).
//
// For every (expert, chunk of <= 16 tokens) segment, y[rows, m] = dequant(W)
// x[m, K] with fp32 accumulation, followed by one of three epilogues: plain
// bf16 store (single linear), bias + interleaved SwiGLU into the FC2 operand
// (FC1), bias into the expert-sorted slot buffer (FC2).
//
// Design (B200):
//  * The weights are streamed from HBM once per segment: one pass over the
//    codes serves all tokens routed to the expert, the remedy the QMoE note
//    gives for the per-token GEMV relaunch ("inner loop over tokens").
//  * Work = (segment, 16-row tile, k-unit of 64 columns; 128 for ternary).
//    With at least as many tiles as CTAs, CTA c takes a balanced range of
//    whole tiles; with fewer, a balanced range of units (stream-K), and tiles
//    split between CTAs are finished by the last CTA to arrive (atomic ticket,
//    no spin-wait), summing partials in CTA order: deterministic either way.
//  * Inside a CTA, up to 8 consecutive tiles form a sub-panel; its k-units go
//    round-robin to 8 warps.  Each warp runs its own TMA bulk-copy pipeline
//    (cp.async.bulk + mbarrier, no tensor map, no multicast) of stages holding
//    the sub-panel's codes, scales and the activation fragments of that
//    k-unit.  Each activation fragment is reused by every tile of the stage,
//    and the MMAs of all tiles of a k-step are issued back to back so their
//    latencies overlap.
//  * Codes become bf16 MMA operands with LOP3 magic numbers (unpack.cuh) and
//    are multiplied on the tensor cores (mma.sync m16n8k16, tokens in N):
//    the CUDA-core budget of sm_100a cannot afford an FMA per weight per
//    token at HBM rate.  The per-block scale is applied to the fp32 partial
//    product of each 64-column block, so the dequantized weight c*s is never
//    rounded.
//  * Programmatic dependent launch: the weights of the first stages are
//    requested before griddepcontrol.wait (they depend only on the routing
//    of an earlier launch), the activations after it.
//  * Per-warp partial sums are reduced through shared memory in warp order.
#pragma once
#include "device_common.cuh"
#include "unpack.cuh"

namespace qmoe {

constexpr int kNW = 8;            // warps per CTA
constexpr int kMaxT = 8;          // tiles per sub-panel
constexpr int kChunkTokens = 16;  // tokens per segment (<= 2 token groups of 8)

enum Epi { EPI_LINEAR = 0, EPI_SWIGLU = 1, EPI_FC2 = 2 };

// One (expert, token chunk) work item.  Fragments of its activation operand
// live at token-group offset xoff of the fragment buffers.
struct Seg {
  int expert;  // weight matrix index
  int m;       // tokens in the chunk, 1..16
  int tg;      // token groups of 8 (1 or 2)
  int slot0;   // first row of the chunk in the expert-sorted slot order (or token index)
  int xoff;    // token-group offset into the fragment buffers
  int pad[3];
};

struct SmallParams {
  const uint8_t* codes;
  unsigned long long codes_stride;   // bytes per matrix
  const uint8_t* scales;
  unsigned long long scales_stride;  // bytes per matrix
  int NT;                            // 16-row tiles per matrix
  int K;
  int KU;                            // k-units per row
  int block;                         // scale block (64 or 128)
  const int* nseg;
  const Seg* segs;
  const uint8_t* xfrag;              // activation fragments: segment at xoff * K * 16 bytes
  int nstages;
  // epilogues
  uint16_t* y;                       // LINEAR: y[token][N]
  int N;
  const uint16_t* bias;              // SWIGLU/FC2: bias + expert * bias_rows (logical rows)
  int bias_rows;
  uint8_t* hfrag;                    // SWIGLU: FC2 activation fragments (K = I)
  int I;
  int h_beta_hi;                     // 4: divide columns k%16 >= 8 by 4 (INT2 / ternary FC2)
  float* yslot;                      // FC2: yslot[slot][H]
  int H;
  float* partials;                   // 2 slots per CTA of 2 token groups * 32 float4
  int* tickets;                      // per (segment, tile), zero before the launch
  unsigned* status;
};

// Stage geometry for a format and token-group count.
template <int FMT, int TG>
struct StageGeom {
  using Tr = FmtTraits<FMT>;
  static constexpr int kBlocksPerKU = Tr::kKUcols / 64;                 // 64-col blocks per k-unit
  static constexpr int kCodeBytes = kMaxT * Tr::kCodeBytes;
  static constexpr int kScaleBytes = kBlocksPerKU * kMaxT * 32;
  static constexpr int kXBytes = kBlocksPerKU * TG * 1024;
  static constexpr int kStageBytes = ((kCodeBytes + kScaleBytes + kXBytes) + 127) / 128 * 128;
  static constexpr int kRedBytes = kNW * kMaxT * TG * 32 * 16;
};

// ---------------------------------------------------------------------------
// Balanced split of n items over G CTAs (32-bit); item boundaries scaled by
// `unit` units (KU for whole tiles, 1 for single k-units).
struct Part {
  unsigned n, q, r, unit;
  __device__ __forceinline__ void init(unsigned n_, unsigned G, unsigned unit_) {
    n = n_;
    q = n_ / G;
    r = n_ - q * G;
    unit = unit_;
  }
  __device__ __forceinline__ unsigned begin(unsigned c) const { return (c * q + min(c, r)) * unit; }
  // CTA whose range holds unit x (x < n * unit).
  __device__ __forceinline__ unsigned owner(unsigned x) const {
    const unsigned i = x / unit;
    const unsigned big = r * (q + 1);
    return i < big ? i / (q + 1) : r + (i - big) / q;
  }
};

// Sub-panel: up to kMaxT consecutive tiles of one segment inside [pos, f1).
struct SubPanel {
  unsigned next;  // first unit after this sub-panel
  int seg, rt0, nt;
  int kf;         // first k-unit of tile 0
  int kl;         // end k-unit of tile nt-1
};

__device__ __forceinline__ void load_subpanel(SubPanel& sp, unsigned pos, unsigned f1, int NT, int KU) {
  const unsigned per_seg = (unsigned)NT * (unsigned)KU;
  const unsigned seg = pos / per_seg;
  const unsigned r = pos - seg * per_seg;
  const unsigned rt = r / (unsigned)KU;
  const unsigned ku = r - rt * (unsigned)KU;
  const unsigned tile_base = seg * per_seg + rt * (unsigned)KU;
  unsigned end = f1;
  const unsigned seg_end = (seg + 1) * per_seg;
  if (seg_end < end) end = seg_end;
  const unsigned cap = tile_base + (unsigned)(kMaxT * KU);
  if (cap < end) end = cap;
  const int nt = (int)((end - tile_base + KU - 1) / (unsigned)KU);
  sp.next = end;
  sp.seg = (int)seg;
  sp.rt0 = (int)rt;
  sp.nt = nt;
  sp.kf = (int)ku;
  sp.kl = (int)(end - (tile_base + (unsigned)(nt - 1) * KU));
}

// Tiles [a, b) of the sub-panel hold k-unit ku (a = 1 when the head tile starts after ku).
__device__ __forceinline__ void active_tiles(const SubPanel& sp, int ku, int& a, int& b) {
  a = ku >= sp.kf ? 0 : 1;
  b = ku < sp.kl ? sp.nt : sp.nt - 1;
}

// Producer iterator over this warp's (sub-panel, k-unit) items; caches the
// current segment so an item costs no global load.
struct ItemIter {
  SubPanel sp;
  Seg sg;
  unsigned f1;
  int ku;
  bool valid;
};

template <int TG>
__device__ __forceinline__ void iter_load_seg(ItemIter& it, const SmallParams& p, int prev_seg) {
  if (it.sp.seg != prev_seg) {
    it.sg = p.segs[it.sp.seg];
    if (it.sg.tg > TG || it.sg.tg < 1) it.sg.tg = TG;  // never overrun the stage buffer (flagged by the consumer)
  }
}

template <int TG>
__device__ __forceinline__ void iter_advance(ItemIter& it, const SmallParams& p, int warp) {
  for (;;) {
    it.ku += kNW;
    if (it.ku >= p.KU) {
      if (it.sp.next >= it.f1) { it.valid = false; return; }
      const int prev = it.sp.seg;
      load_subpanel(it.sp, it.sp.next, it.f1, p.NT, p.KU);
      iter_load_seg<TG>(it, p, prev);
      it.ku = warp;
      if (it.ku >= p.KU) { it.ku = p.KU; continue; }  // this warp has no k-unit here
    }
    int a, b;
    active_tiles(it.sp, it.ku, a, b);
    if (a < b) return;
  }
}

template <int TG>
__device__ __forceinline__ void iter_begin(ItemIter& it, const SmallParams& p, unsigned f0, unsigned f1, int warp) {
  it.f1 = f1;
  it.valid = f0 < f1;
  if (!it.valid) return;
  load_subpanel(it.sp, f0, f1, p.NT, p.KU);
  iter_load_seg<TG>(it, p, -1);
  it.ku = warp - kNW;
  iter_advance<TG>(it, p, warp);
}

// Stage byte count of an item: codes/scales of tiles [0, b) plus the activations.
template <int FMT, int TG>
__device__ __forceinline__ uint32_t stage_bytes(const ItemIter& it) {
  using G = StageGeom<FMT, TG>;
  int a, b;
  active_tiles(it.sp, it.ku, a, b);
  return (uint32_t)(b * FmtTraits<FMT>::kCodeBytes + G::kBlocksPerKU * b * 32 + G::kBlocksPerKU * it.sg.tg * 1024);
}

// Weight part of a stage: codes and scales of tiles [0, b) of the sub-panel at k-unit ku.
template <int FMT, int TG>
__device__ __forceinline__ void issue_weights(const SmallParams& p, const ItemIter& it, uint8_t* stage, uint64_t* bar) {
  using G = StageGeom<FMT, TG>;
  using Tr = FmtTraits<FMT>;
  int a, b;
  active_tiles(it.sp, it.ku, a, b);
  const int tile = it.sp.rt0;
  const uint8_t* csrc = p.codes + (unsigned long long)it.sg.expert * p.codes_stride +
                        ((unsigned long long)it.ku * p.NT + tile) * Tr::kCodeBytes;
  bulk_copy_g2s(stage, csrc, (uint32_t)(b * Tr::kCodeBytes), bar);
#pragma unroll
  for (int bl = 0; bl < G::kBlocksPerKU; ++bl) {
    const int sb = (it.ku * Tr::kKUcols + bl * 64) / p.block;
    const uint8_t* ssrc = p.scales + (unsigned long long)it.sg.expert * p.scales_stride +
                          ((unsigned long long)sb * p.NT + tile) * 32;
    bulk_copy_g2s(stage + G::kCodeBytes + bl * kMaxT * 32, ssrc, (uint32_t)(b * 32), bar);
  }
}

// Activation part of a stage.
template <int FMT, int TG>
__device__ __forceinline__ void issue_acts(const SmallParams& p, const ItemIter& it, uint8_t* stage, uint64_t* bar) {
  using G = StageGeom<FMT, TG>;
  const uint8_t* xsrc = p.xfrag + (unsigned long long)it.sg.xoff * p.K * 16 +
                        (unsigned long long)it.ku * G::kBlocksPerKU * it.sg.tg * 1024;
  bulk_copy_g2s(stage + G::kCodeBytes + G::kScaleBytes, xsrc, (uint32_t)(G::kBlocksPerKU * it.sg.tg * 1024), bar);
}

__device__ __forceinline__ float silu_f(float g) { return g / (1.0f + __expf(-g)); }

__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// Epilogue of one reduced fragment: rows g / g+8 of tile rt, tokens n0, n0+1.
template <int EPI>
__device__ __forceinline__ void epilogue(const SmallParams& p, const Seg& sg, int rt, int tg, int lane,
                                         float4 v) {
  const int g = lane >> 2, q = lane & 3;
  const int n0 = tg * 8 + 2 * q;
  if (EPI == EPI_LINEAR) {
    const int r0 = rt * 16 + g, r1 = r0 + 8;
    if (n0 < sg.m) {
      uint16_t* yr = p.y + (size_t)(sg.slot0 + n0) * p.N;
      yr[r0] = __bfloat16_as_ushort(__float2bfloat16_rn(v.x));
      yr[r1] = __bfloat16_as_ushort(__float2bfloat16_rn(v.z));
    }
    if (n0 + 1 < sg.m) {
      uint16_t* yr = p.y + (size_t)(sg.slot0 + n0 + 1) * p.N;
      yr[r0] = __bfloat16_as_ushort(__float2bfloat16_rn(v.y));
      yr[r1] = __bfloat16_as_ushort(__float2bfloat16_rn(v.w));
    }
  } else if (EPI == EPI_FC2) {
    const int r0 = rt * 16 + g, r1 = r0 + 8;
    float b0 = 0.f, b1 = 0.f;
    if (p.bias) {
      const uint16_t* bp = p.bias + (size_t)sg.expert * p.bias_rows;
      b0 = bf16_to_f(bp[r0]);
      b1 = bf16_to_f(bp[r1]);
    }
    if (n0 < sg.m) {
      float* yr = p.yslot + (size_t)(sg.slot0 + n0) * p.H;
      yr[r0] = v.x + b0;
      yr[r1] = v.z + b1;
    }
    if (n0 + 1 < sg.m) {
      float* yr = p.yslot + (size_t)(sg.slot0 + n0 + 1) * p.H;
      yr[r0] = v.y + b0;
      yr[r1] = v.w + b1;
    }
  } else {  // EPI_SWIGLU: row g = gate j, row g+8 = up j
    const int j = rt * 8 + g;
    float bg = 0.f, bu = 0.f;
    if (p.bias) {
      const uint16_t* bp = p.bias + (size_t)sg.expert * p.bias_rows;
      bg = bf16_to_f(bp[2 * j]);
      bu = bf16_to_f(bp[2 * j + 1]);
    }
    const float h0 = n0 < sg.m ? silu_f(v.x + bg) * (v.z + bu) : 0.f;
    const float h1 = n0 + 1 < sg.m ? silu_f(v.y + bg) * (v.w + bu) : 0.f;
    // FC2 operand fragment position of (token, k = j).
    const int kb = j >> 6, kk = j & 63, ks = kk >> 4, kc = kk & 15;
    const float inv = (kc >= 8 && p.h_beta_hi == 4) ? 0.25f : 1.0f;
    const int reg = ks * 2 + (kc >> 3), half = kc & 1;
    uint16_t* base = reinterpret_cast<uint16_t*>(p.hfrag + (size_t)sg.xoff * p.I * 16);
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int n = n0 + e;
      const int ln = ((n & 7) << 2) | ((kc & 7) >> 1);
      const size_t off = ((((size_t)kb * sg.tg + (n >> 3)) * 32 + ln) * 8 + reg) * 2 + half;
      base[off] = __bfloat16_as_ushort(__float2bfloat16_rn((e ? h1 : h0) * inv));
    }
  }
}

// ---------------------------------------------------------------------------
// One item: tiles [0, NTL) of a stage (NTL = a power of two >= b).  Tiles
// outside [mask_lo, b) contribute with scale 0 (their codes are stale but
// finite), so all NTL tiles run the same straight-line code and the MMAs of a
// k-step for every tile issue back to back.
template <int FMT, int TG, int NTL>
__device__ __forceinline__ void compute_item(const uint8_t* cbuf, const uint32_t* sbuf, const uint8_t* xbuf,
                                             int sg_tg, bool tg2, int lane, int mask_lo, int b,
                                             const uint32_t* lut, float (&acc)[kMaxT][TG][4]) {
  using Tr = FmtTraits<FMT>;
  constexpr int BPK = Tr::kKUcols / 64;
  const uint32_t aconst[4] = {Tr::kConstLo, Tr::kConstLo, Tr::kConstHi, Tr::kConstHi};
  const int g = lane >> 2;
  // activation fragments of each 64-column block and the constant-operand products
  uint32_t bfr[BPK][TG][4][2];
  float corr[BPK][TG][4];
#pragma unroll
  for (int bl = 0; bl < BPK; ++bl)
#pragma unroll
    for (int t = 0; t < TG; ++t) {
#pragma unroll
      for (int e = 0; e < 4; ++e) corr[bl][t][e] = 0.f;
      if (t == 0 || tg2) {
        const uint4* xp = reinterpret_cast<const uint4*>(xbuf + ((size_t)(bl * sg_tg + t) * 32 + lane) * 32);
        const uint4 u0 = xp[0], u1 = xp[1];
        bfr[bl][t][0][0] = u0.x; bfr[bl][t][0][1] = u0.y; bfr[bl][t][1][0] = u0.z; bfr[bl][t][1][1] = u0.w;
        bfr[bl][t][2][0] = u1.x; bfr[bl][t][2][1] = u1.y; bfr[bl][t][3][0] = u1.z; bfr[bl][t][3][1] = u1.w;
#pragma unroll
        for (int k2 = 0; k2 < 4; ++k2) mma_bf16_16816(corr[bl][t], aconst, bfr[bl][t][k2][0], bfr[bl][t][k2][1]);
      } else {
#pragma unroll
        for (int k2 = 0; k2 < 4; ++k2) bfr[bl][t][k2][0] = bfr[bl][t][k2][1] = 0u;
      }
    }
  // per-tile scales (0 outside [mask_lo, b))
  float s_lo[BPK][NTL], s_hi[BPK][NTL];
#pragma unroll
  for (int bl = 0; bl < BPK; ++bl)
#pragma unroll
    for (int i = 0; i < NTL; ++i) {
      const uint32_t sc = sbuf[bl * kMaxT * 8 + i * 8 + g];
      const bool on = i >= mask_lo && i < b;
      s_lo[bl][i] = on ? bf16_lo(sc) : 0.f;
      s_hi[bl][i] = on ? bf16_hi(sc) : 0.f;
    }

  if constexpr (FMT == 3) {
    // ternary: one 13-byte record per tile covers both 64-column blocks
#pragma unroll
    for (int i = 0; i < NTL; ++i) {
      uint32_t am[8][4];
      unpack_tern_record(cbuf + (size_t)i * Tr::kCodeBytes + lane * 13, lut, am);
#pragma unroll
      for (int bl = 0; bl < BPK; ++bl)
#pragma unroll
        for (int t = 0; t < TG; ++t) {
          if (t == 1 && !tg2) continue;
          float tmp[4] = {corr[bl][t][0], corr[bl][t][1], corr[bl][t][2], corr[bl][t][3]};
#pragma unroll
          for (int k2 = 0; k2 < 4; ++k2) mma_bf16_16816(tmp, am[bl * 4 + k2], bfr[bl][t][k2][0], bfr[bl][t][k2][1]);
          acc[i][t][0] = fmaf(s_lo[bl][i], tmp[0], acc[i][t][0]);
          acc[i][t][1] = fmaf(s_lo[bl][i], tmp[1], acc[i][t][1]);
          acc[i][t][2] = fmaf(s_hi[bl][i], tmp[2], acc[i][t][2]);
          acc[i][t][3] = fmaf(s_hi[bl][i], tmp[3], acc[i][t][3]);
        }
    }
  } else {
    constexpr int W = FMT == 2 ? 2 : 4;  // lane words per tile (INT2: 2 k-steps each, INT4: 1)
    uint32_t wd[NTL][W];
#pragma unroll
    for (int i = 0; i < NTL; ++i) {
      if constexpr (FMT == 2) {
        const uint2 w = *reinterpret_cast<const uint2*>(cbuf + (size_t)i * Tr::kCodeBytes + lane * 8);
        wd[i][0] = w.x; wd[i][1] = w.y;
      } else {
        const uint4 w = *reinterpret_cast<const uint4*>(cbuf + (size_t)i * Tr::kCodeBytes + lane * 16);
        wd[i][0] = w.x; wd[i][1] = w.y; wd[i][2] = w.z; wd[i][3] = w.w;
      }
    }
    float tmp[NTL][TG][4];
#pragma unroll
    for (int i = 0; i < NTL; ++i)
#pragma unroll
      for (int t = 0; t < TG; ++t)
#pragma unroll
        for (int e = 0; e < 4; ++e) tmp[i][t][e] = corr[0][t][e];
#pragma unroll
    for (int w = 0; w < W; ++w) {
#pragma unroll
      for (int i = 0; i < NTL; ++i) {
        if constexpr (FMT == 2) {
          uint32_t a0[4], a1[4];
          unpack_int2_word(wd[i][w], a0, a1);
#pragma unroll
          for (int t = 0; t < TG; ++t) {
            if (t == 1 && !tg2) continue;
            mma_bf16_16816(tmp[i][t], a0, bfr[0][t][2 * w][0], bfr[0][t][2 * w][1]);
            mma_bf16_16816(tmp[i][t], a1, bfr[0][t][2 * w + 1][0], bfr[0][t][2 * w + 1][1]);
          }
        } else {
          uint32_t a0[4];
          unpack_int4_word(wd[i][w], a0);
#pragma unroll
          for (int t = 0; t < TG; ++t) {
            if (t == 1 && !tg2) continue;
            mma_bf16_16816(tmp[i][t], a0, bfr[0][t][w][0], bfr[0][t][w][1]);
          }
        }
      }
    }
#pragma unroll
    for (int i = 0; i < NTL; ++i)
#pragma unroll
      for (int t = 0; t < TG; ++t) {
        acc[i][t][0] = fmaf(s_lo[0][i], tmp[i][t][0], acc[i][t][0]);
        acc[i][t][1] = fmaf(s_lo[0][i], tmp[i][t][1], acc[i][t][1]);
        acc[i][t][2] = fmaf(s_hi[0][i], tmp[i][t][2], acc[i][t][2]);
        acc[i][t][3] = fmaf(s_hi[0][i], tmp[i][t][3], acc[i][t][3]);
      }
  }
}

template <int FMT, int TG, int EPI>
__global__ void __launch_bounds__(kNW * 32, 1) qmm_small_kernel(const SmallParams p) {
  using G = StageGeom<FMT, TG>;
  extern __shared__ __align__(128) uint8_t smem[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int NST = p.nstages;

  uint64_t* bars = reinterpret_cast<uint64_t*>(smem);                   // [kNW][NST]
  uint32_t* lut = reinterpret_cast<uint32_t*>(smem + 1024);            // 243 entries (ternary)
  float4* red = reinterpret_cast<float4*>(smem + 2048);                 // [kNW][kMaxT][TG][32]
  uint8_t* stages = smem + 2048 + G::kRedBytes;                         // [kNW][NST][stage]
  __shared__ int s_flag[2];
  __shared__ int s_abort;

  // The segment table comes from a launch at least two back in the stream.
  const int nseg = *p.nseg;
  const unsigned ntiles = (unsigned)nseg * (unsigned)p.NT;
  const bool tile_mode = ntiles >= gridDim.x;
  Part part;
  if (tile_mode) part.init(ntiles, gridDim.x, (unsigned)p.KU);
  else part.init(ntiles * (unsigned)p.KU, gridDim.x, 1u);
  const unsigned f0 = part.begin(blockIdx.x), f1 = part.begin(blockIdx.x + 1);
  if (f0 >= f1) {  // whole CTA idle
    pdl_wait();
    pdl_trigger();
    return;
  }

  if (tid == 0) s_abort = 0;
  if constexpr (FMT == 3)
    for (int i = tid; i < 243; i += blockDim.x) lut[i] = tern_lut_entry(i);
  uint64_t* wbar = bars + warp * NST;
  uint8_t* wstage = stages + (size_t)warp * NST * G::kStageBytes;
  if (lane == 0)
    for (int s = 0; s < NST; ++s) mbar_init(&wbar[s], 1);
  fence_mbar_init();
  __syncthreads();

  // Producer (lane 0): the weights of the first NST items before the
  // dependency wait, their activations after it.
  ItemIter prod;
  int primed = 0;
  if (lane == 0) {
    iter_begin<TG>(prod, p, f0, f1, warp);
    for (int s = 0; s < NST && prod.valid; ++s, ++primed) {
      mbar_arrive_expect_tx(&wbar[s], stage_bytes<FMT, TG>(prod));
      issue_weights<FMT, TG>(p, prod, wstage + s * G::kStageBytes, &wbar[s]);
      iter_advance<TG>(prod, p, warp);
    }
  }
  pdl_wait();
  pdl_trigger();
  if (lane == 0) {
    ItemIter again;
    iter_begin<TG>(again, p, f0, f1, warp);
    for (int s = 0; s < primed; ++s) {
      issue_acts<FMT, TG>(p, again, wstage + s * G::kStageBytes, &wbar[s]);
      iter_advance<TG>(again, p, warp);
    }
  }
  __syncwarp();

  int item = 0;           // this warp's consumed items
  bool aborted = false;   // this warp gave up waiting

  SubPanel sp;
  unsigned pos = f0;
  const int head_tile_glob = (int)(f0 / (unsigned)p.KU);
  int cur_seg = -1;
  Seg sg;
  while (pos < f1) {
    load_subpanel(sp, pos, f1, p.NT, p.KU);
    if (sp.seg != cur_seg) {
      cur_seg = sp.seg;
      sg = p.segs[sp.seg];
      if (sg.tg > TG || sg.tg < 1) {
        if (tid == 0) atomicOr(p.status, kStatusBadSegment);
        sg.tg = TG;
      }
    }
    const bool tg2 = TG == 2 && sg.tg == 2;
    float acc[kMaxT][TG][4];
#pragma unroll
    for (int i = 0; i < kMaxT; ++i)
#pragma unroll
      for (int t = 0; t < TG; ++t)
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[i][t][e] = 0.f;

    for (int ku = warp; ku < p.KU; ku += kNW) {
      int a, b;
      active_tiles(sp, ku, a, b);
      if (a >= b) continue;
      const int s = item % NST;
      const uint32_t par = (uint32_t)(item / NST) & 1u;
      ++item;
      if (!aborted && !mbar_wait_bounded(&wbar[s], par, p.status)) {
        aborted = true;
        s_abort = 1;
      }
      uint8_t* st = wstage + s * G::kStageBytes;
      if (!aborted) {
        const uint8_t* cbuf = st;
        const uint32_t* sbuf = reinterpret_cast<const uint32_t*>(st + G::kCodeBytes);
        const uint8_t* xbuf = st + G::kCodeBytes + G::kScaleBytes;
        if (b > 4) compute_item<FMT, TG, 8>(cbuf, sbuf, xbuf, sg.tg, tg2, lane, a, b, lut, acc);
        else if (b > 2) compute_item<FMT, TG, 4>(cbuf, sbuf, xbuf, sg.tg, tg2, lane, a, b, lut, acc);
        else if (b > 1) compute_item<FMT, TG, 2>(cbuf, sbuf, xbuf, sg.tg, tg2, lane, a, b, lut, acc);
        else compute_item<FMT, TG, 1>(cbuf, sbuf, xbuf, sg.tg, tg2, lane, a, b, lut, acc);
      }
      __syncwarp();
      if (lane == 0 && prod.valid && !aborted) {
        fence_proxy_async_smem();
        mbar_arrive_expect_tx(&wbar[s], stage_bytes<FMT, TG>(prod));
        issue_weights<FMT, TG>(p, prod, st, &wbar[s]);
        issue_acts<FMT, TG>(p, prod, st, &wbar[s]);
        iter_advance<TG>(prod, p, warp);
      }
      __syncwarp();
    }

    // ---- CTA reduction of the sub-panel -------------------------------------
#pragma unroll
    for (int i = 0; i < kMaxT; ++i) {
      if (i >= sp.nt) continue;
#pragma unroll
      for (int t = 0; t < TG; ++t)
        red[((warp * kMaxT + i) * TG + t) * 32 + lane] =
            make_float4(acc[i][t][0], acc[i][t][1], acc[i][t][2], acc[i][t][3]);
    }
    __syncthreads();
    const bool ab = s_abort != 0;
    const int nel = sp.nt * TG * 32;
    const int last_tile = sp.nt - 1;
    const bool head_partial = sp.kf > 0 || (sp.nt == 1 && sp.kl < p.KU);
    const bool tail_partial = sp.kl < p.KU && sp.nt > 1;
#pragma unroll
    for (int r = 0; r < (kMaxT * TG * 32 + kNW * 32 - 1) / (kNW * 32); ++r) {
      const int e = tid + r * kNW * 32;
      if (e >= nel) continue;
      float4 v = red[e];
      for (int w = 1; w < kNW; ++w) {
        const float4 u = red[w * kMaxT * TG * 32 + e];
        v.x += u.x; v.y += u.y; v.z += u.z; v.w += u.w;
      }
      const int i = e / (TG * 32), t = (e / 32) % TG, ln = e % 32;
      if (t == 1 && !tg2) continue;
      const bool partial = (i == 0 && head_partial) || (i == last_tile && tail_partial);
      if (ab) continue;
      if (!partial) {
        epilogue<EPI>(p, sg, sp.rt0 + i, t, ln, v);
      } else {
        const int tglob = sp.seg * p.NT + sp.rt0 + i;
        const int slot = 2 * blockIdx.x + (tglob == head_tile_glob ? 0 : 1);
        reinterpret_cast<float4*>(p.partials)[((size_t)slot * 2 + t) * 32 + ln] = v;
      }
    }
    if (head_partial || tail_partial) {  // only in unit mode
      __threadfence();
      __syncthreads();
      if (tid < 2) {
        s_flag[tid] = 0;
        const bool want = tid == 0 ? head_partial : tail_partial;
        if (want && !ab) {
          const int i = tid == 0 ? 0 : last_tile;
          const int tglob = sp.seg * p.NT + sp.rt0 + i;
          const unsigned T0 = (unsigned)tglob * (unsigned)p.KU;
          const unsigned clo = part.owner(T0), chi = part.owner(T0 + p.KU - 1);
          int ncontrib = 0;
          for (unsigned c = clo; c <= chi; ++c)
            if (part.begin(c + 1) > part.begin(c)) ++ncontrib;
          const int old = atomicAdd(&p.tickets[tglob], 1);
          if (old == ncontrib - 1) {
            s_flag[tid] = 1;
            p.tickets[tglob] = 0;  // leave the ticket clean for the next launch
          }
        }
      }
      __syncthreads();
      if (s_flag[0] || s_flag[1]) {
        __threadfence();
#pragma unroll
        for (int r = 0; r < (kMaxT * TG * 32 + kNW * 32 - 1) / (kNW * 32); ++r) {
          const int e = tid + r * kNW * 32;
          if (e >= nel) continue;
          const int i = e / (TG * 32), t = (e / 32) % TG, ln = e % 32;
          if (t == 1 && !tg2) continue;
          const int which = (i == 0 && head_partial) ? 0 : ((i == last_tile && tail_partial) ? 1 : -1);
          if (which < 0 || !s_flag[which]) continue;
          const int tglob = sp.seg * p.NT + sp.rt0 + i;
          const unsigned T0 = (unsigned)tglob * (unsigned)p.KU;
          const unsigned clo = part.owner(T0), chi = part.owner(T0 + p.KU - 1);
          float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
          for (unsigned c = clo; c <= chi; ++c) {
            const unsigned b0 = part.begin(c), b1 = part.begin(c + 1);
            if (b1 <= b0) continue;
            const int slot = 2 * (int)c + ((int)(b0 / (unsigned)p.KU) == tglob ? 0 : 1);
            const float4 u = __ldcg(reinterpret_cast<const float4*>(p.partials) + ((size_t)slot * 2 + t) * 32 + ln);
            v.x += u.x; v.y += u.y; v.z += u.z; v.w += u.w;
          }
          epilogue<EPI>(p, sg, sp.rt0 + i, t, ln, v);
        }
      }
    }
    __syncthreads();
    pos = sp.next;
  }

  // Drain: if this warp gave up waiting, let its copies in flight land (bounded).
  if (aborted && lane == 0) {
    for (int s = 0; s < NST; ++s) mbar_wait_bounded(&wbar[s], (uint32_t)((item + s) / NST) & 1u, nullptr);
  }
}

}  // namespace qmoe
