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
//  * Work = units of (segment, 16-row tile, k-unit of 64 columns; 128 for
//    ternary).  CTA c of G takes the contiguous unit range [F c/G, F (c+1)/G)
//    in (segment, tile, k) order, so every SM streams the same number of
//    weight bytes whatever the shape (stream-K style balance).  Tiles split
//    between CTAs are finished by the last CTA to arrive (atomic ticket, no
//    spin-wait), summing the partials in CTA order: deterministic.
//  * Inside a CTA, up to 8 consecutive tiles form a sub-panel; its k-units go
//    round-robin to 8 warps.  Each warp runs its own TMA bulk-copy pipeline
//    (cp.async.bulk + mbarrier, no tensor map, no multicast) of stages holding
//    the sub-panel's codes, scales and the activation fragments of that
//    k-unit, and reuses each activation fragment across the 8 tiles.
//  * Codes become bf16 MMA operands with LOP3 magic numbers (unpack.cuh) and
//    are multiplied on the tensor cores (mma.sync m16n8k16, tokens in N) -
//    the CUDA-core budget of sm_100a cannot afford an FMA per weight per
//    token at HBM rate.  The per-block scale is applied to the fp32 partial
//    product of each 64-column block, so the dequantized weight c*s is never
//    rounded.
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
  float* partials;                   // 2 slots per CTA of kMaxTG * 32 float4
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
// Sub-panel iteration over the CTA's unit range [f0, f1).
struct SubPanel {
  long long next;  // first unit after this sub-panel
  int seg, rt0, nt;
  int kf;          // first k-unit of tile 0
  int kl;          // end k-unit of tile nt-1
};

__device__ __forceinline__ void load_subpanel(SubPanel& sp, long long pos, long long f1, int NT, int KU) {
  const long long per_seg = (long long)NT * KU;
  const int seg = (int)(pos / per_seg);
  const long long r = pos - (long long)seg * per_seg;
  const int rt = (int)(r / KU);
  const int ku = (int)(r - (long long)rt * KU);
  const long long tile_base = (long long)seg * per_seg + (long long)rt * KU;
  long long end = f1;
  const long long seg_end = (long long)(seg + 1) * per_seg;
  if (seg_end < end) end = seg_end;
  const long long cap = tile_base + (long long)kMaxT * KU;
  if (cap < end) end = cap;
  const int nt = (int)((end - tile_base + KU - 1) / KU);
  sp.next = end;
  sp.seg = seg;
  sp.rt0 = rt;
  sp.nt = nt;
  sp.kf = ku;
  sp.kl = (int)(end - (tile_base + (long long)(nt - 1) * KU));
}

// Active tiles [a, b) of the sub-panel at k-unit ku.
__device__ __forceinline__ void active_tiles(const SubPanel& sp, int ku, int& a, int& b) {
  a = ku >= sp.kf ? 0 : 1;
  b = ku < sp.kl ? sp.nt : sp.nt - 1;
}

// Warp-level producer/consumer iterator over this warp's (sub-panel, k-unit) items.
struct ItemIter {
  SubPanel sp;
  long long f1;
  int ku;
  bool valid;
};

__device__ __forceinline__ void iter_advance(ItemIter& it, int warp, int NT, int KU) {
  for (;;) {
    it.ku += kNW;
    if (it.ku >= KU) {
      if (it.sp.next >= it.f1) { it.valid = false; return; }
      load_subpanel(it.sp, it.sp.next, it.f1, NT, KU);
      it.ku = warp;
      if (it.ku >= KU) { it.ku = KU; continue; }  // this warp has no k-unit here
    }
    int a, b;
    active_tiles(it.sp, it.ku, a, b);
    if (a < b) return;
  }
}

__device__ __forceinline__ void iter_begin(ItemIter& it, long long f0, long long f1, int warp, int NT, int KU) {
  it.f1 = f1;
  it.valid = f0 < f1;
  if (!it.valid) return;
  load_subpanel(it.sp, f0, f1, NT, KU);
  it.ku = warp - kNW;
  iter_advance(it, warp, NT, KU);
}

// Issue the bulk copies of one item into a stage buffer (called by one lane).
template <int FMT, int TG>
__device__ __forceinline__ void issue_stage(const SmallParams& p, const ItemIter& it, uint8_t* stage,
                                            uint64_t* bar) {
  using G = StageGeom<FMT, TG>;
  using Tr = FmtTraits<FMT>;
  int a, b;
  active_tiles(it.sp, it.ku, a, b);
  Seg sg = p.segs[it.sp.seg];
  if (sg.tg > TG || sg.tg < 1) sg.tg = TG;  // never overrun the stage buffer (flagged by the consumer)
  const int n = b - a;
  const int tile = it.sp.rt0 + a;
  const uint32_t cbytes = (uint32_t)(n * Tr::kCodeBytes);
  const uint32_t sbytes = (uint32_t)(n * 32);
  const uint32_t xbytes = (uint32_t)(G::kBlocksPerKU * sg.tg * 1024);
  mbar_arrive_expect_tx(bar, cbytes + G::kBlocksPerKU * sbytes + xbytes);
  const uint8_t* csrc = p.codes + (unsigned long long)sg.expert * p.codes_stride +
                        ((unsigned long long)it.ku * p.NT + tile) * Tr::kCodeBytes;
  bulk_copy_g2s(stage, csrc, cbytes, bar);
#pragma unroll
  for (int bl = 0; bl < G::kBlocksPerKU; ++bl) {
    const int col = it.ku * Tr::kKUcols + bl * 64;
    const int sb = col / p.block;
    const uint8_t* ssrc = p.scales + (unsigned long long)sg.expert * p.scales_stride +
                          ((unsigned long long)sb * p.NT + tile) * 32;
    bulk_copy_g2s(stage + G::kCodeBytes + bl * kMaxT * 32, ssrc, sbytes, bar);
  }
  const uint8_t* xsrc = p.xfrag + (unsigned long long)sg.xoff * p.K * 16 +
                        (unsigned long long)it.ku * G::kBlocksPerKU * sg.tg * 1024;
  bulk_copy_g2s(stage + G::kCodeBytes + G::kScaleBytes, xsrc, xbytes, bar);
}

__device__ __forceinline__ float silu_f(float g) { return g / (1.0f + __expf(-g)); }

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

// CTA boundaries of the unit range.
__device__ __forceinline__ long long unit_begin(long long F, int G, int c) { return F * c / G; }
__device__ __forceinline__ int cta_of_unit(long long x, long long F, int G) {
  return (int)(((x + 1) * G + F - 1) / F) - 1;
}

template <int FMT, int TG, int EPI>
__global__ void __launch_bounds__(kNW * 32, 1) qmm_small_kernel(const SmallParams p) {
  using G = StageGeom<FMT, TG>;
  using Tr = FmtTraits<FMT>;
  constexpr int BPK = G::kBlocksPerKU;
  extern __shared__ __align__(128) uint8_t smem[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int NST = p.nstages;

  uint64_t* bars = reinterpret_cast<uint64_t*>(smem);                   // [kNW][NST]
  uint32_t* lut = reinterpret_cast<uint32_t*>(smem + 1024);            // 243 entries (ternary)
  float4* red = reinterpret_cast<float4*>(smem + 2048);                 // [kNW][kMaxT][TG][32]
  uint8_t* stages = smem + 2048 + G::kRedBytes;                         // [kNW][NST][stage]
  __shared__ int s_flag[2];
  __shared__ int s_abort;

  const int nseg = *p.nseg;
  const long long F = (long long)nseg * p.NT * p.KU;
  const int Gn = gridDim.x;
  const long long f0 = unit_begin(F, Gn, blockIdx.x), f1 = unit_begin(F, Gn, blockIdx.x + 1);
  if (f0 >= f1) return;  // whole CTA idle

  if (tid == 0) s_abort = 0;
  if constexpr (FMT == 3)
    for (int i = tid; i < 243; i += blockDim.x) lut[i] = tern_lut_entry(i);
  uint64_t* wbar = bars + warp * NST;
  uint8_t* wstage = stages + (size_t)warp * NST * G::kStageBytes;
  if (lane == 0)
    for (int s = 0; s < NST; ++s) mbar_init(&wbar[s], 1);
  fence_mbar_init();
  __syncthreads();

  // Producer: lane 0 keeps NST items in flight.
  ItemIter prod;
  iter_begin(prod, f0, f1, warp, p.NT, p.KU);
  if (lane == 0) {
    for (int s = 0; s < NST && prod.valid; ++s) {
      issue_stage<FMT, TG>(p, prod, wstage + s * G::kStageBytes, &wbar[s]);
      iter_advance(prod, warp, p.NT, p.KU);
    }
  }
  __syncwarp();

  const uint32_t aconst[4] = {Tr::kConstLo, Tr::kConstLo, Tr::kConstHi, Tr::kConstHi};
  int item = 0;           // this warp's consumed items
  bool aborted = false;   // this warp gave up waiting

  SubPanel sp;
  long long pos = f0;
  const int head_tile_glob = (int)(f0 / p.KU);
  while (pos < f1) {
    load_subpanel(sp, pos, f1, p.NT, p.KU);
    Seg sg = p.segs[sp.seg];
    if (sg.tg > TG || sg.tg < 1) {
      if (tid == 0) atomicOr(p.status, kStatusBadSegment);
      sg.tg = TG;
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
        // Activation fragments of every 64-column block of the k-unit and the
        // constant-operand products that remove the code bias (shared by all tiles).
        uint32_t bfr[BPK][TG][4][2];
        float corr[BPK][TG][4];
#pragma unroll
        for (int bl = 0; bl < BPK; ++bl)
#pragma unroll
          for (int t = 0; t < TG; ++t) {
#pragma unroll
            for (int e = 0; e < 4; ++e) corr[bl][t][e] = 0.f;
            if (t == 0 || tg2) {
              const uint4* xp = reinterpret_cast<const uint4*>(xbuf + ((size_t)(bl * sg.tg + t) * 32 + lane) * 32);
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
#pragma unroll
        for (int i = 0; i < kMaxT; ++i) {
          if (i < a || i >= b) continue;
          const int li = i - a;
          uint32_t am[4 * BPK][4];   // A operand of every k-step of the k-unit for this tile
          if constexpr (FMT == 2) {
            const uint2 w = *reinterpret_cast<const uint2*>(cbuf + (size_t)li * Tr::kCodeBytes + lane * 8);
            unpack_int2_word(w.x, am[0], am[1]);
            unpack_int2_word(w.y, am[2], am[3]);
          } else if constexpr (FMT == 4) {
            const uint4 w = *reinterpret_cast<const uint4*>(cbuf + (size_t)li * Tr::kCodeBytes + lane * 16);
            unpack_int4_word(w.x, am[0]);
            unpack_int4_word(w.y, am[1]);
            unpack_int4_word(w.z, am[2]);
            unpack_int4_word(w.w, am[3]);
          } else {
            unpack_tern_record(cbuf + (size_t)li * Tr::kCodeBytes + lane * 13, lut, am);
          }
#pragma unroll
          for (int bl = 0; bl < BPK; ++bl) {
            const uint32_t sc = sbuf[bl * kMaxT * 8 + li * 8 + (lane >> 2)];
            const float s_lo = bf16_lo(sc), s_hi = bf16_hi(sc);
#pragma unroll
            for (int t = 0; t < TG; ++t) {
              if (t == 1 && !tg2) continue;
              float tmp[4] = {corr[bl][t][0], corr[bl][t][1], corr[bl][t][2], corr[bl][t][3]};
#pragma unroll
              for (int k2 = 0; k2 < 4; ++k2)
                mma_bf16_16816(tmp, am[bl * 4 + k2], bfr[bl][t][k2][0], bfr[bl][t][k2][1]);
              acc[i][t][0] = fmaf(s_lo, tmp[0], acc[i][t][0]);
              acc[i][t][1] = fmaf(s_lo, tmp[1], acc[i][t][1]);
              acc[i][t][2] = fmaf(s_hi, tmp[2], acc[i][t][2]);
              acc[i][t][3] = fmaf(s_hi, tmp[3], acc[i][t][3]);
            }
          }
        }
      }
      __syncwarp();
      if (lane == 0 && prod.valid && !aborted) {
        fence_proxy_async_smem();
        issue_stage<FMT, TG>(p, prod, st, &wbar[s]);
        iter_advance(prod, warp, p.NT, p.KU);
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
        reinterpret_cast<float4*>(p.partials)[((size_t)slot * TG + t) * 32 + ln] = v;
      }
    }
    if (head_partial || tail_partial) {
      __threadfence();
      __syncthreads();
      if (tid < 2) {
        s_flag[tid] = 0;
        const bool want = tid == 0 ? head_partial : tail_partial;
        if (want && !ab) {
          const int i = tid == 0 ? 0 : last_tile;
          const int tglob = sp.seg * p.NT + sp.rt0 + i;
          const long long T0 = (long long)tglob * p.KU;
          const int clo = cta_of_unit(T0, F, Gn), chi = cta_of_unit(T0 + p.KU - 1, F, Gn);
          int ncontrib = 0;
          for (int c = clo; c <= chi; ++c)
            if (unit_begin(F, Gn, c + 1) > unit_begin(F, Gn, c)) ++ncontrib;
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
          const long long T0 = (long long)tglob * p.KU;
          const int clo = cta_of_unit(T0, F, Gn), chi = cta_of_unit(T0 + p.KU - 1, F, Gn);
          float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
          for (int c = clo; c <= chi; ++c) {
            const long long b0 = unit_begin(F, Gn, c), b1 = unit_begin(F, Gn, c + 1);
            if (b1 <= b0) continue;
            const int slot = 2 * c + ((int)(b0 / p.KU) == tglob ? 0 : 1);
            const float4 u = __ldcg(reinterpret_cast<const float4*>(p.partials) + ((size_t)slot * TG + t) * 32 + ln);
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
    for (int s = 0; s < NST; ++s) {
      // the stage's current phase may or may not be pending; a bounded wait on
      // either parity returns as soon as the pending one completes
      mbar_wait_bounded(&wbar[s], (uint32_t)((item + s) / NST) & 1u, nullptr);
    }
  }
}

}  // namespace qmoe
