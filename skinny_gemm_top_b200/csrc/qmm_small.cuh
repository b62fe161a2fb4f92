// Small-M quantized expert matmul (the decode hot loop).
//
// For every (expert, chunk of <= 16 tokens) segment, y[rows, m] = dequant(W)
// x[m, K] with fp32 accumulation, followed by one of three epilogues: plain
// bf16 store (single linear), bias + interleaved SwiGLU into bf16 rows of h
// (FC1), bias into the fp32 expert-sorted slot rows (FC2).
//
// Design (B200):
//  * The weights are streamed from HBM once per segment: one pass over the
//    codes serves all tokens routed to the expert, the remedy the QMoE note
//    gives for the per-token GEMV relaunch ("inner loop over tokens").
//  * Work = (segment, 16-row tile, k-unit of 64 columns; 128 for ternary).
//    CTA c takes a balanced range of whole tiles, so no tile is split
//    between CTAs and every output is written once, deterministically.
//  * Inside a CTA, up to 10 consecutive tiles (kTiles) form a sub-panel; its
//    k-units go round-robin to the CTA's warps (12, or 8 for two token
//    groups).  Each warp runs its own stage ring: the codes by one bulk copy
//    (cp.async.bulk + mbarrier, no tensor map, no multicast), the scales and
//    the k-unit's slice of the segment's activation rows by 16-byte
//    cp.async.  B fragments come from those rows through ldmatrix and are
//    reused by every tile of the stage; the MMAs of all tiles of a k-step
//    issue back to back so their latencies overlap.
//  * Codes become bf16 MMA operands with LOP3 magic numbers (unpack.cuh) and
//    are multiplied on the tensor cores (mma.sync m16n8k16, tokens in N):
//    the CUDA-core budget of sm_100a cannot afford an FMA per weight per
//    token at HBM rate.  The per-block scale multiplies the fp32 partial
//    product of each 64-column block, so the dequantized weight c*s is never
//    rounded.
//  * Segment sources: a table written by an earlier routing launch, or fixed
//    chunks of the rows of a single linear.
//  * Programmatic dependent launch: the weights of the first stages are
//    requested before griddepcontrol.wait (they depend only on the routing),
//    the activations after it.
//  * The decode routing (decode_route) used by the decode layer kernel
//    (qmm_slice.cuh) and by qmoe_route lives here too.
#pragma once
#include <cfloat>
#include <climits>

#include "device_common.cuh"
#include "unpack.cuh"

namespace qmoe {

enum Epi { EPI_LINEAR = 0, EPI_SWIGLU = 1, EPI_FC2 = 2 };
enum SegSrc { SRC_TABLE = 0, SRC_LINEAR = 2 };

// Warps per CTA: 12 for one token group (three warps per SM sub-partition
// hide the unpack/MMA latency better than two), 8 for two token groups, whose
// accumulators need more than the 168 registers a 12-warp CTA leaves.
template <int TG>
constexpr int kWarps = TG == 1 ? 12 : 8;
constexpr int kMaxT = 10;         // largest sub-panel (tiles)
// Tiles per sub-panel: 10 for the INT2/INT4 decode and linear kernels (a
// decode layer's FC1 gives a CTA 9-10 tiles: one k-loop instead of 8 + 1..2;
// larger items also help the long linears), 8 otherwise (registers, and the
// larger reduction buffer would cost the general path pipeline stages).
template <int FMT, int TG, int SRC>
constexpr int kTiles = (FMT != 3 && TG == 1 && SRC != SRC_TABLE) ? 10 : 8;
constexpr int kMaxStages = 6;     // stages per consumer warp (barriers: 1024 bytes of shared memory)
constexpr int kChunkTokens = 16;  // tokens per segment (<= 2 token groups of 8)


// Decode batches, routed inside the decode layer kernel: up to 8 tokens, T*k <= 64.
constexpr int kDecMaxT = 8;
constexpr int kDecMaxTK = 64;
constexpr int kMaxExperts = 256;

// One (expert, token chunk) work item.
struct Seg {
  int expert;  // weight matrix index
  int m;       // tokens in the chunk, 1..16
  int tg;      // token groups of 8 (1 or 2)
  int slot0;   // first row of the chunk in the slot order (or first token row)
};

// Routing of a decode batch, computed in shared memory.
struct DecodeRoute {
  int nseg;                      // selected (distinct) experts
  Seg segs[kDecMaxTK];           // one per selected expert, in expert order
  int pos[kDecMaxTK];            // flat index t*k+s -> position in the expert-sorted order
  float w[kDecMaxTK];            // router weight of flat index
  int ids[kDecMaxTK];            // expert of flat index
  int hist[kMaxExperts];         // scratch: entries per expert, then their exclusive prefix
};

struct SmallParams {
  const uint8_t* codes;
  unsigned long long codes_stride;   // bytes per matrix
  const uint8_t* scales;
  unsigned long long scales_stride;  // bytes per matrix
  const uint8_t* zeros;              // affine codes: zero points (scale layout and strides), else null
  int ksplit;                        // single linear: k-unit slices per tile (1: none)
  int KUs;                           // k-units per slice (KU / ksplit)
  float* yacc;                       // ksplit > 1: fp32 output accumulator [T][N], zero at launch
  int* tickets;                      // ksplit > 1: per (token chunk, tile) slice count, zero at launch
  int NT;                            // 16-row tiles per matrix
  int K;
  int KU;                            // k-units per row
  int block;                         // scale block (64 or 128)
  int nstages;
  // segments (SRC_TABLE)
  const int* nseg;
  const Seg* segs;
  // activation rows [*, K] bf16: row of slot s is act_index[s] (or s when null)
  const uint16_t* act;
  const int* act_index;
  int T;                             // SRC_LINEAR: rows
  // epilogues
  uint16_t* y;                       // LINEAR: y[token][N]
  int N;
  const uint16_t* bias;              // SWIGLU/FC2: bias + expert * bias_rows (logical rows)
  int bias_rows;
  uint16_t* hrows;                   // SWIGLU: h[slot][I] bf16
  int I;
  float* yslot;                      // FC2: yslot[slot][H]
  int H;
  int early;                         // 1: segments and weights may be read before griddepcontrol.wait
  unsigned* status;
};

// Stage geometry for a format and token-group count.
template <int FMT, int TG, int SRC, bool AFF = false>
struct StageGeom {
  using Tr = FmtTraits<FMT>;
  static constexpr int kBlocksPerKU = Tr::kKUcols / 64;                 // 64-col blocks per k-unit
  static constexpr int kMT = kTiles<FMT, TG, SRC>;
  static constexpr int kCodeBytes = kMT * Tr::kCodeBytes;
  static constexpr int kScaleBytes = (AFF ? 2 : 1) * kBlocksPerKU * kMT * 32;  // scales (then zero points)
  static constexpr int kActPitch = Tr::kKUcols * 2 + 16;               // padded: conflict-free ldmatrix
  static constexpr int kActBytes = TG * 8 * kActPitch;
  static constexpr int kStageBytes = ((kCodeBytes + kScaleBytes + kActBytes) + 127) / 128 * 128;
  static constexpr int kNW = kWarps<TG>;
  static constexpr int kRedBytes = kNW * kMT * TG * 32 * 16;
};

template <int SRC>
struct SmemHead {
  static constexpr int kFixed = 2048;  // barriers + ternary LUT
};

// ---------------------------------------------------------------------------
// Balanced split of whole tiles over CTAs (32-bit).
struct Part {
  unsigned q, r, unit;
  __device__ __forceinline__ void init(unsigned n, unsigned G, unsigned unit_) {
    q = n / G;
    r = n - q * G;
    unit = unit_;
  }
  __device__ __forceinline__ unsigned begin(unsigned c) const { return (c * q + min(c, r)) * unit; }
};

// This CTA's unit range [f0, f1) (units = tile x k-unit, segment-major).
// With at least two CTAs per segment, every segment gets its own group of
// CTAs (sizes differ by at most one) and its tiles are split within the
// group, so no CTA straddles a segment boundary: a CTA range that did would
// run two sub-panel k-loops.  With fewer, groups of one or two CTAs would be
// unbalanced, and whole tiles are split evenly over the CTAs in
// segment-major order.
__device__ __forceinline__ void cta_range(int nseg, int NT, int KU, unsigned& f0, unsigned& f1) {
  const unsigned G = gridDim.x, c = blockIdx.x;
  if (nseg > 0 && 2u * (unsigned)nseg <= G) {
    const unsigned cps = G / (unsigned)nseg, rem = G % (unsigned)nseg;
    // segments [0, rem) have cps + 1 CTAs, the others cps
    const unsigned big = rem * (cps + 1);
    unsigned seg, j, n;
    if (c < big) {
      seg = c / (cps + 1);
      j = c - seg * (cps + 1);
      n = cps + 1;
    } else {
      seg = rem + (c - big) / cps;
      j = (c - big) - (seg - rem) * cps;
      n = cps;
    }
    const unsigned t0 = (unsigned)NT * j / n, t1 = (unsigned)NT * (j + 1) / n;
    f0 = (seg * (unsigned)NT + t0) * (unsigned)KU;
    f1 = (seg * (unsigned)NT + t1) * (unsigned)KU;
    return;
  }
  Part part;
  part.init((unsigned)nseg * (unsigned)NT, G, (unsigned)KU);
  f0 = part.begin(c);
  f1 = part.begin(c + 1);
}

// Sub-panel: up to cap_tiles consecutive whole tiles of one segment inside [pos, f1).
struct SubPanel {
  unsigned next;  // first unit after this sub-panel
  int seg, rt0, nt;
};

__device__ __forceinline__ void load_subpanel(SubPanel& sp, unsigned pos, unsigned f1, int NT, int KU, int cap_tiles) {
  const unsigned per_seg = (unsigned)NT * (unsigned)KU;
  const unsigned seg = pos / per_seg;
  const unsigned rt = (pos - seg * per_seg) / (unsigned)KU;
  const unsigned tile_base = seg * per_seg + rt * (unsigned)KU;
  unsigned end = f1;
  const unsigned seg_end = (seg + 1) * per_seg;
  if (seg_end < end) end = seg_end;
  const unsigned cap = tile_base + (unsigned)(cap_tiles * KU);
  if (cap < end) end = cap;
  sp.next = end;
  sp.seg = (int)seg;
  sp.rt0 = (int)rt;
  sp.nt = (int)((end - tile_base) / (unsigned)KU);
}

// Segments either come from a table (global or shared memory) or, for a
// single linear, are fixed chunks of kChunkTokens rows.
struct SegSource {
  const Seg* table;
  int rows;  // table == nullptr: number of rows
  __device__ __forceinline__ Seg get(int c) const {
    if (table) return table[c];
    Seg sg;
    sg.expert = 0;
    sg.m = min(kChunkTokens, rows - kChunkTokens * c);
    sg.tg = (sg.m + 7) / 8;
    sg.slot0 = kChunkTokens * c;
    return sg;
  }
};

// Warp-uniform iterator over one warp's (sub-panel, k-unit) items: in every
// sub-panel, warp w takes k-units w, w + kWarps, ...  Caches the segment and,
// per lane n < m, the row of token n.
struct ItemIter {
  SubPanel sp;
  Seg sg;
  unsigned f1;
  int ku;
  int row;     // this lane's activation row (lane < sg.m)
  int cap;     // tiles per sub-panel
  int slice;   // k-unit slice of the sub-panel (single linear split along K)
  bool valid;
};

template <int TG>
__device__ __forceinline__ void iter_load_seg(ItemIter& it, const SmallParams& p, const SegSource& segs,
                                              const int* act_index, int lane) {
  // with a K split, "segment" sp.seg = token chunk * ksplit + slice
  it.sg = segs.get(it.sp.seg / p.ksplit);
  it.slice = it.sp.seg % p.ksplit;
  if (it.sg.tg > TG || it.sg.tg < 1) it.sg.tg = TG;  // never overrun the stage (flagged by the consumer)
  if (it.sg.m > 8 * it.sg.tg) it.sg.m = 8 * it.sg.tg;
  const int s = it.sg.slot0 + (lane < it.sg.m ? lane : 0);
  it.row = act_index ? act_index[s] : s;
}

template <int TG>
__device__ __forceinline__ void iter_advance(ItemIter& it, const SmallParams& p, const SegSource& segs,
                                             const int* act_index, int warp, int lane) {
  it.ku += kWarps<TG>;
  if (it.ku < p.KUs) return;
  for (;;) {
    if (it.sp.next >= it.f1) { it.valid = false; return; }
    const int prev = it.sp.seg;
    load_subpanel(it.sp, it.sp.next, it.f1, p.NT, p.KUs, it.cap);
    if (it.sp.seg != prev) iter_load_seg<TG>(it, p, segs, act_index, lane);
    it.ku = warp;
    if (it.ku < p.KUs) return;
  }
}

template <int TG>
__device__ __forceinline__ void iter_begin(ItemIter& it, const SmallParams& p, const SegSource& segs, const int* act_index,
                                           unsigned f0, unsigned f1, int cap, int warp, int lane) {
  it.f1 = f1;
  it.cap = cap;
  it.valid = f0 < f1;
  if (!it.valid) return;
  load_subpanel(it.sp, f0, f1, p.NT, p.KUs, cap);
  iter_load_seg<TG>(it, p, segs, act_index, lane);
  it.ku = warp;
  if (it.ku >= p.KUs) {
    it.ku = p.KUs - kWarps<TG>;  // so that the advance moves to the next sub-panel
    iter_advance<TG>(it, p, segs, act_index, warp, lane);
  }
}

// Stage fills (issued by the consuming warp itself).  The codes of an item are one contiguous run
// (nt x 256..512 bytes): one TMA bulk copy by lane 0, completing as
// transaction bytes on the stage's full barrier.  Scales and activation rows
// are several pieces of 16..256 bytes: per-lane 16-byte cp.async, each lane
// arriving on the barrier once its copies landed.  Full barrier count: 33
// (lane 0's expect-tx arrival and 32 cp.async arrivals).

// Codes (TMA) and scales (cp.async) of the sub-panel's nt tiles at k-unit ku.
// KS: the matrix is packed QMOE_ROWS_KSPLIT (FC2): an INT2/INT4 k-unit of nt
// tiles is W slabs of nt x 128 bytes, copied by per-lane cp.async into
// [slab][tile][lane] order (ternary records are laid out as in PLAIN).
template <int FMT, int TG, int SRC, bool KS, bool AFF>
__device__ __forceinline__ void issue_weights(const SmallParams& p, const ItemIter& it, uint8_t* stage, uint64_t* bar,
                                              int lane) {
  using G = StageGeom<FMT, TG, SRC, AFF>;
  using Tr = FmtTraits<FMT>;
  const int tile = it.sp.rt0, n = it.sp.nt;
  const int ku = it.slice * p.KUs + it.ku;  // k-unit of the matrix
  if constexpr (KS && FMT != 3) {
    constexpr int W = FMT == 2 ? 2 : 4;
    const int per = n * 8;  // 16-byte pieces per slab
    const uint8_t* base = p.codes + (unsigned long long)it.sg.expert * p.codes_stride;
    for (int c = lane; c < W * per; c += 32) {
      const int w = c / per, j = c - w * per;
      cp_async16(stage + w * (G::kMT * 128) + 16 * j,
                 base + (((unsigned long long)ku * W + w) * p.NT + tile) * 128 + 16 * j);
    }
    if (lane == 0) mbar_arrive(bar);  // the arrival a bulk copy's expect-tx would make
  } else if (lane == 0) {
    const uint8_t* csrc = p.codes + (unsigned long long)it.sg.expert * p.codes_stride +
                          ((unsigned long long)ku * p.NT + tile) * Tr::kCodeBytes;
    const uint32_t bytes = (uint32_t)(n * Tr::kCodeBytes);
    // No proxy fence: the warp's reads of this stage were consumed by its MMAs
    // before the refill is issued.
    mbar_arrive_expect_tx(bar, bytes);
    bulk_copy_g2s(stage, csrc, bytes, bar);
  }
#pragma unroll
  for (int bl = 0; bl < G::kBlocksPerKU; ++bl) {
    const int sb = (ku * Tr::kKUcols + bl * 64) >> (p.block == 128 ? 7 : 6);  // block is 64 or 128
    const uint8_t* ssrc = p.scales + (unsigned long long)it.sg.expert * p.scales_stride +
                          ((unsigned long long)sb * p.NT + tile) * 32;
    if (lane < 2 * n) cp_async16(stage + G::kCodeBytes + bl * G::kMT * 32 + 16 * lane, ssrc + 16 * lane);
    if (AFF && lane < 2 * n)
      cp_async16(stage + G::kCodeBytes + (G::kBlocksPerKU + bl) * G::kMT * 32 + 16 * lane,
                 p.zeros + (ssrc - p.scales) + 16 * lane);
  }
}

// Activation part of a stage: the k-unit slice of each of the segment's m
// token rows (the row of token n is held by lane n of the iterator).
template <int FMT, int TG, int SRC, bool AFF>
__device__ __forceinline__ void issue_acts(const SmallParams& p, const ItemIter& it, uint8_t* stage, int lane) {
  using G = StageGeom<FMT, TG, SRC, AFF>;
  constexpr int kChunks = FmtTraits<FMT>::kKUcols * 2 / 16;  // 16-byte pieces per row slice
  const int total = it.sg.m * kChunks;
  for (int base = 0; base < total; base += 32) {
    const int c = base + lane;
    const int n = c / kChunks, j = c % kChunks;
    const int row = __shfl_sync(0xffffffffu, it.row, n < 32 ? n : 0);
    if (c < total) {
      const uint8_t* src = reinterpret_cast<const uint8_t*>(p.act) + ((unsigned long long)row * p.K) * 2 +
                           (unsigned long long)(it.slice * p.KUs + it.ku) * kChunks * 16 + 16 * j;
      cp_async16(stage + G::kCodeBytes + G::kScaleBytes + n * G::kActPitch + 16 * j, src);
    }
  }
}

__device__ __forceinline__ float silu_f(float g) { return g / (1.0f + __expf(-g)); }


__device__ __forceinline__ void ldmatrix_x4(uint32_t (&r)[4], const void* p) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(smem_addr(p)));
}

// ---------------------------------------------------------------------------
// Routing of a decode batch (T <= 8, T*k <= 64) in shared memory, identical in
// every CTA: top-k with ties to the lower index (-0 equal to +0), softmax over
// the selected logits, positions = stable sort of t*k+s by expert; one
// segment per selected expert, experts in increasing order.  Top-k routing
// and the rows expanded by expert: onnxruntime PR "Enable SM80+ FP16/BF16
// mixed INT2/INT4 QMoE prefill by default", Description.

// Order-preserving key of a logit: a larger key is a larger value; -0 and +0
// are equal; NaN is below every number.
__device__ __forceinline__ uint32_t logit_key(float v) {
  if (v != v) return 0u;
  if (v == 0.f) v = 0.f;
  const uint32_t b = __float_as_uint(v);
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

// The logit of a key (inverse of logit_key up to the sign of zero; NaN stays NaN).
__device__ __forceinline__ float logit_of_key(uint32_t key) {
  return __uint_as_float((key & 0x80000000u) ? (key & 0x7FFFFFFFu) : ~key);
}

// Routing in warp-level steps, every one a register, shuffle or
// shared-memory operation, so that the dependency chain stays short:
//  1. warp t < T: k rounds of a warp arg-max over token t's logits; lane s
//     keeps selection s; softmax over the selected logits in selection order.
//  2. T = 1 (warp 0 goes on without a CTA barrier): the k experts are
//     distinct; the position and the segment of selection s are the rank of
//     its expert among them.
//     T > 1 (warp 0, after a CTA barrier): per expert, the mask of the tokens
//     that selected it (shared-memory atomic OR: the same result in every CTA
//     whatever the order); an entry's rank within its expert is the count of
//     earlier tokens in the mask; a warp scan over the experts gives each
//     entry the entries at lower experts (its position base) and its
//     expert's rank among the selected ones (its segment).
// V = experts per lane (E <= 32 V); decode_route picks the smallest.
// Needs blockDim.x >= 32 T; ends with a CTA barrier.
// Barrier of the threads that route: the whole CTA (NB == 0), else the first
// NB threads on named barrier 1.
template <int NB>
__device__ __forceinline__ void route_sync() {
  if constexpr (NB == 0) __syncthreads();
  else asm volatile("bar.sync 1, %0;" ::"n"(NB) : "memory");
}

template <int V, int NB>
__device__ __noinline__ void decode_route_v(const float* logits, int T, int E, int k, DecodeRoute& R) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int TK = T * k;
  if (warp < T) {
    uint32_t key[V];  // lane holds experts lane + 32j
    unsigned live = 0;
#pragma unroll
    for (int j = 0; j < V; ++j) {
      const int idx = lane + 32 * j;
      key[j] = idx < E ? logit_key(logits[(size_t)warp * E + idx]) : 0u;
      if (idx < E) live |= 1u << j;
    }
    int my_id = 0;
    float my_v = 0.f;
    for (int s = 0; s < k; ++s) {  // (key desc, index asc)
      uint32_t bk = 0;
      int bj = -1;
#pragma unroll
      for (int j = 0; j < V; ++j)
        if (((live >> j) & 1u) && (bj < 0 || key[j] > bk)) { bk = key[j]; bj = j; }
      const uint32_t mk = __reduce_max_sync(0xffffffffu, bj >= 0 ? bk : 0u);
      const int win = __reduce_min_sync(0xffffffffu, (bj >= 0 && bk == mk) ? lane + 32 * bj : INT_MAX);
      if ((win & 31) == lane) live &= ~(1u << (win >> 5));
      if (lane == s) {
        my_id = win;
        my_v = logit_of_key(mk);
      }
    }
    const float ex = expf(my_v - __shfl_sync(0xffffffffu, my_v, 0));
    float sum = 0.f;
    for (int s = 0; s < k; ++s) sum += __shfl_sync(0xffffffffu, ex, s);
    if (lane < k) {
      R.ids[warp * k + lane] = my_id;
      R.w[warp * k + lane] = ex / sum;
    }
    if (T == 1) {
      int rank = 0;
      for (int j = 0; j < k; ++j) rank += __shfl_sync(0xffffffffu, my_id, j) < my_id;
      if (lane < k) {
        R.pos[lane] = rank;
        Seg sg;
        sg.expert = my_id;
        sg.m = 1;
        sg.tg = 1;
        sg.slot0 = rank;
        R.segs[rank] = sg;
      }
      if (lane == 0) R.nseg = k;
    }
  }
  if (T > 1) {
    route_sync<NB>();
    if (warp == 0) {
      int* hist = R.hist;  // per expert: the mask of the tokens that selected it
      const int nb = (E + 31) / 32;  // experts per lane in the scan
      for (int b = lane; b < E; b += 32) hist[b] = 0;
      __syncwarp();
      const int i0 = lane, i1 = lane + 32;
      const int e0 = i0 < TK ? R.ids[i0] : -1, e1 = i1 < TK ? R.ids[i1] : -1;
      const int t0 = i0 / k, t1 = i1 / k;
      if (e0 >= 0) atomicOr(&hist[e0], 1 << t0);
      if (e1 >= 0) atomicOr(&hist[e1], 1 << t1);
      __syncwarp();
      const int mk0 = e0 >= 0 ? hist[e0] : 0, mk1 = e1 >= 0 ? hist[e1] : 0;
      const int before0 = __popc(mk0 & ((1 << t0) - 1)), before1 = __popc(mk1 & ((1 << t1) - 1));
      const int cnt0 = __popc(mk0), cnt1 = __popc(mk1);
      int loc[V];
      int run = 0;  // (entries) | (selected experts) << 16 over this lane's experts
#pragma unroll
      for (int q = 0; q < V; ++q) {
        const int b = lane * nb + q;
        loc[q] = (q < nb && b < E) ? __popc(hist[b]) : 0;
        run += loc[q] | ((loc[q] > 0) << 16);
      }
      __syncwarp();
      int inc = run;
#pragma unroll
      for (int d = 1; d < 32; d <<= 1) {
        const int u = __shfl_up_sync(0xffffffffu, inc, d);
        if (lane >= d) inc += u;
      }
      __syncwarp();
      int ex = inc - run;
#pragma unroll
      for (int q = 0; q < V; ++q) {
        const int b = lane * nb + q;
        if (q < nb && b < E) hist[b] = ex;
        ex += loc[q] | ((loc[q] > 0) << 16);
      }
      __syncwarp();
      const int is[2] = {i0, i1}, es[2] = {e0, e1}, bs[2] = {before0, before1}, cs[2] = {cnt0, cnt1};
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        if (is[h] >= TK) continue;
        const int pre = hist[es[h]], less = pre & 0xFFFF;
        R.pos[is[h]] = less + bs[h];
        if (bs[h] == 0) {
          Seg sg;
          sg.expert = es[h];
          sg.m = cs[h];
          sg.tg = (sg.m + 7) / 8;
          sg.slot0 = less;
          R.segs[pre >> 16] = sg;
        }
      }
      const int nsel = __shfl_sync(0xffffffffu, inc, 31) >> 16;
      if (lane == 0) R.nseg = nsel;
    }
  }
  route_sync<NB>();
}

// (A lane holding 8 experts where 2 would do made the routing of a 64-expert
// layer about 1.5k cycles slower: measured in isolation.)
template <int NB = 0>
__device__ __forceinline__ void decode_route(const float* logits, int T, int E, int k, DecodeRoute& R) {
  if (E <= 64) decode_route_v<2, NB>(logits, T, E, k, R);
  else if (E <= 128) decode_route_v<4, NB>(logits, T, E, k, R);
  else decode_route_v<8, NB>(logits, T, E, k, R);
}

// Epilogue of one reduced fragment: rows g / g+8 of tile rt, tokens n0, n0+1.
template <int EPI>
__device__ __forceinline__ void epilogue(const SmallParams& p, const Seg& sg, int rt, int tg, int lane, float4 v) {
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
    if (n0 < sg.m)
      p.hrows[(size_t)(sg.slot0 + n0) * p.I + j] =
          __bfloat16_as_ushort(__float2bfloat16_rn(silu_f(v.x + bg) * (v.z + bu)));
    if (n0 + 1 < sg.m)
      p.hrows[(size_t)(sg.slot0 + n0 + 1) * p.I + j] =
          __bfloat16_as_ushort(__float2bfloat16_rn(silu_f(v.y + bg) * (v.w + bu)));
  }
}

// ---------------------------------------------------------------------------
// One item: tiles [0, NTL) of a stage (NTL = a power of two >= nt).  Tiles
// at or past nt contribute with scale 0 (their codes are stale but finite),
// so all NTL tiles run the same straight-line code and the MMAs of a k-step
// for every tile issue back to back.
template <int FMT, int TG, int SRC, bool KS, int NTL, bool AFF>
__device__ __forceinline__ void compute_item(const uint8_t* st, bool tg2, int lane, int nt, const uint32_t* lut,
                                             float (&acc)[kTiles<FMT, TG, SRC>][TG][4]) {
  using Tr = FmtTraits<FMT>;
  using G = StageGeom<FMT, TG, SRC, AFF>;
  constexpr int BPK = Tr::kKUcols / 64;
  const uint8_t* cbuf = st;
  const uint32_t* sbuf = reinterpret_cast<const uint32_t*>(st + G::kCodeBytes);
  const uint8_t* abuf = st + G::kCodeBytes + G::kScaleBytes;
  // affine codes: the stored field is u, so the constant operand is -128 in
  // both column classes, and each block adds z * (sum of its activations)
  const uint32_t aconst[4] = {AFF ? kAffConst : Tr::kConstLo, AFF ? kAffConst : Tr::kConstLo,
                              AFF ? kAffConst : Tr::kConstHi, AFF ? kAffConst : Tr::kConstHi};
  const int g = lane >> 2;
  // B fragments from the token rows (ldmatrix: lanes 8j..8j+7 address the
  // rows of matrix j = columns 8j..8j+7 of a 32-column half), columns
  // k%16 >= 8 divided by the code multiplier, and the constant-operand products.
  uint32_t bfr[BPK][TG][4][2];
  float corr[BPK][TG][4];
  float sx[TG][4];  // affine codes (INT2 / INT4: one block per k-unit): sum of the activations
#pragma unroll
  for (int t = 0; t < TG; ++t) sx[t][0] = sx[t][1] = sx[t][2] = sx[t][3] = 0.f;
#pragma unroll
  for (int bl = 0; bl < BPK; ++bl)
#pragma unroll
    for (int t = 0; t < TG; ++t) {
#pragma unroll
      for (int e = 0; e < 4; ++e) corr[bl][t][e] = 0.f;
      if (t == 0 || tg2) {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          uint32_t r[4];
          ldmatrix_x4(r, abuf + (t * 8 + (lane & 7)) * G::kActPitch + (bl * 64 + h * 32 + (lane >> 3) * 8) * 2);
          bfr[bl][t][2 * h][0] = r[0];
          bfr[bl][t][2 * h][1] = r[1];
          bfr[bl][t][2 * h + 1][0] = r[2];
          bfr[bl][t][2 * h + 1][1] = r[3];
        }
        if (Tr::kBetaHi == 4) {
#pragma unroll
          for (int k2 = 0; k2 < 4; ++k2) bfr[bl][t][k2][1] = fma_bf16x2(bfr[bl][t][k2][1], kBf16Quarter, 0x80008000u);
        }
#pragma unroll
        for (int k2 = 0; k2 < 4; ++k2) mma_bf16_16816(corr[bl][t], aconst, bfr[bl][t][k2][0], bfr[bl][t][k2][1]);
        if constexpr (AFF) {
          const uint32_t asum[4] = {kBf16One, kBf16One, sum_const_hi<FMT>(), sum_const_hi<FMT>()};
#pragma unroll
          for (int e = 0; e < 4; ++e) sx[t][e] = 0.f;
#pragma unroll
          for (int k2 = 0; k2 < 4; ++k2) mma_bf16_16816(sx[t], asum, bfr[bl][t][k2][0], bfr[bl][t][k2][1]);
        }
      } else {
#pragma unroll
        for (int k2 = 0; k2 < 4; ++k2) bfr[bl][t][k2][0] = bfr[bl][t][k2][1] = 0u;
      }
    }
  // per-tile scales (0 at or past nt)
  float s_lo[BPK][NTL], s_hi[BPK][NTL];
#pragma unroll
  for (int bl = 0; bl < BPK; ++bl)
#pragma unroll
    for (int i = 0; i < NTL; ++i) {
      const uint32_t sc = sbuf[bl * G::kMT * 8 + i * 8 + g];
      const bool on = i < nt;
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
      if constexpr (KS) {  // [slab][tile][lane]
#pragma unroll
        for (int w = 0; w < W; ++w)
          wd[i][w] = *reinterpret_cast<const uint32_t*>(cbuf + w * (G::kMT * 128) + i * 128 + lane * 4);
      } else if constexpr (FMT == 2) {
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
    if constexpr (AFF) {
      const uint32_t* zbuf = sbuf + G::kBlocksPerKU * G::kMT * 8;
#pragma unroll
      for (int i = 0; i < NTL; ++i) {
        const uint32_t zc = zbuf[i * 8 + g];
        const bool on = i < nt;
        const float zlo = on ? bf16_lo(zc) : 0.f, zhi = on ? bf16_hi(zc) : 0.f;
#pragma unroll
        for (int t = 0; t < TG; ++t) {
          acc[i][t][0] = fmaf(zlo, sx[t][0], acc[i][t][0]);
          acc[i][t][1] = fmaf(zlo, sx[t][1], acc[i][t][1]);
          acc[i][t][2] = fmaf(zhi, sx[t][2], acc[i][t][2]);
          acc[i][t][3] = fmaf(zhi, sx[t][3], acc[i][t][3]);
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

// ---------------------------------------------------------------------------
// One matmul phase of a small-M kernel on the warps' stage rings.  The rings
// (barriers, stage buffers, item counters) are kept in a context that could
// persist across phases of one kernel.
// Single linear split along K: this CTA's fp32 partial of one reduced
// fragment (rows g / g+8 of tile rt, tokens n0, n0+1) added to the output
// accumulator.
__device__ __forceinline__ void linear_partial(const SmallParams& p, const Seg& sg, int rt, int tg, int lane, float4 v) {
  const int g = lane >> 2, q = lane & 3;
  const int n0 = tg * 8 + 2 * q;
  const int r0 = rt * 16 + g, r1 = r0 + 8;
  if (n0 < sg.m) {
    float* yr = p.yacc + (size_t)(sg.slot0 + n0) * p.N;
    atomicAdd(yr + r0, v.x);
    atomicAdd(yr + r1, v.z);
  }
  if (n0 + 1 < sg.m) {
    float* yr = p.yacc + (size_t)(sg.slot0 + n0 + 1) * p.N;
    atomicAdd(yr + r0, v.y);
    atomicAdd(yr + r1, v.w);
  }
}

// After a sub-panel's partials: one ticket per tile; the CTA that adds a
// tile's last slice rounds its rows to bf16.  Ends with a CTA barrier.
__device__ __forceinline__ void linear_tickets(const SmallParams& p, const Seg& sg, int chunk, int rt0, int nt,
                                               bool aborted, int* s_last) {
  const int tid = threadIdx.x;
  if (tid < nt) {
    const int old = atomic_add_acq_rel_gpu(p.tickets + chunk * p.NT + rt0 + tid, 1);
    s_last[tid] = (old == p.ksplit - 1 && !aborted) ? 1 : 0;
  }
  __syncthreads();
  for (int e = tid; e < nt * 16 * sg.m; e += blockDim.x) {
    const int i = e / (16 * sg.m), rem = e - i * 16 * sg.m, n = rem / 16, r = rem % 16;
    if (!s_last[i]) continue;
    const size_t o = (size_t)(sg.slot0 + n) * p.N + (rt0 + i) * 16 + r;
    const float v = *reinterpret_cast<volatile const float*>(p.yacc + o);
    p.y[o] = __bfloat16_as_ushort(__float2bfloat16_rn(v));
  }
  __syncthreads();
}

struct PhaseCtx {
  uint64_t* wfull;  // this warp's full barriers [NST]
  uint8_t* wstage;  // this warp's first stage
  int stride;       // bytes per stage
  int NST;
  int item;         // this warp's consumed items
  int stage;        // item % NST
  uint32_t phase;   // (item / NST) & 1
  int issued;       // this warp's issued items
  int fail_at;      // first item whose wait gave up
  bool aborted;     // this warp gave up waiting
  float4* red;
  const uint32_t* lut;
  int* s_abort;
  int* s_last;     // [kMT] tiles whose last K slice this CTA added (single linear split along K)
};

// Partition, prime (weights, then hook(), then activation rows), stream the
// items, reduce and run the epilogue.  hook() is called by every thread of
// the CTA exactly once (also by CTAs without work): the dependency wait.
template <int FMT, int TG, int EPI, int SRC, bool AFF, class Hook>
__device__ __forceinline__ void run_phase(const SmallParams& p, const SegSource& segs, int nseg, const int* act_index,
                                          PhaseCtx& cx, Hook&& hook) {
  using G = StageGeom<FMT, TG, SRC, AFF>;
  constexpr int kNW = kWarps<TG>;
  constexpr int kCT = kNW * 32;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int NST = cx.NST;

  unsigned f0, f1;
  cta_range(nseg * p.ksplit, p.NT, p.KUs, f0, f1);
  if (f0 >= f1) {  // whole CTA idle in this phase
    hook();
    return;
  }

  // Every warp fills its own ring: the weights of its next NST items before
  // hook(), their activation rows after it.
  ItemIter prod;
  int primed = 0;
  iter_begin<TG>(prod, p, segs, act_index, f0, f1, G::kMT, warp, lane);
  {
    ItemIter it = prod;
    for (int i = 0; i < NST && it.valid && !cx.aborted; ++i, ++primed) {  // (a warp that gave up issues nothing)
      const int s = (cx.issued + i) % NST;
      issue_weights<FMT, TG, SRC, EPI == EPI_FC2, AFF>(p, it, cx.wstage + s * cx.stride, &cx.wfull[s], lane);
      iter_advance<TG>(it, p, segs, act_index, warp, lane);
    }
  }
  hook();
  __syncwarp();
  for (int i = 0; i < primed; ++i) {
    const int s = (cx.issued + i) % NST;
    issue_acts<FMT, TG, SRC, AFF>(p, prod, cx.wstage + s * cx.stride, lane);
    cp_async_arrive(&cx.wfull[s]);
    iter_advance<TG>(prod, p, segs, act_index, warp, lane);
  }
  cx.issued += primed;

  SubPanel sp;
  unsigned pos = f0;
  int cur_seg = -1;
  Seg sg;
  while (pos < f1) {
    load_subpanel(sp, pos, f1, p.NT, p.KUs, G::kMT);
    if (sp.seg != cur_seg) {
      cur_seg = sp.seg;
      sg = segs.get(sp.seg / p.ksplit);
      if (sg.tg > TG || sg.tg < 1 || sg.m > 8 * sg.tg) {
        if (tid == 0) atomicOr(p.status, kStatusBadSegment);
        sg.tg = TG;
        sg.m = min(sg.m, 8 * TG);
      }
    }
    const bool tg2 = TG == 2 && sg.tg == 2;
    float acc[G::kMT][TG][4];
#pragma unroll
    for (int i = 0; i < G::kMT; ++i)
#pragma unroll
      for (int t = 0; t < TG; ++t)
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[i][t][e] = 0.f;

    for (int ku = warp; ku < p.KUs; ku += kNW) {
      const int s = cx.stage;
      const uint32_t par = cx.phase;
      ++cx.item;
      if (++cx.stage == NST) {
        cx.stage = 0;
        cx.phase ^= 1u;
      }
      if (!cx.aborted && __any_sync(0xffffffffu, !mbar_wait_bounded(&cx.wfull[s], par, p.status))) {
        cx.aborted = true;
        cx.fail_at = cx.item - 1;
        *cx.s_abort = 1;
      }
      if (!cx.aborted) {
        const uint8_t* st = cx.wstage + s * cx.stride;
        if (G::kMT > 8 && sp.nt > 8) compute_item<FMT, TG, SRC, EPI == EPI_FC2, G::kMT, AFF>(st, tg2, lane, sp.nt, cx.lut, acc);
        else if (sp.nt > 4) compute_item<FMT, TG, SRC, EPI == EPI_FC2, 8, AFF>(st, tg2, lane, sp.nt, cx.lut, acc);
        else if (sp.nt > 2) compute_item<FMT, TG, SRC, EPI == EPI_FC2, 4, AFF>(st, tg2, lane, sp.nt, cx.lut, acc);
        else if (sp.nt > 1) compute_item<FMT, TG, SRC, EPI == EPI_FC2, 2, AFF>(st, tg2, lane, sp.nt, cx.lut, acc);
        else compute_item<FMT, TG, SRC, EPI == EPI_FC2, 1, AFF>(st, tg2, lane, sp.nt, cx.lut, acc);
      }
      __syncwarp();
      if (prod.valid && !cx.aborted) {
        uint8_t* st = cx.wstage + s * cx.stride;
        issue_weights<FMT, TG, SRC, EPI == EPI_FC2, AFF>(p, prod, st, &cx.wfull[s], lane);
        issue_acts<FMT, TG, SRC, AFF>(p, prod, st, lane);
        cp_async_arrive(&cx.wfull[s]);
        ++cx.issued;
        iter_advance<TG>(prod, p, segs, act_index, warp, lane);
      }
      __syncwarp();
    }

    // ---- CTA reduction of the sub-panel, epilogue ----------------------------
    float4* red = cx.red;
#pragma unroll
    for (int i = 0; i < G::kMT; ++i) {
      if (i >= sp.nt) continue;
#pragma unroll
      for (int t = 0; t < TG; ++t)
        red[((warp * G::kMT + i) * TG + t) * 32 + lane] =
            make_float4(acc[i][t][0], acc[i][t][1], acc[i][t][2], acc[i][t][3]);
    }
    __syncthreads();
    const bool ab = *cx.s_abort != 0;
    const int nel = sp.nt * TG * 32;
#pragma unroll
    for (int r = 0; r < (G::kMT * TG * 32 + kCT - 1) / kCT; ++r) {
      const int e = tid + r * kCT;
      if (e >= nel || ab) continue;
      float4 v = red[e];
      for (int w = 1; w < kNW; ++w) {
        const float4 u = red[w * G::kMT * TG * 32 + e];
        v.x += u.x; v.y += u.y; v.z += u.z; v.w += u.w;
      }
      const int i = e / (TG * 32), t = (e / 32) % TG, ln = e % 32;
      if (t == 1 && !tg2) continue;
      if (EPI == EPI_LINEAR && p.ksplit > 1) linear_partial(p, sg, sp.rt0 + i, t, ln, v);
      else epilogue<EPI>(p, sg, sp.rt0 + i, t, ln, v);
    }
    __syncthreads();
    if (EPI == EPI_LINEAR && p.ksplit > 1) linear_tickets(p, sg, sp.seg / p.ksplit, sp.rt0, sp.nt, ab, cx.s_last);
    pos = sp.next;
  }
}

// Drain: if this warp gave up waiting, let its copies in flight land.
__device__ __forceinline__ void drain_ring(const PhaseCtx& cx, int lane) {
  if (!cx.aborted) return;
  cp_async_wait_all();
  if (lane == 0)
    for (int j = cx.fail_at; j < cx.issued; ++j)  // issued, unconsumed items: their bulk copies (bounded)
      mbar_wait_bounded(&cx.wfull[j % cx.NST], (uint32_t)(j / cx.NST) & 1u, nullptr);
}

// Shared-memory layout of a small-M kernel and the rings' context.
template <int FMT, int TG, int SRC, bool AFF>
struct SmallSmem {
  uint64_t* bars;  // [kNW][NST] full barriers
  uint32_t* lut;   // 243 entries (ternary)
  float4* red;     // [kNW][kMT][TG][32]
  uint8_t* stages; // [kNW][NST][stage]
  __device__ __forceinline__ explicit SmallSmem(uint8_t* smem) {
    bars = reinterpret_cast<uint64_t*>(smem);
    lut = reinterpret_cast<uint32_t*>(smem + 1024);
    red = reinterpret_cast<float4*>(smem + SmemHead<SRC>::kFixed);
    stages = smem + SmemHead<SRC>::kFixed + StageGeom<FMT, TG, SRC, AFF>::kRedBytes;
  }
};

// Ternary table, ring barriers and the phase context (ends with a CTA barrier).
template <int FMT, int TG, int SRC, bool AFF>
__device__ __forceinline__ void init_rings(const SmallSmem<FMT, TG, SRC, AFF>& sm, int NST, int* s_abort,
                                           PhaseCtx& cx) {
  using G = StageGeom<FMT, TG, SRC, AFF>;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) *s_abort = 0;
  if constexpr (FMT == 3)
    for (int i = tid; i < 243; i += blockDim.x) sm.lut[i] = tern_lut_entry(i);
  cx = PhaseCtx{};
  cx.wfull = sm.bars + warp * NST;
  cx.wstage = sm.stages + (size_t)warp * NST * G::kStageBytes;
  cx.stride = G::kStageBytes;
  cx.NST = NST;
  cx.red = sm.red;
  cx.lut = sm.lut;
  cx.s_abort = s_abort;
  if (lane == 0)
    for (int s = 0; s < NST; ++s) mbar_init(&cx.wfull[s], 33);
  fence_mbar_init();
  __syncthreads();
}

template <int FMT, int TG, int EPI, int SRC, bool AFF>
__global__ void __launch_bounds__(kWarps<TG> * 32, 1) qmm_small_kernel(const SmallParams p) {
  extern __shared__ __align__(128) uint8_t smem[];
  const int lane = threadIdx.x & 31;
  const SmallSmem<FMT, TG, SRC, AFF> sm(smem);
  __shared__ int s_abort;
  __shared__ int s_last[kTiles<FMT, TG, SRC>];

  // ---- segments ----
  // With p.early the segment source was written at least two launches back
  // (or is arithmetic), so segments and weights may be read before
  // griddepcontrol.wait; otherwise wait first.
  if (!p.early) pdl_wait();
  int nseg;
  SegSource segs;
  segs.table = nullptr;
  segs.rows = p.T;
  if constexpr (SRC == SRC_LINEAR) {
    nseg = (p.T + kChunkTokens - 1) / kChunkTokens;
  } else {
    nseg = *p.nseg;
    segs.table = p.segs;
  }

  PhaseCtx cx;
  init_rings<FMT, TG, SRC, AFF>(sm, p.nstages, &s_abort, cx);
  cx.s_last = s_last;

  run_phase<FMT, TG, EPI, SRC, AFF>(p, segs, nseg, p.act_index, cx, [&] {
    pdl_wait();
    pdl_trigger();
  });
  drain_ring(cx, lane);
}

}  // namespace qmoe
