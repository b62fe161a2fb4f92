// Internal: host-visible parameters of the decode layer kernel split along the
// expert intermediate dimension (qmm_slice.cuh), and its launcher
// (qmoe_slice.cu).
#pragma once
#include <cstddef>
#include <cstdint>

#include <cuda_runtime.h>

namespace qmoe {

constexpr int kSW = 12;                  // warps per CTA
constexpr int kSChunk = 10;              // FC1 tiles per chunk at most (one cross-warp reduction each)
constexpr int kSRed = 5;                 // FC1 tiles per reduction round
constexpr int kSRT = 11;                 // FC2 row tiles per warp at most
constexpr int kSMaxH = kSW * kSRT * 16;  // 2112: largest H
constexpr int kSMaxChunks = 48;          // chunks per CTA
constexpr int kSNB = 12;                 // items in flight per warp (one barrier each)
constexpr int kSHWin = 8;                // k-steps of h held at once (one ternary granule)

// A chunk: nt FC1 tiles of one expert, starting at tile etile0 of its
// QMOE_ROWS_GATE_UP matrix (8 h columns per tile); its h columns occupy the
// h window from tile hoff on.  After its FC1 it completes ngc FC2 granules of
// the expert, g0 the first.
struct SChunk {
  int expert;  // matrix index (shared experts after the routed ones)
  int wsel;    // rank of the expert among the selected ones; -1: shared expert
  int etile0, nt;
  int g0, ngc;
  int hoff;
  int pad;
};

// Whether a launch of G CTAs over nslots experts of gpe granules each gives
// every expert its own group of CTAs (at least two, and at most 1/8 more
// granules on the busiest CTA than an even split of the granule list).
__host__ __device__ inline bool slice_grouped(int G, int nslots, int gpe) {
  if (nslots < 1 || 2 * nslots > G) return false;
  const int cps = G / nslots;
  const long long grp = (gpe + cps - 1) / cps, even = ((long long)nslots * gpe + G - 1) / G;
  return 8 * grp <= 9 * even;
}

struct SliceParams {
  const uint8_t* c1;  // FC1 codes, QMOE_ROWS_GATE_UP
  unsigned long long c1_stride;
  const uint8_t* s1;
  unsigned long long s1_stride;
  const uint16_t* b1;  // [E + n_shared][2I] or null
  const uint8_t* c2;   // FC2 codes, QMOE_ROWS_KSPLIT
  unsigned long long c2_stride;
  const uint8_t* s2;
  unsigned long long s2_stride;
  const uint16_t* b2;    // [E + n_shared][H] or null
  const uint8_t* z1;     // affine codes: FC1 / FC2 zero points (scale layout and strides), else null
  const uint8_t* z2;
  int aff;               // 1: affine codes (INT2 / INT4)
  int NT1, KU1, block1;  // FC1: 16-row tiles, k-units along H, scale block
  int NT2, block2;       // FC2: 16-row tiles (H / 16), scale block
  int H, I, E, k, n_shared, T;
  int gpe;          // FC2 granules per expert (I / granule columns)
  int ring_bytes;   // per-warp ring of item buffers
  int ngm;          // FC2 granules per item at most
  int xrows;        // rows of x held in shared memory (T, plus a zero row when T < 8)
  const uint16_t* x;    // [T][H] bf16
  const float* logits;  // [T][E]
  uint16_t* y;          // [T][H] bf16
  float* yacc;          // [T][H] fp32, zero at launch
  int* ticket;          // [0]: CTAs done, [1]: CTAs that gave up a wait; zero at launch
  unsigned* status;
  unsigned long long wait_ns;  // limit of every wait in the kernel
  int inject;                  // fault injection (tests): 1 = one wait on a barrier nothing arrives at
};

// Geometry of one launch: ring stages and shared memory for (FC1 format,
// FC2 format, T, H); ok == false when it does not fit.
struct SlicePlan {
  bool ok;
  int ring_bytes, ngm, xrows, gran_cols;
  size_t smem;
};
SlicePlan slice_plan(int f1, int f2, int T, int H, bool aff);

// Upper bound of the chunks one CTA can get, over every count of selected
// experts up to max_routed (host check against kSMaxChunks).
int slice_max_chunks(int f2, int gpe, int n_shared, int max_routed, int grid);

// Launch qmm_slice_kernel<f1, f2> / slice_reset_kernel on st with
// programmatic dependent launch; the reset launch goes first.
cudaError_t slice_launch(int f1, int f2, const SliceParams& p, int grid, size_t smem, cudaStream_t st);
cudaError_t slice_reset_launch(float* yacc, int n4, int* ticket, cudaStream_t st);

}  // namespace qmoe
