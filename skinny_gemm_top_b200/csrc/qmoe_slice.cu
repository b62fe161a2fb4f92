// Instantiations and launcher of the decode layer kernel split along the
// expert intermediate dimension (qmm_slice.cuh).  Its own translation unit:
// the kernel takes the device status word as a parameter.
#include <algorithm>

#include "qmm_slice.cuh"
#include "slice.h"

namespace qmoe {

namespace {

constexpr int kSmemLimit = 227 * 1024;

int fc1_code_bytes(int f) { return f == 2 ? 256 : f == 4 ? 512 : 416; }  // per tile and k-unit
int fc1_blocks_per_ku(int f) { return f == 3 ? 2 : 1; }
int fc2_row_bytes(int f) { return f == 3 ? 416 : 128; }                  // per row tile and granule
int fc2_blocks(int) { return 1; }                                        // scale rows per granule
int fc2_cols(int f) { return f == 4 ? 16 : f == 2 ? 32 : 64; }          // granule width (h columns)
int round128(int v) { return (v + 127) / 128 * 128; }
int chunk_tiles(int f2) { return f2 == 4 ? 10 : 8; }                    // SChunkGeom<f2>::kMT

template <int F1, int F2, bool AFF>
cudaError_t launch_t(const SliceParams& p, int grid, size_t smem, cudaStream_t st) {
  static bool attr_set[64] = {};
  int d = 0;
  cudaGetDevice(&d);
  if (d < 0 || d >= 64) return cudaErrorInvalidDevice;
  if (!attr_set[d]) {
    const cudaError_t e =
        cudaFuncSetAttribute(qmm_slice_kernel<F1, F2, AFF>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemLimit);
    if (e != cudaSuccess) return e;
    attr_set[d] = true;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kSThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, qmm_slice_kernel<F1, F2, AFF>, p);
}

}  // namespace

SlicePlan slice_plan(int f1, int f2, int T, int H, bool aff) {
  SlicePlan pl{};
  pl.ok = false;
  if (T < 1 || T > 8 || H > kSMaxH || H % 64) return pl;
  const int zb = aff ? 2 : 1;  // scale (and zero point) bytes per 16 rows and block
  const int fc1_item = chunk_tiles(f2) * (fc1_code_bytes(f1) + zb * fc1_blocks_per_ku(f1) * 32);
  const int nr_max = (H / 16 + kSW - 1) / kSW;
  const int per_granule = nr_max * (fc2_row_bytes(f2) + zb * fc2_blocks(f2) * 32);
  pl.ngm = std::max(1, std::min(3, 4096 / per_granule));  // FC2 items of about 4 KB
  pl.xrows = T < 8 ? T + 1 : 8;
  pl.gran_cols = fc2_cols(f2);
  const int fixed = SliceSmemLayout::kFixed + round128(pl.xrows * (2 * H + 16));
  pl.ring_bytes = (kSmemLimit - fixed) / kSW / 128 * 128;
  const int item = std::max(fc1_item, pl.ngm * per_granule);
  if (pl.ring_bytes < 2 * item || (size_t)kSW * pl.ring_bytes < (size_t)T * H * 4) return pl;
  pl.smem = (size_t)fixed + (size_t)kSW * pl.ring_bytes;
  pl.ok = true;
  return pl;
}

int slice_max_chunks(int f2, int gpe, int n_shared, int max_routed, int grid) {
  if (gpe < 1 || grid < 1) return 0;
  const int tpg = fc2_cols(f2) / 8;  // FC1 tiles per granule
  const int gmax = std::max(1, chunk_tiles(f2) / tpg);
  long long worst = 0;
  for (int nsel = 1; nsel <= std::max(1, max_routed); ++nsel) {
    const int nslots = n_shared + nsel;
    long long len, pieces;
    if (slice_grouped(grid, nslots, gpe)) {
      len = (gpe + grid / nslots - 1) / (grid / nslots);
      pieces = 1;
    } else {
      len = ((long long)nslots * gpe + grid - 1) / grid;
      pieces = (len + gpe - 1) / gpe + 1;
    }
    const long long n = tpg > chunk_tiles(f2) ? len * (tpg / 8) : (len + gmax - 1) / gmax + pieces;
    worst = std::max(worst, n);
  }
  return (int)std::min<long long>(worst, 1 << 20);
}

cudaError_t slice_launch(int f1, int f2, const SliceParams& p, int grid, size_t smem, cudaStream_t st) {
#define QMOE_SLICE_CASE(A, B) \
  if (f1 == A && f2 == B) return p.aff ? launch_t<A, B, true>(p, grid, smem, st) : launch_t<A, B, false>(p, grid, smem, st);
#define QMOE_SLICE_CASE_SYM(A, B) \
  if (f1 == A && f2 == B) return p.aff ? cudaErrorInvalidValue : launch_t<A, B, false>(p, grid, smem, st);
  QMOE_SLICE_CASE(2, 2)
  QMOE_SLICE_CASE(2, 4)
  QMOE_SLICE_CASE_SYM(2, 3)
  QMOE_SLICE_CASE(4, 2)
  QMOE_SLICE_CASE(4, 4)
  QMOE_SLICE_CASE_SYM(4, 3)
  QMOE_SLICE_CASE_SYM(3, 2)
  QMOE_SLICE_CASE_SYM(3, 4)
  QMOE_SLICE_CASE_SYM(3, 3)
#undef QMOE_SLICE_CASE
#undef QMOE_SLICE_CASE_SYM
  return cudaErrorInvalidValue;
}

cudaError_t slice_reset_launch(float* yacc, int n4, int* ticket, cudaStream_t st) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(std::max(1, std::min(8, (n4 + 1023) / 1024)));
  cfg.blockDim = dim3(256);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, slice_reset_kernel, yacc, n4, ticket);
}

}  // namespace qmoe
