// C ABI of the device entry points: qmoe_route, qmoe_forward, qmoe_linear,
// qmoe_dequant, workspace sizing, stats.  One translation unit holds every
// kernel so that the device status word is a single symbol.
//
// The MoE layer follows the onnxruntime PR "Enable SM80+ FP16/BF16 mixed
// INT2/INT4 QMoE prefill by default" (Description; Current Scope): route,
// expand rows by expert, FC1 with expert bias and interleaved SwiGLU, FC2,
// top-k weighted finalize with FC2 bias, row tiling within a scratch budget.
#include <algorithm>
#include <climits>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <vector>

#include "qmoe.h"
#include "device_common.cuh"
#include "unpack.cuh"
#include "qmm_small.cuh"
#include "qmm_grouped.cuh"
#include "kernels_misc.cuh"
#include "chan.cuh"
#include "slice.h"

#include <cudaTypedefs.h>

namespace qmoe {

__device__ unsigned g_status;

namespace {

constexpr int kMaxDevices = 64;
constexpr size_t kAlign = 256;
constexpr int kSmemLimit = 227 * 1024;

struct DevInfo {
  bool init = false;
  int sms = 0;
  unsigned* status = nullptr;
};
DevInfo g_dev[kMaxDevices];
std::mutex g_mu;
qmoe_stats g_stats = {};

qmoe_status dev_info(DevInfo** out) {
  int d = 0;
  if (cudaGetDevice(&d) != cudaSuccess || d < 0 || d >= kMaxDevices) return QMOE_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_mu);
  DevInfo& di = g_dev[d];
  if (!di.init) {
    if (cudaDeviceGetAttribute(&di.sms, cudaDevAttrMultiProcessorCount, d) != cudaSuccess) return QMOE_ERR_CUDA;
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_status) != cudaSuccess) return QMOE_ERR_CUDA;
    di.status = static_cast<unsigned*>(p);
    di.init = true;
  }
  *out = &di;
  return QMOE_OK;
}

// ---- tracing: CUDA events around each kernel launch ----
enum KernelId { K_ROUTE = 0, K_GATHER, K_FC1_SMALL, K_FC2_SMALL, K_COMBINE, K_LINEAR_SMALL, K_LINEAR_SETUP,
                K_DEQUANT, K_FC1_GROUPED, K_FC2_GROUPED, K_DECODE_RESET, K_DECODE_LAYER, K_LINEAR_GROUPED,
                K_CHAN_SCORE, K_CHAN_SELECT, K_CHAN_EXACT, K_CHAN_RESET, K_COUNT };
// K_DECODE_RESET / K_DECODE_LAYER: slice_reset_kernel / qmm_slice_kernel (the decode layer)
const char* const kKernelNames[K_COUNT] = {"route",        "gather",      "fc1_small",    "fc2_small",
                                           "combine",      "linear_small", "linear_setup", "dequant",
                                           "fc1_grouped",  "fc2_grouped", "decode_reset", "decode_layer",
                                           "linear_grouped", "chan_score", "chan_select", "chan_exact",
                                           "chan_reset"};
struct Tracer {
  bool on = false;
  int cap = 0, n = 0;
  std::vector<cudaEvent_t> ev;
  std::vector<int> ids;
} g_trace;

void record_event(cudaEvent_t e, cudaStream_t st) {
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  cudaStreamIsCapturing(st, &cs);
  if (cs == cudaStreamCaptureStatusActive) cudaEventRecordWithFlags(e, st, cudaEventRecordExternal);
  else cudaEventRecord(e, st);
}

// Brackets one launch with events while tracing is on.
struct TraceScope {
  cudaStream_t st;
  int id, slot = -1;
  TraceScope(cudaStream_t s, int kid) : st(s), id(kid) {
    std::lock_guard<std::mutex> lk(g_mu);
    if (g_trace.on && g_trace.n < g_trace.cap) {
      slot = g_trace.n++;
      g_trace.ids[slot] = id;
      record_event(g_trace.ev[2 * slot], st);
    }
  }
  ~TraceScope() {
    if (slot >= 0) record_event(g_trace.ev[2 * slot + 1], st);
  }
};

// Launch with programmatic dependent launch: the kernel may start while its
// predecessor in the stream finishes; every kernel calls griddepcontrol.wait
// before touching its predecessor's outputs and only then allows its own
// dependents to launch.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                       Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, args...);
}

inline size_t align_up(size_t v) { return (v + kAlign - 1) / kAlign * kAlign; }

bool fmt_ok(int f) { return f == QMOE_INT2 || f == QMOE_INT4 || f == QMOE_TERNARY; }
bool row_order_ok(int r) { return r == QMOE_ROWS_PLAIN || r == QMOE_ROWS_GATE_UP || r == QMOE_ROWS_KSPLIT; }
int ku_cols(int fmt) { return fmt == QMOE_TERNARY ? 128 : 64; }
int beta_hi(int fmt) { return fmt == QMOE_INT4 ? 1 : 4; }
size_t codes_bytes(int fmt, int rows, int K) {
  return fmt == QMOE_TERNARY ? (size_t)rows * (K / 128) * 26 : (size_t)rows * K * fmt / 8;
}
size_t scales_bytes(int rows, int K, int block) { return (size_t)rows * (K / block) * 2; }

qmoe_status check_weights(const qmoe_weights& w, int rows, int K) {
  if (!fmt_ok(w.fmt) || !row_order_ok(w.row_order) || !w.codes || !w.scales) return QMOE_ERR_INVALID_ARG;
  if (w.block != 64 && w.block != 128) return QMOE_ERR_UNSUPPORTED;
  if (rows % 16 || K % 64 || K % w.block) return QMOE_ERR_INVALID_ARG;
  if (w.fmt == QMOE_TERNARY && (w.block != 64 || K % 128)) return QMOE_ERR_UNSUPPORTED;
  if ((reinterpret_cast<uintptr_t>(w.codes) | reinterpret_cast<uintptr_t>(w.scales)) & 15) return QMOE_ERR_INVALID_ARG;
  if (w.zeros) {  // affine codes: INT2 / INT4 only
    if (w.fmt == QMOE_TERNARY) return QMOE_ERR_UNSUPPORTED;
    if (reinterpret_cast<uintptr_t>(w.zeros) & 15) return QMOE_ERR_INVALID_ARG;
  }
  return QMOE_OK;
}

// Workspace plan of one row tile of T tokens.
struct MoEPlan {
  int T, S, TK, max_seg, n_tickets, max_gseg;
  bool grouped, decode;
  SlicePlan slice;  // decode batches
  size_t ids, w, perm, inv, offsets, slot_token, nseg, segs, chunk_counts, yslot, hrows, yacc, ticket, ngseg, gsegs,
      xrows, total;
};

constexpr int kGroupedThreshold = 32;  // AUTO: experts with more tokens take the tcgen05 path
constexpr int kLinearGroupedMinM = 48;  // single linear: from this many rows on, the tcgen05 path

bool grouped_eligible(const qmoe_layer& L) {
  return L.fc1.fmt != QMOE_TERNARY && L.fc2.fmt != QMOE_TERNARY && (2 * L.I) % kGRows == 0 && L.H % kGRows == 0;
}

// Affine codes (zero points): every kernel takes them (INT2 / INT4).
bool affine(const qmoe_layer& L) { return L.fc1.zeros || L.fc2.zeros; }

// Token-count threshold above which an expert runs on the grouped path.
int grouped_threshold(const qmoe_layer& L) {
  if (L.path == QMOE_PATH_SMALL_M || !grouped_eligible(L)) return INT_MAX;
  return L.path == QMOE_PATH_GROUPED ? 0 : kGroupedThreshold;
}

// Single linear on the small-M kernel, split along K when it has fewer than
// 4 16-row tiles per SM (N = 5120: 320 tiles for 148 SMs), into about 8 (tile,
// k-slice) units per SM: slices of at least 12 k-units (one per warp), partial
// sums added into an fp32 accumulator in the workspace, the last slice of a
// tile rounds it to bf16.  (N = 17408, 7.4 tiles per SM, measured slower split.)
constexpr int kLinSplitTiles = 8;
int linear_ksplit(int N, int K, int fmt, int sms) {
  const int NT = N / 16, KU = K / ku_cols(fmt);
  if (2 * NT >= kLinSplitTiles * sms) return 1;
  const int want = (kLinSplitTiles * sms + NT / 2) / NT;
  for (int S = std::min(want, KU / 12); S > 1; --S)
    if (KU % S == 0) return S;
  return 1;
}
size_t linear_split_bytes(int N, int M) {
  return align_up((size_t)M * N * 4) + align_up((size_t)((M + kChunkTokens - 1) / kChunkTokens) * (N / 16) * 4);
}

// Fault injection for tests (qmoe_test_set_fault): the decode kernel's wait
// limit and what to inject.
unsigned long long g_fault_wait_ns = kWaitLimitNs;
int g_fault_inject = 0;

// Decode batches (T <= 8, T*k <= 64, H <= 2112) run as one launch of the
// kernel split along the expert intermediate dimension, which routes in its
// prologue (after a tiny reset launch of its accumulator).
bool decode_eligible(const qmoe_layer& L, int T, int grid, SlicePlan* plan) {
  if (T > kDecMaxT || T * L.k > kDecMaxTK || L.path == QMOE_PATH_GROUPED || L.H > kSMaxH) return false;
  const SlicePlan pl = slice_plan(L.fc1.fmt, L.fc2.fmt, T, L.H, affine(L));
  if (!pl.ok || L.I % pl.gran_cols) return false;
  const int gpe = L.I / pl.gran_cols;
  if (slice_max_chunks(L.fc2.fmt, gpe, L.n_shared, std::min(L.E, T * L.k), grid) > kSMaxChunks) return false;
  if (plan) *plan = pl;
  return true;
}

MoEPlan plan_moe(const qmoe_layer& L, int T, int grid) {
  MoEPlan p{};
  p.T = T;
  p.TK = T * L.k;
  p.S = T * (L.k + L.n_shared);
  p.decode = decode_eligible(L, T, grid, &p.slice);
  p.grouped = !p.decode && T > grouped_threshold(L);
  p.max_seg = std::min(L.E, p.TK) + p.TK / kChunkTokens + L.n_shared * ((T + kChunkTokens - 1) / kChunkTokens);
  size_t o = 0;
  auto take = [&](size_t bytes) { size_t at = o; o = align_up(o + bytes); return at; };
  if (p.decode) {  // the fp32 output accumulator and the last-CTA ticket
    p.yacc = take((size_t)T * L.H * 4);
    p.ticket = take(16);
    p.total = o;
    return p;
  }
  p.yslot = take((size_t)p.S * L.H * 4);
  p.hrows = take((size_t)p.S * L.I * 2 + 16);
  {
    p.ids = take((size_t)p.TK * 4);
    p.w = take((size_t)p.TK * 4);
    p.perm = take((size_t)p.TK * 4);
    p.inv = take((size_t)p.TK * 4);
    p.offsets = take((size_t)(L.E + 1) * 4);
    p.slot_token = take((size_t)p.S * 4);
    p.nseg = take(16);
    p.segs = take((size_t)p.max_seg * sizeof(Seg));
    p.chunk_counts = take((size_t)((T + kRouteChunk - 1) / kRouteChunk) * L.E * 4);
  }
  if (p.grouped) {
    p.max_gseg = std::min(L.E, p.TK) + p.TK / kGTok + L.n_shared * ((T + kGTok - 1) / kGTok);
    p.ngseg = take(16);
    p.gsegs = take((size_t)p.max_gseg * sizeof(GSeg));
    p.xrows = take((size_t)p.S * L.H * 2 + 16);
  }
  p.total = o;
  return p;
}

// ---- TMA tensor maps (driver entry point through the runtime; no libcuda link) ----
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

qmoe_status encode_rows_map(CUtensorMap* map, const void* base, int K, int rows) {
  if (!g_encode) {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess || !fn)
      return QMOE_ERR_CUDA;
    g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  }
  const cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)K * 2};
  const cuuint32_t box[2] = {64, (cuuint32_t)kGTmaRows};
  const cuuint32_t estr[2] = {1, 1};
  CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? QMOE_OK : QMOE_ERR_CUDA;
}

// ---- small-M kernel launch ----
// Dynamic shared memory of a small-M kernel: fixed head, reduction buffer and
// as many ring stages per warp as fit (at most kMaxStages, at least 2).
template <int FMT, int TG, int SRC, bool AFF>
int small_smem(int* nstages) {
  using G = StageGeom<FMT, TG, SRC, AFF>;
  constexpr int kNW = kWarps<TG>;
  const int fixed = SmemHead<SRC>::kFixed + G::kRedBytes;
  const int nst = std::min((kSmemLimit - fixed - 1024) / (kNW * G::kStageBytes), kMaxStages);
  *nstages = nst;
  return nst < 2 ? -1 : fixed + nst * kNW * G::kStageBytes;
}

template <int FMT, int TG, int EPI, int SRC, bool AFF>
qmoe_status launch_small_t(SmallParams prm, int grid, cudaStream_t st) {
  constexpr int kNW = kWarps<TG>;
  int nst = 0;
  const int smem = small_smem<FMT, TG, SRC, AFF>(&nst);
  if (smem < 0) return QMOE_ERR_UNSUPPORTED;
  prm.nstages = nst;
  static bool attr_set[kMaxDevices] = {};
  int d = 0;
  cudaGetDevice(&d);
  if (!attr_set[d]) {
    if (cudaFuncSetAttribute(qmm_small_kernel<FMT, TG, EPI, SRC, AFF>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             smem) != cudaSuccess)
      return QMOE_ERR_CUDA;
    attr_set[d] = true;
  }
  TraceScope ts(st, EPI == EPI_SWIGLU ? K_FC1_SMALL : (EPI == EPI_FC2 ? K_FC2_SMALL : K_LINEAR_SMALL));
  return launch_pdl(qmm_small_kernel<FMT, TG, EPI, SRC, AFF>, dim3(grid), dim3(kNW * 32), smem, st, prm) == cudaSuccess
             ? QMOE_OK
             : QMOE_ERR_CUDA;
}

template <int FMT, int EPI, int SRC, bool AFF>
qmoe_status launch_small_tg(int tg, const SmallParams& prm, int grid, cudaStream_t st) {
  return tg == 1 ? launch_small_t<FMT, 1, EPI, SRC, AFF>(prm, grid, st)
                 : launch_small_t<FMT, 2, EPI, SRC, AFF>(prm, grid, st);
}

// Affine codes (prm.zeros) take their own instantiations (INT2 / INT4).
template <int EPI, int SRC>
qmoe_status launch_small(int fmt, int tg, const SmallParams& prm, int grid, cudaStream_t st) {
  const bool aff = prm.zeros != nullptr;
  if (fmt == QMOE_INT2)
    return aff ? launch_small_tg<2, EPI, SRC, true>(tg, prm, grid, st) : launch_small_tg<2, EPI, SRC, false>(tg, prm, grid, st);
  if (fmt == QMOE_INT4)
    return aff ? launch_small_tg<4, EPI, SRC, true>(tg, prm, grid, st) : launch_small_tg<4, EPI, SRC, false>(tg, prm, grid, st);
  if (aff) return QMOE_ERR_UNSUPPORTED;
  return launch_small_tg<3, EPI, SRC, false>(tg, prm, grid, st);
}

template <int FMT, int EPI, int BT, int CS>
qmoe_status launch_grouped_t(const CUtensorMap& map, const GroupedParams& prm, int grid, cudaStream_t st) {
  constexpr int smem = GGeom<FMT, BT, CS>::kSmem;
  static_assert(smem <= kSmemLimit, "grouped kernel shared memory");
  static bool attr_set[kMaxDevices] = {};
  int d = 0;
  cudaGetDevice(&d);
  if (!attr_set[d]) {
    if (cudaFuncSetAttribute(qmm_grouped_kernel<FMT, EPI, BT, CS>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             smem) != cudaSuccess)
      return QMOE_ERR_CUDA;
    attr_set[d] = true;
  }
  TraceScope ts(st, EPI == EPI_SWIGLU ? K_FC1_GROUPED : (EPI == EPI_FC2 ? K_FC2_GROUPED : K_LINEAR_GROUPED));
  qmm_grouped_kernel<FMT, EPI, BT, CS><<<grid, kGThreads, smem, st>>>(map, prm);
  return cudaGetLastError() == cudaSuccess ? QMOE_OK : QMOE_ERR_CUDA;
}

// Expert tiles: units of up to 256 tokens, a weight ring as deep as the token ring.
template <int EPI>
qmoe_status launch_grouped(int fmt, const CUtensorMap& map, const GroupedParams& prm, int grid, cudaStream_t st) {
  if (fmt == QMOE_INT2) return launch_grouped_t<2, EPI, kGTok, kGStages>(map, prm, grid, st);
  if (fmt == QMOE_INT4) return launch_grouped_t<4, EPI, kGTok, kGStages>(map, prm, grid, st);
  return QMOE_ERR_UNSUPPORTED;
}

// Single linear: units of up to 128 tokens; a weight ring of about 64 KB (28
// INT2 or 16 INT4 stages), the bytes in flight an SM needs for its HBM share.
qmoe_status launch_grouped_linear(int fmt, const CUtensorMap& map, const GroupedParams& prm, int grid,
                                  cudaStream_t st) {
  if (fmt == QMOE_INT2) return launch_grouped_t<2, EPI_LINEAR, kLinBT, 28>(map, prm, grid, st);
  if (fmt == QMOE_INT4) return launch_grouped_t<4, EPI_LINEAR, kLinBT, 16>(map, prm, grid, st);
  return QMOE_ERR_UNSUPPORTED;
}

GroupedParams grouped_params(const qmoe_weights& w, int rows, int K, unsigned* status) {
  GroupedParams p{};
  p.codes = static_cast<const uint8_t*>(w.codes);
  p.codes_stride = codes_bytes(w.fmt, rows, K);
  p.scales = static_cast<const uint8_t*>(w.scales);
  p.scales_stride = scales_bytes(rows, K, w.block);
  p.zeros = static_cast<const uint8_t*>(w.zeros);
  p.NT = rows / 16;
  p.K = K;
  p.block = w.block;
  p.rtiles = rows / kGRows;
  p.status = status;
  return p;
}

SmallParams small_params(const qmoe_weights& w, int rows, int K, unsigned* status) {
  SmallParams p{};
  p.codes = static_cast<const uint8_t*>(w.codes);
  p.codes_stride = codes_bytes(w.fmt, rows, K);
  p.scales = static_cast<const uint8_t*>(w.scales);
  p.scales_stride = scales_bytes(rows, K, w.block);
  p.zeros = static_cast<const uint8_t*>(w.zeros);
  p.NT = rows / 16;
  p.K = K;
  p.KU = K / ku_cols(w.fmt);
  p.ksplit = 1;
  p.KUs = p.KU;
  p.block = w.block;
  p.status = status;
  return p;
}

qmoe_status check_layer(const qmoe_layer* L) {
  if (!L) return QMOE_ERR_INVALID_ARG;
  if (L->H <= 0 || L->I <= 0 || L->E <= 0 || L->k <= 0 || L->n_shared < 0) return QMOE_ERR_INVALID_ARG;
  if (L->E > kMaxExperts || L->k > 32 || L->k > L->E || L->n_shared > 64) return QMOE_ERR_UNSUPPORTED;
  if (L->H % 64 || L->I % 64) return QMOE_ERR_INVALID_ARG;
  if (L->path < QMOE_PATH_AUTO || L->path > QMOE_PATH_GROUPED) return QMOE_ERR_INVALID_ARG;
  if (L->max_row_tile < 0) return QMOE_ERR_INVALID_ARG;
  if (L->fc1.row_order != QMOE_ROWS_GATE_UP || L->fc2.row_order != QMOE_ROWS_KSPLIT) return QMOE_ERR_INVALID_ARG;
  qmoe_status s = check_weights(L->fc1, 2 * L->I, L->H);
  if (s != QMOE_OK) return s;
  s = check_weights(L->fc2, L->H, L->I);
  return s;
}


// ---- channel layer (top-k channel-selective read) ----
struct ChanPlan {
  size_t ids, wts, scores, sel, hist, yacc, ticket, total;  // hist and yacc adjacent (one reset)
};

ChanPlan chan_plan(const qmoe_chan_layer& L, int T, int n_keep) {
  ChanPlan c;
  size_t o = 0;
  c.ids = o;
  o += align_up((size_t)T * L.k * 4);
  c.wts = o;
  o += align_up((size_t)T * L.k * 4);
  c.scores = o;
  o += align_up((size_t)T * L.k * L.I * 4);
  c.sel = o;
  o += align_up((size_t)T * std::max(n_keep, 1) * 4);
  c.hist = o;
  o += (size_t)T * kChanBins * 4;
  c.yacc = o;
  o += align_up((size_t)T * L.H * 4);
  c.ticket = o;
  o += align_up(2 * 4);
  c.total = o;
  return c;
}

qmoe_status chan_check(const qmoe_chan_layer* L, size_t* rec, size_t* sk) {
  if (!L) return QMOE_ERR_INVALID_ARG;
  if (L->k < 1 || L->k > kChanMaxK || L->E < L->k || L->E > 256 || L->I < 1 || L->n_shared < 0)
    return QMOE_ERR_INVALID_ARG;
  if ((size_t)L->k * L->I > (size_t)kChanMaxCand) return QMOE_ERR_UNSUPPORTED;
  qmoe_status s = qmoe_chan_sizes(L->fmt1, L->fmt2, L->H, L->block, rec, sk);
  if (s != QMOE_OK) return s;
  if (L->H > kChanMaxH) return QMOE_ERR_UNSUPPORTED;
  if (!L->records || !L->sketch || !L->dn || !L->signs) return QMOE_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(L->records) | reinterpret_cast<uintptr_t>(L->sketch) |
       reinterpret_cast<uintptr_t>(L->signs)) & 15)
    return QMOE_ERR_INVALID_ARG;
  return QMOE_OK;
}

size_t align_to(size_t v, size_t a) { return (v + a - 1) / a * a; }
// Dynamic shared memory of the score and exact kernels (as laid out in chan.cuh), with
// slack for aligning the wave buffer to 128 bytes.
size_t chan_score_smem(int T, int H, int wave, int skb) {
  return align_to(4 * ((size_t)T * H + (size_t)T * (H / 16)), 16) + 8 * (size_t)wave + 256 + (size_t)wave * skb;
}
int chan_tm(int T) { return T <= 1 ? 1 : T <= 2 ? 2 : T <= 4 ? 4 : 8; }
size_t chan_exact_smem(int T, int H, int f1, int wave, int R) {
  const size_t nc = (size_t)H / (128 / f1);
  return align_to(4 * ((size_t)T * H + T * nc + (size_t)wave * chan_tm(T) + 2 * (size_t)wave), 16) +
         8 * (size_t)wave + 256 + (size_t)wave * R;
}
constexpr size_t kChanSmemBudget = kSmemLimit - 8 * 1024;  // static shared memory of the kernels

template <int NWL>
void (*chan_score_of(int tm))(ChanParams) {
  return tm == 1 ? chan_score_kernel<1, NWL> : tm == 2 ? chan_score_kernel<2, NWL>
         : tm == 4 ? chan_score_kernel<4, NWL> : chan_score_kernel<8, NWL>;
}

template <int TM>
void (*chan_exact_of(int f1, int f2))(ChanParams) {
  if (f1 == QMOE_INT4 && f2 == QMOE_INT4) return chan_exact_kernel<4, 4, TM>;
  if (f1 == QMOE_INT4 && f2 == QMOE_INT2) return chan_exact_kernel<4, 2, TM>;
  if (f1 == QMOE_INT2 && f2 == QMOE_INT4) return chan_exact_kernel<2, 4, TM>;
  return chan_exact_kernel<2, 2, TM>;
}

qmoe_status launch_chan_exact(int f1, int f2, const ChanParams& p, int grid, size_t smem, cudaStream_t st) {
  const int tm = chan_tm(p.T);
  void (*k)(ChanParams) = tm == 1   ? chan_exact_of<1>(f1, f2)
                          : tm == 2 ? chan_exact_of<2>(f1, f2)
                          : tm == 4 ? chan_exact_of<4>(f1, f2)
                                    : chan_exact_of<8>(f1, f2);
  if (cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
    return QMOE_ERR_CUDA;
  TraceScope ts(st, K_CHAN_EXACT);
  return launch_pdl(k, dim3(grid), dim3(kChanThreads), smem, st, p) == cudaSuccess ? QMOE_OK : QMOE_ERR_CUDA;
}

}  // namespace
}  // namespace qmoe

using namespace qmoe;

extern "C" {

const char* qmoe_status_str(int s) {
  switch (s) {
    case QMOE_OK: return "ok";
    case QMOE_ERR_INVALID_ARG: return "invalid argument";
    case QMOE_ERR_UNSUPPORTED: return "unsupported configuration";
    case QMOE_ERR_SCRATCH: return "workspace too small for one token row";
    case QMOE_ERR_CUDA: return "CUDA runtime error";
    case QMOE_ERR_TIMEOUT: return "device wait timed out";
    case QMOE_ERR_STATIC_SCRATCH: return "request needs more than the static scratch (QMOE_STATIC_SCRATCH_BYTES)";
    default: return "unknown status";
  }
}

const char* qmoe_kernel_name(int id) { return id >= 0 && id < K_COUNT ? kKernelNames[id] : "unknown"; }

qmoe_status qmoe_trace_start(int cap) {
  if (cap <= 0 || cap > (1 << 20)) return QMOE_ERR_INVALID_ARG;
  std::lock_guard<std::mutex> lk(g_mu);
  for (cudaEvent_t e : g_trace.ev) cudaEventDestroy(e);
  g_trace.ev.assign(2 * (size_t)cap, nullptr);
  g_trace.ids.assign(cap, -1);
  for (auto& e : g_trace.ev)
    if (cudaEventCreate(&e) != cudaSuccess) {
      g_trace.on = false;
      return QMOE_ERR_CUDA;
    }
  g_trace.cap = cap;
  g_trace.n = 0;
  g_trace.on = true;
  return QMOE_OK;
}

qmoe_status qmoe_trace_stop(void) {
  std::lock_guard<std::mutex> lk(g_mu);
  g_trace.on = false;
  return QMOE_OK;
}

qmoe_status qmoe_trace_read(int cap, int* n, int* kernel_ids, float* ms) {
  if (!n || cap < 0 || (cap > 0 && (!kernel_ids || !ms))) return QMOE_ERR_INVALID_ARG;
  if (cudaDeviceSynchronize() != cudaSuccess) return QMOE_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_mu);
  const int m = std::min(cap, g_trace.n);
  for (int i = 0; i < m; ++i) {
    kernel_ids[i] = g_trace.ids[i];
    float t = -1.f;
    if (cudaEventElapsedTime(&t, g_trace.ev[2 * i], g_trace.ev[2 * i + 1]) != cudaSuccess) t = -1.f;
    ms[i] = t;
  }
  *n = g_trace.n;
  cudaGetLastError();  // an unrecorded event leaves a sticky-free error: clear it
  return QMOE_OK;
}

qmoe_status qmoe_test_set_fault(int inject, unsigned long long wait_limit_ns) {
  if (inject < 0 || inject > 1) return QMOE_ERR_INVALID_ARG;
  qmoe::g_fault_inject = inject;
  qmoe::g_fault_wait_ns = wait_limit_ns ? wait_limit_ns : qmoe::kWaitLimitNs;
  return QMOE_OK;
}

qmoe_status qmoe_get_stats(qmoe_stats* out) {
  if (!out) return QMOE_ERR_INVALID_ARG;
  DevInfo* di;
  qmoe_status s = dev_info(&di);
  if (s != QMOE_OK) return s;
  unsigned v = 0;
  if (cudaMemcpy(&v, di->status, sizeof(v), cudaMemcpyDeviceToHost) != cudaSuccess) return QMOE_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_mu);
  *out = g_stats;
  out->device_status = v;
  return QMOE_OK;
}

qmoe_status qmoe_clear_status(void) {
  DevInfo* di;
  qmoe_status s = dev_info(&di);
  if (s != QMOE_OK) return s;
  return cudaMemset(di->status, 0, sizeof(unsigned)) == cudaSuccess ? QMOE_OK : QMOE_ERR_CUDA;
}

qmoe_status qmoe_route_workspace_size(int T, int E, int k, size_t* bytes) {
  if (!bytes || T <= 0 || E <= 0 || k <= 0) return QMOE_ERR_INVALID_ARG;
  if (E > kMaxExperts || k > 32 || k > E) return QMOE_ERR_UNSUPPORTED;
  *bytes = (T <= kDecMaxT && T * k <= kDecMaxTK) ? 0 : align_up((size_t)((T + kRouteChunk - 1) / kRouteChunk) * E * 4);
  return QMOE_OK;
}

qmoe_status qmoe_route(const float* logits, int T, int E, int k, int32_t* ids, float* weights, int32_t* perm,
                       int32_t* offsets, void* ws, size_t ws_bytes, void* stream) {
  if (!logits || !ids || !weights || !perm || !offsets || T <= 0 || E <= 0 || k <= 0) return QMOE_ERR_INVALID_ARG;
  if (E > kMaxExperts || k > 32 || k > E) return QMOE_ERR_UNSUPPORTED;
  size_t need = 0;
  qmoe_route_workspace_size(T, E, k, &need);
  if (need > ws_bytes || (need && !ws)) return QMOE_ERR_SCRATCH;
  if (reinterpret_cast<uintptr_t>(ws) & 15) return QMOE_ERR_INVALID_ARG;
  DevInfo* di;
  qmoe_status s = dev_info(&di);
  if (s != QMOE_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  TraceScope ts(st, K_ROUTE);
  if (need == 0) {  // decode batch: the decode layer kernel's routing, as one CTA
    route_decode_kernel<<<1, kDecMaxT * 32, 0, st>>>(logits, T, E, k, ids, weights, perm, offsets);
    return cudaGetLastError() == cudaSuccess ? QMOE_OK : QMOE_ERR_CUDA;
  }
  RouteOut o{};
  o.ids = ids;
  o.w = weights;
  o.perm = perm;
  o.offsets = offsets;
  o.status = di->status;
  o.chunk_counts = static_cast<int*>(ws);
  const int nchunks = (T + kRouteChunk - 1) / kRouteChunk;
  if (launch_pdl(route_topk_kernel, dim3(nchunks), dim3(kRouteWarps * 32), 0, st, logits, T, E, k, o) !=
          cudaSuccess ||
      launch_pdl(route_scatter_kernel, dim3(nchunks), dim3(kRouteWarps * 32), 0, st, T, E, k, 0, o) != cudaSuccess)
    return QMOE_ERR_CUDA;
  return QMOE_OK;
}

qmoe_status qmoe_workspace_size(const qmoe_layer* layer, int T, size_t* bytes) {
  qmoe_status s = check_layer(layer);
  if (s != QMOE_OK) return s;
  if (T <= 0 || !bytes) return QMOE_ERR_INVALID_ARG;
  DevInfo* di;
  s = dev_info(&di);
  if (s != QMOE_OK) return s;
  int Tt = T;
  if (layer->max_row_tile > 0) Tt = std::min(Tt, layer->max_row_tile);
  *bytes = plan_moe(*layer, Tt, di->sms).total;
  return QMOE_OK;
}

qmoe_status qmoe_forward(const qmoe_layer* layer, const uint16_t* x, const float* logits, int T, uint16_t* y,
                         void* ws, size_t ws_bytes, void* stream) {
  qmoe_status s = check_layer(layer);
  if (s != QMOE_OK) return s;
  if (!x || !logits || !y || !ws || T <= 0) return QMOE_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(ws) % kAlign) || (reinterpret_cast<uintptr_t>(x) & 15) ||
      (reinterpret_cast<uintptr_t>(y) & 7))
    return QMOE_ERR_INVALID_ARG;
  if (layer->path == QMOE_PATH_GROUPED && !grouped_eligible(*layer)) return QMOE_ERR_UNSUPPORTED;
  DevInfo* di;
  s = dev_info(&di);
  if (s != QMOE_OK) return s;
  const qmoe_layer& L = *layer;
  const int grid = di->sms;
  // Row tile: the largest (<= T, <= max_row_tile) whose workspace fits; halve until it does.
  int Tt = T;
  if (L.max_row_tile > 0) Tt = std::min(Tt, L.max_row_tile);
  while (plan_moe(L, Tt, grid).total > ws_bytes) {
    if (Tt == 1) return QMOE_ERR_SCRATCH;
    Tt = (Tt + 1) / 2;
  }
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* base = static_cast<uint8_t*>(ws);
  int tiles = 0, small = 0, grouped = 0, decode = 0;
  for (int t0 = 0; t0 < T; t0 += Tt) {
    const int tt = std::min(Tt, T - t0);
    const MoEPlan p = plan_moe(L, tt, grid);
    const uint16_t* xt = x + (size_t)t0 * L.H;
    const float* lt = logits + (size_t)t0 * L.E;
    uint16_t* yt = y + (size_t)t0 * L.H;
    if (p.decode) {
      // Decode batch: one launch, split along the experts' intermediate dimension.
      SliceParams sp{};
      sp.c1 = static_cast<const uint8_t*>(L.fc1.codes);
      sp.c1_stride = codes_bytes(L.fc1.fmt, 2 * L.I, L.H);
      sp.s1 = static_cast<const uint8_t*>(L.fc1.scales);
      sp.s1_stride = scales_bytes(2 * L.I, L.H, L.fc1.block);
      sp.b1 = L.fc1.bias;
      sp.c2 = static_cast<const uint8_t*>(L.fc2.codes);
      sp.c2_stride = codes_bytes(L.fc2.fmt, L.H, L.I);
      sp.s2 = static_cast<const uint8_t*>(L.fc2.scales);
      sp.s2_stride = scales_bytes(L.H, L.I, L.fc2.block);
      sp.b2 = L.fc2.bias;
      sp.aff = affine(L) ? 1 : 0;
      sp.z1 = static_cast<const uint8_t*>(L.fc1.zeros);
      sp.z2 = static_cast<const uint8_t*>(L.fc2.zeros);
      sp.NT1 = 2 * L.I / 16;
      sp.KU1 = L.H / ku_cols(L.fc1.fmt);
      sp.block1 = L.fc1.block;
      sp.NT2 = L.H / 16;
      sp.block2 = L.fc2.block;
      sp.H = L.H;
      sp.I = L.I;
      sp.E = L.E;
      sp.k = L.k;
      sp.n_shared = L.n_shared;
      sp.T = tt;
      sp.gpe = L.I / p.slice.gran_cols;
      sp.ring_bytes = p.slice.ring_bytes;
      sp.ngm = p.slice.ngm;
      sp.xrows = p.slice.xrows;
      sp.x = xt;
      sp.logits = lt;
      sp.y = yt;
      sp.yacc = reinterpret_cast<float*>(base + p.yacc);
      sp.ticket = reinterpret_cast<int*>(base + p.ticket);
      sp.status = di->status;
      sp.wait_ns = g_fault_wait_ns;
      sp.inject = g_fault_inject;
      {
        TraceScope ts(st, K_DECODE_RESET);
        if (slice_reset_launch(sp.yacc, tt * L.H / 4, sp.ticket, st) != cudaSuccess) return QMOE_ERR_CUDA;
      }
      {
        TraceScope ts(st, K_DECODE_LAYER);
        if (slice_launch(L.fc1.fmt, L.fc2.fmt, sp, grid, p.slice.smem, st) != cudaSuccess) return QMOE_ERR_CUDA;
      }
      ++tiles;
      ++small;
      ++decode;
      continue;
    }
    float* yslot = reinterpret_cast<float*>(base + p.yslot);
    uint16_t* hrows = reinterpret_cast<uint16_t*>(base + p.hrows);
    SmallParams p1 = small_params(L.fc1, 2 * L.I, L.H, di->status);
    p1.act = xt;
    p1.bias = L.fc1.bias;
    p1.bias_rows = 2 * L.I;
    p1.hrows = hrows;
    p1.I = L.I;
    p1.H = L.H;
    SmallParams p2 = small_params(L.fc2, L.H, L.I, di->status);
    p2.act = hrows;
    p2.act_index = nullptr;
    p2.bias = L.fc2.bias;
    p2.bias_rows = L.H;
    p2.yslot = yslot;
    p2.H = L.H;
    p2.I = L.I;
    RouteOut o{};
    o.ids = reinterpret_cast<int*>(base + p.ids);
    o.w = reinterpret_cast<float*>(base + p.w);
    o.perm = reinterpret_cast<int*>(base + p.perm);
    o.inv = reinterpret_cast<int*>(base + p.inv);
    o.offsets = reinterpret_cast<int*>(base + p.offsets);
    o.slot_token = reinterpret_cast<int*>(base + p.slot_token);
    o.nseg = reinterpret_cast<int*>(base + p.nseg);
    o.segs = reinterpret_cast<Seg*>(base + p.segs);
    o.max_seg = p.max_seg;
    o.thresh = grouped_threshold(L);
    if (p.grouped) {
      o.ngseg = reinterpret_cast<int*>(base + p.ngseg);
      o.gsegs = reinterpret_cast<GSeg*>(base + p.gsegs);
      o.max_gseg = p.max_gseg;
    }
    o.status = di->status;
    o.chunk_counts = reinterpret_cast<int*>(base + p.chunk_counts);
    {
      const int nchunks = (tt + kRouteChunk - 1) / kRouteChunk;
      TraceScope ts(st, K_ROUTE);
      if (launch_pdl(route_topk_kernel, dim3(nchunks), dim3(kRouteWarps * 32), 0, st, lt, tt, L.E, L.k, o) !=
              cudaSuccess ||
          launch_pdl(route_scatter_kernel, dim3(nchunks), dim3(kRouteWarps * 32), 0, st, tt, L.E, L.k, L.n_shared,
                     o) != cudaSuccess)
        return QMOE_ERR_CUDA;
    }
    const int tg = tt <= 8 ? 1 : 2;
    p1.nseg = o.nseg;
    p1.segs = o.segs;
    p1.act_index = o.slot_token;
    p1.early = 0;  // the segment table comes from the routing launch just before
    p2.nseg = o.nseg;
    p2.segs = o.segs;
    p2.early = 1;
    s = launch_small<EPI_SWIGLU, SRC_TABLE>(L.fc1.fmt, tg, p1, grid, st);
    if (s != QMOE_OK) return s;
    CUtensorMap map2;
    GroupedParams g2{};
    if (p.grouped) {
      uint16_t* xrows = reinterpret_cast<uint16_t*>(base + p.xrows);
      {
        TraceScope ts(st, K_GATHER);
        gather_rows_kernel<<<8 * grid, 256, 0, st>>>(xt, L.H, o.slot_token, o.ngseg, o.gsegs,
                                                                            xrows);
        if (cudaGetLastError() != cudaSuccess) return QMOE_ERR_CUDA;
      }
      CUtensorMap map1;
      s = encode_rows_map(&map1, xrows, L.H, p.S);
      if (s != QMOE_OK) return s;
      s = encode_rows_map(&map2, hrows, L.I, p.S);
      if (s != QMOE_OK) return s;
      GroupedParams g1 = grouped_params(L.fc1, 2 * L.I, L.H, di->status);
      g1.ngseg = o.ngseg;
      g1.gsegs = o.gsegs;
      g1.bias = L.fc1.bias;
      g1.bias_rows = 2 * L.I;
      g1.hrows = hrows;
      g1.I = L.I;
      s = launch_grouped<EPI_SWIGLU>(L.fc1.fmt, map1, g1, std::min(p.max_gseg * g1.rtiles, grid), st);
      if (s != QMOE_OK) return s;
      g2 = grouped_params(L.fc2, L.H, L.I, di->status);
      g2.ngseg = o.ngseg;
      g2.gsegs = o.gsegs;
      g2.bias = L.fc2.bias;
      g2.bias_rows = L.H;
      g2.yslot = yslot;
      g2.H = L.H;
    }
    s = launch_small<EPI_FC2, SRC_TABLE>(L.fc2.fmt, tg, p2, grid, st);
    if (s != QMOE_OK) return s;
    if (p.grouped) {
      s = launch_grouped<EPI_FC2>(L.fc2.fmt, map2, g2, std::min(p.max_gseg * g2.rtiles, grid), st);
      if (s != QMOE_OK) return s;
      ++grouped;
    }
    {
      TraceScope ts(st, K_COMBINE);
      if (launch_pdl(combine_kernel, dim3(tt), dim3(256), 0, st, (const float*)yslot, (const float*)o.w,
                     (const int*)o.inv, tt, L.k, L.n_shared, L.H, yt) != cudaSuccess)
        return QMOE_ERR_CUDA;
    }
    ++tiles;
    small += 2;
  }
  std::lock_guard<std::mutex> lk(g_mu);
  g_stats.last_path = grouped ? (L.path == QMOE_PATH_GROUPED ? QMOE_PATH_GROUPED : QMOE_PATH_AUTO) : QMOE_PATH_SMALL_M;
  g_stats.row_tiles = tiles;
  g_stats.row_tile_tokens = Tt;
  g_stats.small_launches = small;
  g_stats.grouped_launches = 2 * grouped;
  return QMOE_OK;
}

qmoe_status qmoe_linear_workspace_size(int N, int K, int M, size_t* bytes) {
  if (N <= 0 || K <= 0 || M <= 0 || N % 16 || K % 64 || !bytes) return QMOE_ERR_INVALID_ARG;
  *bytes = linear_split_bytes(N, M);
  return QMOE_OK;
}

qmoe_status qmoe_linear(const qmoe_weights* w, int N, int K, const uint16_t* x, int M, uint16_t* y, void* ws,
                        size_t ws_bytes, void* stream) {
  if (!w || !x || !y || M <= 0) return QMOE_ERR_INVALID_ARG;
  if (w->row_order != QMOE_ROWS_PLAIN) return QMOE_ERR_INVALID_ARG;
  qmoe_status s = check_weights(*w, N, K);
  if (s != QMOE_OK) return s;
  if (reinterpret_cast<uintptr_t>(x) & 15) return QMOE_ERR_INVALID_ARG;
  DevInfo* di;
  s = dev_info(&di);
  if (s != QMOE_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  SmallParams p = small_params(*w, N, K, di->status);
  p.act = x;
  p.T = M;
  p.y = y;
  p.N = N;
  p.early = 1;  // static weights, arithmetic segments
  // More than one token group: the tcgen05 path, whose cost barely depends on
  // M (the dequantized tile serves up to 256 tokens; the small-M kernel's
  // mma.sync work grows with every group of 8 tokens).
  const bool grouped = M >= kLinearGroupedMinM && N % kGRows == 0 && w->fmt != QMOE_TERNARY;
  if (grouped) {
    CUtensorMap map;
    s = encode_rows_map(&map, x, K, M);
    if (s != QMOE_OK) return s;
    GroupedParams g = grouped_params(*w, N, K, di->status);
    g.y = y;
    g.N = N;
    g.ntok = M;
    const int units = (M + kLinBT - 1) / kLinBT * g.rtiles;
    s = launch_grouped_linear(w->fmt, map, g, std::min(units, di->sms), st);
  } else {
    const int S = linear_ksplit(N, K, w->fmt, di->sms);
    if (S > 1 && ws && ws_bytes >= linear_split_bytes(N, M) && !(reinterpret_cast<uintptr_t>(ws) % kAlign)) {
      p.ksplit = S;
      p.KUs = p.KU / S;
      p.yacc = static_cast<float*>(ws);
      p.tickets = reinterpret_cast<int*>(static_cast<uint8_t*>(ws) + align_up((size_t)M * N * 4));
      const int n4 = M * N / 4, nt = (M + kChunkTokens - 1) / kChunkTokens * (N / 16);
      TraceScope ts(st, K_DECODE_RESET);
      if (launch_pdl(accum_reset_kernel, dim3(std::max(1, std::min(di->sms, (n4 + 255) / 256))), dim3(256), 0, st,
                     p.yacc, n4, p.tickets, nt) != cudaSuccess)
        return QMOE_ERR_CUDA;
    }
    s = launch_small<EPI_LINEAR, SRC_LINEAR>(w->fmt, M <= 8 ? 1 : 2, p, di->sms, st);
  }
  if (s != QMOE_OK) return s;
  std::lock_guard<std::mutex> lk(g_mu);
  g_stats.last_path = grouped ? QMOE_PATH_GROUPED : QMOE_PATH_SMALL_M;
  g_stats.row_tiles = 1;
  g_stats.row_tile_tokens = M;
  g_stats.small_launches = grouped ? 0 : 1;
  g_stats.grouped_launches = grouped ? 1 : 0;
  return QMOE_OK;
}

qmoe_status qmoe_dequant(const qmoe_weights* w, int rows, int K, int n_mats, float* out_f32, uint16_t* out_bf16,
                         void* stream) {
  if (!w || n_mats <= 0 || (!out_f32 && !out_bf16)) return QMOE_ERR_INVALID_ARG;
  const int row_order = w->row_order;
  qmoe_status s = check_weights(*w, rows, K);
  if (s != QMOE_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const unsigned long long cs = codes_bytes(w->fmt, rows, K), ss = scales_bytes(rows, K, w->block);
  const uint8_t* c = static_cast<const uint8_t*>(w->codes);
  const uint8_t* sc = static_cast<const uint8_t*>(w->scales);
  const uint8_t* zc = static_cast<const uint8_t*>(w->zeros);
  const long long items = (long long)n_mats * (K / ku_cols(w->fmt)) * (rows / 16);
  const int grid = (int)std::min<long long>((items + 7) / 8, 65535);
  TraceScope ts(st, K_DEQUANT);
  if (w->fmt == QMOE_INT2)
    dequant_kernel<2><<<grid, 256, 0, st>>>(c, cs, sc, zc, ss, rows / 16, K, w->block, row_order, n_mats, out_f32,
                                            out_bf16);
  else if (w->fmt == QMOE_INT4)
    dequant_kernel<4><<<grid, 256, 0, st>>>(c, cs, sc, zc, ss, rows / 16, K, w->block, row_order, n_mats, out_f32,
                                            out_bf16);
  else
    dequant_kernel<3><<<grid, 256, 0, st>>>(c, cs, sc, nullptr, ss, rows / 16, K, w->block, row_order, n_mats,
                                            out_f32, out_bf16);
  return cudaGetLastError() == cudaSuccess ? QMOE_OK : QMOE_ERR_CUDA;
}

qmoe_status qmoe_chan_workspace_size(const qmoe_chan_layer* layer, int T, int n_keep, size_t* bytes) {
  size_t rec, sk;
  qmoe_status s = chan_check(layer, &rec, &sk);
  if (s != QMOE_OK) return s;
  if (T < 1 || T > kChanMaxT || n_keep < 0 || n_keep > layer->k * layer->I || !bytes) return QMOE_ERR_INVALID_ARG;
  *bytes = chan_plan(*layer, T, n_keep).total;
  return QMOE_OK;
}

qmoe_status qmoe_chan_forward(const qmoe_chan_layer* layer, const uint16_t* x, const float* logits, int T,
                              int n_keep, uint16_t* y, int32_t* sel, float* scores, void* ws, size_t ws_bytes,
                              void* stream) {
  size_t rec, sk;
  qmoe_status s = chan_check(layer, &rec, &sk);
  if (s != QMOE_OK) return s;
  const qmoe_chan_layer& L = *layer;
  if (!x || !logits || !y || !ws || T < 1 || T > kChanMaxT || n_keep < 0 || n_keep > L.k * L.I)
    return QMOE_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(ws) % kAlign) || (reinterpret_cast<uintptr_t>(scores) & 3) ||
      (reinterpret_cast<uintptr_t>(sel) & 3))
    return QMOE_ERR_INVALID_ARG;
  const ChanPlan plan = chan_plan(L, T, n_keep);
  if (ws_bytes < plan.total) return QMOE_ERR_SCRATCH;
  DevInfo* di;
  s = dev_info(&di);
  if (s != QMOE_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* w = static_cast<uint8_t*>(ws);
  ChanParams p = {};
  p.H = L.H;
  p.I = L.I;
  p.E = L.E;
  p.k = L.k;
  p.S = L.n_shared;
  p.T = T;
  p.fmt1 = L.fmt1;
  p.fmt2 = L.fmt2;
  p.block = L.block;
  p.rec_bytes = (int)rec;
  p.sk_bytes = (int)sk;
  p.rec = static_cast<const uint8_t*>(L.records);
  p.sketch = static_cast<const uint8_t*>(L.sketch);
  p.dn = L.dn;
  p.signs = L.signs;
  p.x = x;
  p.logits = logits;
  p.n_keep = n_keep;
  p.ids = reinterpret_cast<int*>(w + plan.ids);
  p.wts = reinterpret_cast<float*>(w + plan.wts);
  p.scores = scores ? scores : reinterpret_cast<float*>(w + plan.scores);
  p.sel = sel ? sel : reinterpret_cast<int*>(w + plan.sel);
  p.hist = reinterpret_cast<int*>(w + plan.hist);
  p.yacc = reinterpret_cast<float*>(w + plan.yacc);
  p.ticket = reinterpret_cast<int*>(w + plan.ticket);
  p.y = y;
  p.inv_sqrt_h = (float)(1.0 / std::sqrt((double)L.H));
  p.wait_ns = g_fault_wait_ns;
  p.inject = g_fault_inject;
  p.status = di->status;

  // scores: every block may hold up to ceil(units / grid) sketch records
  const int g1 = di->sms;
  const int units1 = std::min(L.E, T * L.k) * L.I;
  const size_t fix1 = chan_score_smem(T, L.H, 0, (int)sk);
  if (fix1 + 2 * sk + 8 > kChanSmemBudget) return QMOE_ERR_UNSUPPORTED;
  p.wave_sk = (int)std::min<size_t>((units1 + g1 - 1) / g1, (kChanSmemBudget - fix1) / (sk + 8));
  const size_t smem1 = chan_score_smem(T, L.H, p.wave_sk, (int)sk);
  // exact: shared channels then the selected ones
  const int units3 = L.n_shared * L.I + T * n_keep;
  const int g3 = std::max(1, std::min(di->sms, (units3 + 3) / 4));
  const size_t fix3 = chan_exact_smem(T, L.H, L.fmt1, 0, (int)rec);
  const size_t per3 = rec + 8 + 4 * (chan_tm(T) + 2);
  if (fix3 + 2 * per3 > kChanSmemBudget) return QMOE_ERR_UNSUPPORTED;
  p.wave_rec = (int)std::max<size_t>(1, std::min<size_t>((units3 + g3 - 1) / g3, (kChanSmemBudget - fix3) / per3));
  const size_t smem3 = chan_exact_smem(T, L.H, L.fmt1, p.wave_rec, (int)rec);

  void (*score)(ChanParams) = L.H == 512    ? chan_score_of<1>(chan_tm(T))
                              : L.H == 1024 ? chan_score_of<2>(chan_tm(T))
                                            : chan_score_of<4>(chan_tm(T));
  const size_t smem2 = (size_t)L.k * L.I * 4;
  if (cudaFuncSetAttribute(score, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem1) != cudaSuccess ||
      cudaFuncSetAttribute(chan_select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem2) !=
          cudaSuccess)
    return QMOE_ERR_CUDA;
  {  // the selection histogram, the output accumulator and the tickets start at zero
    const int n4 = (int)(((size_t)T * kChanBins + (size_t)T * L.H) / 4);
    TraceScope ts(st, K_CHAN_RESET);
    if (launch_pdl(accum_reset_kernel, dim3(std::max(1, std::min(di->sms, (n4 + 255) / 256))), dim3(256), 0, st,
                   reinterpret_cast<float*>(p.hist), n4, p.ticket, 2) != cudaSuccess)
      return QMOE_ERR_CUDA;
  }
  {
    TraceScope ts(st, K_CHAN_SCORE);
    if (launch_pdl(score, dim3(g1), dim3(kChanThreads), smem1, st, p) != cudaSuccess)
      return QMOE_ERR_CUDA;
  }
  if (n_keep > 0) {
    TraceScope ts(st, K_CHAN_SELECT);
    if (launch_pdl(chan_select_kernel, dim3(T), dim3(kSelThreads), smem2, st, p) != cudaSuccess)
      return QMOE_ERR_CUDA;
  }
  s = launch_chan_exact(L.fmt1, L.fmt2, p, g3, smem3, st);
  if (s != QMOE_OK) return s;
  std::lock_guard<std::mutex> lk(g_mu);
  g_stats.last_path = QMOE_PATH_SMALL_M;
  g_stats.row_tiles = 1;
  g_stats.row_tile_tokens = T;
  g_stats.small_launches = n_keep > 0 ? 4 : 3;
  g_stats.grouped_launches = 0;
  return QMOE_OK;
}

}  // extern "C"
