/*
 * qmoe.h - C ABI of the B200 (sm_100a) weight-only low-bit quantized MoE
 * expert matmul.
 *
 * What it computes (sources by page and section):
 *   - onnxruntime PR "Enable SM80+ FP16/BF16 mixed INT2/INT4 QMoE prefill by
 *     default", Description / Current Scope: top-k routing, rows expanded by
 *     expert, INT2 (or INT4) FC1 with interleaved fused SwiGLU and expert bias,
 *     INT4 FC2, top-k weighted finalize with FC2 bias; symmetric block
 *     quantization, block 64, no zero points; row tiling under a scratch
 *     budget with an error when even one row does not fit.
 *   - "The QMoE sub-1-bit expert kernel is a GEMV ..." note: the inner loop
 *     over the tokens that share an expert (one pass over the weights serves
 *     all of them).
 *   - "Skip MoE channels ... top-k channel selection" explainer, ternary
 *     sketch paragraph: ternary {-1,0,1} codes with one scale per block.
 *   - MLX issue "2-bit quantized_matmul loses its size advantage over 4-bit
 *     at M >= 3": the single quantized linear y = x W^T, group 128, M = 1..32.
 *
 * Conventions for every entry point:
 *   - Return a qmoe_status; nothing aborts, no C++ exception crosses the ABI.
 *   - Arguments are validated before any launch; a rejected call launches
 *     nothing and writes nothing.
 *   - Device entry points take device pointers and a cudaStream_t passed as
 *     void* (NULL = legacy default stream); they enqueue work and return
 *     without synchronising.  Host entry points (pack, unpack, sizes) are
 *     synchronous and touch host memory only.
 *   - All buffers are owned by the caller.  Device entry points allocate no
 *     memory: scratch comes from the caller's workspace (ws, ws_bytes).
 *   - Errors found on the device (a bounded wait that ran out) are recorded
 *     in a device status word, read back by qmoe_get_stats().
 *   - bf16 values are passed as uint16_t bit patterns.
 */
#ifndef QMOE_H
#define QMOE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  QMOE_OK = 0,
  QMOE_ERR_INVALID_ARG = 1,   /* null pointer, bad size, bad enum value     */
  QMOE_ERR_UNSUPPORTED = 2,   /* valid but outside what the kernels handle  */
  QMOE_ERR_SCRATCH = 3,       /* workspace too small even for one token row */
  QMOE_ERR_CUDA = 4,          /* a CUDA runtime call failed                 */
  QMOE_ERR_TIMEOUT = 5,       /* a device-side bounded wait ran out         */
  QMOE_ERR_STATIC_SCRATCH = 6 /* needs more than QMOE_STATIC_SCRATCH_BYTES  */
} qmoe_status;

/* Weight code formats. */
typedef enum {
  QMOE_INT2 = 2,              /* symmetric, codes -2..1, 16 codes per u32          */
  QMOE_TERNARY = 3,           /* codes -1, 0, 1, 5 trits per byte                   */
  QMOE_INT4 = 4               /* symmetric, codes -8..7, 8 codes per u32            */
} qmoe_fmt;

/* Row order (and code layout) of a packed matrix.
 *   GATE_UP: FC1, whose logical rows interleave gate and up (row 2j = gate j,
 *     row 2j+1 = up j: the fused SwiGLU layout of the onnxruntime PR, Current
 *     Scope "swiglu_fusion=1").
 *   PLAIN:   rows in order (the single linear).
 *   KSPLIT:  rows in order, codes laid out so that a narrow range of K columns
 *     of all rows is one contiguous run (FC2 of a MoE layer, whose K = I is
 *     split across blocks by the decode kernel; see the layout below). */
typedef enum { QMOE_ROWS_PLAIN = 0, QMOE_ROWS_GATE_UP = 1, QMOE_ROWS_KSPLIT = 2 } qmoe_row_order;

/* Expert-compute path selection; AUTO picks per expert by its token count. */
typedef enum { QMOE_PATH_AUTO = 0, QMOE_PATH_SMALL_M = 1, QMOE_PATH_GROUPED = 2 } qmoe_path;

/* ------------------------------------------------------------------------
 * Packed weight format (defined by this library).
 *
 * Quantization of a bf16 matrix W[rows, K] with block size B along K:
 *   INT (bits b in {2,4}): s = bf16_rne(max|w| / 2^(b-1)) per (row, block);
 *     c = clamp(rne(w / s), -2^(b-1), 2^(b-1)-1) computed in double; s == 0
 *     gives c = 0.  Stored code u = c + 2^(b-1).
 *   TERNARY (B = 64): delta = 0.7 * (sum|w| / 64) in double (sum in K order);
 *     t = sign(w) if |w| > delta else 0; s = bf16_rne(mean |w| over the kept
 *     weights), 0 if none.  Stored digit d = t + 1, base 3, 5 digits per byte.
 *
 * Physical layout (rows % 16 == 0).  Rows form tiles of 16 (NT = rows/16);
 * tile row r of tile T is logical row 16T+r (PLAIN) or, for GATE_UP,
 * 16T + 2r (r < 8, gate 8T+r) / 16T + 2(r-8) + 1 (r >= 8, up 8T+r-8).
 * Each lane l (g = l/4, q = l%4) of a 32-lane warp owns the operand
 * fragment of an m16n8k16 MMA: rows g and g+8, k = 16ks + 2q + {0,1} and
 * 16ks + 2q + 8 + {0,1}.
 *   INT2/INT4 codes (GATE_UP, PLAIN): [K/64][NT][32 lanes][W u32], W = 2
 *     (INT2) or 4 (INT4); word w of a lane covers k-steps 2w, 2w+1 (INT2) or
 *     k-step w (INT4) of the 64 columns.  bytes = rows*K*bits/8.  Bit
 *     positions inside a lane's words follow the register order of the
 *     kernels' unpack; qmoe_unpack_host() inverts it.
 *   INT2/INT4 codes (KSPLIT): the same words, slab-major:
 *     [K/64][W][NT][32 lanes][1 u32] = one slab of 32 (INT2) or 16 (INT4)
 *     columns of all rows per (K/64, w), contiguous.
 *   TERNARY codes: [K/128][NT][32 lanes][13 bytes] for every row order (a
 *     lane record is already one slab of 128 columns); bytes = rows*K*13/64
 *     (1.625 bits per weight).
 *   Scales: [K/B][NT][8 u32], u32 g = s(row g) | s(row g+8) << 16 (bf16 bits);
 *     bytes = rows*(K/B)*2.
 * A layer's experts are packed one after another with the same strides.
 * ---------------------------------------------------------------------- */

/* Sizes of one packed matrix.  Requires rows % 16 == 0, K % 64 == 0,
 * block in {64, 128} (ternary: 64, K % 128 == 0; block 128: K % 128 == 0). */
qmoe_status qmoe_pack_size(int fmt, int rows, int K, int block,
                           size_t* codes_bytes, size_t* scales_bytes);

/* Quantize and pack one bf16 matrix w[rows, K] (row-major, host memory) into
 * codes / scales (host memory, sizes from qmoe_pack_size).  Deterministic. */
qmoe_status qmoe_pack(int fmt, int row_order, const uint16_t* w, int rows, int K, int block,
                      void* codes, void* scales);

/* Affine (asymmetric) variant, INT2 / INT4 only: one bf16 scale s and one
 * bf16 zero point z per block, unsigned codes u in [0, 2^bits), w_hat = s*u
 * + z (the (scales, biases) format of the MLX issue "2-bit
 * quantized_matmul loses its size advantage over 4-bit at M >= 3", repro).
 * z = bf16_rne(min w), s = bf16_rne((max w - min w) / (2^bits - 1)), u =
 * clamp(rne((w - z) / s)), all per block in float64 (s == 0 gives u = 0).
 * The codes use the layout and bit positions of qmoe_pack (the stored field
 * is u); zeros use the layout of the scales (sizes from qmoe_pack_size).
 * QMOE_ERR_UNSUPPORTED for ternary. */
qmoe_status qmoe_pack_affine(int fmt, int row_order, const uint16_t* w, int rows, int K, int block,
                             void* codes, void* scales, void* zeros);

/* Inverse of the layout (host): logical signed codes [rows, K] (int8) and
 * bf16 scales [rows, K/block].  Either output may be NULL.  For affine codes
 * codes_out holds u - 2^(bits-1); zeros unpack like scales (pass them as
 * `scales`). */
qmoe_status qmoe_unpack_host(int fmt, int row_order, const void* codes, const void* scales,
                             int rows, int K, int block, int8_t* codes_out, uint16_t* scales_out);

/* One quantized weight set: n matrices of the same shape packed back to back
 * (matrix e at codes + e*codes_bytes, scales + e*scales_bytes) with the row
 * order they were packed with, optional bf16 bias [n][rows] in logical row
 * order (NULL = none), and for affine codes (qmoe_pack_affine) the zero
 * points (NULL = symmetric codes; same layout and strides as the scales).
 * Device pointers, 16-byte aligned. */
typedef struct {
  int fmt;
  int block;
  int row_order;
  const void* codes;
  const void* scales;
  const uint16_t* bias;
  const void* zeros;
} qmoe_weights;

/* Dequantize n_mats packed matrices (device): out_f32[e][rows][K] = c*s
 * (exact; affine: f32_rne(s*u + z)) and/or out_bf16 = bf16_rne(c*s) (affine:
 * bf16_rne(s*u + z), one rounding), logical row order (w->row_order gives
 * the packing).  Debug and parity entry point; uses the hot kernels' unpack
 * routines. */
qmoe_status qmoe_dequant(const qmoe_weights* w, int rows, int K, int n_mats, float* out_f32,
                         uint16_t* out_bf16, void* stream);

/* Routing (device): logits fp32 [T, E] -> ids int32 [T, k] (descending logit,
 * ties to the lower index, -0 equal to +0), weights fp32 [T, k] (softmax over
 * the k selected logits), perm int32 [T*k] (flat index t*k+s at each
 * expert-sorted position; stable), offsets int32 [E+1].  E <= 256,
 * 1 <= k <= min(E, 32).  Logits must be finite.
 * Top-k routing, then "expert maps" and rows expanded by expert: onnxruntime
 * PR "Enable SM80+ FP16/BF16 mixed INT2/INT4 QMoE prefill by default",
 * Description.
 * The routing kernels are the ones qmoe_forward runs: for a decode batch
 * (T <= 8 and T*k <= 64) one CTA with the in-kernel routing of the decode
 * layer kernel; otherwise the two-launch general routing (per-chunk top-k and
 * counts, then the stable scatter), whose per-chunk counts live in ws.
 * ws: device scratch of at least qmoe_route_workspace_size() bytes, 16-byte
 * aligned (NULL allowed when that size is 0); QMOE_ERR_SCRATCH if smaller. */
qmoe_status qmoe_route_workspace_size(int T, int E, int k, size_t* bytes);
qmoe_status qmoe_route(const float* logits, int T, int E, int k, int32_t* ids, float* weights,
                       int32_t* perm, int32_t* offsets, void* ws, size_t ws_bytes, void* stream);

/* One MoE layer.  fc1: E + n_shared matrices [2I, H] packed with
 * QMOE_ROWS_GATE_UP (shared experts after the routed ones); bias [.][2I].
 * fc2: E + n_shared matrices [H, I] packed with QMOE_ROWS_KSPLIT; bias [.][H].
 * Other row orders are rejected (QMOE_ERR_INVALID_ARG).
 * H % 64 == 0, I % 64 == 0; E <= 256; shared experts get every token with
 * weight 1.  max_row_tile bounds the tokens per row tile (0 = none). */
typedef struct {
  int H, I, E, k, n_shared;
  qmoe_weights fc1;
  qmoe_weights fc2;
  int path;
  int max_row_tile;
} qmoe_layer;

/* Workspace for qmoe_forward over T tokens without row tiling. */
qmoe_status qmoe_workspace_size(const qmoe_layer* layer, int T, size_t* bytes);

/* y[T, H] bf16 = MoE(x[T, H] bf16, logits[T, E] fp32).  With ws_bytes below
 * qmoe_workspace_size(T), tokens are processed in row tiles (halved until the
 * tile's workspace fits, explicit partial last tile); QMOE_ERR_SCRATCH when
 * one row does not fit.  ws must be 256-byte aligned, x 16-byte aligned, y
 * 8-byte aligned.
 * A decode batch (T <= 8, T*k <= 64, H <= 2112) runs as one kernel that
 * routes in its prologue and splits every selected expert's intermediate
 * dimension across the SMs; its blocks never wait for one another.  Their
 * partial outputs are summed with fp32 atomic adds, so the summation order,
 * and with it the last bit of an output, can differ between runs.  Larger
 * batches run routing, expert and combine kernels in sequence; their results
 * do not depend on scheduling.  No part of ws needs any initial contents. */
qmoe_status qmoe_forward(const qmoe_layer* layer, const uint16_t* x, const float* logits, int T,
                         uint16_t* y, void* ws, size_t ws_bytes, void* stream);

/* qmoe_forward without a caller workspace, allocating nothing.  The pages
 * describe no counterpart: this is a deployment entry point for callers that
 * own no device allocator or must not call cudaMalloc/cudaFree inside a step
 * (they synchronise the device and can fail under memory pressure).
 * Scratch: a fixed device array of QMOE_STATIC_SCRATCH_BYTES inside the
 * library, one per device.  Arguments and results as qmoe_forward (x, logits,
 * y device pointers; stream a cudaStream_t or NULL).  Errors: those of
 * qmoe_forward, and QMOE_ERR_STATIC_SCRATCH when qmoe_workspace_size(T)
 * exceeds the array (no row tiling; nothing is launched).  The first call on
 * a device resolves the array's address (cudaGetSymbolAddress with that
 * device current) and can load the library's device code: make it before any
 * stream capture.  No scratch value needs to start at any particular value:
 * each call clears what it reads before writing it.  Calls that overlap in
 * time on one device share the array and race: serialise them. */
#define QMOE_STATIC_SCRATCH_BYTES (8u << 20)
qmoe_status qmoe_forward_static(const qmoe_layer* layer, const uint16_t* x, const float* logits, int T,
                                uint16_t* y, void* stream);

/* Single quantized linear y[M, N] bf16 = x[M, K] bf16 @ dequant(W)[N, K]^T,
 * W packed PLAIN (other row orders: QMOE_ERR_INVALID_ARG).  M >= 1.
 * ws (device, 256-byte aligned, contents irrelevant): with at least
 * qmoe_linear_workspace_size() bytes, a shape with few 16-row tiles (such as
 * N = 5120) is split along K over more SMs, its partial sums accumulated in ws
 * in fp32 (their order varies from run to run); with less (or NULL) it runs
 * unsplit.  The MLX issue "2-bit quantized_matmul loses its size advantage
 * over 4-bit at M >= 3", table: K = 5120 -> N = 17408 / 248320, group 128. */
qmoe_status qmoe_linear_workspace_size(int N, int K, int M, size_t* bytes);
qmoe_status qmoe_linear(const qmoe_weights* w, int N, int K, const uint16_t* x, int M,
                        uint16_t* y, void* ws, size_t ws_bytes, void* stream);

/* ---- Top-k channel-selective MoE layer ----
 * "Skip MoE channels for up to 2.69x faster MoE blocks - top-k channel
 * selection" explainer: sketch paragraph (each gate and up row rotated by a
 * randomized Hadamard transform, then three values plus one scale per block
 * of 128 weights), scoring paragraph (score = router weight x down-column
 * norm x |estimated activation|; channels of all routed experts compete in
 * one top-k; the winners are read in full and computed exactly),
 * choosing-k paragraph (a fixed number of channels per token).
 *
 * Channel record, one per expert channel j (record_bytes, a multiple of 16):
 * gate row j (FC1 row 2j) codes, H * fmt1 / 8 bytes; up row j (FC1 row 2j+1)
 * codes; down column j (W2[:, j]) codes, H * fmt2 / 8 bytes; then bf16
 * scales: gate [H / block], up [H / block], down [H / block]; zero padding.
 * Codes are symmetric INT2 / INT4 (stored c + 2^(bits-1)), code i of a row at
 * bit i * bits of its little-endian bytes.  The down column is quantized in
 * blocks of `block` rows (qmoe_pack's FC2 blocks run along I instead), so
 * that one channel is one contiguous read.
 * Sketch record, one per routed expert channel (sketch_bytes, a multiple of
 * 16): the trits t of the rotated gate row, then of the rotated up row, 2 bits
 * each (stored t + 2), same bit order; then bf16 scales, gate [H / 128] and
 * up [H / 128].  Rotation: v' = Had_H (d * v) / sqrt(H), Had_H the Sylvester
 * Hadamard matrix, d the caller's signs.  Ternary rule per block of 128:
 * threshold 0.7 * mean|v'|, t = sign(v') where |v'| exceeds it, else 0;
 * scale = bf16 of the mean |v'| above the threshold (0 if none).
 * dn[j]: fp32 of the Euclidean norm of the dequantized down column j.
 * fmt1, fmt2: QMOE_INT2 or QMOE_INT4 (else QMOE_ERR_INVALID_ARG); block 64 or
 * 128, H a power of two in 512..2048 (else QMOE_ERR_UNSUPPORTED). */
qmoe_status qmoe_chan_sizes(int fmt1, int fmt2, int H, int block, size_t* record_bytes,
                            size_t* sketch_bytes);

/* Host: quantize and pack the I channels of one expert.  w1 [2I, H] bf16 (row
 * 2j gate j, row 2j+1 up j), w2 [H, I] bf16.  records: I * record_bytes.
 * sketch (I * sketch_bytes) and dn (I floats) may be NULL: shared experts
 * need neither.  signs [H]: +1.0f or -1.0f (else QMOE_ERR_INVALID_ARG),
 * needed with a sketch.  QMOE_ERR_INVALID_ARG also for a non-finite norm. */
qmoe_status qmoe_chan_pack(int fmt1, int fmt2, int H, int I, int block, const uint16_t* w1,
                           const uint16_t* w2, const float* signs, void* records, void* sketch,
                           float* dn);

/* A channel layer on the device.  records: [E + n_shared][I] channel records
 * (shared experts after the routed ones), 16-byte aligned; sketch: [E][I]
 * sketch records, 16-byte aligned; dn: [E][I]; signs: [H], 16-byte aligned,
 * the signs the sketch was built with.  1 <= k <= 8, k <= E <= 256, k * I <= 32768. */
typedef struct {
  int H, I, E, k, n_shared;
  int fmt1, fmt2, block;
  const void* records;
  const void* sketch;
  const float* dn;
  const float* signs;
} qmoe_chan_layer;

/* Workspace of qmoe_chan_forward for T tokens and n_keep channels per token. */
qmoe_status qmoe_chan_workspace_size(const qmoe_chan_layer* layer, int T, int n_keep, size_t* bytes);

/* y[T, H] bf16 = for each token, the sum over its n_keep best channels (among
 * the k * I channels of its routed experts, flat index s * I + j with s the
 * routing slot; score descending, ties to the lower index) of
 * w_{t,s} * silu(g_j) * u_j * W2_e[:, j] with g_j, u_j the exact gate and up
 * products, plus the shared experts in full (weight 1).  Routing as
 * qmoe_route: top-k of the fp32 logits (finite), ties to the lower expert,
 * softmax over the k.  1 <= T <= 8, 0 <= n_keep <= k * I; x 16-byte aligned.
 * Scores are computed in fp32 and ranked on their fp32 values.
 * Optional device outputs (NULL to skip, 4-byte aligned): sel[T][n_keep]
 * int32, the selected flat indices in ascending order; scores[T][k * I]
 * fp32.  ws: device, 256-byte aligned, at least qmoe_chan_workspace_size()
 * bytes (else QMOE_ERR_SCRATCH); no initial contents needed.  Three kernels:
 * scoring (routing, rotation, sketch products), selection (one block per
 * token; skipped when n_keep = 0), exact read and combine.  Partial outputs
 * are summed with fp32 atomic adds, so the last bit of y can vary between
 * runs.  A bounded wait that runs out sets QMOE_DEVICE_TIMEOUT and leaves y
 * unwritten. */
qmoe_status qmoe_chan_forward(const qmoe_chan_layer* layer, const uint16_t* x, const float* logits,
                              int T, int n_keep, uint16_t* y, int32_t* sel, float* scores, void* ws,
                              size_t ws_bytes, void* stream);

/* Per-launch GPU timing (tracing).  After qmoe_trace_start(cap) every kernel
 * the library launches - also while the stream is being captured into a CUDA
 * graph - is bracketed by CUDA events, up to cap launches; qmoe_trace_stop()
 * ends recording.  qmoe_trace_read() synchronizes the device and returns per
 * recorded launch its kernel id (qmoe_kernel_name) and duration in ms; for a
 * launch replayed from a graph, the duration of its latest execution. */
qmoe_status qmoe_trace_start(int cap);
qmoe_status qmoe_trace_stop(void);
qmoe_status qmoe_trace_read(int cap, int* n, int* kernel_ids, float* ms);
const char* qmoe_kernel_name(int kernel_id);

typedef struct {
  int last_path;          /* path the last qmoe_forward / qmoe_linear took  */
  int row_tiles;          /* row tiles of the last qmoe_forward             */
  int row_tile_tokens;    /* tokens per full row tile                       */
  int small_launches;     /* small-M expert kernels launched by the last call */
  int grouped_launches;   /* grouped (tcgen05) kernels launched by the last call */
  uint32_t device_status; /* OR of device error flags since the last clear  */
} qmoe_stats;

/* Host-side stats of the last call plus the device status word (this call
 * synchronises the current device to read it). */
qmoe_status qmoe_get_stats(qmoe_stats* out);
qmoe_status qmoe_clear_status(void);
const char* qmoe_status_str(int status);

/* Device status flags (qmoe_stats.device_status). */
#define QMOE_DEVICE_TIMEOUT 1u     /* a bounded device-side wait gave up         */
#define QMOE_DEVICE_BAD_SEGMENT 2u /* a work table overflowed; its excess skipped */

/* Test hook: fault injection for the decode-layer kernel (the qmoe_forward
 * path of T <= 8 tokens) and the exact-read kernel of qmoe_chan_forward.
 * wait_limit_ns bounds every wait of those kernels (0: the default, 2 s).
 * inject = 1 makes one thread of every CTA wait on a barrier that nothing
 * arrives at: the wait runs out, the CTA drops its part of the output, sets
 * QMOE_DEVICE_TIMEOUT and returns, and y is left as it was.  The library stays usable: after qmoe_test_set_fault(0, 0) and
 * qmoe_clear_status() the next call is correct.  Process-wide setting, read
 * at launch; not thread-safe.  QMOE_ERR_INVALID_ARG for another inject. */
qmoe_status qmoe_test_set_fault(int inject, unsigned long long wait_limit_ns);

#ifdef __cplusplus
}
#endif
#endif /* QMOE_H */
