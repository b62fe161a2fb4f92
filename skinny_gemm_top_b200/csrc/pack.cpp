// Host quantizer + packer and its inverse (C ABI: qmoe_pack_size, qmoe_pack,
// qmoe_unpack_host).
//
// Quantization follows the onnxruntime PR "Enable SM80+ FP16/BF16 mixed
// INT2/INT4 QMoE prefill by default", Current Scope (symmetric, no zero
// points, block 64) and, for ternary, the channel-selection explainer's
// ternary sketch (three values plus one scale per block); the exact scale and
// threshold rules are stated in qmoe.h.
#include <cmath>
#include <cstring>
#include <vector>

#include "qmoe.h"
#include "layout.h"

namespace {

double bf16_to_double(uint16_t b) {
  uint32_t u = (uint32_t)b << 16;
  float f;
  std::memcpy(&f, &u, 4);
  return (double)f;
}

// Nearest bf16 (8 significant bits, ties to even) of a finite double.
uint16_t double_to_bf16(double v) {
  if (v == 0.0) return std::signbit(v) ? 0x8000 : 0;
  int e;
  std::frexp(v, &e);                              // v = m * 2^e, 0.5 <= |m| < 1
  int q = (e < -125 ? -125 : e) - 8;              // unit in the last place
  double r = std::nearbyint(std::ldexp(v, -q));   // default rounding: half to even
  double rv = std::ldexp(r, q);
  float f = (float)rv;                            // exact: rv has <= 8 significant bits
  uint32_t u;
  std::memcpy(&u, &f, 4);
  return (uint16_t)(u >> 16);
}

bool fmt_ok(int fmt) { return fmt == QMOE_INT2 || fmt == QMOE_INT4 || fmt == QMOE_TERNARY; }
bool row_order_ok(int r) { return r == QMOE_ROWS_PLAIN || r == QMOE_ROWS_GATE_UP || r == QMOE_ROWS_KSPLIT; }

qmoe_status check_shape(int fmt, int rows, int K, int block) {
  if (!fmt_ok(fmt)) return QMOE_ERR_INVALID_ARG;
  if (rows <= 0 || K <= 0 || rows % 16 || K % 64) return QMOE_ERR_INVALID_ARG;
  if (block != 64 && block != 128) return QMOE_ERR_UNSUPPORTED;
  if (K % block) return QMOE_ERR_INVALID_ARG;
  if (fmt == QMOE_TERNARY && (block != 64 || K % 128)) return QMOE_ERR_UNSUPPORTED;
  return QMOE_OK;
}

size_t codes_bytes_of(int fmt, int rows, int K) {
  if (fmt == QMOE_TERNARY) return (size_t)rows * (K / 128) * 26;  // 13 bytes per 64 weights
  return (size_t)rows * K * fmt / 8;
}

// Affine: one row-block of INT codes u in [0, 2^bits) (written to c as
// small non-negative values), returns the bf16 scale bits, *z the zero point.
uint16_t quantize_block_affine(int fmt, const uint16_t* w, int B, int8_t* c, uint16_t* z) {
  const int umax = (1 << fmt) - 1;
  double lo = bf16_to_double(w[0]), hi = lo;
  for (int i = 1; i < B; ++i) {
    const double v = bf16_to_double(w[i]);
    lo = std::fmin(lo, v);
    hi = std::fmax(hi, v);
  }
  *z = double_to_bf16(lo);
  const double zd = bf16_to_double(*z);
  const uint16_t sb = double_to_bf16((hi - lo) / (double)umax);
  const double s = bf16_to_double(sb);
  for (int i = 0; i < B; ++i) {
    if (s > 0) {
      double q = std::nearbyint((bf16_to_double(w[i]) - zd) / s);
      if (q < 0) q = 0;
      if (q > umax) q = umax;
      c[i] = (int8_t)q;
    } else {
      c[i] = 0;
    }
  }
  return sb;
}

// Quantize one row-block; writes signed codes c[0..B) and returns the bf16 scale bits.
uint16_t quantize_block(int fmt, const uint16_t* w, int B, int8_t* c) {
  if (fmt == QMOE_TERNARY) {
    double sum_abs = 0.0;
    for (int i = 0; i < B; ++i) sum_abs += std::fabs(bf16_to_double(w[i]));
    double delta = 0.7 * (sum_abs / (double)B);
    double sel = 0.0;
    int cnt = 0;
    for (int i = 0; i < B; ++i) {
      double v = bf16_to_double(w[i]);
      double a = std::fabs(v);
      if (a > delta) {
        c[i] = v > 0 ? 1 : -1;
        sel += a;
        ++cnt;
      } else {
        c[i] = 0;
      }
    }
    return cnt ? double_to_bf16(sel / (double)cnt) : 0;
  }
  const int bits = fmt;
  const int qmin = -(1 << (bits - 1)), qmax = (1 << (bits - 1)) - 1;
  double amax = 0.0;
  for (int i = 0; i < B; ++i) amax = std::fmax(amax, std::fabs(bf16_to_double(w[i])));
  uint16_t sb = double_to_bf16(amax / (double)(1 << (bits - 1)));
  double s = bf16_to_double(sb);
  for (int i = 0; i < B; ++i) {
    if (s > 0) {
      double q = std::nearbyint(bf16_to_double(w[i]) / s);
      if (q < qmin) q = qmin;
      if (q > qmax) q = qmax;
      c[i] = (int8_t)q;
    } else {
      c[i] = 0;
    }
  }
  return sb;
}

// Physical position of logical element (tile row tr of tile t, column k) for INT formats:
// returns (word index within the whole codes array, bit shift).
inline void int_position(int fmt, int row_order, int NT, int t, int tr, int k, size_t* word, int* shift) {
  const int kb = k / 64, kk = k % 64;
  const int ks = kk / 16, kc = kk % 16;
  const int hi8 = kc >= 8;                  // f >> 1
  const int q = (kc % 8) / 2, h = kc % 2;
  const int g = tr % 8, rh = tr / 8;        // f & 1
  const int f = rh | (hi8 << 1);
  const int lane = 4 * g + q;
  const int W = fmt == QMOE_INT2 ? 2 : 4;
  int wi, slot;
  if (fmt == QMOE_INT2) {
    wi = ks / 2;
    int m = -1;
    for (int j = 0; j < 8; ++j)
      if (qmoe::kInt2KsF[j][0] == ks % 2 && qmoe::kInt2KsF[j][1] == f) m = j;
    slot = 2 * m + 16 * h;
  } else {
    wi = ks;
    slot = 4 * f + 16 * h;
  }
  *word = row_order == QMOE_ROWS_KSPLIT ? (((size_t)kb * W + wi) * NT + t) * 32 + lane
                                        : (((size_t)kb * NT + t) * 32 + lane) * W + wi;
  *shift = slot;
}

// Ternary: byte offset of the lane record and digit position for logical element.
inline void tern_position(int NT, int t, int tr, int k, size_t* byte, int* pos) {
  const int kp = k / 128, kk = k % 128;
  const int ks = kk / 16, kc = kk % 16;
  const int hi8 = kc >= 8;
  const int q = (kc % 8) / 2, h = kc % 2;
  const int g = tr % 8, rh = tr / 8;
  const int f = rh | (hi8 << 1);
  const int lane = 4 * g + q;
  const int* list = hi8 ? qmoe::kTernHi : qmoe::kTernLo;
  const int reg = list[2 * ks + rh];
  (void)f;
  const int* d = qmoe::kTernRegDigits[reg];
  const int b = h ? d[2] : d[0];
  *pos = h ? d[3] : d[1];
  *byte = (((size_t)kp * NT + t) * 32 + lane) * 13 + b;
}

const int kPow3[5] = {1, 3, 9, 27, 81};

// Per (tile row, column within the 64/128-column unit): word/byte offset inside
// the unit's tile slab and the shift/digit position.
struct PosTable {
  int off[2][16][128];
  int sh[2][16][128];
  PosTable() {
    for (int which = 0; which < 2; ++which)       // 0: INT2 (64 cols), 1: INT4 (64 cols)
      for (int tr = 0; tr < 16; ++tr)
        for (int k = 0; k < 64; ++k) {
          size_t w;
          int s;
          int_position(which == 0 ? QMOE_INT2 : QMOE_INT4, QMOE_ROWS_PLAIN, 1, 0, tr, k, &w, &s);
          off[which][tr][k] = (int)w;
          sh[which][tr][k] = s;
        }
  }
};
struct TernTable {
  int off[16][128];
  int pos[16][128];
  TernTable() {
    for (int tr = 0; tr < 16; ++tr)
      for (int k = 0; k < 128; ++k) {
        size_t b;
        int p;
        tern_position(1, 0, tr, k, &b, &p);
        off[tr][k] = (int)b;
        pos[tr][k] = p;
      }
  }
};
const PosTable& pos_table() { static PosTable t; return t; }
const TernTable& tern_table() { static TernTable t; return t; }

}  // namespace

extern "C" {

qmoe_status qmoe_pack_size(int fmt, int rows, int K, int block, size_t* codes_bytes,
                           size_t* scales_bytes) {
  qmoe_status st = check_shape(fmt, rows, K, block);
  if (st != QMOE_OK) return st;
  if (codes_bytes) *codes_bytes = codes_bytes_of(fmt, rows, K);
  if (scales_bytes) *scales_bytes = (size_t)rows * (K / block) * 2;
  return QMOE_OK;
}

static qmoe_status pack_impl(int fmt, int row_order, const uint16_t* w, int rows, int K, int block, void* codes,
                      void* scales, void* zeros);

qmoe_status qmoe_pack(int fmt, int row_order, const uint16_t* w, int rows, int K, int block,
                      void* codes, void* scales) {
  return pack_impl(fmt, row_order, w, rows, K, block, codes, scales, nullptr);
}

qmoe_status qmoe_pack_affine(int fmt, int row_order, const uint16_t* w, int rows, int K, int block,
                             void* codes, void* scales, void* zeros) {
  if (fmt == QMOE_TERNARY) return QMOE_ERR_UNSUPPORTED;
  if (!zeros) return QMOE_ERR_INVALID_ARG;
  return pack_impl(fmt, row_order, w, rows, K, block, codes, scales, zeros);
}

static qmoe_status pack_impl(int fmt, int row_order, const uint16_t* w, int rows, int K, int block,
                      void* codes, void* scales, void* zeros) {
  qmoe_status st = check_shape(fmt, rows, K, block);
  if (st != QMOE_OK) return st;
  if (!row_order_ok(row_order)) return QMOE_ERR_INVALID_ARG;
  if (!w || !codes || !scales) return QMOE_ERR_INVALID_ARG;
  const int NT = rows / 16, SB = K / block;
  const size_t cbytes = codes_bytes_of(fmt, rows, K);
  uint8_t* cb = static_cast<uint8_t*>(codes);
  uint32_t* sc = static_cast<uint32_t*>(scales);
  if (fmt == QMOE_TERNARY) {
    // every digit starts as 1 (t = 0), which also fills the padding digit
    std::vector<uint8_t> digits(cbytes * 5, 1);
    const TernTable& tt = tern_table();
#pragma omp parallel for schedule(static)
    for (int t = 0; t < NT; ++t) {
      std::vector<int8_t> c(block);
      for (int tr = 0; tr < 16; ++tr) {
        const int lr = qmoe::logical_row(row_order, t, tr);
        for (int b = 0; b < SB; ++b) {
          uint16_t s = quantize_block(fmt, w + (size_t)lr * K + (size_t)b * block, block, c.data());
          uint32_t& slot = sc[((size_t)b * NT + t) * 8 + (tr % 8)];
          if (tr < 8) slot = (slot & 0xFFFF0000u) | s; else slot = (slot & 0xFFFFu) | ((uint32_t)s << 16);
          for (int i = 0; i < block; ++i) {
            const int k = b * block + i;
            const size_t unit = ((size_t)(k / 128) * NT + t) * 32 * 13;
            digits[(unit + tt.off[tr][k % 128]) * 5 + tt.pos[tr][k % 128]] = (uint8_t)(c[i] + 1);
          }
        }
      }
    }
#pragma omp parallel for schedule(static)
    for (size_t i = 0; i < cbytes; ++i) {
      int v = 0;
      for (int p = 0; p < 5; ++p) v += digits[i * 5 + p] * kPow3[p];
      cb[i] = (uint8_t)v;
    }
    return QMOE_OK;
  }
  std::memset(codes, 0, cbytes);
  uint32_t* cw = static_cast<uint32_t*>(codes);
  uint32_t* zc = static_cast<uint32_t*>(zeros);
  const int bias = zeros ? 0 : 1 << (fmt - 1);  // stored field: u (affine) or c + 2^(bits-1)
  const PosTable& pt = pos_table();
  const int which = fmt == QMOE_INT2 ? 0 : 1;
  const int W = fmt == QMOE_INT2 ? 2 : 4;
#pragma omp parallel for schedule(static)
  for (int t = 0; t < NT; ++t) {
    std::vector<int8_t> c(block);
    for (int tr = 0; tr < 16; ++tr) {
      const int lr = qmoe::logical_row(row_order, t, tr);
      for (int b = 0; b < SB; ++b) {
        uint16_t z = 0;
        uint16_t s = zeros ? quantize_block_affine(fmt, w + (size_t)lr * K + (size_t)b * block, block, c.data(), &z)
                           : quantize_block(fmt, w + (size_t)lr * K + (size_t)b * block, block, c.data());
        uint32_t& slot = sc[((size_t)b * NT + t) * 8 + (tr % 8)];
        if (tr < 8) slot = (slot & 0xFFFF0000u) | s; else slot = (slot & 0xFFFFu) | ((uint32_t)s << 16);
        if (zeros) {
          uint32_t& zs = zc[((size_t)b * NT + t) * 8 + (tr % 8)];
          if (tr < 8) zs = (zs & 0xFFFF0000u) | z; else zs = (zs & 0xFFFFu) | ((uint32_t)z << 16);
        }
        for (int i = 0; i < block; ++i) {
          const int k = b * block + i;
          const int off = pt.off[which][tr][k % 64];  // lane * W + word within the 64-column unit
          const size_t idx = row_order == QMOE_ROWS_KSPLIT
                                 ? (((size_t)(k / 64) * W + off % W) * NT + t) * 32 + off / W
                                 : ((size_t)(k / 64) * NT + t) * 32 * W + off;
          cw[idx] |= (uint32_t)(c[i] + bias) << pt.sh[which][tr][k % 64];
        }
      }
    }
  }
  return QMOE_OK;
}

qmoe_status qmoe_unpack_host(int fmt, int row_order, const void* codes, const void* scales, int rows,
                             int K, int block, int8_t* codes_out, uint16_t* scales_out) {
  qmoe_status st = check_shape(fmt, rows, K, block);
  if (st != QMOE_OK) return st;
  if (!row_order_ok(row_order)) return QMOE_ERR_INVALID_ARG;
  if ((codes_out && !codes) || (scales_out && !scales)) return QMOE_ERR_INVALID_ARG;
  const int NT = rows / 16, SB = K / block;
  for (int t = 0; t < NT; ++t)
    for (int tr = 0; tr < 16; ++tr) {
      const int lr = qmoe::logical_row(row_order, t, tr);
      if (scales_out) {
        const uint32_t* sc = static_cast<const uint32_t*>(scales);
        for (int b = 0; b < SB; ++b) {
          uint32_t v = sc[((size_t)b * NT + t) * 8 + (tr % 8)];
          scales_out[(size_t)lr * SB + b] = (uint16_t)(tr < 8 ? (v & 0xFFFF) : (v >> 16));
        }
      }
      if (!codes_out) continue;
      for (int k = 0; k < K; ++k) {
        int8_t c;
        if (fmt == QMOE_TERNARY) {
          size_t byte;
          int pos;
          tern_position(NT, t, tr, k, &byte, &pos);
          int v = static_cast<const uint8_t*>(codes)[byte];
          c = (int8_t)((v / kPow3[pos]) % 3 - 1);
        } else {
          size_t word;
          int shift;
          int_position(fmt, row_order, NT, t, tr, k, &word, &shift);
          uint32_t v = static_cast<const uint32_t*>(codes)[word];
          c = (int8_t)((int)((v >> shift) & ((1u << fmt) - 1)) - (1 << (fmt - 1)));
        }
        codes_out[(size_t)lr * K + k] = c;
      }
    }
  return QMOE_OK;
}


}  // extern "C"

// ---------------------------------------------------------------------------
// Channel layer (top-k channel-selective read): one record per channel holding
// its gate row, up row and down column, and a 2-bit ternary sketch of the
// rotated gate and up rows.  Layouts are stated in qmoe.h.
namespace {

bool chan_fmt_ok(int f) { return f == QMOE_INT2 || f == QMOE_INT4; }

qmoe_status chan_check(int fmt1, int fmt2, int H, int block) {
  if (!chan_fmt_ok(fmt1) || !chan_fmt_ok(fmt2)) return QMOE_ERR_INVALID_ARG;
  if (block != 64 && block != 128) return QMOE_ERR_UNSUPPORTED;
  if (H < 512 || H > 2048 || (H & (H - 1))) return QMOE_ERR_UNSUPPORTED;
  return QMOE_OK;
}

size_t align16(size_t v) { return (v + 15) / 16 * 16; }

// Ternary rule of quantize_block on float64 inputs (the rotated rows are not bf16).
uint16_t ternary_block_f64(const double* w, int B, int8_t* c) {
  double sum_abs = 0.0;
  for (int i = 0; i < B; ++i) sum_abs += std::fabs(w[i]);
  const double delta = 0.7 * (sum_abs / (double)B);
  double sel = 0.0;
  int cnt = 0;
  for (int i = 0; i < B; ++i) {
    const double a = std::fabs(w[i]);
    if (a > delta) {
      c[i] = w[i] > 0 ? 1 : -1;
      sel += a;
      ++cnt;
    } else {
      c[i] = 0;
    }
  }
  return cnt ? double_to_bf16(sel / (double)cnt) : 0;
}

// In-place fast Walsh-Hadamard transform in Sylvester order, then one scaling
// by 1/sqrt(n).  On bf16 inputs every partial sum is exact in float64.
void fwht_scaled(double* v, int n) {
  for (int len = 1; len < n; len <<= 1)
    for (int i = 0; i < n; i += 2 * len)
      for (int j = i; j < i + len; ++j) {
        const double a = v[j], b = v[j + len];
        v[j] = a + b;
        v[j + len] = a - b;
      }
  const double r = 1.0 / std::sqrt((double)n);
  for (int i = 0; i < n; ++i) v[i] *= r;
}

// Packs `n` codes (signed c, stored as c + bias) of `bits` bits little-endian into `out`.
void put_codes(uint8_t* out, const int8_t* c, int n, int bits, int bias) {
  uint32_t* wd = reinterpret_cast<uint32_t*>(out);
  const int per = 32 / bits;
  std::memset(out, 0, (size_t)n * bits / 8);
  for (int i = 0; i < n; ++i) wd[i / per] |= (uint32_t)(c[i] + bias) << ((i % per) * bits);
}

}  // namespace

extern "C" {

qmoe_status qmoe_chan_sizes(int fmt1, int fmt2, int H, int block, size_t* record_bytes, size_t* sketch_bytes) {
  qmoe_status st = chan_check(fmt1, fmt2, H, block);
  if (st != QMOE_OK) return st;
  if (record_bytes) *record_bytes = align16((size_t)2 * H * fmt1 / 8 + (size_t)H * fmt2 / 8 + 3 * (size_t)(H / block) * 2);
  if (sketch_bytes) *sketch_bytes = align16((size_t)2 * H / 4 + 2 * (size_t)(H / 128) * 2);
  return QMOE_OK;
}

qmoe_status qmoe_chan_pack(int fmt1, int fmt2, int H, int I, int block, const uint16_t* w1, const uint16_t* w2,
                           const float* signs, void* records, void* sketch, float* dn) {
  size_t R = 0, SK = 0;
  qmoe_status st = qmoe_chan_sizes(fmt1, fmt2, H, block, &R, &SK);
  if (st != QMOE_OK) return st;
  if (I <= 0 || !w1 || !w2 || !records || (sketch && !signs)) return QMOE_ERR_INVALID_ARG;
  if (sketch)
    for (int i = 0; i < H; ++i)
      if (signs[i] != 1.0f && signs[i] != -1.0f) return QMOE_ERR_INVALID_ARG;
  const int SB = H / block, SKB = H / 128;
  const size_t off_u = (size_t)H * fmt1 / 8, off_d = 2 * off_u, off_s = off_d + (size_t)H * fmt2 / 8;
  uint8_t* rec = static_cast<uint8_t*>(records);
  uint8_t* sk = static_cast<uint8_t*>(sketch);
  bool bad = false;
#pragma omp parallel for schedule(static)
  for (int j = 0; j < I; ++j) {
    std::vector<int8_t> c(H);
    std::vector<uint16_t> col(H);
    std::vector<double> rot(H);
    uint8_t* r = rec + (size_t)j * R;
    std::memset(r, 0, R);
    uint16_t* sc = reinterpret_cast<uint16_t*>(r + off_s);  // gate, up, down scales
    for (int which = 0; which < 2; ++which) {               // 0: gate row 2j, 1: up row 2j+1
      const uint16_t* row = w1 + (size_t)(2 * j + which) * H;
      for (int b = 0; b < SB; ++b) sc[which * SB + b] = quantize_block(fmt1, row + (size_t)b * block, block, &c[(size_t)b * block]);
      put_codes(r + which * off_u, c.data(), H, fmt1, 1 << (fmt1 - 1));
      if (sk) {
        for (int i = 0; i < H; ++i) rot[i] = bf16_to_double(row[i]) * (double)signs[i];
        fwht_scaled(rot.data(), H);
        uint8_t* s = sk + (size_t)j * SK;
        uint16_t* ss = reinterpret_cast<uint16_t*>(s + (size_t)H / 2);
        for (int b = 0; b < SKB; ++b) ss[which * SKB + b] = ternary_block_f64(&rot[(size_t)b * 128], 128, &c[(size_t)b * 128]);
        put_codes(s + which * (size_t)H / 4, c.data(), H, 2, 2);
      }
    }
    for (int i = 0; i < H; ++i) col[i] = w2[(size_t)i * I + j];
    double ss = 0.0;
    for (int b = 0; b < SB; ++b) {
      const uint16_t s = quantize_block(fmt2, &col[(size_t)b * block], block, &c[(size_t)b * block]);
      sc[2 * SB + b] = s;
      const double sd = bf16_to_double(s);
      for (int i = 0; i < block; ++i) {
        const double v = (double)c[(size_t)b * block + i] * sd;
        ss += v * v;
      }
    }
    put_codes(r + off_d, c.data(), H, fmt2, 1 << (fmt2 - 1));
    if (dn) dn[j] = (float)std::sqrt(ss);
    if (!std::isfinite(ss)) bad = true;
  }
  return bad ? QMOE_ERR_INVALID_ARG : QMOE_OK;
}

}  // extern "C"
