// Device unpack of packed weight codes into m16n8k16 A-operand registers.
// The register order is the one layout.h describes for the packer.
//
// Every produced bf16 is 128 + u (columns k%16 < 8 of a k-step) or
// 128 + beta_hi*u (columns k%16 >= 8; beta_hi = 4 for INT2 and ternary, 1 for
// INT4), u = biased code.  The activation operand carries x / beta and a
// constant-operand MMA removes (128 + bias*beta) * x / beta, so the product is
// exactly sum_k c_k x_k in fp32 accumulation.
#pragma once
#include "device_common.cuh"

namespace qmoe {

constexpr uint32_t kMagic = 0x43004300u;          // bf16 pair (128.0, 128.0)
constexpr uint32_t kBf16Sixteenth = 0x3D803D80u;  // (1/16, 1/16)
constexpr uint32_t kBf16Quarter = 0x3E803E80u;    // (1/4, 1/4)
constexpr uint32_t kBf16_120 = 0x42F042F0u;       // (120, 120)
constexpr uint32_t kBf16_96 = 0x42C042C0u;        // (96, 96)
constexpr uint32_t kBf16One = 0x3F803F80u;        // (1, 1)
constexpr uint32_t kBf16NegZero = 0x80008000u;    // (-0, -0): x + (-0) = x for every x

template <int FMT> struct FmtTraits;
template <> struct FmtTraits<2> {             // INT2: codes -2..1, u = c + 2
  static constexpr int kKUcols = 64;          // K columns per k-unit
  static constexpr int kCodeBytes = 256;      // per 16-row tile per k-unit
  static constexpr int kLaneBytes = 8;
  static constexpr int kBetaHi = 4;
  static constexpr uint32_t kConstLo = 0xC302C302u;  // -(128 + 2)     = -130
  static constexpr uint32_t kConstHi = 0xC308C308u;  // -(128 + 2 * 4) = -136
  static constexpr uint32_t kCodeMulHi = 0x3E803E80u;  // 1/4: (128 + 4u) / 4 = 32 + u
  static constexpr uint32_t kCodeSubHi = 0xC208C208u;  // -(32 + 2) = -34
};
template <> struct FmtTraits<4> {             // INT4: codes -8..7, u = c + 8
  static constexpr int kKUcols = 64;
  static constexpr int kCodeBytes = 512;
  static constexpr int kLaneBytes = 16;
  static constexpr int kBetaHi = 1;
  static constexpr uint32_t kConstLo = 0xC308C308u;  // -(128 + 8) = -136
  static constexpr uint32_t kConstHi = 0xC308C308u;
  static constexpr uint32_t kCodeMulHi = 0x3F803F80u;  // 1
  static constexpr uint32_t kCodeSubHi = 0xC308C308u;  // -136
};
template <> struct FmtTraits<3> {             // ternary: t in {-1,0,1}, digit d = t + 1
  static constexpr int kKUcols = 128;
  static constexpr int kCodeBytes = 416;      // 32 lanes x 13 bytes
  static constexpr int kLaneBytes = 13;
  static constexpr int kBetaHi = 4;
  static constexpr uint32_t kConstLo = 0xC301C301u;  // -(128 + 1)     = -129
  static constexpr uint32_t kConstHi = 0xC304C304u;  // -(128 + 1 * 4) = -132
  static constexpr uint32_t kCodeMulHi = 0x3E803E80u;  // 1/4
  static constexpr uint32_t kCodeSubHi = 0xC204C204u;  // -(32 + 1) = -33
};

// Affine codes (zero point per block): the stored field is u itself, so the
// constant parts to remove are 128 (lo columns) and 128 / beta (hi columns
// after the 1/beta multiplier); as a constant MMA operand on beta-divided
// activations both read -128.
constexpr uint32_t kAffConst = 0xC300C300u;  // -128
template <int FMT>
__host__ __device__ constexpr uint32_t aff_sub_hi() {
  return FmtTraits<FMT>::kBetaHi == 4 ? 0xC200C200u /* -32 */ : 0xC300C300u /* -128 */;
}
// Sum of the activations from the beta-divided ones: a constant operand of 1
// (lo columns) and beta (hi columns).
template <int FMT>
__host__ __device__ constexpr uint32_t sum_const_hi() {
  return FmtTraits<FMT>::kBetaHi == 4 ? 0x40804080u /* 4 */ : kBf16One;
}

// INT2: one lane word (16 codes) -> A registers of two consecutive k-steps.
__device__ __forceinline__ void unpack_int2_word(uint32_t w, uint32_t (&a0)[4], uint32_t (&a1)[4]) {
  const uint32_t v1 = w >> 6, v2 = w >> 12;
  const uint32_t r0 = lop3_and_or(w, 0x00030003u, kMagic);    // 128 + u
  const uint32_t r1 = lop3_and_or(w, 0x000C000Cu, kMagic);    // 128 + 4u
  uint32_t r2 = lop3_and_or(w, 0x00300030u, kMagic);          // 128 + 16u
  const uint32_t r3 = lop3_and_or(v1, 0x00030003u, kMagic);
  const uint32_t r4 = lop3_and_or(v1, 0x000C000Cu, kMagic);
  uint32_t r5 = lop3_and_or(v1, 0x00300030u, kMagic);
  const uint32_t r6 = lop3_and_or(v2, 0x00030003u, kMagic);
  const uint32_t r7 = lop3_and_or(v2, 0x000C000Cu, kMagic);
  r2 = fma_bf16x2(r2, kBf16Sixteenth, kBf16_120);            // -> 128 + u
  r5 = fma_bf16x2(r5, kBf16Quarter, kBf16_96);               // -> 128 + 4u
  a0[0] = r0; a0[1] = r2; a0[2] = r1; a0[3] = r4;
  a1[0] = r3; a1[1] = r6; a1[2] = r5; a1[3] = r7;
}

// INT4: one lane word (8 codes) -> A registers of one k-step.
__device__ __forceinline__ void unpack_int4_word(uint32_t w, uint32_t (&a)[4]) {
  a[0] = lop3_and_or(w, 0x000F000Fu, kMagic);
  a[1] = lop3_and_or(w >> 4, 0x000F000Fu, kMagic);
  a[2] = lop3_and_or(w >> 8, 0x000F000Fu, kMagic);
  a[3] = lop3_and_or(w >> 12, 0x000F000Fu, kMagic);
}

// Ternary byte -> its five base-3 digits placed at bits 0,16,2,18,4.
__host__ __device__ constexpr uint32_t tern_lut_entry(int b) {
  return (uint32_t)(b % 3) | ((uint32_t)(b / 3 % 3) << 16) | ((uint32_t)(b / 9 % 3) << 2) |
         ((uint32_t)(b / 27 % 3) << 18) | ((uint32_t)(b / 81 % 3) << 4);
}

// Ternary: one lane record (13 bytes) -> A registers of 8 k-steps (two 64-blocks).
__device__ __forceinline__ void unpack_tern_record(const uint8_t* rec, const uint32_t* lut,
                                                   uint32_t (&a)[8][4]) {
  uint32_t q[32];
#pragma unroll
  for (int p = 0; p < 6; ++p) {
    const uint32_t la = lut[rec[2 * p]], lb = lut[rec[2 * p + 1]];
    q[5 * p + 0] = lop3_and_or(la, 0x00030003u, kMagic);
    q[5 * p + 1] = lop3_and_or(la, 0x000C000Cu, kMagic);
    q[5 * p + 2] = lop3_and_or(lb, 0x00030003u, kMagic);
    q[5 * p + 3] = lop3_and_or(lb, 0x000C000Cu, kMagic);
    const uint32_t t = lop3_and_or(la, 0x00000030u, kMagic);
    const uint32_t q4 = lop3_and_or(lb << 16, 0x00300000u, t);  // 128 + 16d (both halves)
    q[5 * p + 4] = (p % 2 == 0) ? fma_bf16x2(q4, kBf16Sixteenth, kBf16_120)
                                : fma_bf16x2(q4, kBf16Quarter, kBf16_96);
  }
  const uint32_t lc = lut[rec[12]];
  q[30] = lop3_and_or(lc, 0x00030003u, kMagic);
  q[31] = lop3_and_or(lc, 0x000C000Cu, kMagic);
  constexpr int lo[16] = {0, 2, 4, 5, 7, 10, 12, 14, 15, 17, 20, 22, 24, 25, 27, 30};
  constexpr int hi[16] = {1, 3, 6, 8, 9, 11, 13, 16, 18, 19, 21, 23, 26, 28, 29, 31};
#pragma unroll
  for (int ks = 0; ks < 8; ++ks) {
    a[ks][0] = q[lo[2 * ks]];
    a[ks][1] = q[lo[2 * ks + 1]];
    a[ks][2] = q[hi[2 * ks]];
    a[ks][3] = q[hi[2 * ks + 1]];
  }
}

}  // namespace qmoe
