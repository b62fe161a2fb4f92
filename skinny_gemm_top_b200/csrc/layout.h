// Internal: the packed weight layout shared by the host packer and the device
// unpack.  Each table below is the register order of the device unpack in
// unpack.cuh; the packer writes codes where that unpack reads them.
//
// A 16-row tile's operand for one m16n8k16 MMA k-step is held by 32 lanes:
// lane l = 4g + q owns rows g and g+8 and k columns 2q, 2q+1 (fragment
// registers f = 0 row g, f = 1 row g+8) and 2q+8, 2q+9 (f = 2 row g, f = 3
// row g+8); each register carries two bf16 (half h = 0 low, h = 1 high = the
// next k column).
//
// Unpack trick (magic-number conversion, as in FasterTransformer and Kim et
// al. 2022 "Who Says Elephants Can't Run", written from their description):
// OR-ing a 2- or 4-bit field into the low mantissa bits of the bf16 128.0
// (0x4300) gives 128 + u*2^p for a field at mantissa bit p.  The kernels do
// not subtract per weight: columns k%16 < 8 of every k-step carry 128 + u,
// columns k%16 >= 8 carry 128 + 4u (INT2, ternary) or 128 + u (INT4); the
// activation operand is pre-divided by that column multiplier and the
// constant part is removed by one extra MMA per k-step on a constant operand.
#pragma once
#include <cstdint>

namespace qmoe {

constexpr int kTileRows = 16;
constexpr int kKB = 64;              // K columns per fragment block (one MMA k-step x 4)

// INT2: lane word w (0,1) covers k-steps 2w, 2w+1.  Register m (0..7) takes the
// 2-bit fields at bits [2m, 2m+2) (low half) and [16+2m, 18+2m) (high half).
// (ks offset within the word, fragment register f) of register m:
constexpr int kInt2KsF[8][2] = {{0, 0}, {0, 2}, {0, 1}, {1, 0}, {0, 3}, {1, 2}, {1, 1}, {1, 3}};

// INT4: lane word w (0..3) is k-step w; register j (0..3) = fragment register
// f = j, 4-bit fields at bits [4j, 4j+4) and [16+4j, 20+4j).

// TERNARY: a lane's 13-byte record covers 128 K columns (k-steps 0..7, ks < 4
// in the first 64-block).  Register i (0..31) takes digit (byte, pos) for its
// low and high half; kTernRegBytes[i] = {lo byte, lo pos, hi byte, hi pos}.
// Digit pos p of a byte b is floor(b / 3^p) % 3; byte 12, pos 4 is padding (t = 0).
constexpr int kTernRegDigits[32][4] = {
    {0, 0, 0, 1},  {0, 2, 0, 3},  {1, 0, 1, 1},  {1, 2, 1, 3},  {0, 4, 1, 4},
    {2, 0, 2, 1},  {2, 2, 2, 3},  {3, 0, 3, 1},  {3, 2, 3, 3},  {2, 4, 3, 4},
    {4, 0, 4, 1},  {4, 2, 4, 3},  {5, 0, 5, 1},  {5, 2, 5, 3},  {4, 4, 5, 4},
    {6, 0, 6, 1},  {6, 2, 6, 3},  {7, 0, 7, 1},  {7, 2, 7, 3},  {6, 4, 7, 4},
    {8, 0, 8, 1},  {8, 2, 8, 3},  {9, 0, 9, 1},  {9, 2, 9, 3},  {8, 4, 9, 4},
    {10, 0, 10, 1}, {10, 2, 10, 3}, {11, 0, 11, 1}, {11, 2, 11, 3}, {10, 4, 11, 4},
    {12, 0, 12, 1}, {12, 2, 12, 3}};
// Registers whose columns carry 128 + u (k%16 < 8) and 128 + 4u (k%16 >= 8),
// in k-step order: k-step ks uses f0 = kTernLo[2ks], f1 = kTernLo[2ks+1],
// f2 = kTernHi[2ks], f3 = kTernHi[2ks+1].
constexpr int kTernLo[16] = {0, 2, 4, 5, 7, 10, 12, 14, 15, 17, 20, 22, 24, 25, 27, 30};
constexpr int kTernHi[16] = {1, 3, 6, 8, 9, 11, 13, 16, 18, 19, 21, 23, 26, 28, 29, 31};

// Logical row of tile row r (0..15) in tile t.
inline int logical_row(int row_order, int t, int r) {
  if (row_order == 1) return 16 * t + (r < 8 ? 2 * r : 2 * (r - 8) + 1);
  return 16 * t + r;
}

}  // namespace qmoe
