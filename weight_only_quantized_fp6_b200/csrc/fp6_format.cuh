// fp6_format.cuh -- FP6 (e3m2) encoding on the device: the packed layout,
// the bit-splice rebuild of fp16 weights, and the quantizer's rounding.
//
// e3m2 code (low 6 bits of a byte): s = bit 5, e = bits 4..2 (bias 3),
// m = bits 1..0.  Value (-1)^s 2^(e-3)(1+m/4), or (-1)^s 2^-2 (m/4) for e = 0.
//
// Rebuild identity.  Put s at fp16 bit 15 and the five bits e,m at fp16 bits
// 12..8: the fp16 exponent field then equals e and the top two mantissa bits
// equal m, so the half is exactly decode(c) * 2^-12 -- e = 0 codes land on
// fp16 subnormals with the right value.  The layer multiplies by 2^12 once,
// folded into the per-row scale in the fp32 epilogue.
//
// Split (TC-FPx article, "kernel solution redesign": each 6-bit weight is cut
// into a 2-bit and a 4-bit piece held in aligned 32-bit words, rebuilt in
// parallel in registers).  Here the 4-bit piece is e1 e0 m1 m0, which already
// sits at fp16 bits 11..8 after a shift; the 2-bit piece is (s, e2), targets
// fp16 bits 15 and 12.  Two halves are produced per 32-bit operation.
//
// Packed layout (version 1), per tile of 128 rows x 64 columns (6144 bytes,
// tiles stored row-tile major, column-tile minor): row r owns lo words L_q
// (q = 0..7) at byte (q/4)*2048 + r*16 + (q%4)*4 and hi words H_p (p = 0..3)
// at byte 4096 + r*16 + p*4, so a warp reading 16 bytes per row touches 512
// consecutive bytes (no bank conflicts).  Pair j (columns 2j, 2j+1) of the row
// is rebuilt as
//     rotl(H_{j/8}, 12 - 2(j%8)) & 0x90009000   |   shift(L_{j/4}, 8 - 4(j%4)) & 0x0F000F00
// i.e. the nibble of column 2j+h sits at L bits 4(j%4)+16h, e2 at H bit
// 2(j%8)+16h and s at H bit (2(j%8)+3+16h) mod 32.  The eight rotations
// place the 16 two-bit fields of a hi word onto disjoint bit sets.
#pragma once
#include <cstdint>
#include <cuda_fp16.h>

namespace fp6 {

constexpr int kTileRows = 128;
constexpr int kTileCols = 64;
constexpr int kTileBytes = 6144;
constexpr int kLoBytes = 4096;

// Rebuild the 64 fp16 weights (as 32 fp16x2 words, low half = even column) of
// one row of one tile from its 8 lo words and 4 hi words.
__device__ __forceinline__ void splice_row(const uint32_t (&lo)[8], const uint32_t (&hi)[4],
                                           uint32_t (&out)[32]) {
#pragma unroll
  for (int j = 0; j < 32; ++j) {
    const uint32_t h = hi[j >> 3];
    const uint32_t hr = __funnelshift_l(h, h, (12 - 2 * (j & 7)) & 31);
    const uint32_t l = lo[j >> 2];
    const int t = j & 3;
    const uint32_t lr = (t < 2) ? (l << (8 - 4 * t)) : (l >> (4 * t - 8));
    out[j] = (hr & 0x90009000u) | (lr & 0x0F000F00u);
  }
}

// Load the row's fragments from a tile that starts at `tile` (shared or
// global memory, 16-byte aligned).
__device__ __forceinline__ void load_row_fragments(const uint8_t* tile, int r, uint32_t (&lo)[8],
                                                   uint32_t (&hi)[4]) {
  const uint4 a = *reinterpret_cast<const uint4*>(tile + r * 16);
  const uint4 b = *reinterpret_cast<const uint4*>(tile + 2048 + r * 16);
  const uint4 c = *reinterpret_cast<const uint4*>(tile + kLoBytes + r * 16);
  lo[0] = a.x; lo[1] = a.y; lo[2] = a.z; lo[3] = a.w;
  lo[4] = b.x; lo[5] = b.y; lo[6] = b.z; lo[7] = b.w;
  hi[0] = c.x; hi[1] = c.y; hi[2] = c.z; hi[3] = c.w;
}

// Pack 64 codes (columns 0..63 of one tile row) into the row's words.
__device__ __forceinline__ void pack_row(const uint8_t (&c)[64], uint32_t (&lo)[8], uint32_t (&hi)[4]) {
#pragma unroll
  for (int q = 0; q < 8; ++q) lo[q] = 0;
#pragma unroll
  for (int p = 0; p < 4; ++p) hi[p] = 0;
#pragma unroll
  for (int kk = 0; kk < 64; ++kk) {
    const int j = kk >> 1, h = kk & 1, i = j & 7;
    const uint32_t code = c[kk] & 0x3Fu;
    lo[j >> 2] |= (code & 0xFu) << (4 * (j & 3) + 16 * h);
    hi[j >> 3] |= ((code >> 4) & 1u) << (2 * i + 16 * h);
    hi[j >> 3] |= ((code >> 5) & 1u) << ((2 * i + 3 + 16 * h) & 31);
  }
}

// e3m2 magnitude of code c (0..31), exact in fp32.
__host__ __device__ constexpr float e3m2_magnitude(int c) {
  return (c < 4) ? c * 0.0625f
                 : static_cast<float>(1 << ((c >> 2) - 1)) * 0.25f * (1.0f + (c & 3) * 0.25f);
}

// Code of w for the scale s > 0: round |w|/s to the nearest e3m2 magnitude,
// ties to the even code, saturating at 28; sign copied from w.  Decided with
// exact comparisons of |w| against midpoint*s (a product of at most 4 and 11
// significant bits, exact in fp32), which is the rounding of the exact
// quotient |w|/s.
__device__ __forceinline__ uint8_t e3m2_code(float w, float s) {
  const float a = fabsf(w);
  int code = 0;
#pragma unroll
  for (int c = 0; c < 31; ++c) {
    const float mid = 0.5f * (e3m2_magnitude(c) + e3m2_magnitude(c + 1));
    const float t = mid * s;
    const bool up = (a > t) || (a == t && ((c + 1) & 1) == 0);
    code = up ? c + 1 : code;
  }
  return static_cast<uint8_t>(code | (signbit(w) ? 0x20 : 0));
}

}  // namespace fp6
