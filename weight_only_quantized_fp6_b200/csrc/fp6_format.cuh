// fp6_format.cuh -- FP6 (e3m2) encoding on the device: the packed layout,
// the register rebuild of fp16 weights, and the quantizer's rounding; and the
// same for the other formats (FP6 e2m3, FP4 e2m1) at the end.
//
// e3m2 code (low 6 bits of a byte): s = bit 5, e = bits 4..2 (bias 3),
// m = bits 1..0.  Value (-1)^s 2^(e-3)(1+m/4), or (-1)^s 2^-2 (m/4) for e = 0.
// Every value is exact in fp16.
//
// Rebuild.  The TC-FPx article ("kernel solution redesign") cuts each 6-bit
// weight into pieces held in aligned 32-bit words and rebuilds FP16 weights
// in registers, many per operation.  sm_100a converts a pair of e3m2 codes to
// an fp16 pair in one instruction (cvt.rn.f16x2.e3m2x2), reading the low six
// bits of each of the two bytes and ignoring their top two bits; the layout
// below is cut for it.  Of every 16 codes of a row, 12 stay whole in the low
// six bits of a byte and are converted straight from the loaded words; the
// other 4 are cut into three 2-bit pieces kept in the top two bits of those
// bytes and gathered with two masked merges and three shifts into one more
// word of byte containers.  Per row of a tile: 32 conversions and 20 integer
// operations for 64 weights.
//
// Packed layout (version 2), per tile of 128 rows x 64 columns (6144 bytes,
// tiles stored row-tile major, column-tile minor): row r owns words F_w
// (w = 0..11) at byte (w/4)*2048 + r*16 + (w%4)*4, so a warp reading 16 bytes
// per row touches 512 consecutive bytes (no bank conflicts).  Column kk of
// the tile is position i = kk%16 of group g = kk/16 (words F_{3g..3g+2}):
//     i < 12: the whole code in bits 8b..8b+5 of F_{3g + i/4}, b = i%4;
//     i >= 12: b = i - 12; code bits 2j, 2j+1 (j = 0..2) in bits 8b+6, 8b+7
//              of F_{3g + j}.
#pragma once
#include <cstdint>
#include <cuda_fp16.h>

namespace fp6 {

constexpr int kTileRows = 128;
constexpr int kTileCols = 64;
constexpr int kTileBytes = 6144;
constexpr int kRowWords = 12;

// Two e3m2 codes (the low six bits of bytes 0 and 1, resp. 2 and 3, of w) to
// two fp16 pairs: o0 = (byte 0, byte 1), o1 = (byte 2, byte 3), low half first.
__device__ __forceinline__ void cvt_e3m2x4(uint32_t w, uint32_t& o0, uint32_t& o1) {
  asm("{\n\t.reg .b16 l, h;\n\tmov.b32 {l, h}, %2;\n\t"
      "cvt.rn.f16x2.e3m2x2 %0, l;\n\tcvt.rn.f16x2.e3m2x2 %1, h;\n\t}"
      : "=r"(o0), "=r"(o1)
      : "r"(w));
}

// The cut codes of one 16-column group (words f0, f1, f2) gathered into the
// low six bits of four bytes: code bits 5,4 sit in the top bits of f2, bits
// 3,2 in f1, bits 1,0 in f0.
__device__ __forceinline__ uint32_t gather_cut(uint32_t f0, uint32_t f1, uint32_t f2) {
  const uint32_t u1 = (f2 & 0xC0C0C0C0u) | ((f1 >> 2) & 0x3F3F3F3Fu);
  const uint32_t u2 = (u1 & 0xF0F0F0F0u) | ((f0 >> 4) & 0x0F0F0F0Fu);
  return u2 >> 2;
}

// Rebuild the 64 fp16 weights (as 32 fp16x2 words, low half = even column)
// of one row of one tile from its 12 words: decode(c) exactly.
__device__ __forceinline__ void splice_row(const uint32_t (&F)[kRowWords], uint32_t (&out)[32]) {
#pragma unroll
  for (int g = 0; g < 4; ++g) {
    const uint32_t f0 = F[3 * g], f1 = F[3 * g + 1], f2 = F[3 * g + 2];
    cvt_e3m2x4(f0, out[8 * g + 0], out[8 * g + 1]);
    cvt_e3m2x4(f1, out[8 * g + 2], out[8 * g + 3]);
    cvt_e3m2x4(f2, out[8 * g + 4], out[8 * g + 5]);
    cvt_e3m2x4(gather_cut(f0, f1, f2), out[8 * g + 6], out[8 * g + 7]);
  }
}

// Load the row's 12 words from a tile that starts at `tile` (shared or
// global memory, 16-byte aligned).
__device__ __forceinline__ void load_row_words(const uint8_t* tile, int r, uint32_t (&F)[kRowWords]) {
#pragma unroll
  for (int u = 0; u < 3; ++u) {
    const uint4 a = *reinterpret_cast<const uint4*>(tile + u * 2048 + r * 16);
    F[4 * u + 0] = a.x;
    F[4 * u + 1] = a.y;
    F[4 * u + 2] = a.z;
    F[4 * u + 3] = a.w;
  }
}

// Pack 64 codes (columns 0..63 of one tile row) into the row's 12 words.
__device__ __forceinline__ void pack_row(const uint8_t (&c)[64], uint32_t (&F)[kRowWords]) {
#pragma unroll
  for (int w = 0; w < kRowWords; ++w) F[w] = 0;
#pragma unroll
  for (int kk = 0; kk < 64; ++kk) {
    const int g = kk >> 4, i = kk & 15;
    const uint32_t code = c[kk] & 0x3Fu;
    if (i < 12) {
      F[3 * g + (i >> 2)] |= code << (8 * (i & 3));
    } else {
      const int b = i - 12;
#pragma unroll
      for (int j = 0; j < 3; ++j) F[3 * g + j] |= ((code >> (2 * j)) & 3u) << (8 * b + 6);
    }
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

// ---- formats ------------------------------------------------------------
// The FP6-LLM pages describe one design for float weights of several widths.
// Two more formats share this machinery, each with one fp16 scale per row:
//   FP6 e2m3: s = bit 5, e = bits 4..3 (bias 1), m = bits 2..0, largest 7.5;
//             the same 6-bit layout, converted by cvt.rn.f16x2.e2m3x2.
//   FP4 e2m1: s = bit 3, e = bits 2..1 (bias 1), m = bit 0, largest 6;
//             tiles of 128 rows x 64 columns in 4096 bytes: row r owns words
//             F_w (w = 0..7) at byte (w/4)*2048 + r*16 + (w%4)*4, and column
//             kk sits in bits 4(kk%8) .. 4(kk%8)+3 of F_{kk/8} (each byte holds
//             two codes, low nibble first), converted by cvt.rn.f16x2.e2m1x2.
//   FP5 e2m2: s = bit 4, e = bits 3..2 (bias 1), m = bits 1..0, largest 7.
//             Every e2m2 value is the e2m3 value of the code shifted left by
//             one, so the rebuild forms those e2m3 codes in bytes and converts
//             them with cvt.rn.f16x2.e2m3x2.  Tiles of 128 rows x 64 columns in
//             5120 bytes, each code cut 4+1: row r owns eight words P_w of
//             4-bit pieces (the code's top four bits) at byte
//             (w/4)*2048 + r*16 + (w%4)*4 and two words Q_q of 1-bit pieces
//             (its lowest bit) at byte 4096 + r*8 + q*4.  Column kk is
//             position i = kk%32 of half q = kk/32; with v = i/8, h = (i%8)/4,
//             b = i%4 its top bits sit at bits 8b+4h.. of P_{4q+v} and its low
//             bit at bit 8b+2v+h of Q_q.  A P word shifted by two (left for
//             the low nibbles, right for the high ones) puts four top pieces
//             in bits 5..2 of four bytes, and Q shifted by 2v-1 (2v) puts
//             their low bits in bit 1: the e2m3 codes, ready to convert.
enum class Fmt : int { E3M2 = 0, E2M3 = 1, E2M1 = 2, E2M2 = 3, S24 = 4 };

// Per-thread state a format's rebuild needs besides the packed words, made
// once by make_aux() (by every lane of a warp, since the 2:4 format's rebuild
// reads it across lanes).  The float formats need none.
struct NoAux {};

// Store a row's words into a tile laid out as 2048-byte blocks of 16 bytes
// per row (first 4*(W/4) words), then, for W = 10, one 1024-byte block of
// 8 bytes per row.
template <int W>
__device__ __forceinline__ void store_row_words(uint8_t* tile, int r, const uint32_t (&F)[W]) {
#pragma unroll
  for (int u = 0; u < W / 4; ++u)
    *reinterpret_cast<uint4*>(tile + u * 2048 + r * 16) = make_uint4(F[4 * u], F[4 * u + 1], F[4 * u + 2], F[4 * u + 3]);
  if constexpr (W % 4 == 2)
    *reinterpret_cast<uint2*>(tile + (W / 4) * 2048 + r * 8) = make_uint2(F[W - 2], F[W - 1]);
}

// Two e2m3 codes per 16-bit half of w (low six bits of each byte), as
// cvt_e3m2x4 does for e3m2.
__device__ __forceinline__ void cvt_e2m3x4(uint32_t w, uint32_t& o0, uint32_t& o1) {
  asm("{\n\t.reg .b16 l, h;\n\tmov.b32 {l, h}, %2;\n\t"
      "cvt.rn.f16x2.e2m3x2 %0, l;\n\tcvt.rn.f16x2.e2m3x2 %1, h;\n\t}"
      : "=r"(o0), "=r"(o1)
      : "r"(w));
}

// Eight e2m1 codes (two per byte, low nibble first) to four fp16 pairs.
__device__ __forceinline__ void cvt_e2m1x8(uint32_t w, uint32_t (&o)[4]) {
  asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\tmov.b32 {b0, b1, b2, b3}, %4;\n\t"
      "cvt.rn.f16x2.e2m1x2 %0, b0;\n\tcvt.rn.f16x2.e2m1x2 %1, b1;\n\t"
      "cvt.rn.f16x2.e2m1x2 %2, b2;\n\tcvt.rn.f16x2.e2m1x2 %3, b3;\n\t}"
      : "=r"(o[0]), "=r"(o[1]), "=r"(o[2]), "=r"(o[3])
      : "r"(w));
}

template <Fmt F>
struct Format;

template <>
struct Format<Fmt::E3M2> {
  using Aux = NoAux;
  __device__ static Aux make_aux() { return {}; }
  static constexpr int kTileBytes = 6144;
  static constexpr int kRowWords = 12;
  static constexpr int kMags = 32;          // magnitudes; the sign bit is kMags
  static constexpr float kMax = 28.0f;
  __host__ __device__ static constexpr float magnitude(int c) { return e3m2_magnitude(c); }
  __device__ static void load(const uint8_t* tile, int r, uint32_t (&F)[kRowWords]) { load_row_words(tile, r, F); }
  __device__ static void rebuild(const uint32_t (&F)[kRowWords], uint32_t (&out)[32]) { splice_row(F, out); }
  __device__ static void pack(const uint8_t (&c)[64], uint32_t (&F)[kRowWords]) { pack_row(c, F); }
  __device__ static void store(uint8_t* tile, int r, const uint32_t (&F)[kRowWords]) { store_row_words(tile, r, F); }
};

template <>
struct Format<Fmt::E2M3> {
  using Aux = NoAux;
  __device__ static Aux make_aux() { return {}; }
  static constexpr int kTileBytes = 6144;
  static constexpr int kRowWords = 12;
  static constexpr int kMags = 32;
  static constexpr float kMax = 7.5f;
  __host__ __device__ static constexpr float magnitude(int c) {
    return (c < 8) ? c * 0.125f : static_cast<float>(1 << ((c >> 3) - 1)) * (1.0f + (c & 7) * 0.125f);
  }
  __device__ static void load(const uint8_t* tile, int r, uint32_t (&F)[kRowWords]) { load_row_words(tile, r, F); }
  __device__ static void rebuild(const uint32_t (&F)[kRowWords], uint32_t (&out)[32]) {
#pragma unroll
    for (int g = 0; g < 4; ++g) {
      const uint32_t f0 = F[3 * g], f1 = F[3 * g + 1], f2 = F[3 * g + 2];
      cvt_e2m3x4(f0, out[8 * g + 0], out[8 * g + 1]);
      cvt_e2m3x4(f1, out[8 * g + 2], out[8 * g + 3]);
      cvt_e2m3x4(f2, out[8 * g + 4], out[8 * g + 5]);
      cvt_e2m3x4(gather_cut(f0, f1, f2), out[8 * g + 6], out[8 * g + 7]);
    }
  }

  __device__ static void pack(const uint8_t (&c)[64], uint32_t (&F)[kRowWords]) { pack_row(c, F); }
  __device__ static void store(uint8_t* tile, int r, const uint32_t (&F)[kRowWords]) { store_row_words(tile, r, F); }
};

template <>
struct Format<Fmt::E2M1> {
  using Aux = NoAux;
  __device__ static Aux make_aux() { return {}; }
  static constexpr int kTileBytes = 4096;
  static constexpr int kRowWords = 8;
  static constexpr int kMags = 8;
  static constexpr float kMax = 6.0f;
  __host__ __device__ static constexpr float magnitude(int c) {
    return (c < 2) ? c * 0.5f : static_cast<float>(1 << ((c >> 1) - 1)) * (1.0f + (c & 1) * 0.5f);
  }
  __device__ static void load(const uint8_t* tile, int r, uint32_t (&F)[kRowWords]) {
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const uint4 a = *reinterpret_cast<const uint4*>(tile + u * 2048 + r * 16);
      F[4 * u + 0] = a.x;
      F[4 * u + 1] = a.y;
      F[4 * u + 2] = a.z;
      F[4 * u + 3] = a.w;
    }
  }
  __device__ static void rebuild(const uint32_t (&F)[kRowWords], uint32_t (&out)[32]) {
#pragma unroll
    for (int w = 0; w < 8; ++w) {
      uint32_t o[4];
      cvt_e2m1x8(F[w], o);
#pragma unroll
      for (int b = 0; b < 4; ++b) out[4 * w + b] = o[b];
    }
  }

  __device__ static void pack(const uint8_t (&c)[64], uint32_t (&F)[kRowWords]) {
#pragma unroll
    for (int w = 0; w < kRowWords; ++w) F[w] = 0;
#pragma unroll
    for (int kk = 0; kk < 64; ++kk) F[kk >> 3] |= (c[kk] & 0xFu) << (4 * (kk & 7));
  }
  __device__ static void store(uint8_t* tile, int r, const uint32_t (&F)[kRowWords]) { store_row_words(tile, r, F); }
};

template <>
struct Format<Fmt::E2M2> {
  using Aux = NoAux;
  __device__ static Aux make_aux() { return {}; }
  static constexpr int kTileBytes = 5120;
  static constexpr int kRowWords = 10;
  static constexpr int kMags = 16;
  static constexpr float kMax = 7.0f;
  __host__ __device__ static constexpr float magnitude(int c) {
    return (c < 4) ? c * 0.25f : static_cast<float>(1 << ((c >> 2) - 1)) * (1.0f + (c & 3) * 0.25f);
  }
  __device__ static void load(const uint8_t* tile, int r, uint32_t (&F)[kRowWords]) {
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const uint4 a = *reinterpret_cast<const uint4*>(tile + u * 2048 + r * 16);
      F[4 * u + 0] = a.x;
      F[4 * u + 1] = a.y;
      F[4 * u + 2] = a.z;
      F[4 * u + 3] = a.w;
    }
    const uint2 q = *reinterpret_cast<const uint2*>(tile + 4096 + r * 8);
    F[8] = q.x;
    F[9] = q.y;
  }
  __device__ static void rebuild(const uint32_t (&F)[kRowWords], uint32_t (&out)[32]) {
#pragma unroll
    for (int q = 0; q < 2; ++q) {
      const uint32_t Q = F[8 + q];
#pragma unroll
      for (int v = 0; v < 4; ++v) {
        const uint32_t P = F[4 * q + v];
        const uint32_t lo_bits = (v == 0) ? (Q << 1) : (Q >> (2 * v - 1));
        const uint32_t lo = ((P << 2) & 0x3C3C3C3Cu) | (lo_bits & 0x02020202u);
        const uint32_t hi = ((P >> 2) & 0x3C3C3C3Cu) | ((Q >> (2 * v)) & 0x02020202u);
        cvt_e2m3x4(lo, out[16 * q + 4 * v + 0], out[16 * q + 4 * v + 1]);
        cvt_e2m3x4(hi, out[16 * q + 4 * v + 2], out[16 * q + 4 * v + 3]);
      }
    }
  }

  __device__ static void pack(const uint8_t (&c)[64], uint32_t (&F)[kRowWords]) {
#pragma unroll
    for (int w = 0; w < kRowWords; ++w) F[w] = 0;
#pragma unroll
    for (int kk = 0; kk < 64; ++kk) {
      const int q = kk >> 5, i = kk & 31, v = i >> 3, h = (i >> 2) & 1, b = i & 3;
      F[4 * q + v] |= ((c[kk] >> 1) & 0xFu) << (8 * b + 4 * h);
      F[8 + q] |= (c[kk] & 1u) << (8 * b + 2 * v + h);
    }
  }
  __device__ static void store(uint8_t* tile, int r, const uint32_t (&F)[kRowWords]) { store_row_words(tile, r, F); }
};

// ---- 2:4 sparse INT4 (Sparse-Marlin) ----------------------------------------
// In each group of four consecutive weights of a row two are kept; each kept
// weight is a signed 4-bit code q (two's complement, -8..7) and its value is
// scale * q.  Tiles of 128 rows x 64 columns in 3072 bytes: row r owns four
// code words V_w at byte r*16 + 4w and two position words P_h at byte
// 2048 + r*8 + 4h.  Group j (0..15) of the tile row keeps its two codes in
// byte j%4 of V_{j/4} (the first kept weight in the low nibble) and its two
// positions i0 < i1 in bits 4(j%8) .. 4(j%8)+3 of P_{j/8} (i0 in the low two
// bits).
//
// Rebuild of a group: the two nibbles go into the low bits of two fp16 words
// 0x6400 | (q ^ 8), i.e. 1024 + q + 8, and one half-precision subtraction of
// 1032 leaves q exactly.  The pair is then placed at positions i0 and i1 of
// the group's four columns by two byte permutes, whose selectors depend on
// the position nibble alone: lane l of every warp holds the selectors of
// nibble l % 16 (make_aux), and a shuffle fetches those of the group's nibble.
template <>
struct Format<Fmt::S24> {
  static constexpr int kTileBytes = 3072;
  static constexpr int kRowWords = 6;       // V_0..V_3, P_0, P_1
  struct Aux {
    uint32_t sel;   // low 16 bits: selector of columns 0,1; high: columns 2,3
  };
  __device__ static Aux make_aux() {
    const int m = static_cast<int>(threadIdx.x & 15);
    const int i0 = m & 3, i1 = m >> 2;
    uint32_t sel = 0;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      // column k takes half 0 (first kept code), half 1 (second) or half 2
      // (bytes 4, 5: the permute's second operand, zero)
      const uint32_t h = (k == i0) ? 0u : (k == i1) ? 1u : 2u;
      sel |= ((2 * h) | ((2 * h + 1) << 4)) << (8 * k);
    }
    return {sel};
  }
  __device__ static void load(const uint8_t* tile, int r, uint32_t (&F)[kRowWords]) {
    const uint4 v = *reinterpret_cast<const uint4*>(tile + r * 16);
    const uint2 q = *reinterpret_cast<const uint2*>(tile + 2048 + r * 8);
    F[0] = v.x;
    F[1] = v.y;
    F[2] = v.z;
    F[3] = v.w;
    F[4] = q.x;
    F[5] = q.y;
  }
  __device__ static void rebuild(const uint32_t (&F)[kRowWords], uint32_t (&out)[32], const Aux& aux) {
    const __half2 k1032 = __halves2half2(__ushort_as_half(0x6408u), __ushort_as_half(0x6408u));
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      const uint32_t lo = F[w] & 0x0F0F0F0Fu;           // first kept code of each group
      const uint32_t hi = (F[w] >> 4) & 0x0F0F0F0Fu;    // second
#pragma unroll
      for (int b = 0; b < 4; ++b) {
        const int j = 4 * w + b;
        uint32_t h = __byte_perm(lo, hi, b | (b << 4) | ((4 + b) << 8) | ((4 + b) << 12));
        h = (h & 0x000F000Fu) ^ 0x64086408u;
        const __half2 v = __hsub2(*reinterpret_cast<const __half2*>(&h), k1032);
        const uint32_t vb = *reinterpret_cast<const uint32_t*>(&v);
        const uint32_t sel = __shfl_sync(0xffffffffu, aux.sel, static_cast<int>(F[4 + (j >> 3)] >> (4 * (j & 7))), 16);
        out[2 * j] = __byte_perm(vb, 0u, sel);
        out[2 * j + 1] = __byte_perm(vb, 0u, sel >> 16);
      }
    }
  }
};

// Rebuild through a format's per-thread state (the float formats have none).
template <Fmt F>
__device__ __forceinline__ void rebuild_row(const uint32_t (&W)[Format<F>::kRowWords], uint32_t (&out)[32],
                                            const typename Format<F>::Aux& aux) {
  if constexpr (F == Fmt::S24) {
    Format<F>::rebuild(W, out, aux);
  } else {
    (void)aux;
    Format<F>::rebuild(W, out);
  }
}

// Code of w for the scale s > 0 in format F: |w|/s rounded to the nearest
// magnitude, ties to the even code, saturating at the largest; sign copied
// from w.  Decided with exact comparisons of |w| against midpoint*s (few
// significant bits, exact in fp32), which is the rounding of the exact
// quotient |w|/s.
template <Fmt F>
__device__ __forceinline__ uint8_t quant_code(float w, float s) {
  using Fm = Format<F>;
  const float a = fabsf(w);
  int code = 0;
#pragma unroll
  for (int c = 0; c < Fm::kMags - 1; ++c) {
    const float mid = 0.5f * (Fm::magnitude(c) + Fm::magnitude(c + 1));
    const float t = mid * s;
    const bool up = (a > t) || (a == t && ((c + 1) & 1) == 0);
    code = up ? c + 1 : code;
  }
  return static_cast<uint8_t>(code | (signbit(w) ? Fm::kMags : 0));
}

}  // namespace fp6
