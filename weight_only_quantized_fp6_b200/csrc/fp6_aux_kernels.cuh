// fp6_aux_kernels.cuh -- offline quantization, pre-packing, and stand-alone
// dequantization kernels.
#pragma once
#include <cstdint>
#include <cuda_fp16.h>

#include "fp6_format.cuh"

namespace fp6 {

__device__ unsigned int g_quant_error;  // bit 0: non-finite weight; bit 1: scale out of fp16 range
constexpr unsigned int kQuantNonfinite = 1u;
constexpr unsigned int kQuantScaleRange = 2u;

// One CTA per weight row: max |w| (rejecting NaN/inf), the fp16 scale
// fp16_rne(fp32(max/largest)) (largest = 28 for e3m2), then one code per
// weight.
template <int THREADS, Fmt F = Fmt::E3M2>
__global__ void __launch_bounds__(THREADS) quantize_kernel(const float* __restrict__ W, int64_t K,
                                                           uint8_t* __restrict__ codes,
                                                           uint16_t* __restrict__ scales) {
  const int64_t n = blockIdx.x;
  const float* row = W + n * K;
  float amax = 0.0f;
  bool bad = false;
  for (int64_t k = threadIdx.x; k < K; k += THREADS) {
    const float w = row[k];
    bad |= !isfinite(w);
    amax = fmaxf(amax, fabsf(w));
  }
  __shared__ float s_max[THREADS / 32];
  __shared__ int s_bad[THREADS / 32];
  __shared__ float s_scale;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
  const int any_bad = __any_sync(0xffffffffu, bad);
  if ((threadIdx.x & 31) == 0) {
    s_max[threadIdx.x >> 5] = amax;
    s_bad[threadIdx.x >> 5] = any_bad;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    float m = 0.0f;
    int b = 0;
    for (int i = 0; i < THREADS / 32; ++i) {
      m = fmaxf(m, s_max[i]);
      b |= s_bad[i];
    }
    float scale = 0.0f;
    uint16_t sbits = 0;
    if (b) {
      atomicOr(&g_quant_error, kQuantNonfinite);
    } else if (m > 0.0f) {
      const __half h = __float2half_rn(m / Format<F>::kMax);
      sbits = __half_as_ushort(h);
      const uint16_t mag = sbits & 0x7FFFu;
      if (mag >= 0x7C00u || mag == 0) atomicOr(&g_quant_error, kQuantScaleRange);
      scale = __half2float(h);
    }
    scales[n] = sbits;
    s_scale = scale;
  }
  __syncthreads();
  const float s = s_scale;
  uint8_t* crow = codes + n * K;
  if (s > 0.0f && isfinite(s)) {
    for (int64_t k = threadIdx.x; k < K; k += THREADS) crow[k] = quant_code<F>(row[k], s);
  } else {
    for (int64_t k = threadIdx.x; k < K; k += THREADS) crow[k] = 0;
  }
}

// One thread per (row, 64-column tile): read 64 codes, write the row's 48
// bytes (32 for FP4, 40 for FP5) of the packed tile.
template <Fmt F = Fmt::E3M2>
__global__ void __launch_bounds__(256) prepack_kernel(const uint8_t* __restrict__ codes, int64_t N,
                                                      int64_t K, uint8_t* __restrict__ packed) {
  const int64_t KT = K / kTileCols;
  const int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (idx >= N * KT) return;
  // consecutive threads take consecutive rows of the same tile (coalesced writes)
  const int64_t kt = idx / N;
  const int64_t n = idx % N;
  const uint8_t* src = codes + n * K + kt * kTileCols;
  uint8_t c[64];
#pragma unroll
  for (int v = 0; v < 4; ++v) {
    const uint4 u = *reinterpret_cast<const uint4*>(src + 16 * v);
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int b = 0; b < 16; ++b) c[16 * v + b] = static_cast<uint8_t>(w[b >> 2] >> (8 * (b & 3)));
  }
  using Fm = Format<F>;
  uint32_t Fw[Fm::kRowWords];
  Fm::pack(c, Fw);
  uint8_t* tile = packed + ((n / kTileRows) * KT + kt) * Fm::kTileBytes;
  Fm::store(tile, static_cast<int>(n % kTileRows), Fw);
}

// Dequantize to fp16.  Without scales: the code's value exactly (decode(c),
// or q for the 2:4 format).  With scales: fp16_rne(value * s), the product
// formed exactly in fp32 (at most 4 + 11 significant bits).
//
// A unit of work is 32 consecutive rows of one 64-column tile, taken by one
// warp: each lane rebuilds its row's 64 weights, the warp stages the 32 rows
// (128 bytes each) in shared memory, and then stores them row by row, eight
// lanes per 128-byte row, so every store instruction writes four whole rows.
// Warps stride over the units, so every lane takes part in every shuffle.
constexpr int kDequantWarps = 8;
template <Fmt F = Fmt::E3M2>
__global__ void __launch_bounds__(32 * kDequantWarps) dequant_kernel(const uint8_t* __restrict__ packed,
                                                                     const uint16_t* __restrict__ scales,
                                                                     int64_t N, int64_t K,
                                                                     uint16_t* __restrict__ W16) {
  using Fm = Format<F>;
  __shared__ uint4 stage[kDequantWarps][32][9];   // a 128-byte row padded to 144 bytes: no bank conflicts
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int64_t KT = K / kTileCols;
  const int64_t groups = N / 32;
  const int64_t units = groups * KT;
  const auto aux = Fm::make_aux();
  for (int64_t u = static_cast<int64_t>(blockIdx.x) * kDequantWarps + warp; u < units;
       u += static_cast<int64_t>(gridDim.x) * kDequantWarps) {
    const int64_t kt = u / groups;
    const int64_t n0 = (u - kt * groups) * 32;
    const int64_t n = n0 + lane;
    const uint8_t* tile = packed + ((n / kTileRows) * KT + kt) * Fm::kTileBytes;
    uint32_t Fw[Fm::kRowWords], w[32];
    Fm::load(tile, static_cast<int>(n % kTileRows), Fw);
    rebuild_row<F>(Fw, w, aux);
    const float mul = scales ? __half2float(__ushort_as_half(scales[n])) : 1.0f;
#pragma unroll
    for (int v = 0; v < 8; ++v) {
      uint32_t o[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const __half2 h2 = *reinterpret_cast<const __half2*>(&w[4 * v + e]);
        const float2 f = __half22float2(h2);
        const __half2 r2 = __floats2half2_rn(f.x * mul, f.y * mul);
        o[e] = *reinterpret_cast<const uint32_t*>(&r2);
      }
      stage[warp][lane][v] = make_uint4(o[0], o[1], o[2], o[3]);
    }
    __syncwarp();
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int row = 4 * i + (lane >> 3), chunk = lane & 7;
      *reinterpret_cast<uint4*>(W16 + (n0 + row) * K + kt * kTileCols + chunk * 8) = stage[warp][row][chunk];
    }
    __syncwarp();
  }
}

// ---- 2:4 sparse INT4 (Sparse-Marlin) --------------------------------------------
// Code of a kept weight w for the scale s: round-half-even(w / s) clamped to
// [-8, 7], decided with exact comparisons of |w| against (m + 1/2) * s (at
// most 4 + 11 significant bits: exact in fp32), which is the rounding of the
// exact quotient.  A zero scale (all-zero row) gives 0.
__device__ __forceinline__ int s24_code(float w, float s) {
  if (!(s > 0.0f)) return 0;
  const float a = fabsf(w);
  int mag = 0;
#pragma unroll
  for (int m = 0; m < 8; ++m) {
    const float t = (static_cast<float>(m) + 0.5f) * s;
    const bool up = (a > t) || (a == t && ((m + 1) & 1) == 0);
    mag = up ? m + 1 : mag;
  }
  return signbit(w) ? -mag : (mag > 7 ? 7 : mag);
}

// One CTA per weight row: max |w| (rejecting NaN/inf) and the fp16 scale
// fp16_rne(fp32(max / 7)); then, per group of four consecutive weights, the
// two with the largest |w| are kept (ties to the lower position) and coded.
//   q [N, K/2] int8: the kept codes of each group in position order
//   pos [N, K/2] uint8: their positions 0..3 in the group
template <int THREADS>
__global__ void __launch_bounds__(THREADS) s24_quantize_kernel(const float* __restrict__ W, int64_t K,
                                                               int8_t* __restrict__ q, uint8_t* __restrict__ pos,
                                                               uint16_t* __restrict__ scales) {
  const int64_t n = blockIdx.x;
  const float* row = W + n * K;
  float amax = 0.0f;
  bool bad = false;
  for (int64_t k = threadIdx.x; k < K; k += THREADS) {
    const float w = row[k];
    bad |= !isfinite(w);
    amax = fmaxf(amax, fabsf(w));
  }
  __shared__ float s_max[THREADS / 32];
  __shared__ int s_bad[THREADS / 32];
  __shared__ float s_scale;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
  const int any_bad = __any_sync(0xffffffffu, bad);
  if ((threadIdx.x & 31) == 0) {
    s_max[threadIdx.x >> 5] = amax;
    s_bad[threadIdx.x >> 5] = any_bad;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    float m = 0.0f;
    int b = 0;
    for (int i = 0; i < THREADS / 32; ++i) {
      m = fmaxf(m, s_max[i]);
      b |= s_bad[i];
    }
    float scale = 0.0f;
    uint16_t sbits = 0;
    if (b) {
      atomicOr(&g_quant_error, kQuantNonfinite);
    } else if (m > 0.0f) {
      const __half h = __float2half_rn(m / 7.0f);
      sbits = __half_as_ushort(h);
      const uint16_t mag = sbits & 0x7FFFu;
      if (mag >= 0x7C00u || mag == 0) atomicOr(&g_quant_error, kQuantScaleRange);
      else scale = __half2float(h);
    }
    scales[n] = sbits;
    s_scale = scale;
  }
  __syncthreads();
  const float s = s_scale;
  for (int64_t j = threadIdx.x; j < K / 4; j += THREADS) {
    const float4 v = reinterpret_cast<const float4*>(row)[j];
    const float w[4] = {v.x, v.y, v.z, v.w};
    int best = 0;
#pragma unroll
    for (int i = 1; i < 4; ++i)
      if (fabsf(w[i]) > fabsf(w[best])) best = i;           // strict: ties keep the lower position
    int second = -1;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      if (i == best) continue;
      if (second < 0 || fabsf(w[i]) > fabsf(w[second])) second = i;
    }
    const int i0 = best < second ? best : second, i1 = best < second ? second : best;
    const int64_t o = n * (K / 2) + 2 * j;
    q[o] = static_cast<int8_t>(s24_code(w[i0], s));
    q[o + 1] = static_cast<int8_t>(s24_code(w[i1], s));
    pos[o] = static_cast<uint8_t>(i0);
    pos[o + 1] = static_cast<uint8_t>(i1);
  }
}

// One thread per (row, 64-column tile): the row's sixteen groups into its
// four code words and two position words (see Format<Fmt::S24>).
__global__ void __launch_bounds__(256) s24_prepack_kernel(const int8_t* __restrict__ q,
                                                          const uint8_t* __restrict__ pos, int64_t N,
                                                          int64_t K, uint8_t* __restrict__ packed) {
  const int64_t KT = K / kTileCols;
  const int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (idx >= N * KT) return;
  const int64_t kt = idx / N;
  const int64_t n = idx % N;
  const int64_t o = n * (K / 2) + kt * 32;                  // the tile row's 16 groups, two entries each
  uint8_t qc[32], pc[32];
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const uint4 a = reinterpret_cast<const uint4*>(q + o)[h];
    const uint4 b = reinterpret_cast<const uint4*>(pos + o)[h];
    const uint32_t aw[4] = {a.x, a.y, a.z, a.w}, bw[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
    for (int e = 0; e < 16; ++e) {
      qc[16 * h + e] = static_cast<uint8_t>(aw[e >> 2] >> (8 * (e & 3)));
      pc[16 * h + e] = static_cast<uint8_t>(bw[e >> 2] >> (8 * (e & 3)));
    }
  }
  uint32_t V[4] = {0, 0, 0, 0}, P[2] = {0, 0};
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    const uint32_t codes = (qc[2 * j] & 0xFu) | ((qc[2 * j + 1] & 0xFu) << 4);
    V[j >> 2] |= codes << (8 * (j & 3));
    const uint32_t meta = (pc[2 * j] & 3u) | ((pc[2 * j + 1] & 3u) << 2);
    P[j >> 3] |= meta << (4 * (j & 7));
  }
  uint8_t* tile = packed + ((n / kTileRows) * KT + kt) * Format<Fmt::S24>::kTileBytes;
  const int r = static_cast<int>(n % kTileRows);
  *reinterpret_cast<uint4*>(tile + r * 16) = make_uint4(V[0], V[1], V[2], V[3]);
  *reinterpret_cast<uint2*>(tile + 2048 + r * 8) = make_uint2(P[0], P[1]);
}

}  // namespace fp6
