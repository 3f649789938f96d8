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

// One thread per (row, tile): splice the row's 64 weights and write them as
// fp16.  Without scales: decode(c) exactly.  With scales: fp16_rne(decode * s),
// the product formed exactly in fp32 (at most 4 + 11 significant bits).
template <Fmt F = Fmt::E3M2>
__global__ void __launch_bounds__(256) dequant_kernel(const uint8_t* __restrict__ packed,
                                                      const uint16_t* __restrict__ scales, int64_t N,
                                                      int64_t K, uint16_t* __restrict__ W16) {
  const int64_t KT = K / kTileCols;
  const int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (idx >= N * KT) return;
  const int64_t kt = idx / N;
  const int64_t n = idx % N;
  using Fm = Format<F>;
  const uint8_t* tile = packed + ((n / kTileRows) * KT + kt) * Fm::kTileBytes;
  uint32_t Fw[Fm::kRowWords], w[32];
  Fm::load(tile, static_cast<int>(n % kTileRows), Fw);
  Fm::rebuild(Fw, w);
  const float mul = scales ? __half2float(__ushort_as_half(scales[n])) : 1.0f;
  uint16_t* dst = W16 + n * K + kt * kTileCols;
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
    *reinterpret_cast<uint4*>(dst + 8 * v) = make_uint4(o[0], o[1], o[2], o[3]);
  }
}

}  // namespace fp6
