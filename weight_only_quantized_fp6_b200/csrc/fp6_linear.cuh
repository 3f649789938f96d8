// fp6_linear.cuh -- the fused FP6 x FP16 linear layer for sm_100a.
//
// y[M,N] = x[M,K] . (scale (.) decode(W[N,K]))^T, fp32 accumulation, fp16 out.
//
// The TC-FPx design (article section "kernel solution redesign") keeps the
// dequantization and the tensor-core product in one kernel, rebuilds FP16
// weights with bit-parallel SIMT work in registers, and overlaps the two with
// a software pipeline.  On sm_100a this becomes a warp-specialised persistent
// kernel:
//
//   warp 0        producer: one bulk copy of the 6144-byte packed tile and one
//                 TMA tile copy of the activations (128-byte swizzle, rows
//                 beyond M zero-filled) per 64-column step into a smem ring;
//   warp 1        owns TMEM; one lane issues tcgen05.mma (M=128 weight rows,
//                 N = NCOL tokens, K=16) with the weights as the TMEM A operand
//                 and the activations as the smem B operand;
//   warps 2..9    two dequant warpgroups taking alternate steps: each thread
//                 owns one weight row (its TMEM lane), reads its 48 packed
//                 bytes, splices 64 fp16 weights (decode * 2^-12) and writes
//                 them to TMEM with tcgen05.st; warpgroup 0 also runs the
//                 epilogue (tcgen05.ld of the fp32 accumulator, * scale * 2^12,
//                 fp16 store, or the split-K partial and fix-up).
//
// Work split: the (token tile, row tile, 64-column step) iterations are laid
// out row-tile major and cut into G contiguous, equal ranges, one per
// persistent CTA (G = number of SMs).  A row tile whose steps span several
// CTAs is finished by the last of them to arrive (atomic counter), which sums
// the partials in CTA order: results are deterministic and no CTA waits on
// another.  A split tile's counter is indexed by its first contributing CTA,
// which is unique among split tiles and below G, so the counters occupy a
// fixed region of the workspace that no partial ever overlaps.
#pragma once
#include <cstdint>
#include <cuda.h>
#include <cuda_fp16.h>

#include "fp6_format.cuh"
#include "ptx.cuh"

namespace fp6 {

constexpr int kAStages = 4;      // TMEM ring of dequantized weight tiles (32 columns each)
constexpr int kDeqGroups = 2;    // dequant warpgroups
constexpr int kLinearThreads = 64 + 128 * kDeqGroups;
constexpr int kMaxGrid = 1024;   // persistent CTAs at most (one per SM)
constexpr int kCounterBytes = kMaxGrid * 4;

template <int NCOL>
struct LinearShape {
  static_assert(NCOL == 16 || NCOL == 32 || NCOL == 64 || NCOL == 128 || NCOL == 256, "NCOL");
  static constexpr int kXBytes = NCOL * 128;                   // NCOL rows x 64 fp16
  static constexpr int kStageBytes = kXBytes + kTileBytes;     // multiple of 1024
  static constexpr int kStages = (NCOL == 16) ? 24 : (NCOL == 32) ? 19 : (NCOL == 64) ? 13
                               : (NCOL == 128) ? 8 : 5;
  static constexpr int kDCol = kAStages * 32;                  // accumulator column
  static constexpr uint32_t kTmemCols = (kDCol + NCOL <= 256) ? 256u : 512u;
  static constexpr int kBarrierBytes = 1024;
  static constexpr int kSmemBytes = kStages * kStageBytes + kBarrierBytes + 1024;  // + alignment slack
  static_assert(kStageBytes % 1024 == 0, "stage alignment");
};

struct LinearParams {
  const uint8_t* packed;
  const uint16_t* scales;
  uint16_t* y;
  float* partials;       // [2*G][NCOL][128] fp32
  uint32_t* counters;    // [kMaxGrid], indexed by a split tile's first CTA; zero on entry and exit
  int M, N, K;
  int n_tiles, m_tiles, k_tiles;
  long long total_iters;
  int grid;
};

// First iteration of CTA c's range.
__host__ __device__ __forceinline__ long long range_begin(int c, long long total, int G) {
  return static_cast<long long>(c) * total / G;
}
// CTA whose range holds iteration i:  max{c : range_begin(c) <= i}.
__host__ __device__ __forceinline__ int range_owner(long long i, long long total, int G) {
  return static_cast<int>(((i + 1) * G + total - 1) / total - 1);
}
// Partial slot of CTA c's segment in tile t: 0 for the tile its range starts
// in, 1 for the tile its range ends in (only those two can be partial).
__host__ __device__ __forceinline__ int partial_slot(int c, long long t, long long total, int G, int KT) {
  return 2 * c + ((range_begin(c, total, G) / KT == t) ? 0 : 1);
}

// Every lane of the warp waits; the warp continues only if all lanes saw the
// phase complete, so a timeout never leaves a .sync.aligned op divergent.
__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, volatile int* abort) {
  const bool ok = wait_bounded(bar, parity, abort);
  return __all_sync(0xffffffffu, ok) != 0;
}

template <int NCOL>
__global__ void __launch_bounds__(kLinearThreads, 1)
    fp6_linear_kernel(const __grid_constant__ CUtensorMap tmap_x, const LinearParams p) {
  using S = LinearShape<NCOL>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* bar_area = smem + S::kStages * S::kStageBytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(bar_area);
  uint64_t* empty = full + S::kStages;
  uint64_t* afull = empty + S::kStages;
  uint64_t* aempty = afull + kAStages;
  uint64_t* dfull = aempty + kAStages;
  uint64_t* dempty = dfull + 1;
  uint64_t* done = dempty + 1;
  uint64_t* epi = done + 1;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(epi + 1);
  volatile int* s_last = reinterpret_cast<volatile int*>(tmem_holder + 1);
  volatile int* s_abort = s_last + 1;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int G = p.grid;
  const int c = blockIdx.x;
  const long long total = p.total_iters;
  const int KT = p.k_tiles;
  const long long it0 = range_begin(c, total, G);
  const long long it1 = range_begin(c + 1, total, G);
  const int n_local = static_cast<int>(it1 - it0);
  const long long tile_first = it0 / KT;
  const int k_first = static_cast<int>(it0 - tile_first * KT);

  if (threadIdx.x == 0) {
    for (int s = 0; s < S::kStages; ++s) {
      mbar_init(smem_u32(&full[s]), 1);
      mbar_init(smem_u32(&empty[s]), 4 + 1);   // 4 dequant warps + 1 MMA commit
    }
    for (int a = 0; a < kAStages; ++a) {
      mbar_init(smem_u32(&afull[a]), 4);
      mbar_init(smem_u32(&aempty[a]), 1);
    }
    mbar_init(smem_u32(dfull), 1);
    mbar_init(smem_u32(dempty), 4);
    mbar_init(smem_u32(done), 1);
    mbar_init(smem_u32(epi), 4);   // the 4 warps of dequant group 0
    *s_last = 0;
    *s_abort = 0;
    fence_barrier_init();
    fence_proxy_async_smem();
  }
  if (warp == 0 && lane == 0) prefetch_tensormap(&tmap_x);
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_holder), S::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;

  if (warp == 0) {
    // ---------------- producer ----------------
    if (lane == 0) {
      const uint64_t pol_w = policy_evict_first();
      const uint64_t pol_x = policy_evict_last();
      int issued = 0;
      int k = k_first;
      long long tile = tile_first;
      for (int li = 0; li < n_local; ++li, k = (k + 1 == KT) ? 0 : k + 1, tile += (k == 0)) {
        const int s = li % S::kStages;
        if (li >= S::kStages &&
            !wait_bounded(smem_u32(&empty[s]), ((li / S::kStages) - 1) & 1, s_abort))
          break;
        const int nt = static_cast<int>(tile / p.m_tiles);
        const int mt = static_cast<int>(tile - static_cast<long long>(nt) * p.m_tiles);
        uint8_t* stage = smem + s * S::kStageBytes;
        const uint32_t fb = smem_u32(&full[s]);
        mbar_arrive_expect_tx(fb, S::kXBytes + kTileBytes);
        tma_load_2d(smem_u32(stage), &tmap_x, fb, k * kTileCols, mt * NCOL, pol_x);
        bulk_load(smem_u32(stage + S::kXBytes),
                  p.packed + (static_cast<long long>(nt) * KT + k) * kTileBytes, kTileBytes, fb, pol_w);
        ++issued;
      }
      // Leave no copy in flight: the last issued copy of every stage has landed.
      const int first = issued > S::kStages ? issued - S::kStages : 0;
      volatile int never = 0;
      for (int li = first; li < issued; ++li)
        wait_bounded(smem_u32(&full[li % S::kStages]), (li / S::kStages) & 1, &never);
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_f16_f32(128, NCOL);
      const uint32_t d_tmem = tmem + S::kDCol;
      int sg = 0;
      int k = k_first;
      for (int li = 0; li < n_local; ++li, k = (k + 1 == KT) ? 0 : k + 1) {
        const bool seg_first = (li == 0) || (k == 0);
        const bool seg_last = (li == n_local - 1) || (k == KT - 1);
        const int s = li % S::kStages;
        const int a = li % kAStages;
        if (seg_first && sg > 0 && !wait_bounded(smem_u32(dempty), (sg - 1) & 1, s_abort)) break;
        if (!wait_bounded(smem_u32(&full[s]), (li / S::kStages) & 1, s_abort)) break;
        if (!wait_bounded(smem_u32(&afull[a]), (li / kAStages) & 1, s_abort)) break;
        tc_fence_after();
        const uint64_t bdesc = smem_desc_sw128(smem_u32(smem + s * S::kStageBytes));
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          // K = 16 per MMA: 8 TMEM columns of A, 32 bytes along the swizzled B rows
          mma_f16_ts(d_tmem, tmem + a * 32 + kk * 8, bdesc + static_cast<uint64_t>(kk * 2), idesc,
                     (seg_first && kk == 0) ? 0u : 1u);
        }
        tc_commit(smem_u32(&empty[s]));
        tc_commit(smem_u32(&aempty[a]));
        if (seg_last) {
          tc_commit(smem_u32(dfull));
          ++sg;
        }
      }
      // All issued MMAs have finished before TMEM is released.
      tc_commit(smem_u32(done));
      volatile int never = 0;
      wait_bounded(smem_u32(done), 0, &never);
    }
  } else {
    // ---------------- dequant warpgroups (+ epilogue on group 0) ----------------
    const int g = (warp - 2) >> 2;
    const int quad = warp & 3;               // TMEM lanes 32*quad .. 32*quad+31
    const int r = quad * 32 + lane;          // weight row within the tile
    const uint32_t lane_base = static_cast<uint32_t>(quad * 32) << 16;
    int sg = 0;
    int ep = 0;
    int k = k_first;
    long long tile = tile_first;
    for (int li = 0; li < n_local; ++li, k = (k + 1 == KT) ? 0 : k + 1, tile += (k == 0)) {
      const bool seg_last = (li == n_local - 1) || (k == KT - 1);
      if ((li & 1) == g) {
        const int s = li % S::kStages;
        const int a = li % kAStages;
        if (!warp_wait(smem_u32(&full[s]), (li / S::kStages) & 1, s_abort)) break;
        uint32_t lo[8], hi[4], w[32];
        load_row_fragments(smem + s * S::kStageBytes + S::kXBytes, r, lo, hi);
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&empty[s]));
        if (li >= kAStages && !warp_wait(smem_u32(&aempty[a]), ((li / kAStages) - 1) & 1, s_abort))
          break;
        tc_fence_after();
        splice_row(lo, hi, w);
        tmem_st_32x32b_x32(tmem + lane_base + a * 32, w);
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&afull[a]));
      }
      if (g == 0 && seg_last) {
        // ---------------- epilogue for the segment ending at li ----------------
        if (!warp_wait(smem_u32(dfull), sg & 1, s_abort)) break;
        tc_fence_after();
        const int nt = static_cast<int>(tile / p.m_tiles);
        const int mt = static_cast<int>(tile - static_cast<long long>(nt) * p.m_tiles);
        const int n = nt * kTileRows + r;
        const int m0 = mt * NCOL;
        const float mul = __half2float(__ushort_as_half(p.scales[n])) * 4096.0f;
        const int c_lo = range_owner(tile * KT, total, G);
        const int c_hi = range_owner(tile * KT + KT - 1, total, G);
        const bool split = c_lo != c_hi;
        float* mine = p.partials + static_cast<long long>(partial_slot(c, tile, total, G, KT)) * NCOL * 128;
        for (int c0 = 0; c0 < NCOL; c0 += 16) {
          uint32_t v[16];
          tmem_ld_32x32b_x16(tmem + lane_base + S::kDCol + c0, v);
          tmem_wait_ld();
          if (c0 + 16 >= NCOL) {
            // accumulator fully read: the next segment may overwrite it
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(dempty));
          }
          if (split) {
#pragma unroll
            for (int j = 0; j < 16; ++j) mine[(c0 + j) * 128 + r] = __uint_as_float(v[j]);
          } else {
#pragma unroll
            for (int j = 0; j < 16; ++j) {
              const int m = m0 + c0 + j;
              if (m < p.M)
                p.y[static_cast<long long>(m) * p.N + n] =
                    __half_as_ushort(__float2half_rn(__uint_as_float(v[j]) * mul));
            }
          }
        }
        if (split) {
          // Publish this CTA's partial, then count arrivals; the last CTA of the
          // tile sums every partial in CTA order.  Warps of the group meet on an
          // mbarrier (bounded wait) rather than bar.sync, so an aborted warp
          // can never strand the others.
          __threadfence();
          __syncwarp();
          if (lane == 0) mbar_arrive(smem_u32(epi));
          if (!warp_wait(smem_u32(epi), ep & 1, s_abort)) break;
          ++ep;
          if (warp == 2 && lane == 0) {
            __threadfence();
            const unsigned int prev = atomicAdd(&p.counters[c_lo], 1u);
            *s_last = (prev == static_cast<unsigned int>(c_hi - c_lo)) ? 1 : 0;
          }
          __syncwarp();
          if (lane == 0) mbar_arrive(smem_u32(epi));
          if (!warp_wait(smem_u32(epi), ep & 1, s_abort)) break;
          ++ep;
          if (*s_last) {
            __threadfence();
            for (int col = 0; col < NCOL; ++col) {
              const int m = m0 + col;
              if (m >= p.M) break;
              float acc = 0.0f;
              for (int cc = c_lo; cc <= c_hi; ++cc) {
                const float* src = p.partials +
                                   static_cast<long long>(partial_slot(cc, tile, total, G, KT)) * NCOL * 128;
                acc += __ldcg(src + col * 128 + r);
              }
              p.y[static_cast<long long>(m) * p.N + n] = __half_as_ushort(__float2half_rn(acc * mul));
            }
            if (warp == 2 && lane == 0) p.counters[c_lo] = 0u;
          }
        }
        ++sg;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, S::kTmemCols);
  }
}

}  // namespace fp6
