// fp6_linear_wave.cuh -- the fused FP6 x FP16 linear layer for many token
// tiles (prefill), sm_100a: the general kernel's pipeline (fp6_linear.cuh:
// same warp roles, rings, shapes and barriers) with whole tiles per CTA.
//
// CTA c takes the output tiles c, c + G, c + 2G, ... and every K step of
// each, so no tile is split and the epilogue stores y directly.  The tiles
// are numbered in bands of `band` token tiles: within a band the token tile
// runs fastest, then the row tile.  The G tiles that run at the same time
// then span about G / band row tiles and `band` token tiles and, moving
// through K together, share every weight and activation slice through L2,
// where the stream-K ranges (row-tile major) have each CTA stream its row
// tiles once per token tile.  The planner uses this kernel only when the last
// wave of tiles is nearly full.
#pragma once
#include <cstdint>
#include <cuda.h>
#include <cuda_fp16.h>

#include "fp6_format.cuh"
#include "fp6_linear.cuh"
#include "ptx.cuh"

namespace fp6 {

// Row and token tile of tile t in the banded order.
__device__ __forceinline__ void wave_tile_coords(long long t, int NT, int MT, int band, int* nt, int* mt) {
  const long long per_band = static_cast<long long>(band) * NT;
  const int b = static_cast<int>(t / per_band);
  const int r = static_cast<int>(t - b * per_band);
  const int width = min(band, MT - b * band);
  *nt = r / width;
  *mt = b * band + (r - *nt * width);
}

// Walks a CTA's steps: tiles c, c + G, ..., every step of each.
struct WaveCursor {
  int ks, nt, mt;
  long long tile;
  int G, KS, NT, MT, band;
  __device__ __forceinline__ WaveCursor(long long tile0, int G_, int KS_, int NT_, int MT_, int band_)
      : ks(0), tile(tile0), G(G_), KS(KS_), NT(NT_), MT(MT_), band(band_) {
    wave_tile_coords(tile, NT, MT, band, &nt, &mt);
  }
  __device__ __forceinline__ void next() {
    if (++ks == KS) {
      ks = 0;
      tile += G;
      wave_tile_coords(tile, NT, MT, band, &nt, &mt);
    }
  }
};

template <int NCOL, Fmt F = Fmt::E3M2>
__global__ void __launch_bounds__(kLinearThreads, 1)
    fp6_linear_wave_kernel(const __grid_constant__ CUtensorMap tmap_x, const LinearParams p) {
  using S = LinearShape<NCOL, F>;
  using Fm = Format<F>;
  constexpr int kR = S::kR;
  constexpr int kRX = S::kRX;
  constexpr int kSW = S::kSW;
  constexpr int kISS = S::kIssuers;
  constexpr int kL = S::kL;
  constexpr int kEC = S::kEC;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S::kBarOff);
  uint64_t* wfull = bars;
  uint64_t* wempty = wfull + kSW;
  uint64_t* xfull = wempty + kSW;                 // x stage landed (producer arrive + tx)
  uint64_t* ready = xfull + kRX;                  // step ready (its dequant group)
  uint64_t* freed = ready + kL;                   // step's MMAs complete (issuer commits)
  uint64_t* dfull = freed + kL;
  uint64_t* dempty = dfull + 1;
  uint64_t* done = dempty + 1;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + S::kNumBars);
  volatile int* s_abort = reinterpret_cast<volatile int*>(tmem_holder + 1);
  volatile int* s_never = s_abort + 1;            // an abort flag nothing raises (final drains)

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int G = p.grid;
  const int c = blockIdx.x;
  const int KS = p.k_steps;
  const int T = p.T;
  const int KT = p.k_tiles;
  const int NT = p.n_tiles;
  const int MT = p.m_tiles;
  const int band = min(4, MT);
  const long long tiles = static_cast<long long>(NT) * MT;
  const int nseg = tiles > c ? static_cast<int>((tiles - 1 - c) / G) + 1 : 0;   // this CTA's tiles
  const int n_local = nseg * KS;

  grid_launch_dependents();

  // Barrier set-up as in the general kernel (without its split-tile copy
  // barriers).
  if (threadIdx.x < S::kNumBars) {
    const int b = threadIdx.x;
    const int bx = 2 * kSW, br = bx + kRX, bf = br + kL, bd = bf + kL;
    uint32_t count = 1;                                       // wfull, xfull: producer arrive + tx
    if (b >= kSW && b < bx) count = 4;                        // wempty: the reading group's 4 warps
    else if (b >= br && b < bf) count = 4;                    // ready: the step's dequant group
    else if (b >= bf && b < bd) count = kISS;                 // freed: issuer commits
    else if (b == bd) count = kISS;                           // dfull
    else if (b == bd + 1) count = 4;                          // dempty: epilogue warps
    else if (b == bd + 2) count = kISS;                       // done
    mbar_init(smem_u32(&bars[b]), count);
    fence_barrier_init();
  }
  if (threadIdx.x == 0) {
    *s_abort = 0;
    *s_never = 0;
  }
  if (warp == kXProdWarp && lane == 0) prefetch_tensormap(&tmap_x);
  if (warp == 0) {
    tmem_alloc(smem_u32(tmem_holder), kTmemCols);
    tmem_relinquish();
  }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;

  if (warp == kWProdWarp) {
    // ---------------- weight producer ----------------
    const uint64_t pol = policy_evict_first();
    WaveCursor cur(c, G, KS, NT, MT, band);
    const uint32_t bytes = static_cast<uint32_t>(T) * Fm::kTileBytes;
    int issued = 0;
    for (int li = 0; li < n_local; ++li, cur.next()) {
      const int s = li % kSW;
      if (li >= kSW && !warp_wait(smem_u32(&wempty[s]), ((li / kSW) - 1) & 1, s_abort)) break;
      if (lane == 0) {
        const uint32_t fb = smem_u32(&wfull[s]);
        mbar_arrive_expect_tx(fb, bytes);
        bulk_load(smem_u32(smem + S::kWOff + s * S::kWStage),
                  p.packed + (static_cast<long long>(cur.nt) * KT + static_cast<long long>(cur.ks) * T) * Fm::kTileBytes,
                  bytes, fb, pol);
      }
      __syncwarp();
      ++issued;
    }
    // Leave no copy in flight: the last copy issued into every stage has landed.
    for (int li = issued > kSW ? issued - kSW : 0; li < issued; ++li)
      warp_wait(smem_u32(&wfull[li % kSW]), (li / kSW) & 1, s_never);
  } else if (warp == kXProdWarp) {
    // ---------------- activation producer ----------------
    grid_dependency_wait();                  // x is written by earlier work in the stream
    const uint64_t pol = policy_evict_last();
    WaveCursor cur(c, G, KS, NT, MT, band);
    const uint32_t bytes = static_cast<uint32_t>(T) * S::kXTile;
    int issued = 0;
    for (int li = 0; li < n_local; ++li, cur.next()) {
      const int s = li % kRX;
      // the stage's previous step (li - RX) has had its MMAs
      if (li >= kRX && !warp_wait(smem_u32(&freed[(li - kRX) % kL]), ((li - kRX) / kL) & 1, s_abort)) break;
      if (lane == 0) {
        const uint32_t fb = smem_u32(&xfull[s]);
        mbar_arrive_expect_tx(fb, bytes);
        tma_load_3d(smem_u32(smem + s * S::kXStage), &tmap_x, fb, 0, cur.mt * NCOL, cur.ks * T, pol);
      }
      __syncwarp();
      ++issued;
    }
    for (int li = issued > kRX ? issued - kRX : 0; li < issued; ++li)
      warp_wait(smem_u32(&xfull[li % kRX]), (li / kRX) & 1, s_never);
  } else if (warp < kISS) {
    // ---------------- MMA issuer `warp`: its k-slices or its token half of every tile ----------------
    constexpr uint32_t idesc = idesc_f16_f32(128, S::kIssN);
    constexpr int kSlice = S::kIssSlices;
    const int kk0 = S::kNSplit ? 0 : warp * kSlice;
    const uint32_t d_tmem = tmem + S::kDCol + warp * (S::kNSplit ? S::kIssN : NCOL);
    const uint32_t b_off = S::kNSplit ? warp * S::kIssN * 128 : 0;   // its tokens' rows of the x tile
    // The loop runs in lane 0 alone: a barrier test by one lane costs about
    // 13 cycles against about 110 for a whole warp, and a warp issues
    // tcgen05.mma at one per ~50 cycles whichever lanes issue, so per-step
    // warp-wide waits would cost the tensor pipe its feed.
    if (lane == 0) {
      int sg = 0;
      int ks = 0;
      for (int li = 0; li < n_local; ++li, ks = (ks + 1 == KS) ? 0 : ks + 1) {
        const bool seg_first = (ks == 0);
        const bool seg_last = (ks == KS - 1);
        const int s = li % kR;
        const int sx = li % kRX;
        if (seg_first && sg > 0 && !wait_bounded(smem_u32(dempty), (sg - 1) & 1, s_abort)) break;
        if (!wait_bounded(smem_u32(&ready[li % kL]), (li / kL) & 1, s_abort)) break;
        {
          tc_fence_after();
          const uint64_t bdesc0 = smem_desc_sw128(smem_u32(smem + sx * S::kXStage) + b_off);
          const uint32_t a0 = tmem + s * S::kSlotCols;
          for (int t = 0; t < T; ++t) {
            const uint64_t bdesc = bdesc0 + static_cast<uint64_t>(t * (S::kXTile >> 4));
#pragma unroll
            for (int j = 0; j < kSlice; ++j) {
              const int kk = kk0 + j;
              mma_f16_ts(d_tmem, a0 + t * 32 + kk * 8, bdesc + static_cast<uint64_t>(kk * 2), idesc,
                         (seg_first && t == 0 && j == 0) ? 0u : 1u);
            }
          }
          tc_commit(smem_u32(&freed[li % kL]));
          if (seg_last) tc_commit(smem_u32(dfull));
        }
        if (seg_last) ++sg;
      }
      // All issued MMAs have finished before TMEM is released.
      tc_commit(smem_u32(done));
      wait_bounded(smem_u32(done), 0, s_never);
    }
    __syncwarp();
  } else if (warp >= kFirstDeqWarp) {
    // ---------------- dequant warpgroups ----------------
    const int g = (warp - kFirstDeqWarp) >> 2;
    const int quad = warp & 3;               // TMEM lanes 32*quad .. 32*quad+31
    const int r = quad * 32 + lane;          // weight row within the tile
    const uint32_t lane_base = static_cast<uint32_t>(quad * 32) << 16;
    const auto aux = Fm::make_aux();
    for (int li = g; li < n_local; li += kDeqGroups) {
      const int sw = li % kSW;
      const int s = li % kR;
      if (!warp_wait(smem_u32(&wfull[sw]), (li / kSW) & 1, s_abort)) break;
      if (li >= kR && !warp_wait(smem_u32(&freed[(li - kR) % kL]), ((li - kR) / kL) & 1, s_abort)) break;
      tc_fence_after();
      const uint8_t* wst = smem + S::kWOff + sw * S::kWStage;
      for (int t = 0; t < T; ++t) {
        uint32_t Fw[Fm::kRowWords], w[32];
        Fm::load(wst + t * Fm::kTileBytes, r, Fw);
        rebuild_row<F>(Fw, w, aux);
        tmem_st_32x32b_x32(tmem + lane_base + s * S::kSlotCols + t * 32, w);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&wempty[sw]));   // smem fragments read
      tmem_wait_st();
      // The step's x stage has landed too: the issuer then waits on one barrier.
      if (!warp_wait(smem_u32(&xfull[li % kRX]), (li / kRX) & 1, s_abort)) break;
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&ready[li % kL]));
    }
  } else if (warp >= kEpiWarp && warp < kEpiWarp + 4) {
    // ---------------- epilogue warpgroup: this CTA's tiles in order ----------------
    grid_dependency_wait();                  // y may be in use before this kernel
    const int quad = warp & 3;
    const int r = quad * 32 + lane;
    const uint32_t lane_base = static_cast<uint32_t>(quad * 32) << 16;
    for (int sg = 0; sg < nseg; ++sg) {
      const long long tile = c + static_cast<long long>(sg) * G;
      if (!warp_wait(smem_u32(dfull), sg & 1, s_abort)) break;
      tc_fence_after();
      int nt, mt;
      wave_tile_coords(tile, NT, MT, band, &nt, &mt);
      const int n = nt * kTileRows + r;
      const int m0 = mt * NCOL;
      const int mcount = min(NCOL, p.M - m0);
      const float mul = __half2float(__ushort_as_half(p.scales[n]));
      for (int c0 = 0; c0 < NCOL; c0 += kEC) {
        constexpr int kAcc = S::kAccIssuers;
        uint32_t v[kAcc][kEC];
#pragma unroll
        for (int i = 0; i < kAcc; ++i) tmem_ld_cols<kEC>(tmem + lane_base + S::kDCol + i * NCOL + c0, v[i]);
        tmem_wait_ld();
        float acc[kEC];
#pragma unroll
        for (int j = 0; j < kEC; ++j) {
          float a = __uint_as_float(v[0][j]);
#pragma unroll
          for (int i = 1; i < kAcc; ++i) a += __uint_as_float(v[i][j]);
          acc[j] = a;
        }
        if (c0 + kEC >= NCOL) {
          // accumulators fully read: the next tile may overwrite them
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(smem_u32(dempty));
        }
        store_y_pairs<kEC>(p.y, acc, mul, m0 + c0, mcount - c0, p.N, n, lane);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace fp6
