// fp6_linear_decode.cuh -- the FP6 x FP16 linear layer for one token tile of
// at most 32 tokens (decode), sm_100a.
//
// Same product and the same work split as fp6_linear_kernel (fp6_linear.cuh):
// y[M,N] = x[M,K] . (scale (.) decode(W[N,K]))^T, fp32 accumulation, fp16 out,
// persistent CTAs over equal ranges of (row tile, step) iterations, split
// tiles finished, in CTA order, by the CTA holding their first steps.  What differs is the
// pipeline, shaped for the memory-bound regime where the tensor core is nearly
// idle and the integer pipe (the FP6 -> FP16 splice) and synchronisation
// latency are what remain:
//
//   warps 0..4G-1 G dequant groups of four warps (one per TMEM lane
//                 quadrant), taking every G-th step (G = 3; G = 2 for 64 token
//                 columns, where three groups' TMEM would not fit).  A group splices its
//                 step's T tiles into one of its own two TMEM slots, meets on a
//                 hardware named barrier, and one warp of the group (quadrant
//                 g, so the three groups issue from three different SM
//                 sub-partitions) issues the step's 4T MMAs into the group's
//                 own accumulator.  No hand-off to a separate issuer warp: the
//                 step's dequant-to-MMA path is one barrier, and the slot it
//                 refills next was released by the group's own commit two
//                 steps earlier, long done.
//   warps 4G..    epilogue warpgroup (four warps): per segment, the G group
//                 accumulators summed in group order, * scale, fp16
//                 store or split-K partial and fix-up.  Accumulators are double
//                 buffered across segments where TMEM has room (16 token
//                 columns), single buffered otherwise.
//   next warp     weight producer: one bulk copy of T packed tiles per step.
//   last warp     activation producer: one TMA box per step (T column tiles
//                 of NCOL rows x 64 columns, 128-byte swizzle, rows at or
//                 beyond M filled with zeros by the copy) into an smem ring.
//                 One copy per step, not one per tile: the copies of one
//                 issuing warp are served one after another, about 0.3 us
//                 each, which is as long as a step takes.  Completion is
//                 counted in bytes on each stage's barrier, so a stage is ready
//                 as soon as its own copies land, whatever was issued after.
//
// Ring ownership keeps every mbarrier's waits in phase order: weight stages
// (SW) and x stages (RX) are multiples of G, so each stage is always used
// by the same group; TMEM slots and accumulators belong to one group.
//
// Named barriers cannot time out, so the group loops never leave early: a
// warp whose bounded wait gave up (the abort flag is raised) skips its work
// but still runs every later barrier, and every other wait returns at once.
#pragma once
#include <cstdint>
#include <cuda.h>
#include <cuda_fp16.h>

#include "fp6_format.cuh"
#include "fp6_linear.cuh"
#include "ptx.cuh"

namespace fp6 {


template <int NCOL, Fmt F = Fmt::E3M2>
struct DecodeShape {
  static_assert(NCOL == 16 || NCOL == 32 || NCOL == 64, "decode variants: 16, 32 or 64 token columns");
  // dequant groups: three, or two where three groups' TMEM slots and
  // accumulators would not fit in the 512 columns (64 token columns)
  static constexpr int kGroups = (NCOL == 64) ? 2 : 3;
  static constexpr int kEpiWarp = 4 * kGroups;              // four epilogue warps
  static constexpr int kWProdWarp = kEpiWarp + 4;
  static constexpr int kXProdWarp = kWProdWarp + 1;
  static constexpr int kThreads = 32 * (kXProdWarp + 1);   // 576 (three groups) or 448
  static constexpr int kTMax = 2;                           // tiles per step, at most
  static constexpr int kXTile = NCOL * 128;                 // NCOL rows x 64 fp16, 128-byte swizzled
  static constexpr int kXStage = kTMax * kXTile;
  static constexpr int kTileBytes = Format<F>::kTileBytes;
  static constexpr int kWStage = kTMax * kTileBytes;
  static constexpr int kRX = (NCOL == 16) ? 9 : (NCOL == 32) ? 6 : 4;   // x stages
  // weight stages: 15 (12) of 6-bit tiles; the same bytes in FP4 tiles
  static constexpr int kSW = ((NCOL == 16) ? 15 : 12) * 6144 / kTileBytes / kGroups * kGroups;
  static constexpr int kSlots = 2 * kGroups;               // TMEM slots: two per group
  static constexpr int kSlotCols = kTMax * 32;
  static constexpr int kDCol = kSlots * kSlotCols;          // accumulators after the slots
  // accumulator sets: two (segments alternate) when they fit in TMEM
  // MMA-issuing warps per group: each issues the k-slices 4/kIss*i .. of every
  // tile of the step into its own accumulator.  One thread issues one MMA in
  // about 160 cycles, so two issuers halve the group's issue time where TMEM
  // has room for their accumulators (16 token columns).
  static constexpr int kIss = (NCOL == 16) ? 2 : 1;
  static constexpr int kSets = (kDCol + 2 * kGroups * kIss * NCOL <= static_cast<int>(kTmemCols)) ? 2 : 1;
  static constexpr int kAccCols = kSets * kGroups * kIss * NCOL;   // [set][group][issuer][NCOL]
  static constexpr int kWOff = kRX * kXStage;
  static constexpr int kBarOff = kWOff + kSW * kWStage;
  // wfull, wempty [SW]; xfull, xempty [RX]; slot free [6]; dfull, dempty [2]; epi [2]; done
  static constexpr int kNumBars = 2 * kSW + 2 * kRX + kSlots + 2 + 2 + 2 + 1;
  static constexpr int kBarrierBytes = 1024;
  static constexpr int kSmemBytes = kBarOff + kBarrierBytes + 1024;  // + alignment slack
  static_assert(kSW % kGroups == 0 && kRX % kGroups == 0, "stages owned by one group");
  static_assert(kDCol + kAccCols <= static_cast<int>(kTmemCols), "TMEM budget");
  static_assert(kXTile % 1024 == 0 && kTileBytes % 1024 == 0, "1024-byte aligned tiles");
  static_assert(kNumBars * 8 + 32 <= kBarrierBytes, "barrier area");
  static_assert(kSmemBytes <= 232448, "shared memory");
};

// Local step range [a, b] of segment sg (the CTA's steps in tile tile_first + sg).
__device__ __forceinline__ void segment_range(int sg, long long tile_first, long long s0, int KS, int n_local,
                                              int* a, int* b) {
  const long long t = tile_first + sg;
  const long long lo = t * KS - s0, hi = (t + 1) * KS - s0 - 1;
  *a = lo < 0 ? 0 : static_cast<int>(lo);
  *b = hi > n_local - 1 ? n_local - 1 : static_cast<int>(hi);
}

// First step of group g (steps li with li % 3 == g) at or after a.
__device__ __forceinline__ int group_first(int g, int a, int groups) {
  return a + ((g - a % groups) + groups) % groups;
}

template <int NCOL, Fmt F = Fmt::E3M2>
__global__ void __launch_bounds__(DecodeShape<NCOL, F>::kThreads, 1)
    fp6_linear_decode_kernel(const __grid_constant__ CUtensorMap tmap_x, const LinearParams p) {
  using S = DecodeShape<NCOL, F>;
  using Fm = Format<F>;
  constexpr int kSW = S::kSW;
  constexpr int kRX = S::kRX;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S::kBarOff);
  uint64_t* wfull = bars;
  uint64_t* wempty = wfull + kSW;
  uint64_t* xfull = wempty + kSW;
  uint64_t* xempty = xfull + kRX;
  uint64_t* slotfree = xempty + kRX;              // [6]: a group's MMAs on the slot are done
  uint64_t* dfull = slotfree + S::kSlots;         // [2]: a segment's accumulators are complete
  uint64_t* dempty = dfull + 2;                   // [2]: the epilogue has read them
  uint64_t* epi = dempty + 2;                     // [2]: fix-up meeting (epi[0] only)
  uint64_t* done = epi + 2;                       // every MMA finished (before TMEM release)
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + S::kNumBars);
  volatile int* s_last = reinterpret_cast<volatile int*>(tmem_holder + 1);  // [2]
  volatile int* s_abort = s_last + 2;
  volatile int* s_never = s_abort + 1;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int G = p.grid;
  const int c = blockIdx.x;
  const long long total = p.total_steps;
  const int KS = p.k_steps;
  const int T = p.T;
  const int KT = p.k_tiles;
  const long long s0 = range_begin(c, total, G);
  const long long s1 = range_begin(c + 1, total, G);
  const int n_local = static_cast<int>(s1 - s0);
  const long long tile_first = s0 / KS;
  const long long tile_last = (s1 - 1) / KS;
  const int nseg = static_cast<int>(tile_last - tile_first + 1);

  grid_launch_dependents();

  if (threadIdx.x < S::kNumBars) {
    const int b = threadIdx.x;
    const int bx = 2 * kSW, bs = bx + 2 * kRX, bd = bs + S::kSlots;
    uint32_t count = 1;                                       // wfull, xfull
    if (b >= kSW && b < bx) count = 4;                        // wempty: the group's four warps
    else if (b >= bx + kRX && b < bd) count = S::kIss;        // xempty, slotfree: the group's issuers
    else if (b >= bd && b < bd + 2) count = S::kGroups * S::kIss;  // dfull: one arrival per issuer
    else if (b >= bd + 2 && b < bd + 6) count = 4;            // dempty, epi: epilogue warps
    else if (b == bd + 6) count = S::kGroups * S::kIss;       // done: one commit per issuer
    mbar_init(smem_u32(&bars[b]), count);
    fence_barrier_init();
  }
  if (threadIdx.x == 0) {
    s_last[0] = 0;
    s_last[1] = 0;
    *s_abort = 0;
    *s_never = 0;
  }
  if (warp == S::kXProdWarp && lane == 0) prefetch_tensormap(&tmap_x);
  if (warp == 0) {
    tmem_alloc(smem_u32(tmem_holder), kTmemCols);
    tmem_relinquish();
  }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;

  if (warp == S::kWProdWarp) {
    // ---------------- weight producer ----------------
    const uint64_t pol = policy_evict_first();
    StepCursor cur(s0, KS, 1);
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
    for (int li = issued > kSW ? issued - kSW : 0; li < issued; ++li)
      warp_wait(smem_u32(&wfull[li % kSW]), (li / kSW) & 1, s_never);
  } else if (warp == S::kXProdWarp) {
    // ---------------- activation producer ----------------
    grid_dependency_wait();                  // x is written by earlier work in the stream
    const uint64_t pol = policy_evict_last();
    const uint32_t bytes = static_cast<uint32_t>(T) * S::kXTile;
    int ks = static_cast<int>(s0 - tile_first * KS);
    int issued = 0;
    for (int li = 0; li < n_local; ++li, ks = (ks + 1 == KS) ? 0 : ks + 1) {
      const int s = li % kRX;
      if (li >= kRX && !warp_wait(smem_u32(&xempty[s]), ((li / kRX) - 1) & 1, s_abort)) break;
      if (lane == 0) {
        const uint32_t fb = smem_u32(&xfull[s]);
        mbar_arrive_expect_tx(fb, bytes);
        tma_load_3d(smem_u32(smem + s * S::kXStage), &tmap_x, fb, 0, 0, ks * T, pol);
      }
      __syncwarp();
      ++issued;
    }
    // Leave no copy in flight.
    for (int li = issued > kRX ? issued - kRX : 0; li < issued; ++li)
      warp_wait(smem_u32(&xfull[li % kRX]), (li / kRX) & 1, s_never);
  } else if (warp < 4 * S::kGroups) {
    // ---------------- dequant groups, each issuing its own MMAs ----------------
    const int g = warp >> 2;
    const int quad = warp & 3;               // TMEM lanes 32*quad .. 32*quad+31
    const int r = quad * 32 + lane;          // weight row within the tile
    // issuer index of this warp in its group (-1: not an issuer); the issuers
    // of the three groups sit on different SM sub-partitions
    const int iss = (quad == g) ? 0 : (S::kIss == 2 && quad == ((g + 2) & 3)) ? 1 : -1;
    const bool issuer = iss >= 0;
    constexpr int kSlice = 4 / S::kIss;      // k-slices of a tile per issuer
    const int kk0 = (iss < 0 ? 0 : iss) * kSlice;
    const uint32_t lane_base = static_cast<uint32_t>(quad * 32) << 16;
    constexpr uint32_t idesc = idesc_f16_f32(128, NCOL);
    bool ok = true;
    int j = 0;                               // this group's steps so far
    for (int sg = 0; sg < nseg; ++sg) {
      int a, b;
      segment_range(sg, tile_first, s0, KS, n_local, &a, &b);
      const int set = sg % S::kSets;
      const uint32_t d_tmem = tmem + S::kDCol + ((set * S::kGroups + g) * S::kIss + (iss < 0 ? 0 : iss)) * NCOL;
      // The accumulators of this set were last used kSets segments ago: the
      // epilogue must have read them before the first MMA or arrival.
      if (issuer && sg >= S::kSets)
        ok = warp_wait(smem_u32(&dempty[set]), ((sg / S::kSets) - 1) & 1, s_abort) && ok;
      bool first = true;
      for (int li = group_first(g, a, S::kGroups); li <= b; li += S::kGroups, ++j) {
        const int sw = li % kSW;
        const int sx = li % kRX;
        const int slot = 2 * g + (j & 1);
        ok = warp_wait(smem_u32(&wfull[sw]), (li / kSW) & 1, s_abort) && ok;
        if (j >= 2) ok = warp_wait(smem_u32(&slotfree[slot]), ((j >> 1) - 1) & 1, s_abort) && ok;
        tc_fence_after();
        if (ok) {
          const uint8_t* wst = smem + S::kWOff + sw * S::kWStage;
          for (int t = 0; t < T; ++t) {
            uint32_t Fw[Fm::kRowWords], w[32];
            Fm::load(wst + t * Fm::kTileBytes, r, Fw);
            Fm::rebuild(Fw, w);
            tmem_st_32x32b_x32(tmem + lane_base + slot * S::kSlotCols + t * 32, w);
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&wempty[sw]));   // smem fragments read
        tmem_wait_st();
        tc_fence_before();
        named_bar_sync(1 + g, 128);                          // the slot is written by all four warps
        if (issuer) {
          ok = warp_wait(smem_u32(&xfull[sx]), (li / kRX) & 1, s_abort) && ok;
          if (lane == 0) {
            tc_fence_after();
            if (ok) {
              const uint64_t bdesc0 = smem_desc_sw128(smem_u32(smem + sx * S::kXStage));
              const uint32_t a0 = tmem + slot * S::kSlotCols;
              for (int t = 0; t < T; ++t) {
                const uint64_t bdesc = bdesc0 + static_cast<uint64_t>(t * (S::kXTile >> 4));
#pragma unroll
                for (int q = 0; q < kSlice; ++q) {
                  const int kk = kk0 + q;
                  mma_f16_ts(d_tmem, a0 + t * 32 + kk * 8, bdesc + static_cast<uint64_t>(kk * 2), idesc,
                             (first && t == 0 && q == 0) ? 0u : 1u);
                }
              }
            }
            tc_commit(smem_u32(&slotfree[slot]));
            tc_commit(smem_u32(&xempty[sx]));
          }
          __syncwarp();
        }
        first = false;
      }
      // One arrival per group and segment: the commit covers this group's
      // MMAs into the set; a group with no step in the segment just arrives.
      if (issuer) {
        if (lane == 0) {
          if (!first) tc_commit(smem_u32(&dfull[set]));
          else mbar_arrive(smem_u32(&dfull[set]));
        }
        __syncwarp();
      }
    }
    if (issuer) {
      if (lane == 0) tc_commit(smem_u32(done));
      __syncwarp();
      warp_wait(smem_u32(done), 0, s_never);
    }
  } else if (warp >= S::kEpiWarp && warp < S::kEpiWarp + 4) {
    // ---------------- epilogue warpgroup: segments in order ----------------
    // A split row tile is finished by its first CTA c_lo, which reaches the
    // tile at the end of its range; every later contributor reaches it at the
    // start of its own range, publishes its partial there (release add on the
    // tile's counter) and moves on.  The finishing CTA waits for those
    // partials and sums them (in CTA order) while its own MMAs still run, so
    // the end of its range costs one TMEM read and the store of y.  Each
    // epilogue warp of a contributor releases its 32 rows with one add, so the
    // counter reaches 4 per contributor.
    grid_dependency_wait();                  // y, partials and counters may be in use before this kernel
    const int quad = warp & 3;
    const int r = quad * 32 + lane;
    const uint32_t lane_base = static_cast<uint32_t>(quad * 32) << 16;
    const int mcount = min(NCOL, p.M);
    for (int sg = 0; sg < nseg; ++sg) {
      const long long tile = tile_first + sg;
      const int set = sg % S::kSets;
      int a, b;
      segment_range(sg, tile_first, s0, KS, n_local, &a, &b);
      const int n = static_cast<int>(tile) * kTileRows + r;
      const float mul = __half2float(__ushort_as_half(p.scales[n]));
      const int c_lo = range_owner(tile * KS, total, G);
      const int c_hi = range_owner(tile * KS + KS - 1, total, G);
      const bool split = c_lo != c_hi;
      const bool finisher = (c == c_lo);
      float pre[NCOL];
#pragma unroll
      for (int j = 0; j < NCOL; ++j) pre[j] = 0.0f;
      if (split && finisher) {
        // the other contributors' partials, summed in CTA order
        if (!wait_counter(&p.counters[c_lo], 4u * static_cast<unsigned int>(c_hi - c_lo), s_abort)) break;
        for (int cc = c_lo + 1; cc <= c_hi; ++cc) {
          const float* src = p.partials + static_cast<long long>(cc) * NCOL * 128 + r;
#pragma unroll
          for (int j = 0; j < NCOL; ++j)
            if (j < mcount) pre[j] += __ldcg(src + j * 128);
        }
        // Reset the counter for the next launch once all four warps have seen
        // it complete (a CTA finishes at most one split tile: one meeting).
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&epi[0]));
        if (quad == 0 && warp_wait(smem_u32(&epi[0]), 0, s_abort) && lane == 0) p.counters[c_lo] = 0u;
      }
      if (!warp_wait(smem_u32(&dfull[set]), (sg / S::kSets) & 1, s_abort)) break;
      tc_fence_after();
      float* part = p.partials + static_cast<long long>(c) * NCOL * 128 + r;
#pragma unroll
      for (int ch = 0; ch < NCOL / 8; ++ch) {
        const int c0 = ch * 8;
        if (c0 >= mcount) break;
        float acc[8];
#pragma unroll
        for (int jj = 0; jj < 8; ++jj) acc[jj] = 0.0f;
        // groups in order: the sum is the same on every run
        for (int g = 0; g < S::kGroups; ++g) {
          if (group_first(g, a, S::kGroups) > b) continue;   // no step of group g in this segment
          for (int i = 0; i < S::kIss; ++i) {
            uint32_t v[8];
            tmem_ld_32x32b_x8(tmem + lane_base + S::kDCol + ((set * S::kGroups + g) * S::kIss + i) * NCOL + c0, v);
            tmem_wait_ld();
#pragma unroll
            for (int jj = 0; jj < 8; ++jj) acc[jj] += __uint_as_float(v[jj]);
          }
        }
        if (split && !finisher) {
#pragma unroll
          for (int jj = 0; jj < 8; ++jj) __stcg(part + (c0 + jj) * 128, acc[jj]);
        } else {
#pragma unroll
          for (int jj = 0; jj < 8; ++jj) {
            const float v = pre[c0 + jj] + acc[jj];
            if (c0 + jj < mcount)
              p.y[static_cast<long long>(c0 + jj) * p.N + n] = __half_as_ushort(__float2half_rn(v * mul));
          }
        }
      }
      // accumulators read: the set may be reused kSets segments on
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&dempty[set]));
      if (split && !finisher) {
        __syncwarp();                        // the warp's partial rows are written
        if (lane == 0) red_release_add(&p.counters[c_lo], 1u);
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
