// fp6_linear_decode.cuh -- the FP6 x FP16 linear layer for one token tile of
// at most 64 tokens (decode), sm_100a.
//
// Same product and the same work split as fp6_linear_kernel (fp6_linear.cuh):
// y[M,N] = x[M,K] . (scale (.) decode(W[N,K]))^T, fp32 accumulation, fp16 out,
// persistent CTAs over equal ranges of (row tile, step) iterations.  What
// differs is the pipeline, shaped for the memory-bound regime where the
// tensor core is nearly idle and the integer pipe (the FP6 -> FP16 splice)
// and synchronisation latency are what remain:
//
//   warps 0..4G-1 G dequant groups of four warps (one per TMEM lane
//                 quadrant), taking every G-th step (G = 3; G = 2 for 64 token
//                 columns, where three groups' TMEM would not fit).  A group splices its
//                 step's T tiles into one of its own two TMEM slots; each warp
//                 then reports the slot written on an mbarrier and goes on to
//                 the next step, so splicing never waits for MMA issue.
//   warps 4G..    epilogue warpgroup (four warps): per segment, the group
//                 accumulators summed in a fixed order, * scale, fp16
//                 store or split-K partial and fix-up.  Accumulators are double
//                 buffered across segments where TMEM has room (16 token
//                 columns), single buffered otherwise.
//   next warps    MMA issuers, kIss per group (two for 16 token columns, else
//                 one): each waits for its group's slot and the step's
//                 activations, issues its share of the step's 4T MMAs into its
//                 own accumulator and commits, which frees the slot and the x
//                 stage.  One thread issues an MMA in about 50 cycles, and
//                 several issuing warps overlap, so the issue of one group's
//                 step overlaps the splicing of the next.
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
// (SW) are a multiple of G and x stages are the TMEM slots, so each stage is
// always used by the same group; slots and accumulators belong to one group.
//
// Split row tiles.  A row tile whose steps span CTAs c_lo .. c_hi is finished
// by exactly one of them, and no CTA ever waits for another (so nothing
// depends on the CTAs of a launch being resident at the same time).  Each
// epilogue warp (32 rows) has its own counter per tile.  Every contributor
// after c_lo reaches the tile at the start of its range, writes its partial
// sums and adds one to the counter (release).  c_lo reaches the tile at the
// end of its range; if the counter shows every other contributor (acquire),
// it sums their partials with its own accumulators and stores y.  Otherwise
// it writes its own partial and adds one as well, and whichever contributor's
// add completes the count sums the partials.  The sum is always formed in the
// same order (contributors c_lo+1 .. c_hi, then c_lo), so results are
// bit-reproducible whichever CTA finishes the tile.  The finisher resets the
// counter to zero for the next launch.
//
// The role loops never leave early: a warp whose bounded wait gave up (the
// abort flag is raised) skips its work but still makes every later arrival,
// and every other wait returns at once.
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
  // MMA-issuing warps per group: each issues the k-slices 4/kIss*i .. of every
  // tile of the step into its own accumulator.  Two issuers per group where
  // TMEM has room for their accumulators (16 token columns).
  static constexpr int kIss = (NCOL == 16) ? 2 : 1;
  static constexpr int kEpiWarp = 4 * kGroups;              // four epilogue warps
  static constexpr int kIssWarp = kEpiWarp + 4;             // kGroups * kIss issuer warps
  static constexpr int kWProdWarp = kIssWarp + kGroups * kIss;
  static constexpr int kXProdWarp = kWProdWarp + 1;
  static constexpr int kThreads = 32 * (kXProdWarp + 1);   // 768, 672 or 512
  static constexpr int kTMax = 2;                           // tiles per step, at most
  static constexpr int kXTile = NCOL * 128;                 // NCOL rows x 64 fp16, 128-byte swizzled
  static constexpr int kXStage = kTMax * kXTile;
  static constexpr int kTileBytes = Format<F>::kTileBytes;
  static constexpr int kWStage = kTMax * kTileBytes;
  // x stages: one per TMEM slot.  Step li uses slot and x stage
  // 2*(li % G) + ((li / G) & 1); both are free again once the step's MMAs
  // have completed, which one commit per issuer reports.
  static constexpr int kRX = 2 * kGroups;
  // weight stages: 15 (12) of 6-bit tiles; the same bytes in FP4 tiles
  static constexpr int kSW = ((NCOL == 16) ? 15 : 12) * 6144 / kTileBytes / kGroups * kGroups;
  static constexpr int kSlots = 2 * kGroups;               // TMEM slots: two per group
  static constexpr int kSlotCols = kTMax * 32;
  static constexpr int kDCol = kSlots * kSlotCols;          // accumulators after the slots
  // accumulator sets: two (segments alternate) when they fit in TMEM
  static constexpr int kSets = (kDCol + 2 * kGroups * kIss * NCOL <= static_cast<int>(kTmemCols)) ? 2 : 1;
  static constexpr int kAccCols = kSets * kGroups * kIss * NCOL;   // [set][group][issuer][NCOL]
  static constexpr int kWOff = kRX * kXStage;
  static constexpr int kBarOff = kWOff + kSW * kWStage;
  // wfull, wempty [SW]; xfull [RX]; slot free [slots] (frees the x stage too);
  // slot ready [slots]; dfull, dempty [2]; done
  static constexpr int kNumBars = 2 * kSW + kRX + 2 * kSlots + 2 + 2 + 1;
  static constexpr int kBarrierBytes = 1024;
  static constexpr int kSmemBytes = kBarOff + kBarrierBytes + 1024;  // + alignment slack
  static_assert(kSW % kGroups == 0 && kRX == kSlots, "stages owned by one group; one x stage per slot");
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

// Partial sums of a split tile, [2G][NCOL][128] fp32: slot 2c for the tile a
// CTA's range starts in, 2c + 1 for the one it ends in.
template <int NCOL>
__device__ __forceinline__ float* decode_partial(float* partials, int slot, int r) {
  return partials + static_cast<long long>(slot) * NCOL * 128 + r;
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
  uint64_t* slotfree = xfull + kRX;               // [slots]: a step's MMAs are done (slot and x stage free)
  uint64_t* slotready = slotfree + S::kSlots;     // [slots]: the group's four warps have written the slot
  uint64_t* dfull = slotready + S::kSlots;        // [2]: a segment's accumulators are complete
  uint64_t* dempty = dfull + 2;                   // [2]: the epilogue has read them
  uint64_t* done = dempty + 2;                    // every MMA finished (before TMEM release)
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + S::kNumBars);
  volatile int* s_abort = reinterpret_cast<volatile int*>(tmem_holder + 1);
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
    const int bx = 2 * kSW, bs = bx + kRX, br = bs + S::kSlots, bd = br + S::kSlots;
    uint32_t count = 1;                                       // wfull, xfull
    if (b >= kSW && b < bx) count = 4;                        // wempty: the group's four warps
    else if (b >= bs && b < br) count = S::kIss;              // slotfree: the group's issuers
    else if (b >= br && b < bd) count = 4;                    // slotready: the group's four warps
    else if (b >= bd && b < bd + 2) count = S::kGroups * S::kIss;  // dfull: one arrival per issuer
    else if (b >= bd + 2 && b < bd + 4) count = 4;            // dempty: epilogue warps
    else if (b == bd + 4) count = S::kGroups * S::kIss;       // done: one commit per issuer
    mbar_init(smem_u32(&bars[b]), count);
    fence_barrier_init();
  }
  if (threadIdx.x == 0) {
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
      const int jg = li / S::kGroups;                         // the step's index in its group
      const int s = 2 * (li - jg * S::kGroups) + (jg & 1);
      if (li >= kRX && !warp_wait(smem_u32(&slotfree[s]), ((jg >> 1) - 1) & 1, s_abort)) break;
      if (lane == 0) {
        const uint32_t fb = smem_u32(&xfull[s]);
        mbar_arrive_expect_tx(fb, bytes);
        tma_load_3d(smem_u32(smem + s * S::kXStage), &tmap_x, fb, 0, 0, ks * T, pol);
      }
      __syncwarp();
      ++issued;
    }
    // Leave no copy in flight.
    for (int li = issued > kRX ? issued - kRX : 0; li < issued; ++li) {
      const int jg = li / S::kGroups;
      warp_wait(smem_u32(&xfull[2 * (li - jg * S::kGroups) + (jg & 1)]), (jg >> 1) & 1, s_never);
    }
  } else if (warp < 4 * S::kGroups) {
    // ---------------- dequant groups ----------------
    // Group g takes the steps li = g, g + G, ...: it splices each step's T
    // tiles into its TMEM slot 2g + (j & 1) (j = li / G), then every warp
    // reports the slot written and moves on to the next step; the group's
    // issuer warps take it from there.
    const int g = warp >> 2;
    const int quad = warp & 3;               // TMEM lanes 32*quad .. 32*quad+31
    const int r = quad * 32 + lane;          // weight row within the tile
    const uint32_t lane_base = static_cast<uint32_t>(quad * 32) << 16;
    const auto aux = Fm::make_aux();
    bool ok = true;
    int j = 0;                               // this group's steps so far
    for (int li = g; li < n_local; li += S::kGroups, ++j) {
      const int sw = li % kSW;
      const int slot = 2 * g + (j & 1);           // also the x stage
      ok = warp_wait(smem_u32(&wfull[sw]), (li / kSW) & 1, s_abort) && ok;
      if (j >= 2) ok = warp_wait(smem_u32(&slotfree[slot]), ((j >> 1) - 1) & 1, s_abort) && ok;
      tc_fence_after();
      if (ok) {
        const uint8_t* wst = smem + S::kWOff + sw * S::kWStage;
        static_assert(S::kTMax == 2, "two tiles per step at most");
        // both tiles' words first, so the second tile's loads overlap the
        // first tile's rebuild
        uint32_t F0[Fm::kRowWords], F1[Fm::kRowWords], w[32];
        Fm::load(wst, r, F0);
        if (T > 1) Fm::load(wst + Fm::kTileBytes, r, F1);
        rebuild_row<F>(F0, w, aux);
        tmem_st_32x32b_x32(tmem + lane_base + slot * S::kSlotCols, w);
        if (T > 1) {
          rebuild_row<F>(F1, w, aux);
          tmem_st_32x32b_x32(tmem + lane_base + slot * S::kSlotCols + 32, w);
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&wempty[sw]));   // smem fragments read
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&slotready[slot]));
    }
  } else if (warp >= S::kIssWarp && warp < S::kIssWarp + S::kGroups * S::kIss) {
    // ---------------- MMA issuers, kIss per group ----------------
    const int ii = warp - S::kIssWarp;
    const int g = ii / S::kIss;
    const int iss = ii - g * S::kIss;
    constexpr int kSlice = 4 / S::kIss;      // k-slices of a tile per issuer
    const int kk0 = iss * kSlice;
    constexpr uint32_t idesc = idesc_f16_f32(128, NCOL);
    bool ok = true;
    int j = 0;                               // this group's steps so far
    for (int sg = 0; sg < nseg; ++sg) {
      int a, b;
      segment_range(sg, tile_first, s0, KS, n_local, &a, &b);
      const int set = sg % S::kSets;
      const uint32_t d_tmem = tmem + S::kDCol + ((set * S::kGroups + g) * S::kIss + iss) * NCOL;
      // The accumulators of this set were last used kSets segments ago: the
      // epilogue must have read them before the first MMA or arrival.
      if (sg >= S::kSets) ok = warp_wait(smem_u32(&dempty[set]), ((sg / S::kSets) - 1) & 1, s_abort) && ok;
      bool first = true;
      for (int li = group_first(g, a, S::kGroups); li <= b; li += S::kGroups, ++j) {
        const int slot = 2 * g + (j & 1);
        ok = warp_wait(smem_u32(&slotready[slot]), (j >> 1) & 1, s_abort) && ok;
        ok = warp_wait(smem_u32(&xfull[slot]), (j >> 1) & 1, s_abort) && ok;
        if (lane == 0) {
          tc_fence_after();
          if (ok) {
            const uint64_t bdesc0 = smem_desc_sw128(smem_u32(smem + slot * S::kXStage));
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
        }
        __syncwarp();
        first = false;
      }
      // One arrival per issuer and segment: the commit covers this issuer's
      // MMAs into the set; an issuer with no step in the segment just arrives.
      if (lane == 0) {
        if (!first) tc_commit(smem_u32(&dfull[set]));
        else mbar_arrive(smem_u32(&dfull[set]));
      }
      __syncwarp();
    }
    if (lane == 0) tc_commit(smem_u32(done));
    __syncwarp();
    warp_wait(smem_u32(done), 0, s_never);
  } else if (warp >= S::kEpiWarp && warp < S::kEpiWarp + 4) {
    // ---------------- epilogue warpgroup: segments in order ----------------
    // Split row tiles: see the fix-up protocol at the top of this file.
    grid_dependency_wait();                  // y, partials and counters may be in use before this kernel
    const int quad = warp & 3;
    const int r = quad * 32 + lane;
    const uint32_t lane_base = static_cast<uint32_t>(quad * 32) << 16;
    const int mcount = min(NCOL, p.M);
    for (int sg = 0; sg < nseg; ++sg) {
      const long long tile = tile_first + sg;
      const int set = sg % S::kSets;
      const uint32_t dpar = (sg / S::kSets) & 1;
      int a, b;
      segment_range(sg, tile_first, s0, KS, n_local, &a, &b);
      const int n = static_cast<int>(tile) * kTileRows + r;
      const float mul = __half2float(__ushort_as_half(p.scales[n]));
      const int c_lo = range_owner(tile * KS, total, G);
      const int c_hi = range_owner(tile * KS + KS - 1, total, G);
      const bool split = c_lo != c_hi;
      const bool finisher = (c == c_lo);
      const unsigned int need = static_cast<unsigned int>(c_hi - c_lo);   // adds of the later contributors
      unsigned int* cnt = p.counters + 4 * c_lo + quad;
      uint16_t* ybase = p.y + n;

      // This segment's own sums, columns c0 .. c0+7: the accumulators of the
      // groups (and their issuers) added in a fixed order.
      auto own8 = [&](int c0, float (&acc)[8]) {
#pragma unroll
        for (int jj = 0; jj < 8; ++jj) acc[jj] = 0.0f;
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
      };
      // Partials of contributors c_lo+1 .. c_hi summed in CTA order, columns
      // c0 .. c0+15 (those below mcount): one contributor's 16 loads are in
      // flight together, one L2 round trip per contributor and 16 columns.
      auto others16 = [&](int c0, float (&q)[16]) {
#pragma unroll
        for (int jj = 0; jj < 16; ++jj) q[jj] = 0.0f;
        for (int cc = c_lo + 1; cc <= c_hi; ++cc) {
          const float* src = decode_partial<NCOL>(p.partials, 2 * cc, r) + c0 * 128;
          float v[16];
#pragma unroll
          for (int jj = 0; jj < 16; ++jj) v[jj] = (c0 + jj < mcount) ? __ldcg(src + jj * 128) : 0.0f;
#pragma unroll
          for (int jj = 0; jj < 16; ++jj) q[jj] += v[jj];
        }
      };
      auto store8 = [&](int c0, const float (&v)[8]) {
#pragma unroll
        for (int jj = 0; jj < 8; ++jj)
          if (c0 + jj < mcount)
            ybase[static_cast<long long>(c0 + jj) * p.N] = __half_as_ushort(__float2half_rn(v[jj] * mul));
      };
      // The accumulators of this set are read: the issuers may reuse them.
      auto release = [&]() {
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&dempty[set]));
      };
      // Write this CTA's partial (slot 2c + which), release the accumulators
      // and add one to the counter; true when this add completed the count
      // (every other contributor, c_lo included, had counted), making this
      // warp the one that finishes the tile, from the partials in memory.
      auto publish = [&](int which) -> bool {
        float* mine = decode_partial<NCOL>(p.partials, 2 * c + which, r);
#pragma unroll
        for (int c0 = 0; c0 < NCOL; c0 += 8) {
          if (c0 >= mcount) break;
          float acc[8];
          own8(c0, acc);
#pragma unroll
          for (int jj = 0; jj < 8; ++jj) __stcg(mine + (c0 + jj) * 128, acc[jj]);
        }
        // The lanes' partial stores are ordered before lane 0's add by the
        // warp barrier, and its release publishes them with its own.
        release();
        unsigned int old = 0;
        if (lane == 0) old = atom_add_acq_rel(cnt, 1u);
        const bool last = __shfl_sync(0xffffffffu, old, 0) == need;
        if (last) (void)ld_acquire(cnt);      // every lane acquires the others' partials
        return last;
      };
      // The whole tile from the partials in memory: contributors c_lo+1 ..
      // c_hi in CTA order, then c_lo's.
      auto finish_from_partials = [&]() {
        const float* lo = decode_partial<NCOL>(p.partials, 2 * c_lo + 1, r);
#pragma unroll
        for (int c0 = 0; c0 < NCOL; c0 += 16) {
          if (c0 >= mcount) break;
          float q[16], v[16];
          others16(c0, q);
#pragma unroll
          for (int jj = 0; jj < 16; ++jj) v[jj] = (c0 + jj < mcount) ? __ldcg(lo + (c0 + jj) * 128) : 0.0f;
#pragma unroll
          for (int h = 0; h < 16; h += 8) {
            float w[8];
#pragma unroll
            for (int jj = 0; jj < 8; ++jj) w[jj] = q[h + jj] + v[h + jj];
            store8(c0 + h, w);
          }
        }
        __syncwarp();
        if (lane == 0) *cnt = 0u;            // every contributor has counted: reset for the next launch
      };
      // Every later contributor has counted (each lane acquires on its own).
      auto all_counted = [&]() -> bool {
        return __all_sync(0xffffffffu, ld_acquire(cnt) == need) != 0;
      };

      if (!split) {
        if (!warp_wait(smem_u32(&dfull[set]), dpar, s_abort)) break;
        tc_fence_after();
#pragma unroll
        for (int c0 = 0; c0 < NCOL; c0 += 8) {
          if (c0 >= mcount) break;
          float acc[8];
          own8(c0, acc);
          store8(c0, acc);
        }
        release();
      } else if (finisher) {
        // The others' partials, 16 columns at a time.  With 16 token columns
        // that is all of them: sum them while this CTA's last MMAs still run,
        // as soon as all are there.
        float pre[16];
        bool pre_ok = false;
        if constexpr (NCOL == 16) {
          while (true) {
            if (all_counted()) {
              others16(0, pre);
              pre_ok = true;
              break;
            }
            const bool fin = mbar_try_wait(smem_u32(&dfull[set]), dpar);
            if (__any_sync(0xffffffffu, fin || *s_abort)) break;
            __nanosleep(128);
          }
        }
        if (!warp_wait(smem_u32(&dfull[set]), dpar, s_abort)) break;
        tc_fence_after();
        if (pre_ok || all_counted()) {
#pragma unroll
          for (int c0 = 0; c0 < NCOL; c0 += 16) {
            if (c0 >= mcount) break;
            if (!pre_ok) others16(c0, pre);
#pragma unroll
            for (int h = 0; h < 16; h += 8) {
              if (c0 + h >= mcount) break;
              float acc[8];
              own8(c0 + h, acc);
#pragma unroll
              for (int jj = 0; jj < 8; ++jj) acc[jj] = pre[h + jj] + acc[jj];
              store8(c0 + h, acc);
            }
          }
          release();
          __syncwarp();
          if (lane == 0) *cnt = 0u;          // every contributor has counted: reset for the next launch
        } else if (publish(1)) {
          // Not every partial was there; they all are now, after this one.
          finish_from_partials();
        }
      } else {
        // A later contributor (this tile is where its range starts).
        if (!warp_wait(smem_u32(&dfull[set]), dpar, s_abort)) break;
        tc_fence_after();
        // If c_lo and every other contributor counted before this one, this
        // warp finishes the tile, in the order c_lo would.
        if (publish(0)) finish_from_partials();
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
