// fp6_linear.cuh -- the fused FP6 x FP16 linear layer for sm_100a.
//
// y[M,N] = x[M,K] . (scale (.) decode(W[N,K]))^T, fp32 accumulation, fp16 out.
//
// The TC-FPx design (article section "kernel solution redesign") keeps the
// dequantization and the tensor-core product in one kernel, rebuilds FP16
// weights with bit-parallel SIMT work in registers, and overlaps the two with
// a software pipeline.  On sm_100a this becomes a warp-specialised persistent
// kernel.  Per 64-column step ("iteration") of a 128-row weight tile:
//
//   warp 20       weight producer: one 6144-byte bulk copy of the packed tile
//                 into a smem ring (SW stages);
//   warp 21       activation producer: one TMA tile copy of x (NCOL rows x 64,
//                 128-byte swizzle, rows beyond M zero-filled) into a smem ring
//                 of R stages;
//   warps 8..19   three dequant warpgroups taking every third iteration: each
//                 thread owns one weight row (its TMEM lane), reads its 48
//                 packed bytes, splices 64 fp16 weights (decode * 2^-12) and
//                 stores them into a ring of R TMEM slots (tcgen05.st);
//   warps 0..3    MMA issuers.  tcgen05.mma (M = 128, K = 16) costs a warp
//                 about 47 cycles to issue whatever N is, so at small N one
//                 issuer cannot keep up with HBM; NISS issuers each take a
//                 k-slice of every step (K/NISS) into their own fp32
//                 accumulator in TMEM, A from the TMEM slot, B = x from smem;
//   warps 4..7    the epilogue warpgroup: per segment (the iterations of one
//                 tile this CTA owns), tcgen05.ld of the NISS accumulators,
//                 summed in a fixed order, * scale * 2^12, fp16 store, or the
//                 split-K partial and fix-up.
//
// An iteration's x stage and TMEM slot are released together by the issuers'
// commits on one "consumed" barrier.  Every mbarrier has consumers that wait on
// its phases in order (a ring slot always belongs to the same dequant group:
// SW and R are multiples of the group count), so no wait can alias a phase two
// steps ahead.
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

constexpr int kDeqGroups = 3;                 // dequant warpgroups
constexpr int kEpiWarp = 4;                   // warps 4..7
constexpr int kFirstDeqWarp = 8;              // warps 8..19
constexpr int kWProdWarp = kFirstDeqWarp + 4 * kDeqGroups;   // 20
constexpr int kXProdWarp = kWProdWarp + 1;                   // 21
constexpr int kLinearThreads = 32 * (kXProdWarp + 1);        // 704
constexpr int kMaxGrid = 1024;                // persistent CTAs at most (one per SM)
constexpr int kCounterBytes = kMaxGrid * 4;
constexpr uint32_t kTmemCols = 512;

template <int NCOL>
struct LinearShape {
  static_assert(NCOL == 16 || NCOL == 32 || NCOL == 64 || NCOL == 128 || NCOL == 256, "NCOL");
  static constexpr int kXBytes = NCOL * 128;   // NCOL rows x 64 fp16, 128-byte swizzled
  static constexpr int kIssuers = (NCOL <= 32) ? 4 : (NCOL == 64) ? 2 : 1;
  static constexpr int kR = (NCOL <= 64) ? 12 : (NCOL == 128) ? 6 : 3;      // x stages = TMEM slots
  static constexpr int kSW = (NCOL == 16) ? 27 : (NCOL == 32) ? 24 : 18;   // weight stages
  static constexpr int kDCol = kR * 32;        // accumulators after the TMEM slot ring
  static constexpr int kWOff = kR * kXBytes;   // weight ring after the x ring
  static constexpr int kBarOff = kWOff + kSW * kTileBytes;
  static constexpr int kBarrierBytes = 1024;
  static constexpr int kSmemBytes = kBarOff + kBarrierBytes + 1024;  // + alignment slack
  static_assert(kXBytes % 1024 == 0 && kTileBytes % 1024 == 0, "1024-byte aligned stages");
  static_assert(kSW % kDeqGroups == 0 && kR % kDeqGroups == 0, "ring slots owned by one group");
  static_assert(kDCol + kIssuers * NCOL <= static_cast<int>(kTmemCols), "TMEM budget");
  static_assert((2 * kSW + 3 * kR + 6) * 8 + 32 <= kBarrierBytes, "barrier area");
  static_assert(kSmemBytes <= 232448, "shared memory");
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

// Walks the CTA's iterations: the 64-column step k and the tile's (row tile,
// token tile) coordinates, advanced without divisions.
struct IterCursor {
  int k, nt, mt;
  int KT, MT;
  __device__ __forceinline__ IterCursor(long long it0, int KT_, int MT_) : KT(KT_), MT(MT_) {
    const long long tile = it0 / KT_;
    k = static_cast<int>(it0 - tile * KT_);
    nt = static_cast<int>(tile / MT_);
    mt = static_cast<int>(tile - static_cast<long long>(nt) * MT_);
  }
  __device__ __forceinline__ void next() {
    if (++k == KT) {
      k = 0;
      if (++mt == MT) {
        mt = 0;
        ++nt;
      }
    }
  }
};

template <int NCOL>
__global__ void __launch_bounds__(kLinearThreads, 1)
    fp6_linear_kernel(const __grid_constant__ CUtensorMap tmap_x, const LinearParams p) {
  using S = LinearShape<NCOL>;
  constexpr int kR = S::kR;
  constexpr int kSW = S::kSW;
  constexpr int kISS = S::kIssuers;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* wfull = reinterpret_cast<uint64_t*>(smem + S::kBarOff);
  uint64_t* wempty = wfull + kSW;
  uint64_t* xfull = wempty + kSW;
  uint64_t* afull = xfull + kR;
  uint64_t* consumed = afull + kR;                // x stage + TMEM slot free (issuer commits)
  uint64_t* dfull = consumed + kR;
  uint64_t* dempty = dfull + 1;
  uint64_t* done = dempty + 1;
  uint64_t* epi = done + 1;                       // [2]: fix-up meeting of the first / last split segment
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(epi + 2);
  volatile int* s_last = reinterpret_cast<volatile int*>(tmem_holder + 1);  // [2]
  volatile int* s_abort = s_last + 2;
  volatile int* s_never = s_abort + 1;            // an abort flag nothing raises (final drains)

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int G = p.grid;
  const int c = blockIdx.x;
  const long long total = p.total_iters;
  const int KT = p.k_tiles;
  const int MT = p.m_tiles;
  const long long it0 = range_begin(c, total, G);
  const long long it1 = range_begin(c + 1, total, G);
  const int n_local = static_cast<int>(it1 - it0);
  const long long tile_first = it0 / KT;
  const long long tile_last = (it1 - 1) / KT;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kSW; ++s) {
      mbar_init(smem_u32(&wfull[s]), 1);
      mbar_init(smem_u32(&wempty[s]), 4);      // the 4 warps of the group that read it
    }
    for (int s = 0; s < kR; ++s) {
      mbar_init(smem_u32(&xfull[s]), 1);
      mbar_init(smem_u32(&afull[s]), 4);       // the 4 warps of the group that wrote it
      mbar_init(smem_u32(&consumed[s]), kISS); // one commit per issuer
    }
    mbar_init(smem_u32(dfull), kISS);
    mbar_init(smem_u32(dempty), 4);
    mbar_init(smem_u32(done), kISS);
    mbar_init(smem_u32(&epi[0]), 4);
    mbar_init(smem_u32(&epi[1]), 4);
    s_last[0] = 0;
    s_last[1] = 0;
    *s_abort = 0;
    *s_never = 0;
    fence_barrier_init();
    fence_proxy_async_smem();
  }
  if (warp == kXProdWarp && lane == 0) prefetch_tensormap(&tmap_x);
  if (warp == 0) {
    tmem_alloc(smem_u32(tmem_holder), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;

  if (warp == kWProdWarp) {
    // ---------------- weight producer ----------------
    if (lane == 0) {
      const uint64_t pol = policy_evict_first();
      IterCursor cur(it0, KT, MT);
      int issued = 0;
      for (int li = 0; li < n_local; ++li, cur.next()) {
        const int s = li % kSW;
        if (li >= kSW && !wait_bounded(smem_u32(&wempty[s]), ((li / kSW) - 1) & 1, s_abort)) break;
        const uint32_t fb = smem_u32(&wfull[s]);
        mbar_arrive_expect_tx(fb, kTileBytes);
        bulk_load(smem_u32(smem + S::kWOff + s * kTileBytes),
                  p.packed + (static_cast<long long>(cur.nt) * KT + cur.k) * kTileBytes, kTileBytes, fb, pol);
        ++issued;
      }
      // Leave no copy in flight: the last copy issued into every stage has landed.
      for (int li = issued > kSW ? issued - kSW : 0; li < issued; ++li)
        wait_bounded(smem_u32(&wfull[li % kSW]), (li / kSW) & 1, s_never);
    }
  } else if (warp == kXProdWarp) {
    // ---------------- activation producer ----------------
    if (lane == 0) {
      const uint64_t pol = policy_evict_last();
      IterCursor cur(it0, KT, MT);
      int issued = 0;
      for (int li = 0; li < n_local; ++li, cur.next()) {
        const int s = li % kR;
        if (li >= kR && !wait_bounded(smem_u32(&consumed[s]), ((li / kR) - 1) & 1, s_abort)) break;
        const uint32_t fb = smem_u32(&xfull[s]);
        mbar_arrive_expect_tx(fb, S::kXBytes);
        tma_load_2d(smem_u32(smem + s * S::kXBytes), &tmap_x, fb, cur.k * kTileCols, cur.mt * NCOL, pol);
        ++issued;
      }
      for (int li = issued > kR ? issued - kR : 0; li < issued; ++li)
        wait_bounded(smem_u32(&xfull[li % kR]), (li / kR) & 1, s_never);
    }
  } else if (warp < kISS) {
    // ---------------- MMA issuer `warp`: k-slice [warp*4/kISS, (warp+1)*4/kISS) of every step ----------------
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_f16_f32(128, NCOL);
      constexpr int kSlice = 4 / kISS;
      const int kk0 = warp * kSlice;
      const uint32_t d_tmem = tmem + S::kDCol + warp * NCOL;
      int sg = 0;
      int k = static_cast<int>(it0 - tile_first * KT);
      for (int li = 0; li < n_local; ++li, k = (k + 1 == KT) ? 0 : k + 1) {
        const bool seg_first = (li == 0) || (k == 0);
        const bool seg_last = (li == n_local - 1) || (k == KT - 1);
        const int s = li % kR;
        if (seg_first && sg > 0 && !wait_bounded(smem_u32(dempty), (sg - 1) & 1, s_abort)) break;
        if (!wait_bounded(smem_u32(&xfull[s]), (li / kR) & 1, s_abort)) break;
        if (!wait_bounded(smem_u32(&afull[s]), (li / kR) & 1, s_abort)) break;
        tc_fence_after();
        const uint64_t bdesc = smem_desc_sw128(smem_u32(smem + s * S::kXBytes));
#pragma unroll
        for (int j = 0; j < kSlice; ++j) {
          const int kk = kk0 + j;
          // K = 16 per MMA: 8 TMEM columns of A, 32 bytes along the swizzled B rows
          mma_f16_ts(d_tmem, tmem + s * 32 + kk * 8, bdesc + static_cast<uint64_t>(kk * 2), idesc,
                     (seg_first && j == 0) ? 0u : 1u);
        }
        tc_commit(smem_u32(&consumed[s]));
        if (seg_last) {
          tc_commit(smem_u32(dfull));
          ++sg;
        }
      }
      // All issued MMAs have finished before TMEM is released.
      tc_commit(smem_u32(done));
      wait_bounded(smem_u32(done), 0, s_never);
    }
  } else if (warp >= kFirstDeqWarp) {
    // ---------------- dequant warpgroups ----------------
    const int g = (warp - kFirstDeqWarp) >> 2;
    const int quad = warp & 3;               // TMEM lanes 32*quad .. 32*quad+31
    const int r = quad * 32 + lane;          // weight row within the tile
    const uint32_t lane_base = static_cast<uint32_t>(quad * 32) << 16;
    for (int li = g; li < n_local; li += kDeqGroups) {
      const int sw = li % kSW;
      const int s = li % kR;
      if (!warp_wait(smem_u32(&wfull[sw]), (li / kSW) & 1, s_abort)) break;
      uint32_t lo[8], hi[4], w[32];
      load_row_fragments(smem + S::kWOff + sw * kTileBytes, r, lo, hi);
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&wempty[sw]));
      if (li >= kR && !warp_wait(smem_u32(&consumed[s]), ((li / kR) - 1) & 1, s_abort)) break;
      tc_fence_after();
      splice_row(lo, hi, w);
      tmem_st_32x32b_x32(tmem + lane_base + s * 32, w);
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&afull[s]));
    }
  } else if (warp >= kEpiWarp && warp < kEpiWarp + 4) {
    // ---------------- epilogue warpgroup: segments in order ----------------
    const int quad = warp & 3;
    const int r = quad * 32 + lane;
    const bool leader = (warp == kEpiWarp) && lane == 0;
    const uint32_t lane_base = static_cast<uint32_t>(quad * 32) << 16;
    int sg = 0;
    for (long long tile = tile_first; tile <= tile_last; ++tile, ++sg) {
      if (!warp_wait(smem_u32(dfull), sg & 1, s_abort)) break;
      tc_fence_after();
      const int nt = static_cast<int>(tile / MT);
      const int mt = static_cast<int>(tile - static_cast<long long>(nt) * MT);
      const int n = nt * kTileRows + r;
      const int m0 = mt * NCOL;
      const int mcount = min(NCOL, p.M - m0);
      const float mul = __half2float(__ushort_as_half(p.scales[n])) * 4096.0f;
      const int c_lo = range_owner(tile * KT, total, G);
      const int c_hi = range_owner(tile * KT + KT - 1, total, G);
      const bool split = c_lo != c_hi;
      const int which = (tile == tile_first) ? 0 : 1;   // this CTA's first or last segment
      float* part = p.partials + static_cast<long long>(2 * c + which) * NCOL * 128;
      for (int c0 = 0; c0 < NCOL; c0 += 8) {
        float acc[8];
#pragma unroll
        for (int i = 0; i < kISS; ++i) {
          uint32_t v[8];
          tmem_ld_32x32b_x8(tmem + lane_base + S::kDCol + i * NCOL + c0, v);
          tmem_wait_ld();
#pragma unroll
          for (int j = 0; j < 8; ++j) acc[j] = (i == 0) ? __uint_as_float(v[j]) : acc[j] + __uint_as_float(v[j]);
        }
        if (c0 + 8 >= NCOL) {
          // accumulators fully read: the next segment may overwrite them
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(smem_u32(dempty));
        }
        if (split) {
#pragma unroll
          for (int j = 0; j < 8; ++j) part[(c0 + j) * 128 + r] = acc[j];
        } else {
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            if (c0 + j < mcount)
              p.y[static_cast<long long>(m0 + c0 + j) * p.N + n] = __half_as_ushort(__float2half_rn(acc[j] * mul));
          }
        }
      }
      if (split) {
        // Publish this CTA's partial, then count arrivals; the last CTA of the
        // tile sums every partial in CTA order.  The group's warps meet on an
        // mbarrier (bounded wait), never on bar.sync, so an aborted warp cannot
        // strand the others.  Each of the CTA's (at most two) split segments
        // has its own meeting barrier.
        const uint32_t eb = smem_u32(&epi[which]);
        __threadfence();
        __syncwarp();
        if (lane == 0) mbar_arrive(eb);
        if (!warp_wait(eb, 0, s_abort)) break;
        if (leader) {
          __threadfence();
          const unsigned int prev = atomicAdd(&p.counters[c_lo], 1u);
          s_last[which] = (prev == static_cast<unsigned int>(c_hi - c_lo)) ? 1 : 0;
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(eb);
        if (!warp_wait(eb, 1, s_abort)) break;
        if (s_last[which]) {
          __threadfence();
          for (int c0 = 0; c0 < mcount; c0 += 8) {
            float acc[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) acc[j] = 0.0f;
            for (int cc = c_lo; cc <= c_hi; ++cc) {
              const float* src = p.partials +
                                 static_cast<long long>(partial_slot(cc, tile, total, G, KT)) * NCOL * 128 +
                                 c0 * 128 + r;
              float v[8];
#pragma unroll
              for (int j = 0; j < 8; ++j) v[j] = __ldcg(src + j * 128);
#pragma unroll
              for (int j = 0; j < 8; ++j) acc[j] += v[j];
            }
#pragma unroll
            for (int j = 0; j < 8; ++j)
              if (c0 + j < mcount)
                p.y[static_cast<long long>(m0 + c0 + j) * p.N + n] = __half_as_ushort(__float2half_rn(acc[j] * mul));
          }
          if (leader) p.counters[c_lo] = 0u;
        }
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
