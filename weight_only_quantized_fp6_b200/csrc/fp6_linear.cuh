// fp6_linear.cuh -- the fused FP6 x FP16 linear layer for sm_100a.
//
// y[M,N] = x[M,K] . (scale (.) decode(W[N,K]))^T, fp32 accumulation, fp16 out.
//
// The TC-FPx design (article section "kernel solution redesign") keeps the
// dequantization and the tensor-core product in one kernel, rebuilds FP16
// weights with bit-parallel SIMT work in registers, and overlaps the two with
// a software pipeline.  On sm_100a this becomes a warp-specialised persistent
// kernel.  The unit of the pipeline is a "step": T consecutive 64-column tiles
// of one 128-row weight tile (T = 1, 2 or 4), so that per-step
// synchronisation is amortised over T tiles.
//
//   warp 20       weight producer: one bulk copy of the step's T packed tiles
//                 (contiguous, T * 6144 bytes) into a smem ring (SW stages);
//   warp 21       activation producer into a ring of RX stages: one TMA box
//                 per step (T column tiles of NCOL rows x 64 columns, 128-byte
//                 swizzle, rows beyond M zero-filled);
//   warps 8..19   three dequant warpgroups taking every third step: each thread
//                 owns one weight row (its TMEM lane), reads its 48 packed bytes
//                 per tile, rebuilds 64 fp16 weights (decode(c), exact) and stores
//                 them into the step's TMEM slot (tcgen05.st);
//   warps 0..3    MMA issuers (tcgen05.mma M = 128, K = 16; A from the TMEM
//                 slot, B = x from smem): one for 128 token columns (N = 128),
//                 two for 256, each issuing the MMAs of its 128 tokens into
//                 its half of the fp32 accumulator in TMEM;
//   warps 4..7    the epilogue warpgroup: per segment (the steps of one tile
//                 that this CTA owns), tcgen05.ld of the accumulator, * scale,
//                 fp16 store, or the split-K partial and fix-up (with the
//                 dequant warps' help at the end of the range).
//
// Rings: packed weights (SW smem stages, filled by the weight producer,
// released by the dequant group), x (RX smem stages) and dequantized weights
// (R TMEM slots).  The MMA issuer is the one serial thread of the pipeline
// (an MMA issue costs it about 100 cycles, a barrier test or commit 80-130),
// so it handles one barrier of each kind per step: the step's dequant group
// waits for the step's x stage to land before it signals "ready", and one
// commit per step ("freed") releases both the x stage and the TMEM slot.
// Those two barriers form a ring of L = lcm(R, RX) steps.  Every mbarrier's
// waiters wait on its phases in order (a weight stage, TMEM slot or step
// barrier always belongs to the same dequant group: SW, R and L are multiples
// of the group count), so no wait can alias a phase two steps ahead.
//
// Work split: the (token tile, row tile, step) iterations are laid out
// row-tile major and cut into G contiguous, equal ranges, one per persistent
// CTA (G = number of SMs).  A row tile whose steps span several CTAs is
// finished by the last of them to arrive (atomic counter), which sums the
// partials in CTA order: results are deterministic and no CTA waits on
// another.  A split tile's counter is indexed by its first contributing CTA,
// which is unique among split tiles and below G, so the counters occupy a
// fixed region of the workspace that no partial ever overlaps.
//
// Launch: programmatic dependent launch.  The kernel may start while the
// previous kernel in the stream is finishing: barrier set-up, TMEM allocation
// and the stream of packed weights overlap its tail.  Reads of x and scales
// and every write (y, partials, counters) come after griddepcontrol.wait, i.e.
// after the previous kernel has completed and its writes are visible.  A
// previous kernel that never signals early completion (every kernel of this
// library but this one, and ordinary kernels) only lets this kernel start once
// it has finished, so packed weights written by it are seen too; packed
// weights must not be produced by a kernel that does signal early completion.
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
constexpr int kCounterBytes = kMaxGrid * 16;   // up to four counters per CTA
constexpr uint32_t kTmemCols = 512;

constexpr int gcd_int(int a, int b) { return b == 0 ? a : gcd_int(b, a % b); }
constexpr int lcm_int(int a, int b) { return a / gcd_int(a, b) * b; }

template <int NCOL, Fmt F = Fmt::E3M2>
struct LinearShape {
  static_assert(NCOL == 16 || NCOL == 32 || NCOL == 64 || NCOL == 128 || NCOL == 256, "NCOL");
  static constexpr int kTMax = (NCOL <= 32) ? 4 : (NCOL <= 128) ? 2 : 1;   // tiles per step, at most
  static constexpr int kXTile = NCOL * 128;                 // NCOL rows x 64 fp16, 128-byte swizzled
  static constexpr int kXStage = kTMax * kXTile;
  static constexpr int kTileBytes = Format<F>::kTileBytes;
  static constexpr int kWStage = kTMax * kTileBytes;
  // MMA-issuing warps.  Up to 64 token columns each takes a k-slice of every
  // tile into its own accumulator (summed in the epilogue).  At 256 columns
  // two issuers split the tokens instead (N = 128 each, every k-slice, one
  // accumulator in two column halves): one thread issues an MMA in about
  // 100 cycles, so a second issuing thread is what lets the tensor pipe run
  // at its rate.
  static constexpr int kIssuers = (NCOL <= 32) ? 4 : (NCOL == 64) ? 2 : (NCOL == 256) ? 2 : 1;
  static constexpr bool kNSplit = NCOL == 256;
  static constexpr int kIssN = kNSplit ? NCOL / kIssuers : NCOL;        // MMA N of one issuer
  static constexpr int kIssSlices = kNSplit ? 4 : 4 / kIssuers;         // k-slices per tile and issuer
  static constexpr int kAccIssuers = kNSplit ? 1 : kIssuers;            // accumulators the epilogue sums
  static constexpr int kAccCols = kNSplit ? NCOL : kIssuers * NCOL;
  static constexpr int kRX = (NCOL == 16) ? 8 : (NCOL == 32) ? 4 : 3;     // x stages (>= 3)
  // weight stages of 6-bit tiles; the same bytes in FP4 tiles
  static constexpr int kSW = ((NCOL <= 32) ? 6 : (NCOL == 64) ? 12 : (NCOL == 128) ? 9 : 18) * 6144 / kTileBytes /
                             kDeqGroups * kDeqGroups;
  static constexpr int kR = (kTMax == 4) ? 3 : 6;           // TMEM slots
  static constexpr int kSlotCols = kTMax * 32;              // TMEM columns of one slot
  static constexpr int kDCol = kR * kSlotCols;              // accumulators after the slots
  static constexpr int kWOff = kRX * kXStage;               // weight ring after the x ring
  static constexpr int kBarOff = kWOff + kSW * kWStage;
  // Step barriers, a ring of kL (a multiple of the x stages and of the TMEM
  // slots): "ready" (the step's dequant group has written its TMEM slot and
  // seen its x stage land) and "freed" (the step's MMAs have completed).
  static constexpr int kL = lcm_int(kR, kRX);
  // wfull, wempty [SW]; xfull [RX]; ready, freed [L]; dfull, dempty, done
  static constexpr int kNumBars = 2 * kSW + kRX + 2 * kL + 3;
  // columns per TMEM read in the epilogue: kAccIssuers reads of kEC 32-bit columns
  static constexpr int kEC = 32 / kAccIssuers;
  // Split-tile fix-up at the end of a CTA's range, when every ring is idle:
  // the epilogue warp and the three dequant warps of each row quarter (16
  // warps) each own kFixBufs buffers (2 KB: one contributor's 16 partial
  // columns of the quarter's 32 rows) in the rings' space, each with a copy
  // barrier after the kNumBars above; then one "go" barrier per quarter.
  static constexpr int kFixCols = 16;     // the shared-memory reads take 16 columns
  static constexpr int kFixBlock = kFixCols * 32 * 4;
  static constexpr int kFixWarps = 4 * (1 + kDeqGroups);
  static constexpr int kFixBytes = kBarOff / kFixWarps / kFixBlock * kFixBlock;
  static constexpr int kFixBufs = (kFixBytes / kFixBlock < 16) ? kFixBytes / kFixBlock : 16;
  static constexpr int kAllBars = kNumBars + kFixWarps * kFixBufs + 4;
  static constexpr int kBarrierBytes = 2048;
  static constexpr int kSmemBytes = kBarOff + kBarrierBytes + 1024;  // + alignment slack
  static_assert(kXTile % 1024 == 0 && kTileBytes % 1024 == 0, "1024-byte aligned tiles");
  static_assert(kSW % kDeqGroups == 0 && kR % kDeqGroups == 0, "ring slots owned by one group");
  // A dequant group waiting for step li's x stage finds the stage's previous
  // fill (step li - RX) complete: it was its own step, or it precedes step
  // li - R, whose MMAs have completed.  So no parity wait can alias.
  static_assert(kRX % kDeqGroups == 0 || kRX >= kR, "x stage phases seen in order");
  static_assert(kDCol + kAccCols <= static_cast<int>(kTmemCols), "TMEM budget");
  static_assert(kFixBufs >= 2, "fix-up buffers");
  static_assert(kAllBars * 8 + 32 <= kBarrierBytes, "barrier area");
  static_assert(kAllBars <= kLinearThreads, "one thread per barrier at set-up");
  static_assert(kSmemBytes <= 232448, "shared memory");
};

struct LinearParams {
  const uint16_t* x;     // [M,K] fp16 (the kernels read it through the tensor map)
  const uint8_t* packed;
  const uint16_t* scales;
  uint16_t* y;
  float* partials;       // [2*G][4][NCOL][32] fp32: slot, row quarter, column, row
  uint32_t* counters;    // [kMaxGrid], indexed by a split tile's first CTA; zero on entry and exit
  int M, N, K;
  int n_tiles, m_tiles, k_tiles;   // k_tiles = K / 64
  int T;                           // tiles per step (divides k_tiles, <= kTMax)
  int k_steps;                     // k_tiles / T
  long long total_steps;           // n_tiles * m_tiles * k_steps
  int grid;
};

// First step of CTA c's range.
__host__ __device__ __forceinline__ long long range_begin(int c, long long total, int G) {
  return static_cast<long long>(c) * total / G;
}
// CTA whose range holds step i:  max{c : range_begin(c) <= i}.
__host__ __device__ __forceinline__ int range_owner(long long i, long long total, int G) {
  return static_cast<int>(((i + 1) * G + total - 1) / total - 1);
}
// First float of the partial of slot `slot` for row quarter q (32 rows):
// NCOL columns of 32 consecutive floats, 128 * NCOL contiguous bytes.
__host__ __device__ __forceinline__ long long partial_offset(int slot, int q, int ncol) {
  return (static_cast<long long>(slot) * 4 + q) * ncol * 32;
}
// Partial slot of CTA c's segment in tile t (KS steps per tile): 0 for the
// tile its range starts in, 1 for the tile its range ends in (only those two
// can be partial).
__host__ __device__ __forceinline__ int partial_slot(int c, long long t, long long total, int G, int KS) {
  return 2 * c + ((range_begin(c, total, G) / KS == t) ? 0 : 1);
}
// The same slot for contributor cc of split tile t (first contributor c_lo),
// without divisions: t is the first tile of every contributor after c_lo,
// and c_lo's first tile exactly when lo_first (its range starts at t's first
// step).
__host__ __device__ __forceinline__ int split_slot(int cc, int c_lo, bool lo_first) {
  return cc == c_lo ? 2 * c_lo + (lo_first ? 0 : 1) : 2 * cc;
}

// Rows n of a warp's lanes, columns (tokens) m0 + j, j < C, of y as fp16
// (v[j] * mul, rounded to nearest even), stored for j < count.  Lanes l and
// l ^ 1 swap one value per column pair so that each stores two adjacent rows
// of one token as one 32-bit word.  n is the row of an even lane at l & ~1;
// y and N keep every such word 4-byte aligned.
template <int C>
__device__ __forceinline__ void store_y_pairs(uint16_t* y, const float (&v)[C], float mul, long long m0, int count,
                                              int N, int n, int lane) {
  static_assert(C % 2 == 0, "column pairs");
  const int odd = lane & 1;
  uint32_t* yw = reinterpret_cast<uint32_t*>(y) + (((m0 + odd) * N + (n - odd)) >> 1);
  const long long step = N;                     // two tokens, in 32-bit words
  // Eight pairs at a time: their conversions and exchanges first, then the
  // stores, so no store waits on the latency of the next pair's shuffle.
  constexpr int P = (C / 2 < 8) ? C / 2 : 8;
  static_assert((C / 2) % P == 0, "pair groups");
#pragma unroll
  for (int q0 = 0; q0 < C / 2; q0 += P) {
    uint32_t keep[P], send[P];
#pragma unroll
    for (int q = 0; q < P; ++q) {
      const uint32_t ha = __half_as_ushort(__float2half_rn(v[2 * (q0 + q)] * mul));
      const uint32_t hb = __half_as_ushort(__float2half_rn(v[2 * (q0 + q) + 1] * mul));
      keep[q] = odd ? hb : ha;
      send[q] = odd ? ha : hb;
    }
#pragma unroll
    for (int q = 0; q < P; ++q) send[q] = __shfl_xor_sync(0xffffffffu, send[q], 1);
#pragma unroll
    for (int q = 0; q < P; ++q) {
      // even lane: (own, neighbour's) at token 2q, rows n, n+1; odd lane:
      // (neighbour's, own) at token 2q+1, rows n-1, n
      const uint32_t word = odd ? (send[q] | (keep[q] << 16)) : (keep[q] | (send[q] << 16));
      if (2 * (q0 + q) + odd < count) yw[(q0 + q) * step] = word;
    }
  }
}

// C 32-bit TMEM columns of the warp's 32 lanes (C = 8, 16 or 32).
template <int C>
__device__ __forceinline__ void tmem_ld_cols(uint32_t taddr, uint32_t (&v)[C]) {
  if constexpr (C == 32) tmem_ld_32x32b_x32(taddr, v);
  else if constexpr (C == 16) tmem_ld_32x32b_x16(taddr, v);
  else tmem_ld_32x32b_x8(taddr, v);
}

// Every lane of the warp waits; the warp continues only if all lanes saw the
// phase complete, so a timeout never leaves a .sync.aligned op divergent.
__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, volatile int* abort) {
  const bool ok = wait_bounded(bar, parity, abort);
  return __all_sync(0xffffffffu, ok) != 0;
}


// Walks the CTA's steps: the step index within the tile and the tile's (row
// tile, token tile) coordinates, advanced without divisions.
struct StepCursor {
  int ks, nt, mt;
  int KS, MT;
  __device__ __forceinline__ StepCursor(long long s0, int KS_, int MT_) : KS(KS_), MT(MT_) {
    const long long tile = s0 / KS_;
    ks = static_cast<int>(s0 - tile * KS_);
    nt = static_cast<int>(tile / MT_);
    mt = static_cast<int>(tile - static_cast<long long>(nt) * MT_);
  }
  __device__ __forceinline__ void next() {
    if (++ks == KS) {
      ks = 0;
      if (++mt == MT) {
        mt = 0;
        ++nt;
      }
    }
  }
};

__device__ __forceinline__ void grid_dependency_wait() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
}
__device__ __forceinline__ void grid_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void fence_acq_rel_gpu() {
  asm volatile("fence.acq_rel.gpu;" ::: "memory");
}

// Finishes column blocks rank, rank + 4, ... (kFixCols columns each, below
// mcount) of a split tile, for the 32 rows of one row quarter, at the end of
// the CTA's range (every ring idle, this CTA's accumulator final): its own
// sums come from TMEM (dacc), the other contributors' partials by bulk copies
// into this warp's kFixBufs buffers (shared addresses buf, barriers bar), all
// summed in CTA order c_lo .. c_hi, then scaled and stored.  False if a wait
// gave up.
template <int NCOL, class S>
__device__ __forceinline__ bool finish_blocks(const LinearParams& p, int c, int c_lo, int c_hi, bool lo_first, int quad,
                                              int lane, int rank, uint32_t dacc, uint32_t bar, uint32_t buf, int m0,
                                              int mcount, int n, float mul, volatile int* abort, volatile int* never) {
  constexpr int FC = S::kFixCols;
  const int nm = c_hi - c_lo;                        // contributors read from memory
  const int nblk_all = (mcount + FC - 1) / FC;
  const int nblk = rank < nblk_all ? (nblk_all - rank + 3) / 4 : 0;
  const int items = nblk * nm;                       // item k: this warp's block k / nm, other k % nm
  auto issue = [&](int k) {                          // lane 0
    const int o = k % nm;
    const int cc = c_lo + o + ((c_lo + o >= c) ? 1 : 0);
    const int blk = rank + 4 * (k / nm);
    const int b = k % S::kFixBufs;
    mbar_arrive_expect_tx(bar + b * 8, static_cast<uint32_t>(S::kFixBlock));
    bulk_load(buf + b * S::kFixBlock,
              p.partials + partial_offset(split_slot(cc, c_lo, lo_first), quad, NCOL) + blk * FC * 32,
              static_cast<uint32_t>(S::kFixBlock), bar + b * 8, policy_evict_first());
  };
  int issued = min(items, S::kFixBufs);
  if (lane == 0) {
    fence_proxy_async_all();                         // the acquired partials, for the copies
    for (int k = 0; k < issued; ++k) issue(k);
  }
  __syncwarp();
  int k = 0;
  bool ok = true;
  for (int kb = 0; kb < nblk && ok; ++kb) {
    const int blk = rank + 4 * kb;
    float acc[FC];
#pragma unroll
    for (int j = 0; j < FC; ++j) acc[j] = 0.0f;
    for (int cc = c_lo; cc <= c_hi; ++cc) {
      if (cc == c) {
        uint32_t v[FC];
        tmem_ld_cols<FC>(dacc + blk * FC, v);
        tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < FC; ++j) acc[j] += __uint_as_float(v[j]);
        continue;
      }
      const int b = k % S::kFixBufs;
      if (!warp_wait(bar + b * 8, (k / S::kFixBufs) & 1, abort)) {
        ok = false;
        break;
      }
      float v[FC];
      ld_shared_f32x16_stride128(buf + b * S::kFixBlock + lane * 4, v);
#pragma unroll
      for (int j = 0; j < FC; ++j) acc[j] += v[j];
      __syncwarp();                                  // every lane has read the buffer: refill it
      if (k + S::kFixBufs < items) {
        if (lane == 0) issue(k + S::kFixBufs);
        ++issued;
      }
      ++k;
    }
    if (ok) store_y_pairs<FC>(p.y, acc, mul, m0 + blk * FC, mcount - blk * FC, p.N, n, lane);
  }
  // Leave no copy in flight.
  for (; k < issued; ++k) warp_wait(bar + (k % S::kFixBufs) * 8, (k / S::kFixBufs) & 1, never);
  return ok;
}

template <int NCOL, Fmt F = Fmt::E3M2>
__global__ void __launch_bounds__(kLinearThreads, 1)
    fp6_linear_kernel(const __grid_constant__ CUtensorMap tmap_x, const LinearParams p) {
  using S = LinearShape<NCOL, F>;
  using Fm = Format<F>;
  constexpr int kR = S::kR;
  constexpr int kRX = S::kRX;
  constexpr int kSW = S::kSW;
  constexpr int kISS = S::kIssuers;
  constexpr int kL = S::kL;
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
  uint64_t* fixbar = done + 1;                    // [16][kFixBufs]: fix-up copies, per warp (quarter, rank)
  uint64_t* fixgo = fixbar + S::kFixWarps * S::kFixBufs;   // [4]: a quarter's fix-up posted
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + S::kAllBars);
  volatile int* s_abort = reinterpret_cast<volatile int*>(tmem_holder + 1);
  volatile int* s_never = s_abort + 1;            // an abort flag nothing raises (final drains)
  volatile int* s_fixgo = s_never + 1;            // [4]: 1 if the quarter's last tile is finished here

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int G = p.grid;
  const int c = blockIdx.x;
  const long long total = p.total_steps;
  const int KS = p.k_steps;
  const int T = p.T;
  const int KT = p.k_tiles;
  const int MT = p.m_tiles;
  const long long s0 = range_begin(c, total, G);
  const long long s1 = range_begin(c + 1, total, G);
  const int n_local = static_cast<int>(s1 - s0);
  const long long tile_first = s0 / KS;
  const long long tile_last = (s1 - 1) / KS;

  // Let the next kernel in the stream be scheduled as early as possible.
  grid_launch_dependents();

  // Barrier set-up, one thread per barrier.
  static_assert(S::kAccIssuers == 1, "the general kernel runs 128 or 256 token columns (one accumulator)");
  if (threadIdx.x < S::kAllBars) {
    const int b = threadIdx.x;
    const int bx = 2 * kSW, br = bx + kRX, bf = br + kL, bd = bf + kL;
    uint32_t count = 1;                                       // wfull, xfull: producer arrive + tx
    if (b >= kSW && b < bx) count = 4;                        // wempty: the reading group's 4 warps
    else if (b >= br && b < bf) count = 4;                    // ready: the step's dequant group
    else if (b >= bf && b < bd) count = kISS;                 // freed: issuer commits
    else if (b == bd) count = kISS;                           // dfull
    else if (b == bd + 1) count = 4;                          // dempty: epilogue warps
    else if (b == bd + 2) count = kISS;                       // done
    else if (b >= bd + 3) count = 1;                          // fix-up copies (arrive + tx), go
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

  // Producer and issuer loops run on whole warps: every lane waits on the
  // barriers (the warp stays converged) and lane 0 alone issues the copy, MMA
  // or commit.
  if (warp == kWProdWarp) {
    // ---------------- weight producer ----------------
    const uint64_t pol = policy_evict_first();
    StepCursor cur(s0, KS, MT);
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
    StepCursor cur(s0, KS, MT);
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
      int ks = static_cast<int>(s0 - tile_first * KS);
      for (int li = 0; li < n_local; ++li, ks = (ks + 1 == KS) ? 0 : ks + 1) {
        const bool seg_first = (li == 0) || (ks == 0);
        const bool seg_last = (li == n_local - 1) || (ks == KS - 1);
        const int s = li % kR;
        const int sx = li % kRX;
        if (seg_first && sg > 0 && !wait_bounded(smem_u32(dempty), (sg - 1) & 1, s_abort)) break;
        if (!wait_bounded(smem_u32(&ready[li % kL]), (li / kL) & 1, s_abort)) break;
        {
          tc_fence_after();
          const uint64_t bdesc0 = smem_desc_sw128(smem_u32(smem + sx * S::kXStage) + b_off);
          const uint32_t a0 = tmem + s * S::kSlotCols;
          for (int t = 0; t < T; ++t) {
            // B descriptor of tile t: start address advances by kXTile bytes (>> 4)
            const uint64_t bdesc = bdesc0 + static_cast<uint64_t>(t * (S::kXTile >> 4));
#pragma unroll
            for (int j = 0; j < kSlice; ++j) {
              const int kk = kk0 + j;
              // K = 16 per MMA: 8 TMEM columns of A, 32 bytes along the swizzled B rows
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
    // The end of the range: help finish the CTA's last tile if the epilogue
    // warp of this row quarter finishes it (blocks 1 + g, 5 + g, ...).
    if (warp_wait(smem_u32(&fixgo[quad]), 0, s_abort) && s_fixgo[quad]) {
      tc_fence_after();
      const long long tile = tile_last;
      const int nt = static_cast<int>(tile / MT);
      const int mt = static_cast<int>(tile - static_cast<long long>(nt) * MT);
      const int n = nt * kTileRows + r;
      const int c_lo = range_owner(tile * KS, total, G);
      const int rank = 1 + g;
      finish_blocks<NCOL, S>(p, c, c_lo, range_owner(tile * KS + KS - 1, total, G),
                             range_begin(c_lo, total, G) == tile * KS, quad, lane, rank,
                             tmem + lane_base + S::kDCol, smem_u32(fixbar) + (quad * 4 + rank) * S::kFixBufs * 8,
                             smem_u32(smem) + (quad * 4 + rank) * S::kFixBytes, mt * NCOL, min(NCOL, p.M - mt * NCOL),
                             n, __half2float(__ushort_as_half(p.scales[n])), s_abort, s_never);
    }
  } else if (warp >= kEpiWarp && warp < kEpiWarp + 4) {
    // ---------------- epilogue warpgroup: segments in order ----------------
    // A split tile is finished without any wait on another CTA or warp.  Each
    // epilogue warp (32 rows) counts on its own counter, p.counters[4*c_lo + q]:
    //  - c_lo (the CTA holding the tile's first steps; for c_lo that is always
    //    its last segment) finishes the tile at once if every later
    //    contributor has counted; otherwise it publishes its partial and counts;
    //  - a later contributor publishes its partial and counts;
    //  - the one whose count completes the set (c_lo's and all later ones)
    //    finishes the tile.
    // Finishing sums the partials in CTA order c_lo .. c_hi, this CTA's own
    // from TMEM when its accumulator still holds it (its last segment: no
    // MMA follows), so y does not depend on which CTA finishes.  In the last
    // segment every ring is idle and the other contributors' partials come in
    // by bulk copies into that space, all in flight together; otherwise by
    // loads, 32 columns of one contributor per round trip.
    grid_dependency_wait();                  // y, partials and counters may be in use before this kernel
    const int quad = warp & 3;
    const int r = quad * 32 + lane;
    const uint32_t lane_base = static_cast<uint32_t>(quad * 32) << 16;
    const uint32_t dacc = tmem + lane_base + S::kDCol;
    bool posted = false;                     // the quarter's dequant warps have been told
    int sg = 0;
    for (long long tile = tile_first; tile <= tile_last; ++tile, ++sg) {
      if (!warp_wait(smem_u32(dfull), sg & 1, s_abort)) break;
      tc_fence_after();
      const int nt = static_cast<int>(tile / MT);
      const int mt = static_cast<int>(tile - static_cast<long long>(nt) * MT);
      const int n = nt * kTileRows + r;
      const int m0 = mt * NCOL;
      const int mcount = min(NCOL, p.M - m0);
      const float mul = __half2float(__ushort_as_half(p.scales[n]));
      const int c_lo = range_owner(tile * KS, total, G);
      const int c_hi = range_owner(tile * KS + KS - 1, total, G);
      const bool last_seg = tile == tile_last;

      // 32 accumulator columns from c0 (this CTA's own sums for the segment).
      auto own32 = [&](int c0, float (&a)[32]) {
        uint32_t v[32];
        tmem_ld_32x32b_x32(dacc + c0, v);
        tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < 32; ++j) a[j] = __uint_as_float(v[j]);
      };
      // The accumulator is read: the next segment's MMAs may overwrite it.
      auto release_acc = [&]() {
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(dempty));
      };

      if (c_lo == c_hi) {
        for (int c0 = 0; c0 < NCOL; c0 += 32) {
          float a[32];
          own32(c0, a);
          if (c0 + 32 >= NCOL) release_acc();
          store_y_pairs<32>(p.y, a, mul, m0 + c0, mcount - c0, p.N, n, lane);
        }
        continue;
      }

      const unsigned int need = static_cast<unsigned int>(c_hi - c_lo);   // adds of the later contributors
      unsigned int* cnt = p.counters + 4 * c_lo + quad;
      const bool lo_first = range_begin(c_lo, total, G) == tile * KS;
      auto part_of = [&](int cc) -> const float* {
        return p.partials + partial_offset(split_slot(cc, c_lo, lo_first), quad, NCOL);
      };
      bool finish;
      if (c == c_lo && __all_sync(0xffffffffu, ld_acquire(cnt) == need)) {
        finish = true;                       // every later partial is there
      } else {
        // Publish this CTA's partial, then count (release).  The lanes' stores
        // are ordered before lane 0's add by the warp barrier, and its release
        // publishes them with its own.
        float* mine = p.partials + partial_offset(2 * c + ((tile == tile_first) ? 0 : 1), quad, NCOL) + lane;
        for (int c0 = 0; c0 < NCOL; c0 += 16) {
          uint32_t v[16];
          tmem_ld_32x32b_x16(dacc + c0, v);
          tmem_wait_ld();
#pragma unroll
          for (int j = 0; j < 16; ++j) __stcg(mine + (c0 + j) * 32, __uint_as_float(v[j]));
        }
        release_acc();
        unsigned int old = 0;
        if (lane == 0) old = atom_add_acq_rel(cnt, 1u);
        finish = __shfl_sync(0xffffffffu, old, 0) == need;
        if (finish) (void)ld_acquire(cnt);   // every lane acquires the others' partials
      }
      if (!finish) continue;

      bool ok = true;
      if (last_seg) {
        // Post the tile to the quarter's dequant warps (no MMA or ring use
        // follows), then take this warp's share: blocks 0, 4, 8, ...
        if (lane == 0) {
          s_fixgo[quad] = 1;
          mbar_arrive(smem_u32(&fixgo[quad]));
        }
        posted = true;
        ok = finish_blocks<NCOL, S>(p, c, c_lo, c_hi, lo_first, quad, lane, 0, dacc,
                                    smem_u32(fixbar) + quad * 4 * S::kFixBufs * 8,
                                    smem_u32(smem) + quad * 4 * S::kFixBytes, m0, mcount, n, mul, s_abort, s_never);
      } else {
        // Every partial from memory (this CTA's too: its accumulator may
        // already hold the next segment's sums), 16 columns of one
        // contributor per round trip.
        for (int c0 = 0; c0 < mcount; c0 += 16) {
          float acc[16];
#pragma unroll
          for (int j = 0; j < 16; ++j) acc[j] = 0.0f;
          for (int cc = c_lo; cc <= c_hi; ++cc) {
            const float* src = part_of(cc) + c0 * 32 + lane;
            float v[16];
#pragma unroll
            for (int j = 0; j < 16; ++j) v[j] = __ldcg(src + j * 32);
#pragma unroll
            for (int j = 0; j < 16; ++j) acc[j] += v[j];
          }
          store_y_pairs<16>(p.y, acc, mul, m0 + c0, mcount - c0, p.N, n, lane);
        }
      }
      if (!ok) break;
      __syncwarp();
      if (lane == 0) *cnt = 0u;              // every contributor has counted: reset for the next launch
    }
    if (!posted && lane == 0) {              // nothing for the dequant warps to help with
      s_fixgo[quad] = 0;
      mbar_arrive(smem_u32(&fixgo[quad]));
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
