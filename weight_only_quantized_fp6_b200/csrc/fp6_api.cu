// fp6_api.cu -- the C ABI of libfp6.so (declared in include/fp6.h).
// Validates arguments on the host, picks the launch configuration, encodes
// the activation tensor map and launches the kernels on the caller's stream.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>
#include <cstdlib>
#include <cstring>
#include <mutex>

#include "fp6.h"
#include "fp6_aux_kernels.cuh"
#include "fp6_linear.cuh"
#include "fp6_linear_decode.cuh"
#include "fp6_linear_wave.cuh"

namespace fp6 {
// A wait that can never complete: the mbarrier expects one arrival that no
// thread makes.  The bounded wait gives up after its time limit, raises the
// device error word and returns; the kernel then exits normally.
__global__ void wait_timeout_kernel() {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bar), 1);
    abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();
  warp_wait(smem_u32(&bar), 0, &abort_flag);
}
}  // namespace fp6

namespace {

using fp6::DecodeShape;
using fp6::Fmt;
using fp6::LinearShape;

constexpr int kMaxDevices = 64;

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

fp6_status check_shape(int64_t N, int64_t K) {
  if (N < 0 || K < 0) return FP6_ERR_INVALID_ARG;
  if (N % fp6::kTileRows != 0 || K % fp6::kTileCols != 0) return FP6_ERR_UNSUPPORTED_SHAPE;
  if (N > (int64_t(1) << 30) || K > (int64_t(1) << 30)) return FP6_ERR_UNSUPPORTED_SHAPE;
  return FP6_OK;
}

fp6_status cuda_status(cudaError_t e) { return e == cudaSuccess ? FP6_OK : FP6_ERR_CUDA; }

// ---- host-side fault injection (tests of the error paths; no GPU fault) ------
// FP6_FAULT_INJECT=<point>[:<count>] makes the named host step report failure
// the next <count> times it runs (every time without a count), as if the CUDA
// call behind it had failed: "encode" (the activation tensor map), "launch"
// (a kernel launch: nothing is enqueued), "sync" (the quantizer's stream
// synchronisation).  The caller sees FP6_ERR_CUDA; no kernel is started.
struct FaultPlan {
  char point[16] = {0};
  long long left = 0;   // < 0: unlimited
};
FaultPlan g_fault;
std::once_flag g_fault_once;
std::mutex g_fault_mu;

bool fault(const char* point) {
  std::call_once(g_fault_once, [] {
    const char* v = std::getenv("FP6_FAULT_INJECT");
    if (!v || !*v) return;
    const char* colon = std::strchr(v, ':');
    const size_t n = colon ? static_cast<size_t>(colon - v) : std::strlen(v);
    if (n == 0 || n >= sizeof(g_fault.point)) return;
    std::memcpy(g_fault.point, v, n);
    g_fault.left = colon ? std::atoll(colon + 1) : -1;
  });
  if (g_fault.point[0] == 0 || std::strcmp(g_fault.point, point) != 0) return false;
  std::lock_guard<std::mutex> lk(g_fault_mu);
  if (g_fault.left == 0) return false;
  if (g_fault.left > 0) --g_fault.left;
  return true;
}

// ---- per-device cached properties ------------------------------------------
struct DeviceInfo {
  int sms = 0;
  bool attrs_set[5][10] = {};  // [format][kernel variant]: shared-memory limit raised
};
DeviceInfo g_dev[kMaxDevices];
std::mutex g_mu;

int current_device_sms(int* dev_out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 0;
  *dev_out = dev;
  std::lock_guard<std::mutex> lk(g_mu);
  if (g_dev[dev].sms == 0) {
    int v = 0;
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
    g_dev[dev].sms = v;
  }
  return g_dev[dev].sms;
}

// ---- tensor-map encoder from the driver (no link-time libcuda dependency) ---
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// ---- launch plan --------------------------------------------------------------
struct Plan {
  int ncol = 16;
  int stages = 0;
  int grid = 0;
  int n_tiles = 0, m_tiles = 0, k_tiles = 0;
  int T = 1;        // 64-column tiles per pipeline step
  int k_steps = 0;  // steps per (row tile, token tile)
  long long tiles = 0;
  long long total = 0;  // steps in all
  size_t counter_bytes = 0;
  size_t partial_bytes = 0;
  bool wave = false;  // whole tiles per CTA (fp6_linear_wave.cuh) instead of stream-K ranges
};

int pick_ncol(int64_t M) {
  if (M <= 16) return 16;
  if (M <= 32) return 32;
  if (M <= 64) return 64;
  if (M <= 128) return 128;
  return 256;
}

// One token tile of up to 64 columns runs the decode kernel
// (fp6_linear_decode.cuh), wider or several token tiles the general kernel
// (fp6_linear.cuh).
int tmax_for(int ncol) {
  switch (ncol) {
    case 16: return DecodeShape<16>::kTMax;
    case 32: return DecodeShape<32>::kTMax;
    case 64: return DecodeShape<64>::kTMax;
    case 128: return LinearShape<128>::kTMax;
    default: return LinearShape<256>::kTMax;
  }
}

int stages_for(int ncol) {
  switch (ncol) {
    case 16: return DecodeShape<16>::kSW;
    case 32: return DecodeShape<32>::kSW;
    case 64: return DecodeShape<64>::kSW;
    case 128: return LinearShape<128>::kSW;
    default: return LinearShape<256>::kSW;
  }
}

// Pipeline steps of one launch at most: the kernels index steps with 64-bit
// arithmetic (range bounds multiply a step index by the grid size) and count
// a CTA's own steps in 32 bits.
constexpr long long kMaxTotalSteps = 1LL << 40;

// The launch plan for an M x N x K problem (shape already checked) on `sms`
// multiprocessors.  FP6_ERR_UNSUPPORTED_SHAPE when the problem has more
// pipeline steps than the kernels can count.
fp6_status make_plan(int64_t M, int64_t N, int64_t K, int sms, Plan* pl) {
  pl->ncol = pick_ncol(M);
  pl->stages = stages_for(pl->ncol);
  pl->n_tiles = static_cast<int>(N / fp6::kTileRows);
  pl->m_tiles = static_cast<int>((M + pl->ncol - 1) / pl->ncol);
  pl->k_tiles = static_cast<int>(K / fp6::kTileCols);
  pl->tiles = static_cast<long long>(pl->n_tiles) * pl->m_tiles;   // < 2^23 * 2^27
  // widest step (power of two up to the variant's limit) that divides K/64
  pl->T = tmax_for(pl->ncol);
  while (pl->T > 1 && pl->k_tiles % pl->T != 0) pl->T >>= 1;
  pl->k_steps = pl->k_tiles / pl->T;
  if (pl->k_steps > 0 && pl->tiles > kMaxTotalSteps / pl->k_steps) return FP6_ERR_UNSUPPORTED_SHAPE;
  pl->total = pl->tiles * pl->k_steps;
  if (pl->total <= 0) {
    pl->grid = 0;
    return FP6_OK;
  }
  pl->grid = static_cast<int>(std::min<long long>(std::min(sms, fp6::kMaxGrid), pl->total));
  if ((pl->total + pl->grid - 1) / pl->grid > INT32_MAX) return FP6_ERR_UNSUPPORTED_SHAPE;
  // Many tiles and a nearly full last wave (at most 5 % of the CTA-tile slots
  // idle): whole tiles per CTA, which share weights and activations through
  // L2; otherwise the stream-K ranges balance the work exactly.
  if (pl->ncol > 64) {
    const long long G = std::min(sms, fp6::kMaxGrid);
    const long long waves = (pl->tiles + G - 1) / G;
    if (pl->tiles >= G && waves * G * 100 <= pl->tiles * 105) {
      pl->wave = true;
      pl->grid = static_cast<int>(G);
    }
  }
  pl->counter_bytes = fp6::kCounterBytes;
  pl->partial_bytes = static_cast<size_t>(2) * pl->grid * pl->ncol * 128 * sizeof(float);
  return FP6_OK;
}

// Launches one variant with programmatic dependent launch: the kernel may
// begin while the previous kernel in the stream finishes (see the kernel's
// grid-dependency rules).
template <int NCOL, Fmt F>
fp6_status launch_linear(const CUtensorMap& map, const fp6::LinearParams& prm, cudaStream_t stream, int dev) {
  auto kern = fp6::fp6_linear_kernel<NCOL, F>;
  const int smem = LinearShape<NCOL, F>::kSmemBytes;
  const int threads = fp6::kLinearThreads;
  const int idx = NCOL == 16 ? 0 : NCOL == 32 ? 1 : NCOL == 64 ? 2 : NCOL == 128 ? 3 : 4;
  {
    std::lock_guard<std::mutex> lk(g_mu);
    if (!g_dev[dev].attrs_set[static_cast<int>(F)][idx]) {
      if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
        return FP6_ERR_CUDA;
      g_dev[dev].attrs_set[static_cast<int>(F)][idx] = true;
    }
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned int>(prm.grid));
  cfg.blockDim = dim3(static_cast<unsigned int>(threads));
  cfg.dynamicSmemBytes = static_cast<size_t>(smem);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (fault("launch") || cudaLaunchKernelEx(&cfg, kern, map, prm) != cudaSuccess) return FP6_ERR_CUDA;
  return cuda_status(cudaGetLastError());
}

// The wave-schedule kernel (whole tiles per CTA), launched the same way.
template <int NCOL, Fmt F>
fp6_status launch_wave(const CUtensorMap& map, const fp6::LinearParams& prm, cudaStream_t stream, int dev) {
  auto kern = fp6::fp6_linear_wave_kernel<NCOL, F>;
  const int smem = LinearShape<NCOL, F>::kSmemBytes;
  const int idx = NCOL == 128 ? 8 : 9;
  {
    std::lock_guard<std::mutex> lk(g_mu);
    if (!g_dev[dev].attrs_set[static_cast<int>(F)][idx]) {
      if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
        return FP6_ERR_CUDA;
      g_dev[dev].attrs_set[static_cast<int>(F)][idx] = true;
    }
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned int>(prm.grid));
  cfg.blockDim = dim3(static_cast<unsigned int>(fp6::kLinearThreads));
  cfg.dynamicSmemBytes = static_cast<size_t>(smem);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (fault("launch") || cudaLaunchKernelEx(&cfg, kern, map, prm) != cudaSuccess) return FP6_ERR_CUDA;
  return cuda_status(cudaGetLastError());
}

// The decode kernel (one token tile of at most 64 columns), launched the same way.
template <int NCOL, Fmt F>
fp6_status launch_decode(const CUtensorMap& map, const fp6::LinearParams& prm, cudaStream_t stream, int dev) {
  auto kern = fp6::fp6_linear_decode_kernel<NCOL, F>;
  const int smem = DecodeShape<NCOL, F>::kSmemBytes;
  const int idx = NCOL == 16 ? 5 : NCOL == 32 ? 6 : 7;
  {
    std::lock_guard<std::mutex> lk(g_mu);
    if (!g_dev[dev].attrs_set[static_cast<int>(F)][idx]) {
      if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
        return FP6_ERR_CUDA;
      g_dev[dev].attrs_set[static_cast<int>(F)][idx] = true;
    }
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned int>(prm.grid));
  cfg.blockDim = dim3(static_cast<unsigned int>(DecodeShape<NCOL, F>::kThreads));
  cfg.dynamicSmemBytes = static_cast<size_t>(smem);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (fault("launch") || cudaLaunchKernelEx(&cfg, kern, map, prm) != cudaSuccess) return FP6_ERR_CUDA;
  return cuda_status(cudaGetLastError());
}

// Packed bytes of an N x K weight in format f (shape already checked).
size_t packed_bytes_of(Fmt f, int64_t N, int64_t K) {
  const size_t nk = static_cast<size_t>(N) * static_cast<size_t>(K);
  switch (f) {
    case Fmt::E2M1: return nk / 2;
    case Fmt::E2M2: return nk / 8 * 5;
    case Fmt::S24: return nk / 8 * 3;
    default: return nk / 4 * 3;
  }
}

bool fmt_of(int fmt, Fmt* out) {
  if (fmt < 0 || fmt > 3) return false;
  *out = static_cast<Fmt>(fmt);
  return true;
}

template <Fmt F>
fp6_status quantize_impl(const float* W, int64_t N, int64_t K, uint8_t* codes, uint16_t* scales,
                        cudaStream_t stream) {
  if (N < 0 || K < 0) return FP6_ERR_INVALID_ARG;
  if (N == 0) return FP6_OK;
  if (N > INT32_MAX) return FP6_ERR_UNSUPPORTED_SHAPE;
  if (!scales || (K > 0 && (!W || !codes))) return FP6_ERR_INVALID_ARG;
  if (!aligned16(W) || !aligned16(codes) || !aligned16(scales)) return FP6_ERR_MISALIGNED;
  const unsigned int zero = 0;
  cudaError_t e = cudaMemcpyToSymbolAsync(fp6::g_quant_error, &zero, sizeof(zero), 0,
                                          cudaMemcpyHostToDevice, stream);
  if (e != cudaSuccess) return FP6_ERR_CUDA;
  fp6::quantize_kernel<256, F><<<static_cast<unsigned int>(N), 256, 0, stream>>>(W, K, codes, scales);
  if (cudaGetLastError() != cudaSuccess) return FP6_ERR_CUDA;
  unsigned int flags = 0;
  e = cudaMemcpyFromSymbolAsync(&flags, fp6::g_quant_error, sizeof(flags), 0, cudaMemcpyDeviceToHost, stream);
  if (e != cudaSuccess) return FP6_ERR_CUDA;
  // (the synchronisation itself always runs: the flag copy above writes into `flags`)
  if (cudaStreamSynchronize(stream) != cudaSuccess || fault("sync")) return FP6_ERR_CUDA;
  if (flags & fp6::kQuantNonfinite) return FP6_ERR_NONFINITE;
  if (flags & fp6::kQuantScaleRange) return FP6_ERR_SCALE_RANGE;
  return FP6_OK;
}

template <Fmt F>
fp6_status prepack_impl(const uint8_t* codes, int64_t N, int64_t K, void* packed, size_t packed_bytes,
                       cudaStream_t stream) {
  fp6_status st = check_shape(N, K);
  if (st != FP6_OK) return st;
  if (N == 0 || K == 0) return FP6_OK;
  if (!codes || !packed) return FP6_ERR_INVALID_ARG;
  if (packed_bytes < packed_bytes_of(F, N, K)) return FP6_ERR_INVALID_ARG;
  if (!aligned16(codes) || !aligned16(packed)) return FP6_ERR_MISALIGNED;
  const int64_t work = N * (K / fp6::kTileCols);
  const int64_t blocks = (work + 255) / 256;
  fp6::prepack_kernel<F><<<static_cast<unsigned int>(blocks), 256, 0, stream>>>(
      codes, N, K, static_cast<uint8_t*>(packed));
  return cuda_status(cudaGetLastError());
}

template <Fmt F>
fp6_status dequant_impl(const void* packed, const uint16_t* scales, int64_t N, int64_t K, uint16_t* W16,
                       cudaStream_t stream) {
  fp6_status st = check_shape(N, K);
  if (st != FP6_OK) return st;
  if (N == 0 || K == 0) return FP6_OK;
  if (!packed || !W16) return FP6_ERR_INVALID_ARG;
  if (!aligned16(packed) || !aligned16(W16) || (scales && !aligned16(scales))) return FP6_ERR_MISALIGNED;
  const int64_t units = (N / 32) * (K / fp6::kTileCols);   // 32 rows of one tile per warp
  const int64_t blocks = std::min<int64_t>((units + fp6::kDequantWarps - 1) / fp6::kDequantWarps, 1 << 20);
  fp6::dequant_kernel<F><<<static_cast<unsigned int>(blocks), 32 * fp6::kDequantWarps, 0, stream>>>(
      static_cast<const uint8_t*>(packed), scales, N, K, W16);
  return cuda_status(cudaGetLastError());
}

template <Fmt F>
fp6_status linear_impl(const uint16_t* x, const void* packed, const uint16_t* scales, int64_t M, int64_t N,
                      int64_t K, uint16_t* y, void* workspace, size_t workspace_bytes, cudaStream_t stream) {
  fp6_status st = check_shape(N, K);
  if (st != FP6_OK) return st;
  if (M < 0) return FP6_ERR_INVALID_ARG;
  if (M > INT32_MAX) return FP6_ERR_UNSUPPORTED_SHAPE;
  if (M == 0 || N == 0) return FP6_OK;
  if (!y) return FP6_ERR_INVALID_ARG;
  if (!aligned16(y)) return FP6_ERR_MISALIGNED;
  if (K == 0) {  // empty sum
    return cuda_status(cudaMemsetAsync(y, 0, static_cast<size_t>(M) * N * sizeof(uint16_t), stream));
  }
  if (!x || !packed || !scales) return FP6_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(packed) || !aligned16(scales)) return FP6_ERR_MISALIGNED;
  int dev = 0;
  const int sms = current_device_sms(&dev);
  if (sms <= 0) return FP6_ERR_CUDA;
  Plan pl;
  st = make_plan(M, N, K, sms, &pl);
  if (st != FP6_OK) return st;
  const size_t need = pl.counter_bytes + pl.partial_bytes;
  if (workspace_bytes < need || (need > 0 && workspace == nullptr)) return FP6_ERR_WORKSPACE;
  if (need > 0 && !aligned16(workspace)) return FP6_ERR_MISALIGNED;

  fp6::LinearParams prm;
  prm.x = x;
  prm.packed = static_cast<const uint8_t*>(packed);
  prm.scales = scales;
  prm.y = y;
  prm.counters = static_cast<uint32_t*>(workspace);
  prm.partials = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + pl.counter_bytes);
  prm.M = static_cast<int>(M);
  prm.N = static_cast<int>(N);
  prm.K = static_cast<int>(K);
  prm.n_tiles = pl.n_tiles;
  prm.m_tiles = pl.m_tiles;
  prm.k_tiles = pl.k_tiles;
  prm.T = pl.T;
  prm.k_steps = pl.k_steps;
  prm.total_steps = pl.total;
  prm.grid = pl.grid;
  EncodeTiledFn encode = get_encode_fn();
  if (!encode) return FP6_ERR_CUDA;
  CUtensorMap map;
  std::memset(&map, 0, sizeof(map));
  // x as [K/64][M][64] (column tile, row, column): one box of T column tiles x
  // NCOL rows per pipeline step; rows >= M read as zero
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(fp6::kTileCols), static_cast<cuuint64_t>(M),
                              static_cast<cuuint64_t>(K / fp6::kTileCols)};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(K) * sizeof(uint16_t),
                                 static_cast<cuuint64_t>(fp6::kTileCols) * sizeof(uint16_t)};
  const cuuint32_t box[3] = {static_cast<cuuint32_t>(fp6::kTileCols), static_cast<cuuint32_t>(pl.ncol),
                             static_cast<cuuint32_t>(pl.T)};
  const cuuint32_t estr[3] = {1, 1, 1};
  const CUresult cr = encode(&map, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3, const_cast<uint16_t*>(x), dims, strides, box,
                             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (cr != CUDA_SUCCESS || fault("encode")) return FP6_ERR_CUDA;

  switch (pl.ncol) {
    case 16: return launch_decode<16, F>(map, prm, stream, dev);
    case 32: return launch_decode<32, F>(map, prm, stream, dev);
    case 64: return launch_decode<64, F>(map, prm, stream, dev);
    case 128: return pl.wave ? launch_wave<128, F>(map, prm, stream, dev) : launch_linear<128, F>(map, prm, stream, dev);
    default: return pl.wave ? launch_wave<256, F>(map, prm, stream, dev) : launch_linear<256, F>(map, prm, stream, dev);
  }
}

}  // namespace

extern "C" {

const char* fp6_status_string(fp6_status s) {
  switch (s) {
    case FP6_OK: return "FP6_OK";
    case FP6_ERR_INVALID_ARG: return "FP6_ERR_INVALID_ARG";
    case FP6_ERR_UNSUPPORTED_SHAPE: return "FP6_ERR_UNSUPPORTED_SHAPE";
    case FP6_ERR_MISALIGNED: return "FP6_ERR_MISALIGNED";
    case FP6_ERR_NONFINITE: return "FP6_ERR_NONFINITE";
    case FP6_ERR_SCALE_RANGE: return "FP6_ERR_SCALE_RANGE";
    case FP6_ERR_WORKSPACE: return "FP6_ERR_WORKSPACE";
    case FP6_ERR_LAYOUT_VERSION: return "FP6_ERR_LAYOUT_VERSION";
    case FP6_ERR_CUDA: return "FP6_ERR_CUDA";
    case FP6_ERR_TIMEOUT: return "FP6_ERR_TIMEOUT";
  }
  return "FP6_ERR_UNKNOWN";
}

size_t fp6_packed_bytes(int64_t N, int64_t K) {
  if (check_shape(N, K) != FP6_OK) return 0;
  return packed_bytes_of(Fmt::E3M2, N, K);
}

fp6_status fp6_quantize(const float* W, int64_t N, int64_t K, uint8_t* codes, uint16_t* scales,
                        cudaStream_t stream) {
  return quantize_impl<Fmt::E3M2>(W, N, K, codes, scales, stream);
}

fp6_status fp6_prepack(const uint8_t* codes, int64_t N, int64_t K, void* packed, size_t packed_bytes,
                       cudaStream_t stream) {
  return prepack_impl<Fmt::E3M2>(codes, N, K, packed, packed_bytes, stream);
}

fp6_status fp6_dequant(const void* packed, const uint16_t* scales, int64_t N, int64_t K, uint16_t* W16,
                       cudaStream_t stream) {
  return dequant_impl<Fmt::E3M2>(packed, scales, N, K, W16, stream);
}

fp6_status fp6_linear_plan(int64_t M, int64_t N, int64_t K, int64_t out[5]) {
  if (!out) return FP6_ERR_INVALID_ARG;
  fp6_status st = check_shape(N, K);
  if (st != FP6_OK) return st;
  if (M < 0) return FP6_ERR_INVALID_ARG;
  if (M > INT32_MAX) return FP6_ERR_UNSUPPORTED_SHAPE;
  int dev = 0;
  const int sms = current_device_sms(&dev);
  if (sms <= 0) return FP6_ERR_CUDA;
  Plan pl;
  st = make_plan(M, N, K, sms, &pl);
  if (st != FP6_OK) return st;
  out[0] = pl.ncol;
  out[1] = pl.stages;
  out[2] = pl.grid;
  out[3] = pl.tiles;
  out[4] = pl.total;
  return FP6_OK;
}

fp6_status fp6_linear_plan_for_sms(int64_t M, int64_t N, int64_t K, int sms, int64_t out[7]) {
  if (!out) return FP6_ERR_INVALID_ARG;
  fp6_status st = check_shape(N, K);
  if (st != FP6_OK) return st;
  if (M < 0 || sms <= 0) return FP6_ERR_INVALID_ARG;
  if (M > INT32_MAX) return FP6_ERR_UNSUPPORTED_SHAPE;
  Plan pl;
  st = make_plan(M, N, K, sms, &pl);
  if (st != FP6_OK) return st;
  out[0] = pl.ncol;
  out[1] = pl.stages;
  out[2] = pl.grid;
  out[3] = pl.tiles;
  out[4] = pl.total;
  out[5] = pl.T;
  out[6] = pl.wave ? 1 : 0;
  return FP6_OK;
}

size_t fp6_linear_workspace_bytes(int64_t M, int64_t N, int64_t K) {
  if (check_shape(N, K) != FP6_OK || M < 0 || M > INT32_MAX) return 0;
  int dev = 0;
  const int sms = current_device_sms(&dev);
  if (sms <= 0) return 0;
  Plan pl;
  if (make_plan(M, N, K, sms, &pl) != FP6_OK || pl.grid == 0) return 0;
  return pl.counter_bytes + pl.partial_bytes;
}

fp6_status fp6_linear(const uint16_t* x, const void* packed, const uint16_t* scales, int64_t M, int64_t N,
                      int64_t K, uint16_t* y, void* workspace, size_t workspace_bytes, cudaStream_t stream) {
  return linear_impl<Fmt::E3M2>(x, packed, scales, M, N, K, y, workspace, workspace_bytes, stream);
}

// ---- other formats (fpx_format) -----------------------------------------------
size_t fpx_packed_bytes(fpx_format fmt, int64_t N, int64_t K) {
  Fmt f;
  if (!fmt_of(fmt, &f) || check_shape(N, K) != FP6_OK) return 0;
  return packed_bytes_of(f, N, K);
}

fp6_status fpx_quantize(fpx_format fmt, const float* W, int64_t N, int64_t K, uint8_t* codes, uint16_t* scales,
                        cudaStream_t stream) {
  Fmt f;
  if (!fmt_of(fmt, &f)) return FP6_ERR_INVALID_ARG;
  switch (f) {
    case Fmt::E3M2: return quantize_impl<Fmt::E3M2>(W, N, K, codes, scales, stream);
    case Fmt::E2M3: return quantize_impl<Fmt::E2M3>(W, N, K, codes, scales, stream);
    case Fmt::E2M1: return quantize_impl<Fmt::E2M1>(W, N, K, codes, scales, stream);
    default: return quantize_impl<Fmt::E2M2>(W, N, K, codes, scales, stream);
  }
}

fp6_status fpx_prepack(fpx_format fmt, const uint8_t* codes, int64_t N, int64_t K, void* packed,
                       size_t packed_bytes, cudaStream_t stream) {
  Fmt f;
  if (!fmt_of(fmt, &f)) return FP6_ERR_INVALID_ARG;
  switch (f) {
    case Fmt::E3M2: return prepack_impl<Fmt::E3M2>(codes, N, K, packed, packed_bytes, stream);
    case Fmt::E2M3: return prepack_impl<Fmt::E2M3>(codes, N, K, packed, packed_bytes, stream);
    case Fmt::E2M1: return prepack_impl<Fmt::E2M1>(codes, N, K, packed, packed_bytes, stream);
    default: return prepack_impl<Fmt::E2M2>(codes, N, K, packed, packed_bytes, stream);
  }
}

fp6_status fpx_dequant(fpx_format fmt, const void* packed, const uint16_t* scales, int64_t N, int64_t K,
                       uint16_t* W16, cudaStream_t stream) {
  Fmt f;
  if (!fmt_of(fmt, &f)) return FP6_ERR_INVALID_ARG;
  switch (f) {
    case Fmt::E3M2: return dequant_impl<Fmt::E3M2>(packed, scales, N, K, W16, stream);
    case Fmt::E2M3: return dequant_impl<Fmt::E2M3>(packed, scales, N, K, W16, stream);
    case Fmt::E2M1: return dequant_impl<Fmt::E2M1>(packed, scales, N, K, W16, stream);
    default: return dequant_impl<Fmt::E2M2>(packed, scales, N, K, W16, stream);
  }
}

fp6_status fpx_linear(fpx_format fmt, const uint16_t* x, const void* packed, const uint16_t* scales, int64_t M,
                      int64_t N, int64_t K, uint16_t* y, void* workspace, size_t workspace_bytes,
                      cudaStream_t stream) {
  Fmt f;
  if (!fmt_of(fmt, &f)) return FP6_ERR_INVALID_ARG;
  switch (f) {
    case Fmt::E3M2: return linear_impl<Fmt::E3M2>(x, packed, scales, M, N, K, y, workspace, workspace_bytes, stream);
    case Fmt::E2M3: return linear_impl<Fmt::E2M3>(x, packed, scales, M, N, K, y, workspace, workspace_bytes, stream);
    case Fmt::E2M1: return linear_impl<Fmt::E2M1>(x, packed, scales, M, N, K, y, workspace, workspace_bytes, stream);
    default: return linear_impl<Fmt::E2M2>(x, packed, scales, M, N, K, y, workspace, workspace_bytes, stream);
  }
}

// ---- 2:4 sparse INT4 (Sparse-Marlin) ------------------------------------------
size_t s24_packed_bytes(int64_t N, int64_t K) {
  if (check_shape(N, K) != FP6_OK) return 0;
  return packed_bytes_of(Fmt::S24, N, K);
}

fp6_status s24_quantize(const float* W, int64_t N, int64_t K, int8_t* q, uint8_t* pos, uint16_t* scales,
                        cudaStream_t stream) {
  if (N < 0 || K < 0) return FP6_ERR_INVALID_ARG;
  if (K % 4 != 0) return FP6_ERR_UNSUPPORTED_SHAPE;
  if (N == 0) return FP6_OK;
  if (N > INT32_MAX) return FP6_ERR_UNSUPPORTED_SHAPE;
  if (!scales || (K > 0 && (!W || !q || !pos))) return FP6_ERR_INVALID_ARG;
  if (!aligned16(W) || !aligned16(q) || !aligned16(pos) || !aligned16(scales)) return FP6_ERR_MISALIGNED;
  const unsigned int zero = 0;
  cudaError_t e = cudaMemcpyToSymbolAsync(fp6::g_quant_error, &zero, sizeof(zero), 0,
                                          cudaMemcpyHostToDevice, stream);
  if (e != cudaSuccess) return FP6_ERR_CUDA;
  fp6::s24_quantize_kernel<256><<<static_cast<unsigned int>(N), 256, 0, stream>>>(W, K, q, pos, scales);
  if (cudaGetLastError() != cudaSuccess) return FP6_ERR_CUDA;
  unsigned int flags = 0;
  e = cudaMemcpyFromSymbolAsync(&flags, fp6::g_quant_error, sizeof(flags), 0, cudaMemcpyDeviceToHost, stream);
  if (e != cudaSuccess) return FP6_ERR_CUDA;
  // (the synchronisation itself always runs: the flag copy above writes into `flags`)
  if (cudaStreamSynchronize(stream) != cudaSuccess || fault("sync")) return FP6_ERR_CUDA;
  if (flags & fp6::kQuantNonfinite) return FP6_ERR_NONFINITE;
  if (flags & fp6::kQuantScaleRange) return FP6_ERR_SCALE_RANGE;
  return FP6_OK;
}

fp6_status s24_prepack(const int8_t* q, const uint8_t* pos, int64_t N, int64_t K, void* packed,
                       size_t packed_bytes, cudaStream_t stream) {
  fp6_status st = check_shape(N, K);
  if (st != FP6_OK) return st;
  if (N == 0 || K == 0) return FP6_OK;
  if (!q || !pos || !packed) return FP6_ERR_INVALID_ARG;
  if (packed_bytes < packed_bytes_of(Fmt::S24, N, K)) return FP6_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(pos) || !aligned16(packed)) return FP6_ERR_MISALIGNED;
  const int64_t work = N * (K / fp6::kTileCols);
  const int64_t blocks = (work + 255) / 256;
  fp6::s24_prepack_kernel<<<static_cast<unsigned int>(blocks), 256, 0, stream>>>(q, pos, N, K,
                                                                                   static_cast<uint8_t*>(packed));
  return cuda_status(cudaGetLastError());
}

fp6_status s24_dequant(const void* packed, const uint16_t* scales, int64_t N, int64_t K, uint16_t* W16,
                       cudaStream_t stream) {
  return dequant_impl<Fmt::S24>(packed, scales, N, K, W16, stream);
}

fp6_status s24_linear(const uint16_t* x, const void* packed, const uint16_t* scales, int64_t M, int64_t N,
                      int64_t K, uint16_t* y, void* workspace, size_t workspace_bytes, cudaStream_t stream) {
  return linear_impl<Fmt::S24>(x, packed, scales, M, N, K, y, workspace, workspace_bytes, stream);
}

// ---- stored packed weights: the blob header ------------------------------------
}  // extern "C"

namespace {

struct HeaderFields {
  uint32_t version, tile_bytes;
  size_t payload;
};

bool header_fields(int fmt, int64_t N, int64_t K, HeaderFields* h) {
  Fmt f;
  if (fmt == FPX_S24) {
    f = Fmt::S24;
    h->version = FP6_LAYOUT_VERSION_S24;
  } else if (fmt_of(fmt, &f)) {
    h->version = (f == Fmt::E2M1) ? FP6_LAYOUT_VERSION_E2M1
               : (f == Fmt::E2M2) ? FP6_LAYOUT_VERSION_E2M2 : FP6_LAYOUT_VERSION_E3M2;
  } else {
    return false;
  }
  h->tile_bytes = static_cast<uint32_t>(packed_bytes_of(f, fp6::kTileRows, fp6::kTileCols));
  h->payload = packed_bytes_of(f, N, K);
  return true;
}

void put32(uint8_t* p, uint32_t v) { std::memcpy(p, &v, 4); }
void put64(uint8_t* p, uint64_t v) { std::memcpy(p, &v, 8); }

}  // namespace

extern "C" {

fp6_status fp6_packed_header(fpx_format fmt, int64_t N, int64_t K, void* header) {
  if (!header) return FP6_ERR_INVALID_ARG;
  HeaderFields h;
  if (!header_fields(fmt, N, K, &h)) return FP6_ERR_INVALID_ARG;
  const fp6_status st = check_shape(N, K);
  if (st != FP6_OK) return st;
  uint8_t* b = static_cast<uint8_t*>(header);
  std::memset(b, 0, FP6_PACKED_HEADER_BYTES);
  std::memcpy(b, "FP6W", 4);
  put32(b + 4, h.version);
  put32(b + 8, static_cast<uint32_t>(fmt));
  put32(b + 12, FP6_PACKED_HEADER_BYTES);
  put64(b + 16, static_cast<uint64_t>(N));
  put64(b + 24, static_cast<uint64_t>(K));
  put32(b + 32, fp6::kTileRows);
  put32(b + 36, fp6::kTileCols);
  put32(b + 40, h.tile_bytes);
  put32(b + 44, 2);
  put64(b + 48, h.payload);
  return FP6_OK;
}

fp6_status fp6_packed_header_check(const void* header, fpx_format fmt, int64_t N, int64_t K) {
  if (!header) return FP6_ERR_INVALID_ARG;
  uint8_t want[FP6_PACKED_HEADER_BYTES];
  const fp6_status st = fp6_packed_header(fmt, N, K, want);
  if (st == FP6_ERR_UNSUPPORTED_SHAPE) return FP6_ERR_LAYOUT_VERSION;   // no blob of this library has that shape
  if (st != FP6_OK) return st;
  return std::memcmp(want, header, FP6_PACKED_HEADER_BYTES) == 0 ? FP6_OK : FP6_ERR_LAYOUT_VERSION;
}

fp6_status fp6_get_device_status(cudaStream_t stream) {
  unsigned int word = 0;
  const unsigned int zero = 0;
  if (cudaMemcpyFromSymbolAsync(&word, fp6::g_error_word, sizeof(word), 0, cudaMemcpyDeviceToHost, stream) !=
      cudaSuccess)
    return FP6_ERR_CUDA;
  if (cudaMemcpyToSymbolAsync(fp6::g_error_word, &zero, sizeof(zero), 0, cudaMemcpyHostToDevice, stream) !=
      cudaSuccess)
    return FP6_ERR_CUDA;
  if (cudaStreamSynchronize(stream) != cudaSuccess) return FP6_ERR_CUDA;
  return (word & fp6::kErrTimeout) ? FP6_ERR_TIMEOUT : FP6_OK;
}

fp6_status fp6_selftest_wait_timeout(cudaStream_t stream) {
  fp6::wait_timeout_kernel<<<1, 32, 0, stream>>>();
  return cuda_status(cudaGetLastError());
}

// ---- allocation-free variant -------------------------------------------------
// Some callers cannot allocate device memory when they run the layer: a plugin
// inside an engine that owns every byte of device memory, or a latency-bound
// loop where cudaMalloc (which may synchronize the device) is not allowed.
// fp6_linear_noalloc gives them the same layer with its scratch (split-K
// counters and partial sums) in a fixed array that lives in this library's
// device image on every GPU that loads it.
}  // extern "C"

namespace {

constexpr size_t kNoAllocScratchBytes = size_t(16) << 20;   // 16 MiB per device
static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];

// Device address of the scratch array in the current device's context.  The
// array's host-side name is only a stand-in and must never be handed to a
// kernel.  Looked up on every call (it allocates nothing and costs little), so
// a context that was destroyed and created again, in which the module and
// its array may sit elsewhere, is never given a stale address.
fp6_status noalloc_scratch(void** out) {
  void* ptr = nullptr;
  if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess || ptr == nullptr) return FP6_ERR_CUDA;
  *out = ptr;
  return FP6_OK;
}

}  // namespace

extern "C" {

fp6_status fp6_linear_noalloc(const uint16_t* x, const void* packed, const uint16_t* scales, int64_t M, int64_t N,
                              int64_t K, uint16_t* y, cudaStream_t stream) {
  fp6_status st = check_shape(N, K);
  if (st != FP6_OK) return st;
  if (M < 0) return FP6_ERR_INVALID_ARG;
  if (M == 0 || N == 0) return FP6_OK;
  const size_t need = fp6_linear_workspace_bytes(M, N, K);
  if (need > kNoAllocScratchBytes) return FP6_ERR_WORKSPACE;  // beyond the fixed scratch: use fp6_linear
  void* scratch = nullptr;
  st = noalloc_scratch(&scratch);
  if (st != FP6_OK) return st;
  if (need > 0) {
    // The array keeps the previous call's contents: the split-K counters must
    // start at zero, so clear them on the caller's stream first.
    if (cudaMemsetAsync(scratch, 0, fp6::kCounterBytes, stream) != cudaSuccess) return FP6_ERR_CUDA;
  }
  return fp6_linear(x, packed, scales, M, N, K, y, scratch, kNoAllocScratchBytes, stream);
}

}  // extern "C"
