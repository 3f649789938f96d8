/*
 * fp6.h -- C ABI of libfp6.so: FP6 (e3m2) x FP16 weight-only linear layer on
 * NVIDIA B200 (sm_100a).
 *
 * The method (FP6-LLM abstract; TC-FPx article, section "kernel solution
 * redesign"): weights are quantized offline to 6-bit floats, pre-packed into
 * aligned 32-bit words (three of every four codes whole in the low six bits
 * of a byte, the fourth cut into 2-bit pieces kept in the bytes' top bits;
 * see fp6_prepack), and at run time a single kernel rebuilds FP16 weights in
 * registers and multiplies them with FP16 activations on tensor cores.
 *
 * Format.  A code is the low 6 bits of a byte: sign (bit 5), exponent e (bits
 * 4..2, bias 3), mantissa m (bits 1..0).  Value: (-1)^s 2^(e-3) (1 + m/4) for
 * e > 0, (-1)^s 2^-2 (m/4) for e = 0.  No inf/NaN; largest magnitude 28.
 * One FP16 scale per output row n:  W[n,k] ~= scale[n] * decode(code[n,k]).
 *
 * Conventions for every entry point.
 *  - Pointers are DEVICE pointers owned by the caller; the library never
 *    allocates or frees device memory.  Matrices are row-major and dense.
 *  - Every pointer must be 16-byte aligned (else FP6_ERR_MISALIGNED).
 *  - Shapes: N % 128 == 0 and K % 64 == 0 (else FP6_ERR_UNSUPPORTED_SHAPE);
 *    sizes are non-negative (else FP6_ERR_INVALID_ARG).  A zero-sized problem
 *    is a no-op that returns FP6_OK (fp6_linear with K == 0 writes y = 0).
 *  - Work is enqueued on `stream` (a cudaStream_t; NULL = legacy default
 *    stream) and runs asynchronously, except where a function says it
 *    synchronizes.  Argument errors are returned before anything is enqueued.
 *    A failed launch returns FP6_ERR_CUDA.
 *  - fp16 values are passed as their 16-bit patterns (uint16_t).
 */
#ifndef FP6_H_
#define FP6_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

struct CUstream_st; /* cudaStream_t is `struct CUstream_st *` */

typedef enum {
    FP6_OK = 0,
    FP6_ERR_INVALID_ARG = 1,       /* null pointer, negative size, bad buffer size */
    FP6_ERR_UNSUPPORTED_SHAPE = 2, /* N % 128 != 0 or K % 64 != 0, or too large */
    FP6_ERR_MISALIGNED = 3,        /* a pointer is not 16-byte aligned */
    FP6_ERR_NONFINITE = 4,         /* fp6_quantize met a NaN or infinite weight */
    FP6_ERR_SCALE_RANGE = 5,       /* fp6_quantize: max|w|/28 overflows or underflows fp16 */
    FP6_ERR_WORKSPACE = 6,         /* workspace missing or smaller than required */
    FP6_ERR_LAYOUT_VERSION = 7,    /* a stored packed blob's header does not match this library's layout */
    FP6_ERR_CUDA = 8,              /* a CUDA runtime call or launch failed */
    FP6_ERR_TIMEOUT = 9            /* a kernel's bounded wait ran out (see fp6_get_device_status) */
} fp6_status;

/* Human-readable name of a status code (static string, never NULL). */
const char *fp6_status_string(fp6_status status);

/* Bytes of the packed weight buffer for an N x K matrix: exactly 3*N*K/4
 * (six bits per weight, no header).  Returns 0 for unsupported shapes. */
size_t fp6_packed_bytes(int64_t N, int64_t K);

/*
 * fp6_quantize -- offline FP6 quantization (FP6-LLM abstract: weights are
 * quantized to 6-bit floats).  Per row n:
 *     scale[n]  = fp16_rne( fp32( max_k |W[n,k]| / 28 ) )
 *     code[n,k] = nearest e3m2 value to W[n,k] / scale[n], ties to even
 *                 mantissa, saturating at +-28, sign bit copied from W
 * A row of zeros gets scale 0 and codes 0.
 *   W       [N,K] fp32, device, read-only
 *   codes   [N,K] uint8, device, written (one code per byte, bits 7..6 zero)
 *   scales  [N]   fp16 bit patterns, device, written
 * SYNCHRONIZES the stream to report FP6_ERR_NONFINITE (a NaN/inf weight) or
 * FP6_ERR_SCALE_RANGE (a scale that overflows or underflows fp16); on those
 * errors the outputs are unspecified.  Any N >= 0, K >= 0 is accepted.
 */
fp6_status fp6_quantize(const float *W, int64_t N, int64_t K,
                        uint8_t *codes, uint16_t *scales, struct CUstream_st *stream);

/*
 * fp6_prepack -- bit-level pre-packing (TC-FPx article: weights reorganised
 * before inference, each 6-bit weight cut into pieces stored in aligned
 * 32-bit words, fragments reordered so that the run-time rebuild is
 * parallel).  Layout version 2, cut for the sm_100a instruction that converts
 * two byte-held e3m2 codes (low six bits of each byte) to two fp16 values:
 *   tiles of 128 rows x 64 columns, tile (nt, kt) at byte (nt*(K/64)+kt)*6144;
 *   inside a tile, row r owns 12 words F_w at byte (w/4)*2048 + r*16 + (w%4)*4.
 *   Tile column kk is position i = kk%16 of group g = kk/16 (words F_{3g..3g+2}):
 *   i < 12: the whole code in bits 8b..8b+5 of F_{3g+i/4}, b = i%4;
 *   i >= 12: b = i-12, code bits 2j and 2j+1 (j = 0,1,2) in bits 8b+6 and
 *   8b+7 of F_{3g+j}.  Words are little-endian.
 *   codes   [N,K] uint8, device (bits 7..6 ignored)
 *   packed  device buffer of packed_bytes >= fp6_packed_bytes(N,K), written
 */
fp6_status fp6_prepack(const uint8_t *codes, int64_t N, int64_t K,
                       void *packed, size_t packed_bytes, struct CUstream_st *stream);

/*
 * fp6_dequant -- rebuild fp16 weights from packed codes (the "disguise FP6 as
 * FP16" step of the TC-FPx article, run on its own; used for testing and for
 * the separate dequant + GEMM comparison).
 *   scales == NULL:  W16[n,k] = fp16(decode(code))            (exact)
 *   scales != NULL:  W16[n,k] = fp16_rne(decode(code) * scale[n])
 *   W16 [N,K] fp16 bit patterns, device, written
 */
fp6_status fp6_dequant(const void *packed, const uint16_t *scales, int64_t N, int64_t K,
                       uint16_t *W16, struct CUstream_st *stream);

/* Bytes of workspace fp6_linear needs for this problem on the current device
 * (0 when the problem is empty or unsupported).  The first 16384 bytes of a
 * workspace hold counters that must be ZERO before its first use (cudaMemset
 * once); every completed call leaves them zero again, whatever the problem
 * size, so one zeroed buffer of the largest size needed serves every shape.
 * After a call that reported FP6_ERR_TIMEOUT, zero them again. */
size_t fp6_linear_workspace_bytes(int64_t M, int64_t N, int64_t K);

/*
 * fp6_linear -- y[M,N] = x[M,K] . (scale (.) decode(W))^T, fp32 accumulation,
 * fp16 output (round to nearest even).  FP6-LLM abstract (W6A16 inference);
 * TC-FPx article (dequantization fused with the tensor-core product, software
 * pipeline overlapping the two).
 *   x        [M,K] fp16 bit patterns, device, read-only
 *   packed   output of fp6_prepack for the [N,K] weight, device, read-only
 *   scales   [N] fp16 bit patterns, device, read-only
 *   y        [M,N] fp16 bit patterns, device, written
 *   workspace  device buffer of at least fp6_linear_workspace_bytes(M,N,K)
 *              bytes (zeroed once before first use, see above); may be NULL
 *              only when that size is 0
 * Concurrent calls must not share a workspace.  Deterministic: the same
 * inputs give the same bits on every run.  No block of the kernel waits on
 * another, so the call completes however many of its blocks run at once
 * (other streams' kernels, an MPS limit or a green context may hold SMs).
 * Launch: programmatic dependent launch.  The kernel may start before the
 * previous kernel in the stream has finished and begins streaming `packed`
 * then; x, scales and every output are touched only after that kernel has
 * completed.  A previous kernel that does not signal early completion (all
 * other entry points of this library and ordinary kernels) delays the start
 * until it has finished, so it may write `packed`; a kernel that does signal
 * early completion must not be the one that writes `packed` just before.
 */
fp6_status fp6_linear(const uint16_t *x, const void *packed, const uint16_t *scales,
                      int64_t M, int64_t N, int64_t K, uint16_t *y,
                      void *workspace, size_t workspace_bytes, struct CUstream_st *stream);

/* Reads and clears the device error word that kernels set when a bounded wait
 * runs out (returns FP6_ERR_TIMEOUT then, else FP6_OK).  Synchronizes `stream`. */
fp6_status fp6_get_device_status(struct CUstream_st *stream);

/*
 * fp6_selftest_wait_timeout -- failure-detection self-test; the FP6-LLM pages
 * have no counterpart.  Enqueues a one-warp kernel that waits on an mbarrier
 * nothing ever arrives on, through the same bounded wait the linear kernels
 * use.  The wait gives up after its limit (about 2 s), sets the device error
 * word and the kernel exits: the next fp6_get_device_status on the stream
 * returns FP6_ERR_TIMEOUT (and clears the word), and the context stays usable.
 * Returns FP6_ERR_CUDA if the launch fails, else FP6_OK.
 */
fp6_status fp6_selftest_wait_timeout(struct CUstream_st *stream);

/*
 * fp6_linear_noalloc -- fp6_linear for callers that cannot allocate device
 * memory while the layer runs (for example a plugin inside an engine that owns
 * all device memory, or a latency-critical loop where cudaMalloc, which may
 * synchronize the device, is not allowed).  The FP6-LLM pages have no
 * counterpart: this is a convenience of this library.
 *   Same arguments and result as fp6_linear, without the workspace: the
 *   scratch lives in a fixed 16 MiB array inside the library's device image,
 *   present on every GPU that loads the library until the process exits.
 *   A problem whose fp6_linear_workspace_bytes exceed 16 MiB returns
 *   FP6_ERR_WORKSPACE; use fp6_linear for it.  The workspace grows with the
 *   token tile and the SM count, not with N or K: on a 148-SM B200 every
 *   M <= 64 fits and every M > 64 with at least 148 pipeline steps (for
 *   example any Llama-70B- or OPT-30B-sized layer) does not.
 *   Each call looks up the array's device address in the current context
 *   (cudaGetSymbolAddress, which allocates nothing); the first call on a
 *   device may load the library's device code, so make it before capturing a
 *   stream.  Each call clears the counters it needs with cudaMemsetAsync on
 *   `stream`; it never allocates or frees.
 *   All calls on a device share the one array: calls that may overlap on the
 *   GPU (different streams without ordering between them) race and give wrong
 *   results.
 */
fp6_status fp6_linear_noalloc(const uint16_t *x, const void *packed, const uint16_t *scales,
                              int64_t M, int64_t N, int64_t K, uint16_t *y, struct CUstream_st *stream);

/* Launch configuration fp6_linear would use (for tests and benchmarks):
 * out[0] = MMA N-tile (tokens per tile), out[1] = weight pipeline stages,
 * out[2] = persistent CTAs, out[3] = number of (token, row) tiles,
 * out[4] = pipeline steps in total (a step is one to four 64-column tiles).
 * Returns FP6_OK or an argument error. */
fp6_status fp6_linear_plan(int64_t M, int64_t N, int64_t K, int64_t out[5]);

/* The same plan for a device with `sms` multiprocessors, computed on the host
 * alone (no CUDA call; for tests and capacity planning):
 * out[0..4] as fp6_linear_plan, out[5] = 64-column tiles per step (T),
 * out[6] = 1 when the wave-schedule kernel (whole tiles per CTA) runs, else 0.
 * Returns FP6_OK or an argument error (sms <= 0 is FP6_ERR_INVALID_ARG). */
fp6_status fp6_linear_plan_for_sms(int64_t M, int64_t N, int64_t K, int sms, int64_t out[7]);

/*
 * Other float formats -- the FP6-LLM pages present the design as one for
 * float weights of several bit widths (TC-FPx: "x" bits); these entry points
 * run the same pipeline for two more formats, with the same conventions,
 * status codes, workspace (fp6_linear_workspace_bytes) and launch rules as
 * the fp6_* functions.  Each has one FP16 scale per row,
 *     scale[n] = fp16_rne( fp32( max_k |W[n,k]| / largest ) ),
 * codes rounded to nearest with ties to even mantissa and saturating.
 *   FPX_E3M2  the FP6 e3m2 format above (fpx_* with it = the fp6_* calls).
 *   FPX_E2M3  FP6: sign bit 5, exponent bits 4..3 (bias 1), mantissa bits
 *             2..0; value (-1)^s 2^(e-1) (1 + m/8), or (-1)^s m/8 for e = 0;
 *             largest 7.5.  Packed exactly like e3m2 (layout version 2).
 *   FPX_E2M1  FP4: sign bit 3, exponent bits 2..1 (bias 1), mantissa bit 0;
 *             value (-1)^s 2^(e-1) (1 + m/2), or (-1)^s m/2 for e = 0;
 *             largest 6.  Packed N*K/2 bytes: tiles of 128 rows x 64
 *             columns, tile (nt, kt) at byte (nt*(K/64)+kt)*4096; inside a
 *             tile row r owns 8 words F_w at byte (w/4)*2048 + r*16 +
 *             (w%4)*4, and column kk is the 4-bit field at bits
 *             4*(kk%8) .. 4*(kk%8)+3 of F_{kk/8} (little-endian words: byte
 *             (kk%8)/2 of the word, low nibble for even kk).
 *   FPX_E2M2  FP5: sign bit 4, exponent bits 3..2 (bias 1), mantissa bits
 *             1..0; value (-1)^s 2^(e-1) (1 + m/4), or (-1)^s m/4 for e = 0;
 *             largest 7.  Packed 5*N*K/8 bytes, each code cut into a 4-bit
 *             and a 1-bit piece: tiles of 128 rows x 64 columns, tile
 *             (nt, kt) at byte (nt*(K/64)+kt)*5120; inside a tile row r owns
 *             8 words P_w of 4-bit pieces at byte (w/4)*2048 + r*16 + (w%4)*4
 *             and 2 words Q_q of 1-bit pieces at byte 4096 + r*8 + q*4.
 *             Column kk is position i = kk%32 of half q = kk/32; with
 *             v = i/8, h = (i%8)/4, b = i%4, the code's top four bits are
 *             bits 8b+4h .. 8b+4h+3 of P_{4q+v} and its lowest bit is bit
 *             8b+2v+h of Q_q.
 * Codes in the [N,K] code buffers are one per byte (unused high bits zero on
 * output, ignored on input).  An unknown fmt returns FP6_ERR_INVALID_ARG
 * (fpx_packed_bytes returns 0).
 */
typedef enum { FPX_E3M2 = 0, FPX_E2M3 = 1, FPX_E2M1 = 2, FPX_E2M2 = 3,
               FPX_S24 = 4 /* the 2:4 sparse INT4 format: header functions only (compute via s24_*) */
} fpx_format;

size_t fpx_packed_bytes(fpx_format fmt, int64_t N, int64_t K);
fp6_status fpx_quantize(fpx_format fmt, const float *W, int64_t N, int64_t K,
                        uint8_t *codes, uint16_t *scales, struct CUstream_st *stream);
fp6_status fpx_prepack(fpx_format fmt, const uint8_t *codes, int64_t N, int64_t K,
                       void *packed, size_t packed_bytes, struct CUstream_st *stream);
fp6_status fpx_dequant(fpx_format fmt, const void *packed, const uint16_t *scales, int64_t N, int64_t K,
                       uint16_t *W16, struct CUstream_st *stream);
fp6_status fpx_linear(fpx_format fmt, const uint16_t *x, const void *packed, const uint16_t *scales,
                      int64_t M, int64_t N, int64_t K, uint16_t *y,
                      void *workspace, size_t workspace_bytes, struct CUstream_st *stream);

/*
 * 2:4 structured-sparse INT4 weights (NEXT-4; the Sparse-Marlin post: 4-bit
 * weights with 2:4 sparsity, metadata giving the kept positions, per-row
 * quantization statistics).  The post fixes none of the details; these
 * entry points take the plain readings:
 *   pruning  in each group of 4 consecutive weights of a row (k = 4j..4j+3)
 *            the two with the largest |w| are kept, ties to the lower position;
 *   scale    scale[n] = fp16_rne( fp32( max_k |W[n,k]| / 7 ) );
 *   codes    q = round-half-even(w / scale) clamped to [-8, 7];
 *   value    scale * q at the kept positions, 0 elsewhere.
 * Same conventions, status codes, workspace (fp6_linear_workspace_bytes) and
 * launch rules as the fp6_* functions.  The layer runs through the same fused
 * kernels, whose rebuild expands each group's two codes to four fp16 values.
 */

/* 3*N*K/8 bytes (two 4-bit codes and two 2-bit positions per four weights);
 * 0 for unsupported shapes. */
size_t s24_packed_bytes(int64_t N, int64_t K);

/* W [N,K] fp32 (K % 4 == 0, else FP6_ERR_UNSUPPORTED_SHAPE) ->
 *   q      [N,K/2] int8, device: the two kept codes of each group, in position order
 *   pos    [N,K/2] uint8, device: their positions 0..3 within the group (pos[2j] < pos[2j+1])
 *   scales [N] fp16 bit patterns, device
 * SYNCHRONIZES the stream to report FP6_ERR_NONFINITE or FP6_ERR_SCALE_RANGE,
 * as fp6_quantize.  A row of zeros gets scale 0, codes 0 and positions 0, 1. */
fp6_status s24_quantize(const float *W, int64_t N, int64_t K, int8_t *q, uint8_t *pos,
                        uint16_t *scales, struct CUstream_st *stream);

/* q, pos as produced by s24_quantize -> packed, s24_packed_bytes(N,K) bytes:
 *   tiles of 128 rows x 64 columns, tile (nt, kt) at byte (nt*(K/64)+kt)*3072;
 *   row r of a tile owns four code words V_w at byte r*16 + 4w and two
 *   position words P_h at byte 2048 + r*8 + 4h.  Group j (0..15) of the tile
 *   row keeps its codes in byte j%4 of V_{j/4} (first code in the low nibble,
 *   4-bit two's complement) and its positions in bits 4(j%8)..4(j%8)+3 of
 *   P_{j/8} (i0 in the low two bits, i1 in the next two).  Little-endian. */
fp6_status s24_prepack(const int8_t *q, const uint8_t *pos, int64_t N, int64_t K,
                       void *packed, size_t packed_bytes, struct CUstream_st *stream);

/* Dense fp16 weights: fp16(q) at the kept positions without scales,
 * fp16_rne(scale * q) with them; +0 at the pruned positions. */
fp6_status s24_dequant(const void *packed, const uint16_t *scales, int64_t N, int64_t K,
                       uint16_t *W16, struct CUstream_st *stream);

/* y[M,N] = x[M,K] . (scale (.) v)^T with v the dense code values, fp32
 * accumulation, fp16 output; arguments and workspace as fp6_linear. */
fp6_status s24_linear(const uint16_t *x, const void *packed, const uint16_t *scales,
                      int64_t M, int64_t N, int64_t K, uint16_t *y,
                      void *workspace, size_t workspace_bytes, struct CUstream_st *stream);

/*
 * Stored packed weights.  The TC-FPx article's weights are pre-packed once,
 * before inference, so a packed buffer is typically written to disk and read
 * back by a later process, perhaps of another version of this library.  The
 * device buffers the kernels read carry no header (their layout is fixed by
 * the entry points above); a stored blob is the 64-byte header below, then
 * the fp16 scales (2*N bytes), then the packed bytes.  The header records
 * what the bytes are, so a blob packed under another layout is rejected
 * instead of being decoded wrongly.
 *
 * Header (little-endian; FP6_PACKED_HEADER_BYTES = 64):
 *   bytes  0.. 3  magic "FP6W"
 *   bytes  4.. 7  uint32 layout version of the format (FP6_LAYOUT_VERSION_*)
 *   bytes  8..11  uint32 format (fpx_format, FPX_S24 for the 2:4 format)
 *   bytes 12..15  uint32 header bytes (64)
 *   bytes 16..23  int64 N          bytes 24..31  int64 K
 *   bytes 32..35  uint32 tile rows (128)     bytes 36..39  uint32 tile columns (64)
 *   bytes 40..43  uint32 bytes per packed tile
 *   bytes 44..47  uint32 bytes per row scale (2: fp16)
 *   bytes 48..55  uint64 packed bytes (fpx_packed_bytes / s24_packed_bytes)
 *   bytes 56..63  zero
 */
#define FP6_PACKED_HEADER_BYTES 64
#define FP6_LAYOUT_VERSION_E3M2 2   /* also FPX_E2M3: whole codes in byte containers, cut codes in top bits */
#define FP6_LAYOUT_VERSION_E2M1 1
#define FP6_LAYOUT_VERSION_E2M2 1
#define FP6_LAYOUT_VERSION_S24 1

/* Writes the header of an N x K weight in format fmt into `header` (HOST
 * memory, FP6_PACKED_HEADER_BYTES bytes).  FP6_ERR_INVALID_ARG for a NULL
 * header or an unknown format, FP6_ERR_UNSUPPORTED_SHAPE for a shape the
 * format cannot pack.  No CUDA call. */
fp6_status fp6_packed_header(fpx_format fmt, int64_t N, int64_t K, void *header);

/* Checks a stored header (HOST memory) against what this library would write
 * for (fmt, N, K): FP6_OK if it matches in every field; FP6_ERR_LAYOUT_VERSION
 * if the magic, the header size, the layout version, the format, the shape,
 * the tile geometry or the payload size differ; FP6_ERR_INVALID_ARG for a NULL
 * header or an unknown format.  No CUDA call. */
fp6_status fp6_packed_header_check(const void *header, fpx_format fmt, int64_t N, int64_t K);

#ifdef __cplusplus
}
#endif

#endif /* FP6_H_ */
