/*
 * libhadq -- online Hadamard rotation of activations, fused with the
 * round-to-nearest quantizer that consumes them.  CUDA, sm_100a (B200).
 *
 * Operation (every entry point): each row x of a row-major [rows x n] matrix
 * becomes y = x . diag(H_b, ..., H_b) / sqrt(b), where H_b is the Sylvester
 * Hadamard matrix built by the doubling H -> [[H, H], [H, -H]] in natural
 * order ("Rotation Transform", AutoRound docs, section 1.5 "Deterministic vs
 * random Hadamard") and b is the rotation block: b = n for a full rotation,
 * or a power of 2 dividing n for the block-diagonal rotation_size / per-Linear
 * block_size modes (same page, sections 1.2 and 2.1; block 0 or n means full,
 * as block_size None / -1 does there).  The positions that apply it online --
 * R1 residual stream, R3 per-head Q/K after RoPE, R4 down_proj input -- are
 * section 1.1 of that page; the rows are "arbitrary leading dimensions, final
 * dimension = in_features" ("orbitquant 0.2.0", Quantize An Instantiated
 * Module).  H_b / sqrt(b) is symmetric and its own inverse.
 *
 * Conventions shared by all entry points
 *   - Device pointers unless the name says host.  All pointers must be
 *     16-byte aligned (HADQ_ERR_MISALIGNED otherwise).
 *   - Rows are contiguous with stride n elements.
 *   - rows == 0 is a valid empty call: nothing is launched, HADQ_OK.
 *   - Supported sizes: n a multiple of 8 and of b, with b either a power of
 *     2, 1 <= b <= 8192, or b = K * 2^m, K in {12, 20, 28, 36, 52, 60, 108},
 *     2^m >= 64, b <= 32768 (the non-power-of-2 sizes of "Rotation
 *     Transform" section 1.5: H_b = H_K (x) H_(2^m), H_K the Paley II
 *     Hadamard matrix of order K -- the page names these K but prints no
 *     matrix, so this is the construction used).  Other sizes return
 *     HADQ_ERR_UNSUPPORTED (a K * 2^m size) or HADQ_ERR_INVALID_ARG (no
 *     Hadamard matrix of that order here).
 *   - The caller owns every buffer; the library allocates nothing.
 *   - Calls are asynchronous on `stream` (a cudaStream_t; NULL = the legacy
 *     default stream).  The caller synchronizes before reading results.
 *   - All argument checks run on the host before anything is launched.  A
 *     failing call launches nothing and leaves every output untouched (the
 *     validate-then-apply rule of the apply_spinquant docstring).  There is
 *     no CPU fallback and no alternative backend.
 *   - Non-finite inputs give unspecified (but memory-safe) outputs.
 *   - hadq_last_error() gives a one-line reason for the calling thread's
 *     most recent failure.
 */
#ifndef HADQ_H
#define HADQ_H

#include <stdint.h>

#if defined(__GNUC__)
#define HADQ_API __attribute__((visibility("default")))
#else
#define HADQ_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum hadq_status {
  HADQ_OK = 0,
  HADQ_ERR_INVALID_ARG = 1,   /* null pointer, negative size, bad block/group, overlapping buffers */
  HADQ_ERR_UNSUPPORTED = 2,   /* valid by the definition but outside what the kernels cover */
  HADQ_ERR_MISALIGNED = 3,    /* a pointer is not 16-byte aligned */
  HADQ_ERR_CUDA = 4           /* the CUDA runtime reported an error at launch or copy */
} hadq_status;

typedef enum hadq_dtype {
  HADQ_F32 = 0,               /* IEEE binary32 */
  HADQ_BF16 = 1               /* bfloat16 (stored as 16-bit patterns) */
} hadq_dtype;

typedef enum hadq_fmt {
  HADQ_INT4_SYM = 0,          /* symmetric int4 RTN per group, fp16 scales */
  HADQ_INT8_SYM = 1,          /* symmetric int8 RTN per token (row), fp32 scale */
  HADQ_MXFP4 = 2,             /* E2M1 codes, E8M0 shared exponent per 32 */
  HADQ_NVFP4 = 3,             /* E2M1 codes, FP8 E4M3 scale per 16 */
  HADQ_MXFP4_BLOCKED = 4,     /* HADQ_MXFP4, scales in the tiled GEMM layout */
  HADQ_NVFP4_BLOCKED = 5      /* HADQ_NVFP4, scales in the tiled GEMM layout */
} hadq_fmt;

typedef enum hadq_sign_side {
  HADQ_SIGNS_AFTER = 0,       /* R = H_b diag(s) / sqrt(b): the random Hadamard matrix */
  HADQ_SIGNS_BEFORE = 1       /* R = diag(s) H_b / sqrt(b): its transpose and inverse */
} hadq_sign_side;

/*
 * hadq_rotate: out = x . diag(H_b) / sqrt(b), rotation only.
 *   x        [rows x n] of x_dtype (read only)
 *   out      [rows x n] of out_dtype; out == x (in place) is allowed when the
 *            dtypes match, any other overlap is HADQ_ERR_INVALID_ARG
 *   block    0 or n = full rotation, else a power of 2 dividing n
 * Values are computed in fp32 (butterfly of fp32 adds, one fp32 scaling by
 * fp32(1/sqrt(b))); bf16 output is rounded to nearest even.
 */
HADQ_API hadq_status hadq_rotate(const void* x, hadq_dtype x_dtype, int64_t rows, int64_t n, int64_t block,
                        void* out, hadq_dtype out_dtype, void* stream);

/*
 * hadq_rotate_inverse: the inverse rotation.  H_b / sqrt(b) is symmetric and
 * involutory (H H^T = b I), so this is the same operation as hadq_rotate;
 * rotating twice returns x up to fp32 rounding ("Rotation Transform",
 * introduction: R R^T = I).
 */
HADQ_API hadq_status hadq_rotate_inverse(const void* x, hadq_dtype x_dtype, int64_t rows, int64_t n, int64_t block,
                                void* out, hadq_dtype out_dtype, void* stream);

/*
 * hadq_rotate_quant: rotate, then quantize with round-to-nearest, in one pass
 * (each input byte read once, codes and scales written once).  The quantizer
 * is the RTN of "Pre-Process (Rotation Preprocessing)" (Workflow note: wbits,
 * groupsize, sym) or the MXFP4 target of "Rotation Transform" (introduction,
 * section 2.1).  With y the rotated row and m the absmax of a group:
 *
 *   HADQ_INT4_SYM  group in {32, 64, 128}, group | n.
 *                  scale s = fp16_rne(m / 7) (fp32 m / 7, then to fp16);
 *                  q = clamp(rne(y / s), -7, 7); s == 0 or inf -> q = 0.
 *                  codes:  [rows x n/2] bytes, two's-complement nibbles,
 *                          element 2i in the low nibble of byte i.
 *                  scales: [rows x n/group] fp16.
 *   HADQ_INT8_SYM  per token: group must be 0 or n; n <= 32768.
 *                  s = fp32(m / 127); q = clamp(rne(y / s), -127, 127).
 *                  codes:  [rows x n] int8.   scales: [rows] fp32.
 *   HADQ_MXFP4     group must be 0 or 32; n a multiple of 32.
 *                  e = clamp(floor(log2 m) - 2, -127, 127) (m == 0 -> -127);
 *                  code = E2M1 rne(y / 2^e), saturating at +/-6, sign bit 3.
 *                  codes:  [rows x n/2] bytes, element 2i in the low nibble.
 *                  scales: [rows x n/32] bytes = e + 127 (E8M0).
 *   HADQ_NVFP4     group must be 0 or 16; n a multiple of 16.  The pages name
 *                  the scheme and its block of 16 ("Rotation Transform",
 *                  introduction and section 2.1) but not its encoding;
 *                  reading: NVIDIA's public NVFP4 definition, single-level here
 *                  (per-tensor scale 1; see hadq_rotate_quant_nvfp4):
 *                  s = E4M3(m / 6), round half to even, saturating at 448;
 *                  code = E2M1 rne(y / s), saturating at +/-6, sign bit 3;
 *                  s == 0 -> codes 0.
 *                  codes:  [rows x n/2] bytes, element 2i in the low nibble.
 *                  scales: [rows x n/16] E4M3 bytes.
 *   HADQ_MXFP4_BLOCKED, HADQ_NVFP4_BLOCKED
 *                  the same codes and scale values, the scales written in the
 *                  layout block-scaled tensor-core GEMMs read, so the codes go
 *                  straight into a W4A4 / MXFP4 product (the consumer after
 *                  the rotation; reading: the "1D block scaling factors"
 *                  layout of NVIDIA's public cuBLAS documentation).  With C
 *                  scale columns per row (n/32 or n/16), rows padded to
 *                  R = 128 * ceil(rows / 128): 128 x 4 tiles of 512 bytes in
 *                  the order (row / 128, column / 4); inside a tile scale
 *                  (r, c) at byte (r % 32) * 16 + ((r / 32) % 4) * 4 + c % 4.
 *                  scales: R x C bytes; the entries of the padding rows are
 *                  written as 0.  Served by the tensor-core kernels: bf16
 *                  input at full size 4096 or 8192, blocks of 128 .. 2048
 *                  (unsigned above 128), and blocks of K * 2^m with
 *                  2^m >= 128 (unsigned); HADQ_ERR_UNSUPPORTED otherwise,
 *                  with RPBH, and under HADQ_IMPL_BUTTERFLY.
 *
 * Codes are computed from the fp32 rotation z (y = z / sqrt(b)) with the
 * stored scale s: the factor f = (1/sqrt(b)) / s is a correctly rounded fp32
 * quotient, and the exact product z * f is rounded once onto the integer grid
 * (int4, int8; a fused multiply-add) or onto fp32 and then to E2M1 (MXFP4,
 * NVFP4).  Scales are correctly rounded fp32 quotients m / 7, m / 127, m / 6
 * before their rounding to fp16 / E4M3.
 * codes and scales must not overlap x or each other.
 */
HADQ_API hadq_status hadq_rotate_quant(const void* x, hadq_dtype x_dtype, int64_t rows, int64_t n, int64_t block,
                              hadq_fmt fmt, int64_t group, void* codes, void* scales, void* stream);

/*
 * hadq_rotate_quant_nvfp4: HADQ_NVFP4 with its per-tensor (second-level)
 * scale t: the block scales and codes are those of y / t, so dequantization
 * is code * s * t.  t must be finite and > 0 (HADQ_ERR_INVALID_ARG
 * otherwise); t = 1 is hadq_rotate_quant with HADQ_NVFP4.  A caller that
 * uses the full E4M3 range sets t = amax(y) / (6 * 448) from a calibrated or
 * previously measured amax.  Buffers, checks and errors as hadq_rotate_quant.
 */
HADQ_API hadq_status hadq_rotate_quant_nvfp4(const void* x, hadq_dtype x_dtype, int64_t rows, int64_t n,
                                             int64_t block, float tensor_scale, void* codes, void* scales,
                                             void* stream);

/*
 * Random Hadamard ("Rotation Transform", AutoRound docs, section 1.5:
 * random_hadamard_matrix(size) = H @ diag(+/-1) / sqrt(N); section 1.2:
 * random_r1..random_r4 use it in place of the deterministic matrix; section
 * 1.7: the +/-1 signs are persisted as int8).  Every b-element block of a row
 * is multiplied by the same R:
 *   side HADQ_SIGNS_AFTER   R = H_b diag(s) / sqrt(b): output column j of the
 *                           block times s_j (the random Hadamard matrix);
 *   side HADQ_SIGNS_BEFORE  R = diag(s) H_b / sqrt(b): input column j times
 *                           s_j, then the transform -- the transpose, so
 *                           applying AFTER then BEFORE with the same signs
 *                           gives x back; it is also the order of the
 *                           Rademacher signs ahead of the block FWHT in
 *                           orbitquant's RPBH rotation ("orbitquant 0.2.0").
 *   signs   device pointer to b int8 values (b = the block, n when block is
 *           0 / -1 / n), 16-byte aligned; entry j < 0 means s_j = -1, any
 *           other value +1.  Read only; it must not overlap an output.  May be
 *           null when rows == 0.
 * Everything else (shapes, formats, alignment, errors, asynchrony) is as for
 * hadq_rotate / hadq_rotate_quant.  The quantizer sees the signed rotation,
 * so for AFTER the scales equal the unsigned ones and the codes of negated
 * columns are negated (MXFP4: sign bit flipped unless the value is exactly 0).
 */
HADQ_API hadq_status hadq_rotate_signed(const void* x, hadq_dtype x_dtype, int64_t rows, int64_t n, int64_t block,
                                        const int8_t* signs, hadq_sign_side side, void* out, hadq_dtype out_dtype,
                                        void* stream);

HADQ_API hadq_status hadq_rotate_quant_signed(const void* x, hadq_dtype x_dtype, int64_t rows, int64_t n,
                                              int64_t block, const int8_t* signs, hadq_sign_side side,
                                              hadq_fmt fmt, int64_t group, void* codes, void* scales, void* stream);

/*
 * RPBH rotation ("orbitquant 0.2.0", Method Conformance: RPBH permutation,
 * Rademacher signs, block FWHT and orthonormal scaling).  For every row,
 *     v_e = x[perm[e]] * s_e          (e = 0 .. n - 1),
 *     out = v . diag(H_b, ..., H_b) / sqrt(b),
 * i.e. the columns are gathered through the permutation, signed, and rotated
 * block by block as hadq_rotate does.
 *   perm    device pointer to n int32: a permutation of 0 .. n - 1 (the page
 *           gives no rule for choosing it; the caller supplies it).  Entries
 *           outside 0 .. n - 1 are clamped: memory-safe, result unspecified.
 *   signs   device pointer to n int8, one per column; negative = -1.
 *   block   0 / n = full, else a power of 2 dividing n, or K * 2^m as for
 *           hadq_rotate; n must be a multiple of 64 and at most 32768.
 * perm and signs are 16-byte aligned and must not overlap an output; x and
 * out may be the same buffer (equal dtypes).  Other rules as hadq_rotate /
 * hadq_rotate_quant.  hadq_rotate_quant_rpbh quantizes the RPBH rotation
 * with any hadq_fmt.
 */
HADQ_API hadq_status hadq_rotate_rpbh(const void* x, hadq_dtype x_dtype, int64_t rows, int64_t n, int64_t block,
                                      const int32_t* perm, const int8_t* signs, void* out, hadq_dtype out_dtype,
                                      void* stream);

HADQ_API hadq_status hadq_rotate_quant_rpbh(const void* x, hadq_dtype x_dtype, int64_t rows, int64_t n, int64_t block,
                                            const int32_t* perm, const int8_t* signs, hadq_fmt fmt, int64_t group,
                                            void* codes, void* scales, void* stream);

/*
 * hadq_rotate_quant_codebook: orbitquant's online activation quantizer
 * ("orbitquant 0.2.0", Method Conformance: online per-token norm, normalized
 * activation rotation, nearest-centroid quantization, rescaling).  For every
 * row, y = the rotation (RPBH when perm and signs are given, else the plain
 * block rotation of hadq_rotate), r = ||y||_2, and element e codes the index
 * of the nearest centroid of y_e / r: the number of thresholds strictly below
 * it (the thresholds are the midpoints of adjacent centroids; a value exactly
 * on one takes the lower index).  Dequantization is r * centroid[code].
 *   bits        2 or 4
 *   thresholds  device pointer to 2^bits - 1 ascending doubles, usually
 *               those hadq_codebook(n, bits) returns (the codebook for rows
 *               of length n), copied to the device by the caller
 *   codes       [rows x n * bits / 8] bytes; code i of a byte in bits
 *               [i * bits, (i + 1) * bits), element 0 lowest
 *   norms       [rows] fp32: r
 *   perm, signs both null (plain rotation) or both given (RPBH, as above)
 * n must be a multiple of 64 and at most 32768.  The norm is accumulated in
 * double and the comparison of y_e with r * t_j is exact for the fp32 y_e,
 * so a code differs from the exactly computed one only through the fp32
 * rotation's own rounding.  Buffers 16-byte aligned, no overlaps; other
 * rules as hadq_rotate_quant.
 */
HADQ_API hadq_status hadq_rotate_quant_codebook(const void* x, hadq_dtype x_dtype, int64_t rows, int64_t n,
                                                int64_t block, const int32_t* perm, const int8_t* signs, int bits,
                                                const double* thresholds, void* codes, float* norms, void* stream);

/*
 * hadq_rotate_quant_host: the same operation on HOST buffers.  Enqueues on
 * `stream`: copy x_host -> x_dev, hadq_rotate_quant on the device buffers,
 * copy codes_dev -> codes_host and scales_dev -> scales_host.  The caller
 * provides the device staging buffers (sizes as for hadq_rotate_quant) and
 * synchronizes `stream` before reading the host outputs.  Host buffers
 * should be page-locked for the copies to be asynchronous.  Argument checks
 * cover both the host and the device buffers and run before anything is
 * enqueued.
 */
HADQ_API hadq_status hadq_rotate_quant_host(const void* x_host, hadq_dtype x_dtype, int64_t rows, int64_t n, int64_t block,
                                   hadq_fmt fmt, int64_t group, void* codes_host, void* scales_host,
                                   void* x_dev, void* codes_dev, void* scales_dev, void* stream);

/*
 * hadq_rotate_quant_host_static: hadq_rotate_quant_host for callers that
 * cannot allocate device memory.  Some callers cannot call cudaMalloc at all:
 * a host-only C or Fortran application that links libhadq but manages no
 * device memory, or a plugin inside a framework whose allocator owns every
 * device byte (allocating behind its back breaks its pooling and budget).
 * This entry point allocates nothing: it stages x, codes and scales in a
 * 32 MiB array that the library itself declares as static device memory, so
 * the caller passes only host buffers (page-locked for asynchronous copies).
 * There is no counterpart on the pages: it is a deployment variant of the
 * host-buffer entry point above, with the same operation and results.
 *
 *   - Sizes: input bytes + code bytes + scale bytes, each rounded up to 256,
 *     must not exceed 32 MiB (e.g. 2048 x 4096 bf16 with int4 g128 fits);
 *     larger calls return HADQ_ERR_UNSUPPORTED and do nothing.
 *   - The static array exists once per GPU that loads the library and lives
 *     until the process exits.  The first call on a device looks up its
 *     device address (a one-time set-up per device, made with that device
 *     current); make that first call before any stream capture.
 *   - Every call on a device shares the one array.  Calls whose work overlaps
 *     on the GPU (for example on two streams without ordering between them)
 *     race on it: order them on one stream or synchronize between them.
 *     Nothing in the array has to start at zero: each call's copy fills the
 *     input region and its kernel writes every code and scale byte.
 *   - Otherwise as hadq_rotate_quant_host: enqueued on `stream`, the caller
 *     synchronizes before reading codes_host / scales_host.
 */
HADQ_API hadq_status hadq_rotate_quant_host_static(const void* x_host, hadq_dtype x_dtype, int64_t rows, int64_t n,
                                                   int64_t block, hadq_fmt fmt, int64_t group, void* codes_host,
                                                   void* scales_host, void* stream);

/*
 * hadq_codebook: the unit-sphere Lloyd-Max codebook of "orbitquant 0.2.0"
 * (Features: exact unit-sphere Lloyd-Max codebooks; Method Conformance: one
 * fixed codebook per input dimension and bit width).  A rotated, normalized
 * row behaves as a uniform unit vector in R^d; one coordinate then has the
 * density (1 - t^2)^((d - 3) / 2) on [-1, 1] (normalized), and the codebook
 * is the minimum mean-square-error quantizer of that density with 2^bits
 * levels (Lloyd's iteration, in double precision, on the host).
 *   d           the row length the codebook serves (>= 2)
 *   bits        1 .. 8
 *   centroids   host array of 2^bits doubles, ascending (written)
 *   thresholds  host array of 2^bits - 1 doubles: the midpoints of adjacent
 *               centroids, the decision boundaries (written)
 * Synchronous, no CUDA call, nothing allocated on the device.
 * HADQ_ERR_INVALID_ARG for a bad d, bits or a null pointer.
 */
HADQ_API hadq_status hadq_codebook(int64_t d, int bits, double* centroids, double* thresholds);

/* Bytes of the code and scale outputs of hadq_rotate_quant for these sizes
 * (0 for an invalid combination; the blocked formats count the padding rows). */
HADQ_API int64_t hadq_codes_bytes(int64_t rows, int64_t n, hadq_fmt fmt);
HADQ_API int64_t hadq_scales_bytes(int64_t rows, int64_t n, hadq_fmt fmt, int64_t group);

/* Static description of a status code. */
HADQ_API const char* hadq_status_string(hadq_status status);

/* One-line reason for the calling thread's most recent failed call ("" if none). */
HADQ_API const char* hadq_last_error(void);

/* Fault bits recorded by kernels whose bounded internal waits ran out (0 when
 * every wait completed; -1 if the flag could not be read).  Synchronous:
 * call after the work of interest has completed.  `clear` != 0 resets the
 * flags.  No paper counterpart: a diagnostic of this implementation. */
HADQ_API int hadq_device_faults(int clear);

/* Library version as MAJOR * 10000 + MINOR * 100 + PATCH. */
HADQ_API int hadq_version(void);

/*
 * Implementation choice.  Two implementations compute the same operation:
 * the tensor-core kernels (tcgen05 MMA with H_128 for the high index bits,
 * operands staged by TMA) and the CUDA-core butterfly kernels.  The tensor-core
 * kernels cover bf16 input at full size 4096 / 8192 and at block 128 (every
 * format and sign variant), blocks of 256 .. 2048 (block or full size; no
 * signs, no per-token int8), RPBH at full size 4096, blocks of K * 2^m with
 * 2^m >= 128 and
 * K * 2^m / 128 <= 128 chunks (no signs or permutation; rotation outputs,
 * int4, MXFP4, NVFP4, and per-token int8 when the block is the whole row);
 * every other call runs the
 * butterfly (staged) kernels whatever the choice.
 *   HADQ_IMPL_AUTO       the default: the tensor-core kernels wherever they apply
 *   HADQ_IMPL_TENSOR     the same (named for callers that want to say so)
 *   HADQ_IMPL_BUTTERFLY  the butterfly kernels everywhere
 * Results agree within the parity tolerances, not bit for bit (the two sum in
 * different orders).  hadq_set_impl is process-wide and takes effect for calls
 * made after it returns; it returns HADQ_ERR_INVALID_ARG for any other value.
 * No paper counterpart: it exists so that both implementations can be tested
 * and measured on the same shapes.
 */
typedef enum hadq_impl {
  HADQ_IMPL_AUTO = 0,
  HADQ_IMPL_BUTTERFLY = 1,
  HADQ_IMPL_TENSOR = 2
} hadq_impl;

HADQ_API hadq_status hadq_set_impl(hadq_impl impl);
HADQ_API hadq_impl hadq_get_impl(void);

#ifdef __cplusplus
}
#endif

#endif /* HADQ_H */
