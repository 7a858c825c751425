/*
 * mx.h — C ABI of libmx.so: OCP Microscaling (MX) block-32 quantization of
 * bf16 tensors on NVIDIA B200 (sm_100a).
 *
 * Sources restated (page titles; sections in brackets):
 *  [AX] "[Axolotl] MXFP4 quantization support" (PR #3375 analysis) [2: config,
 *       block_size must be 32 else ValueError; torch.float4_e2m1fn_x2 packs two
 *       E2M1 codes per byte] [3: activation and weight share one fake-quantizer].
 *  [VL] "[vLLM] MXFP8/MXFP4: microscaling format quantization" [MXFP8: block-32
 *       scaling: contiguous weight -> (fp8 elements, uint8 scales), dynamic
 *       scheme only] [MXFP4: uint8 storage, two FP4 values per byte, last dim
 *       halved] [MX format table: E4M3/E5M2, E3M2/E2M3, E2M1 and INT8
 *       elements, E8M0 scale, block 32, one scale byte per 32 elements].
 *  [UP] "Unveiling the Potential of Quantization with MXFP4: Strategies for
 *       Quantization Error Reduction" [technical summary 1: E8M0 = 2^k only]
 *       [2.A Overflow-Aware Scaling] [2.B Macro Block Scaling] [3-4: QSNR]
 *       [5: OAS and MBS generalize to MXFP6 and MXFP8].
 *  [BQ] "BATQuant: Outlier-resilient MXFP4 Quantization via Learnable
 *       Block-wise Optimization" [technical summary 2: block-wise affine
 *       transform matched to the MX block; GPK: block matrix = B_j (x) A with
 *       A shared and B_j private; block-wise learnable clipping].
 *
 * Layout (every call): x is row-major contiguous [rows, cols] bf16, cols a
 * multiple of 32 (16 for the block-16 formats); block b of row r is elements
 * [32b, 32b+32) of that row ([16b, 16b+16) for the block-16 formats).
 * A 3-D tensor [E, R, C] is passed as rows = E*R, cols = C.
 *   codes  MXFP4 (and the block-16 formats): uint8 [rows, cols/2], element 2j in the low nibble and 2j+1
 *                 in the high nibble of byte j; bit 3 of a nibble is the sign.
 *          other formats: uint8 [rows, cols], one code per element (E4M3,
 *                 E5M2, INT8: the whole byte; E3M2 / E2M3: the low 6 bits,
 *                 bit 5 the sign, bits 6-7 zero).
 *   scales uint8 [rows, cols/32], E8M0: byte s means 2^(s-127); 255 is NaN.
 *   macro  uint8 [rows, cols/128] (MBS only): k, the macro factor f = 1 + k/256
 *          of the 128-element macro block [128m, 128m+128) of the row.
 *
 * Ownership: the caller allocates and owns every buffer (device memory unless
 * stated). The library allocates nothing and keeps no state between calls.
 * Streams: every call enqueues its kernels on `stream` (a cudaStream_t passed
 * as void*; NULL = the legacy default stream) and returns without waiting.
 * Errors: arguments are checked on the host before anything is enqueued; on
 * any error nothing is launched and no output is written. A failed launch
 * returns MX_ERR_CUDA. Faults inside a kernel surface at the caller's next
 * synchronisation, as usual for CUDA. Kernels never trap or assert; the
 * streaming kernels never wait on flags, and the GEMM kernels' waits on their
 * own barriers are bounded in time (see mx_gemm). All entry points are
 * thread-safe.
 * Empty inputs (rows == 0 or cols == 0) are valid and launch nothing (except
 * that mx_block_error still zeroes its totals).
 * Alignment: x, grad_y, grad_x, y and out must be 32-byte aligned (the
 * kernels move 32 bytes per lane), codes 16-byte; block_sse 4-byte, totals
 * 8-byte; scales and macro have no requirement. (torch allocations are
 * 512-byte aligned; a view that starts mid-buffer may not be.)
 */
#ifndef MX_H_
#define MX_H_

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Element formats ([VL] MX format table: MXFP8 E4M3/E5M2, MXFP6 E3M2/E2M3,
 * MXFP4 E2M1, MXINT8 INT8; block 32 and an E8M0 scale for all), and two
 * block-16 comparison formats. emax is the exponent of the largest power of
 * two the element holds. */
typedef enum {
  MX_FMT_E2M1 = 0, /* MXFP4: magnitudes {0, .5, 1, 1.5, 2, 3, 4, 6} ([UP] 2.A: max 6.0), emax 2 */
  MX_FMT_E4M3 = 1, /* MXFP8: E4M3fn (bias 7, no Inf, S.1111.111 = NaN), max 448, emax 8 */
  MX_FMT_E5M2 = 2, /* MXFP8: E5M2 (bias 15, IEEE Inf/NaN at exponent 31), max 57344, emax 15 */
  MX_FMT_E3M2 = 3, /* MXFP6: E3M2 (bias 3, no Inf/NaN), max 28, emax 4 */
  MX_FMT_E2M3 = 4, /* MXFP6: E2M3 (bias 1, no Inf/NaN), max 7.5, emax 2 */
  MX_FMT_INT8 = 5, /* MXINT8: two's complement i read as i * 2^-6, |i| <= 127, emax 0 */
  /* The two comparison formats of [UP] 1's MXFP4/NVFP4 gap analysis: E2M1
   * elements in 16-element blocks (cols a multiple of 16; scales
   * [rows, cols/16]). */
  MX_FMT_E2M1_B16 = 6, /* MXFP4 at block 16: E8M0 scales, every base rule; MBS over the eight
                        * 16-element sub-blocks of each 128-element macro block ([UP] 2.B's
                        * 1x16 base blocks) */
  MX_FMT_NVFP4 = 7     /* E4M3 scale s = amax / 6 rounded to nearest even and saturated
                        * (no tensor-level scale), elements RNE_sat(x / s); scaling
                        * MX_SCALE_FLOOR only (the one rule); a zero scale keeps only
                        * the signs; a NaN/Inf block gets the E4M3 NaN byte 0x7F */
} mx_format_t;

/* Scale selection. Low 4 bits: the base rule; bits 4-5: Macro Block Scaling.
 * emax is the exponent of the element's largest power of two (mx_format_t)
 * and e = floor(log2 amax) of the block. Every rule clamps E to [-127, 127];
 * an all-zero block gets E = -127 (byte 0); a block holding NaN or Inf gets
 * byte 255 and element codes NaN for FP8 (S.1111.111, S.11111.11), only the
 * sign for FP4 and FP6, and 0 for INT8. */
typedef enum {
  /* OCP rule 2^(e - emax): amax lands in [2^emax, 2^(emax+1)), e.g. [4, 8)
   * for E2M1 or [256, 512) for E4M3; values above the largest element
   * saturate. Every format. */
  MX_SCALE_FLOOR = 0,
  /* [UP] 2.A's "existing" scale: the smallest 2^E with amax <= maxv * 2^E
   * (no element saturates, within the E8M0 range). Every format. */
  MX_SCALE_CEIL = 1,
  /* [UP] 2.A as a rule on the mantissa bits: under the no-overflow scale a
   * block max in (3.0, 3.5] of the 6.0 range is mapped to (6.0, 7.0] instead,
   * i.e. E = e - 2 when the amax significand is at most 1.75, else e - 1. FP4. */
  MX_SCALE_OAS_RULE = 2,
  /* Overflow-Aware Scaling as a per-block minimum-SSE choice between the
   * FLOOR exponent and FLOOR + 1 (exact comparison; a tie keeps FLOOR). The
   * float elements: FP4, and ([UP] 5: OAS generalizes to MXFP6/MXFP8) E4M3,
   * E5M2, E3M2, E2M3; not INT8. */
  MX_SCALE_OAS = 3,
  /* [UP] 2.B Macro Block Scaling, OR-able with MX_SCALE_FLOOR or MX_SCALE_OAS;
   * FP4 only; cols must be a multiple of 128. Each 128-element macro block
   * gets a factor f = 1 + k/256 (k stored in `macro`); each 32-block inside it
   * takes its exponent from floor(log2(amax / f)) and its elements are rounded
   * as x / (f * 2^E). STATIC: the smallest k that maps the macro-block max to
   * at most 6. DYNAMIC: the k in 0..255 with the smallest macro-block SSE
   * (double, summed in element order; a tie keeps the smaller k). */
  MX_MBS_STATIC = 1 << 4,
  MX_MBS_DYNAMIC = 2 << 4,
  /* Layout flag, OR-able with any of the above for mx_quantize and
   * mx_fake_quant_fwd (and in mx_dequantize's flags): the E8M0 bytes are
   * written (read) in the tiled layout that block-scaled tensor-core GEMMs
   * on sm_100 consume (the one cuBLASLt's 1-D block-scaling-factor layout
   * documents) instead of plain [rows, cols/block]. Rows are padded to 128
   * and block columns to 4; the scale of row r, block column j sits at byte
   *   ((r / 128) * T + j / 4) * 512 + (r % 32) * 16 + ((r / 32) % 4) * 4 + j % 4,
   * T = ceil(cols / (4 * block)) tiles per 128-row band. Padding bytes are zero.
   * mx_scale_bytes gives the buffer size. Macro factors keep their layout. */
  MX_SCALES_MMA = 1 << 8
} mx_scaling_t;

typedef enum {
  MX_OK = 0,
  MX_ERR_INVALID_ARG = 1, /* NULL required pointer, negative or oversized shape */
  MX_ERR_SHAPE = 2,       /* cols % 32 != 0, or cols % 128 != 0 with MBS ([AX] 2) */
  MX_ERR_ALIGN = 3,       /* a pointer below its stated alignment */
  MX_ERR_UNSUPPORTED = 4, /* unknown format/scaling, or a scaling the format lacks */
  MX_ERR_CUDA = 5,        /* a kernel launch or stream operation failed */
  MX_ERR_TOO_LARGE = 6    /* mx_quant_gemm_noalloc: the problem exceeds its fixed scratch */
} mx_status_t;

/* Quantize ([VL] MXFP8/MXFP4 sections; [UP] 2.A/2.B for the scaling modes).
 * x: device bf16 [rows, cols]. codes: device, FP4 rows*cols/2 bytes, every
 * other format rows*cols bytes (FP6 codes in the low 6 bits, bits 6-7 zero). scales: device uint8 [rows, cols/32]. macro: device uint8
 * [rows, cols/128] when scaling has an MBS bit (required then), else ignored
 * and may be NULL. Elements: round to nearest, ties to the even code, values
 * past the largest magnitude saturate, the sign is kept (small negatives -> -0). */
int mx_quantize(const void* x, int64_t rows, int64_t cols, int format, int scaling,
                void* codes, uint8_t* scales, uint8_t* macro, void* stream);

/* Bytes of the scale buffer of a [rows, cols] tensor in `format`: rows *
 * cols / block, or the padded size of the MX_SCALES_MMA layout when `scaling`
 * has that flag. -1 for an invalid format or shape. Host only. */
int64_t mx_scale_bytes(int64_t rows, int64_t cols, int format, int scaling);

/* Dequantize: out = value(code) * f * 2^(scale - 127), f = 1 + k/256 from
 * `macro` (NULL means f = 1; FP4 only). out_fp32 (flags): bit 0 clear: bf16
 * (rounded to nearest even; exact for FP4 without MBS); set: float (exact);
 * MX_SCALES_MMA: `scales` is in the tiled layout (see mx_scaling_t). A scale byte of
 * 255 or an FP8 NaN code gives the canonical NaN (0x7FC0 / 0x7FC00000); an
 * E5M2 Inf code gives +-Inf. */
int mx_dequantize(const void* codes, const uint8_t* scales, const uint8_t* macro,
                  int64_t rows, int64_t cols, int format, int out_fp32, void* out,
                  void* stream);

/* QAT fake-quantization forward ([AX] 2-3): y = dequantize(quantize(x)) as
 * bf16, in one pass. scales_out (nullable): the E8M0 bytes, as mx_quantize. */
int mx_fake_quant_fwd(const void* x, int64_t rows, int64_t cols, int format, int scaling,
                      void* y, uint8_t* scales_out, void* stream);

/* Straight-through backward of the fake-quantizer: grad_x = grad_y where
 * |x| <= maxv * X (X = f * 2^E, the scale the forward uses for that block;
 * inclusive), else +0. NaN x, and every element of a NaN/Inf block, give +0.
 * The grad_y bits pass unchanged. */
int mx_fake_quant_bwd(const void* x, const void* grad_y, int64_t rows, int64_t cols,
                      int format, int scaling, void* grad_x, void* stream);

/* Quantization error ([UP] 3-4, QSNR): d = x - y with y the exact dequantized
 * value (float, not rounded to bf16) under `scaling`. block_sse (nullable):
 * device float [rows, cols/32], the per-block sum of d^2. totals: device
 * double[2] = {sum d^2, sum x^2}; the call zeroes it on the stream first and
 * then accumulates (atomically: the last bits may vary run to run). MSE =
 * totals[0] / (rows*cols); SQNR dB = 10 log10(totals[1] / totals[0]). */
int mx_block_error(const void* x, int64_t rows, int64_t cols, int format, int scaling,
                   float* block_sse, double* totals, void* stream);

/* BATQuant apply step ([BQ] 2), alone or fused with MX quantization.
 * Each 32-element block j of every row is multiplied on the right by
 * P_j = B_j (x) A: with i = p*a + q (p < b, q < a, a*b = 32),
 *   y[r*a+s] = sum_p B_j[p][r] * Z[p][s],  Z[p][s] = sum_q x[p*a+q] * A[q][s].
 * Then, when thresholds are given and the block's 32 values are all finite,
 * each value is clipped: t = y < lo ? lo : y; y = t > hi ? hi : t, with
 * lo = beta_min[j] * min(block), hi = beta_max[j] * max(block) (fp32 products;
 * thresholds >= 0 expected, e.g. a sigmoid of the learned parameter). The
 * result is rounded to bf16 (nearest even; NaN -> 0x7FC0).
 * Arithmetic (fixed, so that results are reproducible bit for bit): fp32,
 * IEEE (no flush to zero); every sum is a chain of fused multiply-adds in
 * ascending index order starting from -0, except that a sum whose index runs
 * over both 16-element halves of the block (the sum over p when b >= 2, over
 * q when a = 32) is the fp32 sum of the lower half's chain and the upper
 * half's chain.
 *   a_dim        a, one of 1, 2, 4, 8, 16, 32 (b = 32 / a).
 *   A            device float [a, a], row-major A[q][s]; 16-byte aligned.
 *   B            device float [cols/32, b, b], row-major B_j[p][r]; 16-byte aligned.
 *   beta_min/max device float [cols/32], 4-byte aligned; both NULL = no clip
 *                (exactly one NULL is MX_ERR_INVALID_ARG).
 * mx_bat_apply writes y_bf16 [rows, cols] (32-byte aligned).
 * mx_bat_quantize writes what mx_quantize writes for that y, for the 32-element
 * formats and every scaling except MBS-Dynamic (MX_ERR_UNSUPPORTED; run
 * mx_bat_apply, then mx_quantize), MX_SCALES_MMA included. Other errors as
 * mx_quantize; a_dim not in the list or a NULL A / B is MX_ERR_INVALID_ARG. */
int mx_bat_apply(const void* x, int64_t rows, int64_t cols, int a_dim, const float* A,
                 const float* B, const float* beta_min, const float* beta_max, void* y_bf16,
                 void* stream);
int mx_bat_quantize(const void* x, int64_t rows, int64_t cols, int a_dim, const float* A,
                    const float* B, const float* beta_min, const float* beta_max, int format,
                    int scaling, void* codes, uint8_t* scales, uint8_t* macro, void* stream);

/* Block-scaled MXFP4 GEMM on the tensor cores, the consumer of the MX
 * tensors ([UP] 2.B and 4: the scale work beside the tensor-core GEMM; [VL]
 * MXFP4 MoE section: SM100 kernels consume MXFP4 operands with E8M0 scales):
 *   D[M, N] = A[M, K] . B[N, K]^T,
 * A and B MXFP4 (E2M1 elements, one E8M0 scale per 32 elements along K), the
 * products summed in fp32 by tcgen05.mma.kind::mxf4.block_scale (the
 * tensor cores' summation order is not specified; results agree with the
 * exact product within fp32 rounding and are bit-exact where every partial
 * sum is exact), D written as bf16 (nearest even) or, with out_fp32 = 1, as
 * float. Row-major everywhere:
 *   b_codes   device uint8 [N, K/2], as mx_quantize writes MXFP4 codes
 *             (16-byte aligned).
 *   b_scales  device uint8, B's scales in the MX_SCALES_MMA layout
 *             (mx_scale_bytes(N, K, MX_FMT_E2M1, MX_SCALES_MMA) bytes;
 *             16-byte aligned).
 *   d         device [M, N] bf16 or float (16-byte aligned).
 *   status    device int32 or NULL: set nonzero if one of the kernel's waits
 *             ran out (a kernel fault, not a result; the output is then
 *             undefined). Never cleared by the library.
 * Shapes: K a multiple of 256, N a multiple of 8 (MX_ERR_SHAPE); M up to
 * 8,388,480. M == 0 or N == 0 does nothing; K == 0 writes zeros.
 * mx_gemm: A pre-quantized, a_codes [M, K/2] (16-byte aligned) and a_scales
 * in the MX_SCALES_MMA layout (16-byte aligned).
 * mx_quant_gemm: A given as bf16 [M, K] (32-byte aligned) and quantized to
 * MXFP4 within the call with `scaling` (MX_SCALE_FLOOR, CEIL, OAS_RULE or
 * OAS; no MBS: its factors are not powers of two, which a block-scaled MMA
 * cannot apply), exactly as mx_quantize would quantize it. a_codes_out
 * ([M, K/2], 16-byte aligned) and a_scales_out (MX_SCALES_MMA layout,
 * 16-byte aligned, padding zeroed), each nullable, receive A's quantized
 * form. Two forms:
 *  - staged (default): one cooperative launch quantizes A into those buffers
 *    (into stream-ordered scratch for a NULL one, taken from a memory pool
 *    the library keeps per device) and runs the GEMM on them, read back
 *    mostly from L2. When the GEMM's tiles fit in one wave every warp
 *    quantizes, then a grid-wide barrier; otherwise six extra warps per CTA
 *    quantize while the GEMM runs, each 128-row band of A counted as it
 *    completes (a per-band counter in the scratch) so that its tiles start
 *    as soon as their band is ready. The scratch's stream-ordered
 *    allocation costs about 2 us of GPU time per call; small, latency-bound
 *    calls save it by passing both buffers.
 *  - out_fp32 | MX_GEMM_A_ON_CHIP: A is quantized inside the GEMM's prologue
 *    and the GEMM never reads it from memory; a thread-block cluster of up
 *    to 4 CTAs shares each quantized tile through distributed shared memory.
 * Other errors as mx_quantize. */
enum { MX_GEMM_A_ON_CHIP = 1 << 9 /* OR-ed into mx_quant_gemm's out_fp32 */ };
int mx_gemm(const void* a_codes, const uint8_t* a_scales, const void* b_codes,
            const uint8_t* b_scales, int64_t M, int64_t N, int64_t K, int out_fp32, void* d,
            int* status, void* stream);
int mx_quant_gemm(const void* a_bf16, int scaling, const void* b_codes, const uint8_t* b_scales,
                  int64_t M, int64_t N, int64_t K, int out_fp32, void* d, void* a_codes_out,
                  uint8_t* a_scales_out, int* status, void* stream);

/* mx_quant_gemm without allocation. The paper has no counterpart: this entry
 * point serves callers that may not allocate device memory while they run,
 * such as a serving process that reserves all its device memory at start-up
 * and keeps it fixed, or a runtime without stream-ordered memory pools. The
 * default mx_quant_gemm takes A's quantized form and its per-band counters
 * from a pool; this one takes them from one array of
 * MX_NOALLOC_SCRATCH_BYTES in the library's device memory, which every GPU
 * that loads the library holds until the process exits. Same arguments,
 * result and errors as mx_quant_gemm in its default (staged) form, without
 * A's output buffers or the on-chip flag (out_fp32 is 0 or 1), and
 *  - MX_ERR_TOO_LARGE unless the scratch fits:
 *      M K / 2 (codes, rounded up to 256) + ceil(M / 128) K * 4 (tiled
 *      scales, rounded up to 256) + 8 ceil(M / 128) (counters)
 *      <= MX_NOALLOC_SCRATCH_BYTES;
 *    e.g. 4096 x 3072 fits, 8192 x 8192 does not.
 *  - The first call on a device looks up the array's device address
 *    (cudaGetSymbolAddress) with that device current; make it before any
 *    stream capture.
 *  - Every call shares the array and leaves its bytes there; each call
 *    clears, on its stream, the parts that must start at zero. Calls that
 *    overlap on the GPU (other streams, other host threads) race on it and
 *    give wrong results: order them on one stream or with events. */
#define MX_NOALLOC_SCRATCH_BYTES (9u << 20)
int mx_quant_gemm_noalloc(const void* a_bf16, int scaling, const void* b_codes,
                          const uint8_t* b_scales, int64_t M, int64_t N, int64_t K, int out_fp32,
                          void* d, int* status, void* stream);

/* Static description of a status code (never NULL). */
const char* mx_status_string(int status);

/* Library ABI version, (major << 16) | minor. */
int mx_version(void);

#ifdef __cplusplus
}
#endif

#endif /* MX_H_ */
