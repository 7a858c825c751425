// C entry points of libmx.so (declared in include/mx.h): argument checks on
// the host, then one launch on the caller's stream. Nothing is allocated and
// no state is kept between calls.
//
// The checks restate the sources' interface: block size 32 or an error
// ("[Axolotl] MXFP4 quantization support", 2: a ValueError unless the block
// size is 32), contiguous row-major input with the block along the last
// dimension ("[vLLM] MXFP8/MXFP4", MXFP8 block-32 scaling), dynamic scaling
// only (scales always come from the live tensor; there is no static-scale
// argument), packed FP4 with the last dimension halved ("[vLLM]", MXFP4).

#include <cstdint>

#include "mx.h"
#include "mx_launch.h"

namespace {

// Largest element count accepted: keeps every byte offset far inside int64.
constexpr int64_t kMaxElems = int64_t(1) << 40;

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// Elements per scale: 16 for the block-16 formats, else 32.
int block_of(int format) { return (format == MX_FMT_E2M1_B16 || format == MX_FMT_NVFP4) ? 16 : 32; }

int check_shape(int64_t rows, int64_t cols, bool mbs, int block = 32) {
  if (rows < 0 || cols < 0) return MX_ERR_INVALID_ARG;
  if (cols % block != 0) return MX_ERR_SHAPE;
  if (mbs && cols % 128 != 0) return MX_ERR_SHAPE;
  if (rows > 0 && cols > 0 && rows > kMaxElems / cols) return MX_ERR_INVALID_ARG;
  return MX_OK;
}

// Format and scaling combinations the kernels implement.
bool known_format(int format) { return format >= MX_FMT_E2M1 && format <= MX_FMT_NVFP4; }

int check_mode(int format, int scaling) {
  if (!known_format(format)) return MX_ERR_UNSUPPORTED;
  if (scaling < 0 || (scaling & ~0x3F) != 0) return MX_ERR_UNSUPPORTED;
  const int rule = scaling & 0xF;
  const int mbs = scaling >> 4;
  if (rule > MX_SCALE_OAS || mbs > 2) return MX_ERR_UNSUPPORTED;
  if (format == MX_FMT_NVFP4) return scaling == MX_SCALE_FLOOR ? MX_OK : MX_ERR_UNSUPPORTED;
  if (format == MX_FMT_E2M1_B16)   // MBS as for MXFP4: over FLOOR or OAS
    return (mbs == 0 || rule == MX_SCALE_FLOOR || rule == MX_SCALE_OAS) ? MX_OK : MX_ERR_UNSUPPORTED;
  if (format != MX_FMT_E2M1) {
    // one-byte formats: FLOOR, CEIL, and OAS for the float elements
    if (mbs != 0 || rule == MX_SCALE_OAS_RULE) return MX_ERR_UNSUPPORTED;
    if (format == MX_FMT_INT8 && rule == MX_SCALE_OAS) return MX_ERR_UNSUPPORTED;
  }
  if (mbs != 0 && rule != MX_SCALE_FLOOR && rule != MX_SCALE_OAS) return MX_ERR_UNSUPPORTED;
  return MX_OK;
}

int from_cuda(cudaError_t e) { return e == cudaSuccess ? MX_OK : MX_ERR_CUDA; }

// The scale map of a call; flags holds MX_SCALES_MMA or not.
mxk::ScaleMap scale_map(int64_t cols, int flags, int block) {
  mxk::ScaleMap m{0, 0, 0.0};
  if (flags & MX_SCALES_MMA) {
    m.bpr = cols / block;
    m.nct = (m.bpr + 3) / 4;
    m.inv = 1.0 / static_cast<double>(m.bpr);
  }
  return m;
}

int64_t scale_bytes(int64_t rows, int64_t cols, int flags, int block) {
  if (!(flags & MX_SCALES_MMA)) return rows * (cols / block);
  return (rows + 127) / 128 * 128 * ((cols / block + 3) / 4 * 4);
}

// The tiled layout pads rows to 128 and block columns to 4; the padding must
// read as zero bytes, so it is cleared on the stream before the kernel writes
// the real scales.
cudaError_t clear_padding(uint8_t* scales, int64_t rows, int64_t cols, int flags, int block,
                          cudaStream_t st) {
  if (!(flags & MX_SCALES_MMA) || !scales) return cudaSuccess;
  if (rows % 128 == 0 && (cols / block) % 4 == 0) return cudaSuccess;
  return cudaMemsetAsync(scales, 0, static_cast<size_t>(scale_bytes(rows, cols, flags, block)), st);
}

}  // namespace

extern "C" {

int mx_version(void) { return (1 << 16) | 0; }

const char* mx_status_string(int status) {
  switch (status) {
    case MX_OK: return "ok";
    case MX_ERR_INVALID_ARG: return "invalid argument (null pointer or bad shape)";
    case MX_ERR_SHAPE: return "cols must be a multiple of 32 (of 128 with macro block scaling)";
    case MX_ERR_ALIGN: return "pointer is not aligned as required";
    case MX_ERR_UNSUPPORTED: return "unsupported format / scaling combination";
    case MX_ERR_CUDA: return "CUDA launch or stream operation failed";
    case MX_ERR_TOO_LARGE: return "problem larger than the fixed scratch of the no-allocation entry point";
    default: return "unknown status";
  }
}

int64_t mx_scale_bytes(int64_t rows, int64_t cols, int format, int scaling) {
  if (!known_format(format)) return -1;
  const int block = block_of(format);
  if (rows < 0 || cols < 0 || cols % block != 0) return -1;
  if (rows > 0 && cols > 0 && rows > kMaxElems / cols) return -1;
  return scale_bytes(rows, cols, scaling & MX_SCALES_MMA, block);
}

int mx_quantize(const void* x, int64_t rows, int64_t cols, int format, int scaling, void* codes,
                uint8_t* scales, uint8_t* macro, void* stream) {
  const int layout = scaling & MX_SCALES_MMA;
  scaling &= ~MX_SCALES_MMA;
  int st = check_mode(format, scaling);
  if (st != MX_OK) return st;
  const bool mbs = (scaling >> 4) != 0;
  st = check_shape(rows, cols, mbs, block_of(format));
  if (st != MX_OK) return st;
  const int64_t n = rows * cols;
  if (n == 0) return MX_OK;
  if (!x || !codes || !scales || (mbs && !macro)) return MX_ERR_INVALID_ARG;
  if (!aligned(x, 32) || !aligned(codes, 16)) return MX_ERR_ALIGN;
  const auto cs = static_cast<cudaStream_t>(stream);
  if (clear_padding(scales, rows, cols, layout, block_of(format), cs) != cudaSuccess) return MX_ERR_CUDA;
  return from_cuda(mxk::launch_quantize(x, n, format, scaling, codes, scales, mbs ? macro : nullptr,
                                        scale_map(cols, layout, block_of(format)), cs));
}

int mx_dequantize(const void* codes, const uint8_t* scales, const uint8_t* macro, int64_t rows,
                  int64_t cols, int format, int out_fp32, void* out, void* stream) {
  if (!known_format(format)) return MX_ERR_UNSUPPORTED;
  if (format != MX_FMT_E2M1 && format != MX_FMT_E2M1_B16 && macro) return MX_ERR_UNSUPPORTED;
  if ((out_fp32 & ~(1 | MX_SCALES_MMA)) != 0) return MX_ERR_INVALID_ARG;
  const int layout = out_fp32 & MX_SCALES_MMA;
  out_fp32 &= 1;
  int st = check_shape(rows, cols, macro != nullptr, block_of(format));
  if (st != MX_OK) return st;
  const int64_t n = rows * cols;
  if (n == 0) return MX_OK;
  if (!codes || !scales || !out) return MX_ERR_INVALID_ARG;
  if (!aligned(codes, 16) || !aligned(out, 32)) return MX_ERR_ALIGN;
  return from_cuda(mxk::launch_dequantize(codes, scales, macro, n, format, out_fp32, out,
                                          scale_map(cols, layout, block_of(format)),
                                          static_cast<cudaStream_t>(stream)));
}

int mx_fake_quant_fwd(const void* x, int64_t rows, int64_t cols, int format, int scaling, void* y,
                      uint8_t* scales_out, void* stream) {
  const int layout = scaling & MX_SCALES_MMA;
  scaling &= ~MX_SCALES_MMA;
  int st = check_mode(format, scaling);
  if (st != MX_OK) return st;
  st = check_shape(rows, cols, (scaling >> 4) != 0, block_of(format));
  if (st != MX_OK) return st;
  const int64_t n = rows * cols;
  if (n == 0) return MX_OK;
  if (!x || !y) return MX_ERR_INVALID_ARG;
  if (!aligned(x, 32) || !aligned(y, 32)) return MX_ERR_ALIGN;
  const auto cs = static_cast<cudaStream_t>(stream);
  if (clear_padding(scales_out, rows, cols, layout, block_of(format), cs) != cudaSuccess) return MX_ERR_CUDA;
  return from_cuda(mxk::launch_fake_fwd(x, n, format, scaling, y, scales_out,
                                        scale_map(cols, layout, block_of(format)), cs));
}

int mx_fake_quant_bwd(const void* x, const void* grad_y, int64_t rows, int64_t cols, int format,
                      int scaling, void* grad_x, void* stream) {
  int st = check_mode(format, scaling);
  if (st != MX_OK) return st;
  st = check_shape(rows, cols, (scaling >> 4) != 0, block_of(format));
  if (st != MX_OK) return st;
  const int64_t n = rows * cols;
  if (n == 0) return MX_OK;
  if (!x || !grad_y || !grad_x) return MX_ERR_INVALID_ARG;
  if (!aligned(x, 32) || !aligned(grad_y, 32) || !aligned(grad_x, 32)) return MX_ERR_ALIGN;
  return from_cuda(mxk::launch_fake_bwd(x, grad_y, n, format, scaling, grad_x,
                                        static_cast<cudaStream_t>(stream)));
}

int mx_block_error(const void* x, int64_t rows, int64_t cols, int format, int scaling,
                   float* block_sse, double* totals, void* stream) {
  int st = check_mode(format, scaling);
  if (st != MX_OK) return st;
  st = check_shape(rows, cols, (scaling >> 4) != 0, block_of(format));
  if (st != MX_OK) return st;
  if (!totals) return MX_ERR_INVALID_ARG;
  if (!aligned(totals, 8)) return MX_ERR_ALIGN;
  const int64_t n = rows * cols;
  if (n != 0) {
    if (!x) return MX_ERR_INVALID_ARG;
    if (!aligned(x, 32) || (block_sse && !aligned(block_sse, 4))) return MX_ERR_ALIGN;
  }
  return from_cuda(mxk::launch_block_error(x, n, format, scaling, block_sse, totals,
                                           static_cast<cudaStream_t>(stream)));
}

}  // extern "C"

namespace {

// Shared checks of the BATQuant parameters.
int check_bat(int64_t rows, int64_t cols, int a_dim, const float* A, const float* B,
              const float* beta_min, const float* beta_max) {
  if (a_dim != 1 && a_dim != 2 && a_dim != 4 && a_dim != 8 && a_dim != 16 && a_dim != 32)
    return MX_ERR_INVALID_ARG;
  if ((beta_min == nullptr) != (beta_max == nullptr)) return MX_ERR_INVALID_ARG;
  if (rows == 0 || cols == 0) return MX_OK;
  if (!A || !B) return MX_ERR_INVALID_ARG;
  if (!aligned(A, 16) || !aligned(B, 16)) return MX_ERR_ALIGN;
  if (beta_min && (!aligned(beta_min, 4) || !aligned(beta_max, 4))) return MX_ERR_ALIGN;
  return MX_OK;
}

}  // namespace

extern "C" {

int mx_bat_apply(const void* x, int64_t rows, int64_t cols, int a_dim, const float* A,
                 const float* B, const float* beta_min, const float* beta_max, void* y,
                 void* stream) {
  int st = check_shape(rows, cols, false);
  if (st != MX_OK) return st;
  st = check_bat(rows, cols, a_dim, A, B, beta_min, beta_max);
  if (st != MX_OK) return st;
  const int64_t n = rows * cols;
  if (n == 0) return MX_OK;
  if (!x || !y) return MX_ERR_INVALID_ARG;
  if (!aligned(x, 32) || !aligned(y, 32)) return MX_ERR_ALIGN;
  return from_cuda(mxk::launch_bat(x, rows, cols, a_dim, A, B, beta_min, beta_max, 0, 0, nullptr,
                                   nullptr, nullptr, y, mxk::ScaleMap{0, 0, 0.0},
                                   static_cast<cudaStream_t>(stream)));
}

int mx_bat_quantize(const void* x, int64_t rows, int64_t cols, int a_dim, const float* A,
                    const float* B, const float* beta_min, const float* beta_max, int format,
                    int scaling, void* codes, uint8_t* scales, uint8_t* macro, void* stream) {
  const int layout = scaling & MX_SCALES_MMA;
  scaling &= ~MX_SCALES_MMA;
  int st = check_mode(format, scaling);
  if (st != MX_OK) return st;
  if (block_of(format) != 32 || (scaling >> 4) == 2) return MX_ERR_UNSUPPORTED;
  const bool mbs = (scaling >> 4) != 0;
  st = check_shape(rows, cols, mbs);
  if (st != MX_OK) return st;
  st = check_bat(rows, cols, a_dim, A, B, beta_min, beta_max);
  if (st != MX_OK) return st;
  const int64_t n = rows * cols;
  if (n == 0) return MX_OK;
  if (!x || !codes || !scales || (mbs && !macro)) return MX_ERR_INVALID_ARG;
  if (!aligned(x, 32) || !aligned(codes, 16)) return MX_ERR_ALIGN;
  const auto cs = static_cast<cudaStream_t>(stream);
  if (clear_padding(scales, rows, cols, layout, 32, cs) != cudaSuccess) return MX_ERR_CUDA;
  return from_cuda(mxk::launch_bat(x, rows, cols, a_dim, A, B, beta_min, beta_max, format, scaling,
                                   codes, scales, mbs ? macro : nullptr, nullptr,
                                   scale_map(cols, layout, 32), cs));
}

}  // extern "C"

namespace {

// Shared checks of the block-scaled GEMM entry points. K must hold whole
// 256-element K-blocks; N a multiple of 8 (16-byte output stores); the grid's
// row count bounds M.
int check_gemm(int64_t M, int64_t N, int64_t K, int out_fp32, const void* b_codes,
               const uint8_t* b_scales, const void* d) {
  if (M < 0 || N < 0 || K < 0) return MX_ERR_INVALID_ARG;
  if (K % 256 != 0 || N % 8 != 0) return MX_ERR_SHAPE;
  if (M > (int64_t(65535) * 128) || N > (int64_t(1) << 31) || K > (int64_t(1) << 31))
    return MX_ERR_INVALID_ARG;
  if ((M > 0 && K > kMaxElems / M) || (N > 0 && K > kMaxElems / N) ||
      (M > 0 && N > kMaxElems / M))
    return MX_ERR_INVALID_ARG;
  if (out_fp32 != 0 && out_fp32 != 1) return MX_ERR_INVALID_ARG;
  if (M == 0 || N == 0) return MX_OK;
  if (!d) return MX_ERR_INVALID_ARG;
  if (!aligned(d, 16)) return MX_ERR_ALIGN;
  if (K == 0) return MX_OK;
  if (!b_codes || !b_scales) return MX_ERR_INVALID_ARG;
  if (!aligned(b_codes, 16) || !aligned(b_scales, 16)) return MX_ERR_ALIGN;
  return MX_OK;
}

// K == 0: the product is all zeros.
int gemm_zero(int64_t M, int64_t N, int out_fp32, void* d, cudaStream_t st) {
  return from_cuda(cudaMemsetAsync(d, 0, static_cast<size_t>(M * N * (out_fp32 ? 4 : 2)), st));
}

}  // namespace

extern "C" {

int mx_gemm(const void* a_codes, const uint8_t* a_scales, const void* b_codes,
            const uint8_t* b_scales, int64_t M, int64_t N, int64_t K, int out_fp32, void* d,
            int* status, void* stream) {
  int st = check_gemm(M, N, K, out_fp32, b_codes, b_scales, d);
  if (st != MX_OK || M == 0 || N == 0) return st;
  const auto cs = static_cast<cudaStream_t>(stream);
  if (K == 0) return gemm_zero(M, N, out_fp32, d, cs);
  if (!a_codes || !a_scales) return MX_ERR_INVALID_ARG;
  if (!aligned(a_codes, 16) || !aligned(a_scales, 16) || (status && !aligned(status, 4)))
    return MX_ERR_ALIGN;
  return from_cuda(mxk::launch_gemm(a_codes, a_scales, 0, false, b_codes, b_scales, M, N, K,
                                    out_fp32, d, nullptr, nullptr, status, cs));
}

int mx_quant_gemm(const void* a_bf16, int scaling, const void* b_codes, const uint8_t* b_scales,
                  int64_t M, int64_t N, int64_t K, int out_fp32, void* d, void* a_codes_out,
                  uint8_t* a_scales_out, int* status, void* stream) {
  if (scaling < MX_SCALE_FLOOR || scaling > MX_SCALE_OAS) return MX_ERR_UNSUPPORTED;
  const bool on_chip = (out_fp32 & MX_GEMM_A_ON_CHIP) != 0;
  out_fp32 &= ~MX_GEMM_A_ON_CHIP;
  int st = check_gemm(M, N, K, out_fp32, b_codes, b_scales, d);
  if (st != MX_OK || M == 0 || N == 0) return st;
  const auto cs = static_cast<cudaStream_t>(stream);
  if (K == 0) return gemm_zero(M, N, out_fp32, d, cs);
  if (!a_bf16) return MX_ERR_INVALID_ARG;
  if (!aligned(a_bf16, 32) || (a_codes_out && !aligned(a_codes_out, 16)) ||
      (a_scales_out && !aligned(a_scales_out, 16)) || (status && !aligned(status, 4)))
    return MX_ERR_ALIGN;
  // the tiled layout's padding rows read as zero bytes
  if (clear_padding(a_scales_out, M, K, MX_SCALES_MMA, 32, cs) != cudaSuccess) return MX_ERR_CUDA;
  return from_cuda(mxk::launch_gemm(a_bf16, nullptr, scaling, on_chip, b_codes, b_scales, M, N, K,
                                    out_fp32, d, a_codes_out, a_scales_out, status, cs));
}

// The staged quantize + GEMM for callers that may not allocate: its scratch
// is the library's fixed device array instead of the stream-ordered pool.
int mx_quant_gemm_noalloc(const void* a_bf16, int scaling, const void* b_codes,
                          const uint8_t* b_scales, int64_t M, int64_t N, int64_t K, int out_fp32,
                          void* d, int* status, void* stream) {
  if (scaling < MX_SCALE_FLOOR || scaling > MX_SCALE_OAS) return MX_ERR_UNSUPPORTED;
  int st = check_gemm(M, N, K, out_fp32, b_codes, b_scales, d);
  if (st != MX_OK || M == 0 || N == 0) return st;
  const auto cs = static_cast<cudaStream_t>(stream);
  if (K == 0) return gemm_zero(M, N, out_fp32, d, cs);
  if (!a_bf16) return MX_ERR_INVALID_ARG;
  if (!aligned(a_bf16, 32) || (status && !aligned(status, 4))) return MX_ERR_ALIGN;
  if (!mxk::noalloc_fits(M, K)) return MX_ERR_TOO_LARGE;
  return from_cuda(mxk::launch_quant_gemm_noalloc(a_bf16, scaling, b_codes, b_scales, M, N, K,
                                                  out_fp32, d, status, cs));
}

}  // extern "C"
