// Internal launchers of libmx (not part of the public ABI). Arguments are
// already validated by the C entry points; n = rows * cols elements.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

namespace mxk {

// Where the E8M0 byte of block b (row-major block index) lives: bpr == 0 is
// the plain [rows, cols/32] array; otherwise the tiled layout of block-scaled
// tensor-core operands (128 rows x 4 block columns per 512-byte tile, tiles
// row-major with nct tiles per tile row, inside a tile the byte
// (r % 32) * 16 + ((r / 32) % 4) * 4 + (j % 4)).
struct ScaleMap {
  int64_t bpr;   // blocks per row (cols / 32), or 0 for the plain layout
  int64_t nct;   // tiles per tile row: ceil(bpr / 4)
  double inv;    // 1 / bpr, rounded (for the row index of a block)
};

cudaError_t launch_quantize(const void* x, int64_t n, int fmt, int scaling, void* codes,
                            uint8_t* scales, uint8_t* macro, ScaleMap sm, cudaStream_t st);
cudaError_t launch_dequantize(const void* codes, const uint8_t* scales, const uint8_t* macro,
                              int64_t n, int fmt, int out_fp32, void* out, ScaleMap sm,
                              cudaStream_t st);
cudaError_t launch_fake_fwd(const void* x, int64_t n, int fmt, int scaling, void* y,
                            uint8_t* scales_out, ScaleMap sm, cudaStream_t st);
cudaError_t launch_fake_bwd(const void* x, const void* gy, int64_t n, int fmt, int scaling,
                            void* gx, cudaStream_t st);
// BATQuant: y != null writes the transformed bf16 rows; else quantizes them.
cudaError_t launch_bat(const void* x, int64_t rows, int64_t cols, int a_dim, const float* A,
                       const float* B, const float* beta_min, const float* beta_max, int fmt,
                       int scaling, void* codes, uint8_t* scales, uint8_t* macro, void* y,
                       ScaleMap sm, cudaStream_t st);
// Block-scaled MXFP4 GEMM D = A B^T: A pre-quantized (codes + tiled scales)
// when a_scales != null, else bf16 quantized with rule a_rule within the
// launch: staged through a_codes_out / a_scales_out (scratch for a null one),
// or on chip (a_on_chip; a non-null buffer then receives its part).
cudaError_t launch_gemm(const void* a, const uint8_t* a_scales, int a_rule, bool a_on_chip,
                        const void* b_codes, const uint8_t* b_scales, int64_t M, int64_t N,
                        int64_t K, int out_fp32, void* d, void* a_codes_out,
                        uint8_t* a_scales_out, int* status, cudaStream_t st);
// mx_quant_gemm_noalloc: the staged quantize + GEMM with its scratch in the
// library's fixed device array (noalloc_fits: the problem fits it).
bool noalloc_fits(int64_t M, int64_t K);
cudaError_t launch_quant_gemm_noalloc(const void* a, int a_rule, const void* b_codes,
                                      const uint8_t* b_scales, int64_t M, int64_t N, int64_t K,
                                      int out_fp32, void* d, int* status, cudaStream_t st);
cudaError_t launch_block_error(const void* x, int64_t n, int fmt, int scaling, float* block_sse,
                               double* totals, cudaStream_t st);

}  // namespace mxk
