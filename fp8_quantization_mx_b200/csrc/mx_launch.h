// Internal launchers of libmx (not part of the public ABI). Arguments are
// already validated by the C entry points; n = rows * cols elements.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

namespace mxk {

cudaError_t launch_quantize(const void* x, int64_t n, int fmt, int scaling, void* codes,
                            uint8_t* scales, uint8_t* macro, cudaStream_t st);
cudaError_t launch_dequantize(const void* codes, const uint8_t* scales, const uint8_t* macro,
                              int64_t n, int fmt, int out_fp32, void* out, cudaStream_t st);
cudaError_t launch_fake_fwd(const void* x, int64_t n, int fmt, int scaling, void* y,
                            uint8_t* scales_out, cudaStream_t st);
cudaError_t launch_fake_bwd(const void* x, const void* gy, int64_t n, int fmt, int scaling,
                            void* gx, cudaStream_t st);
cudaError_t launch_block_error(const void* x, int64_t n, int fmt, int scaling, float* block_sse,
                               double* totals, cudaStream_t st);

}  // namespace mxk
