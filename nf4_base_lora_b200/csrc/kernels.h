// Internal launchers of libnf4lora (host-side declarations, C++ linkage).
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

namespace nf4lora {

cudaError_t launch_nf4_quantize(const float* W, int64_t n, uint8_t* codes, int8_t* qscale,
                                float* scale2, float* scale_mean, float* ws_absmax,
                                double* ws_tile_sums, int num_sms, cudaStream_t stream);

cudaError_t launch_nf4_dequantize(const uint8_t* codes, const int8_t* qscale, const float* scale2,
                                  const float* scale_mean, int64_t n, uint16_t* out, int num_sms,
                                  cudaStream_t stream);

// Few-token (M <= 16) rank-r intermediates as bf16 hi | lo pairs; each
// releases its dependent launch as soon as it starts.
cudaError_t launch_few_down(const uint16_t* X, const uint16_t* A, int M, int K, int r, int r64, float s,
                            uint16_t* T2, float* T_saved, cudaStream_t stream);
cudaError_t launch_few_v(const uint16_t* dY, const uint16_t* B, int M, int N, int r, int r64, float s,
                         uint16_t* V2, cudaStream_t stream);

}  // namespace nf4lora
