// Internal interface between the C ABI (api.cu) and the layer orchestration
// (layer.cu).  Host-side, C++ linkage.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

namespace nf4lora {

// The split-K heuristics size their grids for this many SMs (B200: 148), so
// that workspace sizes depend only on the problem shape.
constexpr int kPlanSMs = 148;

struct LayerCtx {
    const uint8_t* codes;
    const int8_t* qscale;
    const float* scale2;
    const float* scale_mean;
    const float* absmax;  // fp32 block scales, or NULL (the double-quantised scales above)
    int64_t d_out;
    int64_t d_in;
    int num_sms;
    cudaStream_t stream;
};

int64_t fwd_workspace_bytes(int64_t M, int64_t d_out, int64_t d_in, int r, int num_sms);
int64_t bwd_workspace_bytes(int64_t M, int64_t d_out, int64_t d_in, int r, int num_sms);

// The CUDA error of the last failed launch of the calling thread (then reset).
cudaError_t layer_last_cuda_error();

// Return 0 on success, -1 if a tensor map could not be encoded, -2 if a
// launch failed.
int layer_fwd(const LayerCtx& c, const uint16_t* A, const uint16_t* B, int r, float s, const uint16_t* X,
              int64_t M, uint16_t* Y, float* T_saved, uint8_t* ws);
int layer_bwd(const LayerCtx& c, const uint16_t* A, const uint16_t* B, int r, float s, const uint16_t* X,
              const float* T_saved, const uint16_t* dY, int64_t M, uint16_t* dX, uint16_t* dA,
              uint16_t* dB, int accumulate, uint8_t* ws);

}  // namespace nf4lora
