// Internal launchers of libnf4lora (host-side declarations, C++ linkage).
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

namespace nf4lora {

// Double quantisation: qscale, scale2, scale_mean and both workspaces set.
// ws_warp_sums holds 8 fp64 values per tile of 256 blocks, then one per
// segment of 2048 tiles and a 4-byte ticket.
// fp32 block scales: qscale, scale2, scale_mean and ws_warp_sums NULL, and
// ws_absmax is the tensor's absmax array (the stored scales).
cudaError_t launch_nf4_quantize(const float* W, int64_t n, uint8_t* codes, int8_t* qscale,
                                float* scale2, float* scale_mean, float* ws_absmax,
                                double* ws_warp_sums, int num_sms, cudaStream_t stream);

// absmax NULL: double-quantised scales; else the fp32 block scales.
cudaError_t launch_nf4_dequantize(const uint8_t* codes, const int8_t* qscale, const float* scale2,
                                  const float* scale_mean, const float* absmax, int64_t n, uint16_t* out,
                                  int num_sms, cudaStream_t stream);

// AdamW step of up to kAdamwMaxTensors adapter tensors per launch (fp32
// master p, bf16 copy p16 or NULL, bf16 gradient g, fp32 moments m, v; n
// elements each; pointers 16-byte aligned).
constexpr int kAdamwMaxTensors = 8;
struct AdamwBatch {
    float* p[kAdamwMaxTensors];
    uint16_t* p16[kAdamwMaxTensors];
    const uint16_t* g[kAdamwMaxTensors];
    float* m[kAdamwMaxTensors];
    float* v[kAdamwMaxTensors];
    int64_t n[kAdamwMaxTensors];
    int count;
};
// decay = 1 - lr wd; b1, omb1 = 1 - b1, b2, omb2 = 1 - b2;
// step_size = lr / (1 - b1^t); inv_sqrt_bc2 = 1 / sqrt(1 - b2^t); eps.
struct AdamwConsts {
    float decay, b1, omb1, b2, omb2, step_size, inv_sqrt_bc2, eps;
};
cudaError_t launch_adamw(const AdamwBatch& b, const AdamwConsts& c, int num_sms, cudaStream_t stream);

// W'[N, K] fp32 = fp32(W_hat + s B A) from an encoded weight and the adapter
// (rank sum in fp64, ascending j).
cudaError_t launch_merge_lora(const uint8_t* codes, const int8_t* qscale, const float* scale2,
                              const float* scale_mean, const float* absmax, const uint16_t* A, const uint16_t* B,
                              int r, int64_t N,
                              int64_t K, float s, float* out, cudaStream_t stream);

// Few-token (M <= 16) rank-r intermediates as bf16 hi | lo pairs; each is a
// programmatic dependent of the kernel before it and releases its own
// dependent once it has waited for that kernel.
cudaError_t launch_few_down(const uint16_t* X, const uint16_t* A, int M, int K, int r, int r64, float s,
                            uint16_t* T2, float* T_saved, cudaStream_t stream);
cudaError_t launch_few_v(const uint16_t* dY, const uint16_t* B, int M, int N, int r, int r64, float s,
                         uint16_t* V2, cudaStream_t stream);

// Few-token (M <= 16) fused products on warp-level tensor instructions with
// the weight decoded in registers (fewmma.cu).
struct FewArgs {
    const uint16_t* act;       // forward: X [M, K]; input grad: dY [M, N]
    const uint8_t* codes;      // packed NF4 codes [N, K / 2]
    const int8_t* qscale;      // [N K / 64]
    const float* scale2;       // [ceil(N K / 64 / 256)]
    const float* scale_mean;   // [1]
    const float* absmax;       // [N K / 64] fp32 block scales, or NULL (double-quantised scales)
    int M, N, K;               // tokens, d_out, d_in
    const uint16_t* ext_act;   // T2 / V2 [M, 2 r64] (bf16 hi | lo)
    const uint16_t* ext_w;     // forward: B [N, r]; input grad: A [r, K]
    int r, r64;
    uint16_t* out;             // forward: Y [M, N]; input grad: dX [M, K]
    int pdl;                   // launched as a programmatic dependent of the ext_act producer
};
int few_max_split(bool forward);
// Plan of the few-token forward (fewfwd.cu): clusters of cs CTAs along the
// contraction, O weight octets per cluster, the ring of quad stages and the
// shared-memory layout.
struct FewFwdPlan {
    int cs;          // CTAs per cluster (1 or 2), splitting the block quads
    int O;           // weight octets (8 rows) per cluster
    int clusters;
    int nq0;         // block quads of rank 0 (rank 1 takes the rest)
    int WQ;          // quad slots: warps w with w % WQ equal share a quad
    int NR;          // ring stages
    int nbox, box_rows, code_bytes;  // TMA boxes of the codes of one stage
    int xbox_rows, xbox_bytes;       // TMA box of one activation block: 16 token rows (8 when M <= 8)
    int slot;        // bytes per stage (codes + activations), a multiple of 1024
    int qrow, q_bytes, step_bytes, t2_bytes, b_bytes, recv_bytes;
    int smem;        // dynamic shared memory
};
bool few_fwd_plan(int M, int N, int K, int r, int num_sms, bool fp32_scales, FewFwdPlan* out);
// map_codes: the packed codes as bytes [N, K / 2], box {128 bytes, plan.box_rows
// rows}, 128-byte swizzle; map_x: the activations as bf16 [M, K], box {64, 16},
// 128-byte swizzle
cudaError_t launch_few_fwd(const CUtensorMap& map_codes, const CUtensorMap& map_x, const FewArgs& a,
                           const FewFwdPlan& p, cudaStream_t stream);
// map_codes: the packed codes as bytes [N, K / 2], box {64 bytes, 256 rows},
// 64-byte swizzle
cudaError_t launch_few_dx(const CUtensorMap& map_codes, const FewArgs& a, int splits, cudaStream_t stream);

}  // namespace nf4lora
