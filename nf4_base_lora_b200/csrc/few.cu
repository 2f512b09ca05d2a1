// Rank-r intermediates for few tokens (M <= 16), on CUDA cores:
//   T = s X A^T   (forward, "第 04 篇：QLoRA 原理" §6.3, the LoRA down product)
//   V = s dY B    (backward, §2.4, the input-gradient branch through B)
// Each writes the bf16 hi | lo pair the tensor-core extension steps consume
// (and T in fp32 for reuse by the backward) and lets the fused dequant-GEMM
// that follows launch at once (programmatic dependent launch): the GEMM
// streams and decodes the weight while these run, and waits for them only
// before its extension steps.  The contraction is split over a thread-block
// cluster and summed through distributed shared memory in rank order.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "common.cuh"
#include "kernels.h"
#include "trace.h"

namespace nf4lora {

namespace {

constexpr int kMaxFewTokens = 16;

__device__ __forceinline__ void allow_dependents() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

__device__ __forceinline__ float bf16_lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t v) { return __uint_as_float(v & 0xffff0000u); }

__device__ __forceinline__ void store_split(uint16_t* dst_hi, uint16_t* dst_lo, float v) {
    const __nv_bfloat16 hi = __float2bfloat16_rn(v);
    const __nv_bfloat16 lo = __float2bfloat16_rn(v - __bfloat162float(hi));
    *dst_hi = *reinterpret_cast<const uint16_t*>(&hi);
    *dst_lo = *reinterpret_cast<const uint16_t*>(&lo);
}

constexpr int kDownSplit = 4;   // cluster size along K for T
constexpr int kVSplit = 8;      // cluster size along d_out for V

// T: cluster (1, kDownSplit) per column j of T (j < r64; j >= r written as
// zeros).  CTA rank ks covers k in [ks K / kDownSplit, (ks + 1) K / kDownSplit);
// thread t accumulates k = k0 + 8t, k0 + 8t + 1024, ... for every token.
__global__ void __launch_bounds__(128) k_few_down(const uint16_t* __restrict__ X, const uint16_t* __restrict__ A,
                                                  int M, int K, int r, int r64, float s,
                                                  uint16_t* __restrict__ T2, float* __restrict__ T_saved) {
    allow_dependents();
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int j = blockIdx.x;
    const int ks = static_cast<int>(cluster_ctarank());
    const int k_len = (K / 8 + kDownSplit - 1) / kDownSplit * 8;
    const int k0 = ks * k_len;
    const int k1 = min(K, k0 + k_len);
    float acc[kMaxFewTokens];
#pragma unroll
    for (int m = 0; m < kMaxFewTokens; ++m) acc[m] = 0.0f;
    if (j < r) {
        for (int k = k0 + tid * 8; k < k1; k += 128 * 8) {
            const uint4 a = __ldg(reinterpret_cast<const uint4*>(A + static_cast<int64_t>(j) * K + k));
            const float af[8] = {bf16_lo(a.x), bf16_hi(a.x), bf16_lo(a.y), bf16_hi(a.y),
                                 bf16_lo(a.z), bf16_hi(a.z), bf16_lo(a.w), bf16_hi(a.w)};
#pragma unroll
            for (int m = 0; m < kMaxFewTokens; ++m) {
                if (m < M) {
                    const uint4 x = __ldg(reinterpret_cast<const uint4*>(X + static_cast<int64_t>(m) * K + k));
                    float d = acc[m];
                    d = fmaf(bf16_lo(x.x), af[0], d);
                    d = fmaf(bf16_hi(x.x), af[1], d);
                    d = fmaf(bf16_lo(x.y), af[2], d);
                    d = fmaf(bf16_hi(x.y), af[3], d);
                    d = fmaf(bf16_lo(x.z), af[4], d);
                    d = fmaf(bf16_hi(x.z), af[5], d);
                    d = fmaf(bf16_lo(x.w), af[6], d);
                    d = fmaf(bf16_hi(x.w), af[7], d);
                    acc[m] = d;
                }
            }
        }
    }
    __shared__ float red[4][kMaxFewTokens];
    __shared__ float part[kMaxFewTokens];
#pragma unroll
    for (int m = 0; m < kMaxFewTokens; ++m) {
        float v = acc[m];
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
        if (lane == 0) red[warp][m] = v;
    }
    __syncthreads();
    if (tid < kMaxFewTokens) part[tid] = ((red[0][tid] + red[1][tid]) + red[2][tid]) + red[3][tid];
    cluster_sync_all();
    if (ks == 0 && tid < M) {
        float t[kDownSplit];
#pragma unroll
        for (int rk = 0; rk < kDownSplit; ++rk) t[rk] = ld_cluster_f32(cluster_map(smem_u32(&part[tid]), rk));
        float v = 0.0f;
#pragma unroll
        for (int rk = 0; rk < kDownSplit; ++rk) v += t[rk];
        v *= s;
        uint16_t* row = T2 + static_cast<int64_t>(tid) * 2 * r64;
        store_split(row + j, row + r64 + j, v);
        if (T_saved != nullptr && j < r) T_saved[static_cast<int64_t>(tid) * r + j] = v;
    }
    cluster_sync_all();
}

// V: cluster (1, kVSplit) per 4 columns of V; CTA rank ns covers rows
// n in [ns N / kVSplit, (ns + 1) N / kVSplit); thread t takes rows t, t + 128, ...
__global__ void __launch_bounds__(128) k_few_v(const uint16_t* __restrict__ dY, const uint16_t* __restrict__ B,
                                               int M, int N, int r, int r64, float s, uint16_t* __restrict__ V2) {
    allow_dependents();
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int j0 = blockIdx.x * 4;
    const int ns = static_cast<int>(cluster_ctarank());
    const int n_len = (N + kVSplit - 1) / kVSplit;
    const int n0 = ns * n_len;
    const int n1 = min(N, n0 + n_len);
    float acc[kMaxFewTokens][4];
#pragma unroll
    for (int m = 0; m < kMaxFewTokens; ++m)
#pragma unroll
        for (int q = 0; q < 4; ++q) acc[m][q] = 0.0f;
    if (j0 < r) {
#pragma unroll 4
        for (int n = n0 + tid; n < n1; n += 128) {
            const uint2 b = __ldg(reinterpret_cast<const uint2*>(B + static_cast<int64_t>(n) * r + j0));
            const float bf[4] = {bf16_lo(b.x), bf16_hi(b.x), bf16_lo(b.y), bf16_hi(b.y)};
#pragma unroll
            for (int m = 0; m < kMaxFewTokens; ++m) {
                if (m < M) {
                    const float d = __uint_as_float(static_cast<uint32_t>(__ldg(dY + static_cast<int64_t>(m) * N + n))
                                                    << 16);
#pragma unroll
                    for (int q = 0; q < 4; ++q) acc[m][q] = fmaf(d, bf[q], acc[m][q]);
                }
            }
        }
    }
    __shared__ float red[4][kMaxFewTokens][4];
    __shared__ float part[kMaxFewTokens][4];
#pragma unroll
    for (int m = 0; m < kMaxFewTokens; ++m)
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            float v = acc[m][q];
#pragma unroll
            for (int o = 16; o >= 1; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
            if (lane == 0) red[warp][m][q] = v;
        }
    __syncthreads();
    if (tid < 4 * kMaxFewTokens) {
        const int m = tid >> 2, q = tid & 3;
        part[m][q] = ((red[0][m][q] + red[1][m][q]) + red[2][m][q]) + red[3][m][q];
    }
    cluster_sync_all();
    if (ns == 0 && tid < 4 * M) {
        const int m = tid >> 2, q = tid & 3, j = j0 + q;
        float t[kVSplit];
#pragma unroll
        for (int rk = 0; rk < kVSplit; ++rk) t[rk] = ld_cluster_f32(cluster_map(smem_u32(&part[m][q]), rk));
        float v = 0.0f;
#pragma unroll
        for (int rk = 0; rk < kVSplit; ++rk) v += t[rk];
        v *= s;
        uint16_t* row = V2 + static_cast<int64_t>(m) * 2 * r64;
        if (j < r64) store_split(row + j, row + r64 + j, j < r ? v : 0.0f);
    }
    cluster_sync_all();
}

}  // namespace

static cudaLaunchConfig_t cluster_config(dim3 grid, int split, cudaLaunchAttribute* attr, cudaStream_t stream) {
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = grid;
    cfg.blockDim = dim3(128);
    cfg.stream = stream;
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 1;
    attr[0].val.clusterDim.y = split;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cfg;
}

cudaError_t launch_few_down(const uint16_t* X, const uint16_t* A, int M, int K, int r, int r64, float s,
                            uint16_t* T2, float* T_saved, cudaStream_t stream) {
    cudaLaunchAttribute attr[1];
    cudaLaunchConfig_t cfg = cluster_config(dim3(r64, kDownSplit), kDownSplit, attr, stream);
    TraceScope trace("few_lora_down", stream);
    return cudaLaunchKernelEx(&cfg, k_few_down, X, A, M, K, r, r64, s, T2, T_saved);
}

cudaError_t launch_few_v(const uint16_t* dY, const uint16_t* B, int M, int N, int r, int r64, float s,
                         uint16_t* V2, cudaStream_t stream) {
    cudaLaunchAttribute attr[1];
    cudaLaunchConfig_t cfg = cluster_config(dim3(r64 / 4, kVSplit), kVSplit, attr, stream);
    TraceScope trace("few_lora_v", stream);
    return cudaLaunchKernelEx(&cfg, k_few_v, dY, B, M, N, r, r64, s, V2);
}

}  // namespace nf4lora
