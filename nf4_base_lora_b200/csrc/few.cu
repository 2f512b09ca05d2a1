// Rank-r intermediates for few tokens (M <= 16):
//   T = s X A^T   (forward, "第 04 篇：QLoRA 原理" §6.3, the LoRA down product;
//                  warp-level tensor instructions)
//   V = s dY B    (backward, §2.4, the input-gradient branch through B; CUDA cores)
// Each writes the bf16 hi | lo pair the fused products' extension steps
// consume (and T in fp32 for reuse by the backward) and lets the fused
// dequant-GEMM that follows launch early (programmatic dependent launch): the
// GEMM streams and decodes the weight while these run, and waits for them only
// before its extension steps.  The contraction is split over a thread-block
// cluster and summed through distributed shared memory in rank order.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>
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

// T on the warp-level tensor instructions: D[t, j] = sum_k X[t, k] A[j, k]
// (m16n8k16: A operand = X, 16 tokens x 16 k; B operand = 8 rows of A).
// CTA (x, z) computes columns 16x .. 16x + 15 of T over the z-th of up to 8
// slices of K; the slices of one column group form a cluster.  A CTA copies
// its part of X and its 16 rows of A (up to 512 k at a time) into shared
// memory with asynchronous copies issued all at once, and releases the
// dependent launch as soon as they are requested, so that these loads queue
// ahead of the dependent kernel's.  The CTAs are small (four warps, 37 KB of
// shared memory) and many (one per SM for r = 64), so that the loads are
// spread over SMs and the CTAs share SMs with the dependent kernel's.  Warp w
// takes every fourth 16-wide chunk; partials are added in a fixed order: the
// four warps in shared memory, then the cluster ranks by rank 0 reading the
// others' shared memory.
constexpr int kDownThreads = 128;
constexpr int kDownMaxSplit = 8;
constexpr int kDownBatch = 512;                 // k per staged slice
constexpr int kDownStride = kDownBatch + 8;     // row stride (elements): 1040 bytes, conflict-free fragments
constexpr int kDownSmem = 2 * kMaxFewTokens * kDownStride * 2 + 4 * kMaxFewTokens * 16 * 4;

__device__ __forceinline__ void mma_m16n8k16(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                             uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void cp_async16(void* smem_dst, const void* src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(smem_dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() {
    asm volatile("cp.async.commit_group;\n\tcp.async.wait_group 0;" ::: "memory");
}

__global__ void __launch_bounds__(kDownThreads) k_few_down(const uint16_t* __restrict__ X,
                                                            const uint16_t* __restrict__ A, int M, int K, int r,
                                                            int r64, float s, uint16_t* __restrict__ T2,
                                                            float* __restrict__ T_saved) {
    extern __shared__ __align__(16) uint8_t smem[];
    uint16_t* sX = reinterpret_cast<uint16_t*>(smem);                // [16][kDownStride]
    uint16_t* sA = sX + kMaxFewTokens * kDownStride;                 // [16][kDownStride]
    float* s_w = reinterpret_cast<float*>(sA + 16 * kDownStride);    // [4 warps][16 t][16 j]
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, g = lane >> 2, q = lane & 3;
    const int splits = static_cast<int>(gridDim.z);
    const int rank = static_cast<int>(cluster_ctarank());
    const int j0 = 16 * blockIdx.x;  // this CTA's columns of T
    const int bpr = K / 64;
    const int per = bpr / splits, extra = bpr % splits;
    const int k_begin = 64 * (rank * per + (rank < extra ? rank : extra));
    const int k_end = k_begin + 64 * (per + (rank < extra ? 1 : 0));
    float acc[2][4] = {{0.0f, 0.0f, 0.0f, 0.0f}, {0.0f, 0.0f, 0.0f, 0.0f}};

    bool released = false;
    for (int k0 = k_begin; k0 < k_end; k0 += kDownBatch) {
        const int kn = min(kDownBatch, k_end - k0);  // a multiple of 64
        const int pieces = kn / 8;                   // 16-byte pieces per row
        __syncthreads();                             // the previous slice is no longer read
        for (int i = tid; i < 2 * kMaxFewTokens * pieces; i += kDownThreads) {
            const int row = i / pieces, pc = i - row * pieces;
            if (row < kMaxFewTokens) {
                uint16_t* dst = sX + row * kDownStride + pc * 8;
                if (row < M) cp_async16(dst, X + static_cast<int64_t>(row) * K + k0 + pc * 8);
                else *reinterpret_cast<uint4*>(dst) = make_uint4(0, 0, 0, 0);
            } else {
                const int j = j0 + row - kMaxFewTokens;
                uint16_t* dst = sA + (row - kMaxFewTokens) * kDownStride + pc * 8;
                if (j < r) cp_async16(dst, A + static_cast<int64_t>(j) * K + k0 + pc * 8);
                else *reinterpret_cast<uint4*>(dst) = make_uint4(0, 0, 0, 0);
            }
        }
        if (!released) {
            allow_dependents();
            released = true;
        }
        cp_async_wait_all();
        __syncthreads();
        const uint16_t* xr0 = sX + g * kDownStride + 2 * q;
        const uint16_t* xr8 = xr0 + 8 * kDownStride;
        const uint16_t* ar0 = sA + g * kDownStride + 2 * q;  // columns j0 .. j0 + 7
        const uint16_t* ar1 = ar0 + 8 * kDownStride;         // columns j0 + 8 .. j0 + 15
#pragma unroll 4
        for (int c = warp; c < kn / 16; c += 4) {
            const int k = 16 * c;
            const uint32_t a0 = *reinterpret_cast<const uint32_t*>(xr0 + k), a1 = *reinterpret_cast<const uint32_t*>(xr8 + k);
            const uint32_t a2 = *reinterpret_cast<const uint32_t*>(xr0 + k + 8), a3 = *reinterpret_cast<const uint32_t*>(xr8 + k + 8);
            mma_m16n8k16(acc[0], a0, a1, a2, a3, *reinterpret_cast<const uint32_t*>(ar0 + k),
                         *reinterpret_cast<const uint32_t*>(ar0 + k + 8));
            mma_m16n8k16(acc[1], a0, a1, a2, a3, *reinterpret_cast<const uint32_t*>(ar1 + k),
                         *reinterpret_cast<const uint32_t*>(ar1 + k + 8));
        }
    }
    if (!released) allow_dependents();

    // acc[u]: tokens g (0, 1) and g + 8 (2, 3) at columns 8u + 2q + {0, 1}; the
    // four warps' partials added in order by warp 0 into s_w[0]
#pragma unroll
    for (int u = 0; u < 2; ++u) {
        float* dst = s_w + warp * 256;
        const int j = 8 * u + 2 * q;
        dst[g * 16 + j] = acc[u][0];
        dst[g * 16 + j + 1] = acc[u][1];
        dst[(g + 8) * 16 + j] = acc[u][2];
        dst[(g + 8) * 16 + j + 1] = acc[u][3];
    }
    __syncthreads();
    for (int i = tid; i < 256; i += kDownThreads) s_w[i] = ((s_w[i] + s_w[256 + i]) + s_w[512 + i]) + s_w[768 + i];
    cluster_sync_all();  // every rank's partial (s_w[0 .. 255]) is complete and visible
    if (rank == 0) {
        for (int i = tid; i < M * 16; i += kDownThreads) {
            const int t = i >> 4, jl = i & 15, j = j0 + jl;
            float part[kDownMaxSplit];
            const uint32_t addr = smem_u32(&s_w[t * 16 + jl]);
#pragma unroll
            for (int rk = 1; rk < kDownMaxSplit; ++rk)
                if (rk < splits) part[rk] = ld_cluster_f32(cluster_map(addr, rk));
            float v = s_w[t * 16 + jl];
#pragma unroll
            for (int rk = 1; rk < kDownMaxSplit; ++rk)
                if (rk < splits) v += part[rk];
            v *= s;
            if (j < r64) {
                uint16_t* row = T2 + static_cast<int64_t>(t) * 2 * r64;
                store_split(row + j, row + r64 + j, j < r ? v : 0.0f);
                if (T_saved != nullptr && j < r) T_saved[static_cast<int64_t>(t) * r + j] = v;
            }
        }
    }
    cluster_sync_all();  // rank 0 has read the other ranks' shared memory
}

constexpr int kVSplit = 8;      // cluster size along d_out for V

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
    if (M < 1 || M > kMaxFewTokens || K % 64 != 0 || r64 > 256) return cudaErrorInvalidValue;
    static bool configured[64] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64 || !configured[dev]) {
        e = cudaFuncSetAttribute(k_few_down, cudaFuncAttributeMaxDynamicSharedMemorySize, kDownSmem);
        if (e != cudaSuccess) return e;
        // the same shared-memory carveout as the dependent kernel, so that an SM
        // running this kernel can also take a CTA of that one
        e = cudaFuncSetAttribute(k_few_down, cudaFuncAttributePreferredSharedMemoryCarveout,
                                 cudaSharedmemCarveoutMaxShared);
        if (e != cudaSuccess) return e;
        if (dev >= 0 && dev < 64) configured[dev] = true;
    }
    const int splits = std::max(1, std::min(kDownMaxSplit, K / 64));
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(r64 / 16, 1, splits);
    cfg.blockDim = dim3(kDownThreads);
    cfg.dynamicSmemBytes = kDownSmem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 1;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = splits;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    TraceScope trace("few_lora_down", stream);
    return cudaLaunchKernelEx(&cfg, k_few_down, X, A, M, K, r, r64, s, T2, T_saved);
}

cudaError_t launch_few_v(const uint16_t* dY, const uint16_t* B, int M, int N, int r, int r64, float s,
                         uint16_t* V2, cudaStream_t stream) {
    static bool configured[64] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64 || !configured[dev]) {
        // the dependent kernel's shared-memory carveout (see launch_few_down)
        e = cudaFuncSetAttribute(k_few_v, cudaFuncAttributePreferredSharedMemoryCarveout,
                                 cudaSharedmemCarveoutMaxShared);
        if (e != cudaSuccess) return e;
        if (dev >= 0 && dev < 64) configured[dev] = true;
    }
    cudaLaunchAttribute attr[1];
    cudaLaunchConfig_t cfg = cluster_config(dim3(r64 / 4, kVSplit), kVSplit, attr, stream);
    TraceScope trace("few_lora_v", stream);
    return cudaLaunchKernelEx(&cfg, k_few_v, dY, B, M, N, r, r64, s, V2);
}

}  // namespace nf4lora
