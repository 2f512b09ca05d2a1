// Rank-r intermediates for few tokens (M <= 16):
//   T = s X A^T   (forward, "第 04 篇：QLoRA 原理" §6.3, the LoRA down product)
//   V = s dY B    (backward, §2.4, the input-gradient branch through B)
// Each writes the bf16 hi | lo pair the fused products' extension steps
// consume (and T in fp32 for reuse by the backward) and lets the fused
// dequant-GEMM that follows launch early (programmatic dependent launch): the
// GEMM streams and decodes the weight while these run, and waits for them only
// before its extension steps.  The contraction is split over a thread-block
// cluster and summed through distributed shared memory in rank order.
//
// Both are themselves programmatic dependents of the kernel before them (the
// previous fused GEMM releases its dependents when it starts): their CTAs
// start early and ask L2 for their rows of the LoRA factor (a prefetch only:
// the factor may have been written by that very kernel, an optimizer step for
// instance), then wait for the preceding kernel to finish before they read
// anything.  They release their own dependent right after that wait, so the
// fused GEMM that follows may read the activations and the encoded weight
// before its own wait.
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

// Asks L2 for `bytes` (a multiple of 16) from a 16-byte aligned address, in
// pieces of at most 32 KB.
__device__ __forceinline__ void prefetch_l2_pieces(const void* src, uint32_t bytes) {
    const uint8_t* p = static_cast<const uint8_t*>(src);
    for (uint32_t off = 0; off < bytes; off += 32768u) prefetch_l2_bulk(p + off, min(32768u, bytes - off));
}

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
// its 16 rows of A and its part of X (up to 512 k at a time) into shared
// memory with asynchronous copies issued all at once, after the wait for the
// preceding kernel (the rows of A were asked into L2 before it), and the
// dependent launch is released right after that wait.  The CTAs are small (four warps, 37 KB of
// shared memory) and many, so that the loads are spread over SMs (the
// dependent forward's CTAs hold an SM's whole register file, so they start on
// an SM once these have left it).  Warp w
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

    // this CTA's rows of A over its K slice, into L2 while the preceding kernel runs
    if (tid < 16 && j0 + tid < r && k_begin < k_end)
        prefetch_l2_pieces(A + static_cast<int64_t>(j0 + tid) * K + k_begin,
                           static_cast<uint32_t>(2 * (k_end - k_begin)));
    pdl_wait();                // the preceding kernel's writes (X, or A itself) are complete and visible
    pdl_launch_dependents();   // the fused GEMM may start: everything before it is complete
    for (int k0 = k_begin; k0 < k_end; k0 += kDownBatch) {
        const int kn = min(kDownBatch, k_end - k0);  // a multiple of 64
        const int pieces = kn / 8;                   // 16-byte pieces per row
        __syncthreads();                             // the previous slice is no longer read
        for (int i = tid; i < kMaxFewTokens * pieces; i += kDownThreads) {
            const int row = i / pieces, pc = i - row * pieces, j = j0 + row;
            uint16_t* dst = sA + row * kDownStride + pc * 8;
            if (j < r) cp_async16(dst, A + static_cast<int64_t>(j) * K + k0 + pc * 8);
            else *reinterpret_cast<uint4*>(dst) = make_uint4(0, 0, 0, 0);
        }
        for (int i = tid; i < kMaxFewTokens * pieces; i += kDownThreads) {
            const int row = i / pieces, pc = i - row * pieces;
            uint16_t* dst = sX + row * kDownStride + pc * 8;
            if (row < M) cp_async16(dst, X + static_cast<int64_t>(row) * K + k0 + pc * 8);
            else *reinterpret_cast<uint4*>(dst) = make_uint4(0, 0, 0, 0);
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

// V on the warp-level tensor instructions: D[t, j] = sum_n dY[t, n] B[n, j]
// (m16n8k16: A operand = dY, 16 tokens x 16 n; B operand = B[n][j] read
// transposed from shared memory with ldmatrix.trans).  The same layout as the
// T kernel: CTA (x, z) computes columns 16x .. 16x + 15 of V over the z-th of
// up to 8 slices of d_out, the slices of one column group form a cluster, the
// slice of B and of dY (up to 256 rows at a time) comes in by asynchronous
// copies issued at once after the wait for the preceding kernel (the rows of B
// were asked into L2 before it), and the dependent launch is released right
// after that wait.
constexpr int kVBatch = 256;                    // rows of B per staged slice (small enough to share an SM with the dX kernel)
constexpr int kVYStride = kVBatch + 8;          // dY staging row stride (elements)
constexpr int kVBStride = 24;                   // B staging row stride (elements): 48 bytes, conflict-free ldmatrix
constexpr int kVSmem = kMaxFewTokens * kVYStride * 2 + kVBatch * kVBStride * 2 + 4 * kMaxFewTokens * 16 * 4;

__device__ __forceinline__ void ldmatrix_x2_trans(uint32_t addr, uint32_t& r0, uint32_t& r1) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x2.trans.shared.b16 {%0, %1}, [%2];" : "=r"(r0), "=r"(r1) : "r"(addr));
}

__global__ void __launch_bounds__(kDownThreads) k_few_v(const uint16_t* __restrict__ dY,
                                                         const uint16_t* __restrict__ B, int M, int N, int r,
                                                         int r64, float s, uint16_t* __restrict__ V2) {
    extern __shared__ __align__(16) uint8_t smem[];
    uint16_t* sY = reinterpret_cast<uint16_t*>(smem);             // [16][kVYStride]
    uint16_t* sB = sY + kMaxFewTokens * kVYStride;               // [kVBatch][kVBStride]: rows n, columns j0 .. j0 + 15
    float* s_w = reinterpret_cast<float*>(sB + kVBatch * kVBStride);  // [4 warps][16 t][16 j]
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, g = lane >> 2, q = lane & 3;
    const int splits = static_cast<int>(gridDim.z);
    const int rank = static_cast<int>(cluster_ctarank());
    const int j0 = 16 * blockIdx.x;
    const int nq = (N + 15) / 16;  // 16-row chunks of d_out
    const int per = nq / splits, extra = nq % splits;
    const int n_begin = 16 * (rank * per + (rank < extra ? rank : extra));
    const int n_end = n_begin + 16 * (per + (rank < extra ? 1 : 0));
    float acc[2][4] = {{0.0f, 0.0f, 0.0f, 0.0f}, {0.0f, 0.0f, 0.0f, 0.0f}};

    // this CTA's rows of B (all r columns of each, contiguous), into L2 while the preceding kernel runs
    if (tid == 0 && n_begin < n_end && j0 < r) {
        const int rows = min(n_end, N) - n_begin;
        if (rows > 0)
            prefetch_l2_pieces(B + static_cast<int64_t>(n_begin) * r, static_cast<uint32_t>(2 * rows * r));
    }
    pdl_wait();                // the preceding kernel's writes (dY, or B itself) are complete and visible
    pdl_launch_dependents();   // the fused GEMM may start: everything before it is complete
    for (int n0 = n_begin; n0 < n_end; n0 += kVBatch) {
        const int nn = min(kVBatch, n_end - n0);  // a multiple of 16
        __syncthreads();                          // the previous slice is no longer read
        // B[n0 : n0 + nn, j0 : j0 + 16] in 16-byte pieces (r is a multiple of 8)
        for (int i = tid; i < nn * 2; i += kDownThreads) {
            const int row = i >> 1, h = i & 1, n = n0 + row, j = j0 + 8 * h;
            uint16_t* dst = sB + row * kVBStride + 8 * h;
            if (n < N && j < r) cp_async16(dst, B + static_cast<int64_t>(n) * r + j);
            else *reinterpret_cast<uint4*>(dst) = make_uint4(0, 0, 0, 0);
        }
        // dY[:, n0 : n0 + nn] in 16-byte pieces (N is a multiple of 8)
        for (int i = tid; i < kMaxFewTokens * (nn / 8); i += kDownThreads) {
            const int t = i / (nn / 8), pc = i - t * (nn / 8), n = n0 + 8 * pc;
            uint16_t* dst = sY + t * kVYStride + 8 * pc;
            if (t < M && n < N) cp_async16(dst, dY + static_cast<int64_t>(t) * N + n);
            else *reinterpret_cast<uint4*>(dst) = make_uint4(0, 0, 0, 0);
        }
        cp_async_wait_all();
        __syncthreads();
        const uint16_t* y0 = sY + g * kVYStride + 2 * q;
        const uint16_t* y8 = y0 + 8 * kVYStride;
        const int mi = lane >> 3, li = lane & 7;  // ldmatrix.x2: matrix mi (rows 8 mi .. 8 mi + 7 of the chunk)
#pragma unroll 4
        for (int c = warp; c < nn / 16; c += 4) {
            const int k = 16 * c;
            const uint32_t a0 = *reinterpret_cast<const uint32_t*>(y0 + k), a1 = *reinterpret_cast<const uint32_t*>(y8 + k);
            const uint32_t a2 = *reinterpret_cast<const uint32_t*>(y0 + k + 8), a3 = *reinterpret_cast<const uint32_t*>(y8 + k + 8);
            const uint32_t brow = smem_u32(sB + (k + 8 * (mi & 1) + li) * kVBStride);
            uint32_t b0, b1, c0, c1;
            ldmatrix_x2_trans(brow, b0, b1);        // columns j0 .. j0 + 7
            ldmatrix_x2_trans(brow + 16, c0, c1);   // columns j0 + 8 .. j0 + 15
            mma_m16n8k16(acc[0], a0, a1, a2, a3, b0, b1);
            mma_m16n8k16(acc[1], a0, a1, a2, a3, c0, c1);
        }
    }

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
    cluster_sync_all();
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
            uint16_t* row = V2 + static_cast<int64_t>(t) * 2 * r64;
            if (j < r64) store_split(row + j, row + r64 + j, j < r ? v : 0.0f);
        }
    }
    cluster_sync_all();
}

}  // namespace

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
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 1;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = splits;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    TraceScope trace("few_lora_down", stream);
    return cudaLaunchKernelEx(&cfg, k_few_down, X, A, M, K, r, r64, s, T2, T_saved);
}

cudaError_t launch_few_v(const uint16_t* dY, const uint16_t* B, int M, int N, int r, int r64, float s,
                         uint16_t* V2, cudaStream_t stream) {
    if (M < 1 || M > kMaxFewTokens || N % 8 != 0 || r % 8 != 0 || r64 > 256) return cudaErrorInvalidValue;
    static bool configured[64] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64 || !configured[dev]) {
        e = cudaFuncSetAttribute(k_few_v, cudaFuncAttributeMaxDynamicSharedMemorySize, kVSmem);
        if (e != cudaSuccess) return e;
        // the dependent kernel's shared-memory carveout (see launch_few_down)
        e = cudaFuncSetAttribute(k_few_v, cudaFuncAttributePreferredSharedMemoryCarveout,
                                 cudaSharedmemCarveoutMaxShared);
        if (e != cudaSuccess) return e;
        if (dev >= 0 && dev < 64) configured[dev] = true;
    }
    const int splits = std::max(1, std::min(kDownMaxSplit, (N + 15) / 16));
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(r64 / 16, 1, splits);
    cfg.blockDim = dim3(kDownThreads);
    cfg.dynamicSmemBytes = kVSmem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 1;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = splits;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    TraceScope trace("few_lora_v", stream);
    return cudaLaunchKernelEx(&cfg, k_few_v, dY, B, M, N, r, r64, s, V2);
}

}  // namespace nf4lora
