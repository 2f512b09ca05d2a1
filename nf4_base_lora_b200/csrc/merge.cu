// Adapter merge for deployment ("第 04 篇：QLoRA 原理" §12.3: fold the adapter
// into the base, W + s B A, then encode the result again; §12.4: the
// effective weight is the dequantised base plus the adapter):
//
//   W'[n, k] = fp32( W_hat[n, k] + s * sum_j B[n, j] A[j, k] )
//
// W_hat is the bf16 dequantisation of the stored encoding (the fp32 original
// is gone).  Each product of two bf16 values is exact in fp64; the rank-r sum
// runs in fp64 in ascending j (a fused multiply-add per term, which rounds
// exactly like an addition of the exact product), then one fp64 multiply by
// s, one fp64 add of W_hat and one rounding to fp32.  Every step is IEEE and
// in a fixed order, so W' is bit-for-bit the stated value.
//
// The fp64 multiply-adds bound the kernel (n * r of them against 4.5 bytes
// of memory traffic per weight).  A CTA computes a 128 x 64 tile of W': the
// factor slices of 16 ranks at a time are staged in shared memory as fp64
// (B transposed), and each thread keeps 8 rows x 4 columns of fp64 sums; the
// epilogue decodes the tile's codes (one 64-block per row) and writes fp32
// rows.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "common.cuh"
#include "kernels.h"
#include "nf4_levels.cuh"
#include "trace.h"

namespace nf4lora {

namespace {

constexpr int kMergeRows = 128;  // rows n per CTA
constexpr int kMergeCols = 64;   // columns k per CTA: one 64-block of each row
constexpr int kMergeRanks = 16;  // ranks j per staged slice

__global__ void __launch_bounds__(256) k_merge_lora(const uint8_t* __restrict__ codes,
                                                   const int8_t* __restrict__ qscale,
                                                   const float* __restrict__ scale2,
                                                   const float* __restrict__ scale_mean,
                                                   const float* __restrict__ absmax,
                                                   const uint16_t* __restrict__ A, const uint16_t* __restrict__ B,
                                                   int r, int64_t N, int64_t K, float s,
                                                   float* __restrict__ out) {
    __shared__ __align__(16) double sA[kMergeRanks][kMergeCols];  // A[j0 + jj][k0 + c]
    __shared__ __align__(16) double sB[kMergeRanks][kMergeRows];  // B[n0 + rr][j0 + jj], transposed
    __shared__ float s_lvl[16];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    if (tid < 16) s_lvl[tid] = nf4_level(tid);
    const int ty = lane >> 4, tx = lane & 15;
    const int64_t n0 = static_cast<int64_t>(blockIdx.y) * kMergeRows;
    const int64_t k0 = static_cast<int64_t>(blockIdx.x) * kMergeCols;
    const int rb = 16 * warp + 8 * ty;  // this thread's first row in the tile (8 rows)
    // this thread's columns: 2 tx, 2 tx + 1 and 32 + 2 tx, 33 + 2 tx, so that the
    // 16-byte reads of eight consecutive lanes cover 128 contiguous bytes
    const int cb = 2 * tx;

    double acc[8][4];
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int c = 0; c < 4; ++c) acc[i][c] = 0.0;

    for (int j0 = 0; j0 < r; j0 += kMergeRanks) {
        const int nj = min(kMergeRanks, r - j0);
        __syncthreads();  // the previous slice is no longer read
        for (int i = tid; i < kMergeRanks * kMergeCols; i += 256) {
            const int jj = i / kMergeCols, c = i % kMergeCols;
            sA[jj][c] = jj < nj ? static_cast<double>(bf16_bits_to_float(A[static_cast<int64_t>(j0 + jj) * K + k0 + c]))
                                : 0.0;
        }
        for (int i = tid; i < kMergeRanks * kMergeRows; i += 256) {
            const int jj = i / kMergeRows, rr = i % kMergeRows;  // consecutive lanes: consecutive rows (no conflicts)
            const int64_t n = n0 + rr;
            sB[jj][rr] = (jj < nj && n < N) ? static_cast<double>(bf16_bits_to_float(B[n * r + j0 + jj])) : 0.0;
        }
        __syncthreads();
        for (int jj = 0; jj < nj; ++jj) {
            const double2 a01 = *reinterpret_cast<const double2*>(&sA[jj][cb]);
            const double2 a23 = *reinterpret_cast<const double2*>(&sA[jj][32 + cb]);
            const double a[4] = {a01.x, a01.y, a23.x, a23.y};
            double b[8];
#pragma unroll
            for (int i = 0; i < 8; i += 2) {
                const double2 t = *reinterpret_cast<const double2*>(&sB[jj][rb + i]);
                b[i] = t.x;
                b[i + 1] = t.y;
            }
#pragma unroll
            for (int i = 0; i < 8; ++i)
#pragma unroll
                for (int c = 0; c < 4; ++c) acc[i][c] = __fma_rn(b[i], a[c], acc[i][c]);
        }
    }

    // epilogue: W_hat of the tile's block in each row, then the merged value
    const float mu = absmax ? 0.0f : *scale_mean;
    const int64_t bpr = K / 64, blk = k0 / 64;
    const double sd = static_cast<double>(s);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const int64_t n = n0 + rb + i;
        if (n >= N) break;
        const int64_t bi = n * bpr + blk;
        const float sc = absmax ? absmax[bi] : nf4_block_scale(qscale[bi], scale2[bi >> 8], mu);
        // codes of elements k0 + cb, + 1 and k0 + 32 + cb, + 1 of row n: one byte
        // each, the even element in the high nibble
        const uint8_t* row = codes + (n * K + k0) / 2;
        const uint32_t b0 = row[cb / 2], b1 = row[16 + cb / 2];
        const uint32_t code[4] = {b0 >> 4, b0 & 15u, b1 >> 4, b1 & 15u};
        float o[4];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            const float w_hat = __bfloat162float(__float2bfloat16_rn(__fmul_rn(s_lvl[code[c]], sc)));
            o[c] = __double2float_rn(__dadd_rn(static_cast<double>(w_hat), __dmul_rn(sd, acc[i][c])));
        }
        *reinterpret_cast<float2*>(out + n * K + k0 + cb) = make_float2(o[0], o[1]);
        *reinterpret_cast<float2*>(out + n * K + k0 + 32 + cb) = make_float2(o[2], o[3]);
    }
}

}  // namespace

cudaError_t launch_merge_lora(const uint8_t* codes, const int8_t* qscale, const float* scale2,
                              const float* scale_mean, const float* absmax, const uint16_t* A, const uint16_t* B,
                              int r, int64_t N, int64_t K, float s, float* out, cudaStream_t stream) {
    if (N < 1 || K < 64 || K % 64 != 0 || r < 1) return cudaErrorInvalidValue;
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(static_cast<unsigned>(K / kMergeCols), static_cast<unsigned>((N + kMergeRows - 1) / kMergeRows));
    cfg.blockDim = dim3(256);
    cfg.stream = stream;
    TraceScope trace("nf4_merge_lora", stream);
    return cudaLaunchKernelEx(&cfg, k_merge_lora, codes, qscale, scale2, scale_mean, absmax, A, B, r, N, K, s, out);
}

}  // namespace nf4lora
