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
// rows (codes and block scales fetched into shared memory at the start).
// The bf16 rows of the next slice travel by 16-byte asynchronous
// copies into a staging buffer while the current slice is multiplied, so the
// fp64 pipe does not wait for global loads between slices (B's rows are
// copied this way when r is a multiple of 8, which makes every row of B start
// on 16 bytes; otherwise B is read element by element at each slice).
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

__device__ __forceinline__ void cp_async16(void* smem_dst, const void* src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(smem_dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }

// VEC_B: r is a multiple of 8, so the 8-rank pieces of B's rows start on 16 bytes.
template <bool VEC_B>
__global__ void __launch_bounds__(256, 2) k_merge_lora(const uint8_t* __restrict__ codes,
                                                      const int8_t* __restrict__ qscale,
                                                      const float* __restrict__ scale2,
                                                      const float* __restrict__ scale_mean,
                                                      const float* __restrict__ absmax,
                                                      const uint16_t* __restrict__ A, const uint16_t* __restrict__ B,
                                                      int r, int64_t N, int64_t K, float s,
                                                      float* __restrict__ out) {
    __shared__ __align__(16) double sA[kMergeRanks][kMergeCols];  // A[j0 + jj][k0 + c]
    __shared__ __align__(16) double sB[kMergeRanks][kMergeRows];  // B[n0 + rr][j0 + jj], transposed
    __shared__ __align__(16) uint16_t stA[kMergeRanks][kMergeCols];  // bf16 staging of the next slice of A
    __shared__ __align__(16) uint16_t stB[kMergeRows][kMergeRanks];  // and of B (VEC_B only), row-major
    __shared__ __align__(16) uint8_t s_codes[kMergeRows][kMergeCols / 2];  // the tile's codes
    __shared__ float s_sc[kMergeRows];  // fp32 scale of each row's block
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
    // staging roles: threads 0..127 copy one 16-byte piece of A (rank row
    // tid / 8, columns 8 (tid % 8) ..), every thread one 8-rank piece of B
    // (row tid % 128, ranks 8 (tid / 128) ..)
    const int a_jj = tid >> 3, a_c = 8 * (tid & 7);
    const int b_rr = tid & 127, b_h = tid >> 7;

    // copies of the slice that starts at rank j0 into the staging buffers;
    // rank rows at or past r, and rows of B at or past N, are not copied (the
    // conversion below writes zeros for them)
    auto stage = [&](int j0) {
        if (tid < 128 && j0 + a_jj < r) cp_async16(&stA[a_jj][a_c], A + static_cast<int64_t>(j0 + a_jj) * K + k0 + a_c);
        if (VEC_B && n0 + b_rr < N && j0 + 8 * b_h < r)
            cp_async16(&stB[b_rr][8 * b_h], B + (n0 + b_rr) * r + j0 + 8 * b_h);
        cp_async_commit();
    };

    double acc[8][4];
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int c = 0; c < 4; ++c) acc[i][c] = 0.0;

    // the epilogue's inputs come in with the first slice: the tile's codes
    // (32 bytes of each row, in the first slice's copy group) and each row's
    // block scale
    const int64_t bpr = K / 64, blk = k0 / 64;
    {
        const int rr = tid >> 1, h = tid & 1;
        if (n0 + rr < N) cp_async16(&s_codes[rr][16 * h], codes + ((n0 + rr) * K + k0) / 2 + 16 * h);
    }
    if (tid < kMergeRows) {
        const int64_t n = n0 + tid;
        float sc = 0.0f;
        if (n < N) {
            const int64_t bi = n * bpr + blk;
            sc = absmax ? absmax[bi] : nf4_block_scale(qscale[bi], scale2[bi >> 8], *scale_mean);
        }
        s_sc[tid] = sc;
    }
    stage(0);
    for (int j0 = 0; j0 < r; j0 += kMergeRanks) {
        const int nj = min(kMergeRanks, r - j0);
        cp_async_wait_all();
        __syncthreads();  // the staged slice is visible, and the previous slice is no longer read
        {
            // A: 4 consecutive columns of one rank row per thread
            const int jj = tid >> 4, c = 4 * (tid & 15);
            const uint2 v = *reinterpret_cast<const uint2*>(&stA[jj][c]);
            const bool live = jj < nj;
            const double2 lo = make_double2(live ? static_cast<double>(bf16_bits_to_float(v.x & 0xffffu)) : 0.0,
                                            live ? static_cast<double>(bf16_bits_to_float(v.x >> 16)) : 0.0);
            const double2 hi = make_double2(live ? static_cast<double>(bf16_bits_to_float(v.y & 0xffffu)) : 0.0,
                                            live ? static_cast<double>(bf16_bits_to_float(v.y >> 16)) : 0.0);
            *reinterpret_cast<double2*>(&sA[jj][c]) = lo;
            *reinterpret_cast<double2*>(&sA[jj][c + 2]) = hi;
        }
        if (VEC_B) {
            // B: the thread's own 8-rank piece, written transposed
            const uint4 v = *reinterpret_cast<const uint4*>(&stB[b_rr][8 * b_h]);
            const uint32_t w[4] = {v.x, v.y, v.z, v.w};
            const bool row_live = n0 + b_rr < N;
#pragma unroll
            for (int t = 0; t < 8; ++t) {
                const int jj = 8 * b_h + t;
                const uint32_t bits = (t & 1) ? (w[t >> 1] >> 16) : (w[t >> 1] & 0xffffu);
                sB[jj][b_rr] = (row_live && jj < nj) ? static_cast<double>(bf16_bits_to_float(bits)) : 0.0;
            }
        } else {
            for (int i = tid; i < kMergeRanks * kMergeRows; i += 256) {
                const int jj = i / kMergeRows, rr = i % kMergeRows;  // consecutive lanes: consecutive rows
                const int64_t n = n0 + rr;
                sB[jj][rr] = (jj < nj && n < N) ? static_cast<double>(bf16_bits_to_float(B[n * r + j0 + jj])) : 0.0;
            }
        }
        __syncthreads();  // sA / sB hold the slice; the staging buffers are free
        if (j0 + kMergeRanks < r) stage(j0 + kMergeRanks);  // lands while this slice is multiplied
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
    const double sd = static_cast<double>(s);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const int64_t n = n0 + rb + i;
        if (n >= N) break;
        const float sc = s_sc[rb + i];
        // codes of elements k0 + cb, + 1 and k0 + 32 + cb, + 1 of row n: one byte
        // each, the even element in the high nibble
        const uint8_t* row = s_codes[rb + i];
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
    if (r % 8 == 0)
        return cudaLaunchKernelEx(&cfg, k_merge_lora<true>, codes, qscale, scale2, scale_mean, absmax, A, B, r, N, K, s,
                                  out);
    return cudaLaunchKernelEx(&cfg, k_merge_lora<false>, codes, qscale, scale2, scale_mean, absmax, A, B, r, N, K, s,
                              out);
}

}  // namespace nf4lora
