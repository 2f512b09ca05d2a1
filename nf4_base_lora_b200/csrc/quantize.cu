// NF4 + double-quantisation encoder and the materialising decoder.
//
// Encoding of one fp32 weight ("第 04 篇：QLoRA 原理" §3.4, §4.3, §5.2; the
// compassingai.com QLoRA page, "NF4 量化機制詳解"), three launches:
//   k_nf4_encode   per 64-block: absmax (half-warp shuffle reduction), IEEE
//                  divide, nearest-level code, nibble packing; per tile of 256
//                  blocks: the fp64 pairwise-tree partial sum of the absmax.
//   k_dq_mean      fp64 pairwise tree over the tile sums -> mean (1 CTA).
//   k_dq_quantize  per group of 256 scales: max |a - mean| and the int8 codes.
// HBM-bound: 4 bytes read and ~0.52 bytes written per weight.
#include <cstdint>

#include "common.cuh"
#include "kernels.h"
#include "nf4_levels.cuh"
#include "trace.h"

namespace nf4lora {

namespace {

constexpr int kTileBlocks = 256;  // = one double-quantisation group

// Code of x: the number of thresholds m_j (ascending, j = 0..14) strictly
// below x, by a 4-step binary search over the thresholds held in shared memory
// (m[15] = +inf pads the table).
__device__ __forceinline__ uint32_t nf4_code(float x, const float* m) {
    uint32_t i = (x > m[7]) ? 8u : 0u;
    i += (x > m[i + 3]) ? 4u : 0u;
    i += (x > m[i + 1]) ? 2u : 0u;
    i += (x > m[i]) ? 1u : 0u;
    return i;
}

__global__ void __launch_bounds__(256) k_nf4_encode(const float* __restrict__ W, int64_t n_blocks,
                                                   uint8_t* __restrict__ codes,
                                                   float* __restrict__ absmax,
                                                   double* __restrict__ tile_sums) {
    __shared__ float s_mid[16];
    __shared__ double s_sum[kTileBlocks];
    const int tid = threadIdx.x;
    if (tid < 15) {
        s_mid[tid] = __fmul_rn(__fadd_rn(nf4_level(tid), nf4_level(tid + 1)), 0.5f);
    } else if (tid == 15) {
        s_mid[15] = __int_as_float(0x7f800000);
    }
    __syncthreads();
    const int lane = tid & 31, warp = tid >> 5;
    const int half = lane >> 4, sub = lane & 15;
    const int64_t n_tiles = (n_blocks + kTileBlocks - 1) / kTileBlocks;

    for (int64_t tile = blockIdx.x; tile < n_tiles; tile += gridDim.x) {
        // warp w owns blocks [32w, 32w + 32) of the tile, two per step
#pragma unroll 4
        for (int it = 0; it < 16; ++it) {
            const int local = warp * 32 + it * 2 + half;
            const int64_t b = tile * kTileBlocks + local;
            float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
            const bool valid = b < n_blocks;
            if (valid) v = __ldcs(reinterpret_cast<const float4*>(W + b * 64) + sub);
            float a = fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w)));
#pragma unroll
            for (int o = 8; o >= 1; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
            uint32_t c0 = 7, c1 = 7, c2 = 7, c3 = 7;
            if (a != 0.0f) {
                c0 = nf4_code(__fdiv_rn(v.x, a), s_mid);
                c1 = nf4_code(__fdiv_rn(v.y, a), s_mid);
                c2 = nf4_code(__fdiv_rn(v.z, a), s_mid);
                c3 = nf4_code(__fdiv_rn(v.w, a), s_mid);
            }
            if (valid) {
                // byte k holds (even element << 4) | odd element
                const uint16_t packed =
                    static_cast<uint16_t>(((c0 << 4) | c1) | (((c2 << 4) | c3) << 8));
                reinterpret_cast<uint16_t*>(codes + b * 32)[sub] = packed;
                if (sub == 0) absmax[b] = a;
            }
            if (sub == 0) s_sum[local] = valid ? static_cast<double>(a) : 0.0;
        }
        __syncthreads();
        // fp64 pairwise tree over the tile's 256 scales (zero-padded: x + 0 == x
        // keeps the carried-up elements of a short tail unchanged)
        for (int stride = 1; stride < kTileBlocks; stride <<= 1) {
            const int idx = tid * 2 * stride;
            if (idx < kTileBlocks) s_sum[idx] = __dadd_rn(s_sum[idx], s_sum[idx + stride]);
            __syncthreads();
        }
        if (tid == 0) tile_sums[tile] = s_sum[0];
        __syncthreads();
    }
}

// One CTA: pairwise tree over the tile sums (zero-padded to a power of two,
// processed in aligned segments of 2048), then mean = fp32(sum / n_b).
__global__ void __launch_bounds__(1024) k_dq_mean(const double* __restrict__ tile_sums,
                                                  int64_t n_tiles, int64_t n_blocks,
                                                  float* __restrict__ mean_out) {
    constexpr int kSeg = 2048;
    __shared__ double s[kSeg];
    __shared__ double s_segs[kSeg];
    const int tid = threadIdx.x;
    const int64_t n_segs = (n_tiles + kSeg - 1) / kSeg;  // <= kSeg for any supported size
    for (int64_t seg = 0; seg < n_segs; ++seg) {
        for (int i = tid; i < kSeg; i += blockDim.x) {
            const int64_t g = seg * kSeg + i;
            s[i] = g < n_tiles ? tile_sums[g] : 0.0;
        }
        __syncthreads();
        for (int stride = 1; stride < kSeg; stride <<= 1) {
            for (int idx = tid * 2 * stride; idx < kSeg; idx += blockDim.x * 2 * stride)
                s[idx] = __dadd_rn(s[idx], s[idx + stride]);
            __syncthreads();
        }
        if (tid == 0) s_segs[seg] = s[0];
        __syncthreads();
    }
    for (int i = tid; i < kSeg; i += blockDim.x)
        if (i >= n_segs) s_segs[i] = 0.0;
    __syncthreads();
    int width = 1;
    while (width < n_segs) width <<= 1;
    for (int stride = 1; stride < width; stride <<= 1) {
        for (int idx = tid * 2 * stride; idx < width; idx += blockDim.x * 2 * stride)
            s_segs[idx] = __dadd_rn(s_segs[idx], s_segs[idx + stride]);
        __syncthreads();
    }
    if (tid == 0) *mean_out = __double2float_rn(__ddiv_rn(s_segs[0], static_cast<double>(n_blocks)));
}

// One warp per group of 256 first-level scales; lane l owns scales
// [8l, 8l + 8) of the group.
__global__ void __launch_bounds__(256) k_dq_quantize(const float* __restrict__ absmax,
                                                    int64_t n_blocks,
                                                    const float* __restrict__ mean_ptr,
                                                    int8_t* __restrict__ qscale,
                                                    float* __restrict__ scale2) {
    const int lane = threadIdx.x & 31;
    const int64_t g = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
    const int64_t n_groups = (n_blocks + kTileBlocks - 1) / kTileBlocks;
    if (g >= n_groups) return;
    const float mu = *mean_ptr;
    const int64_t b0 = g * kTileBlocks + lane * 8;
    float d[8];
    float m = 0.0f;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const int64_t b = b0 + i;
        d[i] = b < n_blocks ? __fsub_rn(absmax[b], mu) : 0.0f;
        m = fmaxf(m, fabsf(d[i]));
    }
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if (lane == 0) scale2[g] = m;
    int8_t q[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        float r = 0.0f;
        if (m != 0.0f) {
            r = rintf(__fmul_rn(__fdiv_rn(d[i], m), 127.0f));
            r = fminf(fmaxf(r, -127.0f), 127.0f);
        }
        q[i] = static_cast<int8_t>(r);
    }
    if (b0 + 8 <= n_blocks) {
        uint2 packed;
        packed.x = (uint32_t(uint8_t(q[0]))) | (uint32_t(uint8_t(q[1])) << 8) |
                   (uint32_t(uint8_t(q[2])) << 16) | (uint32_t(uint8_t(q[3])) << 24);
        packed.y = (uint32_t(uint8_t(q[4]))) | (uint32_t(uint8_t(q[5])) << 8) |
                   (uint32_t(uint8_t(q[6])) << 16) | (uint32_t(uint8_t(q[7])) << 24);
        *reinterpret_cast<uint2*>(qscale + b0) = packed;
    } else {
        for (int i = 0; i < 8; ++i)
            if (b0 + i < n_blocks) qscale[b0 + i] = q[i];
    }
}

// Materialising decoder: each thread decodes 16 weights (8 code bytes) of one
// block; w_hat = bf16_rne(level[code] * s_b).
__global__ void __launch_bounds__(256) k_nf4_dequantize(const uint8_t* __restrict__ codes,
                                                       const int8_t* __restrict__ qscale,
                                                       const float* __restrict__ scale2,
                                                       const float* __restrict__ mean_ptr,
                                                       int64_t n, uint16_t* __restrict__ out) {
    __shared__ float s_lut[16];
    if (threadIdx.x < 16) s_lut[threadIdx.x] = nf4_level(threadIdx.x);
    __syncthreads();
    const float mu = *mean_ptr;
    const int64_t n_units = n / 16;
    for (int64_t u = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; u < n_units;
         u += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int64_t b = u >> 2;  // 4 units per 64-block
        const float s = nf4_block_scale(qscale[b], scale2[b >> 8], mu);
        const uint2 c = __ldcs(reinterpret_cast<const uint2*>(codes) + u);
        uint32_t o[8];
#pragma unroll
        for (int w = 0; w < 2; ++w) {
            const uint32_t x = w == 0 ? c.x : c.y;
#pragma unroll
            for (int byte = 0; byte < 4; ++byte) {
                const uint32_t hi = (x >> (8 * byte + 4)) & 15u, lo = (x >> (8 * byte)) & 15u;
                o[w * 4 + byte] = pack_bf16x2(__fmul_rn(s_lut[hi], s), __fmul_rn(s_lut[lo], s));
            }
        }
        uint4* dst = reinterpret_cast<uint4*>(out + u * 16);
        __stcs(dst, make_uint4(o[0], o[1], o[2], o[3]));
        __stcs(dst + 1, make_uint4(o[4], o[5], o[6], o[7]));
    }
}

}  // namespace

static cudaLaunchConfig_t config(int64_t grid, int block, cudaStream_t stream) {
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(static_cast<unsigned>(grid));
    cfg.blockDim = dim3(block);
    cfg.stream = stream;
    return cfg;
}

cudaError_t launch_nf4_quantize(const float* W, int64_t n, uint8_t* codes, int8_t* qscale,
                                float* scale2, float* scale_mean, float* ws_absmax,
                                double* ws_tile_sums, int num_sms, cudaStream_t stream) {
    const int64_t n_blocks = n / 64;
    const int64_t n_tiles = (n_blocks + kTileBlocks - 1) / kTileBlocks;
    const int64_t grid1 = n_tiles < int64_t(num_sms) * 8 ? n_tiles : int64_t(num_sms) * 8;
    cudaError_t e;
    {
        TraceScope trace("nf4_encode", stream);
        cudaLaunchConfig_t cfg = config(grid1, 256, stream);
        e = cudaLaunchKernelEx(&cfg, k_nf4_encode, W, n_blocks, codes, ws_absmax, ws_tile_sums);
        if (e != cudaSuccess) return e;
    }
    {
        TraceScope trace("dq_mean", stream);
        cudaLaunchConfig_t cfg = config(1, 1024, stream);
        e = cudaLaunchKernelEx(&cfg, k_dq_mean, static_cast<const double*>(ws_tile_sums), n_tiles, n_blocks,
                               scale_mean);
        if (e != cudaSuccess) return e;
    }
    {
        TraceScope trace("dq_quantize", stream);
        cudaLaunchConfig_t cfg = config((n_tiles + 7) / 8, 256, stream);
        e = cudaLaunchKernelEx(&cfg, k_dq_quantize, static_cast<const float*>(ws_absmax), n_blocks,
                               static_cast<const float*>(scale_mean), qscale, scale2);
    }
    return e;
}

cudaError_t launch_nf4_dequantize(const uint8_t* codes, const int8_t* qscale, const float* scale2,
                                  const float* scale_mean, int64_t n, uint16_t* out, int num_sms,
                                  cudaStream_t stream) {
    const int64_t units = n / 16;
    int64_t grid = (units + 255) / 256;
    if (grid > int64_t(num_sms) * 16) grid = int64_t(num_sms) * 16;
    TraceScope trace("nf4_dequantize", stream);
    cudaLaunchConfig_t cfg = config(grid, 256, stream);
    return cudaLaunchKernelEx(&cfg, k_nf4_dequantize, codes, qscale, scale2, scale_mean, n, out);
}

}  // namespace nf4lora
