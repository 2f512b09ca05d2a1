// NF4 + double-quantisation encoder and the materialising decoder.
//
// Without double quantisation ("第 04 篇" §5.1: one fp32 scale per block of
// 64, 0.5 bit per weight) only k_nf4_encode runs, writing the fp32 absmax of
// every block as the stored scale.
//
// Encoding of one fp32 weight ("第 04 篇：QLoRA 原理" §3.4, §4.3, §5.2; the
// compassingai.com QLoRA page, "NF4 量化機制詳解"), three launches:
//   k_nf4_encode   per 64-block: absmax (quad shuffle reduction), nearest-level
//                  code, nibble packing; per run of 32 blocks (one warp's part
//                  of a tile of 256): the fp64 pairwise-tree partial sum.
//   k_dq_mean      the rest of the fp64 pairwise tree -> mean (1 CTA).
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

// The pairwise tree over the 32 lanes' values (level l adds lane pairs
// 2^l apart within aligned runs): lane 0 returns the sum of the run.
__device__ __forceinline__ double pairwise_warp(double v) {
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const double u = __shfl_down_sync(0xffffffffu, v, o);
        if ((threadIdx.x & (2 * o - 1)) == 0) v = __dadd_rn(v, u);
    }
    return v;
}

// Code of x = w / a (IEEE fp32 division): the number of thresholds m_j
// (ascending, j = 0..14, m_j = (level_j + level_j+1) / 2) strictly below x.
__device__ __noinline__ uint32_t nf4_code_exact(float w, float a, const float* m) {
    const float x = __fdiv_rn(w, a);
    uint32_t c = 0;
#pragma unroll
    for (int j = 0; j < 15; ++j) c += x > m[j] ? 1u : 0u;
    return c;
}

// The code without the division, for a normal absmax a: x' = w * fl(1/a)
// lies within 2 ulp of fl(w / a).  Bucket b (0..31) covers [-1 + b/16,
// -1 + (b+1)/16): the thresholds are more than 1/16 apart and none lies within
// 1e-3 of a bucket edge, so each bucket holds at most one threshold thr (if
// none, take any value above 1) above `base` others, and base + (x > thr) is
// the code of every x in the bucket or within rounding distance of it.  The bucket index is
// floor(16 x' + 16): one fused multiply-add adds 1.5 * 2^23 + 16 (an integer,
// exact in fp32, where the fp32 spacing is 1) and rounds toward -inf, so the
// low bits of the result are exactly that floor; -1 and 32, reachable only by
// rounding at x' = -1 and +1, index copies of buckets 0 and 31 (table entries
// 63 and 32).
// A table entry is one 32-bit word, so the 32 lanes of a warp never meet on a
// bank unless they read the same entry: the fp32 threshold with its low four
// mantissa bits replaced by `base` (a change of less than 16 ulp, under 1e-6
// for |thr| < 1), or 2.0 with `base` in those bits for a bucket without one.
// Where x' falls within 2e-6 of that value the exact division decides (the
// true threshold is within 1e-6 of it and x' within 2.4e-7 of fl(w / a)), so
// the result is always the code of fl(w / a).

// Paired fp32 instructions (two lanes of one register pair, each rounded as
// its scalar form).
__device__ __forceinline__ uint64_t f2_pack(float lo, float hi) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}
__device__ __forceinline__ void f2_unpack(uint64_t v, float& lo, float& hi) {
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t f2_mul_rn(uint64_t a, uint64_t b) {
    uint64_t r;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}
__device__ __forceinline__ uint64_t f2_fma_rm(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t r;
    asm("fma.rm.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
    return r;
}
__device__ __forceinline__ uint64_t f2_sub_rn(uint64_t a, uint64_t b) {
    uint64_t r;
    asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}

// The code of two weights by the method above, with the multiplies, the
// bucket FMA and the threshold differences done as paired instructions (the
// same roundings as their scalar forms).
__device__ __forceinline__ void nf4_code_fast2(float w0, float w1, uint64_t rinv2, const uint32_t* bkt,
                                               bool& unsure, uint32_t& c0, uint32_t& c1) {
    constexpr uint64_t k16 = 0x4180000041800000ull;    // (16, 16)
    constexpr uint64_t kOff = 0x4B4000104B400010ull;   // (1.5 * 2^23 + 16) twice
    const uint64_t x2 = f2_mul_rn(f2_pack(w0, w1), rinv2);
    float t0, t1, x0, x1;
    f2_unpack(f2_fma_rm(x2, k16, kOff), t0, t1);
    f2_unpack(x2, x0, x1);
    const uint32_t e0 = bkt[__float_as_int(t0) & 63], e1 = bkt[__float_as_int(t1) & 63];
    const float thr0 = __uint_as_float(e0), thr1 = __uint_as_float(e1);
    float d0, d1;
    f2_unpack(f2_sub_rn(x2, f2_pack(thr0, thr1)), d0, d1);
    unsure |= fabsf(d0) <= 2.0e-6f;
    unsure |= fabsf(d1) <= 2.0e-6f;
    c0 = (e0 & 15u) + (x0 > thr0 ? 1u : 0u);
    c1 = (e1 & 15u) + (x1 > thr1 ? 1u : 0u);
}

// Four lanes per 64-block, eight blocks (a "unit") per warp step: lane
// (g, s) of the warp holds four 16-byte pieces of block g, pieces
// (s + 4 (k + (g & 1))) mod 16 for k = 0..3, so each load instruction of a
// warp reads eight whole 64-byte runs, and the absmax needs two shuffle
// levels.  A CTA of 8 warps takes one tile of 256 blocks: warp w its blocks
// [32 w, 32 w + 32), one unit per step, four steps; the loop over units is
// unrolled by two, so each warp has two units of loads in flight.
//
// The fp64 pairwise tree of the absmax values runs per warp: a warp's 32
// blocks of a tile are one aligned run of the tree, whose five levels it adds
// with shuffles (three across its eight block groups, two over its four
// steps); the warp's sum goes to warp_sums[8 tile + warp], and the mean kernel
// adds the three levels above.  No warp ever waits for another, so each
// streams its blocks at its own pace.
__global__ void __launch_bounds__(256, 3) k_nf4_encode(const float* __restrict__ W, int64_t n_blocks,
                                                   uint8_t* __restrict__ codes,
                                                   float* __restrict__ absmax,
                                                   double* __restrict__ warp_sums,
                                                   unsigned int* __restrict__ mean_ticket) {
    __shared__ float s_mid[16];
    __shared__ uint32_t s_bkt[64];
    const int tid = threadIdx.x;
    const int lane = tid & 31, warp = tid >> 5;
    const int grp = lane >> 2, sub = lane & 3;
    if (mean_ticket != nullptr && blockIdx.x == 0 && tid == 0) *mean_ticket = 0u;  // for the mean kernel after this one
    pdl_launch_dependents();  // the mean kernel may take an SM as soon as one frees; it waits for this grid
    if (tid < 15) {
        s_mid[tid] = __fmul_rn(__fadd_rn(nf4_level(tid), nf4_level(tid + 1)), 0.5f);
    } else if (tid >= 64 && tid < 128) {
        const int idx = tid - 64;
        const int bi = idx < 32 ? idx : (idx == 32 ? 31 : 0);  // 32: rounding above +1; 63: below -1
        const float lo = -1.0f + 0.0625f * static_cast<float>(bi), hi = lo + 0.0625f;
        float thr = 2.0f;
        uint32_t base = 0;
        for (int j = 0; j < 15; ++j) {
            const float m = __fmul_rn(__fadd_rn(nf4_level(j), nf4_level(j + 1)), 0.5f);
            if (m < lo) ++base;
            else if (m < hi) thr = m;
        }
        s_bkt[idx] = (__float_as_uint(thr) & ~15u) | base;
    }
    __syncthreads();  // the tables (the only CTA-wide wait)

    const int64_t n_tiles = (n_blocks + kTileBlocks - 1) / kTileBlocks;
    // the warp's units: u = 4 k + it is step it of tile blockIdx.x + k gridDim.x
    const int64_t tiles_here = blockIdx.x < n_tiles ? (n_tiles - 1 - blockIdx.x) / gridDim.x + 1 : 0;
    const uint32_t n_u = static_cast<uint32_t>(4 * tiles_here);
    const int64_t tile_step = static_cast<int64_t>(gridDim.x) * kTileBlocks;
    int pc[4];  // the lane's pieces
#pragma unroll
    for (int k = 0; k < 4; ++k) pc[k] = (sub + 4 * (k + (grp & 1))) & 15;
    double run_lo = 0.0, run = 0.0;  // levels 4 and 5 of the warp's run
    int64_t b0 = static_cast<int64_t>(blockIdx.x) * kTileBlocks + warp * 32;  // first block of unit u
#pragma unroll 2
    for (uint32_t u = 0; u < n_u; ++u) {
        const int it = static_cast<int>(u & 3);
        const int64_t b = b0 + grp;
        const bool valid = b < n_blocks;
        {
            // ask L2 for the same unit of this CTA's next tile (four units
            // ahead): lane l < 16 one 128-byte line of it, so the loads that
            // follow there find their lines in L2
            const int64_t pb = b0 + tile_step + (lane >> 1);
            if (lane < 16 && pb < n_blocks)
                asm volatile("prefetch.global.L2 [%0];" ::"l"(W + pb * 64 + (lane & 1) * 32));
        }
        float v[16];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            float4 q = make_float4(0.f, 0.f, 0.f, 0.f);
            if (valid) q = __ldcs(reinterpret_cast<const float4*>(W + b * 64) + pc[k]);
            v[4 * k] = q.x;
            v[4 * k + 1] = q.y;
            v[4 * k + 2] = q.z;
            v[4 * k + 3] = q.w;
        }
        float a = 0.0f;
#pragma unroll
        for (int i = 0; i < 16; ++i) a = fmaxf(a, fabsf(v[i]));
        a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, 1));
        a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, 2));
        // codes: an all-zero block (rinv = 0) lands every weight at x = 0,
        // code 7; an absmax below 1e-37 (1 / a not a normal fp32) takes the
        // exact division
        bool unsure = a != 0.0f && !(a >= 1.0e-37f);
        const float rinv = a >= 1.0e-37f ? __frcp_rn(a) : 0.0f;
        const uint64_t rinv2 = f2_pack(rinv, rinv);
        uint32_t c[16];
#pragma unroll
        for (int i = 0; i < 16; i += 2) nf4_code_fast2(v[i], v[i + 1], rinv2, s_bkt, unsure, c[i], c[i + 1]);
        if (unsure) {  // rare: near a threshold, or a tiny absmax
#pragma unroll
            for (int i = 0; i < 16; ++i) c[i] = nf4_code_exact(v[i], a, s_mid);
        }
        if (valid) {
            // piece p holds elements 4p .. 4p + 3: code bytes 2p, 2p + 1
            // (byte = (even element << 4) | odd element)
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const uint32_t packed = (c[4 * k] << 4) | c[4 * k + 1] | (((c[4 * k + 2] << 4) | c[4 * k + 3]) << 8);
                reinterpret_cast<uint16_t*>(codes + b * 32)[pc[k]] = static_cast<uint16_t>(packed);
            }
            if (sub == 0) absmax[b] = a;
        }
        // the tree (zero-padded: x + 0 == x keeps a short tail's sums
        // unchanged): block it * 8 + grp of the run; levels 1-3 pair the
        // groups grp ^ 1, ^ 2, ^ 4 (lanes 4, 8, 16 apart), levels 4-5 the steps
        double t = valid ? static_cast<double>(a) : 0.0;
        t = __dadd_rn(t, __shfl_xor_sync(0xffffffffu, t, 4));
        t = __dadd_rn(t, __shfl_xor_sync(0xffffffffu, t, 8));
        t = __dadd_rn(t, __shfl_xor_sync(0xffffffffu, t, 16));
        if (it == 0 || it == 2) {
            run_lo = t;
        } else if (it == 1) {
            run = __dadd_rn(run_lo, t);
        } else {
            run = __dadd_rn(run, __dadd_rn(run_lo, t));
            // without double quantisation (warp_sums NULL) there is no mean to form
            if (warp_sums != nullptr && lane == 0) warp_sums[(b0 >> 8) * 8 + warp] = run;
        }
        b0 += it == 3 ? tile_step - 24 : 8;
    }
}

// Sum of tile t from its eight warp sums: the top three levels of the tile's
// tree, ((w0 + w1) + (w2 + w3)) + ((w4 + w5) + (w6 + w7)).
__device__ __forceinline__ double tile_sum(const double* warp_sums, int64_t t) {
    const double2* w = reinterpret_cast<const double2*>(warp_sums + 8 * t);
    const double2 a = __ldcg(w), b = __ldcg(w + 1), c = __ldcg(w + 2), d = __ldcg(w + 3);
    return __dadd_rn(__dadd_rn(__dadd_rn(a.x, a.y), __dadd_rn(b.x, b.y)),
                     __dadd_rn(__dadd_rn(c.x, c.y), __dadd_rn(d.x, d.y)));
}

// The pairwise tree over 2048 values by 1024 threads: level 1 in each thread,
// five in each warp, five in warp 0 over the 32 warp sums.  Value i is
// src[i] (from_warp_sums false) or the sum of tile i (true), zero at or
// beyond `count`.  Returns the sum in thread 0.
__device__ __forceinline__ double pairwise_2048(const double* src, int64_t count, double* s_w,
                                                bool from_warp_sums) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    auto value = [&](int64_t i) {
        if (i >= count) return 0.0;
        return from_warp_sums ? tile_sum(src, i) : __ldcg(src + i);
    };
    const double x0 = value(2 * tid);
    const double x1 = value(2 * tid + 1);
    double v = pairwise_warp(__dadd_rn(x0, x1));
    if (lane == 0) s_w[warp] = v;
    __syncthreads();
    if (warp == 0) v = pairwise_warp(s_w[lane]);
    __syncthreads();  // s_w is free again
    return v;
}

// One CTA of 1024 threads per aligned segment of 2048 tiles: the pairwise
// tree over the segment's tile sums (each formed from the encoder's eight warp
// sums; zero-padded to a power of two), written to seg_sums; the CTA that
// finishes last (by a ticket the encoder reset to 0) adds the segment sums
// with the same tree and writes mean = fp32(sum / n_b).
constexpr int kSeg = 2048;
__global__ void __launch_bounds__(1024) k_dq_mean(const double* __restrict__ warp_sums,
                                                  int64_t n_tiles, int64_t n_blocks,
                                                  double* __restrict__ seg_sums, unsigned int* __restrict__ ticket,
                                                  float* __restrict__ mean_out) {
    __shared__ double s_w[32];
    __shared__ int s_last;
    const int64_t n_segs = (n_tiles + kSeg - 1) / kSeg;  // <= kSeg for any supported size
    const int64_t seg = blockIdx.x;
    pdl_wait();                // the encoder's warp sums (and absmax) are complete and visible
    pdl_launch_dependents();   // so the scale quantiser may start and load the absmax values
    const double v = pairwise_2048(warp_sums + 8 * seg * kSeg, n_tiles - seg * kSeg, s_w, true);
    if (threadIdx.x == 0) {
        seg_sums[seg] = v;
        __threadfence();  // the segment sum before the ticket
        s_last = atomicAdd(ticket, 1u) == static_cast<unsigned int>(n_segs - 1);
    }
    __syncthreads();
    if (!s_last) return;
    __threadfence();      // every other segment's sum is visible after its ticket
    const double total = pairwise_2048(seg_sums, n_segs, s_w, false);
    if (threadIdx.x == 0) *mean_out = __double2float_rn(__ddiv_rn(total, static_cast<double>(n_blocks)));
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
    const int64_t b0 = g * kTileBlocks + lane * 8;
    // the absmax values were written by the encoder, which had finished before
    // the mean kernel released this one; the mean itself needs the wait
    float x[8];
    if (b0 + 8 <= n_blocks) {
        const float4 u0 = __ldcg(reinterpret_cast<const float4*>(absmax + b0));
        const float4 u1 = __ldcg(reinterpret_cast<const float4*>(absmax + b0) + 1);
        x[0] = u0.x; x[1] = u0.y; x[2] = u0.z; x[3] = u0.w;
        x[4] = u1.x; x[5] = u1.y; x[6] = u1.z; x[7] = u1.w;
    } else {
#pragma unroll
        for (int i = 0; i < 8; ++i) x[i] = b0 + i < n_blocks ? __ldcg(absmax + b0 + i) : 0.0f;
    }
    pdl_wait();
    const float mu = *mean_ptr;
    float d[8];
    float m = 0.0f;
#pragma unroll
    for (int i = 0; i < 8; ++i) d[i] = b0 + i < n_blocks ? __fsub_rn(x[i], mu) : 0.0f;
#pragma unroll
    for (int i = 0; i < 8; ++i) m = fmaxf(m, fabsf(d[i]));
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
// block; w_hat = bf16_rne(level[code] * s_b), with s_b restored from the
// double-quantised scales or, when absmax is given, the block's fp32 absmax.
__global__ void __launch_bounds__(256) k_nf4_dequantize(const uint8_t* __restrict__ codes,
                                                       const int8_t* __restrict__ qscale,
                                                       const float* __restrict__ scale2,
                                                       const float* __restrict__ mean_ptr,
                                                       const float* __restrict__ absmax,
                                                       int64_t n, uint16_t* __restrict__ out) {
    __shared__ float s_lut[16];
    if (threadIdx.x < 16) s_lut[threadIdx.x] = nf4_level(threadIdx.x);
    __syncthreads();
    const float mu = absmax ? 0.0f : *mean_ptr;
    const int64_t n_units = n / 16;
    for (int64_t u = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; u < n_units;
         u += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int64_t b = u >> 2;  // 4 units per 64-block
        const float s = absmax ? absmax[b] : nf4_block_scale(qscale[b], scale2[b >> 8], mu);
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

// A programmatic dependent of the kernel before it on the stream (it waits
// for that kernel with griddepcontrol.wait before reading its results).
static cudaLaunchAttribute g_pdl_attr = [] {
    cudaLaunchAttribute a{};
    a.id = cudaLaunchAttributeProgrammaticStreamSerialization;
    a.val.programmaticStreamSerializationAllowed = 1;
    return a;
}();

cudaError_t launch_nf4_quantize(const float* W, int64_t n, uint8_t* codes, int8_t* qscale,
                                float* scale2, float* scale_mean, float* ws_absmax,
                                double* ws_warp_sums, int num_sms, cudaStream_t stream) {
    const int64_t n_blocks = n / 64;
    const int64_t n_tiles = (n_blocks + kTileBlocks - 1) / kTileBlocks;
    // three CTAs per SM (at most 85 registers a thread): every CTA resident at once
    const int64_t grid1 = n_tiles < int64_t(num_sms) * 3 ? n_tiles : int64_t(num_sms) * 3;
    // after the warp sums: the segment sums and the mean kernel's ticket
    const int64_t n_segs = (n_tiles + kSeg - 1) / kSeg;
    double* seg_sums = ws_warp_sums ? ws_warp_sums + 8 * n_tiles : nullptr;
    unsigned int* ticket = ws_warp_sums ? reinterpret_cast<unsigned int*>(seg_sums + n_segs) : nullptr;
    cudaError_t e;
    {
        TraceScope trace("nf4_encode", stream);
        cudaLaunchConfig_t cfg = config(grid1, 256, stream);
        e = cudaLaunchKernelEx(&cfg, k_nf4_encode, W, n_blocks, codes, ws_absmax, ws_warp_sums, ticket);
        if (e != cudaSuccess) return e;
    }
    if (qscale == nullptr) return e;  // fp32 block scales: ws_absmax is the output
    {
        TraceScope trace("dq_mean", stream);
        cudaLaunchConfig_t cfg = config(n_segs, 1024, stream);
        cfg.attrs = &g_pdl_attr;
        cfg.numAttrs = 1;
        e = cudaLaunchKernelEx(&cfg, k_dq_mean, static_cast<const double*>(ws_warp_sums), n_tiles, n_blocks,
                               seg_sums, ticket, scale_mean);
        if (e != cudaSuccess) return e;
    }
    {
        TraceScope trace("dq_quantize", stream);
        cudaLaunchConfig_t cfg = config((n_tiles + 7) / 8, 256, stream);
        cfg.attrs = &g_pdl_attr;
        cfg.numAttrs = 1;
        e = cudaLaunchKernelEx(&cfg, k_dq_quantize, static_cast<const float*>(ws_absmax), n_blocks,
                               static_cast<const float*>(scale_mean), qscale, scale2);
    }
    return e;
}

cudaError_t launch_nf4_dequantize(const uint8_t* codes, const int8_t* qscale, const float* scale2,
                                  const float* scale_mean, const float* absmax, int64_t n, uint16_t* out,
                                  int num_sms, cudaStream_t stream) {
    const int64_t units = n / 16;
    int64_t grid = (units + 255) / 256;
    if (grid > int64_t(num_sms) * 16) grid = int64_t(num_sms) * 16;
    TraceScope trace("nf4_dequantize", stream);
    cudaLaunchConfig_t cfg = config(grid, 256, stream);
    return cudaLaunchKernelEx(&cfg, k_nf4_dequantize, codes, qscale, scale2, scale_mean, absmax, n, out);
}

}  // namespace nf4lora
