// Warp-specialised tcgen05 GEMM engine for the NF4-LoRA linear layer.
//
//   D[rows, cols] (fp32, TMEM) = sum_k A[rows, k] * B[cols, k]
//                              + sum_j A_ext[rows, j] * B_ext[cols, j]
//
// One CTA computes a 128 x BN tile (MMA M = 128, N = BN) over a range of
// 64-wide k-steps ("split"), followed -- in split 0 only -- by the extension
// k-steps that carry the rank-r LoRA product, so that X W_hat^T + T B^T (or
// dY W_hat + V A) lands in ONE accumulator without a second pass over the
// output.  The rank-r activation (T or V) is held as a pair of bf16 arrays,
// hi = bf16(v) and lo = bf16(v - hi), side by side; the extension runs over
// [hi | lo] while the LoRA weight tile is re-read for the second half
// (ext_wrap), which keeps ~16 mantissa bits of the fp32 intermediate.
//
// Each operand tile is either
//   * copied by TMA from a bf16 tensor (128-byte swizzle, K-major or
//     MN-major canonical layout), or
//   * DECODED from NF4: TMA stages the packed code bytes, decode warps read
//     them with the block scales, restore w_hat = bf16(level[code] * s_b)
//     ("第 04 篇：QLoRA 原理" §6.1: unpack, restore the scale in two levels,
//     look up, scale, convert to the compute dtype) and write the bf16 tile
//     straight into the swizzled operand layout in shared memory.  The weight
//     never exists in bf16 in device memory.  The same decode serves the
//     forward (K-major: rows of W_hat are MMA rows) and the input gradient
//     (MN-major: rows of W_hat are the contraction), because each decode unit
//     is one (weight row, 64-block) = one 128-byte row of a swizzle atom in
//     both layouts.
//
// Warp roles: warp 0 = TMA producer (one lane), warp 1 = TMEM allocator and
// MMA issuer (one lane), warps 2.. = decoders, then epilogue (TMEM -> regs ->
// global).  Stages are ring-buffered with mbarriers: full (TMA bytes landed),
// dec (decoded tile written), empty (MMAs that read the stage completed).
// Every wait is bounded (see common.cuh).
#pragma once

#include <cstdint>

#include "common.cuh"
#include "nf4_levels.cuh"

namespace nf4lora {

enum OpSrc : int { SRC_TMA_K = 0, SRC_TMA_MN = 1, SRC_DEC_K = 2, SRC_DEC_MN = 3 };
enum EpiKind : int { EPI_BF16 = 0, EPI_F32_PART = 1, EPI_F32_PART_T = 2 };

struct GemmArgs {
    int rows;           // valid rows of D over the whole problem
    int cols;           // valid columns of D
    int k_main;         // 64-wide main k-steps in total
    int k_per_split;    // main k-steps per grid.z slice
    int k_ext;          // extension k-steps (grid.z slice 0 only)
    int ext_wrap_a;     // extension k-step j reads A_ext at (j % ext_wrap_a) when > 0
    int ext_wrap_b;     // ... and B_ext at (j % ext_wrap_b) when > 0
    // NF4 operand
    const int8_t* qscale;
    const float* scale2;
    const float* scale_mean;
    int64_t w_rows;           // d_out of the encoded weight
    int64_t w_blocks_per_row; // d_in / 64
    // epilogue
    float alpha;
    uint16_t* out;      // EPI_BF16: out[row * ldo + col]
    int64_t ldo;
    float* part;        // EPI_F32_PART: part[z * part_slice + row * ldp + col]
    int64_t ldp;        // EPI_F32_PART_T: part[z * part_slice + col * ldp + row]
    int64_t part_slice;
};

template <int SRC>
struct OpTraits {
    static constexpr bool kDecoded = (SRC == SRC_DEC_K || SRC == SRC_DEC_MN);
    static constexpr bool kMN = (SRC == SRC_TMA_MN || SRC == SRC_DEC_MN);
};

template <int BN, int ASRC, int BSRC, int AE_MN, int BE_MN, int EPI>
struct GemmConfig {
    static constexpr int kBM = 128;
    static constexpr int kBK = 64;
    static constexpr bool kDecA = OpTraits<ASRC>::kDecoded;
    static constexpr bool kDecB = OpTraits<BSRC>::kDecoded;
    static_assert(!(kDecA && kDecB), "at most one decoded operand");
    static constexpr bool kHasDec = kDecA || kDecB;
    static constexpr int kABytes = kBM * kBK * 2;             // 16 KB
    static constexpr int kBBytes = BN * kBK * 2;
    static constexpr int kDecMN = kDecA ? kBM : (kDecB ? BN : 0);  // decoded tile's M/N width
    static constexpr int kCBytes = kDecMN * 32;               // packed codes per stage
    static constexpr int kStageBytes = kABytes + kBBytes + kCBytes;
    static constexpr int kStagesRaw = (225 * 1024) / kStageBytes;
    static constexpr int kStages = kStagesRaw > 8 ? 8 : kStagesRaw;
    static_assert(kStages >= 2, "tile too large");
    static constexpr int kDecThreads = kDecMN;                // one (row, block) unit each
    static constexpr int kDecWarps = kDecThreads / 32;
    static constexpr int kWorkWarps = kDecWarps > 4 ? kDecWarps : 4;
    static constexpr int kThreads = 64 + 32 * kWorkWarps;
    static constexpr int kTmemCols = BN < 32 ? 32 : BN;
    static constexpr int kSmemBytes = kStages * kStageBytes + 1024;
    // transaction bytes of one stage
    static constexpr int kTxMain = (kDecA ? kCBytes : kABytes) + (kDecB ? kCBytes : kBBytes);
    static constexpr int kTxExt = kABytes + kBBytes;
    static constexpr uint32_t kIdescMain =
        make_idesc_bf16(kBM, BN, OpTraits<ASRC>::kMN ? 1 : 0, OpTraits<BSRC>::kMN ? 1 : 0);
    static constexpr uint32_t kIdescExt = make_idesc_bf16(kBM, BN, AE_MN, BE_MN);
};

// Descriptor of k-substep kk (16 elements of K) of a 64-deep swizzled tile.
__device__ __forceinline__ uint64_t tile_desc(uint32_t base, bool mn_major, int kk) {
    if (mn_major) return make_sw128_desc(base + kk * 2048, 8192, 1024);  // 16 K-rows of 128 B
    return make_sw128_desc(base + kk * 32, 16, 1024);                   // 16 elements = 32 B
}

// Decode one (weight row, 64-block) unit: 32 packed bytes -> 64 bf16 written
// as 8 swizzled 16-byte chunks of one 128-byte row.
__device__ __forceinline__ void decode_unit(const uint8_t* src, float s, uint8_t* dst_row, int swz,
                                            const float* lut) {
    const uint4 c0 = *reinterpret_cast<const uint4*>(src);
    const uint4 c1 = *reinterpret_cast<const uint4*>(src + 16);
    const uint32_t words[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        const uint32_t x = words[j];  // 8 codes: byte b = (elem 2b << 4) | elem 2b+1
        uint32_t o[4];
#pragma unroll
        for (int b = 0; b < 4; ++b) {
            const float ev = __fmul_rn(lut[(x >> (8 * b + 4)) & 15u], s);
            const float od = __fmul_rn(lut[(x >> (8 * b)) & 15u], s);
            o[b] = pack_bf16x2(ev, od);
        }
        *reinterpret_cast<uint4*>(dst_row + ((j ^ swz) << 4)) = make_uint4(o[0], o[1], o[2], o[3]);
    }
}

__device__ __forceinline__ void zero_row(uint8_t* dst_row) {
#pragma unroll
    for (int j = 0; j < 8; ++j) *reinterpret_cast<uint4*>(dst_row + (j << 4)) = make_uint4(0, 0, 0, 0);
}

// Bounded wait that ignores the abort flag: used only to drain copies that
// are still in flight when a CTA gives up.
__device__ __forceinline__ void mbar_drain(uint64_t* bar, uint32_t parity) {
    const uint64_t t0 = global_timer_ns();
    while (!mbar_try_wait(bar, parity)) {
        if (global_timer_ns() - t0 > kWaitLimitNs / 20) break;
    }
}

template <int BN, int ASRC, int BSRC, int AE_MN, int BE_MN, int EPI>
__global__ void __launch_bounds__(GemmConfig<BN, ASRC, BSRC, AE_MN, BE_MN, EPI>::kThreads, 1)
    k_gemm(const __grid_constant__ CUtensorMap map_a, const __grid_constant__ CUtensorMap map_b,
           const __grid_constant__ CUtensorMap map_ae, const __grid_constant__ CUtensorMap map_be,
           const GemmArgs args) {
    using C = GemmConfig<BN, ASRC, BSRC, AE_MN, BE_MN, EPI>;
    constexpr int S = C::kStages;
    extern __shared__ uint8_t smem_raw[];
    __shared__ uint64_t bar_full[S], bar_dec[S], bar_empty[S], bar_accum;
    __shared__ uint32_t s_tmem;
    __shared__ int s_abort;
    __shared__ float s_lut[16];

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base_u32 = (raw + 1023u) & ~1023u;
    uint8_t* base = smem_raw + (base_u32 - raw);
    auto a_tile = [&](int s) { return base + s * C::kABytes; };
    auto b_tile = [&](int s) { return base + S * C::kABytes + s * C::kBBytes; };
    auto c_tile = [&](int s) { return base + S * (C::kABytes + C::kBBytes) + s * C::kCBytes; };

    const int r0 = blockIdx.x * C::kBM;
    const int c0 = blockIdx.y * BN;
    const int z = blockIdx.z;
    const int kb_begin = z * args.k_per_split;
    int kb_end = kb_begin + args.k_per_split;
    if (kb_end > args.k_main) kb_end = args.k_main;
    const int n_main = kb_end > kb_begin ? kb_end - kb_begin : 0;
    const int n_ext = (z == 0) ? args.k_ext : 0;
    const int n_iter = n_main + n_ext;

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(&bar_full[s], 1);
            mbar_init(&bar_dec[s], C::kDecWarps > 0 ? C::kDecWarps : 1);
            mbar_init(&bar_empty[s], 1);
        }
        mbar_init(&bar_accum, 1);
        s_abort = 0;
        fence_barrier_init();
    }
    if (threadIdx.x < 16) s_lut[threadIdx.x] = nf4_level(threadIdx.x);
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&map_a);
        tma_prefetch_desc(&map_b);
        if (n_ext > 0) {
            tma_prefetch_desc(&map_ae);
            tma_prefetch_desc(&map_be);
        }
    }
    if (warp == 1) {
        tmem_alloc(&s_tmem, C::kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_d = s_tmem;
    volatile int* abort_flag = &s_abort;

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            int issued = 0;
            for (int it = 0; it < n_iter; ++it) {
                const int s = it % S;
                const uint32_t ph = (it / S) & 1u;
                if (it >= S && !mbar_wait(&bar_empty[s], ph ^ 1u, abort_flag)) break;
                if (*abort_flag) break;
                uint64_t* bar = &bar_full[s];
                if (it < n_main) {
                    const int kb = kb_begin + it;
                    mbar_arrive_expect_tx(bar, C::kTxMain);
                    // operand A
                    if constexpr (ASRC == SRC_TMA_K) {
                        tma_load_2d(a_tile(s), &map_a, bar, kb * 64, r0);
                    } else if constexpr (ASRC == SRC_TMA_MN) {
                        tma_load_2d(a_tile(s), &map_a, bar, r0, kb * 64);
                        tma_load_2d(a_tile(s) + 8192, &map_a, bar, r0 + 64, kb * 64);
                    } else if constexpr (ASRC == SRC_DEC_K) {
                        tma_load_2d(c_tile(s), &map_a, bar, kb * 32, r0);
                    } else {
                        tma_load_2d(c_tile(s), &map_a, bar, r0 / 2, kb * 64);
                    }
                    // operand B
                    if constexpr (BSRC == SRC_TMA_K) {
                        tma_load_2d(b_tile(s), &map_b, bar, kb * 64, c0);
                    } else if constexpr (BSRC == SRC_TMA_MN) {
#pragma unroll
                        for (int c = 0; c < BN / 64; ++c)
                            tma_load_2d(b_tile(s) + c * 8192, &map_b, bar, c0 + c * 64, kb * 64);
                    } else if constexpr (BSRC == SRC_DEC_K) {
                        tma_load_2d(c_tile(s), &map_b, bar, kb * 32, c0);
                    } else {
                        tma_load_2d(c_tile(s), &map_b, bar, c0 / 2, kb * 64);
                    }
                } else {
                    const int j = it - n_main;
                    const int ja = args.ext_wrap_a > 0 ? j % args.ext_wrap_a : j;
                    const int jb = args.ext_wrap_b > 0 ? j % args.ext_wrap_b : j;
                    mbar_arrive_expect_tx(bar, C::kTxExt);
                    if constexpr (AE_MN) {
                        tma_load_2d(a_tile(s), &map_ae, bar, r0, ja * 64);
                        tma_load_2d(a_tile(s) + 8192, &map_ae, bar, r0 + 64, ja * 64);
                    } else {
                        tma_load_2d(a_tile(s), &map_ae, bar, ja * 64, r0);
                    }
                    if constexpr (BE_MN) {
#pragma unroll
                        for (int c = 0; c < BN / 64; ++c)
                            tma_load_2d(b_tile(s) + c * 8192, &map_be, bar, c0 + c * 64, jb * 64);
                    } else {
                        tma_load_2d(b_tile(s), &map_be, bar, jb * 64, c0);
                    }
                }
                ++issued;
            }
            if (*abort_flag) {
                // let the copies already issued land before the CTA exits
                const int first = issued > S ? issued - S : 0;
                for (int it = first; it < issued; ++it) mbar_drain(&bar_full[it % S], (it / S) & 1u);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            for (int it = 0; it < n_iter; ++it) {
                const int s = it % S;
                const uint32_t ph = (it / S) & 1u;
                if (!mbar_wait(&bar_full[s], ph, abort_flag)) break;
                const bool is_main = it < n_main;
                if (C::kHasDec && is_main && !mbar_wait(&bar_dec[s], ph, abort_flag)) break;
                tc_fence_after();
                const uint32_t a_base = smem_u32(a_tile(s));
                const uint32_t b_base = smem_u32(b_tile(s));
                const bool a_mn = is_main ? OpTraits<ASRC>::kMN : (AE_MN != 0);
                const bool b_mn = is_main ? OpTraits<BSRC>::kMN : (BE_MN != 0);
                const uint32_t idesc = is_main ? C::kIdescMain : C::kIdescExt;
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) {
                    mma_bf16_ss(tmem_d, tile_desc(a_base, a_mn, kk), tile_desc(b_base, b_mn, kk), idesc,
                                (it > 0 || kk > 0) ? 1u : 0u);
                }
                mma_commit(&bar_empty[s]);
            }
            mma_commit(&bar_accum);
        }
    } else {
        const int ew = warp - 2;
        // ------------------------------------------------------------ decoders
        if constexpr (C::kHasDec) {
            if (ew < C::kDecWarps) {
                const int dt = threadIdx.x - 64;
                const float mu = *args.scale_mean;
                constexpr bool kMNdec = C::kDecA ? (ASRC == SRC_DEC_MN) : (BSRC == SRC_DEC_MN);
                constexpr int kCB = C::kDecMN / 64;           // 64-blocks across the decoded tile
                const int tile_mn0 = C::kDecA ? r0 : c0;
                for (int it = 0; it < n_main; ++it) {
                    const int s = it % S;
                    const uint32_t ph = (it / S) & 1u;
                    const int kb = kb_begin + it;
                    int64_t wrow, wblk;
                    int dst_off, swz;
                    if constexpr (!kMNdec) {
                        wrow = tile_mn0 + dt;
                        wblk = kb;
                        dst_off = dt * 128;
                        swz = dt & 7;
                    } else {
                        const int n_local = dt / kCB, c = dt % kCB;
                        wrow = static_cast<int64_t>(kb) * 64 + n_local;
                        wblk = tile_mn0 / 64 + c;
                        dst_off = c * 8192 + n_local * 128;
                        swz = n_local & 7;
                    }
                    const bool valid = wrow < args.w_rows && wblk < args.w_blocks_per_row;
                    float sc = 0.0f;
                    if (valid) {
                        const int64_t bidx = wrow * args.w_blocks_per_row + wblk;
                        sc = nf4_block_scale(__ldg(args.qscale + bidx), __ldg(args.scale2 + (bidx >> 8)), mu);
                    }
                    if (!mbar_wait(&bar_full[s], ph, abort_flag)) break;
                    uint8_t* dst = (C::kDecA ? a_tile(s) : b_tile(s)) + dst_off;
                    if (valid) decode_unit(c_tile(s) + dt * 32, sc, dst, swz, s_lut);
                    else zero_row(dst);
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&bar_dec[s]);
                }
            }
        }
        // ------------------------------------------------------------ epilogue
        const int q = warp & 3;                       // TMEM lane quadrant of this warp
        constexpr int kColSplit = C::kWorkWarps / 4;  // warps sharing one quadrant
        const int part_idx = ew / 4;
        const int cw = BN / kColSplit;
        const int cbeg = part_idx * cw;
        const bool ok = mbar_wait(&bar_accum, 0, abort_flag);
        tc_fence_after();
        if (ok && !*abort_flag) {
            const int row = r0 + q * 32 + lane;
            const bool row_ok = row < args.rows;
            for (int cc = cbeg; cc < cbeg + cw; cc += 32) {
                uint32_t v[32];
                tmem_ld_32x32b_x32(tmem_d + (static_cast<uint32_t>(q * 32) << 16) + cc, v);
                tmem_ld_wait();
                const int col = c0 + cc;
                if constexpr (EPI == EPI_BF16) {
                    if (row_ok) {
                        uint16_t* dst = args.out + static_cast<int64_t>(row) * args.ldo + col;
                        if (col + 32 <= args.cols) {
#pragma unroll
                            for (int j = 0; j < 32; j += 8) {
                                uint4 pk;
                                pk.x = pack_bf16x2(__uint_as_float(v[j]) * args.alpha, __uint_as_float(v[j + 1]) * args.alpha);
                                pk.y = pack_bf16x2(__uint_as_float(v[j + 2]) * args.alpha, __uint_as_float(v[j + 3]) * args.alpha);
                                pk.z = pack_bf16x2(__uint_as_float(v[j + 4]) * args.alpha, __uint_as_float(v[j + 5]) * args.alpha);
                                pk.w = pack_bf16x2(__uint_as_float(v[j + 6]) * args.alpha, __uint_as_float(v[j + 7]) * args.alpha);
                                *reinterpret_cast<uint4*>(dst + j) = pk;
                            }
                        } else {
#pragma unroll
                            for (int j = 0; j < 32; ++j) {
                                if (col + j < args.cols) {
                                    __nv_bfloat16 h = __float2bfloat16_rn(__uint_as_float(v[j]) * args.alpha);
                                    dst[j] = *reinterpret_cast<uint16_t*>(&h);
                                }
                            }
                        }
                    }
                } else if constexpr (EPI == EPI_F32_PART) {
                    if (row_ok) {
                        float* dst = args.part + z * args.part_slice + static_cast<int64_t>(row) * args.ldp + col;
                        if (col + 32 <= args.cols) {
#pragma unroll
                            for (int j = 0; j < 32; j += 4)
                                *reinterpret_cast<float4*>(dst + j) =
                                    make_float4(__uint_as_float(v[j]), __uint_as_float(v[j + 1]),
                                                __uint_as_float(v[j + 2]), __uint_as_float(v[j + 3]));
                        } else {
#pragma unroll
                            for (int j = 0; j < 32; ++j)
                                if (col + j < args.cols) dst[j] = __uint_as_float(v[j]);
                        }
                    }
                } else {
                    if (row_ok) {
                        float* dst = args.part + z * args.part_slice + row;
#pragma unroll
                        for (int j = 0; j < 32; ++j)
                            if (col + j < args.cols) dst[static_cast<int64_t>(col + j) * args.ldp] = __uint_as_float(v[j]);
                    }
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_d, C::kTmemCols);
    }
}

}  // namespace nf4lora
