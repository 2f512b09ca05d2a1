// Few-token (M <= 16) fused NF4-LoRA input gradient on warp-level tensor
// instructions (mma.sync m16n8k16, bf16 in, fp32 accumulate), the weight
// decoded on chip and never written back to memory ("第 04 篇：QLoRA 原理"
// §2.4: the frozen base still passes the input gradient).  The forward
// counterpart is in fewfwd.cu.
//
// Split-K: the CTAs that share one output tile form a thread-block cluster
// along grid.z.  Inside a CTA every warp puts its fp32 partials into shared
// memory and each thread adds up four outputs (the warps of a column block,
// in order); every CTA of rank > 0 then pushes its partial tile into a slot of
// rank 0 (distributed shared memory) before a cluster barrier, after which
// rank 0 adds the slots in rank order and writes bf16 rows.  The rank-r
// extension, once the kernel that produced V2 has finished (programmatic
// dependent launch), is shared out among the ranks.  The summation order is
// fixed, so the result is the same on every run.
//
// Launch overlap: the kernel releases its own dependents as soon as it starts
// and asks L2 for the rows of A its extension will read.  It reads dY and the
// encoded weight before its own wait: the rank-r kernel it depends on
// released it only after waiting for the kernel before that, so every
// earlier write is complete; global loads go through L2 (ld.global.cg),
// never a possibly stale L1 line.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "common.cuh"
#include "decode.cuh"
#include "kernels.h"
#include "nf4_levels.cuh"
#include "trace.h"

namespace nf4lora {

namespace {

constexpr int kThreads = 512;      // 16 warps
constexpr int kTile = 128;         // weight rows per CTA
constexpr int kTok = 16;           // token rows of the MMA
constexpr int kMaxSplit = 8;       // CTAs per cluster (portable cluster size)
constexpr int kPartFloats = kTile * kTok;  // one CTA's partial tile, fp32

__device__ __forceinline__ void mma_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                          uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Even split of `total` units over `parts`; part p gets [begin, end).
__device__ __forceinline__ void split_range(int total, int parts, int p, int& begin, int& end) {
    const int per = total / parts, extra = total % parts;
    begin = p * per + (p < extra ? p : extra);
    end = begin + per + (p < extra ? 1 : 0);
}

// row stride (floats) of the per-warp partial tiles [token][row] gathered for
// the reduction: 132 puts the 8 x 4 (row, token) pairs of a fragment store in
// distinct banks and keeps the rows 16-byte aligned
constexpr int kSumStride = 132;

// ---------------------------------------------------------------- input gradient
// dX^T[k, t] = sum_n W_hat[n, k] dY[t, n] + sum_j [A ; A][j, k] V2[t, j]:
// tensor-instruction roles A = 16 columns k x 16 rows n of W_hat (transposed),
// B = 16 rows n x 8 tokens (dY), D = 16 columns x 8 tokens.  The operand pairs
// of A run along n, i.e. across two code bytes of different rows, so the
// decode goes through shared memory: each thread decodes one whole 64-block
// of one weight row (one scale) with the register codebook into its warp's
// padded tile [32 rows][64 + 8], and ldmatrix.trans hands out the transposed
// pairs.  Warp w works on 64-column block (w & 1) of the CTA's 128 columns and
// on every eighth 32-row chunk of the CTA's rows (w >> 1); the codes of up to
// 1024 rows x 128 columns come in by TMA (64-byte swizzle) in four boxes.
constexpr int kDxRowsSeg = 1024;
constexpr int kDxTileStride = 144;                 // bytes per tile row: 64 bf16 + 16 bytes padding
constexpr int kDxTileBytes = 32 * kDxTileStride;   // one warp's tile
constexpr int kDxYStride = kDxRowsSeg + 8;         // dY staging, elements (2064 bytes: conflict-free)
constexpr int kDxMaxSplit = 4;
constexpr int kDxSmem = 1024 + kDxRowsSeg * 64 + 16 * kDxTileBytes + kTok * kDxYStride * 2 +
                        (kDxMaxSplit - 1) * kPartFloats * 4;
static_assert(8 * kTok * kSumStride * 4 <= 16 * kDxTileBytes, "the partial tiles reuse the decode tiles");
static_assert(kTok * (2 * 256 + 8) <= kTok * kDxYStride, "V2 staging reuses the dY staging");

__device__ __forceinline__ void ldmatrix_x4_trans(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                                  uint32_t& r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}

// The MMAs of one 32-row chunk held in the warp's tile, against activation
// rows row0 .. row0 + 31 of the staged [16][ystride] array.
__device__ __forceinline__ void dx_chunk_mma(float (&acc)[4][2][4], uint32_t tile_u32, const uint16_t* sy,
                                             int ystride, int row0, int lane, bool two_halves) {
    const int g = lane >> 2, q = lane & 3;
    const int mi = lane >> 3, i = lane & 7;  // ldmatrix: this lane's row address of matrix mi
#pragma unroll
    for (int s = 0; s < 2; ++s) {
        const uint16_t* y0 = sy + g * ystride + row0 + 16 * s + 2 * q;
        const uint16_t* y8 = y0 + 8 * ystride;
        const uint32_t b0 = *reinterpret_cast<const uint32_t*>(y0), b1 = *reinterpret_cast<const uint32_t*>(y0 + 8);
        const uint32_t c0 = *reinterpret_cast<const uint32_t*>(y8), c1 = *reinterpret_cast<const uint32_t*>(y8 + 8);
        const uint32_t row_addr = tile_u32 + (16 * s + 8 * (mi >> 1) + i) * kDxTileStride + 16 * (mi & 1);
#pragma unroll
        for (int m = 0; m < 4; ++m) {
            uint32_t a0, a1, a2, a3;
            ldmatrix_x4_trans(row_addr + 32 * m, a0, a1, a2, a3);
            mma_16816(acc[m][0], a0, a1, a2, a3, b0, b1);
            if (two_halves) mma_16816(acc[m][1], a0, a1, a2, a3, c0, c1);
        }
    }
}

__global__ void __maxnreg__(112) k_few_dx(const __grid_constant__ CUtensorMap map_codes, const FewArgs a) {
    extern __shared__ __align__(16) uint8_t smem_raw[];
    __shared__ uint64_t bar_c[4];
    __shared__ int s_abort;
    pdl_launch_dependents();
    // [codes: kDxRowsSeg rows x 64 B, 64-byte swizzle][16 warp tiles; after the
    //  loop the partial tiles][dY staging][slots for the other ranks' partial tiles]
    const uint32_t raw = smem_u32(smem_raw);
    uint8_t* s_codes = smem_raw + (((raw + 1023u) & ~1023u) - raw);
    uint8_t* s_tiles = s_codes + kDxRowsSeg * 64;
    uint16_t* sY = reinterpret_cast<uint16_t*>(s_tiles + 16 * kDxTileBytes);
    float* s_part = reinterpret_cast<float*>(sY + kTok * kDxYStride);  // [kDxMaxSplit - 1][2048]

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, g = lane >> 2, q = lane & 3;
    const int cb = warp & 1, rw = warp >> 1;
    const int splits = static_cast<int>(gridDim.z);
    const int rank = static_cast<int>(cluster_ctarank());
    const int M = a.M, N = a.N, K = a.K;
    const int bpr = K / 64;
    const int blk = 2 * blockIdx.x + cb;
    const bool blk_ok = blk < bpr;
    int ch0, ch1;  // this rank's 32-row chunks
    split_range((N + 31) / 32, splits, rank, ch0, ch1);
    auto issue_codes = [&](int sc0, int sc1) {
        for (int b = 0; 8 * b < sc1 - sc0; ++b) {
            mbar_arrive_expect_tx(&bar_c[b], 256 * 64);
            tma_load_2d(s_codes + b * 256 * 64, &map_codes, &bar_c[b], 64 * blockIdx.x, 32 * (sc0 + 8 * b));
        }
    };
    if (tid == 0) {
        for (int b = 0; b < 4; ++b) mbar_init(&bar_c[b], 1);
        s_abort = 0;
        fence_barrier_init();
        if (ch0 < ch1) {
            tma_prefetch_desc(&map_codes);
            issue_codes(ch0, min(ch1, ch0 + kDxRowsSeg / 32));
        }
    } else if (tid >= 32 && tid < 32 + a.r && a.ext_act != nullptr) {
        // row tid - 32 of A over the CTA's one or two 64-column blocks
        const int j = tid - 32;
        prefetch_l2_bulk(a.ext_w + static_cast<int64_t>(j) * K + 128 * blockIdx.x,
                         2 * static_cast<int>(blockIdx.x) + 1 < bpr ? 256u : 128u);
    }
    const bool two_halves = M > 8;
    float acc[4][2][4];
#pragma unroll
    for (int m = 0; m < 4; ++m)
#pragma unroll
        for (int h = 0; h < 2; ++h)
#pragma unroll
            for (int e = 0; e < 4; ++e) acc[m][h][e] = 0.0f;
    __syncthreads();
    cluster_arrive_relaxed();  // barriers initialised (made visible by the init fence)
    const bool fp32_scales = a.absmax != nullptr;  // no double quantisation
    const float mu = fp32_scales ? 0.0f : __ldcg(a.scale_mean);
    volatile int* abort_flag = &s_abort;
    uint8_t* my_tile = s_tiles + warp * kDxTileBytes;
    const uint32_t my_tile_u32 = smem_u32(my_tile);

    int seg_i = 0, issued_seg = 0, issued_boxes = ch0 < ch1 ? (min(ch1, ch0 + kDxRowsSeg / 32) - ch0 + 7) / 8 : 0;
    for (int sc0 = ch0; sc0 < ch1; sc0 += kDxRowsSeg / 32, ++seg_i) {
        const int sc1 = min(ch1, sc0 + kDxRowsSeg / 32);
        const int rows = 32 * (sc1 - sc0);  // staged rows (the last ones may lie beyond N)
        if (seg_i > 0) {
            __syncthreads();  // the previous segment's codes, tiles and dY are no longer read
            if (*abort_flag) break;
            if (tid == 0) issue_codes(sc0, sc1);
            issued_seg = seg_i;
            issued_boxes = (sc1 - sc0 + 7) / 8;
        }
        // dY[:, 32 sc0 : 32 sc1] (rows >= N, tokens >= M as zeros) and this thread's scales
        // a token row has `per` 8-byte pieces (256 in a full segment)
        const int per = rows / 4;
        uint2 yv[8];
#pragma unroll
        for (int p = 0; p < 8; ++p) {
            const int i = tid + p * kThreads, t = per == 256 ? (i >> 8) : i / per, pc = i - t * per;
            const int n = 32 * sc0 + 4 * pc;
            yv[p] = make_uint2(0, 0);
            if (t < M && n < N) yv[p] = __ldcg(reinterpret_cast<const uint2*>(a.act + static_cast<int64_t>(t) * N + n));
        }
        int qv[4];
        float a2v[4];
#pragma unroll
        for (int it = 0; it < 4; ++it) {
            const int c = sc0 + rw + 8 * it, n = 32 * c + lane;
            const bool ok = c < sc1 && n < N && blk_ok;
            const int64_t bi = static_cast<int64_t>(n) * bpr + blk;
            qv[it] = ok && !fp32_scales ? static_cast<int>(__ldcg(a.qscale + bi)) : 0;
            a2v[it] = ok ? __ldcg(fp32_scales ? a.absmax + bi : a.scale2 + (bi >> 8)) : 0.0f;
        }
#pragma unroll
        for (int p = 0; p < 8; ++p) {
            const int i = tid + p * kThreads, t = per == 256 ? (i >> 8) : i / per, pc = i - t * per;
            if (t < kTok) *reinterpret_cast<uint2*>(sY + t * kDxYStride + 4 * pc) = yv[p];
        }
        __syncthreads();
#pragma unroll 1
        for (int it = 0; it < 4; ++it) {
            const int c = sc0 + rw + 8 * it;
            if (c >= sc1) break;
            const int lr = 32 * (c - sc0) + lane;  // staged row of this thread
            if (!mbar_wait(&bar_c[(c - sc0) / 8], seg_i & 1, abort_flag)) break;
            const int n = 32 * c + lane;
            const bool ok = n < N && blk_ok;
            const float sc =
                ok ? (fp32_scales ? a2v[it] : nf4_block_scale(static_cast<int8_t>(qv[it]), a2v[it], mu)) : 0.0f;
            // the row's 32 code bytes of block cb: 16-byte chunks 2 cb, 2 cb + 1, swizzled by row
            const uint8_t* crow = s_codes + lr * 64;
            const int sw = (lr >> 1) & 3;
            const uint4 u0 = *reinterpret_cast<const uint4*>(crow + (((2 * cb) ^ sw) << 4));
            const uint4 u1 = *reinterpret_cast<const uint4*>(crow + (((2 * cb + 1) ^ sw) << 4));
            const uint32_t w[8] = {u0.x, u0.y, u0.z, u0.w, u1.x, u1.y, u1.z, u1.w};
            uint32_t d[32];
            nf4_decode_block(w, sc, d);
            uint4* trow = reinterpret_cast<uint4*>(my_tile + lane * kDxTileStride);
#pragma unroll
            for (int j = 0; j < 8; ++j) trow[j] = make_uint4(d[4 * j], d[4 * j + 1], d[4 * j + 2], d[4 * j + 3]);
            __syncwarp();
            dx_chunk_mma(acc, my_tile_u32, sY, kDxYStride, 32 * (c - sc0), lane, two_halves);
            __syncwarp();
        }
    }
    if (tid == 0 && *abort_flag) {
        for (int b = 0; b < issued_boxes; ++b) mbar_drain(&bar_c[b], issued_seg & 1);
    }

    // rank-r extension: the rows of [A ; A] as 32-row chunks through the same
    // tiles, against V2 staged in place of dY, once the kernel producing V2
    // has finished; the chunks are dealt round-robin to the ranks, which add
    // them to the partials they push
    if (a.pdl) pdl_wait();
    if (a.ext_act != nullptr) {
        const int vstride = 2 * a.r64 + 8;
        __syncthreads();  // dY staging and tiles are free
        for (int i = tid; i < kTok * (2 * a.r64 / 4); i += kThreads) {
            const int t = i / (2 * a.r64 / 4), pc = i - t * (2 * a.r64 / 4);
            uint2 v = make_uint2(0, 0);
            if (t < M) v = __ldcg(reinterpret_cast<const uint2*>(a.ext_act + static_cast<int64_t>(t) * 2 * a.r64) + pc);
            *reinterpret_cast<uint2*>(sY + t * vstride + 4 * pc) = v;
        }
        __syncthreads();
        for (int c = rank + splits * rw; c < 2 * a.r64 / 32; c += 8 * splits) {
            const int j = (32 * c + lane) % a.r64;  // row of A (the same in both halves)
            uint4* trow = reinterpret_cast<uint4*>(my_tile + lane * kDxTileStride);
            const uint4* arow = reinterpret_cast<const uint4*>(a.ext_w + static_cast<int64_t>(j) * K + 64 * blk);
#pragma unroll
            for (int k = 0; k < 8; ++k) trow[k] = (j < a.r && blk_ok) ? __ldcg(arow + k) : make_uint4(0, 0, 0, 0);
            __syncwarp();
            dx_chunk_mma(acc, my_tile_u32, sY, vstride, 32 * c, lane, two_halves);
            __syncwarp();
        }
    }

    // every warp's partials into shared memory (the tiles are free),
    // s_sum[row warp][token][local column]; then thread tid adds up token
    // tid / 32, columns 4 (tid % 32) .. + 3: the eight row warps in order
    __syncthreads();
    float* s_sum = reinterpret_cast<float*>(s_tiles);
    {
        float* dst = s_sum + rw * kTok * kSumStride;
        // acc[m][h]: columns 64 cb + 16m + g (e = 0, 1) and + 8 (e = 2, 3), tokens 2q + 8h + (e & 1)
#pragma unroll
        for (int m = 0; m < 4; ++m)
#pragma unroll
            for (int h = 0; h < 2; ++h)
#pragma unroll
                for (int e = 0; e < 4; ++e)
                    dst[(2 * q + 8 * h + (e & 1)) * kSumStride + 64 * cb + 16 * m + g + 8 * (e >> 1)] = acc[m][h][e];
    }
    __syncthreads();
    const int ot = tid >> 5, ocol = 4 * (tid & 31);
    float4 o = *reinterpret_cast<const float4*>(s_sum + ot * kSumStride + ocol);
#pragma unroll
    for (int w = 1; w < 8; ++w) {
        const float4 v = *reinterpret_cast<const float4*>(s_sum + (w * kTok + ot) * kSumStride + ocol);
        o.x += v.x;
        o.y += v.y;
        o.z += v.z;
        o.w += v.w;
    }
    // ranks > 0 push into rank 0's slots; the cluster barrier (every CTA has
    // started, then every push is visible) orders them before rank 0's sums,
    // and no CTA touches another's shared memory after it
    cluster_wait_acquire();
    if (rank != 0)
        st_cluster_f4(cluster_map(smem_u32(s_part + (rank - 1) * kPartFloats + 4 * tid), 0), o.x, o.y, o.z, o.w);
    cluster_arrive_release();
    cluster_wait_acquire();
    if (rank == 0) {
        for (int rk = 1; rk < splits; ++rk) {
            const float4 v = *reinterpret_cast<const float4*>(s_part + (rk - 1) * kPartFloats + 4 * tid);
            o.x += v.x;
            o.y += v.y;
            o.z += v.z;
            o.w += v.w;
        }
        // columns 128 x + ocol .. + 3 lie in block 2x (ocol < 64) or 2x + 1
        const bool col_ok = ocol < 64 || 2 * static_cast<int>(blockIdx.x) + 1 < bpr;
        if (ot < M && col_ok) {
            uint2 packed;
            packed.x = pack_bf16x2(o.x, o.y);
            packed.y = pack_bf16x2(o.z, o.w);
            *reinterpret_cast<uint2*>(a.out + static_cast<int64_t>(ot) * K + 128 * blockIdx.x + ocol) = packed;
        }
    }
}

// `configured`: per-device flags of this kernel (both kernels have the same
// type, so the flags cannot live in the template)
template <typename Kern, typename... Params>
cudaError_t launch_cluster(Kern kern, bool (&configured)[64], int smem, const char* name, const FewArgs& a, int tiles,
                           int splits, cudaStream_t stream, const Params&... params) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64 || !configured[dev]) {
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e != cudaSuccess) return e;
        e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, cudaSharedmemCarveoutMaxShared);
        if (e != cudaSuccess) return e;
        if (dev >= 0 && dev < 64) configured[dev] = true;
    }
    if (splits < 1 || splits > kMaxSplit) return cudaErrorInvalidValue;
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(tiles, 1, splits);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    int n = 0;
    attr[n].id = cudaLaunchAttributeClusterDimension;
    attr[n].val.clusterDim.x = 1;
    attr[n].val.clusterDim.y = 1;
    attr[n].val.clusterDim.z = splits;
    ++n;
    if (a.pdl) {
        attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[n].val.programmaticStreamSerializationAllowed = 1;
        ++n;
    }
    cfg.attrs = attr;
    cfg.numAttrs = n;
    TraceScope trace(name, stream);
    return cudaLaunchKernelEx(&cfg, kern, params..., a);
}

}  // namespace

int few_max_split(bool forward) { return forward ? kMaxSplit : kDxMaxSplit; }

cudaError_t launch_few_dx(const CUtensorMap& map_codes, const FewArgs& a, int splits, cudaStream_t stream) {
    if (a.M < 1 || a.M > kTok || a.K % 64 != 0 || a.N % 8 != 0 || splits > (a.N + 31) / 32 || splits > kDxMaxSplit ||
        a.r64 > 256)
        return cudaErrorInvalidValue;
    static bool configured[64] = {};
    return launch_cluster(k_few_dx, configured, kDxSmem, "nf4_gemm_dx_few", a, (a.K + 127) / 128, splits, stream,
                          map_codes);
}

}  // namespace nf4lora
