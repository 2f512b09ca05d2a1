// Warp-specialised tcgen05 GEMM engine for the NF4-LoRA linear layer.
//
//   D[rows, cols] (fp32, TMEM) = sum_k A[rows, k] * B[cols, k]
//                              + sum_j A_ext[rows, j] * B_ext[cols, j]
//
// One CTA computes a (128 MSUB) x BN tile -- MSUB accumulators of 128 x BN
// (MMA M = 128, N = BN) that share every B tile -- over a range of
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
// global).  With two decode teams, team t decodes the k-steps t, t + 2, ...  Two rings of shared-memory stages, each with mbarriers:
//   load ring   (deep, small slots): the TMA-copied operand and the packed
//               codes; full = bytes landed, empty = MMAs that read it done;
//   decode ring (shallow, one decoded bf16 tile per slot): dfull = decode
//               warps wrote it, dempty = MMAs that read it done.
// The deep load ring keeps many HBM requests in flight while only a few
// decoded tiles occupy shared memory.  Every wait is bounded (common.cuh).
//
// Split-K over few tokens: the splits of one tile form a thread-block cluster
// along grid.z; every CTA of rank > 0 pushes its fp32 partial tile straight
// into a shared-memory slot of rank 0 (distributed shared memory) and arrives
// on an mbarrier there; rank 0 adds the slots in rank order -- no atomics, no
// round trip through global memory, the same sum on every run.
#pragma once

#include <cstdint>

#include "common.cuh"
#include "decode.cuh"
#include "nf4_levels.cuh"

namespace nf4lora {

enum OpSrc : int { SRC_TMA_K = 0, SRC_TMA_MN = 1, SRC_DEC_K = 2, SRC_DEC_MN = 3 };
enum EpiKind : int { EPI_BF16 = 0, EPI_F32_PART = 1, EPI_F32_PART_T = 2, EPI_CLUSTER_BF16_T = 3 };

struct GemmArgs {
    int rows;           // valid rows of D over the whole problem
    int cols;           // valid columns of D
    int k_main;         // 64-wide main k-steps in total
    int k_per_split;    // main k-steps per grid.z slice
    int k_ext;          // extension k-steps (grid.z slice 0 only)
    int ext_wrap_a;     // extension k-step j reads A_ext at (j % ext_wrap_a) when > 0
    int ext_wrap_b;     // ... and B_ext at (j % ext_wrap_b) when > 0
    int cols_fastest;   // 1: grid.x walks the column tiles and grid.y the row tiles (else the reverse)
    // NF4 operand
    const int8_t* qscale;
    const float* scale2;
    const float* scale_mean;
    const float* absmax;      // fp32 block scales, or NULL (double-quantised scales above)
    int64_t w_rows;           // d_out of the encoded weight
    int64_t w_blocks_per_row; // d_in / 64
    // epilogue
    float alpha;
    uint16_t* out;      // EPI_BF16: out[row * ldo + col]; EPI_CLUSTER_BF16_T: out[col * ldo + row]
    int64_t ldo;
    float* part;        // EPI_F32_PART: part[z * part_slice + row * ldp + col];
                        // EPI_CLUSTER_BF16_T: [tile][split][128][BN] fp32 slots
    int64_t ldp;        // EPI_F32_PART_T: part[z * part_slice + col * ldp + row]
    int64_t part_slice;
    // 1: the kernel runs as a programmatic dependent of the previous kernel on
    // the stream, which produces the extension operand (the producer waits
    // for it before the extension steps only; the main operands come from
    // kernels that completed before that one started).
    int pdl;
    // 1: a programmatic dependent that waits for the previous kernel before
    // anything else (it reads or overwrites what that kernel may still use).
    int wait_first;
};

template <int SRC>
struct OpTraits {
    static constexpr bool kDecoded = (SRC == SRC_DEC_K || SRC == SRC_DEC_MN);
    static constexpr bool kMN = (SRC == SRC_TMA_MN || SRC == SRC_DEC_MN);
};

template <int BN, int ASRC, int BSRC, int AE_MN, int BE_MN, int EPI, int LSTAGES = 0, int DSTAGES = 0, int TEAMS = 1,
          int MSUB = 1>
struct GemmConfig {
    static constexpr int kBM = 128;                           // rows of one MMA / accumulator
    static constexpr int kMSub = MSUB;                        // accumulators (128-row sub-tiles) per CTA
    static constexpr int kRows = kBM * MSUB;                  // rows of D per CTA
    static constexpr int kBK = 64;
    static constexpr bool kDecA = OpTraits<ASRC>::kDecoded;
    static constexpr bool kDecB = OpTraits<BSRC>::kDecoded;
    static_assert(!(kDecA && kDecB), "at most one decoded operand");
    static constexpr bool kHasDec = kDecA || kDecB;
    static constexpr int kTeams = kHasDec ? TEAMS : 1;
    static constexpr int kABytes = kRows * kBK * 2;           // 16 KB per sub-tile
    static constexpr int kBBytes = BN * kBK * 2;
    static constexpr int kDecMN = kDecA ? kRows : (kDecB ? BN : 0);  // decoded tile's M/N width
    static constexpr int kCBytes = kDecMN * 32;               // packed codes per k-step
    // load slot: [A tile or A codes | B tile or B codes]; decode slot: the decoded tile
    static constexpr int kLoadA = kDecA ? kCBytes : kABytes;
    static constexpr int kLoadB = kDecB ? kCBytes : kBBytes;
    static constexpr int kLoadSlot = kLoadA + kLoadB;
    static constexpr int kDecSlot = kDecA ? kABytes : (kDecB ? kBBytes : 0);
    static constexpr int kDS = kHasDec ? (DSTAGES > 0 ? DSTAGES : 3 * kTeams) : 1;
    static_assert(kDS % kTeams == 0, "each team must own whole decode slots");
    // cluster split-K: rank 0 receives the partial tiles of ranks 1 .. kPushMax - 1
    static constexpr int kPushMax = 4;
    static constexpr int kPartBytes = EPI == EPI_CLUSTER_BF16_T ? (kPushMax - 1) * kBM * BN * 4 : 0;
    static constexpr int kBudget = 225 * 1024 - (kHasDec ? kDS * kDecSlot : 0) - kPartBytes;
    static constexpr int kLSRaw = kBudget / kLoadSlot;
    static constexpr int kLSCap = kHasDec ? 2 * kDS : 8;
    static constexpr int kLSAuto = kLSRaw < kLSCap ? kLSRaw : kLSCap;
    static constexpr int kLS = LSTAGES > 0 ? LSTAGES : (kLSAuto > 8 ? 8 : kLSAuto);
    static_assert(kLS >= 2, "tile too large");
    // The producer runs at most kLS k-steps ahead of the MMAs.  Its first
    // parity wait on a decode slot (extension k-steps) is unambiguous only if
    // it cannot be two phases ahead of that slot, i.e. kLS <= 2 * kDS.
    static_assert(!kHasDec || kLS <= 2 * kDS, "load ring too deep for the decode ring");
    static_assert(kLoadA % 1024 == 0 && kLoadSlot % 1024 == 0 && kDecSlot % 1024 == 0, "swizzle alignment");
    static constexpr int kTeamThreads = kDecMN;               // one (row, block) unit each
    static constexpr int kTeamWarps = kTeamThreads / 32;
    static constexpr int kDecWarps = kTeamWarps * kTeams;
    static constexpr int kWorkWarps = kDecWarps > 4 ? kDecWarps : 4;
    static constexpr int kThreads = 64 + 32 * kWorkWarps;
    // Few-token tiles (N = 16) rotate their MMAs over kAcc independent
    // accumulators: one small MMA finishes long before the next one on the same
    // accumulator could start, so a single chain would leave the tensor core
    // idle.  The epilogue adds the accumulators in a fixed order.
    static constexpr int kAcc = EPI == EPI_CLUSTER_BF16_T ? 8 : 1;
    static_assert(kAcc == 1 || MSUB == 1, "rotating accumulators or two sub-tiles, not both");
    static constexpr int kAccCols = BN * MSUB * kAcc;
    static constexpr int kTmemCols = kAccCols <= 32 ? 32 : kAccCols <= 64 ? 64 : kAccCols <= 128 ? 128 : kAccCols <= 256 ? 256 : 512;
    static_assert(kAccCols <= 512, "accumulators exceed tensor memory");
    static_assert(MSUB == 1 || (ASRC == SRC_TMA_K && !AE_MN && EPI == EPI_BF16), "two sub-tiles: K-major A, bf16 out");
    static constexpr int kSmemBytes = kLS * kLoadSlot + (kHasDec ? kDS * kDecSlot : 0) + kPartBytes + 1024;
    // CTAs per SM the configuration is built for (registers are capped to fit)
    static constexpr int kMinBlocks = kSmemBytes <= 110 * 1024 ? 2 : 1;
    static constexpr int kTxMain = kLoadA + kLoadB;            // bytes TMA lands per main k-step
    static constexpr int kTxExt = kABytes + kBBytes;           // per extension k-step
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

// The same decode with the codebook held in registers (csrc/decode.cuh): no
// shared-memory reads, so the shared-memory port stays free for TMA, the
// decoded stores and the MMAs.
__device__ __forceinline__ void decode_unit_reg(const uint8_t* src, float s, uint8_t* dst_row, int swz) {
    uint32_t P[4], H[4];
    nf4_table(s, P, H);
    const uint4 c0 = *reinterpret_cast<const uint4*>(src);
    const uint4 c1 = *reinterpret_cast<const uint4*>(src + 16);
    const uint32_t words[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        uint32_t o[4];
        nf4_lookup4(words[j], P, H, o[0], o[1]);
        nf4_lookup4(words[j] >> 16, P, H, o[2], o[3]);
        *reinterpret_cast<uint4*>(dst_row + ((j ^ swz) << 4)) = make_uint4(o[0], o[1], o[2], o[3]);
    }
}

// Codebook used by the engine's decode warps: registers (true) or a 16-word
// shared-memory table (false).
constexpr bool kRegisterCodebook = true;

__device__ __forceinline__ void zero_row(uint8_t* dst_row) {
#pragma unroll
    for (int j = 0; j < 8; ++j) *reinterpret_cast<uint4*>(dst_row + (j << 4)) = make_uint4(0, 0, 0, 0);
}

// Programmatic dependent launch: block until the preceding kernel on the
// stream has completed and its writes are visible (returns at once when the
// kernel was not launched as a dependent).
__device__ __forceinline__ void grid_dependency_wait() {
    asm volatile("griddepcontrol.wait;" ::: "memory");
}

__device__ __forceinline__ void named_barrier_sync(int id, int threads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

template <int BN, int ASRC, int BSRC, int AE_MN, int BE_MN, int EPI, int LSTAGES = 0, int DSTAGES = 0, int TEAMS = 1,
          int MSUB = 1>
__global__ void __launch_bounds__(GemmConfig<BN, ASRC, BSRC, AE_MN, BE_MN, EPI, LSTAGES, DSTAGES, TEAMS, MSUB>::kThreads,
                                  GemmConfig<BN, ASRC, BSRC, AE_MN, BE_MN, EPI, LSTAGES, DSTAGES, TEAMS, MSUB>::kMinBlocks)
    k_gemm(const __grid_constant__ CUtensorMap map_a, const __grid_constant__ CUtensorMap map_b,
           const __grid_constant__ CUtensorMap map_ae, const __grid_constant__ CUtensorMap map_be,
           const GemmArgs args) {
    using C = GemmConfig<BN, ASRC, BSRC, AE_MN, BE_MN, EPI, LSTAGES, DSTAGES, TEAMS, MSUB>;
    constexpr int LS = C::kLS;
    constexpr int DS = C::kDS;
    constexpr int kEpiThreads = C::kWorkWarps * 32;
    extern __shared__ uint8_t smem_raw[];
    __shared__ uint64_t bar_full[LS], bar_empty[LS], bar_dfull[DS], bar_dempty[DS], bar_accum, bar_part;
    __shared__ uint32_t s_tmem;
    __shared__ int s_abort;
    __shared__ float s_lut[16];

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    bool cluster_waited = false;  // this thread has passed the cluster barrier's first phase
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base_u32 = (raw + 1023u) & ~1023u;
    uint8_t* base = smem_raw + (base_u32 - raw);
    auto load_slot = [&](int it) { return base + (it % LS) * C::kLoadSlot; };
    auto dec_slot = [&](int it) { return base + LS * C::kLoadSlot + (it % DS) * C::kDecSlot; };
    // operand tiles and codes of iteration `it`
    auto a_buf = [&](int it) { return C::kDecA ? dec_slot(it) : load_slot(it); };
    auto b_buf = [&](int it) { return C::kDecB ? dec_slot(it) : load_slot(it) + C::kLoadA; };
    auto codes_buf = [&](int it) { return load_slot(it) + (C::kDecA ? 0 : C::kLoadA); };

    // consecutive CTAs share their B operand (row tiles fastest) or their A
    // operand (column tiles fastest): the one they share is read from DRAM
    // about once, the other once per wave of CTAs
    const int r0 = (args.cols_fastest ? blockIdx.y : blockIdx.x) * C::kRows;
    const int c0 = (args.cols_fastest ? blockIdx.x : blockIdx.y) * BN;
    const int z = blockIdx.z;
    int kb_begin, kb_end;
    if constexpr (EPI == EPI_CLUSTER_BF16_T) {
        // spread main + extension k-steps evenly over the splits, split 0
        // (which also runs the extension) taking correspondingly fewer main ones
        const int splits = static_cast<int>(gridDim.z);
        const int total = args.k_main + args.k_ext;
        const int per = total / splits, extra = total % splits;
        auto start = [&](int zz) {  // first iteration index (main + ext numbering) of split zz
            return zz * per + (zz < extra ? zz : extra);
        };
        const int it0 = start(z), it1 = start(z + 1);
        // split 0 owns iterations [0, it1): its k_ext extension steps come first in
        // this numbering, so its main range is [0, it1 - k_ext)
        kb_begin = z == 0 ? 0 : it0 - args.k_ext;
        kb_end = it1 - args.k_ext;
        if (kb_end > args.k_main) kb_end = args.k_main;
        if (kb_begin < 0) kb_begin = 0;
    } else {
        kb_begin = z * args.k_per_split;
        kb_end = kb_begin + args.k_per_split;
        if (kb_end > args.k_main) kb_end = args.k_main;
    }
    const int n_main = kb_end > kb_begin ? kb_end - kb_begin : 0;
    const int n_ext = (z == 0) ? args.k_ext : 0;
    const int n_iter = n_main + n_ext;

    // the next kernel on the stream may be scheduled once every CTA of this
    // grid has started (it waits for this grid's completion before it reads
    // anything this grid writes)
    if (args.wait_first) grid_dependency_wait();
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

    if (threadIdx.x == 0) {
        for (int i = 0; i < LS; ++i) {
            mbar_init(&bar_full[i], 1);
            mbar_init(&bar_empty[i], 1);
        }
        for (int i = 0; i < DS; ++i) {
            mbar_init(&bar_dfull[i], C::kTeamWarps > 0 ? C::kTeamWarps : 1);
            mbar_init(&bar_dempty[i], 1);
        }
        mbar_init(&bar_accum, 1);
        // rank 0 of a split-K cluster: one arrival per row from every other rank
        mbar_init(&bar_part, gridDim.z > 1 ? (gridDim.z - 1) * C::kBM : 1);
        s_abort = 0;
        fence_barrier_init();
    }
    if (threadIdx.x < 16) s_lut[threadIdx.x] = nf4_level(threadIdx.x);
    // thread 0 initialised the barriers and is the producer: it goes straight
    // on to issue copies while the other threads wait for the barriers here
    // (non-aligned barrier forms: lane 0 of warp 0 arrives while its other
    // lanes wait)
    if (threadIdx.x == 0) {
        asm volatile("barrier.arrive 3, %0;" ::"r"(C::kThreads) : "memory");
    } else {
        asm volatile("barrier.sync 3, %0;" ::"r"(C::kThreads) : "memory");
    }
    volatile int* abort_flag = &s_abort;
    // split-K cluster: announce that this CTA's barriers are initialised; the
    // matching wait comes before the first access to another CTA's memory
    if constexpr (EPI == EPI_CLUSTER_BF16_T) cluster_arrive_release();

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        // (starts while warp 1 is still allocating tensor memory)
        if (lane == 0) {
            tma_prefetch_desc(&map_a);
            tma_prefetch_desc(&map_b);
            if (n_ext > 0) {
                tma_prefetch_desc(&map_ae);
                tma_prefetch_desc(&map_be);
            }
            int issued = 0;
            for (int it = 0; it < n_iter; ++it) {
                if (it >= LS && !mbar_wait(&bar_empty[it % LS], ((it / LS) & 1u) ^ 1u, abort_flag)) break;
                if (*abort_flag) break;
                uint64_t* bar = &bar_full[it % LS];
                if (it < n_main) {
                    const int kb = kb_begin + it;
                    mbar_arrive_expect_tx(bar, C::kTxMain);
                    // operand A
                    if constexpr (ASRC == SRC_TMA_K) {
#pragma unroll
                        for (int ms = 0; ms < MSUB; ++ms)
                            tma_load_2d(a_buf(it) + ms * (C::kBM * 128), &map_a, bar, kb * 64, r0 + ms * C::kBM);
                    } else if constexpr (ASRC == SRC_TMA_MN) {
                        tma_load_2d(a_buf(it), &map_a, bar, r0, kb * 64);
                        tma_load_2d(a_buf(it) + 8192, &map_a, bar, r0 + 64, kb * 64);
                    } else if constexpr (ASRC == SRC_DEC_K) {
                        tma_load_2d(codes_buf(it), &map_a, bar, kb * 32, r0);
                    } else {
                        tma_load_2d(codes_buf(it), &map_a, bar, r0 / 2, kb * 64);
                    }
                    // operand B
                    if constexpr (BSRC == SRC_TMA_K) {
                        tma_load_2d(b_buf(it), &map_b, bar, kb * 64, c0);
                    } else if constexpr (BSRC == SRC_TMA_MN) {
#pragma unroll
                        for (int c = 0; c < BN / 64; ++c)
                            tma_load_2d(b_buf(it) + c * 8192, &map_b, bar, c0 + c * 64, kb * 64);
                    } else if constexpr (BSRC == SRC_DEC_K) {
                        tma_load_2d(codes_buf(it), &map_b, bar, kb * 32, c0);
                    } else {
                        tma_load_2d(codes_buf(it), &map_b, bar, c0 / 2, kb * 64);
                    }
                } else {
                    const int j = it - n_main;
                    // an extension tile on the decoded side lands in a decode slot
                    if (C::kHasDec && it >= DS &&
                        !mbar_wait(&bar_dempty[it % DS], ((it / DS) & 1u) ^ 1u, abort_flag))
                        break;
                    // the extension operand comes from the preceding kernel
                    if (j == 0 && args.pdl) grid_dependency_wait();
                    const int ja = args.ext_wrap_a > 0 ? j % args.ext_wrap_a : j;
                    const int jb = args.ext_wrap_b > 0 ? j % args.ext_wrap_b : j;
                    mbar_arrive_expect_tx(bar, C::kTxExt);
                    if constexpr (AE_MN) {
                        tma_load_2d(a_buf(it), &map_ae, bar, r0, ja * 64);
                        tma_load_2d(a_buf(it) + 8192, &map_ae, bar, r0 + 64, ja * 64);
                    } else {
#pragma unroll
                        for (int ms = 0; ms < MSUB; ++ms)
                            tma_load_2d(a_buf(it) + ms * (C::kBM * 128), &map_ae, bar, ja * 64, r0 + ms * C::kBM);
                    }
                    if constexpr (BE_MN) {
#pragma unroll
                        for (int c = 0; c < BN / 64; ++c)
                            tma_load_2d(b_buf(it) + c * 8192, &map_be, bar, c0 + c * 64, jb * 64);
                    } else {
                        tma_load_2d(b_buf(it), &map_be, bar, jb * 64, c0);
                    }
                }
                ++issued;
            }
            if (*abort_flag) {
                // let the copies already issued land before the CTA exits
                const int first = issued > LS ? issued - LS : 0;
                for (int it = first; it < issued; ++it) mbar_drain(&bar_full[it % LS], (it / LS) & 1u);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ TMEM + MMA issuer
        tmem_alloc(&s_tmem, C::kTmemCols);
        tmem_relinquish();
        tc_fence_before();
        // hand the tensor-memory address to the epilogue warps
        asm volatile("bar.arrive 2, %0;" ::"r"(32 + kEpiThreads) : "memory");
        __syncwarp();
        tc_fence_after();
        const uint32_t tmem_d = s_tmem;
        if (lane == 0) {
            for (int it = 0; it < n_iter; ++it) {
                if (!mbar_wait(&bar_full[it % LS], (it / LS) & 1u, abort_flag)) break;
                const bool is_main = it < n_main;
                if (C::kHasDec && is_main && !mbar_wait(&bar_dfull[it % DS], (it / DS) & 1u, abort_flag)) break;
                tc_fence_after();
                const uint32_t a_base = smem_u32(a_buf(it));
                const uint32_t b_base = smem_u32(b_buf(it));
                const bool a_mn = is_main ? OpTraits<ASRC>::kMN : (AE_MN != 0);
                const bool b_mn = is_main ? OpTraits<BSRC>::kMN : (BE_MN != 0);
                const uint32_t idesc = is_main ? C::kIdescMain : C::kIdescExt;
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) {
                    const uint64_t bdesc = tile_desc(b_base, b_mn, kk);
#pragma unroll
                    for (int ms = 0; ms < MSUB; ++ms) {  // sub-tile ms: rows 128 ms.., columns ms BN..
                        const int mi = it * 4 + kk;      // MMA index; with kAcc > 1 it picks the accumulator
                        const uint32_t dcol = C::kAcc > 1 ? (mi % C::kAcc) * BN : ms * BN;
                        const uint32_t accumulate = C::kAcc > 1 ? (mi >= C::kAcc ? 1u : 0u) : (mi > 0 ? 1u : 0u);
                        mma_bf16_ss(tmem_d + dcol, tile_desc(a_base + ms * C::kBM * 128, a_mn, kk), bdesc, idesc,
                                    accumulate);
                    }
                }
                mma_commit(&bar_empty[it % LS]);
                if (C::kHasDec) mma_commit(&bar_dempty[it % DS]);
            }
            mma_commit(&bar_accum);
        }
    } else {
        const int ew = warp - 2;
        // ------------------------------------------------------------ decoders
        if constexpr (C::kHasDec) {
            if (ew < C::kDecWarps) {
                const int team = ew / C::kTeamWarps;
                const int dt = threadIdx.x - 64 - team * C::kTeamThreads;
                // fp32 block scales (no double quantisation) when absmax is set
                const bool fp32_scales = args.absmax != nullptr;
                const float mu = fp32_scales ? 0.0f : __ldg(args.scale_mean);
                constexpr bool kMNdec = C::kDecA ? (ASRC == SRC_DEC_MN) : (BSRC == SRC_DEC_MN);
                constexpr int kCB = C::kDecMN / 64;           // 64-blocks across the decoded tile
                const int tile_mn0 = C::kDecA ? r0 : c0;
                // MN-major: this thread's unit is (k-row n_local of the step, block c
                // of the tile).  The eight threads of a quarter warp take eight
                // consecutive rows (their swizzled 16-byte stores hit eight
                // different bank groups) and blocks spread so that their 32-byte
                // code reads land at most two to a bank group.
                int n_local = dt, cblk = 0;
                if constexpr (kMNdec) {
                    const int qw = dt >> 3, i = dt & 7;
                    n_local = 8 * (qw / kCB) + i;
                    cblk = ((i * kCB) / 4 + qw % kCB) % kCB;
                }
                // (weight row, 64-block) decoded by this thread at main step `it`
                auto unit = [&](int it, int64_t& wrow, int64_t& wblk) {
                    const int kb = kb_begin + it;
                    if constexpr (!kMNdec) {
                        wrow = tile_mn0 + dt;
                        wblk = kb;
                    } else {
                        wrow = static_cast<int64_t>(kb) * 64 + n_local;
                        wblk = tile_mn0 / 64 + cblk;
                    }
                };
                int dst_off, swz, code_off;
                if constexpr (!kMNdec) {
                    dst_off = dt * 128;
                    swz = dt & 7;
                    code_off = dt * 32;
                } else {
                    dst_off = cblk * 8192 + n_local * 128;
                    swz = n_local & 7;
                    code_off = (n_local * kCB + cblk) * 32;  // codes tile: [64 k-rows][kCB blocks x 32 bytes]
                }
                // Block scales are prefetched kPf of this team's steps ahead
                // into registers, so no decode waits on a dependent load.
                constexpr int kPf = 4;
                constexpr int kStride = C::kTeams;
                int8_t q_pf[kPf];
                float a2_pf[kPf];
                bool ok_pf[kPf];
                auto fetch = [&](int it, int slot) {
                    int64_t wrow, wblk;
                    unit(it, wrow, wblk);
                    ok_pf[slot] = it < n_main && wrow < args.w_rows && wblk < args.w_blocks_per_row;
                    if (ok_pf[slot]) {
                        const int64_t bidx = wrow * args.w_blocks_per_row + wblk;
                        if (fp32_scales) {
                            q_pf[slot] = 0;
                            a2_pf[slot] = __ldg(args.absmax + bidx);
                        } else {
                            q_pf[slot] = __ldg(args.qscale + bidx);
                            a2_pf[slot] = __ldg(args.scale2 + (bidx >> 8));
                        }
                    }
                };
#pragma unroll
                for (int u = 0; u < kPf; ++u) fetch(team + u * kStride, u);
                bool stop = false;
                for (int base_it = team; base_it < n_main && !stop; base_it += kPf * kStride) {
#pragma unroll
                    for (int u = 0; u < kPf; ++u) {
                        const int it = base_it + u * kStride;
                        if (it >= n_main) break;
                        const bool valid = ok_pf[u];
                        const float sc =
                            valid ? (fp32_scales ? a2_pf[u] : nf4_block_scale(q_pf[u], a2_pf[u], mu)) : 0.0f;
                        fetch(it + kPf * kStride, u);
                        if (!mbar_wait(&bar_full[it % LS], (it / LS) & 1u, abort_flag) ||
                            (it >= DS && !mbar_wait(&bar_dempty[it % DS], ((it / DS) & 1u) ^ 1u, abort_flag))) {
                            stop = true;
                            break;
                        }
                        uint8_t* dst = dec_slot(it) + dst_off;
                        if (!valid) zero_row(dst);
                        else if constexpr (kRegisterCodebook) decode_unit_reg(codes_buf(it) + code_off, sc, dst, swz);
                        else decode_unit(codes_buf(it) + code_off, sc, dst, swz, s_lut);
                        fence_proxy_async_smem();
                        __syncwarp();
                        if (lane == 0) mbar_arrive(&bar_dfull[it % DS]);
                    }
                }
            }
        }
        // ------------------------------------------------------------ epilogue
        asm volatile("bar.sync 2, %0;" ::"r"(32 + kEpiThreads) : "memory");
        tc_fence_after();
        const uint32_t tmem_d = s_tmem;
        const int q = warp & 3;                       // TMEM lane quadrant of this warp
        constexpr int kColSplit = C::kWorkWarps / 4;  // warps sharing one quadrant
        const int part_idx = ew / 4;
        const int cw = BN / kColSplit;
        const int cbeg = part_idx * cw;
        const bool ok = mbar_wait(&bar_accum, 0, abort_flag);
        tc_fence_after();
        if constexpr (EPI != EPI_CLUSTER_BF16_T) if (ok && !*abort_flag) {
          for (int ms = 0; ms < MSUB; ++ms) {
            const int row = r0 + ms * C::kBM + q * 32 + lane;
            const bool row_ok = row < args.rows;
            for (int cc = cbeg; cc < cbeg + cw; cc += 32) {
                uint32_t v[32];
                tmem_ld_32x32b_x32(tmem_d + (static_cast<uint32_t>(q * 32) << 16) + ms * BN + cc, v);
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
                } else {  // EPI_F32_PART_T
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
        if constexpr (EPI == EPI_CLUSTER_BF16_T) {
            // ranks > 0 push their fp32 partial tile into slot rank - 1 of
            // rank 0; rank 0 adds the slots to its own tile in rank order
            if (ew < 4) {
                const int rl = q * 32 + lane;  // row within the tile
                const uint32_t rank = cluster_ctarank();
                const int splits = static_cast<int>(gridDim.z);
                float* s_part = reinterpret_cast<float*>(base + LS * C::kLoadSlot + DS * C::kDecSlot);
                const bool have = ok && !*abort_flag;
                // this CTA's partial: the used accumulators added in index order
                float part[BN];
#pragma unroll
                for (int j = 0; j < BN; ++j) part[j] = 0.0f;
                if (have) {
                    const int used = n_iter * 4 < C::kAcc ? n_iter * 4 : C::kAcc;
                    static_assert(32 % BN == 0 && (C::kAcc * BN) % 32 == 0, "accumulator loads of 32 columns");
#pragma unroll
                    for (int c = 0; c < C::kAcc * BN; c += 32) {
                        uint32_t v[32];
                        tmem_ld_32x32b_x32(tmem_d + (static_cast<uint32_t>(q * 32) << 16) + c, v);
                        tmem_ld_wait();
#pragma unroll
                        for (int j = 0; j < 32; ++j)
                            if ((c + j) / BN < used) part[(c + j) % BN] += __uint_as_float(v[j]);
                    }
                }
                if (rank != 0) {
                    cluster_wait_acquire();  // rank 0's barrier is initialised
                    cluster_waited = true;
                    if (have) {
                        const uint32_t dst = cluster_map(smem_u32(s_part + ((rank - 1) * C::kBM + rl) * BN), 0);
#pragma unroll
                        for (int j = 0; j < BN; j += 4)
                            st_cluster_f4(dst + 4 * j, part[j], part[j + 1], part[j + 2], part[j + 3]);
                    }
                    // arrive even without data, so that rank 0 never waits out
                    // the time limit for a rank that gave up (the device status
                    // word already reports it)
                    mbar_arrive_remote(cluster_map(smem_u32(&bar_part), 0));
                } else {
                    const bool got = splits == 1 || mbar_wait_cluster(&bar_part, 0, abort_flag);
                    if (have && got && !*abort_flag) {
                        float acc[BN];
#pragma unroll
                        for (int j = 0; j < BN; ++j) acc[j] = part[j];
                        for (int rk = 1; rk < splits; ++rk) {
                            const float4* src = reinterpret_cast<const float4*>(s_part + ((rk - 1) * C::kBM + rl) * BN);
#pragma unroll
                            for (int j = 0; j < BN / 4; ++j) {
                                const float4 t = src[j];
                                acc[4 * j] += t.x;
                                acc[4 * j + 1] += t.y;
                                acc[4 * j + 2] += t.z;
                                acc[4 * j + 3] += t.w;
                            }
                        }
                        const int row = r0 + rl;
                        if (row < args.rows) {
#pragma unroll
                            for (int j = 0; j < BN; ++j) {
                                if (j < args.cols) {
                                    const __nv_bfloat16 h = __float2bfloat16_rn(acc[j] * args.alpha);
                                    args.out[static_cast<int64_t>(j) * args.ldo + row] =
                                        *reinterpret_cast<const uint16_t*>(&h);
                                }
                            }
                        }
                    }
                }
            }
        }
    }

    if constexpr (EPI == EPI_CLUSTER_BF16_T) {
        // no CTA leaves while another may still write into its shared memory
        if (!cluster_waited) cluster_wait_acquire();
        cluster_arrive_release();
        cluster_wait_acquire();
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(s_tmem, C::kTmemCols);
    }
}

}  // namespace nf4lora
