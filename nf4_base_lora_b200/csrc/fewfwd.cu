// Few-token (M <= 16) fused NF4-LoRA forward:
//
//   Y[t, n] = sum_k X[t, k] W_hat[n, k] + sum_j T2[t, j] [B | B][n, j]
//
// ("第 04 篇：QLoRA 原理" §2.3 decode on demand, §6.1-§6.3; T2 holds the
// rank-r intermediate s X A^T as a bf16 hi | lo pair.)
//
// With at most 16 tokens the layer is a streamed matrix-vector product: per
// weight the GPU reads 4.127 bits and decodes them, and the 16 dot products
// are a small tail.  The kernel is built so that every SM streams from the
// first cycle to the last:
//
// * Partition.  Weight rows go in octets (8 rows); a thread-block cluster of
//   two CTAs owns O consecutive octets and splits the contraction in two
//   halves of whole block quads (4 x 64 weights).  74 clusters of two fill
//   the 148 SMs of a B200, and octet granularity keeps them within one octet
//   of even (4096 rows: 7 octets per cluster).
// * Streaming.  The CTA's quads go through a ring of stages, each stage one
//   quad: the packed codes of all O octets and the quad's four 64-column
//   activation boxes of the token rows, all by TMA with the 128-byte swizzle,
//   completing on the stage's barrier (rows beyond M and blocks beyond K read
//   as zeros).  Thread 0 initialises the barriers and issues the first two
//   stages before the CTA barrier; after it, lane 0 of warp w issues stages
//   w, w + 16, ... of the rest that fit the ring, so every stage that fits
//   is in flight from the start; where the ring is shorter than the CTA's
//   quads, the last warp to finish with a stage refills it.  Lanes 1 .. 31 of
//   every warp stage the block-scale codes and the second-level steps
//   a2 / 127 of the CTA's rows once in shared memory (or the fp32 block
//   scales of the format without double quantisation).
// * Decode.  Each lane holds the 16 scaled levels of one (row, block) as byte
//   planes in registers (csrc/decode.cuh) and turns four codes into two
//   bf16 pairs with eight byte permutes; the pairs are the A operand of the
//   warp-level tensor instruction (mma.sync m16n8k16, bf16 in, fp32
//   accumulate: 16 weight rows, the rows g and g + 8 of an octet pair, by 16
//   columns) whose B operand is eight tokens of activations.  Lane (g, q) of
//   a warp covers rows g and g + 8 of a pair and block q of a quad; the
//   16-wide contraction of each MMA takes four consecutive columns of every
//   lane's block, so one scale serves a lane for a whole block.  Lane q walks
//   its block's words in the order j ^ 2q (its code words are loaded in that
//   order), which puts the 16-byte activation loads of a quarter warp (two
//   tokens, four blocks) on eight different bank groups of the swizzled
//   boxes; the 8-byte code loads of a half warp are conflict-free too.
// * Reduction.  Warps of one pair group add their partials in shared memory
//   in a fixed order; the two CTAs of a cluster then each finish half the
//   octets: the other half's partials go to the peer through distributed
//   shared memory, and the owner adds the two and writes bf16 rows.  The
//   rank-r term is computed by the owner for its octets once the kernel
//   producing T2 has finished (programmatic dependent launch; lane 0 of the
//   last warp that issues a first stage also copies the owner's rows of B,
//   then waits for that kernel and copies T2).  The summation order is
//   fixed, so the result is the same on every run.
//
// Launch overlap: the kernel releases its own dependents as soon as it starts,
// and reads the activations, the encoded weight and B before its wait: the
// rank-r kernel it depends on released it only after waiting for the kernel
// before that, so every earlier write is complete.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>

#include "common.cuh"
#include "decode.cuh"
#include "kernels.h"
#include "nf4_levels.cuh"
#include "trace.h"

namespace nf4lora {

namespace {

constexpr int kWarps = 16;                        // consumer warps
constexpr int kThreads = kWarps * 32;
constexpr int kTok = 16;
constexpr int kXBox = kTok * 128;                 // one block of activations: 16 token rows x 64 bf16
constexpr int kXStage = 4 * kXBox;                // a quad: 8192 bytes
constexpr int kMaxRing = 24;
constexpr int kMaxPPW = 4;                        // octet pairs per warp (largest instance)
constexpr int kMaxBoxRows = 256;
constexpr int kStageLoads = 8;                    // scale codes per thread per staging round
constexpr int kEarly = 2;                         // stages thread 0 issues before the CTA barrier
constexpr int kSmemLimit = 227 * 1024 - 1024;  // room for the static barriers

__device__ __forceinline__ void mma_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                          uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Shared-memory loads by 32-bit shared address.  Volatile, so that they stay
// after the barrier waits that make the asynchronous copies visible.
__device__ __forceinline__ uint4 lds128(uint32_t addr) {
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
    return v;
}
__device__ __forceinline__ uint2 lds64(uint32_t addr) {
    uint2 v;
    asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(addr));
    return v;
}
__device__ __forceinline__ float lds_f32(uint32_t addr) {
    float v;
    asm volatile("ld.shared.f32 %0, [%1];" : "=f"(v) : "r"(addr));
    return v;
}
__device__ __forceinline__ int lds_s8(uint32_t addr) {
    int v;
    asm volatile("ld.shared.s8 %0, [%1];" : "=r"(v) : "r"(addr));
    return v;
}

// Four codes -> two bf16 pairs with the selectors precomputed for a whole
// code word: sel = w & 0x77777777 (index within an 8-entry half), pick =
// ((w >> 1) & 0x44444444) | 0x32103210 (entry from the upper half if bit 3).
__device__ __forceinline__ void lookup4_sel(uint32_t sel, uint32_t pick, const uint32_t (&P)[4],
                                            const uint32_t (&H)[4], uint32_t& p0, uint32_t& p1) {
    const uint32_t lo = __byte_perm(__byte_perm(P[0], P[1], sel), __byte_perm(P[2], P[3], sel), pick);
    const uint32_t hi = __byte_perm(__byte_perm(H[0], H[1], sel), __byte_perm(H[2], H[3], sel), pick);
    p0 = __byte_perm(lo, hi, 0x4051);
    p1 = __byte_perm(lo, hi, 0x6273);
}

struct Geometry {
    int rank, cl, oct0, Oc, row0, rows, qa, nqc, kb0, kb1, nbc, own0, own1;
};

__device__ __forceinline__ Geometry geometry(const FewArgs& a, const FewFwdPlan& p) {
    Geometry G;
    G.rank = p.cs > 1 ? static_cast<int>(cluster_ctarank()) : 0;
    G.cl = static_cast<int>(blockIdx.x) / p.cs;
    const int noct = a.N / 8;
    G.oct0 = G.cl * p.O;
    G.Oc = min(p.O, noct - G.oct0);
    G.row0 = 8 * G.oct0;
    G.rows = 8 * G.Oc;
    const int nb = a.K / 64, nq = (nb + 3) / 4;
    G.qa = G.rank == 0 ? 0 : p.nq0;
    const int qb = (p.cs == 1 || G.rank == 1) ? nq : p.nq0;
    G.nqc = qb - G.qa;
    G.kb0 = 4 * G.qa;
    G.kb1 = min(nb, 4 * qb);
    G.nbc = G.kb1 - G.kb0;
    // octets this CTA finishes (adds the peer's partials, the rank-r term, writes Y)
    const int half = p.cs > 1 ? (G.Oc + 1) / 2 : G.Oc;
    G.own0 = G.rank == 0 ? 0 : half;
    G.own1 = G.rank == 0 ? half : G.Oc;
    return G;
}

template <int PPW, bool TWO>
__global__ void __launch_bounds__(kThreads, 1) k_few_fwd(const __grid_constant__ CUtensorMap map_codes,
                                                          const __grid_constant__ CUtensorMap map_x, const FewArgs a,
                                                          const FewFwdPlan p) {
    // only 16-byte alignment is guaranteed (and declared: a larger __align__
    // would let the compiler drop the round-up below); TMA boxes with the
    // 128-byte swizzle need 1024-byte aligned shared addresses
    extern __shared__ __align__(16) uint8_t smem_raw[];
    __shared__ uint64_t bar_full[kMaxRing], bar_lora, bar_b, bar_staged;
    __shared__ int s_done[kMaxRing];   // warps finished with the stage's current contents
    __shared__ int s_fills[kMaxRing];  // fills issued into each stage
    __shared__ int s_abort, s_lora;
    pdl_launch_dependents();
    const uint32_t raw = smem_u32(smem_raw);
    uint8_t* base = smem_raw + (((raw + 1023u) & ~1023u) - raw);
    uint8_t* ring = base;                                               // NR x slot
    int8_t* s_q = reinterpret_cast<int8_t*>(ring + p.NR * p.slot);       // [rows][qrow]
    float* s_step = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(s_q) + p.q_bytes);  // [ngroups]
    uint16_t* s_t2 = reinterpret_cast<uint16_t*>(reinterpret_cast<uint8_t*>(s_step) + p.step_bytes);  // [M][2 r64]
    uint16_t* s_b = reinterpret_cast<uint16_t*>(reinterpret_cast<uint8_t*>(s_t2) + p.t2_bytes);       // owned rows of B
    float* s_recv = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(s_b) + p.b_bytes);           // peer partials

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, g = lane >> 2, q = lane & 3;
    const Geometry G = geometry(a, p);
    const int M = a.M, N = a.N, K = a.K, bpr = K / 64;
    const int WP = kWarps / p.WQ;
    const int P = (G.Oc + 1) / 2;  // octet pairs of this CTA
    const bool lora = a.ext_act != nullptr && G.own1 > G.own0;
    constexpr bool two = TWO;      // tokens 8 .. 15 exist (M > 8)
    const int n_first = min(p.NR, G.nqc);  // stages issued at the start

    // one stage: the codes of the O octets and the quad's four activation
    // blocks (rows beyond M and blocks beyond K read as zeros), by one thread
    auto issue_stage = [&](int i) {
        const int slot = i % p.NR;
        const int quad = G.qa + i;
        uint8_t* st = ring + slot * p.slot;
        mbar_arrive_expect_tx(&bar_full[slot], p.code_bytes + 4 * p.xbox_bytes);
        for (int b = 0; b < p.nbox; ++b)
            if (NF4_CHECK(in_smem(st + b * p.box_rows * 128, p.box_rows * 128, ring, int64_t(p.NR) * p.slot, 1024),
                          12))
                tma_load_2d(st + b * p.box_rows * 128, &map_codes, &bar_full[slot], 128 * quad,
                            G.row0 + b * p.box_rows);
        uint8_t* xs = st + p.code_bytes;
        for (int b = 0; b < 4; ++b)
            if (NF4_CHECK(in_smem(xs + b * kXBox, kXBox, st, p.slot, 1024), 11))
                tma_load_2d(xs + b * kXBox, &map_x, &bar_full[slot], 256 * quad + 64 * b, 0);
        s_fills[slot] += 1;
    };

    // thread 0 initialises the barriers and puts the first stages in flight
    // before anything else, so that the weight stream starts at once
    if (tid == 0) {
        tma_prefetch_desc(&map_codes);
        tma_prefetch_desc(&map_x);
        for (int i = 0; i < p.NR; ++i) {
            mbar_init(&bar_full[i], 1);
            s_done[i] = 0;
            s_fills[i] = 0;
        }
        mbar_init(&bar_lora, 1);
        mbar_init(&bar_b, 1);
        mbar_init(&bar_staged, kWarps * 31);  // lanes 1 .. 31 of every warp stage the scales
        s_abort = 0;
        s_lora = 0;
        fence_barrier_init();
        for (int i = 0; i < min(n_first, kEarly); ++i) issue_stage(i);
    }

    // lanes 1 .. 31 of every warp stage the block-scale codes and the
    // second-level steps of the CTA's rows; their first loads are issued
    // before any copy of the weight stream, so that they are not queued
    // behind it
    const bool stager = lane != 0;
    const int sidx = warp * 31 + lane - 1, nst = kWarps * 31;
    const int nq_el = G.rows * G.nbc;
    // e / nbc = umulhi(e, magic), exact for e < 2^32 / nbc; nbc = 1 is e itself
    // (its magic, 2^32, does not fit in 32 bits)
    const uint32_t magic = G.nbc > 1 ? 0xFFFFFFFFu / static_cast<uint32_t>(G.nbc) + 1u : 0u;
    const int g0s = (G.row0 * bpr + G.kb0) >> 8;
    const int g1s = ((G.row0 + G.rows - 1) * bpr + G.kb1 - 1) >> 8;
    // fp32 block scales (no double quantisation): staged as floats after the
    // CTA barrier, and no second-level steps
    const bool fp32_scales = a.absmax != nullptr;
    int8_t v[kStageLoads];
    float a2 = 0.0f;
    if (stager && !fp32_scales) {
        if (sidx <= g1s - g0s) a2 = __ldcg(a.scale2 + g0s + sidx);
#pragma unroll
        for (int u = 0; u < kStageLoads; ++u) {
            const int e = u * nst + sidx;
            v[u] = 0;
            if (e < nq_el) {
                const int lr = G.nbc > 1 ? static_cast<int>(__umulhi(static_cast<uint32_t>(e), magic)) : e;
                v[u] = __ldcg(a.qscale + (G.row0 + lr) * bpr + G.kb0 + (e - lr * G.nbc));
            }
        }
    }
    const float mu = fp32_scales ? 0.0f : __ldcg(a.scale_mean);
    __syncthreads();
    if (p.cs > 1) cluster_arrive_relaxed();  // barriers initialised; the peer may address this CTA after its wait
    volatile int* abort_flag = &s_abort;

    if (lane == 0) {
        // the rest of the first stages, spread over the warps (the ring may
        // be deeper than there are warps)
        for (int i = warp; i < n_first; i += kWarps)
            if (i >= kEarly) issue_stage(i);
        if (warp == min(n_first, kWarps) - 1 && lora) {
            // the owner's rows of B (written before the kernel this one depends
            // on released it), then T2 once that kernel has finished
            const uint32_t bb = static_cast<uint32_t>(8 * (G.own1 - G.own0) * 2 * a.r);
            const uint16_t* bsrc = a.ext_w + static_cast<int64_t>(G.row0 + 8 * G.own0) * a.r;
            mbar_arrive_expect_tx(&bar_b, bb);
            if (NF4_CHECK(in_smem(s_b, bb, s_b, p.b_bytes, 16) && in_span(bsrc, bb, a.ext_w, int64_t(N) * a.r * 2, 16),
                          13))
                bulk_load(s_b, bsrc, bb, &bar_b);
            if (a.pdl) pdl_wait();
            const uint32_t t2b = static_cast<uint32_t>(M * 4 * a.r64);
            mbar_arrive_expect_tx(&bar_lora, t2b);
            if (NF4_CHECK(in_smem(s_t2, t2b, s_t2, p.t2_bytes, 16) &&
                              in_span(a.ext_act, t2b, a.ext_act, int64_t(M) * 4 * a.r64, 16),
                          13))
                bulk_load(s_t2, a.ext_act, t2b, &bar_lora);
            s_lora = 1;
        }
    } else if (fp32_scales) {
        float* s_qf = reinterpret_cast<float*>(s_q);
        for (int e = sidx; e < nq_el; e += nst) {
            const int lr = G.nbc > 1 ? static_cast<int>(__umulhi(static_cast<uint32_t>(e), magic)) : e;
            const int qi = lr * p.qrow + (e - lr * G.nbc);
            if (NF4_CHECK(4 * (qi + 1) <= p.q_bytes, 14))
                s_qf[qi] = __ldcg(a.absmax + (G.row0 + lr) * bpr + G.kb0 + (e - lr * G.nbc));
        }
        mbar_arrive(&bar_staged);
    } else {
        // store the first round; later rounds (large row counts only) load and
        // store in turn
        for (int e0 = 0; e0 < nq_el; e0 += nst * kStageLoads) {
            if (e0 > 0) {
#pragma unroll
                for (int u = 0; u < kStageLoads; ++u) {
                    const int e = e0 + u * nst + sidx;
                    v[u] = 0;
                    if (e < nq_el) {
                        const int lr = G.nbc > 1 ? static_cast<int>(__umulhi(static_cast<uint32_t>(e), magic)) : e;
                        v[u] = __ldcg(a.qscale + (G.row0 + lr) * bpr + G.kb0 + (e - lr * G.nbc));
                    }
                }
            }
#pragma unroll
            for (int u = 0; u < kStageLoads; ++u) {
                const int e = e0 + u * nst + sidx;
                if (e < nq_el) {
                    const int lr = G.nbc > 1 ? static_cast<int>(__umulhi(static_cast<uint32_t>(e), magic)) : e;
                    const int qi = lr * p.qrow + (e - lr * G.nbc);
                    if (NF4_CHECK(qi < p.q_bytes, 14)) s_q[qi] = v[u];
                }
            }
        }
        for (int e = sidx; e <= g1s - g0s; e += nst)
            if (NF4_CHECK(4 * (e + 1) <= p.step_bytes, 15))
                s_step[e] = __fdiv_rn(e == sidx ? a2 : __ldcg(a.scale2 + g0s + e), 127.0f);
        mbar_arrive(&bar_staged);  // releases the stores above to the waiting threads
    }
    const int g0 = g0s;
    mbar_wait(&bar_staged, 0, abort_flag);

    const int wq = warp % p.WQ, wp = warp / p.WQ;
    // acc[pp][h]: rows g, g + 8 of pair pp (octets 2 pr, 2 pr + 1) x tokens 8 h + 2q, + 1
    float acc[PPW][2][4];
#pragma unroll
    for (int pp = 0; pp < PPW; ++pp)
#pragma unroll
        for (int h = 0; h < 2; ++h)
#pragma unroll
            for (int e = 0; e < 4; ++e) acc[pp][h][e] = 0.0f;

    const uint32_t ring_s = smem_u32(ring);
    const uint32_t sq_s = smem_u32(s_q), sstep_s = smem_u32(s_step);
    // the lane's 8-byte code pieces of its block in the order jj ^ q (a row's
    // 16-byte chunks are swizzled by the row index, which is g modulo 8)
    uint32_t coff[4];
#pragma unroll
    for (int jj = 0; jj < 4; ++jj) {
        const int pw = jj ^ q;
        coff[jj] = static_cast<uint32_t>((((2 * q + (pw >> 1)) ^ g) << 4) + 8 * (pw & 1));
    }
    for (int i = wq; i < G.nqc; i += p.WQ) {
        const int slot = i % p.NR;
        if (!mbar_wait(&bar_full[slot], (i / p.NR) & 1, abort_flag)) break;
        const uint32_t st_s = ring_s + slot * p.slot;
        const uint8_t* st = ring + slot * p.slot;  // the same stage, for the debug checks
        (void)st;
        const int bl = 4 * i + q;                    // this lane's block, relative to kb0
        const bool blk_ok = G.kb0 + bl < G.kb1;
        // block q, token g (g + 8: + 1024); the 16-byte chunk of word j is
        // j ^ 2q, stored at chunk j ^ 2q ^ g of the swizzled row (x0 is
        // 128-byte aligned, so the XOR reaches only the chunk bits)
        const uint32_t x0 = (st_s + p.code_bytes + q * kXBox + g * 128) | (((2 * q) ^ g) << 4);
#pragma unroll
        for (int pp = 0; pp < PPW; ++pp) {
            const int pr = wp + pp * WP;
            if (pr < P) {  // the same for the whole warp
                const bool has1 = 2 * pr + 1 < G.Oc;
                uint32_t PT[2][4], HT[2][4], w[2][8];
#pragma unroll
                for (int o = 0; o < 2; ++o) {
                    const int lr = 16 * pr + 8 * o + g;  // local row; lr & 7 == g
                    const bool row_ok = o == 0 || has1;  // the second octet of the pair may not exist
                    float sc = 0.0f;
                    if (blk_ok && row_ok) {
                        const int bi = (G.row0 + lr) * bpr + G.kb0 + bl;
                        const int qi = lr * p.qrow + bl;
                        const int si = (bi >> 8) - g0;
                        if (fp32_scales) {
                            if (NF4_CHECK(4 * (qi + 1) <= p.q_bytes, 3))
                                sc = lds_f32(sq_s + 4 * static_cast<uint32_t>(qi));
                        } else if (NF4_CHECK(qi < p.q_bytes, 3) &&
                                   NF4_CHECK(si >= 0 && 4 * (si + 1) <= p.step_bytes, 4)) {
                            sc = __fadd_rn(__fmul_rn(static_cast<float>(lds_s8(sq_s + qi)),
                                                     lds_f32(sstep_s + 4 * static_cast<uint32_t>(si))),
                                           mu);
                        }
                    }
                    nf4_table(sc, PT[o], HT[o]);
                    const uint32_t crow = st_s + lr * 128;
                    const bool cok = row_ok && NF4_CHECK(in_smem(st + lr * 128, 128, st, p.code_bytes, 16), 1);
#pragma unroll
                    for (int jj = 0; jj < 4; ++jj) {
                        uint2 c = make_uint2(0, 0);
                        if (cok) c = lds64(crow + coff[jj]);
                        w[o][2 * jj] = c.x;
                        w[o][2 * jj + 1] = c.y;
                    }
                }
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    // word j of the walk = stored word j ^ 2q of the lane's block and
                    // the activations of the same 16-byte chunk
                    const uint32_t xj = x0 ^ static_cast<uint32_t>(j << 4);
                    const uint4 xa = lds128(xj);                                       // tokens 0 .. 7
                    const uint4 xb = two ? lds128(xj + 1024) : make_uint4(0, 0, 0, 0);  // tokens 8 .. 15
                    uint32_t r0[4], r1[4];  // A fragments of the two chunks: rows g, g + 8
                    {
                        const uint32_t sel = w[0][j] & 0x77777777u;
                        const uint32_t pick = ((w[0][j] >> 1) & 0x44444444u) | 0x32103210u;
                        lookup4_sel(sel, pick, PT[0], HT[0], r0[0], r0[2]);
                        lookup4_sel(sel >> 16, pick >> 16, PT[0], HT[0], r1[0], r1[2]);
                    }
                    {
                        // a missing second octet has zero codes and a zero table
                        const uint32_t sel = w[1][j] & 0x77777777u;
                        const uint32_t pick = ((w[1][j] >> 1) & 0x44444444u) | 0x32103210u;
                        lookup4_sel(sel, pick, PT[1], HT[1], r0[1], r0[3]);
                        lookup4_sel(sel >> 16, pick >> 16, PT[1], HT[1], r1[1], r1[3]);
                    }
                    mma_16816(acc[pp][0], r0[0], r0[1], r0[2], r0[3], xa.x, xa.y);
                    mma_16816(acc[pp][0], r1[0], r1[1], r1[2], r1[3], xa.z, xa.w);
                    if (two) {
                        mma_16816(acc[pp][1], r0[0], r0[1], r0[2], r0[3], xb.x, xb.y);
                        mma_16816(acc[pp][1], r1[0], r1[1], r1[2], r1[3], xb.z, xb.w);
                    }
                }
            }
        }
        __syncwarp();
        if (lane == 0 && i + p.NR < G.nqc) {
            // the last of the WP warps done with this stage refills it: their
            // reads are ordered before the counter, and the copies after it
            __threadfence_block();
            if (atomicAdd(&s_done[slot], 1) == WP - 1) {
                s_done[slot] = 0;
                __threadfence_block();
                fence_proxy_async_smem();
                issue_stage(i + p.NR);
            }
        }
    }

    // rank-r term for the octets this CTA finishes: 16-wide chunks of
    // [B | B] (rows) x [T2 hi | T2 lo]^T dealt to the warps of each pair group
    if (lora && !*abort_flag) {
        if (mbar_wait(&bar_b, 0, abort_flag) && mbar_wait(&bar_lora, 0, abort_flag)) {
            const int nch = a.r64 / 8;
            const int rs = a.r;
#pragma unroll
            for (int pp = 0; pp < PPW; ++pp) {
                const int pr = wp + pp * WP;
                const bool own0 = 2 * pr >= G.own0 && 2 * pr < G.own1;
                const bool own1 = 2 * pr + 1 >= G.own0 && 2 * pr + 1 < G.own1;
                if (pr < P && (own0 || own1)) {
                    for (int ch = wq; ch < nch; ch += p.WQ) {
                        const int j0 = 16 * ch + 2 * q;
                        uint32_t af[4];  // rows g (octet 2 pr), g + 8 (octet 2 pr + 1) of [B | B]
#pragma unroll
                        for (int u = 0; u < 4; ++u) {
                            const int o = u & 1, h = u >> 1;
                            const bool ok = o == 0 ? own0 : own1;
                            const int lrb = 8 * (2 * pr + o - G.own0) + g;  // row within the staged B rows
                            const int jj = (j0 + 8 * h) % a.r64;             // column of B (the same in both halves)
                            uint32_t lo = 0u, hi = 0u;
                            if (ok) {
                                const uint16_t* br = s_b + lrb * rs;
                                if (jj < rs && NF4_CHECK(in_smem(br + jj, 2, s_b, p.b_bytes, 2), 6)) lo = br[jj];
                                if (jj + 1 < rs && NF4_CHECK(in_smem(br + jj + 1, 2, s_b, p.b_bytes, 2), 6)) hi = br[jj + 1];
                            }
                            af[u] = lo | (hi << 16);
                        }
#pragma unroll
                        for (int h = 0; h < 2; ++h) {
                            if (h == 0 || two) {
                                const uint16_t* t0 = s_t2 + (g + 8 * h) * 2 * a.r64 + j0;
                                const bool tok = g + 8 * h < M && NF4_CHECK(in_smem(t0, 20, s_t2, p.t2_bytes, 4), 5);
                                const uint32_t b0 = tok ? *reinterpret_cast<const uint32_t*>(t0) : 0u;
                                const uint32_t b1 = tok ? *reinterpret_cast<const uint32_t*>(t0 + 8) : 0u;
                                mma_16816(acc[pp][h], af[0], af[1], af[2], af[3], b0, b1);
                            }
                        }
                    }
                }
            }
        }
    }

    // every copy issued has landed (each stage was waited for; the rank-r
    // operands too, unless a wait gave up: then drain them here)
    __syncthreads();
    if (tid == 0 && *abort_flag) {
        for (int sl = 0; sl < p.NR; ++sl)
            if (s_fills[sl] > 0) mbar_drain(&bar_full[sl], (s_fills[sl] - 1) & 1);
        if (s_lora) mbar_drain(&bar_lora, 0);
        if (lora) mbar_drain(&bar_b, 0);
    }
    __syncthreads();
    // partials of every warp into the (free) ring: s_red[wq][octet][token][8 rows]
    {
        float* s_red = reinterpret_cast<float*>(ring);
#pragma unroll
        for (int pp = 0; pp < PPW; ++pp) {
            const int pr = wp + pp * WP;
            if (pr < P) {
#pragma unroll
                for (int h = 0; h < 2; ++h) {
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int oc = 2 * pr + (e >> 1), t = 8 * h + 2 * q + (e & 1);
                        if (oc < G.Oc) {
                            float* d = s_red + (wq * G.Oc + oc) * 128 + t * 8 + g;
                            if (NF4_CHECK(in_smem(d, 4, ring, int64_t(p.NR) * p.slot, 4), 7)) *d = acc[pp][h][e];
                        }
                    }
                }
            }
        }
    }
    // ---------------------------------------------------------------- reduction (all threads)
    __syncthreads();
    const float* s_red = reinterpret_cast<const float*>(ring);
    // element e of [octet][token][8 rows], two rows per thread per pass
    const int half_elems = G.Oc * 64;
    const int own_lo = G.own0 * 64, own_hi = G.own1 * 64;
    if (p.cs > 1) {
        cluster_wait_acquire();  // the peer CTA has started: its shared memory may be written
        const int peer = G.rank ^ 1;
        const int peer_own0 = G.rank == 0 ? G.own1 : 0;  // the peer finishes the octets this CTA does not
        for (int e = tid; e < half_elems; e += kThreads) {
            if (e >= own_lo && e < own_hi) continue;
            float v0 = 0.0f, v1 = 0.0f;
            for (int z = 0; z < p.WQ; ++z) {
                const float* sp = s_red + z * G.Oc * 128 + 2 * e;
                if (!NF4_CHECK(in_smem(sp, 8, ring, int64_t(p.NR) * p.slot, 8), 8)) continue;
                const float2 v = *reinterpret_cast<const float2*>(sp);
                v0 += v.x;
                v1 += v.y;
            }
            const int le = e - peer_own0 * 64;  // index in the peer's receive buffer
            if (!NF4_CHECK(in_smem(s_recv + 2 * le, 8, s_recv, p.recv_bytes, 8), 9)) continue;
            const uint32_t dst = cluster_map(smem_u32(s_recv + 2 * le), peer);
            asm volatile("st.shared::cluster.v2.f32 [%0], {%1, %2};" ::"r"(dst), "f"(v0), "f"(v1) : "memory");
        }
        cluster_arrive_release();
        cluster_wait_acquire();
    }
    for (int e = own_lo + tid; e < own_hi; e += kThreads) {
        float v0 = 0.0f, v1 = 0.0f;
        for (int z = 0; z < p.WQ; ++z) {
            const float* sp = s_red + z * G.Oc * 128 + 2 * e;
            if (!NF4_CHECK(in_smem(sp, 8, ring, int64_t(p.NR) * p.slot, 8), 8)) continue;
            const float2 v = *reinterpret_cast<const float2*>(sp);
            v0 += v.x;
            v1 += v.y;
        }
        if (p.cs > 1 && NF4_CHECK(in_smem(s_recv + 2 * (e - own_lo), 8, s_recv, p.recv_bytes, 8), 9)) {
            const float2 pv = *reinterpret_cast<const float2*>(s_recv + 2 * (e - own_lo));
            // rank 0's partial first, then rank 1's, on both CTAs
            if (G.rank == 0) {
                v0 += pv.x;
                v1 += pv.y;
            } else {
                v0 = pv.x + v0;
                v1 = pv.y + v1;
            }
        }
        const int oc = e / 64, rem = e % 64, t = rem / 4, nl = 2 * (rem % 4);
        // e covers rows nl, nl + 1 of token t in octet oc: [token][8 rows] -> 2 e = t * 8 + nl
        const int n = G.row0 + 8 * oc + nl;
        uint16_t* yp = a.out + static_cast<int64_t>(t) * N + n;
        if (t < M && NF4_CHECK(in_span(yp, 4, a.out, int64_t(M) * N * 2, 4), 10))
            *reinterpret_cast<uint32_t*>(yp) = pack_bf16x2(v0, v1);
    }
}

// Per-device cache of the number of co-resident clusters of two.
int max_clusters_of_two(int smem) {
    static int cached[64] = {};
    static int cached_smem[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
    if (cached[dev] > 0 && cached_smem[dev] == smem) return cached[dev];
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(2 * 64);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, k_few_fwd<kMaxPPW, true>, &cfg) != cudaSuccess) n = 0;
    cached[dev] = n;
    cached_smem[dev] = smem;
    return n;
}

template <int PPW, bool TWO>
bool configure_kernel() {
    cudaFuncAttributes fa{};
    if (cudaFuncGetAttributes(&fa, k_few_fwd<PPW, TWO>) != cudaSuccess || fa.maxThreadsPerBlock < kThreads)
        return false;
    return cudaFuncSetAttribute(k_few_fwd<PPW, TWO>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemLimit) ==
               cudaSuccess &&
           cudaFuncSetAttribute(k_few_fwd<PPW, TWO>, cudaFuncAttributePreferredSharedMemoryCarveout,
                                cudaSharedmemCarveoutMaxShared) == cudaSuccess;
}

bool configure(int dev) {
    static bool configured[64] = {};
    if (dev < 0 || dev >= 64) return false;
    if (!configured[dev]) {
        if (!configure_kernel<2, false>() || !configure_kernel<4, false>() || !configure_kernel<2, true>() ||
            !configure_kernel<4, true>())
            return false;
        configured[dev] = true;
    }
    return true;
}

}  // namespace

// Host plan: cluster size, octets per CTA, quad slots per pair group, ring
// depth and the shared-memory layout (see the kernel's comment).
bool few_fwd_plan(int M, int N, int K, int r, int num_sms, bool fp32_scales, FewFwdPlan* out) {
    if (M < 1 || M > kTok || N % 8 != 0 || K % 64 != 0 || r < 1 || r > 256) return false;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || !configure(dev)) return false;
    const int noct = N / 8, nb = K / 64, nq = (nb + 3) / 4;
    const int r64 = (r + 63) / 64 * 64;
    FewFwdPlan p{};
    p.cs = nq >= 2 ? 2 : 1;
    int slots = num_sms;
    if (p.cs == 2) {
        const int mc = max_clusters_of_two(kSmemLimit);
        slots = mc > 0 ? mc : num_sms / 2;
    }
    p.O = (noct + slots - 1) / slots;
    p.clusters = (noct + p.O - 1) / p.O;
    p.nq0 = p.cs == 2 ? (nq + 1) / 2 : nq;
    const int nqc = p.cs == 2 ? p.nq0 : nq;
    const int nbc = std::min(nb, 4 * nqc);
    // TMA boxes of at most 256 rows, a multiple of 8 rows each (1024-byte
    // swizzle atoms); together they cover the CTA's 8 O rows
    p.nbox = (8 * p.O + kMaxBoxRows - 1) / kMaxBoxRows;
    p.box_rows = 8 * ((p.O + p.nbox - 1) / p.nbox);
    p.code_bytes = p.nbox * p.box_rows * 128;
    p.xbox_rows = M > 8 ? 16 : 8;
    p.xbox_bytes = p.xbox_rows * 128;
    p.slot = (p.code_bytes + kXStage + 1023) / 1024 * 1024;
    p.qrow = nbc;
    p.q_bytes = (8 * p.O * p.qrow * (fp32_scales ? 4 : 1) + 15) / 16 * 16;
    const int64_t ngroups = (int64_t(8) * p.O * nb) / 256 + 2;
    p.step_bytes = static_cast<int>((ngroups * 4 + 15) / 16 * 16);
    p.t2_bytes = M * 4 * r64;
    const int own = p.cs == 2 ? (p.O + 1) / 2 : p.O;
    p.b_bytes = (8 * own * 2 * r + 15) / 16 * 16;
    p.recv_bytes = p.cs == 2 ? 8 * own * kTok * 4 : 0;
    const int fixed = 1024 + p.q_bytes + p.step_bytes + p.t2_bytes + p.b_bytes + p.recv_bytes;
    const int P = (p.O + 1) / 2;
    for (int wq : {8, 4, 2, 1}) {
        if (wq > nqc && wq > 1) continue;
        const int wp = kWarps / wq;
        if ((P + wp - 1) / wp > kMaxPPW) continue;
        const int nr = std::min({nqc, kMaxRing, (kSmemLimit - fixed) / p.slot});
        if (nr < wq) continue;
        // the partials of the reduction reuse the ring
        if (int64_t(wq) * p.O * 512 > int64_t(nr) * p.slot) continue;
        p.WQ = wq;
        p.NR = nr;
        p.smem = fixed + nr * p.slot;
        *out = p;
        return true;
    }
    return false;
}

cudaError_t launch_few_fwd(const CUtensorMap& map_codes, const CUtensorMap& map_x, const FewArgs& a,
                           const FewFwdPlan& p, cudaStream_t stream) {
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(p.clusters * p.cs);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = p.smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    int n = 0;
    attr[n].id = cudaLaunchAttributeClusterDimension;
    attr[n].val.clusterDim.x = p.cs;
    attr[n].val.clusterDim.y = 1;
    attr[n].val.clusterDim.z = 1;
    ++n;
    if (a.pdl) {
        attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[n].val.programmaticStreamSerializationAllowed = 1;
        ++n;
    }
    cfg.attrs = attr;
    cfg.numAttrs = n;
    TraceScope trace("nf4_gemm_fwd_few", stream);
    const int P = (p.O + 1) / 2, WP = kWarps / p.WQ;
    const bool two = a.M > 8;
    if ((P + WP - 1) / WP <= 2)
        return two ? cudaLaunchKernelEx(&cfg, k_few_fwd<2, true>, map_codes, map_x, a, p)
                   : cudaLaunchKernelEx(&cfg, k_few_fwd<2, false>, map_codes, map_x, a, p);
    return two ? cudaLaunchKernelEx(&cfg, k_few_fwd<4, true>, map_codes, map_x, a, p)
               : cudaLaunchKernelEx(&cfg, k_few_fwd<4, false>, map_codes, map_x, a, p);
}

}  // namespace nf4lora
