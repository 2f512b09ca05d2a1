// Host orchestration of the NF4-LoRA linear layer on the tcgen05 engine.
//
// Forward   ("第 04 篇：QLoRA 原理" §6.1-§6.3):
//   1. T = s X A^T (fp32, kept as a bf16 hi|lo pair)  LoRA down: tcgen05, split-K
//   2. Y = X W_hat^T + T B^T                    fused dequant-GEMM, LoRA up as
//                                               extension k-steps of the same
//                                               accumulator
// Backward  (§2.4: input gradient through the frozen base; no dW):
//   1. V = s dY B (bf16 hi|lo pair)             tcgen05, split-K over d_out
//   2. dX = dY W_hat + V A                      fused dequant-GEMM (MN-major
//                                               decode of the same codes)
//   3. dB = dY^T T,  dA = V^T X                 tcgen05, split over tokens,
//                                               deterministic fixed-order sum
// Few tokens (M <= 16) run the fused GEMMs "swapped": weight rows fill the
// 128-wide MMA M and tokens the N = 16 side, split-K over all SMs, so the
// weight stream (4.127 bits per weight) sets the pace.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cstring>
#include <mutex>

#include "gemm.cuh"
#include "kernels.h"
#include "layer.h"
#include "trace.h"

namespace nf4lora {

// The CUDA error behind the last failed launch of this thread (for messages).
static thread_local cudaError_t t_launch_error = cudaSuccess;
static cudaError_t note(cudaError_t e) {
    if (e != cudaSuccess) t_launch_error = e;
    return e;
}
cudaError_t layer_last_cuda_error() {
    const cudaError_t e = t_launch_error;
    t_launch_error = cudaSuccess;
    return e;
}

// ------------------------------------------------------------------ tensor maps
static PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

// bf16 matrix [outer, inner] with row stride ld (elements), 128-byte swizzle,
// box {64, box_outer}.
static bool map_bf16(CUtensorMap* m, const void* ptr, uint64_t inner, uint64_t outer, uint64_t ld,
                     uint32_t box_outer) {
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {inner, outer};
    cuuint64_t strides[1] = {ld * 2};
    cuuint32_t box[2] = {64, box_outer};
    cuuint32_t estr[2] = {1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Packed NF4 codes viewed as bytes [d_out, d_in / 2], box {box_inner bytes, box_outer rows}.
static bool map_codes(CUtensorMap* m, const uint8_t* codes, int64_t d_out, int64_t d_in,
                      uint32_t box_inner, uint32_t box_outer,
                      CUtensorMapSwizzle swizzle = CU_TENSOR_MAP_SWIZZLE_NONE) {
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(d_in / 2), static_cast<cuuint64_t>(d_out)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(d_in / 2)};
    cuuint32_t box[2] = {box_inner, box_outer};
    cuuint32_t estr[2] = {1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(codes), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// ------------------------------------------------------------------ launch
template <int BN, int ASRC, int BSRC, int AE, int BE, int EPI, int LSTAGES = 0, int DSTAGES = 0, int TEAMS = 1,
          int MSUB = 1>
static cudaError_t launch(const char* name, const CUtensorMap& a, const CUtensorMap& b, const CUtensorMap& ae,
                          const CUtensorMap& be, const GemmArgs& args, dim3 grid, cudaStream_t st,
                          int cluster_z = 1) {
    using C = GemmConfig<BN, ASRC, BSRC, AE, BE, EPI, LSTAGES, DSTAGES, TEAMS, MSUB>;
    auto kern = k_gemm<BN, ASRC, BSRC, AE, BE, EPI, LSTAGES, DSTAGES, TEAMS, MSUB>;
    // rank 0 of a split-K cluster has partial-tile slots for kPushMax - 1 other ranks
    if (EPI == EPI_CLUSTER_BF16_T && (static_cast<int>(grid.z) > C::kPushMax || cluster_z != static_cast<int>(grid.z)))
        return note(cudaErrorInvalidValue);
    // the shared-memory opt-in is per device; set it once (also keeps it out of
    // stream captures)
    static bool configured[64] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return note(e);
    if (dev < 0 || dev >= 64 || !configured[dev]) {
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
        if (e != cudaSuccess) return note(e);
        // all of the unified L1/shared array as shared memory, so that two
        // ~100 KB CTAs (and clusters of them) fit on one SM
        e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout,
                                 cudaSharedmemCarveoutMaxShared);
        if (e != cudaSuccess) return note(e);
        if (dev >= 0 && dev < 64) configured[dev] = true;
    }
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = grid;
    cfg.blockDim = dim3(C::kThreads);
    cfg.dynamicSmemBytes = C::kSmemBytes;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    int n_attr = 0;
    if (args.pdl || args.wait_first) {
        // may start while the previous kernel on the stream still runs; the
        // kernel waits for it (griddepcontrol.wait) where it needs its output
        attr[n_attr].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[n_attr].val.programmaticStreamSerializationAllowed = 1;
        ++n_attr;
    }
    if (cluster_z > 1) {
        // the split-K slices of one tile form a cluster along grid.z
        attr[n_attr].id = cudaLaunchAttributeClusterDimension;
        attr[n_attr].val.clusterDim.x = 1;
        attr[n_attr].val.clusterDim.y = 1;
        attr[n_attr].val.clusterDim.z = cluster_z;
        ++n_attr;
    }
    cfg.attrs = n_attr ? attr : nullptr;
    cfg.numAttrs = n_attr;
    TraceScope trace(name, st);
    return note(cudaLaunchKernelEx(&cfg, kern, a, b, ae, be, args));
}

// Fixed-order sum over the split-K slices of an fp32 partial buffer:
//   v[r, c] = alpha * sum_z (part[z][r, c] + part[z][r, c + fold])   (fold 0: no second term)
// written as bf16 (optionally added to the bf16 already there), or -- in split
// mode (lo_off > 0) -- as the pair hi = bf16(v), lo = bf16(v - hi) at columns c
// and c + lo_off; optionally also as fp32 into out32 for c < out32_cols.
struct ReduceArgs {
    const float* part;
    int splits;
    int64_t slice;
    int rows;
    int cols;
    int64_t ldp;
    int64_t fold;
    float alpha;
    uint16_t* out;
    int64_t ldo;
    int64_t lo_off;
    int accumulate;
    float* out32;
    int64_t ldo32;
    int pdl;  // launched as a programmatic dependent: waits for the previous kernel first
    int out32_cols;
};

__global__ void k_reduce_splits(const ReduceArgs a) {
    if (a.pdl) asm volatile("griddepcontrol.wait;" ::: "memory");  // the partials are complete
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    const int64_t total = static_cast<int64_t>(a.rows) * a.cols;
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < total;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int64_t r = i / a.cols, c = i % a.cols;
        const float* p = a.part + r * a.ldp + c;
        float acc = 0.0f;
        for (int z = 0; z < a.splits; ++z) {
            acc += p[z * a.slice];
            if (a.fold) acc += p[z * a.slice + a.fold];
        }
        const float v = acc * a.alpha;
        uint16_t* o = a.out + r * a.ldo + c;
        if (a.lo_off > 0) {
            const __nv_bfloat16 hi = __float2bfloat16_rn(v);
            const __nv_bfloat16 lo = __float2bfloat16_rn(v - __bfloat162float(hi));
            o[0] = *reinterpret_cast<const uint16_t*>(&hi);
            o[a.lo_off] = *reinterpret_cast<const uint16_t*>(&lo);
        } else {
            const float w = a.accumulate ? v + bf16_bits_to_float(o[0]) : v;
            const __nv_bfloat16 h = __float2bfloat16_rn(w);
            o[0] = *reinterpret_cast<const uint16_t*>(&h);
        }
        if (a.out32 != nullptr && c < a.out32_cols) a.out32[r * a.ldo32 + c] = v;
    }
}

static cudaError_t reduce(const ReduceArgs& a, int num_sms, cudaStream_t st) {
    const int64_t total = static_cast<int64_t>(a.rows) * a.cols;
    int64_t grid = (total + 255) / 256;
    grid = std::min<int64_t>(grid, int64_t(num_sms) * 8);
    if (grid < 1) grid = 1;
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(static_cast<unsigned>(grid));
    cfg.blockDim = dim3(256);
    cfg.stream = st;
    cudaLaunchAttribute attr{};
    if (a.pdl) {
        attr.id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr.val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = &attr;
        cfg.numAttrs = 1;
    }
    TraceScope trace("reduce_splits", st);
    return note(cudaLaunchKernelEx(&cfg, k_reduce_splits, a));
}

static ReduceArgs reduce_args(const float* part, int splits, int64_t slice, int rows, int cols, int64_t ldp,
                              float alpha, uint16_t* out, int64_t ldo) {
    ReduceArgs a{};
    a.pdl = 1;  // it follows the split-K GEMM that wrote the partials
    a.part = part;
    a.splits = splits;
    a.slice = slice;
    a.rows = rows;
    a.cols = cols;
    a.ldp = ldp;
    a.alpha = alpha;
    a.out = out;
    a.ldo = ldo;
    return a;
}

// T2 / V2 [M, 2 r64] = (hi | lo) split of an fp32 [M, r] array, zero beyond r.
__global__ void k_split_from_f32(const float* __restrict__ src, int64_t M, int r, int r64,
                                 uint16_t* __restrict__ dst) {
    const int64_t total = M * r64;
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < total;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int64_t m = i / r64;
        const int j = static_cast<int>(i % r64);
        const float v = j < r ? src[m * r + j] : 0.0f;
        const __nv_bfloat16 hi = __float2bfloat16_rn(v);
        const __nv_bfloat16 lo = __float2bfloat16_rn(v - __bfloat162float(hi));
        dst[m * 2 * r64 + j] = *reinterpret_cast<const uint16_t*>(&hi);
        dst[m * 2 * r64 + r64 + j] = *reinterpret_cast<const uint16_t*>(&lo);
    }
}

// ------------------------------------------------------------------ split sizing
struct Split {
    int splits;
    int k_per_split;
};

// Split k_steps over grid.z so that tiles * splits fills about `target` CTAs,
// each split keeping at least `min_steps` k-steps; never leaves a split empty.
static Split choose_split(int tiles, int k_steps, int target, int min_steps) {
    int s = std::max(1, target / std::max(1, tiles));
    s = std::min(s, std::max(1, k_steps / std::max(1, min_steps)));
    int kps = (k_steps + s - 1) / s;
    s = (k_steps + kps - 1) / kps;
    return {s, kps};
}

static inline int64_t align256(int64_t b) { return (b + 255) & ~int64_t(255); }
static inline int round64(int r) { return (r + 63) / 64 * 64; }
static inline int ceil_div(int64_t a, int64_t b) { return static_cast<int>((a + b - 1) / b); }
static int bn_for(int cols) { return cols <= 64 ? 64 : (cols <= 128 ? 128 : 256); }

// Bytes of an encoded weight (codes, int8 scales, group scales), close enough
// to choose a tile order.
static inline int64_t weight_bytes_approx(int64_t d_out, int64_t d_in) { return d_out * d_in * 33 / 64; }

// The grid of a fused GEMM: row tiles x column tiles, the column tiles along
// grid.x when g.cols_fastest is set.
static inline dim3 tile_grid(int row_tiles, int col_tiles, const GemmArgs& g) {
    return g.cols_fastest ? dim3(col_tiles, row_tiles, 1) : dim3(row_tiles, col_tiles, 1);
}

static constexpr int kSmallM = 16;

// Many-token fused GEMMs: 256-row CTA tiles (two accumulators sharing each
// decoded weight tile, which halves the decode work per MMA) once there are
// enough of them to cover every SM, else 128-row tiles.
static bool wide_tiles(int64_t M, int64_t cols, int sms) {
    return int64_t(ceil_div(M, 256)) * ceil_div(cols, 256) >= sms;
}
// 256 x 256 tiles: 4 load slots of 40 KB + 2 decoded tiles of 32 KB, one per
// decode team, teams on alternate k-steps
static constexpr int kWideLoad = 4;
static constexpr int kWideDec = 2;
static constexpr int kWideTeams = 2;
// Split of the contraction of the few-token kernels: the splits of one tile
// form a cluster; as many (up to the cluster limit) as keep every tile's
// cluster resident at once with one CTA per SM.
static int few_splits(int tiles, int units, int sms, bool forward) {
    return std::max(1, std::min({few_max_split(forward), sms / std::max(1, tiles), units}));
}

static FewArgs few_args(const LayerCtx& c, const uint16_t* act, int M, const uint16_t* ext_act,
                        const uint16_t* ext_w, int r, int r64, uint16_t* out) {
    FewArgs a{};
    a.act = act;
    a.codes = c.codes;
    a.qscale = c.qscale;
    a.scale2 = c.scale2;
    a.scale_mean = c.scale_mean;
    a.absmax = c.absmax;
    a.M = M;
    a.N = static_cast<int>(c.d_out);
    a.K = static_cast<int>(c.d_in);
    a.ext_act = ext_act;
    a.ext_w = ext_w;
    a.r = r;
    a.r64 = r64;
    a.out = out;
    a.pdl = 1;
    return a;
}

// The splits each split-K GEMM uses (the workspace query and the calls share them).
static Split split_down(int64_t M, int64_t d_in, int sms) {
    return choose_split(ceil_div(M, 128), ceil_div(d_in, 64), sms, 4);
}
static Split split_v(int64_t M, int64_t d_out, int sms) {
    return choose_split(ceil_div(M, 128), ceil_div(d_out, 64), sms, 4);
}
static Split split_tokens(int64_t rows, int r64, int64_t M, int sms) {
    const int tiles = ceil_div(rows, 128) * ceil_div(2 * r64, bn_for(2 * r64));
    return choose_split(tiles, ceil_div(M, 64), sms, 4);
}

// ------------------------------------------------------------------ layer ops
struct Maps {
    CUtensorMap a, b, ae, be;
    Maps() { std::memset(this, 0, sizeof(*this)); }
};

template <int EPI, int ASRC, int BSRC>
static cudaError_t launch_lora_gemm(const char* name, int bn, const Maps& m, const GemmArgs& args, dim3 grid,
                                    cudaStream_t st) {
    switch (bn) {
        case 64: return launch<64, ASRC, BSRC, 0, 0, EPI>(name, m.a, m.b, m.ae, m.be, args, grid, st);
        case 128: return launch<128, ASRC, BSRC, 0, 0, EPI>(name, m.a, m.b, m.ae, m.be, args, grid, st);
        default: return launch<256, ASRC, BSRC, 0, 0, EPI>(name, m.a, m.b, m.ae, m.be, args, grid, st);
    }
}

// T2[M, 2 r64] = hi | lo of s X A^T (zero columns beyond r); optional fp32 T_saved[M, r].
static int lora_down(const LayerCtx& c, const uint16_t* A, int r, float s, const uint16_t* X, int64_t M,
                     uint16_t* T2, float* T_saved, float* part) {
    const int r64 = round64(r), bn = bn_for(r64);
    Maps m;
    if (!map_bf16(&m.a, X, c.d_in, M, c.d_in, 128) || !map_bf16(&m.b, A, c.d_in, r, c.d_in, bn)) return -1;
    const Split sp = split_down(M, c.d_in, c.num_sms);
    GemmArgs g{};
    g.wait_first = 1;  // it overwrites the split-K partials the kernels before it used
    g.rows = static_cast<int>(M);
    g.cols = r64;
    g.k_main = ceil_div(c.d_in, 64);
    g.k_per_split = sp.k_per_split;
    g.part = part;
    g.ldp = r64;
    g.part_slice = M * r64;
    dim3 grid(ceil_div(M, 128), ceil_div(r64, bn), sp.splits);
    if (launch_lora_gemm<EPI_F32_PART, SRC_TMA_K, SRC_TMA_K>("lora_down", bn, m, g, grid, c.stream) != cudaSuccess) return -2;
    ReduceArgs ra = reduce_args(part, sp.splits, M * r64, static_cast<int>(M), r64, r64, s, T2, 2 * r64);
    ra.lo_off = r64;
    ra.out32 = T_saved;
    ra.ldo32 = r;
    ra.out32_cols = r;
    return reduce(ra, c.num_sms, c.stream) == cudaSuccess ? 0 : -2;
}

static int64_t fwd_core_bytes(int64_t M, int64_t d_out, int64_t d_in, int r, int num_sms) {
    (void)d_out;
    const int r64 = round64(r);
    const int64_t part = M <= kSmallM ? 0 : int64_t(split_down(M, d_in, num_sms).splits) * M * r64;
    return align256(M * r64 * 4) + align256(part * 4);
}

// The layer for a rank that is a multiple of 8 (B's rows, r bf16, are then
// whole 16-byte units, as the tensor maps and the vector loads need).
static int layer_fwd_r8(const LayerCtx& c, const uint16_t* A, const uint16_t* B, int r, float s,
                        const uint16_t* X, int64_t M, uint16_t* Y, float* T_saved, uint8_t* ws) {
    const int r64 = round64(r), kx = r64 / 64;
    uint16_t* T2 = reinterpret_cast<uint16_t*>(ws);
    float* part = reinterpret_cast<float*>(ws + align256(M * r64 * 4));
    Maps m;
    GemmArgs g{};
    g.qscale = c.qscale;
    g.scale2 = c.scale2;
    g.scale_mean = c.scale_mean;
    g.absmax = c.absmax;
    g.w_rows = c.d_out;
    g.w_blocks_per_row = c.d_in / 64;
    g.k_main = ceil_div(c.d_in, 64);
    g.k_ext = 2 * kx;
    g.alpha = 1.0f;
    if (M <= kSmallM) {
        // T (hi | lo) first; the fused product as its programmatic dependent
        // streams and decodes the weight meanwhile and waits for T only before
        // the rank-r extension.
        if (note(launch_few_down(X, A, static_cast<int>(M), static_cast<int>(c.d_in), r, r64, s, T2, T_saved,
                                 c.stream)) != cudaSuccess)
            return -2;
        const FewArgs fa = few_args(c, X, static_cast<int>(M), T2, B, r, r64, Y);
        FewFwdPlan fp;
        if (!few_fwd_plan(static_cast<int>(M), static_cast<int>(c.d_out), static_cast<int>(c.d_in), r, c.num_sms,
                          c.absmax != nullptr, &fp))
        {
            note(cudaErrorInvalidConfiguration);
            return -2;
        }
        if (!map_codes(&m.a, c.codes, c.d_out, c.d_in, 128, static_cast<uint32_t>(fp.box_rows),
                       CU_TENSOR_MAP_SWIZZLE_128B) ||
            !map_bf16(&m.b, X, c.d_in, M, c.d_in, static_cast<uint32_t>(fp.xbox_rows)))
            return -1;
        return note(launch_few_fwd(m.a, m.b, fa, fp, c.stream)) == cudaSuccess ? 0 : -2;
    }
    int rc = lora_down(c, A, r, s, X, M, T2, T_saved, part);
    if (rc) return rc;
    if (!map_bf16(&m.a, X, c.d_in, M, c.d_in, 128) || !map_codes(&m.b, c.codes, c.d_out, c.d_in, 32, 256) ||
        !map_bf16(&m.ae, T2, 2 * r64, M, 2 * r64, 128) || !map_bf16(&m.be, B, r, c.d_out, r, 256))
        return -1;
    g.ext_wrap_b = kx;
    g.pdl = 1;  // T (hi | lo) comes from the reduction just launched
    g.rows = static_cast<int>(M);
    g.cols = static_cast<int>(c.d_out);
    g.k_per_split = g.k_main;
    g.out = Y;
    g.ldo = c.d_out;
    // re-read the smaller operand once per wave: X (2 M K bytes) or the codes
    // (about 0.52 N K bytes)
    g.cols_fastest = 2 * M * c.d_in > weight_bytes_approx(c.d_out, c.d_in) ? 1 : 0;
    cudaError_t e;
    if (wide_tiles(M, c.d_out, c.num_sms)) {
        e = launch<256, SRC_TMA_K, SRC_DEC_K, 0, 0, EPI_BF16, kWideLoad, kWideDec, kWideTeams, 2>(
            "nf4_gemm_fwd", m.a, m.b, m.ae, m.be, g, tile_grid(ceil_div(M, 256), ceil_div(c.d_out, 256), g),
            c.stream);
    } else {
        e = launch<256, SRC_TMA_K, SRC_DEC_K, 0, 0, EPI_BF16>("nf4_gemm_fwd", m.a, m.b, m.ae, m.be, g,
                                                             tile_grid(ceil_div(M, 128), ceil_div(c.d_out, 256), g),
                                                             c.stream);
    }
    return e == cudaSuccess ? 0 : -2;
}

static int64_t bwd_core_bytes(int64_t M, int64_t d_out, int64_t d_in, int r, int num_sms) {
    const int r64 = round64(r);
    int64_t part = int64_t(split_down(M, d_in, num_sms).splits) * M * r64;
    part = std::max<int64_t>(part, int64_t(split_v(M, d_out, num_sms).splits) * M * r64);
    part = std::max<int64_t>(part, int64_t(split_tokens(d_out, r64, M, num_sms).splits) * d_out * 2 * r64);
    part = std::max<int64_t>(part, int64_t(split_tokens(d_in, r64, M, num_sms).splits) * d_in * 2 * r64);
    return 2 * align256(M * r64 * 4) + align256(part * 4);
}

static int layer_bwd_r8(const LayerCtx& c, const uint16_t* A, const uint16_t* B, int r, float s,
                        const uint16_t* X, const float* T_saved, const uint16_t* dY, int64_t M, uint16_t* dX,
                        uint16_t* dA, uint16_t* dB, int accumulate, uint8_t* ws) {
    const int r64 = round64(r), kx = r64 / 64;
    uint16_t* V2 = reinterpret_cast<uint16_t*>(ws);
    uint16_t* T2 = reinterpret_cast<uint16_t*>(ws + align256(M * r64 * 4));
    float* part = reinterpret_cast<float*>(ws + 2 * align256(M * r64 * 4));
    const bool few = M <= kSmallM;

    // ---- V = s dY B, held as hi | lo: D[m, j] = sum_n dY[m, n] B[n, j]
    if (few && (dX != nullptr || dA != nullptr)) {
        if (note(launch_few_v(dY, B, static_cast<int>(M), static_cast<int>(c.d_out), r, r64, s, V2, c.stream)) !=
            cudaSuccess)
            return -2;
    } else if (dX != nullptr || dA != nullptr) {
        const int bn = bn_for(r64);
        Maps m;
        if (!map_bf16(&m.a, dY, c.d_out, M, c.d_out, 128) || !map_bf16(&m.b, B, r, c.d_out, r, 64)) return -1;
        const Split sp = split_v(M, c.d_out, c.num_sms);
        GemmArgs g{};
        g.wait_first = 1;
        g.rows = static_cast<int>(M);
        g.cols = r64;
        g.k_main = ceil_div(c.d_out, 64);
        g.k_per_split = sp.k_per_split;
        g.part = part;
        g.ldp = r64;
        g.part_slice = M * r64;
        dim3 grid(ceil_div(M, 128), ceil_div(r64, bn), sp.splits);
        if (launch_lora_gemm<EPI_F32_PART, SRC_TMA_K, SRC_TMA_MN>("lora_v", bn, m, g, grid, c.stream) != cudaSuccess) return -2;
        ReduceArgs ra = reduce_args(part, sp.splits, M * r64, static_cast<int>(M), r64, r64, s, V2, 2 * r64);
        ra.lo_off = r64;
        if (reduce(ra, c.num_sms, c.stream) != cudaSuccess) return -2;
    }

    // ---- dX = dY W_hat + V A
    if (dX != nullptr) {
        Maps m;
        GemmArgs g{};
        g.qscale = c.qscale;
        g.scale2 = c.scale2;
        g.scale_mean = c.scale_mean;
    g.absmax = c.absmax;
        g.w_rows = c.d_out;
        g.w_blocks_per_row = c.d_in / 64;
        g.k_main = ceil_div(c.d_out, 64);
        g.k_ext = 2 * kx;
        g.alpha = 1.0f;
        if (few) {
            // a programmatic dependent of the V kernel just launched
            const FewArgs fa = few_args(c, dY, static_cast<int>(M), V2, A, r, r64, dX);
            const int splits = few_splits(ceil_div(c.d_in, 128), ceil_div(c.d_out, 32), c.num_sms, false);
            if (!map_codes(&m.a, c.codes, c.d_out, c.d_in, 64, 256, CU_TENSOR_MAP_SWIZZLE_64B)) return -1;
            if (note(launch_few_dx(m.a, fa, splits, c.stream)) != cudaSuccess) return -2;
        } else {
            if (!map_bf16(&m.a, dY, c.d_out, M, c.d_out, 128) || !map_codes(&m.b, c.codes, c.d_out, c.d_in, 128, 64) ||
                !map_bf16(&m.ae, V2, 2 * r64, M, 2 * r64, 128) || !map_bf16(&m.be, A, c.d_in, r, c.d_in, 64))
                return -1;
            g.ext_wrap_b = kx;
            g.pdl = 1;  // V (hi | lo) comes from the reduction just launched
            g.rows = static_cast<int>(M);
            g.cols = static_cast<int>(c.d_in);
            g.k_per_split = g.k_main;
            g.out = dX;
            g.ldo = c.d_in;
            // re-read the smaller operand once per wave: dY (2 M N bytes) or the
            // codes (about 0.52 N K bytes)
            g.cols_fastest = 2 * M * c.d_out > weight_bytes_approx(c.d_out, c.d_in) ? 1 : 0;
            cudaError_t e;
            if (wide_tiles(M, c.d_in, c.num_sms)) {
                e = launch<256, SRC_TMA_K, SRC_DEC_MN, 0, 1, EPI_BF16, kWideLoad, kWideDec, kWideTeams, 2>(
                    "nf4_gemm_dx", m.a, m.b, m.ae, m.be, g, tile_grid(ceil_div(M, 256), ceil_div(c.d_in, 256), g),
                    c.stream);
            } else {
                e = launch<256, SRC_TMA_K, SRC_DEC_MN, 0, 1, EPI_BF16>(
                    "nf4_gemm_dx", m.a, m.b, m.ae, m.be, g, tile_grid(ceil_div(M, 128), ceil_div(c.d_in, 256), g),
                    c.stream);
            }
            if (e != cudaSuccess) return -2;
        }
    }

    const int bn2 = bn_for(2 * r64);  // the (hi | lo) operand is 2 r64 wide
    // ---- dB = dY^T T: D[n, c] = sum_m dY[m, n] T2[m, c], then dB[n, j] = D[n, j] + D[n, j + r64]
    if (dB != nullptr) {
        if (T_saved != nullptr) {
            TraceScope trace("split_t", c.stream);
            cudaLaunchConfig_t cfg{};
            cfg.gridDim = dim3(static_cast<unsigned>(std::min<int64_t>((M * r64 + 255) / 256, c.num_sms * 8)));
            cfg.blockDim = dim3(256);
            cfg.stream = c.stream;
            if (note(cudaLaunchKernelEx(&cfg, k_split_from_f32, T_saved, M, r, r64, T2)) != cudaSuccess) return -2;
        } else if (few) {
            if (note(launch_few_down(X, A, static_cast<int>(M), static_cast<int>(c.d_in), r, r64, s, T2, nullptr,
                                     c.stream)) != cudaSuccess)
                return -2;
        } else {
            int rc = lora_down(c, A, r, s, X, M, T2, nullptr, part);
            if (rc) return rc;
        }
        Maps m;
        if (!map_bf16(&m.a, dY, c.d_out, M, c.d_out, 64) || !map_bf16(&m.b, T2, 2 * r64, M, 2 * r64, 64)) return -1;
        const Split sp = split_tokens(c.d_out, r64, M, c.num_sms);
        GemmArgs g{};
        g.wait_first = 1;
        g.rows = static_cast<int>(c.d_out);
        g.cols = 2 * r64;
        g.k_main = ceil_div(M, 64);
        g.k_per_split = sp.k_per_split;
        g.part = part;
        g.ldp = 2 * r64;
        g.part_slice = c.d_out * 2 * r64;
        dim3 grid(ceil_div(c.d_out, 128), ceil_div(2 * r64, bn2), sp.splits);
        if (launch_lora_gemm<EPI_F32_PART, SRC_TMA_MN, SRC_TMA_MN>("lora_db", bn2, m, g, grid, c.stream) != cudaSuccess) return -2;
        ReduceArgs ra = reduce_args(part, sp.splits, c.d_out * 2 * r64, static_cast<int>(c.d_out), r, 2 * r64, 1.0f, dB, r);
        ra.fold = r64;
        ra.accumulate = accumulate;
        if (reduce(ra, c.num_sms, c.stream) != cudaSuccess) return -2;
    }

    // ---- dA = V^T X: D[k, c] = sum_m X[m, k] V2[m, c], stored transposed, dA[j, k] = D[k, j] + D[k, j + r64]
    if (dA != nullptr) {
        Maps m;
        if (!map_bf16(&m.a, X, c.d_in, M, c.d_in, 64) || !map_bf16(&m.b, V2, 2 * r64, M, 2 * r64, 64)) return -1;
        const Split sp = split_tokens(c.d_in, r64, M, c.num_sms);
        GemmArgs g{};
        g.wait_first = 1;
        g.rows = static_cast<int>(c.d_in);
        g.cols = 2 * r64;
        g.k_main = ceil_div(M, 64);
        g.k_per_split = sp.k_per_split;
        g.part = part;
        g.ldp = c.d_in;
        g.part_slice = int64_t(2 * r64) * c.d_in;
        dim3 grid(ceil_div(c.d_in, 128), ceil_div(2 * r64, bn2), sp.splits);
        if (launch_lora_gemm<EPI_F32_PART_T, SRC_TMA_MN, SRC_TMA_MN>("lora_da", bn2, m, g, grid, c.stream) != cudaSuccess)
            return -2;
        ReduceArgs ra = reduce_args(part, sp.splits, int64_t(2 * r64) * c.d_in, r, static_cast<int>(c.d_in), c.d_in,
                                    1.0f, dA, c.d_in);
        ra.fold = int64_t(r64) * c.d_in;
        ra.accumulate = accumulate;
        if (reduce(ra, c.num_sms, c.stream) != cudaSuccess) return -2;
    }
    return 0;
}

// ------------------------------------------------------------------ any rank
// A rank that is not a multiple of 8 runs as the next multiple r8 on padded
// copies in the workspace: A with zero rows r .. r8-1, B with zero columns,
// T_saved with zero columns; dA and dB are produced padded and their first r
// rows / columns copied out (copied in first when accumulating).  The zero
// rows and columns add exact zeros to every product and sum, so the results
// are those of rank r.

// dst[i, j] (dst_rows x dst_cols, leading dimension ld_dst) = src[i, j] for
// i < src_rows and j < src_cols, else 0.
template <typename T>
__global__ void k_repack(const T* __restrict__ src, int64_t src_rows, int src_cols, int64_t ld_src,
                         T* __restrict__ dst, int64_t dst_rows, int dst_cols, int64_t ld_dst) {
    const int64_t total = dst_rows * dst_cols;
    for (int64_t e = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; e < total;
         e += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int64_t i = e / dst_cols;
        const int j = static_cast<int>(e - i * dst_cols);
        dst[i * ld_dst + j] = (i < src_rows && j < src_cols) ? src[i * ld_src + j] : T(0);
    }
}

template <typename T>
static cudaError_t repack(const T* src, int64_t src_rows, int src_cols, int64_t ld_src, T* dst, int64_t dst_rows,
                          int dst_cols, int64_t ld_dst, int num_sms, cudaStream_t st) {
    const int64_t total = dst_rows * dst_cols;
    if (total <= 0) return cudaSuccess;
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(static_cast<unsigned>(std::min<int64_t>((total + 255) / 256, int64_t(num_sms) * 8)));
    cfg.blockDim = dim3(256);
    cfg.stream = st;
    TraceScope trace("repack_rank", st);
    return note(cudaLaunchKernelEx(&cfg, k_repack<T>, src, src_rows, src_cols, ld_src, dst, dst_rows, dst_cols,
                                   ld_dst));
}

static inline int round8(int r) { return (r + 7) / 8 * 8; }

// Padded copies after the core workspace: A [r8, d_in], B [d_out, r8],
// T [M, r8] (fp32), and for the backward dA [r8, d_in], dB [d_out, r8].
struct RankPad {
    uint16_t* A;
    uint16_t* B;
    float* T;
    uint16_t* dA;
    uint16_t* dB;
    int64_t bytes;
};

static RankPad rank_pad(uint8_t* base, int64_t M, int64_t d_out, int64_t d_in, int r, bool backward) {
    RankPad p{};
    if (r % 8 == 0) return p;
    const int r8 = round8(r);
    int64_t off = 0;
    auto take = [&](int64_t bytes) {
        uint8_t* q = base ? base + off : nullptr;
        off += align256(bytes);
        return q;
    };
    p.A = reinterpret_cast<uint16_t*>(take(int64_t(r8) * d_in * 2));
    p.B = reinterpret_cast<uint16_t*>(take(d_out * r8 * 2));
    p.T = reinterpret_cast<float*>(take(M * r8 * 4));
    if (backward) {
        p.dA = reinterpret_cast<uint16_t*>(take(int64_t(r8) * d_in * 2));
        p.dB = reinterpret_cast<uint16_t*>(take(d_out * r8 * 2));
    }
    p.bytes = off;
    return p;
}

int64_t fwd_workspace_bytes(int64_t M, int64_t d_out, int64_t d_in, int r, int num_sms) {
    return fwd_core_bytes(M, d_out, d_in, r, num_sms) + rank_pad(nullptr, M, d_out, d_in, r, false).bytes;
}

int64_t bwd_workspace_bytes(int64_t M, int64_t d_out, int64_t d_in, int r, int num_sms) {
    return bwd_core_bytes(M, d_out, d_in, r, num_sms) + rank_pad(nullptr, M, d_out, d_in, r, true).bytes;
}

int layer_fwd(const LayerCtx& c, const uint16_t* A, const uint16_t* B, int r, float s, const uint16_t* X,
              int64_t M, uint16_t* Y, float* T_saved, uint8_t* ws) {
    if (r % 8 == 0) return layer_fwd_r8(c, A, B, r, s, X, M, Y, T_saved, ws);
    const int r8 = round8(r);
    const RankPad p = rank_pad(ws + fwd_core_bytes(M, c.d_out, c.d_in, r, c.num_sms), M, c.d_out, c.d_in, r, false);
    if (repack(A, r, static_cast<int>(c.d_in), c.d_in, p.A, r8, static_cast<int>(c.d_in), c.d_in, c.num_sms,
               c.stream) != cudaSuccess ||
        repack(B, c.d_out, r, r, p.B, c.d_out, r8, r8, c.num_sms, c.stream) != cudaSuccess)
        return -2;
    const int rc = layer_fwd_r8(c, p.A, p.B, r8, s, X, M, Y, T_saved ? p.T : nullptr, ws);
    if (rc) return rc;
    if (T_saved && repack<float>(p.T, M, r8, r8, T_saved, M, r, r, c.num_sms, c.stream) != cudaSuccess) return -2;
    return 0;
}

int layer_bwd(const LayerCtx& c, const uint16_t* A, const uint16_t* B, int r, float s, const uint16_t* X,
              const float* T_saved, const uint16_t* dY, int64_t M, uint16_t* dX, uint16_t* dA, uint16_t* dB,
              int accumulate, uint8_t* ws) {
    if (r % 8 == 0) return layer_bwd_r8(c, A, B, r, s, X, T_saved, dY, M, dX, dA, dB, accumulate, ws);
    const int r8 = round8(r);
    const int d_in = static_cast<int>(c.d_in);
    const RankPad p = rank_pad(ws + bwd_core_bytes(M, c.d_out, c.d_in, r, c.num_sms), M, c.d_out, c.d_in, r, true);
    if (repack(A, r, d_in, c.d_in, p.A, r8, d_in, c.d_in, c.num_sms, c.stream) != cudaSuccess ||
        repack(B, c.d_out, r, r, p.B, c.d_out, r8, r8, c.num_sms, c.stream) != cudaSuccess ||
        (T_saved && repack<float>(T_saved, M, r, r, p.T, M, r8, r8, c.num_sms, c.stream) != cudaSuccess) ||
        (accumulate && dA && repack(dA, r, d_in, c.d_in, p.dA, r8, d_in, c.d_in, c.num_sms, c.stream) != cudaSuccess) ||
        (accumulate && dB && repack(dB, c.d_out, r, r, p.dB, c.d_out, r8, r8, c.num_sms, c.stream) != cudaSuccess))
        return -2;
    const int rc = layer_bwd_r8(c, p.A, p.B, r8, s, X, T_saved ? p.T : nullptr, dY, M, dX, dA ? p.dA : nullptr,
                                dB ? p.dB : nullptr, accumulate, ws);
    if (rc) return rc;
    if ((dA && repack(p.dA, r8, d_in, c.d_in, dA, r, d_in, c.d_in, c.num_sms, c.stream) != cudaSuccess) ||
        (dB && repack(p.dB, c.d_out, r8, r8, dB, c.d_out, r, r, c.num_sms, c.stream) != cudaSuccess))
        return -2;
    return 0;
}

}  // namespace nf4lora
