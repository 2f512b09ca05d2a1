// The adapter's optimizer step: AdamW over the trainable tensors A and B
// ("第 04 篇：QLoRA 原理" §7.3: two fp32 moments m, v per trainable parameter;
// §8.3: an fp32 master copy of the adapter beside the bf16 one the layer
// reads).  The pages print no update rule; this is decoupled-weight-decay
// AdamW with bias-corrected moments (t counted from 1):
//
//   p <- p (1 - lr wd)
//   m <- b1 m + (1 - b1) g
//   v <- b2 v + (1 - b2) g^2
//   p <- p - lr / (1 - b1^t) * m / (sqrt(v) / sqrt(1 - b2^t) + eps)
//
// per element in fp32, with the step's constants formed on the host in fp64
// and rounded once.  Elementwise and HBM-bound: 28 bytes per parameter (fp32
// p, m, v read and written, the bf16 gradient read, the bf16 copy written),
// moved as 16-byte vectors.  One launch covers up to kAdamwMaxTensors tensors
// (grid.y), each swept by a grid-stride loop.
#include <cuda_runtime.h>

#include <cstdint>

#include "common.cuh"
#include "kernels.h"
#include "trace.h"

namespace nf4lora {

namespace {

__device__ __forceinline__ void adamw_one(float& p, float g, float& m, float& v, const AdamwConsts& c) {
    p = __fmul_rn(p, c.decay);
    m = __fadd_rn(__fmul_rn(c.b1, m), __fmul_rn(c.omb1, g));
    v = __fadd_rn(__fmul_rn(c.b2, v), __fmul_rn(c.omb2, __fmul_rn(g, g)));
    const float denom = __fadd_rn(__fmul_rn(__fsqrt_rn(v), c.inv_sqrt_bc2), c.eps);
    p = __fsub_rn(p, __fmul_rn(c.step_size, __fdiv_rn(m, denom)));
}

__global__ void __launch_bounds__(256) k_adamw(const AdamwBatch b, const AdamwConsts c) {
    const int i = blockIdx.y;
    const int64_t n = b.n[i];
    float* P = b.p[i];
    uint16_t* P16 = b.p16[i];
    const uint16_t* G = b.g[i];
    float* Mo = b.m[i];
    float* Vo = b.v[i];
    const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
    const int64_t first = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    const int64_t n4 = n / 4;
    for (int64_t u = first; u < n4; u += stride) {
        float4 p = __ldcs(reinterpret_cast<const float4*>(P) + u);
        float4 m = __ldcs(reinterpret_cast<const float4*>(Mo) + u);
        float4 v = __ldcs(reinterpret_cast<const float4*>(Vo) + u);
        const uint2 g = __ldcs(reinterpret_cast<const uint2*>(G) + u);
        adamw_one(p.x, bf16_bits_to_float(static_cast<uint16_t>(g.x)), m.x, v.x, c);
        adamw_one(p.y, bf16_bits_to_float(static_cast<uint16_t>(g.x >> 16)), m.y, v.y, c);
        adamw_one(p.z, bf16_bits_to_float(static_cast<uint16_t>(g.y)), m.z, v.z, c);
        adamw_one(p.w, bf16_bits_to_float(static_cast<uint16_t>(g.y >> 16)), m.w, v.w, c);
        __stcs(reinterpret_cast<float4*>(P) + u, p);
        __stcs(reinterpret_cast<float4*>(Mo) + u, m);
        __stcs(reinterpret_cast<float4*>(Vo) + u, v);
        if (P16 != nullptr)
            __stcs(reinterpret_cast<uint2*>(P16) + u, make_uint2(pack_bf16x2(p.x, p.y), pack_bf16x2(p.z, p.w)));
    }
    for (int64_t e = 4 * n4 + first; e < n; e += stride) {  // the last n % 4 elements
        float p = P[e], m = Mo[e], v = Vo[e];
        adamw_one(p, bf16_bits_to_float(G[e]), m, v, c);
        P[e] = p;
        Mo[e] = m;
        Vo[e] = v;
        if (P16 != nullptr) {
            const __nv_bfloat16 h = __float2bfloat16_rn(p);
            P16[e] = *reinterpret_cast<const uint16_t*>(&h);
        }
    }
}

}  // namespace

cudaError_t launch_adamw(const AdamwBatch& b, const AdamwConsts& c, int num_sms, cudaStream_t stream) {
    if (b.count < 1 || b.count > kAdamwMaxTensors) return cudaErrorInvalidValue;
    int64_t most = 0;
    for (int i = 0; i < b.count; ++i) most = b.n[i] > most ? b.n[i] : most;
    if (most == 0) return cudaSuccess;
    // enough CTAs for eight per SM over all tensors of the launch, at least one per tensor
    int64_t gx = (most / 4 + 255) / 256;
    const int64_t cap = (static_cast<int64_t>(num_sms) * 8 + b.count - 1) / b.count;
    if (gx > cap) gx = cap;
    if (gx < 1) gx = 1;
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(static_cast<unsigned>(gx), static_cast<unsigned>(b.count));
    cfg.blockDim = dim3(256);
    cfg.stream = stream;
    TraceScope trace("lora_adamw", stream);
    return cudaLaunchKernelEx(&cfg, k_adamw, b, c);
}

}  // namespace nf4lora
