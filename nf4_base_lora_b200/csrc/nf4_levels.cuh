// The 16 NF4 levels in ascending order (index = 4-bit code), as printed in
// "第 04 篇：QLoRA 原理" (jupiter-lab.pages.dev) §4.3, the bitsandbytes table
// quoted there: standard-normal quantiles with equal-probability bins on each
// half, built separately so that 0 is exact, normalised to [-1, 1].
#pragma once

namespace nf4lora {

// One copy per translation unit in the constant bank.  Kernels that index it
// with per-thread codes copy it to shared memory first, where the 16 words
// sit in 16 different banks, so any pattern of lookups is conflict-free.
static __constant__ float kNf4Levels[16] = {
    -1.0000000f, -0.6961928f, -0.5250731f, -0.3949175f, -0.2844414f, -0.1847734f,
    -0.0910500f, 0.0000000f,  0.0795803f,  0.1609302f,  0.2461123f,  0.3379152f,
    0.4407098f,  0.5626170f,  0.7229568f,  1.0000000f};

// Restored first-level scale of block b: s_b = q_b * (a2_g / 127) + mean,
// each step an IEEE fp32 operation rounded once ("第 04 篇：QLoRA 原理" §6.1).
__device__ __forceinline__ float nf4_block_scale(int8_t q, float a2, float mean) {
    const float step = __fdiv_rn(a2, 127.0f);
    return __fadd_rn(__fmul_rn(static_cast<float>(q), step), mean);
}

}  // namespace nf4lora
