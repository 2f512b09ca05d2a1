// The 16 NF4 levels in ascending order (index = 4-bit code), as printed in
// "第 04 篇：QLoRA 原理" (jupiter-lab.pages.dev) §4.3, the bitsandbytes table
// quoted there: standard-normal quantiles with equal-probability bins on each
// half, built separately so that 0 is exact, normalised to [-1, 1].
#pragma once

namespace nf4lora {

// Level j as an immediate (no constant-bank table).  Kernels that index the
// levels with per-thread codes copy them to shared memory first, where the 16
// words sit in 16 different banks, so any pattern of lookups is conflict-free.
__device__ __forceinline__ float nf4_level(int j) {
    switch (j) {
        case 0: return -1.0000000f;
        case 1: return -0.6961928f;
        case 2: return -0.5250731f;
        case 3: return -0.3949175f;
        case 4: return -0.2844414f;
        case 5: return -0.1847734f;
        case 6: return -0.0910500f;
        case 7: return 0.0000000f;
        case 8: return 0.0795803f;
        case 9: return 0.1609302f;
        case 10: return 0.2461123f;
        case 11: return 0.3379152f;
        case 12: return 0.4407098f;
        case 13: return 0.5626170f;
        case 14: return 0.7229568f;
        default: return 1.0000000f;
    }
}

// Restored first-level scale of block b: s_b = q_b * (a2_g / 127) + mean,
// each step an IEEE fp32 operation rounded once ("第 04 篇：QLoRA 原理" §6.1).
__device__ __forceinline__ float nf4_block_scale(int8_t q, float a2, float mean) {
    const float step = __fdiv_rn(a2, 127.0f);
    return __fadd_rn(__fmul_rn(static_cast<float>(q), step), mean);
}

}  // namespace nf4lora
