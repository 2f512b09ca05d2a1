// Register-codebook decode of one NF4 block (64 weights, one restored scale):
// the 16 scaled levels bf16(level_j * s) ("第 04 篇：QLoRA 原理" §6.1: look
// up, scale, convert to the compute dtype) are formed once and split into
// byte planes (P: low bytes, H: high bytes, four entries per register); each
// group of four codes is then looked up with byte permutes, entries 0-7 and
// 8-15 separately and merged on bit 3 of the code.  No memory is read.
#pragma once

#include <cstdint>

#include "common.cuh"
#include "nf4_levels.cuh"

namespace nf4lora {

// The byte planes of the table for scale s.
__device__ __forceinline__ void nf4_table(float s, uint32_t (&P)[4], uint32_t (&H)[4]) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const uint32_t t0 = pack_bf16x2(__fmul_rn(nf4_level(4 * i), s), __fmul_rn(nf4_level(4 * i + 1), s));
        const uint32_t t1 = pack_bf16x2(__fmul_rn(nf4_level(4 * i + 2), s), __fmul_rn(nf4_level(4 * i + 3), s));
        P[i] = __byte_perm(t0, t1, 0x6420);
        H[i] = __byte_perm(t0, t1, 0x7531);
    }
}

// Two code bytes in the low 16 bits of xs (byte b = element 2b in the high
// nibble, 2b + 1 in the low one; nibbles low first: e1 e0 e3 e2) to the bf16
// pairs p0 = (e0, e1) and p1 = (e2, e3), the first element in the low half.
__device__ __forceinline__ void nf4_lookup4(uint32_t xs, const uint32_t (&P)[4], const uint32_t (&H)[4],
                                            uint32_t& p0, uint32_t& p1) {
    const uint32_t sel = xs & 0x7777u;                      // index within 0-7 / 8-15
    const uint32_t pick = ((xs >> 1) & 0x4444u) | 0x3210u;  // byte i from the 8-15 half if bit 3
    const uint32_t lo = __byte_perm(__byte_perm(P[0], P[1], sel), __byte_perm(P[2], P[3], sel), pick);
    const uint32_t hi = __byte_perm(__byte_perm(H[0], H[1], sel), __byte_perm(H[2], H[3], sel), pick);
    p0 = __byte_perm(lo, hi, 0x4051);  // lo.b1 hi.b1 lo.b0 hi.b0
    p1 = __byte_perm(lo, hi, 0x6273);  // lo.b3 hi.b3 lo.b2 hi.b2
}

// w: the block's 32 packed bytes as 8 words.  out[i] = (w_2i, w_2i+1) as
// bf16, w_2i in the low half.
__device__ __forceinline__ void nf4_decode_block(const uint32_t (&w)[8], float s, uint32_t (&out)[32]) {
    uint32_t P[4], H[4];
    nf4_table(s, P, H);
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        nf4_lookup4(w[j], P, H, out[4 * j], out[4 * j + 1]);
        nf4_lookup4(w[j] >> 16, P, H, out[4 * j + 2], out[4 * j + 3]);
    }
}

}  // namespace nf4lora
