/*
 * CPU oracle for the NF4 + double-quantisation encoding of a frozen base
 * weight (QLoRA).  TEST INFRASTRUCTURE ONLY: the tests, the smoke check and
 * the benchmark's CPU-baseline leg call it; the product path never does.
 *
 * Plain C99, one element at a time, in the order the method states.  It
 * shares no code, header, table or constant with the CUDA library.  Compiled
 * with -ffp-contract=off so that every float operation below rounds exactly
 * once, as written.
 *
 * Sources (web pages about QLoRA):
 *   [QP] "第 04 篇：QLoRA 原理", jupiter-lab.pages.dev
 *   [CA] "QLoRA" concept page, compassingai.com (zh-hant)
 *
 * Every function is pinned by tests in tests/test_oracle_*.py against values
 * the pages print, closed forms or brute force; see the header of each.
 */
#include <math.h>
#include <stdint.h>
#include <stddef.h>
#include <stdlib.h>
#include <string.h>

#define NF4_BLOCK 64    /* first-level block, [QP] §3.4 and §4.4 */
#define DQ_BLOCK 256    /* second-level block, [QP] §5.2 */

/* ------------------------------------------------------------------ */
/* Codebook                                                            */
/* ------------------------------------------------------------------ */

/* The 16 NF4 levels as printed in [QP] §4.3 (the bitsandbytes lookup table
 * shown there, 7 decimals).  Converted to fp32 by the C compiler's
 * correctly-rounded decimal conversion. */
static const float NF4_LEVELS[16] = {
    -1.0000000f, -0.6961928f, -0.5250731f, -0.3949175f,
    -0.2844414f, -0.1847734f, -0.0910500f,  0.0000000f,
     0.0795803f,  0.1609302f,  0.2461123f,  0.3379152f,
     0.4407098f,  0.5626170f,  0.7229568f,  1.0000000f};

void oracle_nf4_levels(float out[16]) {
    memcpy(out, NF4_LEVELS, sizeof(NF4_LEVELS));
}

/* Lower tail Phi(x) = erfc(-x / sqrt 2) / 2 and upper tail 1 - Phi(x) =
 * erfc(x / sqrt 2) / 2, both with libm's erfc (each accurate in its own tail). */
static double norm_lower(double x) { return 0.5 * erfc(-x / sqrt(2.0)); }
static double norm_upper(double x) { return 0.5 * erfc(x / sqrt(2.0)); }

/* Inverse standard normal CDF by bisection, which needs only that the CDF is
 * continuous and strictly increasing: 200 halvings of [-40, 40] reach the
 * double grid.  Below 1/2 the lower tail is compared with p; above it the
 * upper tail is compared with 1 - p (exact for p >= 1/2), so both tails keep
 * full relative precision. */
double oracle_norm_ppf(double p) {
    if (!(p > 0.0 && p < 1.0)) return NAN;
    double lo = -40.0, hi = 40.0, q = 1.0 - p;
    for (int it = 0; it < 200; ++it) {
        double mid = 0.5 * (lo + hi);
        if (mid == lo || mid == hi) break;
        int below = (p < 0.5) ? (norm_lower(mid) < p) : (norm_upper(mid) > q);
        if (below) lo = mid; else hi = mid;
    }
    return 0.5 * (lo + hi);
}

/* Build the 16 levels from standard-normal quantiles ([QP] §4.2-§4.3, [CA]
 * "NF4 量化機制詳解"): equal-probability points on each half of the axis,
 * built separately so that 0 is exact, one half taking one more point;
 * merged, sorted and divided by the largest magnitude so the ends are +-1.
 *
 * The pages strip the formula of the end point.  Reading taken: the
 * probability grid runs from delta = 1 - (1/32 + 1/30)/2 down to 1/2, 9 points
 * on the positive side and 8 on the negative side, the point at 1/2 (which
 * maps to 0) dropped from each and a single 0 added. */
void oracle_nf4_build_codebook(double out[16]) {
    const double delta = 1.0 - 0.5 * (1.0 / 32.0 + 1.0 / 30.0);
    double v[16];
    int n = 0;
    for (int i = 0; i < 8; ++i) {            /* linspace(delta, 1/2, 9)[:-1] */
        double p = delta + (0.5 - delta) * (double)i / 8.0;
        v[n++] = oracle_norm_ppf(p);
    }
    for (int i = 0; i < 7; ++i) {            /* -(linspace(delta, 1/2, 8)[:-1]) */
        double p = delta + (0.5 - delta) * (double)i / 7.0;
        v[n++] = -oracle_norm_ppf(p);
    }
    v[n++] = 0.0;
    /* insertion sort, ascending */
    for (int i = 1; i < 16; ++i) {
        double key = v[i];
        int j = i - 1;
        while (j >= 0 && v[j] > key) { v[j + 1] = v[j]; --j; }
        v[j + 1] = key;
    }
    double vmax = 0.0;
    for (int i = 0; i < 16; ++i) if (fabs(v[i]) > vmax) vmax = fabs(v[i]);
    for (int i = 0; i < 16; ++i) out[i] = v[i] / vmax;
}

/* Decision thresholds between neighbouring levels: m_j = (c_j + c_{j+1}) / 2
 * evaluated in fp32 (one rounded add, then an exact halving). */
void oracle_nf4_midpoints(float out[15]) {
    for (int j = 0; j < 15; ++j) {
        float s = NF4_LEVELS[j] + NF4_LEVELS[j + 1];
        out[j] = s * 0.5f;
    }
}

/* ------------------------------------------------------------------ */
/* First-level quantisation: blockwise absmax, nearest level, packing   */
/* ------------------------------------------------------------------ */

int64_t oracle_num_blocks(int64_t n) { return (n + NF4_BLOCK - 1) / NF4_BLOCK; }
int64_t oracle_num_groups(int64_t n) {
    return (oracle_num_blocks(n) + DQ_BLOCK - 1) / DQ_BLOCK;
}

/* a_b = max |w_i| over each block of 64 consecutive elements of the
 * row-major flattened tensor; the last block may be short.  [QP] §3.4,
 * §4.4; [CA] step 2. */
void oracle_nf4_absmax(const float* w, int64_t n, float* absmax) {
    int64_t nb = oracle_num_blocks(n);
#pragma omp parallel for schedule(static)
    for (int64_t b = 0; b < nb; ++b) {
        int64_t lo = b * NF4_BLOCK, hi = lo + NF4_BLOCK < n ? lo + NF4_BLOCK : n;
        float m = 0.0f;
        for (int64_t i = lo; i < hi; ++i) {
            float a = fabsf(w[i]);
            if (a > m) m = a;
        }
        absmax[b] = m;
    }
}

/* One 4-bit code per element: normalise x = w / a_b (IEEE fp32 division,
 * rounded once) and take the nearest level, realised as the number of
 * thresholds strictly below x.  A value exactly on a threshold therefore goes
 * to the lower level (reading: the pages do not state the tie rule).  An
 * all-zero block (a_b == 0) encodes every element as level 7, the exact 0.
 * [QP] §3.2 (index of the nearest codebook point), §4.3 (encoding);
 * [CA] step 3. */
void oracle_nf4_encode(const float* w, int64_t n, const float* absmax,
                       uint8_t* codes) {
    float mid[15];
    oracle_nf4_midpoints(mid);
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) {
        float a = absmax[i / NF4_BLOCK];
        uint8_t code = 7;
        if (a != 0.0f) {
            float x = w[i] / a;
            code = 0;
            for (int j = 0; j < 15; ++j) if (x > mid[j]) ++code;
        }
        codes[i] = code;
    }
}

/* Two codes per byte ([QP] §2.1).  Reading for the unstated nibble order:
 * the even element goes to the high nibble.  An odd element count leaves the
 * low nibble of the last byte zero. */
void oracle_nf4_pack(const uint8_t* codes, int64_t n, uint8_t* packed) {
    for (int64_t i = 0; i < (n + 1) / 2; ++i) {
        uint8_t hi = codes[2 * i];
        uint8_t lo = (2 * i + 1 < n) ? codes[2 * i + 1] : 0;
        packed[i] = (uint8_t)((hi << 4) | lo);
    }
}

void oracle_nf4_unpack(const uint8_t* packed, int64_t n, uint8_t* codes) {
    for (int64_t i = 0; i < n; ++i) {
        uint8_t byte = packed[i / 2];
        codes[i] = (i % 2 == 0) ? (uint8_t)(byte >> 4) : (uint8_t)(byte & 15);
    }
}

/* ------------------------------------------------------------------ */
/* Second-level (double) quantisation of the block scales               */
/* ------------------------------------------------------------------ */

/* mu = mean of all first-level scales of the tensor ([QP] §5.2: the scales
 * are positive, so their mean is subtracted first).  Reading for the unstated
 * summation order: the sum is formed in fp64 by a pairwise tree, level by
 * level, s'[i] = s[2i] + s[2i+1], an odd last element carried up unchanged;
 * then mu = fp32(sum / n_b). */
float oracle_dq_mean(const float* absmax, int64_t nb) {
    if (nb <= 0) return 0.0f;
    double* buf = (double*)malloc((size_t)nb * sizeof(double));
    for (int64_t i = 0; i < nb; ++i) buf[i] = (double)absmax[i];
    int64_t len = nb;
    while (len > 1) {
        int64_t half = len / 2;
        for (int64_t i = 0; i < half; ++i) buf[i] = buf[2 * i] + buf[2 * i + 1];
        if (len % 2) { buf[half] = buf[len - 1]; len = half + 1; }
        else len = half;
    }
    double total = buf[0];
    free(buf);
    return (float)(total / (double)nb);
}

/* Per group g of 256 consecutive scales (the last group may be short):
 * d_b = a_b - mu (fp32), a2_g = max |d_b|, and the symmetric 8-bit code
 * q_b = rint((d_b / a2_g) * 127) with round-half-even, in [-127, 127].
 * A group with a2_g == 0 stores q_b = 0.  [QP] §5.2 (centre, then symmetric
 * 8-bit, second block 256, one fp32 scale per group), §3.3.
 * Reading: "8-bit" is a linear int8 with 127 steps per side; the
 * compassingai page's FP8 is not taken (see the design notes). */
void oracle_dq_quantize(const float* absmax, int64_t nb, float mu, int8_t* q,
                        float* a2) {
    int64_t ng = (nb + DQ_BLOCK - 1) / DQ_BLOCK;
#pragma omp parallel for schedule(static)
    for (int64_t g = 0; g < ng; ++g) {
        int64_t lo = g * DQ_BLOCK, hi = lo + DQ_BLOCK < nb ? lo + DQ_BLOCK : nb;
        float m = 0.0f;
        for (int64_t b = lo; b < hi; ++b) {
            float d = absmax[b] - mu;
            if (fabsf(d) > m) m = fabsf(d);
        }
        a2[g] = m;
        for (int64_t b = lo; b < hi; ++b) {
            if (m == 0.0f) { q[b] = 0; continue; }
            float d = absmax[b] - mu;
            float t = (d / m) * 127.0f;
            float r = rintf(t);             /* default rounding mode: half-even */
            if (r > 127.0f) r = 127.0f;
            if (r < -127.0f) r = -127.0f;
            q[b] = (int8_t)r;
        }
    }
}

/* Restored first-level scale ([QP] §6.1, double dequantisation, and §5.4):
 * s_b = q_b * (a2_g / 127) + mu, as a rounded fp32 multiply followed by a
 * rounded fp32 add (no fused multiply-add). */
void oracle_dq_scales(const int8_t* q, const float* a2, float mu, int64_t nb,
                      float* s_hat) {
#pragma omp parallel for schedule(static)
    for (int64_t b = 0; b < nb; ++b) {
        float step = a2[b / DQ_BLOCK] / 127.0f;
        float prod = (float)q[b] * step;
        s_hat[b] = prod + mu;
    }
}

/* fp32 -> bfloat16 bit pattern, round to nearest, ties to even (the compute
 * dtype of [QP] §6.2).  NaN maps to a quiet NaN. */
uint16_t oracle_bf16_bits(float x) {
    uint32_t u;
    memcpy(&u, &x, 4);
    if ((u & 0x7f800000u) == 0x7f800000u && (u & 0x007fffffu))
        return (uint16_t)((u >> 16) | 0x40u);
    uint32_t lsb = (u >> 16) & 1u;
    u += 0x7fffu + lsb;
    return (uint16_t)(u >> 16);
}

/* Dequantised weight, bit-exact definition: w_hat = bf16(c[code] * s_b), one
 * rounded fp32 multiply then one rounding to bfloat16.  [QP] §6.1 (unpack,
 * restore the scale in two levels, look up, scale, convert to the compute
 * dtype). */
void oracle_nf4_dequantize(const uint8_t* packed, const int8_t* q,
                           const float* a2, float mu, int64_t n,
                           uint16_t* w_bf16) {
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) {
        int64_t b = i / NF4_BLOCK;
        float step = a2[b / DQ_BLOCK] / 127.0f;
        float s = (float)q[b] * step + mu;
        uint8_t byte = packed[i / 2];
        uint8_t code = (i % 2 == 0) ? (uint8_t)(byte >> 4) : (uint8_t)(byte & 15);
        float v = NF4_LEVELS[code] * s;
        w_bf16[i] = oracle_bf16_bits(v);
    }
}

/* Dequantised weight from plain fp32 block scales (the encoding without
 * double quantisation, [QP] §5.1: one 32-bit scale per block of 64):
 * w_hat = bf16(c[code] * s_b) with s_b = scale[b], the same look-up, scale
 * and conversion as above without the two-level restore. */
void oracle_nf4_dequantize_scales(const uint8_t* packed, const float* scale,
                                  int64_t n, uint16_t* w_bf16) {
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) {
        float s = scale[i / NF4_BLOCK];
        uint8_t byte = packed[i / 2];
        uint8_t code = (i % 2 == 0) ? (uint8_t)(byte >> 4) : (uint8_t)(byte & 15);
        float v = NF4_LEVELS[code] * s;
        w_bf16[i] = oracle_bf16_bits(v);
    }
}

/* Whole encoding of one tensor, in the pages' order. */
void oracle_nf4_quantize(const float* w, int64_t n, uint8_t* packed,
                         int8_t* q, float* a2, float* mu_out, float* absmax_ws,
                         uint8_t* codes_ws) {
    int64_t nb = oracle_num_blocks(n);
    oracle_nf4_absmax(w, n, absmax_ws);
    oracle_nf4_encode(w, n, absmax_ws, codes_ws);
    oracle_nf4_pack(codes_ws, n, packed);
    float mu = oracle_dq_mean(absmax_ws, nb);
    oracle_dq_quantize(absmax_ws, nb, mu, q, a2);
    *mu_out = mu;
}

/* Storage of one encoded tensor in bytes: n/2 code bytes, one int8 scale per
 * block, one fp32 second-level scale per group and one fp32 mean ([QP] §5.3,
 * §8.1). */
int64_t oracle_packed_bytes(int64_t n) {
    return (n + 1) / 2 + oracle_num_blocks(n) + 4 * oracle_num_groups(n) + 4;
}

/* Storage without double quantisation: n/2 code bytes and one fp32 scale per
 * block ([QP] §5.1: 32 bits per 64 weights, 0.5 bit per weight). */
int64_t oracle_packed_bytes_nodq(int64_t n) {
    return (n + 1) / 2 + 4 * oracle_num_blocks(n);
}
