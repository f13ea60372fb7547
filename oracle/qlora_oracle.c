/*
 * Plain, slow CPU oracle for the QLoRA frozen-base codec.
 *
 * TEST INFRASTRUCTURE ONLY. Only tests/, __graft_entry__.smoke() and the
 * cpu_baseline / reference leg of bench.py may load this code. The product
 * library never links it, and this file includes nothing from the product.
 *
 * Every routine restates a step described on the QLoRA pages:
 *   - "4-bit NormalFloat" (promptingindex.com, "Finetuning 65B Models on a
 *     Single GPU", NF4 section) and the formulation's symbol list on
 *     intvml.com "DL0087 QLoRA: 4-bit Quantized LoRA" (levels at normal
 *     quantiles, rescaled to [-1,1] with an exact zero);
 *   - "Blockwise Absmax Scaling" (intvml.com, component 2): blocks of 64
 *     weights, one absmax constant per block;
 *   - "Double Quantization" (intvml.com, component 3; promptingindex.com,
 *     "Double Quantization and Paged Optimizers"): the constants quantized
 *     to 8 bits with one fp32 scale per 256 constants;
 *   - dequantization to bf16 just before the matmul (intvml.com, opening
 *     paragraph and Figure 1).
 * Where the pages are silent the plain reading chosen is written beside the
 * step (table offset, tie-break, nibble order, 8-bit code map, zero blocks).
 *
 * Build: gcc -O2 -fno-fast-math -ffp-contract=off -fexcess-precision=standard
 *        -mfpmath=sse -shared -fPIC (x86-64: all float arithmetic is IEEE
 *        binary32 with round-to-nearest-even, no contraction).
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

#define ORACLE_BLOCK 64      /* weights per absmax constant            */
#define ORACLE_DQ_BLOCK 256  /* absmax constants per second-level scale */

/* ---------------------------------------------------------------- bf16 -- */

/* bf16 bit pattern -> binary32 value (exact: bf16 is the top half of fp32). */
static float bf16_to_float(uint16_t h) {
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

/* binary32 -> bf16 with round-to-nearest-even, done on the bit pattern.
 * NaN maps to the canonical quiet NaN 0x7FC0 (inputs are finite anyway). */
static uint16_t float_to_bf16_rne(float f) {
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    if ((u & 0x7F800000u) == 0x7F800000u && (u & 0x007FFFFFu) != 0u)
        return (uint16_t)0x7FC0u;
    uint32_t lsb = (u >> 16) & 1u;
    u += 0x7FFFu + lsb;
    return (uint16_t)(u >> 16);
}

/* binary32 -> IEEE 754 binary16 (1 sign, 5 exponent bits of bias 15, 10
 * fraction bits) with round-to-nearest-even, on the bit patterns:
 *   |f| >= 65520 (half-way above the largest finite 65504) -> inf;
 *   2^-14 <= |f|: normal, the 23-bit fraction rounded to 10 bits (a carry
 *                 out of the fraction correctly bumps the exponent);
 *   |f| <  2^-14: subnormal, |f| / 2^-24 rounded to an integer (2^-24 is
 *                 the subnormal unit; 1024 units become the least normal).
 * NaN maps to the quiet NaN 0x7E00 with the input's sign. */
static uint16_t float_to_f16_rne(float f) {
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    uint16_t sign = (uint16_t)((u >> 16) & 0x8000u);
    uint32_t a = u & 0x7FFFFFFFu;
    if (a > 0x7F800000u) return (uint16_t)(sign | 0x7E00u);
    if (a >= 0x477FF000u) return (uint16_t)(sign | 0x7C00u);
    if (a >= 0x38800000u) {
        uint32_t e = (a >> 23) - 127u + 15u;
        uint32_t frac = a & 0x7FFFFFu;
        uint32_t h = (e << 10) | (frac >> 13);
        uint32_t rem = frac & 0x1FFFu;
        if (rem > 0x1000u || (rem == 0x1000u && (h & 1u))) h += 1u;
        return (uint16_t)(sign | h);
    }
    uint32_t E = a >> 23;             /* biased binary32 exponent, <= 112 here */
    if (E < 102u) return sign;        /* |f| < 2^-25: rounds to (signed) zero */
    uint32_t sig = (a & 0x7FFFFFu) | 0x800000u;  /* |f| = sig * 2^(E - 150)  */
    uint32_t shift = 126u - E;        /* |f| / 2^-24 = sig / 2^shift, 14..24 */
    uint32_t h = sig >> shift;
    uint32_t rem = sig & ((1u << shift) - 1u);
    uint32_t half = 1u << (shift - 1u);
    if (rem > half || (rem == half && (h & 1u))) h += 1u;
    return (uint16_t)(sign | h);
}

/* -------------------------------------------------------- NF4 levels ---- */

/* Standard normal CDF in long double. */
static long double std_normal_cdf(long double z) {
    return 0.5L * erfcl(-z / sqrtl(2.0L));
}

/* Standard normal quantile by plain bisection on the CDF (long double).
 * 200 halvings of [-40, 40] reach far below long-double resolution. */
static long double std_normal_quantile(long double p) {
    long double lo = -40.0L, hi = 40.0L;
    for (int it = 0; it < 200; ++it) {
        long double mid = 0.5L * (lo + hi);
        if (std_normal_cdf(mid) < p) lo = mid; else hi = mid;
    }
    return 0.5L * (lo + hi);
}

/*
 * The 16 NF4 levels, ascending.
 *
 * The pages fix: 16 levels at quantiles of N(0,1), each level covering equal
 * probability mass, rescaled into [-1, 1], with an exact zero. Sixteen is
 * even, so a symmetric set cannot hold 0: the reading taken here splits the
 * codes 7 (negative) + 1 (zero) + 8 (positive). Each side takes its
 * quantiles at probabilities evenly spaced from delta down towards 1/2
 * (8 positive probabilities on a 9-point grid and 7 negative ones on an
 * 8-point grid, the 1/2 end point dropped), so each side's levels cut the
 * half-line into equal-mass pieces. delta (the outermost probability; the
 * pages give none) is the mean of the last-bin centres for 15 and 16
 * equal-mass bins: delta = ((1 - 1/30) + (1 - 1/32)) / 2. Dividing by
 * quantile(delta) puts the extremes at exactly -1 and +1.
 */
void oracle_nf4_levels(float out[16]) {
    const long double delta = 0.5L * ((1.0L - 1.0L / 30.0L) + (1.0L - 1.0L / 32.0L));
    const long double zmax = std_normal_quantile(delta);
    /* negative side: 7 levels, most negative first */
    for (int i = 0; i < 7; ++i) {
        long double p = delta + (long double)i * (0.5L - delta) / 7.0L;
        out[i] = (float)(-std_normal_quantile(p) / zmax);
    }
    out[7] = 0.0f;
    /* positive side: 8 levels, largest (j = 0) stored last */
    for (int j = 0; j < 8; ++j) {
        long double p = delta + (long double)j * (0.5L - delta) / 8.0L;
        out[15 - j] = (float)(std_normal_quantile(p) / zmax);
    }
}

/*
 * The 8-bit code map for the absmax constants: 256 values, ascending.
 * The pages say only "8-bit" with one fp32 scale per 256 constants, and the
 * storage count (4 + 0.125 + 0.002 bits) leaves no room for a stored offset.
 * Absmax constants are >= 0, so the reading taken is the unsigned linear map
 * T8[k] = k / 255 (rounded once to fp32). Any other ascending map can be
 * passed in its place.
 */
void oracle_dq_levels(float out[256]) {
    for (int k = 0; k < 256; ++k)
        out[k] = (float)((double)k / 255.0);
}

/* ------------------------------------------------- nearest-level encode - */

/* Index of the nearest level by the midpoint rule: the count of midpoints
 * strictly below x, midpoints formed in fp32 as (L[i] + L[i+1]) * 0.5.
 * A value exactly on a midpoint goes to the lower level (pages silent). */
static int nearest_level(float x, const float *levels, int n) {
    int code = 0;
    for (int i = 0; i + 1 < n; ++i) {
        float mid = (levels[i] + levels[i + 1]) * 0.5f;
        if (x > mid) code += 1;
    }
    return code;
}

int oracle_nearest_level(float x, const float *levels, int n) {
    return nearest_level(x, levels, n);
}

/* ------------------------------------------- blockwise absmax + encode -- */

/*
 * absmax[b] = max |w| over block b, the 64 consecutive elements
 * w[64b .. 64b+63] of the row-major [N, K] weight (K % 64 == 0, so no block
 * crosses a row). Exact in fp32: it is a max of bf16 values.
 */
void oracle_absmax(const uint16_t *w, int64_t n_elems, float *absmax) {
    int64_t nb = n_elems / ORACLE_BLOCK;
    for (int64_t b = 0; b < nb; ++b) {
        float m = 0.0f;
        for (int e = 0; e < ORACLE_BLOCK; ++e) {
            float v = fabsf(bf16_to_float(w[b * ORACLE_BLOCK + e]));
            if (v > m) m = v;
        }
        absmax[b] = m;
    }
}

/*
 * NF4 codes for every element, packed two per byte: element 2j in the low
 * nibble of byte j, element 2j+1 in the high nibble (pages silent on order).
 * x = w / absmax (IEEE fp32 division); an all-zero block (absmax 0) encodes
 * every element as x = 0, i.e. the index of the exact-zero level.
 */
void oracle_encode_nf4(const uint16_t *w, int64_t n_elems, const float *absmax,
                       const float levels[16], uint8_t *packed) {
    for (int64_t e = 0; e < n_elems; e += 2) {
        int codes[2];
        for (int h = 0; h < 2; ++h) {
            float c = absmax[(e + h) / ORACLE_BLOCK];
            float x = (c == 0.0f) ? 0.0f : bf16_to_float(w[e + h]) / c;
            codes[h] = nearest_level(x, levels, 16);
        }
        packed[e / 2] = (uint8_t)(codes[0] | (codes[1] << 4));
    }
}

/* ------------------------------------------------- double quantization -- */

/*
 * Second-level quantization of the absmax constants: consecutive groups of
 * 256 constants in global block order (the last group may be shorter).
 * S[g] = max of the group (fp32; the constants are non-negative),
 * q = nearest 8-bit level of c / S[g] by the same midpoint rule.
 * A group of zeros (S = 0) encodes x = 0.
 */
void oracle_double_quant(const float *absmax, int64_t nb, const float t8[256],
                         uint8_t *q, float *scale2) {
    int64_t ng = (nb + ORACLE_DQ_BLOCK - 1) / ORACLE_DQ_BLOCK;
    for (int64_t g = 0; g < ng; ++g) {
        int64_t lo = g * ORACLE_DQ_BLOCK;
        int64_t hi = lo + ORACLE_DQ_BLOCK < nb ? lo + ORACLE_DQ_BLOCK : nb;
        float s = 0.0f;
        for (int64_t b = lo; b < hi; ++b)
            if (absmax[b] > s) s = absmax[b];
        scale2[g] = s;
        for (int64_t b = lo; b < hi; ++b) {
            float x = (s == 0.0f) ? 0.0f : absmax[b] / s;
            q[b] = (uint8_t)nearest_level(x, t8, 256);
        }
    }
}

/* --------------------------------------------------------- dequantize -- */

/*
 * W'[e] = bf16_rne( L[code_e] * c'_b ),  c'_b = T8[q_b] * S[b / 256],
 * both products in fp32. Dequantization uses the double-quantized constant
 * c' (the stored state is (q, S); the fp32 absmax is not kept).
 */
void oracle_dequant(const uint8_t *packed, const uint8_t *q, const float *scale2,
                    int64_t n_elems, const float levels[16], const float t8[256],
                    uint16_t *w_out) {
    for (int64_t e = 0; e < n_elems; ++e) {
        int64_t b = e / ORACLE_BLOCK;
        float cprime = t8[q[b]] * scale2[b / ORACLE_DQ_BLOCK];
        int code = (e & 1) ? (packed[e / 2] >> 4) : (packed[e / 2] & 0x0F);
        float v = levels[code] * cprime;
        w_out[e] = float_to_bf16_rne(v);
    }
}

/* The same dequantization with an fp16 result (the pages' other 16-bit
 * compute type, systemoverflow.com "QLoRA ... at Extreme Scale"):
 * W'[e] = f16_rne( L[code_e] * c'_b ), the products as above. */
void oracle_dequant_f16(const uint8_t *packed, const uint8_t *q, const float *scale2,
                        int64_t n_elems, const float levels[16], const float t8[256],
                        uint16_t *w_out) {
    for (int64_t e = 0; e < n_elems; ++e) {
        int64_t b = e / ORACLE_BLOCK;
        float cprime = t8[q[b]] * scale2[b / ORACLE_DQ_BLOCK];
        int code = (e & 1) ? (packed[e / 2] >> 4) : (packed[e / 2] & 0x0F);
        float v = levels[code] * cprime;
        w_out[e] = float_to_f16_rne(v);
    }
}

void oracle_f32_to_f16(const float *f, int64_t n, uint16_t *out) {
    for (int64_t i = 0; i < n; ++i) out[i] = float_to_f16_rne(f[i]);
}

/* The double-quantized constants c'_b alone (used by the round-trip pins). */
void oracle_dq_constants(const uint8_t *q, const float *scale2, int64_t nb,
                         const float t8[256], float *cprime) {
    for (int64_t b = 0; b < nb; ++b)
        cprime[b] = t8[q[b]] * scale2[b / ORACLE_DQ_BLOCK];
}

/* bf16 <-> fp32 helpers exported for the tests' own use. */
void oracle_bf16_to_f32(const uint16_t *h, int64_t n, float *out) {
    for (int64_t i = 0; i < n; ++i) out[i] = bf16_to_float(h[i]);
}

void oracle_f32_to_bf16(const float *f, int64_t n, uint16_t *out) {
    for (int64_t i = 0; i < n; ++i) out[i] = float_to_bf16_rne(f[i]);
}
