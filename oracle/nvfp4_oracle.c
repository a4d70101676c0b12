/*
 * nvfp4_oracle.c — plain, slow CPU oracle for BF16 -> NVFP4 quantization.
 *
 * TEST INFRASTRUCTURE ONLY (see nvfp4_oracle.h): used by the tests, the smoke check and the
 * bench's CPU-baseline leg, never by the product path. No code is shared with the CUDA side.
 *
 * The algorithm follows the Four Over Six page's technical summary in its own order:
 *   Problem definition: NVFP4 = E2M1 values {0, 0.5, 1, 1.5, 2, 3, 4, 6} with steps
 *     0.5 on [0,2], 1 on [2,4], 2 on [4,6]; standard quantization scales each block so its
 *     maximum lands on 6.
 *   Core mechanism: a block may instead be scaled so its maximum lands on 4.
 *   Adaptive block scaling algorithm: quantize each block twice (target 6 and target 4),
 *     compute each version's error against the original high-precision values, keep the
 *     version with the smaller error under one of three rules (max error, MAE, MSE).
 *   Implementation details: block scales are FP8 E4M3 under a global tensor scale alpha;
 *     in Four Over Six mode alpha is built from FP8 max 256 instead of 448, because a
 *     target-4 block needs a 1.5x larger E4M3 scale than a target-6 block.
 * Block size 16 along the last dimension: QAD page, technical summary §3.3.
 *
 * Where the pages leave a step open, the reading used is written beside the step.
 */
#include "nvfp4_oracle.h"

#include <float.h>
#include <math.h>
#include <string.h>

static float f32_from_bits(uint32_t u) { float f; memcpy(&f, &u, sizeof f); return f; }
static uint32_t bits_from_f32(float f) { uint32_t u; memcpy(&u, &f, sizeof u); return u; }

/* ---- BF16 ------------------------------------------------------------------------------ */

float nvo_bf16_to_f32(uint16_t b) { return f32_from_bits((uint32_t)b << 16); }

/* Value of a BF16 bit pattern in binary64, with the all-ones-exponent pattern read as 2^128
 * (the overflow threshold IEEE round-to-nearest uses). */
static double bf16_value_for_rounding(uint16_t b) {
    if ((b & 0x7FFFu) == 0x7F80u) return (b & 0x8000u) ? -ldexp(1.0, 128) : ldexp(1.0, 128);
    return (double)nvo_bf16_to_f32(b);
}

uint16_t nvo_f32_to_bf16_rne(float f) {
    uint32_t u = bits_from_f32(f);
    if (isnan(f)) return (uint16_t)((u >> 16) | 0x0040u);      /* outside the contract */
    if (isinf(f)) return (uint16_t)(u >> 16);
    /* The two BF16 neighbours: `lo` truncates toward zero, `hi` is the next one away. */
    uint16_t lo = (uint16_t)(u >> 16);
    uint16_t hi = (uint16_t)(lo + 1u);
    double v = (double)f;
    double below = fabs(v - bf16_value_for_rounding(lo));        /* exact in binary64 */
    double above = fabs(bf16_value_for_rounding(hi) - v);
    if (below < above) return lo;
    if (above < below) return hi;
    return (lo & 1u) ? hi : lo;                                   /* tie: even mantissa */
}

/* ---- E4M3 (block scale) --------------------------------------------------------------- */

uint8_t nvo_f32_to_e4m3_satfinite(float t) {
    uint8_t sign = signbit(t) ? 0x80u : 0x00u;
    double a = fabs((double)t);
    if (isnan(t)) return (uint8_t)(sign | 0x7Fu);                 /* outside the contract */
    double v;
    if (isinf(t)) {
        v = 448.0;
    } else if (a == 0.0) {
        return sign;
    } else {
        int e;
        frexp(a, &e);
        e -= 1;                         /* a = m * 2^e, m in [1, 2) */
        if (e < -6) e = -6;             /* below 2^-6 the lattice step stays 2^-9 (subnormals) */
        double step = ldexp(1.0, e - 3);  /* 3 mantissa bits */
        v = rint(a / step) * step;        /* a/step is exact; rint rounds half to even */
        if (v > 448.0) v = 448.0;         /* satfinite */
    }
    if (v < ldexp(1.0, -6)) {             /* subnormal: v = n * 2^-9, n in 0..7 */
        return (uint8_t)(sign | (uint8_t)(v / ldexp(1.0, -9)));
    }
    int e;
    double m = frexp(v, &e);              /* v = m * 2^e, m in [0.5, 1) */
    int exp_field = (e - 1) + 7;
    int man = (int)((m * 2.0 - 1.0) * 8.0);   /* exact: v has at most 4 significant bits */
    return (uint8_t)(sign | (uint8_t)(exp_field << 3) | (uint8_t)man);
}

float nvo_e4m3_to_f32(uint8_t s) {
    int exp_field = (s >> 3) & 0xF;
    int man = s & 0x7;
    double v;
    if ((s & 0x7Fu) == 0x7Fu) return NAN;
    if (exp_field == 0) v = man * ldexp(1.0, -9);
    else v = (1.0 + man / 8.0) * ldexp(1.0, exp_field - 7);
    return (float)((s & 0x80u) ? -v : v);
}

/* ---- E2M1 (element values) ------------------------------------------------------------ */

uint8_t nvo_f32_to_e2m1_satfinite(float y) {
    uint8_t sign = signbit(y) ? 0x8u : 0x0u;
    double a = fabs((double)y);
    double v;
    if (isnan(y)) return (uint8_t)(sign | 0x7u);                  /* outside the contract */
    if (isinf(y)) {
        v = 6.0;
    } else {
        /* Step sizes of the E2M1 grid (Problem definition): 0.5 below 2, 1 on [2,4), 2 from 4. */
        double step = (a < 2.0) ? 0.5 : (a < 4.0 ? 1.0 : 2.0);
        v = rint(a / step) * step;
        if (v > 6.0) v = 6.0;
    }
    /* magnitude index: 0, 0.5, 1, 1.5, 2 -> 0..4; 3 -> 5; 4 -> 6; 6 -> 7 */
    uint8_t idx;
    if (v <= 2.0) idx = (uint8_t)(v * 2.0);
    else if (v == 3.0) idx = 5;
    else if (v == 4.0) idx = 6;
    else idx = 7;
    return (uint8_t)(sign | idx);
}

float nvo_e2m1_to_f32(uint8_t c) {
    int idx = c & 0x7;
    int ebits = idx >> 1, mbit = idx & 1;
    double v = (ebits == 0) ? 0.5 * mbit : (1.0 + 0.5 * mbit) * ldexp(1.0, ebits - 1);
    return (float)((c & 0x8u) ? -v : v);
}

void nvo_f32_to_e2m1_array(const float* in, uint8_t* out, int64_t n) {
    for (int64_t i = 0; i < n; ++i) out[i] = nvo_f32_to_e2m1_satfinite(in[i]);
}

void nvo_f32_to_e4m3_array(const float* in, uint8_t* out, int64_t n) {
    for (int64_t i = 0; i < n; ++i) out[i] = nvo_f32_to_e4m3_satfinite(in[i]);
}

void nvo_f32_to_bf16_array(const float* in, uint16_t* out, int64_t n) {
    for (int64_t i = 0; i < n; ++i) out[i] = nvo_f32_to_bf16_rne(in[i]);
}

/* ---- one block, one candidate --------------------------------------------------------- */

void nvo_block_candidate(const float x[16], float alpha, float K, int rule, nvo_candidate* c) {
    /* Block maximum |x| (exact). */
    float m = 0.0f;
    for (int i = 0; i < 16; ++i) {
        float a = fabsf(x[i]);
        if (a > m) m = a;
    }
    /* Block scale: the E4M3 value that maps the block max onto K, i.e. m / (K * alpha),
     * rounded to nearest-even and saturated at 448 (Implementation details: E4M3 scale
     * factor; reading: the "cvt family" rounds to nearest with satfinite). */
    c->beta = K * alpha;
    c->t = (c->beta > 0.0f) ? m / c->beta : 0.0f;
    c->s = nvo_f32_to_e4m3_satfinite(c->t);
    /* Decode scale and encode factor. Reading: elements are scaled by one reciprocal per
     * block; the clamp keeps 0 * inf out when d is tiny. */
    c->d = nvo_e4m3_to_f32(c->s) * alpha;
    if (c->d > 0.0f) {
        float r = 1.0f / c->d;
        c->r = (r > FLT_MAX) ? FLT_MAX : r;
    } else {
        c->r = 0.0f;
    }
    /* Element codes, dequantized values and errors against the original values
     * (Adaptive block scaling algorithm: error computation). */
    float acc[2] = {0.0f, 0.0f};
    float emax = 0.0f;
    for (int i = 0; i < 16; ++i) {
        float y = x[i] * c->r;
        c->code[i] = nvo_f32_to_e2m1_satfinite(y);
        float v = nvo_e2m1_to_f32(c->code[i]);
        c->q[i] = v * c->d;
        /* Reading: the error is the exact difference between the original value and the
         * dequantized value v * d, rounded once (a fused multiply-add). */
        c->e[i] = fmaf(-v, c->d, x[i]);
        float ae = fabsf(c->e[i]);
        /* Rules (Adaptive block scaling algorithm: selection rule). Reading: sums are not
         * divided by 16 (an exact scaling that cannot change the choice) and are accumulated
         * in two running sums, one over even and one over odd element indices, each in
         * increasing index order, added at the end. */
        switch (rule) {
            case NVO_RULE_MAXERR: if (ae > emax) emax = ae; break;
            case NVO_RULE_MAE:    acc[i & 1] = acc[i & 1] + ae; break;
            default:              acc[i & 1] = fmaf(c->e[i], c->e[i], acc[i & 1]); break;
        }
    }
    c->err = (rule == NVO_RULE_MAXERR) ? emax : acc[0] + acc[1];
}

/* ---- tensors ------------------------------------------------------------------------- */

void nvo_amax(const uint16_t* x, int64_t groups, int64_t rows, int64_t cols, float* amax) {
    int64_t per_group = rows * cols;
    for (int64_t g = 0; g < groups; ++g) {
        float m = 0.0f;
        for (int64_t i = 0; i < per_group; ++i) {
            float a = fabsf(nvo_bf16_to_f32(x[g * per_group + i]));
            if (a > m) m = a;
        }
        amax[g] = m;
    }
}

/* Global tensor scale (Implementation details): alpha = amax / (6 * M), M the FP8 E4M3
 * maximum the tensor scale is built from. Reading: alpha is the decode-side scale, so a
 * stored value is v * s * alpha. */
static float tensor_scale_with_max(float amax, float fp8_max) {
    float six_m = 6.0f * fp8_max;           /* 2688 or 1536, exact */
    return amax / six_m;
}

float nvo_tensor_scale(float amax, int mode) {
    return tensor_scale_with_max(amax, mode == NVO_FOUR_OVER_SIX ? 256.0f : 448.0f);
}

void nvo_quantize_ex(const uint16_t* x, int64_t groups, int64_t rows, int64_t cols,
                     const float* amax, float fp8_max, int cand_mask, int rule,
                     uint8_t* codes, uint8_t* scales, float* tscale, uint8_t* choice, uint16_t* fq) {
    int64_t blocks_per_group = rows * cols / 16;
    int64_t nblocks = groups * blocks_per_group;
    if (choice) memset(choice, 0, (size_t)((nblocks + 7) / 8));
    for (int64_t g = 0; g < groups; ++g) {
        float alpha = tensor_scale_with_max(amax[g], fp8_max);
        if (tscale) tscale[g] = alpha;
        for (int64_t bl = 0; bl < blocks_per_group; ++bl) {
            int64_t b = g * blocks_per_group + bl;
            float xb[16];
            for (int i = 0; i < 16; ++i) xb[i] = nvo_bf16_to_f32(x[b * 16 + i]);
            nvo_candidate c6, c4;
            const nvo_candidate* chosen;
            int four = 0;
            if (cand_mask == 1) {
                nvo_block_candidate(xb, alpha, 6.0f, rule, &c6);
                chosen = &c6;
            } else if (cand_mask == 2) {
                nvo_block_candidate(xb, alpha, 4.0f, rule, &c4);
                chosen = &c4;
                four = 1;
            } else {
                nvo_block_candidate(xb, alpha, 6.0f, rule, &c6);
                nvo_block_candidate(xb, alpha, 4.0f, rule, &c4);
                /* Keep the smaller error; reading: ties keep target 6, the standard format. */
                four = (c4.err < c6.err);
                chosen = four ? &c4 : &c6;
            }
            if (codes)
                for (int j = 0; j < 8; ++j)
                    codes[b * 8 + j] = (uint8_t)(chosen->code[2 * j] | (chosen->code[2 * j + 1] << 4));
            if (scales) scales[b] = chosen->s;
            if (choice && four) choice[b / 8] |= (uint8_t)(1u << (b % 8));
            if (fq)
                for (int i = 0; i < 16; ++i) fq[b * 16 + i] = nvo_f32_to_bf16_rne(chosen->q[i]);
        }
    }
}

void nvo_quantize(const uint16_t* x, int64_t groups, int64_t rows, int64_t cols,
                  const float* amax, int mode, int rule,
                  uint8_t* codes, uint8_t* scales, float* tscale, uint8_t* choice, uint16_t* fq) {
    if (mode == NVO_FOUR_OVER_SIX)
        nvo_quantize_ex(x, groups, rows, cols, amax, 256.0f, 3, rule, codes, scales, tscale, choice, fq);
    else
        nvo_quantize_ex(x, groups, rows, cols, amax, 448.0f, 1, rule, codes, scales, tscale, choice, fq);
}

void nvo_dequantize(const uint8_t* codes, const uint8_t* scales, const float* tscale,
                    int64_t groups, int64_t rows, int64_t cols, uint16_t* y) {
    int64_t blocks_per_group = rows * cols / 16;
    for (int64_t g = 0; g < groups; ++g) {
        for (int64_t bl = 0; bl < blocks_per_group; ++bl) {
            int64_t b = g * blocks_per_group + bl;
            float d = nvo_e4m3_to_f32(scales[b]) * tscale[g];
            for (int i = 0; i < 16; ++i) {
                uint8_t byte = codes[b * 8 + i / 2];
                uint8_t c = (i & 1) ? (uint8_t)(byte >> 4) : (uint8_t)(byte & 0xF);
                y[b * 16 + i] = nvo_f32_to_bf16_rne(nvo_e2m1_to_f32(c) * d);
            }
        }
    }
}

/* ---- QAD distillation loss (see the header) -------------------------------------------- */

void nvo_qad_kl(const uint16_t* teacher, const uint16_t* student, int64_t rows, int64_t vocab, double tau,
                double grad_scale, double* kl, double* grad) {
    for (int64_t r = 0; r < rows; ++r) {
        const uint16_t* t = teacher + r * vocab;
        const uint16_t* s = student + r * vocab;
        /* log-sum-exp of each row, shifted by its maximum */
        double mt = -INFINITY, ms = -INFINITY;
        for (int64_t v = 0; v < vocab; ++v) {
            double a = nvo_bf16_to_f32(t[v]) / tau, b = nvo_bf16_to_f32(s[v]) / tau;
            if (a > mt) mt = a;
            if (b > ms) ms = b;
        }
        double zt = 0.0, zs = 0.0;
        for (int64_t v = 0; v < vocab; ++v) {
            zt += exp(nvo_bf16_to_f32(t[v]) / tau - mt);
            zs += exp(nvo_bf16_to_f32(s[v]) / tau - ms);
        }
        double lse_t = mt + log(zt), lse_s = ms + log(zs);
        double acc = 0.0;
        for (int64_t v = 0; v < vocab; ++v) {
            double a = nvo_bf16_to_f32(t[v]) / tau, b = nvo_bf16_to_f32(s[v]) / tau;
            double logp = a - lse_t, logq = b - lse_s;
            double p = exp(logp), q = exp(logq);
            acc += p * (logp - logq);
            if (grad) grad[r * vocab + v] = grad_scale * (q - p);
        }
        kl[r] = acc;
    }
}
