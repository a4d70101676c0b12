/*
 * nvfp4_oracle.h — plain, slow CPU oracle for BF16 -> NVFP4 block-scaled quantization
 * (standard "scale-6" NVFP4 and Four Over Six adaptive block scaling).
 *
 * TEST INFRASTRUCTURE ONLY. Nothing on the product path may include, link or call this file:
 * only the test suite, the smoke check and the bench's CPU-baseline leg use it. It shares no
 * code, header, table or constant with the CUDA library.
 *
 * Sources (web pages, cited by title and section):
 *   [FOS]  "Four Over Six: More Accurate NVFP4 Quantization with Adaptive Block Scaling"
 *          (Cook, Guo, Xiao, Lin, Han), gist.science explainer, technical summary:
 *          Problem definition (問題定義), Method › Core mechanism (中核メカニズム),
 *          Method › Adaptive block scaling algorithm (適応的ブロックスケーリングアルゴリズム),
 *          Implementation details (実装詳細).
 *   [QAD]  "Quantization-Aware Distillation for NVFP4 Inference Accuracy Recovery",
 *          gist.science explainer, technical summary §3.3 (NVFP4 block size 16).
 *   [N35]  "NVIDIA、「Nemotron 3.5 Lightning」のNVFP4量子化手法を公開" news article, section on the
 *          two-stage QAD process (the student's forward runs through simulated quantization).
 *
 * Arithmetic: IEEE-754 binary32, round-to-nearest-even for every operation, no fused
 * multiply-add except the explicit fmaf calls (the error x - v*d and the MSE sum),
 * subnormals kept (no FTZ/DAZ).
 * Built with -O2 -fno-fast-math -ffp-contract=off. The narrow formats (E2M1, E4M3, BF16)
 * are converted by exact lattice arithmetic in binary64, written from their definitions.
 *
 * Parity status: every function here is pinned by tests/test_oracle_pins.py (worked examples
 * from the pages, closed forms, exhaustive nearest-value searches, exact-rational brute force,
 * library routines). No function is "parity unpinned".
 */
#ifndef NVFP4_ORACLE_H
#define NVFP4_ORACLE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Modes and rules; the numbers match the public library's enums by value only. */
enum { NVO_SCALE6 = 0, NVO_FOUR_OVER_SIX = 1 };
enum { NVO_RULE_MAXERR = 0, NVO_RULE_MAE = 1, NVO_RULE_MSE = 2 };

/* ---- scalar format conversions ------------------------------------------------------ */

/* BF16 bits -> binary32 (exact). */
float nvo_bf16_to_f32(uint16_t b);
/* binary32 -> BF16 bits, round to nearest, ties to even; overflow rounds to +-inf as IEEE. */
uint16_t nvo_f32_to_bf16_rne(float f);

/* binary32 -> E4M3 (bias 7, 3 mantissa bits, max finite 448, no inf) bits, round to nearest,
 * ties to even, saturating to +-448 ("satfinite"). NaN input is outside the contract. */
uint8_t nvo_f32_to_e4m3_satfinite(float t);
/* E4M3 bits -> binary32 (exact; 0x7F/0xFF are NaN). */
float nvo_e4m3_to_f32(uint8_t s);

/* binary32 -> 4-bit E2M1 code (bit 3 = sign of the input, bits 0-2 = magnitude index into
 * {0, 0.5, 1, 1.5, 2, 3, 4, 6}), round to nearest, ties to even, saturating to +-6.
 * The sign bit copies the input's sign bit, so inputs in (-0.25, -0] give code 0x8. */
uint8_t nvo_f32_to_e2m1_satfinite(float y);
/* 4-bit E2M1 code -> binary32 (exact). */
float nvo_e2m1_to_f32(uint8_t c);

/* Element-wise array versions of the conversions above (for exhaustive comparisons). */
void nvo_f32_to_e2m1_array(const float* in, uint8_t* out, int64_t n);
void nvo_f32_to_e4m3_array(const float* in, uint8_t* out, int64_t n);
void nvo_f32_to_bf16_array(const float* in, uint16_t* out, int64_t n);

/* ---- one 16-element block, one candidate ---------------------------------------------- */

typedef struct {
    float    beta;      /* K * alpha (rounded once)                                     */
    float    t;         /* block max / beta (rounded once), 0 when beta == 0            */
    uint8_t  s;         /* E4M3 block scale bits                                        */
    float    d;         /* decode scale f32(s) * alpha (rounded once)                   */
    float    r;         /* encode factor: 0 if d == 0, else min(1/d, FLT_MAX)            */
    uint8_t  code[16];  /* E2M1 codes of x_i * r                                        */
    float    q[16];     /* dequantized values v(code_i) * d (rounded once)              */
    float    e[16];     /* errors x_i - v(code_i) * d (exact difference, rounded once)  */
    float    err;       /* the rule's error: max|e|, sum|e| or sum e^2 (see below)       */
} nvo_candidate;

/* Quantize one block of 16 binary32 values (each exactly a BF16 value) with target block
 * maximum K (6 or 4) under tensor scale alpha, and score it with `rule`. */
void nvo_block_candidate(const float x[16], float alpha, float K, int rule, nvo_candidate* out);

/* ---- whole tensors ------------------------------------------------------------------ */

/* amax[g] = max |x| over group g of a [groups, rows, cols] BF16 tensor (exact). */
void nvo_amax(const uint16_t* x, int64_t groups, int64_t rows, int64_t cols, float* amax);

/* alpha = amax / (6 * M), M = 448 (scale-6) or 256 (Four Over Six). */
float nvo_tensor_scale(float amax, int mode);

/* Quantize a [groups, rows, cols] BF16 tensor (cols % 16 == 0) given per-group amax.
 * Outputs (each may be NULL to skip it):
 *   codes  [groups*rows*cols/2]  element 2j in the low nibble, 2j+1 in the high nibble
 *   scales [groups*rows*cols/16] E4M3 bits, row-major
 *   tscale [groups]              alpha
 *   choice [ceil(nblocks/8)]     bit b (LSB-first) set iff block b chose target max 4;
 *                                all zero in scale-6 mode
 *   fq     [groups*rows*cols]    BF16 bits of the chosen candidate's dequantized values */
void nvo_quantize(const uint16_t* x, int64_t groups, int64_t rows, int64_t cols,
                  const float* amax, int mode, int rule,
                  uint8_t* codes, uint8_t* scales, float* tscale, uint8_t* choice, uint16_t* fq);

/* Same, with the FP8 maximum M and the candidate set given explicitly: cand_mask bit 0 =
 * target max 6, bit 1 = target max 4 (at least one bit). Exposed for the special-case pins. */
void nvo_quantize_ex(const uint16_t* x, int64_t groups, int64_t rows, int64_t cols,
                     const float* amax, float fp8_max, int cand_mask, int rule,
                     uint8_t* codes, uint8_t* scales, float* tscale, uint8_t* choice, uint16_t* fq);

/* y = bf16_rne(v(code) * (f32(scale) * alpha)), per element. */
void nvo_dequantize(const uint8_t* codes, const uint8_t* scales, const float* tscale,
                    int64_t groups, int64_t rows, int64_t cols, uint16_t* y);

/* ---- QAD distillation loss ---------------------------------------------------------------
 * "Quantization-Aware Distillation for NVFP4 Inference Accuracy Recovery", technical summary
 * §2 (method): the student (NVFP4, run through simulated quantization) is trained to match
 * the frozen BF16 teacher's output distribution, loss L = D_KL(p_teacher || p_student).
 * Per row r of [rows, vocab] BF16 logits, with temperature tau:
 *   p = softmax(teacher / tau), q = softmax(student / tau),
 *   kl[r] = sum_v p_v (log p_v - log q_v)                      (natural log, binary64)
 *   grad[r, v] = grad_scale * (q_v - p_v)   (d kl / d student_v = (q_v - p_v) / tau; the
 *                                            caller folds 1/tau and any mean into grad_scale)
 * grad may be NULL. Everything is computed in binary64 from the BF16 inputs. */
void nvo_qad_kl(const uint16_t* teacher, const uint16_t* student, int64_t rows, int64_t vocab, double tau,
                double grad_scale, double* kl, double* grad);

#ifdef __cplusplus
}
#endif
#endif
