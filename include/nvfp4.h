/*
 * nvfp4.h — C ABI of libnvfp4.so: BF16 -> NVFP4 block-scaled quantization on NVIDIA B200
 * (sm_100a), with standard "scale-6" blocks and Four Over Six adaptive block scaling; the
 * block-scaled FP4 GEMM on the tensor cores that consumes it (optionally quantizing the
 * activations inside its prologue); and the distillation loss of a QAD student.
 *
 * Sources (web pages, cited by title and section):
 *   [FOS] "Four Over Six: More Accurate NVFP4 Quantization with Adaptive Block Scaling"
 *         (gist.science explainer), technical summary: Problem definition; Method > Core
 *         mechanism; Method > Adaptive block scaling algorithm; Implementation details.
 *   [QAD] "Quantization-Aware Distillation for NVFP4 Inference Accuracy Recovery"
 *         (gist.science explainer), technical summary §3.3: NVFP4 blocks of 16 values.
 *   [N35] "NVIDIA、「Nemotron 3.5 Lightning」のNVFP4量子化手法を公開" (news article), two-stage
 *         QAD section: the student's forward pass runs through simulated quantization.
 *   [MO]  "NVIDIA Model Optimizerを用いたNemotron 3.5 Lightning NVFP4とQADの開発" (blog), NVFP4
 *         and QAD sections.
 *
 * The number format. A tensor x of BF16 values, viewed as [groups, rows, cols] row-major, is
 * cut into blocks of 16 consecutive elements along the last dimension ([QAD] §3.3). Each
 * group g has an FP32 tensor scale alpha_g; each block b has an FP8 E4M3 scale s_b; each
 * element is a 4-bit E2M1 code c (sign bit 3, magnitude index bits 0-2 into the grid
 * {0, 0.5, 1, 1.5, 2, 3, 4, 6}, [FOS] Problem definition). The stored value is
 *     v(c) * s_b * alpha_g.
 *
 * The computation (every operation IEEE binary32, round to nearest even):
 *     alpha  = amax_g / (6 * M),  M = 448 in scale-6 mode, 256 in Four Over Six mode
 *              ([FOS] Implementation details: 256 instead of 448 leaves room for the 1.5x
 *              larger scale of a target-4 block)
 *     for each candidate target maximum K (scale-6 mode: K = 6; Four Over Six: K = 6 and 4,
 *     [FOS] Core mechanism and Adaptive block scaling algorithm: quantize twice):
 *       beta = K * alpha;  t = m_b / beta (0 if beta <= 0), m_b = max |x| over the block
 *       s    = E4M3(t), round to nearest even, saturating at 448
 *       d    = f32(s) * alpha;  r = (d > 0) ? min(1 / d, FLT_MAX) : 0
 *       c_i  = E2M1(x_i * r), round to nearest even, saturating at 6, sign kept
 *       q_i  = v(c_i) * d;  e_i = x_i - v(c_i) * d, the exact difference rounded once
 *              (a fused multiply-add): the error against the original values
 *       err  = MAXERR: max |e_i|;  MAE: S(|e_i|);  MSE: S(e_i^2) with fused multiply-add,
 *              where S sums even-indexed and odd-indexed terms in two running sums (each in
 *              increasing index order, starting from +0) and then adds the two
 *     Four Over Six keeps target 4 iff err_4 < err_6 (ties keep 6, the standard format),
 *     under one of the three rules of [FOS] Adaptive block scaling algorithm.
 * Results are bit-identical to the CPU oracle that ships with the tests.
 *
 * Conventions for every entry point
 *   - All tensor pointers are DEVICE pointers owned by the caller. The library allocates no
 *     memory and never synchronizes the host: work is enqueued on `stream` (0 = the legacy
 *     default stream) and completes in stream order. Its only state between calls is a
 *     per-device cache of device attributes (SM count, occupancies, the symbol address below,
 *     the driver's tensor-map encoder, which kernels have had their dynamic shared-memory
 *     limit raised for the 64 KiB decode table) and one static device word per device: the grid-wide
 *     barrier counter of nvfp4_amax_quantize / nvfp4_amax_fakequant calls made without a
 *     workspace.
 *   - Shapes: groups >= 1, rows >= 0, cols >= 0 with cols % 16 == 0. An empty tensor
 *     (rows == 0 or cols == 0) is valid; each function states what it writes for one.
 *   - Alignment: BF16 tensors (x, y) 32 bytes, codes 8 bytes, choice/amax/tscale 4 bytes.
 *     Memory from cudaMalloc or torch satisfies all of these.
 *   - Inputs must be finite and amax values finite and >= 0; NaN/Inf inputs do not fault but
 *     give unspecified outputs. Output buffers must not overlap inputs or each other.
 *   - Errors: argument errors are detected on the host and returned before anything is
 *     enqueued (no output is touched). A launch failure returns NVFP4_ERR_CUDA. Kernels
 *     contain no device-side assert or trap. The only waits are the GEMM's mbarrier waits on
 *     its own copies and tensor-core work, and the grid-wide barrier of the one-launch amax +
 *     quantize kernel (every CTA resident by a cooperative launch). Each is bounded (about two
 *     seconds) and reports a timeout through the caller's status word.
 *   - Buffers must live on the device that is current for the calling thread.
 */
#ifndef NVFP4_H
#define NVFP4_H

#include <stdint.h>
#include <cuda_runtime_api.h>

#if defined(__GNUC__)
#define NVFP4_API __attribute__((visibility("default")))
#else
#define NVFP4_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    NVFP4_OK = 0,
    NVFP4_ERR_NULL = 1,    /* a required pointer is NULL                                 */
    NVFP4_ERR_SHAPE = 2,   /* groups < 1, negative rows/cols, cols % 16 != 0, or overflow */
    NVFP4_ERR_ALIGN = 3,   /* a pointer violates the alignment rule above                 */
    NVFP4_ERR_MODE = 4,    /* unknown nvfp4_mode                                          */
    NVFP4_ERR_RULE = 5,    /* unknown nvfp4_rule (checked in Four Over Six mode only)     */
    NVFP4_ERR_CUDA = 6,    /* the CUDA runtime reported an error while enqueuing          */
    NVFP4_ERR_VALUE = 7    /* a scalar argument is out of range (nvfp4_qad_kl)            */
} nvfp4_status;

/* Block-scale selection ([FOS] Problem definition; Core mechanism). */
typedef enum {
    NVFP4_SCALE6 = 0,          /* standard NVFP4: every block's maximum maps to 6, M = 448 */
    NVFP4_FOUR_OVER_SIX = 1    /* per block, the better of max 6 and max 4, M = 256        */
} nvfp4_mode;

/* Error rule for Four Over Six ([FOS] Adaptive block scaling algorithm). */
typedef enum {
    NVFP4_RULE_MAXERR = 0,     /* smaller maximum absolute error                           */
    NVFP4_RULE_MAE = 1,        /* smaller mean absolute error                              */
    NVFP4_RULE_MSE = 2         /* smaller mean squared error                               */
} nvfp4_rule;

/* Per-group absolute maximum (the input of the global tensor scale, [FOS] Implementation
 * details). amax[g] = max |x| over group g, exactly (a BF16 value as binary32).
 *   x     [groups, rows, cols] BF16 bits, 32-byte aligned          (in)
 *   amax  [groups] float                                            (out)
 * Enqueues a zero-fill of amax followed by one reduction kernel. An empty tensor writes
 * amax = 0 for every group. */
NVFP4_API nvfp4_status nvfp4_amax(const uint16_t* x, int64_t groups, int64_t rows, int64_t cols,
                        float* amax, cudaStream_t stream);

/* Quantize to NVFP4 ([FOS] Problem definition, Core mechanism, Adaptive block scaling
 * algorithm, Implementation details). One kernel, one pass over x.
 *   x       [groups, rows, cols] BF16 bits, 32-byte aligned                        (in)
 *   amax    [groups] float, e.g. from nvfp4_amax, or a calibrated static value:
 *           a value below the true maximum saturates the largest blocks              (in)
 *   mode    NVFP4_SCALE6 or NVFP4_FOUR_OVER_SIX
 *   rule    error rule; ignored (not validated) in scale-6 mode
 *   codes   [groups*rows*cols/2] bytes: element 2j in the low nibble of byte j,
 *           element 2j+1 in the high nibble, 8-byte aligned                          (out)
 *   scales  [groups*rows*cols/16] E4M3 bytes, one per block, row-major              (out)
 *   tscale  [groups] float alpha_g                                                  (out)
 *   choice  NULL, or [ceil(groups*rows*cols/16 / 8)] bytes, 4-byte aligned: bit b%8 of
 *           byte b/8 set iff block b (flat index) kept target 4; all zero in scale-6 (out)
 * An empty tensor writes tscale[g] = alpha of amax[g] for every group (nothing else). */
NVFP4_API nvfp4_status nvfp4_quantize(const uint16_t* x, int64_t groups, int64_t rows, int64_t cols,
                            const float* amax, nvfp4_mode mode, nvfp4_rule rule,
                            uint8_t* codes, uint8_t* scales, float* tscale, uint8_t* choice,
                            cudaStream_t stream);

/* Dequantize NVFP4 to BF16: y_i = bf16_rne(v(c_i) * (f32(s_b) * alpha_g)), the values the
 * stored tensor represents ([FOS] Problem definition; block and tensor scales of
 * Implementation details).
 *   codes, scales, tscale as written by nvfp4_quantize                              (in)
 *   y       [groups, rows, cols] BF16 bits, 32-byte aligned                          (out)
 * An empty tensor does nothing. */
NVFP4_API nvfp4_status nvfp4_dequantize(const uint8_t* codes, const uint8_t* scales, const float* tscale,
                              int64_t groups, int64_t rows, int64_t cols, uint16_t* y,
                              cudaStream_t stream);

/* Fake quantization (quantize then dequantize in one pass): the simulated-quantization
 * forward of a QAD student ([N35] two-stage QAD section). Bit-identical to
 * nvfp4_quantize followed by nvfp4_dequantize, without materialising the codes.
 *   x, amax, mode, rule as for nvfp4_quantize                                         (in)
 *   y       [groups, rows, cols] BF16 bits, 32-byte aligned                           (out)
 *   choice  NULL or the choice bitmap as for nvfp4_quantize                           (out)
 * An empty tensor does nothing. */
NVFP4_API nvfp4_status nvfp4_fakequant(const uint16_t* x, int64_t groups, int64_t rows, int64_t cols,
                             const float* amax, nvfp4_mode mode, nvfp4_rule rule,
                             uint16_t* y, uint8_t* choice, cudaStream_t stream);

/* Bit set in a quantizer's status word when the grid-wide wait of nvfp4_amax_quantize or
 * nvfp4_amax_fakequant timed out (about two seconds) in at least one CTA. The outputs other
 * than amax are then undefined: a CTA whose wait ran out writes nothing, but CTAs that saw
 * the last arrival before their own limit go on and write their tiles, so the outputs may be
 * partly written. */
#define NVFP4_QUANT_TIMEOUT 2u

/* nvfp4_amax followed by nvfp4_quantize in one launch, usable without any allocation. The
 * pages have no counterpart for this entry point: it computes exactly what nvfp4_amax and
 * nvfp4_quantize compute (outputs bit-identical to the two calls) and exists for callers that
 * want one launch, or that cannot allocate device memory.
 * Every CTA reduces max |x| over exactly the tiles it then quantizes, all CTAs meet at a
 * grid-wide barrier (a cooperative launch keeps them resident), and the quantization re-reads
 * the tiles, from L2 when the tensor fits there (126 MB). The barrier needs one 32-bit counter
 * of scratch memory, whatever the tensor's shape.
 *   x, groups, rows, cols, mode, rule, codes, scales, tscale, choice as nvfp4_quantize (in/out)
 *   amax       [groups] float, 4-byte aligned: max |x| per group, written here          (out)
 *   workspace  NULL, or one 4-byte-aligned device word (the counter), zero-filled by the
 *              call in stream order before the launch. With NULL the call allocates nothing:
 *              it uses a static device word of the library (one per device that loads the
 *              library, held until the process exits), for callers that cannot call
 *              cudaMalloc: code running while a CUDA graph is being captured in the global
 *              capture mode (where cudaMalloc is not allowed), serving runtimes that reserve
 *              all device memory for their own pool up front, and plain C callers handed
 *              device buffers with no allocator of their own. The first NULL-workspace call on
 *              a device looks the word's device address up (cudaGetSymbolAddress, with that
 *              device current) and caches it, so make that first call before any stream
 *              capture. Every NULL-workspace call on a device shares the word (the call
 *              zero-fills it first): such calls must not overlap on the GPU (different
 *              streams), or their barriers race; calls with their own workspaces may overlap.
 *              No shape is refused for lack of scratch: one word is all any call needs.
 *                                                                                (scratch)
 *   status     NULL, or a device word; NVFP4_QUANT_TIMEOUT is or-ed in on a timed-out
 *              grid-wide wait                                                        (in/out)
 * Group layouts the grouped quantizer does not take (several groups whose block count is not
 * a multiple of 32), empty tensors, and devices that refuse the cooperative launch (the grid
 * cannot be resident at once) run as the two separate launches (the counter is then not
 * used). Errors as nvfp4_quantize; NVFP4_ERR_CUDA also when the static
 * word's address cannot be obtained. */
NVFP4_API nvfp4_status nvfp4_amax_quantize(const uint16_t* x, int64_t groups, int64_t rows, int64_t cols,
                                           nvfp4_mode mode, nvfp4_rule rule, float* amax, uint8_t* codes,
                                           uint8_t* scales, float* tscale, uint8_t* choice, uint32_t* workspace,
                                           uint32_t* status, cudaStream_t stream);

/* nvfp4_amax followed by nvfp4_fakequant in one launch, as nvfp4_amax_quantize.
 *   y  [groups, rows, cols] BF16 bits, 32-byte aligned                                  (out) */
NVFP4_API nvfp4_status nvfp4_amax_fakequant(const uint16_t* x, int64_t groups, int64_t rows, int64_t cols,
                                            nvfp4_mode mode, nvfp4_rule rule, float* amax, uint16_t* y,
                                            uint8_t* choice, uint32_t* workspace, uint32_t* status,
                                            cudaStream_t stream);

/* Quantize a [rows, cols] BF16 matrix for a Blackwell block-scaled FP4 tensor-core GEMM, in
 * which it is the K-major operand (cols = K). NVFP4 weights and activations are run on
 * Blackwell's native FP4 tensor cores ("NVIDIA Model Optimizerを用いたNemotron 3.5 Lightning
 * NVFP4とQADの開発", section on Nemotron 3.5 Lightning and NVFP4; "Nemotron-3 Nano NVFP4" blog
 * §2). Same arithmetic, codes, tensor scale and choice bits as nvfp4_quantize with one group;
 * only the scale layout differs: the scales of row r, block column c (c = k / 16) are stored
 * in tiles of 128 rows x 4 block columns, 512 bytes each, tile (r / 128, c / 4) at byte
 * ((r / 128) * ceil(cols / 64) + c / 4) * 512, and inside the tile at byte
 * (r % 32) * 16 + ((r % 128) / 32) * 4 + c % 4 (the tiled 1-D block-scaling layout of cuBLASLt).
 *   scales  [roundup(rows, 128) * roundup(cols / 16, 4)] bytes; the padding is zero-filled
 *           (one cudaMemsetAsync before the kernel)                                    (out)
 * rows * cols / 16 must be below 2^30 (else NVFP4_ERR_SHAPE). The library has no counterpart
 * on the pages for the layout itself; it is the operand format of the FP4 GEMMs they run. */
NVFP4_API nvfp4_status nvfp4_quantize_gemm(const uint16_t* x, int64_t rows, int64_t cols, const float* amax,
                                           nvfp4_mode mode, nvfp4_rule rule, uint8_t* codes, uint8_t* scales,
                                           float* tscale, uint8_t* choice, cudaStream_t stream);

/* Bit set in a GEMM's status word when one of the kernel's bounded waits for the tensor core
 * timed out (about two seconds); the kernel then stops, lets the copies it already issued land
 * (again bounded), frees its tensor memory and leaves y partly written. */
#define NVFP4_GEMM_TIMEOUT 1u

/* Block-scaled FP4 GEMM on the 5th-generation tensor cores (tcgen05, kind::mxf4nvf4 with
 * 16-element E4M3 scale blocks): y[m, n] = alpha_x * alpha_w * sum_k Xq[m, k] * Wq[n, k], FP32,
 * row-major. NVFP4 operands run on Blackwell's FP4 tensor cores ("Four Over Six",
 * Implementation details; "NVIDIA Model Optimizerを用いたNemotron 3.5 Lightning NVFP4とQADの開発",
 * NVFP4 section). Both operands are K-major NVFP4 as written by nvfp4_quantize_gemm:
 *   x_codes [m, k/2], x_scales tiled, x_tscale [1] alpha_x      (in, device)
 *   w_codes [n, k/2], w_scales tiled, w_tscale [1] alpha_w      (in, device)
 *   y       [m, n] FP32                                          (out, device)
 *   status  nullable device word; NVFP4_GEMM_TIMEOUT is or-ed in on a timed-out wait (in/out)
 * m >= 0 is any row count, n a multiple of 128 and k of 256 (else NVFP4_ERR_SHAPE); codes and
 * scales 16-byte aligned, y 32-byte aligned; the tensor-map encoder of the driver must be available (else
 * NVFP4_ERR_CUDA). The accumulation is FP32 inside the tensor core, so y agrees
 * with the exact product to within FP32 accumulation error, not bit for bit. Shapes whose m
 * and n are multiples of 256 run on clusters of two CTAs (tcgen05 cta_group::2, one 256 x 256
 * output tile per pair, bit-identical to the one-CTA kernel), or on one CTA per tile when
 * the device refuses the cluster launch. */
NVFP4_API nvfp4_status nvfp4_gemm(const uint8_t* x_codes, const uint8_t* x_scales, const float* x_tscale,
                                  const uint8_t* w_codes, const uint8_t* w_scales, const float* w_tscale,
                                  int64_t m, int64_t n, int64_t k, float* y, uint32_t* status,
                                  cudaStream_t stream);

/* The same GEMM with a BF16 result and, fused into its epilogue, the absolute maximum of that
 * result: the tensor amax from which the next quantization of y derives its FP32 tensor scale
 * ("Four Over Six", Implementation details), so that quantizing y takes one pass over it and
 * no nvfp4_amax read (the reproducible workflow lets the user choose dynamic or static scales:
 * "NVIDIA、「Nemotron 3.5 Lightning」のNVFP4量子化手法を公開", section on the released workflow).
 *   y       [m, n] BF16 bits, y[i, j] = BF16 round-to-nearest-even of the binary32 value
 *           nvfp4_gemm writes at [i, j]; 32-byte aligned                          (out, device)
 *   y_amax  NULL, or [1] float: max |y| over the BF16 values written, exactly (equal to
 *           nvfp4_amax of y; NaN if a y is NaN); 4-byte aligned; zero-filled first in stream
 *           order (cudaMemsetAsync), so an empty product leaves 0                 (out, device)
 * Operands, shapes, status and errors as nvfp4_gemm. */
NVFP4_API nvfp4_status nvfp4_gemm_bf16(const uint8_t* x_codes, const uint8_t* x_scales, const float* x_tscale,
                                       const uint8_t* w_codes, const uint8_t* w_scales, const float* w_tscale,
                                       int64_t m, int64_t n, int64_t k, uint16_t* y, float* y_amax,
                                       uint32_t* status, cudaStream_t stream);

/* The same GEMM with the activation operand quantized inside the kernel's prologue from BF16
 * x [m, k] (32-byte aligned) with its amax x_amax [1] (device), in `mode` under `rule`,
 * exactly as nvfp4_quantize_gemm would quantize it (the pages apply Four Over Six to the
 * activations: "Four Over Six", Results). y equals nvfp4_gemm on nvfp4_quantize_gemm's
 * output bit for bit. */
NVFP4_API nvfp4_status nvfp4_gemm_quantize_x(const uint16_t* x, const float* x_amax, nvfp4_mode mode,
                                             nvfp4_rule rule, const uint8_t* w_codes, const uint8_t* w_scales,
                                             const float* w_tscale, int64_t m, int64_t n, int64_t k, float* y,
                                             uint32_t* status, cudaStream_t stream);

/* Distillation loss of quantization-aware distillation ("Quantization-Aware Distillation for
 * NVFP4 Inference Accuracy Recovery", technical summary §2: the NVFP4 student, whose forward
 * runs through simulated quantization (nvfp4_fakequant), is trained against the frozen BF16
 * teacher with L = D_KL(p_teacher || p_student)). For every row r of [rows, vocab] logits:
 *   p = softmax(teacher[r] / tau), q = softmax(student[r] / tau)
 *   kl[r]      = sum_v p_v (ln p_v - ln q_v)                    (nats)
 *   grad[r, v] = BF16(grad_scale * (q_v - p_v))   (d kl[r] / d student[r, v] = (q_v - p_v) / tau:
 *                pass grad_scale = 1 / (tau * rows) for the gradient of the mean loss)
 *   teacher, student  [rows, vocab] BF16 bits, 2-byte aligned (16-byte aligned rows with
 *                     vocab % 8 == 0 take the vectorised path)                     (in)
 *   kl                [rows] float, 4-byte aligned                                (out)
 *   grad              NULL, or [rows, vocab] BF16 bits, 2-byte aligned            (out)
 * Arithmetic in binary32 with an online (single read) softmax per row and the hardware base-2
 * exponential; the results agree with the binary64 definition to about 1e-6 of the loss's
 * magnitude (tests/test_gpu_5_qad_kl.py states the bounds). tau must be finite and > 0,
 * grad_scale finite (else NVFP4_ERR_VALUE); vocab >= 1; logits must be finite. rows == 0 does
 * nothing. One kernel; a second read of each row when grad is requested. */
NVFP4_API nvfp4_status nvfp4_qad_kl(const uint16_t* teacher, const uint16_t* student, int64_t rows, int64_t vocab,
                                    float tau, float grad_scale, float* kl, uint16_t* grad, cudaStream_t stream);

/* Static description of a status code (never NULL). */
NVFP4_API const char* nvfp4_status_string(nvfp4_status status);

/* Library version: major * 10000 + minor * 100 + patch. */
NVFP4_API int nvfp4_version(void);

#ifdef __cplusplus
}
#endif
#endif /* NVFP4_H */
