// block.cuh — per-block arithmetic of the NVFP4 quantizer (sm_100a), shared by the
// quantizer kernels and the prologue of the block-scaled FP4 GEMM.
//
// Layout in HBM: x is a flat array of 16-element BF16 blocks (32 bytes each); block b of the
// flat index belongs to group b / blocks_per_group. Per block the quantizer writes 8 bytes of
// codes, 1 byte of E4M3 scale and 1 choice bit; the fake-quant variant writes 32 bytes of BF16.
//
// The quantizer is issue-bound, not memory-bound, so the per-block arithmetic is kept small:
//  - block scales without a division: lo = RN(m * RN(RN(1/beta) (1 - 2^-20))) and
//    hi = RN(m * RN(RN(1/beta) (1 + 2^-20))) bracket the exact quotient RN(m/beta), so when
//    E4M3(lo) == E4M3(hi) the scale is proven; otherwise the quotient sits at the E4M3
//    rounding boundary between the two codes, and one comparison of m with the group's
//    threshold for the upper code decides (kernels with a shared-memory table), or one exact
//    fused multiply-add (the generic kernel);
//  - the decode scale d = RN(f32(s) * alpha) and its reciprocal for every E4M3 code s, and the
//    thresholds, come from tables per group in shared memory (kernels whose CTAs work inside
//    one group at a time), or are computed per block (the generic kernel);
//  - packed .f32x2 arithmetic, three-input max, and 32-bit in-group indices.
#pragma once

#include <float.h>
#include <stdint.h>

#include "ptx.cuh"

namespace nvfp4 {

constexpr int kThreads = 256;

enum Rule : int { kMaxErr = 0, kMae = 1, kMse = 2 };

// Group lookup for the generic kernel: g = b / blocks_per_group. Division by an invariant
// integer with a precomputed multiplier (exact for b < 2^31); the 64-bit quotient otherwise.
struct GroupDiv {
    int64_t bpg;          // blocks per group
    uint32_t mul;         // ceil(2^(31 + l) / bpg), l = ceil(log2 bpg)
    uint32_t shift;       // l - 1
    int mode;             // 0: single group, 1: bpg == 1, 2: multiplier, 3: 64-bit divide

    __device__ __forceinline__ int64_t operator()(int64_t b) const {
        switch (mode) {
            case 0: return 0;
            case 1: return b;
            case 2: return static_cast<int64_t>(__umulhi(static_cast<uint32_t>(b), mul) >> shift);
            default: return b / bpg;
        }
    }
};

struct QuantParams {
    uint32_t ident = 0x3210u;   // identity byte selector, passed at run time (e2m1x8_and_decode)
    const uint16_t* x;
    const float* amax;
    uint8_t* codes;      // codes output (quantize) or nullptr (fake-quant)
    uint8_t* scales;
    float* tscale;
    uint8_t* choice;     // nullable
    uint16_t* y;         // fake-quant output or nullptr
    int64_t nblocks;
    int64_t choice_bytes;
    int64_t groups;
    GroupDiv gdiv;
    // tiled scale layout of block-scaled GEMM operands (one group, a [rows, 16 * bpr] matrix):
    // blocks per row, multiply-shift divisor for it (exact below 2^31), 4-column tiles per row
    uint32_t bpr, bpr_mul, bpr_shift, n_ct;
};

struct DequantParams {
    const uint8_t* codes;
    const uint8_t* scales;
    const float* tscale;
    uint16_t* y;
    int64_t nblocks;
    int64_t groups;
    GroupDiv gdiv;
};

// ---- small helpers ------------------------------------------------------------------------------

__device__ __forceinline__ float max3(float a, float b, float c) {
    float r;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}

__device__ __forceinline__ float recip_clamped(float d) {
    return d > 0.0f ? fminf(__frcp_rn(d), FLT_MAX) : 0.0f;
}

// Per-group constants: alpha = amax / (6 M), beta_K = K * alpha, and the bracket factors
// yl_K = RN(RN(1/beta_K) * (1 - 2^-20)), yh_K = RN(RN(1/beta_K) * (1 + 2^-20)) used to bracket
// the block-scale quotients (`fast` when both betas lie in [2^-90, 2^125]: every factor is a
// normal number, and the boundary test of block_scales is exact).
struct GroupCtx {
    float alpha, beta6, beta4, yl6, yh6, yl4, yh4;
    bool fast;
    uint32_t ident;   // the kernel argument's identity byte selector (e2m1x8_and_decode)
    uint32_t lane8, dtab;   // decode table (candidate_tab): (lane % 16) * 8 and the table's shared address
};

template <bool FOUR>
__device__ __forceinline__ GroupCtx make_group(float amax, float six_m, uint32_t ident) {
    GroupCtx c;
    c.ident = ident;
    c.alpha = __fdiv_rn(amax, six_m);
    c.beta6 = __fmul_rn(6.0f, c.alpha);
    c.beta4 = __fmul_rn(4.0f, c.alpha);
    const float lo = FOUR ? c.beta4 : c.beta6;
    c.fast = lo >= 0x1p-90f && c.beta6 <= 0x1p125f;
    constexpr float kLo = 1.0f - 0x1p-20f, kHi = 1.0f + 0x1p-20f;
    const float y6 = c.fast ? __frcp_rn(c.beta6) : 0.0f, y4 = c.fast ? __frcp_rn(c.beta4) : 0.0f;
    c.yl6 = __fmul_rn(y6, kLo);
    c.yh6 = __fmul_rn(y6, kHi);
    c.yl4 = __fmul_rn(y4, kLo);
    c.yh4 = __fmul_rn(y4, kHi);
    return c;
}

// The smallest BF16 value m >= 0 with E4M3(RN(m / beta)) >= s, as binary32 (+inf when no
// finite m reaches code s, or beta <= 0; 0 for s = 0). Code s is reached past the E4M3
// rounding boundary M between codes s - 1 and s (their midpoint, at most 5 significant bits):
// with ties going to the even code, E4M3(t) >= s iff t >= M (s even) or t > M (s odd).
// For t = RN(m / beta): t >= M iff m / beta >= H, H the midpoint between M and the binary32
// number below it (a quotient exactly at H rounds to M, whose significand is even), and t > M
// iff m / beta > H', H' the midpoint between M and the binary32 number above it. beta * H is
// exact in binary64 (24 + 26 significant bits), so the threshold is that product rounded up to
// binary32 and then up to BF16 (the smallest BF16 value at or above it), one BF16 step higher
// when the comparison is strict and the product is itself that BF16 value.
__device__ __forceinline__ float e4m3_threshold(uint32_t s, float beta) {
    if (s == 0u) return 0.0f;
    if (s >= 127u || !(beta > 0.0f)) return __int_as_float(0x7F800000);
    const float2 v = e4m3x2_to_float2((s - 1u) | (s << 8));
    const float M = 0.5f * (v.x + v.y);
    const bool odd = s & 1u;
    const float nb = __uint_as_float(__float_as_uint(M) + (odd ? 1u : 0xFFFFFFFFu));
    const double h = 0.5 * (static_cast<double>(M) + static_cast<double>(nb));
    const double V = static_cast<double>(beta) * h;
    const uint32_t b = __float_as_uint(__double2float_ru(V));
    uint32_t t = (b + 0xFFFFu) & 0xFFFF0000u;
    if (odd && static_cast<double>(__uint_as_float(t)) == V) t += 0x10000u;
    return __uint_as_float(t);
}

// E4M3(RN(m / beta)) when the bracket gave adjacent codes s_lo < s_hi (the conversions of lo
// and hi). The E4M3 rounding boundary M between them has at most 5 significant bits and
// hi lies in [M, M (1 + 2^-19)], so M is hi truncated to 5 significant bits. With t =
// RN(m / beta), u = the binary32 gap above M and M even in binary32:
//   s_lo even (ties go down): s_hi iff t > M iff m / beta > M + u / 2,
//   s_lo odd  (ties go up):   s_hi iff t >= M iff m / beta >= M - u / 2
// (M is a power of two only between codes 0 and 1, where the smaller gap below M does not
// matter). Multiplying by beta > 0 compares d = m - beta M with +-beta u / 2. Where
// |m - beta M| <= 2^-18 m, beta M is a 29-bit multiple of 2^(e_beta + e_M - 27) >= 2^-149
// (beta >= 2^-90, M >= 2^-10), so d needs at most 12 bits and the fused multiply-add is
// exact; beta u / 2 = beta 2^(e_M - 24) is exact as well.
__device__ __forceinline__ uint32_t scale_at_boundary(float m, float beta, float hi, uint32_t s_lo, uint32_t s_hi) {
    const float mid = __uint_as_float(__float_as_uint(hi) & 0xFFF80000u);
    const float d = __fmaf_rn(-beta, mid, m);
    const float bu = __fmul_rn(beta, __uint_as_float((__float_as_uint(mid) & 0x7F800000u) - (24u << 23)));
    return (s_lo & 1u) ? (d >= -bu ? s_hi : s_lo) : (d > bu ? s_hi : s_lo);
}

// E4M3(RN(m / beta_6)) in the low byte and E4M3(RN(m / beta_4)) in the high byte.
// lo = RN(m * yl) and hi = RN(m * yh) carry three roundings of at most 2^-24 each on top of
// the factors 1 -+ 2^-20, so lo < m/beta * (1 - 2^-21) < RN(m / beta) < hi whenever the
// products are normal; below 2^-126 every one of them converts to E4M3 zero, and an overflow
// saturates to 448 like the quotient it bounds. E4M3 rounding is monotone, so equal
// conversions of lo and hi are the exact scale; different ones are adjacent codes (E4M3
// boundaries lie at least 2^-4 apart, relatively), and scale_at_boundary decides between
// them: with a threshold table (thr, see fill_scale_tables), the exact code is s_lo plus
// [m >= threshold of s_lo + 1]; without one, scale_at_boundary. For data on a coarse grid,
// such as BF16 block maxima over a tensor scale with a short binary expansion, RN(m / beta)
// falls exactly on an E4M3 boundary for a few percent of the blocks, so most warps meet one:
// the threshold comparison keeps that path to a few instructions. Outside the factors' valid
// range the exact division decides.
template <bool FOUR>
__device__ __forceinline__ uint32_t block_scales(float m, const GroupCtx& c, const float* thr = nullptr) {
    if (c.fast) {
        if (FOUR) {
            const float2 lo = mul2(make_float2(m, m), make_float2(c.yl6, c.yl4));
            const float2 hi = mul2(make_float2(m, m), make_float2(c.yh6, c.yh4));
            const uint32_t wl = e4m3x2(lo.x, lo.y), wh = e4m3x2(hi.x, hi.y);
            if (wl == wh) return wl;
            uint32_t s6 = wl & 0xFFu, s4 = wl >> 8;
            if (thr != nullptr) {
                s6 += m >= thr[s6 + 1u] ? 1u : 0u;
                s4 += m >= thr[128u + s4 + 1u] ? 1u : 0u;
                return s6 | (s4 << 8);
            }
            if (s6 != (wh & 0xFFu)) s6 = scale_at_boundary(m, c.beta6, hi.x, s6, wh & 0xFFu);
            if (s4 != (wh >> 8)) s4 = scale_at_boundary(m, c.beta4, hi.y, s4, wh >> 8);
            return s6 | (s4 << 8);
        } else {
            const float2 b = mul2(make_float2(m, m), make_float2(c.yl6, c.yh6));
            const uint32_t b6 = e4m3x2(b.x, b.y);
            if ((b6 & 0xFFu) == (b6 >> 8)) return b6 & 0xFFu;
            if (thr != nullptr) return (b6 & 0xFFu) + (m >= thr[(b6 & 0xFFu) + 1u] ? 1u : 0u);
            return scale_at_boundary(m, c.beta6, b.y, b6 & 0xFFu, b6 >> 8);
        }
    }
    const float t6 = c.beta6 > 0.0f ? __fdiv_rn(m, c.beta6) : 0.0f;
    const float t4 = FOUR ? (c.beta4 > 0.0f ? __fdiv_rn(m, c.beta4) : 0.0f) : 0.0f;
    return e4m3x2(t6, t4);
}

// Decode scale and encode factor for E4M3 code s: d = RN(f32(s) * alpha), r = min(1/d, FLT_MAX).
__device__ __forceinline__ float2 scale_entry(uint32_t s, float alpha) {
    const float d = __fmul_rn(e4m3x2_to_float2(s).x, alpha);
    return make_float2(d, recip_clamped(d));
}

// Per-group tables in shared memory (256 float2 = 2 KiB), built by the first 256 threads of a
// CTA: entries 0-127, (d, 1/d) by E4M3 code (code 127, not produced, repeats 126); then, as
// floats, the thresholds e4m3_threshold(s, beta_6) for s = 0..127 and (Four Over Six) those
// for beta_4. The thresholds are only built, and only read, when the bracket is in use.
template <bool FOUR>
__device__ __forceinline__ void fill_scale_tables(float2* tab, const GroupCtx& gc, uint32_t tid) {
    if (tid < 128u) {
        tab[tid] = scale_entry(tid == 127u ? 126u : tid, gc.alpha);
    } else if (tid < 256u && gc.fast) {
        float* thr = reinterpret_cast<float*>(tab + 128);
        thr[tid - 128u] = e4m3_threshold(tid - 128u, gc.beta6);
        if (FOUR) thr[tid] = e4m3_threshold(tid - 128u, gc.beta4);
    }
}

// One candidate (target maximum K) of one block: its codes, their exact values as f16x2
// words, and the rule's error. e_i = x_i - v_i * d is one fused multiply-add (the exact
// difference, rounded once). MAE/MSE keep two running sums, one over even and one over odd
// element indices (for MSE the two lanes of a packed pair), added at the end.
template <int RULE>
__device__ __forceinline__ float candidate(const float2 (&x)[8], float r, float d, uint32_t& c_lo,
                                           uint32_t& c_hi, uint32_t (&h)[8], uint32_t ident) {
    const float2 rr = make_float2(r, r), nd = make_float2(-d, -d);
    float2 y[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) y[j] = mul2(x[j], rr);
    c_lo = e2m1x8_and_decode(y[0], y[1], y[2], y[3], h[0], h[1], h[2], h[3], ident);
    c_hi = e2m1x8_and_decode(y[4], y[5], y[6], y[7], h[4], h[5], h[6], h[7], ident);
    float2 acc = make_float2(0.0f, 0.0f);
    float emax = 0.0f;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        const float2 e = fma2(f16x2_to_float2(h[j]), nd, x[j]);
        if (RULE == kMse) {
            acc = fma2(e, e, acc);
        } else if (RULE == kMae) {
            acc.x = __fadd_rn(acc.x, fabsf(e.x));
            acc.y = __fadd_rn(acc.y, fabsf(e.y));
        } else {
            emax = max3(emax, fabsf(e.x), fabsf(e.y));
        }
    }
    return RULE == kMaxErr ? emax : __fadd_rn(acc.x, acc.y);
}

// Decode table in shared memory (dynamic, kDecodeTableBytes = 64 KiB): for every E2M1 byte e
// (two codes) the binary32 values of both codes, in 16 copies at e * 256 + c * 8 (c < 16), so
// that the 16 lanes of a shared-memory phase (lane l reads copy l % 16) each read their own
// bank pair whatever bytes they look up. One byte permutation forms a lookup's address: the
// code byte into bits 8-15 and (lane % 16) * 8 into bits 0-7; the second half of each 256-byte
// row is not used. The values are the hardware decode's (cvt.rn.f16x2.e2m1x2, widened).
constexpr uint32_t kDecodeTableBytes = 65536;

// Work item j (0..255) decodes the four rows 4q .. 4q+3 (q = j / 4) with one conversion word
// and writes copies 4k .. 4k+3 (k = j % 4) of each as two 16-byte stores; odd q writes its two
// stores in the other order, so the 8 lanes of a 16-byte store phase hit distinct banks.
__device__ __forceinline__ void fill_decode_table(float2* dect) {
    float4* t4 = reinterpret_cast<float4*>(dect);   // a row is 16 float4; copies 2i, 2i+1 share one
    for (uint32_t j = threadIdx.x; j < 256u; j += blockDim.x) {
        const uint32_t q = j >> 2, k = j & 3u, o = q & 1u;
        uint32_t h[4];
        e2m1x8_to_f16x2(0x03020100u + q * 0x04040404u, h[0], h[1], h[2], h[3]);
#pragma unroll
        for (int m = 0; m < 4; ++m) {
            const float2 v = f16x2_to_float2(h[m]);
            const float4 vv = make_float4(v.x, v.y, v.x, v.y);
            float4* row = t4 + (4u * q + m) * 16u + 2u * k;
            row[o] = vv;
            row[1u - o] = vv;
        }
    }
}

// candidate() with the code values read from the decode table instead of decoded and widened:
// per pair of elements one byte permutation and one 8-byte shared-memory load replace a decode,
// its byte extraction and two widening additions (about 2 instructions fewer per pair, and
// the ALU and FMA pipes lose work to the load pipe). Same values, same error, bit for bit.
template <int RULE>
__device__ __forceinline__ float candidate_tab(const float2 (&x)[8], float r, float d, uint32_t& c_lo,
                                               uint32_t& c_hi, uint32_t lane8, uint32_t dtab) {
    const float2 rr = make_float2(r, r), nd = make_float2(-d, -d);
    float2 y[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) y[j] = mul2(x[j], rr);
    c_lo = e2m1x8(y[0], y[1], y[2], y[3]);
    c_hi = e2m1x8(y[4], y[5], y[6], y[7]);
    float2 acc = make_float2(0.0f, 0.0f);
    float emax = 0.0f;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        const uint32_t w = j < 4 ? c_lo : c_hi;
        const float2 v = lds_f2(dtab + __byte_perm(w, lane8, 0x5504u | ((j & 3) << 4)));
        const float2 e = fma2(v, nd, x[j]);
        if (RULE == kMse) {
            acc = fma2(e, e, acc);
        } else if (RULE == kMae) {
            acc.x = __fadd_rn(acc.x, fabsf(e.x));
            acc.y = __fadd_rn(acc.y, fabsf(e.y));
        } else {
            emax = max3(emax, fabsf(e.x), fabsf(e.y));
        }
    }
    return RULE == kMaxErr ? emax : __fadd_rn(acc.x, acc.y);
}

// Quantize the block in `w` (eight BF16 pairs) into registers: the kept candidate's codes
// (clo: elements 0-7, chi: 8-15, element 2j in the low nibble), its E4M3 scale s and decode
// scale d, and (FQ) its values as f16x2 words in h. Returns whether target 4 was kept.
// TABLE: d, 1/d and the scale thresholds come from `tab` (fill_scale_tables). DEC: code values
// come from the decode table (gc.dtab; not with FQ, which keeps the decoded words).
template <bool FOUR, int RULE, bool FQ, bool TABLE, bool DEC = false>
__device__ __forceinline__ bool quantize_block_regs(const uint32_t (&w)[8], const GroupCtx& gc, const float2* tab,
                                                    uint32_t& clo, uint32_t& chi, uint32_t& s, float& dsel,
                                                    uint32_t (&h)[8]) {
    float2 x[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) x[j] = unpack_bf16x2(w[j]);
    // max of the 16 |x_i|: a depth-3 tree of 3-input max (the same value as a running max)
    const float m01 = max3(fabsf(x[0].x), fabsf(x[0].y), fabsf(x[1].x));
    const float m02 = max3(fabsf(x[1].y), fabsf(x[2].x), fabsf(x[2].y));
    const float m03 = max3(fabsf(x[3].x), fabsf(x[3].y), fabsf(x[4].x));
    const float m04 = max3(fabsf(x[4].y), fabsf(x[5].x), fabsf(x[5].y));
    const float m05 = max3(fabsf(x[6].x), fabsf(x[6].y), fabsf(x[7].x));
    const float m = fmaxf(max3(m01, m02, m03), max3(m04, m05, fabsf(x[7].y)));
    const uint32_t s2 = block_scales<FOUR>(m, gc, TABLE ? reinterpret_cast<const float*>(tab + 128) : nullptr);
    const uint32_t i6 = __byte_perm(s2, 0u, 0x4440), i4 = __byte_perm(s2, 0u, 0x4441);
    const float2 e6 = TABLE ? tab[i6] : scale_entry(i6, gc.alpha);
    const float err6 = DEC ? candidate_tab<RULE>(x, e6.y, e6.x, clo, chi, gc.lane8, gc.dtab)
                           : candidate<RULE>(x, e6.y, e6.x, clo, chi, h, gc.ident);
    s = i6;
    dsel = e6.x;
    bool four = false;
    if (FOUR) {
        const float2 e4 = TABLE ? tab[i4] : scale_entry(i4, gc.alpha);
        uint32_t c4lo, c4hi, h4[8];
        const float err4 = DEC ? candidate_tab<RULE>(x, e4.y, e4.x, c4lo, c4hi, gc.lane8, gc.dtab)
                               : candidate<RULE>(x, e4.y, e4.x, c4lo, c4hi, h4, gc.ident);
        four = err4 < err6;   // ties keep target 6
        if (four) {
            clo = c4lo;
            chi = c4hi;
            s = i4;
            dsel = e4.x;
        }
        if (FQ) {
#pragma unroll
            for (int j = 0; j < 8; ++j) h[j] = four ? h4[j] : h[j];
        }
    }
    return four;
}

// Quantize the block in `w` and store its codes + scale (or fake-quant BF16); returns whether
// target 4 was kept. ok = false (a lane past the end of the group) computes but stores nothing
// and returns false.
template <bool FOUR, int RULE, bool FQ, bool TABLE, bool DEC = false>
__device__ __forceinline__ bool quantize_block(const uint32_t (&w)[8], const GroupCtx& gc, const float2* tab,
                                               uint8_t* codes8, uint8_t* scale1, uint16_t* y16, bool ok = true) {
    uint32_t clo, chi, s, h[8];
    float dsel;
    const bool four = quantize_block_regs<FOUR, RULE, FQ, TABLE, DEC>(w, gc, tab, clo, chi, s, dsel, h);
    if (FQ) {   // q = RN(v * d) of the kept candidate, rounded to BF16
        const float2 dd = make_float2(dsel, dsel);
        uint32_t out[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) out[j] = bf16x2(mul2(f16x2_to_float2(h[j]), dd));
        if (ok) st32(y16, out);
    } else if (ok) {
        st8(codes8, clo, chi);
        *scale1 = static_cast<uint8_t>(s);
    }
    return four && ok;
}

// Byte offset of local block a's scale in the tiled layout: 128-row x 4-column tiles of 512
// bytes, tile (row / 128, col / 4) at ((row / 128) * n_ct + col / 4) * 512, and inside a tile
// row r, column c at (r % 32) * 16 + (r / 32) * 4 + c.
__device__ __forceinline__ uint32_t tiled_scale_offset(uint32_t a, const QuantParams& p) {
    const uint32_t row = p.bpr == 1u ? a : __umulhi(a, p.bpr_mul) >> p.bpr_shift;
    const uint32_t col = a - row * p.bpr;
    return (((row >> 7) * p.n_ct + (col >> 2)) << 9) + ((row & 31u) << 4) + (((row >> 5) & 3u) << 2) + (col & 3u);
}

// Store one warp's 32 choice bits (the word starting at flat block `first`, a multiple of 32).
__device__ __forceinline__ void store_choice(uint8_t* choice, int64_t choice_bytes, int64_t first, uint32_t bits) {
    const int64_t byte0 = first >> 3;
    if (byte0 + 4 <= choice_bytes) {
        *reinterpret_cast<uint32_t*>(choice + byte0) = bits;
    } else {
        for (int k = 0; byte0 + k < choice_bytes; ++k) choice[byte0 + k] = static_cast<uint8_t>(bits >> (8 * k));
    }
}

}  // namespace nvfp4
