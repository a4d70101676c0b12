// kernels.cuh — sm_100a kernels of the NVFP4 quantizer.
//
// Layout in HBM: x is a flat array of 16-element BF16 blocks (32 bytes each); block b of the
// flat index belongs to group b / blocks_per_group. Per block the quantizer writes 8 bytes of
// codes, 1 byte of E4M3 scale and 1 choice bit; the fake-quant variant writes 32 bytes of BF16.
//
// One thread owns one block at a time: a warp reads 1 KiB of contiguous input per step with
// 32-byte vector loads and writes 256 contiguous bytes of codes, 32 bytes of scales and one
// 32-bit word of choice bits (a warp ballot). Grids are persistent (a multiple of the SM
// count) and each thread prefetches its next block before working on the current one.
//
// The quantizer is issue-bound, not memory-bound, so the per-block arithmetic is kept small:
//  - block scales without a division: t' = m * RN(1/beta) is within a few ulps of the exact
//    quotient RN(m/beta), so when E4M3(t' * (1 - 2^-20)) == E4M3(t' * (1 + 2^-20)) the
//    scale is proven; otherwise (rare) the exact division decides;
//  - the decode scale d = RN(f32(s) * alpha) and its reciprocal for every E4M3 code s come
//    from a 128-entry table per group in shared memory (kernels whose CTAs work inside one
//    group at a time), or are computed per block (the generic kernel);
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
// the block-scale quotients (valid when both betas lie in [2^-125, 2^125], so that every
// factor is a normal number).
struct GroupCtx {
    float alpha, beta6, beta4, yl6, yh6, yl4, yh4;
    bool fast;
};

template <bool FOUR>
__device__ __forceinline__ GroupCtx make_group(float amax, float six_m) {
    GroupCtx c;
    c.alpha = __fdiv_rn(amax, six_m);
    c.beta6 = __fmul_rn(6.0f, c.alpha);
    c.beta4 = __fmul_rn(4.0f, c.alpha);
    const float lo = FOUR ? c.beta4 : c.beta6;
    c.fast = lo >= 0x1p-125f && c.beta6 <= 0x1p125f;
    constexpr float kLo = 1.0f - 0x1p-20f, kHi = 1.0f + 0x1p-20f;
    const float y6 = c.fast ? __frcp_rn(c.beta6) : 0.0f, y4 = c.fast ? __frcp_rn(c.beta4) : 0.0f;
    c.yl6 = __fmul_rn(y6, kLo);
    c.yh6 = __fmul_rn(y6, kHi);
    c.yl4 = __fmul_rn(y4, kLo);
    c.yh4 = __fmul_rn(y4, kHi);
    return c;
}

// E4M3(RN(m / beta_6)) in the low byte and E4M3(RN(m / beta_4)) in the high byte.
// lo = RN(m * yl) and hi = RN(m * yh) carry three roundings of at most 2^-24 each on top of
// the factors 1 -+ 2^-20, so lo < m/beta * (1 - 2^-21) < RN(m / beta) < hi whenever the
// products are normal; below 2^-126 every one of them converts to E4M3 zero, and an overflow
// saturates to 448 like the quotient it bounds. E4M3 rounding is monotone, so equal
// conversions of lo and hi are the exact scale. Near a rounding boundary (about one block in
// 2^15), or outside the factors' valid range, the exact division decides.
template <bool FOUR>
__device__ __forceinline__ uint32_t block_scales(float m, const GroupCtx& c) {
    if (c.fast) {
        if (FOUR) {
            const float2 lo = mul2(make_float2(m, m), make_float2(c.yl6, c.yl4));
            const float2 hi = mul2(make_float2(m, m), make_float2(c.yh6, c.yh4));
            const uint32_t wl = e4m3x2(lo.x, lo.y), wh = e4m3x2(hi.x, hi.y);
            if (wl == wh) return wl;
        } else {
            const float2 b = mul2(make_float2(m, m), make_float2(c.yl6, c.yh6));
            const uint32_t b6 = e4m3x2(b.x, b.y);
            if ((b6 & 0xFFu) == (b6 >> 8)) return b6 & 0xFFu;
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

// One candidate (target maximum K) of one block: its codes, their exact values as f16x2
// words, and the rule's error. e_i = x_i - v_i * d is one fused multiply-add (the exact
// difference, rounded once). MAE/MSE keep two running sums, one over even and one over odd
// element indices (for MSE the two lanes of a packed pair), added at the end.
template <int RULE>
__device__ __forceinline__ float candidate(const float2 (&x)[8], float r, float d, uint32_t& c_lo,
                                           uint32_t& c_hi, uint32_t (&h)[8]) {
    const float2 rr = make_float2(r, r), nd = make_float2(-d, -d);
    float2 y[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) y[j] = mul2(x[j], rr);
    c_lo = e2m1x8_and_decode(y[0], y[1], y[2], y[3], h[0], h[1], h[2], h[3]);
    c_hi = e2m1x8_and_decode(y[4], y[5], y[6], y[7], h[4], h[5], h[6], h[7]);
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

// Quantize the block in `w` (eight BF16 pairs). Stores its codes + scale (or fake-quant
// BF16) and returns whether target 4 was kept. TABLE: d and 1/d come from `tab`. ok = false
// (a lane past the end of the group) computes but stores nothing and returns false.
template <bool FOUR, int RULE, bool FQ, bool TABLE>
__device__ __forceinline__ bool quantize_block(const uint32_t (&w)[8], const GroupCtx& gc, const float2* tab,
                                               uint8_t* codes8, uint8_t* scale1, uint16_t* y16, bool ok = true) {
    float2 x[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) x[j] = unpack_bf16x2(w[j]);
    // max over {0, |x_i|}: depth-3 tree of 3-input max (the same value as a running max)
    const float m01 = max3(0.0f, fabsf(x[0].x), fabsf(x[0].y));
    const float m02 = max3(fabsf(x[1].x), fabsf(x[1].y), fabsf(x[2].x));
    const float m03 = max3(fabsf(x[2].y), fabsf(x[3].x), fabsf(x[3].y));
    const float m04 = max3(fabsf(x[4].x), fabsf(x[4].y), fabsf(x[5].x));
    const float m05 = max3(fabsf(x[5].y), fabsf(x[6].x), fabsf(x[6].y));
    const float m06 = max3(fabsf(x[7].x), fabsf(x[7].y), 0.0f);
    const float m = fmaxf(max3(m01, m02, m03), max3(m04, m05, m06));
    const uint32_t s2 = block_scales<FOUR>(m, gc);
    const uint32_t i6 = __byte_perm(s2, 0u, 0x4440), i4 = __byte_perm(s2, 0u, 0x4441);
    const float2 e6 = TABLE ? tab[i6] : scale_entry(i6, gc.alpha);
    uint32_t clo, chi, h[8];
    const float err6 = candidate<RULE>(x, e6.y, e6.x, clo, chi, h);
    uint32_t s = i6;
    float dsel = e6.x;
    bool four = false;
    if (FOUR) {
        const float2 e4 = TABLE ? tab[i4] : scale_entry(i4, gc.alpha);
        uint32_t c4lo, c4hi, h4[8];
        const float err4 = candidate<RULE>(x, e4.y, e4.x, c4lo, c4hi, h4);
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

// ---- amax --------------------------------------------------------------------------------------

// amax[g] = max |x| over group g. BF16 magnitudes compare like their bit patterns, so the
// reduction runs on (bits & 0x7FFF) as packed unsigned 16-bit pairs; the result's bits
// shifted left by 16 are the binary32 value, and binary32 values >= 0 order like their bits,
// so the per-CTA results combine with an unsigned atomicMax into the zero-filled output.
__global__ void __launch_bounds__(kThreads) amax_kernel(const uint16_t* __restrict__ x, int64_t groups,
                                                        int64_t chunks_per_group, float* __restrict__ amax) {
    __shared__ uint32_t warp_max[kThreads / 32];
    const int64_t stride = static_cast<int64_t>(gridDim.x) * kThreads;
    for (int64_t g = blockIdx.y; g < groups; g += gridDim.y) {
        const uint16_t* base = x + g * chunks_per_group * 16;
        uint32_t m2 = 0;
        int64_t i = static_cast<int64_t>(blockIdx.x) * kThreads + threadIdx.x;
        // four independent 32-byte loads in flight per thread
        for (; i + 3 * stride < chunks_per_group; i += 4 * stride) {
            uint32_t v[4][8];
#pragma unroll
            for (int u = 0; u < 4; ++u) ld32_stream(base + (i + u * stride) * 16, v[u]);
#pragma unroll
            for (int u = 0; u < 4; ++u)
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    uint32_t a = v[u][k] & 0x7FFF7FFFu;
                    asm("max.u16x2 %0, %0, %1;" : "+r"(m2) : "r"(a));
                }
        }
        for (; i < chunks_per_group; i += stride) {
            uint32_t v[8];
            ld32_stream(base + i * 16, v);
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                uint32_t a = v[k] & 0x7FFF7FFFu;
                asm("max.u16x2 %0, %0, %1;" : "+r"(m2) : "r"(a));
            }
        }
        uint32_t m = max(m2 & 0xFFFFu, m2 >> 16);
        m = __reduce_max_sync(0xFFFFFFFFu, m);
        const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
        if (lane == 0) warp_max[warp] = m;
        __syncthreads();
        if (warp == 0) {
            uint32_t v = lane < kThreads / 32 ? warp_max[lane] : 0u;
            v = __reduce_max_sync(0xFFFFFFFFu, v);
            if (lane == 0 && v != 0) atomicMax(reinterpret_cast<unsigned int*>(amax + g), v << 16);
        }
        __syncthreads();
    }
}

// ---- quantize / fake-quant: CTAs inside one group at a time (scale table in shared memory) ------

// Grid: x = CTAs per group, y = groups (looping when there are more than gridDim.y).
// Each warp works on tiles of 64 consecutive blocks of its group: lane t quantizes blocks t and
// t + 32 of the tile, so both 32-byte loads, both code stores and both scale stores of a warp
// are contiguous, and each half-tile's 32 choice bits are one ballot word. The next tile's
// blocks are loaded into registers before the current ones are worked on: in 4/6 mode into a
// second register set (the loop is unrolled twice so the two sets swap roles without copies),
// in scale-6 mode into one set that is copied, which keeps that kernel within 64 registers.
// The last, partial tile runs the same code with its stores predicated off.
// Requires every group to start on a 32-block boundary of the flat index (one group, or
// blocks_per_group % 32 == 0) and blocks_per_group < 2^30.
// SWZ: scales go to the tiled GEMM layout (one group only).
// One warp tile (64 blocks) of one group; lane t works on blocks 64 tile + t and + 32.
template <bool FOUR, int RULE, bool FQ, bool SWZ>
__device__ __forceinline__ void quant_tile(const QuantParams& p, const GroupCtx& gc, const float2* tab,
                                           uint32_t tile, uint32_t lane, uint32_t bpg, uint8_t* cg, uint8_t* sg,
                                           uint16_t* yg, uint32_t* chw, int64_t base,
                                           const uint32_t (&ca)[8], const uint32_t (&cb)[8]) {
    const uint32_t a = (tile << 6) + lane;
    const bool oka = a < bpg, okb = a + 32u < bpg;
    // the second block's addresses are the first one's plus constant offsets (32 blocks)
    uint8_t* c0 = FQ ? nullptr : cg + static_cast<size_t>(a) * 8;
    uint8_t* s0 = FQ ? nullptr : sg + a;
    uint16_t* y0 = FQ ? yg + static_cast<size_t>(a) * 16 : nullptr;
    const bool fa = quantize_block<FOUR, RULE, FQ, true>(ca, gc, tab, c0, SWZ ? p.scales + tiled_scale_offset(a, p) : s0,
                                                         y0, oka);
    const bool fb = quantize_block<FOUR, RULE, FQ, true>(cb, gc, tab, FQ ? nullptr : c0 + 256,
                                                         SWZ ? p.scales + tiled_scale_offset(a + 32u, p) : (FQ ? nullptr : s0 + 32),
                                                         FQ ? y0 + 512 : nullptr, okb);
    if (p.choice != nullptr) {
        const uint32_t bits_a = __ballot_sync(0xFFFFFFFFu, fa);
        const uint32_t bits_b = __ballot_sync(0xFFFFFFFFu, fb);
        const uint32_t w = 2u * tile + lane;
        if (lane < 2u && (w << 5) < bpg) {
            const uint32_t bits = lane ? bits_b : bits_a;
            if ((w << 5) + 32u <= bpg) chw[w] = bits;   // all 32 blocks of the word exist
            else store_choice(p.choice, p.choice_bytes, base + (static_cast<int64_t>(w) << 5), bits);
        }
    }
}

// Load a lane's two blocks of a tile. Lanes past the group's end (bpg >= 1) re-read its last
// block, so every register the tile computes on holds defined data; their stores are off.
__device__ __forceinline__ void load_tile(const uint16_t* xg, uint32_t tile, uint32_t lane, uint32_t bpg,
                                          uint32_t (&ra)[8], uint32_t (&rb)[8]) {
    const uint32_t a = (tile << 6) + lane, last = bpg - 1u;
    ld32_stream(xg + static_cast<size_t>(min(a, last)) * 16, ra);
    ld32_stream(xg + static_cast<size_t>(min(a + 32u, last)) * 16, rb);
}

template <bool FOUR, int RULE, bool FQ, bool SWZ = false>
__global__ void __launch_bounds__(kThreads, FOUR ? 2 : 4) quantize_grouped_kernel(const QuantParams p) {
    constexpr float kSixM = FOUR ? 1536.0f : 2688.0f;   // 6 * 256 or 6 * 448
    __shared__ float2 tab[128];
    const uint32_t lane = threadIdx.x & 31u;
    const uint32_t bpg = static_cast<uint32_t>(p.gdiv.bpg);
    const uint32_t ntiles = (bpg + 63u) >> 6;
    const uint32_t warps = gridDim.x * (kThreads / 32);
    const uint32_t warp0 = blockIdx.x * (kThreads / 32) + (threadIdx.x >> 5);
    for (int64_t g = blockIdx.y; g < p.groups; g += gridDim.y) {
        const GroupCtx gc = make_group<FOUR>(__ldg(p.amax + g), kSixM);
        __syncthreads();                       // the previous group's table is no longer read
        if (threadIdx.x < 128) tab[threadIdx.x] = scale_entry(threadIdx.x == 127 ? 126u : threadIdx.x, gc.alpha);
        if (!FQ && blockIdx.x == 0 && threadIdx.x == 0) p.tscale[g] = gc.alpha;
        __syncthreads();
        const int64_t base = g * static_cast<int64_t>(bpg);
        const uint16_t* xg = p.x + base * 16;
        uint8_t* cg = FQ ? nullptr : p.codes + base * 8;
        uint8_t* sg = FQ ? nullptr : p.scales + base;
        uint16_t* yg = FQ ? p.y + base * 16 : nullptr;
        uint32_t* chw = reinterpret_cast<uint32_t*>(p.choice) + (base >> 5);   // base is a multiple of 32
        uint32_t tile = warp0;
        uint32_t a0[8], a1[8];
        if (tile < ntiles) load_tile(xg, tile, lane, bpg, a0, a1);
        if constexpr (!FOUR) {   // one prefetch buffer: two would not fit the 64-register budget
            for (; tile < ntiles; tile += warps) {
                uint32_t b0[8], b1[8];
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    b0[k] = a0[k];
                    b1[k] = a1[k];
                }
                if (tile + warps < ntiles) load_tile(xg, tile + warps, lane, bpg, a0, a1);
                quant_tile<FOUR, RULE, FQ, SWZ>(p, gc, tab, tile, lane, bpg, cg, sg, yg, chw, base, b0, b1);
            }
        } else {
            uint32_t b0[8], b1[8];
            while (tile < ntiles) {
                uint32_t nt = tile + warps;
                if (nt < ntiles) load_tile(xg, nt, lane, bpg, b0, b1);
                quant_tile<FOUR, RULE, FQ, SWZ>(p, gc, tab, tile, lane, bpg, cg, sg, yg, chw, base, a0, a1);
                tile = nt;
                if (tile >= ntiles) break;
                nt = tile + warps;
                if (nt < ntiles) load_tile(xg, nt, lane, bpg, a0, a1);
                quant_tile<FOUR, RULE, FQ, SWZ>(p, gc, tab, tile, lane, bpg, cg, sg, yg, chw, base, b0, b1);
                tile = nt;
            }
        }
    }
}

// ---- quantize / fake-quant: flat grid over all blocks (any group layout) ------------------------

template <bool FOUR, int RULE, bool FQ>
__global__ void __launch_bounds__(kThreads) quantize_kernel(const QuantParams p) {
    constexpr float kSixM = FOUR ? 1536.0f : 2688.0f;
    const int64_t stride = static_cast<int64_t>(gridDim.x) * kThreads;
    const int64_t nb_pad = (p.nblocks + 31) & ~int64_t(31);
    const int lane = threadIdx.x & 31;
    int64_t b = static_cast<int64_t>(blockIdx.x) * kThreads + threadIdx.x;

    int64_t g_end = 0;
    GroupCtx gc{};

    uint32_t nxt[8];
    if (b < p.nblocks) ld32_stream(p.x + b * 16, nxt);

    for (; b < nb_pad; b += stride) {
        uint32_t cur[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) cur[k] = nxt[k];
        const int64_t bn = b + stride;
        if (bn < p.nblocks) ld32_stream(p.x + bn * 16, nxt);

        bool four = false;
        if (b < p.nblocks) {
            if (b >= g_end) {   // entering a new group
                const int64_t g = p.gdiv(b);
                const int64_t g_start = g * p.gdiv.bpg;
                g_end = g_start + p.gdiv.bpg;
                gc = make_group<FOUR>(__ldg(p.amax + g), kSixM);
                if (!FQ && b == g_start) p.tscale[g] = gc.alpha;
            }
            four = quantize_block<FOUR, RULE, FQ, false>(cur, gc, nullptr, FQ ? nullptr : p.codes + b * 8,
                                                         FQ ? nullptr : p.scales + b, FQ ? p.y + b * 16 : nullptr);
        }
        if (p.choice != nullptr) {
            const uint32_t bits = __ballot_sync(0xFFFFFFFFu, four);
            if (lane == 0) store_choice(p.choice, p.choice_bytes, b - lane, bits);
        }
    }
}

// ---- dequantize ------------------------------------------------------------------------------

__global__ void __launch_bounds__(kThreads, 4) dequantize_kernel(const DequantParams p) {
    const int64_t stride = static_cast<int64_t>(gridDim.x) * kThreads;
    int64_t b = static_cast<int64_t>(blockIdx.x) * kThreads + threadIdx.x;
    int64_t g_end = 0;
    float alpha = 0.0f;
    uint32_t nlo = 0, nhi = 0, ns = 0;
    if (b < p.nblocks) {
        ld8_stream(p.codes + b * 8, nlo, nhi);
        ns = ld1_stream(p.scales + b);
    }
    for (; b < p.nblocks; b += stride) {
        const uint32_t clo = nlo, chi = nhi, s = ns;
        const int64_t bn = b + stride;
        if (bn < p.nblocks) {
            ld8_stream(p.codes + bn * 8, nlo, nhi);
            ns = ld1_stream(p.scales + bn);
        }
        if (b >= g_end) {
            const int64_t g = p.gdiv(b);
            g_end = g * p.gdiv.bpg + p.gdiv.bpg;
            alpha = __ldg(p.tscale + g);
        }
        const float d = __fmul_rn(e4m3x2_to_float2(s).x, alpha);
        const float2 dd = make_float2(d, d);
        uint32_t h[8];
        e2m1x8_to_f16x2(clo, h[0], h[1], h[2], h[3]);
        e2m1x8_to_f16x2(chi, h[4], h[5], h[6], h[7]);
        uint32_t out[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) out[j] = bf16x2(mul2(f16x2_to_float2(h[j]), dd));
        st32(p.y + b * 16, out);
    }
}

}  // namespace nvfp4
