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
#pragma once

#include <float.h>
#include <stdint.h>

#include "ptx.cuh"

namespace nvfp4 {

constexpr int kThreads = 256;

enum Rule : int { kMaxErr = 0, kMae = 1, kMse = 2 };

// Group lookup: g = b / blocks_per_group. Division by an invariant integer with a
// precomputed multiplier (exact for b < 2^31); the 64-bit quotient is the fallback.
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
    GroupDiv gdiv;
};

struct DequantParams {
    const uint8_t* codes;
    const uint8_t* scales;
    const float* tscale;
    uint16_t* y;
    int64_t nblocks;
    GroupDiv gdiv;
};

// ---- amax --------------------------------------------------------------------------------

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
            uint32_t w = lane < kThreads / 32 ? warp_max[lane] : 0u;
            w = __reduce_max_sync(0xFFFFFFFFu, w);
            if (lane == 0 && w != 0) atomicMax(reinterpret_cast<unsigned int*>(amax + g), w << 16);
        }
        __syncthreads();
    }
}

// ---- quantize / fake-quant -----------------------------------------------------------------

// One candidate (target maximum K) of one block: its codes, their exact values as f16x2
// words, and the rule's error. e_i = x_i - v_i * d is one fused multiply-add (the exact
// difference, rounded once). The two running sums of MAE/MSE are the two lanes of a packed
// pair (even and odd element indices), added at the end.
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
            acc = add2(acc, make_float2(fabsf(e.x), fabsf(e.y)));
        } else {
            emax = fmaxf(emax, fmaxf(fabsf(e.x), fabsf(e.y)));
        }
    }
    return RULE == kMaxErr ? emax : __fadd_rn(acc.x, acc.y);
}

__device__ __forceinline__ float recip_clamped(float d) {
    return d > 0.0f ? fminf(__frcp_rn(d), FLT_MAX) : 0.0f;
}

// FOUR: Four Over Six (two candidates) or scale-6 (one). FQ: write fake-quant BF16 instead of
// codes + scales + tensor scale.
template <bool FOUR, int RULE, bool FQ>
__global__ void __launch_bounds__(kThreads) quantize_kernel(const QuantParams p) {
    constexpr float kSixM = FOUR ? 1536.0f : 2688.0f;   // 6 * 256 or 6 * 448
    const int64_t stride = static_cast<int64_t>(gridDim.x) * kThreads;
    const int64_t nb_pad = (p.nblocks + 31) & ~int64_t(31);
    const int lane = threadIdx.x & 31;
    int64_t b = static_cast<int64_t>(blockIdx.x) * kThreads + threadIdx.x;

    int64_t g_start = 0, g_end = 0;
    float alpha = 0.0f, beta6 = 0.0f, beta4 = 0.0f;

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
            if (b >= g_end) {   // entering a new group: its tensor scale and the two betas
                const int64_t g = p.gdiv(b);
                g_start = g * p.gdiv.bpg;
                g_end = g_start + p.gdiv.bpg;
                alpha = __fdiv_rn(__ldg(p.amax + g), kSixM);
                beta6 = __fmul_rn(6.0f, alpha);
                beta4 = __fmul_rn(4.0f, alpha);
                if (!FQ && b == g_start) p.tscale[g] = alpha;
            }
            float2 x[8];
            float m = 0.0f;
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                x[j] = unpack_bf16x2(cur[j]);
                m = fmaxf(m, fmaxf(fabsf(x[j].x), fabsf(x[j].y)));
            }
            // block scales of both candidates with one paired E4M3 conversion
            const float t6 = beta6 > 0.0f ? __fdiv_rn(m, beta6) : 0.0f;
            const float t4 = FOUR ? (beta4 > 0.0f ? __fdiv_rn(m, beta4) : 0.0f) : 0.0f;
            const uint32_t s2 = e4m3x2(t6, t4);
            const float2 sf = e4m3x2_to_float2(s2);
            const float d6 = __fmul_rn(sf.x, alpha);
            uint32_t c6lo, c6hi, h[8];
            const float err6 = candidate<RULE>(x, recip_clamped(d6), d6, c6lo, c6hi, h);
            uint32_t clo = c6lo, chi = c6hi, s = s2 & 0xFFu;
            float dsel = d6;
            if (FOUR) {
                const float d4 = __fmul_rn(sf.y, alpha);
                uint32_t c4lo, c4hi, h4[8];
                const float err4 = candidate<RULE>(x, recip_clamped(d4), d4, c4lo, c4hi, h4);
                four = err4 < err6;   // ties keep target 6
                if (four) {
                    clo = c4lo;
                    chi = c4hi;
                    s = s2 >> 8;
                    dsel = d4;
                }
#pragma unroll
                for (int j = 0; j < 8; ++j) h[j] = four ? h4[j] : h[j];
            }
            if (FQ) {   // q = RN(v * d) of the kept candidate, rounded to BF16
                const float2 dd = make_float2(dsel, dsel);
                uint32_t out[8];
#pragma unroll
                for (int j = 0; j < 8; ++j) out[j] = bf16x2(mul2(f16x2_to_float2(h[j]), dd));
                st32(p.y + b * 16, out);
            } else {
                st8(p.codes + b * 8, clo, chi);
                p.scales[b] = static_cast<uint8_t>(s);
            }
        }
        if (p.choice != nullptr) {
            const uint32_t bits = __ballot_sync(0xFFFFFFFFu, four);
            if (lane == 0) {
                const int64_t byte0 = (b - lane) >> 3;   // first block of the warp is a multiple of 32
                if (byte0 + 4 <= p.choice_bytes) {
                    *reinterpret_cast<uint32_t*>(p.choice + byte0) = bits;
                } else {
                    for (int k = 0; byte0 + k < p.choice_bytes; ++k)
                        p.choice[byte0 + k] = static_cast<uint8_t>(bits >> (8 * k));
                }
            }
        }
    }
}

// ---- dequantize ------------------------------------------------------------------------------

__global__ void __launch_bounds__(kThreads) dequantize_kernel(const DequantParams p) {
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
