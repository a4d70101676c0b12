// qad_kl.cu — fused distillation loss of quantization-aware distillation on sm_100a.
//
// "Quantization-Aware Distillation for NVFP4 Inference Accuracy Recovery", technical summary
// §2: the NVFP4 student (whose forward runs through simulated quantization, i.e. the
// fake-quant output of this library) is trained against the frozen BF16 teacher with
// L = D_KL(p_teacher || p_student) over the output vocabulary.
//
// Per row (one token), with t = teacher / tau and s = student / tau in base-2 log units
// (t2 = t * log2(e)):
//   pass 1 (online, one read of both rows): running maxima mT, mS, normalisers
//     ZT = sum 2^(t2 - mT), ZS = sum 2^(s2 - mS) and AT = sum 2^(t2 - mT) * (t2 - s2);
//     KL = ln2 * (AT / ZT - (mT + log2 ZT) + (mS + log2 ZS))
//   pass 2 (optional): grad_v = grad_scale * (q_v - p_v), p_v = 2^(t2 - lseT2), q_v likewise,
//     stored as BF16.
// One CTA per row; threads stride over the row with 16-byte loads (8 logits) when the vocab
// is a multiple of 8, else element by element.
#include <cuda_runtime.h>
#include <float.h>
#include <stdint.h>

#include "../../include/nvfp4.h"

namespace {

constexpr int kKlThreads = 256;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kNone = -FLT_MAX;      // "no element yet": 2^(kNone - m) == 0 for any finite m

__device__ __forceinline__ float ex2(float x) {
    float r;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
    return r;
}

// Running softmax statistics of a row segment.
struct Stats {
    float mt, zt, at, ms, zs;
};

__device__ __forceinline__ void add_logit(Stats& st, float t2, float s2) {
    if (t2 > st.mt) {                      // rescale to the new teacher maximum
        const float c = ex2(st.mt - t2);
        st.zt *= c;
        st.at *= c;
        st.mt = t2;
    }
    if (s2 > st.ms) {
        st.zs *= ex2(st.ms - s2);
        st.ms = s2;
    }
    const float et = ex2(t2 - st.mt);
    st.zt += et;
    st.at = fmaf(et, t2 - s2, st.at);
    st.zs += ex2(s2 - st.ms);
}

__device__ __forceinline__ Stats merge(const Stats& a, const Stats& b) {
    Stats r;
    r.mt = fmaxf(a.mt, b.mt);
    const float ca = ex2(a.mt - r.mt), cb = ex2(b.mt - r.mt);
    r.zt = a.zt * ca + b.zt * cb;
    r.at = a.at * ca + b.at * cb;
    r.ms = fmaxf(a.ms, b.ms);
    r.zs = a.zs * ex2(a.ms - r.ms) + b.zs * ex2(b.ms - r.ms);
    return r;
}

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

__device__ __forceinline__ uint16_t to_bf16(float f) {
    uint16_t r;
    asm("cvt.rn.bf16.f32 %0, %1;" : "=h"(r) : "f"(f));
    return r;
}

__device__ __forceinline__ uint32_t to_bf16x2(float lo, float hi) {
    uint32_t r;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}

__device__ __forceinline__ uint4 ld16(const void* p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.b32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

}  // namespace

namespace {

// Eight teacher and student logits (one 16-byte load of each): one rescale per row segment
// per eight logits, then the eight terms.
__device__ __forceinline__ void add8(Stats& st, const uint4& a, const uint4& b, float scale2) {
    const uint32_t wa[4] = {a.x, a.y, a.z, a.w}, wb[4] = {b.x, b.y, b.z, b.w};
    float t2[8], s2[8];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        t2[2 * k] = bf16_lo(wa[k]) * scale2;
        t2[2 * k + 1] = bf16_hi(wa[k]) * scale2;
        s2[2 * k] = bf16_lo(wb[k]) * scale2;
        s2[2 * k + 1] = bf16_hi(wb[k]) * scale2;
    }
    float mt = st.mt, ms = st.ms;
#pragma unroll
    for (int k = 0; k < 8; ++k) {
        mt = fmaxf(mt, t2[k]);
        ms = fmaxf(ms, s2[k]);
    }
    const float ct = ex2(st.mt - mt), cs = ex2(st.ms - ms);
    float zt = st.zt * ct, at = st.at * ct, zs = st.zs * cs;
#pragma unroll
    for (int k = 0; k < 8; ++k) {
        const float et = ex2(t2[k] - mt);
        zt += et;
        at = fmaf(et, t2[k] - s2[k], at);
        zs += ex2(s2[k] - ms);
    }
    st = Stats{mt, zt, at, ms, zs};
}

template <bool VEC, bool GRAD>
__global__ void __launch_bounds__(kKlThreads) qad_kl_kernel(const uint16_t* __restrict__ teacher,
                                                            const uint16_t* __restrict__ student, int64_t rows,
                                                            int64_t vocab, float scale2, float grad_scale,
                                                            float* __restrict__ kl, uint16_t* __restrict__ grad) {
    __shared__ Stats part[kKlThreads / 32];
    __shared__ float lse[2];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    for (int64_t r = blockIdx.x; r < rows; r += gridDim.x) {
        const uint16_t* t = teacher + r * vocab;
        const uint16_t* s = student + r * vocab;
        Stats st{kNone, 0.0f, 0.0f, kNone, 0.0f};
        if (VEC) {
            const int64_t nvec = vocab >> 3;
            for (int64_t i = threadIdx.x; i < nvec; i += kKlThreads) add8(st, ld16(t + i * 8), ld16(s + i * 8), scale2);
        } else {
            for (int64_t i = threadIdx.x; i < vocab; i += kKlThreads)
                add_logit(st, __uint_as_float(uint32_t(t[i]) << 16) * scale2, __uint_as_float(uint32_t(s[i]) << 16) * scale2);
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
            Stats o;
            o.mt = __shfl_xor_sync(0xFFFFFFFFu, st.mt, off);
            o.zt = __shfl_xor_sync(0xFFFFFFFFu, st.zt, off);
            o.at = __shfl_xor_sync(0xFFFFFFFFu, st.at, off);
            o.ms = __shfl_xor_sync(0xFFFFFFFFu, st.ms, off);
            o.zs = __shfl_xor_sync(0xFFFFFFFFu, st.zs, off);
            st = merge(st, o);
        }
        if (lane == 0) part[warp] = st;
        __syncthreads();
        if (threadIdx.x == 0) {
            Stats tot = part[0];
            for (int w = 1; w < kKlThreads / 32; ++w) tot = merge(tot, part[w]);
            const float lt = tot.mt + log2f(tot.zt), ls = tot.ms + log2f(tot.zs);
            kl[r] = kLn2 * (tot.at / tot.zt - lt + ls);
            lse[0] = lt;
            lse[1] = ls;
        }
        __syncthreads();
        if (GRAD) {
            const float lt = lse[0], ls = lse[1];
            uint16_t* g = grad + r * vocab;
            if (VEC) {
                const int64_t nvec = vocab >> 3;
                for (int64_t i = threadIdx.x; i < nvec; i += kKlThreads) {
                    const uint4 a = ld16(t + i * 8), b = ld16(s + i * 8);
                    const uint32_t wa[4] = {a.x, a.y, a.z, a.w}, wb[4] = {b.x, b.y, b.z, b.w};
                    uint32_t o[4];
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        const float g0 = grad_scale * (ex2(fmaf(bf16_lo(wb[k]), scale2, -ls)) -
                                                       ex2(fmaf(bf16_lo(wa[k]), scale2, -lt)));
                        const float g1 = grad_scale * (ex2(fmaf(bf16_hi(wb[k]), scale2, -ls)) -
                                                       ex2(fmaf(bf16_hi(wa[k]), scale2, -lt)));
                        o[k] = to_bf16x2(g0, g1);
                    }
                    asm volatile("st.global.v4.b32 [%0], {%1,%2,%3,%4};" ::"l"(g + i * 8), "r"(o[0]), "r"(o[1]),
                                 "r"(o[2]), "r"(o[3])
                                 : "memory");
                }
            } else {
                for (int64_t i = threadIdx.x; i < vocab; i += kKlThreads) {
                    const float tv = __uint_as_float(uint32_t(t[i]) << 16), sv = __uint_as_float(uint32_t(s[i]) << 16);
                    g[i] = to_bf16(grad_scale * (ex2(fmaf(sv, scale2, -ls)) - ex2(fmaf(tv, scale2, -lt))));
                }
            }
        }
        __syncthreads();   // part[] and lse[] are reused by the next row
    }
}

template <bool VEC, bool GRAD>
nvfp4_status launch_kl(const uint16_t* t, const uint16_t* s, int64_t rows, int64_t vocab, float tau,
                       float grad_scale, float* kl, uint16_t* grad, cudaStream_t stream) {
    const int64_t grid = rows < (int64_t(1) << 20) ? rows : (int64_t(1) << 20);
    qad_kl_kernel<VEC, GRAD><<<static_cast<unsigned>(grid), kKlThreads, 0, stream>>>(t, s, rows, vocab, kLog2e / tau,
                                                                                    grad_scale, kl, grad);
    return cudaGetLastError() == cudaSuccess ? NVFP4_OK : NVFP4_ERR_CUDA;
}

bool aligned_to(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

}  // namespace

extern "C" nvfp4_status nvfp4_qad_kl(const uint16_t* teacher, const uint16_t* student, int64_t rows, int64_t vocab,
                                     float tau, float grad_scale, float* kl, uint16_t* grad, cudaStream_t stream) {
    if (rows < 0 || vocab < 1 || (rows > 0 && vocab > (int64_t(1) << 62) / rows)) return NVFP4_ERR_SHAPE;
    if (!(tau > 0.0f) || !(tau <= FLT_MAX) || !(grad_scale == grad_scale) || grad_scale > FLT_MAX ||
        grad_scale < -FLT_MAX)
        return NVFP4_ERR_VALUE;
    if (rows == 0) return NVFP4_OK;
    if (teacher == nullptr || student == nullptr || kl == nullptr) return NVFP4_ERR_NULL;
    if (!aligned_to(teacher, 2) || !aligned_to(student, 2) || !aligned_to(kl, 4) || (grad && !aligned_to(grad, 2)))
        return NVFP4_ERR_ALIGN;
    const bool vec = vocab % 8 == 0 && aligned_to(teacher, 16) && aligned_to(student, 16) &&
                     (grad == nullptr || aligned_to(grad, 16));
    if (vec) {
        return grad ? launch_kl<true, true>(teacher, student, rows, vocab, tau, grad_scale, kl, grad, stream)
                    : launch_kl<true, false>(teacher, student, rows, vocab, tau, grad_scale, kl, grad, stream);
    }
    return grad ? launch_kl<false, true>(teacher, student, rows, vocab, tau, grad_scale, kl, grad, stream)
                : launch_kl<false, false>(teacher, student, rows, vocab, tau, grad_scale, kl, grad, stream);
}
