// ptx.cuh — thin inline-PTX wrappers used by the NVFP4 kernels (sm_100a only).
//
// Conversions use the Blackwell cvt family ("Four Over Six ...", Implementation details:
// the kernel is built on cvt instructions): f32 -> E2M1 pairs and f32 -> E4M3 pairs with
// round-to-nearest-even and satfinite, and the exact widening conversions back to f16. f16 and
// BF16 values are widened to binary32 by mixed-precision additions (sm_100), which run on the
// FMA pipes: in the quantizer the ALU pipe is the busier one.
// Arithmetic that decides a code or a choice is IEEE binary32 round-to-nearest; the packed
// .f32x2 forms are lane-wise IEEE (sm_100+), so they give the same bits as scalar code.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

namespace nvfp4 {

// ---- memory ------------------------------------------------------------------------------

// 32-byte streaming load (read-only path, no L1 allocation, 256-byte L2 prefetch).
__device__ __forceinline__ void ld32_stream(const void* p, uint32_t (&v)[8]) {
    asm volatile("ld.global.nc.L1::no_allocate.L2::256B.v8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                 : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]),
                   "=r"(v[7])
                 : "l"(p));
}

__device__ __forceinline__ void ld8_stream(const void* p, uint32_t& a, uint32_t& b) {
    asm volatile("ld.global.nc.L1::no_allocate.v2.b32 {%0,%1}, [%2];" : "=r"(a), "=r"(b) : "l"(p));
}

__device__ __forceinline__ uint32_t ld1_stream(const uint8_t* p) {
    uint16_t v;
    asm volatile("ld.global.nc.L1::no_allocate.b8 %0, [%1];" : "=h"(v) : "l"(p));
    return v & 0xFFu;
}

__device__ __forceinline__ void st32(void* p, const uint32_t (&v)[8]) {
    asm volatile("st.global.v8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"l"(p), "r"(v[0]), "r"(v[1]),
                 "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7])
                 : "memory");
}

__device__ __forceinline__ void st8(void* p, uint32_t a, uint32_t b) {
    asm volatile("st.global.v2.b32 [%0], {%1,%2};" ::"l"(p), "r"(a), "r"(b) : "memory");
}

// ---- packed binary32 arithmetic (IEEE per lane, no contraction) ---------------------------

__device__ __forceinline__ float2 mul2(float2 a, float2 b) {
    float2 d;
    asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
        "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
        "mul.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(d.x), "=f"(d.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
    return d;
}

__device__ __forceinline__ float2 sub2(float2 a, float2 b) {
    float2 d;
    asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
        "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
        "sub.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(d.x), "=f"(d.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
    return d;
}

__device__ __forceinline__ float2 add2(float2 a, float2 b) {
    float2 d;
    asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
        "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
        "add.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(d.x), "=f"(d.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
    return d;
}

// d = a * b + c per lane, one rounding.
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) {
    float2 d;
    asm("{\n\t.reg .b64 ra, rb, rc, rd;\n\t"
        "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\tmov.b64 rc, {%6, %7};\n\t"
        "fma.rn.f32x2 rd, ra, rb, rc;\n\tmov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(d.x), "=f"(d.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
    return d;
}

// gpu-scope acquire loads (values written by other CTAs of the same launch)
__device__ __forceinline__ uint32_t ld_acquire_u32(const uint32_t* p) {
    uint32_t v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ float ld_acquire_f32(const float* p) {
    return __uint_as_float(ld_acquire_u32(reinterpret_cast<const uint32_t*>(p)));
}

// ---- format conversions ------------------------------------------------------------------

// Eight binary32 values -> eight E2M1 codes packed as in e2m1x8_and_decode, without the decode
// (the conversions write their bytes straight into the word).
__device__ __forceinline__ uint32_t e2m1x8(float2 p0, float2 p1, float2 p2, float2 p3) {
    uint32_t r;
    asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
        "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
        : "=r"(r)
        : "f"(p0.x), "f"(p0.y), "f"(p1.x), "f"(p1.y), "f"(p2.x), "f"(p2.y), "f"(p3.x), "f"(p3.y));
    return r;
}

// 8-byte shared-memory load (volatile: stays after the barrier that publishes the table).
__device__ __forceinline__ float2 lds_f2(uint32_t a) {
    float2 v;
    asm volatile("ld.shared.v2.f32 {%0, %1}, [%2];" : "=f"(v.x), "=f"(v.y) : "r"(a));
    return v;
}

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// Eight packed E2M1 codes loaded from memory -> four f16x2 words (exact); word j holds
// elements 2j (low half) and 2j+1 (high half).
__device__ __forceinline__ void e2m1x8_to_f16x2(uint32_t w, uint32_t& h0, uint32_t& h1, uint32_t& h2,
                                                uint32_t& h3) {
    asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
        "mov.b32 {b0, b1, b2, b3}, %4;\n\t"
        "cvt.rn.f16x2.e2m1x2 %0, b0;\n\t"
        "cvt.rn.f16x2.e2m1x2 %1, b1;\n\t"
        "cvt.rn.f16x2.e2m1x2 %2, b2;\n\t"
        "cvt.rn.f16x2.e2m1x2 %3, b3;\n\t}"
        : "=r"(h0), "=r"(h1), "=r"(h2), "=r"(h3)
        : "r"(w));
}

// Eight binary32 values (four pairs p[j] = (element 2j, element 2j+1)) -> eight E2M1 codes
// packed so that element k sits in bits [4k, 4k+4) (the low nibble of each byte holds the
// even element; cvt ... d, a, b puts a in the high nibble and b in the low nibble), and the
// codes' exact values as four f16x2 words (word j: element 2j low, 2j+1 high).
// The four conversions write their bytes straight into the packed word; the decode then reads
// the word's bytes. The word passes through a byte permutation whose selector is the identity
// 0x3210 given at run time (`ident`, a kernel argument), so the compiler treats it as an
// arbitrary word: letting the compiler forward the conversions' bytes into the decode
// instead (the same code without the permutation) decoded bytes 2 and 3 as zeros with CUDA
// 12.9 for sm_100a, and decoding each byte before packing costs about three more
// instructions per word.
__device__ __forceinline__ uint32_t e2m1x8_and_decode(float2 p0, float2 p1, float2 p2, float2 p3, uint32_t& h0,
                                                      uint32_t& h1, uint32_t& h2, uint32_t& h3, uint32_t ident) {
    uint32_t r;
    asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
        "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
        : "=r"(r)
        : "f"(p0.x), "f"(p0.y), "f"(p1.x), "f"(p1.y), "f"(p2.x), "f"(p2.y), "f"(p3.x), "f"(p3.y));
    e2m1x8_to_f16x2(__byte_perm(r, 0u, ident), h0, h1, h2, h3);
    return r;
}

// f16 pair -> two binary32 (exact): each half widened by a mixed-precision addition of -0
// (f16 + f32 -> f32), which runs on the FMA pipes and leaves the ALU to the conversions.
__device__ __forceinline__ float2 f16x2_to_float2(uint32_t h) {
    float2 r;
    asm("{\n\t.reg .b16 a, b;\n\tmov.b32 {a, b}, %2;\n\t"
        "add.rn.f32.f16 %0, a, 0f80000000;\n\tadd.rn.f32.f16 %1, b, 0f80000000;\n\t}"
        : "=f"(r.x), "=f"(r.y)
        : "r"(h));
    return r;
}

// Two non-negative binary32 values -> two E4M3 bytes (round to nearest even, satfinite):
// the result's low byte holds `lo`, the high byte holds `hi`.
__device__ __forceinline__ uint32_t e4m3x2(float lo, float hi) {
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
    return r;
}

// Two E4M3 bytes (low byte -> .x, high byte -> .y) -> binary32 (exact).
__device__ __forceinline__ float2 e4m3x2_to_float2(uint32_t s2) {
    uint32_t h;
    uint16_t s = static_cast<uint16_t>(s2);
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h) : "h"(s));
    return f16x2_to_float2(h);
}

// Two binary32 -> BF16x2 bits, round to nearest even (low half = a).
__device__ __forceinline__ uint32_t bf16x2(float2 v) {
    __nv_bfloat162 b = __floats2bfloat162_rn(v.x, v.y);
    return *reinterpret_cast<uint32_t*>(&b);
}

// BF16x2 bits -> two binary32 (exact), by mixed-precision additions of -0 like f16x2_to_float2
// (x + -0 is x for every finite x, zeros keep their sign).
__device__ __forceinline__ float2 unpack_bf16x2(uint32_t w) {
    float2 r;
    asm("{\n\t.reg .b16 a, b;\n\tmov.b32 {a, b}, %2;\n\t"
        "add.rn.f32.bf16 %0, a, 0f80000000;\n\tadd.rn.f32.bf16 %1, b, 0f80000000;\n\t}"
        : "=f"(r.x), "=f"(r.y)
        : "r"(w));
    return r;
}

}  // namespace nvfp4
