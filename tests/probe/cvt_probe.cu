// cvt_probe.cu — TEST INFRASTRUCTURE: runs single hardware instructions element-wise so the
// tests can compare them with the oracle's scalar definitions (rounding, ties, saturation,
// sign of zero) and with IEEE host arithmetic. Not part of the product library.
#include <cuda_runtime.h>
#include <cuda_fp16.h>
#include <cuda_bf16.h>
#include <stdint.h>

namespace {

__global__ void k_e2m1(const float* in, uint8_t* out, int64_t n) {
    for (int64_t i = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; i < n; i += int64_t(gridDim.x) * blockDim.x) {
        uint16_t r;
        // the probed value goes to the low nibble (second source operand)
        asm("{ .reg .b8 t; cvt.rn.satfinite.e2m1x2.f32 t, %1, %2; cvt.u16.u8 %0, t; }"
            : "=h"(r) : "f"(0.0f), "f"(in[i]));
        out[i] = static_cast<uint8_t>(r & 0xF);
    }
}

__global__ void k_e2m1_hi(const float* in, uint8_t* out, int64_t n) {
    for (int64_t i = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; i < n; i += int64_t(gridDim.x) * blockDim.x) {
        uint16_t r;
        // the probed value goes to the high nibble (first source operand)
        asm("{ .reg .b8 t; cvt.rn.satfinite.e2m1x2.f32 t, %1, %2; cvt.u16.u8 %0, t; }"
            : "=h"(r) : "f"(in[i]), "f"(0.0f));
        out[i] = static_cast<uint8_t>((r >> 4) & 0xF);
    }
}

__global__ void k_e4m3(const float* in, uint8_t* out, int64_t n) {
    for (int64_t i = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; i < n; i += int64_t(gridDim.x) * blockDim.x) {
        uint16_t r;
        asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(0.0f), "f"(in[i]));
        out[i] = static_cast<uint8_t>(r & 0xFF);
    }
}

// all 256 E2M1 byte pairs -> f16x2 -> two floats; all 65536 E4M3 pairs likewise
__global__ void k_decode(float* e2m1_out /*512*/, float* e4m3_out /*131072*/) {
    int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i < 256) {
        uint32_t h;
        uint16_t b = static_cast<uint16_t>(i);
        asm("{ .reg .b8 t; cvt.u8.u16 t, %1; cvt.rn.f16x2.e2m1x2 %0, t; }" : "=r"(h) : "h"(b));
        __half2 v = *reinterpret_cast<__half2*>(&h);
        e2m1_out[2 * i] = __low2float(v);
        e2m1_out[2 * i + 1] = __high2float(v);
    }
    if (i < 65536) {
        uint32_t h;
        uint16_t s = static_cast<uint16_t>(i);
        asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h) : "h"(s));
        __half2 v = *reinterpret_cast<__half2*>(&h);
        e4m3_out[2 * i] = __low2float(v);
        e4m3_out[2 * i + 1] = __high2float(v);
    }
}

__global__ void k_bf16(const float* in, uint16_t* out, int64_t n) {
    for (int64_t i = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; i < n; i += int64_t(gridDim.x) * blockDim.x) {
        __nv_bfloat16 b = __float2bfloat16_rn(in[i]);
        out[i] = *reinterpret_cast<uint16_t*>(&b);
    }
}

// op: 0 rcp_rn(a), 1 div_rn(a, b), 2 mul.rn.f32x2, 3 sub.rn.f32x2, 4 add.rn.f32x2, 5 fma.rn.f32x2(a, b, c),
// 6 c - a*b written as mul.rn.f32x2 then sub.rn.f32x2 (two roundings expected),
// 7 c - a*b written as fma.rn.f32x2(a, b, -0) then sub.rn.f32x2 (two roundings)
__global__ void k_arith(int op, const float* a, const float* b, const float* c, float* out, int64_t n) {
    for (int64_t i = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; i < n / 2; i += int64_t(gridDim.x) * blockDim.x) {
        float a0 = a[2 * i], a1 = a[2 * i + 1], b0 = b[2 * i], b1 = b[2 * i + 1], c0 = c[2 * i], c1 = c[2 * i + 1];
        float r0, r1;
        switch (op) {
            case 0: r0 = __frcp_rn(a0); r1 = __frcp_rn(a1); break;
            case 1: r0 = __fdiv_rn(a0, b0); r1 = __fdiv_rn(a1, b1); break;
            case 2:
                asm("{ .reg .b64 x, y, z; mov.b64 x, {%2, %3}; mov.b64 y, {%4, %5}; mul.rn.f32x2 z, x, y; mov.b64 {%0, %1}, z; }"
                    : "=f"(r0), "=f"(r1) : "f"(a0), "f"(a1), "f"(b0), "f"(b1));
                break;
            case 3:
                asm("{ .reg .b64 x, y, z; mov.b64 x, {%2, %3}; mov.b64 y, {%4, %5}; sub.rn.f32x2 z, x, y; mov.b64 {%0, %1}, z; }"
                    : "=f"(r0), "=f"(r1) : "f"(a0), "f"(a1), "f"(b0), "f"(b1));
                break;
            case 4:
                asm("{ .reg .b64 x, y, z; mov.b64 x, {%2, %3}; mov.b64 y, {%4, %5}; add.rn.f32x2 z, x, y; mov.b64 {%0, %1}, z; }"
                    : "=f"(r0), "=f"(r1) : "f"(a0), "f"(a1), "f"(b0), "f"(b1));
                break;
            case 5:
                asm("{ .reg .b64 x, y, w, z; mov.b64 x, {%2, %3}; mov.b64 y, {%4, %5}; mov.b64 w, {%6, %7}; fma.rn.f32x2 z, x, y, w; mov.b64 {%0, %1}, z; }"
                    : "=f"(r0), "=f"(r1) : "f"(a0), "f"(a1), "f"(b0), "f"(b1), "f"(c0), "f"(c1));
                break;
            case 6: {
                float p0, p1;
                asm("{ .reg .b64 x, y, z; mov.b64 x, {%2, %3}; mov.b64 y, {%4, %5}; mul.rn.f32x2 z, x, y; mov.b64 {%0, %1}, z; }"
                    : "=f"(p0), "=f"(p1) : "f"(a0), "f"(a1), "f"(b0), "f"(b1));
                asm("{ .reg .b64 x, y, z; mov.b64 x, {%2, %3}; mov.b64 y, {%4, %5}; sub.rn.f32x2 z, x, y; mov.b64 {%0, %1}, z; }"
                    : "=f"(r0), "=f"(r1) : "f"(c0), "f"(c1), "f"(p0), "f"(p1));
                break;
            }
            default: {
                float p0, p1;
                asm("{ .reg .b64 x, y, w, z; mov.b64 x, {%2, %3}; mov.b64 y, {%4, %5}; mov.b64 w, {%6, %6}; fma.rn.f32x2 z, x, y, w; mov.b64 {%0, %1}, z; }"
                    : "=f"(p0), "=f"(p1) : "f"(a0), "f"(a1), "f"(b0), "f"(b1), "f"(-0.0f));
                asm("{ .reg .b64 x, y, z; mov.b64 x, {%2, %3}; mov.b64 y, {%4, %5}; sub.rn.f32x2 z, x, y; mov.b64 {%0, %1}, z; }"
                    : "=f"(r0), "=f"(r1) : "f"(c0), "f"(c1), "f"(p0), "f"(p1));
                break;
            }
        }
        out[2 * i] = r0;
        out[2 * i + 1] = r1;
    }
}

int status() { return cudaGetLastError() == cudaSuccess ? 0 : 1; }
unsigned grid(int64_t n) { int64_t g = (n + 255) / 256; return static_cast<unsigned>(g < 4096 ? (g < 1 ? 1 : g) : 4096); }

}  // namespace

extern "C" {
int probe_e2m1(const float* in, uint8_t* out, int64_t n, int high) {
    if (high) k_e2m1_hi<<<grid(n), 256>>>(in, out, n); else k_e2m1<<<grid(n), 256>>>(in, out, n);
    return status();
}
int probe_e4m3(const float* in, uint8_t* out, int64_t n) { k_e4m3<<<grid(n), 256>>>(in, out, n); return status(); }
int probe_decode(float* e2m1_out, float* e4m3_out) { k_decode<<<256, 256>>>(e2m1_out, e4m3_out); return status(); }
int probe_bf16(const float* in, uint16_t* out, int64_t n) { k_bf16<<<grid(n), 256>>>(in, out, n); return status(); }
int probe_arith(int op, const float* a, const float* b, const float* c, float* out, int64_t n) {
    k_arith<<<grid(n / 2), 256>>>(op, a, b, c, out, n);
    return status();
}
int probe_sync(void) { return cudaDeviceSynchronize() == cudaSuccess ? 0 : 1; }
}
