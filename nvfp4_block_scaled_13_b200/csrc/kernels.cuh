// kernels.cuh — sm_100a kernels of the NVFP4 quantizer: amax, quantize / fake-quant (a
// grouped kernel whose CTAs work inside one group at a time, and a flat one for any group
// layout) and dequantize.
//
// Grids are persistent (a multiple of the SM count). In the grouped kernel a warp owns tiles
// of 64 consecutive blocks: it reads 2 KiB of contiguous input per tile with 32-byte vector
// loads, prefetched one tile ahead, and writes 512 contiguous bytes of codes, 64 bytes of
// scales and two 32-bit words of choice bits (warp ballots).
#pragma once

#include "block.cuh"

namespace nvfp4 {

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

// Each warp works on tiles of 64 consecutive blocks of one group (the grid is described at
// quantize_grouped_kernel): lane t quantizes blocks t and
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
template <bool FOUR, int RULE, bool FQ, bool SWZ, bool DEC = false>
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
    const bool fa = quantize_block<FOUR, RULE, FQ, true, DEC>(ca, gc, tab, c0, SWZ ? p.scales + tiled_scale_offset(a, p) : s0,
                                                         y0, oka);
    const bool fb = quantize_block<FOUR, RULE, FQ, true, DEC>(cb, gc, tab, FQ ? nullptr : c0 + 256,
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

// Tiles tile, tile + stride, ... below tend of group g, with the group's scale table built
// first (every thread of the CTA takes part: the table is shared). write_tscale: this CTA
// stores the group's tensor scale.
// FRESH: the amax was written during this launch (by other CTAs), so it is read with a
// gpu-scope acquire load rather than through the read-only cache.
template <bool FOUR, int RULE, bool FQ, bool SWZ, bool FRESH = false, bool DEC = false>
__device__ __forceinline__ void quant_segment(const QuantParams& p, float2* tab, int64_t g, uint32_t tile,
                                              uint32_t tend, uint32_t stride, uint32_t lane, bool write_tscale,
                                              uint32_t dtab = 0, float2* dect = nullptr, bool fill_dec = false) {
    constexpr float kSixM = FOUR ? 1536.0f : 2688.0f;   // 6 * 256 or 6 * 448
    const uint32_t bpg = static_cast<uint32_t>(p.gdiv.bpg);
    const int64_t base = g * static_cast<int64_t>(bpg);
    const uint16_t* xg = p.x + base * 16;
    uint32_t a0[8], a1[8];
    if (tile < tend) load_tile(xg, tile, lane, bpg, a0, a1);   // in flight while the tables are built
    if constexpr (DEC) {
        if (fill_dec) fill_decode_table(dect);   // once per CTA; the barrier below publishes it
    }
    GroupCtx gc = make_group<FOUR>(FRESH ? ld_acquire_f32(p.amax + g) : __ldg(p.amax + g), kSixM, p.ident);
    gc.lane8 = (lane & 15u) * 8u;
    gc.dtab = dtab;
    __syncthreads();                       // the previous group's table is no longer read
    fill_scale_tables<FOUR>(tab, gc, threadIdx.x);
    if (!FQ && write_tscale && threadIdx.x == 0) p.tscale[g] = gc.alpha;
    __syncthreads();
    uint8_t* cg = FQ ? nullptr : p.codes + base * 8;
    uint8_t* sg = FQ ? nullptr : p.scales + base;
    uint16_t* yg = FQ ? p.y + base * 16 : nullptr;
    uint32_t* chw = reinterpret_cast<uint32_t*>(p.choice) + (base >> 5);   // base is a multiple of 32
    if constexpr (!FOUR) {   // one prefetch buffer: two would not fit the 64-register budget
        for (; tile < tend; tile += stride) {
            uint32_t b0[8], b1[8];
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                b0[k] = a0[k];
                b1[k] = a1[k];
            }
            if (tile + stride < tend) load_tile(xg, tile + stride, lane, bpg, a0, a1);
            quant_tile<FOUR, RULE, FQ, SWZ, DEC>(p, gc, tab, tile, lane, bpg, cg, sg, yg, chw, base, b0, b1);
        }
    } else {
        uint32_t b0[8], b1[8];
        while (tile < tend) {
            uint32_t nt = tile + stride;
            if (nt < tend) load_tile(xg, nt, lane, bpg, b0, b1);
            quant_tile<FOUR, RULE, FQ, SWZ, DEC>(p, gc, tab, tile, lane, bpg, cg, sg, yg, chw, base, a0, a1);
            tile = nt;
            if (tile >= tend) break;
            nt = tile + stride;
            if (nt < tend) load_tile(xg, nt, lane, bpg, a0, a1);
            quant_tile<FOUR, RULE, FQ, SWZ, DEC>(p, gc, tab, tile, lane, bpg, cg, sg, yg, chw, base, b0, b1);
            tile = nt;
        }
    }
}

// One group: grid (x, 1), every warp of the grid strides over the group's tiles, so the warps
// in flight read neighbouring tiles. Several groups: grid (x, 1), CTA b takes the contiguous
// range [b T / x, (b + 1) T / x) of the T = groups * tiles_per_group tiles in group order, as
// one segment per group it touches (its warps stride by the CTA's 8 warps inside a segment),
// so every CTA slot works and the ranges differ by at most one tile.
template <bool FOUR, int RULE, bool FQ, bool SWZ = false>
__global__ void __launch_bounds__(kThreads, FOUR ? 2 : 4) quantize_grouped_kernel(const QuantParams p) {
    __shared__ float2 tab[256];   // scale tables (fill_scale_tables)
    extern __shared__ __align__(16) float2 dect[];   // decode table (Four Over Six codes): 64 KiB dynamic
    constexpr bool kDec = FOUR && !FQ;
    if (kDec) {
        // a launch without the table's dynamic shared memory would read past it: do nothing
        uint32_t dyn;
        asm("mov.u32 %0, %%dynamic_smem_size;" : "=r"(dyn));
        if (dyn < kDecodeTableBytes) return;
    }
    const uint32_t dtab = kDec ? smem_addr(dect) : 0u;
    const uint32_t lane = threadIdx.x & 31u;
    const uint32_t bpg = static_cast<uint32_t>(p.gdiv.bpg);
    const uint32_t ntiles = (bpg + 63u) >> 6;
    constexpr uint32_t kWarps = kThreads / 32;
    const uint32_t w = threadIdx.x >> 5;
    // one call site for both layouts (the inlined tile loop is large; a second copy costs issue)
    const bool one = p.groups == 1;
    const int64_t total = p.groups * static_cast<int64_t>(ntiles);
    const int64_t begin = one ? 0 : total * blockIdx.x / gridDim.x;
    const int64_t end = one ? ntiles : total * (blockIdx.x + 1) / gridDim.x;
    const uint32_t first = one ? blockIdx.x * kWarps + w : w, stride = one ? gridDim.x * kWarps : kWarps;
    for (int64_t t = begin; t < end;) {
        const int64_t g = t / ntiles;
        const uint32_t t0 = static_cast<uint32_t>(t - g * ntiles);
        const uint32_t t1 = static_cast<uint32_t>(min(end - g * ntiles, static_cast<int64_t>(ntiles)));
        quant_segment<FOUR, RULE, FQ, SWZ, false, kDec>(p, tab, g, t0 + first, t1, stride, lane,
                                                        one ? blockIdx.x == 0 : t0 == 0, dtab, dect, t == begin);
        t = g * ntiles + t1;
    }
}

// ---- amax and quantize / fake-quant in one launch (a grid-wide wait between them) -------------

// Max |x| (as BF16 magnitude bits, packed pairs) over the lane's blocks of tiles tile, tile +
// stride, ... below tend of one group (the tiles the same lane quantizes afterwards).
__device__ __forceinline__ uint32_t segment_max2(const uint16_t* xg, uint32_t tile, uint32_t tend, uint32_t stride,
                                                 uint32_t lane, uint32_t bpg) {
    uint32_t m2 = 0;
    for (; tile < tend; tile += stride) {
        uint32_t a[8], b[8];
        load_tile(xg, tile, lane, bpg, a, b);
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            asm("max.u16x2 %0, %0, %1;" : "+r"(m2) : "r"(a[k] & 0x7FFF7FFFu));
            asm("max.u16x2 %0, %0, %1;" : "+r"(m2) : "r"(b[k] & 0x7FFF7FFFu));
        }
    }
    return m2;
}

// Maximum over the CTA of one value per thread, combined into *out with an unsigned atomic
// maximum (binary32 values >= 0 order like their bits). Every thread of the CTA calls it.
__device__ __forceinline__ void cta_max_to(uint32_t* red, uint32_t v, float* out) {
    v = __reduce_max_sync(0xFFFFFFFFu, v);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (lane == 0) red[warp] = v;
    __syncthreads();
    if (warp == 0) {
        uint32_t w = lane < kThreads / 32 ? red[lane] : 0u;
        w = __reduce_max_sync(0xFFFFFFFFu, w);
        if (lane == 0 && w != 0) atomicMax(reinterpret_cast<unsigned int*>(out), w << 16);
    }
    __syncthreads();
}

// Quantize (or fake-quantize) with the group amaxes found in the same launch: every CTA first
// reduces max |x| over exactly the tiles it quantizes afterwards into p.amax (zero-filled
// before the launch), then all CTAs meet at a grid-wide barrier on *arrive (zero-filled
// before the launch), then they quantize as quantize_grouped_kernel does, re-reading their
// tiles (from L2 when the tensor fits there). The grid must be co-resident (a cooperative
// launch). The barrier waits for `expected` arrivals (the library passes gridDim.x). Its wait
// is bounded (about two seconds): on timeout the CTA or-s NVFP4_QUANT_TIMEOUT into *status
// (nullable) and quantizes nothing.
template <bool FOUR, int RULE, bool FQ>
__global__ void __launch_bounds__(kThreads, FOUR ? 2 : 4) quantize_amax_kernel(const QuantParams p, uint32_t* arrive,
                                                                                uint32_t* status, uint32_t expected) {
    __shared__ float2 tab[256];   // scale tables (fill_scale_tables)
    __shared__ uint32_t red[kThreads / 32];
    __shared__ uint32_t go;
    const uint32_t lane = threadIdx.x & 31u;
    const uint32_t bpg = static_cast<uint32_t>(p.gdiv.bpg);
    const uint32_t ntiles = (bpg + 63u) >> 6;
    constexpr uint32_t kWarps = kThreads / 32;
    const uint32_t w = threadIdx.x >> 5;
    const bool one = p.groups == 1;
    const int64_t total = p.groups * static_cast<int64_t>(ntiles);
    const int64_t begin = one ? 0 : total * blockIdx.x / gridDim.x;
    const int64_t end = one ? ntiles : total * (blockIdx.x + 1) / gridDim.x;
    const uint32_t first = one ? blockIdx.x * kWarps + w : w, stride = one ? gridDim.x * kWarps : kWarps;
    float* amax = const_cast<float*>(p.amax);
    for (int64_t t = begin; t < end;) {   // phase 1: this CTA's share of every group's amax
        const int64_t g = t / ntiles;
        const uint32_t t0 = static_cast<uint32_t>(t - g * ntiles);
        const uint32_t t1 = static_cast<uint32_t>(min(end - g * ntiles, static_cast<int64_t>(ntiles)));
        const uint32_t m2 = segment_max2(p.x + g * static_cast<int64_t>(bpg) * 16, t0 + first, t1, stride, lane, bpg);
        cta_max_to(red, max(m2 & 0xFFFFu, m2 >> 16), amax + g);
        t = g * ntiles + t1;
    }
    if (threadIdx.x == 0) {   // grid-wide barrier: release this CTA's maxima, wait for every CTA
        __threadfence();
        atomicAdd(arrive, 1u);
        uint32_t ok = 1;
        const unsigned long long t0 = clock64();
        while (ld_acquire_u32(arrive) < expected) {
            if (clock64() - t0 > 4000000000ull) {
                ok = 0;
                if (status != nullptr) atomicOr(status, NVFP4_QUANT_TIMEOUT);
                break;
            }
            __nanosleep(64);
        }
        go = ok;
    }
    __syncthreads();
    if (!go) return;
    for (int64_t t = begin; t < end;) {   // phase 2: quantize with the finished amaxes
        const int64_t g = t / ntiles;
        const uint32_t t0 = static_cast<uint32_t>(t - g * ntiles);
        const uint32_t t1 = static_cast<uint32_t>(min(end - g * ntiles, static_cast<int64_t>(ntiles)));
        quant_segment<FOUR, RULE, FQ, false, true>(p, tab, g, t0 + first, t1, stride, lane,
                                                   one ? blockIdx.x == 0 : t0 == 0);
        t = g * ntiles + t1;
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
                gc = make_group<FOUR>(__ldg(p.amax + g), kSixM, p.ident);
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

// Thread i dequantizes blocks 2i and 2i + 1 per step (grid-strided over pairs): two 8-byte code
// loads and two scale bytes, prefetched one step ahead, and 64 contiguous bytes of BF16 out, so
// a warp reads 512 contiguous bytes of codes and writes 2 KiB. The two blocks of a pair may sit
// in different groups; each looks its tensor scale up when it passes the cached group end.
__global__ void __launch_bounds__(kThreads, 4) dequantize_kernel(const DequantParams p) {
    const int64_t npairs = (p.nblocks + 1) >> 1;
    const int64_t stride = static_cast<int64_t>(gridDim.x) * kThreads;
    int64_t i = static_cast<int64_t>(blockIdx.x) * kThreads + threadIdx.x;
    int64_t g_end = 0;
    float alpha = 0.0f;
    uint32_t n0lo = 0, n0hi = 0, n1lo = 0, n1hi = 0, ns0 = 0, ns1 = 0;
    if (i < npairs) {
        ld8_stream(p.codes + i * 16, n0lo, n0hi);
        ns0 = ld1_stream(p.scales + 2 * i);
        if (2 * i + 1 < p.nblocks) {
            ld8_stream(p.codes + i * 16 + 8, n1lo, n1hi);
            ns1 = ld1_stream(p.scales + 2 * i + 1);
        }
    }
    for (; i < npairs; i += stride) {
        const uint32_t c[2][2] = {{n0lo, n0hi}, {n1lo, n1hi}}, sc[2] = {ns0, ns1};
        const int64_t in = i + stride;
        if (in < npairs) {
            ld8_stream(p.codes + in * 16, n0lo, n0hi);
            ns0 = ld1_stream(p.scales + 2 * in);
            if (2 * in + 1 < p.nblocks) {
                ld8_stream(p.codes + in * 16 + 8, n1lo, n1hi);
                ns1 = ld1_stream(p.scales + 2 * in + 1);
            }
        }
#pragma unroll
        for (int k = 0; k < 2; ++k) {
            const int64_t b = 2 * i + k;
            if (b >= p.nblocks) break;
            if (b >= g_end) {
                const int64_t g = p.gdiv(b);
                g_end = g * p.gdiv.bpg + p.gdiv.bpg;
                alpha = __ldg(p.tscale + g);
            }
            const float d = __fmul_rn(e4m3x2_to_float2(sc[k]).x, alpha);
            const float2 dd = make_float2(d, d);
            uint32_t h[8];
            e2m1x8_to_f16x2(c[k][0], h[0], h[1], h[2], h[3]);
            e2m1x8_to_f16x2(c[k][1], h[4], h[5], h[6], h[7]);
            uint32_t out[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) out[j] = bf16x2(mul2(f16x2_to_float2(h[j]), dd));
            st32(p.y + b * 16, out);
        }
    }
}

}  // namespace nvfp4
