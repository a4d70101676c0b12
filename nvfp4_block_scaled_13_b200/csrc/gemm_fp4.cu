// gemm_fp4.cu — block-scaled FP4 GEMM on the 5th-generation tensor cores of sm_100a:
//
//     Y[m, n] = alpha_x * alpha_w * sum_k Xq[m, k] * Wq[n, k]        (FP32 out, row-major)
//
// with NVFP4 operands: E2M1 values, one E4M3 scale per 16 consecutive elements along K and
// one FP32 tensor scale per operand ("Four Over Six", Problem definition and Implementation
// details: NVFP4 weights and activations run on Blackwell's FP4 tensor cores, and applying
// 4/6 to the activations alone recovers most of the accuracy). The activation operand Xq
// either comes in quantized (codes + scales in the tiled layout of nvfp4_quantize_gemm), or is
// quantized from BF16 inside this kernel, in the GEMM's prologue, with the same per-block
// arithmetic as nvfp4_quantize (scale-6 or Four Over Six under a max / MAE / MSE rule).
//
// One CTA computes a 128 x 256 tile of Y with warp-specialised roles over a 4-stage ring of
// K slices (256 elements: four MMAs of K = 64) in shared memory:
//   warp 0 (one lane)  TMA: B codes (and A codes when pre-quantized) as 128-byte swizzled
//                      tiles completing on the stage's "full" mbarrier, and the operands'
//                      512-byte scale tiles as bulk copies completing on its "sffull" one
//                      (on "full" as well in the prologue variant);
//   warps 6-10         (prologue variant) quantize the stage's 128 x 256 BF16 activations
//                      into the swizzled A tile and its scale tiles, then arrive on "full";
//   last warps (lane 0; two, or one in the prologue variant) wait for "sffull", copy the
//                      stage's scale tiles into tensor memory (tcgen05.cp.32x128b.warpx4, each
//                      lane those of its share of the four MMAs) and commit the copies to the
//                      stage's "sfready" mbarrier;
//   warp 1 (one lane)  waits for "sfready" and "full", issues four
//                      tcgen05.mma.kind::mxf4nvf4.block_scale.block16 into the FP32
//                      accumulator in tensor memory, and commits them to the stage's "empty"
//                      mbarrier, which releases the slot to the producers.
// m and n multiples of 256 run on pairs of CTAs instead (gemm_fp4_pair_kernel, below).
// The epilogue (warps 2-9, two per 32-lane quarter of tensor memory and 128 columns each; in
// the prologue variant warps 2-5, one per quarter) reads the accumulator with tcgen05.ld,
// releases it to the MMA lane and scales it by alpha_x * alpha_w while it stores. Every mbarrier wait is bounded: on
// timeout the kernel records NVFP4_GEMM_TIMEOUT in the status word, every role stops, the
// CTA frees its tensor memory and returns.
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>
#include <string.h>

#include "../../include/nvfp4.h"
#include "block.cuh"

namespace {

using namespace nvfp4;

constexpr int kBM = 128, kBN = 256, kBK = 256;    // CTA tile and K slice (elements)
constexpr int kStages = 4;
constexpr int kQuantWarps = 5;                    // prologue variant: warps 6..10
constexpr uint32_t kTmemCols = 512;
// tensor memory: accumulator columns 0..255; per stage, A scales 4 x 4 columns from 256 and
// B scales 4 x 8 columns from 320
constexpr uint32_t kColSfa = 256, kColSfb = 320;
// shared memory per stage: A codes 128 rows x 128 bytes, B codes 256 x 128 (128-byte
// swizzled, 1024-byte aligned), A scale tiles 4 x 512 bytes, B scale tiles 8 x 512 bytes
constexpr uint32_t kABytes = kBM * 128, kBBytes = kBN * 128;
constexpr uint32_t kSfaBytes = 4 * 512, kSfbBytes = 8 * 512;
constexpr uint32_t kStageBytes = kABytes + kBBytes + kSfaBytes + kSfbBytes;   // 55296, a multiple of 1024
constexpr uint32_t kDynSmem = kStages * kStageBytes + 1024;                   // + alignment slack
constexpr unsigned long long kWaitCycles = 4000000000ull;                     // about two seconds at 2 GHz

// ---- PTX wrappers -------------------------------------------------------------------------------

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.b32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}

// Bounded wait for the mbarrier phase with the given parity to complete (the clock is read
// once per 64 polls, so that the common case costs one try_wait).
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity) {
    if (mbar_try_wait(bar, parity)) return true;
    const unsigned long long t0 = clock64();
    for (;;) {
#pragma unroll 1
        for (int i = 0; i < 64; ++i)
            if (mbar_try_wait(bar, parity)) return true;
        if (clock64() - t0 > kWaitCycles) return false;
    }
}

__device__ __forceinline__ void fence_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}

__device__ __forceinline__ void tmem_alloc(uint32_t dst_smem, uint32_t ncols) {   // whole warp
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem), "r"(ncols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {     // whole warp
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

// Shared-memory matrix descriptor, K-major without swizzle: core matrices of 8 rows x 16 bytes
// (128 contiguous bytes); `lbo` = bytes between the two 16-byte K chunks of one MMA, `sbo` =
// bytes between 8-row groups; version 1 (Blackwell) in bits 46-47, layout type 0.
__device__ __forceinline__ uint64_t smem_desc(uint32_t addr, uint32_t lbo, uint32_t sbo) {
    uint64_t d = 0;
    d |= static_cast<uint64_t>((addr >> 4) & 0x3FFFu);
    d |= static_cast<uint64_t>((lbo >> 4) & 0x3FFFu) << 16;
    d |= static_cast<uint64_t>((sbo >> 4) & 0x3FFFu) << 32;
    d |= static_cast<uint64_t>(1) << 46;
    return d;
}

// The same for a K-major operand written with the 128-byte swizzle (TMA's SWIZZLE_128B):
// rows of 128 bytes, 8-row atoms of 1024 bytes (SBO), layout type 2; the MMA with K offset j
// (32 bytes each) starts 32 j bytes into the 1024-byte-aligned atom.
__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t addr) {
    uint64_t d = 0;
    d |= static_cast<uint64_t>((addr >> 4) & 0x3FFFu);
    d |= static_cast<uint64_t>(1) << 16;
    d |= static_cast<uint64_t>(1024 >> 4) << 32;
    d |= static_cast<uint64_t>(1) << 46;
    d |= static_cast<uint64_t>(2) << 61;
    return d;
}

__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

// 2-D tiled TMA load of box {x, y} (x in bytes along K) into shared memory.
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, int32_t x, int32_t y,
                                            uint32_t bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];"
        ::"r"(dst), "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar)
        : "memory");
}

// Contiguous bulk copy (16-byte aligned, multiple of 16 bytes) into shared memory.
__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
                 ::"r"(dst), "l"(src), "r"(bytes), "r"(bar)
                 : "memory");
}

// Instruction descriptor of kind::mxf4nvf4 with 16-element E4M3 scale blocks: A and B E2M1
// (format 1), both K-major, scale format E4M3 (0), M = 128, N = 256, dense, K = 64.
constexpr uint32_t kIdesc = (1u << 7) | (1u << 10) | (static_cast<uint32_t>(kBN >> 3) << 17) |
                            (static_cast<uint32_t>(kBM >> 4) << 24);

// 32 rows x 16 bytes of scale factors (one 512-byte tile) -> 4 TMEM columns, replicated to
// the four 32-lane quarters; row i of the tile lands in lane i (+32 q), column c, byte j
// holding the scale of row i + 32 c and K block j of the MMA.
__device__ __forceinline__ void tmem_copy_sf(uint32_t taddr, uint64_t desc) {
    asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(desc) : "memory");
}

__device__ __forceinline__ void mma_fp4(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                        uint32_t sfa_tmem, uint32_t sfb_tmem, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%5], [%6], p;\n\t}"
        ::"r"(d_tmem), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem)
        : "memory");
}

__device__ __forceinline__ void mma_commit(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
                 : "memory");
}

// 32 lanes x 64 consecutive 32-bit columns of tensor memory -> 64 registers per thread; the
// registers are valid after tmem_wait_ld().
__device__ __forceinline__ void tmem_ld64(uint32_t taddr, uint32_t (&r)[64]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x64.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,"
        "%32,%33,%34,%35,%36,%37,%38,%39,%40,%41,%42,%43,%44,%45,%46,%47,"
        "%48,%49,%50,%51,%52,%53,%54,%55,%56,%57,%58,%59,%60,%61,%62,%63}, [%64];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
          "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31]),
          "=r"(r[32]), "=r"(r[33]), "=r"(r[34]), "=r"(r[35]), "=r"(r[36]), "=r"(r[37]), "=r"(r[38]), "=r"(r[39]),
          "=r"(r[40]), "=r"(r[41]), "=r"(r[42]), "=r"(r[43]), "=r"(r[44]), "=r"(r[45]), "=r"(r[46]), "=r"(r[47]),
          "=r"(r[48]), "=r"(r[49]), "=r"(r[50]), "=r"(r[51]), "=r"(r[52]), "=r"(r[53]), "=r"(r[54]), "=r"(r[55]),
          "=r"(r[56]), "=r"(r[57]), "=r"(r[58]), "=r"(r[59]), "=r"(r[60]), "=r"(r[61]), "=r"(r[62]), "=r"(r[63])
        : "r"(taddr));
}

__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// 8 consecutive FP32 outputs (a 32-byte sector), each accumulator word times alpha.
__device__ __forceinline__ void st_v8f(float* dst, const uint32_t* r, float alpha) {
    asm volatile("st.global.v8.f32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"l"(dst),
                 "f"(__uint_as_float(r[0]) * alpha), "f"(__uint_as_float(r[1]) * alpha),
                 "f"(__uint_as_float(r[2]) * alpha), "f"(__uint_as_float(r[3]) * alpha),
                 "f"(__uint_as_float(r[4]) * alpha), "f"(__uint_as_float(r[5]) * alpha),
                 "f"(__uint_as_float(r[6]) * alpha), "f"(__uint_as_float(r[7]) * alpha)
                 : "memory");
}

// 16 consecutive outputs as BF16 (one 32-byte sector), each accumulator word times alpha rounded
// to binary32 and then to BF16 (so each equals the BF16 rounding of the FP32 output). `mag`
// collects the largest |alpha * acc| as binary32 bits: non-negative floats order like their
// bits, and a NaN sorts above infinity.
__device__ __forceinline__ void st_v16bf(uint16_t* dst, const uint32_t* r, float alpha, uint32_t& mag) {
    uint32_t w[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const float a = __uint_as_float(r[2 * i]) * alpha, b = __uint_as_float(r[2 * i + 1]) * alpha;
        mag = max(mag, max(__float_as_uint(a) & 0x7FFFFFFFu, __float_as_uint(b) & 0x7FFFFFFFu));
        w[i] = bf16x2(make_float2(a, b));
    }
    asm volatile("st.global.v8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"l"(dst), "r"(w[0]), "r"(w[1]), "r"(w[2]),
                 "r"(w[3]), "r"(w[4]), "r"(w[5]), "r"(w[6]), "r"(w[7])
                 : "memory");
}

__device__ __forceinline__ void sts16(uint32_t addr, uint4 v) {
    asm volatile("st.shared.v4.b32 [%0], {%1,%2,%3,%4};" ::"r"(addr), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
                 : "memory");
}

__device__ __forceinline__ void sts16b(uint32_t addr, uint16_t v) {
    asm volatile("st.shared.b16 [%0], %1;" ::"r"(addr), "h"(v) : "memory");
}

// After a timed-out wait: let the copies this producer issued land before the CTA exits. Slot
// s last received slice s + kStages * j (j = (issued - 1 - s) / stages); its barriers complete
// the phase of parity j & 1 once those bytes have arrived. Each wait is bounded.
__device__ __forceinline__ void drain_copies(uint32_t full0, uint32_t sff0, bool scales_apart, int issued,
                                             int stages) {
    for (int s = 0; s < stages && s < issued; ++s) {
        const uint32_t parity = static_cast<uint32_t>((issued - 1 - s) / stages) & 1u;
        mbar_wait(full0 + 8 * s, parity);
        if (scales_apart) mbar_wait(sff0 + 8 * s, parity);
    }
}

// ---- pairs of CTAs (a cluster of two, tcgen05 cta_group::2) ----

__device__ __forceinline__ uint32_t cluster_rank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}

// Address of this CTA's shared variable at `addr` in the shared memory of cluster CTA `rank`.
__device__ __forceinline__ uint32_t map_rank(uint32_t addr, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
    return r;
}

__device__ __forceinline__ void cluster_sync_all() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_bar) {
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_bar) : "memory");
}

// 2-D tiled TMA load into this CTA's shared memory whose completion is counted on the pair
// leader's mbarrier (`bar` is a cluster address). Each CTA loads only its own tiles.
__device__ __forceinline__ void tma_load_2d_pair(uint32_t dst, const CUtensorMap* map, int32_t x, int32_t y,
                                                 uint32_t bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes "
        "[%0], [%1, {%2, %3}], [%4];"
        ::"r"(dst), "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar)
        : "memory");
}

__device__ __forceinline__ void tmem_alloc_pair(uint32_t dst_smem, uint32_t ncols) {   // one warp per CTA
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem), "r"(ncols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

// tmem_copy_sf in both CTAs of the pair: each copies from its own shared memory at the same
// offset into its own tensor memory.
__device__ __forceinline__ void tmem_copy_sf_pair(uint32_t taddr, uint64_t desc) {
    asm volatile("tcgen05.cp.cta_group::2.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(desc) : "memory");
}

__device__ __forceinline__ void mma_fp4_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                             uint32_t sfa_tmem, uint32_t sfb_tmem, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%5], [%6], p;\n\t}"
        ::"r"(d_tmem), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem)
        : "memory");
}

// Arrive on the mbarrier at the same offset in both CTAs of the pair once the tcgen05
// operations this thread issued so far have completed.
__device__ __forceinline__ void mma_commit_both(uint32_t bar) {
    asm volatile(
        "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;"
        ::"r"(bar), "h"(static_cast<uint16_t>(3))
        : "memory");
}

// The same on this CTA's mbarrier only.
__device__ __forceinline__ void mma_commit_pair(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
                 : "memory");
}

}  // namespace


namespace {

struct GemmParams {
    uint32_t ident = 0x3210u;  // prologue variant: identity byte selector (e2m1x8_and_decode)
    const uint16_t* x;        // prologue variant: BF16 activations [m, k] (32-byte aligned)
    const float* x_amax;      // prologue variant: amax of x, [1]
    const uint8_t* x_scales;  // pre-quantized variant: tiled scales of x
    const float* x_tscale;    // pre-quantized variant: alpha_x, [1]
    const uint8_t* w_scales;  // tiled scales of w
    const float* w_tscale;    // alpha_w, [1]
    float* y;                 // [m, n] FP32, or
    uint16_t* y16;            // [m, n] BF16 (nvfp4_gemm_bf16)
    float* y_amax;            // nullable, nvfp4_gemm_bf16: max |y|, zero-filled before the launch
    uint32_t* status;         // nullable; NVFP4_GEMM_TIMEOUT is or-ed in on a timed-out wait
    int64_t m, n, k;
};

// Persistent: grid = min(tiles, SMs), CTA b takes output tiles b, b + grid, ... in row-major
// tile order (tm = t / (n / 256), tn = t % (n / 256)). tmap_a / tmap_b: the codes of x / w as
// [rows, k/2] byte matrices, boxes of 128 bytes x 128 (A) or 256 (B) rows, 128-byte swizzle
// (tmap_a unused in the prologue variant). Warps: 0 producer lane, 1 MMA lane (and tensor-memory
// allocation), 2-9 epilogue (2-5 in the prologue variant; tensor-memory lane quarter = warp % 4),
// 6-10 quantizers (prologue variant), and lane 0 of the last warps (10-11; 11 in the prologue
// variant) copies each slice's scales into tensor memory. The
// ring of K slices runs on across tiles, so the next tile's operands stream in
// while the epilogue drains the accumulator; the MMA lane waits for "accumulator empty" (all
// epilogue warps) before a tile's first MMA.
// epilogue warps: eight (two per tensor-memory lane quarter, 128 columns each) when operands come
// in quantized; four in the prologue variant, whose quantizer warps need the registers
template <bool QUANT>
__host__ __device__ constexpr int epi_warps() { return QUANT ? 4 : 8; }
// scale-copy warps (the last ones): two when operands come in quantized, each issuing the
// copies of two of a slice's four MMAs; one in the prologue variant
template <bool QUANT>
__host__ __device__ constexpr int sf_warps() { return QUANT ? 1 : 2; }
template <bool QUANT>
__host__ __device__ constexpr int gemm_threads() {
    return 32 * (2 + epi_warps<QUANT>() + (QUANT ? kQuantWarps : 0) + sf_warps<QUANT>());
}

template <bool QUANT, bool FOUR, int RULE, bool BF16 = false>
__global__ void __launch_bounds__(gemm_threads<QUANT>(), 1)
    gemm_fp4_kernel(const __grid_constant__ CUtensorMap tmap_a, const __grid_constant__ CUtensorMap tmap_b,
                    const GemmParams p) {
    static_assert(!(QUANT && BF16), "the BF16 output is built for pre-quantized operands");
    extern __shared__ uint8_t smem_raw[];
    __shared__ __align__(8) uint64_t full[kStages], empty[kStages], sfready[kStages], sffull[kStages], acc_full,
        acc_empty, drain;
    __shared__ uint32_t tmem_base_sh;
    __shared__ volatile uint32_t stop_sh;
    __shared__ float2 tab[256];   // the prologue's scale tables (fill_scale_tables)
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int64_t n_ct = p.k / 64;                   // scale tiles per 128 rows
    const int nk = static_cast<int>(p.k / kBK);
    // ragged edges: the last row tile may hold fewer than 128 rows of A (TMA fills the rest
    // with zeros and the epilogue stores only rows below m), and n a multiple of 128 may end
    // in a half tile (its second 128 rows of B are zeros and its columns are not stored)
    const int64_t ntn = (p.n + kBN - 1) / kBN, ntiles = ((p.m + kBM - 1) / kBM) * ntn;
    const uint32_t sbase = (smem_u32(smem_raw) + 1023u) & ~1023u;
    const uint32_t full0 = smem_u32(&full[0]), empty0 = smem_u32(&empty[0]), sfr0 = smem_u32(&sfready[0]);
    // pre-quantized operands: the slice's scale tiles complete on "sffull", its code tiles on
    // "full", so the scale copies into tensor memory start while the codes still stream in; in
    // the prologue variant the quantizer warps write the A scales, and everything uses "full"
    const uint32_t sff0 = QUANT ? full0 : smem_u32(&sffull[0]);
    const uint32_t accf = smem_u32(&acc_full), acce = smem_u32(&acc_empty), drain_bar = smem_u32(&drain);
    constexpr int kSfWarp0 = gemm_threads<QUANT>() / 32 - sf_warps<QUANT>();   // first scale-copy warp

    if (warp == 1) tmem_alloc(smem_u32(&tmem_base_sh), kTmemCols);
    if (tid == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(full0 + 8 * s, QUANT ? 1 + kQuantWarps : 1);
            mbar_init(empty0 + 8 * s, 1);
            mbar_init(sfr0 + 8 * s, sf_warps<QUANT>());
            mbar_init(smem_u32(&sffull[s]), 1);
        }
        mbar_init(accf, 1);
        mbar_init(acce, epi_warps<QUANT>());
        mbar_init(drain_bar, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        stop_sh = 0;
    }
    GroupCtx gc{};
    if (QUANT) {
        constexpr float kSixM = FOUR ? 1536.0f : 2688.0f;
        gc = make_group<FOUR>(__ldg(p.x_amax), kSixM, p.ident);
        fill_scale_tables<FOUR>(tab, gc, static_cast<uint32_t>(tid));
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tmem_base_sh;

    if (warp == 0) {
        if (lane == 0) {   // producer: TMA and bulk copies into the ring, tile after tile
            int g = 0;
            for (int64_t t = blockIdx.x; t < ntiles && !stop_sh; t += gridDim.x) {
                const int64_t tm = t / ntn, tn = t % ntn;
                for (int ks = 0; ks < nk; ++ks, ++g) {
                    const int s = g % kStages;
                    const uint32_t u = static_cast<uint32_t>(g / kStages);
                    if (g >= kStages && !mbar_wait(empty0 + 8 * s, (u - 1) & 1)) {
                        stop_sh = 1;
                        break;
                    }
                    const uint32_t fb = full0 + 8 * s, sA = sbase + s * kStageBytes, sB = sA + kABytes;
                    const uint32_t sSFA = sB + kBBytes, sSFB = sSFA + kSfaBytes;
                    const bool b_hi = (2 * tn + 1) * 128 < p.n;   // the tile's second 128 rows of B exist
                    const uint32_t sb = sff0 + 8 * s;   // == fb in the prologue variant
                    const uint32_t sf_bytes = (QUANT ? 0u : kSfaBytes) + (b_hi ? kSfbBytes : kSfbBytes / 2);
                    if (QUANT) {
                        mbar_expect_tx(fb, kBBytes + sf_bytes);
                    } else {
                        mbar_expect_tx(sb, sf_bytes);   // the small scale tiles first
                        mbar_expect_tx(fb, kABytes + kBBytes);
                        bulk_load(sSFA, p.x_scales + (tm * n_ct + 4 * ks) * 512, kSfaBytes, sb);
                    }
                    bulk_load(sSFB, p.w_scales + (2 * tn * n_ct + 4 * ks) * 512, kSfbBytes / 2, sb);
                    if (b_hi)
                        bulk_load(sSFB + kSfbBytes / 2, p.w_scales + ((2 * tn + 1) * n_ct + 4 * ks) * 512,
                                  kSfbBytes / 2, sb);
                    if (!QUANT) tma_load_2d(sA, &tmap_a, ks * (kBK / 2), static_cast<int32_t>(tm * kBM), fb);
                    tma_load_2d(sB, &tmap_b, ks * (kBK / 2), static_cast<int32_t>(tn * kBN), fb);
                }
            }
            if (stop_sh) drain_copies(full0, sff0, !QUANT, g, kStages);
        }
    } else if (warp == 1) {
        if (lane == 0) {   // MMA issuer: one thread issues every tcgen05 instruction, so its per-slice
                           // work is kept to a few instructions: the ring slots are unrolled and their
                           // descriptors and tensor-memory addresses are immediates off per-slot bases
            const int64_t my_tiles = (ntiles - blockIdx.x + gridDim.x - 1) / gridDim.x;
            const int64_t total = my_tiles * nk;
            const uint64_t dA0 = smem_desc_sw128(sbase), dB0 = smem_desc_sw128(sbase + kABytes);
            constexpr uint64_t kSlot = kStageBytes >> 4;   // descriptor start-address units per slot
            int64_t gg = 0;
            int ks = 0, tile_j = 0;
            uint32_t phase = 0;
            bool ok = true;
            while (gg < total && ok) {
#pragma unroll
                for (int s = 0; s < kStages; ++s) {
                    if (gg >= total) break;
                    if (ks == 0 && tile_j > 0) {   // the epilogue has drained tile tile_j - 1
                        if (!mbar_wait(acce, static_cast<uint32_t>(tile_j - 1) & 1)) {
                            ok = false;
                            break;
                        }
                    }
                    if (!mbar_wait(sfr0 + 8 * s, phase) ||   // scales copied into tensor memory
                        (!QUANT && !mbar_wait(full0 + 8 * s, phase))) {   // code tiles landed
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t ca = tmem + kColSfa + 16 * s, cb = tmem + kColSfb + 32 * s;
#pragma unroll
                    for (int jj = 0; jj < 4; ++jj)
                        mma_fp4(tmem, dA0 + s * kSlot + 2 * jj, dB0 + s * kSlot + 2 * jj, kIdesc, ca + 4 * jj,
                                cb + 8 * jj, (ks | jj) != 0);
                    mma_commit(empty0 + 8 * s);
                    ++gg;
                    if (++ks == nk) {
                        ks = 0;
                        ++tile_j;
                        mma_commit(accf);   // the tile's accumulator is complete once these MMAs are
                    }
                }
                phase ^= 1;
            }
            if (!ok) stop_sh = 1;
            mma_commit(drain_bar);   // arrives when every MMA issued above has completed
            if (!mbar_wait(drain_bar, 0)) stop_sh = 1;
        }
    } else if (warp >= kSfWarp0) {
        if (lane == 0) {   // scale copies into tensor memory, one slice at a time, off the MMA lane
            constexpr int kPer = 4 / sf_warps<QUANT>();   // MMAs whose scales this lane copies
            const int j0 = (warp - kSfWarp0) * kPer;
            const int64_t my_tiles = (ntiles - blockIdx.x + gridDim.x - 1) / gridDim.x;
            const int64_t total = my_tiles * nk;
            const uint64_t dSA0 = smem_desc(sbase + kABytes + kBBytes, 16, 128);
            const uint64_t dSB0 = smem_desc(sbase + kABytes + kBBytes + kSfaBytes, 16, 128);
            constexpr uint64_t kSlot = kStageBytes >> 4;
            int64_t gg = 0;
            uint32_t phase = 0;
            bool ok = true;
            while (gg < total && ok) {
#pragma unroll
                for (int s = 0; s < kStages; ++s) {
                    if (gg >= total) break;
                    // slice gg's scale tiles land only after the MMAs that last read this slot's
                    // scale columns have finished (the producer refilled the slot after "empty")
                    if (!mbar_wait(sff0 + 8 * s, phase)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t ca = tmem + kColSfa + 16 * s, cb = tmem + kColSfb + 32 * s;
#pragma unroll
                    for (int i = 0; i < kPer; ++i) {
                        const int jj = j0 + i;
                        tmem_copy_sf(ca + 4 * jj, dSA0 + s * kSlot + 32 * jj);
                        tmem_copy_sf(cb + 8 * jj, dSB0 + s * kSlot + 32 * jj);             // B rows 0..127
                        tmem_copy_sf(cb + 8 * jj + 4, dSB0 + s * kSlot + 128 + 32 * jj);   // 128..255
                    }
                    mma_commit(sfr0 + 8 * s);   // "scales ready" once these copies have completed
                    ++gg;
                }
                phase ^= 1;
            }
            if (!ok) stop_sh = 1;
        }
    } else if (warp < 2 + epi_warps<QUANT>()) {   // epilogue: warp w reads tensor-memory lane quarter w % 4
        const int q = warp & 3;
        int j = 0;
        for (int64_t t = blockIdx.x; t < ntiles && !stop_sh; t += gridDim.x, ++j) {
            const int64_t tm = t / ntn, tn = t % ntn;
            uint32_t ok = 1;
            if (lane == 0) ok = mbar_wait(accf, j & 1);
            if (!__shfl_sync(0xFFFFFFFFu, ok, 0)) {
                stop_sh = 1;
                break;
            }
            tc_fence_after();
            const float alpha = (QUANT ? gc.alpha : __ldg(p.x_tscale)) * __ldg(p.w_tscale);
            const int64_t row = tm * kBM + 32 * q + lane;
            const bool row_ok = row < p.m, full_n = tn * kBN + kBN <= p.n;
            float* yr = BF16 ? nullptr : p.y + (row_ok ? row : 0) * p.n + tn * kBN;
            const uint32_t trow = tmem + (static_cast<uint32_t>(32 * q) << 16);
            uint32_t r0[64], r1[64];
            if constexpr (epi_warps<QUANT>() == 8) {
                // this warp's 128 columns come out of tensor memory in two loads; the accumulator
                // is released before any store, so the next tile's MMAs overlap all of them
                const int c0 = (warp - 2) >> 2 ? 128 : 0;
                tmem_ld64(trow + c0, r0);
                tmem_ld64(trow + c0 + 64, r1);
                tmem_wait_ld();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(acce);
                if constexpr (BF16) {
                    // BF16 output with its amax fused in: rounding is monotone and symmetric, so
                    // max |BF16(v)| = BF16(max |v|), one rounding per warp and tile
                    uint32_t mag = 0;
                    if (row_ok && (c0 == 0 || full_n)) {
                        uint16_t* yb = p.y16 + (row_ok ? row : 0) * p.n + tn * kBN + c0;
#pragma unroll
                        for (int e = 0; e < 64; e += 16) st_v16bf(yb + e, r0 + e, alpha, mag);
#pragma unroll
                        for (int e = 0; e < 64; e += 16) st_v16bf(yb + 64 + e, r1 + e, alpha, mag);
                    }
                    if (p.y_amax != nullptr) {
#pragma unroll
                        for (int o = 16; o > 0; o >>= 1) mag = max(mag, __shfl_xor_sync(0xFFFFFFFFu, mag, o));
                        if (lane == 0 && mag != 0)
                            atomicMax(reinterpret_cast<unsigned int*>(p.y_amax),
                                      __float_as_uint(__bfloat162float(__float2bfloat16_rn(__uint_as_float(mag)))));
                    }
                } else if (row_ok && (c0 == 0 || full_n)) {
#pragma unroll
                    for (int e = 0; e < 64; e += 8) st_v8f(yr + c0 + e, r0 + e, alpha);   // whole 32-byte sectors
#pragma unroll
                    for (int e = 0; e < 64; e += 8) st_v8f(yr + c0 + 64 + e, r1 + e, alpha);
                }
            } else {
                // four chunks of 64 columns: the next chunk's load is in flight while this one is
                // stored, and the accumulator is released as soon as the last load has landed
                tmem_ld64(trow, r0);
                tmem_wait_ld();
                tmem_ld64(trow + 64, r1);
                if (row_ok) {
#pragma unroll
                    for (int e = 0; e < 64; e += 8) st_v8f(yr + e, r0 + e, alpha);
                }
                tmem_wait_ld();
                tmem_ld64(trow + 128, r0);
                if (row_ok) {
#pragma unroll
                    for (int e = 0; e < 64; e += 8) st_v8f(yr + 64 + e, r1 + e, alpha);
                }
                tmem_wait_ld();
                tmem_ld64(trow + 192, r1);
                if (row_ok && full_n) {
#pragma unroll
                    for (int e = 0; e < 64; e += 8) st_v8f(yr + 128 + e, r0 + e, alpha);
                }
                tmem_wait_ld();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(acce);
                if (row_ok && full_n) {
#pragma unroll
                    for (int e = 0; e < 64; e += 8) st_v8f(yr + 192 + e, r1 + e, alpha);
                }
            }
        }
    } else if (QUANT) {   // warps 6-10: quantize each slice's activations into the A tile
        const int qt = tid - 192;
        int g = 0;
        for (int64_t t = blockIdx.x; t < ntiles && !stop_sh; t += gridDim.x) {
            const int64_t tm = t / ntn;
            bool ok = true;
            for (int ks = 0; ks < nk; ++ks, ++g) {
                const int s = g % kStages;
                const uint32_t u = static_cast<uint32_t>(g / kStages);
                if (g >= kStages) {
                    uint32_t w = 1;
                    if (lane == 0) w = mbar_wait(empty0 + 8 * s, (u - 1) & 1);
                    if (!__shfl_sync(0xFFFFFFFFu, w, 0)) {
                        ok = false;
                        break;
                    }
                }
                const uint32_t sA = sbase + s * kStageBytes, sSFA = sA + kABytes + kBBytes;
                // 1024 chunks of 32 elements (two blocks): chunk c = row c / 8, K chunk c % 8
                for (int c = qt; c < 1024; c += 32 * kQuantWarps) {
                    const int r = c >> 3, kc = c & 7;
                    const int64_t row = tm * kBM + r;
                    uint32_t w0[8] = {}, w1[8] = {}, c0lo, c0hi, c1lo, c1hi, s0, s1, h[8];
                    float d;
                    if (row < p.m) {   // rows past m quantize as zeros (codes 0, scale 0)
                        const uint16_t* xs = p.x + row * p.k + ks * kBK + kc * 32;
                        ld32_stream(xs, w0);
                        ld32_stream(xs + 16, w1);
                    }
                    quantize_block_regs<FOUR, RULE, false, true>(w0, gc, tab, c0lo, c0hi, s0, d, h);
                    quantize_block_regs<FOUR, RULE, false, true>(w1, gc, tab, c1lo, c1hi, s1, d, h);
                    // 128-byte swizzle: 16-byte chunk kc of row r at r * 128 + (kc ^ (r % 8)) * 16
                    sts16(sA + r * 128 + ((kc ^ (r & 7)) << 4), make_uint4(c0lo, c0hi, c1lo, c1hi));
                    // scale tile of MMA kc / 2: row r, K block j at (r % 32) * 16 + (r / 32) * 4 + j
                    sts16b(sSFA + (kc >> 1) * 512 + (r & 31) * 16 + (r >> 5) * 4 + (kc & 1) * 2,
                           static_cast<uint16_t>(s0 | (s1 << 8)));
                }
                fence_async_smem();   // the stores are read by the tensor core (async proxy)
                __syncwarp();
                if (lane == 0) mbar_arrive(full0 + 8 * s);
            }
            if (!ok) {
                stop_sh = 1;
                break;
            }
        }
    }
    tc_fence_before();
    __syncthreads();   // every role has left its loop; the MMA lane has drained the tensor core
    if (stop_sh && tid == 0 && p.status != nullptr) atomicOr(p.status, NVFP4_GEMM_TIMEOUT);
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem, kTmemCols);
}

// ---- pairs of CTAs on one 256 x 256 tile (tcgen05 cta_group::2) --------------------------------

// A cluster of two CTAs on two SMs owns a 256 x 256 output tile. CTA rank r loads rows 128 r..
// of the tile's 256 A rows (its accumulator's rows) and rows 128 r.. of its 256 B rows; the
// leader (rank 0) issues tcgen05.mma.cta_group::2 (M 256, N 256), which takes A from each CTA's
// own shared memory and B from both, and accumulates into each CTA's tensor memory. Per CTA
// and K slice the ring holds 38 KiB instead of 54 for the same MMA work: a third less traffic
// from L2, which the single-CTA kernel draws at about 12 TB/s against a measured read
// bandwidth of 15-17 TB/s. Each CTA stages the scales of its own A rows and of all 256 B rows
// (its accumulator needs them all); two lanes of the leader (warps 10 and 11, two MMAs' scales
// each) move both CTAs' scales into their tensor memory with tcgen05.cp.cta_group::2 as soon
// as the scale tiles have landed ("sffull", separate from the code tiles' "full"). Used by
// nvfp4_gemm and nvfp4_gemm_bf16 when m and n are multiples of 256; bit-identical to the
// single-CTA kernel.
constexpr int kStagesP = 5;
constexpr uint32_t kAP = 128 * 128, kBP = 128 * 128, kSfaP = 4 * 512, kSfbP = 8 * 512;
constexpr uint32_t kStageP = kAP + kBP + kSfaP + kSfbP;             // 38912, a multiple of 1024
constexpr uint32_t kDynSmemP = kStagesP * kStageP + 1024;
constexpr uint32_t kColSfaP = 256, kColSfbP = 256 + 16 * kStagesP;  // 256..335, 336..495
constexpr uint32_t kIdescP = (1u << 7) | (1u << 10) | (static_cast<uint32_t>(256 >> 3) << 17) |
                             (static_cast<uint32_t>(256 >> 4) << 24);
constexpr int kWarpsP = 12;   // producer, MMA, eight epilogue warps, two scale-copy warps
static_assert(kColSfbP + 32 * kStagesP <= kTmemCols, "tensor-memory columns");

// Grid: clusters of 2; cluster c takes 256 x 256 tiles c, c + clusters, ... (tm = t / (n / 256),
// tn = t % (n / 256)). tmap_a / tmap_b: codes as [rows, k/2] bytes in boxes of 128 bytes x 128
// rows, 128-byte swizzle; tmap_sa / tmap_sb: the tiled scale buffers viewed as
// [rows * k / 4096, 256] bytes in boxes of 256 bytes x 8 rows (the four 512-byte scale tiles of
// a 128-row tile and a 256-element K slice).
template <bool BF16>
__global__ void __launch_bounds__(32 * kWarpsP, 1)
    gemm_fp4_pair_kernel(const __grid_constant__ CUtensorMap tmap_a, const __grid_constant__ CUtensorMap tmap_b,
                         const __grid_constant__ CUtensorMap tmap_sa, const __grid_constant__ CUtensorMap tmap_sb,
                         const GemmParams p) {
    extern __shared__ uint8_t smem_raw[];
    __shared__ __align__(8) uint64_t full[kStagesP], empty[kStagesP], sfready[kStagesP], sffull[kStagesP], acc_full,
        acc_empty, drain;
    __shared__ uint32_t tmem_base_sh;
    __shared__ volatile uint32_t stop_sh;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const uint32_t rank = cluster_rank();
    const int64_t n_ct4 = p.k / 256;   // 2 KiB runs of scale tiles per 128 rows
    const int nk = static_cast<int>(p.k / kBK);
    const int64_t ntn = p.n / 256, ntiles = (p.m / 256) * ntn;
    const int64_t cluster_id = blockIdx.x >> 1, nclusters = gridDim.x >> 1;
    const uint32_t sbase = (smem_u32(smem_raw) + 1023u) & ~1023u;
    const uint32_t full0 = smem_u32(&full[0]), empty0 = smem_u32(&empty[0]), sfr0 = smem_u32(&sfready[0]);
    const uint32_t accf = smem_u32(&acc_full), acce = smem_u32(&acc_empty), drain_bar = smem_u32(&drain);
    const uint32_t sff0 = smem_u32(&sffull[0]);
    const uint32_t full0_lead = map_rank(full0, 0), acce_lead = map_rank(acce, 0), sff0_lead = map_rank(sff0, 0);

    if (warp == 1) tmem_alloc_pair(smem_u32(&tmem_base_sh), kTmemCols);
    if (tid == 0) {
        for (int s = 0; s < kStagesP; ++s) {
            mbar_init(full0 + 8 * s, 1);   // the leader's counts both CTAs' bytes
            mbar_init(empty0 + 8 * s, 1);
            mbar_init(sfr0 + 8 * s, 2);
            mbar_init(sff0 + 8 * s, 1);
        }
        mbar_init(accf, 1);
        mbar_init(acce, 16);               // the leader's: eight epilogue warps in each CTA
        mbar_init(drain_bar, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        stop_sh = 0;
    }
    tc_fence_before();
    cluster_sync_all();   // both CTAs' barriers are initialised and their tensor memory allocated
    tc_fence_after();
    const uint32_t tmem = tmem_base_sh;

    if (warp == 0) {
        if (lane == 0) {   // producer: this CTA's tiles into its ring, completion on the leader's "full"
            int g = 0;
            for (int64_t t = cluster_id; t < ntiles && !stop_sh; t += nclusters) {
                const int64_t tm = t / ntn, tn = t % ntn;
                const int64_t rt_a = 2 * tm + rank, rt_b = 2 * tn;   // 128-row tiles
                for (int ks = 0; ks < nk; ++ks, ++g) {
                    const int s = g % kStagesP;
                    const uint32_t u = static_cast<uint32_t>(g / kStagesP);
                    if (g >= kStagesP && !mbar_wait(empty0 + 8 * s, (u - 1) & 1)) {
                        stop_sh = 1;
                        break;
                    }
                    const uint32_t fb = full0_lead + 8 * s, sb = sff0_lead + 8 * s;
                    const uint32_t sA = sbase + s * kStageP, sB = sA + kAP;
                    const uint32_t sSFA = sB + kBP, sSFB = sSFA + kSfaP;
                    if (rank == 0) {   // both CTAs' bytes: the scale tiles on "sffull", the codes on "full"
                        mbar_expect_tx(sff0 + 8 * s, 2 * (kSfaP + kSfbP));
                        mbar_expect_tx(full0 + 8 * s, 2 * (kAP + kBP));
                    }
                    tma_load_2d_pair(sSFA, &tmap_sa, 0, static_cast<int32_t>((rt_a * n_ct4 + ks) * 8), sb);
                    tma_load_2d_pair(sSFB, &tmap_sb, 0, static_cast<int32_t>((rt_b * n_ct4 + ks) * 8), sb);
                    tma_load_2d_pair(sSFB + kSfbP / 2, &tmap_sb, 0,
                                     static_cast<int32_t>(((rt_b + 1) * n_ct4 + ks) * 8), sb);
                    tma_load_2d_pair(sA, &tmap_a, ks * (kBK / 2), static_cast<int32_t>(rt_a * 128), fb);
                    tma_load_2d_pair(sB, &tmap_b, ks * (kBK / 2), static_cast<int32_t>((rt_b + rank) * 128), fb);
                }
            }
            // the leader's barriers count both CTAs' bytes; the closing cluster barrier keeps the
            // other CTA (and its shared memory) alive until then
            if (stop_sh && rank == 0) drain_copies(full0, sff0, true, g, kStagesP);
        }
    } else if (warp == 1) {
        if (lane == 0 && rank == 0) {   // MMA issuer (leader only), slots unrolled as in the single-CTA kernel
            const int64_t my_tiles = (ntiles - cluster_id + nclusters - 1) / nclusters;
            const int64_t total = my_tiles * nk;
            const uint64_t dA0 = smem_desc_sw128(sbase), dB0 = smem_desc_sw128(sbase + kAP);
            constexpr uint64_t kSlot = kStageP >> 4;
            int64_t gg = 0;
            int ks = 0, tile_j = 0;
            uint32_t phase = 0;
            bool ok = true;
            while (gg < total && ok) {
#pragma unroll
                for (int s = 0; s < kStagesP; ++s) {
                    if (gg >= total) break;
                    if (ks == 0 && tile_j > 0) {   // both CTAs' epilogues have drained tile tile_j - 1
                        if (!mbar_wait(acce, static_cast<uint32_t>(tile_j - 1) & 1)) {
                            ok = false;
                            break;
                        }
                    }
                    if (!mbar_wait(sfr0 + 8 * s, phase) || !mbar_wait(full0 + 8 * s, phase)) {   // scales, codes
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t ca = tmem + kColSfaP + 16 * s, cb = tmem + kColSfbP + 32 * s;
#pragma unroll
                    for (int jj = 0; jj < 4; ++jj)
                        mma_fp4_pair(tmem, dA0 + s * kSlot + 2 * jj, dB0 + s * kSlot + 2 * jj, kIdescP, ca + 4 * jj,
                                     cb + 8 * jj, (ks | jj) != 0);
                    mma_commit_both(empty0 + 8 * s);   // releases the slot in both CTAs
                    ++gg;
                    if (++ks == nk) {
                        ks = 0;
                        ++tile_j;
                        mma_commit_both(accf);
                    }
                }
                phase ^= 1;
            }
            if (!ok) stop_sh = 1;
            mma_commit_pair(drain_bar);
            if (!mbar_wait(drain_bar, 0)) stop_sh = 1;
        }
    } else if (warp >= kWarpsP - 2) {
        if (lane == 0 && rank == 0) {   // scale copies into both CTAs' tensor memory (leader only)
            const int j0 = (warp - (kWarpsP - 2)) * 2;   // this lane copies the scales of MMAs j0, j0 + 1
            const int64_t my_tiles = (ntiles - cluster_id + nclusters - 1) / nclusters;
            const int64_t total = my_tiles * nk;
            const uint64_t dSA0 = smem_desc(sbase + kAP + kBP, 16, 128);
            const uint64_t dSB0 = smem_desc(sbase + kAP + kBP + kSfaP, 16, 128);
            constexpr uint64_t kSlot = kStageP >> 4;
            int64_t gg = 0;
            uint32_t phase = 0;
            bool ok = true;
            while (gg < total && ok) {
#pragma unroll
                for (int s = 0; s < kStagesP; ++s) {
                    if (gg >= total) break;
                    // the leader's "full" completes once both CTAs' bytes have landed, which is
                    // after the MMAs that last read this slot's scale columns have finished
                    if (!mbar_wait(sff0 + 8 * s, phase)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t ca = tmem + kColSfaP + 16 * s, cb = tmem + kColSfbP + 32 * s;
#pragma unroll
                    for (int i = 0; i < 2; ++i) {
                        const int jj = j0 + i;
                        tmem_copy_sf_pair(ca + 4 * jj, dSA0 + s * kSlot + 32 * jj);
                        tmem_copy_sf_pair(cb + 8 * jj, dSB0 + s * kSlot + 32 * jj);             // B rows 0..127
                        tmem_copy_sf_pair(cb + 8 * jj + 4, dSB0 + s * kSlot + 128 + 32 * jj);   // 128..255
                    }
                    mma_commit_pair(sfr0 + 8 * s);
                    ++gg;
                }
                phase ^= 1;
            }
            if (!ok) stop_sh = 1;
        }
    } else {   // epilogue, warps 2-9: lane quarter warp % 4, columns 0..127 (warps 2-5) or 128..255
        const int q = warp & 3;
        const int c0 = warp >= 6 ? 128 : 0;
        int j = 0;
        for (int64_t t = cluster_id; t < ntiles && !stop_sh; t += nclusters, ++j) {
            const int64_t tm = t / ntn, tn = t % ntn;
            uint32_t ok = 1;
            if (lane == 0) ok = mbar_wait(accf, j & 1);
            if (!__shfl_sync(0xFFFFFFFFu, ok, 0)) {
                stop_sh = 1;
                break;
            }
            tc_fence_after();
            const float alpha = __ldg(p.x_tscale) * __ldg(p.w_tscale);
            const int64_t off = (tm * 256 + 128 * rank + 32 * q + lane) * p.n + tn * 256 + c0;
            const uint32_t trow = tmem + (static_cast<uint32_t>(32 * q) << 16) + c0;
            uint32_t r0[64], r1[64];
            tmem_ld64(trow, r0);
            tmem_ld64(trow + 64, r1);
            tmem_wait_ld();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(acce_lead);   // the accumulator is free before any store
            if constexpr (BF16) {   // BF16 result and its amax, as in the single-CTA kernel
                uint32_t mag = 0;
                uint16_t* yb = p.y16 + off;
#pragma unroll
                for (int e = 0; e < 64; e += 16) st_v16bf(yb + e, r0 + e, alpha, mag);
#pragma unroll
                for (int e = 0; e < 64; e += 16) st_v16bf(yb + 64 + e, r1 + e, alpha, mag);
                if (p.y_amax != nullptr) {
#pragma unroll
                    for (int o = 16; o > 0; o >>= 1) mag = max(mag, __shfl_xor_sync(0xFFFFFFFFu, mag, o));
                    if (lane == 0 && mag != 0)
                        atomicMax(reinterpret_cast<unsigned int*>(p.y_amax),
                                  __float_as_uint(__bfloat162float(__float2bfloat16_rn(__uint_as_float(mag)))));
                }
            } else {
                float* yr = p.y + off;
#pragma unroll
                for (int e = 0; e < 64; e += 8) st_v8f(yr + e, r0 + e, alpha);
#pragma unroll
                for (int e = 0; e < 64; e += 8) st_v8f(yr + 64 + e, r1 + e, alpha);
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    cluster_sync_all();   // the leader has drained the MMAs that write both CTAs' tensor memory
    if (stop_sh && tid == 0 && p.status != nullptr) atomicOr(p.status, NVFP4_GEMM_TIMEOUT);
    tc_fence_after();
    if (warp == 1) tmem_dealloc_pair(tmem, kTmemCols);
}

// ---- host side -----------------------------------------------------------------------------------

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    if (fn == nullptr) {
        void* f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(f);
    }
    return fn;
}

// Tensor map of a [rows, row_bytes] byte matrix read in boxes of 128 bytes x box_rows rows
// with the 128-byte swizzle.
bool codes_map(CUtensorMap* map, const void* base, int64_t rows, int64_t row_bytes, uint32_t box_rows) {
    EncodeTiledFn enc = encode_fn();
    if (enc == nullptr) return false;
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(row_bytes), static_cast<cuuint64_t>(rows)};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(row_bytes)};
    const cuuint32_t box[2] = {128u, box_rows};
    const cuuint32_t estr[2] = {1u, 1u};
    return enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <bool QUANT, bool FOUR, int RULE, bool BF16 = false>
nvfp4_status launch_gemm(const CUtensorMap& ma, const CUtensorMap& mb, const GemmParams& p, cudaStream_t stream) {
    auto kernel = gemm_fp4_kernel<QUANT, FOUR, RULE, BF16>;
    // per device, so set on every launch (cheap)
    if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kDynSmem) != cudaSuccess)
        return NVFP4_ERR_CUDA;
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return NVFP4_ERR_CUDA;
    const int64_t tiles = ((p.m + kBM - 1) / kBM) * ((p.n + kBN - 1) / kBN);
    const unsigned grid = static_cast<unsigned>(tiles < sms ? tiles : sms);   // one CTA per SM
    kernel<<<grid, gemm_threads<QUANT>(), kDynSmem, stream>>>(ma, mb, p);
    return cudaGetLastError() == cudaSuccess ? NVFP4_OK : NVFP4_ERR_CUDA;
}

// Tensor map of a tiled scale buffer of `rows` operand rows (a multiple of 128) and k columns
// (a multiple of 256), viewed as [rows * k / 4096, 256] bytes and read in boxes of 256 bytes x 8
// rows: the 2 KiB run of four 512-byte scale tiles that a 128-row tile and a 256-element K slice
// own.
bool scales_map(CUtensorMap* map, const void* base, int64_t rows, int64_t k) {
    EncodeTiledFn enc = encode_fn();
    if (enc == nullptr) return false;
    const cuuint64_t dims[2] = {256u, static_cast<cuuint64_t>(rows / 128 * (k / 32))};
    const cuuint64_t strides[1] = {256u};
    const cuuint32_t box[2] = {256u, 8u};
    const cuuint32_t estr[2] = {1u, 1u};
    return enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// A pair launch that was refused (no cluster of two can be resident, or the launch failed).
constexpr nvfp4_status kPairRefused = static_cast<nvfp4_status>(1000);

// Clusters of two CTAs that can be resident at once on the current device (a GPC with an odd
// number of SMs leaves one unpaired), found once per device.
int pair_clusters() {
    static int cached[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) return 0;
    if (dev < 64 && cached[dev] > 0) return cached[dev];
    int sms = 0, active = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.gridDim = dim3(2);
    cfg.blockDim = dim3(32 * kWarpsP);
    cfg.dynamicSmemBytes = kDynSmemP;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaOccupancyMaxActiveClusters(&active, gemm_fp4_pair_kernel<false>, &cfg) != cudaSuccess || active < 1) {
        cudaGetLastError();
        active = sms / 2;
    }
    if (dev < 64) cached[dev] = active;
    return active;
}

template <bool BF16>
nvfp4_status launch_gemm_pair(const CUtensorMap& ma, const CUtensorMap& mb, const CUtensorMap& msa,
                              const CUtensorMap& msb, const GemmParams& p, cudaStream_t stream) {
    if (cudaFuncSetAttribute(gemm_fp4_pair_kernel<BF16>, cudaFuncAttributeMaxDynamicSharedMemorySize, kDynSmemP) !=
        cudaSuccess)
        return NVFP4_ERR_CUDA;
    const int active = pair_clusters();
    if (active < 1) return kPairRefused;
    const int64_t tiles = (p.m / 256) * (p.n / 256);
    const int64_t clusters = tiles < active ? tiles : active;
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.gridDim = dim3(static_cast<unsigned>(2 * clusters));
    cfg.blockDim = dim3(32 * kWarpsP);
    cfg.dynamicSmemBytes = kDynSmemP;
    cfg.stream = stream;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, gemm_fp4_pair_kernel<BF16>, ma, mb, msa, msb, p) != cudaSuccess) {
        cudaGetLastError();   // cluster launch refused: the caller runs the one-CTA kernel
        return kPairRefused;
    }
    return cudaGetLastError() == cudaSuccess ? NVFP4_OK : NVFP4_ERR_CUDA;
}

// The pair kernel takes shapes whose 256 x 256 tiles cover the output exactly and whose scale
// views have row counts that fit the tensor map's 32-bit coordinates.
bool use_pair(int64_t m, int64_t n, int64_t k) {
    return m % 256 == 0 && n % 256 == 0 && m / 128 * (k / 32) < (int64_t(1) << 31) &&
           n / 128 * (k / 32) < (int64_t(1) << 31);
}

bool aligned16(const void* q) { return (reinterpret_cast<uintptr_t>(q) & 15u) == 0; }
bool aligned4(const void* q) { return (reinterpret_cast<uintptr_t>(q) & 3u) == 0; }

nvfp4_status check_gemm_shape(int64_t m, int64_t n, int64_t k) {
    if (m < 0 || n < 0 || k < 0) return NVFP4_ERR_SHAPE;
    if (n % 128 || k % kBK) return NVFP4_ERR_SHAPE;
    if (k > (int64_t(1) << 30) || m > (int64_t(1) << 31) || n > (int64_t(1) << 31)) return NVFP4_ERR_SHAPE;
    return NVFP4_OK;
}

}  // namespace

namespace {

// nvfp4_gemm and nvfp4_gemm_bf16: exactly one of y (FP32) and y16 (BF16) is set.
nvfp4_status gemm_prequantized(const uint8_t* x_codes, const uint8_t* x_scales, const float* x_tscale,
                               const uint8_t* w_codes, const uint8_t* w_scales, const float* w_tscale, int64_t m,
                               int64_t n, int64_t k, float* y, uint16_t* y16, float* y_amax, uint32_t* status,
                               cudaStream_t stream) {
    const nvfp4_status st = check_gemm_shape(m, n, k);
    if (st != NVFP4_OK) return st;
    if (y_amax != nullptr && !aligned4(y_amax)) return NVFP4_ERR_ALIGN;
    const bool empty = m == 0 || n == 0;
    if (!empty) {
        if (!x_codes || !x_scales || !x_tscale || !w_codes || !w_scales || !w_tscale || (!y && !y16))
            return NVFP4_ERR_NULL;
        const uintptr_t yp = y != nullptr ? reinterpret_cast<uintptr_t>(y) : reinterpret_cast<uintptr_t>(y16);
        if (!aligned16(x_codes) || !aligned16(x_scales) || !aligned16(w_codes) || !aligned16(w_scales) ||
            (yp & 31u) || !aligned4(x_tscale) || !aligned4(w_tscale) || !aligned4(status))
            return NVFP4_ERR_ALIGN;
        if (k == 0) return NVFP4_ERR_SHAPE;
    }
    // the amax is an atomic maximum over the tiles: it starts from +0 in stream order
    if (y_amax != nullptr && cudaMemsetAsync(y_amax, 0, sizeof(float), stream) != cudaSuccess) return NVFP4_ERR_CUDA;
    if (empty) return NVFP4_OK;
    const bool pair = use_pair(m, n, k);
    CUtensorMap ma, mb, msa, msb;
    if (!codes_map(&ma, x_codes, m, k / 2, pair ? 128u : static_cast<uint32_t>(kBM)) ||
        !codes_map(&mb, w_codes, n, k / 2, pair ? 128u : static_cast<uint32_t>(kBN)))
        return NVFP4_ERR_CUDA;
    if (pair && (!scales_map(&msa, x_scales, m, k) || !scales_map(&msb, w_scales, n, k))) return NVFP4_ERR_CUDA;
    GemmParams p{};
    p.x_scales = x_scales;
    p.x_tscale = x_tscale;
    p.w_scales = w_scales;
    p.w_tscale = w_tscale;
    p.y = y;
    p.y16 = y16;
    p.y_amax = y_amax;
    p.status = status;
    p.m = m;
    p.n = n;
    p.k = k;
    if (pair) {
        const nvfp4_status ps = y16 != nullptr ? launch_gemm_pair<true>(ma, mb, msa, msb, p, stream)
                                               : launch_gemm_pair<false>(ma, mb, msa, msb, p, stream);
        if (ps != kPairRefused) return ps;
        // the one-CTA kernel reads B in boxes of 256 rows
        if (!codes_map(&ma, x_codes, m, k / 2, kBM) || !codes_map(&mb, w_codes, n, k / 2, kBN)) return NVFP4_ERR_CUDA;
    }
    if (y16 != nullptr) return launch_gemm<false, true, kMse, true>(ma, mb, p, stream);
    return launch_gemm<false, true, kMse>(ma, mb, p, stream);
}

}  // namespace

extern "C" nvfp4_status nvfp4_gemm(const uint8_t* x_codes, const uint8_t* x_scales, const float* x_tscale,
                                   const uint8_t* w_codes, const uint8_t* w_scales, const float* w_tscale,
                                   int64_t m, int64_t n, int64_t k, float* y, uint32_t* status,
                                   cudaStream_t stream) {
    return gemm_prequantized(x_codes, x_scales, x_tscale, w_codes, w_scales, w_tscale, m, n, k, y, nullptr, nullptr,
                             status, stream);
}

extern "C" nvfp4_status nvfp4_gemm_bf16(const uint8_t* x_codes, const uint8_t* x_scales, const float* x_tscale,
                                        const uint8_t* w_codes, const uint8_t* w_scales, const float* w_tscale,
                                        int64_t m, int64_t n, int64_t k, uint16_t* y, float* y_amax,
                                        uint32_t* status, cudaStream_t stream) {
    return gemm_prequantized(x_codes, x_scales, x_tscale, w_codes, w_scales, w_tscale, m, n, k, nullptr, y, y_amax,
                             status, stream);
}

extern "C" nvfp4_status nvfp4_gemm_quantize_x(const uint16_t* x, const float* x_amax, nvfp4_mode mode,
                                              nvfp4_rule rule, const uint8_t* w_codes, const uint8_t* w_scales,
                                              const float* w_tscale, int64_t m, int64_t n, int64_t k, float* y,
                                              uint32_t* status, cudaStream_t stream) {
    const nvfp4_status st = check_gemm_shape(m, n, k);
    if (st != NVFP4_OK) return st;
    if (mode != NVFP4_SCALE6 && mode != NVFP4_FOUR_OVER_SIX) return NVFP4_ERR_MODE;
    if (rule != NVFP4_RULE_MAXERR && rule != NVFP4_RULE_MAE && rule != NVFP4_RULE_MSE) return NVFP4_ERR_RULE;
    if (m == 0 || n == 0) return NVFP4_OK;
    if (!x || !x_amax || !w_codes || !w_scales || !w_tscale || !y) return NVFP4_ERR_NULL;
    if ((reinterpret_cast<uintptr_t>(x) & 31u) || !aligned16(w_codes) || !aligned16(w_scales) ||
        (reinterpret_cast<uintptr_t>(y) & 31u) ||
        !aligned4(x_amax) || !aligned4(w_tscale) || !aligned4(status))
        return NVFP4_ERR_ALIGN;
    if (k == 0) return NVFP4_ERR_SHAPE;
    CUtensorMap ma, mb;
    memset(&ma, 0, sizeof(ma));
    if (!codes_map(&mb, w_codes, n, k / 2, kBN)) return NVFP4_ERR_CUDA;
    GemmParams p{};
    p.x = x;
    p.x_amax = x_amax;
    p.w_scales = w_scales;
    p.w_tscale = w_tscale;
    p.y = y;
    p.status = status;
    p.m = m;
    p.n = n;
    p.k = k;
    if (mode == NVFP4_SCALE6) return launch_gemm<true, false, kMse>(ma, mb, p, stream);
    switch (rule) {
        case NVFP4_RULE_MAXERR: return launch_gemm<true, true, kMaxErr>(ma, mb, p, stream);
        case NVFP4_RULE_MAE: return launch_gemm<true, true, kMae>(ma, mb, p, stream);
        default: return launch_gemm<true, true, kMse>(ma, mb, p, stream);
    }
}
