// nvfp4_api.cu — the C ABI declared in include/nvfp4.h: argument validation, launch
// configuration and kernel dispatch. No allocation, no host synchronization, no state
// beyond a per-device cache of launch limits (and of the dynamic shared-memory allowance set
// once per device for the kernels that hold the 64 KiB decode table).
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cstdint>

#include "../../include/nvfp4.h"
#include "kernels.cuh"

namespace {

using nvfp4::GroupDiv;
using nvfp4::kThreads;

constexpr int kMaxDevices = 64;

// Launch limits of one device: SM count and resident CTAs per SM for each kernel family.
struct DeviceInfo {
    std::atomic<int> sms{0};
};
DeviceInfo g_dev[kMaxDevices];

int sm_count() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) return 148;
    if (dev >= kMaxDevices) {
        int n = 0;
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
        return n > 0 ? n : 148;
    }
    int n = g_dev[dev].sms.load(std::memory_order_relaxed);
    if (n == 0) {
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
        g_dev[dev].sms.store(n, std::memory_order_relaxed);
    }
    return n;
}

// Resident CTAs per SM for a kernel, cached per kernel and device. The kernel is a template
// argument so that every kernel gets its own cache: the quantizer's instantiations share one
// function type, and a cache keyed by the type would hand one kernel's occupancy to another.
template <auto kernel>
int ctas_per_sm(size_t dyn_smem = 0) {
    static std::atomic<int> cache[kMaxDevices];
    int dev = 0;
    cudaGetDevice(&dev);
    int v = (dev >= 0 && dev < kMaxDevices) ? cache[dev].load(std::memory_order_relaxed) : 0;
    if (v == 0) {
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&v, kernel, kThreads, dyn_smem) != cudaSuccess || v <= 0)
            v = 1;
        if (dev >= 0 && dev < kMaxDevices) cache[dev].store(v, std::memory_order_relaxed);
    }
    return v;
}

// Dynamic shared memory of the grouped quantizer: the decode table for Four Over Six codes.
template <bool FOUR, bool FQ>
constexpr size_t quant_dyn_smem() { return (FOUR && !FQ) ? nvfp4::kDecodeTableBytes : 0; }

// Lets `kernel` use `bytes` of dynamic shared memory on the current device (set once per device).
template <auto kernel>
bool allow_dyn_smem(size_t bytes) {
    if (bytes <= 48 * 1024) return true;
    static std::atomic<int> done[kMaxDevices];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) return false;
    if (dev < kMaxDevices && done[dev].load(std::memory_order_acquire)) return true;
    if (cudaFuncSetAttribute(reinterpret_cast<const void*>(kernel), cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(bytes)) != cudaSuccess) {
        cudaGetLastError();
        return false;
    }
    if (dev < kMaxDevices) done[dev].store(1, std::memory_order_release);
    return true;
}

// Persistent grid: enough CTAs to fill every SM at full occupancy, never more than the work.
template <auto kernel>
unsigned grid_for(int64_t work_items) {
    const int64_t full = static_cast<int64_t>(sm_count()) * ctas_per_sm<kernel>();
    const int64_t need = (work_items + kThreads - 1) / kThreads;
    const int64_t g = need < full ? need : full;
    return static_cast<unsigned>(g < 1 ? 1 : g);
}

GroupDiv make_gdiv(int64_t groups, int64_t bpg, int64_t nblocks) {
    GroupDiv d{};
    d.bpg = bpg;
    if (groups == 1) {
        d.mode = 0;
    } else if (bpg == 1) {
        d.mode = 1;
    } else if (nblocks < (int64_t(1) << 31) && bpg < (int64_t(1) << 31)) {
        // q = floor(b * m / 2^(31 + l)) with m = ceil(2^(31 + l) / bpg), l = ceil(log2 bpg):
        // exact for every b < 2^31, and m < 2^32 because bpg > 2^(l - 1).
        uint32_t l = 0;
        while ((int64_t(1) << l) < bpg) ++l;
        const unsigned __int128 num = (unsigned __int128)1 << (31 + l);
        d.mul = static_cast<uint32_t>((num + bpg - 1) / bpg);
        d.shift = l - 1;
        d.mode = 2;
    } else {
        d.mode = 3;
    }
    return d;
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

// Shared shape check. Returns NVFP4_OK and the element count, or an error.
nvfp4_status check_shape(int64_t groups, int64_t rows, int64_t cols, int64_t* numel) {
    if (groups < 1 || rows < 0 || cols < 0 || cols % 16 != 0) return NVFP4_ERR_SHAPE;
    const int64_t lim = int64_t(1) << 62;
    if (rows > 0 && cols > lim / rows) return NVFP4_ERR_SHAPE;
    const int64_t per = rows * cols;
    if (per > 0 && groups > lim / per) return NVFP4_ERR_SHAPE;
    *numel = groups * per;
    return NVFP4_OK;
}

nvfp4_status launch_status() {
    return cudaGetLastError() == cudaSuccess ? NVFP4_OK : NVFP4_ERR_CUDA;
}

// Grid of the grouped quantize kernel (one row of CTAs): one group takes enough CTAs for one
// warp tile per warp, at most `full` (the resident CTAs); several groups take one CTA per
// resident slot, at most one per warp tile of the whole tensor, and the kernel splits the
// tiles of all groups into equal contiguous ranges.
dim3 grouped_grid(int64_t full, int64_t groups, int64_t bpg) {
    constexpr int64_t kWarps = kThreads / 32;
    const int64_t ntiles = (bpg + 63) / 64;
    const int64_t want = groups == 1 ? (ntiles + kWarps - 1) / kWarps : groups * ntiles;
    return dim3(static_cast<unsigned>(std::max<int64_t>(1, std::min(full, want))), 1u);
}

template <bool FOUR, int RULE, bool FQ>
nvfp4_status launch_quant(const nvfp4::QuantParams& p, cudaStream_t stream) {
    const int64_t bpg = p.gdiv.bpg;
    const bool grouped = (p.groups == 1 || bpg % 32 == 0) && bpg < (int64_t(1) << 30);
    if (grouped) {
        // CTAs work inside one group at a time, with the group's scale table in shared memory
        constexpr auto kernel = nvfp4::quantize_grouped_kernel<FOUR, RULE, FQ>;
        constexpr size_t dyn = quant_dyn_smem<FOUR, FQ>();
        if (!allow_dyn_smem<kernel>(dyn)) return NVFP4_ERR_CUDA;
        const dim3 grid = grouped_grid(static_cast<int64_t>(sm_count()) * ctas_per_sm<kernel>(dyn), p.groups, bpg);
        kernel<<<grid, kThreads, dyn, stream>>>(p);
    } else {
        constexpr auto kernel = nvfp4::quantize_kernel<FOUR, RULE, FQ>;
        const unsigned grid = grid_for<kernel>(p.nblocks);
        kernel<<<grid, kThreads, 0, stream>>>(p);
    }
    return launch_status();
}

template <bool FQ>
nvfp4_status dispatch_quant(nvfp4_mode mode, nvfp4_rule rule, const nvfp4::QuantParams& p, cudaStream_t s) {
    if (mode == NVFP4_SCALE6) return launch_quant<false, nvfp4::kMse, FQ>(p, s);
    switch (rule) {
        case NVFP4_RULE_MAXERR: return launch_quant<true, nvfp4::kMaxErr, FQ>(p, s);
        case NVFP4_RULE_MAE: return launch_quant<true, nvfp4::kMae, FQ>(p, s);
        default: return launch_quant<true, nvfp4::kMse, FQ>(p, s);
    }
}

// Internal: a cooperative or cluster launch was refused, and the caller takes its other path.
constexpr nvfp4_status NVFP4_ERR_UNSUPPORTED_LAUNCH = static_cast<nvfp4_status>(1000);

// Scratch of nvfp4_amax_quantize / nvfp4_amax_fakequant calls made without a workspace: the
// grid-wide barrier's arrival counter, one 32-bit word (the most any call needs, whatever the
// tensor's size). A __device__ variable exists once on every device that loads the library and
// lives until the process exits, so these calls allocate nothing; calls that use it must not
// overlap on the GPU (they would share the counter).
constexpr int kNoAllocScratchWords = 1;
static __device__ __align__(256) uint32_t g_amax_quant_scratch[kNoAllocScratchWords];

// Device address of g_amax_quant_scratch on the current device. In host code the symbol is a
// host-side stand-in, not a device address, so it is looked up once per device (with that
// device current: the first call on a device does it) and cached.
nvfp4_status noalloc_scratch(uint32_t** out) {
    static std::atomic<uintptr_t> addr[kMaxDevices];
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) return NVFP4_ERR_CUDA;
    uintptr_t a = dev < kMaxDevices ? addr[dev].load(std::memory_order_acquire) : 0;
    if (a == 0) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_amax_quant_scratch) != cudaSuccess || p == nullptr) {
            cudaGetLastError();
            return NVFP4_ERR_CUDA;
        }
        a = reinterpret_cast<uintptr_t>(p);
        if (dev < kMaxDevices) addr[dev].store(a, std::memory_order_release);
    }
    *out = reinterpret_cast<uint32_t*>(a);
    return NVFP4_OK;
}

template <bool FOUR, int RULE, bool FQ>
nvfp4_status launch_quant_amax(const nvfp4::QuantParams& p, uint32_t* arrive, uint32_t* status, cudaStream_t stream) {
    constexpr auto kernel = nvfp4::quantize_amax_kernel<FOUR, RULE, FQ>;
    // every CTA must be resident for the grid-wide barrier: a cooperative launch of at most
    // the resident CTAs (it fails instead of hanging if they do not fit)
    const dim3 grid = grouped_grid(static_cast<int64_t>(sm_count()) * ctas_per_sm<kernel>(), p.groups, p.gdiv.bpg);
    nvfp4::QuantParams pp = p;
    uint32_t expected = grid.x;   // every CTA of the grid arrives at the barrier
    void* args[] = {&pp, &arrive, &status, &expected};
    if (cudaLaunchCooperativeKernel(reinterpret_cast<const void*>(kernel), grid, dim3(kThreads), args, 0, stream) !=
        cudaSuccess) {
        cudaGetLastError();   // refused (e.g. the grid cannot be resident): the caller runs two launches
        return NVFP4_ERR_UNSUPPORTED_LAUNCH;
    }
    return launch_status();
}

template <bool FQ>
nvfp4_status dispatch_quant_amax(nvfp4_mode mode, nvfp4_rule rule, const nvfp4::QuantParams& p, uint32_t* arrive,
                                 uint32_t* status, cudaStream_t s) {
    if (mode == NVFP4_SCALE6) return launch_quant_amax<false, nvfp4::kMse, FQ>(p, arrive, status, s);
    switch (rule) {
        case NVFP4_RULE_MAXERR: return launch_quant_amax<true, nvfp4::kMaxErr, FQ>(p, arrive, status, s);
        case NVFP4_RULE_MAE: return launch_quant_amax<true, nvfp4::kMae, FQ>(p, arrive, status, s);
        default: return launch_quant_amax<true, nvfp4::kMse, FQ>(p, arrive, status, s);
    }
}

template <bool FOUR, int RULE>
nvfp4_status launch_quant_gemm(const nvfp4::QuantParams& p, cudaStream_t stream) {
    constexpr auto kernel = nvfp4::quantize_grouped_kernel<FOUR, RULE, false, true>;
    constexpr size_t dyn = quant_dyn_smem<FOUR, false>();
    if (!allow_dyn_smem<kernel>(dyn)) return NVFP4_ERR_CUDA;
    kernel<<<grouped_grid(static_cast<int64_t>(sm_count()) * ctas_per_sm<kernel>(dyn), 1, p.nblocks), kThreads,
             dyn, stream>>>(p);
    return launch_status();
}

nvfp4_status dispatch_quant_gemm(nvfp4_mode mode, nvfp4_rule rule, const nvfp4::QuantParams& p, cudaStream_t s) {
    if (mode == NVFP4_SCALE6) return launch_quant_gemm<false, nvfp4::kMse>(p, s);
    switch (rule) {
        case NVFP4_RULE_MAXERR: return launch_quant_gemm<true, nvfp4::kMaxErr>(p, s);
        case NVFP4_RULE_MAE: return launch_quant_gemm<true, nvfp4::kMae>(p, s);
        default: return launch_quant_gemm<true, nvfp4::kMse>(p, s);
    }
}

nvfp4_status check_mode_rule(nvfp4_mode mode, nvfp4_rule rule) {
    if (mode != NVFP4_SCALE6 && mode != NVFP4_FOUR_OVER_SIX) return NVFP4_ERR_MODE;
    if (mode == NVFP4_FOUR_OVER_SIX && rule != NVFP4_RULE_MAXERR && rule != NVFP4_RULE_MAE && rule != NVFP4_RULE_MSE)
        return NVFP4_ERR_RULE;
    return NVFP4_OK;
}

// alpha_g = amax_g / (6 M) for empty tensors (no blocks to quantize).
__global__ void tensor_scale_only_kernel(const float* amax, float* tscale, int64_t groups, float six_m) {
    for (int64_t g = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; g < groups; g += int64_t(gridDim.x) * blockDim.x)
        tscale[g] = __fdiv_rn(amax[g], six_m);
}

// nvfp4_amax_quantize (y == nullptr) and nvfp4_amax_fakequant (y != nullptr).
nvfp4_status amax_quant_impl(const uint16_t* x, int64_t groups, int64_t rows, int64_t cols, nvfp4_mode mode,
                             nvfp4_rule rule, float* amax, uint8_t* codes, uint8_t* scales, float* tscale,
                             uint16_t* y, uint8_t* choice, uint32_t* workspace, uint32_t* status, cudaStream_t stream) {
    const bool fq = y != nullptr;
    if (amax == nullptr || (!fq && tscale == nullptr)) return NVFP4_ERR_NULL;
    int64_t n = 0;
    nvfp4_status st = check_shape(groups, rows, cols, &n);
    if (st != NVFP4_OK) return st;
    if (n > 0 && (x == nullptr || (!fq && (codes == nullptr || scales == nullptr)))) return NVFP4_ERR_NULL;
    st = check_mode_rule(mode, rule);
    if (st != NVFP4_OK) return st;
    if (!aligned(amax, 4) || (tscale && !aligned(tscale, 4)) || (choice && !aligned(choice, 4)) ||
        (workspace && !aligned(workspace, 4)) || (status && !aligned(status, 4)))
        return NVFP4_ERR_ALIGN;
    if (n > 0 && (!aligned(x, 32) || (!fq && !aligned(codes, 8)) || (fq && !aligned(y, 32)))) return NVFP4_ERR_ALIGN;
    const int64_t bpg = rows * cols / 16;
    if (n == 0 || !((groups == 1 || bpg % 32 == 0) && bpg < (int64_t(1) << 30))) {
        // empty tensors and group layouts the one-launch kernel does not take: the two passes
        st = nvfp4_amax(x, groups, rows, cols, amax, stream);
        if (st != NVFP4_OK) return st;
        return fq ? nvfp4_fakequant(x, groups, rows, cols, amax, mode, rule, y, choice, stream)
                  : nvfp4_quantize(x, groups, rows, cols, amax, mode, rule, codes, scales, tscale, choice, stream);
    }
    if (workspace == nullptr) {
        st = noalloc_scratch(&workspace);
        if (st != NVFP4_OK) return st;
    }
    if (cudaMemsetAsync(amax, 0, static_cast<size_t>(groups) * sizeof(float), stream) != cudaSuccess ||
        cudaMemsetAsync(workspace, 0, sizeof(uint32_t), stream) != cudaSuccess)
        return NVFP4_ERR_CUDA;
    nvfp4::QuantParams p{};
    p.x = x;
    p.amax = amax;
    p.codes = fq ? nullptr : codes;
    p.scales = fq ? nullptr : scales;
    p.tscale = fq ? nullptr : tscale;
    p.choice = choice;
    p.y = y;
    p.nblocks = n / 16;
    p.choice_bytes = (p.nblocks + 7) / 8;
    p.groups = groups;
    p.gdiv = make_gdiv(groups, bpg, p.nblocks);
    st = fq ? dispatch_quant_amax<true>(mode, rule, p, workspace, status, stream)
            : dispatch_quant_amax<false>(mode, rule, p, workspace, status, stream);
    if (st != NVFP4_ERR_UNSUPPORTED_LAUNCH) return st;
    st = nvfp4_amax(x, groups, rows, cols, amax, stream);   // the two launches
    if (st != NVFP4_OK) return st;
    return fq ? nvfp4_fakequant(x, groups, rows, cols, amax, mode, rule, y, choice, stream)
              : nvfp4_quantize(x, groups, rows, cols, amax, mode, rule, codes, scales, tscale, choice, stream);
}

}  // namespace

extern "C" {

nvfp4_status nvfp4_amax(const uint16_t* x, int64_t groups, int64_t rows, int64_t cols, float* amax,
                        cudaStream_t stream) {
    if (amax == nullptr) return NVFP4_ERR_NULL;
    int64_t n = 0;
    nvfp4_status st = check_shape(groups, rows, cols, &n);
    if (st != NVFP4_OK) return st;
    if (n > 0 && x == nullptr) return NVFP4_ERR_NULL;
    if (!aligned(amax, 4) || (n > 0 && !aligned(x, 32))) return NVFP4_ERR_ALIGN;
    if (cudaMemsetAsync(amax, 0, static_cast<size_t>(groups) * sizeof(float), stream) != cudaSuccess)
        return NVFP4_ERR_CUDA;
    if (n == 0) return launch_status();
    const int64_t chunks = rows * cols / 16;
    const int64_t full = static_cast<int64_t>(sm_count()) * ctas_per_sm<nvfp4::amax_kernel>();
    int64_t per_group = full / groups;
    if (per_group < 1) per_group = 1;
    const int64_t need = (chunks + kThreads - 1) / kThreads;
    if (per_group > need) per_group = need;
    const int64_t gy = groups < 65535 ? groups : 65535;
    dim3 grid(static_cast<unsigned>(per_group), static_cast<unsigned>(gy));
    nvfp4::amax_kernel<<<grid, kThreads, 0, stream>>>(x, groups, chunks, amax);
    return launch_status();
}

nvfp4_status nvfp4_quantize(const uint16_t* x, int64_t groups, int64_t rows, int64_t cols, const float* amax,
                            nvfp4_mode mode, nvfp4_rule rule, uint8_t* codes, uint8_t* scales, float* tscale,
                            uint8_t* choice, cudaStream_t stream) {
    if (amax == nullptr || tscale == nullptr) return NVFP4_ERR_NULL;
    int64_t n = 0;
    nvfp4_status st = check_shape(groups, rows, cols, &n);
    if (st != NVFP4_OK) return st;
    if (n > 0 && (x == nullptr || codes == nullptr || scales == nullptr)) return NVFP4_ERR_NULL;
    st = check_mode_rule(mode, rule);
    if (st != NVFP4_OK) return st;
    if (!aligned(amax, 4) || !aligned(tscale, 4) || (choice && !aligned(choice, 4))) return NVFP4_ERR_ALIGN;
    if (n > 0 && (!aligned(x, 32) || !aligned(codes, 8))) return NVFP4_ERR_ALIGN;
    const float six_m = mode == NVFP4_FOUR_OVER_SIX ? 1536.0f : 2688.0f;
    if (n == 0) {
        const unsigned grid = static_cast<unsigned>((groups + kThreads - 1) / kThreads < 1024 ? (groups + kThreads - 1) / kThreads : 1024);
        tensor_scale_only_kernel<<<grid, kThreads, 0, stream>>>(amax, tscale, groups, six_m);
        return launch_status();
    }
    nvfp4::QuantParams p{};
    p.x = x;
    p.amax = amax;
    p.codes = codes;
    p.scales = scales;
    p.tscale = tscale;
    p.choice = choice;
    p.y = nullptr;
    p.nblocks = n / 16;
    p.choice_bytes = (p.nblocks + 7) / 8;
    p.groups = groups;
    p.gdiv = make_gdiv(groups, rows * cols / 16, p.nblocks);
    return dispatch_quant<false>(mode, rule, p, stream);
}

nvfp4_status nvfp4_fakequant(const uint16_t* x, int64_t groups, int64_t rows, int64_t cols, const float* amax,
                             nvfp4_mode mode, nvfp4_rule rule, uint16_t* y, uint8_t* choice, cudaStream_t stream) {
    if (amax == nullptr) return NVFP4_ERR_NULL;
    int64_t n = 0;
    nvfp4_status st = check_shape(groups, rows, cols, &n);
    if (st != NVFP4_OK) return st;
    if (n > 0 && (x == nullptr || y == nullptr)) return NVFP4_ERR_NULL;
    st = check_mode_rule(mode, rule);
    if (st != NVFP4_OK) return st;
    if (!aligned(amax, 4) || (choice && !aligned(choice, 4))) return NVFP4_ERR_ALIGN;
    if (n > 0 && (!aligned(x, 32) || !aligned(y, 32))) return NVFP4_ERR_ALIGN;
    if (n == 0) return NVFP4_OK;
    nvfp4::QuantParams p{};
    p.x = x;
    p.amax = amax;
    p.choice = choice;
    p.y = y;
    p.nblocks = n / 16;
    p.choice_bytes = (p.nblocks + 7) / 8;
    p.groups = groups;
    p.gdiv = make_gdiv(groups, rows * cols / 16, p.nblocks);
    return dispatch_quant<true>(mode, rule, p, stream);
}

nvfp4_status nvfp4_amax_quantize(const uint16_t* x, int64_t groups, int64_t rows, int64_t cols, nvfp4_mode mode,
                                 nvfp4_rule rule, float* amax, uint8_t* codes, uint8_t* scales, float* tscale,
                                 uint8_t* choice, uint32_t* workspace, uint32_t* status, cudaStream_t stream) {
    return amax_quant_impl(x, groups, rows, cols, mode, rule, amax, codes, scales, tscale, nullptr, choice, workspace,
                           status, stream);
}

nvfp4_status nvfp4_amax_fakequant(const uint16_t* x, int64_t groups, int64_t rows, int64_t cols, nvfp4_mode mode,
                                  nvfp4_rule rule, float* amax, uint16_t* y, uint8_t* choice, uint32_t* workspace,
                                  uint32_t* status, cudaStream_t stream) {
    if (y == nullptr) {   // y selects the fake-quant variant inside; check it here
        int64_t n = 0;
        const nvfp4_status st = check_shape(groups, rows, cols, &n);
        if (st != NVFP4_OK) return st;
        if (n > 0) return NVFP4_ERR_NULL;
        if (amax == nullptr) return NVFP4_ERR_NULL;
        return nvfp4_amax(x, groups, rows, cols, amax, stream);
    }
    return amax_quant_impl(x, groups, rows, cols, mode, rule, amax, nullptr, nullptr, nullptr, y, choice, workspace,
                           status, stream);
}

nvfp4_status nvfp4_dequantize(const uint8_t* codes, const uint8_t* scales, const float* tscale, int64_t groups,
                              int64_t rows, int64_t cols, uint16_t* y, cudaStream_t stream) {
    int64_t n = 0;
    nvfp4_status st = check_shape(groups, rows, cols, &n);
    if (st != NVFP4_OK) return st;
    if (n == 0) return NVFP4_OK;
    if (codes == nullptr || scales == nullptr || tscale == nullptr || y == nullptr) return NVFP4_ERR_NULL;
    if (!aligned(codes, 8) || !aligned(tscale, 4) || !aligned(y, 32)) return NVFP4_ERR_ALIGN;
    nvfp4::DequantParams p{};
    p.codes = codes;
    p.scales = scales;
    p.tscale = tscale;
    p.y = y;
    p.nblocks = n / 16;
    p.groups = groups;
    p.gdiv = make_gdiv(groups, rows * cols / 16, p.nblocks);
    const unsigned grid = grid_for<nvfp4::dequantize_kernel>((p.nblocks + 1) / 2);   // one pair per thread
    nvfp4::dequantize_kernel<<<grid, kThreads, 0, stream>>>(p);
    return launch_status();
}

nvfp4_status nvfp4_quantize_gemm(const uint16_t* x, int64_t rows, int64_t cols, const float* amax, nvfp4_mode mode,
                                 nvfp4_rule rule, uint8_t* codes, uint8_t* scales, float* tscale, uint8_t* choice,
                                 cudaStream_t stream) {
    if (amax == nullptr || tscale == nullptr) return NVFP4_ERR_NULL;
    int64_t n = 0;
    nvfp4_status st = check_shape(1, rows, cols, &n);
    if (st != NVFP4_OK) return st;
    if (n / 16 >= (int64_t(1) << 30)) return NVFP4_ERR_SHAPE;
    if (n > 0 && (x == nullptr || codes == nullptr || scales == nullptr)) return NVFP4_ERR_NULL;
    st = check_mode_rule(mode, rule);
    if (st != NVFP4_OK) return st;
    if (!aligned(amax, 4) || !aligned(tscale, 4) || (choice && !aligned(choice, 4))) return NVFP4_ERR_ALIGN;
    if (n > 0 && (!aligned(x, 32) || !aligned(codes, 8))) return NVFP4_ERR_ALIGN;
    if (n == 0) {
        const float six_m = mode == NVFP4_FOUR_OVER_SIX ? 1536.0f : 2688.0f;
        tensor_scale_only_kernel<<<1, kThreads, 0, stream>>>(amax, tscale, 1, six_m);
        return launch_status();
    }
    const int64_t bpr = cols / 16;
    const int64_t n_ct = (bpr + 3) / 4;
    const int64_t padded = (rows + 127) / 128 * 128 * n_ct * 4;
    if (cudaMemsetAsync(scales, 0, static_cast<size_t>(padded), stream) != cudaSuccess) return NVFP4_ERR_CUDA;
    nvfp4::QuantParams p{};
    p.x = x;
    p.amax = amax;
    p.codes = codes;
    p.scales = scales;
    p.tscale = tscale;
    p.choice = choice;
    p.nblocks = n / 16;
    p.choice_bytes = (p.nblocks + 7) / 8;
    p.groups = 1;
    p.gdiv = make_gdiv(1, p.nblocks, p.nblocks);
    p.bpr = static_cast<uint32_t>(bpr);
    p.n_ct = static_cast<uint32_t>(n_ct);
    if (bpr > 1) {
        // row = floor(a * m / 2^(31 + l)), m = ceil(2^(31 + l) / bpr), l = ceil(log2 bpr): exact for a < 2^31
        uint32_t l = 0;
        while ((int64_t(1) << l) < bpr) ++l;
        const unsigned __int128 num = (unsigned __int128)1 << (31 + l);
        p.bpr_mul = static_cast<uint32_t>((num + bpr - 1) / bpr);
        p.bpr_shift = l - 1;
    }
    return dispatch_quant_gemm(mode, rule, p, stream);
}

const char* nvfp4_status_string(nvfp4_status status) {
    switch (status) {
        case NVFP4_OK: return "ok";
        case NVFP4_ERR_NULL: return "a required pointer is NULL";
        case NVFP4_ERR_SHAPE: return "invalid shape (groups >= 1, rows/cols >= 0, cols % 16 == 0, size limit)";
        case NVFP4_ERR_ALIGN: return "misaligned pointer (BF16 tensors 32 B, codes 8 B, floats and choice 4 B)";
        case NVFP4_ERR_MODE: return "unknown nvfp4_mode";
        case NVFP4_ERR_RULE: return "unknown nvfp4_rule";
        case NVFP4_ERR_CUDA: return "CUDA runtime error while enqueuing work";
        case NVFP4_ERR_VALUE: return "scalar argument out of range (tau > 0 and finite, grad_scale finite)";
        default: return "unknown nvfp4_status";
    }
}

int nvfp4_version(void) { return 100; }

}  // extern "C"
