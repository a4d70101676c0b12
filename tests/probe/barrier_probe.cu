// barrier_probe.cu — TEST INFRASTRUCTURE: launches the library's one-launch amax + quantize
// kernel (one group, Four Over Six, MSE) with a chosen number of expected arrivals at its
// grid-wide barrier. The library passes the grid size; one more makes the bounded wait run out
// on purpose, so a test can check the timeout path (status bit set, outputs other than amax
// untouched, the launch completes) without faulting or hanging anything. Not part of the
// product library.
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/nvfp4.h"
#include "../../nvfp4_block_scaled_13_b200/csrc/kernels.cuh"

extern "C" int probe_amax_quantize(const uint16_t* x, int64_t rows, int64_t cols, float* amax, uint8_t* codes,
                                   uint8_t* scales, float* tscale, uint8_t* choice, uint32_t* arrive,
                                   uint32_t* status, uint32_t extra, uint32_t* grid_out) {
    const int64_t nb = rows * cols / 16;
    if (rows <= 0 || cols <= 0 || cols % 16 != 0 || nb >= (int64_t(1) << 30)) return -1;
    constexpr auto kernel = nvfp4::quantize_amax_kernel<true, nvfp4::kMse, false>;
    int dev = 0, sms = 0, per_sm = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, nvfp4::kThreads, 0) != cudaSuccess)
        return -2;
    // the library's grid for one group: one warp tile per warp, at most the resident CTAs
    const int64_t ntiles = (nb + 63) / 64, want = (ntiles + 7) / 8, full = int64_t(sms) * per_sm;
    const unsigned grid = static_cast<unsigned>(want < full ? want : full);
    nvfp4::QuantParams p{};
    p.x = x;
    p.amax = amax;
    p.codes = codes;
    p.scales = scales;
    p.tscale = tscale;
    p.choice = choice;
    p.nblocks = nb;
    p.choice_bytes = (nb + 7) / 8;
    p.groups = 1;
    p.gdiv.bpg = nb;
    p.gdiv.mode = 0;
    if (cudaMemset(amax, 0, sizeof(float)) != cudaSuccess || cudaMemset(arrive, 0, sizeof(uint32_t)) != cudaSuccess)
        return -3;
    uint32_t expected = grid + extra;
    void* args[] = {&p, &arrive, &status, &expected};
    *grid_out = grid;
    const cudaError_t e = cudaLaunchCooperativeKernel(reinterpret_cast<const void*>(kernel), dim3(grid),
                                                      dim3(nvfp4::kThreads), args, 0, nullptr);
    return static_cast<int>(e);
}
