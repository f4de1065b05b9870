// Device helpers shared by the kernels of the CUDA path.
#pragma once
#include <cstdint>
#include <cuda_runtime.h>

#define ROSA_FULL_MASK 0xffffffffu

namespace rosa {

__host__ __device__ __forceinline__ int64_t ceil_div64(int64_t a, int64_t b) { return (a + b - 1) / b; }
__host__ __device__ __forceinline__ int ceil_div(int a, int b) { return (a + b - 1) / b; }

__device__ __forceinline__ unsigned lanemask_lt() {
    unsigned m;
    asm volatile("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
    return m;
}

// Exclusive prefix sum over one value per thread of a block of exactly
// NT threads (NT a multiple of 32, <= 1024).  `warp_sums` needs NT/32 + 1 slots.
// Returns this thread's exclusive prefix; *total receives the block total.
template <int NT>
__device__ __forceinline__ uint32_t block_exclusive_scan(uint32_t v, uint32_t *warp_sums, uint32_t *total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    uint32_t x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        uint32_t y = __shfl_up_sync(ROSA_FULL_MASK, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) warp_sums[warp] = x;
    __syncthreads();
    if (warp == 0) {
        uint32_t w = (lane < NT / 32) ? warp_sums[lane] : 0;
        uint32_t ws = w;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            uint32_t y = __shfl_up_sync(ROSA_FULL_MASK, ws, o);
            if (lane >= o) ws += y;
        }
        if (lane < NT / 32) warp_sums[lane] = ws - w;   // exclusive warp offsets
        if (lane == NT / 32 - 1) warp_sums[NT / 32] = ws;
    }
    __syncthreads();
    uint32_t r = warp_sums[warp] + x - v;
    if (total) *total = warp_sums[NT / 32];
    __syncthreads();
    return r;
}

}  // namespace rosa
