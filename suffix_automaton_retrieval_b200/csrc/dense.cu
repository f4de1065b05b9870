// Streaming kernels of the ROSA retrieval step: binary discretisation with
// multi-route packing, and the read-out (gather) of value rows at tau.
//
// "ROSA-Tuning" (arXiv 2602.02499): section 3.2 Eqs. (10)-(15) for the
// discretisation, section 4.1 for the route layout (channel c = r*M + j),
// appendix C.4 and Eq. (17) for the read-out and its mask.
//
// Both kernels are HBM-bound copies/reductions: 16-byte vector loads where
// alignment allows, shared-memory staging so that both the read and the
// write side are coalesced, streaming stores for outputs nobody re-reads.
#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "common.cuh"
#include "kernels.h"

namespace rosa {

// ---------------------------------------------------------------------------
// Discretisation
// ---------------------------------------------------------------------------

namespace {

constexpr int kDiscTT = 32;     // positions per tile
constexpr int kDiscCC = 512;    // channel budget per tile (rounded down to a multiple of M)
constexpr int kDiscThreads = 256;

__device__ __forceinline__ uint8_t positive_bit(uint16_t h) {
    // I[x > 0] on the bf16 value: the exact float conversion then a strict compare.
    return __bfloat162float(__ushort_as_bfloat16(h)) > 0.0f ? 1 : 0;
}

// grid: (t tiles, channel tiles, B x tensors); tensor i = blockIdx.z / B
// reads x_i and writes sym_i (the query and key projections share a launch).
__global__ void __launch_bounds__(kDiscThreads)
discretize_kernel(const uint16_t *__restrict__ x0, const uint16_t *__restrict__ x1, int B, int T, int C, int M,
                  int CC, bool vec, uint8_t *__restrict__ sym0, uint8_t *__restrict__ sym1) {
    // rows padded by one word: the packing phase reads a column (32 positions of
    // one channel), which would otherwise hit a single bank 32 times
    __shared__ uint8_t bits[kDiscTT][kDiscCC + 4];
    const int which = blockIdx.z >= (unsigned)B;
    const int b = blockIdx.z - which * B;
    const uint16_t *__restrict__ x = which ? x1 : x0;
    uint8_t *__restrict__ sym = which ? sym1 : sym0;
    const int t0 = blockIdx.x * kDiscTT;
    const int c0 = blockIdx.y * CC;
    const int cc = min(CC, C - c0);
    const int tt = min(kDiscTT, T - t0);
    const uint16_t *xb = x + ((int64_t)b * T + t0) * C + c0;

    if (vec) {
        // cc % 8 == 0 and rows are 16-byte aligned: 8 channels per load.
        const int per_row = cc / 8;
        for (int i = threadIdx.x; i < tt * per_row; i += kDiscThreads) {
            const int r = i / per_row, c8 = i - r * per_row;
            const uint4 w = __ldg(reinterpret_cast<const uint4 *>(xb + (int64_t)r * C) + c8);
            const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
            for (int h = 0; h < 4; ++h) {
                bits[r][c8 * 8 + 2 * h] = positive_bit((uint16_t)(ws[h] & 0xffffu));
                bits[r][c8 * 8 + 2 * h + 1] = positive_bit((uint16_t)(ws[h] >> 16));
            }
        }
    } else {
        for (int i = threadIdx.x; i < tt * cc; i += kDiscThreads) {
            const int r = i / cc, c = i - r * cc;
            bits[r][c] = positive_bit(xb[(int64_t)r * C + c]);
        }
    }
    __syncthreads();

    // One symbol per (route, position); consecutive threads take consecutive
    // positions so each warp writes 32 consecutive bytes of one route row.
    const int routes = cc / M;
    const int R = C / M;
    const int r0 = c0 / M;
    for (int i = threadIdx.x; i < routes * kDiscTT; i += kDiscThreads) {
        const int rl = i / kDiscTT, t = i - rl * kDiscTT;
        if (t >= tt) continue;
        unsigned a = 0;
        for (int j = 0; j < M; ++j) a |= (unsigned)bits[t][rl * M + j] << j;
        sym[((int64_t)b * R + r0 + rl) * T + t0 + t] = (uint8_t)a;
    }
}

}  // namespace

cudaError_t launch_discretize(const uint16_t *const *x, uint8_t *const *sym, int count, int B, int T, int C,
                              int M, cudaStream_t stream) {
    if (B == 0 || T == 0 || count < 1) return cudaSuccess;
    int CC = (kDiscCC / M) * M;
    if (CC > C) CC = C;
    // vector path: every tile starts on a 16-byte boundary and covers whole 8-channel groups
    bool vec = (C % 8 == 0) && (CC % 8 == 0);
    for (int i = 0; i < count; ++i) vec = vec && (reinterpret_cast<uintptr_t>(x[i]) % 16 == 0);
    dim3 grid((unsigned)ceil_div(T, kDiscTT), (unsigned)ceil_div(C, CC), (unsigned)(B * count));
    discretize_kernel<<<grid, kDiscThreads, 0, stream>>>(x[0], x[count - 1], B, T, C, M, CC, vec, sym[0],
                                                         sym[count - 1]);
    return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// Gather (read-out at tau)
// ---------------------------------------------------------------------------

namespace {

constexpr int kGatherTT = 8;        // positions per tile: one 32-byte sector of end_idx per route
constexpr int kGatherRC = 512;      // routes staged per pass
constexpr int kGatherThreads = 256;

__device__ __forceinline__ uint4 ld_nc_v4(const void *p) {
    uint4 r;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "l"(p));
    return r;
}

__device__ __forceinline__ void st_cs_v4(void *p, uint4 v) {
    asm volatile("st.global.cs.v4.u32 [%0], {%1,%2,%3,%4};" ::"l"(p), "r"(v.x), "r"(v.y), "r"(v.z),
                 "r"(v.w)
                 : "memory");
}

// grid: (t tiles, B).  16-byte path: d, rho, row stride multiples of 8 elements.
__global__ void __launch_bounds__(kGatherThreads)
gather_kernel_v4(const uint16_t *__restrict__ V, int64_t vrow, int64_t rho,
                 const int32_t *__restrict__ end_idx, int R, int T, int d,
                 uint16_t *__restrict__ out) {
    __shared__ int32_t tau_s[kGatherRC][kGatherTT];
    const int b = blockIdx.y;
    const int t0 = blockIdx.x * kGatherTT;
    const int tt = min(kGatherTT, T - t0);
    const int d8 = d / 8;
    for (int rb = 0; rb < R; rb += kGatherRC) {
        const int rc = min(kGatherRC, R - rb);
        __syncthreads();
        for (int i = threadIdx.x; i < rc * kGatherTT; i += kGatherThreads) {
            const int r = i / kGatherTT, t = i - r * kGatherTT;
            tau_s[r][t] = (t < tt) ? end_idx[((int64_t)b * R + rb + r) * T + t0 + t] : -1;
        }
        __syncthreads();
        const int per_t = rc * d8;                   // 16-byte chunks per position and pass
        const int total = tt * per_t;
        for (int i0 = threadIdx.x; i0 < total; i0 += 4 * kGatherThreads) {
            uint4 v[4];
            uint16_t *dst[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int i = i0 + u * kGatherThreads;
                dst[u] = nullptr;
                if (i < total) {
                    const int t = i / per_t, rem = i - t * per_t;
                    const int r = rem / d8, m8 = rem - r * d8;
                    const int e = tau_s[r][t];
                    dst[u] = out + (((int64_t)b * T + t0 + t) * R + rb + r) * d + m8 * 8;
                    if (e >= 0 && e < T - 1) {
                        const uint16_t *src = V + ((int64_t)b * T + e + 1) * vrow + (int64_t)(rb + r) * rho + m8 * 8;
                        v[u] = ld_nc_v4(src);
                    } else {
                        v[u] = make_uint4(0, 0, 0, 0);
                    }
                }
            }
#pragma unroll
            for (int u = 0; u < 4; ++u)
                if (dst[u]) st_cs_v4(dst[u], v[u]);
        }
    }
}

// Element-wise fallback for shapes or pointers that break 16-byte alignment.
__global__ void __launch_bounds__(kGatherThreads)
gather_kernel_scalar(const uint16_t *__restrict__ V, int64_t vrow, int64_t rho,
                     const int32_t *__restrict__ end_idx, int R, int T, int d,
                     uint16_t *__restrict__ out) {
    const int b = blockIdx.y;
    const int t0 = blockIdx.x * kGatherTT;
    const int tt = min(kGatherTT, T - t0);
    const int64_t per_t = (int64_t)R * d;
    for (int64_t i = threadIdx.x; i < tt * per_t; i += kGatherThreads) {
        const int t = (int)(i / per_t);
        const int64_t rem = i - t * per_t;
        const int r = (int)(rem / d), m = (int)(rem - (int64_t)r * d);
        const int e = end_idx[((int64_t)b * R + r) * T + t0 + t];
        uint16_t val = 0;
        if (e >= 0 && e < T - 1) val = V[((int64_t)b * T + e + 1) * vrow + (int64_t)r * rho + m];
        out[((int64_t)b * T + t0 + t) * per_t + rem] = val;
    }
}

}  // namespace

cudaError_t launch_gather(const uint16_t *V, int64_t vrow, int64_t rho, const int32_t *end_idx,
                          int B, int R, int T, int d, uint16_t *out, cudaStream_t stream) {
    if (B == 0 || T == 0 || R == 0) return cudaSuccess;
    dim3 grid((unsigned)ceil_div(T, kGatherTT), (unsigned)B);
    const bool vec = (d % 8 == 0) && (rho % 8 == 0) && (vrow % 8 == 0) &&
                     (reinterpret_cast<uintptr_t>(V) % 16 == 0) && (reinterpret_cast<uintptr_t>(out) % 16 == 0);
    if (vec)
        gather_kernel_v4<<<grid, kGatherThreads, 0, stream>>>(V, vrow, rho, end_idx, R, T, d, out);
    else
        gather_kernel_scalar<<<grid, kGatherThreads, 0, stream>>>(V, vrow, rho, end_idx, R, T, d, out);
    return cudaGetLastError();
}

}  // namespace rosa
