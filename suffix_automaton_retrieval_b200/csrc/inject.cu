// Read-out embedding and injection on the tensor cores.
//
// "ROSA-Tuning" (arXiv 2602.02499), appendix C.3 (Eqs. 21-22 of the main
// text) with the Eq. (17) mask: the value symbol recalled for route r at
// position (b, t) gives one bit b^ per channel c = r*M + j, the mask
// m = I[tau >= 0], the embedding y_c = m((1 - b^) e0_c + b^ e1_c), and the
// injection inj = W_out y.
//
// One CTA computes a 128-row x BN-column tile of inj (rows are positions
// b*T + t).  For every 64-channel block of K it builds the A tile (y, bf16)
// directly in shared memory from the recalled symbols, so the embedding
// never touches global memory, stages the matching W_out block, and one
// thread issues four tcgen05 MMAs (M = 128, N = BN, K = 16 each) into an
// fp32 accumulator in tensor memory.  The epilogue reads the accumulator
// back with tcgen05.ld, rounds to bf16 and stores the rows.
#include <cstdint>
#include <cstring>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "../../include/rosa.h"
#include "common.cuh"
#include "kernels.h"
#include "umma.cuh"

namespace rosa {
namespace {

constexpr int kInjM = 128;          // rows per tile = UMMA M
constexpr int kInjK = 64;           // channels per K block = one 128-byte swizzle row
constexpr int kInjThreads = 128;    // four warps: one per 32 TMEM lanes in the epilogue
constexpr int kInjMaxN = 256;       // UMMA N limit for M = 128
constexpr uint32_t kWaitPolls = 1u << 24;

struct InjSmem {
    alignas(1024) unsigned char a[kInjM * 128];        // y block, K-major SW128
    alignas(1024) unsigned char b[kInjMaxN * 128];     // W_out block, K-major SW128
    uint16_t e0[kInjK], e1[kInjK];
    int32_t sym[kInjK][kInjM];                         // recalled symbols of the block's routes, per row
    uint64_t mbar;
    uint32_t tmem;
    int failed;
};

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<const uint32_t *>(&v);
}

__global__ void __launch_bounds__(kInjThreads, 1)
inject_kernel(const __grid_constant__ CUtensorMap tmOut, bool tma_out, const int32_t *__restrict__ sym,
              const uint16_t *__restrict__ e0, const uint16_t *__restrict__ e1, const uint16_t *__restrict__ W, int R,
              int M, int T, int D, int BN, int64_t P, bool wvec, uint16_t *__restrict__ out,
              uint32_t *__restrict__ status) {
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    InjSmem &sm = *reinterpret_cast<InjSmem *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int C = R * M;
    const int64_t p0 = (int64_t)blockIdx.x * kInjM;
    const int n0 = blockIdx.y * BN;
    const uint32_t ncols = BN <= 32 ? 32 : (BN <= 64 ? 64 : (BN <= 128 ? 128 : 256));

    if (tid == 0) {
        umma::mbar_init(&sm.mbar, 1);
        umma::fence_mbar_init();
        sm.failed = 0;
    }
    if (warp == 0) umma::tmem_alloc(&sm.tmem, ncols);
    umma::tc_fence_before();
    __syncthreads();
    umma::tc_fence_after();
    const uint32_t tmem = sm.tmem;

    // this thread's row of A: position p = b*T + t
    const int64_t p = p0 + tid;
    const bool row_ok = p < P;
    int64_t sym_row = 0;   // sym index of route 0 at this position
    if (row_ok) {
        const int64_t b = p / T;
        sym_row = b * (int64_t)R * T + (p - b * T);
    }
    const uint32_t idesc = umma::make_idesc_bf16_f32(kInjM, BN);
    const int nkb = ceil_div(C, kInjK);
    for (int kb = 0; kb < nkb; ++kb) {
        const int k0 = kb * kInjK;
        if (tid < kInjK) {
            const int c = k0 + tid;
            sm.e0[tid] = c < C ? e0[c] : 0;
            sm.e1[tid] = c < C ? e1[c] : 0;
        }
        // the symbols of this block's routes for this row: independent loads,
        // coalesced across the warp (consecutive rows are consecutive t)
        const int r0 = k0 / M, nr = min(C - 1, k0 + kInjK - 1) / M - r0 + 1;   // routes touched, <= 64
#pragma unroll 8
        for (int i = 0; i < kInjK; ++i)
            if (i < nr) sm.sym[i][tid] = row_ok ? sym[sym_row + (int64_t)(r0 + i) * T] : -1;
        __syncthreads();
        // A: the embedding of this row's 64 channels, eight per 16-byte chunk
#pragma unroll
        for (int ch = 0; ch < 8; ++ch) {
            uint32_t w[4];
#pragma unroll
            for (int h = 0; h < 4; ++h) {
                uint16_t v2[2];
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const int kk = ch * 8 + h * 2 + e;
                    const int c = k0 + kk;
                    uint16_t v = 0;
                    if (c < C) {
                        const int r = c / M;
                        const int32_t a = sm.sym[r - r0][tid];
                        if (a >= 0) v = ((a >> (c - r * M)) & 1) ? sm.e1[kk] : sm.e0[kk];
                    }
                    v2[e] = v;
                }
                w[h] = (uint32_t)v2[0] | ((uint32_t)v2[1] << 16);
            }
            *reinterpret_cast<uint4 *>(sm.a + umma::sw128_offset(tid, ch * 8)) = make_uint4(w[0], w[1], w[2], w[3]);
        }
        // B: rows n0 .. n0+BN-1 of W_out, channels k0 .. k0+63 (zeros outside)
#pragma unroll 16
        for (int i = tid; i < BN * 8; i += kInjThreads) {
            const int nr = i >> 3, ch = i & 7;
            const int n = n0 + nr, c = k0 + ch * 8;
            uint4 v = make_uint4(0, 0, 0, 0);
            if (n < D) {
                const uint16_t *src = W + (int64_t)n * C + c;
                if (wvec && c + 8 <= C) {
                    v = __ldg(reinterpret_cast<const uint4 *>(src));
                } else {
                    uint16_t t8[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) t8[e] = (c + e < C) ? src[e] : 0;
                    v = make_uint4(t8[0] | (t8[1] << 16), t8[2] | (t8[3] << 16), t8[4] | (t8[5] << 16),
                                   t8[6] | ((uint32_t)t8[7] << 16));
                }
            }
            *reinterpret_cast<uint4 *>(sm.b + umma::sw128_offset(nr, ch * 8)) = v;
        }
        umma::fence_async_smem();
        __syncthreads();
        if (tid == 0) {
            umma::tc_fence_after();
            const uint32_t abase = umma::smem_u32(sm.a), bbase = umma::smem_u32(sm.b);
#pragma unroll
            for (int kk = 0; kk < kInjK / 16; ++kk)
                umma::mma_bf16(tmem, umma::make_kmajor_sw128_desc(abase + kk * 32),
                               umma::make_kmajor_sw128_desc(bbase + kk * 32), idesc, (kb > 0 || kk > 0) ? 1u : 0u);
            umma::mma_commit(&sm.mbar);
        }
        // the tiles are rewritten by the next block: wait for the MMAs to finish reading them
        if (!umma::mbar_wait_bounded(&sm.mbar, (uint32_t)(kb & 1), kWaitPolls)) sm.failed = 1;
        __syncthreads();
        if (sm.failed) break;
    }
    umma::tc_fence_after();
    if (!sm.failed && tma_out) {
        // epilogue through shared memory: each 64-column box of the tile is
        // written row by row (thread = row) in the 128-byte swizzle, so the
        // eight 16-byte chunks of consecutive rows fall in distinct banks, and
        // leaves in one TMA store (rows and columns past the output are clipped).
        // The operand tiles are free now: three box buffers (A, then B twice).
        unsigned char *bufs[3] = {sm.a, sm.b, sm.b + kInjM * 128};
        const uint32_t trow = tmem + ((uint32_t)(warp * 32) << 16);
        for (int c0 = 0, box = 0; c0 < BN && n0 + c0 < D; c0 += 64, ++box) {
            unsigned char *buf = bufs[box % 3];
            if (box >= 3) {   // the buffer's previous store must have read it
                if (tid == 0) umma::tma_store_wait_read();
                __syncthreads();
            }
            uint32_t r[32], w[32];
            umma::tmem_ld_32cols(trow + (uint32_t)c0, r);
#pragma unroll
            for (int j = 0; j < 16; ++j) w[j] = pack_bf16x2(__uint_as_float(r[2 * j]), __uint_as_float(r[2 * j + 1]));
            umma::tmem_ld_32cols(trow + (uint32_t)(c0 + 32), r);
#pragma unroll
            for (int j = 0; j < 16; ++j)
                w[16 + j] = pack_bf16x2(__uint_as_float(r[2 * j]), __uint_as_float(r[2 * j + 1]));
#pragma unroll
            for (int ch = 0; ch < 8; ++ch)
                *reinterpret_cast<uint4 *>(buf + umma::sw128_offset(tid, ch * 8)) =
                    make_uint4(w[4 * ch], w[4 * ch + 1], w[4 * ch + 2], w[4 * ch + 3]);
            umma::fence_async_smem();
            __syncthreads();
            if (tid == 0) umma::tma_store_2d(&tmOut, n0 + c0, (int)p0, buf);
        }
        if (tid == 0) umma::tma_store_wait_read();
    } else if (!sm.failed) {
        // epilogue: warp w owns rows 32w .. 32w+31 of the tile (TMEM lanes)
        const int64_t row = p0 + warp * 32 + lane;
        const bool vec = (D % 8) == 0;
        for (int c0 = 0; c0 < BN; c0 += 32) {
            uint32_t r[32];
            umma::tmem_ld_32cols(tmem + ((uint32_t)(warp * 32) << 16) + (uint32_t)c0, r);
            if (row >= P) continue;
            uint16_t *dst = out + row * D + n0 + c0;
            const int left = D - (n0 + c0);
            if (vec && left >= 32) {
#pragma unroll
                for (int q4 = 0; q4 < 4; ++q4) {
                    uint4 v;
                    v.x = pack_bf16x2(__uint_as_float(r[q4 * 8 + 0]), __uint_as_float(r[q4 * 8 + 1]));
                    v.y = pack_bf16x2(__uint_as_float(r[q4 * 8 + 2]), __uint_as_float(r[q4 * 8 + 3]));
                    v.z = pack_bf16x2(__uint_as_float(r[q4 * 8 + 4]), __uint_as_float(r[q4 * 8 + 5]));
                    v.w = pack_bf16x2(__uint_as_float(r[q4 * 8 + 6]), __uint_as_float(r[q4 * 8 + 7]));
                    reinterpret_cast<uint4 *>(dst)[q4] = v;
                }
            } else {
                for (int j = 0; j < 32 && j < left; ++j) {
                    const __nv_bfloat16 h = __float2bfloat16_rn(__uint_as_float(r[j]));
                    dst[j] = *reinterpret_cast<const uint16_t *>(&h);
                }
            }
        }
    } else if (tid == 0 && status) {
        atomicOr(status, ROSA_DEV_TIMEOUT);
    }
    umma::tc_fence_before();
    __syncthreads();
    if (warp == 0) umma::tmem_dealloc(tmem, ncols);
}

}  // namespace

// Dynamic shared memory of one CTA: the tiles plus alignment slack, and at
// least 80 KB so that no more than two CTAs share an SM (each holds up to
// 256 of its 512 TMEM columns).
size_t inject_smem_bytes() {
    const size_t need = sizeof(InjSmem) + 1024;
    return need > (80u << 10) ? need : (80u << 10);
}

cudaError_t launch_inject(const int32_t *sym, const uint16_t *e0, const uint16_t *e1, const uint16_t *W, int B, int R,
                          int M, int T, int D, uint16_t *out, uint32_t *status, cudaStream_t st) {
    const int64_t P = (int64_t)B * T;
    if (P == 0 || D == 0) return cudaSuccess;
    static bool attr_done[64] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const int smem = (int)inject_smem_bytes();
    if (dev < 0 || dev >= 64 || !attr_done[dev]) {
        e = cudaFuncSetAttribute(inject_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e != cudaSuccess) return e;
        if (dev >= 0 && dev < 64) attr_done[dev] = true;
    }
    // N tile: all of D when it fits one MMA, else 256 (a multiple of 16 in [16, 256])
    int BN = D >= kInjMaxN ? kInjMaxN : ((D + 15) / 16) * 16;
    if (BN < 16) BN = 16;
    const int C = R * M;
    const bool wvec = (C % 8 == 0) && (reinterpret_cast<uintptr_t>(W) % 16 == 0);
    // the output leaves by TMA stores when its rows are 16-byte aligned and BN
    // is a whole number of 64-column boxes
    CUtensorMap tmOut;
    const bool tma_out = (BN % 64 == 0) && make_tmap_bf16_2d(&tmOut, out, (uint64_t)P, (uint64_t)D, kInjM, 64);
    if (!tma_out) memset(&tmOut, 0, sizeof tmOut);
    dim3 grid((unsigned)ceil_div64(P, kInjM), (unsigned)ceil_div(D, BN));
    inject_kernel<<<grid, kInjThreads, smem, st>>>(tmOut, tma_out, sym, e0, e1, W, R, M, T, D, BN, P, wvec, out,
                                                   status);
    return cudaGetLastError();
}

}  // namespace rosa
