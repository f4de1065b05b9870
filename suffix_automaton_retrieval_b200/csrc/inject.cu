// Read-out embedding and injection on the tensor cores.
//
// "ROSA-Tuning" (arXiv 2602.02499), appendix C.3 (Eqs. 21-22 of the main
// text) with the Eq. (17) mask: the value symbol recalled for route r at
// position (b, t) gives one bit b^ per channel c = r*M + j, the mask
// m = I[tau >= 0], the embedding y_c = m((1 - b^) e0_c + b^ e1_c), and the
// injection inj = W_out y.
//
// Main kernel (C <= 512 channels): persistent CTAs, each owning 128-row
// tiles of inj (rows are positions b*T + t).  For a row tile the CTA builds
// the whole A operand (y, bf16, K-major with the 128-byte swizzle) in shared
// memory from the recalled symbols once, so the embedding never touches
// global memory, then walks the output in 128-column tiles: W_out blocks
// arrive by TMA through a three-stage ring, one thread issues the tcgen05
// MMAs into one of two fp32 accumulators in tensor memory, and while the
// tensor cores work on column tile j the eight warps drain tile j-1 (two
// warps per 32 accumulator lanes, one 64-column box each), round to bf16,
// stage the box in the swizzled layout and send it out with a TMA store.
// Wider embeddings (C > 512) use a one-tile-per-CTA kernel.
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
constexpr uint32_t kWaitPolls = umma::kWaitPolls;

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

// One CTA per 128-row x BN-column tile (any C): the A tile is built per
// 64-channel K block, W_out staged by 16-byte loads, four MMAs per block.
__global__ void __launch_bounds__(kInjThreads, 1)
inject_tile_kernel(const __grid_constant__ CUtensorMap tmOut, bool tma_out, const int32_t *__restrict__ sym,
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


// ---- persistent kernel (C <= 512) -------------------------------------------
//
// Warp roles (320 threads):
//   warps 0-7  build the A tile of each row tile, then drain the accumulators
//              of its column tiles (warps w and w + 4 share TMEM lanes
//              32*(w % 4) and take one 64-column box each);
//   warp 8     lane 0 issues the MMAs;
//   warp 9     produces the W_out blocks (lane 0 by TMA, or the whole warp by
//              plain loads when W_out rows are not 16-byte aligned).
// The roles meet only on mbarriers: W_out stage full / empty, accumulator
// full / empty (two accumulators of 128 columns), A full / empty.

constexpr int kIpN = 128;                       // columns per accumulator / column tile
constexpr int kIpWorkers = 256;                 // warps 0-7
constexpr int kIpThreads = kIpWorkers + 64;     // + MMA warp + W_out producer warp
constexpr int kIpStages = 3;                    // W_out blocks in flight
constexpr int kIpMaxKb = 8;                     // K blocks of a resident A tile (C <= 512)
constexpr uint32_t kIpTile = kInjM * 128;       // 16 KB: 128 rows x 64 bf16, K-major SW128

// Shared-memory carve of the persistent kernel, from a 1024-aligned base.
struct IpCarve {
    uint32_t a, w, ob, e0, e1, bars, slot, total;
};

// barriers: wfull[S], wempty[S], accfull[2], accempty[2], afull, aempty, drain
constexpr int kIpBars = 2 * kIpStages + 7;

__host__ __device__ inline IpCarve ip_carve(int nkb) {
    IpCarve c{};
    c.a = 0;
    c.w = c.a + (uint32_t)nkb * kIpTile;
    c.ob = c.w + kIpStages * kIpTile;                // two output boxes (one per worker group)
    c.e0 = c.ob + 2 * kIpTile;
    c.e1 = c.e0 + (uint32_t)nkb * 64 * 2;            // e0, e1 padded with zeros to nkb * 64 channels
    c.bars = c.e1 + (uint32_t)nkb * 64 * 2;          // multiple of 128: 8-byte aligned
    c.slot = c.bars + 8 * kIpBars;
    c.total = c.slot + 16;
    return c;
}

__device__ __forceinline__ void named_bar(int id, int nthreads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(umma::smem_u32(bar)) : "memory");
}

// Bounded wait that also gives up once another role has flagged a failure.
__device__ __forceinline__ bool ip_wait(uint64_t *bar, uint32_t parity, volatile int *failed) {
    for (uint32_t i = 0; i < kWaitPolls; ++i) {
        if (umma::mbar_try_wait(bar, parity)) return true;
        if (*failed) return false;
    }
    *failed = 1;
    return false;
}

// Two bf16 channels of a 32-bit word: e1 where the bit is set, else e0; zero where the mask is clear.
__device__ __forceinline__ uint32_t select_pair(uint32_t z0, uint32_t z1, uint32_t bits, uint32_t mask, int k) {
    const uint32_t bs = (((bits >> k) & 1u) ? 0x0000FFFFu : 0u) | (((bits >> (k + 1)) & 1u) ? 0xFFFF0000u : 0u);
    const uint32_t ms = (((mask >> k) & 1u) ? 0x0000FFFFu : 0u) | (((mask >> (k + 1)) & 1u) ? 0xFFFF0000u : 0u);
    return ((z1 & bs) | (z0 & ~bs)) & ms;
}

__global__ void __launch_bounds__(kIpThreads, 2)
inject_persistent_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmOut, bool tma_w,
                         bool tma_out, const int32_t *__restrict__ sym, const uint16_t *__restrict__ e0,
                         const uint16_t *__restrict__ e1, const uint16_t *__restrict__ W, int R, int M, int T, int D,
                         int64_t P, int nkb, uint16_t *__restrict__ out, uint32_t *__restrict__ status) {
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char *base = reinterpret_cast<unsigned char *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                            ~(uintptr_t)1023);
    const IpCarve cv = ip_carve(nkb);
    unsigned char *sa = base + cv.a, *sw = base + cv.w, *sob = base + cv.ob;
    uint16_t *se0 = reinterpret_cast<uint16_t *>(base + cv.e0), *se1 = reinterpret_cast<uint16_t *>(base + cv.e1);
    uint64_t *wfull = reinterpret_cast<uint64_t *>(base + cv.bars);
    uint64_t *wempty = wfull + kIpStages, *accfull = wfull + 2 * kIpStages, *accempty = accfull + 2;
    uint64_t *afull = accempty + 2, *aempty = afull + 1, *drain = aempty + 1;
    uint32_t *tslot = reinterpret_cast<uint32_t *>(base + cv.slot);
    volatile int *failed = reinterpret_cast<volatile int *>(tslot + 1);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int C = R * M;
    const int nrt = (int)ceil_div64(P, kInjM), NJ = ceil_div(D, kIpN);
    const int my_rt = (nrt - (int)blockIdx.x + (int)gridDim.x - 1) / (int)gridDim.x;
    const int64_t nq = (int64_t)my_rt * NJ;         // column tiles of this CTA
    // CTAs start their column walk at different tiles, so that concurrent
    // stores (and W_out reads) spread over the output's rows instead of all
    // hitting the same offsets
    const int crot = (int)(blockIdx.x % (unsigned)NJ);
    const int64_t total_wb = nq * nkb;              // W_out blocks

    if (tid == 0) {
        for (int s = 0; s < kIpStages; ++s) {
            umma::mbar_init(&wfull[s], 1);
            umma::mbar_init(&wempty[s], 1);
        }
        umma::mbar_init(&accfull[0], 1);
        umma::mbar_init(&accfull[1], 1);
        umma::mbar_init(&accempty[0], kIpWorkers);
        umma::mbar_init(&accempty[1], kIpWorkers);
        umma::mbar_init(afull, kIpWorkers);
        umma::mbar_init(aempty, 1);
        umma::mbar_init(drain, 1);
        umma::fence_mbar_init();
        *failed = 0;
    }
    for (int c = tid; c < nkb * 64; c += kIpThreads) {
        se0[c] = c < C ? e0[c] : 0;
        se1[c] = c < C ? e1[c] : 0;
    }
    if (warp == 0) umma::tmem_alloc(tslot, 2 * kIpN);
    umma::tc_fence_before();
    __syncthreads();
    umma::tc_fence_after();
    const uint32_t tmem = *tslot;

    if (warp == 9) {
        // ---- W_out producer: block x = column tile ((x / nkb) % NJ + crot) % NJ, K block x % nkb
        int64_t issued = 0;
        for (int64_t x = 0; x < total_wb; ++x) {
            const int s = (int)(x % kIpStages);
            if (x >= kIpStages && !ip_wait(&wempty[s], (uint32_t)(((x / kIpStages) + 1) & 1), failed)) break;
            const int64_t u = x % ((int64_t)NJ * nkb);
            const int jj = ((int)(u / nkb) + crot) % NJ, kk = (int)(u % nkb);
            unsigned char *dst = sw + s * kIpTile;
            if (tma_w) {
                if (lane == 0) {
                    umma::mbar_arrive_expect_tx(&wfull[s], kIpTile);
                    umma::tma_load_2d(dst, &tmW, kk * 64, jj * kIpN, &wfull[s]);
                }
            } else {
                for (int e = lane; e < kIpN * 8; e += 32) {
                    const int nr = e >> 3, ch = e & 7;
                    const int n = jj * kIpN + nr, c = kk * 64 + ch * 8;
                    uint16_t t8[8];
#pragma unroll
                    for (int z = 0; z < 8; ++z) t8[z] = (n < D && c + z < C) ? W[(int64_t)n * C + c + z] : 0;
                    *reinterpret_cast<uint4 *>(dst + umma::sw128_offset(nr, ch * 8)) =
                        make_uint4(t8[0] | ((uint32_t)t8[1] << 16), t8[2] | ((uint32_t)t8[3] << 16),
                                   t8[4] | ((uint32_t)t8[5] << 16), t8[6] | ((uint32_t)t8[7] << 16));
                }
                umma::fence_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(&wfull[s]);
            }
            issued = x + 1;
        }
        // no load may still be landing at exit: wait for the last one of each stage
        if (tma_w && lane == 0)
            for (int s = 0; s < kIpStages; ++s)
                if (issued > s) {
                    const int64_t last = s + ((issued - 1 - s) / kIpStages) * kIpStages;
                    if (!umma::mbar_wait_bounded(&wfull[s], (uint32_t)((last / kIpStages) & 1), kWaitPolls)) *failed = 1;
                }
    } else if (warp == 8) {
        // ---- MMA issuer
        if (lane == 0) {
            const uint32_t idesc = umma::make_idesc_bf16_f32(kInjM, kIpN);
            int64_t q = 0, x = 0;
            bool ok = true;
            for (int k = 0; k < my_rt && ok; ++k) {
                ok = ip_wait(afull, (uint32_t)(k & 1), failed);
                for (int j = 0; j < NJ && ok; ++j, ++q) {
                    const int b = (int)(q & 1);
                    if (q >= 2) ok = ip_wait(&accempty[b], (uint32_t)(((q >> 1) + 1) & 1), failed);
                    umma::tc_fence_after();
                    const uint32_t dacc = tmem + (uint32_t)(b * kIpN);
                    for (int kb = 0; kb < nkb && ok; ++kb, ++x) {
                        const int s = (int)(x % kIpStages);
                        ok = ip_wait(&wfull[s], (uint32_t)((x / kIpStages) & 1), failed);
                        if (!ok) break;
                        umma::tc_fence_after();
                        const uint32_t ab = umma::smem_u32(sa + kb * kIpTile), bb = umma::smem_u32(sw + s * kIpTile);
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk)
                            umma::mma_bf16(dacc, umma::make_kmajor_sw128_desc(ab + kk * 32),
                                           umma::make_kmajor_sw128_desc(bb + kk * 32), idesc,
                                           (kb > 0 || kk > 0) ? 1u : 0u);
                        umma::mma_commit(&wempty[s]);
                    }
                    umma::mma_commit(&accfull[b]);
                }
                umma::mma_commit(aempty);
            }
            // every MMA issued has completed before the CTA leaves
            umma::mma_commit(drain);
            if (!umma::mbar_wait_bounded(drain, 0u, kWaitPolls)) *failed = 1;
        }
    } else {
        // ---- workers: A tiles and epilogues
        const int g = warp >> 2, lbase = (warp & 3) * 32;
        const int row = tid & 127, half = tid >> 7;
        const uint32_t lowm = (1u << M) - 1u;
        int64_t q = 0;
        bool ok = true;
        for (int k = 0; k < my_rt && ok; ++k) {
            const int i = (int)blockIdx.x + k * (int)gridDim.x;
            if (k >= 1) ok = ip_wait(aempty, (uint32_t)((k - 1) & 1), failed);
            if (!ok) break;
            // A: row = tid % 128, channels [64 kb + 32 half, +32) of every K block
            {
                const int64_t p = (int64_t)i * kInjM + row;
                const bool valid = p < P;
                const int32_t *srow = sym;
                if (valid) {
                    const int64_t bb = p / T;
                    srow = sym + bb * (int64_t)R * T + (p - bb * T);
                }
                // Symbols of one batch -> the bf16 embedding of 32 channels per K block.
                // One-bit routes: a K block's 32 channels are 32 routes, one batch per
                // block.  Routes of 2+ bits: 32 channels span at most 16 routes, so two
                // K blocks share a batch.  Every load of a batch is issued before the
                // first is used.
                auto emit = [&](int kbd, int cbase, int rlo, int rhi, const int32_t *sv, int first) {
                    uint32_t vb = 0, mm = 0;
#pragma unroll
                    for (int u = 0; u < 16 * (2 - first / 16) && u < 32; ++u) {
                        const int r = rlo + u;
                        if (r <= rhi) {
                            const int32_t av = sv[first + u];
                            const uint32_t bits = av >= 0 ? ((uint32_t)av & lowm) : 0u;
                            const uint32_t mk = av >= 0 ? lowm : 0u;
                            const int pos = r * M - cbase;
                            if (pos >= 0) {
                                vb |= bits << pos;
                                mm |= mk << pos;
                            } else {
                                vb |= bits >> -pos;
                                mm |= mk >> -pos;
                            }
                        }
                    }
#pragma unroll
                    for (int ch = 0; ch < 4; ++ch) {
                        const int k0 = ch * 8;
                        const uint4 z0 = *reinterpret_cast<const uint4 *>(se0 + cbase + k0);
                        const uint4 z1 = *reinterpret_cast<const uint4 *>(se1 + cbase + k0);
                        uint4 v;
                        v.x = select_pair(z0.x, z1.x, vb, mm, k0 + 0);
                        v.y = select_pair(z0.y, z1.y, vb, mm, k0 + 2);
                        v.z = select_pair(z0.z, z1.z, vb, mm, k0 + 4);
                        v.w = select_pair(z0.w, z1.w, vb, mm, k0 + 6);
                        *reinterpret_cast<uint4 *>(sa + kbd * kIpTile + umma::sw128_offset(row, half * 32 + k0)) = v;
                    }
                };
                if (M == 1) {
                    for (int kb = 0; kb < nkb; ++kb) {
                        const int cbase = kb * 64 + half * 32;
                        const int r0 = cbase, r1 = cbase < C ? min(C - 1, cbase + 31) : cbase - 1;
                        int32_t sv[32];
#pragma unroll
                        for (int u = 0; u < 32; ++u)
                            sv[u] = (valid && r0 + u <= r1) ? __ldg(srow + (int64_t)(r0 + u) * T) : -1;
                        emit(kb, cbase, r0, r1, sv, 0);
                    }
                } else {
                    for (int kb = 0; kb < nkb; kb += 2) {
                        const int ca = kb * 64 + half * 32, cb = ca + 64;
                        const int ra0 = ca / M, ra1 = ca < C ? min(C - 1, ca + 31) / M : ra0 - 1;
                        const int rb0 = cb / M, rb1 = (kb + 1 < nkb && cb < C) ? min(C - 1, cb + 31) / M : rb0 - 1;
                        int32_t sv[32];
#pragma unroll
                        for (int u = 0; u < 16; ++u) {
                            sv[u] = (valid && ra0 + u <= ra1) ? __ldg(srow + (int64_t)(ra0 + u) * T) : -1;
                            sv[16 + u] = (valid && rb0 + u <= rb1) ? __ldg(srow + (int64_t)(rb0 + u) * T) : -1;
                        }
                        emit(kb, ca, ra0, ra1, sv, 0);
                        if (kb + 1 < nkb) emit(kb + 1, cb, rb0, rb1, sv, 16);
                    }
                }
                umma::fence_async_smem();
                mbar_arrive(afull);
            }
            // epilogues of this row tile's column tiles
            for (int j = 0; j < NJ; ++j, ++q) {
                const int b = (int)(q & 1);
                const int col0 = ((j + crot) % NJ) * kIpN + g * 64;
                const bool live = col0 < D;
                ok = ip_wait(&accfull[b], (uint32_t)((q >> 1) & 1), failed);
                ok = __all_sync(ROSA_FULL_MASK, ok);
                umma::tc_fence_after();
                const uint32_t ta = tmem + ((uint32_t)lbase << 16) + (uint32_t)(b * kIpN + g * 64);
                const int orow = lbase + lane;
                if (tma_out) {
                    unsigned char *buf = sob + g * kIpTile;
                    if ((tid & 127) == 0) umma::tma_store_wait_read();   // the box's previous store has read it
                    named_bar(1 + g, 128);
                    if (ok && live) {
#pragma unroll
                        for (int h = 0; h < 2; ++h) {
                            uint32_t r[32];
                            umma::tmem_ld_32cols(ta + 32 * h, r);
#pragma unroll
                            for (int c4 = 0; c4 < 4; ++c4) {
                                uint4 v;
                                v.x = pack_bf16x2(__uint_as_float(r[8 * c4 + 0]), __uint_as_float(r[8 * c4 + 1]));
                                v.y = pack_bf16x2(__uint_as_float(r[8 * c4 + 2]), __uint_as_float(r[8 * c4 + 3]));
                                v.z = pack_bf16x2(__uint_as_float(r[8 * c4 + 4]), __uint_as_float(r[8 * c4 + 5]));
                                v.w = pack_bf16x2(__uint_as_float(r[8 * c4 + 6]), __uint_as_float(r[8 * c4 + 7]));
                                *reinterpret_cast<uint4 *>(buf + umma::sw128_offset(orow, 32 * h + 8 * c4)) = v;
                            }
                        }
                    }
                    umma::tc_fence_before();
                    mbar_arrive(&accempty[b]);           // the accumulator may be overwritten
                    umma::fence_async_smem();
                    named_bar(1 + g, 128);
                    if ((tid & 127) == 0 && ok && live) umma::tma_store_2d(&tmOut, col0, i * kInjM, buf);
                } else {
                    if (ok && live) {
                        const int64_t p = (int64_t)i * kInjM + orow;
                        uint16_t *dst = out + p * D + col0;
                        const int left = D - col0;
#pragma unroll
                        for (int h = 0; h < 2; ++h) {
                            uint32_t r[32];
                            umma::tmem_ld_32cols(ta + 32 * h, r);
                            if (p < P) {
#pragma unroll
                                for (int z = 0; z < 32; ++z) {
                                    const __nv_bfloat16 hv = __float2bfloat16_rn(__uint_as_float(r[z]));
                                    if (32 * h + z < left) dst[32 * h + z] = *reinterpret_cast<const uint16_t *>(&hv);
                                }
                            }
                        }
                    }
                    umma::tc_fence_before();
                    mbar_arrive(&accempty[b]);
                }
                if (!ok) break;
            }
        }
        if ((tid & 127) == 0 && tma_out) umma::tma_store_wait_all();
    }
    umma::tc_fence_before();
    __syncthreads();
    if (warp == 0) umma::tmem_dealloc(tmem, 2 * kIpN);
    if (tid == 0 && *failed && status) atomicOr(status, ROSA_DEV_TIMEOUT);
}

size_t ip_smem_bytes(int nkb) { return ip_carve(nkb).total + 1024; }

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
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const int C = R * M;
    const int nkb = ceil_div(C, kInjK);
    if (nkb <= kIpMaxKb) {
        static bool ip_attr[64] = {};
        if (dev < 0 || dev >= 64 || !ip_attr[dev]) {
            e = cudaFuncSetAttribute(inject_persistent_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     (int)ip_smem_bytes(kIpMaxKb));
            if (e != cudaSuccess) return e;
            if (dev >= 0 && dev < 64) ip_attr[dev] = true;
        }
        const int smem = (int)ip_smem_bytes(nkb);
        CUtensorMap tmW, tmOut;
        const bool tma_w = C >= kInjK && make_tmap_bf16_2d(&tmW, W, (uint64_t)D, (uint64_t)C, kInjM, 64);
        const bool tma_out = D >= 64 && make_tmap_bf16_2d(&tmOut, out, (uint64_t)P, (uint64_t)D, kInjM, 64);
        if (!tma_w) memset(&tmW, 0, sizeof tmW);
        if (!tma_out) memset(&tmOut, 0, sizeof tmOut);
        // at most two CTAs per SM: each holds 256 of the SM's 512 tensor-memory columns
        static bool ip_carve_set[64] = {};
        if (dev >= 0 && dev < 64 && !ip_carve_set[dev]) {
            // the whole unified L1 / shared array as shared memory, so that two CTAs fit where they can
            e = cudaFuncSetAttribute(inject_persistent_kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                                     (int)cudaSharedmemCarveoutMaxShared);
            if (e != cudaSuccess) return e;
            ip_carve_set[dev] = true;
        }
        // CTAs per SM from the SM's shared memory and registers (at most two:
        // each CTA holds 256 of the SM's 512 tensor-memory columns)
        static int ip_regs[64] = {};
        if (dev >= 0 && dev < 64 && ip_regs[dev] == 0) {
            cudaFuncAttributes fa;
            if ((e = cudaFuncGetAttributes(&fa, inject_persistent_kernel)) != cudaSuccess) return e;
            ip_regs[dev] = fa.numRegs;
        }
        int smem_sm = 0, smem_rsv = 0, regs_sm = 0;
        if ((e = cudaDeviceGetAttribute(&smem_sm, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev)) != cudaSuccess ||
            (e = cudaDeviceGetAttribute(&smem_rsv, cudaDevAttrReservedSharedMemoryPerBlock, dev)) != cudaSuccess ||
            (e = cudaDeviceGetAttribute(&regs_sm, cudaDevAttrMaxRegistersPerMultiprocessor, dev)) != cudaSuccess)
            return e;
        const int regs = (dev >= 0 && dev < 64) ? ip_regs[dev] : 96;
        const int regs_cta = ((regs * 32 + 255) / 256) * 256 * (kIpThreads / 32);   // per-warp allocation units
        int per_sm = smem_sm / (smem + smem_rsv);
        if (regs_cta > 0) per_sm = min(per_sm, regs_sm / regs_cta);
        per_sm = per_sm < 1 ? 1 : (per_sm > 2 ? 2 : per_sm);
        const int64_t nrt = ceil_div64(P, kInjM);
        const int64_t slots = (int64_t)per_sm * device_sm_count();
        const unsigned grid = (unsigned)(nrt < slots ? nrt : slots);
        inject_persistent_kernel<<<grid, kIpThreads, smem, st>>>(tmW, tmOut, tma_w, tma_out, sym, e0, e1, W, R, M, T,
                                                                  D, P, nkb, out, status);
        return cudaGetLastError();
    }
    static bool attr_done[64] = {};
    const int smem = (int)inject_smem_bytes();
    if (dev < 0 || dev >= 64 || !attr_done[dev]) {
        e = cudaFuncSetAttribute(inject_tile_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e != cudaSuccess) return e;
        if (dev >= 0 && dev < 64) attr_done[dev] = true;
    }
    // N tile: all of D when it fits one MMA, else 256 (a multiple of 16 in [16, 256])
    int BN = D >= kInjMaxN ? kInjMaxN : ((D + 15) / 16) * 16;
    if (BN < 16) BN = 16;
    const bool wvec = (C % 8 == 0) && (reinterpret_cast<uintptr_t>(W) % 16 == 0);
    // the output leaves by TMA stores when its rows are 16-byte aligned and BN
    // is a whole number of 64-column boxes
    CUtensorMap tmOut;
    const bool tma_out = (BN % 64 == 0) && make_tmap_bf16_2d(&tmOut, out, (uint64_t)P, (uint64_t)D, kInjM, 64);
    if (!tma_out) memset(&tmOut, 0, sizeof tmOut);
    dim3 grid((unsigned)ceil_div64(P, kInjM), (unsigned)ceil_div(D, BN));
    inject_tile_kernel<<<grid, kInjThreads, smem, st>>>(tmOut, tma_out, sym, e0, e1, W, R, M, T, D, BN, P, wvec, out,
                                                        status);
    return cudaGetLastError();
}

}  // namespace rosa
