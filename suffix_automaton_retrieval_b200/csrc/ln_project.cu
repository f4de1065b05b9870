// Layer norm, query/key projection and discretisation fused on the tensor
// cores.
//
// "ROSA-Tuning" (arXiv 2602.02499), section 3.2: U = LN(H), Q = U W_q,
// K = U W_k, then the strict threshold I[x > 0] and multi-route packing
// (Eqs. 10-15; channel c = r*M + j carries bit j of route r's symbol).
//
// The layer norm is folded into the contraction:
//   U W = rstd * (H (gamma o W) - mu * colsum(gamma o W)) + beta W,
// with mu and rstd the row's mean and reciprocal standard deviation.  The
// tensor cores therefore consume the raw rows of H, which arrive in shared
// memory by TMA (128-byte swizzle, mbarrier completion, two stages), and the
// same shared-memory tiles give each row's sums of h and h^2.  The scaled
// weights gamma o W are split into bf16 high and low parts (hi + lo carries
// about 16 significant bits) that are multiplied as two halves of one MMA
// (N = 2 x the effective columns), so the weights lose almost nothing to
// bf16.  The epilogue reads both halves from tensor memory, applies the
// fold, thresholds and packs the bits of each route, and writes the symbol
// bytes of the query and key streams.
//
// Effective columns n < C are query channels, C <= n < 2C key channels; a
// CTA covers NE of them (a multiple of both 8 and M, at most 128).
#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "../../include/rosa.h"
#include "common.cuh"
#include "kernels.h"
#include "umma.cuh"

namespace rosa {
namespace {

constexpr int kLnpM = 256;          // rows per CTA: two M = 128 MMAs share each weight block
constexpr int kLnpMmaM = 128;       // rows of one single-CTA MMA (M = 256 exists only for CTA pairs)
constexpr int kLnpK = 64;           // K per block (one 128-byte swizzle row)
constexpr int kLnpThreads = 256;    // one row each for the statistics; warps 4-7 take the second half
constexpr int kLnpStages = 3;
constexpr uint32_t kLnpWaitPolls = umma::kWaitPolls;

int gcd_int(int a, int b) { return b ? gcd_int(b, a % b) : a; }

// Effective columns per CTA: the largest multiple of lcm(M, 8) up to 128.
int lnp_ne(int M) {
    const int l = 8 * M / gcd_int(8, M);
    return (128 / l) * l;
}

struct LnpSmem {
    alignas(1024) unsigned char a[kLnpStages][kLnpM * 128];   // H block (256 rows), K-major SW128
    alignas(1024) unsigned char b[kLnpStages][256 * 128];     // hi / lo weight rows, K-major SW128
    float cs[128], bv[128];                                    // this tile's column constants
    uint64_t full[kLnpStages], done[kLnpStages];
    uint32_t tmem;
    int failed;
};

constexpr int kPrepCols = 32;    // effective columns per prep CTA
constexpr int kPrepK = 128;      // rows of W per prep CTA

struct LnpLayout {
    uint16_t *wp;     // [NT * 2NE rows][D]: per tile NE high rows then NE low rows
    float *cs;        // [ceil(D / kPrepK)][NT * NE]: partial column sums of hi + lo
    float *bv;        // [ceil(D / kPrepK)][NT * NE]: partial beta . W
    size_t bytes;
};

size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

LnpLayout lnp_carve(int D, int C, int M, void *base) {
    const int NE = lnp_ne(M), NT = ceil_div(2 * C, NE);
    LnpLayout L{};
    char *b = static_cast<char *>(base);
    size_t off = 0;
    auto take = [&](size_t n) -> void * {
        void *p = b ? b + off : nullptr;
        off += align256(n);
        return p;
    };
    const int nkc = ceil_div(D, kPrepK);
    L.wp = (uint16_t *)take((size_t)NT * 2 * NE * D * 2);
    L.cs = (float *)take((size_t)nkc * NT * NE * 4);
    L.bv = (float *)take((size_t)nkc * NT * NE * 4);
    L.bytes = off;
    return L;
}

__device__ __forceinline__ uint16_t bf16_bits_rn(float x) {
    const __nv_bfloat16 h = __float2bfloat16_rn(x);
    return *reinterpret_cast<const uint16_t *>(&h);
}

__device__ __forceinline__ float bf16_bits_to_float(uint16_t h) { return __uint_as_float((uint32_t)h << 16); }

// One CTA per 32 effective columns x 128 rows of W (padding columns of the
// last tile write zeros): a warp reads 32 consecutive columns of one row, the
// high and low parts are transposed in shared memory and leave as 256-byte
// row pieces; each CTA writes its partial column sums (the main kernel adds
// the 128-row partials in a fixed order).
__global__ void __launch_bounds__(256)
lnp_prep_kernel(const float *__restrict__ gamma, const float *__restrict__ beta, const uint16_t *__restrict__ Wq,
                const uint16_t *__restrict__ Wk, int D, int C, int NE, int NTNE, uint16_t *__restrict__ wp,
                float *__restrict__ cs, float *__restrict__ bv) {
    __shared__ __align__(16) uint16_t th[kPrepCols][kPrepK + 8], tl[kPrepCols][kPrepK + 8];
    __shared__ float red[2][8][kPrepCols];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int n0 = blockIdx.x * kPrepCols, k0 = blockIdx.y * kPrepK;
    const int n = n0 + lane;
    const bool valid = n < 2 * C;
    float s_cs = 0.f, s_bv = 0.f;
#pragma unroll
    for (int i = warp; i < kPrepK; i += 8) {   // all loads of a thread issued together
        const int k = k0 + i;
        uint16_t h = 0, l = 0;
        if (valid && k < D) {
            const float w = bf16_bits_to_float(n < C ? Wq[(int64_t)k * C + n] : Wk[(int64_t)k * C + n - C]);
            const float ws = (gamma ? gamma[k] : 1.f) * w;
            h = bf16_bits_rn(ws);
            l = bf16_bits_rn(ws - bf16_bits_to_float(h));
            s_cs += bf16_bits_to_float(h) + bf16_bits_to_float(l);
            s_bv += (beta ? beta[k] : 0.f) * w;
        }
        th[lane][i] = h;
        tl[lane][i] = l;
    }
    red[0][warp][lane] = s_cs;
    red[1][warp][lane] = s_bv;
    __syncthreads();
    // rows n0 .. n0+31 of the high and low planes, columns k0 .. k0+255
    const int kn = min(kPrepK, D - k0);
    for (int r = warp; r < kPrepCols; r += 8) {
        const int nn = n0 + r;
        if (nn >= NTNE) break;
        const int tile = nn / NE, cn = nn - tile * NE;
        uint16_t *hi = wp + ((int64_t)tile * 2 * NE + cn) * D + k0;
        uint16_t *lo = wp + ((int64_t)tile * 2 * NE + NE + cn) * D + k0;
        for (int c = lane * 8; c < kn; c += 32 * 8) {   // D % 8 == 0: whole 16-byte pieces
            *reinterpret_cast<uint4 *>(hi + c) = *reinterpret_cast<const uint4 *>(&th[r][c]);
            *reinterpret_cast<uint4 *>(lo + c) = *reinterpret_cast<const uint4 *>(&tl[r][c]);
        }
    }
    if (warp == 0 && n < NTNE) {
        float a = 0.f, c = 0.f;
        for (int w = 0; w < 8; ++w) {
            a += red[0][w][lane];
            c += red[1][w][lane];
        }
        cs[(int64_t)blockIdx.y * NTNE + n] = a;
        bv[(int64_t)blockIdx.y * NTNE + n] = c;
    }
}

__global__ void __launch_bounds__(kLnpThreads, 1)
lnp_kernel(const __grid_constant__ CUtensorMap tmH, const __grid_constant__ CUtensorMap tmW, int64_t P, int T, int D,
           int C, int M, int NE, float eps, const float *__restrict__ cs, const float *__restrict__ bv,
           uint8_t *__restrict__ symq, uint8_t *__restrict__ symk, uint32_t *__restrict__ status) {
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    LnpSmem &sm = *reinterpret_cast<LnpSmem *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    const int tid = threadIdx.x, warp = tid >> 5;
    const int64_t p0 = (int64_t)blockIdx.x * kLnpM;
    const int tile = blockIdx.y;
    const int N = 2 * NE;                               // MMA N: high then low halves
    const uint32_t a_bytes = kLnpM * 128, b_bytes = (uint32_t)N * 128;
    const int nkb = ceil_div(D, kLnpK);

    if (tid == 0) {
        for (int s = 0; s < kLnpStages; ++s) {
            umma::mbar_init(&sm.full[s], 1);
            umma::mbar_init(&sm.done[s], 1);
        }
        umma::fence_mbar_init();
        sm.failed = 0;
    }
    // the epilogue's per-column constants, read once per CTA
    if (tid < NE) {
        const int nkc = ceil_div(D, kPrepK), NTNE = gridDim.y * NE;
        float a = 0.f, c = 0.f;
        for (int kc = 0; kc < nkc; ++kc) {
            a += cs[(int64_t)kc * NTNE + tile * NE + tid];
            c += bv[(int64_t)kc * NTNE + tile * NE + tid];
        }
        sm.cs[tid] = a;
        sm.bv[tid] = c;
    }
    if (warp == 0) umma::tmem_alloc(&sm.tmem, 512);   // accumulators of the two row halves
    umma::tc_fence_before();
    __syncthreads();
    umma::tc_fence_after();
    const uint32_t tmem = sm.tmem;

    if (tid == 0) {
        for (int s = 0; s < kLnpStages && s < nkb; ++s) {
            umma::mbar_arrive_expect_tx(&sm.full[s], a_bytes + b_bytes);
            umma::tma_load_2d(sm.a[s], &tmH, s * kLnpK, (int)p0, &sm.full[s]);
            umma::tma_load_2d(sm.b[s], &tmW, s * kLnpK, tile * N, &sm.full[s]);
        }
    }
    const uint32_t idesc = umma::make_idesc_bf16_f32(kLnpMmaM, N);   // each MMA covers one 128-row half
    float s1 = 0.f, s2 = 0.f;   // this thread's row: sum of h and of h^2
    for (int kb = 0; kb < nkb; ++kb) {
        const int s = kb % kLnpStages;
        if (!umma::mbar_wait_bounded(&sm.full[s], (uint32_t)((kb / kLnpStages) & 1), kLnpWaitPolls)) sm.failed = 1;
        if (!sm.failed) {
            const unsigned char *row = sm.a[s] + tid * 128;
#pragma unroll
            for (int ch = 0; ch < 8; ++ch) {
                const uint4 v = *reinterpret_cast<const uint4 *>(row + ((ch ^ (tid & 7)) << 4));
                const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                for (int h = 0; h < 4; ++h) {
                    const float lo = __uint_as_float(w4[h] << 16), hi = __uint_as_float(w4[h] & 0xffff0000u);
                    s1 += lo + hi;
                    s2 += lo * lo + hi * hi;
                }
            }
        }
        if (tid == 0 && !sm.failed) {
            umma::tc_fence_after();
            const uint32_t abase = umma::smem_u32(sm.a[s]), bbase = umma::smem_u32(sm.b[s]);
#pragma unroll
            for (int half = 0; half < 2; ++half)
#pragma unroll
                for (int kk = 0; kk < kLnpK / 16; ++kk)
                    umma::mma_bf16(tmem + half * 256, umma::make_kmajor_sw128_desc(abase + half * kLnpMmaM * 128 + kk * 32),
                                   umma::make_kmajor_sw128_desc(bbase + kk * 32), idesc, (kb > 0 || kk > 0) ? 1u : 0u);
            umma::mma_commit(&sm.done[s]);
        }
        __syncthreads();   // every row's statistics read of stages up to s is done
        if (sm.failed) break;
        // Refill the previous block's stage with block kb - 1 + kLnpStages once its
        // MMAs have read it: they were issued before this block's, so the tensor
        // pipe keeps this block's MMAs queued while the issuing thread waits.
        const int kp = kb - 1;
        if (kp >= 0 && kp + kLnpStages < nkb && tid == 0) {
            const int sp = kp % kLnpStages;
            if (!umma::mbar_wait_bounded(&sm.done[sp], (uint32_t)((kp / kLnpStages) & 1), kLnpWaitPolls)) {
                sm.failed = 1;
            } else {
                umma::mbar_arrive_expect_tx(&sm.full[sp], a_bytes + b_bytes);
                umma::tma_load_2d(sm.a[sp], &tmH, (kp + kLnpStages) * kLnpK, (int)p0, &sm.full[sp]);
                umma::tma_load_2d(sm.b[sp], &tmW, (kp + kLnpStages) * kLnpK, tile * N, &sm.full[sp]);
            }
        }
    }
    // the last commit covers every MMA of the tile
    if (!sm.failed && nkb > 0) {
        const int kl = nkb - 1;
        if (!umma::mbar_wait_bounded(&sm.done[kl % kLnpStages], (uint32_t)((kl / kLnpStages) & 1), kLnpWaitPolls))
            sm.failed = 1;
    }
    __syncthreads();
    umma::tc_fence_after();
    if (!sm.failed) {
        // epilogue: thread = row; warps 0-3 read the first half's accumulator
        // (TMEM columns 0..255), warps 4-7 the second half's (256..511)
        const int64_t p = p0 + tid;
        const uint32_t tacc = tmem + ((uint32_t)((warp & 3) * 32) << 16) + (uint32_t)((warp >> 2) * 256);
        const float mu = s1 / (float)D;
        const float var = fmaxf(s2 / (float)D - mu * mu, 0.f);
        const float rstd = rsqrtf(var + eps);
        // threshold bits of the NE effective columns, kept in registers: every
        // index into them is a compile-time constant or an explicit select
        uint32_t bits[4] = {0, 0, 0, 0};
#pragma unroll
        for (int w = 0; w < 4; ++w) {
            const int c0 = 32 * w;
            if (c0 < NE) {
                uint32_t h[32], l[32];
                umma::tmem_ld_32cols(tacc + (uint32_t)c0, h);
                umma::tmem_ld_32cols(tacc + (uint32_t)(NE + c0), l);
#pragma unroll
                for (int j = 0; j < 32; ++j) {
                    const int cn = c0 + j;
                    if (cn < NE) {
                        const float acc = __uint_as_float(h[j]) + __uint_as_float(l[j]);
                        const float x = rstd * (acc - mu * sm.cs[cn]) + sm.bv[cn];
                        if (x > 0.f) bits[w] |= 1u << j;
                    }
                }
            }
        }
        if (p < P) {
            const int64_t b = p / T, t = p - b * T;
            const int R = C / M;
            const uint32_t lowm = (1u << M) - 1u;
            // effective column n = tile*NE + cn is bit 0 of route n / M of the query
            // channels (n < C) or route n / M - R of the key channels; M divides NE and C
            int ra = tile * NE / M;
            for (int cn = 0; cn < NE; cn += M, ++ra) {
                const int n = tile * NE + cn;
                if (n >= 2 * C) break;
                // M bits from column cn on (M divides NE, so they may straddle two words)
                const int wd = cn >> 5, o = cn & 31;
                const uint32_t lo = wd == 0 ? bits[0] : wd == 1 ? bits[1] : wd == 2 ? bits[2] : bits[3];
                const uint32_t hi = wd == 0 ? bits[1] : wd == 1 ? bits[2] : wd == 2 ? bits[3] : 0u;
                const uint32_t a = ((lo >> o) | (o ? hi << (32 - o) : 0u)) & lowm;
                const bool isq = ra < R;
                const int r = isq ? ra : ra - R;
                (isq ? symq : symk)[(b * R + r) * (int64_t)T + t] = (uint8_t)a;
            }
        }
    } else if (tid == 0 && status) {
        atomicOr(status, ROSA_DEV_TIMEOUT);
    }
    umma::tc_fence_before();
    __syncthreads();
    if (warp == 0) umma::tmem_dealloc(tmem, 512);
}

size_t lnp_smem_bytes() { return sizeof(LnpSmem) + 1024; }

}  // namespace

size_t ln_project_workspace_bytes(int D, int C, int M) { return lnp_carve(D, C, M, nullptr).bytes; }

cudaError_t launch_ln_project(const uint16_t *H, const float *gamma, const float *beta, const uint16_t *Wq,
                              const uint16_t *Wk, int B, int T, int D, int C, int M, float eps, uint8_t *symq,
                              uint8_t *symk, void *workspace, size_t ws_bytes, uint32_t *status, cudaStream_t st) {
    const LnpLayout L = lnp_carve(D, C, M, workspace);
    if (L.bytes > ws_bytes) return cudaErrorInvalidValue;
    const int64_t P = (int64_t)B * T;
    if (P == 0) return cudaSuccess;
    const int NE = lnp_ne(M), NT = ceil_div(2 * C, NE);
    CUtensorMap tmH, tmW;
    if (!make_tmap_bf16_2d(&tmH, H, (uint64_t)P, (uint64_t)D, kLnpM, 64) ||
        !make_tmap_bf16_2d(&tmW, L.wp, (uint64_t)NT * 2 * NE, (uint64_t)D, (uint32_t)(2 * NE), 64))
        return cudaErrorInvalidValue;
    static bool attr_done[64] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const int smem = (int)lnp_smem_bytes();
    if (dev < 0 || dev >= 64 || !attr_done[dev]) {
        e = cudaFuncSetAttribute(lnp_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e != cudaSuccess) return e;
        if (dev >= 0 && dev < 64) attr_done[dev] = true;
    }
    lnp_prep_kernel<<<dim3((unsigned)ceil_div(NT * NE, kPrepCols), (unsigned)ceil_div(D, kPrepK)), 256, 0, st>>>(
        gamma, beta, Wq, Wk, D, C, NE, NT * NE, L.wp, L.cs, L.bv);
    dim3 grid((unsigned)ceil_div64(P, kLnpM), (unsigned)NT);
    lnp_kernel<<<grid, kLnpThreads, smem, st>>>(tmH, tmW, P, T, D, C, M, NE, eps, L.cs, L.bv, symq, symk, status);
    return cudaGetLastError();
}

}  // namespace rosa
