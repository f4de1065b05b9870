// Run-level retrieval with adjacent folding.
//
// "ROSA-Tuning" (arXiv 2602.02499), section 3.3, the run-length encoding
// paragraph: consecutive equal symbols of a route form one run, the
// automaton and the matching state move only at run boundaries, and a hit
// on a key run maps back to the time axis as the start of the next key run;
// appendix C.5-C.6 keep per-run start indices and precompute per query run.
//
// Both streams fold.  Query run m (start time u_m) takes the retrieval once,
// at u_m, and every t of the run reports it.  Key run l is admissible for it
// iff the next key run starts at s_{l+1} <= u_m - g + 1; since run starts
// increase, that is a prefix l <= X_m of the key runs.  The longest run-level
// match and its most recent key run l* are exactly what the position-level
// matcher computes on the run-symbol streams with bound X_m per query, so
// the path is:
//
//   1. rle_count / rle_scan / rle_write: run starts per 2048-position tile,
//      per-stream offsets, then the run-symbol streams, the run start times
//      and, for keys, the run index of every position;
//   2. rle_bound: X_m = (key run of position u_m - g + 1) - 1;
//   3. the matcher (match.cu) on the run streams with those bounds;
//   4. rle_map: every position t finds its query run m and writes
//      end_idx = s_{l*+1} - 1 (tau = end_idx + 1 is the next run's start),
//      len = the run-level length, sym = v[s_{l*+1}].
//
// Run streams are shorter than T; their tails up to T are padded with
// pseudo-random symbols (a hash of the slot) that can never be used: a
// padded key run has no successor inside the stream, so it is never
// admissible, and padded query runs get the bound -1 and are not read.
// Random padding keeps the sort of the padded items as cheap as that of
// ordinary data (a constant pad would form one long tie).
#include <cstdint>
#include <cuda_runtime.h>

#include "../../include/rosa.h"
#include "common.cuh"
#include "kernels.h"

namespace rosa {
namespace {

constexpr int kRleTile = 2048;
constexpr int kRleThreads = 256;
constexpr int kRleIPT = kRleTile / kRleThreads;   // 8 consecutive positions per thread

struct RleLayout {
    size_t match_off, match_bytes;
    uint8_t *qr, *kr;           // run-symbol streams [S, T]; qr == kr when q == k
    int32_t *qstart, *kstart;   // run start times [S, T]; qstart == kstart when q == k
    int32_t *krun;              // key run index of every position [S, T]
    int32_t *xb;                // bound of every query run [S, T]
    int32_t *rend, *rlen, *rsym;   // run-level matcher outputs [S, T]
    int32_t *tcnt;              // [S][tiles][2]: run starts per tile, then exclusive offsets
    int32_t *nrun;              // [S][2]: runs per stream (0: keys, 1: queries)
    size_t bytes;
};

size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

// The matcher's workspace comes first, so that its status word sits at the
// start of the run-level workspace as well.
RleLayout rle_carve(int S, int T, int K, bool same, void *base) {
    RleLayout L{};
    char *b = static_cast<char *>(base);
    size_t off = 0;
    auto take = [&](size_t bytes) -> void * {
        void *p = b ? b + off : nullptr;
        off += align256(bytes);
        return p;
    };
    L.match_bytes = match_workspace_bytes(S, T, K, same);
    L.match_off = 0;
    take(L.match_bytes);
    const size_t n = (size_t)S * T;
    const int ntile = ceil_div(T, kRleTile);
    L.kr = (uint8_t *)take(n);
    L.qr = same ? L.kr : (uint8_t *)take(n);
    L.kstart = (int32_t *)take(n * 4);
    L.qstart = same ? L.kstart : (int32_t *)take(n * 4);
    L.krun = (int32_t *)take(n * 4);
    L.xb = (int32_t *)take(n * 4);
    L.rend = (int32_t *)take(n * 4);
    L.rlen = (int32_t *)take(n * 4);
    L.rsym = (int32_t *)take(n * 4);
    L.tcnt = (int32_t *)take((size_t)S * ntile * 2 * 4);
    L.nrun = (int32_t *)take((size_t)S * 2 * 4);
    L.bytes = off;
    return L;
}

// Stages positions [p0 - 1, p0 + 2048) of one stream in shared memory and
// returns this thread's run-start flags for its 8 positions (bit u for
// position p0 + 8 * thread + u).
__device__ __forceinline__ unsigned tile_flags(const uint8_t *__restrict__ x, int T, int p0, uint8_t *sb) {
    const int lim = min(kRleTile, T - p0);
    for (int i = threadIdx.x; i <= kRleTile; i += kRleThreads) {
        const int p = p0 - 1 + i;
        sb[i] = (p >= 0 && p < T) ? x[p] : 0;
    }
    __syncthreads();
    unsigned f = 0;
    const int j0 = threadIdx.x * kRleIPT;
#pragma unroll
    for (int u = 0; u < kRleIPT; ++u) {
        const int j = j0 + u;
        if (j < lim && (p0 + j == 0 || sb[j + 1] != sb[j])) f |= 1u << u;
    }
    return f;
}

// Slot j of stream s's padded key (which = 0) or query (which = 1) run
// stream: a symbol below K that no real run depends on, hashed from the slot
// and the side.  The two sides draw independent symbols: identical padded
// tails would share histories as long as the padding and make the suffix
// sorting and the LCP work grow with it.
__device__ __forceinline__ uint8_t pad_symbol(int64_t slot, int K) {
    uint32_t h = (uint32_t)slot * 0x9E3779B1u;
    h ^= h >> 15;
    h *= 0x85EBCA77u;
    h ^= h >> 13;
    return (uint8_t)(h % (uint32_t)K);
}

// grid: S * tiles * streams (keys, then queries when q != k)
__global__ void __launch_bounds__(kRleThreads)
rle_count_kernel(const uint8_t *__restrict__ q, const uint8_t *__restrict__ k, int T, int ntile, int nwhich,
                 int32_t *__restrict__ tcnt) {
    __shared__ uint8_t sb[kRleTile + 1];
    __shared__ int red[kRleThreads / 32];
    const int which = blockIdx.x % nwhich;
    const int st = blockIdx.x / nwhich;
    const int s = st / ntile, tile = st - s * ntile;
    const uint8_t *x = (which ? q : k) + (int64_t)s * T;
    const unsigned f = tile_flags(x, T, tile * kRleTile, sb);
    int c = __popc(f);
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) c += __shfl_xor_sync(ROSA_FULL_MASK, c, o);
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = c;
    __syncthreads();
    if (threadIdx.x == 0) {
        int t = 0;
        for (int w = 0; w < kRleThreads / 32; ++w) t += red[w];
        tcnt[((int64_t)s * ntile + tile) * 2 + which] = t;
    }
}

// One warp per (stream, which): exclusive scan of the tile counts in place,
// the total into nrun.
__global__ void rle_scan_kernel(int S, int ntile, int nwhich, int32_t *__restrict__ tcnt,
                                int32_t *__restrict__ nrun) {
    const int lane = threadIdx.x & 31;
    const int64_t wid = (blockIdx.x * (int64_t)blockDim.x + threadIdx.x) >> 5;
    if (wid >= (int64_t)S * nwhich) return;
    const int s = (int)(wid / nwhich), which = (int)(wid % nwhich);
    int32_t *c = tcnt + (int64_t)s * ntile * 2 + which;
    int carry = 0;
    for (int t0 = 0; t0 < ntile; t0 += 32) {
        const int t = t0 + lane;
        const int v = t < ntile ? c[(int64_t)t * 2] : 0;
        int incl = v;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(ROSA_FULL_MASK, incl, o);
            if (lane >= o) incl += y;
        }
        if (t < ntile) c[(int64_t)t * 2] = carry + incl - v;
        carry += __shfl_sync(ROSA_FULL_MASK, incl, 31);
    }
    if (lane == 0) {
        nrun[s * 2 + which] = carry;
        if (nwhich == 1) nrun[s * 2 + 1] = carry;   // q == k: the same runs
    }
}

// Run symbols and start times; for keys also the run index of every
// position; the padded tail of each run stream.
__global__ void __launch_bounds__(kRleThreads)
rle_write_kernel(const uint8_t *__restrict__ q, const uint8_t *__restrict__ k, int T, int K, int ntile, int nwhich,
                 const int32_t *__restrict__ tcnt, const int32_t *__restrict__ nrun, uint8_t *__restrict__ kr,
                 uint8_t *__restrict__ qr, int32_t *__restrict__ kstart, int32_t *__restrict__ qstart,
                 int32_t *__restrict__ krun) {
    __shared__ uint8_t sb[kRleTile + 1];
    __shared__ uint32_t ws[kRleThreads / 32 + 1];
    const int which = blockIdx.x % nwhich;
    const int st = blockIdx.x / nwhich;
    const int s = st / ntile, tile = st - s * ntile;
    const int p0 = tile * kRleTile;
    const uint8_t *x = (which ? q : k) + (int64_t)s * T;
    uint8_t *rs = (which ? qr : kr) + (int64_t)s * T;
    int32_t *rt = (which ? qstart : kstart) + (int64_t)s * T;
    const unsigned f = tile_flags(x, T, p0, sb);
    const uint32_t before = block_exclusive_scan<kRleThreads>((uint32_t)__popc(f), ws, nullptr);
    const int base = tcnt[((int64_t)s * ntile + tile) * 2 + which] + (int)before;
    const int j0 = threadIdx.x * kRleIPT;
    int run = base - 1;   // run index of the position before this thread's first
#pragma unroll
    for (int u = 0; u < kRleIPT; ++u) {
        const int j = j0 + u;
        if (p0 + j >= T) break;
        if ((f >> u) & 1u) {
            ++run;
            rs[run] = sb[j + 1];
            rt[run] = p0 + j;
        }
        if (which == 0) krun[(int64_t)s * T + p0 + j] = run;
    }
    // this tile's slots of the padded tail
    const int n = nrun[s * 2 + which];
    for (int j = p0 + threadIdx.x; j < min(p0 + kRleTile, T); j += kRleThreads) {
        if (j >= n) {
            rs[j] = pad_symbol((((int64_t)s * T + j) << 1) | which, K);
            rt[j] = T;
        }
    }
}

// Bound of every query run: the last admissible key run, or -1.
__global__ void rle_bound_kernel(int S, int T, int g, const int32_t *__restrict__ nrun,
                                 const int32_t *__restrict__ qstart, const int32_t *__restrict__ krun,
                                 int32_t *__restrict__ xb) {
    const int64_t total = (int64_t)S * T;
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total;
         i += (int64_t)gridDim.x * blockDim.x) {
        const int s = (int)(i / T), m = (int)(i - (int64_t)s * T);
        int X = -1;
        if (m < nrun[s * 2 + 1]) {
            const int p = qstart[i] - g + 1;   // the next key run must start by here
            if (p >= 0) X = krun[(int64_t)s * T + p] - 1;
        }
        xb[i] = X;
    }
}

// Binary alphabet (K = 2): consecutive runs differ, so a folded stream
// alternates and its whole run history is fixed by its last symbol.  The
// run-level suffix of query run m then matches key run l over min(m, l) + 1
// runs when the two symbols agree and not at all otherwise, so the longest
// admissible match ends at the last admissible key run with query run m's
// symbol: X_m or X_m - 1.  Every real run's symbol is also checked against
// the alphabet (the status word of the workspace).
__global__ void rle_binary_kernel(int S, int T, const int32_t *__restrict__ nrun, const uint8_t *__restrict__ qr,
                                  const uint8_t *__restrict__ kr, const int32_t *__restrict__ xb,
                                  int32_t *__restrict__ rend, int32_t *__restrict__ rlen, uint32_t *__restrict__ status) {
    const int64_t total = (int64_t)S * T;
    bool bad = false;
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total;
         i += (int64_t)gridDim.x * blockDim.x) {
        const int s = (int)(i / T), m = (int)(i - (int64_t)s * T);
        const int nk = nrun[s * 2], nq = nrun[s * 2 + 1];
        if (m < nk) bad |= kr[i] >= 2;
        int e = -1, L = 0;
        if (m < nq) {
            const uint8_t d = qr[i];
            bad |= d >= 2;
            const int X = xb[i];
            if (X >= 0) {
                const int l = kr[(int64_t)s * T + X] == d ? X : X - 1;
                if (l >= 0) {
                    e = l;
                    L = min(l, m) + 1;
                }
            }
        }
        rend[i] = e;
        rlen[i] = L;
    }
    if (bad) atomicOr(status, ROSA_DEV_SYMBOL_RANGE);
}

// Every position reads its query run's answer and maps it to the time axis.
__global__ void __launch_bounds__(kRleThreads)
rle_map_kernel(const uint8_t *__restrict__ q, const uint8_t *__restrict__ vs, int T, int ntile, int qwhich,
               const int32_t *__restrict__ tcnt, const int32_t *__restrict__ kstart,
               const int32_t *__restrict__ rend, const int32_t *__restrict__ rlen, int32_t *__restrict__ end_idx,
               int32_t *__restrict__ len, int32_t *__restrict__ sym) {
    __shared__ uint8_t sb[kRleTile + 1];
    __shared__ uint32_t ws[kRleThreads / 32 + 1];
    const int s = blockIdx.x / ntile, tile = blockIdx.x - s * ntile;
    const int p0 = tile * kRleTile;
    const unsigned f = tile_flags(q + (int64_t)s * T, T, p0, sb);
    const uint32_t before = block_exclusive_scan<kRleThreads>((uint32_t)__popc(f), ws, nullptr);
    int run = tcnt[((int64_t)s * ntile + tile) * 2 + qwhich] + (int)before - 1;
    const int64_t so = (int64_t)s * T;
    const int j0 = threadIdx.x * kRleIPT;
    int32_t e[kRleIPT], l[kRleIPT], y[kRleIPT];
#pragma unroll
    for (int u = 0; u < kRleIPT; ++u) {
        const int j = j0 + u;
        e[u] = -1; l[u] = 0; y[u] = -1;
        if (p0 + j >= T) continue;
        if ((f >> u) & 1u) ++run;
        const int L = rlen[so + run];
        if (L > 0) {
            const int tau = kstart[so + rend[so + run] + 1];
            e[u] = tau - 1;
            l[u] = L;
            y[u] = (int32_t)vs[so + tau];
        }
    }
    // coalesced stores: the tile's outputs pass through shared memory, nine
    // words per thread so that a warp's eight-apart stores hit distinct banks
    constexpr int kStride = kRleIPT + 1;
    __shared__ int32_t so_e[kRleThreads * kStride], so_l[kRleThreads * kStride], so_y[kRleThreads * kStride];
#pragma unroll
    for (int u = 0; u < kRleIPT; ++u) {
        so_e[threadIdx.x * kStride + u] = e[u];
        so_l[threadIdx.x * kStride + u] = l[u];
        so_y[threadIdx.x * kStride + u] = y[u];
    }
    __syncthreads();
    const int lim = min(kRleTile, T - p0);
    for (int j = threadIdx.x; j < lim; j += kRleThreads) {
        const int slot = (j / kRleIPT) * kStride + j % kRleIPT;
        end_idx[so + p0 + j] = so_e[slot];
        len[so + p0 + j] = so_l[slot];
        sym[so + p0 + j] = so_y[slot];
    }
}

}  // namespace

size_t match_rle_workspace_bytes(int S, int T, int K, bool same) {
    return rle_carve(S, T, K, same, nullptr).bytes;
}

int match_rle_launch_count(int S, int T, int K, bool same) {
    if (S == 0 || T == 0) return 0;
    return 4 + (K == 2 ? 1 : match_launch_count(S, T, K, same)) + 1;
}

cudaError_t launch_match_rle(const uint8_t *q, const uint8_t *k, const uint8_t *v, int S, int T, int K, int g,
                             int32_t *end_idx, int32_t *len, int32_t *sym, void *workspace, size_t ws_bytes,
                             cudaStream_t st) {
    const bool same = (q == k);
    const RleLayout L = rle_carve(S, T, K, same, workspace);
    if (L.bytes > ws_bytes) return cudaErrorInvalidValue;
    if (S == 0 || T == 0) {
        // still clear the matcher's status word, as the plain entry point does
        return launch_match(L.kr, L.kr, nullptr, S, T, K, g, end_idx, len, sym, workspace, L.match_bytes, st);
    }
    const int ntile = ceil_div(T, kRleTile);
    const int nwhich = same ? 1 : 2;
    const unsigned tiles = (unsigned)((int64_t)S * ntile * nwhich);
    rle_count_kernel<<<tiles, kRleThreads, 0, st>>>(q, k, T, ntile, nwhich, L.tcnt);
    rle_scan_kernel<<<(unsigned)ceil_div(S * nwhich, 8), 256, 0, st>>>(S, ntile, nwhich, L.tcnt, L.nrun);
    rle_write_kernel<<<tiles, kRleThreads, 0, st>>>(q, k, T, K, ntile, nwhich, L.tcnt, L.nrun, L.kr, L.qr, L.kstart,
                                                    L.qstart, L.krun);
    rle_bound_kernel<<<(unsigned)(device_sm_count() * 8), 256, 0, st>>>(S, T, g, L.nrun, L.qstart, L.krun, L.xb);
    cudaError_t e;
    if (K == 2) {
        uint32_t *status = reinterpret_cast<uint32_t *>(static_cast<char *>(workspace) + kStatusOffset);
        if ((e = cudaMemsetAsync(status, 0, sizeof(uint32_t), st)) != cudaSuccess) return e;
        rle_binary_kernel<<<(unsigned)(device_sm_count() * 8), 256, 0, st>>>(S, T, L.nrun, L.qr, L.kr, L.xb, L.rend,
                                                                             L.rlen, status);
    } else {
        e = launch_match(L.qr, L.kr, nullptr, S, T, K, g, L.rend, L.rlen, L.rsym, workspace, L.match_bytes, st, L.xb);
        if (e != cudaSuccess) return e;
    }
    rle_map_kernel<<<(unsigned)((int64_t)S * ntile), kRleThreads, 0, st>>>(q, v ? v : k, T, ntile, same ? 0 : 1,
                                                                           L.tcnt, L.kstart, L.rend, L.rlen, end_idx,
                                                                           len, sym);
    return cudaGetLastError();
}

}  // namespace rosa
