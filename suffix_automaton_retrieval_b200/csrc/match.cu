// Position-parallel exact matcher for the ROSA retrieval destination.
//
// "ROSA-Tuning" (arXiv 2602.02499), section 3.3 Eq. (16) and appendix B.3:
// for every stream and time t, the longest suffix of q[0..t] that occurs in
// the key stream ending at an admissible position i <= t - g, and the most
// recent such end i* (tau = i* + 1; -1 when nothing matches).  The pages run
// one online suffix automaton per stream on a CPU core (sections 2.2, 4.1);
// that is a chain of T dependent steps per stream.  Here the same quantity is
// computed position-parallel:
//
//   D(t, i) = longest common suffix of q[0..t] and k[0..i]
//           = longest common prefix of the reversed prefixes
//             Q_t = q[t] q[t-1] .. q[0]  and  K_i = k[i] k[i-1] .. k[0].
//
// 1. Sort all reversed prefixes of a stream (keys, and queries when q != k)
//    lexicographically: an LSD radix sort on the first D0 symbols packed in a
//    64-bit word, then prefix doubling (sort each tied group by the rank of
//    the prefix h symbols further back) until every group is a single string.
// 2. Adjacent longest-common-prefix array of the sorted order.
// 3. For a query at rank j, LCP with any other rank is the minimum of the
//    adjacent LCPs in between, so the best admissible key lies at the nearest
//    admissible rank on either side: L_t = max of the two.  The admissible
//    keys with LCP >= L_t form a rank interval around j; i* is the largest
//    admissible key position inside it.  Summaries over blocks of 32 and 1024
//    ranks (smallest key position, smallest inner LCP) let long scans skip.
//
// All kernels are stream-segmented: items of stream s occupy [s*n, (s+1)*n).
#include <climits>
#include <cstdint>
#include <mutex>
#include <cuda_runtime.h>

#include "../../include/rosa.h"
#include "common.cuh"
#include "kernels.h"

namespace rosa {
namespace {

constexpr int kRadixThreads = 256;
constexpr int kRadixIPT = 8;
constexpr int kRadixTile = kRadixThreads * kRadixIPT;   // 2048 items per tile
constexpr int kRadixBits = 8;
constexpr int kRadixBins = 1 << kRadixBits;
constexpr int kSmallGroup = 32;        // groups up to this size are sorted by one warp
constexpr int kSmemSortCap = 4096;     // larger groups up to this size sort in shared memory
constexpr int kLargeThreads = 512;
constexpr int kL1 = 32;                // summary block sizes (ranks)
constexpr int kL2 = 1024;
constexpr int kWLeafBits = 5;         // a wavelet leaf holds at most 32 values

int bits_for(int v) {   // number of bits to hold values 0..v
    int b = 0;
    while ((1 << b) <= v) ++b;
    return b;
}

struct Geometry {
    const int32_t *xb;       // per-query admissibility bound [S, T], or null for t - g
    int S, T, K, g, n;
    bool same;
    // Item kinds of a stream, T items each: keys (0), queries (1, unless
    // q == k, when the keys are the queries), then mcf counterfactual branch
    // kinds (bit j of the query symbol flipped).  br0 is the first branch
    // item; allkeys: every item is a key (q == k without branches).
    int mcf, br0, nkinds;
    bool allkeys;
    int bps, D0, idbits, keybits;
    int64_t N;
    int ntps, nb1, nb2;
    int wbits, ntw, nw;      // wavelet matrix: bits of a key position, 2048-element tiles, 64-bit words per stream
    int wlev;                // levels built: the rest (kWLeafBits) is scanned in the leaf
};

Geometry make_geometry(int S, int T, int K, int g, bool same, int mcf = 0) {
    Geometry G{};
    G.S = S; G.T = T; G.K = K; G.g = g; G.same = same;
    G.mcf = mcf;
    G.br0 = same ? T : 2 * T;
    G.nkinds = (same ? 1 : 2) + mcf;
    G.allkeys = same && mcf == 0;
    G.n = G.nkinds * T;
    G.N = (int64_t)S * G.n;
    G.bps = bits_for(K - 1);
    if (G.bps < 1) G.bps = 1;
    // 64-bit sort key: [D0 symbols | item id].  The symbols take at most 40
    // bits (five 8-bit radix passes) and at most what the item id leaves;
    // deeper ties go to prefix doubling.  Strings shorter than D0 (the first
    // D0 positions of a stream) are told apart by their initial place in the
    // array, which the stable sort keeps among equal symbols.
    G.idbits = bits_for(G.n > 0 ? G.n - 1 : 0);
    if (G.idbits < 1) G.idbits = 1;
    const int budget = min(G.bps <= 4 ? 32 : 40, 64 - G.idbits);   // small alphabets: fewer passes pay
    G.D0 = max(1, budget / G.bps);
    G.keybits = G.idbits + G.D0 * G.bps;
    G.ntps = ceil_div(G.n, kRadixTile);
    G.nb1 = ceil_div(G.n, kL1);
    G.nb2 = ceil_div(G.n, kL2);
    int wb = 0;
    while ((1 << wb) < T) ++wb;   // key positions 0..T-1
    G.wbits = wb < 1 ? 1 : wb;
    G.wlev = G.wbits > kWLeafBits ? G.wbits - kWLeafBits : 0;
    G.ntw = ceil_div(T, 2048);
    G.nw = (T >> 6) + 1;
    return G;
}

struct Workspace {
    uint32_t *status;
    int *counts;             // [2 buffers][2 kinds]
    uint64_t *keys[2];
    uint32_t *sa;            // item ids in sorted order (low bits of the sorted keys)
    int32_t *rank;
    int32_t *lcp;
    uint32_t *k2;
    uint32_t *hist;
    int2 *lists[2][2];       // [buffer][0 = small, 1 = large]
    int32_t *minpos1, *emin1, *ein1, *minpos2, *emin2, *ein2;
    int32_t *hard;           // ranks of queries left for the warp-cooperative phase
    int32_t *wq;             // output slots of queries waiting for a wavelet lookup
    int32_t *hardb;          // ranks of queries whose interval runs past their window (long L)
    int32_t *hardw;          // same, short L: waiting for a shared per-tile bound
    int32_t *btask;          // (tile, side, L) bound tasks
    int32_t *btab;           // their results
    int32_t *kcount;         // keys before each rank (q != k)
    int *ktile;              // keys per 2048-rank tile
    uint32_t *wvals[2];      // wavelet level sequences
    int *wcnt;               // [level][stream][tile] ones per wavelet tile
    void *words;             // [stream][level][word] rank directory + bits (16 B each)
    int *wz;                 // [stream][level] zeros per level
    int32_t *flip[3];        // counterfactual runs: flipped-bit end / len / sym [S, T, mcf]
    size_t bytes;
};

size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

// Lays the workspace out from `base` (or only measures it when base == nullptr).
Workspace carve(const Geometry &G, void *base) {
    Workspace W{};
    size_t off = 0;
    char *b = static_cast<char *>(base);
    auto take = [&](size_t bytes) -> void * {
        void *p = b ? b + off : nullptr;
        off += align256(bytes);
        return p;
    };
    const size_t N = (size_t)G.N;
    const size_t list_cap = N / 2 + 1;
    W.status = (uint32_t *)take(256);
    W.counts = (int *)take(64 * sizeof(int));   // list, hard-query and tie counters (cleared with status)
    W.keys[0] = (uint64_t *)take(N * 8);
    W.keys[1] = (uint64_t *)take(N * 8);
    W.sa = (uint32_t *)take(N * 4);
    W.rank = (int32_t *)take(N * 4);
    W.lcp = (int32_t *)take(N * 4);
    W.k2 = (uint32_t *)take(N * 4);
    W.hist = (uint32_t *)take((size_t)G.S * kRadixBins * G.ntps * 4);
    for (int i = 0; i < 2; ++i)
        for (int j = 0; j < 2; ++j) W.lists[i][j] = (int2 *)take(list_cap * sizeof(int2));
    W.minpos1 = (int32_t *)take((size_t)G.S * G.nb1 * 4);
    W.emin1 = (int32_t *)take((size_t)G.S * G.nb1 * 4);
    W.ein1 = (int32_t *)take((size_t)G.S * G.nb1 * 4);
    W.minpos2 = (int32_t *)take((size_t)G.S * G.nb2 * 4);
    W.emin2 = (int32_t *)take((size_t)G.S * G.nb2 * 4);
    W.ein2 = (int32_t *)take((size_t)G.S * G.nb2 * 4);
    W.hard = (int32_t *)take(N * 4);
    const size_t nqueries = (size_t)G.S * G.T * (1 + G.mcf);   // queries and branch queries
    W.wq = (int32_t *)take(nqueries * 4);
    W.hardb = (int32_t *)take(nqueries * 4);
    W.hardw = (int32_t *)take(nqueries * 4);
    const size_t ntiles_resolve = (size_t)G.S * ceil_div(G.n, 1024);
    W.btask = (int32_t *)take(ntiles_resolve * 128 * 4);
    W.btab = (int32_t *)take(ntiles_resolve * 128 * 4);
    W.kcount = (int32_t *)take(N * 4);
    W.ktile = (int *)take((size_t)G.S * G.ntps * 4);
    W.wvals[0] = (uint32_t *)take((size_t)G.S * G.T * 4);
    W.wvals[1] = (uint32_t *)take((size_t)G.S * G.T * 4);
    W.wcnt = (int *)take((size_t)G.wbits * G.S * G.ntw * 4);
    W.words = take((size_t)G.S * G.wbits * G.nw * 16);
    W.wz = (int *)take((size_t)G.S * G.wbits * 4);
    if (G.mcf > 0) {   // counterfactual runs: the flipped-bit results before assembly
        const size_t nf = (size_t)G.S * G.T * G.mcf;
        for (int i = 0; i < 3; ++i) W.flip[i] = (int32_t *)take(nf * 4);
    }
    W.bytes = off;
    return W;
}

// Largest admissible key position for the query at position t of stream s:
// t - g, or the caller's bound where one is given (run-level retrieval).
__device__ __forceinline__ int query_bound(const Geometry &G, int s, int t) {
    return G.xb ? __ldg(G.xb + (int64_t)s * G.T + t) : t - G.g;
}

// Position of item x in its string (keys 0..T-1, then queries).
__device__ __forceinline__ int item_pos(uint32_t x, int T) {
    const int i = (int)x;
    return i < T ? i : (i < 2 * T ? i - T : (int)(x % (uint32_t)T));
}
// Stream of a global item index (item counts stay below 2^31).
__device__ __forceinline__ int stream_of(int64_t gi, int n) { return (int)((uint32_t)gi / (uint32_t)n); }

// ---------------------------------------------------------------------------
// 1a. Round-0 keys: first D0 symbols of the reversed prefix, most significant
//     first, zero-padded past the start, then the item id in the low bits
//     (carried through the sort, never sorted on).
// ---------------------------------------------------------------------------
// One CTA per 2048 positions of one string (a stream's keys or queries).
// The positions and the D0 - 1 symbols before them are staged in shared
// memory; thread t builds the keys of positions 8t .. 8t+7, each from the
// previous one by one shift (the oldest symbol drops out at the bottom), and
// the keys leave through shared memory in coalesced stores.
constexpr int kKeysThreads = 256;
constexpr int kKeysTile = 2048;
constexpr int kMaxD0 = 40;

__global__ void __launch_bounds__(kKeysThreads)
keys0_kernel(const uint8_t *__restrict__ q, const uint8_t *__restrict__ k, Geometry G,
             uint64_t *__restrict__ keys, uint32_t *__restrict__ status) {
    __shared__ uint8_t sb[kMaxD0 + kKeysTile];
    __shared__ uint64_t sk[kKeysThreads * 9];   // 9 words per thread: conflict-free
    const int ntile = ceil_div(G.T, kKeysTile);
    const int sp = blockIdx.x / ntile, tile = blockIdx.x - sp * ntile;
    const int s = sp / G.nkinds, kind = sp - s * G.nkinds;
    const int kind0 = G.same ? 1 : 2;                 // first branch kind
    const int flip = kind >= kind0 ? 1 << (kind - kind0) : 0;   // branch: this query bit flipped
    const uint8_t *a = (kind == 0 ? k : q) + (int64_t)s * G.T;
    const int p0 = tile * kKeysTile;
    const int lim = min(kKeysTile, G.T - p0);
#pragma unroll
    for (int u = 0; u < (kMaxD0 + kKeysTile + kKeysThreads - 1) / kKeysThreads; ++u) {   // all loads in flight
        const int i = u * kKeysThreads + threadIdx.x;
        const int p = p0 - kMaxD0 + i;
        if (i < kMaxD0 + kKeysTile)
            sb[i] = (p >= 0 && p < G.T) ? a[p] : 0;   // zeros before the start pad short strings
    }
    __syncthreads();
    const uint32_t symmask = (1u << G.bps) - 1u;
    const int top = (G.D0 - 1) * G.bps;
    const int j0 = threadIdx.x * 8;
    bool bad = false;
    if (j0 < lim) {
        const uint8_t *e = sb + kMaxD0 + j0;      // e[-m] = symbol at p0 + j0 - m
        uint64_t chars = 0;
        for (int m = 0; m < G.D0; ++m) chars = (chars << G.bps) | ((uint32_t)e[-m] & symmask);
        for (int u = 0; u < 8 && j0 + u < lim; ++u) {
            if (u > 0) chars = (chars >> G.bps) | ((uint64_t)((uint32_t)e[u] & symmask) << top);
            bad |= (uint32_t)e[u] >= (uint32_t)G.K;
            const int x = kind * G.T + p0 + j0 + u;
            uint64_t c = chars;
            if (flip) c ^= (uint64_t)flip << top;       // the branch symbol, then the query history
            sk[threadIdx.x * 9 + u] = (c << G.idbits) | (uint64_t)x;
        }
    }
    if (bad) atomicOr(status, ROSA_DEV_SYMBOL_RANGE);
    __syncthreads();
    // Initial place: the short strings first, by length, then by kind (key,
    // query, branches); then the rest by kind and position.  Equal symbols
    // then sort as (length, item id), the order of the full comparison.
    uint64_t *out = keys + (int64_t)s * G.n;
    const int m0 = min(G.D0, G.T);
    for (int i = threadIdx.x; i < lim; i += kKeysThreads) {
        const int p = p0 + i;
        const int pos = p < m0 ? p * G.nkinds + kind : G.nkinds * m0 + kind * (G.T - m0) + (p - m0);
        out[pos] = sk[(i >> 3) * 9 + (i & 7)];
    }
}

// ---------------------------------------------------------------------------
// 1b. Segmented LSD radix sort, 8-bit digits, tiles of 2048 items that never
//     straddle a stream.  hist layout: [stream][tile-in-stream][digit].
// ---------------------------------------------------------------------------
constexpr int kRadixWarps = kRadixThreads / 32;
constexpr int kWarpItems = kRadixTile / kRadixWarps;   // 256 contiguous items per warp

__global__ void __launch_bounds__(kRadixThreads)
radix_hist_kernel(const uint64_t *__restrict__ keys, Geometry G, int shift, uint32_t *__restrict__ hist) {
    __shared__ uint32_t cnt[kRadixBins];
    const int tile = blockIdx.x;
    const int s = tile / G.ntps, tt = tile - s * G.ntps;
    cnt[threadIdx.x] = 0;
    __syncthreads();
    const int64_t base = (int64_t)s * G.n + (int64_t)tt * kRadixTile;
    const int lim = min(kRadixTile, G.n - tt * kRadixTile);
    uint64_t key[kRadixIPT];
#pragma unroll
    for (int u = 0; u < kRadixIPT; ++u) {   // loads first: eight in flight per thread
        const int i = u * kRadixThreads + threadIdx.x;
        key[u] = i < lim ? keys[base + i] : 0ull;
    }
#pragma unroll
    for (int u = 0; u < kRadixIPT; ++u)
        if (u * kRadixThreads + (int)threadIdx.x < lim) atomicAdd(&cnt[(key[u] >> shift) & (kRadixBins - 1)], 1u);
    __syncthreads();
    hist[((int64_t)s * G.ntps + tt) * kRadixBins + threadIdx.x] = cnt[threadIdx.x];
}

// Per stream: turn the [tile][digit] counts into each tile's first output
// slot per digit (digit-major order, tiles in order within a digit).
__global__ void __launch_bounds__(kRadixBins)
radix_scan_kernel(uint32_t *__restrict__ hist, int ntps) {
    __shared__ uint32_t ws[kRadixBins / 32 + 1];
    uint32_t *h = hist + (int64_t)blockIdx.x * ntps * kRadixBins + threadIdx.x;
    uint32_t total = 0;
    for (int t = 0; t < ntps; ++t) total += h[(int64_t)t * kRadixBins];
    uint32_t run = block_exclusive_scan<kRadixBins>(total, ws, nullptr);
    for (int t = 0; t < ntps; ++t) {
        const uint32_t c = h[(int64_t)t * kRadixBins];
        h[(int64_t)t * kRadixBins] = run;
        run += c;
    }
}

// Stable scatter of one tile.  Warp w owns items [256w, 256w+256) of the
// tile; ranks come from warp-private digit counters, so the whole tile needs
// only three block barriers.
__global__ void __launch_bounds__(kRadixThreads, 4)
radix_scatter_kernel(const uint64_t *__restrict__ kin, uint64_t *__restrict__ kout, Geometry G, int shift,
                     const uint32_t *__restrict__ hist) {
    __shared__ uint64_t sk[kRadixTile];
    __shared__ uint32_t wcnt[kRadixWarps][kRadixBins];   // per-warp digit counts, then per-warp offsets
    __shared__ uint32_t tstart[kRadixBins];
    __shared__ uint32_t gofs[kRadixBins];
    __shared__ uint32_t wsum[kRadixWarps + 1];

    const int tile = blockIdx.x;
    const int s = tile / G.ntps, tt = tile - s * G.ntps;
    const int64_t seg = (int64_t)s * G.n;
    const int64_t base = seg + (int64_t)tt * kRadixTile;
    const int lim = min(kRadixTile, G.n - tt * kRadixTile);
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;

    gofs[threadIdx.x] = hist[((int64_t)s * G.ntps + tt) * kRadixBins + threadIdx.x];
#pragma unroll
    for (int w = 0; w < kRadixWarps; ++w) wcnt[w][threadIdx.x] = 0;
    __syncthreads();

    uint64_t key[kRadixIPT];
    unsigned peer[kRadixIPT];
    const int wbase = warp * kWarpItems;
    const unsigned lt = lanemask_lt();
    // loads first: eight independent loads in flight per thread
#pragma unroll
    for (int u = 0; u < kRadixIPT; ++u) {
        const int i = wbase + u * 32 + lane;
        key[u] = i < lim ? kin[base + i] : 0ull;
    }
    // pass 1: lanes holding the same digit (8 ballots, one per digit bit);
    // each digit's lowest lane adds the group size to the warp's counter
#pragma unroll
    for (int u = 0; u < kRadixIPT; ++u) {
        const bool ok = wbase + u * 32 + lane < lim;
        const unsigned d = (unsigned)(key[u] >> shift) & (kRadixBins - 1);
        unsigned pm = __ballot_sync(ROSA_FULL_MASK, ok);
#pragma unroll
        for (int bit = 0; bit < kRadixBits; ++bit) {
            const unsigned bm = __ballot_sync(ROSA_FULL_MASK, (d >> bit) & 1u);
            pm &= ((d >> bit) & 1u) ? bm : ~bm;
        }
        peer[u] = pm;
        if (ok && (pm & lt) == 0) wcnt[warp][d] += __popc(pm);
        __syncwarp();
    }
    __syncthreads();
    // digit totals -> tile start per digit; per-warp offsets within the digit
    {
        const int d = threadIdx.x;
        uint32_t tot = 0;
#pragma unroll
        for (int w = 0; w < kRadixWarps; ++w) tot += wcnt[w][d];
        const uint32_t st = block_exclusive_scan<kRadixThreads>(tot, wsum, nullptr);
        tstart[d] = st;
        uint32_t run = st;
#pragma unroll
        for (int w = 0; w < kRadixWarps; ++w) {
            const uint32_t c = wcnt[w][d];
            wcnt[w][d] = run;
            run += c;
        }
    }
    __syncthreads();
    // pass 2: place each item at its stable slot in shared memory
#pragma unroll
    for (int u = 0; u < kRadixIPT; ++u) {
        const bool ok = wbase + u * 32 + lane < lim;
        const unsigned d = (unsigned)(key[u] >> shift) & (kRadixBins - 1);
        const unsigned before = __popc(peer[u] & lt);
        if (ok) {
            const uint32_t pos = wcnt[warp][d] + before;
            sk[pos] = key[u];
        }
        __syncwarp();
        if (ok && before == 0) wcnt[warp][d] += __popc(peer[u]);
        __syncwarp();
    }
    __syncthreads();
    for (int j = threadIdx.x; j < lim; j += kRadixThreads) {
        const uint64_t kk = sk[j];
        const int d = (int)((kk >> shift) & (kRadixBins - 1));
        const int64_t dst = seg + gofs[d] + (j - tstart[d]);
        kout[dst] = kk;
    }
}

// ---------------------------------------------------------------------------
// 1c. Groups after round 0: rank = position of the group head; groups of more
//     than one incomplete string (p + 1 > D0) go to the unresolved lists
//     (small: up to kSmallGroup members, large: more).
// ---------------------------------------------------------------------------

// One CTA per 2048-item tile of a stream's round-0 order; thread t owns
// items [8t, 8t+8).  The tile passes through shared memory (9 words per
// thread, conflict-free) so that global loads and stores stay coalesced.
// Group heads (key differs from the previous item) come from a block-wide
// max-scan; a group running in from the previous tile is found by a warp
// search.  The adjacent LCP is written here wherever it cannot change later:
// across different round-0 keys (it depends on the keys only) and inside
// groups of identical complete strings.  Positions inside unresolved groups
// are listed (-1 in lcp); their LCP is taken after doubling.
constexpr int kG0Stride = 9;
__device__ __forceinline__ int g0_slot(int i) { return (i >> 3) * kG0Stride + (i & 7); }

// Round-0 group key: [D0 symbols | available length 0..D0+1], the length
// taken from the item id.  Sorted keys are ascending in it.
constexpr int kAvailBits = 6;   // D0 + 1 <= 41
__device__ __forceinline__ uint64_t g0_key(uint64_t full, const Geometry &G) {
    const int p = item_pos((uint32_t)(full & ((1ull << G.idbits) - 1ull)), G.T);
    return ((full >> G.idbits) << kAvailBits) | (uint64_t)min(p + 1, G.D0 + 1);
}

__global__ void __launch_bounds__(256)
groups0_kernel(const uint64_t *__restrict__ keys, uint32_t *__restrict__ sa, Geometry G, int32_t *__restrict__ rank,
               int32_t *__restrict__ lcp, int2 *small, int2 *large, int *counts_next, int32_t *__restrict__ ties,
               int *tie_count) {
    __shared__ uint64_t sk[256 * kG0Stride];
    __shared__ int32_t so[256 * kG0Stride];
    __shared__ int wmax[8];
    __shared__ uint32_t scan_ws[9];
    __shared__ int list_base[3];
    __shared__ int look;
    const int s = blockIdx.x / G.ntps, tt = blockIdx.x - s * G.ntps;
    const int64_t seg = (int64_t)s * G.n;
    const int j0 = tt * kRadixTile;
    const int lim = min(kRadixTile, G.n - j0);
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const uint64_t idmask = (1ull << G.idbits) - 1ull;
    const uint64_t amask = (1ull << kAvailBits) - 1ull;
    const int base = threadIdx.x * 8;
    for (int i = threadIdx.x; i < lim; i += 256) sk[g0_slot(i)] = keys[seg + j0 + i];
    if (warp == 0) {
        // Head of the group that runs into this tile from the previous one.
        // Keys are sorted, so the group is the run of keys equal to keys[j0]:
        // its head is a lower bound, found 32 positions per step.
        int h = -1;
        if (j0 > 0 && lim > 0) {
            const uint64_t kk = g0_key(keys[seg + j0], G);
            // backward probes j0-1 .. j0-32 first: most runs are short
            const int p0 = j0 - 1 - lane;
            const unsigned ne = ~__ballot_sync(ROSA_FULL_MASK, p0 >= 0 && g0_key(keys[seg + p0], G) == kk);
            int lo, hi;                            // keys[hi] == kk; the head lies in [lo, hi]
            if (ne) lo = hi = j0 - (__ffs(ne) - 1);
            else { lo = 0; hi = j0 - 32; }
            while (lo < hi) {
                const int64_t span = hi - lo;
                const int p = lo + (int)(span * lane / 32);
                const unsigned b = __ballot_sync(ROSA_FULL_MASK, g0_key(keys[seg + p], G) == kk);
                if (b & 1u) { hi = lo; break; }
                const int f = b ? __ffs(b) - 1 : 32;   // first probe inside the run
                const int nlo = lo + (int)(span * (f - 1) / 32) + 1;
                if (f < 32) hi = lo + (int)(span * f / 32);
                lo = nlo;
            }
            if (hi < j0) h = hi;
        }
        look = h;
    }
    __syncthreads();
    uint64_t kv[8];
    uint32_t id[8];
    int hp = -1;
    unsigned headbits = 0;
    uint64_t prev = ~0ull;
    if (base < lim && j0 + base > 0) prev = g0_key(base > 0 ? sk[g0_slot(base - 1)] : keys[seg + j0 - 1], G);
#pragma unroll
    for (int e = 0; e < 8; ++e) {
        const int jl = base + e, j = j0 + jl;
        const bool ok = jl < lim;
        const uint64_t full = ok ? sk[g0_slot(jl)] : 0ull;
        const uint64_t k = g0_key(full, G);
        kv[e] = k;
        id[e] = (uint32_t)(full & idmask);
        if (ok) {
            const bool head = (j == 0) || k != prev;
            if (head) { hp = j; headbits |= 1u << e; }
            int l = -1;   // -1: decided after doubling
            const int a2 = (int)(k & amask);
            if (j == 0) {
                l = 0;
            } else if (head) {
                const int a1 = (int)(prev & amask);
                const uint64_t x = (prev >> kAvailBits) ^ (k >> kAvailBits);
                int diff = G.D0;
                if (x) diff = (__clzll((long long)x) - (64 - G.D0 * G.bps)) / G.bps;
                l = min(diff, min(min(a1, G.D0), min(a2, G.D0)));
            } else if (a2 <= G.D0) {
                l = a2;   // identical complete strings
            }
            so[g0_slot(jl)] = l;
            prev = k;
        }
    }
    // first key after this thread's chunk, for end-of-group tests
    uint64_t nk = ~0ull;
    if (base + 8 < lim) nk = g0_key(sk[g0_slot(base + 8)], G);
    else if (base + 8 == lim && j0 + lim < G.n) nk = g0_key(keys[seg + j0 + lim], G);
    // exclusive max-scan of the threads' last head positions
    int incl = hp;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(ROSA_FULL_MASK, incl, o);
        if (lane >= o) incl = max(incl, y);
    }
    if (lane == 31) wmax[warp] = incl;
    __syncthreads();
    for (int i = threadIdx.x; i < lim; i += 256) lcp[seg + j0 + i] = so[g0_slot(i)];
    int carry = look;
    for (int w2 = 0; w2 < warp; ++w2) carry = max(carry, wmax[w2]);
    const int excl = __shfl_up_sync(ROSA_FULL_MASK, incl, 1);
    if (lane > 0) carry = max(carry, excl);
    __syncthreads();   // so[] is reused for the item ids
    // Pass 1: ranks, and which items end a group to refine or are ties.
    unsigned tiebits = 0, smallbits = 0, largebits = 0;
    int h = carry;
#pragma unroll
    for (int e = 0; e < 8; ++e) {
        const int jl = base + e, j = j0 + jl;
        const bool head = (headbits >> e) & 1u;
        if (head) h = j;
        if (jl < lim) {
            so[g0_slot(jl)] = (int32_t)id[e];
            rank[seg + id[e]] = h;
            const uint64_t next = e < 7 ? (jl + 1 < lim ? kv[e + 1] : ~0ull) : nk;
            const bool last = j + 1 >= G.n || next != kv[e];
            const bool incomplete = (int)(kv[e] & amask) > G.D0;
            if (last && j > h && incomplete) {
                if (j - h + 1 <= kSmallGroup) smallbits |= 1u << e;
                else largebits |= 1u << e;
            }
            if (!head && incomplete) tiebits |= 1u << e;
        }
    }
    // Pass 2: one atomic per list per CTA.  Counts share a word: ties <= 2048
    // (12 bits), group ends <= 1024 (11 bits: a refined group has two members
    // in the tile), ends of groups over 32 members <= 63 (9 bits).
    const uint32_t packed = __popc(tiebits) | (__popc(smallbits) << 12) | (__popc(largebits) << 23);
    uint32_t total;
    const uint32_t ex = block_exclusive_scan<256>(packed, scan_ws, &total);
    if (threadIdx.x == 0) {
        const uint32_t nt = total & 4095u, ns = (total >> 12) & 2047u, nl = total >> 23;
        list_base[0] = nt ? atomicAdd(tie_count, (int)nt) : 0;
        list_base[1] = ns ? atomicAdd(&counts_next[0], (int)ns) : 0;
        list_base[2] = nl ? atomicAdd(&counts_next[1], (int)nl) : 0;
    }
    __syncthreads();
    int it = list_base[0] + (int)(ex & 4095u), is = list_base[1] + (int)((ex >> 12) & 2047u),
        il = list_base[2] + (int)(ex >> 23);
    h = carry;
#pragma unroll
    for (int e = 0; e < 8; ++e) {
        const int j = j0 + base + e;
        if ((headbits >> e) & 1u) h = j;
        if ((tiebits >> e) & 1u) ties[it++] = (int32_t)(seg + j);
        if ((smallbits >> e) & 1u) small[is++] = make_int2((int)(seg + h), j - h + 1);
        if ((largebits >> e) & 1u) large[il++] = make_int2((int)(seg + h), j - h + 1);
    }
    for (int i = threadIdx.x; i < lim; i += 256) sa[seg + j0 + i] = (uint32_t)so[g0_slot(i)];
}

// ---------------------------------------------------------------------------
// 1d. Prefix doubling at depth h: sort each unresolved group by the rank of
//     the same-kind prefix h symbols further back, then split into new groups.
//     Groups of up to 32 members (nearly all of them) take one thread each;
//     larger ones a warp (keys, regroup) and a CTA (sort).  Within a round all
//     keys are read before any rank changes (separate launches).
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint64_t pair_key(uint32_t k2, uint32_t x) { return ((uint64_t)k2 << 32) | x; }

// The item whose string is item x's with its first h symbols removed: the
// same kind h positions back, except that a branch's history is the query's
// (a branch differs from its query only in the first symbol).
__device__ __forceinline__ uint32_t back_item(const Geometry &G, uint32_t x, int64_t h) {
    if ((int)x < G.br0) return x - (uint32_t)h;
    return (uint32_t)((G.same ? 0 : G.T) + item_pos(x, G.T) - h);
}

// Small groups: one thread computes its members' keys and insertion-sorts
// them in place.  Large groups: one warp computes the keys.
__global__ void dbl_keys_sort_kernel(const int2 *__restrict__ small, const int2 *__restrict__ large,
                                     const int *__restrict__ counts, Geometry G, int64_t h, uint32_t *__restrict__ sa,
                                     const int32_t *__restrict__ rank, uint32_t *__restrict__ k2) {
    const int ns = counts[0], nl = counts[1];
    const int64_t tid = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
    const int64_t nth = (int64_t)gridDim.x * blockDim.x;
    for (int64_t gidx = tid; gidx < ns; gidx += nth) {
        const int2 gr = small[gidx];
        const int64_t seg = (gr.x / G.n) * (int64_t)G.n;
        uint32_t *gs = sa + gr.x;
        uint32_t *gk = k2 + gr.x;
        // keys first: the members' rank loads are independent of each other
        for (int m = 0; m < gr.y; ++m) gk[m] = (uint32_t)rank[seg + back_item(G, gs[m], h)];
        for (int m = 1; m < gr.y; ++m) {   // insertion sort of (key, id) pairs
            const uint32_t x = gs[m], kk = gk[m];
            const uint64_t key = pair_key(kk, x);
            int i = m - 1;
            while (i >= 0 && pair_key(gk[i], gs[i]) > key) {
                gk[i + 1] = gk[i];
                gs[i + 1] = gs[i];
                --i;
            }
            gk[i + 1] = kk;
            gs[i + 1] = x;
        }
    }
    const int lane = threadIdx.x & 31;
    for (int64_t gidx = tid >> 5; gidx < nl; gidx += nth >> 5) {
        const int2 gr = large[gidx];
        const int64_t seg = (gr.x / G.n) * (int64_t)G.n;
        for (int m = lane; m < gr.y; m += 32) {
            const uint32_t x = sa[gr.x + m];
            k2[gr.x + m] = (uint32_t)rank[seg + back_item(G, x, h)];
        }
    }
}

// Ascending-only bitonic sort of n keys (virtual +inf padding to a power of 2).
__device__ void bitonic_sort(uint64_t *a, int n) {
    int np2 = 1;
    while (np2 < n) np2 <<= 1;
    for (int kk = 2; kk <= np2; kk <<= 1) {
        const int half = kk >> 1;
        for (int i = threadIdx.x; i < np2 / 2; i += blockDim.x) {
            const int blk = i / half, off = i - blk * half;
            const int lo = blk * kk + off, hi = blk * kk + kk - 1 - off;
            if (hi < n && a[lo] > a[hi]) { const uint64_t t = a[lo]; a[lo] = a[hi]; a[hi] = t; }
        }
        __syncthreads();
        for (int jj = kk >> 2; jj >= 1; jj >>= 1) {
            for (int i = threadIdx.x; i < np2 / 2; i += blockDim.x) {
                const int blk = i / jj, off = i - blk * jj;
                const int lo = blk * 2 * jj + off, hi = lo + jj;
                if (hi < n && a[lo] > a[hi]) { const uint64_t t = a[lo]; a[lo] = a[hi]; a[hi] = t; }
            }
            __syncthreads();
        }
    }
}

// One CTA per group of more than 32: shared memory up to kSmemSortCap, else
// in place in the scratch key buffer (global memory).
__global__ void __launch_bounds__(kLargeThreads)
dbl_sort_large_kernel(const int2 *__restrict__ large, const int *__restrict__ counts,
                      uint32_t *__restrict__ sa, uint32_t *__restrict__ k2, uint64_t *__restrict__ scratch) {
    __shared__ uint64_t buf[kSmemSortCap];
    const int nl = counts[1];
    for (int gidx = blockIdx.x; gidx < nl; gidx += gridDim.x) {
        const int2 gr = large[gidx];
        uint64_t *a = gr.y <= kSmemSortCap ? buf : scratch + gr.x;
        for (int m = threadIdx.x; m < gr.y; m += blockDim.x) a[m] = pair_key(k2[gr.x + m], sa[gr.x + m]);
        __syncthreads();
        bitonic_sort(a, gr.y);
        for (int m = threadIdx.x; m < gr.y; m += blockDim.x) {
            const uint64_t key = a[m];
            sa[gr.x + m] = (uint32_t)key;
            k2[gr.x + m] = (uint32_t)(key >> 32);
        }
        __syncthreads();
    }
}

// Split sorted groups at k2 changes.  New group id = local head position;
// new groups of more than one incomplete string (p + 1 > 2h) go on.  List
// appends take one atomic per warp (per list), not one per group.
__global__ void dbl_regroup_kernel(const int2 *__restrict__ small, const int2 *__restrict__ large,
                                   const int *__restrict__ counts, Geometry G, int64_t h2,
                                   const uint32_t *__restrict__ sa, const uint32_t *__restrict__ k2,
                                   int32_t *__restrict__ rank, int2 *nsmall, int2 *nlarge, int *counts_next) {
    const int ns = counts[0], nl = counts[1];
    const int lane = threadIdx.x & 31;
    const int64_t tid = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
    const int64_t nth = (int64_t)gridDim.x * blockDim.x;
    // Small groups, one per thread; the loop runs warp-uniformly.  A group of
    // at most 32 only splits into small groups.
    for (int64_t gb = tid - lane; gb < ns; gb += nth) {
        const int64_t gidx = gb + lane;
        const int2 gr = gidx < ns ? small[gidx] : make_int2(0, 0);
        const int64_t seg = (gr.x / G.n) * (int64_t)G.n;
        const int jstart = (int)(gr.x - seg);
        int head = 0, npush = 0;
        for (int m = 0; m < gr.y; ++m) {
            const uint32_t kk = k2[gr.x + m];
            if (m > 0 && kk != k2[gr.x + m - 1]) head = m;
            const uint32_t x = sa[gr.x + m];
            rank[seg + x] = jstart + head;
            const bool last = (m == gr.y - 1) || (k2[gr.x + m + 1] != kk);
            if (last && m > head && (int64_t)item_pos(x, G.T) + 1 > h2) ++npush;
        }
        int incl = npush;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(ROSA_FULL_MASK, incl, o);
            if (lane >= o) incl += y;
        }
        int wbase = 0;
        if (lane == 31 && incl) wbase = atomicAdd(&counts_next[0], incl);
        int slot = __shfl_sync(ROSA_FULL_MASK, wbase, 31) + incl - npush;
        if (npush) {
            head = 0;
            for (int m = 0; m < gr.y; ++m) {
                const uint32_t kk = k2[gr.x + m];
                if (m > 0 && kk != k2[gr.x + m - 1]) head = m;
                const bool last = (m == gr.y - 1) || (k2[gr.x + m + 1] != kk);
                if (last && m > head && (int64_t)item_pos(sa[gr.x + m], G.T) + 1 > h2)
                    nsmall[slot++] = make_int2(gr.x + head, m - head + 1);
            }
        }
    }
    for (int64_t gidx = tid >> 5; gidx < nl; gidx += nth >> 5) {
        const int2 gr = large[gidx];
        const int64_t seg = (gr.x / G.n) * (int64_t)G.n;
        const int jstart = (int)(gr.x - seg);
        int carry = jstart;
        for (int m0 = 0; m0 < gr.y; m0 += 32) {
            const int m = m0 + lane;
            const bool ok = m < gr.y;
            const uint32_t kk = ok ? k2[gr.x + m] : 0u;
            const bool head = ok && (m == 0 || k2[gr.x + m - 1] != kk);
            int hp = head ? jstart + m : -1;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int y = __shfl_up_sync(ROSA_FULL_MASK, hp, o);
                if (lane >= o) hp = max(hp, y);
            }
            const int gid = max(hp, carry);
            bool push = false;
            int size = 0;
            if (ok) {
                const uint32_t x = sa[gr.x + m];
                rank[seg + x] = gid;
                const bool last = (m == gr.y - 1) || (k2[gr.x + m + 1] != kk);
                size = jstart + m - gid + 1;
                push = last && size > 1 && (int64_t)item_pos(x, G.T) + 1 > h2;
            }
            const unsigned ms = __ballot_sync(ROSA_FULL_MASK, push && size <= kSmallGroup);
            const unsigned ml = __ballot_sync(ROSA_FULL_MASK, push && size > kSmallGroup);
            int bs = 0, bl = 0;
            if (lane == 0) {
                if (ms) bs = atomicAdd(&counts_next[0], __popc(ms));
                if (ml) bl = atomicAdd(&counts_next[1], __popc(ml));
            }
            bs = __shfl_sync(ROSA_FULL_MASK, bs, 0);
            bl = __shfl_sync(ROSA_FULL_MASK, bl, 0);
            if (push) {
                const int2 ng = make_int2((int)(seg + gid), size);
                if (size <= kSmallGroup) nsmall[bs + __popc(ms & lanemask_lt())] = ng;
                else nlarge[bl + __popc(ml & lanemask_lt())] = ng;
            }
            carry = __shfl_sync(ROSA_FULL_MASK, gid, 31);
        }
    }
}

// ---------------------------------------------------------------------------
// 2. Adjacent LCP of the final order.  groups0 already wrote every position
//    whose neighbours differ in their round-0 keys; the rest lie inside tied
//    groups, whose members share the first D0 symbols.
// ---------------------------------------------------------------------------
constexpr int kLcpSerial = 24;         // symbols past D0 one thread compares before handing off

// Positions listed by groups0 (inside unresolved round-0 groups): their
// neighbours share the first D0 symbols; compare onward in the final order.
__global__ void lcp_ties_kernel(const uint8_t *__restrict__ q, const uint8_t *__restrict__ k, Geometry G,
                                const uint32_t *__restrict__ sa, int32_t *__restrict__ lcp,
                                const int32_t *__restrict__ ties, const int *__restrict__ tie_count,
                                int32_t *__restrict__ long_list, int *long_count) {
    const int nt = *tie_count;
    for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < nt; e += (int64_t)gridDim.x * blockDim.x) {
        const int64_t gi = ties[e];
        const int s = stream_of(gi, G.n);
        const uint32_t x1 = sa[gi - 1], x2 = sa[gi];
        const uint8_t *s1 = ((int)x1 < G.T ? k : q) + (int64_t)s * G.T;
        const uint8_t *s2 = ((int)x2 < G.T ? k : q) + (int64_t)s * G.T;
        const int p1 = item_pos(x1, G.T), p2 = item_pos(x2, G.T);
        int m = G.D0;
        const int lim = min(p1, p2) + 1;
        const int stop = min(lim, G.D0 + kLcpSerial);
        while (m < stop && s1[p1 - m] == s2[p2 - m]) ++m;
        lcp[gi] = m;
        if (m == stop && m < lim) long_list[atomicAdd(long_count, 1)] = (int32_t)gi;   // still equal: a warp finishes it
    }
}

// Four symbols of a stream ending at byte address `e` (the symbol at e in the
// top byte, e-3 in the low byte), from aligned words that lie inside
// [lo, hi); returns false (nothing read) where they would not.
__device__ __forceinline__ bool load4_back(const uint8_t *e, const uint8_t *lo, const uint8_t *hi, uint32_t &v) {
    const uintptr_t a = (uintptr_t)(e - 3);
    const uintptr_t w = a & ~(uintptr_t)3;
    const int sh = (int)(a & 3);
    if (w < (uintptr_t)lo || w + (sh ? 8 : 4) > (uintptr_t)hi) return false;
    const uint32_t w0 = *reinterpret_cast<const uint32_t *>(w);
    const uint32_t w1 = sh ? *reinterpret_cast<const uint32_t *>(w + 4) : 0u;
    v = __funnelshift_r(w0, w1, 8 * sh);
    return true;
}

// Long common prefixes (repeats): one warp per pair, 4 symbols per lane and
// 128 per step, compared as words.
__global__ void lcp_long_kernel(const uint8_t *__restrict__ q, const uint8_t *__restrict__ k, Geometry G,
                                const uint32_t *__restrict__ sa, int32_t *__restrict__ lcp,
                                const int32_t *__restrict__ long_list, const int *__restrict__ long_count) {
    const int nl = *long_count;
    const int lane = threadIdx.x & 31;
    const int64_t wid = (blockIdx.x * (int64_t)blockDim.x + threadIdx.x) >> 5;
    const int64_t nw = ((int64_t)gridDim.x * blockDim.x) >> 5;
    const int64_t total = (int64_t)G.S * G.T;
    for (int64_t e = wid; e < nl; e += nw) {
        const int64_t gi = long_list[e];
        const int s = stream_of(gi, G.n);
        const uint32_t x1 = sa[gi - 1], x2 = sa[gi];
        const uint8_t *b1 = (int)x1 < G.T ? k : q, *b2 = (int)x2 < G.T ? k : q;
        const uint8_t *s1 = b1 + (int64_t)s * G.T, *s2 = b2 + (int64_t)s * G.T;
        const int p1 = item_pos(x1, G.T), p2 = item_pos(x2, G.T);
        const int lim = min(p1, p2) + 1;
        int m = lcp[gi];
        for (;;) {
            const int i0 = m + 4 * lane;   // this lane compares symbols i0 .. i0+3 back from the ends
            int off = 4;                   // first differing symbol within the four (4: none)
            uint32_t v1, v2;
            if (i0 + 3 < lim && load4_back(s1 + p1 - i0, b1, b1 + total, v1) &&
                load4_back(s2 + p2 - i0, b2, b2 + total, v2)) {
                const uint32_t x = v1 ^ v2;
                if (x) off = __clz(x) >> 3;
            } else {
                for (int j = 0; j < 4; ++j) {
                    const int i = i0 + j;
                    if (i >= lim || s1[p1 - i] != s2[p2 - i]) { off = j; break; }
                }
            }
            const unsigned dm = __ballot_sync(ROSA_FULL_MASK, off < 4);
            if (dm) {
                const int f = __ffs(dm) - 1;
                m += 4 * f + __shfl_sync(ROSA_FULL_MASK, off, f);
                break;
            }
            m += 128;
        }
        if (lane == 0) lcp[gi] = m;
    }
}

// ---------------------------------------------------------------------------
// 3a. Block summaries: smallest key position and smallest inner LCP (edges
//     strictly inside the block) per 32 and per 1024 ranks, and the LCP edge
//     entering each 32-block from below.
// ---------------------------------------------------------------------------
// Keys are the items below T (with q == k they are the queries as well).
__device__ __forceinline__ int key_pos_or_inf(uint32_t x, int T) { return (int)x < T ? (int)x : INT_MAX; }

// One CTA of 256 threads per 1024 ranks; thread t loads ranks t + 256u
// (u < 4) up front, so that each warp's u-th group is one 32-rank block.
__global__ void __launch_bounds__(256)
summary_kernel(Geometry G, const uint32_t *__restrict__ sa, const int32_t *__restrict__ lcp,
               int32_t *__restrict__ minpos1, int32_t *__restrict__ emin1, int32_t *__restrict__ ein1,
               int32_t *__restrict__ minpos2, int32_t *__restrict__ emin2, int32_t *__restrict__ ein2) {
    constexpr int kPer = kL2 / 256;
    __shared__ int wpos[kL2 / kL1], wemin[kL2 / kL1], wfirst[kL2 / kL1];
    __shared__ int edge_in;   // LCP edge entering the 1024 ranks
    const int s = blockIdx.x / G.nb2, B2 = blockIdx.x - s * G.nb2;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int64_t seg = (int64_t)s * G.n;
    int pos[kPer], l[kPer];
#pragma unroll
    for (int u = 0; u < kPer; ++u) {
        const int j = B2 * kL2 + u * 256 + threadIdx.x;
        pos[u] = INT_MAX;
        l[u] = INT_MAX;
        if (j < G.n) {
            pos[u] = key_pos_or_inf(sa[seg + j], G.T);
            l[u] = lcp[seg + j];
        }
    }
#pragma unroll
    for (int u = 0; u < kPer; ++u) {
        const int first = __shfl_sync(ROSA_FULL_MASK, l[u], 0);
        const int mp = __reduce_min_sync(ROSA_FULL_MASK, pos[u]);
        const int me = __reduce_min_sync(ROSA_FULL_MASK, lane == 0 ? INT_MAX : l[u]);
        const int blk = u * 8 + warp;   // 32-rank block within the 1024
        const int b1 = B2 * (kL2 / kL1) + blk;
        if (lane == 0) {
            if (b1 < G.nb1) {
                minpos1[(int64_t)s * G.nb1 + b1] = mp;
                emin1[(int64_t)s * G.nb1 + b1] = me;
                ein1[(int64_t)s * G.nb1 + b1] = first;
            }
            wpos[blk] = mp;
            wemin[blk] = me;
            wfirst[blk] = blk == 0 ? INT_MAX : first;
        }
    }
    if (threadIdx.x == 0) edge_in = l[0];
    __syncthreads();
    if (warp == 0) {
        const int p2 = __reduce_min_sync(ROSA_FULL_MASK, wpos[lane]);
        const int e2 = __reduce_min_sync(ROSA_FULL_MASK, min(wemin[lane], wfirst[lane]));
        if (lane == 0) {
            minpos2[(int64_t)s * G.nb2 + B2] = p2;
            emin2[(int64_t)s * G.nb2 + B2] = e2;
            ein2[(int64_t)s * G.nb2 + B2] = edge_in;
        }
    }
}

// ---------------------------------------------------------------------------
// 3b. Wavelet matrix over the key positions in rank order, for the query
//     "largest key position <= X among ranks [lo, hi]" in O(log T).  One
//     stable partition by bit per level, most significant bit first; each
//     level stores its bits with the count of ones before every 64-bit word.
// ---------------------------------------------------------------------------
constexpr int kWTile = 2048;

struct __align__(16) WWord {
    uint32_t cum;
    uint32_t pad;
    unsigned long long bits;
};

// Keys per 2048-rank tile of the sorted order (q != k only).
__global__ void __launch_bounds__(256)
key_tile_count_kernel(Geometry G, const uint32_t *__restrict__ sa, int *__restrict__ ktile) {
    __shared__ int red[8];
    const int s = blockIdx.x / G.ntps, tt = blockIdx.x - s * G.ntps;
    const int64_t base = (int64_t)s * G.n + (int64_t)tt * kRadixTile;
    const int lim = min(kRadixTile, G.n - tt * kRadixTile);
    int c = 0;
    for (int i = threadIdx.x; i < lim; i += 256) c += (int)sa[base + i] < G.T ? 1 : 0;
    c = __reduce_add_sync(ROSA_FULL_MASK, c);
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = c;
    __syncthreads();
    if (threadIdx.x == 0) {
        int t = 0;
        for (int w = 0; w < 8; ++w) t += red[w];
        ktile[(int64_t)s * G.ntps + tt] = t;
    }
}

// Level-0 sequence (key positions in rank order), the exclusive key count
// before every rank (q != k), and the level-0 ones per wavelet tile.  The
// tile's sa loads and the key count of the tiles before it are in flight
// together (a warp sums the per-tile counts), and one scan over the 8 x 8
// (round, warp) key counts gives every thread its offsets.
__global__ void __launch_bounds__(256)
wavelet_compact_kernel(Geometry G, int nbits, const uint32_t *__restrict__ sa, const int *__restrict__ ktile,
                       int32_t *__restrict__ kcount, uint32_t *__restrict__ a0, int *__restrict__ wcnt0) {
    __shared__ int wk[kRadixIPT * 8];     // keys per (round, warp), then exclusive offsets
    __shared__ int pre_s;
    __shared__ int ones[2];
    const int s = blockIdx.x / G.ntps, tt = blockIdx.x - s * G.ntps;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int64_t base = (int64_t)s * G.n + (int64_t)tt * kRadixTile;
    const int lim = min(kRadixTile, G.n - tt * kRadixTile);
    const int ntw = ceil_div(G.T, kWTile);
    uint32_t xs[kRadixIPT];
#pragma unroll
    for (int u = 0; u < kRadixIPT; ++u) {
        const int i = u * 256 + threadIdx.x;
        xs[u] = i < lim ? sa[base + i] : 0u;
    }
    if (warp == 0) {
        int p = 0;
        if (G.allkeys) {
            p = tt * kRadixTile;
        } else {
            for (int i = lane; i < tt; i += 32) p += ktile[(int64_t)s * G.ntps + i];
            p = __reduce_add_sync(ROSA_FULL_MASK, p);
        }
        if (lane == 0) pre_s = p;
    }
    if (threadIdx.x < 2) ones[threadIdx.x] = 0;
    unsigned bal[kRadixIPT];
#pragma unroll
    for (int u = 0; u < kRadixIPT; ++u) {
        const int i = u * 256 + threadIdx.x;
        bal[u] = __ballot_sync(ROSA_FULL_MASK, i < lim && (int)xs[u] < G.T);
        if (lane == 0) wk[u * 8 + warp] = __popc(bal[u]);
    }
    __syncthreads();
    if (warp == 0) {   // exclusive scan of the 64 counts, round-major
        const int c0v = wk[lane], c1v = wk[32 + lane];
        int i0 = c0v, i1 = c1v;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y0 = __shfl_up_sync(ROSA_FULL_MASK, i0, o), y1 = __shfl_up_sync(ROSA_FULL_MASK, i1, o);
            if (lane >= o) { i0 += y0; i1 += y1; }
        }
        const int first = __shfl_sync(ROSA_FULL_MASK, i0, 31);
        wk[lane] = pre_s + i0 - c0v;
        wk[32 + lane] = pre_s + first + i1 - c1v;
    }
    __syncthreads();
    const int t0 = pre_s / kWTile;
    int c0 = 0, c1 = 0;   // level-0 ones landing in wavelet tiles t0 and t0 + 1
#pragma unroll
    for (int u = 0; u < kRadixIPT; ++u) {
        const int i = u * 256 + threadIdx.x;
        const uint32_t x = xs[u];
        const bool key = (bal[u] >> lane) & 1u;
        const int kidx = wk[u * 8 + warp] + __popc(bal[u] & lanemask_lt());
        if (i < lim && !G.allkeys) kcount[base + i] = kidx;
        if (key) {
            a0[(int64_t)s * G.T + kidx] = x;
            if ((x >> (nbits - 1)) & 1u) {
                if (kidx / kWTile == t0) ++c0;
                else ++c1;
            }
        }
    }
    c0 = __reduce_add_sync(ROSA_FULL_MASK, c0);
    c1 = __reduce_add_sync(ROSA_FULL_MASK, c1);
    if (lane == 0) {
        if (c0) atomicAdd(&ones[0], c0);
        if (c1) atomicAdd(&ones[1], c1);
    }
    __syncthreads();
    if (threadIdx.x < 2 && ones[threadIdx.x]) atomicAdd(&wcnt0[(int64_t)s * ntw + t0 + threadIdx.x], ones[threadIdx.x]);
}

__global__ void __launch_bounds__(256)
wavelet_level_kernel(Geometry G, int nbits, int lv, const uint32_t *__restrict__ in, uint32_t *__restrict__ out,
                     int *__restrict__ wcnt, WWord *__restrict__ words, int *__restrict__ wz) {
    // warp w owns elements [256w, 256w + 256) of the tile: its ones count
    // gives the warp's offsets, so the tile needs only two block barriers
    __shared__ uint32_t ballots[kWTile / 32];
    __shared__ int wones[8];
    __shared__ int red_a[8], red_t[8];
    __shared__ int nxt[4];
    const int ntw = ceil_div(G.T, kWTile), nw = (G.T >> 6) + 1;
    const int s = blockIdx.x / ntw, tt = blockIdx.x - s * ntw;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int b = nbits - 1 - lv;
    const int *cnt = wcnt + ((int64_t)lv * G.S + s) * ntw;
    const int lim = min(kWTile, G.T - tt * kWTile);
    const uint32_t *src = in + (int64_t)s * G.T + (int64_t)tt * kWTile;
    uint32_t v[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {   // the tile's values and the tile counts are loaded together
        const int i = warp * 256 + u * 32 + lane;
        v[u] = i < lim ? src[i] : 0u;
    }
    int a = 0, tot = 0;
    for (int i = threadIdx.x; i < ntw; i += 256) {
        const int c = cnt[i];
        tot += c;
        if (i < tt) a += c;
    }
    a = __reduce_add_sync(ROSA_FULL_MASK, a);
    tot = __reduce_add_sync(ROSA_FULL_MASK, tot);
    unsigned bal[8];
    int mine = 0;
#pragma unroll
    for (int u = 0; u < 8; ++u) {
        const int i = warp * 256 + u * 32 + lane;
        bal[u] = __ballot_sync(ROSA_FULL_MASK, i < lim && ((v[u] >> b) & 1u));
        mine += __popc(bal[u]);
    }
    if (lane == 0) {
        red_a[warp] = a;
        red_t[warp] = tot;
        wones[warp] = mine;
#pragma unroll
        for (int u = 0; u < 8; ++u) ballots[warp * 8 + u] = bal[u];
    }
    if (threadIdx.x < 4) nxt[threadIdx.x] = 0;
    __syncthreads();
    int ones_before = 0, total_ones = 0, wpre = 0;
#pragma unroll
    for (int w2 = 0; w2 < 8; ++w2) {
        ones_before += red_a[w2];
        total_ones += red_t[w2];
        if (w2 < warp) wpre += wones[w2];
    }
    const int Z = G.T - total_ones;
    const int zeros_before = tt * kWTile - ones_before;
    // zeros of this tile land in one contiguous range and ones in another, so
    // the next level's per-tile counts touch at most four tiles
    const int zr0 = zeros_before / kWTile, or0 = (Z + ones_before) / kWTile;
    uint32_t *dst = out + (int64_t)s * G.T;
    int run = wpre;
#pragma unroll
    for (int u = 0; u < 8; ++u) {
        const int i = warp * 256 + u * 32 + lane;
        const int bit = (bal[u] >> lane) & 1;
        const int lo1 = run + __popc(bal[u] & lanemask_lt());
        if (i < lim) {
            const int d = bit ? Z + ones_before + lo1 : zeros_before + (i - lo1);
            dst[d] = v[u];
            if (lv + 1 < G.wlev && ((v[u] >> (b - 1)) & 1u)) {
                const int dt = d / kWTile;
                atomicAdd(&nxt[bit ? 2 + (dt - or0) : (dt - zr0)], 1);
            }
        }
        run += __popc(bal[u]);
    }
    if (threadIdx.x < 32) {
        const int k = threadIdx.x;
        const unsigned long long bits =
            (unsigned long long)ballots[2 * k] | ((unsigned long long)ballots[2 * k + 1] << 32);
        const int pc = __popcll(bits);
        int incl = pc;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(ROSA_FULL_MASK, incl, o);
            if (lane >= o) incl += y;
        }
        if (k * 64 < lim) {
            WWord wd;
            wd.cum = (uint32_t)(ones_before + incl - pc);
            wd.pad = 0;
            wd.bits = bits;
            words[((int64_t)s * nbits + lv) * nw + tt * 32 + k] = wd;
        }
    }
    __syncthreads();
    if (lv + 1 < G.wlev && threadIdx.x < 4) {
        const int c = nxt[threadIdx.x];
        const int dt = threadIdx.x < 2 ? zr0 + threadIdx.x : or0 + threadIdx.x - 2;
        if (c) atomicAdd(&wcnt[((int64_t)(lv + 1) * G.S + s) * ntw + dt], c);
    }
    if (threadIdx.x == 0) {
        if (tt == ntw - 1 && (G.T & 63) == 0) {
            WWord wd;
            wd.cum = (uint32_t)total_ones;
            wd.pad = 0;
            wd.bits = 0ull;
            words[((int64_t)s * nbits + lv) * nw + (G.T >> 6)] = wd;
        }
        if (tt == 0) wz[(int64_t)s * nbits + lv] = Z;
    }
}

__device__ __forceinline__ int wrank1(const WWord *W, int i) {
    const uint4 raw = __ldg(reinterpret_cast<const uint4 *>(W + (i >> 6)));
    const unsigned long long bits = ((unsigned long long)raw.w << 32) | raw.z;
    const unsigned long long mask = (i & 63) ? ((1ull << (i & 63)) - 1ull) : 0ull;
    return (int)raw.x + __popcll(bits & mask);
}

// Largest value <= X in positions [l, r) of the level-0 sequence, or -1.
// Only the top nlev bits have levels: a range that shares them holds at most
// 2^(nbits - nlev) values (key positions are distinct), which are read from
// the level-nlev sequence `leaf`.
__device__ int wavelet_max_le(const WWord *W, const int *Z, const uint32_t *leaf, int nbits, int nlev, int nw, int l,
                              int r, int X) {
    if (l >= r || X < 0) return -1;
    const int top = (1 << nbits) - 1;
    if (X > top) X = top;
    int alt_lv = -1, alt_l = 0, alt_r = 0;
    bool alive = true;
    for (int lv = 0; lv < nlev; ++lv) {
        const int b = nbits - 1 - lv;
        const WWord *Wl = W + (int64_t)lv * nw;
        const int ol = wrank1(Wl, l), orr = wrank1(Wl, r);
        const int zl = l - ol, zr = r - orr;
        if ((X >> b) & 1) {
            if (zr > zl) { alt_lv = lv; alt_l = zl; alt_r = zr; }
            l = Z[lv] + ol;
            r = Z[lv] + orr;
        } else {
            l = zl;
            r = zr;
        }
        if (l >= r) { alive = false; break; }
    }
    if (alive) {   // values with X's top nlev bits, eight independent loads at a time
        int best = -1;
        for (int i0 = l; i0 < r; i0 += 8) {
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int v = i0 + u < r ? (int)__ldg(leaf + i0 + u) : -1;
                if (v <= X && v > best) best = v;
            }
        }
        if (best >= 0) return best;
    }
    if (alt_lv < 0) return -1;
    // deepest level where X has a one and the zero side is not empty: every
    // value there is below X; follow ones where possible, then take the leaf's max
    l = alt_l;
    r = alt_r;
    for (int lv = alt_lv + 1; lv < nlev; ++lv) {
        const WWord *Wl = W + (int64_t)lv * nw;
        const int ol = wrank1(Wl, l), orr = wrank1(Wl, r);
        if (orr > ol) {
            l = Z[lv] + ol;
            r = Z[lv] + orr;
        } else {
            l -= ol;
            r -= orr;
        }
    }
    int best = -1;
    for (int i0 = l; i0 < r; i0 += 8) {
#pragma unroll
        for (int u = 0; u < 8; ++u) best = max(best, i0 + u < r ? (int)__ldg(leaf + i0 + u) : -1);
    }
    return best;
}

// ---------------------------------------------------------------------------
// 3c. Per-query resolution.
//     resolve_tile_kernel: a CTA stages 1024 ranks plus 512 on each side (key
//     position, LCP edge) in shared memory and resolves the tile's queries
//     there: the nearest admissible key on each side gives L, binary lifting
//     on a sparse table gives the interval of ranks sharing L symbols, and a
//     scan of that interval gives i* when it spans at most 128 ranks.
//     Wider intervals are parked for wavelet_query_kernel.  Queries whose
//     nearest key lies outside the window go to resolve_hard_kernel (one warp
//     per query over global memory, 32 ranks or 32 blocks per step); interval
//     ends outside the window are found by resolve_bounds_kernel, or once per
//     (tile, side, L) for short L by bound_task/bound_finish_kernel.
// ---------------------------------------------------------------------------
constexpr int kRTile = 1024;
constexpr int kRHalo = 512;
constexpr int kRWin = kRTile + 2 * kRHalo;
constexpr int kRThreads = 512;

struct StreamView {
    const uint32_t *sa;
    const int32_t *lcp;
    const int32_t *mp1, *em1, *ein1, *mp2, *em2, *ein2;
    const int32_t *kcount;
    const WWord *W;
    const int *Z;
    int n, T, nb1, nb2, nbits, nw;
    bool same;
};

__device__ __forceinline__ int kpos(const StreamView &v, int r) { return key_pos_or_inf(v.sa[r], v.T); }

// number of keys at ranks below r (r in [0, n])
__device__ __forceinline__ int kc(const StreamView &v, int r) {
    if (v.same) return r;
    return r < v.n ? v.kcount[r] : v.T;
}

struct ResolveArgs {
    const uint32_t *sa;
    const int32_t *lcp, *mp1, *em1, *ein1, *mp2, *em2, *ein2, *kcount;
    const WWord *words;
    const int *wz;
    const uint32_t *leaf;    // wavelet level-nlev sequence
    int nbits, nlev;
};

__device__ __forceinline__ StreamView make_view(const Geometry &G, int s, const ResolveArgs &A) {
    const int64_t seg = (int64_t)s * G.n;
    const int nw = (G.T >> 6) + 1;
    return StreamView{A.sa + seg, A.lcp + seg, A.mp1 + (int64_t)s * G.nb1, A.em1 + (int64_t)s * G.nb1,
                      A.ein1 + (int64_t)s * G.nb1, A.mp2 + (int64_t)s * G.nb2, A.em2 + (int64_t)s * G.nb2,
                      A.ein2 + (int64_t)s * G.nb2, A.kcount ? A.kcount + seg : nullptr,
                      A.words + (int64_t)s * A.nbits * nw, A.wz + (int64_t)s * A.nbits, G.n, G.T, G.nb1, G.nb2,
                      A.nbits, nw, G.allkeys};
}

// Output slots.  The query at (s, t) writes slot s*T + t of the caller's
// arrays; branch j of (s, t) (query bit j flipped) writes slot
// S*T + (s*T + t)*mcf + j, i.e. entry (s*T + t)*mcf + j of the branch arrays.
// Deferred lookups park their key range in the same slots.
struct Outs {
    int32_t *e0, *l0, *y0;   // [S, T]
    int32_t *e1, *l1, *y1;   // [S, T, mcf]
    int64_t n0;              // S * T
    __device__ __forceinline__ int32_t &E(int64_t o) const { return o < n0 ? e0[o] : e1[o - n0]; }
    __device__ __forceinline__ int32_t &L(int64_t o) const { return o < n0 ? l0[o] : l1[o - n0]; }
    __device__ __forceinline__ int32_t &Y(int64_t o) const { return o < n0 ? y0[o] : y1[o - n0]; }
};

// Slot of query item x (a query or a branch) of stream s.
__device__ __forceinline__ int64_t out_slot(const Geometry &G, int s, uint32_t x) {
    const int t = item_pos(x, G.T);
    if ((int)x < G.br0) return (int64_t)s * G.T + t;
    const int j = ((int)x - G.br0) / G.T;
    return (int64_t)G.S * G.T + ((int64_t)s * G.T + t) * G.mcf + j;
}

// Stream and time of an output slot.
__device__ __forceinline__ void slot_stream_time(const Geometry &G, int64_t o, int &s, int &t) {
    const int64_t n0 = (int64_t)G.S * G.T;
    const int64_t st = o < n0 ? o : (o - n0) / G.mcf;
    s = (int)(st / G.T);
    t = (int)(st - (int64_t)s * G.T);
}

__device__ __forceinline__ void write_result(const uint8_t *vsym, const Outs &O, int64_t o, int64_t srow, int L,
                                             int ib) {
    if (L > 0 && ib >= 0) {
        O.E(o) = ib;
        O.L(o) = L;
        O.Y(o) = (int32_t)vsym[srow + ib + 1];
    } else {
        O.E(o) = -1;
        O.L(o) = 0;
        O.Y(o) = -1;
    }
}

// Staged window of one resolve tile (local ranks 0..kRWin-1):
//   kp[i]  key position of local rank i, INT_MAX for query items and ranks
//          outside the stream;
//   lc[i]  LCP edge between local ranks i-1 and i (0 at the stream start,
//          -1 past the stream end); lc[kRWin] is the edge just past the window;
//   sp[k][i] min(lc[i .. i+2^k-1]) capped to 255 (u8);
//   per query of the tile: local rank qj, item id qt, match length qL.
// Queries are resolved in three uniform phases (see resolve_tile_kernel).
constexpr int kSpLevels = 11;          // lifting reaches 2^11 - 1 ranks: a whole side of the window
constexpr int kProbe = 16;             // ranks a lane probes on each side before its warp helps
constexpr int kNeedWarp = -1;          // qL codes
constexpr int kNeedHard = -2;

constexpr int kWarpScanMax = 128;      // widest interval a warp scans in shared memory
constexpr int kBoundShared = 64;       // match lengths whose out-of-window bounds are shared per tile

struct WinSmem {
    int kp[kRWin];
    int lc[kRWin + 1];
    int qt[kRTile];
    int qL[kRTile];
    int16_t qj[kRTile];
    int16_t bq[kRTile];
    int16_t dlo[kRTile];     // phase D: interval bounds of queries a warp finishes
    int16_t dhi[kRTile];     // (their query indices reuse bq)
    unsigned long long need[2];   // lengths L < 64 whose interval leaves the window below / above
    int nq, nb, nd;
    int bkp[kRWin / 32];     // per 32-rank block: smallest key position,
    int beL[kRWin / 32];     //   LCP minimum crossed walking down through it (lc[32B+1 .. 32B+32]),
    int beR[kRWin / 32];     //   and walking up through it (lc[32B .. 32B+31])
    uint8_t sp[kSpLevels][kRWin];
};

// Parks a query whose interval is too wide to scan: its key range goes into
// the output slots until wavelet_query_kernel replaces it with the answer.
__device__ __forceinline__ void defer_wavelet(const Outs &O, int64_t o, int L, int klo, int khi, int32_t *wq,
                                              int *wq_count) {
    O.L(o) = L;
    O.E(o) = klo;
    O.Y(o) = khi;
    wq[atomicAdd(wq_count, 1)] = (int32_t)o;
}

// Warp-cooperative nearest admissible key in direction dir: the LCP with it
// when that exceeds lim, 0 when the running LCP falls to lim first,
// kNeedHard when the answer lies beyond the window.  The ranks up to the end
// of jl's 32-rank block are scanned directly; beyond it the warp takes 32
// whole blocks per step from their summaries (smallest key position, LCP
// minimum) and scans only the first block that holds an admissible key.
__device__ int warp_nearest_smem(const WinSmem &w, int jl, int X, int dir, int lim, int lane) {
    // The running LCP first drops to <= lim at the first lane whose own edge
    // is <= lim (the carry from earlier steps is > lim, or the scan would have
    // ended), so a ballot finds the stop and one warp min-reduction over the
    // lanes before a hit gives the running LCP there.
    constexpr int kNB = kRWin / 32;
    const unsigned lt = lanemask_lt();
    int blk, cnt0, r;
    if (dir < 0) {
        const int rtop = jl - 1;
        blk = rtop >> 5;
        cnt0 = (rtop & 31) + 1;
        r = rtop - lane;
    } else {
        const int rbot = jl + 1;
        blk = rbot >> 5;
        cnt0 = 32 - (rbot & 31);
        r = rbot + lane;
    }
    int e = lane < cnt0 ? (dir < 0 ? w.lc[r + 1] : w.lc[r]) : INT_MAX;
    const bool valid = lane < cnt0 && w.kp[r] <= X;
    unsigned sm = __ballot_sync(ROSA_FULL_MASK, e <= lim);
    int fs = sm ? __ffs(sm) - 1 : 32;
    const unsigned before_fs = fs < 32 ? ((1u << fs) - 1u) : ROSA_FULL_MASK;
    const unsigned vm = __ballot_sync(ROSA_FULL_MASK, valid) & before_fs;
    if (vm) {
        const int fv = __ffs(vm) - 1;
        return __reduce_min_sync(ROSA_FULL_MASK, lane <= fv ? e : INT_MAX);
    }
    if (fs < 32) return __shfl_sync(ROSA_FULL_MASK, e, fs) == kNeedHard ? kNeedHard : 0;
    int carry = __reduce_min_sync(ROSA_FULL_MASK, e);
    for (int B0 = blk + dir;; B0 += 32 * dir) {   // ends at the window edge at the latest
        const int B = B0 + dir * lane;
        bool has = false;
        if (B >= 0 && B < kNB) {
            e = dir < 0 ? w.beL[B] : w.beR[B];
            has = w.bkp[B] <= X;
        } else if (B == -1 || B == kNB) {   // the edge out of the window, then unknown ranks
            const int edge = B < 0 ? w.lc[0] : w.lc[kRWin];
            e = edge <= lim ? edge : kNeedHard;
        } else {
            e = kNeedHard;
        }
        sm = __ballot_sync(ROSA_FULL_MASK, e <= lim);
        const unsigned hm = __ballot_sync(ROSA_FULL_MASK, has);
        fs = sm ? __ffs(sm) - 1 : 32;
        const int fh = hm ? __ffs(hm) - 1 : 32;
        if (fh < 32 && fh <= fs) {   // the first block with an admissible key, entered above lim
            const int cin = min(carry, __reduce_min_sync(ROSA_FULL_MASK, lane < fh ? e : INT_MAX));
            const int Bh = B0 + dir * fh;
            const int rr = dir < 0 ? 32 * Bh + 31 - lane : 32 * Bh + lane;
            const int e2 = dir < 0 ? w.lc[rr + 1] : w.lc[rr];
            const unsigned sm2 = __ballot_sync(ROSA_FULL_MASK, e2 <= lim);
            const int fs2 = sm2 ? __ffs(sm2) - 1 : 32;
            const unsigned vm2 = __ballot_sync(ROSA_FULL_MASK, w.kp[rr] <= X) &
                                 (fs2 < 32 ? ((1u << fs2) - 1u) : ROSA_FULL_MASK);
            if (!vm2) return 0;
            const int fv2 = __ffs(vm2) - 1;
            return min(cin, __reduce_min_sync(ROSA_FULL_MASK, lane <= fv2 ? e2 : INT_MAX));
        }
        if (fs < 32) return __shfl_sync(ROSA_FULL_MASK, e, fs) == kNeedHard ? kNeedHard : 0;
        carry = min(carry, __reduce_min_sync(ROSA_FULL_MASK, e));
    }
}

// Interval of local ranks around jl whose LCP with jl is >= L.  A side that
// may extend beyond the window is returned as -1.
__device__ void window_bounds(const WinSmem &w, bool at_start, int jl, int L, int &lo, int &hi) {
    if (L < 255) {
        int cur = jl;
#pragma unroll
        for (int k = kSpLevels - 1; k >= 0; --k) {
            const int c = cur - (1 << k);
            if (c >= 0 && w.sp[k][c + 1] >= L) cur = c;
        }
        lo = (cur == 0 && !at_start && w.lc[0] >= L) ? -1 : cur;
        cur = jl;
#pragma unroll
        for (int k = kSpLevels - 1; k >= 0; --k) {
            const int c = cur + (1 << k);
            if (c < kRWin && w.sp[k][cur + 1] >= L) cur = c;
        }
        hi = (cur == kRWin - 1 && w.lc[kRWin] >= L) ? -1 : cur;
    } else {   // long matches: exact edges (such intervals are short)
        int r = jl;
        while (r > 0 && w.lc[r] >= L) --r;
        lo = (r == 0 && !at_start && w.lc[0] >= L) ? -1 : r;
        r = jl;
        while (r + 1 < kRWin && w.lc[r + 1] >= L) ++r;
        hi = (r == kRWin - 1 && w.lc[kRWin] >= L) ? -1 : r;
    }
}

// One CTA per 1024 ranks of a stream, with 512 ranks of context on each side.
//   Phase A: each lane probes 16 ranks on each side of its query for the
//            nearest admissible key (fixed trip count, no divergence).
//   Phase B: queries the probes could not settle get a warp each, scanning
//            32 ranks per step in shared memory.
//   Phase C: each lane finds its interval bounds by binary lifting on the
//            sparse table, then i* by a 16-rank probe; intervals of up to
//            kWarpScanMax ranks go to phase D, wider ones to the wavelet.
//   Phase D: one warp per listed interval, 32 ranks per step.
// Queries whose answer needs ranks outside the window go to the hard lists.
__global__ void __launch_bounds__(kRThreads, 4)
resolve_tile_kernel(Geometry G, ResolveArgs A, const uint8_t *__restrict__ vsym, Outs O, int32_t *__restrict__ hard,
                    int *hard_count, int32_t *__restrict__ hardb, int *hardb_count, int32_t *__restrict__ hardw,
                    int *hardw_count, int32_t *__restrict__ btask, int *btask_count, int32_t *__restrict__ wq,
                    int *wq_count) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    WinSmem &w = *reinterpret_cast<WinSmem *>(smem_raw);
    const int ntr = ceil_div(G.n, kRTile);
    const int s = blockIdx.x / ntr, tt = blockIdx.x - s * ntr;
    const int64_t seg = (int64_t)s * G.n;
    const int w0 = tt * kRTile - kRHalo;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    if (threadIdx.x == 0) { w.nq = 0; w.nb = 0; w.nd = 0; w.need[0] = 0; w.need[1] = 0; }
    {
        // loads first: the window's ranks and edges, five of each per thread
        constexpr int kStage = (kRWin + 1 + kRThreads - 1) / kRThreads;
        uint32_t xs[kStage];
        int ls[kStage];
#pragma unroll
        for (int u = 0; u < kStage; ++u) {
            const int i = u * kRThreads + threadIdx.x;
            const int r = w0 + i;
            const bool in = i <= kRWin && r >= 0 && r < G.n;
            xs[u] = (in && i < kRWin) ? A.sa[seg + r] : 0u;
            ls[u] = in ? A.lcp[seg + r] : -1;
        }
#pragma unroll
        for (int u = 0; u < kStage; ++u) {
            const int i = u * kRThreads + threadIdx.x;
            if (i > kRWin) break;
            const int r = w0 + i;
            const int l = ls[u];
            if (i < kRWin) {
                w.kp[i] = (r >= 0 && r < G.n) ? key_pos_or_inf(xs[u], G.T) : INT_MAX;
                w.sp[0][i] = (uint8_t)(l < 0 ? 0 : (l > 255 ? 255 : l));
            }
            w.lc[i] = l;
        }
    }
    __syncthreads();
    for (int B = warp; B < kRWin / 32; B += kRThreads / 32) {
        const int r = 32 * B + lane;
        const int kmin = __reduce_min_sync(ROSA_FULL_MASK, w.kp[r]);
        const int el = __reduce_min_sync(ROSA_FULL_MASK, w.lc[r + 1]);
        const int er = __reduce_min_sync(ROSA_FULL_MASK, w.lc[r]);
        if (lane == 0) { w.bkp[B] = kmin; w.beL[B] = el; w.beR[B] = er; }
    }
    // sparse table levels, four byte entries per step with byte-wise SIMD minima
    for (int k = 1; k < kSpLevels; ++k) {
        const int h = 1 << (k - 1);
        const uint32_t *prev = reinterpret_cast<const uint32_t *>(w.sp[k - 1]);
        uint32_t *cur = reinterpret_cast<uint32_t *>(w.sp[k]);
        for (int q4 = threadIdx.x; q4 < kRWin / 4; q4 += kRThreads) {
            const int i = q4 * 4;
            const uint32_t a = prev[q4];
            uint32_t b;
            if ((h & 3) == 0) {
                b = (i + h < kRWin) ? prev[q4 + (h >> 2)] : 0u;
            } else {   // h = 1 or 2: bytes i+h .. i+h+3 straddle two words
                const uint32_t lo = prev[q4];
                const uint32_t hi = (q4 + 1 < kRWin / 4) ? prev[q4 + 1] : 0u;
                b = __byte_perm(lo, hi, h == 1 ? 0x4321 : 0x5432);
            }
            uint32_t m = __vminu4(a, b);
            // entries whose range runs past the window stay 0 (never read)
            const int valid = kRWin - (2 * h - 1) - i;   // entries i .. i+valid-1 are in range
            if (valid < 4) m = valid <= 0 ? 0u : (m & (0xffffffffu >> (8 * (4 - valid))));
            cur[q4] = m;
        }
        __syncthreads();
    }
    // compact the tile's query items so that every lane has one to answer
    for (int i0 = 0; i0 < kRTile; i0 += kRThreads) {
        const int i = i0 + threadIdx.x;
        const int j = tt * kRTile + i;
        uint32_t x = 0;
        bool isq = false;
        if (j < G.n) {
            x = A.sa[seg + j];
            isq = G.same || (int)x >= G.T;
        }
        const unsigned bal = __ballot_sync(ROSA_FULL_MASK, isq);
        int base = 0;
        if (lane == 0 && bal) base = atomicAdd(&w.nq, __popc(bal));
        base = __shfl_sync(ROSA_FULL_MASK, base, 0);
        if (isq) {
            const int slot = base + __popc(bal & lanemask_lt());
            w.qj[slot] = (int16_t)(i + kRHalo);
            w.qt[slot] = (int)x;
        }
    }
    __syncthreads();
    const int nq = w.nq;
    // Phase A
    for (int qi = threadIdx.x; qi < nq; qi += kRThreads) {
        const int jl = w.qj[qi];
        const int X = query_bound(G, s, item_pos(w.qt[qi], G.T));
        int L = 0;
        if (X >= 0) {
            int m = INT_MAX, Ll = -1;
#pragma unroll
            for (int k = 1; k <= kProbe; ++k) {
                const int r = jl - k;                  // jl >= kRHalo, so r >= 0
                m = min(m, w.lc[r + 1]);
                const int c = w.kp[r];
                if (Ll < 0) Ll = (m <= 0) ? 0 : (c <= X ? m : -1);
            }
            int Lr = -1;
            if (Ll >= 0) {
                m = INT_MAX;
#pragma unroll
                for (int k = 1; k <= kProbe; ++k) {
                    const int r = jl + k;              // jl + kProbe < kRWin
                    m = min(m, w.lc[r]);
                    const int c = w.kp[r];
                    if (Lr < 0) Lr = (m <= Ll) ? 0 : (c <= X ? m : -1);
                }
            }
            if (Ll < 0 || Lr < 0) {
                L = kNeedWarp;
                w.bq[atomicAdd(&w.nb, 1)] = (int16_t)qi;
            } else {
                L = max(Ll, Lr);
            }
        }
        w.qL[qi] = L;
    }
    __syncthreads();
    // Phase B
    const int nb = w.nb;
    for (int bi = warp; bi < nb; bi += kRThreads / 32) {
        const int qi = w.bq[bi];
        const int jl = w.qj[qi];
        const int X = query_bound(G, s, item_pos(w.qt[qi], G.T));
        const int Ll = warp_nearest_smem(w, jl, X, -1, 0, lane);
        int L = Ll;
        if (Ll != kNeedHard) {
            const int Lr = warp_nearest_smem(w, jl, X, +1, Ll, lane);
            L = Lr == kNeedHard ? kNeedHard : max(Ll, Lr);
        }
        if (lane == 0) w.qL[qi] = L;
    }
    __syncthreads();
    // Phase C
    const bool at_start = w0 <= 0;
    const StreamView v = make_view(G, s, A);
    for (int qi = threadIdx.x; qi < nq; qi += kRThreads) {
        const int jl = w.qj[qi];
        const uint32_t qx = (uint32_t)w.qt[qi];
        const int X = query_bound(G, s, item_pos(qx, G.T));
        const int64_t o = out_slot(G, s, qx);
        const int L = w.qL[qi];
        int lo = 0, hi = -1;
        if (L == kNeedHard) {
            hard[atomicAdd(hard_count, 1)] = (int32_t)(seg + w0 + jl);
            continue;
        }
        if (L > 0) {
            window_bounds(w, at_start, jl, L, lo, hi);
            if (lo < 0 || hi < 0) {
                // L is known; only the interval's far end lies outside the window.  That
                // end depends on (tile, side, L) alone, so short L share one scan.
                O.L(o) = L;
                O.E(o) = lo < 0 ? -1 : w0 + lo;
                O.Y(o) = hi < 0 ? -1 : w0 + hi;
                if (L < kBoundShared) {
                    if (lo < 0) atomicOr(&w.need[0], 1ull << L);
                    if (hi < 0) atomicOr(&w.need[1], 1ull << L);
                    hardw[atomicAdd(hardw_count, 1)] = (int32_t)(seg + w0 + jl);
                } else {
                    hardb[atomicAdd(hardb_count, 1)] = (int32_t)(seg + w0 + jl);
                }
                continue;
            }
        }
        int ib = -1;
        if (L > 0) {
            if (hi - lo < kProbe) {
#pragma unroll
                for (int k = 0; k < kProbe; ++k) {
                    const int r = lo + k;              // lo <= jl < kRWin - kProbe
                    const int c = r <= hi ? w.kp[r] : INT_MAX;
                    if (c <= X) ib = max(ib, c);
                }
            } else if (hi - lo < kWarpScanMax) {
                const int d = atomicAdd(&w.nd, 1);
                w.bq[d] = (int16_t)qi;
                w.dlo[d] = (int16_t)lo;
                w.dhi[d] = (int16_t)hi;
                w.qL[qi] = L;
                continue;
            } else {
                defer_wavelet(O, o, L, kc(v, w0 + lo), kc(v, w0 + hi + 1), wq, wq_count);
                continue;
            }
        }
        write_result(vsym, O, o, (int64_t)s * G.T, L, ib);
    }
    __syncthreads();
    // Phase D: mid-size intervals, 8 lanes each (4 per warp), 8 ranks per step
    const int nd = w.nd;
    {
        constexpr int kSub = 8;
        const int grp = lane / kSub, sl = lane % kSub;
        for (int d0 = warp * (32 / kSub); d0 < nd; d0 += (kRThreads / 32) * (32 / kSub)) {
            const int di = d0 + grp;
            const bool act = di < nd;
            int qi = 0, lo = 0, hi = -1, X = -1;
            if (act) {
                qi = w.bq[di];
                lo = w.dlo[di];
                hi = w.dhi[di];
                X = query_bound(G, s, item_pos(w.qt[qi], G.T));
            }
            int best = -1;
            for (int r = lo + sl; r <= hi; r += kSub) {
                const int c = w.kp[r];
                if (c <= X) best = max(best, c);
            }
#pragma unroll
            for (int o = kSub / 2; o >= 1; o >>= 1) best = max(best, __shfl_xor_sync(ROSA_FULL_MASK, best, o));
            if (act && sl == 0)
                write_result(vsym, O, out_slot(G, s, (uint32_t)w.qt[qi]), (int64_t)s * G.T, w.qL[qi], best);
        }
    }
    // one bound task per (side, L) this tile needs beyond its window
    if (threadIdx.x < 2 * kBoundShared) {
        const int side = threadIdx.x / kBoundShared, L = threadIdx.x % kBoundShared;
        if ((w.need[side] >> L) & 1ull)
            btask[atomicAdd(btask_count, 1)] = (int32_t)(((int64_t)blockIdx.x << 7) | (side << 6) | L);
    }
}

// ---- warp-cooperative scans over global memory ------------------------------


// NEAREST: LCP with the first admissible key in direction dir if > lim, else 0.
// BOUND: the last rank in direction dir whose running LCP stays >= lim.
enum ScanMode { NEAREST = 0, BOUND = 1 };

// One step over up to 32 consecutive ranks: lane i visits first + dir*i when
// i < cnt.  Returns true when the scan has ended (result set).
template <int MODE>
__device__ bool warp_fine(const StreamView &v, int first, int cnt, int dir, int X, int lim, int lane, int &carry,
                          int &result) {
    // carry (the running LCP before this step) is above lim (NEAREST) or at
    // least lim (BOUND), or the scan would have ended: the stop is the first
    // lane whose own edge crosses lim, and a warp min-reduction over the
    // lanes up to a hit gives the running LCP there
    const int r = first + dir * lane;
    const bool act = lane < cnt && r >= 0 && r < v.n;
    int e = INT_MAX;
    bool valid = false;
    if (act) {
        e = dir < 0 ? v.lcp[r + 1] : v.lcp[r];
        if (MODE == NEAREST) valid = kpos(v, r) <= X;
    } else if (lane < cnt) {
        e = -1;   // ran off the stream: ends every scan
    }
    if (MODE == NEAREST) {
        const unsigned stopm = __ballot_sync(ROSA_FULL_MASK, lane < cnt && e <= lim);
        const int fs = stopm ? __ffs(stopm) - 1 : 32;
        const unsigned valm = __ballot_sync(ROSA_FULL_MASK, valid) & (fs < 32 ? ((1u << fs) - 1u) : ROSA_FULL_MASK);
        if (valm) {
            const int fv = __ffs(valm) - 1;
            result = min(carry, __reduce_min_sync(ROSA_FULL_MASK, lane <= fv ? e : INT_MAX));
            return true;
        }
        if (fs < 32) {
            result = 0;
            return true;
        }
    } else {
        const unsigned stopm = __ballot_sync(ROSA_FULL_MASK, lane < cnt && e < lim);
        if (stopm) {
            const int fs = __ffs(stopm) - 1;
            result = first + dir * (fs - 1);
            return true;
        }
        result = first + dir * (cnt - 1);
    }
    carry = min(carry, __reduce_min_sync(ROSA_FULL_MASK, e));
    return false;
}

template <int MODE>
__device__ int warp_scan(const StreamView &v, int j, int dir, int X, int lim, int lane) {
    int carry = INT_MAX;
    int result = MODE == NEAREST ? 0 : j;
    int next = j + dir;
    if (next < 0 || next >= v.n) return result;
    const int cnt = dir < 0 ? (next & (kL1 - 1)) + 1 : kL1 - (next & (kL1 - 1));
    if (warp_fine<MODE>(v, next, cnt, dir, X, lim, lane, carry, result)) return result;
    next += dir * cnt;
    // `next` is now the last (dir < 0) or first (dir > 0) rank of block next / 32
    while (next >= 0 && next < v.n) {
        if ((dir < 0 && (next & (kL2 - 1)) == kL2 - 1) || (dir > 0 && (next & (kL2 - 1)) == 0)) {
            // at a 1024-rank boundary: try to cross up to 32 whole 1024-blocks at once
            const int nb2 = next / kL2;
            const int b2 = nb2 + dir * lane;
            const bool in2 = b2 >= 0 && b2 < v.nb2 && (b2 + 1) * kL2 <= v.n;
            int bm2 = -1;
            bool hv2 = true;
            if (in2) {
                const int edge = dir < 0 ? ((b2 + 1) * kL2 < v.n ? v.ein2[b2 + 1] : INT_MAX) : v.ein2[b2];
                bm2 = min(edge, v.em2[b2]);
                hv2 = v.mp2[b2] <= X;
            }
            // the first stop: the first block that leaves the stream, holds an
            // admissible key, or whose own LCP minimum crosses lim (carry does not)
            const bool st2 = MODE == NEAREST ? (!in2 || hv2 || bm2 <= lim) : (!in2 || bm2 < lim);
            const unsigned sm2 = __ballot_sync(ROSA_FULL_MASK, st2);
            const int f2 = sm2 ? __ffs(sm2) - 1 : 32;
            if (f2 > 0) {
                carry = min(carry, __reduce_min_sync(ROSA_FULL_MASK, lane < f2 ? bm2 : INT_MAX));
                if (MODE == BOUND) {
                    const int bl = nb2 + dir * (f2 - 1);
                    result = dir < 0 ? bl * kL2 : bl * kL2 + kL2 - 1;
                }
                next += dir * kL2 * f2;
                if (f2 == 32) continue;
                if (next < 0 || next >= v.n) break;
            }
        }
        const int nb = next / kL1;
        const int b = nb + dir * lane;
        const bool inside = b >= 0 && b < v.nb1 && (b + 1) * kL1 <= v.n;
        int bm = -1;
        bool has_valid = true;
        if (inside) {
            const int edge = dir < 0 ? ((b + 1) * kL1 < v.n ? v.ein1[b + 1] : INT_MAX) : v.ein1[b];
            bm = min(edge, v.em1[b]);
            has_valid = v.mp1[b] <= X;
        }
        const bool stop_here = MODE == NEAREST ? (!inside || has_valid || bm <= lim) : (!inside || bm < lim);
        const unsigned sm = __ballot_sync(ROSA_FULL_MASK, stop_here);
        const int f = sm ? __ffs(sm) - 1 : 32;
        if (f > 0) {
            carry = min(carry, __reduce_min_sync(ROSA_FULL_MASK, lane < f ? bm : INT_MAX));
            if (MODE == BOUND) {
                const int bl = nb + dir * (f - 1);
                result = dir < 0 ? bl * kL1 : bl * kL1 + kL1 - 1;
            }
            if (f == 32) {
                next += dir * kL1 * 32;
                continue;
            }
        }
        const int bb = nb + dir * f;
        const int first = dir < 0 ? bb * kL1 + kL1 - 1 : bb * kL1;
        if (first < 0 || first >= v.n) break;
        if (warp_fine<MODE>(v, first, kL1, dir, X, lim, lane, carry, result)) return result;
        next = first + dir * kL1;
    }
    return result;
}

// One warp per listed query: scans for L and the interval bounds; the most
// recent admissible end is left to wavelet_query_kernel.
__global__ void resolve_hard_kernel(Geometry G, ResolveArgs A, Outs O,
                                    const int32_t *__restrict__ hard, const int *__restrict__ hard_count,
                                    int32_t *__restrict__ wq, int *wq_count) {
    const int nh = *hard_count;
    const int lane = threadIdx.x & 31;
    const int64_t wid = (blockIdx.x * (int64_t)blockDim.x + threadIdx.x) >> 5;
    const int64_t nw = ((int64_t)gridDim.x * blockDim.x) >> 5;
    for (int64_t h = wid; h < nh; h += nw) {
        const int64_t gi = hard[h];
        const int s = stream_of(gi, G.n);
        const int j = (int)(gi - (int64_t)s * G.n);
        const uint32_t x = A.sa[gi];
        const int X = query_bound(G, s, item_pos(x, G.T));
        const int64_t o = out_slot(G, s, x);
        const StreamView v = make_view(G, s, A);
        const int bl = warp_scan<NEAREST>(v, j, -1, X, 0, lane);
        const int br = warp_scan<NEAREST>(v, j, +1, X, bl, lane);
        const int L = max(bl, br);
        if (L > 0) {
            const int lo = warp_scan<BOUND>(v, j, -1, X, L, lane);
            const int hi = warp_scan<BOUND>(v, j, +1, X, L, lane);
            if (lane == 0) defer_wavelet(O, o, L, kc(v, lo), kc(v, hi + 1), wq, wq_count);
        } else if (lane == 0) {
            O.E(o) = -1;
            O.L(o) = 0;
            O.Y(o) = -1;
        }
    }
}

// Queries whose L is known but whose interval runs past the staged window:
// one warp scans outward from the window edge on each open side, then the
// query is parked for the wavelet lookup.
__global__ void resolve_bounds_kernel(Geometry G, ResolveArgs A, Outs O,
                                      const int32_t *__restrict__ hardb, const int *__restrict__ hardb_count,
                                      int32_t *__restrict__ wq, int *wq_count) {
    const int nh = *hardb_count;
    const int lane = threadIdx.x & 31;
    const int64_t wid = (blockIdx.x * (int64_t)blockDim.x + threadIdx.x) >> 5;
    const int64_t nw = ((int64_t)gridDim.x * blockDim.x) >> 5;
    for (int64_t h = wid; h < nh; h += nw) {
        const int64_t gi = hardb[h];
        const int s = stream_of(gi, G.n);
        const int j = (int)(gi - (int64_t)s * G.n);
        const uint32_t x = A.sa[gi];
        const int X = query_bound(G, s, item_pos(x, G.T));
        const int64_t o = out_slot(G, s, x);
        const int L = O.L(o);
        int lo = O.E(o), hi = O.Y(o);
        const int w0 = (j / kRTile) * kRTile - kRHalo;
        const StreamView v = make_view(G, s, A);
        if (lo < 0) lo = warp_scan<BOUND>(v, w0, -1, X, L, lane);
        if (hi < 0) hi = warp_scan<BOUND>(v, w0 + kRWin - 1, +1, X, L, lane);
        if (lane == 0) {
            O.E(o) = kc(v, lo);
            O.Y(o) = kc(v, hi + 1);
            wq[atomicAdd(wq_count, 1)] = (int32_t)o;
        }
    }
}

// One warp per (tile, side, L): the interval bound beyond the tile's window.
__global__ void bound_task_kernel(Geometry G, ResolveArgs A, const int32_t *__restrict__ btask,
                                  const int *__restrict__ btask_count, int32_t *__restrict__ btab) {
    const int nt = *btask_count;
    const int lane = threadIdx.x & 31;
    const int ntr = ceil_div(G.n, kRTile);
    const int64_t wid = (blockIdx.x * (int64_t)blockDim.x + threadIdx.x) >> 5;
    const int64_t nw = ((int64_t)gridDim.x * blockDim.x) >> 5;
    for (int64_t e = wid; e < nt; e += nw) {
        const int code = btask[e];
        const int tile = code >> 7, side = (code >> 6) & 1, L = code & 63;
        const int s = tile / ntr, tt = tile - s * ntr;
        const int w0 = tt * kRTile - kRHalo;
        const StreamView v = make_view(G, s, A);
        const int r = side ? warp_scan<BOUND>(v, w0 + kRWin - 1, +1, 0, L, lane)
                           : warp_scan<BOUND>(v, w0, -1, 0, L, lane);
        if (lane == 0) btab[(int64_t)tile * 2 * kBoundShared + side * kBoundShared + L] = r;
    }
}

// Queries waiting for a shared bound: fill the open side(s) from the table
// and park the query for the wavelet lookup.
__global__ void bound_finish_kernel(Geometry G, ResolveArgs A, Outs O,
                                    const int32_t *__restrict__ hardw, const int *__restrict__ hardw_count,
                                    const int32_t *__restrict__ btab, int32_t *__restrict__ wq, int *wq_count) {
    const int nh = *hardw_count;
    const int ntr = ceil_div(G.n, kRTile);
    for (int64_t h = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; h < nh; h += (int64_t)gridDim.x * blockDim.x) {
        const int64_t gi = hardw[h];
        const int s = stream_of(gi, G.n);
        const int j = (int)(gi - (int64_t)s * G.n);
        const uint32_t x = A.sa[gi];
        const int64_t o = out_slot(G, s, x);
        const int L = O.L(o);
        const int64_t tb = ((int64_t)s * ntr + j / kRTile) * 2 * kBoundShared;
        int lo = O.E(o), hi = O.Y(o);
        if (lo < 0) lo = btab[tb + L];
        if (hi < 0) hi = btab[tb + kBoundShared + L];
        const StreamView v = make_view(G, s, A);
        O.E(o) = kc(v, lo);
        O.Y(o) = kc(v, hi + 1);
        wq[atomicAdd(wq_count, 1)] = (int32_t)o;
    }
}

// Largest admissible key position inside each parked query's key range.
__global__ void __launch_bounds__(256, 8)
wavelet_query_kernel(Geometry G, ResolveArgs A, const uint8_t *__restrict__ vsym, Outs O,
                                     const int32_t *__restrict__ wq, const int *__restrict__ wq_count) {
    const int nq = *wq_count;
    const int nw = (G.T >> 6) + 1;
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < nq; i += (int64_t)gridDim.x * blockDim.x) {
        const int64_t o = wq[i];
        int s, t;
        slot_stream_time(G, o, s, t);
        const int klo = O.E(o), khi = O.Y(o);
        const WWord *W = A.words + (int64_t)s * A.nbits * nw;
        const int ib = wavelet_max_le(W, A.wz + (int64_t)s * A.nbits, A.leaf + (int64_t)s * G.T, A.nbits, A.nlev, nw,
                                      klo, khi, query_bound(G, s, t));
        O.E(o) = ib;
        O.Y(o) = ib >= 0 ? (int32_t)vsym[(int64_t)s * G.T + ib + 1] : -1;
    }
}


// The resolve tile needs more than 48 KB of shared memory; opt in once per
// device (a host-side attribute, so later calls, captured or not, skip it).
cudaError_t tile_smem_optin() {
    static std::mutex mu;
    static bool done[64] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    std::lock_guard<std::mutex> lock(mu);
    if (dev >= 0 && dev < 64 && done[dev]) return cudaSuccess;
    e = cudaFuncSetAttribute(resolve_tile_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sizeof(WinSmem));
    if (e == cudaSuccess && dev >= 0 && dev < 64) done[dev] = true;
    return e;
}

}  // namespace

int device_sm_count() {
    static std::mutex mu;
    static int sms[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
    std::lock_guard<std::mutex> lock(mu);
    if (sms[dev] == 0) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n < 1) return 148;
        sms[dev] = n;
    }
    return sms[dev];
}

int match_launch_count(int S, int T, int K, bool same, int mcf) {
    if (S == 0 || T == 0) return 0;
    const Geometry G = make_geometry(S, T, K, 1, same, mcf);
    int rounds = 0;
    for (int64_t h = G.D0; h < T; h *= 2) ++rounds;
    const int passes = ceil_div(G.keybits - G.idbits, kRadixBits);
    // keys0 + 3 per radix pass + groups0 + 3 per doubling round + 2 lcp + summary
    // + wavelet (key count unless every item is a key, compaction, one per level)
    // + 6 resolve (+ the counterfactual assembly)
    return 1 + 3 * passes + 1 + 3 * rounds + 3 + (G.allkeys ? 0 : 1) + 1 + G.wlev + 6 + (mcf > 0 ? 1 : 0);
}

size_t match_workspace_bytes(int S, int T, int K, bool same, int mcf) {
    const Geometry G = make_geometry(S, T, K, 1, same, mcf);
    return carve(G, nullptr).bytes;
}

namespace {

// Counterfactual tables [S, T, M, 2] (beta last): the branch that keeps
// query bit j is the ordinary result; the other one is the flipped branch.
__global__ void cf_assemble_kernel(const uint8_t *__restrict__ q, int64_t ST, int M, const int32_t *__restrict__ oe,
                                   const int32_t *__restrict__ ol, const int32_t *__restrict__ oy,
                                   const int32_t *__restrict__ fe, const int32_t *__restrict__ fl,
                                   const int32_t *__restrict__ fy, int32_t *__restrict__ end_cf,
                                   int32_t *__restrict__ len_cf, int32_t *__restrict__ sym_cf) {
    const int64_t total = ST * M;
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total;
         i += (int64_t)gridDim.x * blockDim.x) {
        const int64_t o = i / M;
        const int j = (int)(i - o * M);
        const int keep = (q[o] >> j) & 1;
        const int64_t b = i * 2;
        end_cf[b + keep] = oe[o];
        len_cf[b + keep] = ol[o];
        sym_cf[b + keep] = oy[o];
        end_cf[b + 1 - keep] = fe[i];
        len_cf[b + 1 - keep] = fl[i];
        sym_cf[b + 1 - keep] = fy[i];
    }
}

cudaError_t run_match(const uint8_t *q, const uint8_t *k, const uint8_t *v, const Geometry &G, const Workspace &W,
                      Outs O, cudaStream_t st) {
    cudaError_t err;
    if ((err = cudaMemsetAsync(W.status, 0, 256 + 256, st)) != cudaSuccess) return err;   // status + counts
    if (G.S == 0 || G.T == 0) return cudaSuccess;
    const int T = G.T;
    const uint8_t *vs = v ? v : k;

    // 1a. keys
    keys0_kernel<<<(unsigned)((int64_t)G.S * G.nkinds * ceil_div(T, kKeysTile)), kKeysThreads, 0, st>>>(
        q, k, G, W.keys[0], W.status);
    // 1b. radix sort over the key bits above the item id, 8 bits per pass
    int cur = 0;
    const unsigned tiles = (unsigned)(G.S * G.ntps);
    for (int shift = G.idbits; shift < G.keybits; shift += kRadixBits) {
        radix_hist_kernel<<<tiles, kRadixThreads, 0, st>>>(W.keys[cur], G, shift, W.hist);
        radix_scan_kernel<<<(unsigned)G.S, kRadixBins, 0, st>>>(W.hist, G.ntps);
        radix_scatter_kernel<<<tiles, kRadixThreads, 0, st>>>(W.keys[cur], W.keys[cur ^ 1], G, shift, W.hist);
        cur ^= 1;
    }
    uint64_t *keys = W.keys[cur];
    uint64_t *scratch = W.keys[cur ^ 1];
    uint32_t *sa = W.sa;
    // 1c. round-0 groups (lists buffer 0)
    groups0_kernel<<<tiles, 256, 0, st>>>(keys, sa, G, W.rank, W.lcp, W.lists[0][0], W.lists[0][1], W.counts,
                                          W.kcount, W.counts + 10);
    // 1d. doubling rounds while some string is longer than the sorted depth
    int lb = 0;
    const int sms = device_sm_count();
    const unsigned wgrid = sms * 8;   // 8 CTAs of 8 warps per SM, grid-stride over groups
    for (int64_t h = G.D0; h < T; h *= 2) {
        int *cnt = W.counts + 2 * lb;
        int *cnt_next = W.counts + 2 * (lb ^ 1);
        dbl_keys_sort_kernel<<<wgrid, 256, 0, st>>>(W.lists[lb][0], W.lists[lb][1], cnt, G, h, sa, W.rank, W.k2);
        dbl_sort_large_kernel<<<sms * 2, kLargeThreads, 0, st>>>(W.lists[lb][1], cnt, sa, W.k2, scratch);
        if ((err = cudaMemsetAsync(cnt_next, 0, 2 * sizeof(int), st)) != cudaSuccess) return err;
        dbl_regroup_kernel<<<wgrid, 256, 0, st>>>(W.lists[lb][0], W.lists[lb][1], cnt, G, 2 * h, sa, W.k2, W.rank,
                                                  W.lists[lb ^ 1][0], W.lists[lb ^ 1][1], cnt_next);
        lb ^= 1;
    }
    // 2. LCP
    lcp_ties_kernel<<<sms * 16, 256, 0, st>>>(q, k, G, sa, W.lcp, W.kcount, W.counts + 10, W.hard, W.counts + 6);
    lcp_long_kernel<<<sms * 8, 256, 0, st>>>(q, k, G, sa, W.lcp, W.hard, W.counts + 6);
    // 3a. summaries
    summary_kernel<<<(unsigned)(G.S * G.nb2), 256, 0, st>>>(G, sa, W.lcp, W.minpos1, W.emin1, W.ein1,
                                                           W.minpos2, W.emin2, W.ein2);
    // 3b. wavelet matrix over key positions in rank order
    if ((err = cudaMemsetAsync(W.wcnt, 0, (size_t)G.wbits * G.S * G.ntw * 4, st)) != cudaSuccess) return err;
    if (!G.allkeys) key_tile_count_kernel<<<(unsigned)(G.S * G.ntps), 256, 0, st>>>(G, sa, W.ktile);
    wavelet_compact_kernel<<<(unsigned)(G.S * G.ntps), 256, 0, st>>>(G, G.wbits, sa, W.ktile, W.kcount, W.wvals[0],
                                                                      W.wcnt);
    WWord *words = static_cast<WWord *>(W.words);
    for (int lv = 0; lv < G.wlev; ++lv)
        wavelet_level_kernel<<<(unsigned)(G.S * G.ntw), 256, 0, st>>>(G, G.wbits, lv, W.wvals[lv & 1],
                                                                       W.wvals[(lv + 1) & 1], W.wcnt, words, W.wz);
    // 3c. resolve: thread per query, then warp per query for the long scans
    if ((err = tile_smem_optin()) != cudaSuccess) return err;
    ResolveArgs A{sa, W.lcp, W.minpos1, W.emin1, W.ein1, W.minpos2, W.emin2, W.ein2, G.allkeys ? nullptr : W.kcount,
                  words, W.wz, W.wvals[G.wlev & 1], G.wbits, G.wlev};
    int *hard_count = W.counts + 4;
    int *wq_count = W.counts + 5;
    int *hardb_count = W.counts + 7;
    int *hardw_count = W.counts + 8;
    int *btask_count = W.counts + 9;
    resolve_tile_kernel<<<(unsigned)(G.S * ceil_div(G.n, kRTile)), kRThreads, sizeof(WinSmem), st>>>(
        G, A, vs, O, W.hard, hard_count, W.hardb, hardb_count, W.hardw, hardw_count, W.btask, btask_count, W.wq,
        wq_count);
    resolve_hard_kernel<<<sms * 16, 256, 0, st>>>(G, A, O, W.hard, hard_count, W.wq, wq_count);
    resolve_bounds_kernel<<<sms * 16, 256, 0, st>>>(G, A, O, W.hardb, hardb_count, W.wq, wq_count);
    bound_task_kernel<<<sms * 16, 256, 0, st>>>(G, A, W.btask, btask_count, W.btab);
    bound_finish_kernel<<<sms * 16, 256, 0, st>>>(G, A, O, W.hardw, hardw_count, W.btab, W.wq, wq_count);
    wavelet_query_kernel<<<sms * 16, 256, 0, st>>>(G, A, vs, O, W.wq, wq_count);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_match(const uint8_t *q, const uint8_t *k, const uint8_t *v, int S, int T, int K, int g,
                         int32_t *end_idx, int32_t *len, int32_t *sym, void *workspace, size_t ws_bytes,
                         cudaStream_t st, const int32_t *xbound) {
    Geometry G = make_geometry(S, T, K, g, q == k);
    G.xb = xbound;
    const Workspace W = carve(G, workspace);
    if (W.bytes > ws_bytes) return cudaErrorInvalidValue;
    const Outs O{end_idx, len, sym, nullptr, nullptr, nullptr, (int64_t)S * T};
    return run_match(q, k, v, G, W, O, st);
}

cudaError_t launch_match_cf(const uint8_t *q, const uint8_t *k, const uint8_t *v, int S, int T, int M, int g,
                            int32_t *end_idx, int32_t *len, int32_t *sym, int32_t *end_cf, int32_t *len_cf,
                            int32_t *sym_cf, void *workspace, size_t ws_bytes, cudaStream_t st) {
    const Geometry G = make_geometry(S, T, 1 << M, g, q == k, M);
    const Workspace W = carve(G, workspace);
    if (W.bytes > ws_bytes) return cudaErrorInvalidValue;
    const Outs O{end_idx, len, sym, W.flip[0], W.flip[1], W.flip[2], (int64_t)S * T};
    cudaError_t e = run_match(q, k, v, G, W, O, st);
    if (e != cudaSuccess || S == 0 || T == 0) return e;
    const int64_t ST = (int64_t)S * T;
    cf_assemble_kernel<<<(unsigned)(device_sm_count() * 8), 256, 0, st>>>(
        q, ST, M, end_idx, len, sym, W.flip[0], W.flip[1], W.flip[2], end_cf, len_cf, sym_cf);
    return cudaGetLastError();
}

}  // namespace rosa
