/*
 * rosa.h -- C ABI of the B200-native ROSA retrieval step.
 *
 * The operation is the retrieval stage of "ROSA-Tuning: Enhancing Windowed
 * Attention with Global Recall" (arXiv 2602.02499): binary discretisation of
 * hidden states into multi-route symbol streams (section 3.2), the suffix
 * retrieval destination tau of each position (section 3.3, Eq. 16; appendix
 * B.3), and the read-out of value rows at tau (appendix C.4, Eq. 17).
 *
 * Conventions shared by every call:
 *   - All tensor pointers are DEVICE pointers into memory the caller owns
 *     (cudaMalloc, a torch tensor, ...).  The library allocates nothing and
 *     keeps no state between calls, with one exception: rosa_match_noalloc
 *     (below) takes its scratch from a fixed device array the library
 *     reserves on every GPU that loads it, which keeps the last call's
 *     contents.
 *   - Work is enqueued on `stream` (NULL = the legacy default stream) and the
 *     call returns without waiting for it, except where stated.
 *   - Argument errors are detected on the host before anything is enqueued
 *     and returned as ROSA_ERR_INVALID_ARG / ROSA_ERR_WORKSPACE; launch
 *     failures are returned as ROSA_ERR_CUDA.  No call aborts the process or
 *     throws across the ABI.
 *   - bf16 tensors are passed as pointers to their 16-bit patterns
 *     (rosa_bf16), IEEE bfloat16 layout.
 */
#ifndef ROSA_H_
#define ROSA_H_

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#if defined(__GNUC__)
#define ROSA_API __attribute__((visibility("default")))
#else
#define ROSA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef uint16_t rosa_bf16;

typedef enum {
    ROSA_OK = 0,
    ROSA_ERR_INVALID_ARG = 1,   /* bad shape, range, alignment or NULL pointer */
    ROSA_ERR_WORKSPACE = 2,     /* workspace missing or smaller than required */
    ROSA_ERR_CUDA = 3,          /* a CUDA launch or runtime call failed */
    ROSA_ERR_DEVICE = 4,        /* a device-side check fired (see rosa_match_device_status) */
    ROSA_ERR_INTERNAL = 5
} rosa_status;

/* Human-readable name of a status code (static storage, never NULL). */
ROSA_API const char *rosa_status_string(int status);

/*
 * Binary discretisation and multi-route packing (section 3.2, Eqs. 10-15;
 * route layout of section 4.1).
 *
 *   x    [B, T, C] bf16, row-major (channel fastest).
 *   sym  [B, R, T] uint8, R = C / M, written in full.
 *   sym[b, r, t] = sum_{j<M} I[x[b, t, r*M + j] > 0] * 2^j
 *
 * The threshold is strict: +0, -0 and NaN give bit 0; +inf and positive
 * subnormals give bit 1.  Requires 1 <= M <= 8, C % M == 0, B, T >= 0, C >= 1.
 * Any alignment is accepted (16-byte aligned rows take the vector path).
 */
ROSA_API int rosa_discretize(const rosa_bf16 *x, int B, int T, int C, int M,
                    uint8_t *sym, cudaStream_t stream);

/*
 * rosa_discretize of the query and the key projections (two tensors of the
 * same shape) in one launch: xq -> symq, xk -> symk, each as above.
 * Requires B <= 32767; otherwise the same conditions as rosa_discretize.
 */
ROSA_API int rosa_discretize_pair(const rosa_bf16 *xq, const rosa_bf16 *xk, int B, int T, int C, int M,
                                  uint8_t *symq, uint8_t *symk, cudaStream_t stream);

/*
 * Bytes of workspace rosa_match needs for S streams of length T over an
 * alphabet of K symbols (an upper bound valid whether or not q == k).
 * Returns 0 for invalid sizes.
 */
ROSA_API size_t rosa_match_workspace_size(int S, int T, int K);

/*
 * Suffix retrieval (section 3.3, Eq. 16; appendix B.3), S independent
 * streams (one per batch x route pair, section 4.1).
 *
 *   q, k  [S, T] uint8 query / key symbols, each < K.  Passing the same
 *         pointer for q and k selects the self-retrieval form (q = k), which
 *         needs half the work; distinct pointers with equal contents give the
 *         same result.
 *   v     [S, T] uint8 value symbols, or NULL to read them from k.
 *   g     causal lag >= 1: key end i is admissible at query time t iff
 *         i <= t - g.  g = 2 gives tau = i + 1 <= t - 1, the range of Eq. 16.
 *
 * For every stream s and position t, with L the length of the longest
 * suffix of q[s, 0..t] that ends in k[s, .] at some admissible i, and i* the
 * largest such i:
 *   end_idx[s, t] = i*        (-1 if L = 0)   -- tau = end_idx + 1
 *   len[s, t]     = L
 *   sym[s, t]     = v[s, i*+1] (-1 if L = 0)
 * Outputs are int32 [S, T], written in full.
 *
 * `workspace` is device memory of at least rosa_match_workspace_size(S, T, K)
 * bytes, 256-byte aligned; its contents on entry do not matter and are
 * clobbered.  Calls that share a workspace must not overlap on the GPU.
 * Requires 1 <= K <= 256, g >= 1, S >= 0, T >= 0 and S*T*2 < 2^31.
 * Symbols >= K are a caller error: they are masked to the alphabet's bit
 * width and flagged in the workspace status word (rosa_match_device_status).
 */
ROSA_API int rosa_match(const uint8_t *q, const uint8_t *k, const uint8_t *v,
               int S, int T, int K, int g,
               int32_t *end_idx, int32_t *len, int32_t *sym,
               void *workspace, size_t ws_bytes, cudaStream_t stream);

/*
 * Number of kernel launches one rosa_match call with these arguments
 * enqueues (q_is_k: 1 when q and k are the same pointer).  Host-only; lets a
 * caller account for the work it submits.  Returns -1 for invalid sizes.
 */
ROSA_API int rosa_match_launch_count(int S, int T, int K, int q_is_k);

/*
 * Per-bit counterfactual destinations (section 3.5: every query bit is a
 * discrete decision switch; the branches "force the bit to 0" and "force
 * it to 1" each take one retrieval step from the same history; appendix
 * C.5 precomputes tau^(0), tau^(1) for the gradients).
 *
 * Symbols carry M bits (K = 2^M, 1 <= M <= 8).  For position t, bit j < M
 * and beta in {0, 1}, the branch symbol is q[s, t] with bit j set to beta;
 * q[s, 0..t-1] and the keys stay as they are, and the branch's destination
 * is the ordinary retrieval of that symbol (longest admissible match ending
 * at t, most recent end, same lag g).  The branch that keeps the actual bit
 * is the ordinary result, which is also returned:
 *   end_idx, len, sym  [S, T]        as rosa_match
 *   end_cf, len_cf, sym_cf [S, T, M, 2] int32, beta last:
 *     end_cf[s, t, j, beta] = i*' (-1 if no match), len_cf = L',
 *     sym_cf = v[s, i*' + 1] (-1 if no match)
 * All outputs are written in full.  Requires 1 <= M <= 8, g >= 1,
 * S*T*(2+M) < 2^31 and symbols < 2^M; workspace of at least
 * rosa_match_cf_workspace_size(S, T, M) bytes, 256-byte aligned (status
 * word read with rosa_match_device_status).  Key-bit branches are not
 * computed.
 */
ROSA_API size_t rosa_match_cf_workspace_size(int S, int T, int M);
ROSA_API int rosa_match_cf(const uint8_t *q, const uint8_t *k, const uint8_t *v,
                           int S, int T, int M, int g,
                           int32_t *end_idx, int32_t *len, int32_t *sym,
                           int32_t *end_cf, int32_t *len_cf, int32_t *sym_cf,
                           void *workspace, size_t ws_bytes, cudaStream_t stream);

/* Kernel launches one rosa_match_cf call enqueues (-1 for invalid sizes). */
ROSA_API int rosa_match_cf_launch_count(int S, int T, int M, int q_is_k);

/*
 * Run-level retrieval with adjacent folding (section 3.3, the run-length
 * encoding paragraph; appendix C.5-C.6 for the per-run bookkeeping).
 *
 * Consecutive equal symbols of a stream form one run; both q and k fold.
 * Key runs have symbols c_l and start times s_l, query runs d_m and u_m.
 * The retrieval moves only at run boundaries: query run m is answered once,
 * at its start time u_m, and every t of the run reports that answer.  Key
 * run l is admissible iff the next key run starts at s_{l+1} <= u_m - g + 1
 * (g = 2: tau <= t - 1, read strictly from the past).  With L the longest
 * run-level common suffix of d_0..d_m and c_0..c_l over admissible l, and
 * l* the largest admissible l reaching it, for every t of query run m:
 *   end_idx[s, t] = s_{l*+1} - 1   (-1 if L = 0)   -- tau = end_idx + 1 is
 *                                    the start of the key run after l*
 *   len[s, t]     = L              (counted in runs)
 *   sym[s, t]     = v[s, s_{l*+1}]  (-1 if L = 0)
 * Without adjacent repeats every run is one symbol and this is rosa_match.
 * With K = 2 folded streams alternate, so the answer for query run m is the
 * last admissible key run with d_m's symbol, L = min(l*, m) + 1; the call
 * computes that directly instead of sorting (same results; symbols >= 2 are
 * flagged, and for such streams the outputs of this path are unspecified).
 * Shapes, ownership and errors as for rosa_match; the workspace is at least
 * rosa_match_rle_workspace_size(S, T, K) bytes (256-byte aligned) and its
 * status word is read with rosa_match_device_status.
 */
ROSA_API size_t rosa_match_rle_workspace_size(int S, int T, int K);
ROSA_API int rosa_match_rle(const uint8_t *q, const uint8_t *k, const uint8_t *v,
                            int S, int T, int K, int g,
                            int32_t *end_idx, int32_t *len, int32_t *sym,
                            void *workspace, size_t ws_bytes, cudaStream_t stream);

/* Kernel launches one rosa_match_rle call enqueues (-1 for invalid sizes). */
ROSA_API int rosa_match_rle_launch_count(int S, int T, int K, int q_is_k);

/*
 * Reads the device status word a previous rosa_match (or rosa_match_rle)
 * left in `workspace` (0 = no device-side check fired, otherwise a bit set
 * of ROSA_DEV_*).
 * Synchronises `stream`.  Returns ROSA_OK or ROSA_ERR_CUDA.
 */
#define ROSA_DEV_SYMBOL_RANGE 1u   /* some input symbol was >= K */
#define ROSA_DEV_TIMEOUT 2u        /* a bounded wait inside a kernel ran out */
ROSA_API int rosa_match_device_status(const void *workspace, cudaStream_t stream, uint32_t *status);

/*
 * rosa_match without a workspace argument: the same retrieval, with its
 * scratch memory taken from a fixed device array inside this library
 * (ROSA_NOALLOC_SCRATCH_BYTES, 64 MiB, reserved on every GPU that loads the
 * library until the process exits).  There is no counterpart on the pages;
 * it exists for callers that cannot allocate device memory where they run
 * the retrieval (hosts that own all device allocations, serving loops that
 * must not call cudaMalloc/cudaFree because those can synchronise the
 * device).  Inputs and outputs are the caller's, as for rosa_match.
 *
 * Sizes whose workspace (rosa_match_workspace_size) exceeds the array are
 * rejected with ROSA_ERR_WORKSPACE before anything touches the GPU; the
 * array holds about 500 000 positions (S*T), e.g. 16 streams of 16384 with
 * q != k over 256 symbols.
 * The first call on a device looks up the array's device address (once per
 * device, with that device current); make that first call before any
 * stream capture.  The address is cached for the life of the process: after
 * cudaDeviceReset on a device, do not call this entry point on that device
 * again (the cached address may no longer be the array's).  All calls share
 * the one array and it keeps the last call's contents: calls that overlap on
 * the GPU (different streams or threads) race and must be serialised by the
 * caller.  Symbols >= K are masked and flagged as for rosa_match; the flag
 * is read with rosa_match_noalloc_device_status.
 */
#define ROSA_NOALLOC_SCRATCH_BYTES (64u << 20)
ROSA_API int rosa_match_noalloc(const uint8_t *q, const uint8_t *k, const uint8_t *v,
                                int S, int T, int K, int g,
                                int32_t *end_idx, int32_t *len, int32_t *sym, cudaStream_t stream);

/*
 * The device status word (ROSA_DEV_* bits) the last rosa_match_noalloc call
 * on the current device left in the fixed array; the counterpart of
 * rosa_match_device_status for callers without a workspace.  Synchronises
 * `stream`.  Returns ROSA_OK, ROSA_ERR_INVALID_ARG (NULL status) or
 * ROSA_ERR_CUDA.
 */
ROSA_API int rosa_match_noalloc_device_status(cudaStream_t stream, uint32_t *status);

/*
 * Layer norm, query/key projection and discretisation in one pass, on the
 * tensor cores (section 3.2: U = LN(H), Q = U W_q, K = U W_k, then the
 * strict threshold and packing of Eqs. 10-15).
 *
 *   H       [B, T, D] bf16 hidden states, row-major (16-byte aligned, D % 8 == 0).
 *   gamma, beta [D] float layer-norm scale and shift, or NULL (1 and 0).
 *   Wq, Wk  [D, C] bf16 projections, row-major; C % M == 0.
 *   symq, symk [B, C/M, T] uint8, written in full:
 *     u = gamma * (h - mean(h)) / sqrt(var(h) + eps) + beta  (population variance)
 *     sym[b, r, t] = sum_j I[(u W)[c = r*M + j] > 0] * 2^j
 * The layer norm is folded into the contraction (the kernels multiply the raw
 * rows by gamma o W, kept to about 16 significant bits as a bf16 high + low
 * pair, with fp32 accumulation), so a channel whose exact projection lies
 * within that rounding of zero may take either bit.
 * `workspace` holds the prepared weights: at least
 * rosa_ln_project_workspace_size(D, C, M) bytes, 256-byte aligned.
 * dev_status: optional device word (ROSA_DEV_TIMEOUT if a bounded wait ran out).
 * Requires B, T >= 0, D >= 8, D % 8 == 0, 1 <= M <= 8, C >= M.
 */
ROSA_API size_t rosa_ln_project_workspace_size(int D, int C, int M);
ROSA_API int rosa_ln_project_discretize(const rosa_bf16 *H, const float *gamma, const float *beta,
                                        const rosa_bf16 *Wq, const rosa_bf16 *Wk, int B, int T, int D, int C, int M,
                                        float eps, uint8_t *symq, uint8_t *symk, void *workspace, size_t ws_bytes,
                                        uint32_t *dev_status, cudaStream_t stream);

/*
 * Read-out embedding and injection (appendix C.3, Eqs. 21-22 of the main
 * text, with the Eq. 17 mask), on the tensor cores.
 *
 *   sym    [B*R, T] int32: the recalled value symbol of route r at position
 *          t (rosa_match's sym output; -1 where nothing matched).
 *   e0, e1 [C] bf16, C = R*M: the embedding of a recalled 0 / 1 bit.
 *   W_out  [D, C] bf16, row-major.
 *   inj    [B, T, D] bf16, written in full:
 *     y[b, t, r*M + j] = m * ((1 - bit_j) * e0[r*M + j] + bit_j * e1[r*M + j])
 *       with bit_j = (sym >> j) & 1 and m = I[sym >= 0];
 *     inj[b, t, d] = bf16(sum_c W_out[d, c] * y[b, t, c])  (fp32 accumulation)
 * dev_status: optional device word; ROSA_DEV_TIMEOUT is or-ed into it if a
 * kernel's bounded wait ran out (the affected tiles are not written).
 * Requires B, T >= 0, 1 <= M <= 8, R >= 1, D >= 1; any alignment.  W_out
 * arrives by TMA when C >= 64, C % 8 == 0 and W_out is 16-byte aligned, and
 * inj leaves by TMA stores when D >= 64, D % 8 == 0 and inj is 16-byte
 * aligned; other shapes take plain loads and stores.  With C <= 512 the call
 * runs persistent CTAs that each hold 256 of an SM's 512 tensor-memory
 * columns until they finish (a kernel that holds tensor memory on the same
 * SMs delays them).
 */
ROSA_API int rosa_inject(const int32_t *sym, const rosa_bf16 *e0, const rosa_bf16 *e1, const rosa_bf16 *W_out,
                         int B, int R, int M, int T, int D, rosa_bf16 *inj, uint32_t *dev_status,
                         cudaStream_t stream);

/*
 * Read-out of value rows at tau (appendix C.4 with the Eq. 17 mask).
 *
 *   V        [B, T, *] bf16 rows, row stride v_row_stride elements.
 *   end_idx  [B*R, T] int32 from rosa_match (stream s = b*R + r).
 *   out      [B, T, R*d] bf16, written in full.
 *   out[b, t, r*d + m] = V[b, end_idx[b*R+r, t] + 1, r*v_route_stride + m]
 *                        for m < d, or +0.0 when end_idx = -1.
 * v_route_stride = d reads each route's own slice; 0 makes every route read
 * the same d-wide row.  rosa_match only produces end_idx in [-1, T-2]; any
 * value outside that range is treated like -1 (zero row), so no call reads
 * outside V.  A bit-exact copy: no arithmetic on the values.
 * Requires B, R, T >= 0, d >= 1, v_route_stride >= 0,
 * (R-1)*v_route_stride + d <= v_row_stride.
 */
ROSA_API int rosa_gather(const rosa_bf16 *V, int64_t v_row_stride, int64_t v_route_stride,
                const int32_t *end_idx, int B, int R, int T, int d,
                rosa_bf16 *out, cudaStream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* ROSA_H_ */
