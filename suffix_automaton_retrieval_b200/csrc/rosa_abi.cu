// C ABI of the ROSA retrieval step (declared in include/rosa.h).
// Host-side argument checks, then the launches in dense.cu and match.cu.
#include <cstdint>
#include <cuda_runtime.h>

#include "../../include/rosa.h"
#include "kernels.h"

namespace {

int cuda_status(cudaError_t e) { return e == cudaSuccess ? ROSA_OK : ROSA_ERR_CUDA; }

bool aligned(const void *p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

bool match_sizes_ok(int S, int T, int K) {
    if (S < 0 || T < 0 || K < 1 || K > 256) return false;
    // every item index (2 per position) must fit a signed 32-bit integer
    return (int64_t)S * T * 2 < ((int64_t)1 << 31);
}

}  // namespace

extern "C" {

const char *rosa_status_string(int status) {
    switch (status) {
        case ROSA_OK: return "ROSA_OK";
        case ROSA_ERR_INVALID_ARG: return "ROSA_ERR_INVALID_ARG";
        case ROSA_ERR_WORKSPACE: return "ROSA_ERR_WORKSPACE";
        case ROSA_ERR_CUDA: return "ROSA_ERR_CUDA";
        case ROSA_ERR_DEVICE: return "ROSA_ERR_DEVICE";
        case ROSA_ERR_INTERNAL: return "ROSA_ERR_INTERNAL";
        default: return "ROSA_ERR_UNKNOWN";
    }
}

int rosa_discretize(const rosa_bf16 *x, int B, int T, int C, int M, uint8_t *sym, cudaStream_t stream) {
    if (B < 0 || T < 0 || C < 1 || M < 1 || M > 8 || C % M != 0 || B > 65535) return ROSA_ERR_INVALID_ARG;
    if ((int64_t)B * T > 0 && (!x || !sym)) return ROSA_ERR_INVALID_ARG;
    const uint16_t *xs[1] = {x};
    uint8_t *ss[1] = {sym};
    return cuda_status(rosa::launch_discretize(xs, ss, 1, B, T, C, M, stream));
}

int rosa_discretize_pair(const rosa_bf16 *xq, const rosa_bf16 *xk, int B, int T, int C, int M, uint8_t *symq,
                         uint8_t *symk, cudaStream_t stream) {
    if (B < 0 || T < 0 || C < 1 || M < 1 || M > 8 || C % M != 0 || B > 32767) return ROSA_ERR_INVALID_ARG;
    if ((int64_t)B * T > 0 && (!xq || !xk || !symq || !symk)) return ROSA_ERR_INVALID_ARG;
    const uint16_t *xs[2] = {xq, xk};
    uint8_t *ss[2] = {symq, symk};
    return cuda_status(rosa::launch_discretize(xs, ss, 2, B, T, C, M, stream));
}

size_t rosa_match_workspace_size(int S, int T, int K) {
    if (!match_sizes_ok(S, T, K)) return 0;
    return rosa::match_workspace_bytes(S, T, K, /*same=*/false);
}

int rosa_match(const uint8_t *q, const uint8_t *k, const uint8_t *v, int S, int T, int K, int g,
               int32_t *end_idx, int32_t *len, int32_t *sym, void *workspace, size_t ws_bytes,
               cudaStream_t stream) {
    if (!match_sizes_ok(S, T, K) || g < 1) return ROSA_ERR_INVALID_ARG;
    if ((int64_t)S * T > 0 && (!q || !k || !end_idx || !len || !sym)) return ROSA_ERR_INVALID_ARG;
    if (!workspace || !aligned(workspace, 256)) return ROSA_ERR_WORKSPACE;
    if (ws_bytes < rosa::match_workspace_bytes(S, T, K, q == k)) return ROSA_ERR_WORKSPACE;
    return cuda_status(rosa::launch_match(q, k, v, S, T, K, g, end_idx, len, sym, workspace, ws_bytes, stream));
}

namespace {
bool cf_sizes_ok(int S, int T, int M) {
    if (S < 0 || T < 0 || M < 1 || M > 8) return false;
    // every item index (keys, queries and M branch kinds per position) fits a signed 32-bit integer
    return (int64_t)S * T * (2 + M) < ((int64_t)1 << 31);
}
}  // namespace

size_t rosa_match_cf_workspace_size(int S, int T, int M) {
    if (!cf_sizes_ok(S, T, M)) return 0;
    return rosa::match_workspace_bytes(S, T, 1 << M, /*same=*/false, M);
}

int rosa_match_cf(const uint8_t *q, const uint8_t *k, const uint8_t *v, int S, int T, int M, int g,
                  int32_t *end_idx, int32_t *len, int32_t *sym, int32_t *end_cf, int32_t *len_cf, int32_t *sym_cf,
                  void *workspace, size_t ws_bytes, cudaStream_t stream) {
    if (!cf_sizes_ok(S, T, M) || g < 1) return ROSA_ERR_INVALID_ARG;
    if ((int64_t)S * T > 0 && (!q || !k || !end_idx || !len || !sym || !end_cf || !len_cf || !sym_cf))
        return ROSA_ERR_INVALID_ARG;
    if (!workspace || !aligned(workspace, 256)) return ROSA_ERR_WORKSPACE;
    if (ws_bytes < rosa::match_workspace_bytes(S, T, 1 << M, q == k, M)) return ROSA_ERR_WORKSPACE;
    return cuda_status(rosa::launch_match_cf(q, k, v, S, T, M, g, end_idx, len, sym, end_cf, len_cf, sym_cf,
                                             workspace, ws_bytes, stream));
}

int rosa_match_cf_launch_count(int S, int T, int M, int q_is_k) {
    if (!cf_sizes_ok(S, T, M)) return -1;
    return rosa::match_launch_count(S, T, 1 << M, q_is_k != 0, M);
}

size_t rosa_match_rle_workspace_size(int S, int T, int K) {
    if (!match_sizes_ok(S, T, K)) return 0;
    return rosa::match_rle_workspace_bytes(S, T, K, /*same=*/false);
}

int rosa_match_rle(const uint8_t *q, const uint8_t *k, const uint8_t *v, int S, int T, int K, int g,
                   int32_t *end_idx, int32_t *len, int32_t *sym, void *workspace, size_t ws_bytes,
                   cudaStream_t stream) {
    if (!match_sizes_ok(S, T, K) || g < 1) return ROSA_ERR_INVALID_ARG;
    if ((int64_t)S * T > 0 && (!q || !k || !end_idx || !len || !sym)) return ROSA_ERR_INVALID_ARG;
    if (!workspace || !aligned(workspace, 256)) return ROSA_ERR_WORKSPACE;
    if (ws_bytes < rosa::match_rle_workspace_bytes(S, T, K, q == k)) return ROSA_ERR_WORKSPACE;
    return cuda_status(rosa::launch_match_rle(q, k, v, S, T, K, g, end_idx, len, sym, workspace, ws_bytes, stream));
}

int rosa_match_rle_launch_count(int S, int T, int K, int q_is_k) {
    if (!match_sizes_ok(S, T, K)) return -1;
    return rosa::match_rle_launch_count(S, T, K, q_is_k != 0);
}

int rosa_match_launch_count(int S, int T, int K, int q_is_k) {
    if (!match_sizes_ok(S, T, K)) return -1;
    return rosa::match_launch_count(S, T, K, q_is_k != 0);
}

int rosa_match_device_status(const void *workspace, cudaStream_t stream, uint32_t *status) {
    if (!workspace || !status) return ROSA_ERR_INVALID_ARG;
    uint32_t h = 0;
    cudaError_t e = cudaMemcpyAsync(&h, static_cast<const char *>(workspace) + rosa::kStatusOffset, sizeof h,
                                    cudaMemcpyDeviceToHost, stream);
    if (e == cudaSuccess) e = cudaStreamSynchronize(stream);
    if (e != cudaSuccess) return ROSA_ERR_CUDA;
    *status = h;
    return ROSA_OK;
}

namespace {
bool lnp_sizes_ok(int D, int C, int M) {
    return D >= 8 && D % 8 == 0 && M >= 1 && M <= 8 && C >= M && C % M == 0 && C <= (1 << 16) && D <= (1 << 20);
}
}  // namespace

size_t rosa_ln_project_workspace_size(int D, int C, int M) {
    if (!lnp_sizes_ok(D, C, M)) return 0;
    return rosa::ln_project_workspace_bytes(D, C, M);
}

int rosa_ln_project_discretize(const rosa_bf16 *H, const float *gamma, const float *beta, const rosa_bf16 *Wq,
                               const rosa_bf16 *Wk, int B, int T, int D, int C, int M, float eps, uint8_t *symq,
                               uint8_t *symk, void *workspace, size_t ws_bytes, uint32_t *dev_status,
                               cudaStream_t stream) {
    if (B < 0 || T < 0 || !lnp_sizes_ok(D, C, M) || !(eps >= 0.f)) return ROSA_ERR_INVALID_ARG;
    if ((int64_t)B * T >= ((int64_t)1 << 31)) return ROSA_ERR_INVALID_ARG;
    if ((int64_t)B * T > 0 && (!H || !Wq || !Wk || !symq || !symk || !aligned(H, 16))) return ROSA_ERR_INVALID_ARG;
    if (!workspace || !aligned(workspace, 256)) return ROSA_ERR_WORKSPACE;
    if (ws_bytes < rosa::ln_project_workspace_bytes(D, C, M)) return ROSA_ERR_WORKSPACE;
    return cuda_status(rosa::launch_ln_project(H, gamma, beta, Wq, Wk, B, T, D, C, M, eps, symq, symk, workspace,
                                               ws_bytes, dev_status, stream));
}

int rosa_inject(const int32_t *sym, const rosa_bf16 *e0, const rosa_bf16 *e1, const rosa_bf16 *W_out, int B, int R,
                int M, int T, int D, rosa_bf16 *inj, uint32_t *dev_status, cudaStream_t stream) {
    if (B < 0 || T < 0 || R < 1 || M < 1 || M > 8 || D < 1) return ROSA_ERR_INVALID_ARG;
    if ((int64_t)B * T >= ((int64_t)1 << 31) / 2 || (int64_t)R * M > (1 << 20)) return ROSA_ERR_INVALID_ARG;
    if ((int64_t)B * T > 0 && (!sym || !e0 || !e1 || !W_out || !inj)) return ROSA_ERR_INVALID_ARG;
    return cuda_status(rosa::launch_inject(sym, e0, e1, W_out, B, R, M, T, D, inj, dev_status, stream));
}

int rosa_gather(const rosa_bf16 *V, int64_t v_row_stride, int64_t v_route_stride, const int32_t *end_idx,
                int B, int R, int T, int d, rosa_bf16 *out, cudaStream_t stream) {
    if (B < 0 || R < 0 || T < 0 || d < 1 || v_route_stride < 0 || B > 65535) return ROSA_ERR_INVALID_ARG;
    if (R > 0 && (int64_t)(R - 1) * v_route_stride + d > v_row_stride) return ROSA_ERR_INVALID_ARG;
    if ((int64_t)B * R * T > 0 && (!V || !end_idx || !out)) return ROSA_ERR_INVALID_ARG;
    return cuda_status(rosa::launch_gather(V, v_row_stride, v_route_stride, end_idx, B, R, T, d, out, stream));
}

}  // extern "C"
