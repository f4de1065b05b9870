// Internal launch interface between the C ABI (rosa_abi.cu) and the kernels.
#pragma once
#include <cstddef>
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

namespace rosa {

// Tensor map of a 2-D bf16 tensor [rows][cols] for TMA (tmap.cu): box of
// box_cols (64: one 128-byte swizzle row) x box_rows; false if the encoder is
// unavailable or the rows are not 16-byte aligned.
bool make_tmap_bf16_2d(CUtensorMap *m, const void *base, uint64_t rows, uint64_t cols, uint32_t box_rows,
                       uint32_t box_cols);

// Streaming multiprocessors of the current device (queried once per device);
// grids of grid-stride kernels are sized in multiples of it.
int device_sm_count();

// One launch for `count` (1 or 2) tensors of the same shape.
cudaError_t launch_discretize(const uint16_t *const *x, uint8_t *const *sym, int count, int B, int T, int C,
                              int M, cudaStream_t stream);

cudaError_t launch_gather(const uint16_t *V, int64_t vrow, int64_t rho, const int32_t *end_idx,
                          int B, int R, int T, int d, uint16_t *out, cudaStream_t stream);

// Workspace bytes for the matcher with n items per stream (n = T when q and k
// are the same buffer, 2T otherwise, plus mcf * T counterfactual branches).
size_t match_workspace_bytes(int S, int T, int K, bool same, int mcf = 0);

// xbound: optional [S, T] int32, the largest admissible key position of
// each query (replaces t - g; run-level retrieval passes its own bounds).
cudaError_t launch_match(const uint8_t *q, const uint8_t *k, const uint8_t *v, int S, int T, int K,
                         int g, int32_t *end_idx, int32_t *len, int32_t *sym, void *workspace,
                         size_t ws_bytes, cudaStream_t stream, const int32_t *xbound = nullptr);

// Kernel launches one launch_match (mcf = 0) or launch_match_cf call enqueues.
int match_launch_count(int S, int T, int K, bool same, int mcf = 0);

// The ordinary retrieval plus, for every query bit j < M, the branch with
// that bit flipped (one retrieval step from the same history); the tables
// are [S, T, M, 2] with the forced bit value last.  Alphabet K = 2^M.
cudaError_t launch_match_cf(const uint8_t *q, const uint8_t *k, const uint8_t *v, int S, int T, int M, int g,
                            int32_t *end_idx, int32_t *len, int32_t *sym, int32_t *end_cf, int32_t *len_cf,
                            int32_t *sym_cf, void *workspace, size_t ws_bytes, cudaStream_t stream);

// Run-level retrieval with adjacent folding (rle.cu).
size_t match_rle_workspace_bytes(int S, int T, int K, bool same);
cudaError_t launch_match_rle(const uint8_t *q, const uint8_t *k, const uint8_t *v, int S, int T, int K, int g,
                             int32_t *end_idx, int32_t *len, int32_t *sym, void *workspace, size_t ws_bytes,
                             cudaStream_t stream);
int match_rle_launch_count(int S, int T, int K, bool same);

// Read-out embedding and injection on the tensor cores (inject.cu).
cudaError_t launch_inject(const int32_t *sym, const uint16_t *e0, const uint16_t *e1, const uint16_t *W, int B, int R,
                          int M, int T, int D, uint16_t *out, uint32_t *status, cudaStream_t stream);

// Layer norm + projection + discretisation on the tensor cores (ln_project.cu).
size_t ln_project_workspace_bytes(int D, int C, int M);
cudaError_t launch_ln_project(const uint16_t *H, const float *gamma, const float *beta, const uint16_t *Wq,
                              const uint16_t *Wk, int B, int T, int D, int C, int M, float eps, uint8_t *symq,
                              uint8_t *symk, void *workspace, size_t ws_bytes, uint32_t *status, cudaStream_t stream);

// Offset of the device status word inside a matcher workspace.
constexpr size_t kStatusOffset = 0;

}  // namespace rosa
