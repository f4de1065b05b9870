// Internal launch interface between the C ABI (rosa_abi.cu) and the kernels.
#pragma once
#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>

namespace rosa {

// Streaming multiprocessors of the current device (queried once per device);
// grids of grid-stride kernels are sized in multiples of it.
int device_sm_count();

// One launch for `count` (1 or 2) tensors of the same shape.
cudaError_t launch_discretize(const uint16_t *const *x, uint8_t *const *sym, int count, int B, int T, int C,
                              int M, cudaStream_t stream);

cudaError_t launch_gather(const uint16_t *V, int64_t vrow, int64_t rho, const int32_t *end_idx,
                          int B, int R, int T, int d, uint16_t *out, cudaStream_t stream);

// Workspace bytes for the matcher with n items per stream (n = T when q and k
// are the same buffer, 2T otherwise).
size_t match_workspace_bytes(int S, int T, int K, bool same);

cudaError_t launch_match(const uint8_t *q, const uint8_t *k, const uint8_t *v, int S, int T, int K,
                         int g, int32_t *end_idx, int32_t *len, int32_t *sym, void *workspace,
                         size_t ws_bytes, cudaStream_t stream);

// Kernel launches one launch_match call enqueues.
int match_launch_count(int S, int T, int K, bool same);

// Offset of the device status word inside a matcher workspace.
constexpr size_t kStatusOffset = 0;

}  // namespace rosa
