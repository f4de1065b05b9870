// rosa_match_noalloc: the matcher with its scratch memory in a fixed,
// file-scope device array instead of a caller-provided workspace.
//
// Some callers cannot allocate device memory at the point where they need
// the retrieval: hosts that own every device allocation and give plug-ins no
// allocator, or serving loops that must not call cudaMalloc/cudaFree because
// those calls can synchronise the whole device.  They still pass their own
// input and output buffers; only the scratch space comes from here.
#include <cstdint>
#include <mutex>
#include <cuda_runtime.h>

#include "../../include/rosa.h"
#include "kernels.h"

namespace {

// Every GPU that loads this library reserves this much device memory for the
// array, for the lifetime of the process.
static __device__ __align__(256) unsigned char g_noalloc_scratch[ROSA_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_setup_mutex;
void *g_scratch_ptr[kMaxDevices] = {};

// Device address of the array on the current device, looked up once per
// device.  In host code the array's name is only a stand-in for the symbol,
// so the kernels must be given this address, never the name.
cudaError_t scratch_address(void **out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_setup_mutex);
    if (!g_scratch_ptr[dev]) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess) return e;
        g_scratch_ptr[dev] = p;
    }
    *out = g_scratch_ptr[dev];
    return cudaSuccess;
}

}  // namespace

extern "C" int rosa_match_noalloc(const uint8_t *q, const uint8_t *k, const uint8_t *v, int S, int T, int K,
                                  int g, int32_t *end_idx, int32_t *len, int32_t *sym, cudaStream_t stream) {
    if (S < 0 || T < 0 || K < 1 || K > 256 || g < 1) return ROSA_ERR_INVALID_ARG;
    if ((int64_t)S * T * 2 >= ((int64_t)1 << 31)) return ROSA_ERR_INVALID_ARG;
    if ((int64_t)S * T > 0 && (!q || !k || !end_idx || !len || !sym)) return ROSA_ERR_INVALID_ARG;
    const size_t need = rosa::match_workspace_bytes(S, T, K, q == k);
    if (need > (size_t)ROSA_NOALLOC_SCRATCH_BYTES) return ROSA_ERR_WORKSPACE;   // too large for the fixed array
    void *scratch = nullptr;
    if (scratch_address(&scratch) != cudaSuccess) return ROSA_ERR_CUDA;
    // The matcher clears every counter and status word it relies on before use,
    // so the array's contents from the previous call do not matter.
    return rosa::launch_match(q, k, v, S, T, K, g, end_idx, len, sym, scratch, (size_t)ROSA_NOALLOC_SCRATCH_BYTES,
                              stream) == cudaSuccess
               ? ROSA_OK
               : ROSA_ERR_CUDA;
}

extern "C" int rosa_match_noalloc_device_status(cudaStream_t stream, uint32_t *status) {
    if (!status) return ROSA_ERR_INVALID_ARG;
    void *scratch = nullptr;
    if (scratch_address(&scratch) != cudaSuccess) return ROSA_ERR_CUDA;
    uint32_t h = 0;
    cudaError_t e = cudaMemcpyAsync(&h, static_cast<const char *>(scratch) + rosa::kStatusOffset, sizeof h,
                                    cudaMemcpyDeviceToHost, stream);
    if (e == cudaSuccess) e = cudaStreamSynchronize(stream);
    if (e != cudaSuccess) return ROSA_ERR_CUDA;
    *status = h;
    return ROSA_OK;
}
