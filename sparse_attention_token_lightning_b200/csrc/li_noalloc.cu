// li_indexer_noalloc: the indexer for callers that may not allocate device memory (plugin
// enqueue steps without an allocator, runtimes that forbid allocation after start-up, real-time
// loops). The workspace li_indexer needs comes from a static device array compiled into this
// file instead of from the caller. See include/li.h for the contract.
#include <cstdio>
#include <mutex>

#include "li_internal.cuh"

namespace {

constexpr size_t kScratchBytes = LI_NOALLOC_SCRATCH_BYTES;

// The scratch every li_indexer_noalloc call on a device uses. In host code this name is only a
// handle for cudaGetSymbolAddress, never a device address.
__device__ __align__(256) unsigned char g_noalloc_scratch[kScratchBytes];

constexpr int kMaxDevices = 128;
void *g_scratch_addr[kMaxDevices] = {};
std::mutex g_scratch_mu;

// Device address of the scratch on the current device, looked up once per device.
cudaError_t scratch_address(void **out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    if (!g_scratch_addr[dev]) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess) return e;
        g_scratch_addr[dev] = p;
    }
    *out = g_scratch_addr[dev];
    return cudaSuccess;
}

}  // namespace

extern "C" li_status li_indexer_noalloc(const li_args *args, int32_t *sparse_indices,
                                        float *sparse_values, uint32_t *device_status,
                                        void *stream) {
    size_t need = 0;
    li_status st = li_indexer_workspace_size(args, &need);
    if (st != LI_OK) return st;
    if (need > kScratchBytes) {
        char msg[256];
        snprintf(msg, sizeof msg,
                 "li_indexer_noalloc: this problem needs %zu bytes of workspace but the static "
                 "scratch holds %zu bytes (LI_NOALLOC_SCRATCH_BYTES); call li_indexer with a "
                 "caller-provided workspace instead", need, kScratchBytes);
        li::set_last_error(msg);
        return LI_ERR_WORKSPACE;
    }
    void *scratch = nullptr;
    cudaError_t e = scratch_address(&scratch);
    if (e != cudaSuccess) {
        char msg[256];
        snprintf(msg, sizeof msg, "li_indexer_noalloc: scratch address lookup failed: %s",
                 cudaGetErrorString(e));
        li::set_last_error(msg);
        return LI_ERR_CUDA;
    }
    st = li_indexer(args, nullptr, scratch, kScratchBytes, sparse_indices, sparse_values, stream);
    if (st != LI_OK) return st;
    if (device_status) {
        e = cudaMemcpyAsync(device_status, scratch, sizeof(uint32_t), cudaMemcpyDeviceToDevice,
                            static_cast<cudaStream_t>(stream));
        if (e != cudaSuccess) {
            char msg[256];
            snprintf(msg, sizeof msg, "li_indexer_noalloc: status copy failed: %s",
                     cudaGetErrorString(e));
            li::set_last_error(msg);
            return LI_ERR_CUDA;
        }
    }
    return LI_OK;
}
