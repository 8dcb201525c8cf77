// decode_static.cu -- mlra_decode for callers that cannot allocate device
// memory.
//
// mlra_decode needs a scratch workspace (the split-KV partial outputs, their
// log-sum-exps and the device error word).  Some callers cannot provide one:
// plugins that must not allocate from the host application's memory pools,
// runtimes that have handed all device memory to their own allocator, and
// latency-critical serving loops that forbid allocation after start-up
// (cudaMalloc synchronises the device and can fail under memory pressure).
// This entry point serves them: its scratch is a fixed array in the
// library's own device image, so the call itself allocates nothing.
//
// Costs and limits:
//  - every GPU that loads this library holds kStaticScratchBytes of device
//    memory for the array until the process exits;
//  - a step whose workspace would exceed kStaticScratchBytes is rejected
//    with MLRA_ERR_WORKSPACE (use mlra_decode with your own workspace);
//  - all calls on a device share the one array: calls that may overlap on the
//    GPU (different streams without ordering between them) race and corrupt
//    each other's results;
//  - the first call on each device looks up the array's device address
//    (cudaGetSymbolAddress) with that device current; make that first call
//    before any stream capture begins.
#include <mutex>

#include "common.cuh"
#include "kernels.h"

namespace {

// 8 MiB: holds the partials of every workload in the test suite (the largest,
// 64 sequences x 16 heads x 4 branches x 128 latent columns over 212 slots,
// needs about 7 MB).
constexpr size_t kStaticScratchBytes = size_t(8) << 20;
constexpr int kMaxDevices = 64;

// The scratch.  In host code this name only stands for the symbol: its
// device address comes from cudaGetSymbolAddress below.  Device memory of a
// __device__ array starts zeroed, so the error word at its start and the
// split counters are 0 before the first call; each call clears the error word
// again after copying it out, and the decode kernel returns the counters to 0.
static __device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

std::mutex g_setup_mutex;
void* g_scratch_ptr[kMaxDevices] = {nullptr};

// Device address of the scratch on the current device (looked up once per
// device); nullptr if the lookup fails.
void* scratch_on_current_device() {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    std::lock_guard<std::mutex> lock(g_setup_mutex);
    if (g_scratch_ptr[dev] == nullptr) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_static_scratch) != cudaSuccess || p == nullptr) return nullptr;
        g_scratch_ptr[dev] = p;
    }
    return g_scratch_ptr[dev];
}

}  // namespace

extern "C" {

mlra_status mlra_decode_static_scratch(const mlra_dims* dims, const void* q_lat, const void* q_rope,
                                       const void* latent_cache, const void* rope_cache,
                                       const int32_t* block_table, const int32_t* seqlens,
                                       float scale, float out_scale, void* out,
                                       int32_t* device_status, void* stream) {
    if (mlra_decode_workspace_bytes(dims, 1) == 0) return MLRA_ERR_INVALID_ARG;  // dims alone
    const size_t need = mlra_decode_workspace_bytes(dims, 0);                 // this device's grid
    if (need == 0) return MLRA_ERR_CUDA;
    if (need > kStaticScratchBytes) return MLRA_ERR_WORKSPACE;
    if (device_status != nullptr && (reinterpret_cast<uintptr_t>(device_status) & 3u) != 0)
        return MLRA_ERR_INVALID_ARG;
    void* scratch = scratch_on_current_device();
    if (scratch == nullptr) return MLRA_ERR_CUDA;
    const mlra_status s = mlra_decode(dims, q_lat, q_rope, latent_cache, rope_cache, block_table,
                                      seqlens, scale, out_scale, out, scratch, kStaticScratchBytes,
                                      stream);
    if (s != MLRA_OK) return s;
    // The error word (offset 0 of the workspace layout) goes to the caller,
    // then back to zero for the next call; both are stream-ordered copies
    // and sets, not allocations.
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (device_status != nullptr &&
        cudaMemcpyAsync(device_status, scratch, sizeof(int32_t), cudaMemcpyDeviceToDevice, st) != cudaSuccess)
        return MLRA_ERR_CUDA;
    if (cudaMemsetAsync(scratch, 0, sizeof(int32_t), st) != cudaSuccess) return MLRA_ERR_CUDA;
    return MLRA_OK;
}

}  // extern "C"
