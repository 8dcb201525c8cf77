// decode_static.cu -- mlra_decode for callers that cannot allocate device
// memory.
//
// mlra_decode needs a scratch workspace (the split-KV partial outputs, their
// log-sum-exps, the per-sequence split counters and the device error word).
// Some callers cannot provide one: plugins that must not allocate from the
// host application's memory pools, runtimes that have handed all device
// memory to their own allocator, and latency-critical serving loops that
// forbid allocation after start-up (cudaMalloc synchronises the device and
// can fail under memory pressure).  This entry point serves them: its
// scratch is a fixed array in the library's own device image, so the call
// itself allocates nothing.
//
// Costs and limits:
//  - every GPU that loads this library holds kStaticScratchBytes of device
//    memory for the array until the process exits;
//  - a step whose workspace would exceed kStaticScratchBytes is rejected
//    with MLRA_ERR_WORKSPACE (use mlra_decode with your own workspace);
//  - all calls on a device share the one array: calls that may overlap on the
//    GPU (different streams without ordering between them) race and corrupt
//    each other's results;
//  - every call first clears, stream-ordered, the parts of the array that
//    must start at zero (the error word and the call's split counters), so a
//    call never inherits state from an earlier one, not even from a call
//    whose kernel gave up on a bounded wait;
//  - the array's device address is looked up (cudaGetSymbolAddress) on the
//    first call in each CUDA context, with that context current: make the
//    first call on a device, and the first after a cudaDeviceReset, before
//    any stream capture begins.
#include <cuda.h>

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
// device address comes from cudaGetSymbolAddress below.
static __device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

// Unique id of the current CUDA context (driver entry points reached through
// the runtime, so the library links no driver library).
using CtxGetCurrentFn = CUresult (*)(CUcontext*);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long*);

bool current_context_id(unsigned long long* id) {
    static CtxGetCurrentFn get_current = nullptr;
    static CtxGetIdFn get_id = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_current = reinterpret_cast<CtxGetCurrentFn>(p);
        p = nullptr;
        if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_id = reinterpret_cast<CtxGetIdFn>(p);
    });
    CUcontext ctx = nullptr;
    if (get_current == nullptr || get_id == nullptr || get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr)
        return false;
    return get_id(ctx, id) == CUDA_SUCCESS;
}

struct ScratchAddress {
    unsigned long long ctx_id = 0;
    void* ptr = nullptr;
};
std::mutex g_setup_mutex;
ScratchAddress g_scratch[kMaxDevices];

// Device address of the scratch in the current context, looked up once per
// context: a new context (e.g. after cudaDeviceReset) reloads the module,
// and the array may then sit elsewhere.  nullptr if the lookup fails.
void* scratch_in_current_context() {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    // the runtime makes the device's primary context current on first use
    if (cudaFree(nullptr) != cudaSuccess) return nullptr;
    unsigned long long id = 0;
    if (!current_context_id(&id)) return nullptr;
    std::lock_guard<std::mutex> lock(g_setup_mutex);
    ScratchAddress& s = g_scratch[dev];
    if (s.ptr == nullptr || s.ctx_id != id) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_static_scratch) != cudaSuccess || p == nullptr) return nullptr;
        s.ptr = p;
        s.ctx_id = id;
    }
    return s.ptr;
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
    void* scratch = scratch_in_current_context();
    if (scratch == nullptr) return MLRA_ERR_CUDA;
    mlra::DecodeArgs a;
    const mlra_status s = mlra::decode_tc_args(dims, q_lat, q_rope, latent_cache, rope_cache, block_table,
                                               seqlens, scale, out_scale, out, scratch, kStaticScratchBytes, &a);
    if (s != MLRA_OK) return s;
    // Clear the error word and this call's split counters (the first
    // 256 + 4 * batch * head groups bytes of the workspace layout) before the kernel, so
    // that no earlier call's state -- a stale count left by a kernel that gave
    // up on a bounded wait -- reaches this one.  Stream-ordered, no allocation.
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const size_t clear = reinterpret_cast<char*>(a.seq_cnt + (size_t)dims->batch * mlra::tc_head_groups(dims->heads, dims->d_c)) -
                         static_cast<char*>(scratch);
    if (cudaMemsetAsync(scratch, 0, clear, st) != cudaSuccess) return MLRA_ERR_CUDA;
    if (mlra::launch_decode_tc(a, st) != cudaSuccess) return MLRA_ERR_CUDA;
    // the error word (offset 0) goes to the caller, stream-ordered
    if (device_status != nullptr &&
        cudaMemcpyAsync(device_status, scratch, sizeof(int32_t), cudaMemcpyDeviceToDevice, st) != cudaSuccess)
        return MLRA_ERR_CUDA;
    return MLRA_OK;
}

}  // extern "C"
