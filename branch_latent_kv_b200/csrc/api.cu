// api.cu -- the C ABI declared in include/mlra.h: host-side validation,
// workspace sizing and kernel launches.  No allocation, no synchronisation
// (except mlra_read_device_error), no exceptions across the boundary.
#include <cmath>
#include <cstdint>
#include <cstring>

#include "common.cuh"
#include "kernels.h"

namespace {

using namespace mlra;

bool aligned16(const void* p) { return p != nullptr && (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool is_pow2_in(int v, int lo, int hi) { return v >= lo && v <= hi && (v & (v - 1)) == 0; }

// Structural validity of the dimensions (INVALID_ARG).
mlra_status check_dims(const mlra_dims* d) {
    if (d == nullptr) return MLRA_ERR_INVALID_ARG;
    if (d->batch < 1 || d->heads < 1 || d->branches < 1 || d->d_c < 1 || d->d_r < 1 ||
        d->page_size < 1 || d->max_pages_per_seq < 1 || d->num_pages < 1)
        return MLRA_ERR_INVALID_ARG;
    // every flat index must fit the kernels' 64-bit arithmetic and the
    // 32-bit row coordinates of the cache tensor maps
    if ((int64_t)d->num_pages * d->page_size > INT32_MAX) return MLRA_ERR_INVALID_ARG;
    if ((int64_t)d->max_pages_per_seq * d->page_size > INT32_MAX) return MLRA_ERR_INVALID_ARG;
    if ((int64_t)d->batch * d->max_pages_per_seq > INT32_MAX) return MLRA_ERR_INVALID_ARG;
    // the plan counts cost units in int32
    if (!plan_fits_int32(d->batch, d->page_size, d->max_pages_per_seq)) return MLRA_ERR_INVALID_ARG;
    if (d->batch > kMaxBatch) return MLRA_ERR_UNSUPPORTED;
    return MLRA_OK;
}

// Shapes the tensor-core decode kernel implements.
mlra_status check_tc_coverage(const mlra_dims* d) {
    if (!is_pow2_in(d->page_size, 16, 128)) return MLRA_ERR_UNSUPPORTED;
    if (!decode_tc_supported(d->branches, d->d_c, d->d_r, d->heads)) return MLRA_ERR_UNSUPPORTED;
    // one block of split counters per head group
    if ((int64_t)d->batch * tc_head_groups(d->heads, d->d_c) > kMaxBatch) return MLRA_ERR_UNSUPPORTED;
    return MLRA_OK;
}

// Shapes the CUDA-core decode kernel implements (its shared memory holds the
// whole query block and a 32-token tile).
mlra_status check_simt_coverage(const mlra_dims* d) {
    if (d->d_c % 8 != 0 || d->d_r % 8 != 0 || d->heads > 64) return MLRA_ERR_UNSUPPORTED;
    if ((int64_t)d->branches * d->d_c > 1024 || d->d_r > 256) return MLRA_ERR_UNSUPPORTED;
    if (decode_simt_smem_bytes(d->heads, d->branches, d->d_c, d->d_r) > 232448) return MLRA_ERR_UNSUPPORTED;
    return MLRA_OK;
}

int device_sm_count() {
    static int cache[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) return 0;
    if (dev < 64 && cache[dev] > 0) return cache[dev];
    int sms = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
    if (dev < 64) cache[dev] = sms;
    return sms;
}

mlra_status cuda_status(cudaError_t e) { return e == cudaSuccess ? MLRA_OK : MLRA_ERR_CUDA; }

// The address through which the device reaches `p` (device, managed or
// mapped pinned host memory), or null for memory the device cannot address.
const void* device_address(const void* p) {
    if (p == nullptr) return nullptr;
    cudaPointerAttributes at;
    if (cudaPointerGetAttributes(&at, p) != cudaSuccess) {
        cudaGetLastError();  // clear the error state the failed query leaves
        return nullptr;
    }
    switch (at.type) {
        case cudaMemoryTypeDevice:
        case cudaMemoryTypeManaged:
        case cudaMemoryTypeHost:
            return at.devicePointer;
        default:
            return nullptr;
    }
}


enum class Impl { kTensorCore, kSimt };

// Host validation of a decode call and the kernel arguments it implies.
mlra_status decode_args(Impl impl, const mlra_dims* dims, const void* q_lat, const void* q_rope,
                        const void* latent_cache, const void* rope_cache,
                        const int32_t* block_table, const int32_t* seqlens, float scale,
                        float out_scale, void* out, void* workspace, size_t workspace_bytes,
                        DecodeArgs* a_out) {
    mlra_status s = check_dims(dims);
    if (s != MLRA_OK) return s;
    s = impl == Impl::kTensorCore ? check_tc_coverage(dims) : check_simt_coverage(dims);
    if (s != MLRA_OK) return s;
    if (!aligned16(q_lat) || !aligned16(q_rope) || !aligned16(latent_cache) ||
        !aligned16(rope_cache) || !aligned16(block_table) || !aligned16(seqlens) ||
        !aligned16(out))
        return MLRA_ERR_INVALID_ARG;
    if (!(scale == scale) || !(out_scale == out_scale)) return MLRA_ERR_INVALID_ARG;  // NaN
    if (workspace == nullptr || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
        return MLRA_ERR_WORKSPACE;
    const int ctas = device_sm_count();
    if (ctas <= 0) return MLRA_ERR_CUDA;
    const WorkspaceLayout wl =
        workspace_layout(dims->batch, dims->heads, dims->branches, dims->d_c, ctas);
    if (workspace_bytes < wl.total) return MLRA_ERR_WORKSPACE;

    DecodeArgs& a = *a_out;
    a.q_lat = static_cast<const __nv_bfloat16*>(q_lat);
    a.q_rope = static_cast<const __nv_bfloat16*>(q_rope);
    a.latent = static_cast<const __nv_bfloat16*>(latent_cache);
    a.rope = static_cast<const __nv_bfloat16*>(rope_cache);
    a.block_table = block_table;
    a.seqlens = seqlens;
    a.out = static_cast<__nv_bfloat16*>(out);
    char* ws = static_cast<char*>(workspace);
    a.err = reinterpret_cast<int*>(ws + wl.err_off);
    a.lse_part = reinterpret_cast<float*>(ws + wl.lse_off);
    a.o_part = reinterpret_cast<float*>(ws + wl.o_off);
    a.seq_cnt = reinterpret_cast<int*>(ws + wl.cnt_off);
    a.batch = dims->batch;
    a.heads = dims->heads;
    a.branches = dims->branches;
    a.d_c = dims->d_c;
    a.d_r = dims->d_r;
    a.page_size = dims->page_size;
    a.max_pages = dims->max_pages_per_seq;
    a.num_pages = dims->num_pages;
    a.num_ctas = ctas;
    a.scale_log2 = scale * kLog2e;
    a.out_scale = out_scale;
    a.w_uv = nullptr;
    a.y = nullptr;
    a.d_h = 0;
    return MLRA_OK;
}

mlra_status decode_impl(Impl impl, const mlra_dims* dims, const void* q_lat, const void* q_rope,
                        const void* latent_cache, const void* rope_cache,
                        const int32_t* block_table, const int32_t* seqlens, float scale,
                        float out_scale, void* out, void* workspace, size_t workspace_bytes,
                        void* stream) {
    DecodeArgs a;
    const mlra_status s = decode_args(impl, dims, q_lat, q_rope, latent_cache, rope_cache, block_table,
                                      seqlens, scale, out_scale, out, workspace, workspace_bytes, &a);
    if (s != MLRA_OK) return s;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (impl == Impl::kTensorCore) return cuda_status(launch_decode_tc(a, st));  // merges in-kernel
    mlra_status r = cuda_status(launch_decode_simt(a, st));
    if (r != MLRA_OK) return r;
    return cuda_status(launch_combine(a, st));
}

}  // namespace

namespace mlra {
mlra_status decode_tc_args(const mlra_dims* dims, const void* q_lat, const void* q_rope,
                           const void* latent_cache, const void* rope_cache, const int32_t* block_table,
                           const int32_t* seqlens, float scale, float out_scale, void* out, void* workspace,
                           size_t workspace_bytes, DecodeArgs* a) {
    return decode_args(Impl::kTensorCore, dims, q_lat, q_rope, latent_cache, rope_cache, block_table, seqlens,
                       scale, out_scale, out, workspace, workspace_bytes, a);
}
}  // namespace mlra

extern "C" {

size_t mlra_decode_workspace_bytes(const mlra_dims* dims, int32_t num_ctas) {
    if (check_dims(dims) != MLRA_OK) return 0;
    if (num_ctas <= 0) num_ctas = device_sm_count();
    if (num_ctas <= 0) return 0;
    return workspace_layout(dims->batch, dims->heads, dims->branches, dims->d_c, num_ctas).total;
}

mlra_status mlra_decode(const mlra_dims* dims, const void* q_lat, const void* q_rope,
                        const void* latent_cache, const void* rope_cache,
                        const int32_t* block_table, const int32_t* seqlens, float scale,
                        float out_scale, void* out, void* workspace, size_t workspace_bytes,
                        void* stream) {
    return decode_impl(Impl::kTensorCore, dims, q_lat, q_rope, latent_cache, rope_cache, block_table,
                       seqlens, scale, out_scale, out, workspace, workspace_bytes, stream);
}

mlra_status mlra_decode_up_proj(const mlra_dims* dims, const void* q_lat, const void* q_rope,
                                const void* latent_cache, const void* rope_cache,
                                const int32_t* block_table, const int32_t* seqlens, float scale,
                                float out_scale, void* out, const void* w_uv, int32_t d_h, void* y,
                                void* workspace, size_t workspace_bytes, void* stream) {
    DecodeArgs a;
    mlra_status s = decode_args(Impl::kTensorCore, dims, q_lat, q_rope, latent_cache, rope_cache, block_table,
                                seqlens, scale, out_scale, out, workspace, workspace_bytes, &a);
    if (s != MLRA_OK) return s;
    if (!aligned16(w_uv)) return MLRA_ERR_INVALID_ARG;
    if (d_h != 64 && d_h != 128) return MLRA_ERR_UNSUPPORTED;
    if (dims->batch > kUpProjFusedMaxBatch) return MLRA_ERR_UNSUPPORTED;
    void* y_dev = const_cast<void*>(device_address(y));  // y may be mapped pinned host memory
    if (y_dev == nullptr || !aligned16(y_dev)) return MLRA_ERR_INVALID_ARG;
    a.w_uv = static_cast<const __nv_bfloat16*>(w_uv);
    a.y = static_cast<__nv_bfloat16*>(y_dev);
    a.d_h = d_h;
    const cudaError_t e = launch_decode_tc(a, static_cast<cudaStream_t>(stream));
    if (e == cudaErrorInvalidConfiguration) return MLRA_ERR_UNSUPPORTED;  // staging does not fit
    return cuda_status(e);
}

mlra_status mlra_decode_simt(const mlra_dims* dims, const void* q_lat, const void* q_rope,
                             const void* latent_cache, const void* rope_cache,
                             const int32_t* block_table, const int32_t* seqlens, float scale,
                             float out_scale, void* out, void* workspace, size_t workspace_bytes,
                             void* stream) {
    return decode_impl(Impl::kSimt, dims, q_lat, q_rope, latent_cache, rope_cache, block_table,
                       seqlens, scale, out_scale, out, workspace, workspace_bytes, stream);
}

namespace {

mlra_status up_proj_impl(int32_t batch, int32_t heads, int32_t branches, int32_t d_c, int32_t d_h,
                         const void* out_lat, const void* w_uv, const void* gate, void* y, void* stream) {
    if (batch < 1 || heads < 1 || branches < 1 || d_c < 1 || d_h < 1) return MLRA_ERR_INVALID_ARG;
    if (!aligned16(out_lat) || !aligned16(w_uv) || !aligned16(y)) return MLRA_ERR_INVALID_ARG;
    if (gate != nullptr && (reinterpret_cast<uintptr_t>(gate) & 1u) != 0) return MLRA_ERR_INVALID_ARG;
    if ((int64_t)batch * heads * d_h > INT32_MAX) return MLRA_ERR_INVALID_ARG;
    const int K = branches * d_c;
    if (K % 64 != 0 || K > 512 || (d_h != 64 && d_h != 128)) return MLRA_ERR_UNSUPPORTED;
    void* y_dev = const_cast<void*>(device_address(y));  // y may be mapped pinned host memory
    if (y_dev == nullptr || !aligned16(y_dev)) return MLRA_ERR_INVALID_ARG;
    return cuda_status(launch_up_proj(batch, heads, branches, d_c, d_h,
                                      static_cast<const __nv_bfloat16*>(out_lat),
                                      static_cast<const __nv_bfloat16*>(w_uv),
                                      static_cast<const __nv_bfloat16*>(gate),
                                      static_cast<__nv_bfloat16*>(y_dev),
                                      static_cast<cudaStream_t>(stream)));
}
}  // namespace

mlra_status mlra_up_proj(int32_t batch, int32_t heads, int32_t branches, int32_t d_c, int32_t d_h,
                         const void* out_lat, const void* w_uv, void* y, void* stream) {
    return up_proj_impl(batch, heads, branches, d_c, d_h, out_lat, w_uv, nullptr, y, stream);
}

mlra_status mlra_up_proj_gated(int32_t batch, int32_t heads, int32_t branches, int32_t d_c,
                               int32_t d_h, const void* out_lat, const void* w_uv, const void* gate,
                               void* y, void* stream) {
    if (gate == nullptr) return MLRA_ERR_INVALID_ARG;
    return up_proj_impl(batch, heads, branches, d_c, d_h, out_lat, w_uv, gate, y, stream);
}

size_t mlra_exchange_bytes(int32_t batch, int32_t heads, int32_t branches, int32_t d_c, int32_t d_h,
                           int32_t world) {
    if (batch < 1 || heads < 1 || branches < 1 || d_c < 1 || d_h < 1 || world < 1 || world > kMaxWorld) return 0;
    if ((branches * d_c) % 64 != 0 || branches * d_c > 512) return 0;
    if ((int64_t)batch * heads * d_h > INT32_MAX) return 0;
    return exchange_layout(batch, heads, d_h, world, up_proj_tiles(batch, heads, branches, d_c)).total;
}

mlra_status mlra_exchange_alloc(size_t bytes, void** region, void* ipc_handle) {
    if (region == nullptr || bytes == 0) return MLRA_ERR_INVALID_ARG;
    *region = nullptr;
    void* p = nullptr;
    if (cudaMalloc(&p, bytes) != cudaSuccess) return MLRA_ERR_CUDA;
    if (cudaMemset(p, 0, bytes) != cudaSuccess || cudaDeviceSynchronize() != cudaSuccess) {
        cudaFree(p);
        return MLRA_ERR_CUDA;
    }
    if (ipc_handle != nullptr) {
        static_assert(sizeof(cudaIpcMemHandle_t) == MLRA_IPC_HANDLE_BYTES, "IPC handle size");
        cudaIpcMemHandle_t h;
        if (cudaIpcGetMemHandle(&h, p) != cudaSuccess) {
            cudaFree(p);
            return MLRA_ERR_CUDA;
        }
        std::memcpy(ipc_handle, &h, sizeof(h));
    }
    *region = p;
    return MLRA_OK;
}

mlra_status mlra_exchange_open(const void* ipc_handle, void** region) {
    if (ipc_handle == nullptr || region == nullptr) return MLRA_ERR_INVALID_ARG;
    *region = nullptr;
    cudaIpcMemHandle_t h;
    std::memcpy(&h, ipc_handle, sizeof(h));
    void* p = nullptr;
    if (cudaIpcOpenMemHandle(&p, h, cudaIpcMemLazyEnablePeerAccess) != cudaSuccess) return MLRA_ERR_CUDA;
    *region = p;
    return MLRA_OK;
}

mlra_status mlra_exchange_close(void* region) {
    if (region == nullptr) return MLRA_ERR_INVALID_ARG;
    return cuda_status(cudaIpcCloseMemHandle(region));
}

mlra_status mlra_exchange_free(void* region) {
    if (region == nullptr) return MLRA_ERR_INVALID_ARG;
    return cuda_status(cudaFree(region));
}

mlra_status mlra_exchange_reset(void* region, size_t bytes, void* stream) {
    if (region == nullptr || bytes == 0) return MLRA_ERR_INVALID_ARG;
    return cuda_status(cudaMemsetAsync(region, 0, bytes, static_cast<cudaStream_t>(stream)));
}

mlra_status mlra_up_proj_allreduce(int32_t batch, int32_t heads, int32_t branches, int32_t d_c, int32_t d_h,
                                   const void* out_lat, const void* w_uv, const void* gate, void* y,
                                   void* const* regions, int32_t world, int32_t rank, int32_t ranks_in_launch,
                                   int32_t* device_status, uint64_t wait_limit_ns, void* stream) {
    if (batch < 1 || heads < 1 || branches < 1 || d_c < 1 || d_h < 1) return MLRA_ERR_INVALID_ARG;
    if (world < 1 || world > kMaxWorld || rank < 0 || ranks_in_launch < 1 || rank + ranks_in_launch > world)
        return MLRA_ERR_INVALID_ARG;
    if (!aligned16(out_lat) || !aligned16(w_uv) || !aligned16(y) || !aligned16(regions))
        return MLRA_ERR_INVALID_ARG;
    if (gate != nullptr && (reinterpret_cast<uintptr_t>(gate) & 1u) != 0) return MLRA_ERR_INVALID_ARG;
    if (device_status != nullptr && (reinterpret_cast<uintptr_t>(device_status) & 3u) != 0)
        return MLRA_ERR_INVALID_ARG;
    if (wait_limit_ns == 0) return MLRA_ERR_INVALID_ARG;
    if ((int64_t)batch * ranks_in_launch * heads * d_h > INT32_MAX) return MLRA_ERR_INVALID_ARG;
    const int K = branches * d_c;
    if (K % 64 != 0 || K > 512 || (d_h != 64 && d_h != 128)) return MLRA_ERR_UNSUPPORTED;
    XRankArgs xr;
    xr.regions = regions;
    xr.world = world;
    xr.rank_base = rank;
    xr.tiles = up_proj_tiles(batch, heads, branches, d_c);
    xr.status = device_status;
    xr.limit_ns = wait_limit_ns;
    const cudaError_t e = launch_up_proj_xrank(batch, heads, branches, d_c, d_h,
                                               static_cast<const __nv_bfloat16*>(out_lat),
                                               static_cast<const __nv_bfloat16*>(w_uv),
                                               static_cast<const __nv_bfloat16*>(gate),
                                               static_cast<__nv_bfloat16*>(y), xr, ranks_in_launch,
                                               static_cast<cudaStream_t>(stream));
    if (e == cudaErrorCooperativeLaunchTooLarge) return MLRA_ERR_UNSUPPORTED;
    return cuda_status(e);
}



mlra_status mlra_copy_ranges(int32_t count, const void* const* src, void* const* dst, const uint64_t* bytes,
                             void* stream) {
    if (count < 1 || count > kMaxRanges || src == nullptr || dst == nullptr || bytes == nullptr)
        return MLRA_ERR_INVALID_ARG;
    CopyRanges r;
    r.count = count;
    for (int k = 0; k < count; ++k) {
        if (!aligned16(src[k]) || !aligned16(dst[k])) return MLRA_ERR_INVALID_ARG;
        const void* s_dev = device_address(src[k]);
        void* d_dev = const_cast<void*>(device_address(dst[k]));
        if (s_dev == nullptr || d_dev == nullptr || !aligned16(s_dev) || !aligned16(d_dev))
            return MLRA_ERR_INVALID_ARG;
        // no overlap between any destination and any range
        r.src[k] = s_dev;
        r.dst[k] = d_dev;
        r.bytes[k] = (size_t)bytes[k];
    }
    for (int a = 0; a < count; ++a)
        for (int c = 0; c < count; ++c) {
            const uintptr_t d0 = reinterpret_cast<uintptr_t>(r.dst[a]), d1 = d0 + r.bytes[a];
            const uintptr_t s0 = reinterpret_cast<uintptr_t>(r.src[c]), s1 = s0 + r.bytes[c];
            const uintptr_t e0 = reinterpret_cast<uintptr_t>(r.dst[c]), e1 = e0 + r.bytes[c];
            if (r.bytes[a] && r.bytes[c] && d0 < s1 && s0 < d1) return MLRA_ERR_INVALID_ARG;
            if (a != c && r.bytes[a] && r.bytes[c] && d0 < e1 && e0 < d1) return MLRA_ERR_INVALID_ARG;
        }
    const int sms = device_sm_count();
    if (sms <= 0) return MLRA_ERR_CUDA;
    return cuda_status(launch_copy_ranges(r, sms, static_cast<cudaStream_t>(stream)));
}

mlra_status mlra_prepare(const mlra_dims* dims, int32_t d_h, const void* q_c, const void* q_r,
                         const void* w_uk, const void* c_new, const void* kr_new,
                         const int32_t* seqlens, const int32_t* block_table, float rope_base,
                         void* q_lat, void* q_rope, void* latent_cache, void* rope_cache,
                         int32_t* device_status, void* stream) {
    mlra_status s = check_dims(dims);
    if (s != MLRA_OK) return s;
    if (d_h < 8 || d_h > 256 || d_h % 8 != 0 || dims->d_c % 8 != 0 || dims->d_r % 2 != 0 ||
        dims->d_r > 64)
        return MLRA_ERR_UNSUPPORTED;
    if (!aligned16(q_c) || !aligned16(w_uk) || !aligned16(c_new) || !aligned16(q_lat) ||
        !aligned16(latent_cache) || !aligned16(q_r) || !aligned16(kr_new) || !aligned16(q_rope) ||
        !aligned16(rope_cache) || !aligned16(seqlens) || !aligned16(block_table))
        return MLRA_ERR_INVALID_ARG;
    if (device_status != nullptr && (reinterpret_cast<uintptr_t>(device_status) & 3u) != 0)
        return MLRA_ERR_INVALID_ARG;
    if (!(rope_base > 1.f) || !(rope_base < 3.0e38f)) return MLRA_ERR_INVALID_ARG;
    PrepareArgs a;
    a.q_c = static_cast<const __nv_bfloat16*>(q_c);
    a.q_r = static_cast<const __nv_bfloat16*>(q_r);
    a.w_uk = static_cast<const __nv_bfloat16*>(w_uk);
    a.c_new = static_cast<const __nv_bfloat16*>(c_new);
    a.kr_new = static_cast<const __nv_bfloat16*>(kr_new);
    a.seqlens = seqlens;
    a.block_table = block_table;
    a.q_lat = static_cast<__nv_bfloat16*>(q_lat);
    a.q_rope = static_cast<__nv_bfloat16*>(q_rope);
    a.latent_cache = static_cast<__nv_bfloat16*>(latent_cache);
    a.rope_cache = static_cast<__nv_bfloat16*>(rope_cache);
    a.status = device_status;
    a.batch = dims->batch;
    a.heads = dims->heads;
    a.branches = dims->branches;
    a.d_c = dims->d_c;
    a.d_r = dims->d_r;
    a.d_h = d_h;
    a.page_size = dims->page_size;
    a.max_pages = dims->max_pages_per_seq;
    a.num_pages = dims->num_pages;
    for (int i = 0; i < 32; ++i)
        a.rope_turns[i] = 2 * i < dims->d_r
                              ? std::pow((double)rope_base, -2.0 * i / dims->d_r) / (2.0 * 3.14159265358979323846)
                              : 0.0;
    return cuda_status(launch_prepare(a, static_cast<cudaStream_t>(stream)));
}

mlra_status mlra_read_device_error(void* workspace, void* stream) {
    if (workspace == nullptr) return MLRA_ERR_INVALID_ARG;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (cudaStreamSynchronize(st) != cudaSuccess) return MLRA_ERR_CUDA;
    int code = 0;
    if (cudaMemcpy(&code, workspace, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess)
        return MLRA_ERR_CUDA;
    // A kernel that gave up on a bounded wait may leave split counters set;
    // they sit at a fixed place for every dims (after the error word), so
    // reporting the timeout also clears them and the workspace is usable again.
    const size_t clear = code == MLRA_ERR_DEVICE_TIMEOUT
                             ? workspace_layout(1, 1, 1, 1, 1).lse_off
                             : (code != 0 ? sizeof(int) : 0);
    if (clear != 0 && cudaMemset(workspace, 0, clear) != cudaSuccess) return MLRA_ERR_CUDA;
    return static_cast<mlra_status>(code);
}

const char* mlra_status_string(mlra_status status) {
    switch (status) {
        case MLRA_OK: return "MLRA_OK";
        case MLRA_ERR_INVALID_ARG: return "MLRA_ERR_INVALID_ARG: invalid argument";
        case MLRA_ERR_UNSUPPORTED: return "MLRA_ERR_UNSUPPORTED: shape not implemented";
        case MLRA_ERR_WORKSPACE: return "MLRA_ERR_WORKSPACE: workspace missing or too small";
        case MLRA_ERR_CUDA: return "MLRA_ERR_CUDA: CUDA call or launch failed";
        case MLRA_ERR_DEVICE_BAD_INDEX: return "MLRA_ERR_DEVICE_BAD_INDEX: block-table entry out of range";
        case MLRA_ERR_DEVICE_BAD_SEQLEN: return "MLRA_ERR_DEVICE_BAD_SEQLEN: sequence length out of range";
        case MLRA_ERR_DEVICE_TIMEOUT: return "MLRA_ERR_DEVICE_TIMEOUT: bounded wait expired in a kernel";
    }
    return "MLRA: unknown status";
}

mlra_status mlra_decode_plan(int32_t batch, int32_t page_size, int32_t max_pages_per_seq,
                             const int32_t* seqlens, int32_t num_ctas, int32_t* plan_out,
                             void* stream) {
    if (batch < 1 || page_size < 1 || max_pages_per_seq < 1 || num_ctas < 1) return MLRA_ERR_INVALID_ARG;
    if (!aligned16(seqlens) || !aligned16(plan_out)) return MLRA_ERR_INVALID_ARG;
    if ((int64_t)max_pages_per_seq * page_size > INT32_MAX) return MLRA_ERR_INVALID_ARG;
    if (!plan_fits_int32(batch, page_size, max_pages_per_seq)) return MLRA_ERR_INVALID_ARG;
    return cuda_status(launch_plan_dump(batch, page_size, max_pages_per_seq, seqlens, num_ctas,
                                        plan_out, static_cast<cudaStream_t>(stream)));
}

}  // extern "C"
