// kernels.h -- internal launch interface between the C ABI (api.cu) and the
// kernel translation units.  Not part of the public ABI.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "mlra.h"

namespace mlra {

// Arguments of the decode kernels (everything already validated on the host).
struct DecodeArgs {
    const __nv_bfloat16* q_lat;   // [N, H, B, d_c]
    const __nv_bfloat16* q_rope;  // [N, H, d_r]
    const __nv_bfloat16* latent;  // [pages, P, B, d_c]
    const __nv_bfloat16* rope;    // [pages, P, d_r]
    const int32_t* block_table;   // [N, max_pages]
    const int32_t* seqlens;       // [N]
    __nv_bfloat16* out;           // [N, H, B, d_c]
    float* lse_part;              // [slots, B, H]        log2 domain
    float* o_part;                // [slots, B, d_c, HP]   HP = partial_heads(H)
    int* err;                     // device error word
    int* seq_cnt;                 // [N] split counters of the in-kernel merge (zero between calls)
    int batch, heads, branches, d_c, d_r, page_size, max_pages, num_pages;
    int num_ctas;                 // grid of the split kernel (partial slots = num_ctas + batch)
    float scale_log2;             // scale * log2(e)
    float out_scale;
    // the fused step (mlra_decode_up_proj): after the merges the same launch
    // up-projects the latent output; w_uv null: no up-projection
    const __nv_bfloat16* w_uv;    // [B, d_c, H * d_h]
    __nv_bfloat16* y;             // [N, H * d_h] (device address)
    int d_h;
};

// Host validation of a tensor-core decode call (what mlra_decode checks);
// fills the kernel arguments.  Defined in api.cu.
mlra_status decode_tc_args(const mlra_dims* dims, const void* q_lat, const void* q_rope,
                           const void* latent_cache, const void* rope_cache, const int32_t* block_table,
                           const int32_t* seqlens, float scale, float out_scale, void* out, void* workspace,
                           size_t workspace_bytes, DecodeArgs* a);

// Largest batch of the fused decode + up-projection (its latent rows of one
// head for every sequence are staged in shared memory).
constexpr int kUpProjFusedMaxBatch = 64;

// Split-KV decode on CUDA cores (fp32 FMA).  Writes final outputs of
// single-split sequences and partials of the others.
cudaError_t launch_decode_simt(const DecodeArgs& a, cudaStream_t stream);

// Split-KV decode on the tensor cores (tcgen05 + TMA); see decode_tc.cu.
bool decode_tc_supported(int branches, int d_c, int d_r, int heads);
cudaError_t launch_decode_tc(const DecodeArgs& a, cudaStream_t stream);
size_t decode_simt_smem_bytes(int heads, int branches, int d_c, int d_r);

// Log-sum-exp merge of the partials, out_scale, bf16 cast; zeros and an error
// code for invalid sequences.
cudaError_t launch_combine(const DecodeArgs& a, cudaStream_t stream);

// y = per-branch W_UV up-projection summed over branches, times
// sigmoid(gate) elementwise when gate is not null.
cudaError_t launch_up_proj(int batch, int heads, int branches, int d_c, int d_h,
                           const __nv_bfloat16* out_lat, const __nv_bfloat16* w_uv,
                           const __nv_bfloat16* gate, __nv_bfloat16* y, cudaStream_t stream);

// ---------------------------------------------------------------------------
// Cross-rank branch sum of the branch-sharded up-projection.  Every rank owns
// one exchange region (device memory that every other rank can address):
//   epoch [tiles]                        u32  calls completed, per output tile
//   data  [2][world][batch][heads*d_h]   u64  rank src's fp32 partial in the
//                                             low half, call + 1 in the high half
// A partial and its call tag travel in one 64-bit store, so a reader that
// sees the tag also sees the value: no flags and no fences.  par = call & 1
// double-buffers the data, so a rank that runs ahead into the next call never
// overwrites a value that a slower rank has not yet read.
constexpr int kMaxWorld = 8;

struct ExchangeLayout {
    size_t epoch_off, data_off, total;
};

__host__ __device__ inline ExchangeLayout exchange_layout(int batch, int heads, int d_h, int world, int tiles) {
    ExchangeLayout L;
    L.epoch_off = 0;
    L.data_off = ((size_t)tiles * 4 + 255) & ~size_t(255);
    L.total = L.data_off + (((size_t)2 * world * batch * heads * d_h * 8 + 255) & ~size_t(255));
    return L;
}

struct XRankArgs {
    void* const* regions;  // device array [world]: every rank's exchange region
    int world;             // ranks in the sum (0: no cross-rank sum)
    int rank_base;         // rank computed by blockIdx.z == 0
    int tiles;             // output tiles (CTAs) of one rank's grid
    int* status;           // optional device error word
    unsigned long long limit_ns;  // bound on the wait for the other ranks
};

// Output tiles (CTAs per rank) of the up-projection grid for these sizes.
int up_proj_tiles(int batch, int heads, int branches, int d_c);

// The branch-sharded up-projection: each rank multiplies its own branches,
// then the ranks' fp32 partial sums are exchanged through the regions and
// added in rank order.  ranks_in_launch > 1 runs ranks rank_base ..
// rank_base + ranks_in_launch - 1 in one launch on one device, with their
// out_lat, w_uv and y stacked along the leading dimension.
cudaError_t launch_up_proj_xrank(int batch, int heads, int branches, int d_c, int d_h,
                                 const __nv_bfloat16* out_lat, const __nv_bfloat16* w_uv,
                                 const __nv_bfloat16* gate, __nv_bfloat16* y, const XRankArgs& xr,
                                 int ranks_in_launch, cudaStream_t stream);

// Byte ranges copied by one launch of the SMs (device or mapped pinned host
// memory, 16-byte aligned, validated on the host).
constexpr int kMaxRanges = 8;
struct CopyRanges {
    const void* src[kMaxRanges];
    void* dst[kMaxRanges];
    size_t bytes[kMaxRanges];
    int count;
};
cudaError_t launch_copy_ranges(const CopyRanges& r, int sms, cudaStream_t stream);

// Arguments of the decode pre-step (validated on the host).
struct PrepareArgs {
    const __nv_bfloat16* q_c;     // [N, H, d_h]
    const __nv_bfloat16* q_r;     // [N, H, d_r] unrotated
    const __nv_bfloat16* w_uk;    // [B, H, d_h, d_c]
    const __nv_bfloat16* c_new;   // [N, B, d_c]
    const __nv_bfloat16* kr_new;  // [N, d_r] unrotated
    const int32_t* seqlens;       // [N] lengths including the new token
    const int32_t* block_table;   // [N, max_pages]
    __nv_bfloat16* q_lat;         // [N, H, B, d_c] written
    __nv_bfloat16* q_rope;        // [N, H, d_r] written (rotated)
    __nv_bfloat16* latent_cache;  // [pages, P, B, d_c] one row per sequence written
    __nv_bfloat16* rope_cache;    // [pages, P, d_r] one row per sequence written
    int* status;                  // optional device error word
    int batch, heads, branches, d_c, d_r, d_h, page_size, max_pages, num_pages;
    // RoPE pair i turns by rope_turns[i] * p full turns at position p:
    // rope_base^(-2i/d_r) / (2 pi), formed on the host in fp64
    double rope_turns[32];
};

// Query absorption, rotary embedding and the new token's append.
cudaError_t launch_prepare(const PrepareArgs& a, cudaStream_t stream);
size_t prepare_smem_bytes(int d_h);

// Writes the work partition (see mlra_decode_plan in mlra.h).
cudaError_t launch_plan_dump(int batch, int page_size, int max_pages, const int32_t* seqlens,
                             int num_ctas, int32_t* plan_out, cudaStream_t stream);

}  // namespace mlra
