// kernels.h -- internal launch interface between the C ABI (api.cu) and the
// kernel translation units.  Not part of the public ABI.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

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
};

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
    float rope_base;
};

// Query absorption, rotary embedding and the new token's append.
cudaError_t launch_prepare(const PrepareArgs& a, cudaStream_t stream);
size_t prepare_smem_bytes(int d_h);

// Writes the work partition (see mlra_decode_plan in mlra.h).
cudaError_t launch_plan_dump(int batch, int page_size, int max_pages, const int32_t* seqlens,
                             int num_ctas, int32_t* plan_out, cudaStream_t stream);

}  // namespace mlra
