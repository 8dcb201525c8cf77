// common.cuh -- pieces shared by the MLRA kernels: the split-KV plan, the
// workspace layout, error recording and small numeric helpers.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "mlra.h"

namespace mlra {

// Tokens per work tile.  The tensor-core kernel puts one tile on the M = 128
// rows of its score MMA; the plan, the partials and the combine use the same
// unit so that every kernel agrees on the work partition.
constexpr int kTileTokens = 128;

// log2(e): scores are kept in the base-2 domain so that exp becomes exp2.
constexpr float kLog2e = 1.4426950408889634f;

// ---------------------------------------------------------------------------
// Workspace layout (byte offsets, each region 256-byte aligned):
//   [0, 256)        int32 error word (first device-side error code, else 0)
//   lse partials    fp32 [slots][branches][heads]      (log2 domain)
//   o partials      fp32 [slots][branches][d_c][16]    (normalised per split;
//                   heads innermost, padded to 16: one 64-byte row per column)
// slots = num_ctas + batch: the partial of CTA c for sequence n lives in slot
// c + n (unique because CTA ranges are contiguous and ordered).
// ---------------------------------------------------------------------------
struct WorkspaceLayout {
    size_t err_off, lse_off, o_off, total;
    int slots;
};

__host__ __device__ inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

__host__ __device__ inline WorkspaceLayout workspace_layout(int batch, int heads, int branches,
                                                            int d_c, int num_ctas) {
    WorkspaceLayout w;
    w.slots = num_ctas + batch;
    w.err_off = 0;
    w.lse_off = 256;
    w.o_off = align256(w.lse_off + sizeof(float) * (size_t)w.slots * branches * heads);
    const size_t hp = heads <= 16 ? 16 : (size_t)heads;  // heads padded to 16 (more for the CUDA-core kernel)
    w.total = align256(w.o_off + sizeof(float) * (size_t)w.slots * branches * d_c * hp);
    return w;
}

// Heads per partial row: 16 (or H when H > 16).
__host__ __device__ inline int partial_heads(int heads) { return heads <= 16 ? 16 : heads; }

// Marker stored in a partial's lse when the split met a bad block-table entry.
__device__ __forceinline__ float bad_split_marker() { return __int_as_float(0x7f800000); }  // +inf

__device__ __forceinline__ void record_error(int* err, int code) {
    atomicCAS(err, 0, code);
}

// ---------------------------------------------------------------------------
// Split-KV plan.  Sequence n owns tiles_n = ceil(L_n / 128) tiles, or none if
// L_n is invalid.  The concatenated tile list is cut into num_ctas contiguous
// ranges of chunk = ceil(total / num_ctas) tiles.  Every kernel recomputes
// this from seqlens with the warp routines below (no plan buffer).
// ---------------------------------------------------------------------------
__device__ __forceinline__ bool seqlen_valid(int L, int page_size, int max_pages) {
    return L >= 1 && (long long)L <= (long long)max_pages * page_size;
}

__device__ __forceinline__ int seq_tiles(int L, int page_size, int max_pages) {
    return seqlen_valid(L, page_size, max_pages) ? (L + kTileTokens - 1) / kTileTokens : 0;
}

// Whole warp: total number of tiles.
__device__ inline int warp_total_tiles(const int32_t* seqlens, int batch, int P, int max_pages) {
    const int lane = threadIdx.x & 31;
    int sum = 0;
    for (int n = lane; n < batch; n += 32) sum += seq_tiles(__ldg(seqlens + n), P, max_pages);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
    return sum;
}

// Whole warp: first global tile of sequence n (sum of tiles of sequences < n).
__device__ inline int warp_seq_first_tile(const int32_t* seqlens, int n, int P, int max_pages) {
    const int lane = threadIdx.x & 31;
    int sum = 0;
    for (int m = lane; m < n; m += 32) sum += seq_tiles(__ldg(seqlens + m), P, max_pages);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
    return sum;
}

// Whole warp: the sequence whose tile range contains global tile g (g < total)
// and that sequence's first global tile.
__device__ inline void warp_find_seq(const int32_t* seqlens, int batch, int P, int max_pages,
                                     int g, int* seq_out, int* first_out) {
    const int lane = threadIdx.x & 31;
    int base_cum = 0;
    for (int base = 0; base < batch; base += 32) {
        const int n = base + lane;
        const int t = n < batch ? seq_tiles(__ldg(seqlens + n), P, max_pages) : 0;
        int incl = t;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int v = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += v;
        }
        const int excl = incl - t;
        const unsigned hit = __ballot_sync(0xffffffffu, t > 0 && base_cum + excl <= g &&
                                                            g < base_cum + incl);
        if (hit) {
            const int src = __ffs(hit) - 1;
            *seq_out = base + src;
            *first_out = __shfl_sync(0xffffffffu, base_cum + excl, src);
            return;
        }
        base_cum += __shfl_sync(0xffffffffu, incl, 31);
    }
    *seq_out = -1;
    *first_out = base_cum;
}

__host__ __device__ __forceinline__ int ceil_div(int a, int b) { return (a + b - 1) / b; }

// Round-to-nearest-even fp32 -> bf16 (the cuda_bf16 conversion is RNE).
__device__ __forceinline__ __nv_bfloat16 to_bf16(float x) { return __float2bfloat16_rn(x); }

}  // namespace mlra
