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
//   split counters  int32 [kMaxBatch + 1]              (fixed place)
//   lse partials    fp32 [slots][branches][HP]         (log2 domain; HP = the
//                   head count rounded up to whole head tiles: 16 up to 16
//                   heads, else a multiple of 32)
//   o partials      fp32 [slots][branches][d_c][HP]    (normalised per split;
//                   heads innermost)
// slots = num_ctas + batch: the partial of CTA c for sequence n lives in slot
// c + n (unique because CTA ranges are contiguous and ordered).  The
// tensor-core kernel writes rows of one head tile (T = 16 or 32 heads): with
// G = HP / T head groups, group g owns the G-th part of the bytes, cpg + batch
// slots of T-wide rows (cpg = num_ctas / G), and split counters
// [g batch, (g + 1) batch).
// ---------------------------------------------------------------------------
struct WorkspaceLayout {
    size_t err_off, lse_off, o_off, cnt_off, total;
    int slots;
};

__host__ __device__ inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// Largest batch the library accepts (int32 sequence ids, 16-bit grid rows).
constexpr int kMaxBatch = 65535;

// Heads the tensor-core kernel takes: one tile of 16 heads (its MMA's N), or
// tiles of 32 heads when there are more and a branch is at least 128 wide
// (narrower branches put two in a step, and a softmax thread's registers hold
// 16 heads of one branch or 8 heads of two); at most 128 heads.
constexpr int kMaxTcHeads = 128;
__host__ __device__ inline int tc_head_tile(int heads, int d_c) { return heads <= 16 || d_c < 128 ? 16 : 32; }
__host__ __device__ inline int tc_head_groups(int heads, int d_c) {
    return (heads + tc_head_tile(heads, d_c) - 1) / tc_head_tile(heads, d_c);
}

__host__ __device__ inline WorkspaceLayout workspace_layout(int batch, int heads, int branches,
                                                            int d_c, int num_ctas) {
    WorkspaceLayout w;
    w.slots = num_ctas + batch;
    w.err_off = 0;
    // per-sequence split counters of the tensor-core kernel's merge, at a
    // fixed place sized for the largest batch: calls with other dimensions
    // that reuse the workspace find them where they left them (at zero)
    w.cnt_off = 256;
    w.lse_off = align256(w.cnt_off + sizeof(int) * (size_t)(kMaxBatch + 1));
    const size_t hp = (size_t)tc_head_tile(heads, d_c) * tc_head_groups(heads, d_c);  // heads padded to whole tiles
    w.o_off = align256(w.lse_off + sizeof(float) * (size_t)w.slots * branches * hp);
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
// L_n is invalid.  Work is counted in cost units: a tile costs kTileCost, and
// every sequence adds kSeqCost after its last tile for the per-segment work
// (query load, first-tile setup, epilogue) that a CTA pays each time its range
// enters a new sequence.  Sequence n occupies the cost interval
// [cum_n, cum_n + cost_n), cost_n = kTileCost * tiles_n + kSeqCost, and its
// tile t starts at cum_n + kTileCost * t.  With
//   chunk = kTileCost * max(ceil(total_cost / (num_ctas * kTileCost)), 1)
// CTA c owns the tiles whose start lies in [c * chunk, (c + 1) * chunk): a
// whole number of tiles per window, so no CTA holds more than
// ceil(total_cost / (num_ctas * kTileCost)) tiles (the slowest CTA bounds the
// kernel).  kSeqCost is half a tile: a range that crosses into another
// sequence reloads queries and pays a second epilogue, which the other CTAs'
// pipelines absorb but its own does not entirely.
// Ranges are contiguous in the tile list, and because chunk >= kTileCost
// every CTA between the first and the last owner of a sequence owns at least
// one of its tiles.  Every kernel recomputes this from seqlens with the warp
// routines below (no plan buffer).
// ---------------------------------------------------------------------------
constexpr int kTileCost = 8;
constexpr int kSeqCost = 4;

__device__ __forceinline__ bool seqlen_valid(int L, int page_size, int max_pages) {
    return L >= 1 && (long long)L <= (long long)max_pages * page_size;
}

__device__ __forceinline__ int seq_tiles(int L, int page_size, int max_pages) {
    return seqlen_valid(L, page_size, max_pages) ? (L + kTileTokens - 1) / kTileTokens : 0;
}

__device__ __forceinline__ int seq_cost(int L, int page_size, int max_pages) {
    const int t = seq_tiles(L, page_size, max_pages);
    return t > 0 ? t * kTileCost + kSeqCost : 0;
}

__host__ __device__ __forceinline__ int plan_chunk(int total_cost, int num_ctas) {
    const long long per = ((long long)total_cost + (long long)num_ctas * kTileCost - 1) /
                          ((long long)num_ctas * kTileCost);
    return kTileCost * (per > 1 ? (int)per : 1);
}

// First tile of a sequence (cost start cum, `tiles` tiles) that starts at or
// after position A; `tiles` if none does.
__device__ __forceinline__ int first_tile_at(int cum, int tiles, int A) {
    if (A <= cum) return 0;
    const int t = (A - cum + kTileCost - 1) / kTileCost;
    return t < tiles ? t : tiles;
}

// Whole warp: sum of the costs of sequences [0, n).
__device__ inline int warp_cost_prefix(const int32_t* seqlens, int n, int P, int max_pages) {
    const int lane = threadIdx.x & 31;
    int sum = 0;
    for (int m = lane; m < n; m += 32) sum += seq_cost(__ldg(seqlens + m), P, max_pages);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
    return sum;
}

// Whole warp: the first sequence with a tile starting at or after position A,
// and its cost start (batch and the total cost if there is none).
__device__ inline void warp_find_seq(const int32_t* seqlens, int batch, int P, int max_pages,
                                     int A, int* seq_out, int* cum_out) {
    const int lane = threadIdx.x & 31;
    int base_cum = 0;
    for (int base = 0; base < batch; base += 32) {
        const int n = base + lane;
        const int c = n < batch ? seq_cost(__ldg(seqlens + n), P, max_pages) : 0;
        int incl = c;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int v = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += v;
        }
        const int excl = incl - c;
        // last tile start = cum + cost - kSeqCost - kTileCost
        const unsigned hit = __ballot_sync(0xffffffffu,
                                           c > 0 && base_cum + incl - kSeqCost - kTileCost >= A);
        if (hit) {
            const int src = __ffs(hit) - 1;
            *seq_out = base + src;
            *cum_out = __shfl_sync(0xffffffffu, base_cum + excl, src);
            return;
        }
        base_cum += __shfl_sync(0xffffffffu, incl, 31);
    }
    *seq_out = batch;
    *cum_out = base_cum;
}

// The plan's cost positions are int32: the largest possible total must fit.
inline bool plan_fits_int32(long long batch, long long page_size, long long max_pages) {
    const long long tiles_per_seq = (max_pages * page_size + kTileTokens - 1) / kTileTokens;
    return batch * (tiles_per_seq * kTileCost + kSeqCost) <= (1LL << 30);
}

// CTAs owning the first and the last tile of a sequence (tiles > 0).
__device__ __forceinline__ void seq_owners(int cum, int tiles, int chunk, int* c0, int* c1) {
    *c0 = cum / chunk;
    *c1 = (cum + (tiles - 1) * kTileCost) / chunk;
}

__host__ __device__ __forceinline__ int ceil_div(int a, int b) { return (a + b - 1) / b; }

// Round-to-nearest-even fp32 -> bf16 (the cuda_bf16 conversion is RNE).
__device__ __forceinline__ __nv_bfloat16 to_bf16(float x) { return __float2bfloat16_rn(x); }

}  // namespace mlra
