// combine.cu -- cross-split log-sum-exp merge, output scale and bf16 cast.
//
// A sequence cut into S > 1 splits has, per (branch, head), S normalised
// partial outputs o_s and base-2 log-sum-exps lse_s.  The full softmax output
// is o = sum_s w_s o_s / sum_s w_s with w_s = 2^(lse_s - max_s lse_s); the
// variance-calibration factor ("Mathematical Calibration: Scaling the
// Latents" section of the wispaper.ai MLRA blog page) multiplies the result
// before the bf16 cast.  Sequences with an invalid length get zeros and an
// error code; sequences a single CTA covered were finished by the decode
// kernel and are skipped.
#include "common.cuh"
#include "kernels.h"

namespace mlra {
namespace {

constexpr int kWarps = 4;

__global__ void __launch_bounds__(kWarps * 32) combine_kernel(DecodeArgs a) {
    const int n = blockIdx.x;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int H = a.heads, B = a.branches, d_c = a.d_c;
    const int pair = blockIdx.y * kWarps + warp;  // (b, h) with h fastest
    if (pair >= B * H) return;                    // warp-uniform
    const int b = pair / H, h = pair % H;
    __nv_bfloat16* out = a.out + (((size_t)n * H + h) * B + b) * d_c;

    const int Ln = __ldg(a.seqlens + n);
    const int tiles = seq_tiles(Ln, a.page_size, a.max_pages);
    if (tiles == 0) {
        for (int k = lane; k < d_c; k += 32) out[k] = to_bf16(0.f);
        if (pair == 0 && lane == 0) record_error(a.err, MLRA_ERR_DEVICE_BAD_SEQLEN);
        return;
    }
    const int total = warp_total_tiles(a.seqlens, a.batch, a.page_size, a.max_pages);
    const int chunk = ceil_div(total, a.num_ctas);
    const int first = warp_seq_first_tile(a.seqlens, n, a.page_size, a.max_pages);
    const int c0 = first / chunk, c1 = (first + tiles - 1) / chunk;
    if (c0 == c1) return;

    // max over splits (each lane takes every 32nd split, then a warp max)
    float mx = -INFINITY;
    int bad = 0;
    for (int c = c0 + lane; c <= c1; c += 32) {
        const float l = __ldg(a.lse_part + ((size_t)(c + n) * B + b) * H + h);
        if (l == bad_split_marker()) bad = 1; else mx = fmaxf(mx, l);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        bad |= __shfl_xor_sync(0xffffffffu, bad, o);
    }
    if (bad) {
        for (int k = lane; k < d_c; k += 32) out[k] = to_bf16(0.f);
        if (lane == 0) record_error(a.err, MLRA_ERR_DEVICE_BAD_INDEX);
        return;
    }
    float wsum = 0.f;
    for (int c = c0 + lane; c <= c1; c += 32)
        wsum += exp2f(__ldg(a.lse_part + ((size_t)(c + n) * B + b) * H + h) - mx);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) wsum += __shfl_xor_sync(0xffffffffu, wsum, o);
    const float norm = a.out_scale / wsum;

    for (int k = lane; k < d_c; k += 32) {
        float acc = 0.f;
        for (int c = c0; c <= c1; ++c) {
            const size_t slot = (size_t)c + n;
            const float w = exp2f(__ldg(a.lse_part + (slot * B + b) * H + h) - mx);
            acc = fmaf(w, __ldg(a.o_part + ((slot * B + b) * H + h) * d_c + k), acc);
        }
        out[k] = to_bf16(acc * norm);
    }
}

}  // namespace

cudaError_t launch_combine(const DecodeArgs& a, cudaStream_t stream) {
    dim3 grid(a.batch, ceil_div(a.branches * a.heads, kWarps));
    combine_kernel<<<grid, kWarps * 32, 0, stream>>>(a);
    return cudaGetLastError();
}

}  // namespace mlra
