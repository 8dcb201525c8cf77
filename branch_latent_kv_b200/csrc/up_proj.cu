// up_proj.cu -- per-branch W_UV up-projection and branch sum.
//
//   y[n, h*d_h + j] = sum_b sum_k out_lat[n,h,b,k] * w_uv[b][k][h*d_h + j]
//
// ("The Core Insight" section of the wispaper.ai MLRA blog page: every
// branch is up-projected by its own matrix and the branch outputs are summed
// at the end.)  The branch sum is the K reduction over K = branches * d_c.
// One CTA per (head, group of 8 sequences); thread j owns output column j,
// so the W_UV reads of a warp are contiguous.
#include "common.cuh"
#include "kernels.h"

namespace mlra {
namespace {

constexpr int kSeqPerCta = 8;

__global__ void up_proj_simt_kernel(int batch, int heads, int K, int d_h,
                                    const __nv_bfloat16* __restrict__ out_lat,
                                    const __nv_bfloat16* __restrict__ w_uv,
                                    __nv_bfloat16* __restrict__ y) {
    extern __shared__ float ol[];  // [kSeqPerCta][K]
    const int h = blockIdx.x, n0 = blockIdx.y * kSeqPerCta, j = threadIdx.x;
    for (int i = threadIdx.x; i < kSeqPerCta * K; i += blockDim.x) {
        const int nn = i / K, kk = i % K, n = n0 + nn;
        ol[i] = n < batch ? __bfloat162float(out_lat[((size_t)n * heads + h) * K + kk]) : 0.f;
    }
    __syncthreads();
    float acc[kSeqPerCta];
#pragma unroll
    for (int nn = 0; nn < kSeqPerCta; ++nn) acc[nn] = 0.f;
    const size_t width = (size_t)heads * d_h;
    for (int kk = 0; kk < K; ++kk) {
        const float w = __bfloat162float(w_uv[kk * width + (size_t)h * d_h + j]);
#pragma unroll
        for (int nn = 0; nn < kSeqPerCta; ++nn) acc[nn] = fmaf(ol[nn * K + kk], w, acc[nn]);
    }
#pragma unroll
    for (int nn = 0; nn < kSeqPerCta; ++nn) {
        const int n = n0 + nn;
        if (n < batch) y[(size_t)n * width + (size_t)h * d_h + j] = to_bf16(acc[nn]);
    }
}

}  // namespace

cudaError_t launch_up_proj(int batch, int heads, int branches, int d_c, int d_h,
                           const __nv_bfloat16* out_lat, const __nv_bfloat16* w_uv,
                           __nv_bfloat16* y, cudaStream_t stream) {
    const int K = branches * d_c;
    dim3 grid(heads, ceil_div(batch, kSeqPerCta));
    up_proj_simt_kernel<<<grid, d_h, sizeof(float) * kSeqPerCta * K, stream>>>(batch, heads, K, d_h,
                                                                             out_lat, w_uv, y);
    return cudaGetLastError();
}

}  // namespace mlra
