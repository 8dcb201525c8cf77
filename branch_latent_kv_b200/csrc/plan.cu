// plan.cu -- writes the split-KV work partition that the decode and combine
// kernels recompute internally, so that tests can check it bit for bit.
#include "common.cuh"
#include "kernels.h"

namespace mlra {
namespace {

__global__ void __launch_bounds__(32) plan_dump_kernel(const int32_t* seqlens, int batch, int P,
                                                       int max_pages, int num_ctas, int32_t* plan) {
    const int lane = threadIdx.x;
    const int total = warp_total_tiles(seqlens, batch, P, max_pages);
    const int chunk = total > 0 ? ceil_div(total, num_ctas) : 0;
    for (int c = 0; c < num_ctas; ++c) {
        const int g0 = c * chunk, g1 = min(g0 + chunk, total);
        int n0 = -1, n1 = -1, f;
        if (g0 < g1) {
            warp_find_seq(seqlens, batch, P, max_pages, g0, &n0, &f);
            warp_find_seq(seqlens, batch, P, max_pages, g1 - 1, &n1, &f);
        }
        if (lane == 0) {
            plan[c * 4 + 0] = min(g0, total);
            plan[c * 4 + 1] = max(g1, min(g0, total));
            plan[c * 4 + 2] = n0;
            plan[c * 4 + 3] = n1;
        }
    }
    for (int n = 0; n < batch; ++n) {
        const int tiles = seq_tiles(__ldg(seqlens + n), P, max_pages);
        const int first = warp_seq_first_tile(seqlens, n, P, max_pages);
        if (lane == 0) {
            int32_t* s = plan + num_ctas * 4 + n * 2;
            if (tiles == 0) {
                s[0] = 0;
                s[1] = -1;
            } else {
                s[0] = (first + tiles - 1) / chunk - first / chunk + 1;
                s[1] = first / chunk;
            }
        }
    }
}

}  // namespace

cudaError_t launch_plan_dump(int batch, int page_size, int max_pages, const int32_t* seqlens,
                             int num_ctas, int32_t* plan_out, cudaStream_t stream) {
    plan_dump_kernel<<<1, 32, 0, stream>>>(seqlens, batch, page_size, max_pages, num_ctas, plan_out);
    return cudaGetLastError();
}

}  // namespace mlra
