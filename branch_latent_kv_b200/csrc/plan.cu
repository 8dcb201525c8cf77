// plan.cu -- writes the split-KV work partition that the decode and combine
// kernels recompute internally, so that tests can check it bit for bit.
#include "common.cuh"
#include "kernels.h"

namespace mlra {
namespace {

// One thread walks the sequences; per sequence only its owner CTAs are
// visited, so the walk is O(batch + num_ctas).
__global__ void __launch_bounds__(32) plan_dump_kernel(const int32_t* seqlens, int batch, int P,
                                                       int max_pages, int num_ctas, int32_t* plan) {
    if (threadIdx.x != 0) return;
    int total = 0;
    for (int n = 0; n < batch; ++n) total += seq_cost(seqlens[n], P, max_pages);
    const int chunk = plan_chunk(total, num_ctas);
    for (int c = 0; c < num_ctas; ++c) {
        plan[c * 4 + 0] = 0;
        plan[c * 4 + 1] = 0;
        plan[c * 4 + 2] = -1;
        plan[c * 4 + 3] = -1;
    }
    int cum = 0, g = 0;
    for (int n = 0; n < batch; ++n) {
        const int L = seqlens[n];
        const int tiles = seq_tiles(L, P, max_pages);
        int32_t* s = plan + num_ctas * 4 + n * 2;
        if (tiles == 0) {
            s[0] = 0;
            s[1] = -1;
            continue;
        }
        int c0, c1;
        seq_owners(cum, tiles, chunk, &c0, &c1);
        s[0] = c1 - c0 + 1;
        s[1] = c0;
        for (int c = c0; c <= c1; ++c) {
            const int tb = first_tile_at(cum, tiles, c * chunk);
            const int te = first_tile_at(cum, tiles, (c + 1) * chunk);
            int32_t* p = plan + c * 4;
            if (p[2] < 0) {
                p[0] = g + tb;
                p[2] = n;
            }
            p[1] = g + te;
            p[3] = n;
        }
        cum += seq_cost(L, P, max_pages);
        g += tiles;
    }
}

}  // namespace

cudaError_t launch_plan_dump(int batch, int page_size, int max_pages, const int32_t* seqlens,
                             int num_ctas, int32_t* plan_out, cudaStream_t stream) {
    plan_dump_kernel<<<1, 32, 0, stream>>>(seqlens, batch, page_size, max_pages, num_ctas, plan_out);
    return cudaGetLastError();
}

}  // namespace mlra
