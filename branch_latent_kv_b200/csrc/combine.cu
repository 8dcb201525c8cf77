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
//
// One CTA per (sequence, branch, 32 latent columns); thread (k, q) owns latent
// column k and heads 4q..4q+3, so every split is one independent 16-byte
// load.  The kernel is launched as a programmatic dependent of the decode
// kernel: it works out its sequence's splits from seqlens while the decode
// grid finishes, then waits for it before reading the partials.
#include "common.cuh"
#include "kernels.h"
#include "sm100.cuh"

namespace mlra {
namespace {

constexpr int kThreads = 128;
constexpr int kCols = 32;  // latent columns per CTA

__global__ void __launch_bounds__(kThreads) combine_kernel(DecodeArgs a) {
    extern __shared__ float w_s[];  // [S][HP] weights
    __shared__ int info[3];
    __shared__ int bad_any;
    const int H = a.heads, B = a.branches, d_c = a.d_c, HP = partial_heads(H);
    const int kchunks = ceil_div(d_c, kCols);
    const int kc = blockIdx.x % kchunks, b = (blockIdx.x / kchunks) % B, n = blockIdx.x / (kchunks * B);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int k = kc * kCols + lane;
    sm100::launch_dependents();

    if (tid < 32) {
        const int Ln = __ldg(a.seqlens + n);
        const int tiles = seq_tiles(Ln, a.page_size, a.max_pages);
        int c0 = 0, c1 = -1;
        if (tiles > 0) {
            const int cum = warp_cost_prefix(a.seqlens, n, a.page_size, a.max_pages);
            const int total = cum + warp_cost_prefix(a.seqlens + n, a.batch - n, a.page_size, a.max_pages);
            seq_owners(cum, tiles, plan_chunk(total, a.num_ctas), &c0, &c1);
        }
        if (tid == 0) {
            info[0] = tiles;
            info[1] = c0;
            info[2] = c1 - c0 + 1;
            bad_any = 0;
        }
    }
    __syncthreads();
    const int tiles = info[0], c0 = info[1], S = info[2];
    sm100::wait_prerequisite_grid();  // the decode kernel's partials and outputs are complete
    if (tiles == 0) {  // invalid length: zeros
        if (k < d_c)
            for (int h = warp; h < H; h += kThreads / 32) a.out[(((size_t)n * H + h) * B + b) * d_c + k] = to_bf16(0.f);
        if (tid == 0 && b == 0 && kc == 0) record_error(a.err, MLRA_ERR_DEVICE_BAD_SEQLEN);
        return;
    }
    if (S == 1) return;  // finished by the decode kernel

    // all S x H log-sum-exps in one round of independent loads
    for (int e = tid; e < S * HP; e += kThreads) {
        const int s = e / HP, h = e % HP;
        w_s[e] = h < H ? __ldg(a.lse_part + ((size_t)(c0 + s + n) * B + b) * partial_heads(H) + h) : -INFINITY;
    }
    __syncthreads();
    // weights per head: 2^(lse - max) * out_scale / sum (one warp per head)
    for (int h = warp; h < HP; h += kThreads / 32) {
        if (h >= H) {
            for (int s = lane; s < S; s += 32) w_s[s * HP + h] = 0.f;
            continue;
        }
        float mx = -INFINITY;
        int bad = 0;
        for (int s = lane; s < S; s += 32) {
            const float l = w_s[s * HP + h];
            if (l == bad_split_marker()) bad = 1; else mx = fmaxf(mx, l);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
            bad |= __shfl_xor_sync(0xffffffffu, bad, o);
        }
        float sum = 0.f;
        for (int s = lane; s < S; s += 32) {
            const float w = exp2f(w_s[s * HP + h] - mx);
            w_s[s * HP + h] = w;
            sum += w;
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
        const float norm = a.out_scale / sum;
        for (int s = lane; s < S; s += 32) w_s[s * HP + h] *= norm;
        if (bad && lane == 0) bad_any = 1;
    }
    __syncthreads();
    if (bad_any) {  // a split met a bad block-table entry: zeros
        if (k < d_c)
            for (int h = warp; h < H; h += kThreads / 32) a.out[(((size_t)n * H + h) * B + b) * d_c + k] = to_bf16(0.f);
        if (tid == 0 && kc == 0) record_error(a.err, MLRA_ERR_DEVICE_BAD_INDEX);
        return;
    }
    if (k >= d_c) return;
    const size_t step = (size_t)B * d_c * HP;  // one slot further
    for (int q = warp; q < HP / 4; q += kThreads / 32) {
        const float4* src = reinterpret_cast<const float4*>(
            a.o_part + (((size_t)(c0 + n) * B + b) * d_c + k) * HP + 4 * q);
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 8
        for (int s = 0; s < S; ++s) {
            const float4 v = __ldg(src + s * (step / 4));
            const float4 w = *reinterpret_cast<const float4*>(w_s + s * HP + 4 * q);
            acc.x = fmaf(w.x, v.x, acc.x);
            acc.y = fmaf(w.y, v.y, acc.y);
            acc.z = fmaf(w.z, v.z, acc.z);
            acc.w = fmaf(w.w, v.w, acc.w);
        }
        const float vals[4] = {acc.x, acc.y, acc.z, acc.w};
#pragma unroll
        for (int i = 0; i < 4; ++i)
            if (4 * q + i < H) a.out[(((size_t)n * H + 4 * q + i) * B + b) * d_c + k] = to_bf16(vals[i]);
    }
}

}  // namespace

cudaError_t launch_combine(const DecodeArgs& a, cudaStream_t stream) {
    const size_t smem = sizeof(float) * (size_t)(a.num_ctas + 1) * partial_heads(a.heads);
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(combine_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)a.batch * a.branches * ceil_div(a.d_c, kCols));
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, combine_kernel, a);
}

}  // namespace mlra
