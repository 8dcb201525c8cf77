// prepare.cu -- the decode pre-step: query absorption, rotary embedding of
// the RoPE query and the new token's RoPE key, and the new token's append to
// the paged cache.
//
//   q_lat[n,h,b,k] = sum_j w_uk[b,h,j,k] * q_c[n,h,j]
//     (the key up-projection of branch b, head h folded into the query: only
//     latents are cached -- the TransMLA thread on Hacker News -- and every
//     branch has its own up-projection -- "The Core Insight" section of the
//     wispaper.ai MLRA blog page)
//   rotary embedding at the new token's position p = seqlens[n] - 1, as
//   RoFormer defines it: pair i of a vector turns by p * base^(-2i/d_r)
//   latent_cache[page][slot] = c_new[n], rope_cache[page][slot] = rotated key
//     page = block_table[n][p / P], slot = p mod P
//
// One launch, two kinds of CTA.  Absorption CTAs own (head, branch, 64
// latent columns): the 64 columns of W_UK for that head and branch
// (d_h x 64 bf16) stay in shared memory while 64-sequence chunks of q_c
// stream through; each thread forms dot products over d_h in fp32.  The
// contraction is tiny (N x d_h per output) and its weights (2 MiB at the
// 2.9B shape) are read once, so it is bound by memory and latency, not by
// tensor-core throughput.  Append CTAs take one sequence per warp: lane i
// owns RoPE pair i (angles in fp64, so positions up to 2^31 keep their
// phase), rotates that pair of every head's query and of the new key, and
// the warp copies the new latents in 16-byte units.
#include "common.cuh"
#include "kernels.h"

namespace mlra {
namespace {

constexpr int kPrepThreads = 256;
constexpr int kColBlock = 64;   // latent columns per absorption CTA
constexpr int kSeqChunk = 64;   // sequences per q_c chunk
constexpr int kSeqPerAppendCta = kPrepThreads / 32;

__global__ void __launch_bounds__(kPrepThreads)
prepare_kernel(const PrepareArgs a, int n_abs_ctas) {
    extern __shared__ uint4 prep_smem[];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int H = a.heads, B = a.branches, d_c = a.d_c, d_h = a.d_h;

    if ((int)blockIdx.x < n_abs_ctas) {
        // ------------------------------------------------------------ absorption
        const int kblocks = (d_c + kColBlock - 1) / kColBlock;
        const int hb = blockIdx.x / kblocks, kb = blockIdx.x % kblocks;
        const int h = hb / B, b = hb % B;
        const int k0 = kb * kColBlock, kw = min(kColBlock, d_c - k0);  // kw: a multiple of 8
        __nv_bfloat16* w_s = reinterpret_cast<__nv_bfloat16*>(prep_smem);   // [d_h][64]
        __nv_bfloat16* q_s = w_s + d_h * kColBlock;                          // [64][d_h]
        const int kv = kw / 8;  // 16-byte units per W row
        for (int e = tid; e < d_h * kv; e += kPrepThreads) {
            const int j = e / kv, u = e % kv;
            reinterpret_cast<uint4*>(w_s + j * kColBlock)[u] =
                __ldg(reinterpret_cast<const uint4*>(a.w_uk + (((size_t)b * H + h) * d_h + j) * d_c + k0) + u);
        }
        // thread: latent column pair kp (columns 2kp, 2kp+1 of the block) and
        // sequence group ng; each pass takes two sequences (nn, nn + 8) so
        // every W pair read from shared memory feeds 8 FMAs
        const int kp = tid & 31, ng = tid >> 5;  // ng < 8
        const int qv = d_h / 8;
        for (int n0 = 0; n0 < a.batch; n0 += kSeqChunk) {
            const int nc = min(kSeqChunk, a.batch - n0);
            __syncthreads();  // W is staged; the previous chunk's q_s is no longer read
            for (int e = tid; e < nc * qv; e += kPrepThreads) {
                const int nn = e / qv, u = e % qv;
                reinterpret_cast<uint4*>(q_s + nn * d_h)[u] =
                    __ldg(reinterpret_cast<const uint4*>(a.q_c + ((size_t)(n0 + nn) * H + h) * d_h) + u);
            }
            __syncthreads();
            if (2 * kp < kw) {
                for (int nn = ng; nn < nc; nn += 16) {
                    const bool two = nn + 8 < nc;
                    const __nv_bfloat162* q0 = reinterpret_cast<const __nv_bfloat162*>(q_s + nn * d_h);
                    const __nv_bfloat162* q1 = reinterpret_cast<const __nv_bfloat162*>(q_s + (two ? nn + 8 : nn) * d_h);
                    float a00 = 0.f, a01 = 0.f, a10 = 0.f, a11 = 0.f;  // [sequence][column]
#pragma unroll 4
                    for (int j = 0; j < d_h; j += 2) {
                        const float2 w0 = __bfloat1622float2(reinterpret_cast<const __nv_bfloat162*>(w_s + j * kColBlock)[kp]);
                        const float2 w1 = __bfloat1622float2(reinterpret_cast<const __nv_bfloat162*>(w_s + (j + 1) * kColBlock)[kp]);
                        const float2 x0 = __bfloat1622float2(q0[j / 2]);
                        const float2 x1 = __bfloat1622float2(q1[j / 2]);
                        a00 = fmaf(w0.x, x0.x, fmaf(w1.x, x0.y, a00));
                        a01 = fmaf(w0.y, x0.x, fmaf(w1.y, x0.y, a01));
                        a10 = fmaf(w0.x, x1.x, fmaf(w1.x, x1.y, a10));
                        a11 = fmaf(w0.y, x1.x, fmaf(w1.y, x1.y, a11));
                    }
                    reinterpret_cast<__nv_bfloat162*>(a.q_lat + (((size_t)(n0 + nn) * H + h) * B + b) * d_c + k0)[kp] =
                        __floats2bfloat162_rn(a00, a01);
                    if (two)
                        reinterpret_cast<__nv_bfloat162*>(a.q_lat + (((size_t)(n0 + nn + 8) * H + h) * B + b) * d_c + k0)[kp] =
                            __floats2bfloat162_rn(a10, a11);
                }
            }
        }
        return;
    }

    // ---------------------------------------------------------------- rotary + append
    const int n = ((int)blockIdx.x - n_abs_ctas) * kSeqPerAppendCta + warp;
    if (n >= a.batch) return;
    const int d_r = a.d_r, half = d_r / 2, P = a.page_size;
    const long long p = (long long)__ldg(a.seqlens + n) - 1;
    float c = 1.f, s = 0.f;
    if (lane < half) {
        const double theta = pow((double)a.rope_base, -2.0 * (double)lane / (double)d_r);
        double sd, cd;
        sincos((double)(p < 0 ? 0 : p) * theta, &sd, &cd);
        c = (float)cd;
        s = (float)sd;
    }
    // the RoPE query of every head, 16 heads' loads in flight before their
    // stores (the output may alias nothing, but the compiler cannot know)
    if (lane < half) {
        for (int h0 = 0; h0 < a.heads; h0 += 16) {
            __nv_bfloat162 x[16];
#pragma unroll
            for (int i = 0; i < 16; ++i)
                if (h0 + i < a.heads)
                    x[i] = __ldg(reinterpret_cast<const __nv_bfloat162*>(a.q_r + ((size_t)n * a.heads + h0 + i) * d_r) + lane);
#pragma unroll
            for (int i = 0; i < 16; ++i)
                if (h0 + i < a.heads) {
                    const float x0 = __low2float(x[i]), x1 = __high2float(x[i]);
                    reinterpret_cast<__nv_bfloat162*>(a.q_rope + ((size_t)n * a.heads + h0 + i) * d_r)[lane] =
                        __floats2bfloat162_rn(x0 * c - x1 * s, x0 * s + x1 * c);
                }
        }
    }
    // the append target
    int err = 0;
    int page = -1;
    if (p < 0 || p >= (long long)a.max_pages * P) {
        err = MLRA_ERR_DEVICE_BAD_SEQLEN;
    } else {
        page = __ldg(a.block_table + (size_t)n * a.max_pages + p / P);
        if (page < 0 || page >= a.num_pages) err = MLRA_ERR_DEVICE_BAD_INDEX;
    }
    if (err != 0) {
        if (lane == 0 && a.status != nullptr) record_error(a.status, err);
        return;
    }
    const size_t row = (size_t)page * P + (size_t)(p % P);
    if (lane < half) {
        const __nv_bfloat162 x = reinterpret_cast<const __nv_bfloat162*>(a.kr_new + (size_t)n * d_r + 2 * lane)[0];
        const float x0 = __low2float(x), x1 = __high2float(x);
        reinterpret_cast<__nv_bfloat162*>(a.rope_cache + row * d_r + 2 * lane)[0] =
            __floats2bfloat162_rn(x0 * c - x1 * s, x0 * s + x1 * c);
    }
    const int W = B * d_c, wv = W / 8;
    const uint4* src = reinterpret_cast<const uint4*>(a.c_new + (size_t)n * W);
    uint4* dst = reinterpret_cast<uint4*>(a.latent_cache + row * W);
    for (int u = lane; u < wv; u += 32) dst[u] = __ldg(src + u);
}

}  // namespace

size_t prepare_smem_bytes(int d_h) { return (size_t)d_h * kColBlock * 2 + (size_t)kSeqChunk * d_h * 2; }

cudaError_t launch_prepare(const PrepareArgs& a, cudaStream_t stream) {
    const int kblocks = (a.d_c + kColBlock - 1) / kColBlock;
    const int n_abs = a.heads * a.branches * kblocks;
    const int n_app = (a.batch + kSeqPerAppendCta - 1) / kSeqPerAppendCta;
    const size_t smem = prepare_smem_bytes(a.d_h);
    cudaError_t e = cudaFuncSetAttribute(prepare_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    if (a.status != nullptr) {
        e = cudaMemsetAsync(a.status, 0, sizeof(int), stream);
        if (e != cudaSuccess) return e;
    }
    prepare_kernel<<<n_abs + n_app, kPrepThreads, smem, stream>>>(a, n_abs);
    return cudaGetLastError();
}

}  // namespace mlra
