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
// stream through; warp w multiplies the chunk by columns [8 w, 8 w + 8) on
// the warp-level tensor cores (m16n8k16, bf16 in, fp32 accumulate).  The
// contraction is tiny (34 MFLOP at the 2.9B shape) and its weights (2 MiB)
// are read once, so it is bound by latency: the weights do not depend on
// the preceding kernel and are loaded before the wait for it (the launch is
// a programmatic dependent), the inputs after it (the append reads the
// lengths and block-table entries before the wait too).  Append CTAs take one
// sequence per warp: lane i owns RoPE pair i (the angle formed in turns in
// fp64 and reduced to a fraction of a turn, so positions up to 2^31 keep
// their phase; sine and cosine of that fraction in fp32), rotates that pair
// of every head's query and of the new key, and the warp copies the new
// latents in 16-byte units.
#include "common.cuh"
#include "kernels.h"
#include "sm100.cuh"

namespace mlra {
namespace {

using namespace sm100;

constexpr int kPrepThreads = 256;
constexpr int kColBlock = 64;   // latent columns per absorption CTA
constexpr int kSeqChunk = 64;   // sequences per q_c chunk
constexpr int kSeqPerAppendCta = kPrepThreads / 32;
constexpr int kWP = kColBlock + 8;  // W row stride in shared memory (bf16)

__global__ void __launch_bounds__(kPrepThreads)
prepare_kernel(const PrepareArgs a, int n_abs_ctas) {
    extern __shared__ uint4 prep_smem[];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int H = a.heads, B = a.branches, d_c = a.d_c, d_h = a.d_h;

    launch_dependents();  // the next kernel may set up while this grid runs
    if ((int)blockIdx.x < n_abs_ctas) {
        // ------------------------------------------------------------ absorption
        const int kblocks = (d_c + kColBlock - 1) / kColBlock;
        const int hb = blockIdx.x / kblocks, kb = blockIdx.x % kblocks;
        const int h = hb / B, b = hb % B;
        const int k0 = kb * kColBlock, kw = min(kColBlock, d_c - k0);  // kw: a multiple of 8
        const int DK = (d_h + 15) & ~15, QP = DK + 8;  // K padded to the MMA's 16; q_s row stride
        __nv_bfloat16* w_s = reinterpret_cast<__nv_bfloat16*>(prep_smem);   // [DK][kWP]
        __nv_bfloat16* q_s = w_s + DK * kWP;                                 // [kSeqChunk][QP]
        // W_UK[b][h][j][k0 .. k0 + kw), rows past d_h zero (weights: read
        // before the wait for the preceding grid)
        const int kv = kw / 8;  // 16-byte units per W row
        for (int e = tid; e < DK * kv; e += kPrepThreads) {
            const int j = e / kv, u = e % kv;
            uint4 v = make_uint4(0u, 0u, 0u, 0u);
            if (j < d_h) v = __ldg(reinterpret_cast<const uint4*>(a.w_uk + (((size_t)b * H + h) * d_h + j) * d_c + k0) + u);
            *reinterpret_cast<uint4*>(w_s + j * kWP + 8 * u) = v;
        }
        wait_prerequisite_grid();  // q_c may come from the preceding kernel
        const int g = lane >> 2, tg = lane & 3;
        const int col = 8 * warp;  // this warp's 8 output columns of the block
        const uint16_t* w16 = reinterpret_cast<const uint16_t*>(w_s);
        const int qv = d_h / 8;
        for (int n0 = 0; n0 < a.batch; n0 += kSeqChunk) {
            const int nc = min(kSeqChunk, a.batch - n0), mp = (nc + 15) & ~15;
            __syncthreads();  // W is staged; the previous chunk's q_s is no longer read
            for (int e = tid; e < mp * (DK / 8); e += kPrepThreads) {
                const int nn = e / (DK / 8), u = e % (DK / 8);
                uint4 v = make_uint4(0u, 0u, 0u, 0u);
                if (nn < nc && u < qv)
                    v = __ldg(reinterpret_cast<const uint4*>(a.q_c + ((size_t)(n0 + nn) * H + h) * d_h) + u);
                *reinterpret_cast<uint4*>(q_s + nn * QP + 8 * u) = v;
            }
            __syncthreads();
            if (col >= kw) continue;
            for (int mt = 0; mt < mp / 16; ++mt) {
                float acc[4] = {0.f, 0.f, 0.f, 0.f};
                for (int ks = 0; ks < DK / 16; ++ks) {
                    const int kk = 16 * ks + 2 * tg;
                    // A: sequences x d_h (row-major q_s); B: d_h x 8 columns
                    // (rows kk, kk + 1 and kk + 8, kk + 9 of W, packed in pairs)
                    const __nv_bfloat16* x0 = q_s + (16 * mt + g) * QP + kk;
                    const uint32_t af[4] = {*reinterpret_cast<const uint32_t*>(x0),
                                            *reinterpret_cast<const uint32_t*>(x0 + 8 * QP),
                                            *reinterpret_cast<const uint32_t*>(x0 + 8),
                                            *reinterpret_cast<const uint32_t*>(x0 + 8 * QP + 8)};
                    const uint32_t b0 = (uint32_t)w16[kk * kWP + col + g] | ((uint32_t)w16[(kk + 1) * kWP + col + g] << 16);
                    const uint32_t b1 =
                        (uint32_t)w16[(kk + 8) * kWP + col + g] | ((uint32_t)w16[(kk + 9) * kWP + col + g] << 16);
                    mma_m16n8k16_bf16(acc, af, b0, b1);
                }
                // rows g and g + 8 of the tile, columns col + 2 tg, + 1
#pragma unroll
                for (int r = 0; r < 2; ++r) {
                    const int nn = 16 * mt + g + 8 * r;
                    if (nn < nc)
                        *reinterpret_cast<__nv_bfloat162*>(a.q_lat + (((size_t)(n0 + nn) * H + h) * B + b) * d_c + k0 + col +
                                                           2 * tg) = __floats2bfloat162_rn(acc[2 * r], acc[2 * r + 1]);
                }
            }
        }
        return;
    }

    // ---------------------------------------------------------------- rotary + append
    // The length and the block-table entry are read before the wait for the
    // preceding grid (like w_uk, they must not be written by that kernel), so
    // the position's angle and page are ready when the inputs may be read.
    const int n = ((int)blockIdx.x - n_abs_ctas) * kSeqPerAppendCta + warp;
    if (n >= a.batch) return;
    const int d_r = a.d_r, half = d_r / 2, P = a.page_size;
    const long long p = (long long)__ldg(a.seqlens + n) - 1;
    int err = 0;
    int page = -1;
    if (p < 0 || p >= (long long)a.max_pages * P) {
        err = MLRA_ERR_DEVICE_BAD_SEQLEN;
    } else {
        page = __ldg(a.block_table + (size_t)n * a.max_pages + p / P);
        if (page < 0 || page >= a.num_pages) err = MLRA_ERR_DEVICE_BAD_INDEX;
    }
    float c = 1.f, s = 0.f;
    if (lane < half) {
        // the angle in turns, reduced to [0, 1) in fp64 (2^-24 of a turn or
        // better for every int32 position), then sine and cosine in fp32
        const double t = (double)(p < 0 ? 0 : p) * a.rope_turns[lane];
        sincospif(2.f * (float)(t - floor(t)), &s, &c);
    }
    wait_prerequisite_grid();  // the queries and the new token may come from the preceding kernel
    // every load of the step at once: the new key's pair, the first 16 heads'
    // query pairs, the new latents (up to 4 16-byte units per lane)
    const int W = B * d_c, wv = W / 8;
    const uint4* src = reinterpret_cast<const uint4*>(a.c_new + (size_t)n * W);
    uint4 cv[4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
        if (lane + 32 * i < wv) cv[i] = __ldg(src + lane + 32 * i);
    __nv_bfloat162 kr = __floats2bfloat162_rn(0.f, 0.f), x[16];
    if (lane < half) {
        kr = __ldg(reinterpret_cast<const __nv_bfloat162*>(a.kr_new + (size_t)n * d_r) + lane);
#pragma unroll
        for (int i = 0; i < 16; ++i)
            if (i < a.heads) x[i] = __ldg(reinterpret_cast<const __nv_bfloat162*>(a.q_r + ((size_t)n * a.heads + i) * d_r) + lane);
    }
    // the RoPE query of every head, 16 heads' loads in flight before their
    // stores (the output may alias nothing, but the compiler cannot know)
    if (lane < half) {
        for (int h0 = 0; h0 < a.heads; h0 += 16) {
            if (h0 > 0) {
#pragma unroll
                for (int i = 0; i < 16; ++i)
                    if (h0 + i < a.heads)
                        x[i] = __ldg(reinterpret_cast<const __nv_bfloat162*>(a.q_r + ((size_t)n * a.heads + h0 + i) * d_r) + lane);
            }
#pragma unroll
            for (int i = 0; i < 16; ++i)
                if (h0 + i < a.heads) {
                    const float x0 = __low2float(x[i]), x1 = __high2float(x[i]);
                    reinterpret_cast<__nv_bfloat162*>(a.q_rope + ((size_t)n * a.heads + h0 + i) * d_r)[lane] =
                        __floats2bfloat162_rn(x0 * c - x1 * s, x0 * s + x1 * c);
                }
        }
    }
    // the append (the sequence's queries are written even when it is bad)
    if (err != 0) {
        if (lane == 0 && a.status != nullptr) record_error(a.status, err);
        return;
    }
    const size_t row = (size_t)page * P + (size_t)(p % P);
    if (lane < half) {
        const float x0 = __low2float(kr), x1 = __high2float(kr);
        reinterpret_cast<__nv_bfloat162*>(a.rope_cache + row * d_r + 2 * lane)[0] =
            __floats2bfloat162_rn(x0 * c - x1 * s, x0 * s + x1 * c);
    }
    uint4* dst = reinterpret_cast<uint4*>(a.latent_cache + row * W);
#pragma unroll
    for (int i = 0; i < 4; ++i)
        if (lane + 32 * i < wv) dst[lane + 32 * i] = cv[i];
    for (int u = lane + 128; u < wv; u += 32) dst[u] = __ldg(src + u);
}

}  // namespace

size_t prepare_smem_bytes(int d_h) {
    const size_t dk = (size_t)(d_h + 15) / 16 * 16;
    return dk * kWP * 2 + (size_t)kSeqChunk * (dk + 8) * 2;
}

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
    // programmatic: the CTAs may start (and load the weights) while the
    // preceding kernel in the stream runs; inputs are read after its end
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(n_abs + n_app);
    cfg.blockDim = dim3(kPrepThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, prepare_kernel, a, n_abs);
}

}  // namespace mlra
