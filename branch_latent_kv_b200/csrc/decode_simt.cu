// decode_simt.cu -- split-KV MLRA decode on CUDA cores (fp32 FMA).
//
// One persistent CTA per SM walks its contiguous range of 128-token tiles
// (the shared plan in common.cuh).  Per 32-token sub-tile it gathers the
// paged latent and RoPE rows into shared memory, scores every (head, branch)
// pair against its own branch latent plus the shared RoPE key, updates an
// online softmax per (head, branch) and accumulates the value-absorbed
// output.  This is the straightforward statement of the kernel; the
// tensor-core kernel computes the same partials.
//
// Method: "MLRA: Breaking the Sharding Bottleneck in Latent Attention"
// (wispaper.ai blog), section "The Core Insight: Sum of Branches, Not Sum of
// Keys" -- each latent block is attended independently.
#include "common.cuh"
#include "kernels.h"

namespace mlra {
namespace {

constexpr int kSub = 32;       // tokens per shared-memory sub-tile
constexpr int kThreads = 256;

struct SimtSmem {
    // offsets in floats
    int q, qr, o, c, r, s, m, l, a, total;
};

__host__ __device__ inline SimtSmem simt_layout(int H, int B, int d_c, int d_r) {
    const int W = B * d_c, HB = H * B;
    SimtSmem s;
    s.q = 0;                            // [H][B][d_c]  queries * scale * log2e
    s.qr = s.q + H * W;                 // [H][d_r]
    s.o = s.qr + H * d_r;               // [H][B][d_c]  running output
    s.c = s.o + H * W;                  // [kSub][W + 1] latent rows (padded)
    s.r = s.c + kSub * (W + 1);         // [kSub][d_r + 1]
    s.s = s.r + kSub * (d_r + 1);       // [HB][kSub]   scores, then p
    s.m = s.s + HB * kSub;              // [HB] running max (log2 domain)
    s.l = s.m + HB;                     // [HB] running sum
    s.a = s.l + HB;                     // [HB] rescale factor of this sub-tile
    s.total = s.a + HB;
    return s;
}

__device__ inline float bf16_at(const __nv_bfloat16* p, size_t i) { return __bfloat162float(p[i]); }

__global__ void __launch_bounds__(kThreads) decode_simt_kernel(DecodeArgs a) {
    extern __shared__ float sm[];
    __shared__ int plan[4];  // chunk, first sequence, its cost start
    __shared__ int seg_bad;

    const int H = a.heads, B = a.branches, d_c = a.d_c, d_r = a.d_r, P = a.page_size;
    const int W = B * d_c, HB = H * B;
    const SimtSmem L = simt_layout(H, B, d_c, d_r);
    float* q_s = sm + L.q;
    float* qr_s = sm + L.qr;
    float* o_s = sm + L.o;
    float* c_s = sm + L.c;
    float* r_s = sm + L.r;
    float* s_s = sm + L.s;
    float* m_s = sm + L.m;
    float* l_s = sm + L.l;
    float* a_s = sm + L.a;
    const int tid = threadIdx.x;
    const int cta = blockIdx.x;

    if (tid < 32) {
        const int total = warp_cost_prefix(a.seqlens, a.batch, P, a.max_pages);
        const int chunk = plan_chunk(total, a.num_ctas);
        int n0 = a.batch, cum0 = total;
        if ((long long)cta * chunk < total)
            warp_find_seq(a.seqlens, a.batch, P, a.max_pages, cta * chunk, &n0, &cum0);
        if (tid == 0) { plan[0] = chunk; plan[1] = n0; plan[2] = cum0; }
    }
    __syncthreads();
    const int chunk = plan[0];
    const int A0 = cta * chunk, A1 = A0 + chunk;  // this CTA's cost window

    int n = plan[1], cum = plan[2];
    for (; n < a.batch && cum < A1; ++n) {
        const int Ln = __ldg(a.seqlens + n);
        const int tiles = seq_tiles(Ln, P, a.max_pages);
        if (tiles == 0) continue;
        const int cum_n = cum;
        cum += seq_cost(Ln, P, a.max_pages);
        const int tb = first_tile_at(cum_n, tiles, A0);
        const int te = first_tile_at(cum_n, tiles, A1);
        if (tb >= te) continue;
        const int tok_begin = tb * kTileTokens;
        const int tok_end = min(te * kTileTokens, Ln);
        const int32_t* bt = a.block_table + (size_t)n * a.max_pages;

        // queries, pre-multiplied by scale*log2e so scores are base-2 logits
        for (int i = tid; i < H * W; i += kThreads)
            q_s[i] = bf16_at(a.q_lat, (size_t)n * H * W + i) * a.scale_log2;
        for (int i = tid; i < H * d_r; i += kThreads)
            qr_s[i] = bf16_at(a.q_rope, (size_t)n * H * d_r + i) * a.scale_log2;
        for (int i = tid; i < H * W; i += kThreads) o_s[i] = 0.f;
        for (int i = tid; i < HB; i += kThreads) { m_s[i] = -INFINITY; l_s[i] = 0.f; }
        if (tid == 0) seg_bad = 0;
        __syncthreads();

        for (int tok0 = tok_begin; tok0 < tok_end; tok0 += kSub) {
            // gather kSub token rows (8 bf16 per 16-byte load); rows past the
            // end of the range are zero and never reach the output
            const int cpr = W / 8, rpr = d_r / 8;
            for (int i = tid; i < kSub * (cpr + rpr); i += kThreads) {
                const int row = i / (cpr + rpr), col = i % (cpr + rpr);
                const int t = tok0 + row;
                float v[8];
#pragma unroll
                for (int j = 0; j < 8; ++j) v[j] = 0.f;
                if (t < tok_end) {
                    int page = __ldg(bt + t / P);
                    if (page < 0 || page >= a.num_pages) {
                        seg_bad = 1;
                    } else {
                        const size_t pool_row = (size_t)page * P + t % P;
                        const uint4 raw = col < cpr
                            ? __ldg(reinterpret_cast<const uint4*>(a.latent + pool_row * W) + col)
                            : __ldg(reinterpret_cast<const uint4*>(a.rope + pool_row * d_r) + (col - cpr));
                        const __nv_bfloat16* e = reinterpret_cast<const __nv_bfloat16*>(&raw);
#pragma unroll
                        for (int j = 0; j < 8; ++j) v[j] = __bfloat162float(e[j]);
                    }
                }
                float* dst = col < cpr ? c_s + row * (W + 1) + col * 8
                                       : r_s + row * (d_r + 1) + (col - cpr) * 8;
#pragma unroll
                for (int j = 0; j < 8; ++j) dst[j] = v[j];
            }
            __syncthreads();

            // scores s[hb][t] (base-2 logits); masked tokens get -inf
            for (int i = tid; i < HB * kSub; i += kThreads) {
                const int t = i % kSub, hb = i / kSub;
                const int h = hb / B, b = hb % B;
                float s = -INFINITY;
                if (tok0 + t < tok_end) {
                    const float* q = q_s + h * W + b * d_c;
                    const float* c = c_s + t * (W + 1) + b * d_c;
                    float acc = 0.f;
                    for (int k = 0; k < d_c; ++k) acc = fmaf(q[k], c[k], acc);
                    const float* qr = qr_s + h * d_r;
                    const float* r = r_s + t * (d_r + 1);
                    for (int k = 0; k < d_r; ++k) acc = fmaf(qr[k], r[k], acc);
                    s = acc;
                }
                s_s[hb * kSub + t] = s;
            }
            __syncthreads();

            // online softmax update per (head, branch)
            for (int hb = tid; hb < HB; hb += kThreads) {
                float* s = s_s + hb * kSub;
                float mt = -INFINITY;
                for (int t = 0; t < kSub; ++t) mt = fmaxf(mt, s[t]);
                const float m_old = m_s[hb];
                const float m_new = fmaxf(m_old, mt);
                const float alpha = exp2f(m_old - m_new);  // 0 on the first sub-tile
                float sum = 0.f;
                for (int t = 0; t < kSub; ++t) {
                    const float pt = exp2f(s[t] - m_new);   // masked: exp2(-inf) = 0
                    s[t] = pt;
                    sum += pt;
                }
                l_s[hb] = l_s[hb] * alpha + sum;
                m_s[hb] = m_new;
                a_s[hb] = alpha;
            }
            __syncthreads();

            // o[h][b][:] = alpha * o + sum_t p_t c_b[t]
            for (int e = tid; e < H * W; e += kThreads) {
                const int h = e / W, rem = e % W, b = rem / d_c;
                const int hb = h * B + b;
                const float* p = s_s + hb * kSub;
                float acc = o_s[e] * a_s[hb];
                for (int t = 0; t < kSub; ++t) acc = fmaf(p[t], c_s[t * (W + 1) + rem], acc);
                o_s[e] = acc;
            }
            __syncthreads();
        }

        // epilogue: final output of a single-split sequence, else a partial
        int first_cta, last_cta;
        seq_owners(cum_n, tiles, chunk, &first_cta, &last_cta);
        const bool bad = seg_bad != 0;
        if (bad && tid == 0) record_error(a.err, MLRA_ERR_DEVICE_BAD_INDEX);
        if (first_cta == last_cta) {
            for (int e = tid; e < H * W; e += kThreads) {
                const int h = e / W, b = (e % W) / d_c;
                const float v = bad ? 0.f : a.out_scale * o_s[e] / l_s[h * B + b];
                a.out[(size_t)n * H * W + e] = to_bf16(v);
            }
        } else {
            const size_t slot = (size_t)cta + n;
            for (int e = tid; e < H * W; e += kThreads) {
                const int h = e / W, rem = e % W, b = rem / d_c, k = rem % d_c;
                const float v = bad ? 0.f : o_s[e] / l_s[h * B + b];
                a.o_part[((slot * B + b) * d_c + k) * partial_heads(H) + h] = v;
            }
            for (int hb = tid; hb < HB; hb += kThreads) {
                const int h = hb / B, b = hb % B;
                a.lse_part[(slot * B + b) * partial_heads(H) + h] =
                    bad ? bad_split_marker() : m_s[hb] + log2f(l_s[hb]);
            }
        }
        __syncthreads();
    }
}

}  // namespace

size_t decode_simt_smem_bytes(int heads, int branches, int d_c, int d_r) {
    return sizeof(float) * (size_t)simt_layout(heads, branches, d_c, d_r).total;
}

cudaError_t launch_decode_simt(const DecodeArgs& a, cudaStream_t stream) {
    const size_t smem = decode_simt_smem_bytes(a.heads, a.branches, a.d_c, a.d_r);
    cudaError_t e = cudaFuncSetAttribute(decode_simt_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    decode_simt_kernel<<<a.num_ctas, kThreads, smem, stream>>>(a);
    return cudaGetLastError();
}

}  // namespace mlra
