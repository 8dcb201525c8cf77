// up_proj.cu -- per-branch W_UV up-projection and branch sum on tcgen05.
//
//   y[n, h*d_h + j] = sum_b sum_k out_lat[n,h,b,k] * w_uv[b][k][h*d_h + j]
//
// ("The Core Insight" section of the wispaper.ai MLRA blog page: every
// branch is up-projected by its own matrix and the branch outputs are summed
// at the end.)  The branch sum is the K reduction over K = branches * d_c:
// for head h the product is one GEMM of W_h^T [d_h x K] by X_h^T [K x N].
//
// A cluster of KS CTAs per (head, tile of up to 64 sequences) splits K; each
// CTA multiplies its K range, swap-AB so that the 128 output columns of a
// head are the MMA's M:
//   D[j, n] = sum_K W[K][h*d_h + j] * X[n][h][K]
//   A = W slice, MN-major (j contiguous), 128-byte swizzle, two 64-column boxes
//   B = X slice, K-major (K contiguous), 128-byte swizzle, rows past the
//       batch are zero-filled by TMA
// Every 64-wide K chunk of a CTA's range is loaded at once, each on its own
// mbarrier, so the MMAs start as chunks land.  The KS fp32 partial products
// are summed through distributed shared memory: each CTA stages its
// [128 x nt] partial, then CTA r of the cluster adds up columns
// [r*nt/KS, (r+1)*nt/KS) from all KS CTAs and writes them as bf16.
// Rows j >= d_h (d_h = 64) are computed from neighbouring columns or TMA
// zero fill and discarded.
//
// Optional output gate ("Critical Insight: The Value of 'Gating'" on the same
// page: a gate on the attention output adds a non-linearity; its formula is
// lost in the page text, read here as the usual elementwise sigmoid gate):
//   y[n, c] *= 1 / (1 + exp(-gate[n, c]))   for every output element c,
// applied to the fp32 sum before the bf16 rounding.
//
// Branch sharding ("The Core Insight" section of the same page: the branches
// can live on different GPUs, so under 4-way tensor parallelism each GPU loads
// only its own branch's latents plus the shared RoPE key, 1.5 d_h per token
// against 4.5 d_h for MLA).  Rank r then holds out_lat and W_UV of its
// branches only, and the branch sum crosses the ranks.  In that mode a CTA's
// column slice is not written as y: each CTA stores every fp32 value of its
// slice, paired with the call's tag (call + 1) in one 64-bit word, into slot
// r of every rank's exchange region (plain stores, to peer memory over
// NVLink).  Each rank then reads its own region's slots for the tile, polls
// (with a bound) any word whose tag is not this call's, adds the slots in
// rank order (the same order on every rank, so every rank's y is
// bit-identical) and applies the gate.  The word is single-copy atomic, so a
// reader that sees the tag sees the value: no flags, no fences.  The call
// number of each tile, kept per tile in the region, selects one of two
// buffers, so a rank that runs ahead into the next call never overwrites a
// word that a slower rank has not yet read.
#include <cudaTypedefs.h>

#include "common.cuh"
#include "kernels.h"
#include "peer.cuh"
#include "sm100.cuh"

namespace mlra {
namespace {

using namespace sm100;
using namespace peer;

constexpr int kThreads = 128;
constexpr int kMaxChunks = 8;      // K <= 512
constexpr int kMaxNT = 64;         // sequences per CTA
constexpr int kWChunkBytes = 2 * 64 * 128;  // two 64-column boxes of 64 K rows: 16 KB

struct UpMaps {
    CUtensorMap w;  // w_uv as [K rows][H*d_h columns]
    CUtensorMap x;  // out_lat as [N rows][H*K columns]
};

struct UpSmem {
    uint64_t full[kMaxChunks];
    uint64_t mma_done;
    uint32_t tmem_base;
    uint32_t xr_call;                // cross-rank mode: this tile's call number
    uint8_t* xr_region[kMaxWorld];   // and every rank's exchange region
};

// Row j, columns nn .. nn + 3 of the [128 x nt] fp32 partial, summed over the
// ks CTAs of the cluster (distributed shared memory).
__device__ __forceinline__ float4 cluster_column_sum(uint32_t part_addr, int j, int nt, int nn, int ks) {
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int r = 0; r < ks; ++r) {
        const float4 v = ld_shared_cluster_f4(map_shared_rank(part_addr + (j * nt + nn) * 4, r));
        acc.x += v.x;
        acc.y += v.y;
        acc.z += v.z;
        acc.w += v.w;
    }
    return acc;
}

// kXRank: the cross-rank branch sum (a separate instantiation, so that the
// single-device kernel carries none of its code or registers)
template <bool kXRank>
__global__ void __launch_bounds__(kThreads, 1)
up_proj_tc_kernel(const __grid_constant__ UpMaps maps, int batch, int heads, int K, int d_h, int nt, int ks,
                  const __nv_bfloat16* __restrict__ gate, __nv_bfloat16* __restrict__ y, const XRankArgs xr) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int cpc = K / 64 / ks;                 // K chunks of this CTA
    const int x_chunk_bytes = nt * 128;
    uint8_t* w_s = sm;                           // cpc x 16 KB
    uint8_t* x_s = sm + cpc * kWChunkBytes;      // cpc x nt*128 B
    float* part = reinterpret_cast<float*>(sm);  // [128][nt] fp32 partial, reuses the operand buffers
    // barriers and flags past both the operands and the partial
    UpSmem& ms = *reinterpret_cast<UpSmem*>(sm + max(cpc * (kWChunkBytes + x_chunk_bytes), 128 * nt * 4));
    const uint32_t rank = cluster_ctarank();
    const int h = blockIdx.x / ks, n0 = blockIdx.y * nt;
    // blockIdx.z: which of the ranks stacked into this launch (0 otherwise);
    // its operands start lr * K rows into w_uv and lr * batch rows into out_lat
    const int lr = blockIdx.z;
    y += (size_t)lr * batch * heads * d_h;
    const int c_first = (int)rank * cpc;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t tmem_cols = nt <= 32 ? 32 : 64;

    if (threadIdx.x == 0) {
        for (int c = 0; c < cpc; ++c) mbar_init(&ms.full[c], 1);
        mbar_init(&ms.mma_done, 1);
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc(&ms.tmem_base, tmem_cols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = ms.tmem_base;

    launch_dependents();
    if (warp == 0 && elect_one()) {
        prefetch_tensormap(&maps.w);
        prefetch_tensormap(&maps.x);
        // W_UV does not depend on the preceding kernels: load it first, then
        // wait for the grid that writes out_lat (programmatic dependent launch)
        for (int c = 0; c < cpc; ++c) {
            const int kc = c_first + c;
            mbar_arrive_expect_tx(&ms.full[c], kWChunkBytes + x_chunk_bytes);
            tma_load_2d(w_s + c * kWChunkBytes, &maps.w, h * d_h, lr * K + kc * 64, &ms.full[c]);
            tma_load_2d(w_s + c * kWChunkBytes + kWChunkBytes / 2, &maps.w, h * d_h + 64, lr * K + kc * 64,
                        &ms.full[c]);
        }
        wait_prerequisite_grid();
        for (int c = 0; c < cpc; ++c)
            tma_load_2d(x_s + c * x_chunk_bytes, &maps.x, h * K + (c_first + c) * 64, lr * batch + n0, &ms.full[c]);
        if constexpr (kXRank) {
            // under the GEMM: the regions and this tile's call number (written
            // by the previous call, which the wait above has seen complete)
            for (int p = 0; p < xr.world; ++p) ms.xr_region[p] = static_cast<uint8_t*>(xr.regions[p]);
            const int tile = blockIdx.y * gridDim.x + blockIdx.x;
            uint32_t* epoch = reinterpret_cast<uint32_t*>(ms.xr_region[xr.rank_base + lr]) + tile;
            const uint32_t call = __ldcg(epoch);
            ms.xr_call = call;
            *epoch = call + 1;  // read by the next call only
        }
    }
    if (warp == 1) {
        bool ok = true;
        const uint32_t idesc = idesc_bf16_f32(128, nt, true, false);
        const uint64_t dW = smem_desc(smem_u32(w_s), kWChunkBytes / 2, 1024, kLayoutSw128);  // MN-major
        const uint64_t dX = smem_desc(smem_u32(x_s), 16, 1024, kLayoutSw128);               // K-major
        for (int c = 0; c < cpc && ok; ++c) {
            ok = mbar_wait_warp(&ms.full[c], 0);
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
                if (ok && elect_one())
                    mma_bf16(tmem, dW + ((c * kWChunkBytes + kk * 2048) >> 4),
                             dX + ((c * x_chunk_bytes + kk * 32) >> 4), idesc, (c | kk) ? 1u : 0u);
            __syncwarp();
        }
        if (elect_one()) mma_commit(&ms.mma_done);
        __syncwarp();
    }
    // every copy has landed once the MMAs that read it are done; the wait
    // below also covers the case where an MMA wait gave up (bounded)
    const bool done = mbar_wait(&ms.mma_done, 0);
    if (warp == 0 && lane == 0)
        for (int c = 0; c < cpc; ++c) mbar_wait(&ms.full[c], 0, 200000000ull);
    __syncthreads();
    tc_fence_after();
    // stage this CTA's partial: thread j writes row j (nt fp32)
    const int j = warp * 32 + lane;
    const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
    for (int c0 = 0; c0 < nt; c0 += 16) {
        float v[16];
        tmem_ld16(tmem + lane_off + c0, v);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 16; i += 4)
            *reinterpret_cast<float4*>(part + j * nt + c0 + i) =
                done ? make_float4(v[i], v[i + 1], v[i + 2], v[i + 3]) : make_float4(0.f, 0.f, 0.f, 0.f);
    }
    tc_fence_before();
    cluster_sync();  // every CTA's partial is staged
    // CTA `rank` sums columns [n_lo, n_hi) over the cluster
    const int per = nt / ks;
    const int n_lo = (int)rank * per, n_hi = n_lo + per;
    const uint32_t part_addr = smem_u32(part);
    const size_t HD = (size_t)heads * d_h;
    if constexpr (!kXRank) {
        if (j < d_h) {
            for (int nn = n_lo; nn < n_hi; nn += 4) {
                const float4 acc = cluster_column_sum(part_addr, j, nt, nn, ks);
                const float vals[4] = {acc.x, acc.y, acc.z, acc.w};
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int n = n0 + nn + i;
                    if (n >= batch) continue;
                    const size_t o = (size_t)n * HD + (size_t)h * d_h + j;
                    float v = vals[i];
                    if (gate != nullptr) v *= 1.f / (1.f + expf(-__bfloat162float(gate[o])));
                    y[o] = to_bf16(v);
                }
            }
        }
    } else {
        const int world = xr.world, xrank = xr.rank_base + lr;
        const ExchangeLayout L = exchange_layout(batch, heads, d_h, world, xr.tiles);
        const uint32_t call = ms.xr_call, tag = call + 1;
        const size_t buf = (size_t)(call & 1u) * world;  // first slot of this call's buffer
        if (j < d_h) {
            // push: this rank's slice into slot xrank of every rank's buffer
            for (int nn = n_lo; nn < n_hi; nn += 4) {
                const float4 acc = cluster_column_sum(part_addr, j, nt, nn, ks);
                const float vals[4] = {acc.x, acc.y, acc.z, acc.w};
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int n = n0 + nn + i;
                    if (n >= batch) continue;
                    const size_t o = (size_t)n * HD + (size_t)h * d_h + j;
                    const uint64_t word = (uint64_t)__float_as_uint(vals[i]) | ((uint64_t)tag << 32);
                    for (int p = 0; p < world; ++p)
                        st_relaxed_sys_u64(reinterpret_cast<uint64_t*>(ms.xr_region[p] + L.data_off) +
                                               ((buf + xrank) * batch) * HD + o, word);
                }
            }
            // sum: every rank's slot in rank order, four columns' loads in
            // flight at once; a slot whose tag is not this call's is polled
            // (bounded), and a sum with a missing slot is written as zero
            const uint64_t* data = reinterpret_cast<const uint64_t*>(ms.xr_region[xrank] + L.data_off);
            bool alive = true;
            uint64_t t0 = 0;
            for (int nn = n_lo; nn < n_hi; nn += 4) {
                uint64_t w[4][kMaxWorld];
#pragma unroll
                for (int i = 0; i < 4; ++i)
#pragma unroll
                    for (int src = 0; src < kMaxWorld; ++src)
                        if (src < world && n0 + nn + i < batch)
                            w[i][src] = ld_relaxed_sys_u64(data + ((buf + src) * batch) * HD +
                                                           (size_t)(n0 + nn + i) * HD + (size_t)h * d_h + j);
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int n = n0 + nn + i;
                    if (n >= batch) continue;
                    const size_t o = (size_t)n * HD + (size_t)h * d_h + j;
                    float v = 0.f;
                    bool complete = true;
#pragma unroll
                    for (int src = 0; src < kMaxWorld; ++src) {
                        if (src >= world) break;
                        uint64_t x = w[i][src];
                        while ((uint32_t)(x >> 32) != tag && alive) {
                            const uint64_t now = globaltimer_ns();
                            if (t0 == 0) t0 = now;
                            if (now - t0 > xr.limit_ns) {
                                alive = false;
                                break;
                            }
                            x = ld_relaxed_sys_u64(data + ((buf + src) * batch) * HD + o);
                        }
                        if ((uint32_t)(x >> 32) == tag) v += __uint_as_float((uint32_t)x);
                        else complete = false;
                    }
                    if (!complete) v = 0.f;
                    if (gate != nullptr) v *= 1.f / (1.f + expf(-__bfloat162float(gate[o])));
                    y[o] = to_bf16(v);
                }
            }
            if (!alive && xr.status != nullptr) record_error(xr.status, MLRA_ERR_DEVICE_TIMEOUT);
        }
    }
    cluster_sync();  // no CTA leaves while another still reads its shared memory
    if (warp == 1) tmem_dealloc(tmem, tmem_cols);
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (fn == nullptr) {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    }
    return fn;
}

bool encode(CUtensorMap* map, const void* base, uint64_t inner, uint64_t rows, uint32_t box_inner,
            uint32_t box_rows) {
    auto fn = encode_fn();
    if (fn == nullptr) return false;
    const cuuint64_t dims[2] = {inner, rows};
    const cuuint64_t strides[1] = {inner * 2};
    const cuuint32_t box[2] = {box_inner, box_rows};
    const cuuint32_t estr[2] = {1, 1};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

namespace {

struct UpGrid {
    int ks, nt, cpc;
    size_t smem;
};

UpGrid up_grid(int batch, int branches, int d_c) {
    UpGrid g;
    const int nchunk = branches * d_c / 64;
    g.ks = nchunk % 4 == 0 ? 4 : (nchunk % 2 == 0 ? 2 : 1);  // CTAs splitting K (cluster size)
    // sequences per CTA: a multiple of 16 (MMA N) and of 4 * ks, at most 64
    g.nt = batch >= kMaxNT ? kMaxNT : ceil_div(batch, 16) * 16;
    g.cpc = nchunk / g.ks;
    // operands (the fp32 partial reuses them), then the barriers; 1024 bytes
    // of slack for aligning the base to the 128-byte swizzle atom
    const size_t ops = (size_t)g.cpc * (kWChunkBytes + g.nt * 128), part_bytes = (size_t)128 * g.nt * 4;
    g.smem = (ops > part_bytes ? ops : part_bytes) + sizeof(UpSmem) + 1024;
    return g;
}

cudaError_t launch_impl(int batch, int heads, int branches, int d_c, int d_h, const __nv_bfloat16* out_lat,
                        const __nv_bfloat16* w_uv, const __nv_bfloat16* gate, __nv_bfloat16* y,
                        const XRankArgs& xr, int ranks_in_launch, cudaStream_t stream) {
    const int K = branches * d_c;
    if (K % 64 != 0 || K / 64 > kMaxChunks || ranks_in_launch < 1) return cudaErrorInvalidValue;
    const UpGrid g = up_grid(batch, branches, d_c);
    UpMaps maps;
    if (!encode(&maps.w, w_uv, (uint64_t)heads * d_h, (uint64_t)K * ranks_in_launch, 64, 64) ||
        !encode(&maps.x, out_lat, (uint64_t)heads * K, (uint64_t)batch * ranks_in_launch, 64, (uint32_t)g.nt))
        return cudaErrorInvalidValue;
    const bool xrank = xr.world > 0;
    auto kernel = xrank ? up_proj_tc_kernel<true> : up_proj_tc_kernel<false>;
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)g.smem);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(heads * g.ks, ceil_div(batch, g.nt), ranks_in_launch);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = g.smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = g.ks;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    if (xrank) {
        // a tile waits for the same tile of every other rank: the whole grid
        // must be resident at once, or a waiting CTA could hold the SM that a
        // tile it waits for needs
        int clusters = 0;
        cfg.numAttrs = 1;
        e = cudaOccupancyMaxActiveClusters(&clusters, kernel, &cfg);
        cfg.numAttrs = 2;
        if (e != cudaSuccess) return e;
        const long long need = (long long)heads * ceil_div(batch, g.nt) * ranks_in_launch;
        if (clusters < need) return cudaErrorCooperativeLaunchTooLarge;
    }
    return cudaLaunchKernelEx(&cfg, kernel, maps, batch, heads, K, d_h, g.nt, g.ks, gate, y, xr);
}

}  // namespace

int up_proj_tiles(int batch, int heads, int branches, int d_c) {
    const UpGrid g = up_grid(batch, branches, d_c);
    return heads * g.ks * ceil_div(batch, g.nt);
}

cudaError_t launch_up_proj(int batch, int heads, int branches, int d_c, int d_h,
                           const __nv_bfloat16* out_lat, const __nv_bfloat16* w_uv,
                           const __nv_bfloat16* gate, __nv_bfloat16* y, cudaStream_t stream) {
    XRankArgs none{};
    return launch_impl(batch, heads, branches, d_c, d_h, out_lat, w_uv, gate, y, none, 1, stream);
}

cudaError_t launch_up_proj_xrank(int batch, int heads, int branches, int d_c, int d_h,
                                 const __nv_bfloat16* out_lat, const __nv_bfloat16* w_uv,
                                 const __nv_bfloat16* gate, __nv_bfloat16* y, const XRankArgs& xr,
                                 int ranks_in_launch, cudaStream_t stream) {
    if (xr.world < 1 || xr.world > kMaxWorld || xr.regions == nullptr) return cudaErrorInvalidValue;
    if (xr.tiles != up_proj_tiles(batch, heads, branches, d_c)) return cudaErrorInvalidValue;
    return launch_impl(batch, heads, branches, d_c, d_h, out_lat, w_uv, gate, y, xr, ranks_in_launch, stream);
}

}  // namespace mlra
