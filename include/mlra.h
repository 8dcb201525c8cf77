/*
 * mlra.h -- C ABI of the MLRA decode-attention library (sm_100a, one GPU).
 *
 * Multi-Head Low-Rank Attention keeps B independent latent branches per token
 * (B = 4 for MLRA-4) plus one decoupled RoPE key shared by all branches and
 * heads.  A decode step scores every query head against every branch's
 * latent, runs an independent softmax per (head, branch), forms the
 * value-absorbed latent output of each branch, up-projects each branch with
 * its own W_UV and sums the branches.
 *
 * Sources:
 *  - "MLRA: Breaking the Sharding Bottleneck in Latent Attention"
 *    (wispaper.ai blog), section "The Core Insight: Sum of Branches, Not Sum
 *    of Keys": attention on each latent block independently, outputs summed.
 *  - same page, section "Mathematical Calibration: Scaling the Latents": a
 *    final rescaling factor on the attention output (here `out_scale`).
 *  - "Multi-Head Low-Rank Attention" abstract (arXiv 2603.02188, shd-paper.top
 *    and searcharxiv pages): decoding is bound by moving the KV cache from HBM
 *    to on-chip memory at every step.
 *  - "TransMLA: Multi-head latent attention is all you need" (Hacker News
 *    thread), comment quoting its section 3.3: only the latents are cached.
 *
 * Conventions for every entry point:
 *  - All tensors are dense, row-major, in device memory owned by the caller,
 *    and 16-byte aligned.  bf16 is IEEE bfloat16; results are rounded to
 *    nearest even.
 *  - `stream` is a cudaStream_t passed as void* (NULL = the legacy default
 *    stream).  Work is enqueued asynchronously; no entry point allocates,
 *    frees or synchronises, except mlra_read_device_error and the
 *    exchange-region setup calls (mlra_exchange_*; documented below).
 *  - Arguments are validated on the host before anything is enqueued; a
 *    rejected call enqueues nothing.  No C++ exception crosses this ABI.
 *  - Problems that only the device can see (a bad block-table entry or
 *    sequence length) do not trap: the affected sequence's output is written
 *    as zeros and the first such code is recorded in the workspace error
 *    word, read back with mlra_read_device_error.
 */
#ifndef MLRA_H
#define MLRA_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define MLRA_API __attribute__((visibility("default")))
#else
#define MLRA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    MLRA_OK = 0,
    MLRA_ERR_INVALID_ARG = 1,      /* null/misaligned pointer, bad size, inconsistent dims */
    MLRA_ERR_UNSUPPORTED = 2,      /* valid but outside the shapes the kernels implement */
    MLRA_ERR_WORKSPACE = 3,        /* workspace missing or smaller than required */
    MLRA_ERR_CUDA = 4,             /* a CUDA call or kernel launch failed */
    MLRA_ERR_DEVICE_BAD_INDEX = 5, /* device: block-table entry outside [0, num_pages) */
    MLRA_ERR_DEVICE_BAD_SEQLEN = 6,/* device: seqlen < 1 or > max_pages_per_seq * page_size */
    MLRA_ERR_DEVICE_TIMEOUT = 7    /* device: a bounded wait inside a kernel gave up */
} mlra_status;

/* Shape of one decode step. */
typedef struct {
    int32_t batch;             /* N: sequences, one new query token each            */
    int32_t heads;             /* H: query heads                                     */
    int32_t branches;          /* B: latent branches (4 for MLRA-4, 1 = MLA)         */
    int32_t d_c;               /* latent width of one branch                         */
    int32_t d_r;               /* width of the shared decoupled RoPE key             */
    int32_t page_size;         /* P: tokens per cache page                           */
    int32_t max_pages_per_seq; /* columns of the block table                         */
    int32_t num_pages;         /* pages in the physical pool                         */
} mlra_dims;

/*
 * Bytes of workspace mlra_decode needs for `dims` when its grid has
 * `num_ctas` CTAs; num_ctas <= 0 means "the current device's SM count"
 * (the grid mlra_decode launches).  Pure host computation (the SM count query
 * is the only CUDA call).  Returns 0 if dims are invalid.
 * The workspace holds the device error word, a split counter per sequence
 * (a fixed 256 KB region, so a workspace can serve calls with different
 * dims), the split-KV partial outputs (fp32) and their log-sum-exps.
 * Zero it once before first use (the error word and the counters must start
 * at 0).  Every call that ends without MLRA_ERR_DEVICE_TIMEOUT leaves the
 * counters at 0 again, so it never needs re-zeroing.  A call whose kernel
 * gave up on a bounded wait may leave counters set: mlra_read_device_error
 * clears them when it reports the timeout; a caller that does not read the
 * error must zero the first 256 KB + 256 bytes of the workspace before
 * reusing it.
 */
MLRA_API size_t mlra_decode_workspace_bytes(const mlra_dims* dims, int32_t num_ctas);

/*
 * MLRA decode attention for one step (the value-absorbed latent output of
 * every head and branch).  For sequence n of length L = seqlens[n], token t
 * lives at latent_cache[block_table[n][t / P]][t % P]; for every head h and
 * branch b independently:
 *   s_t = scale * (q_lat[n,h,b,:] . c_b[t] + q_rope[n,h,:] . k_r[t])
 *   out[n,h,b,:] = out_scale * sum_t softmax_t(s)_t * c_b[t]
 * ("The Core Insight" and "Mathematical Calibration" sections of the blog
 * page named above; the RoPE query is one per head, the RoPE key one per
 * token, both shared by the branches and already rotated.)
 *
 *   q_lat        bf16 [batch, heads, branches, d_c]   absorbed no-RoPE queries
 *   q_rope       bf16 [batch, heads, d_r]             RoPE queries
 *   latent_cache bf16 [num_pages, page_size, branches, d_c]
 *   rope_cache   bf16 [num_pages, page_size, d_r]
 *   block_table  int32 [batch, max_pages_per_seq]     page of each block; only
 *                the first ceil(L/P) entries of a row are read
 *   seqlens      int32 [batch]                        device memory
 *   scale        softmax scale applied to the raw dot products
 *   out_scale    variance-calibration factor applied to the output
 *   out          bf16 [batch, heads, branches, d_c]   written
 *   workspace    device buffer of >= mlra_decode_workspace_bytes(dims, 0)
 *                bytes, zeroed before its first use; one call at a time
 *
 * Runs on the tensor cores (tcgen05, operands staged by TMA) as one
 * cooperative kernel (one CTA per SM, all resident; the CTAs that share a
 * sequence merge their partials at the end).  The MMAs take one tile of
 * T heads at a time, T = 16 up to 16 heads, else 32 when d_c >= 128 and 16
 * when d_c = 64: more heads run as ceil(heads / T) groups on as many equal
 * parts of the grid, which walk the same tokens together so that the cache
 * crosses HBM about once (the repeat reads of a line hit L2).  Supported
 * shapes: heads <= 128 with batch * ceil(heads / T) <= 65535;
 * (branches, d_c) in {(2,64), (4,64), (1,128), (2,128),
 * (4,128), (1,256), (2,256), (1,512)}; d_r in {32, 64}; page_size in
 * {16, 32, 64, 128}.  Other shapes return MLRA_ERR_UNSUPPORTED
 * (mlra_decode_simt covers more).
 * Returns MLRA_OK once the kernel is enqueued.
 */
MLRA_API mlra_status mlra_decode(const mlra_dims* dims, const void* q_lat, const void* q_rope,
                        const void* latent_cache, const void* rope_cache,
                        const int32_t* block_table, const int32_t* seqlens, float scale,
                        float out_scale, void* out, void* workspace, size_t workspace_bytes,
                        void* stream);

/*
 * The whole decode step in one launch: mlra_decode's attention and split
 * merge, then the per-branch W_UV up-projection and branch sum of its output
 * (what mlra_up_proj computes; "The Core Insight" section of the blog page:
 * each branch is up-projected by its own matrix and the branch outputs are
 * summed):
 *   y[n, h*d_h + j] = sum_b sum_k out[n,h,b,k] * w_uv[b][k][h*d_h + j]
 * Arguments as mlra_decode, plus
 *   w_uv  bf16 [branches, d_c, heads * d_h]
 *   d_h   64 or 128
 *   y     bf16 [batch, heads * d_h], written; device memory or pinned host
 *         memory the device can map
 * `out` is written exactly as mlra_decode writes it (the same bits).  After
 * the launch's merges the CTAs meet once (a bounded grid-wide wait, reported
 * as MLRA_ERR_DEVICE_TIMEOUT if it expires) and form the heads * d_h / 16
 * blocks of 16 output columns (CTA c takes blocks c, c + grid, ...) in fp32
 * on the warp-level tensor cores.
 * Supported: the shapes of mlra_decode with batch <= 64; other batches
 * return MLRA_ERR_UNSUPPORTED (use mlra_decode and mlra_up_proj).
 */
MLRA_API mlra_status mlra_decode_up_proj(const mlra_dims* dims, const void* q_lat, const void* q_rope,
                                         const void* latent_cache, const void* rope_cache,
                                         const int32_t* block_table, const int32_t* seqlens, float scale,
                                         float out_scale, void* out, const void* w_uv, int32_t d_h, void* y,
                                         void* workspace, size_t workspace_bytes, void* stream);

/*
 * The same operation as mlra_decode, computed by a split-KV kernel on the
 * CUDA cores (fp32 FMA) instead of the tensor cores: same arguments, same
 * workspace, same outputs within the stated tolerance.  It covers more
 * shapes (heads <= 64, d_c and d_r multiples of 8, branches * d_c <= 1024,
 * any page size) at a fraction of the speed, and serves as an independent
 * GPU statement of the kernel for cross-checks.
 */
MLRA_API mlra_status mlra_decode_simt(const mlra_dims* dims, const void* q_lat, const void* q_rope,
                             const void* latent_cache, const void* rope_cache,
                             const int32_t* block_table, const int32_t* seqlens, float scale,
                             float out_scale, void* out, void* workspace, size_t workspace_bytes,
                             void* stream);

/*
 * mlra_decode for callers that cannot allocate device memory.  (An interface
 * addition of this library; the pages describing the method have no
 * counterpart.)  Some callers cannot call cudaMalloc or own a workspace:
 * plugins that must not allocate from the host application's memory pools,
 * runtimes that have handed all device memory to their own allocator, and
 * serving loops that forbid allocation after start-up (cudaMalloc
 * synchronises the device and can fail under memory pressure).  This variant takes no
 * workspace: its scratch is a fixed 8 MiB array inside the library's device
 * image, held on every GPU that loads the library until the process exits.
 *   Arguments as mlra_decode, without workspace/workspace_bytes;
 *   device_status  optional int32 in device memory (4-byte aligned, may be
 *                  NULL): receives the call's device error code (0, or
 *                  MLRA_ERR_DEVICE_*), stream-ordered after the kernels.
 * Returns MLRA_ERR_WORKSPACE when the step needs more scratch than the
 * 8 MiB array holds (mlra_decode_workspace_bytes(dims, 0) > 8 MiB; call
 * mlra_decode with a workspace instead), otherwise what mlra_decode returns.
 * It allocates and frees nothing.  All calls on a device share the array:
 * calls that may overlap on the GPU race and corrupt each other's results,
 * so order them on one stream.  The array keeps the last call's contents;
 * every call first clears, stream-ordered, the parts that must start at zero
 * (the error word and its split counters), so no call inherits state from an
 * earlier one, not even from one whose kernel gave up on a bounded wait.
 * The first call in each CUDA context (on each device, and again after a
 * cudaDeviceReset) looks up the array's address with that context current;
 * make it before any stream capture starts.
 */
MLRA_API mlra_status mlra_decode_static_scratch(const mlra_dims* dims, const void* q_lat,
                             const void* q_rope, const void* latent_cache,
                             const void* rope_cache, const int32_t* block_table,
                             const int32_t* seqlens, float scale, float out_scale, void* out,
                             int32_t* device_status, void* stream);

/*
 * Per-branch W_UV up-projection followed by the branch sum ("The Core
 * Insight" section: each branch is up-projected by its own matrix and the
 * branch outputs are summed at the end):
 *   y[n, h*d_h + j] = sum_b sum_k out_lat[n,h,b,k] * w_uv[b][k][h*d_h + j]
 * fp32 accumulation, bf16 result.
 *   out_lat bf16 [batch, heads, branches, d_c]  (the output of mlra_decode)
 *   w_uv    bf16 [branches, d_c, heads * d_h]
 *   y       bf16 [batch, heads * d_h]           written; device memory or
 *           pinned host memory the device can map (the kernel then writes
 *           the result straight over PCIe, no separate copy)
 * Supported: branches * d_c in {64, 128, ..., 512} (a multiple of 64),
 * d_h in {64, 128}, any batch >= 1.
 */
MLRA_API mlra_status mlra_up_proj(int32_t batch, int32_t heads, int32_t branches, int32_t d_c, int32_t d_h,
                         const void* out_lat, const void* w_uv, void* y, void* stream);

/*
 * mlra_up_proj followed by an elementwise output gate ("Critical Insight:
 * The Value of 'Gating'" section of the blog page: a gate on the attention
 * output; its formula is lost in the page text and is read here as the
 * usual sigmoid gate on each output element):
 *   y[n, c] = sigmoid(gate[n, c]) * sum_b sum_k out_lat[n,h,b,k] * w_uv[b][k][c]
 * with c = h*d_h + j, applied to the fp32 sum before the bf16 rounding.
 *   gate  bf16 [batch, heads * d_h]  gate logits (device memory, not null)
 * Other arguments, shapes and errors as mlra_up_proj.
 */
MLRA_API mlra_status mlra_up_proj_gated(int32_t batch, int32_t heads, int32_t branches, int32_t d_c,
                                        int32_t d_h, const void* out_lat, const void* w_uv,
                                        const void* gate, void* y, void* stream);

/*
 * The decode pre-step for one new token per sequence: the work between the
 * layer's projections and mlra_decode.
 *  1. Query absorption: q_lat[n,h,b,k] = sum_j w_uk[b,h,j,k] * q_c[n,h,j]
 *     (each branch's key up-projection folded into the query, so that
 *     attention runs against the cached latents; "The Core Insight" section
 *     of the blog page: every branch has its own up-projection per head).
 *  2. Rotary embedding (RoFormer's definition; the pages do not specify one)
 *     of the RoPE query and the new token's RoPE key at its position
 *     p = seqlens[n] - 1: pair i = (x[2i], x[2i+1]) turns by the angle
 *     p * rope_base^(-2i/d_r) (the angle formed in turns in fp64, reduced to
 *     a fraction of a turn, its sine and cosine in fp32).
 *  3. Append: latent_cache[page][slot] = c_new[n], rope_cache[page][slot] =
 *     the rotated key, page = block_table[n][p / P], slot = p mod P.
 *   dims         as mlra_decode's (batch, heads, branches, d_c, d_r,
 *                page_size, max_pages_per_seq, num_pages)
 *   d_h          head dimension of q_c (a multiple of 8, at most 256)
 *   q_c          bf16 [batch, heads, d_h]             no-RoPE query per head
 *   q_r          bf16 [batch, heads, d_r]             RoPE query, unrotated
 *   w_uk         bf16 [branches, heads, d_h, d_c]     key up-projections
 *   c_new        bf16 [batch, branches, d_c]          the new token's latents
 *   kr_new       bf16 [batch, d_r]                    its RoPE key, unrotated
 *   seqlens      int32 [batch]  lengths including the new token
 *   block_table  int32 [batch, max_pages_per_seq]
 *   rope_base    e.g. 10000
 *   q_lat        bf16 [batch, heads, branches, d_c]   written (mlra_decode's q_lat)
 *   q_rope       bf16 [batch, heads, d_r]             written (mlra_decode's q_rope)
 *   latent_cache, rope_cache  one row per valid sequence written in place
 *   device_status  optional int32 (device, may be NULL): zeroed, then the
 *                first device-detected problem (MLRA_ERR_DEVICE_BAD_SEQLEN for
 *                seqlens[n] < 1 or beyond the block table,
 *                MLRA_ERR_DEVICE_BAD_INDEX for a page outside the pool); such
 *                a sequence's row is not written (its queries still are)
 * Requires d_c a multiple of 8, d_r even and at most 64, 16-byte aligned
 * arrays.  Allocates nothing; fp32 arithmetic (the absorption on the
 * warp-level tensor cores: bf16 products, fp32 sums), bf16 results.
 * The launch is a programmatic dependent of the preceding kernel in the
 * stream: its CTAs may start while that kernel runs and read w_uk, seqlens
 * and block_table then (every other input only after it has finished), so
 * these three must not be written by that kernel.
 */
MLRA_API mlra_status mlra_prepare(const mlra_dims* dims, int32_t d_h, const void* q_c, const void* q_r,
                                  const void* w_uk, const void* c_new, const void* kr_new,
                                  const int32_t* seqlens, const int32_t* block_table, float rope_base,
                                  void* q_lat, void* q_rope, void* latent_cache, void* rope_cache,
                                  int32_t* device_status, void* stream);

/*
 * Branch-sharded tensor parallelism ("The Core Insight" section of the blog
 * page: the branches can be placed on different GPUs, so each GPU reads only
 * its own branches' latents plus the shared RoPE key -- 1.5 d_h per token
 * against MLA's 4.5 d_h under 4-way tensor parallelism).  Rank r of a group
 * of `world` ranks holds branches [r*B/world, (r+1)*B/world): their slice of
 * the latent cache, q_lat and W_UV, plus a full copy of the RoPE cache and
 * q_rope.  Each rank runs mlra_decode on its branches (with the global
 * out_scale), then mlra_up_proj_allreduce, which multiplies its branches and
 * sums the ranks' products, so that every rank ends with the full y.
 *
 * The cross-rank sum runs inside the up-projection kernel over an exchange
 * region per rank, device memory that every rank maps: each rank stores its
 * fp32 partial products into every rank's region and raises a flag there;
 * each rank waits (bounded) for all flags on its own region and adds the
 * ranks' partials in rank order, so all ranks' y are bit-identical.
 */

/* Size in bytes of one rank's exchange region for these (per-rank) sizes;
 * 0 if the sizes are invalid.  `branches` is the rank's branch count. */
MLRA_API size_t mlra_exchange_bytes(int32_t batch, int32_t heads, int32_t branches, int32_t d_c,
                                    int32_t d_h, int32_t world);

#define MLRA_IPC_HANDLE_BYTES 64

/*
 * Allocates a zeroed exchange region of `bytes` on the current device
 * (cudaMalloc; released with mlra_exchange_free) and, when `ipc_handle` is
 * not NULL, writes the MLRA_IPC_HANDLE_BYTES-byte handle through which the
 * other processes of the group map it.  Synchronises the device, so the
 * zeroing is complete on return.  Every rank must hold its zeroed region
 * before any rank makes its first mlra_up_proj_allreduce call (exchange the
 * handles through a collective that all ranks enter after this returns).
 */
MLRA_API mlra_status mlra_exchange_alloc(size_t bytes, void** region, void* ipc_handle);

/* Maps another process's region from its handle (peer access enabled
 * lazily); unmap with mlra_exchange_close. */
MLRA_API mlra_status mlra_exchange_open(const void* ipc_handle, void** region);
MLRA_API mlra_status mlra_exchange_close(void* region);
MLRA_API mlra_status mlra_exchange_free(void* region);

/* Zeroes a region (asynchronously on `stream`).  After a timeout the ranks'
 * call counters disagree.  To start afresh: every rank synchronises its
 * device, the group meets at a barrier (no kernel can still write into a
 * region), every rank zeroes its own region and synchronises, and the group
 * meets again before the next call. */
MLRA_API mlra_status mlra_exchange_reset(void* region, size_t bytes, void* stream);

/*
 * Branch-sharded up-projection with the cross-rank branch sum:
 *   y[n, c] = sigmoid(gate[n, c])? * sum_{ranks s} sum_{b in s} sum_k out_lat_s[n,h,b,k] * w_uv_s[b][k][c]
 *   out_lat, w_uv   this rank's branches (`branches` of them), layouts as
 *                   mlra_up_proj
 *   gate            optional bf16 [batch, heads * d_h] (NULL: no gate); the
 *                   same values on every rank
 *   y               bf16 [batch, heads * d_h], the full sum, on every rank
 *   regions         DEVICE array of `world` pointers: rank s's exchange region
 *                   as this device addresses it (its own, or mapped with
 *                   mlra_exchange_open); each of size
 *                   mlra_exchange_bytes(batch, heads, branches, d_c, d_h, world)
 *   rank            this rank (0 <= rank < world <= 8)
 *   ranks_in_launch 1 normally.  k > 1 computes ranks rank .. rank + k - 1
 *                   in one launch on this device, with their out_lat, w_uv
 *                   and y stacked along the leading dimension ([k, ...]);
 *                   for checking the exchange on one device
 *   device_status   optional int32 (device, may be NULL): MLRA_ERR_DEVICE_TIMEOUT
 *                   is recorded if another rank's partial does not arrive
 *                   within wait_limit_ns (the tile's y is then written as zeros)
 * Every rank must make the same sequence of calls with the same sizes.  The
 * whole grid must fit on the device at once (a waiting tile must never hold
 * the SM that another tile needs): MLRA_ERR_UNSUPPORTED otherwise.  Shape
 * limits as mlra_up_proj.
 */
MLRA_API mlra_status mlra_up_proj_allreduce(int32_t batch, int32_t heads, int32_t branches, int32_t d_c,
                                            int32_t d_h, const void* out_lat, const void* w_uv,
                                            const void* gate, void* y, void* const* regions, int32_t world,
                                            int32_t rank, int32_t ranks_in_launch, int32_t* device_status,
                                            uint64_t wait_limit_ns, void* stream);

/*
 * Copies `count` (1..8) byte ranges, dst[k] <- src[k] (bytes[k] bytes each),
 * in one kernel launch whose SMs issue the loads and stores.  Every pointer
 * is device memory, managed memory or pinned host memory the device can map
 * (cudaHostAlloc / cudaMallocHost, or registered with cudaHostRegister),
 * 16-byte aligned; no destination may overlap any range.  Host pointers are
 * translated to their device addresses here.  For the host-to-device leg of
 * a serving step: a few small input tensors cross PCIe in one launch instead
 * of one DMA copy (and its setup latency) each.  Pageable host memory is
 * rejected (MLRA_ERR_INVALID_ARG).  Asynchronous on `stream`.
 */
MLRA_API mlra_status mlra_copy_ranges(int32_t count, const void* const* src, void* const* dst,
                                      const uint64_t* bytes, void* stream);

/*
 * Synchronises `stream`, returns the first device-side error code recorded
 * in `workspace` since the last read (MLRA_OK if none) and resets it to 0.
 * When the code is MLRA_ERR_DEVICE_TIMEOUT it also clears the workspace's
 * split counters (a kernel that gave up may have left them set), so the
 * workspace serves the next call.  Returns MLRA_ERR_CUDA if the
 * synchronisation or copy fails.
 */
MLRA_API mlra_status mlra_read_device_error(void* workspace, void* stream);

/* Static, human-readable name of a status code. */
MLRA_API const char* mlra_status_string(mlra_status status);

/*
 * The split-KV work partition mlra_decode uses, written for inspection.
 * Sequence n has tiles_n = ceil(L_n / 128) token tiles (0 if L_n is
 * invalid).  Work is counted in cost units: 8 per tile plus 8 per valid
 * sequence, placed after its last tile, for the per-sequence setup and
 * epilogue.  Sequence n spans [cum_n, cum_n + 8 * tiles_n + 8) and its tile t
 * starts at cum_n + 8 * t; with chunk = max(ceil(total / num_ctas), 8), CTA c
 * owns the tiles that start in [c * chunk, (c + 1) * chunk).  The ranges are
 * contiguous in the list of all tiles.
 *   plan_out int32 device [num_ctas * 4 + batch * 2]:
 *     per CTA c:  first tile (global index), end tile (global), first
 *                 sequence, last sequence touched (0, 0, -1, -1 when the
 *                 CTA owns no tile)
 *     per seq n:  number of CTAs covering it (0 if invalid), first such CTA
 * Returns after enqueueing one small kernel.
 */
MLRA_API mlra_status mlra_decode_plan(int32_t batch, int32_t page_size, int32_t max_pages_per_seq,
                             const int32_t* seqlens, int32_t num_ctas, int32_t* plan_out,
                             void* stream);

#ifdef __cplusplus
}
#endif

#endif /* MLRA_H */
