// decode_tc.cu -- split-KV MLRA decode on the sm_100a tensor cores.
//
// Method ("MLRA: Breaking the Sharding Bottleneck in Latent Attention",
// wispaper.ai blog, section "The Core Insight: Sum of Branches, Not Sum of
// Keys"): every latent branch b is attended independently,
//   s_t = scale * (q_lat[h,b] . c_b[t] + q_rope[h] . k_r[t]),
//   o[h,b] = sum_t softmax_t(s)_t c_b[t]       (values = the same latents),
// with one RoPE key per token shared by all branches and heads.  The
// decoding cost is the HBM -> SRAM movement of the cache at every step
// (abstract of "Multi-Head Low-Rank Attention"), so the kernel streams each
// token's latent and RoPE row through shared memory exactly once.
//
// Organisation (one persistent CTA per SM, 352 threads):
//   warp 0     TMA producer: per 128-token tile, the RoPE tile and, per
//              "pair" of 64-column chunks (128 latent columns), the paged
//              latent rows (one 2-D box per page) into a ring of stages.
//   warp 1     score MMA issuer (one thread) and TMEM owner:
//                S^T_b[t, h]  = C_b[t, :] . Q_b[h, :] + K_r[t, :] . Q_r[h, :]
//                               M = 128 tokens, N = 16 (or 32) heads, K = d_c + d_r
//   warp 6     output MMA issuer (one thread):
//                O^T_b[k, h] += C_b[:, k]^T . P_b[:, h]
//                               M = 128 latent columns, N = 16 (or 32) heads, K = 128 tokens
//              (the same shared-memory tile is the K-major A operand of the
//              score MMA and the MN-major A operand of the output MMA).  An
//              MMA issue stalls the issuing warp for about one MMA's duration,
//              so two issuers keep the tensor pipe busy while either waits.
//   warps 2-5  softmax and epilogue, the first half of the tile's heads, and
//   warps 7-10 the same for the second half (two warps per scheduler, so that
//              each hides the other's latency): a thread owns one token of
//              the tile (a TMEM lane); scores are base-2 logits; each (head, branch) has
//              its own running max, rescaled only when a score exceeds it by
//              more than 2^8 (then the exact column max is reduced and the
//              TMEM accumulator is rescaled); P is written as bf16 to shared
//              memory; at the end of a sequence's range the row sums are
//              reduced and the normalised output (or a split partial with its
//              log-sum-exp) is written.
// Every wait is bounded: a wait that expires records
// MLRA_ERR_DEVICE_TIMEOUT, and the CTA drains its copies and exits.
#include <cudaTypedefs.h>

#include <cstddef>

#include "common.cuh"
#include "kernels.h"
#include "sm100.cuh"

namespace mlra {
namespace {

using namespace sm100;

// Heads per MMA tile (the MMA's N): 16, or 32 when a step has more than 16
// heads; each softmax warpgroup takes half of them.
constexpr int kT = kTileTokens;     // tokens per tile = MMA M
constexpr int kThreads = 352;
constexpr float kRescaleLog2 = 8.0f;
constexpr int kSmemLimit = 232448;  // max dynamic shared memory per CTA on sm_100

template <int NB, int DC, int DR, int HP_>
struct Cfg {
    static constexpr int HP = HP_;                          // heads per tile (MMA N)
    static constexpr int W = NB * DC;                       // latent elements per token
    static constexpr int NCHUNK = W / 64;                   // 64-column (128-byte) chunks
    // A step is the unit of the MMA <-> softmax pipeline: SBR branches whose
    // latents are PPS "pairs" (128 latent columns each); a pair holds BPP
    // branches (two when DC = 64).
    // one pair per step: the ring must hold two steps in flight plus the
    // copies ahead of them, so steps stay as small as the pair layout allows
    static constexpr int SBR = DC >= 128 ? 1 : 128 / DC;           // branches per step
    static constexpr int BPP = DC >= 128 ? 1 : 128 / DC;            // branches per pair
    static constexpr int PPS = SBR * DC / 128 > 0 ? SBR * DC / 128 : 1;  // pairs per step
    static constexpr int NPAIR = W / 128;                           // pairs per tile
    static constexpr int NSTEP = NB / SBR;                          // steps per tile
    static constexpr int CHUNK_BYTES = kT * 128;            // 16 KB
    static constexpr int PAIR_BYTES = 2 * CHUNK_BYTES;      // 32 KB
    static constexpr int ROPE_ROW = DR * 2;                 // 128 or 64 bytes
    static constexpr int ROPE_BYTES = kT * ROPE_ROW;
    static constexpr int Q_CHUNK_BYTES = HP * 128;          // [HP heads x 64 elements]
    static constexpr int Q_BYTES = NCHUNK * Q_CHUNK_BYTES;
    static constexpr int QR_BYTES = HP * ROPE_ROW;                  // [HP heads x d_r]
    static constexpr int QR_SPAN = (QR_BYTES + 1023) / 1024 * 1024;  // keeps the next region aligned
    static constexpr int P_BRANCH_BYTES = kT * HP * 2;      // 4 KB per 16 heads
    static constexpr int P_BYTES = SBR * P_BRANCH_BYTES;   // one P slot (a step)
    static constexpr int MISC_BYTES = HP == 16 ? 4096 : 8192;
    static constexpr int QSET_BYTES = Q_BYTES + QR_SPAN;  // one sequence's queries
    // Pipeline depths: NSP steps may be between their score MMA and their
    // output MMA at once (S slots in TMEM, P slots in shared memory); NROPE
    // RoPE tiles are in flight, so the producer never waits for a tile's RoPE
    // score before it loads the next tile (more slots when a tile is only one
    // or two pairs of latents, so that the RoPE ring is not the shorter one);
    // one query set (a sequence change waits for the previous range's score
    // MMAs, rare: at most two per CTA).  The RoPE score of tile t lives in
    // TMEM slot t % NRS: the score MMA of a tile's first step waits for the
    // output MMA NSP steps back, so the softmax has read every RoPE score
    // more than ceil(NSP / NSTEP) tiles back.
    static constexpr int NSP = NPAIR == 1 ? 4 : 3;
    // (one slot when a tile is four pairs of 32-head steps: a tile's RoPE
    // score is taken at its first step, long before its last pair lands, and
    // the wider queries and probabilities leave no room for a second)
    static constexpr int NROPE = NPAIR == 1 ? 4 : NPAIR == 2 ? 3 : HP == 16 ? 2 : 1;
    static constexpr int NRS = (NSP + NSTEP - 1) / NSTEP > 2 ? (NSP + NSTEP - 1) / NSTEP : 2;
    static constexpr int FIXED = NROPE * ROPE_BYTES + QSET_BYTES + NSP * P_BYTES + MISC_BYTES;
    static constexpr int NSTAGE_FIT = (kSmemLimit - 1024 - FIXED) / PAIR_BYTES;
    static constexpr int NSTAGE = NSTAGE_FIT > 8 ? 8 : NSTAGE_FIT;
    // shared-memory offsets from a 1024-byte aligned base
    static constexpr int OFF_PAIR = 0;
    static constexpr int OFF_ROPE = OFF_PAIR + NSTAGE * PAIR_BYTES;  // RoPE slot r at + r * ROPE_BYTES
    static constexpr int OFF_Q = OFF_ROPE + NROPE * ROPE_BYTES;
    static constexpr int OFF_QR = OFF_Q + Q_BYTES;
    static constexpr int OFF_P = OFF_Q + QSET_BYTES;                  // P slot k at + k * P_BYTES
    static constexpr int OFF_MISC = OFF_P + NSP * P_BYTES;
    static constexpr int SMEM_BYTES = OFF_MISC + MISC_BYTES + 1024;  // + alignment slack
    // TMEM columns: O blocks first, then two S slots, then two slots of the
    // RoPE score shared by all branches of a tile
    static constexpr int O_BLOCKS = NPAIR * BPP;
    static constexpr int S_COL0 = O_BLOCKS * HP;
    static constexpr int S_SLOT_COLS = SBR * HP;
    static constexpr int R_COL0 = S_COL0 + NSP * S_SLOT_COLS;
    static constexpr int TMEM_COLS = R_COL0 + NRS * HP <= 128 ? 128 : R_COL0 + NRS * HP <= 256 ? 256 : 512;
    static_assert(NB % SBR == 0 && (SBR * DC) % 128 == 0, "branches must fill whole steps and pairs");
    static_assert(NSTEP * PPS == NPAIR, "step / pair bookkeeping");
    static_assert(NSTAGE >= PPS, "a step's pairs must fit the stage ring");
    static_assert(R_COL0 + NRS * HP <= TMEM_COLS, "TMEM budget");
    static_assert(HP == 16 || HP == 32, "heads per tile");
    static_assert(SMEM_BYTES <= kSmemLimit, "shared-memory budget");
    static_assert(OFF_QR + QR_BYTES <= OFF_P && OFF_Q + Q_BYTES <= OFF_QR &&
                  OFF_P + NSP * P_BYTES <= OFF_MISC && QSET_BYTES % 1024 == 0 && ROPE_BYTES % 1024 == 0,
                  "shared-memory regions must not overlap");
    static_assert(DR == 32 || DR == 64, "RoPE width");
};

// Barriers and scratch in the MISC region (HP heads per tile, at most 4 branches).
template <int NSTAGE, int HP>
struct Misc {
    uint64_t pair_full[NSTAGE];
    uint64_t pair_empty[NSTAGE];
    uint64_t rope_full[4];  // tile t in RoPE slot t % NROPE: its RoPE keys are in shared memory
    uint64_t rope_empty[4];  // its RoPE score MMA finished
    uint64_t s_full[4];   // step g in slot g % NSP: its scores are in TMEM
    uint64_t p_full[4];   // its probabilities are in shared memory
    uint64_t p_empty[4];  // its output MMA finished (S and P slots free, O up to date)
    uint64_t q_full;      // sequence range r (phase r & 1): its queries are in shared memory
    uint64_t q_empty;     // the score MMAs of a range with a successor have finished
    uint64_t drain[2];
    uint64_t merge_full;  // the split merge's bulk copies have landed
    uint32_t tmem_base;
    int abort_flag;
    int plan[4];      // -, chunk, first sequence, its cost start
    int last_seg[4];  // this CTA's last sequence range: sequence, cost start, tiles (-1: none), c1 merges
    int merge_flag;   // merge: bit 0 a split met a bad page, bit 1 a wait expired
    float red_max[4][2 * HP];  // [quadrant][step branch, head]: column maxima of a rescale
    float red_sum[4][4 * HP];  // [quadrant][group, branch, head]: denominator partials
    alignas(16) float m_run[4 * HP];  // running max per (branch, head), base-2 logits; read as float4
    float inv_l[4 * HP];              // 1 / softmax denominator per (branch, head), epilogue only
};

template <int NSTAGE, int HP>
constexpr bool m_run_aligned() {
    using M = Misc<NSTAGE, HP>;
    return offsetof(M, m_run) % 16 == 0;
}
static_assert(m_run_aligned<5, 16>() && m_run_aligned<4, 16>() && m_run_aligned<6, 16>() &&
                  m_run_aligned<2, 32>() && m_run_aligned<3, 32>() && m_run_aligned<4, 32>(),
              "float4 access to m_run");

struct Maps {
    CUtensorMap lat;   // latent cache rows [pages * P][W]
    CUtensorMap rope;  // RoPE cache rows [pages * P][d_r]
    CUtensorMap q;     // q_lat [batch][H][W]: a 16-head box per 64 columns (heads >= H read as 0)
    CUtensorMap qr;    // q_rope [batch][H][d_r]
};

// Head groups.  The MMAs take one tile of HP heads (N = 16, or 32 when there
// are more than 16 heads); more heads run as ceil(H / HP) groups side by
// side.  CTA g * cpg + i (cpg = grid / groups) runs window i of one cost plan
// over cpg windows for heads [HP g, HP g + HP), so the groups stream the same
// tokens at about the same time and every read of a cache line after the
// first hits L2 (the latents are shared by all heads).  Each group has its own
// partial slots (a block of cpg + batch) and split counters (a block of
// batch); CTAs past groups * cpg only take part in the fused up-projection.
struct HeadGroup {
    int ci, cpg;   // window of this CTA, windows (CTAs) per group
    int h0, hn;    // first head of the group, heads in it
    int slot0;     // first partial slot of the group
    int cnt0;      // first split counter of the group
    bool idle;     // no group: beyond groups * cpg
};

template <int HP>
__device__ __forceinline__ HeadGroup head_group(const DecodeArgs& a) {
    constexpr int kHP = HP;
    HeadGroup hg;
    const int groups = (a.heads + HP - 1) / HP;
    hg.cpg = a.num_ctas / groups;
    const int g = (int)blockIdx.x / hg.cpg;
    hg.ci = (int)blockIdx.x - g * hg.cpg;
    hg.idle = g >= groups;
    hg.h0 = g * kHP;
    hg.hn = hg.idle ? 0 : min(kHP, a.heads - hg.h0);
    hg.slot0 = g * (hg.cpg + a.batch);
    hg.cnt0 = g * a.batch;
    return hg;
}

// 2^x on the special-function unit (ex2.approx, flush-to-zero: results below
// 2^-126 become 0, which only affects probabilities that are negligible).
__device__ __forceinline__ float fast_exp2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// Max over the 32 lanes of a warp of each of 16 values, reduce-scattered:
// the result for column c ends up in lanes 2c and 2c+1.  16 shuffles.
__device__ __forceinline__ float warp_colmax16(const float (&v)[16], int lane) {
    float a8[8], a4[4], a2[2];
#pragma unroll
    for (int i = 0; i < 8; ++i) {  // lanes with bit 4 keep columns 8..15
        const bool hi = lane & 16;
        const float keep = hi ? v[i + 8] : v[i], send = hi ? v[i] : v[i + 8];
        a8[i] = fmaxf(keep, __shfl_xor_sync(0xffffffffu, send, 16));
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const bool hi = lane & 8;
        const float keep = hi ? a8[i + 4] : a8[i], send = hi ? a8[i] : a8[i + 4];
        a4[i] = fmaxf(keep, __shfl_xor_sync(0xffffffffu, send, 8));
    }
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        const bool hi = lane & 4;
        const float keep = hi ? a4[i + 2] : a4[i], send = hi ? a4[i] : a4[i + 2];
        a2[i] = fmaxf(keep, __shfl_xor_sync(0xffffffffu, send, 4));
    }
    const bool hi = lane & 2;
    const float keep = hi ? a2[1] : a2[0], send = hi ? a2[0] : a2[1];
    const float a1 = fmaxf(keep, __shfl_xor_sync(0xffffffffu, send, 2));
    return fmaxf(a1, __shfl_xor_sync(0xffffffffu, a1, 1));
}

// Max over the 32 lanes of a warp of each of 8 values, reduce-scattered:
// the result for column c ends up in lanes 4c..4c+3.  9 shuffles.
__device__ __forceinline__ float warp_colmax8(const float (&v)[8], int lane) {
    float a4[4], a2[2];
#pragma unroll
    for (int i = 0; i < 4; ++i) {  // lanes with bit 4 keep columns 4..7
        const bool hi = lane & 16;
        const float keep = hi ? v[i + 4] : v[i], send = hi ? v[i] : v[i + 4];
        a4[i] = fmaxf(keep, __shfl_xor_sync(0xffffffffu, send, 16));
    }
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        const bool hi = lane & 8;
        const float keep = hi ? a4[i + 2] : a4[i], send = hi ? a4[i] : a4[i + 2];
        a2[i] = fmaxf(keep, __shfl_xor_sync(0xffffffffu, send, 8));
    }
    const bool hi = lane & 4;
    const float keep = hi ? a2[1] : a2[0], send = hi ? a2[0] : a2[1];
    float a1 = fmaxf(keep, __shfl_xor_sync(0xffffffffu, send, 4));
    a1 = fmaxf(a1, __shfl_xor_sync(0xffffffffu, a1, 2));
    return fmaxf(a1, __shfl_xor_sync(0xffffffffu, a1, 1));
}

// The same for a softmax group's N = 8 or 16 heads: column c in lanes
// [c 32 / N, (c + 1) 32 / N).
template <int N>
__device__ __forceinline__ float warp_colmax(const float (&v)[N], int lane) {
    if constexpr (N == 8) return warp_colmax8(v, lane);
    else return warp_colmax16(v, lane);
}

// TMEM loads and stores of a softmax group's N = 8 or 16 columns.
template <int N>
__device__ __forceinline__ void tmem_ld_cols(uint32_t taddr, float (&v)[N]) {
    if constexpr (N == 8) tmem_ld8(taddr, v);
    else tmem_ld16(taddr, v);
}
template <int N>
__device__ __forceinline__ void tmem_st_cols(uint32_t taddr, const float (&v)[N]) {
    if constexpr (N == 8) tmem_st8(taddr, v);
    else tmem_st16(taddr, v);
}

// Sum over the 32 lanes of a warp of each of N values (N = 16, 32, 64, 128),
// reduce-scattered: afterwards, for N >= 32, lane L holds in v[r]
// (r < N/32) the warp total of value N/32*L + r; for N = 16, lanes 2c and
// 2c+1 hold in v[0] the total of value c.  N - 1 + (N < 32) shuffles.
template <int LIVE, int O, int N>
__device__ __forceinline__ void warp_sum_scatter(float (&v)[N], int lane) {
    if constexpr (O >= 1) {
        if constexpr (LIVE >= 2) {
            constexpr int H = LIVE / 2;
#pragma unroll
            for (int i = 0; i < H; ++i) {
                const bool hi = lane & O;
                const float keep = hi ? v[i + H] : v[i], send = hi ? v[i] : v[i + H];
                v[i] = keep + __shfl_xor_sync(0xffffffffu, send, O);
            }
            warp_sum_scatter<H, O / 2, N>(v, lane);
        } else {
            v[0] += __shfl_xor_sync(0xffffffffu, v[0], O);
            warp_sum_scatter<1, O / 2, N>(v, lane);
        }
    }
}

struct bool4_t {
    bool x, y, z, w;
};

template <int DR>
__device__ __forceinline__ uint64_t rope_desc(uint32_t addr) {
    return DR == 64 ? smem_desc(addr, 16, 1024, kLayoutSw128) : smem_desc(addr, 16, 512, kLayoutSw64);
}

// The sequence walk every role performs identically: the next sequence n
// (cost start cum) with tiles [tb, te) in this CTA's cost window [A0, A1).
// next_len holds seqlens[n], loaded one range ahead (first_len starts it).
// The caller advances past the range with finish_segment.
__device__ __forceinline__ int first_len(const DecodeArgs& a, int n) {
    return n < a.batch ? __ldg(a.seqlens + n) : 0;
}

__device__ __forceinline__ bool next_segment(const DecodeArgs& a, int& n, int& cum, int A0, int A1,
                                             int& L, int& tiles, int& tb, int& te, int& next_len) {
    while (n < a.batch && cum < A1) {
        L = next_len;
        next_len = n + 1 < a.batch ? __ldg(a.seqlens + n + 1) : 0;
        tiles = seq_tiles(L, a.page_size, a.max_pages);
        if (tiles > 0) {
            tb = first_tile_at(cum, tiles, A0);
            te = first_tile_at(cum, tiles, A1);
            if (tb < te) return true;
            cum += tiles * kTileCost + kSeqCost;
        }
        ++n;
    }
    return false;
}

__device__ __forceinline__ void finish_segment(int& n, int& cum, int tiles) {
    cum += tiles * kTileCost + kSeqCost;
    ++n;
}

// The sequence of the CTA's next range after sequence n (cost start cum,
// `tiles` tiles) in its window [A0, A1), or -1 if n is its last.
__device__ __forceinline__ int next_range_seq(const DecodeArgs& a, int n, int cum, int tiles, int A0, int A1) {
    int c = cum + tiles * kTileCost + kSeqCost;
    for (int m = n + 1; m < a.batch && c < A1; ++m) {
        const int t = seq_tiles(__ldg(a.seqlens + m), a.page_size, a.max_pages);
        if (t > 0) {
            if (first_tile_at(c, t, A0) < first_tile_at(c, t, A1)) return m;
            c += t * kTileCost + kSeqCost;
        }
    }
    return -1;
}

// One sequence's queries (latent and RoPE, the 16 head rows from h0; rows
// past the last head read as zero) into the query buffer, completing `full`;
// issued by one thread.
template <class C>
__device__ __forceinline__ void load_queries(const Maps& maps, uint8_t* sm, uint64_t& full, int seq, int h0) {
    uint8_t* qd = sm + C::OFF_Q;
    mbar_arrive_expect_tx(&full, C::Q_BYTES + C::QR_BYTES);
    for (int c = 0; c < C::NCHUNK; ++c) tma_load_3d(qd + c * C::Q_CHUNK_BYTES, &maps.q, c * 64, h0, seq, &full);
    tma_load_3d(qd + C::Q_BYTES, &maps.qr, 0, h0, seq, &full);
}

// End of the kernel, all threads: the merge of split sequences.
//
// Sequence n with S > 1 splits (CTAs c0..c1) is merged by the CTAs whose
// range ends in it: c0..c1-1 always, c1 when n is also its last sequence.
// Each such CTA waits until all S splits have counted their partials into
// seq_cnt[n], then combines rows [i R / G, (i+1) R / G) of the R = NB * DC
// (branch, latent column) rows, i = c - c0, G the group size:
//   o = out_scale * sum_s w_s o_s / sum_s w_s,  w_s = 2^(lse_s - max_s lse_s)
// per (branch, head) -- the log-sum-exp merge of independent softmax
// partitions, summed in split order.  The S log-sum-exp rows (consecutive
// slots) and each split's slice of partial rows (contiguous) arrive by bulk
// copies.  A CTA leaves the count as soon as its wait is over (the count
// guards only the wait; the partials stay in place until the next launch),
// and the last of the S + G counts returns seq_cnt[n] to zero.  The arithmetic
// is laid out for latency: every thread loads its values for up to 8 splits
// at once before combining them.
template <int NB, int DC, int HP>
__device__ __forceinline__ void merge_tail(const DecodeArgs& a, const HeadGroup& grp, int n, int cum, int tiles,
                                           bool c1_member, int chunk, float* w_s, int* flag, uint64_t* bar) {
    constexpr int kHP = HP;
    constexpr int QD = HP / 4;    // head quads of a row
    constexpr int HB = NB * kHP;  // (branch, head) columns of a split's log-sum-exp row
    constexpr int R = NB * DC;    // (branch, latent column) rows
    const int tid = threadIdx.x;
    const int H = a.heads;

    if (n < 0) return;
    int c0, c1;
    seq_owners(cum, tiles, chunk, &c0, &c1);
    const int S = c1 - c0 + 1;
    if (S == 1) return;  // written by the epilogue
    // c1 belongs to the group when no later tile is its own (the next valid
    // sequence starts in a later window); worked out at the range's start
    const int G = c1_member ? S : S - 1;
    const int gi = grp.ci - c0;  // 0 <= gi < G: n is this CTA's last sequence
    const int r0 = (int)((long long)gi * R / G), r1 = (int)((long long)(gi + 1) * R / G);
    const int rows = r1 - r0;
    const size_t slot_c0 = (size_t)grp.slot0 + c0 + n;  // the partial slot of split 0
    int* cnt = a.seq_cnt + grp.cnt0 + n;
    float* part_s = w_s + S * HB;  // [S][rows][16 heads]
    // wait until every split of n has counted its partials
    if (tid == 0) {
        const uint64_t t0 = globaltimer_ns();
        bool ok = true;
        while (ld_acquire_gpu(cnt) < S) {
            if (globaltimer_ns() - t0 > 2000000000ull) {
                ok = false;
                break;
            }
            __nanosleep(32);
        }
        if (!ok) {
            *flag = 2;
            record_error(a.err, MLRA_ERR_DEVICE_TIMEOUT);
        }
    }
    __syncthreads();
    if (*flag & 2) return;
    int departed = 0;
    if (tid < 32) {
        // the partials were published by generic stores and acquired by
        // thread 0 (ordered before this warp by the barrier); the copies read
        // them through the async proxy
        fence_proxy_async_global();
        if (tid == 0) {
            mbar_arrive_expect_tx(bar, (uint32_t)(S * HB + S * rows * kHP) * 4u);
            bulk_load(w_s, a.lse_part + slot_c0 * HB, (uint32_t)(S * HB) * 4u, bar);
        }
        __syncwarp();
        if (rows > 0)
            for (int sp = tid; sp < S; sp += 32)
                bulk_load(part_s + (size_t)sp * rows * kHP, a.o_part + ((slot_c0 + sp) * R + r0) * kHP,
                          (uint32_t)rows * kHP * 4u, bar);
        // this CTA leaves the count (its result is needed only at the end)
        if (tid == 0) departed = atomicAdd(cnt, 1);
    }
    if (!mbar_wait(bar, 0)) {
        // never expected: report it, and give the copies a last bounded
        // chance to land before this CTA's shared memory goes away
        if (tid == 0) record_error(a.err, MLRA_ERR_DEVICE_TIMEOUT);
        mbar_wait(bar, 0, 200000000ull);
        return;
    }
    // weights out_scale * 2^(lse - max) / sum, two threads per (branch, head)
    // column, each over every other split, eight splits' values in flight
    static_assert(2 * HB <= kThreads && HB % 16 == 0, "two threads per column in whole warps");
    if (tid < 2 * HB) {
        const int col = tid >> 1, half = tid & 1;
        float mx = -INFINITY;
        bool bad = false;
        for (int s0 = half; s0 < S; s0 += 16) {
            float v[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) v[j] = s0 + 2 * j < S ? w_s[(s0 + 2 * j) * HB + col] : -INFINITY;
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                bad |= v[j] == bad_split_marker();
                if (v[j] != bad_split_marker()) mx = fmaxf(mx, v[j]);
            }
        }
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
        bad = __shfl_xor_sync(0xffffffffu, (int)bad, 1) != 0 || bad;
        float sum = 0.f;
        for (int s0 = half; s0 < S; s0 += 16) {
            float v[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) v[j] = s0 + 2 * j < S ? w_s[(s0 + 2 * j) * HB + col] : -INFINITY;
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                v[j] = bad ? 0.f : fast_exp2(v[j] - mx);
                sum += v[j];
            }
#pragma unroll
            for (int j = 0; j < 8; ++j)
                if (s0 + 2 * j < S) w_s[(s0 + 2 * j) * HB + col] = v[j];
        }
        sum += __shfl_xor_sync(0xffffffffu, sum, 1);
        const float norm = bad ? 0.f : a.out_scale / sum;
        for (int s0 = half; s0 < S; s0 += 16) {
#pragma unroll
            for (int j = 0; j < 8; ++j)
                if (s0 + 2 * j < S) w_s[(s0 + 2 * j) * HB + col] *= norm;
        }
        if (bad && half == 0 && col % kHP < grp.hn) atomicOr(flag, 1);
    }
    __syncthreads();
    const bool bad = *flag & 1;
    if (bad && tid == 0) record_error(a.err, MLRA_ERR_DEVICE_BAD_INDEX);

    // items (row, head quad), quads fastest: conflict-free 16-byte reads; the
    // weighted sum over the splits in split order, eight splits' loads at once
    for (int e = tid; e < rows * QD; e += kThreads) {
        const int lr = e / QD, q = e % QD, row = r0 + lr;
        const int b = row / DC, k = row % DC;
        const float* w = w_s + b * kHP + 4 * q;
        const float* src = part_s + lr * kHP + 4 * q;
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int s0 = 0; s0 < S; s0 += 8) {
            float4 v[8], wv[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const bool in = s0 + j < S;
                v[j] = in ? *reinterpret_cast<const float4*>(src + (size_t)(s0 + j) * rows * kHP)
                          : make_float4(0.f, 0.f, 0.f, 0.f);
                wv[j] = in ? *reinterpret_cast<const float4*>(w + (s0 + j) * HB) : make_float4(0.f, 0.f, 0.f, 0.f);
            }
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                acc.x = fmaf(wv[j].x, v[j].x, acc.x);
                acc.y = fmaf(wv[j].y, v[j].y, acc.y);
                acc.z = fmaf(wv[j].z, v[j].z, acc.z);
                acc.w = fmaf(wv[j].w, v[j].w, acc.w);
            }
        }
        if (bad) acc = make_float4(0.f, 0.f, 0.f, 0.f);
        __nv_bfloat16* dst = a.out + (((size_t)n * H + grp.h0) * NB + b) * DC + k;
        const float v4[4] = {acc.x, acc.y, acc.z, acc.w};
#pragma unroll
        for (int j = 0; j < 4; ++j)
            if (4 * q + j < grp.hn) dst[(size_t)(4 * q + j) * NB * DC] = to_bf16(v4[j]);
    }
    if (tid == 0 && departed == S + G - 1) *cnt = 0;
}

// ------------------------------------------------------------------ fused up-projection
// The fused step (mlra_decode_up_proj): after the launch's merges, CTA c
// computes the 16 output columns [16 cb, 16 cb + 16) of each column block
// cb = c, c + grid, ... below H d_h / 16 of
//   y[n, h d_h + j] = sum_b sum_k out[n, h, b, k] W_UV[b][k][h d_h + j]
// for every sequence n: the per-branch up-projection summed over the
// branches is one K = B d_c reduction ("The Core Insight" section of the
// wispaper.ai MLRA page: each branch is up-projected by its own matrix and
// the branch outputs are summed).  Every CTA counts itself into a grid
// counter once its merge duty is done (the spare word after the split
// counters); the up-projection CTAs wait (bounded) for all of them, read the
// latent output of the block's head for every sequence (rows padded to a
// multiple of 16 with zeros) and multiply it on the warp-level tensor cores
// (m16n8k16, fp32 accumulate) with K split over the warps; the warps' sums
// meet in shared memory, in warp order.  The first block's weight columns are
// copied asynchronously before the CTA's merge and waited for after the wait
// (a further block's, when there are more blocks than CTAs, after the block
// before it).
constexpr int kUpMaxBatch = kUpProjFusedMaxBatch;

template <int K>
struct UpTile {
    static constexpr int KP = K + 8;                       // row stride (bf16): conflict-free fragment reads
    static constexpr int W_BYTES = K * 16 * 2;             // the 16 weight columns, [K][16]
    static constexpr int X_BYTES = kUpMaxBatch * KP * 2;   // latent rows, [N padded][KP]
    static constexpr int RED_BYTES = (kThreads / 32) * kUpMaxBatch * 16 * 4;
    static constexpr int BYTES = W_BYTES + X_BYTES + RED_BYTES;
};

// The CTA's 16 weight columns into wt [K][16] (at the end of the ring), by
// asynchronous 16-byte copies that land while the merge runs (waited for in
// up_proj_tail).
template <int NB, int DC>
__device__ __forceinline__ void up_stage_weights(const DecodeArgs& a, __nv_bfloat16* wt, int cb) {
    constexpr int K = NB * DC;
    const int cols = a.heads * a.d_h;
    const int h = cb / (a.d_h / 16), j0 = (cb % (a.d_h / 16)) * 16;
    const __nv_bfloat16* src = a.w_uv + (size_t)h * a.d_h + j0;
    for (int e = threadIdx.x; e < 2 * K; e += kThreads) {
        const int k = e >> 1, half = e & 1;
        cp_async16(wt + k * 16 + 8 * half, src + (size_t)k * cols + 8 * half);
    }
}

template <int NB, int DC>
__device__ __forceinline__ void up_proj_tail(const DecodeArgs& a, uint8_t* ring, __nv_bfloat16* wt, int* flag) {
    constexpr int K = NB * DC;
    using T = UpTile<K>;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int N = a.batch, H = a.heads, ncb = H * a.d_h / 16;
    const int workers = ncb < a.num_ctas ? ncb : a.num_ctas;
    int* gcnt = a.seq_cnt + kMaxBatch;
    __syncthreads();  // the CTA's merge is done (and its weight columns staged)
    if (tid == 0) red_add_release_gpu(gcnt, 1);
    if ((int)blockIdx.x >= ncb) return;
    int departed = 0;
    if (tid == 0) {
        const uint64_t t0 = globaltimer_ns();
        bool ok = true;
        while (ld_acquire_gpu(gcnt) < a.num_ctas) {
            if (globaltimer_ns() - t0 > 2000000000ull) {
                ok = false;
                break;
            }
            __nanosleep(32);
        }
        if (ok) departed = atomicAdd(gcnt, 1);  // (the counter guards only this wait)
        else {
            *flag |= 4;
            record_error(a.err, MLRA_ERR_DEVICE_TIMEOUT);
        }
    }
    const int Np = (N + 15) & ~15;
    __nv_bfloat16* xs = reinterpret_cast<__nv_bfloat16*>(ring);
    float* red = reinterpret_cast<float*>(ring + T::X_BYTES);
    for (int cb = blockIdx.x; cb < ncb; cb += a.num_ctas) {
        if (cb != (int)blockIdx.x) {
            __syncthreads();  // the block before is done with wt, xs and red
            up_stage_weights<NB, DC>(a, wt, cb);
        }
        const int h = cb / (a.d_h / 16), j0 = (cb % (a.d_h / 16)) * 16;
        if (cb == (int)blockIdx.x) {
            cp_async_wait_all();  // this thread's weight copies (issued before the merge)
            __syncthreads();
            if (*flag & 4) return;
        }
        // out[n][h][0..K) for every sequence: asynchronous 16-byte copies, all
        // in flight at once (rows past N zero)
        for (int e = tid; e < Np * (K / 8); e += kThreads) {
            const int n = e / (K / 8), u = e % (K / 8);
            if (n < N)
                cp_async16(xs + n * T::KP + 8 * u, a.out + ((size_t)n * H + h) * K + 8 * u);
            else
                *reinterpret_cast<uint4*>(xs + n * T::KP + 8 * u) = make_uint4(0u, 0u, 0u, 0u);
        }
        cp_async_wait_all();
        __syncthreads();
        const int g = lane >> 2, tg = lane & 3;
        float acc[4][2][4];
#pragma unroll
        for (int mt = 0; mt < 4; ++mt)
#pragma unroll
            for (int t = 0; t < 2; ++t)
#pragma unroll
                for (int i = 0; i < 4; ++i) acc[mt][t][i] = 0.f;
        for (int ks = warp; ks < K / 16; ks += kThreads / 32) {
            const int kb = 16 * ks + 2 * tg;
            // B (K x 8, column n = output column 8 t + g): rows kb, kb + 1 and
            // kb + 8, kb + 9 of the [K][16] weight tile, packed in pairs
            uint32_t bf[2][2];
            const uint16_t* wt16 = reinterpret_cast<const uint16_t*>(wt);
#pragma unroll
            for (int t = 0; t < 2; ++t) {
                const int col = 8 * t + g;
                bf[t][0] = (uint32_t)wt16[kb * 16 + col] | ((uint32_t)wt16[(kb + 1) * 16 + col] << 16);
                bf[t][1] = (uint32_t)wt16[(kb + 8) * 16 + col] | ((uint32_t)wt16[(kb + 9) * 16 + col] << 16);
            }
#pragma unroll
            for (int mt = 0; mt < 4; ++mt) {
                if (16 * mt >= Np) break;
                const __nv_bfloat16* x0 = xs + (16 * mt + g) * T::KP + kb;
                const uint32_t af[4] = {*reinterpret_cast<const uint32_t*>(x0),
                                        *reinterpret_cast<const uint32_t*>(x0 + 8 * T::KP),
                                        *reinterpret_cast<const uint32_t*>(x0 + 8),
                                        *reinterpret_cast<const uint32_t*>(x0 + 8 * T::KP + 8)};
#pragma unroll
                for (int t = 0; t < 2; ++t) mma_m16n8k16_bf16(acc[mt][t], af, bf[t][0], bf[t][1]);
            }
        }
        // the warps' partial sums: red[warp][row][16 columns]
#pragma unroll
        for (int mt = 0; mt < 4; ++mt) {
            if (16 * mt >= Np) break;
#pragma unroll
            for (int t = 0; t < 2; ++t) {
                float* r = red + ((size_t)warp * kUpMaxBatch + 16 * mt + g) * 16 + 8 * t + 2 * tg;
                r[0] = acc[mt][t][0];
                r[1] = acc[mt][t][1];
                r[8 * 16] = acc[mt][t][2];
                r[8 * 16 + 1] = acc[mt][t][3];
            }
        }
        __syncthreads();
        for (int e = tid; e < N * 16; e += kThreads) {
            const int n = e >> 4, j = e & 15;
            float v = 0.f;
#pragma unroll
            for (int w = 0; w < kThreads / 32; ++w) v += red[((size_t)w * kUpMaxBatch + n) * 16 + j];
            a.y[(size_t)n * H * a.d_h + h * a.d_h + j0 + j] = to_bf16(v);
        }
    }
    if (tid == 0 && departed == a.num_ctas + workers - 1) *gcnt = 0;
}

template <int NB, int DC, int DR, int HP>
__global__ void __launch_bounds__(kThreads, 1)
decode_tc_kernel(const __grid_constant__ Maps maps, const __grid_constant__ DecodeArgs a) {
    using C = Cfg<NB, DC, DR, HP>;
    using M = Misc<C::NSTAGE, HP>;
    constexpr int kHP = HP;       // heads per tile (the MMAs' N)
    constexpr int kHG = HP / 2;   // heads per softmax warpgroup
    static_assert(sizeof(M) <= C::MISC_BYTES, "barriers and scratch fit the MISC region");
    static_assert(C::NSP <= 4 && C::NROPE <= 4, "barrier arrays of Misc");
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    M& misc = *reinterpret_cast<M*>(sm + C::OFF_MISC);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int P = a.page_size;
    const HeadGroup grp = head_group<HP>(a);

    if (warp == 0 && lane < 4) {
        // descriptor fetches overlap the set-up below
        prefetch_tensormap(lane == 0 ? &maps.lat : lane == 1 ? &maps.rope : lane == 2 ? &maps.q : &maps.qr);
    }
    if (threadIdx.x == 0) {
        for (int i = 0; i < C::NSTAGE; ++i) {
            mbar_init(&misc.pair_full[i], 1);
            mbar_init(&misc.pair_empty[i], 1);
        }
        for (int i = 0; i < C::NROPE; ++i) {
            mbar_init(&misc.rope_full[i], 1);
            mbar_init(&misc.rope_empty[i], 1);
        }
        mbar_init(&misc.drain[0], 1);
        mbar_init(&misc.drain[1], 1);
        for (int i = 0; i < C::NSP; ++i) {
            mbar_init(&misc.s_full[i], 1);
            mbar_init(&misc.p_full[i], 8);  // the eight softmax warps
            mbar_init(&misc.p_empty[i], 1);
        }
        mbar_init(&misc.q_full, 1);
        mbar_init(&misc.merge_full, 1);
        mbar_init(&misc.q_empty, 1);
        misc.abort_flag = 0;
        misc.last_seg[0] = -1;
        misc.merge_flag = 0;
        fence_barrier_init();
    }
    launch_dependents();  // a dependent kernel may be scheduled as CTAs retire
    // Warp 0 computes the plan and goes straight on to its copies; the other
    // warps allocate TMEM and meet it (named barrier 2) for the plan.
    int n_first, cum_first;
    if (warp == 0) {
        // the inputs may come from the preceding kernel (programmatic launch)
        wait_prerequisite_grid();
        const int total = warp_cost_prefix(a.seqlens, a.batch, P, a.max_pages);
        const int chunk = plan_chunk(total, grp.cpg);
        n_first = a.batch;
        cum_first = total;
        if (!grp.idle && (long long)grp.ci * chunk < total)
            warp_find_seq(a.seqlens, a.batch, P, a.max_pages, grp.ci * chunk, &n_first, &cum_first);
        if (lane == 0) {
            misc.plan[1] = chunk;
            misc.plan[2] = n_first;
            misc.plan[3] = cum_first;
        }
        __syncwarp();
        named_bar_arrive<2, kThreads>();
    } else {
        if (warp == 1) {
            tmem_alloc(&misc.tmem_base, C::TMEM_COLS);
            tmem_relinquish();
        }
        tc_fence_before();
        named_bar_sync<2, kThreads>();
        tc_fence_after();
        n_first = misc.plan[2];
        cum_first = misc.plan[3];
        if (warp == 6) {
            // sequences with an invalid length: zeros and an error code,
            // sequence m by CTA m mod grid (this warp is idle until the first
            // probabilities of its CTA are ready)
            const int R = NB * DC;
            for (int m = blockIdx.x; m < a.batch; m += a.num_ctas) {
                if (seq_tiles(__ldg(a.seqlens + m), P, a.max_pages) > 0) continue;
                __nv_bfloat162* dst = reinterpret_cast<__nv_bfloat162*>(a.out + (size_t)m * a.heads * R);
                for (int e = lane; e < a.heads * R / 2; e += 32) dst[e] = __floats2bfloat162_rn(0.f, 0.f);
                if (lane == 0) record_error(a.err, MLRA_ERR_DEVICE_BAD_SEQLEN);
            }
        }
    }
    const int chunk = misc.plan[1];
    const int A0 = grp.ci * chunk, A1 = A0 + chunk;  // this CTA's cost window
    const uint32_t tmem = misc.tmem_base;                // (warp 0 never uses it)
    volatile int* abort_flag = &misc.abort_flag;

    if (n_first < a.batch) {
        if (warp == 0) {
            // ------------------------------------------------------------ producer
            int n = n_first, cum = cum_first, next_len = first_len(a, n);
            int L, tiles, tb, te;
            uint32_t pc = 0, tc = 0, sc = 0;
            // the cache is read once per step: its lines go first, and the
            // block table, lengths, queries and partials stay in L2 (with
            // head groups every line is read once per group, at about the
            // same time: normal priority)
            const uint64_t stream_policy = grp.cpg == a.num_ctas ? l2_policy_evict_first() : l2_policy_evict_normal();
            bool ok = true;
            while (ok && next_segment(a, n, cum, A0, A1, L, tiles, tb, te, next_len)) {
                // the first range's queries; a later range's are loaded by the
                // score MMA warp once the range before has its last scores, so
                // the copies of the cache never wait for the query buffer
                // (the range's first window of block-table entries is in flight
                // meanwhile: a lane per entry, a window of 32 pages)
                const int32_t* bt = a.block_table + (size_t)n * a.max_pages;
                int win_base = tb * kT / P, win_val = 0;
                if (win_base + lane < a.max_pages) win_val = __ldg(bt + win_base + lane);
                if (lane == 0 && sc == 0) load_queries<C>(maps, sm, misc.q_full, n, grp.h0);
                win_val = (win_val >= 0 && win_val < a.num_pages) ? win_val : 0;  // bad entries are reported by the softmax warps
                ++sc;
                for (int j = tb; j < te && ok; ++j) {
                    const int tok0 = j * kT;
                    const int valid = min(kT, L - tok0);
                    const int npages = ceil_div(valid, P);
                    const int page0 = tok0 / P;
                    if (page0 < win_base || page0 + npages > win_base + 32) {
                        win_base = page0;
                        const int idx = page0 + lane;
                        const int v = idx < a.max_pages ? __ldg(bt + idx) : 0;
                        win_val = (v >= 0 && v < a.num_pages) ? v : 0;  // bad entries are reported by the softmax warps
                    }
                    const int rs = tc % C::NROPE;  // RoPE slot of this tile
                    if (lane == 0) {
                        if (tc >= (uint32_t)C::NROPE) ok = mbar_wait(&misc.rope_empty[rs], ((tc / C::NROPE) - 1) & 1);
                        if (ok) mbar_arrive_expect_tx(&misc.rope_full[rs], npages * P * C::ROPE_ROW);
                    }
                    ok = __shfl_sync(0xffffffffu, ok, 0);
                    if (!ok) break;
                    for (int q = 0; q < npages; ++q) {
                        const int page = __shfl_sync(0xffffffffu, win_val, page0 + q - win_base);
                        if (lane == 0)
                            tma_load_2d_hint(sm + C::OFF_ROPE + rs * C::ROPE_BYTES + q * P * C::ROPE_ROW, &maps.rope,
                                             0, page * P, &misc.rope_full[rs], stream_policy);
                    }
                    ++tc;
                    for (int sp = 0; sp < C::NSTEP * C::PPS && ok; ++sp) {
                        const int stage = pc % C::NSTAGE;
                        if (lane == 0) {
                            ok = mbar_wait(&misc.pair_empty[stage], ((pc / C::NSTAGE) & 1) ^ 1);
                            if (ok) mbar_arrive_expect_tx(&misc.pair_full[stage], 2 * npages * P * 128);
                        }
                        ok = __shfl_sync(0xffffffffu, ok, 0);
                        if (!ok) break;
                        const int chunk0 = sp * 2;  // pairs are consecutive 128-column groups
                        for (int q = 0; q < npages; ++q) {
                            const int page = __shfl_sync(0xffffffffu, win_val, page0 + q - win_base);
                            if (lane == 0) {
                                uint8_t* dst = sm + C::OFF_PAIR + stage * C::PAIR_BYTES + q * P * 128;
                                tma_load_2d_hint(dst, &maps.lat, chunk0 * 64, page * P, &misc.pair_full[stage],
                                                 stream_policy);
                                tma_load_2d_hint(dst + C::CHUNK_BYTES, &maps.lat, chunk0 * 64 + 64, page * P,
                                                 &misc.pair_full[stage], stream_policy);
                            }
                        }
                        ++pc;
                    }
                    ok = __shfl_sync(0xffffffffu, ok && !*abort_flag, 0);
                }
                finish_segment(n, cum, tiles);
            }
            if (!ok) {
                if (lane == 0) {
                    record_error(a.err, MLRA_ERR_DEVICE_TIMEOUT);
                    *abort_flag = 1;
                }
            }
            // drain: wait (bounded) for the copies issued last, so that no
            // TMA write lands after this CTA has exited
            if (lane == 0) {
                for (uint32_t i = 0; i < (uint32_t)C::NSTAGE && i < pc; ++i) {
                    const uint32_t k = pc - 1 - i;
                    mbar_wait(&misc.pair_full[k % C::NSTAGE], (k / C::NSTAGE) & 1, 200000000ull);
                }
                for (uint32_t i = 0; i < (uint32_t)C::NROPE && i < tc; ++i) {
                    const uint32_t k = tc - 1 - i;
                    mbar_wait(&misc.rope_full[k % C::NROPE], (k / C::NROPE) & 1, 200000000ull);
                }
                if (sc > 0) mbar_wait(&misc.q_full, (sc - 1) & 1, 200000000ull);
            }
        } else if (warp == 1) {
            // ------------------------------------------------------------ score MMA issuer
            // (the whole warp walks the schedule; the elected lane issues)
            constexpr uint32_t IDESC_S = idesc_bf16_f32(128, kHP, false, false);
            const uint32_t sm_base = smem_u32(sm);
            // Descriptor bases; every operand below is a base plus a byte
            // offset >> 4 (the start-address field never overflows: all
            // addresses are below 256 KB).
            const uint64_t dA_s = smem_desc(sm_base + C::OFF_PAIR, 16, 1024, kLayoutSw128);  // K-major
            const uint64_t dQ = smem_desc(sm_base + C::OFF_Q, 16, 1024, kLayoutSw128);
            const uint64_t dQR = rope_desc<DR>(sm_base + C::OFF_QR);
            const uint64_t dR = rope_desc<DR>(sm_base + C::OFF_ROPE);
            int n = n_first, cum = cum_first, next_len = first_len(a, n);
            int L, tiles, tb, te;
            uint32_t gs = 0, tc = 0, sc = 0, qe = 0;
            uint32_t stage = 0, phase = 0;  // ring position of the next pair to consume
            bool ok = true;
            while (ok && next_segment(a, n, cum, A0, A1, L, tiles, tb, te, next_len)) {
                ok = mbar_wait_warp(&misc.q_full, sc & 1);
                tc_fence_after();
                for (int j = tb; j < te && ok; ++j) {
                    const uint32_t rs = tc % C::NROPE;
                    ok = mbar_wait_warp(&misc.rope_full[rs], (tc / C::NROPE) & 1);
#pragma unroll 1
                    for (int st = 0; st < C::NSTEP && ok; ++st) {
                        // the step's first pair, then its S slot (and the P slot the
                        // softmax fills next): free once the output MMA NSP steps
                        // back is done
                        ok = mbar_wait_warp(&misc.pair_full[stage], phase);
                        const uint32_t slot = gs % C::NSP;
                        if (ok && gs >= (uint32_t)C::NSP)
                            ok = mbar_wait_warp(&misc.p_empty[slot], ((gs / C::NSP) - 1) & 1);
                        if (!ok) break;
                        tc_fence_after();
                        if (st == 0) {
                            // RoPE score of the tile, shared by every branch
                            const uint32_t dRt = tmem + C::R_COL0 + (tc % C::NRS) * kHP;
                            const uint64_t dRs = dR + ((rs * C::ROPE_BYTES) >> 4);
#pragma unroll
                            for (int kk = 0; kk < DR / 16; ++kk)
                                if (elect_one()) mma_bf16(dRt, dRs + kk * 2, dQR + kk * 2, IDESC_S, kk ? 1u : 0u);
                            if (elect_one()) mma_commit(&misc.rope_empty[rs]);
                            __syncwarp();
                        }
                        const uint32_t dS = tmem + C::S_COL0 + slot * C::S_SLOT_COLS;
                        // this step's branches start at chunk st*SBR*(DC/64) of the token row
                        const uint64_t dQs = dQ + ((st * C::SBR * (DC / 64) * C::Q_CHUNK_BYTES) >> 4);
                        // each pair's MMAs as soon as it lands: chunk lc = 2 pp + hf of
                        // the step is column chunk c of branch g of the step
#pragma unroll 1
                        for (int pp = 0; pp < C::PPS && ok; ++pp) {
                            if (pp > 0) {
                                ok = mbar_wait_warp(&misc.pair_full[stage], phase);
                                if (!ok) break;
                                tc_fence_after();
                            }
#pragma unroll
                            for (int hf = 0; hf < 2; ++hf) {
                                const int lc = 2 * pp + hf;
                                const int g = lc / (DC / 64), c = lc % (DC / 64);
                                const uint64_t a0 = dA_s + ((stage * C::PAIR_BYTES + hf * C::CHUNK_BYTES) >> 4);
                                const uint64_t q0 = dQs + ((lc * C::Q_CHUNK_BYTES) >> 4);
#pragma unroll
                                for (int kk = 0; kk < 4; ++kk)
                                    if (elect_one())
                                        mma_bf16(dS + g * kHP, a0 + kk * 2, q0 + kk * 2, IDESC_S, (c | kk) ? 1u : 0u);
                            }
                            if (++stage == (uint32_t)C::NSTAGE) {
                                stage = 0;
                                phase ^= 1;
                            }
                        }
                        if (!ok) break;
                        if (elect_one()) mma_commit(&misc.s_full[slot]);
                        __syncwarp();
                        ++gs;
                    }
                    ++tc;
                    if (__shfl_sync(0xffffffffu, *abort_flag, 0)) ok = false;
                }
                // a next range: its queries replace these once this range's
                // score MMAs have finished
                const int nn = next_range_seq(a, n, cum, tiles, A0, A1);
                if (ok && nn >= 0) {
                    if (elect_one()) mma_commit(&misc.q_empty);
                    __syncwarp();
                    ok = mbar_wait_warp(&misc.q_empty, qe & 1);
                    ++qe;
                    if (ok && elect_one()) load_queries<C>(maps, sm, misc.q_full, nn, grp.h0);
                    __syncwarp();
                }
                ++sc;
                finish_segment(n, cum, tiles);
            }
            if (!ok && lane == 0) {
                record_error(a.err, MLRA_ERR_DEVICE_TIMEOUT);
                *abort_flag = 1;
            }
            // drain: every MMA issued above completes before TMEM is freed
            if (elect_one()) mma_commit(&misc.drain[0]);
            __syncwarp();
            mbar_wait(&misc.drain[0], 0, 200000000ull);
            __syncwarp();
        } else if (warp == 6) {
            // ------------------------------------------------------------ output MMA issuer
            constexpr uint32_t IDESC_PV = idesc_bf16_f32(128, kHP, true, true);
            const uint32_t sm_base = smem_u32(sm);
            const uint64_t dA_pv = smem_desc(sm_base + C::OFF_PAIR, C::CHUNK_BYTES, 1024, kLayoutSw128);  // MN-major
            const uint64_t dP = smem_desc(sm_base + C::OFF_P, 128, 2048, kLayoutNone);
            int n = n_first, cum = cum_first, next_len = first_len(a, n);
            int L, tiles, tb, te;
            uint32_t gs = 0;
            uint32_t stage = 0;  // ring position of the step's first pair
            bool ok = true;
            while (ok && next_segment(a, n, cum, A0, A1, L, tiles, tb, te, next_len)) {
                for (int j = tb; j < te && ok; ++j) {
#pragma unroll 1
                    for (int st = 0; st < C::NSTEP; ++st) {
                        const uint32_t slot = gs % C::NSP;
                        ok = mbar_wait_warp(&misc.p_full[slot], (gs / C::NSP) & 1);
                        if (!ok) break;
                        tc_fence_after();
                        const uint64_t b0 = dP + ((slot * C::P_BYTES) >> 4);
#pragma unroll
                        for (int p = 0; p < C::PPS; ++p) {
                            uint32_t sp = stage + p;
                            if (sp >= (uint32_t)C::NSTAGE) sp -= C::NSTAGE;
                            const uint64_t a0 = dA_pv + ((sp * C::PAIR_BYTES) >> 4);
#pragma unroll
                            for (int g2 = 0; g2 < C::BPP; ++g2) {
                                // branch of the step whose P multiplies this pair (rows of the
                                // other branch of a shared pair are discarded later)
                                const int gl = DC >= 128 ? p * 128 / DC : p * C::BPP + g2;
                                const uint32_t d = tmem + ((st * C::PPS + p) * C::BPP + g2) * kHP;
#pragma unroll
                                for (int kt = 0; kt < kT / 16; ++kt)
                                    if (elect_one())
                                        mma_bf16(d, a0 + (kt * 2048 >> 4), b0 + ((gl * C::P_BRANCH_BYTES + kt * 256) >> 4),
                                                 IDESC_PV, (j == tb && kt == 0) ? 0u : 1u);
                            }
                            // the pair's stage is free once its MMAs (and all before) finish
                            if (elect_one()) mma_commit(&misc.pair_empty[sp]);
                        }
                        if (elect_one()) mma_commit(&misc.p_empty[slot]);
                        __syncwarp();
                        stage += C::PPS;
                        if (stage >= (uint32_t)C::NSTAGE) stage -= C::NSTAGE;
                        ++gs;
                    }
                    if (__shfl_sync(0xffffffffu, *abort_flag, 0)) ok = false;
                }
                finish_segment(n, cum, tiles);
            }
            if (!ok && lane == 0) {
                record_error(a.err, MLRA_ERR_DEVICE_TIMEOUT);
                *abort_flag = 1;
            }
            if (elect_one()) mma_commit(&misc.drain[1]);
            __syncwarp();
            mbar_wait(&misc.drain[1], 0, 200000000ull);
            __syncwarp();
        } else {
            // ------------------------------------------------------------ softmax + epilogue
            // Two groups of four warps (warps 2-5 and 7-10), one warp of each
            // per TMEM lane quadrant: group sg owns heads [8 sg, 8 sg + 8) of
            // every score and output column block.  The groups share no
            // running max, denominator or rescale (those are per head); they
            // meet only in a P slot (each writes its 8 heads of a token's row
            // and arrives on p_full) and at the kernel's end.  Two warps per
            // scheduler hide each other's latency chains.
            const int sg = warp >= 7;                        // softmax group
            const int hoff = kHG * sg;                       // its first head column
            const uint32_t gbar = 3 + sg;                    // its named barrier (128 threads)
            const int quad = warp & 3;                       // TMEM lane quadrant of this warp
            const int row = quad * 32 + lane;                // token (S) / latent row (O)
            const int stid = (warp - (sg ? 7 : 2)) * 32 + lane;  // 0..127 within the group
            const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
            const int H = a.heads;
            int n = n_first, cum = cum_first, next_len = first_len(a, n);
            int L, tiles, tb, te;
            uint32_t gs = 0, sc = 0, tcnt = 0;  // steps, ranges, tiles so far
            // This thread's share of the softmax denominators, one row per
            // branch.  The step loop is not unrolled: after each step the rows
            // rotate by G so that the current step's branches are rows 0..G-1.
            float l[NB][kHG];
            bool dead = false;
            int pend_a = -1, pend_b = -1;  // split ranges not yet counted (thread stid 0)

            while (!dead && next_segment(a, n, cum, A0, A1, L, tiles, tb, te, next_len)) {
                // block-table entries of the range must name real pages: each
                // thread checks its own token's page once per tile (the load is
                // issued at the tile's start and consumed at its end)
                bool bad = false;
                const int32_t* bt = a.block_table + (size_t)n * a.max_pages;
                // for the merge at the kernel's end: whether the CTA owning
                // this sequence's last tile also merges it (no later sequence
                // starts in its window); worked out now, off the critical path
                int c1_member = 1;
                if (sg == 0 && stid == 0) {
                    const int c1 = (cum + (tiles - 1) * kTileCost) / chunk;
                    for (int m = n + 1; m < a.batch; ++m) {
                        if (seq_tiles(__ldg(a.seqlens + m), a.page_size, a.max_pages) == 0) continue;
                        c1_member = (cum + tiles * kTileCost + kSeqCost) / chunk != c1;
                        break;
                    }
                }
#pragma unroll
                for (int b = 0; b < NB; ++b)
#pragma unroll
                    for (int i = 0; i < kHG; ++i) l[b][i] = 0.f;

                for (int j = tb; j < te && !dead; ++j) {
                    const int valid = min(kT, L - j * kT);
                    const bool masked = row >= valid;
                    const int page = masked ? 0 : __ldg(bt + (j * kT + row) / P);
                    float r[kHG];  // this token's RoPE score per head, shared by the tile's branches
#pragma unroll 1
                    for (int st = 0; st < C::NSTEP; ++st) {
                        const uint32_t slot = gs % C::NSP;
                        const bool ok = mbar_wait(&misc.s_full[slot], (gs / C::NSP) & 1);
                        tc_fence_after();

                        float x[C::SBR][kHG];
                        if (st == 0) tmem_ld_cols<kHG>(tmem + lane_off + C::R_COL0 + (tcnt % C::NRS) * kHP + hoff, r);
#pragma unroll
                        for (int g = 0; g < C::SBR; ++g)
                            tmem_ld_cols<kHG>(tmem + lane_off + C::S_COL0 + slot * C::S_SLOT_COLS + g * kHP + hoff, x[g]);
                        tmem_wait_ld();
#pragma unroll
                        for (int g = 0; g < C::SBR; ++g)
#pragma unroll
                            for (int i = 0; i < kHG; ++i)
                                x[g][i] = masked ? -INFINITY : (x[g][i] + r[i]) * a.scale_log2;
                        float* m_step = &misc.m_run[st * C::SBR * kHP + hoff];  // [g * kHP + i]
                        if (j == tb) {
                            // first tile of the range: token 0 (always valid) sets the
                            // reference maxima; larger scores take the exact path below
                            if (stid == 0) {
#pragma unroll
                                for (int g = 0; g < C::SBR; ++g)
#pragma unroll
                                    for (int i = 0; i < kHG; ++i) m_step[g * kHP + i] = x[g][i];
                            }
                            named_bar_sync_id<128>(gbar);
                        }
                        float m[C::SBR][kHG];
#pragma unroll
                        for (int g = 0; g < C::SBR; ++g)
#pragma unroll
                            for (int i = 0; i < kHG; i += 4) {
                                const float4 v = *reinterpret_cast<const float4*>(m_step + g * kHP + i);
                                m[g][i] = v.x;
                                m[g][i + 1] = v.y;
                                m[g][i + 2] = v.z;
                                m[g][i + 3] = v.w;
                            }
                        bool need = false;
#pragma unroll
                        for (int g = 0; g < C::SBR; ++g)
#pragma unroll
                            for (int i = 0; i < kHG; ++i) need |= x[g][i] > m[g][i] + kRescaleLog2;
                        if (named_bar_or_id<128>(gbar, need || !ok)) {
                            if (named_bar_or_id<128>(gbar, !ok)) {
                                dead = true;
                                break;
                            }
                            // exact column max over the tile's 128 tokens: a warp
                            // reduce-scatter leaves column lane / (32 / kHG) in each lane
                            constexpr int CSPAN = 32 / kHG;
#pragma unroll
                            for (int g = 0; g < C::SBR; ++g) {
                                const float v = warp_colmax<kHG>(x[g], lane);
                                if ((lane & (CSPAN - 1)) == 0) misc.red_max[quad][g * kHP + hoff + lane / CSPAN] = v;
                            }
                            named_bar_sync_id<128>(gbar);
                            float alpha[C::SBR][kHG];
#pragma unroll
                            for (int g = 0; g < C::SBR; ++g)
#pragma unroll
                                for (int i = 0; i < kHG; ++i) {
                                    const int c = g * kHP + hoff + i;
                                    const float tmax = fmaxf(fmaxf(misc.red_max[0][c], misc.red_max[1][c]),
                                                             fmaxf(misc.red_max[2][c], misc.red_max[3][c]));
                                    const float mnew = fmaxf(m[g][i], tmax);
                                    alpha[g][i] = fast_exp2(m[g][i] - mnew);
                                    m[g][i] = mnew;
                                    l[g][i] *= alpha[g][i];
                                }
                            // every thread read the old maxima before the barrier above; the
                            // barrier below publishes the new ones (and frees red_max)
                            if (stid == 0) {
#pragma unroll
                                for (int g = 0; g < C::SBR; ++g)
#pragma unroll
                                    for (int i = 0; i < kHG; ++i) m_step[g * kHP + i] = m[g][i];
                            }
                            named_bar_sync_id<128>(gbar);
                            if (j > tb) {
                                // O holds earlier tiles of this range: rescale this
                                // group's columns once the previous output MMA has finished
                                const bool ok2 = mbar_wait(&misc.p_empty[(gs - 1) % C::NSP], ((gs - 1) / C::NSP) & 1);
                                if (named_bar_or_id<128>(gbar, !ok2)) {
                                    dead = true;
                                    break;
                                }
                                tc_fence_after();
#pragma unroll
                                for (int p = 0; p < C::PPS; ++p)
#pragma unroll
                                    for (int g2 = 0; g2 < C::BPP; ++g2) {
                                        const int gl = DC >= 128 ? p * 128 / DC : p * C::BPP + g2;
                                        const uint32_t col = ((st * C::PPS + p) * C::BPP + g2) * kHP + hoff;
                                        float o[kHG];
                                        tmem_ld_cols<kHG>(tmem + lane_off + col, o);
                                        tmem_wait_ld();
#pragma unroll
                                        for (int i = 0; i < kHG; ++i) o[i] *= alpha[gl][i];
                                        tmem_st_cols<kHG>(tmem + lane_off + col, o);
                                    }
                                tmem_wait_st();
                            }
                        }
                        // probabilities -> bf16 P (MN-major, 8x8 core matrices of 8
                        // heads at a stride of 2048 bytes; this group's kHG heads are
                        // the core matrices from kHG / 8 sg)
                        uint8_t* p_slot = sm + C::OFF_P + slot * C::P_BYTES;
#pragma unroll
                        for (int g = 0; g < C::SBR; ++g) {
                            uint32_t packed[kHG / 2];
#pragma unroll
                            for (int i = 0; i < kHG; i += 2) {
                                const float p0 = fast_exp2(x[g][i] - m[g][i]);
                                const float p1 = fast_exp2(x[g][i + 1] - m[g][i + 1]);
                                l[g][i] += p0;
                                l[g][i + 1] += p1;
                                __nv_bfloat162 pr = __floats2bfloat162_rn(p0, p1);
                                packed[i / 2] = *reinterpret_cast<uint32_t*>(&pr);
                            }
                            uint8_t* dst = p_slot + g * C::P_BRANCH_BYTES + (row >> 3) * 128 + (row & 7) * 16 +
                                           sg * (kHG / 8) * 2048;
#pragma unroll
                            for (int c8 = 0; c8 < kHG / 8; ++c8)
                                *reinterpret_cast<uint4*>(dst + c8 * 2048) =
                                    make_uint4(packed[4 * c8], packed[4 * c8 + 1], packed[4 * c8 + 2], packed[4 * c8 + 3]);
                        }
                        // rows past the end of the sequence (stale or poisoned data)
                        // become zero before the output MMA reads them: this group
                        // clears chunk sg of each of the step's pairs
                        if (masked) {
#pragma unroll
                            for (int p = 0; p < C::PPS; ++p) {
                                uint8_t* pair = sm + C::OFF_PAIR + ((gs * C::PPS + p) % C::NSTAGE) * C::PAIR_BYTES;
#pragma unroll
                                for (int u = 0; u < 8; ++u)
                                    *reinterpret_cast<uint4*>(pair + sg * C::CHUNK_BYTES + row * 128 + u * 16) =
                                        make_uint4(0, 0, 0, 0);
                            }
                        }
                        fence_proxy_async_smem();
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive(&misc.p_full[slot]);
                        // rotate the denominator rows: the next step's branches first
#pragma unroll
                        for (int r2 = 0; r2 < C::SBR; ++r2) {
                            float t[kHG];
#pragma unroll
                            for (int i = 0; i < kHG; ++i) t[i] = l[0][i];
#pragma unroll
                            for (int b = 0; b + 1 < NB; ++b)
#pragma unroll
                                for (int i = 0; i < kHG; ++i) l[b][i] = l[b + 1][i];
#pragma unroll
                            for (int i = 0; i < kHG; ++i) l[NB - 1][i] = t[i];
                        }
                        ++gs;
                    }
                    bad |= page < 0 || page >= a.num_pages;
                    ++tcnt;
                }
                if (dead) break;

                // ---------------------------------------------------- epilogue
                // denominators (final once the last probabilities are written):
                // warp reduce-scatter, then the four warps through shared memory
                // (this group's 32 columns of red_sum), while the range's last
                // output MMA may still run
                constexpr int NV = NB * kHG;  // (branch, head) values of the group
                static_assert(2 * NV <= 4 * kHP, "the groups' denominators fit red_sum");
                {
                    float f[NV];
#pragma unroll
                    for (int b = 0; b < NB; ++b)
#pragma unroll
                        for (int i = 0; i < kHG; ++i) f[b * kHG + i] = l[b][i];
                    warp_sum_scatter<NV, 16, NV>(f, lane);
                    if constexpr (NV >= 32) {  // lane L holds values (NV / 32) L + r
#pragma unroll
                        for (int r2 = 0; r2 < NV / 32; ++r2) misc.red_sum[quad][NV * sg + (NV / 32) * lane + r2] = f[r2];
                    } else {
                        constexpr int SPAN = 32 / NV;  // lanes holding one value's total
                        if ((lane & (SPAN - 1)) == 0) misc.red_sum[quad][NV * sg + lane / SPAN] = f[0];
                    }
                }
                bad = named_bar_or_id<128>(gbar, bad);  // also publishes red_sum
                // one window holds every tile of the sequence: no split
                const bool single = cum >= A0 && cum + (tiles - 1) * kTileCost < A1;
                const size_t slot = (size_t)grp.slot0 + grp.ci + n;
                if (stid < NV) {
                    const int c = NV * sg + stid;
                    const float lt = misc.red_sum[0][c] + misc.red_sum[1][c] + misc.red_sum[2][c] + misc.red_sum[3][c];
                    const int b = stid / kHG, i = hoff + stid % kHG;
                    misc.inv_l[b * kHP + i] = 1.0f / lt;
                    if (!single)  // all 16 columns (padded heads too): the merge reads whole rows
                        a.lse_part[(slot * NB + b) * kHP + i] =
                            bad ? bad_split_marker() : misc.m_run[b * kHP + i] + __log2f(lt);
                }
                // the range's last output MMA (the barrier below also publishes inv_l)
                {
                    const bool ok = mbar_wait(&misc.p_empty[(gs - 1) % C::NSP], ((gs - 1) / C::NSP) & 1);
                    if (named_bar_or_id<128>(gbar, !ok)) {
                        dead = true;
                        break;
                    }
                }
                tc_fence_after();
                // outputs: a block of TMEM holds 128 latent rows x 16 heads of one
                // branch (or two branches of 64 rows when DC = 64); this group
                // reads its 8 heads of every block before a single wait
                constexpr int WIDTH = DC >= 128 ? 128 : DC;  // valid rows per block
                float o[C::O_BLOCKS][kHG];
#pragma unroll
                for (int blk = 0; blk < C::O_BLOCKS; ++blk) tmem_ld_cols<kHG>(tmem + lane_off + blk * kHP + hoff, o[blk]);
                tmem_wait_ld();
#pragma unroll
                for (int blk = 0; blk < C::O_BLOCKS; ++blk) {
                    const int g2 = blk % C::BPP, gp = blk / C::BPP;  // pair of the tile, branch in it
                    const int row0 = g2 * WIDTH;                     // first valid row of the block
                    const int b = (gp * 128 + row0) / DC;            // branch of the block
                    const int k = (gp * 128 + row0) % DC + (row - row0);  // latent column of this row
                    const bool mine = row >= row0 && row < row0 + WIDTH;
                    if (!mine) continue;
                    const float* inv = &misc.inv_l[b * kHP + hoff];
#pragma unroll
                    for (int i = 0; i < kHG; ++i) o[blk][i] = bad ? 0.f : o[blk][i] * inv[i];
                    if (single) {
                        __nv_bfloat16* dst = a.out + (((size_t)n * H + grp.h0 + hoff) * NB + b) * DC + k;
#pragma unroll
                        for (int i = 0; i < kHG; ++i)
                            if (hoff + i < grp.hn) dst[(size_t)i * NB * DC] = to_bf16(o[blk][i] * a.out_scale);
                    } else {
                        // partial layout [slot][branch][k][kHP heads]: this group's
                        // heads are 32-byte stores of 8
                        float* dst = a.o_part + ((slot * NB + b) * DC + k) * kHP + hoff;
#pragma unroll
                        for (int c8 = 0; c8 < kHG / 8; ++c8)
                            st_global_v8(dst + 8 * c8, o[blk][8 * c8], o[blk][8 * c8 + 1], o[blk][8 * c8 + 2],
                                         o[blk][8 * c8 + 3], o[blk][8 * c8 + 4], o[blk][8 * c8 + 5], o[blk][8 * c8 + 6],
                                         o[blk][8 * c8 + 7]);
                    }
                }
                if (bad && stid == 0) record_error(a.err, MLRA_ERR_DEVICE_BAD_INDEX);
                tc_fence_before();
                named_bar_sync_id<128>(gbar);  // inv_l and red_sum are reused by the next range
                if (stid == 0) {
                    // a split's partials are complete: counted for the merge when
                    // this CTA's work ends (only its first and last ranges can be
                    // splits, and their merges wait for the kernel's end anyway;
                    // a fence here would stall the pipeline)
                    if (!single) {
                        if (pend_a < 0) pend_a = n; else pend_b = n;
                    }
                    if (sg == 0) {
                        misc.last_seg[0] = n;
                        misc.last_seg[1] = cum;
                        misc.last_seg[2] = tiles;
                        misc.last_seg[3] = c1_member;
                    }
                }
                ++sc;
                finish_segment(n, cum, tiles);
            }
            if (dead && stid == 0) {
                record_error(a.err, MLRA_ERR_DEVICE_TIMEOUT);
                *abort_flag = 1;
            }
            // both groups' partial stores precede this barrier; then one
            // release fence makes them visible before both counts (none when
            // either group gave up: the CTA then skips its merges too)
            const bool any_dead = named_bar_or<5, 2 * 128>(dead);
            if (!any_dead && sg == 0 && stid == 0 && pend_a >= 0) {
                fence_acq_rel_gpu();
                red_add_relaxed_gpu(a.seq_cnt + grp.cnt0 + pend_a, 1);
                if (pend_b >= 0) red_add_relaxed_gpu(a.seq_cnt + grp.cnt0 + pend_b, 1);
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem, C::TMEM_COLS);
    if (*abort_flag) return;
    // every region below MISC (ring, RoPE slots, queries, probabilities) is
    // free from here on: the merge stages its partials at its start, the
    // fused up-projection its weight columns at its end
    __nv_bfloat16* wt = reinterpret_cast<__nv_bfloat16*>(sm + C::OFF_MISC - UpTile<NB * DC>::W_BYTES);
    const bool fused = a.w_uv != nullptr;
    if (fused && (int)blockIdx.x < a.heads * a.d_h / 16) up_stage_weights<NB, DC>(a, wt, blockIdx.x);
    merge_tail<NB, DC, HP>(a, grp, misc.last_seg[0], misc.last_seg[1], misc.last_seg[2], misc.last_seg[3] != 0, chunk,
                       reinterpret_cast<float*>(sm + C::OFF_PAIR), &misc.merge_flag, &misc.merge_full);
    if (fused) up_proj_tail<NB, DC>(a, sm + C::OFF_PAIR, wt, &misc.merge_flag);
}

// ------------------------------------------------------------------ host side
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

bool encode_2d(CUtensorMap* map, const void* base, uint64_t inner, uint64_t rows, uint32_t box_inner,
               uint32_t box_rows, CUtensorMapSwizzle swizzle) {
    auto fn = encode_fn();
    if (fn == nullptr) return false;
    const cuuint64_t dims[2] = {inner, rows};
    const cuuint64_t strides[1] = {inner * 2};
    const cuuint32_t box[2] = {box_inner, box_rows};
    const cuuint32_t estr[2] = {1, 1};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool encode_3d(CUtensorMap* map, const void* base, uint64_t inner, uint64_t mid, uint64_t outer,
               uint32_t box_inner, uint32_t box_mid, CUtensorMapSwizzle swizzle) {
    auto fn = encode_fn();
    if (fn == nullptr) return false;
    const cuuint64_t dims[3] = {inner, mid, outer};
    const cuuint64_t strides[2] = {inner * 2, inner * mid * 2};
    const cuuint32_t box[3] = {box_inner, box_mid, 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int NB, int DC, int DR, int HP>
cudaError_t launch_cfg(const DecodeArgs& a, cudaStream_t stream) {
    using C = Cfg<NB, DC, DR, HP>;
    constexpr int kHP = HP;
    Maps maps;
    const uint64_t rows = (uint64_t)a.num_pages * a.page_size;
    const uint32_t box_rows = (uint32_t)a.page_size;
    if (!encode_2d(&maps.lat, a.latent, (uint64_t)C::W, rows, 64, box_rows, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !encode_2d(&maps.rope, a.rope, (uint64_t)DR, rows, DR, box_rows,
                   DR == 64 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B) ||
        !encode_3d(&maps.q, a.q_lat, (uint64_t)C::W, (uint64_t)a.heads, (uint64_t)a.batch, 64, kHP,
                   CU_TENSOR_MAP_SWIZZLE_128B) ||
        !encode_3d(&maps.qr, a.q_rope, (uint64_t)DR, (uint64_t)a.heads, (uint64_t)a.batch, DR, kHP,
                   DR == 64 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B))
        return cudaErrorInvalidValue;
    auto kernel = decode_tc_kernel<NB, DC, DR, HP>;
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    // the merge stages below MISC, for every S <= grid splits of a sequence:
    // the log-sum-exp rows (S NB kHP floats) and S row slices of at most
    // ceil(R / (S - 1)) rows of kHP floats (a member's share: at least S - 1
    // members divide the R rows)
    size_t merge_bytes = 0;
    for (int S = 2; S <= a.num_ctas; ++S) {
        const size_t rows = ((size_t)C::W + S - 2) / (S - 1);
        const size_t bytes = sizeof(float) * ((size_t)S * NB * kHP + (size_t)S * rows * kHP);
        merge_bytes = bytes > merge_bytes ? bytes : merge_bytes;
    }
    const size_t room = (size_t)C::OFF_MISC;  // all shared memory below MISC, idle after the main loop
    if (merge_bytes > room) return cudaErrorInvalidConfiguration;
    // the fused up-projection: weight columns at the ring's end (staged while
    // the merge uses its start), then its rows and sums from the start
    if (a.w_uv != nullptr &&
        (merge_bytes + UpTile<NB * DC>::W_BYTES > room || (size_t)UpTile<NB * DC>::BYTES > room))
        return cudaErrorInvalidConfiguration;
    // Cooperative: every CTA is resident at once, so the merge's wait for the
    // other splits of a sequence always ends.
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(a.num_ctas);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = C::SMEM_BYTES;
    cfg.stream = stream;
    // Programmatic: the CTAs of this launch may set up (barriers, TMEM) on SMs
    // the preceding kernel has released, and wait for its completion only
    // before reading inputs.
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    return cudaLaunchKernelEx(&cfg, kernel, maps, a);
}

// The head tile of a shape: 16 heads, or 32 when there are more and a
// branch is at least 128 wide (no 32-head instantiation for narrower ones).
template <int NB, int DC>
cudaError_t launch_shape(const DecodeArgs& a, cudaStream_t stream) {
    if constexpr (DC >= 128) {
        if (tc_head_tile(a.heads, DC) == 32)
            return a.d_r == 64 ? launch_cfg<NB, DC, 64, 32>(a, stream) : launch_cfg<NB, DC, 32, 32>(a, stream);
    }
    return a.d_r == 64 ? launch_cfg<NB, DC, 64, 16>(a, stream) : launch_cfg<NB, DC, 32, 16>(a, stream);
}

}  // namespace

bool decode_tc_supported(int branches, int d_c, int d_r, int heads) {
    if (heads > kMaxTcHeads || (d_r != 32 && d_r != 64)) return false;
    switch (d_c) {
        case 64: return branches == 2 || branches == 4;
        case 128: return branches == 1 || branches == 2 || branches == 4;
        case 256: return branches == 1 || branches == 2;
        case 512: return branches == 1;
    }
    return false;
}

cudaError_t launch_decode_tc(const DecodeArgs& a, cudaStream_t stream) {
#define MLRA_TC_CASE(NB_, DC_) \
    if (a.branches == NB_ && a.d_c == DC_) return launch_shape<NB_, DC_>(a, stream);
    MLRA_TC_CASE(2, 64)
    MLRA_TC_CASE(4, 64)
    MLRA_TC_CASE(1, 128)
    MLRA_TC_CASE(2, 128)
    MLRA_TC_CASE(4, 128)
    MLRA_TC_CASE(1, 256)
    MLRA_TC_CASE(2, 256)
    MLRA_TC_CASE(1, 512)
#undef MLRA_TC_CASE
    return cudaErrorInvalidValue;
}

}  // namespace mlra
