/*
 * mlra_oracle.c -- plain, slow, fp64 CPU statement of MLRA decode attention.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path (the CUDA library
 * and its Python binding) may include, link or call this file.  Only the
 * test-suite, the smoke check and the CPU-baseline leg of the benchmark use
 * it.  It shares no code, header or constant with the CUDA sources.
 *
 * What it computes (the plain definition, no blocking, no online softmax):
 *
 *   For every sequence n with length L = seqlens[n] and every token t < L:
 *     page = block_table[n][t / P], slot = t mod P
 *     c_b[t] = latent_cache[page][slot][b][0:d_c]   (branch b's own latent)
 *     k_r[t] = rope_cache[page][slot][0:d_r]        (one RoPE key, shared)
 *   For every head h and branch b, independently:
 *     s_t  = scale * (q_lat[n,h,b] . c_b[t] + q_rope[n,h] . k_r[t])
 *     m    = max_t s_t                            (first pass)
 *     p_t  = exp(s_t - m) / sum_u exp(s_u - m)    (second pass)
 *     o    = sum_t p_t c_b[t]                     (values = the same latents)
 *     out[n,h,b,:] = out_scale * o
 *     lse[n,h,b]   = m + log(sum_u exp(s_u - m))  (natural log)
 *
 * Sources (the pages this follows):
 *  - "MLRA: Breaking the Sharding Bottleneck in Latent Attention" (wispaper.ai
 *    blog), section "The Core Insight: Sum of Branches, Not Sum of Keys":
 *    attention is computed on each latent block independently and the branch
 *    outputs are summed afterwards (the sum is in oracle_mlra_up_proj, after
 *    each branch's own up-projection).
 *  - same page, section "Mathematical Calibration: Scaling the Latents": a
 *    final rescaling factor multiplies the attention output (its symbol is
 *    lost in the text we have, so it is the argument out_scale).
 *  - "TransMLA: Multi-head latent attention is all you need" (Hacker News
 *    thread), the comment quoting section 3.3: only the latent
 *    representations are cached, so scores and values are taken against the
 *    latents directly after the key/value up-projections are absorbed.
 *
 * Readings of what the pages leave open (each is a library argument or a
 * layout choice; they are listed with reasons in the design notes):
 *  - one RoPE query per head and one RoPE key per token, both shared by all
 *    branches, already rotated upstream;
 *  - scale and out_scale are arguments;
 *  - L < 1, L > max_pages_per_seq * P, or a block-table entry outside
 *    [0, num_pages) make that sequence invalid: its outputs are set to 0, its
 *    lse to -inf, and the first such problem is returned as an error code
 *    (5 = bad page index, 6 = bad sequence length).
 *
 * Inputs may be given either as bf16 bit patterns (uint16) or as doubles;
 * bf16 -> double is exact, so both forms describe the same numbers.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_OK 0
#define ORACLE_ERR_ARG 1
#define ORACLE_ERR_BAD_INDEX 5
#define ORACLE_ERR_BAD_SEQLEN 6

/* Element type of an input array. */
#define ORACLE_BF16 0
#define ORACLE_F64 1

static double bf16_bits_to_double(uint16_t bits)
{
    uint32_t u = ((uint32_t)bits) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

static double load(const void* base, int64_t i, int kind)
{
    if (kind == ORACLE_BF16) return bf16_bits_to_double(((const uint16_t*)base)[i]);
    return ((const double*)base)[i];
}

/* Validity of one sequence: 0, or the error code that invalidates it. */
static int check_sequence(int32_t n, int32_t page_size, int32_t max_pages_per_seq,
                          int32_t num_pages, const int32_t* block_table,
                          const int32_t* seqlens)
{
    int64_t L = seqlens[n];
    if (L < 1 || L > (int64_t)max_pages_per_seq * page_size) return ORACLE_ERR_BAD_SEQLEN;
    int64_t used_pages = (L + page_size - 1) / page_size;
    for (int64_t j = 0; j < used_pages; ++j) {
        int32_t page = block_table[(int64_t)n * max_pages_per_seq + j];
        if (page < 0 || page >= num_pages) return ORACLE_ERR_BAD_INDEX;
    }
    return ORACLE_OK;
}

/*
 * Decode attention for the sequences listed in seq_ids (all of them when
 * seq_ids is NULL).  Layouts, all dense row-major:
 *   q_lat        [batch, heads, branches, d_c]
 *   q_rope       [batch, heads, d_r]
 *   latent_cache [num_pages, page_size, branches, d_c]
 *   rope_cache   [num_pages, page_size, d_r]
 *   block_table  [batch, max_pages_per_seq]   int32
 *   seqlens      [batch]                      int32
 *   out          [batch, heads, branches, d_c] double (listed sequences only)
 *   lse          [batch, heads, branches]      double, may be NULL
 * Returns 0, ORACLE_ERR_ARG, or the first per-sequence error code met (in
 * seq_ids order).
 */
int oracle_mlra_decode(int32_t batch, int32_t heads, int32_t branches, int32_t d_c,
                       int32_t d_r, int32_t page_size, int32_t max_pages_per_seq,
                       int32_t num_pages, int input_kind, const void* q_lat,
                       const void* q_rope, const void* latent_cache,
                       const void* rope_cache, const int32_t* block_table,
                       const int32_t* seqlens, double scale, double out_scale,
                       const int32_t* seq_ids, int32_t n_ids, double* out, double* lse)
{
    if (batch < 1 || heads < 1 || branches < 1 || d_c < 1 || d_r < 0 || page_size < 1 ||
        max_pages_per_seq < 1 || num_pages < 1)
        return ORACLE_ERR_ARG;
    if (input_kind != ORACLE_BF16 && input_kind != ORACLE_F64) return ORACLE_ERR_ARG;
    if (seq_ids == NULL) n_ids = batch;

    const int64_t row = (int64_t)branches * d_c; /* latent elements per token */
    int first_error = ORACLE_OK;

    for (int32_t i = 0; i < n_ids; ++i) {
        int32_t n = seq_ids ? seq_ids[i] : i;
        if (n < 0 || n >= batch) return ORACLE_ERR_ARG;
        int err = check_sequence(n, page_size, max_pages_per_seq, num_pages, block_table, seqlens);
        if (err != ORACLE_OK) {
            if (first_error == ORACLE_OK) first_error = err;
            for (int64_t j = 0; j < (int64_t)heads * row; ++j) out[(int64_t)n * heads * row + j] = 0.0;
            if (lse)
                for (int64_t j = 0; j < (int64_t)heads * branches; ++j)
                    lse[(int64_t)n * heads * branches + j] = -INFINITY;
            continue;
        }
        const int64_t L = seqlens[n];

        /* token t -> row of the pool: page * P + slot */
        int64_t* pool_row = (int64_t*)malloc(sizeof(int64_t) * L);
        for (int64_t t = 0; t < L; ++t) {
            int64_t page = block_table[(int64_t)n * max_pages_per_seq + t / page_size];
            pool_row[t] = page * page_size + t % page_size;
        }

        #pragma omp parallel for schedule(dynamic, 1)
        for (int64_t hb = 0; hb < (int64_t)heads * branches; ++hb) {
            const int64_t h = hb / branches, b = hb % branches;
            const int64_t q_off = (((int64_t)n * heads + h) * branches + b) * d_c;
            const int64_t qr_off = ((int64_t)n * heads + h) * d_r;
            double* s = (double*)malloc(sizeof(double) * L);
            double* acc = (double*)calloc((size_t)d_c, sizeof(double));

            /* pass 1: scores and their maximum */
            double m = -INFINITY;
            for (int64_t t = 0; t < L; ++t) {
                const int64_t c_off = pool_row[t] * row + b * d_c;
                const int64_t r_off = pool_row[t] * d_r;
                double dot = 0.0;
                for (int64_t k = 0; k < d_c; ++k)
                    dot += load(q_lat, q_off + k, input_kind) * load(latent_cache, c_off + k, input_kind);
                for (int64_t k = 0; k < d_r; ++k)
                    dot += load(q_rope, qr_off + k, input_kind) * load(rope_cache, r_off + k, input_kind);
                s[t] = scale * dot;
                if (s[t] > m) m = s[t];
            }
            /* pass 2: normaliser and probability-weighted sum of latents */
            double denom = 0.0;
            for (int64_t t = 0; t < L; ++t) denom += exp(s[t] - m);
            for (int64_t t = 0; t < L; ++t) {
                const double p = exp(s[t] - m) / denom;
                const int64_t c_off = pool_row[t] * row + b * d_c;
                for (int64_t k = 0; k < d_c; ++k) acc[k] += p * load(latent_cache, c_off + k, input_kind);
            }
            for (int64_t k = 0; k < d_c; ++k) out[q_off + k] = out_scale * acc[k];
            if (lse) lse[((int64_t)n * heads + h) * branches + b] = m + log(denom);
            free(acc);
            free(s);
        }
        free(pool_row);
    }
    return first_error;
}

/*
 * Per-branch W_UV up-projection followed by the branch sum:
 *   y[n, h*d_h + j] = sum_b sum_k out_lat[n,h,b,k] * w_uv[b][k][h*d_h + j]
 * ("The Core Insight" section of the blog page above: the branch outputs are
 * summed at the end; each branch has its own up-projection.)
 *   out_lat [batch, heads, branches, d_c] double
 *   w_uv    [branches, d_c, heads*d_h]    bf16 bits or double (input_kind)
 *   y       [batch, heads*d_h]            double
 */
int oracle_mlra_up_proj(int32_t batch, int32_t heads, int32_t branches, int32_t d_c,
                        int32_t d_h, int input_kind, const double* out_lat, const void* w_uv,
                        double* y)
{
    if (batch < 1 || heads < 1 || branches < 1 || d_c < 1 || d_h < 1) return ORACLE_ERR_ARG;
    if (input_kind != ORACLE_BF16 && input_kind != ORACLE_F64) return ORACLE_ERR_ARG;
    const int64_t width = (int64_t)heads * d_h;
    #pragma omp parallel for schedule(static)
    for (int64_t nh = 0; nh < (int64_t)batch * heads; ++nh) {
        const int64_t n = nh / heads, h = nh % heads;
        for (int64_t j = 0; j < d_h; ++j) {
            double sum = 0.0;
            for (int64_t b = 0; b < branches; ++b)
                for (int64_t k = 0; k < d_c; ++k)
                    sum += out_lat[((n * heads + h) * branches + b) * d_c + k] *
                           load(w_uv, (b * d_c + k) * width + h * d_h + j, input_kind);
            y[n * width + h * d_h + j] = sum;
        }
    }
    return ORACLE_OK;
}

/*
 * Output gate ("Critical Insight: The Value of 'Gating'" section of the blog
 * page above: a gate on the attention output adds a non-linearity; its
 * formula is lost in the page text, read as the usual elementwise sigmoid
 * gate):
 *   y[i] = y[i] / (1 + exp(-gate[i]))     for i < count
 *   gate  bf16 bits or double (input_kind), y double (in place)
 */
int oracle_mlra_gate(int64_t count, int input_kind, const void* gate, double* y)
{
    if (count < 0) return ORACLE_ERR_ARG;
    if (input_kind != ORACLE_BF16 && input_kind != ORACLE_F64) return ORACLE_ERR_ARG;
    for (int64_t i = 0; i < count; ++i)
        y[i] = y[i] / (1.0 + exp(-load(gate, i, input_kind)));
    return ORACLE_OK;
}

/*
 * Decode pre-step: the work between the layer's projections and the decode
 * attention for one new token per sequence.
 *
 *  1. Query absorption (the key up-projection folded into the query; the
 *     "TransMLA" Hacker News thread quotes that only latents are cached and
 *     attention runs against them after absorption; "The Core Insight" of the
 *     blog page: each branch b has its own up-projection per head h):
 *        q_lat[n,h,b,k] = sum_j w_uk[b,h,j,k] * q_c[n,h,j]
 *  2. Rotary position embedding of the RoPE query and of the new token's
 *     shared RoPE key at the new token's position p = seqlens[n] - 1, as
 *     RoFormer defines it (pairs of adjacent dimensions rotated):
 *        theta_i = base^(-2 i / d_r),  a = p * theta_i,  i < d_r / 2
 *        x'[2i]   = x[2i] cos a - x[2i+1] sin a
 *        x'[2i+1] = x[2i] sin a + x[2i+1] cos a
 *  3. Append: the new token's latents c_new[n] and rotated key go to
 *     page = block_table[n][p / P], slot = p mod P.
 *
 *   q_c     [batch, heads, d_h]            w_uk [branches, heads, d_h, d_c]
 *   q_r     [batch, heads, d_r] (unrotated) kr_new [batch, d_r] (unrotated)
 *   inputs as bf16 bits or doubles (input_kind)
 *   q_lat   [batch, heads, branches, d_c] double (written)
 *   q_rope  [batch, heads, d_r]           double (written, rotated)
 *   kr_rot  [batch, d_r]                  double (written, rotated)
 *   dest    [batch, 2] int32: (page, slot) the new token goes to, or (-1, -1)
 *           when seqlens[n] < 1, p >= max_pages_per_seq * P or the page is
 *           outside [0, num_pages) (the first such problem is returned:
 *           6 = bad length, 5 = bad page)
 */
int oracle_mlra_prepare(int32_t batch, int32_t heads, int32_t branches, int32_t d_c, int32_t d_h,
                        int32_t d_r, int32_t page_size, int32_t max_pages_per_seq,
                        int32_t num_pages, int input_kind, const void* q_c, const void* q_r,
                        const void* w_uk, const void* kr_new, const int32_t* seqlens,
                        const int32_t* block_table, double rope_base, double* q_lat,
                        double* q_rope, double* kr_rot, int32_t* dest)
{
    if (batch < 1 || heads < 1 || branches < 1 || d_c < 1 || d_h < 1 || d_r < 2 || d_r % 2 ||
        page_size < 1 || max_pages_per_seq < 1 || num_pages < 1 || !(rope_base > 1.0))
        return ORACLE_ERR_ARG;
    if (input_kind != ORACLE_BF16 && input_kind != ORACLE_F64) return ORACLE_ERR_ARG;
    int status = ORACLE_OK;
    for (int64_t n = 0; n < batch; ++n) {
        for (int64_t h = 0; h < heads; ++h)
            for (int64_t b = 0; b < branches; ++b)
                for (int64_t k = 0; k < d_c; ++k) {
                    double sum = 0.0;
                    for (int64_t j = 0; j < d_h; ++j)
                        sum += load(w_uk, ((b * heads + h) * d_h + j) * d_c + k, input_kind) *
                               load(q_c, (n * heads + h) * d_h + j, input_kind);
                    q_lat[((n * heads + h) * branches + b) * d_c + k] = sum;
                }
        const int64_t p = (int64_t)seqlens[n] - 1;
        for (int64_t i = 0; i < d_r / 2; ++i) {
            const double a = (double)(p < 0 ? 0 : p) * pow(rope_base, -2.0 * (double)i / (double)d_r);
            const double c = cos(a), sn = sin(a);
            for (int64_t h = 0; h < heads; ++h) {
                const int64_t o = (n * heads + h) * d_r + 2 * i;
                const double x0 = load(q_r, o, input_kind), x1 = load(q_r, o + 1, input_kind);
                q_rope[o] = x0 * c - x1 * sn;
                q_rope[o + 1] = x0 * sn + x1 * c;
            }
            const double k0 = load(kr_new, n * d_r + 2 * i, input_kind);
            const double k1 = load(kr_new, n * d_r + 2 * i + 1, input_kind);
            kr_rot[n * d_r + 2 * i] = k0 * c - k1 * sn;
            kr_rot[n * d_r + 2 * i + 1] = k0 * sn + k1 * c;
        }
        dest[2 * n] = dest[2 * n + 1] = -1;
        if (p < 0 || p >= (int64_t)max_pages_per_seq * page_size) {
            if (status == ORACLE_OK) status = ORACLE_ERR_BAD_SEQLEN;
            continue;
        }
        const int32_t page = block_table[n * (int64_t)max_pages_per_seq + p / page_size];
        if (page < 0 || page >= num_pages) {
            if (status == ORACLE_OK) status = ORACLE_ERR_BAD_INDEX;
            continue;
        }
        dest[2 * n] = page;
        dest[2 * n + 1] = (int32_t)(p % page_size);
    }
    return status;
}

/* Threads OpenMP will use (1 when built without OpenMP). */
#ifdef _OPENMP
#include <omp.h>
int oracle_num_threads(void) { return omp_get_max_threads(); }
void oracle_set_num_threads(int n) { if (n > 0) omp_set_num_threads(n); }
#else
int oracle_num_threads(void) { return 1; }
void oracle_set_num_threads(int n) { (void)n; }
#endif
