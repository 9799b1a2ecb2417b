/*
 * msa_oracle.c -- plain, slow, float64 CPU oracle of the MiniMax Sparse
 * Attention (MSA) decode path.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test-suite, the smoke check and the
 * benchmark's CPU-baseline leg may load this library.  It shares no code,
 * header, table or helper with the CUDA library: every format decoder and
 * every step below is written out again here from its definition.
 *
 * Source of the method: the vLLM blog post "vLLM 為 MiniMax-M3.1-Flash 提供
 * Day-0 支援" (hot.atechcom.net), cited below as [post, "<section>"]:
 *   - "MSA primer": 128-token blocks; one index query per GQA group scores
 *     every cached key against one shared index-key head; max-pool to one
 *     score per block; exact attention over the top 16 blocks, the most
 *     recent block always kept, at most 2,048 keys per query.
 *   - "What is new in the MiniMax-M3.1 architecture": NVFP4 KV cache for
 *     both the indexer and the attention path.
 *   - "NVIDIA Blackwell optimized MSA kernels": the query stays FP8, the
 *     NVFP4 cache is dequantised to FP8 (E4M3) and fed to an FP8 MMA; each
 *     E2M1 value times its E4M3 scale is therefore re-rounded to E4M3.
 *   - "NVIDIA Rubin optimized MSA": names that E4M3 re-rounding explicitly.
 * Number formats (the pages name them only): OCP "Microscaling Formats (MX)
 * v1.0" -- FP4 E2M1 (no inf/NaN, max 6) and FP8 E4M3 (bias 7, subnormals,
 * max 448, S.1111.111 = NaN, no infinities).
 *
 * Readings where the pages are silent (each one is listed in the design
 * notes): raw dot-product index score; 16 selected blocks in total including
 * the forced latest one; ties broken by the lower block id; a query sees
 * every cached key up to and including its own position; a partially filled
 * last block pools and attends only over its valid tokens; the per-tensor
 * fp32 scale is applied after the E4M3 re-rounding.
 *
 * Cache layout read here (the library's layout, restated, not included):
 *   index keys NVFP4: data [page][128 tok][64 B], scale [page][128 tok][8 B]
 *   index keys FP8  : data [page][128 tok][128 B]
 *   K and V  NVFP4  : data [page][4 kv][128 tok][64 B], scale [page][4][128][8]
 *   element d of a 128-vector: byte d/2, low nibble for even d, high for odd;
 *   scale byte s covers elements 16s .. 16s+15.
 *   logical block i of sequence b lives in page page_table[b*max_pages+i]
 *   (or page b*max_pages+i when page_table is NULL).
 * Parallelism: plain pthreads over independent (sequence, token) rows.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORC_BLOCK 128   /* tokens per block  [post, "MSA primer"] */
#define ORC_TOPK 16     /* blocks attended   [post, "MSA primer"] */
#define ORC_D 128       /* head dim          [post, "MSA primer"] */
#define ORC_G 4         /* KV heads = GQA groups = index queries per token */
#define ORC_HPG 16      /* query heads per group */
#define ORC_HQ (ORC_G * ORC_HPG)

/* ------------------------------------------------------------------------ */
/* Number formats (OCP MX v1.0)                                              */
/* ------------------------------------------------------------------------ */

/* FP4 E2M1: bit 3 sign, bits 2..1 exponent (bias 1), bit 0 mantissa. */
double orc_e2m1(unsigned code)
{
    unsigned e = (code >> 1) & 3u, m = code & 1u;
    double mag = (e == 0) ? 0.5 * m : ldexp(1.0 + 0.5 * m, (int)e - 1);
    return (code & 8u) ? -mag : mag;
}

/* FP8 E4M3: bit 7 sign, bits 6..3 exponent (bias 7), bits 2..0 mantissa;
 * exponent 0 is subnormal (m * 2^-9); S.1111.111 is NaN; no infinities. */
double orc_e4m3(unsigned byte)
{
    unsigned e = (byte >> 3) & 15u, m = byte & 7u;
    double mag;
    if (e == 15 && m == 7) return NAN;
    mag = (e == 0) ? ldexp((double)m, -9) : ldexp(1.0 + m / 8.0, (int)e - 7);
    return (byte & 0x80u) ? -mag : mag;
}

/* Round a real to E4M3: round to nearest, ties to even, on the E4M3 grid
 * (subnormals included); magnitudes above 448 saturate to 448; NaN -> 0x7F.
 * This is the re-rounding step of [post, "NVIDIA Blackwell optimized MSA
 * kernels"] and [post, "NVIDIA Rubin optimized MSA"]. */
unsigned orc_e4m3_round(double x)
{
    unsigned sign, e_field, m;
    double a, n;
    int e;
    if (isnan(x)) return 0x7Fu;
    sign = signbit(x) ? 0x80u : 0u;
    a = fabs(x);
    if (a >= 448.0) return sign | 0x7Eu;
    if (a < ldexp(1.0, -6)) {                 /* subnormal range, quantum 2^-9 */
        n = nearbyint(ldexp(a, 9));           /* ties to even (default mode) */
        if (n >= 8.0) return sign | 0x08u;    /* rounded up to 2^-6 */
        return sign | (unsigned)n;
    }
    frexp(a, &e);                              /* a = f * 2^e, f in [0.5,1) */
    e -= 1;                                    /* a in [2^e, 2^(e+1)) */
    n = nearbyint(ldexp(a, 3 - e));            /* in [8, 16] */
    if (n >= 16.0) { n = 8.0; e += 1; }
    m = (unsigned)n - 8u;
    e_field = (unsigned)(e + 7);
    if (e_field > 15u || (e_field == 15u && m > 6u)) return sign | 0x7Eu;
    return sign | (e_field << 3) | m;
}

/* One NVFP4 element before the per-tensor scale:
 * E4M3( RNE_sat( e2m1(code) * e4m3(scale) ) ), returned as its real value. */
double orc_nvfp4_elem(unsigned code, unsigned scale_byte)
{
    double prod = orc_e2m1(code) * orc_e4m3(scale_byte);  /* exact in f64 */
    return orc_e4m3(orc_e4m3_round(prod));
}

/* Nibble d of a packed 128-element FP4 row. */
static unsigned nib(const uint8_t* row, int d)
{
    uint8_t by = row[d >> 1];
    return (d & 1) ? (by >> 4) : (by & 15u);
}

/* Decode one packed NVFP4 row of 128 elements into v[] (no tensor scale). */
static void decode_nvfp4_row(const uint8_t* data64, const uint8_t* scale8, double* v)
{
    for (int d = 0; d < ORC_D; ++d) v[d] = orc_nvfp4_elem(nib(data64, d), scale8[d / 16]);
}

/* ------------------------------------------------------------------------ */
/* Cache description                                                         */
/* ------------------------------------------------------------------------ */

typedef struct {
    const uint8_t *idx_data, *idx_scale;     /* idx_scale unused for FP8 */
    const uint8_t *k_data, *k_scale, *v_data, *v_scale;
    double s_idx, s_k, s_v;
    int64_t num_pages;
    int idx_mode;                            /* 0: NVFP4 index keys, 1: FP8,
                                                2: NVFP4 scored at exact value */
    const int32_t* page_table;               /* [B][max_pages] or NULL */
    int64_t max_pages;
    const int32_t* seq_lens;                 /* [B] */
    int batch, q_tokens;
} orc_cache;

/* Physical page of logical block blk of sequence b, or -1 if out of range. */
static int64_t page_of(const orc_cache* c, int b, int64_t blk)
{
    int64_t p;
    if (blk < 0 || blk >= c->max_pages) return -1;
    p = c->page_table ? (int64_t)c->page_table[(int64_t)b * c->max_pages + blk]
                      : (int64_t)b * c->max_pages + blk;
    if (p < 0 || p >= c->num_pages) return -1;
    return p;
}

/* Index key of logical token j of sequence b (no tensor scale).
 * Mode 2 is the exact variant of [post, "NVIDIA Rubin optimized MSA"]: the
 * NVFP4 keys are converted to FP16 and scored with an FP16 MMA, so the scores
 * carry no E4M3 re-rounding; e2m1 * e4m3 is exact in FP16 (at most 5
 * significant bits, magnitude 2^-10 .. 2688), hence the key is that product. */
static int index_key(const orc_cache* c, int b, int64_t j, double* v)
{
    int64_t p = page_of(c, b, j / ORC_BLOCK);
    int64_t r = j % ORC_BLOCK;
    if (p < 0) return -1;
    if (c->idx_mode == 1) {
        const uint8_t* row = c->idx_data + (p * ORC_BLOCK + r) * ORC_D;
        for (int d = 0; d < ORC_D; ++d) v[d] = orc_e4m3(row[d]);
    } else if (c->idx_mode == 2) {
        const uint8_t* row = c->idx_data + (p * ORC_BLOCK + r) * 64;
        const uint8_t* sc = c->idx_scale + (p * ORC_BLOCK + r) * 8;
        for (int d = 0; d < ORC_D; ++d) v[d] = orc_e2m1(nib(row, d)) * orc_e4m3(sc[d / 16]);
    } else {
        decode_nvfp4_row(c->idx_data + (p * ORC_BLOCK + r) * 64,
                         c->idx_scale + (p * ORC_BLOCK + r) * 8, v);
    }
    return 0;
}

/* K (kv=0) or V (kv=1) row of KV head g at logical token j (no tensor scale). */
static int kv_row(const orc_cache* c, int kv, int b, int g, int64_t j, double* v)
{
    int64_t p = page_of(c, b, j / ORC_BLOCK);
    int64_t r = j % ORC_BLOCK;
    int64_t row = (p * ORC_G + g) * ORC_BLOCK + r;
    if (p < 0) return -1;
    decode_nvfp4_row((kv ? c->v_data : c->k_data) + row * 64,
                     (kv ? c->v_scale : c->k_scale) + row * 8, v);
    return 0;
}

/* 0-based position of query token t of sequence b: the cached length counts
 * the T new tokens, so the last query sits at L_b - 1. */
static int64_t query_pos(const orc_cache* c, int b, int t)
{
    return (int64_t)c->seq_lens[b] - c->q_tokens + t;
}

static int row_ok(const orc_cache* c, int b, int t)
{
    int64_t L;
    if (b < 0 || b >= c->batch || t < 0 || t >= c->q_tokens) return 0;
    L = c->seq_lens[b];
    return L >= c->q_tokens && L <= c->max_pages * ORC_BLOCK;
}

/* ------------------------------------------------------------------------ */
/* Tiny parallel-for over rows (pthreads)                                    */
/* ------------------------------------------------------------------------ */

typedef void (*row_fn)(void* ctx, int64_t row);
typedef struct { row_fn fn; void* ctx; int64_t n, next; pthread_mutex_t mu; } pfor_t;

static void* pfor_worker(void* arg)
{
    pfor_t* P = (pfor_t*)arg;
    for (;;) {
        int64_t r;
        pthread_mutex_lock(&P->mu);
        r = P->next++;
        pthread_mutex_unlock(&P->mu);
        if (r >= P->n) break;
        P->fn(P->ctx, r);
    }
    return NULL;
}

static int g_threads = 1;
void orc_set_threads(int n) { g_threads = n < 1 ? 1 : (n > 256 ? 256 : n); }
int orc_get_threads(void) { return g_threads; }

static void parallel_rows(row_fn fn, void* ctx, int64_t n)
{
    pfor_t P;
    pthread_t th[256];
    int k, nt = g_threads < n ? g_threads : (int)(n > 0 ? n : 1);
    P.fn = fn; P.ctx = ctx; P.n = n; P.next = 0;
    pthread_mutex_init(&P.mu, NULL);
    if (nt <= 1) { pfor_worker(&P); pthread_mutex_destroy(&P.mu); return; }
    for (k = 0; k < nt; ++k) pthread_create(&th[k], NULL, pfor_worker, &P);
    for (k = 0; k < nt; ++k) pthread_join(th[k], NULL);
    pthread_mutex_destroy(&P.mu);
}

/* ------------------------------------------------------------------------ */
/* Step 1: indexer token scores                                              */
/*   s[j] = s_qi * s_idx * sum_d qi[d] * k_idx[j][d],  j <= pos              */
/* [post, "MSA primer"]: one index query per GQA group, one shared index-key */
/* head, every cached key scored.                                            */
/* ------------------------------------------------------------------------ */

typedef struct {
    const orc_cache* c;
    const uint8_t* qi;          /* [B][T][4][128] E4M3 */
    double s_qi;
    const int32_t *rows_b, *rows_t;
    int64_t ctx_cap;            /* row stride of the token-score output */
    double* scores;             /* [rows][4][ctx_cap] */
    double* block_scores;       /* [rows][4][max_pages] */
    int* status;
} idx_ctx;

static void indexer_row(void* vctx, int64_t row)
{
    idx_ctx* X = (idx_ctx*)vctx;
    const orc_cache* c = X->c;
    int b = X->rows_b[row], t = X->rows_t[row];
    double q[ORC_G][ORC_D], k[ORC_D];
    int64_t pos, j, i;
    if (!row_ok(c, b, t)) { X->status[row] = -1; return; }
    pos = query_pos(c, b, t);
    for (int g = 0; g < ORC_G; ++g)
        for (int d = 0; d < ORC_D; ++d)
            q[g][d] = orc_e4m3(X->qi[(((int64_t)b * c->q_tokens + t) * ORC_G + g) * ORC_D + d]);
    if (X->block_scores)
        for (int g = 0; g < ORC_G; ++g)
            for (i = 0; i < c->max_pages; ++i)
                X->block_scores[(row * ORC_G + g) * c->max_pages + i] = -INFINITY;
    for (j = 0; j <= pos; ++j) {
        if (index_key(c, b, j, k)) { X->status[row] = -2; return; }
        for (int g = 0; g < ORC_G; ++g) {
            double acc = 0.0, s;
            for (int d = 0; d < ORC_D; ++d) acc += q[g][d] * k[d];
            s = X->s_qi * c->s_idx * acc;
            if (X->scores && j < X->ctx_cap) X->scores[(row * ORC_G + g) * X->ctx_cap + j] = s;
            /* Step 2, max-pool over the valid tokens of block j/128 [post, "MSA primer"] */
            if (X->block_scores) {
                double* S = &X->block_scores[(row * ORC_G + g) * c->max_pages + j / ORC_BLOCK];
                if (s > *S) *S = s;
            }
        }
    }
    X->status[row] = 0;
}

/* Token scores and/or block scores for the listed (b, t) rows.
 * scores: [n_rows][4][ctx_cap] (entries j > pos untouched) or NULL;
 * block_scores: [n_rows][4][max_pages], -inf for blocks with no valid key.
 * Returns 0, or the negative status of the first bad row. */
int orc_indexer(const orc_cache* c, const uint8_t* qi, double s_qi,
                const int32_t* rows_b, const int32_t* rows_t, int64_t n_rows,
                double* scores, int64_t ctx_cap, double* block_scores)
{
    idx_ctx X;
    int* st = (int*)calloc((size_t)(n_rows > 0 ? n_rows : 1), sizeof(int));
    int rc = 0;
    X.c = c; X.qi = qi; X.s_qi = s_qi; X.rows_b = rows_b; X.rows_t = rows_t;
    X.ctx_cap = ctx_cap; X.scores = scores; X.block_scores = block_scores; X.status = st;
    parallel_rows(indexer_row, &X, n_rows);
    for (int64_t r = 0; r < n_rows; ++r) if (st[r] && !rc) rc = st[r];
    free(st);
    return rc;
}

/* ------------------------------------------------------------------------ */
/* Step 3: block selection                                                   */
/* [post, "MSA primer"]: the top 16 blocks, the most recent always kept.     */
/* Reading: 16 in total; others ranked by (score desc, block id asc); a      */
/* query whose visible context has <= 16 blocks takes all of them.           */
/* Output ids ascending, padded with -1.                                     */
/* ------------------------------------------------------------------------ */

/* Does block a rank before block b?  (higher score, then lower id) */
static int ranks_before(const double* S, int64_t a, int64_t b)
{
    if (S[a] > S[b]) return 1;
    if (S[a] < S[b]) return 0;
    return a < b;
}

/* Select for one (row, group).  nb = number of visible blocks. */
static void select_one(const double* S, int64_t nb, int32_t* sel)
{
    int64_t chosen[ORC_TOPK];
    int n = 0;
    if (nb <= ORC_TOPK) {
        for (int64_t i = 0; i < nb; ++i) chosen[n++] = i;
    } else {
        int64_t latest = nb - 1;
        chosen[n++] = latest;
        /* 15 rounds of "best remaining" -- a plain selection by definition */
        for (int r = 0; r < ORC_TOPK - 1; ++r) {
            int64_t best = -1;
            for (int64_t i = 0; i < latest; ++i) {
                int taken = 0;
                for (int k = 0; k < n; ++k) if (chosen[k] == i) { taken = 1; break; }
                if (taken) continue;
                if (best < 0 || ranks_before(S, i, best)) best = i;
            }
            chosen[n++] = best;
        }
    }
    /* ascending ids */
    for (int a = 0; a < n; ++a)
        for (int b2 = a + 1; b2 < n; ++b2)
            if (chosen[b2] < chosen[a]) { int64_t tmp = chosen[a]; chosen[a] = chosen[b2]; chosen[b2] = tmp; }
    for (int k = 0; k < ORC_TOPK; ++k) sel[k] = k < n ? (int32_t)chosen[k] : -1;
}

/* block_scores: [n_rows][4][max_pages]; sel: [n_rows][4][16]. */
int orc_select(const orc_cache* c, const int32_t* rows_b, const int32_t* rows_t, int64_t n_rows,
               const double* block_scores, int32_t* sel)
{
    for (int64_t r = 0; r < n_rows; ++r) {
        int b = rows_b[r], t = rows_t[r];
        int64_t nb;
        if (!row_ok(c, b, t)) return -1;
        nb = query_pos(c, b, t) / ORC_BLOCK + 1;
        for (int g = 0; g < ORC_G; ++g)
            select_one(block_scores + (r * ORC_G + g) * c->max_pages, nb,
                       sel + (r * ORC_G + g) * ORC_TOPK);
    }
    return 0;
}

/* ------------------------------------------------------------------------ */
/* Step 4: exact attention over the selected blocks                         */
/* [post, "MSA primer"] and Figure 1 caption: every query head of a group   */
/* attends over its group's selected blocks.  Query head h uses KV head h/16.*/
/*   z_j = scale * s_q * s_k * q.k_j  over selected j <= pos                */
/*   o   = s_v * sum_j softmax(z)_j v_j                                     */
/* ------------------------------------------------------------------------ */

typedef struct {
    const orc_cache* c;
    const uint8_t* q;           /* [B][T][64][128] E4M3 */
    double s_q, softmax_scale;
    const int32_t *rows_b, *rows_t;
    const int32_t* sel;         /* [rows][4][16] */
    double* out;                /* [rows][64][128] */
    int* status;
} att_ctx;

static void attention_row(void* vctx, int64_t row)
{
    att_ctx* X = (att_ctx*)vctx;
    const orc_cache* c = X->c;
    int b = X->rows_b[row], t = X->rows_t[row];
    int64_t pos, nkeys;
    double *K, *V, *z;
    if (!row_ok(c, b, t)) { X->status[row] = -1; return; }
    pos = query_pos(c, b, t);
    K = (double*)malloc(sizeof(double) * ORC_TOPK * ORC_BLOCK * ORC_D);
    V = (double*)malloc(sizeof(double) * ORC_TOPK * ORC_BLOCK * ORC_D);
    z = (double*)malloc(sizeof(double) * ORC_TOPK * ORC_BLOCK);
    for (int g = 0; g < ORC_G; ++g) {
        const int32_t* s = X->sel + (row * ORC_G + g) * ORC_TOPK;
        /* gather the keys of the selected blocks that the query may see */
        nkeys = 0;
        for (int k = 0; k < ORC_TOPK; ++k) {
            if (s[k] < 0) continue;
            for (int64_t r = 0; r < ORC_BLOCK; ++r) {
                int64_t j = (int64_t)s[k] * ORC_BLOCK + r;
                if (j > pos) break;
                if (kv_row(c, 0, b, g, j, K + nkeys * ORC_D) ||
                    kv_row(c, 1, b, g, j, V + nkeys * ORC_D)) { X->status[row] = -2; goto done; }
                ++nkeys;
            }
        }
        for (int hh = 0; hh < ORC_HPG; ++hh) {
            int h = g * ORC_HPG + hh;
            double qv[ORC_D], zmax = -INFINITY, denom = 0.0;
            double* o = X->out + (row * ORC_HQ + h) * ORC_D;
            for (int d = 0; d < ORC_D; ++d)
                qv[d] = orc_e4m3(X->q[(((int64_t)b * c->q_tokens + t) * ORC_HQ + h) * ORC_D + d]);
            for (int64_t n = 0; n < nkeys; ++n) {
                double acc = 0.0;
                for (int d = 0; d < ORC_D; ++d) acc += qv[d] * K[n * ORC_D + d];
                z[n] = X->softmax_scale * X->s_q * c->s_k * acc;
                if (z[n] > zmax) zmax = z[n];
            }
            for (int64_t n = 0; n < nkeys; ++n) { z[n] = exp(z[n] - zmax); denom += z[n]; }
            for (int d = 0; d < ORC_D; ++d) {
                double acc = 0.0;
                for (int64_t n = 0; n < nkeys; ++n) acc += z[n] * V[n * ORC_D + d];
                o[d] = nkeys ? c->s_v * acc / denom : 0.0;
            }
        }
    }
    X->status[row] = 0;
done:
    free(K); free(V); free(z);
}

int orc_attention(const orc_cache* c, const uint8_t* q, double s_q, double softmax_scale,
                  const int32_t* rows_b, const int32_t* rows_t, int64_t n_rows,
                  const int32_t* sel, double* out)
{
    att_ctx X;
    int* st = (int*)calloc((size_t)(n_rows > 0 ? n_rows : 1), sizeof(int));
    int rc = 0;
    X.c = c; X.q = q; X.s_q = s_q; X.softmax_scale = softmax_scale;
    X.rows_b = rows_b; X.rows_t = rows_t; X.sel = sel; X.out = out; X.status = st;
    parallel_rows(attention_row, &X, n_rows);
    for (int64_t r = 0; r < n_rows; ++r) if (st[r] && !rc) rc = st[r];
    free(st);
    return rc;
}

/* ------------------------------------------------------------------------ */
/* Helpers exposed for the pins                                              */
/* ------------------------------------------------------------------------ */

/* Decode a whole NVFP4 row (128 elements) -- used by the pins to compare the
 * oracle's decoder against an independent library conversion. */
void orc_decode_nvfp4_row(const uint8_t* data64, const uint8_t* scale8, double* out128)
{
    decode_nvfp4_row(data64, scale8, out128);
}

/* ------------------------------------------------------------------------ */
/* Writing new tokens into the cache (NVFP4 / FP8 encode)                    */
/* ------------------------------------------------------------------------ */
/* The step before the decode path: the T new tokens' K, V and index key are
 * quantised into the paged cache ([post, "What is new in the MiniMax-M3.1
 * architecture"]: NVFP4 KV cache for indexer and attention; [post, "QKV GEMM
 * + norm + RoPE + KV insert fusion"] names the insertion).  The pages do not
 * spell out the quantiser; the reading taken (listed in the design notes):
 *   per 16 elements   r  = amax / (6 * s_t)              (fp32 arithmetic)
 *                     sb = E4M3 of r, nearest, ties to even, saturating
 *                     u  = e4m3(sb) * s_t                 (fp32)
 *   per element       y  = x / u                          (fp32)
 *                     code = nearest E2M1 magnitude of |y|, ties to the even
 *                     code, saturating at 6; sign bit set for x < 0 unless
 *                     the magnitude is 0; u == 0 gives code 0.
 *   FP8 index keys    E4M3 of x / s_idx (fp32), nearest-even, saturating.
 * The divisions whose results decide the codes are done in fp32, the
 * precision a kernel takes them in, so that both sides decide alike. */

/* Nearest E2M1 magnitude code (0..7) of y >= 0: the grid point at the
 * smallest distance; on a tie the code with mantissa bit 0. */
unsigned orc_e2m1_round(double y)
{
    unsigned best = 0;
    double bd = INFINITY;
    if (!(y > 0.0)) return 0u;
    if (y >= 6.0) return 7u;                  /* saturates at the largest value */
    for (unsigned c = 0; c < 8u; ++c) {
        const double d = fabs(y - orc_e2m1(c));
        if (d < bd || (d == bd && (c & 1u) == 0u)) { bd = d; best = c; }
    }
    return best;
}

/* One 128-element row x (fp32 values) -> packed codes [64] + scales [8]. */
void orc_nvfp4_encode_row(const float* x, float s_t, uint8_t* data64, uint8_t* scale8)
{
    volatile float six_st = 6.0f * s_t;       /* volatile: one fp32 rounding each */
    for (int j = 0; j < ORC_D / 16; ++j) {
        float amax = 0.0f;
        for (int i = 0; i < 16; ++i) {
            const float a = fabsf(x[16 * j + i]);
            if (a > amax) amax = a;
        }
        volatile float r = amax / six_st;
        const unsigned sb = orc_e4m3_round((double)r);
        volatile float u = (float)orc_e4m3(sb) * s_t;
        scale8[j] = (uint8_t)sb;
        for (int i = 0; i < 16; ++i) {
            const int d = 16 * j + i;
            unsigned code = 0u;
            if (u != 0.0f) {
                volatile float y = x[d] / u;
                code = orc_e2m1_round(fabs((double)y));
                if (code != 0u && x[d] < 0.0f) code |= 8u;
            }
            if (d & 1) data64[d >> 1] = (uint8_t)((data64[d >> 1] & 0x0Fu) | (code << 4));
            else data64[d >> 1] = (uint8_t)((data64[d >> 1] & 0xF0u) | code);
        }
    }
}

/* One 128-element row -> FP8 E4M3 bytes. */
void orc_fp8_encode_row(const float* x, float s_t, uint8_t* out128)
{
    for (int d = 0; d < ORC_D; ++d) {
        volatile float y = x[d] / s_t;
        out128[d] = (uint8_t)orc_e4m3_round((double)y);
    }
}

/* Write the T new tokens of every sequence (positions L-T .. L-1) into the
 * cache c (whose buffers the caller owns and lets this function write):
 * k_new, v_new [B][T][4][128], idx_new [B][T][128], fp32 values; s_* are the
 * cache's fp32 tensor scales.  Returns -1 if a position has no page. */
int orc_kv_insert(const orc_cache* c, const float* k_new, const float* v_new,
                  const float* idx_new, float s_idx, float s_k, float s_v)
{
    int rc = 0;
    for (int b = 0; b < c->batch; ++b) {
        for (int t = 0; t < c->q_tokens; ++t) {
            const int64_t pos = query_pos(c, b, t);
            const int64_t p = page_of(c, b, pos / ORC_BLOCK);
            const int64_t slot = pos % ORC_BLOCK;
            const int64_t tok = (int64_t)b * c->q_tokens + t;
            if (p < 0 || !row_ok(c, b, t)) { rc = -1; continue; }
            for (int g = 0; g < ORC_G; ++g) {
                const int64_t r = (p * ORC_G + g) * ORC_BLOCK + slot;
                orc_nvfp4_encode_row(k_new + (tok * ORC_G + g) * ORC_D, s_k,
                                     (uint8_t*)c->k_data + r * 64, (uint8_t*)c->k_scale + r * 8);
                orc_nvfp4_encode_row(v_new + (tok * ORC_G + g) * ORC_D, s_v,
                                     (uint8_t*)c->v_data + r * 64, (uint8_t*)c->v_scale + r * 8);
            }
            {
                const int64_t r = p * ORC_BLOCK + slot;
                if (c->idx_mode == 1)
                    orc_fp8_encode_row(idx_new + tok * ORC_D, s_idx, (uint8_t*)c->idx_data + r * 128);
                else
                    orc_nvfp4_encode_row(idx_new + tok * ORC_D, s_idx, (uint8_t*)c->idx_data + r * 64,
                                         (uint8_t*)c->idx_scale + r * 8);
            }
        }
    }
    return rc;
}
