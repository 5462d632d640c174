/*
 * oracle.c -- plain, slow, fp64 reference for paged-KV GQA decode attention
 * with dynamic split-KV scheduling.
 *
 * TEST INFRASTRUCTURE ONLY. Only the tests, the smoke check and the bench's
 * CPU-baseline / reference arm may load this library. The CUDA path shares no
 * code with it: no headers, helpers, tables or constants.
 *
 * What it follows:
 *  - "PaddlePaddle/HALOps" README, Highlights, GQA attention item: decode over
 *    a paged KV cache, BF16 / FP8 KV, GQA, speculative decoding, split-KV.
 *  - "HPC-Ops: Tencent's CUDA Kernel Library for LLM Inference Hot Paths",
 *    section "How the kernels are organized around specific workload shapes":
 *    uniform KV tiles, greedy bin-packing of the tiles onto CTAs before each
 *    decode step, and a combine kernel that merges the split results.
 *  The attention itself is plain scaled-dot-product attention, which the pages
 *  take for granted; it is written out below by its definition, in fp64, with an
 *  explicit full softmax (no blocking, no online rescaling, no split).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

typedef struct {
    int32_t batch, q_tokens, n_q_heads, n_kv_heads, head_dim, page_size, num_pages, max_pages_per_seq;
    int32_t kv_fp8;              /* 0: K/V hold bf16 bit patterns, 1: OCP E4M3 codes */
    int32_t pad_;
    double sm_scale;
    const uint16_t *q;           /* bf16 bits [B][T][Hq][d] */
    const void *k_pages;         /* [num_pages][Hkv][P][d] */
    const void *v_pages;
    const float *kv_scales;      /* [2][num_pages][Hkv]: K scales, then V scales (FP8 only) */
    const int32_t *page_table;   /* [B][max_pages_per_seq] */
    const int32_t *seq_lens;     /* [B] */
    /* block-sparse decode (NULL: every key may be seen): bit i % 32 of word i / 32 of row
     * (b * Hkv + h) keeps tile i = keys [i * tile_len, (i + 1) * tile_len) of (b, h) */
    const uint32_t *tile_mask;
    int32_t mask_words, tile_len;
} oracle_problem;

/* Whether key j of (b, h) lies in a kept tile ("HPC-Ops ...", "How the kernels are organized
 * around specific workload shapes": sparse attention skips the KV tiles its precomputed block
 * mask masks out). */
static int key_kept(const oracle_problem *pr, int b, int h, int64_t j)
{
    if (!pr->tile_mask) return 1;
    int64_t i = j / pr->tile_len;
    uint32_t w = pr->tile_mask[((int64_t)b * pr->n_kv_heads + h) * pr->mask_words + i / 32];
    return (int)((w >> (i % 32)) & 1u);
}

/* bf16 -> double: the bf16 bit pattern is the top half of an IEEE binary32. */
static double bf16_value(uint16_t h)
{
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* OCP 8-bit floating point, E4M3 "fn" variant: 1 sign bit, 4 exponent bits
 * (bias 7), 3 mantissa bits; exponent 0 encodes subnormals m/8 * 2^-6; the
 * all-ones exponent is a normal binade except mantissa 111, which is NaN; no
 * infinities. */
double oracle_e4m3_value(uint8_t code)
{
    int s = code >> 7, e = (code >> 3) & 15, m = code & 7;
    double v;
    if (e == 15 && m == 7) return NAN;
    if (e == 0) v = ldexp((double)m, -9);             /* (m/8) * 2^(1-7) */
    else v = ldexp(8.0 + m, e - 10);                  /* (1 + m/8) * 2^(e-7) */
    return s ? -v : v;
}

/* Element c of the K (which=0) or V (which=1) vector of token j of request b,
 * KV head h: the page is page_table[b][j / P], the slot j % P. */
static double kv_elem(const oracle_problem *pr, int which, int b, int h, int64_t j, int c)
{
    const int P = pr->page_size, d = pr->head_dim, Hkv = pr->n_kv_heads;
    int32_t page = pr->page_table[(int64_t)b * pr->max_pages_per_seq + j / P];
    int64_t idx = (((int64_t)page * Hkv + h) * P + (j % P)) * d + c;
    const void *pool = which ? pr->v_pages : pr->k_pages;
    if (!pr->kv_fp8) return bf16_value(((const uint16_t *)pool)[idx]);
    double scale = (double)pr->kv_scales[(int64_t)which * pr->num_pages * Hkv + (int64_t)page * Hkv + h];
    return oracle_e4m3_value(((const uint8_t *)pool)[idx]) * scale;
}

/* Attention of query row (b, t, qh) over the keys j in [j_lo, j_hi) that the
 * row may see. The T query tokens are the last T tokens of the request's KV, so
 * token t sees keys 0 .. Lb - T + t (bottom-right causal). Writes out_row[d]
 * and *lse (natural log). With no visible key: out = 0, lse = -inf. If weights
 * is given, the softmax weight of each visible key (in key order) is written
 * there. Returns the number of visible keys. */
int64_t oracle_attend(const oracle_problem *pr, int b, int t, int qh, int64_t j_lo, int64_t j_hi,
                      double *out_row, double *lse, double *weights)
{
    const int d = pr->head_dim, T = pr->q_tokens, G = pr->n_q_heads / pr->n_kv_heads;
    const int h = qh / G;                                   /* contiguous query-head groups */
    const int64_t Lb = pr->seq_lens[b];
    int64_t last = Lb - T + t;                              /* last visible key */
    int64_t lo = j_lo < 0 ? 0 : j_lo;
    int64_t hi = j_hi < last + 1 ? j_hi : last + 1;
    int64_t n = 0;
    const uint16_t *qrow = pr->q + (((int64_t)b * T + t) * pr->n_q_heads + qh) * d;
    double *s;
    int64_t *key;
    int c;
    for (c = 0; c < d; ++c) out_row[c] = 0.0;
    if (hi <= lo) { *lse = -INFINITY; return 0; }
    key = (int64_t *)malloc((size_t)(hi - lo) * sizeof(int64_t));  /* the visible keys, in order */
    for (int64_t j = lo; j < hi; ++j)
        if (key_kept(pr, b, h, j)) key[n++] = j;
    if (n == 0) { *lse = -INFINITY; free(key); return 0; }
    s = (double *)malloc((size_t)n * sizeof(double));
    /* scores s_j = sm_scale * <q, k_j> */
    for (int64_t i = 0; i < n; ++i) {
        double acc = 0.0;
        for (c = 0; c < d; ++c) acc += bf16_value(qrow[c]) * kv_elem(pr, 0, b, h, key[i], c);
        s[i] = pr->sm_scale * acc;
    }
    /* explicit full softmax */
    double m = s[0];
    for (int64_t i = 1; i < n; ++i) if (s[i] > m) m = s[i];
    double Z = 0.0;
    for (int64_t i = 0; i < n; ++i) Z += exp(s[i] - m);
    for (int64_t i = 0; i < n; ++i) {
        double w = exp(s[i] - m) / Z;
        if (weights) weights[i] = w;
        for (c = 0; c < d; ++c) out_row[c] += w * kv_elem(pr, 1, b, h, key[i], c);
    }
    *lse = m + log(Z);
    free(s);
    free(key);
    return n;
}

/* Every query row: out [B][T][Hq][d], lse [B][T][Hq]. */
int oracle_decode(const oracle_problem *pr, double *out, double *lse, int nthreads)
{
    const int B = pr->batch, T = pr->q_tokens, Hq = pr->n_q_heads, d = pr->head_dim;
    const int64_t rows = (int64_t)B * T * Hq;
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#pragma omp parallel for schedule(dynamic, 1)
#endif
    for (int64_t r = 0; r < rows; ++r) {
        int b = (int)(r / ((int64_t)T * Hq)), t = (int)((r / Hq) % T), qh = (int)(r % Hq);
        oracle_attend(pr, b, t, qh, 0, pr->seq_lens[b], out + r * d, lse + r, NULL);
    }
    return 0;
}

/* Selected rows only: rows[3*i .. 3*i+2] = (b, t, qh); out [n][d], lse [n]. */
int oracle_decode_rows(const oracle_problem *pr, const int32_t *rows, int64_t n, double *out, double *lse,
                       int nthreads)
{
    const int d = pr->head_dim;
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#pragma omp parallel for schedule(dynamic, 1)
#endif
    for (int64_t i = 0; i < n; ++i) {
        int b = rows[3 * i], t = rows[3 * i + 1], qh = rows[3 * i + 2];
        oracle_attend(pr, b, t, qh, 0, pr->seq_lens[b], out + i * d, lse + i, NULL);
    }
    return 0;
}

int oracle_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/*
 * Planner reference: the greedy bin-packing of uniform KV tiles onto n_bins CTAs.
 *
 *  1. Tiles: for each pair (b, h) in lexicographic order, n_b = ceil(Lb / tl)
 *     tiles [i*tl, min((i+1)*tl, Lb)), i = 0 .. n_b-1. Cost = tokens in the tile.
 *  2. Order: stable sort of the tiles by cost, largest first (ties keep the
 *     lexicographic order).
 *  3. Greedy: each tile in that order goes to the bin with the least load so far
 *     (ties: lowest bin index); the bin's load grows by the tile's cost.
 *  4. Within a bin, tiles keep the order in which they were assigned.
 *  Partial-result slot of tile (b, h, i) = pair_off[b*Hkv + h] + i, where pair_off
 *  is the exclusive prefix sum of n_b over pairs; a tile that covers its whole
 *  request (n_b == 1) writes the final output and gets slot -1.
 *
 * Output per tile (8 int32): b, h, tok_begin, tok_end, seq_len, slot, i, 0.
 * Returns the number of tiles, or -1 if it exceeds capacity (nothing written).
 */
typedef struct { int64_t cost; int64_t idx; } tile_key;

static int cmp_tile(const void *a, const void *b)
{
    const tile_key *x = (const tile_key *)a, *y = (const tile_key *)b;
    if (x->cost != y->cost) return x->cost > y->cost ? -1 : 1;   /* larger cost first */
    return x->idx < y->idx ? -1 : (x->idx > y->idx);             /* stable */
}

int64_t oracle_plan_masked(const int32_t *seq_lens, const uint32_t *mask, int mask_words, int B, int Hkv,
                           int tl, int n_bins, int64_t capacity, int32_t *bin_off, int32_t *units,
                           int32_t *pair_off);

int64_t oracle_plan(const int32_t *seq_lens, int B, int Hkv, int tl, int n_bins, int64_t capacity,
                    int32_t *bin_off, int32_t *units, int32_t *pair_off)
{
    return oracle_plan_masked(seq_lens, NULL, 0, B, Hkv, tl, n_bins, capacity, bin_off, units, pair_off);
}

/* Block-sparse variant: only the tiles whose mask bit is set (row b * Hkv + h of mask, words
 * of 32 tiles) enter the work list; a pair's kept tiles are numbered j = 0, 1, ... in tile
 * order, its partial slots are pair_off[pair] + j (a pair with one kept tile writes the final
 * output: slot -1), and unit field 6 is the tile's index i among all tiles of the pair. */
int64_t oracle_plan_masked(const int32_t *seq_lens, const uint32_t *mask, int mask_words, int B, int Hkv,
                           int tl, int n_bins, int64_t capacity, int32_t *bin_off, int32_t *units,
                           int32_t *pair_off)
{
    int64_t U = 0, p, k;
#define KEPT(b, h, i) (!mask || ((mask[((int64_t)(b) * Hkv + (h)) * mask_words + (i) / 32] >> ((i) % 32)) & 1u))
    for (int b = 0; b < B; ++b) {
        int64_t nb = ((int64_t)seq_lens[b] + tl - 1) / tl;
        for (int h = 0; h < Hkv; ++h) {
            pair_off[(int64_t)b * Hkv + h] = (int32_t)U;
            for (int64_t i = 0; i < nb; ++i) U += KEPT(b, h, i) ? 1 : 0;
        }
    }
    pair_off[(int64_t)B * Hkv] = (int32_t)U;
    if (U > capacity) return -1;

    int32_t *tb = (int32_t *)malloc(sizeof(int32_t) * 8 * (U ? U : 1));
    tile_key *key = (tile_key *)malloc(sizeof(tile_key) * (U ? U : 1));
    int64_t u = 0;
    for (int b = 0; b < B; ++b) {
        int64_t Lb = seq_lens[b], nb = (Lb + tl - 1) / tl;
        for (int h = 0; h < Hkv; ++h) {
            int64_t p0 = pair_off[(int64_t)b * Hkv + h], m = pair_off[(int64_t)b * Hkv + h + 1] - p0, j = 0;
            for (int64_t i = 0; i < nb; ++i) {
                if (!KEPT(b, h, i)) continue;
                int64_t beg = i * tl, end = (i + 1) * tl < Lb ? (i + 1) * tl : Lb;
                int32_t *r = tb + 8 * u;
                r[0] = b; r[1] = h; r[2] = (int32_t)beg; r[3] = (int32_t)end; r[4] = (int32_t)Lb;
                r[5] = m == 1 ? -1 : (int32_t)(p0 + j);
                r[6] = (int32_t)i; r[7] = 0;
                key[u].cost = end - beg; key[u].idx = u;
                ++u; ++j;
            }
        }
    }
#undef KEPT
    qsort(key, (size_t)U, sizeof(tile_key), cmp_tile);

    int64_t *load = (int64_t *)calloc((size_t)n_bins, sizeof(int64_t));
    int32_t *count = (int32_t *)calloc((size_t)n_bins, sizeof(int32_t));
    int32_t *bin_of = (int32_t *)malloc(sizeof(int32_t) * (U ? U : 1));
    int32_t *rank_in_bin = (int32_t *)malloc(sizeof(int32_t) * (U ? U : 1));
    for (p = 0; p < U; ++p) {
        int64_t best = 0;
        for (k = 1; k < n_bins; ++k) if (load[k] < load[best]) best = k;
        bin_of[key[p].idx] = (int32_t)best;
        rank_in_bin[key[p].idx] = count[best]++;
        load[best] += key[p].cost;
    }
    bin_off[0] = 0;
    for (k = 0; k < n_bins; ++k) bin_off[k + 1] = bin_off[k] + count[k];
    for (u = 0; u < U; ++u) memcpy(units + 8 * ((int64_t)bin_off[bin_of[u]] + rank_in_bin[u]), tb + 8 * u,
                                   8 * sizeof(int32_t));
    free(tb); free(key); free(load); free(count); free(bin_of); free(rank_in_bin);
    return U;
}

/* ------------------------------------------------------------------------------------------
 * Fused pre-processing of a decode step: rotary position embedding of the new q and k, and
 * the append of the new K/V rows into their pages ("PaddlePaddle/HALOps" README, Highlights,
 * GQA attention item: fused pre/post-processing around paged-KV decode). The pages name this
 * step without defining it; the reading written out here:
 *  - rotate-half rotary embedding: for i < d/2, theta_i = base^(-2i/d), and the pair
 *    (x_i, x_{i+d/2}) of a row at position pos becomes
 *    (x_i cos(pos theta_i) - x_{i+d/2} sin(pos theta_i), x_{i+d/2} cos(pos theta_i) + x_i sin(pos theta_i));
 *  - the T new tokens of request b sit at positions Lb - T + t, t < T (seq_lens already
 *    counts them, as the decode does);
 *  - rotated q goes to q_out; rotated k and unchanged v go to page page_table[b][pos / P],
 *    slot pos % P, of their KV head; stored values are the bf16 nearest to the fp64 result;
 *  - a token with pos < 0 has no slot: nothing is written for it and its q row is the
 *    rotation at position 0 (the identity).
 * ------------------------------------------------------------------------------------------ */

/* The rotation of one row of d values at position pos, in fp64. */
void oracle_rope_row(const double *x, int d, double pos, double base, double *y)
{
    int half = d / 2;
    for (int i = 0; i < half; ++i) {
        double theta = pow(base, -2.0 * i / d);
        double c = cos(pos * theta), s = sin(pos * theta);
        y[i] = x[i] * c - x[i + half] * s;
        y[i + half] = x[i + half] * c + x[i] * s;
    }
}

/* The bf16 (8 significant bits, binary32's exponent range) nearest to v, ties to even, as its
 * bit pattern; rounded in one step from the double (no detour through binary32). */
uint16_t oracle_bf16_bits(double v)
{
    if (isnan(v)) return 0x7fc0;
    int sgn = signbit(v) ? 1 : 0;
    double a = fabs(v), r;
    if (a == 0.0) return (uint16_t)(sgn << 15);
    int e;
    frexp(a, &e);                     /* a = m 2^e, m in [0.5, 1) */
    if (e < -125) e = -125;           /* below the normal range the spacing stays 2^-133 */
    r = ldexp(rint(ldexp(a, 8 - e)), e - 8);
    if (r >= 0x1p128) return (uint16_t)((sgn << 15) | 0x7f80);
    float f = (float)r;               /* exact: r has at most 8 significant bits */
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    return (uint16_t)((u >> 16) | (uint32_t)(sgn << 15));
}

/* Applies the pre-processing to bf16 inputs. q_new [B][T][Hq][d], k_new / v_new [B][T][Hkv][d]
 * (bf16 bits); q_out [B][T][Hq][d]; k_pages / v_pages [num_pages][Hkv][P][d] (bf16 bits,
 * updated in place). Returns the number of (token, KV head) rows written, or -1 if a page id
 * read for a written row lies outside [0, num_pages) or past the page-table row. */
int64_t oracle_append_rope(const uint16_t *q_new, const uint16_t *k_new, const uint16_t *v_new,
                           const int32_t *page_table, const int32_t *seq_lens, int B, int T, int Hq,
                           int Hkv, int d, int P, int num_pages, int mpps, double base, uint16_t *q_out,
                           uint16_t *k_pages, uint16_t *v_pages)
{
    double *x = (double *)malloc(sizeof(double) * (size_t)d);
    double *y = (double *)malloc(sizeof(double) * (size_t)d);
    int64_t written = 0;
    for (int b = 0; b < B; ++b)
        for (int t = 0; t < T; ++t) {
            int64_t pos = (int64_t)seq_lens[b] - T + t;
            double rpos = pos < 0 ? 0.0 : (double)pos;
            for (int qh = 0; qh < Hq; ++qh) {
                size_t o = (((size_t)b * T + t) * Hq + qh) * d;
                for (int c = 0; c < d; ++c) x[c] = bf16_value(q_new[o + c]);
                oracle_rope_row(x, d, rpos, base, y);
                for (int c = 0; c < d; ++c) q_out[o + c] = oracle_bf16_bits(y[c]);
            }
            if (pos < 0) continue;
            if (pos / P >= mpps) { written = -1; goto done; }
            int32_t pid = page_table[(int64_t)b * mpps + pos / P];
            if (pid < 0 || pid >= num_pages) { written = -1; goto done; }
            for (int h = 0; h < Hkv; ++h) {
                size_t in = (((size_t)b * T + t) * Hkv + h) * d;
                size_t dst = (((size_t)pid * Hkv + h) * P + (size_t)(pos % P)) * d;
                for (int c = 0; c < d; ++c) x[c] = bf16_value(k_new[in + c]);
                oracle_rope_row(x, d, (double)pos, base, y);
                for (int c = 0; c < d; ++c) {
                    k_pages[dst + c] = oracle_bf16_bits(y[c]);
                    v_pages[dst + c] = v_new[in + c];
                }
                ++written;
            }
        }
done:
    free(x);
    free(y);
    return written;
}
