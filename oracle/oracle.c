/*
 * fp64 CPU oracle for decode attention over a paged KV cache.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path links, loads or calls
 * this file: only the tests, the package's smoke check and the bench's CPU
 * baseline leg do.  It shares no code, header, table or helper with the CUDA
 * library.
 *
 * It computes the plain definition, in double precision, one query row at a
 * time, with no blocking, fusion or reordering:
 *
 *   for sequence b, query position i in [0, L) and query head h:
 *     p      = T_b - L + i                 (position of the query token; the L
 *                                           new tokens are the last L tokens of
 *                                           the cache, so row i sees t <= p)
 *     k_t    = key of token t for head h   (gathered through the block table:
 *                                           page = block_table[b][t / S],
 *                                           slot = t mod S)
 *     s_t    = scale * <q_{b,i,h}, k_t>    for t in the visible range
 *     lse    = ln sum_t exp(s_t)           (natural log; -inf if nothing is visible)
 *     out    = sum_t exp(s_t - lse) v_t    (0 if nothing is visible)
 *
 * The variants differ only in what k_t and v_t are ("Hardware-Efficient
 * Attention for Fast Decoding", section 3 and the Figure 2 caption):
 *   GQA  group g = h / (h_q / h_kv); k = K[g], v = V[g]           (m_kv = 2)
 *   GTA  group g = h / (h_q / h_kv); k = [tied[g][0 : d_h - d_r] ++ rope],
 *        v = tied[g] (all d_h dims); rope is one slice per token shared by
 *        every head                                                  (m_kv = 1)
 *   GLA  latent head c = h / (h_q / h_c); k = [latent[c] ++ rope], v = latent[c]
 *        (absorbed form; MLA is h_c = 1)
 *
 * Inputs are raw bf16 bit patterns (uint16) widened exactly to double.  An
 * optional per-sequence token window [lo, hi) restricts the visible tokens
 * further; it exists to check split-KV partials against the whole.
 *
 * LSE combine ("softmax denominator" decomposition, as Hydragen uses it):
 *   lse = ln sum_s exp(lse_s);  out = sum_s exp(lse_s - lse) out_s.
 *
 * RoPE (rotate-half convention, pairs (j, j + d_r/2), theta_j = base^(-2j/d_r),
 * 0-based absolute position); the decode step itself never rotates.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

static double bf16_to_f64(uint16_t h)
{
    uint32_t u = ((uint32_t)h) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

enum { ORC_GQA = 0, ORC_GTA = 1, ORC_GLA = 2 };

typedef struct {
    int variant;
    int B, L, h_q, h_kv, d, d_r, S, max_pages;
    const uint16_t *q;       /* [B, L, h_q, d_qk] */
    const uint16_t *c0;      /* GQA: K  [P, S, h_kv, d];  GTA: tied [P, S, h_kv, d];  GLA: latent [P, S, h_c, d] */
    const uint16_t *c1;      /* GQA: V  [P, S, h_kv, d];  GTA/GLA: rope [P, S, d_r] */
    const int32_t *block_table;  /* [B, max_pages] */
    const int32_t *seqlens;      /* [B] */
    double scale;
} orc_problem;

static int d_qk_of(const orc_problem *p)
{
    return p->variant == ORC_GLA ? p->d + p->d_r : p->d;
}

/* Key element j of token t (logical position in sequence b) for head h. */
static double key_elem(const orc_problem *p, int b, int t, int h, int j)
{
    int page = p->block_table[(size_t)b * p->max_pages + t / p->S];
    int slot = t % p->S;
    size_t tok = (size_t)page * p->S + slot;
    int grp = h / (p->h_q / p->h_kv);
    switch (p->variant) {
    case ORC_GQA:
        return bf16_to_f64(p->c0[(tok * p->h_kv + grp) * p->d + j]);
    case ORC_GTA: {
        int nope = p->d - p->d_r;
        if (j < nope) return bf16_to_f64(p->c0[(tok * p->h_kv + grp) * p->d + j]);
        return bf16_to_f64(p->c1[tok * p->d_r + (j - nope)]);
    }
    default:
        if (j < p->d) return bf16_to_f64(p->c0[(tok * p->h_kv + grp) * p->d + j]);
        return bf16_to_f64(p->c1[tok * p->d_r + (j - p->d)]);
    }
}

/* Value element j (j < d) of token t for head h. */
static double value_elem(const orc_problem *p, int b, int t, int h, int j)
{
    int page = p->block_table[(size_t)b * p->max_pages + t / p->S];
    int slot = t % p->S;
    size_t tok = (size_t)page * p->S + slot;
    int grp = h / (p->h_q / p->h_kv);
    if (p->variant == ORC_GQA) return bf16_to_f64(p->c1[(tok * p->h_kv + grp) * p->d + j]);
    return bf16_to_f64(p->c0[(tok * p->h_kv + grp) * p->d + j]);
}

/*
 * One query row: fills out_row[d] and *lse_out.  `s` is caller scratch of at
 * least (hi - lo) doubles.
 */
static void attend_row(const orc_problem *p, int b, int i, int h, int lo, int hi,
                       double *s, double *out_row, double *lse_out)
{
    int dqk = d_qk_of(p);
    int T = p->seqlens[b];
    int pos = T - p->L + i;              /* visible tokens: t <= pos */
    int end = hi < pos + 1 ? hi : pos + 1;
    const uint16_t *q = p->q + (((size_t)b * p->L + i) * p->h_q + h) * dqk;
    int n = end - lo;
    for (int j = 0; j < p->d; ++j) out_row[j] = 0.0;
    if (n <= 0) {
        *lse_out = -INFINITY;
        return;
    }
    double m = -INFINITY;
    for (int t = lo; t < end; ++t) {
        double acc = 0.0;
        for (int j = 0; j < dqk; ++j) acc += bf16_to_f64(q[j]) * key_elem(p, b, t, h, j);
        s[t - lo] = p->scale * acc;
        if (s[t - lo] > m) m = s[t - lo];
    }
    double denom = 0.0;
    for (int t = lo; t < end; ++t) denom += exp(s[t - lo] - m);
    double lse = m + log(denom);
    for (int t = lo; t < end; ++t) {
        double w = exp(s[t - lo] - lse);
        for (int j = 0; j < p->d; ++j) out_row[j] += w * value_elem(p, b, t, h, j);
    }
    *lse_out = lse;
}

/*
 * Decode for the sequences listed in b_list[0..nb) (all B when b_list is NULL,
 * nb = B).  out is [nb, L, h_q, d] and lse is [nb, L, h_q], compact over the
 * list.  tok_lo / tok_hi (per listed sequence, may be NULL) bound the tokens
 * each sequence contributes to [lo, hi) on top of the causal rule.
 * Returns the number of OpenMP threads used.
 */
int orc_decode(int variant, int B, int L, int h_q, int h_kv, int d, int d_r, int S,
               int max_pages, const uint16_t *q, const uint16_t *c0, const uint16_t *c1,
               const int32_t *block_table, const int32_t *seqlens, double scale,
               const int32_t *b_list, int nb, const int32_t *tok_lo, const int32_t *tok_hi,
               double *out, double *lse, int num_threads)
{
    orc_problem p = {variant, B, L, h_q, h_kv, d, d_r, S, max_pages, q, c0, c1,
                     block_table, seqlens, scale};
    if (b_list == NULL) nb = B;
    int maxT = 0;
    for (int k = 0; k < nb; ++k) {
        int b = b_list ? b_list[k] : k;
        if (seqlens[b] > maxT) maxT = seqlens[b];
    }
    long total = (long)nb * L * h_q;
    int used = 1;
#ifdef _OPENMP
    if (num_threads <= 0) num_threads = omp_get_max_threads();
#pragma omp parallel num_threads(num_threads)
    {
#pragma omp single
        used = omp_get_num_threads();
#else
    (void)num_threads;
    {
#endif
        double *s = (double *)malloc(sizeof(double) * (size_t)(maxT > 0 ? maxT : 1));
#ifdef _OPENMP
#pragma omp for schedule(dynamic, 1)
#endif
        for (long r = 0; r < total; ++r) {
            int h = (int)(r % h_q);
            int i = (int)((r / h_q) % L);
            int k = (int)(r / ((long)h_q * L));
            int b = b_list ? b_list[k] : k;
            int lo = tok_lo ? tok_lo[k] : 0;
            int hi = tok_hi ? tok_hi[k] : seqlens[b];
            attend_row(&p, b, i, h, lo, hi, s, out + (size_t)r * d, lse + r);
        }
        free(s);
    }
    return used;
}

/*
 * LSE combine of nsplit partial results over `rows` query rows of width d_v.
 * part_out [nsplit, rows, d_v], part_lse [nsplit, rows] -> out [rows, d_v],
 * lse [rows].  A split with lse = -inf (nothing visible) has weight 0; if all
 * are -inf the result is out = 0, lse = -inf.
 */
void orc_combine(int nsplit, int rows, int d_v, const double *part_out, const double *part_lse,
                 double *out, double *lse)
{
    for (int r = 0; r < rows; ++r) {
        double m = -INFINITY;
        for (int s = 0; s < nsplit; ++s)
            if (part_lse[(size_t)s * rows + r] > m) m = part_lse[(size_t)s * rows + r];
        for (int j = 0; j < d_v; ++j) out[(size_t)r * d_v + j] = 0.0;
        if (m == -INFINITY) {
            lse[r] = -INFINITY;
            continue;
        }
        double sum = 0.0;
        for (int s = 0; s < nsplit; ++s) sum += exp(part_lse[(size_t)s * rows + r] - m);
        double L = m + log(sum);
        for (int s = 0; s < nsplit; ++s) {
            double w = exp(part_lse[(size_t)s * rows + r] - L);
            if (w == 0.0) continue;
            for (int j = 0; j < d_v; ++j)
                out[(size_t)r * d_v + j] += w * part_out[((size_t)s * rows + r) * d_v + j];
        }
        lse[r] = L;
    }
}

/* Rotate x[d_r] to absolute position `pos` (rotate-half pairs). */
void orc_rope(const double *x, int d_r, double pos, double base, double *y)
{
    int half = d_r / 2;
    for (int j = 0; j < half; ++j) {
        double theta = pow(base, -2.0 * j / d_r);
        double c = cos(pos * theta), s = sin(pos * theta);
        y[j] = x[j] * c - x[j + half] * s;
        y[j + half] = x[j + half] * c + x[j] * s;
    }
}
