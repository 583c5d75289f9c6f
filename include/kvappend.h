/*
 * kvappend — the step before decode: write the new tokens' states into their paged
 * cache slots, rotating the RoPE slices, and rotate the queries.
 *
 * "Hardware-Efficient Attention for Fast Decoding" (section 3.3.1 for GTA, 3.3.2 for
 * GLA; Figure 2) stores per token, per variant:
 *   GQA  a K head and a V head per group; RoPE is applied to the key's last d_r dims
 *        (d_r = d: the whole key, the GQA baseline's "full RoPE");
 *   GTA  one tied state per group (stored as is) and one d_r-wide RoPE key slice per
 *        token shared by all heads (rotated);
 *   GLA  h_c latent heads (stored as is) and one shared d_r-wide RoPE key slice
 *        (rotated).  MLA is h_c = 1.
 * The pages rotate the RoPE part without fixing the convention; this library uses
 * rotate-half pairs: for j in [0, d_r/2), with theta_j = rope_base^(-2 j / d_r) and
 * angle a = position * theta_j,
 *   y[j]          = x[j] cos a - x[j + d_r/2] sin a
 *   y[j + d_r/2]  = x[j + d_r/2] cos a + x[j] sin a.
 * Angles, sines, cosines and the rotation are computed in fp64 and the result is
 * rounded once to bf16 (round to nearest even), so a stored value differs from the
 * exactly rotated one by at most half a bf16 ulp plus the fp64 error of sin and cos.
 *
 * Memory: all pointers are DEVICE pointers owned by the caller; nothing is allocated.
 *   new-token inputs  bf16 [N, heads, dim] contiguous (RoPE slices [N, d_r]); inputs
 *                     and caches 16-byte aligned, dims multiples of 8
 *   positions         int32 [N]: absolute position of each new token (the RoPE angle)
 *   slot_mapping      int32 [N]: destination row in the cache viewed as
 *                     [num_pages * page_size, heads, dim], i.e. physical_page *
 *                     page_size + offset; a negative entry skips the token (padding)
 *   caches            as in kvdecode.h, page-major [num_pages, page_size, heads, dim]
 *   num_rows          num_pages * page_size; a token whose slot is at or past it is
 *                     not written
 *   error_word        optional device uint32 (may be NULL, e.g. the first word of a
 *                     decode workspace); KVD_DEVERR_BAD_PAGE is OR-ed into it when a
 *                     slot is out of range
 * Rows named twice in one call are written in an unspecified order.
 *
 * Execution: asynchronous on `stream`, no host synchronisation, graph-capturable.
 * Errors: KVD_OK or a negative KVD_ERR_* code (nothing launched).
 */
#ifndef KVAPPEND_H
#define KVAPPEND_H

#include <stdint.h>

#include "kvdecode.h"

#ifdef __cplusplus
extern "C" {
#endif

typedef struct {
    const void *k_new, *v_new;   /* bf16 [N, h_kv, d] */
    void *k_cache, *v_cache;     /* bf16 [num_rows, h_kv, d] */
    const int32_t *positions, *slot_mapping;
    uint32_t *error_word;
    int32_t N, h_kv, d, d_r, num_rows;
    float rope_base;             /* 10000 in the pages' models */
} kvd_gqa_append_params;

typedef struct {
    const void *tied_new;        /* bf16 [N, h_kv, d_h] */
    const void *rope_new;        /* bf16 [N, d_r], not yet rotated */
    void *tied_cache, *rope_cache;
    const int32_t *positions, *slot_mapping;
    uint32_t *error_word;
    int32_t N, h_kv, d_h, d_r, num_rows;
    float rope_base;
} kvd_gta_append_params;

typedef struct {
    const void *latent_new;      /* bf16 [N, h_c, d_c] */
    const void *rope_new;        /* bf16 [N, d_r], not yet rotated */
    void *latent_cache, *rope_cache;
    const int32_t *positions, *slot_mapping;
    uint32_t *error_word;
    int32_t N, h_c, d_c, d_r, num_rows;
    float rope_base;
} kvd_gla_append_params;

/* Write N new tokens into the caches (rotating the RoPE part). */
int kvd_gqa_append(const kvd_gqa_append_params *p, kvd_stream_t stream);
int kvd_gta_append(const kvd_gta_append_params *p, kvd_stream_t stream);
int kvd_gla_append(const kvd_gla_append_params *p, kvd_stream_t stream);

/*
 * Rotate the RoPE dims [rope_off, rope_off + d_r) of every head of q in place, for
 * the decode call that follows: q is bf16 [B, L, heads, d_qk] and row (b, i) sits at
 * position seqlens[b] - L + i (the convention of kvdecode.h; rows of a sequence with
 * fewer than L tokens are left as they are).  GQA with full RoPE: rope_off = 0,
 * d_r = d; GTA: rope_off = d_h - d_r; GLA: rope_off = d_c.
 */
int kvd_rope_q(void *q, const int32_t *seqlens, int32_t B, int32_t L, int32_t heads, int32_t d_qk,
               int32_t rope_off, int32_t d_r, float rope_base, kvd_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* KVAPPEND_H */
