/*
 * kvdecode — decode-phase attention over a paged KV cache on NVIDIA B200 (sm_100a).
 *
 * Variants, as defined in "Hardware-Efficient Attention for Fast Decoding"
 * (Zadouri, Strauss, Dao; section 3 "Methodology", Figure 2 caption):
 *   GQA  query heads split into h_kv groups; each group reads its own K and V
 *        head (m_kv = 2).  MQA (h_kv = 1) and MHA (h_kv = h_q) are special cases.
 *   GTA  grouped-tied attention: one tied state per group is the value (all d_h
 *        dims) and its first d_h - d_r dims are the non-RoPE half of the key;
 *        the RoPE half of the key is one d_r-wide slice per token shared by all
 *        heads (m_kv = 1).
 *   GLA  grouped latent attention in absorbed form: h_c latent heads of width
 *        d_c plus one shared d_r-wide RoPE key; query head h attends latent head
 *        h / (h_q / h_c) with key = [latent ++ rope] and value = latent.  MLA is
 *        the h_c = 1 case.
 *
 * For sequence b with T_b = seqlens[b] cached tokens (the L new query tokens
 * are the last L of them), query row i in [0, L) and head h:
 *   visible tokens t <= T_b - L + i;  s_t = scale * <q, k_t>;
 *   lse = ln sum_t exp(s_t);  out = sum_t exp(s_t - lse) v_t.
 * A row that sees no token gets out = 0 and lse = -inf.
 *
 * Memory (all pointers are DEVICE pointers owned by the caller; the library
 * never allocates, frees or keeps them after the call returns):
 *   q            bf16 [B, L, h_q, d_qk] contiguous
 *                  GQA d_qk = d; GTA d_qk = d_h laid out [q_nope (d_h - d_r) ++ q_rope (d_r)];
 *                  GLA d_qk = d_c + d_r laid out [q_latent (d_c) ++ q_rope (d_r)]
 *   caches       bf16, page-major: [num_pages, page_size, heads, dim] contiguous
 *                  GQA k_cache, v_cache [P, S, h_kv, d]
 *                  GTA tied_cache [P, S, h_kv, d_h], rope_cache [P, S, d_r]
 *                  GLA latent_cache [P, S, h_c, d_c], rope_cache [P, S, d_r]
 *                RoPE is applied when tokens are written (rotated keys are
 *                stored, q arrives rotated); decode does no rotation.
 *   block_table  int32 [B, max_pages]: physical page of logical page i of b.
 *                Entries at or past ceil(T_b / page_size) are never read.
 *   seqlens      int32 [B], 0 <= T_b <= max_pages * page_size, and T_b >= L
 *                when T_b > 0.
 *   out          bf16 [B, L, h_q, d_v] (d_v = d, d_h or d_c), round to nearest even
 *   lse          fp32 [B, L, h_q], natural log of the softmax denominator of the
 *                scaled scores
 *   workspace    device scratch of at least kvd_*_workspace_size() bytes, 256-byte
 *                aligned, ZEROED ONCE before its first use (cudaMemset).  It holds
 *                the split-KV partials and a sticky device error word; calls
 *                that overlap on the GPU must not share one workspace.
 * q, caches and (for GLA) out must be 16-byte aligned (TMA, vector stores); out
 * 8-byte aligned for GQA/GTA; the int32 and fp32 arrays 4-byte aligned.
 *
 * Execution: every entry point is asynchronous on `stream`; there is no host
 * synchronisation and no allocation, so a call can be captured in a CUDA graph.
 * Split planning runs on the device from seqlens: the (sequence, 16-token tile)
 * stream is cut into `num_parts` equal contiguous parts (0 = one per SM, or per
 * SM pair for the latent kernel), each processed by one CTA; sequences cut into
 * several parts are merged by an LSE-combine kernel.
 *
 * Errors: functions return KVD_OK (0) or a negative KVD_ERR_* code and do not
 * launch anything on a host-side validation error.  Faults detected on the
 * device (a block-table entry outside [0, num_pages), an invalid seqlen, a
 * bounded wait that ran out) never trap: the kernel records a flag in the
 * workspace's error word, substitutes a safe value (page 0, a clamped length)
 * or stops early, and kvd_read_device_error() reports it.
 */
#ifndef KVDECODE_H
#define KVDECODE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st *kvd_stream_t; /* same handle as cudaStream_t; NULL = legacy default stream */

enum {
    KVD_OK = 0,
    KVD_ERR_INVALID_ARG = -1,        /* null/misaligned pointer, inconsistent sizes */
    KVD_ERR_UNSUPPORTED_SHAPE = -2,  /* head dims or group size outside the compiled set */
    KVD_ERR_WORKSPACE_TOO_SMALL = -3,
    KVD_ERR_CUDA = -4,               /* a CUDA runtime call or launch failed */
    KVD_ERR_DEVICE = -5              /* kvd_read_device_error found flags set */
};

/* Device error-word bits reported by kvd_read_device_error(). */
enum {
    KVD_DEVERR_TIMEOUT = 1u,     /* a bounded pipeline wait ran out; output incomplete */
    KVD_DEVERR_BAD_PAGE = 2u,    /* block_table entry outside [0, num_pages); page 0 was read instead */
    KVD_DEVERR_BAD_SEQLEN = 4u   /* seqlens[b] < 0, > max_pages*page_size, or 0 < T_b < L; clamped */
};

/*
 * GQA (and MQA/MHA).  d in {64, 128}; h_q % h_kv == 0; (h_q / h_kv) * L <= 32; any
 * page_size >= 1: pages holding whole 16- or 32-token tiles are loaded with one tensor-map box
 * per tile, smaller pages (down to one token) or sizes that are not a multiple of 16 are
 * gathered token by token (slower; the same results).
 */
typedef struct {
    const void *q;            /* bf16 [B, L, h_q, d] */
    const void *k_cache;      /* bf16 [num_pages, page_size, h_kv, d] */
    const void *v_cache;      /* bf16 [num_pages, page_size, h_kv, d] */
    const int32_t *block_table;
    const int32_t *seqlens;
    void *out;                /* bf16 [B, L, h_q, d] */
    float *lse;               /* fp32 [B, L, h_q] */
    int32_t B, L, h_q, h_kv, d, page_size, num_pages, max_pages;
    float scale;              /* softmax scale applied to q.k */
    int32_t num_parts;        /* 0 = auto */
} kvd_gqa_params;

/*
 * GTA.  d_h in {64, 128}, d_r in {32, 64}, d_r <= d_h, (d_h - d_r) % 16 == 0;
 * other limits as GQA.
 */
typedef struct {
    const void *q;            /* bf16 [B, L, h_q, d_h] = [nope ++ rope] */
    const void *tied_cache;   /* bf16 [num_pages, page_size, h_kv, d_h] */
    const void *rope_cache;   /* bf16 [num_pages, page_size, d_r] */
    const int32_t *block_table;
    const int32_t *seqlens;
    void *out;                /* bf16 [B, L, h_q, d_h] */
    float *lse;               /* fp32 [B, L, h_q] */
    int32_t B, L, h_q, h_kv, d_h, d_r, page_size, num_pages, max_pages;
    float scale;
    int32_t num_parts;
} kvd_gta_params;

/*
 * GLA / MLA (absorbed).  d_c in {256, 512}, d_r == 64, h_q % h_c == 0, h_q / h_c divides or is
 * a multiple of 128, (h_q / h_c) * L <= 8192; any page_size >= 1.  GLA (d_c 256) loads a
 * tile (96 tokens with at most 64 query rows per latent head, 64 with more) in boxes of
 * gcd(tile, page_size) tokens when that is at least 16, MLA whole 64-token tiles when
 * page_size is a multiple of 64; other page sizes are gathered token by token.
 */
typedef struct {
    const void *q;            /* bf16 [B, L, h_q, d_c + d_r] = [latent ++ rope] */
    const void *latent_cache; /* bf16 [num_pages, page_size, h_c, d_c] */
    const void *rope_cache;   /* bf16 [num_pages, page_size, d_r] */
    const int32_t *block_table;
    const int32_t *seqlens;
    void *out;                /* bf16 [B, L, h_q, d_c] */
    float *lse;               /* fp32 [B, L, h_q] */
    int32_t B, L, h_q, h_c, d_c, d_r, page_size, num_pages, max_pages;
    float scale;
    int32_t num_parts;
} kvd_gla_params;

/* Bytes of workspace the matching decode call needs (0 on invalid params). */
size_t kvd_gqa_workspace_size(const kvd_gqa_params *p);
size_t kvd_gta_workspace_size(const kvd_gta_params *p);
size_t kvd_gla_workspace_size(const kvd_gla_params *p);

/* Decode entry points: plan, decode and combine kernels on `stream`. */
int kvd_gqa_decode(const kvd_gqa_params *p, void *workspace, size_t workspace_bytes, kvd_stream_t stream);
int kvd_gta_decode(const kvd_gta_params *p, void *workspace, size_t workspace_bytes, kvd_stream_t stream);
int kvd_gla_decode(const kvd_gla_params *p, void *workspace, size_t workspace_bytes, kvd_stream_t stream);

/*
 * Allocation-free GTA decode (no counterpart in the paper: an interface for
 * callers that cannot provide a workspace).  Serving engines that have already
 * split all of HBM between KV pages and their own arenas cannot allocate more
 * device memory per call, and code that calls this while a stream is captured
 * in global mode may not call cudaMalloc at all.  This entry computes exactly
 * what kvd_gta_decode() computes, with the workspace in a fixed 8 MiB device
 * array inside the library (held by every GPU that loads the library until the
 * process exits).  It allocates and frees nothing.
 *   - Every call looks up that array's device address in the current context
 *     (a host-side lookup; the first one on a device also loads the library's
 *     device code there, so make the first call on each device before any
 *     stream capture).
 *   - Calls whose split partials need more than 8 MiB (see
 *     kvd_gta_workspace_size) are rejected with KVD_ERR_WORKSPACE_TOO_SMALL and
 *     launch nothing.
 *   - Every call on a device shares the one array and leaves its contents
 *     behind; nothing in it needs to start at zero, but calls that overlap on
 *     the GPU (different streams, no ordering between them) race on it.
 *   - Device error flags land in the shared array and cannot be read back; use
 *     kvd_gta_decode() with a workspace to inspect them.
 */
int kvd_gta_decode_noalloc(const kvd_gta_params *p, kvd_stream_t stream);

/*
 * Shared-prefix attention (GTA) for cascade decoding: every one of the B x L query rows
 * attends every token of ONE prefix that the whole batch shares, with no causal mask (the
 * prefix precedes all queries).  The prefix is read once per KV group for the whole batch:
 * the q rows of all sequences that share a group form one tensor-core tile (Hydragen-style
 * batching of a shared prefix; the pages' shared-prefix decoding).
 *   p->q            bf16 [B, L, h_q, d_h] as in kvd_gta_decode (q_rope already rotated)
 *   p->tied_cache, p->rope_cache, p->page_size, p->num_pages: as in kvd_gta_decode
 *   p->block_table  int32 [1, max_pages]: the prefix's pages
 *   p->seqlens      int32 [1]: the prefix length T_p (T_p = 0: out = 0, lse = -inf)
 *   p->out, p->lse  as in kvd_gta_decode: the state of each row over the prefix alone
 * Requires d_h = 128, d_r = 64 and (h_q / h_kv) * B * L <= 8192.  The continuation (each
 * sequence's own tokens) is decoded by kvd_gta_decode on its own pages; kvd_merge_states then
 * gives attention over prefix + continuation.  Workspace as for kvd_gta_decode, sized by
 * kvd_gta_prefix_workspace_size.
 */
size_t kvd_gta_prefix_workspace_size(const kvd_gta_params *p);
int kvd_gta_prefix_decode(const kvd_gta_params *p, void *workspace, size_t ws_bytes, kvd_stream_t stream);

/*
 * Merge two attention states of the same query rows over disjoint key sets, e.g. a prefix
 * shared by the whole batch and each sequence's own continuation (cascade decoding; the
 * combine step of "Hardware-Efficient Attention for Fast Decoding", section 3.3.2, applied
 * to two parts).  With m = max(lse_a, lse_b):
 *   lse = m + ln(e^(lse_a - m) + e^(lse_b - m)),
 *   out = e^(lse_a - lse) out_a + e^(lse_b - lse) out_b,
 * a state with lse = -inf weighs nothing, and two empty states give out = 0, lse = -inf.
 * out_a, out_b, out: bf16 [rows, d_v] (device, 16-byte aligned, d_v a multiple of 8);
 * lse_a, lse_b, lse: fp32 [rows] (device).  out / lse may be out_a / lse_a (in place).
 * Arithmetic in fp32, out rounded to bf16.  Asynchronous on `stream`.
 */
int kvd_merge_states(const void *out_a, const float *lse_a, const void *out_b, const float *lse_b, void *out,
                     float *lse, int32_t rows, int32_t d_v, kvd_stream_t stream);

/*
 * Split plan for inspection and tests.  Cuts the (sequence, tile) stream of
 * seqlens[B] (device pointer) with `tile` tokens per tile into num_parts parts
 * exactly as the decode kernels do and writes, for part c, up to `cap` records
 * of 6 int32 {b, tile_begin, tile_end, split_index, num_splits, slot} at
 * segments[c * cap * 6 ...] and the record count at counts[c] (device
 * pointers).  A count above `cap` means records were dropped.  seg_cost >= 0:
 * each non-empty sequence counts as seg_cost extra tiles placed before its
 * own when the stream is cut into parts of equal size (the GLA kernels plan
 * with 3 for at most 64 rows per latent head and 7 for more, GTA with
 * 128 / tile, the others with 0).
 */
int kvd_plan(const int32_t *seqlens, int32_t B, int32_t tile, int32_t seg_cost, int32_t max_tokens,
             int32_t num_parts, int32_t *segments, int32_t *counts, int32_t cap, kvd_stream_t stream);

/* The same plan computed on the host from host memory; returns KVD_OK. */
int kvd_plan_host(const int32_t *seqlens, int32_t B, int32_t tile, int32_t seg_cost, int32_t max_tokens,
                  int32_t num_parts, int32_t *segments, int32_t *counts, int32_t cap);

/*
 * Synchronises `stream`, reads the workspace's device error word into *flags
 * (KVD_DEVERR_* bits) and clears it.  Returns KVD_OK, KVD_ERR_DEVICE when any
 * flag was set, or KVD_ERR_CUDA.
 */
int kvd_read_device_error(void *workspace, kvd_stream_t stream, uint32_t *flags);

/*
 * Test knobs, process-wide, read at launch time; not for production use.
 *   KVD_DEBUG_WAIT_LIMIT_NS    limit of one bounded pipeline wait (default 2e9 ns)
 *   KVD_DEBUG_SKIP_FIRST_LOAD  nonzero: the first tile's copy is never issued, so
 *                              the consumers' bounded wait runs out and the call
 *                              reports KVD_DEVERR_TIMEOUT (exercises the timeout
 *                              path without any fault)
 */
enum { KVD_DEBUG_WAIT_LIMIT_NS = 1, KVD_DEBUG_SKIP_FIRST_LOAD = 2 };
int kvd_debug_set(int knob, long long value);

/*
 * Measurement hook, process-wide: when both are non-null (cudaEvent_t handles),
 * every decode call records `before_main` on its stream just before launching
 * its main decode kernel and `after_main` just after it, so that a benchmark can
 * time that kernel alone with events.  Pass NULLs to turn it off.
 */
int kvd_profile_events(void *before_main, void *after_main);

/*
 * Measurement helper (no counterpart in the paper): reads `bytes` of device memory at
 * `buf` once with streaming 16-byte loads on `stream` (grid: blocks_per_sm x the SM count,
 * 512 threads each) and writes nothing but, practically never, an increment of *sink
 * (device memory).  Timed with events around it, it gives the read-only rate of the
 * device memory, the ceiling a decode kernel that only reads the KV cache streams
 * against.  `buf` 16-byte aligned, `bytes` a multiple of 16; KVD_ERR_INVALID_ARG
 * otherwise.  Asynchronous; allocates nothing.
 */
int kvd_read_stream(const void *buf, size_t bytes, unsigned long long *sink, int blocks_per_sm,
                    kvd_stream_t stream);

/* Number of SMs of the current device (the default part count), or a negative code. */
int kvd_num_sms(void);

/* Static description of a status code. */
const char *kvd_status_string(int status);

/* Library version as major*10000 + minor*100 + patch. */
int kvd_version(void);

#ifdef __cplusplus
}
#endif

#endif /* KVDECODE_H */
