// C-ABI entry points: validation, workspace sizing, TMA descriptors, launches.
#include <cuda.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cmath>
#include <cstring>
#include <mutex>

#include "common.cuh"
#include "kernels.h"
#include "kvdecode.h"

using namespace kvd;

namespace kvd {
// SM count of the calling thread's current device, looked up once per device.
int num_sms_current() {
    static std::atomic<int> cache[64];  // zero-initialised (static storage)
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return -1;
    const bool cached = dev >= 0 && dev < 64;
    if (cached) {
        const int c = cache[dev].load(std::memory_order_relaxed);
        if (c > 0) return c;
    }
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return -1;
    if (cached) cache[dev].store(n, std::memory_order_relaxed);
    return n;
}
}  // namespace kvd

namespace {

// Dynamic shared memory the decode kernels may ask for (the SM's 227 KB less
// the static arrays and the 1 KB alignment slack).
constexpr size_t SMEM_BUDGET = 220 * 1024;

std::atomic<int> g_debug_flags{0};
std::atomic<void *> g_ev_before{nullptr}, g_ev_after{nullptr};

void record(std::atomic<void *> &ev, cudaStream_t st) {
    void *e = ev.load();
    if (e && g_ev_before.load() && g_ev_after.load()) cudaEventRecord((cudaEvent_t)e, st);
}
std::atomic<long long> g_wait_limit_ns{(long long)WAIT_LIMIT_NS};

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = (EncodeTiledFn)p;
    });
    return fn;
}

bool encode(CUtensorMap *m, const void *base, int rank, const cuuint64_t *dims, const cuuint64_t *strides,
            const cuuint32_t *box, CUtensorMapSwizzle sw) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    cuuint32_t es[5] = {1, 1, 1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, (cuuint32_t)rank, const_cast<void *>(base), dims, strides, box,
              es, CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool aligned(const void *p, size_t a) { return ((uintptr_t)p % a) == 0; }
size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// ----------------------------------------------------------------------------- GQA / GTA
struct GroupPlan {
    int gpc, n_sub, parts, nt, nstage, tile;
    int seg_cost;  // plan: units a segment start costs, in tiles
    bool gather;
    uint32_t stage_bytes, stage_bytes_tx;
    size_t ws_bytes;
};

// Shared validation and sizing for the GQA/GTA kernel.  tied: GTA.
int plan_group(bool tied, const void *q, const void *c0, const void *c1, const int32_t *bt, const int32_t *sl,
               const void *out, const float *lse, int B, int L, int h_q, int h_kv, int d, int d_r, int S, int P,
               int max_pages, float scale, int num_parts, GroupPlan *gp) {
    if (B < 0 || L < 1 || h_q < 1 || h_kv < 1 || S < 1 || P < 1 || max_pages < 1 || num_parts < 0)
        return KVD_ERR_INVALID_ARG;
    if (!std::isfinite(scale)) return KVD_ERR_INVALID_ARG;
    if (h_q % h_kv) return KVD_ERR_INVALID_ARG;
    if (!q || !c0 || !c1 || !bt || !sl || !out || !lse) return KVD_ERR_INVALID_ARG;
    if (!aligned(q, 16) || !aligned(c0, 16) || !aligned(c1, 16) || !aligned(out, 8) || !aligned(lse, 4) ||
        !aligned(bt, 4) || !aligned(sl, 4))
        return KVD_ERR_INVALID_ARG;
    if (d != 64 && d != 128) return KVD_ERR_UNSUPPORTED_SHAPE;
    if (tied) {
        if ((d_r != 32 && d_r != 64) || d_r > d || (d - d_r) % 16) return KVD_ERR_UNSUPPORTED_SHAPE;
    }
    if ((long long)P * S >= (1ll << 31) || (long long)max_pages * S >= (1ll << 31)) return KVD_ERR_UNSUPPORTED_SHAPE;
    const int R = (h_q / h_kv) * L;
    int nt = R <= 8 ? 1 : R <= 16 ? 2 : R <= 32 ? 4 : 0;
    if (!nt) return KVD_ERR_UNSUPPORTED_SHAPE;
    int gpc = 1;
    for (int g = 8; g >= 1; --g)
        if (h_kv % g == 0) {
            gpc = g;
            break;
        }
    // 32-token stages (two independent MMA chains per wait) when a page holds whole 32-token
    // tiles and at least three stages fit; otherwise 16-token stages.
    auto stage_tx = [&](int tt) -> uint32_t {
        const uint32_t kvt = (uint32_t)gpc * d * tt * 2;
        return tied ? kvt + tt * d_r * 2 : 2 * kvt;
    };
    // Pages that hold whole tiles are loaded with one box per operand; smaller (or ragged)
    // pages are gathered row by row (four rows per TMA).
    const bool fits32 = nt == 1 && 3 * round_up(stage_tx(32), 1024) <= SMEM_BUDGET - 1024;
    int tile = TILE;
    bool gather = false;
    if (S % 32 == 0 && fits32) {
        tile = 32;
    } else if (S % TILE) {
        gather = true;
        tile = fits32 ? 32 : TILE;
    }
    const uint32_t tx = stage_tx(tile);
    const uint32_t stage = (uint32_t)round_up(tx, 1024);
    int nstage = (int)((SMEM_BUDGET - 1024) / stage);
    if (nstage > MAX_STAGES) nstage = MAX_STAGES;
    if (nstage < 2) return KVD_ERR_UNSUPPORTED_SHAPE;
    const int n_sub = h_kv / gpc;
    int parts = num_parts;
    if (parts == 0) {
        const int sms = num_sms_current();
        if (sms <= 0) return KVD_ERR_CUDA;
        parts = sms / n_sub > 0 ? sms / n_sub : 1;
    }
    const size_t slots = (size_t)B + parts - 1;
    const size_t rows = (size_t)L * h_q;
    gp->gpc = gpc;
    gp->n_sub = n_sub;
    gp->parts = parts;
    gp->nt = nt;
    gp->nstage = nstage;
    gp->tile = tile;
    // GTA: a segment start (q rows, the ring's refill, the epilogue) costs about as much as
    // streaming 128 tokens; the split plan counts it (measured on B 32 with 1k..8k contexts:
    // 68.8 us against 72.7 us without).  GQA streams twice the bytes per token and measured no
    // gain from it.
    gp->seg_cost = tied ? 128 / tile : 0;
    gp->gather = gather;
    gp->stage_bytes = stage;
    gp->stage_bytes_tx = tx;
    gp->ws_bytes = WS_HEADER + round_up(slots * rows * 4, 256) + slots * rows * d * 4;
    return KVD_OK;
}

int run_group(bool tied, const void *q, const void *c0, const void *c1, const int32_t *bt, const int32_t *sl,
              void *out, float *lse, int B, int L, int h_q, int h_kv, int d, int d_r, int S, int P, int max_pages,
              float scale, int num_parts, void *ws, size_t ws_bytes, cudaStream_t st) {
    GroupPlan gp;
    int rc = plan_group(tied, q, c0, c1, bt, sl, out, lse, B, L, h_q, h_kv, d, d_r, S, P, max_pages, scale,
                        num_parts, &gp);
    if (rc != KVD_OK) return rc;
    if (!ws || !aligned(ws, 256)) return KVD_ERR_INVALID_ARG;
    if (ws_bytes < gp.ws_bytes) return KVD_ERR_WORKSPACE_TOO_SMALL;
    if (B == 0) return KVD_OK;

    CUtensorMap m0, m1;
    const cuuint64_t tokens = (cuuint64_t)P * S;
    if (gp.gather) {
        memset(&m0, 0, sizeof(m0));  // rows are copied with cp.async; no tensor maps
        memset(&m1, 0, sizeof(m1));
    } else {
        cuuint64_t dims[3] = {64, tokens, (cuuint64_t)h_kv * d / 64};
        cuuint64_t strides[2] = {(cuuint64_t)h_kv * d * 2, 128};
        cuuint32_t box[3] = {64, (cuuint32_t)gp.tile, (cuuint32_t)(gp.gpc * d / 64)};
        if (!encode(&m0, c0, 3, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B)) return KVD_ERR_CUDA;
        if (!tied && !encode(&m1, c1, 3, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B)) return KVD_ERR_CUDA;
        if (tied) {
            cuuint64_t rdims[2] = {(cuuint64_t)d_r, tokens};
            cuuint64_t rstrides[1] = {(cuuint64_t)d_r * 2};
            cuuint32_t rbox[2] = {(cuuint32_t)d_r, (cuuint32_t)gp.tile};
            if (!encode(&m1, c1, 2, rdims, rstrides, rbox,
                        d_r == 64 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B))
                return KVD_ERR_CUDA;
        }
    }

    const size_t slots = (size_t)B + gp.parts - 1;
    const size_t rows = (size_t)L * h_q;
    uint8_t *w = (uint8_t *)ws;
    GroupArgs a;
    a.q = (const __nv_bfloat16 *)q;
    a.block_table = bt;
    a.seqlens = sl;
    a.out = (__nv_bfloat16 *)out;
    a.lse = lse;
    a.err = (uint32_t *)w;
    a.ws_lse = (float *)(w + WS_HEADER);
    a.ws_o = (float *)(w + WS_HEADER + round_up(slots * rows * 4, 256));
    a.B = B;
    a.L = L;
    a.h_q = h_q;
    a.h_kv = h_kv;
    a.page_size = S;
    a.num_pages = P;
    a.max_pages = max_pages;
    a.tile = gp.tile;
    a.seg_cost = gp.seg_cost;
    a.gather = gp.gather ? 1 : 0;
    a.cache0 = c0;
    a.cache1 = c1;
    a.gpc = gp.gpc;
    a.n_sub = gp.n_sub;
    a.parts = gp.parts;
    a.nstage = gp.nstage;
    a.stage_bytes = gp.stage_bytes;
    a.stage_bytes_tx = gp.stage_bytes_tx;
    a.scale_log2 = scale * 1.4426950408889634f;
    a.wait_limit_ns = (uint64_t)g_wait_limit_ns.load();
    a.debug_flags = g_debug_flags.load();
    const size_t smem = (size_t)gp.nstage * gp.stage_bytes + 1024;
    record(g_ev_before, st);
    cudaError_t e = launch_group_decode(tied, d, tied ? d_r : 0, gp.nt, m0, m1, a, gp.parts * gp.n_sub, smem, st);
    if (e != cudaSuccess) return KVD_ERR_CUDA;
    record(g_ev_after, st);

    CombineArgs c;
    c.seqlens = sl;
    c.ws_lse = a.ws_lse;
    c.ws_o = a.ws_o;
    c.out = (__nv_bfloat16 *)out;
    c.lse = lse;
    c.B = B;
    c.L = L;
    c.tile = gp.tile;
    c.seg_cost = gp.seg_cost;
    c.max_tokens = max_pages * S;
    c.parts = gp.parts;
    c.rows = (int)rows;
    c.d_v = d;
    if (launch_combine(c, st) != cudaSuccess) return KVD_ERR_CUDA;
    return KVD_OK;
}

// ----------------------------------------------------------------------------- GLA / MLA
// Shared memory a block may hold in total on sm_100 (227 KB).
constexpr size_t SMEM_PER_BLOCK = 232448;
// Static shared memory of the latent kernel is below this.
constexpr size_t LATENT_STATIC_SMEM = 4096;

struct LatentPlan {
    int spread;  // rows per lane quadrant when the rows are spread (0: not spread)
    bool gather;
    bool narrow;  // at most 64 rows per latent head of width 256: the narrow kernel
    bool m128;    // more rows per latent head of width 256: the 128-row kernel, one CTA per 128 rows
    int tile;     // tokens per plan tile
    int box_tok;  // narrow and 128-row kernels, box path: tokens per TMA box
    int seg_cost; // plan: units a segment start costs, in tiles
    LatentShape shape;
    bool pair;
    int n_rt, n_vc, n_sub, parts, nstage, rb;
    size_t smem, ws_bytes;
};

int plan_latent(const kvd_gla_params *p, LatentPlan *lp) {
    if (p->B < 0 || p->L < 1 || p->h_q < 1 || p->h_c < 1 || p->page_size < 1 || p->num_pages < 1 ||
        p->max_pages < 1 || p->num_parts < 0)
        return KVD_ERR_INVALID_ARG;
    if (!std::isfinite(p->scale) || p->h_q % p->h_c) return KVD_ERR_INVALID_ARG;
    if (!p->q || !p->latent_cache || !p->rope_cache || !p->block_table || !p->seqlens || !p->out || !p->lse)
        return KVD_ERR_INVALID_ARG;
    if (!aligned(p->q, 16) || !aligned(p->latent_cache, 16) || !aligned(p->rope_cache, 16) || !aligned(p->out, 16) ||
        !aligned(p->lse, 4) || !aligned(p->block_table, 4) || !aligned(p->seqlens, 4))
        return KVD_ERR_INVALID_ARG;
    if (p->d_r != 64) return KVD_ERR_UNSUPPORTED_SHAPE;
    LatentShape sh = latent_shape(p->d_c);
    if (sh.tok == 0) return KVD_ERR_UNSUPPORTED_SHAPE;
    // pages that do not hold whole tiles are gathered token by token
    lp->gather = p->page_size % sh.tok != 0;
    const int g = p->h_q / p->h_c;
    if (!(128 % g == 0 || g % 128 == 0)) return KVD_ERR_UNSUPPORTED_SHAPE;
    const long long R = (long long)g * p->L;
    if ((long long)p->num_pages * p->page_size >= (1ll << 31) || (long long)p->max_pages * p->page_size >= (1ll << 31) ||
        (long long)p->B * p->L * p->h_q >= (1ll << 31) || R > 128 * 64)
        return KVD_ERR_UNSUPPORTED_SHAPE;
    lp->shape = sh;
    lp->n_rt = (int)((R + 127) / 128);
    lp->pair = p->d_c == 512;  // CTA pairs split the key dimension instead of the value
    lp->n_vc = lp->pair ? 1 : p->d_c / 256;
    lp->n_sub = p->h_c * lp->n_rt * lp->n_vc;
    const int ctas_per_sub = lp->pair ? 2 : 1;
    // the GLA kernel spreads at most 64 rows evenly over the four TMEM lane quadrants
    // (rpq = 4, 8 or 16 rows each), which needs the q rows in rpq-row runs that stay inside one
    // query position (g % rpq == 0)
    lp->spread = 0;
    if (!lp->pair && R <= 64)
        for (int rpq = 4; rpq <= 16; rpq *= 2)
            if (4 * rpq >= R && g % rpq == 0) {
                lp->spread = rpq;
                break;
            }
    lp->rb = lp->spread ? lp->spread : (g < 128 ? g : 128);
    lp->tile = sh.tok;
    lp->box_tok = 0;
    lp->seg_cost = 0;
    lp->narrow = !lp->pair && p->d_c == 256 && R <= 64;
    lp->m128 = !lp->pair && p->d_c == 256 && R > 64;
    if (lp->narrow || lp->m128) {
        // narrow: rows spread over the four lane quadrants, ceil(R / 4) each; 128-row kernel: row
        // 128 k + n at TMEM lane n of the k-th CTA of a latent head.  The tile is cut into boxes of
        // the largest size that divides both the tile and the page (at least 16 tokens), else
        // gathered token by token
        lp->spread = lp->narrow ? (int)((R + 3) / 4) : 0;
        lp->tile = lp->narrow ? narrow_tile_tokens() : m128_tile_tokens();
        int gcd = lp->tile, b2 = p->page_size;
        while (b2) {
            const int t = gcd % b2;
            gcd = b2;
            b2 = t;
        }
        lp->box_tok = gcd >= 16 ? gcd : 0;
        lp->gather = lp->box_tok == 0;
        lp->seg_cost = lp->narrow ? narrow_seg_cost() : m128_seg_cost();
        lp->nstage = 0;
        lp->smem = lp->narrow ? narrow_smem_bytes() : m128_smem_bytes();
    }
    if (!lp->narrow && !lp->m128) {
        const size_t fixed = SMEM_PER_BLOCK - LATENT_STATIC_SMEM - 1024 - sh.q_bytes - sh.p_bytes;
        int nstage = (int)(fixed / sh.stage_bytes);
        if (nstage > MAX_STAGES) nstage = MAX_STAGES;
        if (nstage < 2) return KVD_ERR_UNSUPPORTED_SHAPE;
        lp->nstage = nstage;
        lp->smem = 1024 + sh.q_bytes + (size_t)nstage * sh.stage_bytes + sh.p_bytes;
    }
    int parts = p->num_parts;
    if (parts == 0) {
        const int sms = num_sms_current();
        if (sms <= 0) return KVD_ERR_CUDA;
        parts = sms / (lp->n_sub * ctas_per_sub) > 0 ? sms / (lp->n_sub * ctas_per_sub) : 1;
    }
    lp->parts = parts;
    const size_t slots = (size_t)p->B + parts - 1;
    const size_t rows = (size_t)p->L * p->h_q;
    lp->ws_bytes = WS_HEADER + round_up(slots * rows * 4, 256) + slots * rows * p->d_c * 4;
    return KVD_OK;
}

int run_latent(const kvd_gla_params *p, void *ws, size_t ws_bytes, cudaStream_t st) {
    LatentPlan lp;
    int rc = plan_latent(p, &lp);
    if (rc != KVD_OK) return rc;
    if (!ws || !aligned(ws, 256)) return KVD_ERR_INVALID_ARG;
    if (ws_bytes < lp.ws_bytes) return KVD_ERR_WORKSPACE_TOO_SMALL;
    if (p->B == 0) return KVD_OK;

    const int d_qk = p->d_c + p->d_r;
    const int kch = d_qk / 64;
    const cuuint64_t tokens = (cuuint64_t)p->num_pages * p->page_size;
    CUtensorMap qm, lm, rm;
    if (lp.narrow || lp.m128) {
        memset(&qm, 0, sizeof(qm));  // q rows are copied by the kernel's softmax warps
        memset(&lm, 0, sizeof(lm));
        memset(&rm, 0, sizeof(rm));
        if (!lp.gather) {
            const cuuint32_t nch = lp.box_tok == lp.tile ? (cuuint32_t)(p->d_c / 64) : 1u;
            cuuint64_t dims[3] = {64, tokens, (cuuint64_t)p->h_c * p->d_c / 64};
            cuuint64_t strides[2] = {(cuuint64_t)p->h_c * p->d_c * 2, 128};
            cuuint32_t box[3] = {64, (cuuint32_t)lp.box_tok, nch};
            if (!encode(&lm, p->latent_cache, 3, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B))
                return KVD_ERR_CUDA;
            cuuint64_t rdims[2] = {64, tokens};
            cuuint64_t rstrides[1] = {128};
            cuuint32_t rbox[2] = {64, (cuuint32_t)lp.box_tok};
            if (!encode(&rm, p->rope_cache, 2, rdims, rstrides, rbox, CU_TENSOR_MAP_SWIZZLE_128B))
                return KVD_ERR_CUDA;
        }
    } else {
        {
            cuuint64_t dims[3] = {64, (cuuint64_t)p->B * p->L * p->h_q, (cuuint64_t)kch};
            cuuint64_t strides[2] = {(cuuint64_t)d_qk * 2, 128};
            cuuint32_t box[3] = {64, (cuuint32_t)lp.rb, 1};
            if (!encode(&qm, p->q, 3, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B)) return KVD_ERR_CUDA;
        }
        if (lp.gather) {
            memset(&lm, 0, sizeof(lm));  // gathered tiles are copied with cp.async: no cache maps
            memset(&rm, 0, sizeof(rm));
        } else {
            {
                cuuint64_t dims[3] = {64, tokens, (cuuint64_t)p->h_c * p->d_c / 64};
                cuuint64_t strides[2] = {(cuuint64_t)p->h_c * p->d_c * 2, 128};
                cuuint32_t box[3] = {64, (cuuint32_t)lp.shape.tok, (cuuint32_t)(p->d_c / 64)};
                if (!encode(&lm, p->latent_cache, 3, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B))
                    return KVD_ERR_CUDA;
            }
            {
                cuuint64_t dims[2] = {64, tokens};
                cuuint64_t strides[1] = {128};
                cuuint32_t box[2] = {64, (cuuint32_t)lp.shape.tok};
                if (!encode(&rm, p->rope_cache, 2, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B))
                    return KVD_ERR_CUDA;
            }
        }
    }
    const size_t slots = (size_t)p->B + lp.parts - 1;
    const size_t rows = (size_t)p->L * p->h_q;
    uint8_t *w = (uint8_t *)ws;
    LatentArgs a;
    a.q = (const __nv_bfloat16 *)p->q;
    a.block_table = p->block_table;
    a.seqlens = p->seqlens;
    a.out = (__nv_bfloat16 *)p->out;
    a.lse = p->lse;
    a.err = (uint32_t *)w;
    a.ws_lse = (float *)(w + WS_HEADER);
    a.ws_o = (float *)(w + WS_HEADER + round_up(slots * rows * 4, 256));
    a.B = p->B;
    a.L = p->L;
    a.h_q = p->h_q;
    a.h_c = p->h_c;
    a.page_size = p->page_size;
    a.num_pages = p->num_pages;
    a.max_pages = p->max_pages;
    a.n_sub = lp.n_sub;
    a.n_rt = lp.n_rt;
    a.row_spread = lp.spread;
    a.noncausal = 0;
    a.box_tok = lp.box_tok;
    a.seg_cost = lp.seg_cost;
    a.gather = lp.gather ? 1 : 0;
    a.cache0 = p->latent_cache;
    a.cache1 = p->rope_cache;
    a.parts = lp.parts;
    a.nstage = lp.nstage;
    a.scale_log2 = p->scale * 1.4426950408889634f;
    a.wait_limit_ns = (uint64_t)g_wait_limit_ns.load();
    a.debug_flags = g_debug_flags.load();
    record(g_ev_before, st);
    if (lp.pair) {
        CUtensorMap qrm, lm2, rm2;
        {   // q's rope dims in 32-wide halves (64-byte rows, 64 B swizzle)
            cuuint64_t dims[3] = {32, (cuuint64_t)p->B * p->L * p->h_q, (cuuint64_t)d_qk / 32};
            cuuint64_t strides[2] = {(cuuint64_t)d_qk * 2, 64};
            cuuint32_t box[3] = {32, (cuuint32_t)lp.rb, 1};
            if (!encode(&qrm, p->q, 3, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_64B)) return KVD_ERR_CUDA;
        }
        if (lp.gather) {
            memset(&lm2, 0, sizeof(lm2));
            memset(&rm2, 0, sizeof(rm2));
        }
        if (!lp.gather) {   // four 64-wide latent chunks (one CTA's half of a latent head) per box
            cuuint64_t dims[3] = {64, tokens, (cuuint64_t)p->h_c * p->d_c / 64};
            cuuint64_t strides[2] = {(cuuint64_t)p->h_c * p->d_c * 2, 128};
            cuuint32_t box[3] = {64, (cuuint32_t)lp.shape.tok, 4};
            if (!encode(&lm2, p->latent_cache, 3, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B))
                return KVD_ERR_CUDA;
        }
        if (!lp.gather) {   // 32-wide halves of the rope rows
            cuuint64_t dims[2] = {64, tokens};
            cuuint64_t strides[1] = {128};
            cuuint32_t box[2] = {32, (cuuint32_t)lp.shape.tok};
            if (!encode(&rm2, p->rope_cache, 2, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_64B)) return KVD_ERR_CUDA;
        }
        if (launch_mla_pair(qm, qrm, lm2, rm2, a, lp.parts * lp.n_sub * 2, lp.smem, st) != cudaSuccess)
            return KVD_ERR_CUDA;
    } else if (lp.narrow) {
        if (launch_gla_narrow(lm, rm, a, lp.parts * lp.n_sub, st) != cudaSuccess) return KVD_ERR_CUDA;
    } else if (lp.m128) {
        if (launch_gla_m128(lm, rm, a, lp.parts * lp.n_sub, st) != cudaSuccess) return KVD_ERR_CUDA;
    } else {
        return KVD_ERR_UNSUPPORTED_SHAPE;  // d_c 256 takes one of the two kernels above
    }
    record(g_ev_after, st);

    CombineArgs c;
    c.seqlens = p->seqlens;
    c.ws_lse = a.ws_lse;
    c.ws_o = a.ws_o;
    c.out = (__nv_bfloat16 *)p->out;
    c.lse = p->lse;
    c.B = p->B;
    c.L = p->L;
    c.tile = lp.tile;
    c.seg_cost = lp.seg_cost;
    c.max_tokens = p->max_pages * p->page_size;
    c.parts = lp.parts;
    c.rows = (int)rows;
    c.d_v = p->d_c;
    if (launch_combine(c, st) != cudaSuccess) return KVD_ERR_CUDA;
    return KVD_OK;
}

}  // namespace

extern "C" {

size_t kvd_gla_workspace_size(const kvd_gla_params *p) {
    if (!p) return 0;
    LatentPlan lp;
    if (plan_latent(p, &lp) != KVD_OK) return 0;
    return lp.ws_bytes;
}

int kvd_gla_decode(const kvd_gla_params *p, void *ws, size_t ws_bytes, kvd_stream_t stream) {
    if (!p) return KVD_ERR_INVALID_ARG;
    return run_latent(p, ws, ws_bytes, (cudaStream_t)stream);
}

size_t kvd_gqa_workspace_size(const kvd_gqa_params *p) {
    if (!p) return 0;
    GroupPlan gp;
    if (plan_group(false, p->q, p->k_cache, p->v_cache, p->block_table, p->seqlens, p->out, p->lse, p->B, p->L,
                   p->h_q, p->h_kv, p->d, 0, p->page_size, p->num_pages, p->max_pages, p->scale, p->num_parts,
                   &gp) != KVD_OK)
        return 0;
    return gp.ws_bytes;
}

size_t kvd_gta_workspace_size(const kvd_gta_params *p) {
    if (!p) return 0;
    GroupPlan gp;
    if (plan_group(true, p->q, p->tied_cache, p->rope_cache, p->block_table, p->seqlens, p->out, p->lse, p->B,
                   p->L, p->h_q, p->h_kv, p->d_h, p->d_r, p->page_size, p->num_pages, p->max_pages, p->scale,
                   p->num_parts, &gp) != KVD_OK)
        return 0;
    return gp.ws_bytes;
}

int kvd_gqa_decode(const kvd_gqa_params *p, void *ws, size_t ws_bytes, kvd_stream_t stream) {
    if (!p) return KVD_ERR_INVALID_ARG;
    return run_group(false, p->q, p->k_cache, p->v_cache, p->block_table, p->seqlens, p->out, p->lse, p->B, p->L,
                     p->h_q, p->h_kv, p->d, 0, p->page_size, p->num_pages, p->max_pages, p->scale, p->num_parts, ws,
                     ws_bytes, (cudaStream_t)stream);
}

int kvd_gta_decode(const kvd_gta_params *p, void *ws, size_t ws_bytes, kvd_stream_t stream) {
    if (!p) return KVD_ERR_INVALID_ARG;
    return run_group(true, p->q, p->tied_cache, p->rope_cache, p->block_table, p->seqlens, p->out, p->lse, p->B,
                     p->L, p->h_q, p->h_kv, p->d_h, p->d_r, p->page_size, p->num_pages, p->max_pages, p->scale,
                     p->num_parts, ws, ws_bytes, (cudaStream_t)stream);
}

// ----------------------------------------------------------------------------- GTA prefix
// All B x L query rows attend one shared prefix (no causal mask) on the latent kernel: one
// pseudo-sequence whose q positions are the batch's rows, state = a tied group (key: its first
// 64 dims and the rope slice; value: all 128 dims).
struct PrefixPlan {
    LatentShape shape;
    bool gather;
    int n_rt, n_sub, parts, nstage, rb, rows_pos;
    size_t smem, ws_bytes;
};

int plan_prefix(const kvd_gta_params *p, PrefixPlan *pp) {
    if (p->B < 0 || p->L < 1 || p->h_q < 1 || p->h_kv < 1 || p->page_size < 1 || p->num_pages < 1 ||
        p->max_pages < 1 || p->num_parts < 0)
        return KVD_ERR_INVALID_ARG;
    if (!std::isfinite(p->scale) || p->h_q % p->h_kv) return KVD_ERR_INVALID_ARG;
    if (!p->q || !p->tied_cache || !p->rope_cache || !p->block_table || !p->seqlens || !p->out || !p->lse)
        return KVD_ERR_INVALID_ARG;
    if (!aligned(p->q, 16) || !aligned(p->tied_cache, 16) || !aligned(p->rope_cache, 16) || !aligned(p->out, 16) ||
        !aligned(p->lse, 4) || !aligned(p->block_table, 4) || !aligned(p->seqlens, 4))
        return KVD_ERR_INVALID_ARG;
    if (p->d_h != 128 || p->d_r != 64) return KVD_ERR_UNSUPPORTED_SHAPE;
    const int g = p->h_q / p->h_kv;
    if (!(128 % g == 0 || g % 128 == 0)) return KVD_ERR_UNSUPPORTED_SHAPE;
    const long long rows_pos = (long long)p->B * p->L;  // query positions of the pseudo-sequence
    const long long R = (long long)g * rows_pos;
    if ((long long)p->num_pages * p->page_size >= (1ll << 31) || (long long)p->max_pages * p->page_size >= (1ll << 31) ||
        rows_pos * p->h_q >= (1ll << 31) || R > 128 * 64)
        return KVD_ERR_UNSUPPORTED_SHAPE;
    pp->shape = tied_prefix_shape();
    pp->gather = p->page_size % pp->shape.tok != 0;
    pp->rows_pos = (int)rows_pos;
    pp->n_rt = (int)((R + 127) / 128);
    pp->n_sub = p->h_kv * pp->n_rt;
    pp->rb = g < 128 ? g : 128;
    const size_t fixed = SMEM_PER_BLOCK - LATENT_STATIC_SMEM - 1024 - pp->shape.q_bytes;
    int nstage = (int)(fixed / pp->shape.stage_bytes);
    if (nstage > MAX_STAGES) nstage = MAX_STAGES;
    if (nstage < 2) return KVD_ERR_UNSUPPORTED_SHAPE;
    pp->nstage = nstage;
    pp->smem = 1024 + pp->shape.q_bytes + (size_t)nstage * pp->shape.stage_bytes;
    int parts = p->num_parts;
    if (parts == 0) {
        const int sms = num_sms_current();
        if (sms <= 0) return KVD_ERR_CUDA;
        parts = sms / pp->n_sub > 0 ? sms / pp->n_sub : 1;
    }
    pp->parts = parts;
    const size_t slots = (size_t)parts;  // one pseudo-sequence: slot = part
    const size_t rows = (size_t)rows_pos * p->h_q;
    pp->ws_bytes = WS_HEADER + round_up(slots * rows * 4, 256) + slots * rows * 128 * 4;
    return KVD_OK;
}

size_t kvd_gta_prefix_workspace_size(const kvd_gta_params *p) {
    PrefixPlan pp;
    return (p && plan_prefix(p, &pp) == KVD_OK) ? pp.ws_bytes : 0;
}

int kvd_gta_prefix_decode(const kvd_gta_params *p, void *ws, size_t ws_bytes, kvd_stream_t stream) {
    if (!p) return KVD_ERR_INVALID_ARG;
    PrefixPlan pp;
    int rc = plan_prefix(p, &pp);
    if (rc != KVD_OK) return rc;
    if (!ws || !aligned(ws, 256)) return KVD_ERR_INVALID_ARG;
    if (ws_bytes < pp.ws_bytes) return KVD_ERR_WORKSPACE_TOO_SMALL;
    if (p->B == 0) return KVD_OK;
    cudaStream_t st = (cudaStream_t)stream;
    const cuuint64_t tokens = (cuuint64_t)p->num_pages * p->page_size;
    CUtensorMap qm, lm, rm;
    {
        cuuint64_t dims[3] = {64, (cuuint64_t)pp.rows_pos * p->h_q, 2};
        cuuint64_t strides[2] = {(cuuint64_t)p->d_h * 2, 128};
        cuuint32_t box[3] = {64, (cuuint32_t)pp.rb, 1};
        if (!encode(&qm, p->q, 3, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B)) return KVD_ERR_CUDA;
    }
    if (pp.gather) {
        memset(&lm, 0, sizeof(lm));
        memset(&rm, 0, sizeof(rm));
    } else {
        cuuint64_t dims[3] = {64, tokens, (cuuint64_t)p->h_kv * 2};
        cuuint64_t strides[2] = {(cuuint64_t)p->h_kv * p->d_h * 2, 128};
        cuuint32_t box[3] = {64, (cuuint32_t)pp.shape.tok, 2};
        if (!encode(&lm, p->tied_cache, 3, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B)) return KVD_ERR_CUDA;
        cuuint64_t rdims[2] = {64, tokens};
        cuuint64_t rstrides[1] = {128};
        cuuint32_t rbox[2] = {64, (cuuint32_t)pp.shape.tok};
        if (!encode(&rm, p->rope_cache, 2, rdims, rstrides, rbox, CU_TENSOR_MAP_SWIZZLE_128B)) return KVD_ERR_CUDA;
    }
    const size_t slots = (size_t)pp.parts;
    const size_t rows = (size_t)pp.rows_pos * p->h_q;
    uint8_t *w = (uint8_t *)ws;
    LatentArgs a;
    memset(&a, 0, sizeof(a));
    a.q = (const __nv_bfloat16 *)p->q;
    a.block_table = p->block_table;
    a.seqlens = p->seqlens;
    a.out = (__nv_bfloat16 *)p->out;
    a.lse = p->lse;
    a.err = (uint32_t *)w;
    a.ws_lse = (float *)(w + WS_HEADER);
    a.ws_o = (float *)(w + WS_HEADER + round_up(slots * rows * 4, 256));
    a.B = 1;
    a.L = pp.rows_pos;
    a.h_q = p->h_q;
    a.h_c = p->h_kv;
    a.page_size = p->page_size;
    a.num_pages = p->num_pages;
    a.max_pages = p->max_pages;
    a.n_sub = pp.n_sub;
    a.n_rt = pp.n_rt;
    a.row_spread = 0;
    a.noncausal = 1;
    a.box_tok = 0;
    a.seg_cost = 0;
    a.gather = pp.gather ? 1 : 0;
    a.cache0 = p->tied_cache;
    a.cache1 = p->rope_cache;
    a.parts = pp.parts;
    a.nstage = pp.nstage;
    a.scale_log2 = p->scale * 1.4426950408889634f;
    a.wait_limit_ns = (uint64_t)g_wait_limit_ns.load();
    a.debug_flags = g_debug_flags.load();
    record(g_ev_before, st);
    if (launch_tied_prefix(qm, lm, rm, a, pp.parts * pp.n_sub, pp.smem, st) != cudaSuccess) return KVD_ERR_CUDA;
    record(g_ev_after, st);
    CombineArgs c;
    c.seqlens = p->seqlens;
    c.ws_lse = a.ws_lse;
    c.ws_o = a.ws_o;
    c.out = (__nv_bfloat16 *)p->out;
    c.lse = p->lse;
    c.B = 1;
    c.L = 1;  // the plan of a non-causal pseudo-sequence (every position sees all tokens)
    c.tile = pp.shape.tok;
    c.seg_cost = 0;
    c.max_tokens = p->max_pages * p->page_size;
    c.parts = pp.parts;
    c.rows = (int)rows;
    c.d_v = 128;
    if (launch_combine(c, st) != cudaSuccess) return KVD_ERR_CUDA;
    return KVD_OK;
}

int kvd_merge_states(const void *out_a, const float *lse_a, const void *out_b, const float *lse_b, void *out,
                     float *lse, int32_t rows, int32_t d_v, kvd_stream_t stream) {
    if (rows < 0 || d_v <= 0 || d_v % 8) return KVD_ERR_INVALID_ARG;
    if (!out_a || !out_b || !out || !lse_a || !lse_b || !lse) return KVD_ERR_INVALID_ARG;
    if (!aligned(out_a, 16) || !aligned(out_b, 16) || !aligned(out, 16) || !aligned(lse_a, 4) || !aligned(lse_b, 4) ||
        !aligned(lse, 4))
        return KVD_ERR_INVALID_ARG;
    return launch_merge(out_a, lse_a, out_b, lse_b, out, lse, rows, d_v, (cudaStream_t)stream) == cudaSuccess
               ? KVD_OK
               : KVD_ERR_CUDA;
}

int kvd_plan(const int32_t *seqlens, int32_t B, int32_t tile, int32_t seg_cost, int32_t max_tokens,
             int32_t num_parts, int32_t *segments, int32_t *counts, int32_t cap, kvd_stream_t stream) {
    if (B < 0 || tile < 1 || seg_cost < 0 || max_tokens < 0 || num_parts < 1 || cap < 0) return KVD_ERR_INVALID_ARG;
    if ((B > 0 && !seqlens) || !counts || (cap > 0 && !segments)) return KVD_ERR_INVALID_ARG;
    return launch_plan(seqlens, B, tile, seg_cost, max_tokens, 1, num_parts, segments, counts, cap,
                       (cudaStream_t)stream) ==
                   cudaSuccess
               ? KVD_OK
               : KVD_ERR_CUDA;
}

int kvd_plan_host(const int32_t *seqlens, int32_t B, int32_t tile, int32_t seg_cost, int32_t max_tokens,
                  int32_t num_parts, int32_t *segments, int32_t *counts, int32_t cap) {
    if (B < 0 || tile < 1 || seg_cost < 0 || max_tokens < 0 || num_parts < 1 || cap < 0) return KVD_ERR_INVALID_ARG;
    if ((B > 0 && !seqlens) || !counts || (cap > 0 && !segments)) return KVD_ERR_INVALID_ARG;
    int64_t N = 0;
    for (int b = 0; b < B; ++b) N += units_of(tiles_of(clamp_len(seqlens[b], max_tokens, 1, nullptr), tile), seg_cost);
    const int64_t P = N < num_parts ? N : num_parts;
    for (int c = 0; c < num_parts; ++c) {
        int cnt = 0;
        if (N > 0 && c < P) {
            const int64_t lo = part_begin(c, N, P), hi = part_begin(c + 1, N, P);
            int64_t run = 0;  // units before sequence b
            for (int b = 0; b < B && run < hi; ++b) {
                const int32_t n = tiles_of(clamp_len(seqlens[b], max_tokens, 1, nullptr), tile);
                const int64_t cu = run + units_of(n, seg_cost) - n;  // the unit of b's first tile
                if (n > 0 && cu < hi && cu + n > lo) {
                    if (cnt < cap) {
                        Seg s = make_seg(b, cu, n, lo, hi, c, N, P);
                        int32_t *o = segments + ((size_t)c * cap + cnt) * 6;
                        o[0] = s.b;
                        o[1] = s.t0;
                        o[2] = s.t1;
                        o[3] = s.split;
                        o[4] = s.nsplit;
                        o[5] = s.slot;
                    }
                    ++cnt;
                }
                run += units_of(n, seg_cost);
            }
        }
        counts[c] = cnt;
    }
    return KVD_OK;
}

int kvd_read_device_error(void *ws, kvd_stream_t stream, uint32_t *flags) {
    if (!ws || !flags) return KVD_ERR_INVALID_ARG;
    cudaStream_t st = (cudaStream_t)stream;
    uint32_t v = 0;
    if (cudaMemcpyAsync(&v, ws, sizeof v, cudaMemcpyDeviceToHost, st) != cudaSuccess) return KVD_ERR_CUDA;
    if (cudaMemsetAsync(ws, 0, sizeof v, st) != cudaSuccess) return KVD_ERR_CUDA;
    if (cudaStreamSynchronize(st) != cudaSuccess) return KVD_ERR_CUDA;
    *flags = v;
    return v ? KVD_ERR_DEVICE : KVD_OK;
}

int kvd_profile_events(void *before_main, void *after_main) {
    if ((before_main == nullptr) != (after_main == nullptr)) return KVD_ERR_INVALID_ARG;
    g_ev_before.store(before_main);
    g_ev_after.store(after_main);
    return KVD_OK;
}

int kvd_num_sms(void) {
    const int n = num_sms_current();
    return n > 0 ? n : KVD_ERR_CUDA;
}

int kvd_debug_set(int knob, long long value) {
    switch (knob) {
        case KVD_DEBUG_WAIT_LIMIT_NS:
            if (value <= 0) return KVD_ERR_INVALID_ARG;
            g_wait_limit_ns.store(value);
            return KVD_OK;
        case KVD_DEBUG_SKIP_FIRST_LOAD:
            if (value)
                g_debug_flags.fetch_or(DEBUG_SKIP_FIRST_LOAD);
            else
                g_debug_flags.fetch_and(~DEBUG_SKIP_FIRST_LOAD);
            return KVD_OK;
        default:
            return KVD_ERR_INVALID_ARG;
    }
}

const char *kvd_status_string(int s) {
    switch (s) {
        case KVD_OK: return "ok";
        case KVD_ERR_INVALID_ARG: return "invalid argument";
        case KVD_ERR_UNSUPPORTED_SHAPE: return "unsupported shape";
        case KVD_ERR_WORKSPACE_TOO_SMALL: return "workspace too small";
        case KVD_ERR_CUDA: return "CUDA error";
        case KVD_ERR_DEVICE: return "device error flag set";
        default: return "unknown status";
    }
}

int kvd_version(void) { return 100; }

}  // extern "C"

// ----------------------------------------------------------------------------- allocation-free GTA entry
// Some callers cannot hand us a workspace: a serving engine that has already
// carved all of HBM into KV pages and its own arenas (so any further device
// allocation can fail, or fragment memory it manages), or code that issues
// this call while a stream is being captured in global mode, where
// cudaMalloc is not a legal call.  For them kvd_gta_decode_noalloc() runs the
// same kernels as kvd_gta_decode() with the workspace placed in this fixed
// device array, which every GPU that loads the library holds until the
// process exits.
namespace {

constexpr size_t NOALLOC_WS_BYTES = 8u << 20;  // 8 MiB
static __device__ __align__(256) uint8_t g_noalloc_ws[NOALLOC_WS_BYTES];

// Device address of g_noalloc_ws in the current context.  Host code must not use
// the symbol itself as a pointer: on the host it names a stand-in, not device
// memory.  The address is looked up on every call (a host-side table lookup once
// the module is loaded), so a context that was reset and recreated gets the new
// array's address rather than a stale one.  The first lookup on a device loads
// the library's device code there.
void *noalloc_workspace(int *status) {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_ws) != cudaSuccess || !p) {
        *status = KVD_ERR_CUDA;
        return nullptr;
    }
    *status = KVD_OK;
    return p;
}

}  // namespace

extern "C" int kvd_gta_decode_noalloc(const kvd_gta_params *p, kvd_stream_t stream) {
    if (!p) return KVD_ERR_INVALID_ARG;
    GroupPlan gp;
    int rc = plan_group(true, p->q, p->tied_cache, p->rope_cache, p->block_table, p->seqlens, p->out, p->lse, p->B,
                        p->L, p->h_q, p->h_kv, p->d_h, p->d_r, p->page_size, p->num_pages, p->max_pages, p->scale,
                        p->num_parts, &gp);
    if (rc != KVD_OK) return rc;
    if (gp.ws_bytes > NOALLOC_WS_BYTES) return KVD_ERR_WORKSPACE_TOO_SMALL;
    void *ws = noalloc_workspace(&rc);
    if (rc != KVD_OK) return rc;
    return run_group(true, p->q, p->tied_cache, p->rope_cache, p->block_table, p->seqlens, p->out, p->lse, p->B,
                     p->L, p->h_q, p->h_kv, p->d_h, p->d_r, p->page_size, p->num_pages, p->max_pages, p->scale,
                     p->num_parts, ws, NOALLOC_WS_BYTES, (cudaStream_t)stream);
}
