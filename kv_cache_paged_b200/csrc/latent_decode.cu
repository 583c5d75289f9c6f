// Latent-style attention over a paged cache on 5th-generation tensor cores (tcgen05,
// accumulators in tensor memory), for one state shared by 128-row blocks of query rows with a
// 64-token tile and q's rows loaded by TMA.  It serves the batched shared-prefix pass of GTA
// (kvd_gta_prefix_decode): the state is one tied group (d_h 128), the key its first 64 dims plus
// the 64-wide rope slice, and all B x L rows of a KV group's heads attend the prefix once,
// without the causal mask.  (GLA decode itself runs on gla_narrow_kernel, at most 64 rows per
// latent head, and gla_m128_kernel, more rows; MLA on the CTA-pair kernel.)
//
// "Hardware-Efficient Attention for Fast Decoding", section 3.3.2 gives the absorbed form this
// follows: query head h attends state c = h / (h_q / h_c) with key [state_c ++ rope] and value
// state_c.  The rows of a state share every loaded row, so the step is a dense contraction.
//
// One CTA owns one contiguous part of the (sequence, TOK-token tile) stream, one state c and
// one 128-row block of the (q position, head) rows.  Roles:
//   warp 0      producer: q's rope chunk of the segment, then per tile one 3-D TMA for
//               the latent rows and one for the rope rows (128 B swizzle), into an
//               n-stage mbarrier ring; block-table entries a warp at a time.  Pages that
//               do not hold whole tiles are gathered token by token with cp.async by
//               warps 0, 2 and 3 into the same layout.
//   warp 1      MMA issuer (one thread): S = Q K^T into one of two TMEM S buffers
//               (M 128 rows, N TOK tokens, K d_c + d_r; q's latent part is the A operand
//               from tensor memory, its rope chunk from shared memory), then O += P V
//               (N d_c, K TOK, V read MN-major straight from the latent tile, P the A
//               operand from tensor memory); completion reported with tcgen05.commit.
//   warps 4..7  softmax, one thread per row (TMEM lane): load the S row, mask, fp32 online
//               softmax in base 2 with a lazy rescale (O in TMEM is rescaled only when the
//               running max grows by more than 2^8), write P as bf16 pairs over S in the
//               same TMEM columns; at segment start they write q's latent part into TMEM;
//               epilogue out / lse or split partials.
// Tensor memory (512 columns): O [0, d_c), the two S/P buffers [d_c, d_c + 2 TOK), q's
// key part (bf16 pairs) after them.
#include <cuda_bf16.h>

#include "common.cuh"
#include "kernels.h"

namespace kvd {

namespace {

constexpr int LMAXSEG = 32;
constexpr int NSMX = 4;  // softmax warps, one per TMEM lane quadrant
constexpr int NGATHER = 3;  // warps that copy gathered tiles (0, 2, 3)
constexpr int LTHREADS = 32 * (4 + NSMX);  // warp 0 producer, 1 MMA, 2-3 idle, 4.. softmax
constexpr float RESCALE_LOG2 = 8.f;

// DC: width of the stored state the value reads (GLA: one latent head, 256; the GTA prefix
// path: one tied group, 128); KL: its 64-wide chunks that are also key dims (GLA: all four;
// GTA: the first, the non-RoPE half of the key).  The key is those chunks plus the 64-wide rope.
template <int DC, int TOK, int KL>
struct LatCfg {
    static constexpr int DV = DC;                         // value columns (fp32 accumulator columns)
    static constexpr int NV = DC / 64;                    // 64-wide chunks of the state in a stage
    static constexpr int KCH = NV + 1;                    // stage chunks: state, then rope
    static constexpr int NVC = 1;                         // value slices
    static constexpr uint32_t Q_BYTES = 128 * 128;        // q's rope chunk: 128 rows x 128 B
    static constexpr uint32_t CHUNK = TOK * 128;          // one 64-dim chunk of a tile
    static constexpr uint32_t STAGE = KCH * CHUNK;
    static constexpr uint32_t S_COL = DV;                 // TMEM columns of the two S buffers
    static constexpr uint32_t Q_COL = DV + 2 * TOK;       // TMEM columns of q's key part (bf16 pairs)
    static constexpr int DQK = KL * 64 + 64;              // q row: key part of the state, then rope
    static_assert(KL <= NV && Q_COL + KL * 32 <= 512, "q's key part must fit in tensor memory");
};

template <int DC, int TOK, int KL>
__global__ void __launch_bounds__(LTHREADS, 1)
    latent_decode_kernel(const __grid_constant__ CUtensorMap qmap, const __grid_constant__ CUtensorMap latmap,
                         const __grid_constant__ CUtensorMap ropemap, const LatentArgs a) {
    using C = LatCfg<DC, TOK, KL>;
    constexpr int DV = C::DV;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    __shared__ uint64_t full_bar[MAX_STAGES], empty_bar[MAX_STAGES];
    __shared__ uint64_t qfull_bar, qtm_bar, qempty_bar, sfull_bar[2], pfull_bar[2], end_bar;
    __shared__ Seg segs[LMAXSEG];
    __shared__ int nseg_sh, more_sh;
    __shared__ volatile int abort_sh;
    __shared__ uint32_t tmem_sh;

    uint8_t *smem = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    uint8_t *q_s = smem;
    uint8_t *stage_s = smem + C::Q_BYTES;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int part = blockIdx.x / a.n_sub, sub = blockIdx.x % a.n_sub;
    const int vc = sub % C::NVC;
    const int rt = (sub / C::NVC) % a.n_rt;
    const int c = sub / (C::NVC * a.n_rt);
    const int g = a.h_q / a.h_c;
    const int R = g * a.L;
    const int max_tokens = a.max_pages * a.page_size;
    const int nstage = a.nstage;
    const uint64_t lim_ns = a.wait_limit_ns;

    if (threadIdx.x == 0) {
        for (int s = 0; s < nstage; ++s) {
            mbar_init(&full_bar[s], a.gather ? 32 * NGATHER : 1);  // gathered: one arrival per gather lane
            mbar_init(&empty_bar[s], 1);
        }
        mbar_init(&qfull_bar, 1);  // q's rope chunk (TMA)
        mbar_init(&qtm_bar, 4);    // q's latent part written into tensor memory by softmax warps 4..7
        mbar_init(&qempty_bar, 1);
        for (int s = 0; s < 2; ++s) {
            mbar_init(&sfull_bar[s], 1);
            mbar_init(&pfull_bar[s], NSMX);  // one arrival per softmax warp
        }
        mbar_init(&end_bar, 1);
        abort_sh = 0;
        fence_mbar_init();
    }
    if (warp == 1) tmem_alloc(&tmem_sh, 512);
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&qmap);
        if (!a.gather) {
            tma_prefetch_desc(&latmap);
            tma_prefetch_desc(&ropemap);
        }
    }
    pdl_launch_dependents();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tmem_sh;

    // counters that persist across segment-list rounds
    uint32_t p_issued = 0, p_qloads = 0;                    // producer
    uint32_t m_tile = 0, m_s = 0, m_pv = 0, m_q = 0;        // MMA issuer
    uint32_t x_tile = 0, x_s = 0, x_pv = 0, x_q = 0;  // softmax

    for (int skip = 0;; skip += LMAXSEG) {
        if (warp == 0) {
            int cnt = 0;
            plan_walk(a.seqlens, a.B, TOK, a.seg_cost, max_tokens, a.noncausal ? 1 : a.L, part, a.parts, a.err, [&](const Seg &s) {
                if (cnt >= skip && cnt < skip + LMAXSEG) segs[cnt - skip] = s;
                ++cnt;
            });
            if (lane == 0) {
                nseg_sh = cnt - skip < LMAXSEG ? (cnt - skip > 0 ? cnt - skip : 0) : LMAXSEG;
                more_sh = cnt > skip + LMAXSEG;
            }
        }
        __syncthreads();
        const int nseg = nseg_sh;

        if (warp == 0 || (a.gather && (warp == 2 || warp == 3))) {
            // ================================================================ producer(s)
            // warp 0: q's rope chunk per segment and the KV tiles; with gathered tiles warps 2
            // and 3 copy their share of every tile too
            const int gw = warp == 0 ? 0 : warp - 1;
            const uint64_t pol = policy_evict_first();
            bool stop = false;
            const int rb = a.row_spread ? a.row_spread : (g < 128 ? g : 128);  // q rows per TMA box
            const int rows_tile = min(R - rt * 128, 128);          // valid rows of this row block
            for (int si = 0; si < nseg && !stop; ++si) {
                const Seg sg = segs[si];
                if (warp == 0 && !mbar_wait_warp(&qempty_bar, (p_qloads & 1) ^ 1, &abort_sh, a.err, lim_ns)) {
                    stop = true;
                    break;
                }
                if (warp == 0 && lane == 0) {
                    mbar_arrive_expect_tx(&qfull_bar, (uint32_t)rows_tile * 128);
                    for (int run = 0; run * rb < rows_tile; ++run) {
                        const int n0 = rt * 128 + run * rb;
                        const int i = n0 / g, h0 = n0 % g;
                        const int row = (sg.b * a.L + i) * a.h_q + c * g + h0;
                        // spread rows: run k (rows k * row_spread ..) lands at lanes 32k .. (see the softmax)
                        const int srow = a.row_spread ? run * 32 : run * rb;
                        tma_load_3d(q_s + srow * 128, &qmap, &qfull_bar, 0, row, KL, pol);
                    }
                }
                if (warp == 0) ++p_qloads;
                const int32_t *bt = a.block_table + (size_t)sg.b * a.max_pages;
                if (a.gather) {
                    // Pages smaller than the tile (down to one token) or not a multiple of it: the
                    // NGATHER gather warps (0, 2, 3) split the tile's tokens k = gw, gw + NGATHER, ..;
                    // lane i resolves the cache row of the warp's i-th token (a tile ahead), then
                    // the warp copies each token's latent and rope rows with 16-byte cp.async into
                    // the layout the box loads produce; every lane arrives on the stage barrier
                    // when its copies have landed.
                    const int T = clamp_len(__ldg(a.seqlens + sg.b), max_tokens, a.L, nullptr);
                    const __nv_bfloat16 *lat = (const __nv_bfloat16 *)a.cache0 + (size_t)c * DC;
                    const __nv_bfloat16 *rope = (const __nv_bfloat16 *)a.cache1;
                    const int nk = (TOK - gw + NGATHER - 1) / NGATHER;
                    auto tok_of = [&](int t) { return min(t * TOK + gw + NGATHER * lane, T - 1); };
                    int nxt = lane < nk ? __ldg(bt + tok_of(sg.t0) / a.page_size) : 0;
                    for (int t = sg.t0; t < sg.t1 && !stop; ++t) {
                        int pg = nxt;
                        if (t + 1 < sg.t1 && lane < nk) nxt = __ldg(bt + tok_of(t + 1) / a.page_size);
                        const uint32_t stage = p_issued % nstage;
                        if (!mbar_wait_warp(&empty_bar[stage], ((p_issued / nstage) & 1) ^ 1, &abort_sh, a.err,
                                            lim_ns)) {
                            stop = true;
                            break;
                        }
                        int myrow = 0;  // cache row of this warp's lane-th token (past T_b: repeat)
                        if (lane < nk) {
                            if (pg < 0 || pg >= a.num_pages) {
                                set_error(a.err, DEVERR_BAD_PAGE);
                                pg = 0;
                            }
                            myrow = pg * a.page_size + tok_of(t) % a.page_size;
                        }
                        if (!(a.debug_flags & DEBUG_SKIP_FIRST_LOAD) || p_issued != 0) {
                            const uint32_t st = smem_u32(stage_s + (size_t)stage * C::STAGE);
                            gather_tile<DC / 64, 8>(st, C::CHUNK, lat, (size_t)a.h_c * DC, rope, 64,
                                                    st + (DC / 64) * C::CHUNK, myrow, gw, NGATHER, nk, lane, pol);
                            cp_async_arrive(&full_bar[stage]);
                        }
                        ++p_issued;
                    }
                    continue;
                }
                const int tpp = a.page_size / TOK;
                const int p_first = sg.t0 / tpp, p_last = (sg.t1 - 1) / tpp;
                for (int pb = p_first; pb <= p_last && !stop; pb += 32) {
                    int page = 0;
                    if (pb + lane <= p_last) {
                        page = __ldg(bt + pb + lane);
                        if (page < 0 || page >= a.num_pages) {
                            set_error(a.err, DEVERR_BAD_PAGE);
                            page = 0;
                        }
                    }
                    const int t_lo = max(sg.t0, pb * tpp), t_hi = min(sg.t1, (pb + 32) * tpp);
                    for (int t = t_lo; t < t_hi; ++t) {
                        const int pg = __shfl_sync(0xffffffffu, page, t / tpp - pb);
                        const uint32_t stage = p_issued % nstage;
                        if (!mbar_wait_warp(&empty_bar[stage], ((p_issued / nstage) & 1) ^ 1, &abort_sh, a.err,
                                            lim_ns)) {
                            stop = true;
                            break;
                        }
                        if (lane == 0) {
                            uint8_t *st = stage_s + (size_t)stage * C::STAGE;
                            const int row = pg * a.page_size + (t % tpp) * TOK;
                            mbar_arrive_expect_tx(&full_bar[stage], C::STAGE);
                            if (!(a.debug_flags & DEBUG_SKIP_FIRST_LOAD) || p_issued != 0) {
                                tma_load_3d(st, &latmap, &full_bar[stage], 0, row, c * (DC / 64), pol);
                                tma_load_2d(st + (DC / 64) * C::CHUNK, &ropemap, &full_bar[stage], 0, row, pol);
                            }
                        }
                        ++p_issued;
                    }
                }
            }
            if (stop) {
                // let every copy already issued land before the CTA can exit
                volatile int never = 0;
                if (a.gather) {
                    asm volatile("cp.async.wait_all;" ::: "memory");  // this lane's copies
                } else {
                    const uint32_t lo = p_issued > (uint32_t)nstage ? p_issued - nstage : 0;
                    for (uint32_t k = lo; k < p_issued; ++k)
                        mbar_wait_warp(&full_bar[k % nstage], (k / nstage) & 1, &never, nullptr, lim_ns);
                }
                if (p_qloads) mbar_wait_warp(&qfull_bar, (p_qloads - 1) & 1, &never, nullptr, lim_ns);
            }
        } else if (warp == 1) {
            // ================================================================ MMA issuer
            if (lane == 0) {
                constexpr uint32_t idesc_s = umma_idesc_bf16(128, TOK, false, false);
                constexpr uint32_t idesc_pv = umma_idesc_bf16(128, DV, false, true);
                const uint32_t st0 = smem_u32(stage_s);
                const uint64_t dq0 = umma_desc(smem_u32(q_s), 16, 1024, 2);
                bool ok = true;
                auto issue_s = [&](uint32_t gt) -> bool {
                    const uint32_t stage = gt % nstage;
                    if (!mbar_wait_one(&full_bar[stage], (gt / nstage) & 1, &abort_sh, a.err, lim_ns)) return false;
                    // S(j) goes into buffer j & 1, over P(j - 2): the MMAs of one thread run in
                    // issue order, so this product, issued after the P.V product of tile j - 2,
                    // cannot overwrite that P before it is read
                    const uint32_t sb = m_s & 1;
                    tc_fence_after();
                    // gathered rows were written by cp.async (the generic proxy); the tensor core reads
                    // them through the async proxy, so order the two before the MMAs
                    if (a.gather) fence_proxy_async();
                    const uint32_t d = tmem + C::S_COL + sb * TOK;
                    // descriptors advance by (byte offset >> 4) in their low word: one add per MMA
                    const uint64_t dk0 = umma_desc(st0 + stage * C::STAGE, 16, 1024, 2);
#pragma unroll
                    for (int kc = 0; kc < KL; ++kc)  // key chunks of the state: q from tensor memory
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk)
                            umma_bf16_ts(d, tmem + C::Q_COL + kc * 32 + kk * 8,
                                         dk0 + (uint64_t)((kc * C::CHUNK + kk * 32) >> 4), idesc_s, (kc | kk) != 0);
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)  // rope chunk: q from shared memory
                        umma_bf16(d, dq0 + (uint64_t)((kk * 32) >> 4),
                                  dk0 + (uint64_t)((C::NV * C::CHUNK + kk * 32) >> 4), idesc_s, 1u);
                    umma_commit(&sfull_bar[sb]);
                    ++m_s;
                    return true;
                };
                for (int si = 0; si < nseg && ok; ++si) {
                    const int n = segs[si].t1 - segs[si].t0;
                    if (!mbar_wait_one(&qfull_bar, m_q & 1, &abort_sh, a.err, lim_ns)) break;
                    if (!mbar_wait_one(&qtm_bar, m_q & 1, &abort_sh, a.err, lim_ns)) break;
                    ++m_q;
                    tc_fence_after();
                    if (!issue_s(m_tile)) break;
                    if (n == 1) umma_commit(&qempty_bar);
                    for (int j = 0; j < n; ++j) {
                        if (j + 1 < n) {
                            if (!issue_s(m_tile + j + 1)) {
                                ok = false;
                                break;
                            }
                            if (j + 1 == n - 1) umma_commit(&qempty_bar);
                        }
                        const uint32_t pb = m_pv & 1;
                        if (!mbar_wait_one(&pfull_bar[pb], (m_pv >> 1) & 1, &abort_sh, a.err, lim_ns)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                        const uint32_t stage = (m_tile + j) % nstage;
                        const uint64_t dv0 = umma_desc(st0 + stage * C::STAGE + vc * C::NV * C::CHUNK, C::CHUNK, 1024, 2);
                        const uint32_t pa = tmem + C::S_COL + pb * TOK;  // P(j) over S(j)
#pragma unroll
                        for (int kk = 0; kk < TOK / 16; ++kk)
                            umma_bf16_ts(tmem, pa + kk * 8, dv0 + (uint64_t)(kk * 128), idesc_pv,
                                         (j > 0 || kk > 0) ? 1u : 0u);
                        umma_commit(&empty_bar[stage]);  // the stage is free and P.V j is done
                        ++m_pv;
                    }
                    m_tile += n;
                }
            }
            __syncwarp();
        } else if (warp >= 4) {
            // ================================================================ softmax / epilogue
            // Four warps, one thread per row: warp w reads TMEM lanes 32 (w % 4) .. + 31 and the
            // whole 64-token S row of its thread, so no row value crosses threads.  When a CTA has
            // at most 64 rows (GLA-2 at q_len 1: 64; GLA-8: 16 L) they are spread evenly over the
            // four lane quadrants, row_spread rows each (row n at lane 32 (n / row_spread) +
            // n % row_spread), so that each of the four warps, one per SM sub-partition, holds
            // a quarter of them.
            const int st_id = threadIdx.x - 128;         // 0 .. 127
            const int r = (warp & 3) * 32 + lane;        // TMEM lane
            const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
            const bool spread = a.row_spread != 0;
            const int n_row = spread ? ((lane < a.row_spread) ? (warp & 3) * a.row_spread + lane : R) : rt * 128 + r;
            const bool row_ok = n_row < R;
            const bool warp_live = spread || rt * 128 + (warp & 3) * 32 < R;  // some row of this warp is real
            const int i_row = row_ok ? n_row / g : 0;
            const int head = row_ok ? c * g + n_row % g : 0;
            bool ok = true;
            // wait until P.V number k has completed (O settled): the commit that frees tile k's
            // stage.  Every earlier P.V is complete by then (P(k) needed S(k), issued after P.V
            // k - 2), so the barrier is at most one phase short of the one waited for.
            auto wait_pv = [&](uint32_t k) -> bool {
                return mbar_wait_warp(&empty_bar[k % nstage], (k / nstage) & 1, &abort_sh, a.err, lim_ns);
            };
            for (int si = 0; si < nseg && ok; ++si) {
                const Seg sg = segs[si];
                const int b = sg.b;
                const int T = clamp_len(__ldg(a.seqlens + b), max_tokens, a.L, nullptr);
                // causal: row (i, h) sees t <= T - L + i; non-causal (prefix): every row sees all T
                const int lim = row_ok ? (a.noncausal ? T - 1 : T - a.L + i_row) : -1;
                const int lim_all = a.noncausal ? T - 1 : T - a.L;  // visible to every row
                {
                    // q's latent part of this segment's rows -> tensor memory (the A operand of
                    // the score product), once the previous segment's score MMAs are done with it
                    if (!mbar_wait_warp(&qempty_bar, (x_q & 1) ^ 1, &abort_sh, a.err, lim_ns)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint4 *src =
                        row_ok ? (const uint4 *)(a.q + ((size_t)(b * a.L + i_row) * a.h_q + head) * C::DQK) : nullptr;
#pragma unroll 1
                    for (int part16 = 0; part16 < KL * 2; ++part16) {
                        uint32_t w[16];
#pragma unroll
                        for (int k = 0; k < 4; ++k) {
                            const uint4 v = src ? __ldg(src + part16 * 4 + k) : make_uint4(0, 0, 0, 0);
                            w[4 * k] = v.x;
                            w[4 * k + 1] = v.y;
                            w[4 * k + 2] = v.z;
                            w[4 * k + 3] = v.w;
                        }
                        tmem_st16u(tmem + lane_base + C::Q_COL + part16 * 16, w);
                    }
                    tmem_st_wait();
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&qtm_bar);
                }
                ++x_q;
                // l: sum of the fp32 P (gives lse); lq: sum of the bf16-rounded P the product
                // uses (normalises O: a convex combination of the rounded weights).
                float m_ref = -INFINITY, l = 0.f, lq = 0.f;
                for (int tile = sg.t0; tile < sg.t1; ++tile) {
                    const int tok0 = tile * TOK;
                    const uint32_t sb = x_s & 1;
                    if (!mbar_wait_warp(&sfull_bar[sb], (x_s >> 1) & 1, &abort_sh, a.err, lim_ns)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    float s[TOK];
                    float mx = -INFINITY;
                    if (warp_live) {
#pragma unroll
                        for (int h = 0; h < TOK / 32; ++h) {
                            float t32[32];
                            tmem_ld32(tmem + lane_base + C::S_COL + sb * TOK + 32 * h, t32);
#pragma unroll
                            for (int k = 0; k < 32; ++k) s[32 * h + k] = t32[k];
                        }
                    }
                    ++x_s;
                    // no column masked; the same for every lane of the warp (rows past R are
                    // handled by forcing their maximum to -inf: their S is garbage, never used)
                    const bool full = tile * TOK + TOK - 1 <= lim_all;
                    if (warp_live) {
                        mx = tile_max(s, full, tok0, lim, a.scale_log2);
                        if (!row_ok) mx = -INFINITY;
                    }
                    float alpha = 1.f;
                    bool need = false;
                    if (mx != -INFINITY) {
                        if (m_ref == -INFINITY) {
                            m_ref = mx;  // nothing visible before: O and the sums hold zeros
                        } else if (mx > m_ref + RESCALE_LOG2) {
                            alpha = ex2(m_ref - mx);
                            need = true;
                            m_ref = mx;
                        }
                    }
                    if (__any_sync(0xffffffffu, need)) {
                        // O is settled once the previous P.V (and so every earlier one) is done
                        if (x_pv > 0 && !wait_pv(x_pv - 1)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                        l *= alpha;
                        lq *= alpha;
#pragma unroll 1
                        for (int ch = 0; ch < DV / 32; ++ch) {
                            float o[32];
                            tmem_ld32(tmem + lane_base + ch * 32, o);
#pragma unroll
                            for (int k = 0; k < 32; ++k) o[k] *= alpha;
                            tmem_st32(tmem + lane_base + ch * 32, o);
                        }
                        tmem_st_wait();
                    }
                    if (warp_live) l += tile_exp(s, full, tok0, lim, a.scale_log2, m_ref);

                    // tokens past T_b in this tile hold garbage: zero their value rows (P is 0 there,
                    // but 0 * NaN would still poison the product)
                    const uint32_t stage = x_tile % nstage;
                    const int ttok0 = tile * TOK;
                    if (ttok0 + TOK > T) {
                        const int k0 = max(T - ttok0, 0);
                        uint8_t *v0 = stage_s + (size_t)stage * C::STAGE + (size_t)vc * C::NV * C::CHUNK;
                        const int units = (TOK - k0) * C::NV * 8;  // 16-byte units: rows x chunks x 8
                        for (int u = st_id; u < units; u += 32 * NSMX) {
                            const int row = k0 + u / (C::NV * 8), ch = (u / 8) % C::NV, k = u & 7;
                            *(uint4 *)(v0 + ch * C::CHUNK + row * 128 + k * 16) = make_uint4(0, 0, 0, 0);
                        }
                    }
                    // P (bf16 pairs) over S in buffer x_pv & 1 (this thread has read its S row)
                    if (warp_live) {
                        const uint32_t pa = tmem + lane_base + C::S_COL + sb * TOK;
                        float sum = 0.f, sum2 = 0.f;
#pragma unroll
                        for (int h = 0; h < TOK / 32; ++h) {
                            uint32_t w[16];
#pragma unroll
                            for (int k = 0; k < 16; ++k) {
                                w[k] = pack_bf16(s[32 * h + 2 * k], s[32 * h + 2 * k + 1]);
                                sum += bf16_lo(w[k]);
                                sum2 += bf16_hi(w[k]);
                            }
                            tmem_st16u(pa + 16 * h, w);
                        }
                        tmem_st_wait();
                        lq += sum + sum2;
                    }
                    if (ttok0 + TOK > T) fence_proxy_async();  // the zeroed value rows above
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&pfull_bar[x_pv & 1]);
                    ++x_pv;
                    ++x_tile;
                }
                if (!ok) break;

                // ---- epilogue: O is final once the last P.V completes
                if (!wait_pv(x_pv - 1)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const float inv = lq > 0.f ? 1.f / lq : 0.f;
                const float lse_v = l > 0.f ? (m_ref + lg2(l)) * 0.69314718055994530942f : -INFINITY;
                const size_t rows_b = (size_t)a.L * a.h_q;
                const size_t r_out = (size_t)i_row * a.h_q + head;
                if (warp_live) {
#pragma unroll 1
                    for (int ch = 0; ch < DV / 32; ++ch) {
                        float o[32];
                        const int col = ch * 32;
                        tmem_ld32(tmem + lane_base + col, o);
                        if (!row_ok) continue;
                        if (sg.nsplit == 1) {
                            uint4 *op = (uint4 *)(a.out + ((size_t)b * rows_b + r_out) * DC + vc * DV + col);
#pragma unroll
                            for (int k = 0; k < 4; ++k)
                                op[k] = make_uint4(pack_bf16(o[8 * k] * inv, o[8 * k + 1] * inv),
                                                   pack_bf16(o[8 * k + 2] * inv, o[8 * k + 3] * inv),
                                                   pack_bf16(o[8 * k + 4] * inv, o[8 * k + 5] * inv),
                                                   pack_bf16(o[8 * k + 6] * inv, o[8 * k + 7] * inv));
                        } else {
                            float4 *op =
                                (float4 *)(a.ws_o + ((size_t)sg.slot * rows_b + r_out) * DC + vc * DV + col);
#pragma unroll
                            for (int k = 0; k < 8; ++k)
                                op[k] = make_float4(o[4 * k] * inv, o[4 * k + 1] * inv, o[4 * k + 2] * inv,
                                                    o[4 * k + 3] * inv);
                        }
                    }
                }
                if (row_ok && vc == 0) {
                    if (sg.nsplit == 1)
                        a.lse[(size_t)b * rows_b + r_out] = lse_v;
                    else
                        a.ws_lse[(size_t)sg.slot * rows_b + r_out] = lse_v;
                }
                tc_fence_before();
            }
        }
        __syncthreads();
        if (!more_sh || abort_sh) break;
        __syncthreads();
    }

    // every MMA issued by this CTA has completed before tensor memory is released
    if (warp == 1 && lane == 0) {
        volatile int never = 0;
        umma_commit(&end_bar);
        mbar_wait_one(&end_bar, 0, &never, nullptr, lim_ns);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem, 512);
}

template <int DC, int TOK, int KL>
cudaError_t launch_t(const CUtensorMap &qm, const CUtensorMap &lm, const CUtensorMap &rm, const LatentArgs &a,
                     int grid, size_t smem, cudaStream_t st) {
    auto k = latent_decode_kernel<DC, TOK, KL>;
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    k<<<grid, LTHREADS, smem, st>>>(qm, lm, rm, a);
    return cudaGetLastError();
}

}  // namespace

LatentShape latent_shape(int d_c) {
    LatentShape s{};
    if (d_c == 256) {
        s.tok = 64;
        s.q_bytes = LatCfg<256, 64, 4>::Q_BYTES;
        s.stage_bytes = LatCfg<256, 64, 4>::STAGE;
        s.p_bytes = 0;
    } else if (d_c == 512) {  // the CTA-pair kernel of latent_pair.cu
        s.tok = 64;
        s.q_bytes = mla_pair_fixed_smem();
        s.stage_bytes = mla_pair_stage_bytes();
        s.p_bytes = 0;
    }
    return s;
}

LatentShape tied_prefix_shape() {
    LatentShape s{};
    s.tok = 64;
    s.q_bytes = LatCfg<128, 64, 1>::Q_BYTES;
    s.stage_bytes = LatCfg<128, 64, 1>::STAGE;
    s.p_bytes = 0;
    return s;
}

cudaError_t launch_tied_prefix(const CUtensorMap &qm, const CUtensorMap &lm, const CUtensorMap &rm,
                               const LatentArgs &a, int grid, size_t smem, cudaStream_t st) {
    return launch_t<128, 64, 1>(qm, lm, rm, a, grid, smem, st);
}

}  // namespace kvd
