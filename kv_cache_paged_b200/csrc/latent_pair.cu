// MLA decode (absorbed, d_c = 512) on a pair of CTAs that split the key dimension.
//
// "Hardware-Efficient Attention for Fast Decoding", section 3.3.2 with h_c latent heads of
// width d_c = 512 (MLA: h_c = 1).  The fp32 accumulator of 128 query rows x 512 value
// columns alone fills tensor memory, so the value columns are split over two CTAs.  Rather
// than have both CTAs compute the same 128 x 576 score product, the pair (a thread-block
// cluster of 2) splits the 576-wide key dimension as well: CTA k holds q's latent dims
// [256k, 256k + 256) and rope dims [32k, 32k + 32),
// loads only those columns of each 64-token tile (36 KB), computes a partial score
// S_k = Q_k K_k^T on tcgen05 and swaps it with its peer through distributed shared memory.
// Both CTAs then hold the same S = S_0 + S_1 (fp32 addition commutes, so the sums agree bit
// for bit), run the same softmax and accumulate O for their own 256 latent columns, which are
// exactly the latent columns they loaded.  Every byte of the cache is read once per pair.
//
// Roles per CTA: warps 0..3 send (one per TMEM lane quadrant: write q's latent half into tensor
// memory at the start of each sequence, then per tile load this CTA's partial S and bulk-copy it
// into the peer's receive buffer, one 32-token half at a time), warps 4..7 softmax (one thread
// per row: it adds the peer's partial from the receive buffer to its own from tensor memory),
// warp 8 TMA producer, warp 9 MMA issuer (one thread); warps 10 and 11 exist to help warp 8
// gather tiles token by token with cp.async when pages do not hold whole tiles.
// Tensor memory: O [0, 256), two S buffers [256, 384) with P(j) written over S(j) as bf16 pairs,
// and q's latent half [384, 512) as the A operand of the score product.  Keeping q there leaves
// shared memory for four 36 KB KV stages next to the exchange buffers.  Every wait is bounded.
#include <cuda_bf16.h>

#include "common.cuh"
#include "kernels.h"

namespace kvd {

namespace {

constexpr int PMAXSEG = 32;
constexpr int PTOK = 64;                                  // tokens per tile
constexpr int PDV = 256;                                  // value columns per CTA
constexpr int P_DQK = 576;                                // q row: 512 latent + 64 rope
constexpr uint32_t P_QBYTES = 128 * 64;                  // q rope half: 128 rows x 64 B (shared memory)
constexpr uint32_t P_CHUNK = PTOK * 128;                  // one 64-dim chunk of a tile
constexpr uint32_t P_STAGE = 4 * P_CHUNK + PTOK * 64;     // latent half + rope half
constexpr uint32_t P_XHALF = 128 * 32 * 4;               // one 32-token half of a partial S tile (fp32)
constexpr uint32_t P_XBYTES = 4 * P_XHALF;                // send and receive buffers, one per half
constexpr int P_NSB = 2;                                  // S buffers (P is written over its S)
constexpr uint32_t P_SCOL = PDV;                          // S buffers [256, 384)
constexpr uint32_t P_QCOL = PDV + P_NSB * PTOK;           // q latent half [384, 512), bf16 pairs
constexpr int P_NSMX = 4;                                 // softmax warps, one thread per row
constexpr int W_PROD = 4 + P_NSMX, W_MMA = 5 + P_NSMX;
constexpr int P_NGATHER = 3;  // warps that copy gathered tiles: the producer and the last two
constexpr int P_THREADS = 32 * (6 + P_NSMX + P_NGATHER - 1);
constexpr float P_RESCALE_LOG2 = 8.f;

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(P_THREADS, 1)
    mla_pair_kernel(const __grid_constant__ CUtensorMap qmap, const __grid_constant__ CUtensorMap qrmap,
                    const __grid_constant__ CUtensorMap latmap, const __grid_constant__ CUtensorMap ropemap,
                    const LatentArgs a) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    __shared__ uint64_t full_bar[MAX_STAGES], empty_bar[MAX_STAGES];
    __shared__ uint64_t qfull_bar, qtm_bar, qempty_bar, pfull_bar[P_NSB], end_bar;
    __shared__ uint64_t sfull_bar[P_NSB], sread_bar[P_NSB];
    __shared__ uint64_t xfull_bar[2], xfree_bar[2];
    // teardown drain: psent_sh[w][h] = halves h the peer's send warp w copied into this CTA;
    // xseen_sh[h] = phases of xfull_bar[h] this CTA has seen complete
    __shared__ uint32_t psent_sh[4][2], xseen_sh[2];
    __shared__ Seg segs[PMAXSEG];
    __shared__ int nseg_sh, more_sh;
    __shared__ volatile int abort_sh;
    __shared__ uint32_t tmem_sh;

    uint8_t *smem = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    uint8_t *q_s = smem;
    uint8_t *send_s = smem + P_QBYTES;                      // this CTA's partial S, per half
    uint8_t *recv_s = send_s + 2 * P_XHALF;                 // the peer's partial S, per half
    uint8_t *stage_s = send_s + P_XBYTES;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t kr = cluster_rank();                     // 0 or 1: which half of the key
    const uint32_t peer = kr ^ 1u;
    const int pair = blockIdx.x >> 1;
    const int part = pair / a.n_sub, sub = pair % a.n_sub;
    const int rt = sub % a.n_rt;
    const int c = sub / a.n_rt;
    const int g = a.h_q / a.h_c;
    const int R = g * a.L;
    const int max_tokens = a.max_pages * a.page_size;
    const int nstage = a.nstage;
    const uint64_t lim_ns = a.wait_limit_ns;

    if (threadIdx.x == 0) {
        for (int s = 0; s < nstage; ++s) {
            mbar_init(&full_bar[s], a.gather ? 32 * P_NGATHER : 1);  // gathered: one arrival per gather lane
            mbar_init(&empty_bar[s], 1);
        }
        mbar_init(&qfull_bar, 1);   // q rope half (TMA)
        mbar_init(&qtm_bar, 4);     // q latent half written into tensor memory by the send warps
        mbar_init(&qempty_bar, 1);
        for (int s = 0; s < 2; ++s) {
            mbar_init(&pfull_bar[s], P_NSMX);
        }
        for (int s = 0; s < P_NSB; ++s) {
            mbar_init(&sfull_bar[s], 1);    // partial S computed (MMA commit)
            mbar_init(&sread_bar[s], 4);    // partial S read by the send warps (P may overwrite it)
        }
        mbar_init(&end_bar, 1);
        // per 32-token half h of a tile: xfull[h] takes one local arrival that arms the expected
        // bytes and is completed by the peer's bulk copies (16 KB); xfree[h] takes one arrival
        // from each of the peer's softmax warps
        for (int h = 0; h < 2; ++h) {
            mbar_init(&xfull_bar[h], 1);
            mbar_init(&xfree_bar[h], P_NSMX);
            mbar_arrive_expect_tx(&xfull_bar[h], P_XHALF);  // armed for the first tile
        }
        abort_sh = 0;
        for (int k = 0; k < 8; ++k) psent_sh[k / 2][k % 2] = 0;
        xseen_sh[0] = xseen_sh[1] = 0;
        fence_mbar_init();
    }
    if (warp == W_MMA) tmem_alloc(&tmem_sh, 512);
    if (warp == W_PROD && lane == 0) {
        tma_prefetch_desc(&qrmap);
        if (!a.gather) {
            tma_prefetch_desc(&latmap);
            tma_prefetch_desc(&ropemap);
        }
    }
    pdl_launch_dependents();
    tc_fence_before();
    cluster_sync();  // both CTAs' barriers are initialised before any remote arrival
    tc_fence_after();
    const uint32_t tmem = tmem_sh;

    uint32_t p_issued = 0, p_qloads = 0;
    uint32_t m_tile = 0, m_q = 0;
    uint32_t x_tile = 0, x_s = 0, x_pv = 0;            // softmax
    uint32_t e_t = 0, e_q = 0;                          // send
    uint32_t sent[2] = {0, 0};                          // send: halves copied to the peer

    for (int skip = 0;; skip += PMAXSEG) {
        if (warp == W_PROD) {
            int cnt = 0;
            plan_walk(a.seqlens, a.B, PTOK, a.seg_cost, max_tokens, a.L, part, a.parts, a.err, [&](const Seg &s) {
                if (cnt >= skip && cnt < skip + PMAXSEG) segs[cnt - skip] = s;
                ++cnt;
            });
            if (lane == 0) {
                nseg_sh = cnt - skip < PMAXSEG ? (cnt - skip > 0 ? cnt - skip : 0) : PMAXSEG;
                more_sh = cnt > skip + PMAXSEG;
            }
        }
        __syncthreads();
        const int nseg = nseg_sh;

        if (warp == W_PROD || (a.gather && warp > W_MMA)) {
            // ================================================================ producer(s)
            // W_PROD: q's rope half per segment and the KV tiles; with gathered tiles the warps
            // after W_MMA copy their share of every tile too
            const int gw = warp == W_PROD ? 0 : warp - W_MMA;
            const uint64_t pol = policy_evict_first();
            bool stop = false;
            const int rb = g < 128 ? g : 128;
            const int rows_tile = min(R - rt * 128, 128);
            for (int si = 0; si < nseg && !stop; ++si) {
                const Seg sg = segs[si];
                if (warp == W_PROD && !mbar_wait_warp(&qempty_bar, (p_qloads & 1) ^ 1, &abort_sh, a.err, lim_ns)) {
                    stop = true;
                    break;
                }
                if (warp == W_PROD && lane == 0) {
                    mbar_arrive_expect_tx(&qfull_bar, (uint32_t)rows_tile * 64);
                    for (int run = 0; run * rb < rows_tile; ++run) {
                        const int n0 = rt * 128 + run * rb;
                        const int i = n0 / g, h0 = n0 % g;
                        const int row = (sg.b * a.L + i) * a.h_q + c * g + h0;
                        tma_load_3d(q_s + run * rb * 64, &qrmap, &qfull_bar, 0, row, 16 + kr, pol);
                    }
                }
                if (warp == W_PROD) ++p_qloads;
                const int32_t *bt = a.block_table + (size_t)sg.b * a.max_pages;
                if (a.gather) {
                    // Pages smaller than the tile or not a multiple of it: as the GLA kernel's
                    // gather (P_NGATHER warps split the tile's tokens), but only this CTA's latent
                    // half (dims 256 kr ..) and rope half (dims 32 kr .., 64-byte rows).
                    const int T = clamp_len(__ldg(a.seqlens + sg.b), max_tokens, a.L, nullptr);
                    const __nv_bfloat16 *lat = (const __nv_bfloat16 *)a.cache0 + (size_t)c * 512 + kr * PDV;
                    const __nv_bfloat16 *rope = (const __nv_bfloat16 *)a.cache1 + kr * 32;
                    const int nk = (PTOK - gw + P_NGATHER - 1) / P_NGATHER;
                    auto tok_of = [&](int t) { return min(t * PTOK + gw + P_NGATHER * lane, T - 1); };
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
                            const uint32_t st = smem_u32(stage_s + (size_t)stage * P_STAGE);
                            gather_tile<4, 4>(st, P_CHUNK, lat, (size_t)a.h_c * 512, rope, 64, st + 4 * P_CHUNK,
                                              myrow, gw, P_NGATHER, nk, lane, pol);
                            cp_async_arrive(&full_bar[stage]);
                        }
                        ++p_issued;
                    }
                    continue;
                }
                const int tpp = a.page_size / PTOK;
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
                            uint8_t *st = stage_s + (size_t)stage * P_STAGE;
                            const int row = pg * a.page_size + (t % tpp) * PTOK;
                            mbar_arrive_expect_tx(&full_bar[stage], P_STAGE);
                            if (!(a.debug_flags & DEBUG_SKIP_FIRST_LOAD) || p_issued != 0) {
                                tma_load_3d(st, &latmap, &full_bar[stage], 0, row, c * 8 + 4 * kr, pol);
                                tma_load_2d(st + 4 * P_CHUNK, &ropemap, &full_bar[stage], 32 * kr, row, pol);
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
        } else if (warp == W_MMA) {
            // ================================================================ MMA issuer
            if (lane == 0) {
                constexpr uint32_t idesc_s = umma_idesc_bf16(128, PTOK, false, false);
                constexpr uint32_t idesc_pv = umma_idesc_bf16(128, PDV, false, true);
                const uint32_t st0 = smem_u32(stage_s);
                const uint64_t dqr = umma_desc(smem_u32(q_s), 16, 512, 4);  // rope half, 64 B swizzle
                bool ok = true;
                // S(j) goes into buffer j % 2, where P(j - 2) was: the MMAs of one thread run in
                // issue order, so the score product of tile j, issued after the P.V product of
                // tile j - 2, cannot overwrite that P before it is read
                auto issue_s = [&](uint32_t gt) -> bool {
                    const uint32_t stage = gt % nstage;
                    if (!mbar_wait_one(&full_bar[stage], (gt / nstage) & 1, &abort_sh, a.err, lim_ns)) return false;
                    tc_fence_after();
                    // gathered rows were written by cp.async (the generic proxy); the tensor core reads
                    // them through the async proxy, so order the two before the MMAs
                    if (a.gather) fence_proxy_async();
                    const uint32_t d = tmem + P_SCOL + (gt % P_NSB) * PTOK;
                    const uint64_t dk0 = umma_desc(st0 + stage * P_STAGE, 16, 1024, 2);
                    const uint64_t dkr = umma_desc(st0 + stage * P_STAGE + 4 * P_CHUNK, 16, 512, 4);
#pragma unroll
                    for (int ch = 0; ch < 4; ++ch)
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk)
                            umma_bf16_ts(d, tmem + P_QCOL + ch * 32 + kk * 8,
                                         dk0 + (uint64_t)((ch * P_CHUNK + kk * 32) >> 4), idesc_s, (ch | kk) != 0);
#pragma unroll
                    for (int kk = 0; kk < 2; ++kk)
                        umma_bf16(d, dqr + (uint64_t)(kk * 2), dkr + (uint64_t)(kk * 2), idesc_s, 1u);
                    umma_commit(&sfull_bar[gt % P_NSB]);
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
                            if (j + 1 == n - 1) umma_commit(&qempty_bar);  // q is free once these finish
                        }
                        const uint32_t pb = (m_tile + j) % P_NSB;
                        if (!mbar_wait_one(&pfull_bar[pb], ((m_tile + j) / P_NSB) & 1, &abort_sh, a.err, lim_ns)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                        const uint32_t stage = (m_tile + j) % nstage;
                        const uint64_t dv0 = umma_desc(st0 + stage * P_STAGE, P_CHUNK, 1024, 2);
                        const uint32_t pa = tmem + P_SCOL + pb * PTOK;
#pragma unroll
                        for (int kk = 0; kk < PTOK / 16; ++kk)
                            umma_bf16_ts(tmem, pa + kk * 8, dv0 + (uint64_t)(kk * 128), idesc_pv,
                                         (j > 0 || kk > 0) ? 1u : 0u);
                        umma_commit(&empty_bar[stage]);
                    }
                    m_tile += n;
                }
            }
            __syncwarp();
        } else if (warp < 4) {
            // ================================================================ send
            // thread = row.  Each 32-token half of the row's partial S is staged in this CTA's
            // send buffer (16-byte chunks XOR-swizzled by row), then one bulk copy per warp and
            // half moves the warp's 32 rows (4 KB) into the peer's receive buffer.
            const int r = warp * 32 + lane;
            const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
            const uint32_t peer_recv = mapa_shared(smem_u32(recv_s), peer);
            const uint32_t peer_xfull[2] = {mapa_shared(smem_u32(&xfull_bar[0]), peer),
                                            mapa_shared(smem_u32(&xfull_bar[1]), peer)};
            const int n_row = rt * 128 + r;
            bool ok = true;
            for (int si = 0; si < nseg && ok; ++si) {
                const int n = segs[si].t1 - segs[si].t0;
                // q's latent half for this segment's rows goes into tensor memory (the A operand
                // of the score product) once the previous segment's score MMAs are done with it
                if (!mbar_wait_warp(&qempty_bar, (e_q & 1) ^ 1, &abort_sh, a.err, lim_ns)) break;
                ++e_q;
                tc_fence_after();
                {
                    const uint4 *src = nullptr;
                    if (n_row < R) {
                        const int i = n_row / g, h = n_row % g;
                        src = (const uint4 *)(a.q + ((size_t)(segs[si].b * a.L + i) * a.h_q + c * g + h) * P_DQK +
                                              kr * PDV);
                    }
#pragma unroll 1
                    for (int part16 = 0; part16 < 8; ++part16) {
                        uint32_t w[16];
#pragma unroll
                        for (int k = 0; k < 4; ++k) {
                            const uint4 v = src ? __ldg(src + part16 * 4 + k) : make_uint4(0, 0, 0, 0);
                            w[4 * k] = v.x;
                            w[4 * k + 1] = v.y;
                            w[4 * k + 2] = v.z;
                            w[4 * k + 3] = v.w;
                        }
                        tmem_st16u(tmem + lane_base + P_QCOL + part16 * 16, w);
                    }
                    tmem_st_wait();
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&qtm_bar);
                for (int j = 0; j < n && ok; ++j, ++e_t) {
                    const uint32_t sb = e_t % P_NSB;
                    if (!mbar_wait_warp(&sfull_bar[sb], (e_t / P_NSB) & 1, &abort_sh, a.err, lim_ns)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t sa = tmem + lane_base + P_SCOL + sb * PTOK;
                    float sp[2][32];
                    tmem_ld32(sa, sp[0]);
                    tmem_ld32(sa + 32, sp[1]);
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&sread_bar[sb]);
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        // the peer has read the previous tile's half h, so both this CTA's send
                        // buffer (the copy's source) and the peer's receive buffer are free
                        if (e_t > 0 &&
                            !mbar_wait_warp_cluster(&xfree_bar[h], (e_t - 1) & 1, &abort_sh, a.err, lim_ns)) {
                            ok = false;
                            break;
                        }
                        const uint32_t row = smem_u32(send_s + h * P_XHALF) + r * 128;
#pragma unroll
                        for (int c8 = 0; c8 < 8; ++c8)
                            asm volatile("st.shared.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(row + ((c8 ^ (r & 7)) << 4)),
                                         "f"(sp[h][4 * c8]), "f"(sp[h][4 * c8 + 1]), "f"(sp[h][4 * c8 + 2]),
                                         "f"(sp[h][4 * c8 + 3])
                                         : "memory");
                        fence_proxy_async();
                        __syncwarp();
                        if (lane == 0)
                            bulk_copy_to_peer(peer_recv + h * P_XHALF + warp * 4096,
                                              smem_u32(send_s + h * P_XHALF) + warp * 4096, 4096, peer_xfull[h]);
                        ++sent[h];
                    }
                }
            }
        } else if (warp >= 4 && warp < 4 + P_NSMX) {
            // ================================================================ softmax / epilogue
            // One thread per row (TMEM lane): the whole 64-token S row, so no row value crosses
            // threads.  The peer's partial arrives in two 32-token halves.
            const int st_id = threadIdx.x - 128;
            const int r = (warp & 3) * 32 + lane;
            const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
            const int n_row = rt * 128 + r;
            const bool row_ok = n_row < R;
            const bool warp_live = rt * 128 + (warp & 3) * 32 < R;
            const uint32_t peer_xfree[2] = {mapa_shared(smem_u32(&xfree_bar[0]), peer),
                                            mapa_shared(smem_u32(&xfree_bar[1]), peer)};
            const int i_row = row_ok ? n_row / g : 0;
            const int head = row_ok ? c * g + n_row % g : 0;
            bool ok = true;
            // P.V number k has completed (O settled): the commit that frees tile k's stage.  Every
            // earlier P.V is complete by then (P(k) needed S(k), issued after P.V k - 2), so the
            // barrier is at most one phase short of the one waited for.
            auto wait_pv = [&](uint32_t k) -> bool {
                return mbar_wait_warp(&empty_bar[k % nstage], (k / nstage) & 1, &abort_sh, a.err, lim_ns);
            };
            for (int si = 0; si < nseg && ok; ++si) {
                const Seg sg = segs[si];
                const int b = sg.b;
                const int T = clamp_len(__ldg(a.seqlens + b), max_tokens, a.L, nullptr);
                const int lim = row_ok ? T - a.L + i_row : -1;
                float m_ref = -INFINITY, l = 0.f, lq = 0.f;
                for (int tile = sg.t0; tile < sg.t1; ++tile) {
                    const int tok0 = tile * PTOK;
                    const uint32_t sb = x_s % P_NSB;
                    if (!mbar_wait_warp(&sfull_bar[sb], (x_s / P_NSB) & 1, &abort_sh, a.err, lim_ns)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    float s[PTOK];
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        float t32[32];
                        tmem_ld32(tmem + lane_base + P_SCOL + sb * PTOK + 32 * h, t32);
#pragma unroll
                        for (int k = 0; k < 32; ++k) s[32 * h + k] = t32[k];
                    }
                    // S = own partial + the peer's (the peer adds in the opposite order; fp32
                    // addition commutes, so both CTAs see the same S bit for bit)
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        if (!mbar_wait_warp_cluster(&xfull_bar[h], x_s & 1, &abort_sh, a.err, lim_ns)) {
                            ok = false;
                            break;
                        }
                        // the phase is complete: arm the next tile's before any warp frees the buffer
                        if (threadIdx.x == 128) {
                            mbar_arrive_expect_tx(&xfull_bar[h], P_XHALF);
                            *(volatile uint32_t *)&xseen_sh[h] = x_s + 1;
                        }
                        const uint32_t row = smem_u32(recv_s + h * P_XHALF) + r * 128;
#pragma unroll
                        for (int c8 = 0; c8 < 8; ++c8) {
                            float4 v;
                            asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];"
                                         : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
                                         : "r"(row + ((c8 ^ (r & 7)) << 4))
                                         : "memory");
                            s[32 * h + 4 * c8] += v.x;
                            s[32 * h + 4 * c8 + 1] += v.y;
                            s[32 * h + 4 * c8 + 2] += v.z;
                            s[32 * h + 4 * c8 + 3] += v.w;
                        }
                        __syncwarp();
                        if (lane == 0) mbar_arrive_cluster(peer_xfree[h]);
                    }
                    if (!ok) break;
                    ++x_s;

                    float mx = -INFINITY;
                    // no column masked; the same for every lane of the warp (rows past R: -inf)
                    const bool full = tile * PTOK + PTOK - 1 <= T - a.L;
                    if (warp_live) {
                        mx = tile_max(s, full, tok0, lim, a.scale_log2);
                        if (!row_ok) mx = -INFINITY;
                    }
                    float alpha = 1.f;
                    bool need = false;
                    if (mx != -INFINITY) {
                        if (m_ref == -INFINITY) {
                            m_ref = mx;
                        } else if (mx > m_ref + P_RESCALE_LOG2) {
                            alpha = ex2(m_ref - mx);
                            need = true;
                            m_ref = mx;
                        }
                    }
                    if (__any_sync(0xffffffffu, need)) {
                        if (x_pv > 0 && !wait_pv(x_pv - 1)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                        l *= alpha;
                        lq *= alpha;
#pragma unroll 1
                        for (int ch = 0; ch < PDV / 32; ++ch) {
                            float o[32];
                            tmem_ld32(tmem + lane_base + ch * 32, o);
#pragma unroll
                            for (int k = 0; k < 32; ++k) o[k] *= alpha;
                            tmem_st32(tmem + lane_base + ch * 32, o);
                        }
                        tmem_st_wait();
                    }
                    if (warp_live) l += tile_exp(s, full, tok0, lim, a.scale_log2, m_ref);
                    // value rows of tokens past T_b hold garbage: zero them (0 * NaN would poison O)
                    const uint32_t stage = x_tile % nstage;
                    const int ttok0 = tile * PTOK;
                    if (ttok0 + PTOK > T) {
                        const int k0 = max(T - ttok0, 0);
                        uint8_t *v0 = stage_s + (size_t)stage * P_STAGE;
                        const int units = (PTOK - k0) * 4 * 8;
                        for (int u = st_id; u < units; u += 32 * P_NSMX) {
                            const int row = k0 + u / 32, ch = (u / 8) & 3, k = u & 7;
                            *(uint4 *)(v0 + ch * P_CHUNK + row * 128 + k * 16) = make_uint4(0, 0, 0, 0);
                        }
                    }
                    // P(j) is written over S(j): the send warps must have read it too
                    if (!mbar_wait_warp(&sread_bar[sb], (x_pv / P_NSB) & 1, &abort_sh, a.err, lim_ns)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    if (warp_live) {
                        const uint32_t pa = tmem + lane_base + P_SCOL + sb * PTOK;
                        float sum = 0.f, sum2 = 0.f;
#pragma unroll
                        for (int h = 0; h < 2; ++h) {
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
                    if (ttok0 + PTOK > T) fence_proxy_async();
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&pfull_bar[x_pv & 1]);
                    ++x_pv;
                    ++x_tile;
                }
                if (!ok) break;

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
                    for (int ch = 0; ch < PDV / 32; ++ch) {
                        float o[32];
                        const int col = ch * 32;
                        tmem_ld32(tmem + lane_base + col, o);
                        if (!row_ok) continue;
                        const int gcol = kr * PDV + col;
                        if (sg.nsplit == 1) {
                            uint4 *op = (uint4 *)(a.out + ((size_t)b * rows_b + r_out) * 512 + gcol);
#pragma unroll
                            for (int k = 0; k < 4; ++k)
                                op[k] = make_uint4(pack_bf16(o[8 * k] * inv, o[8 * k + 1] * inv),
                                                   pack_bf16(o[8 * k + 2] * inv, o[8 * k + 3] * inv),
                                                   pack_bf16(o[8 * k + 4] * inv, o[8 * k + 5] * inv),
                                                   pack_bf16(o[8 * k + 6] * inv, o[8 * k + 7] * inv));
                        } else {
                            float4 *op = (float4 *)(a.ws_o + ((size_t)sg.slot * rows_b + r_out) * 512 + gcol);
#pragma unroll
                            for (int k = 0; k < 8; ++k)
                                op[k] = make_float4(o[4 * k] * inv, o[4 * k + 1] * inv, o[4 * k + 2] * inv,
                                                    o[4 * k + 3] * inv);
                        }
                    }
                }
                if (row_ok && kr == 0) {
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

    if (warp == W_MMA && lane == 0) {
        volatile int never = 0;
        umma_commit(&end_bar);
        mbar_wait_one(&end_bar, 0, &never, nullptr, lim_ns);
    }
    // Teardown.  A CTA that gave up early (a wait ran out) may still have one of the peer's bulk
    // copies landing in its receive buffer: the peer copies a tile's half only after this CTA
    // freed the previous tile's, so at most the half of tile xseen_sh[h] can be in flight, from
    // the send warps whose count passes it.  Each send warp tells the peer how many halves it
    // copied; the receiver completes the bytes of the copies that were never issued and waits
    // (bounded) for the issued ones, and only then may either CTA exit.
    if (warp < 4 && lane == 0)
        for (int h = 0; h < 2; ++h)
            asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(mapa_shared(smem_u32(&psent_sh[warp][h]), peer)),
                         "r"(sent[h])
                         : "memory");
    tc_fence_before();
    __syncthreads();
    cluster_sync();  // the peer's send counts are visible; nobody sends any more
    if (threadIdx.x == 0) {
        volatile int never = 0;
        for (int h = 0; h < 2; ++h) {
            const uint32_t f = xseen_sh[h];
            uint32_t n = 0;
            for (int w = 0; w < 4; ++w) n += psent_sh[w][h] > f ? 1u : 0u;
            if (n > 0) {
                if (n < 4) mbar_complete_tx(&xfull_bar[h], (4 - n) * 4096);
                mbar_wait_one(&xfull_bar[h], f & 1, &never, nullptr, lim_ns);
            }
        }
    }
    __syncthreads();
    cluster_sync();  // every copy into either CTA's shared memory has landed
    tc_fence_after();
    if (warp == W_MMA) tmem_dealloc(tmem, 512);
}

}  // namespace

uint32_t mla_pair_fixed_smem() { return P_QBYTES + P_XBYTES; }
uint32_t mla_pair_stage_bytes() { return P_STAGE; }

cudaError_t launch_mla_pair(const CUtensorMap &qm, const CUtensorMap &qrm, const CUtensorMap &lm,
                            const CUtensorMap &rm, const LatentArgs &a, int grid, size_t smem, cudaStream_t st) {
    cudaError_t e = cudaFuncSetAttribute(mla_pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    mla_pair_kernel<<<grid, P_THREADS, smem, st>>>(qm, qrm, lm, rm, a);
    return cudaGetLastError();
}

}  // namespace kvd
