// GLA decode (absorbed form) for latent heads attended by at most 64 query rows: GLA-2 at
// q_len 1 (64 heads per latent head), GLA-8 up to q_len 4 (16 heads per latent head).
//
// "Hardware-Efficient Attention for Fast Decoding", section 3.3.2: h_c latent heads of
// width d_c = 256 plus one shared RoPE key of width 64; query head h attends latent head
// c = h / (h_q / h_c) with key [latent_c ++ rope] and value latent_c.  With at most 64 rows
// per latent head the step sits at ~h_q FLOPs per byte (GLA-2), below the ridge: the kernel
// is built to stream the cache at the HBM rate with the tensor work hidden under it.
//
// Tensor-core shape.  A 128-row MMA would be half padding, and an M = 64 MMA occupies the
// tensor pipe as long as an M = 128 one, so the rows are not what to spend it on: what costs
// is the number of score MMAs per token, set by N (tokens per tile).  The tile is TOK tokens
// (96: three stages fit next to q), the score product S = Q K^T is M = 64 (rows), N = TOK,
// K = 320 (20 MMAs, both operands in shared memory), and O += P V is M = 64, N = 256,
// K = TOK (P read from tensor memory, V MN-major straight from the latent tile).  An M = 64
// accumulator fills TMEM lanes 0-15 of each 32-lane quadrant: O takes columns [0, 256) and
// the two S/P buffers the TOK columns each after it.
//
// One CTA owns one contiguous part of the (sequence, TOK-token tile) stream and one latent
// head.  Roles:
//   warps 0,2,3 producers: per tile the latent and rope rows of each page box by TMA (128 B
//               swizzle) into an NSTAGE ring, boxes spread over the three warps; block-table
//               entries one lane per box.  Pages that are not whole boxes are gathered token by
//               token with cp.async by five warps (0, 2, 3, 8, 9: the gather instantiation of
//               the kernel has 320 threads).
//   warp 1      MMA issuer (one thread).
//   warps 4..7  softmax, two threads per row (lanes l and l + 16 of the quadrant's warp take
//               the first and second half of the row's TOK scores through the half-warp
//               split TMEM shape), fp32 online softmax in base 2 with a lazy rescale of O;
//               they also copy each segment's q rows into shared memory with cp.async (the
//               next segment's as soon as the current one's last score product is done) and
//               write the epilogue.
// Rows: at most 16 per quadrant, row n of the latent head at quadrant n / rq, slot n % rq
// (rq = ceil(R / 4)), i.e. MMA row 16 (n / rq) + n % rq and TMEM lane 32 (n / rq) + n % rq.
#include <cuda_bf16.h>

#include "common.cuh"
#include "kernels.h"

namespace kvd {

namespace {

constexpr int NARROW_TOK = 96;  // tokens per tile
constexpr int NMAXSEG = 32;
constexpr int NSMX = 4;     // softmax warps
// GW producer warps: 0, 2, 3 and, for gathered tiles, 8 .. GW + 4 (warps 4-7 are the softmax
// warps: their lane quadrant is warp % 4)
constexpr int BOX_WARPS = 3;
constexpr int GATHER_WARPS = 5;
template <int GW>
constexpr int narrow_threads() { return 32 * (4 + NSMX + GW - 3); }
constexpr float RESCALE_LOG2 = 8.f;
constexpr int PF = 2;       // tiles ahead of the load that the producer prefetches into L2

template <int TOK>
struct NarrowCfg {
    static constexpr int DC = 256;                    // latent width (value columns)
    static constexpr int NV = DC / 64;                // 64-wide latent chunks
    static constexpr int KCH = NV + 1;                // key chunks: latent, then rope
    static constexpr int DQK = DC + 64;               // q row: latent part, then rope
    static constexpr uint32_t QCHUNK = 64 * 128;      // one 64-dim chunk of q (64 MMA rows)
    static constexpr uint32_t Q_BYTES = KCH * QCHUNK; // 40 KB
    static constexpr uint32_t CHUNK = TOK * 128;      // one 64-dim chunk of a tile
    static constexpr uint32_t STAGE = KCH * CHUNK;
    static constexpr int NSTAGE = TOK == 96 ? 3 : 2;
    static constexpr uint32_t SMEM = 1024 + Q_BYTES + NSTAGE * STAGE;
    static constexpr int NS = TOK / 2;                // scores of a row held by one thread
    static constexpr uint32_t S_COL = DC;             // S/P buffers after O (columns [0, DC))
    static constexpr uint32_t TMEM_COLS = 512;
    static_assert(TOK % 32 == 0 && S_COL + 2 * TOK <= TMEM_COLS, "two S buffers next to O");
    static_assert(SMEM <= 226 * 1024, "shared memory");
};

// Scores of this thread's half row: NS consecutive columns from col (lanes 0-15) and from
// col + NS (lanes 16-31) of the 16 TMEM lanes at taddr.
template <int NS>
__device__ __forceinline__ void load_half_row(uint32_t taddr, float (&s)[NS]) {
    if constexpr (NS == 48) {
        uint32_t a[32], b[16];
        tmem_ld16x2_32_nw<48>(taddr, a);
        tmem_ld16x2_16_nw<48>(taddr + 32, b);
        tmem_ld_wait();
#pragma unroll
        for (int k = 0; k < 32; ++k) s[k] = __uint_as_float(a[k]);
#pragma unroll
        for (int k = 0; k < 16; ++k) s[32 + k] = __uint_as_float(b[k]);
    } else {
        static_assert(NS == 64, "half rows of 48 or 64 scores");
        uint32_t a[32], b[32];
        tmem_ld16x2_32_nw<64>(taddr, a);
        tmem_ld16x2_32_nw<64>(taddr + 32, b);
        tmem_ld_wait();
#pragma unroll
        for (int k = 0; k < 32; ++k) {
            s[k] = __uint_as_float(a[k]);
            s[32 + k] = __uint_as_float(b[k]);
        }
    }
}

// This thread's NS / 2 packed bf16 pairs of P over its half of the S buffer at taddr
// (lanes 0-15: packed columns [0, NS / 2), lanes 16-31: [NS / 2, NS)).
template <int NS>
__device__ __forceinline__ void store_half_row(uint32_t taddr, const uint32_t (&w)[NS / 2]) {
    if constexpr (NS == 48) {
        uint32_t a[16], b[8];
#pragma unroll
        for (int k = 0; k < 16; ++k) a[k] = w[k];
#pragma unroll
        for (int k = 0; k < 8; ++k) b[k] = w[16 + k];
        tmem_st16x2_16u<24>(taddr, a);
        tmem_st16x2_8u<24>(taddr + 16, b);
    } else {
        uint32_t a[16], b[16];
#pragma unroll
        for (int k = 0; k < 16; ++k) {
            a[k] = w[k];
            b[k] = w[16 + k];
        }
        tmem_st16x2_16u<32>(taddr, a);
        tmem_st16x2_16u<32>(taddr + 16, b);
    }
}

template <int TOK, int GW>
__global__ void __launch_bounds__(narrow_threads<GW>(), 1)
    gla_narrow_kernel(const __grid_constant__ CUtensorMap latmap, const __grid_constant__ CUtensorMap ropemap,
                      const LatentArgs a) {
    using C = NarrowCfg<TOK>;
    constexpr int NST = C::NSTAGE;
    constexpr int NS = C::NS;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    __shared__ uint64_t full_bar[NST], empty_bar[NST];
    __shared__ uint64_t qfull_bar, sfull_bar[2], pfull_bar[2], end_bar;
    __shared__ Seg segs[NMAXSEG];
    __shared__ int nseg_sh, more_sh;
    __shared__ volatile int abort_sh;
    __shared__ uint32_t tmem_sh;

    uint8_t *smem = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    uint8_t *q_s = smem;
    uint8_t *stage_s = smem + C::Q_BYTES;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int part = blockIdx.x / a.h_c, c = blockIdx.x % a.h_c;
    const int g = a.h_q / a.h_c;
    const int R = g * a.L;
    const int rq = a.row_spread;  // rows per lane quadrant, 4 rq >= R, rq <= 16
    const int max_tokens = a.max_pages * a.page_size;
    const uint64_t lim_ns = a.wait_limit_ns;

    if (threadIdx.x == 0) {
        for (int s = 0; s < NST; ++s) {
            mbar_init(&full_bar[s], a.gather ? 32 * GW : 1);  // gathered: one arrival per gather lane
            mbar_init(&empty_bar[s], 1);
        }
        mbar_init(&qfull_bar, 32 * NSMX);  // one cp.async arrival per softmax thread
        for (int s = 0; s < 2; ++s) {
            mbar_init(&sfull_bar[s], 1);
            mbar_init(&pfull_bar[s], NSMX);  // one arrival per softmax warp
        }
        mbar_init(&end_bar, 1);
        abort_sh = 0;
        fence_mbar_init();
    }
    if (warp == 1) tmem_alloc(&tmem_sh, C::TMEM_COLS);
    if (warp == 0 && lane == 0 && !a.gather) {
        tma_prefetch_desc(&latmap);
        tma_prefetch_desc(&ropemap);
    }
    pdl_launch_dependents();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tmem_sh;

    // counters that persist across segment-list rounds
    uint32_t p_issued = 0;                          // producer
    uint32_t m_tile = 0, m_s = 0, m_pv = 0, m_q = 0;  // MMA issuer
    uint32_t x_tile = 0, x_s = 0, x_pv = 0;         // softmax

    // softmax thread geometry: quadrant qd, half of the row's scores, row slot in the quadrant
    const int qd = warp & 3;
    const int half = lane >> 4, rl = lane & 15;
    const bool smx_warp = warp >= 4 && warp < 8;
    const int n_row = (smx_warp && rl < rq) ? qd * rq + rl : R;
    const bool row_ok = n_row < R;
    const bool warp_live = qd * rq < R;  // some row of this warp is real
    const int i_row = row_ok ? n_row / g : 0;
    const int head = row_ok ? c * g + n_row % g : 0;
    const uint32_t s_lanes = (uint32_t)(qd * 32) << 16;  // rows: lanes 0-15 of the quadrant

    // q rows of sequence b into shared memory (MMA row 16 qd + rl), this thread's half of the
    // row's 40 16-byte units; every softmax thread arrives on qfull once its copies landed
    const uint64_t q_pol = smx_warp ? policy_evict_first() : 0;
    auto load_q = [&](int b) {
        if (row_ok) {
            const __nv_bfloat16 *src = a.q + ((size_t)(b * a.L + i_row) * a.h_q + head) * C::DQK;
            const uint32_t dst = smem_u32(q_s);
            const uint32_t m = (uint32_t)(16 * qd + rl);
#pragma unroll 4
            for (int u = 20 * half; u < 20 * half + 20; ++u)
                cp_async16(dst + (uint32_t)(u >> 3) * C::QCHUNK + sw128(m, (uint32_t)(u & 7)), src + u * 8, q_pol);
        }
        cp_async_arrive(&qfull_bar);
    };

    for (int skip = 0;; skip += NMAXSEG) {
        if (warp == 0) {
            int cnt = 0;
            plan_walk(a.seqlens, a.B, TOK, a.seg_cost, max_tokens, a.L, part, a.parts, a.err, [&](const Seg &s) {
                if (cnt >= skip && cnt < skip + NMAXSEG) segs[cnt - skip] = s;
                ++cnt;
            });
            if (lane == 0) {
                nseg_sh = cnt - skip < NMAXSEG ? (cnt - skip > 0 ? cnt - skip : 0) : NMAXSEG;
                more_sh = cnt > skip + NMAXSEG;
            }
        }
        __syncthreads();
        const int nseg = nseg_sh;

        if (warp == 0 || warp == 2 || warp == 3 || warp >= 8) {
            // ================================================================ producer(s)
            const int gw = warp == 0 ? 0 : (warp < 4 ? warp - 1 : warp - 5);
            const uint64_t pol = policy_evict_first();
            const uint64_t pol_rope = policy_evict_normal();
            bool stop = false;
            for (int si = 0; si < nseg && !stop; ++si) {
                const Seg sg = segs[si];
                const int T = clamp_len(__ldg(a.seqlens + sg.b), max_tokens, a.L, nullptr);
                const int32_t *bt = a.block_table + (size_t)sg.b * a.max_pages;
                if (a.gather) {
                    // the gather warps split a tile's tokens k = gw, gw + GW, ..; lane i resolves the
                    // cache row of the warp's i-th token (a tile ahead) and the warp copies each
                    // token's latent and rope rows into the box layout; every lane arrives on the
                    // stage barrier once its copies have landed
                    static_assert(TOK <= 32 * GW, "one token per gather lane");
                    const __nv_bfloat16 *lat = (const __nv_bfloat16 *)a.cache0 + (size_t)c * C::DC;
                    const __nv_bfloat16 *rope = (const __nv_bfloat16 *)a.cache1;
                    const int nk = (TOK - gw + GW - 1) / GW;
                    auto tok_of = [&](int t) { return min(t * TOK + gw + GW * lane, T - 1); };
                    int nxt = lane < nk ? __ldg(bt + tok_of(sg.t0) / a.page_size) : 0;
                    for (int t = sg.t0; t < sg.t1 && !stop; ++t) {
                        int pg = nxt;
                        if (t + 1 < sg.t1 && lane < nk) nxt = __ldg(bt + tok_of(t + 1) / a.page_size);
                        const uint32_t stage = p_issued % NST;
                        if (!mbar_wait_warp(&empty_bar[stage], ((p_issued / NST) & 1) ^ 1, &abort_sh, a.err,
                                            lim_ns)) {
                            stop = true;
                            break;
                        }
                        int myrow = 0;
                        if (lane < nk) {
                            if (pg < 0 || pg >= a.num_pages) {
                                set_error(a.err, DEVERR_BAD_PAGE);
                                pg = 0;
                            }
                            myrow = pg * a.page_size + tok_of(t) % a.page_size;
                        }
                        if (!(a.debug_flags & DEBUG_SKIP_FIRST_LOAD) || p_issued != 0) {
                            const uint32_t st = smem_u32(stage_s + (size_t)stage * C::STAGE);
                            gather_tile<C::NV, 8>(st, C::CHUNK, lat, (size_t)a.h_c * C::DC, rope, 64,
                                                  st + C::NV * C::CHUNK, myrow, gw, GW, nk, lane, pol);
                            cp_async_arrive(&full_bar[stage]);
                        }
                        ++p_issued;
                    }
                    continue;
                }
                // box path: a tile is nbox boxes of box_tok tokens, each inside one page; boxes
                // that start at or past T are not loaded (their rows are masked and zeroed).  The
                // three warps 0, 2, 3 issue the boxes together (box k by warp k % 3, lane k / 3):
                // a TMA instruction costs its warp ~0.1k cycles of issue per active lane, and a
                // tile's 5 nbox copies from one warp fell behind the stream
                const int box_tok = a.box_tok;
                const int nbox = TOK / box_tok;
                const int kbox = gw + GW * lane;  // this lane's box of every tile
                // block-table entries are read two tiles ahead of their use, so that their latency
                // overlaps the stage waits; NO_BOX marks a box past T_b
                constexpr int NO_BOX = -2147483647 - 1;
                auto raw_entry = [&](int t) -> int {
                    const int tok = t * TOK + kbox * box_tok;
                    return (t < sg.t1 && kbox < nbox && tok < T) ? __ldg(bt + tok / a.page_size) : NO_BOX;
                };
                auto cache_row = [&](int raw, int t) -> int {  // cache row of this lane's box of tile t
                    if (raw == NO_BOX) return -1;
                    if (raw < 0 || raw >= a.num_pages) {
                        set_error(a.err, DEVERR_BAD_PAGE);
                        raw = 0;
                    }
                    return raw * a.page_size + (t * TOK + kbox * box_tok) % a.page_size;
                };
                // warp 0 also brings the pages of tile t + PF into L2 when it loads tile t, so that
                // their load a stage release later finds them there: whole pages (every latent head
                // and the rope rows) with one untiled bulk prefetch each, by the first latent head's
                // CTA only (the others read the same pages at about the same time)
                const bool pf_warp = warp == 0 && c == 0;
                const size_t lat_page = (size_t)a.page_size * a.h_c * C::DC * 2, rope_page = (size_t)a.page_size * 128;
                int pf_next_page = -1;  // logical page index prefetched next (pages already done: below)
                auto raw_page = [&](int t) -> int {  // lane j: the j-th page of tile t
                    const int p0 = t * TOK / a.page_size, p1 = (min(t * TOK + TOK, T) - 1) / a.page_size;
                    return (pf_warp && t < sg.t1 && p0 + lane <= p1) ? __ldg(bt + p0 + lane) : NO_BOX;
                };
                int raw_ld = raw_entry(sg.t0), raw_nx = raw_entry(sg.t0 + 1);
                int raw_pf = raw_page(sg.t0 + PF), raw_pf_nx = raw_page(sg.t0 + PF + 1);
                for (int t = sg.t0; t < sg.t1 && !stop; ++t) {
                    const int row = cache_row(raw_ld, t);
                    const int pf = raw_pf;
                    raw_ld = raw_nx;
                    raw_nx = raw_entry(t + 2);
                    raw_pf = raw_pf_nx;
                    raw_pf_nx = raw_page(t + PF + 2);
                    const uint32_t stage = p_issued % NST;
                    if (!mbar_wait_warp(&empty_bar[stage], ((p_issued / NST) & 1) ^ 1, &abort_sh, a.err, lim_ns)) {
                        stop = true;
                        break;
                    }
                    if (warp == 0 && lane == 0) {
                        const int nb = min(nbox, (T - t * TOK + box_tok - 1) / box_tok);
                        mbar_arrive_expect_tx(&full_bar[stage], (uint32_t)(nb * box_tok * C::DQK * 2));
                    }
                    if (row >= 0 && (!(a.debug_flags & DEBUG_SKIP_FIRST_LOAD) || p_issued != 0)) {
                        uint8_t *st = stage_s + (size_t)stage * C::STAGE + (size_t)kbox * box_tok * 128;
                        if (box_tok == TOK) {  // one box of all four latent chunks
                            tma_load_3d(st, &latmap, &full_bar[stage], 0, row, c * C::NV, pol);
                        } else {
#pragma unroll
                            for (int ch = 0; ch < C::NV; ++ch)
                                tma_load_3d(st + ch * C::CHUNK, &latmap, &full_bar[stage], 0, row, c * C::NV + ch, pol);
                        }
                        // the rope rows are read by every latent head's CTA: no evict-first hint
                        tma_load_2d(st + C::NV * C::CHUNK, &ropemap, &full_bar[stage], 0, row, pol_rope);
                    }
                    if (pf_warp && t + PF < sg.t1) {
                        // the pages of tile t + PF not prefetched yet (a page can span two tiles)
                        const int p0 = (t + PF) * TOK / a.page_size;
                        const int p1 = (min((t + PF) * TOK + TOK, T) - 1) / a.page_size;
                        const int pg = pf < 0 || pf >= a.num_pages ? 0 : pf;
                        if (p0 + lane <= p1 && p0 + lane >= pf_next_page) {
                            bulk_prefetch_l2((const uint8_t *)a.cache0 + (size_t)pg * lat_page, (uint32_t)lat_page);
                            bulk_prefetch_l2((const uint8_t *)a.cache1 + (size_t)pg * rope_page, (uint32_t)rope_page);
                        }
                        pf_next_page = p1 + 1;
                    }
                    ++p_issued;
                }
            }
            if (stop) {
                // let every copy already issued land before the CTA can exit
                volatile int never = 0;
                if (a.gather) {
                    asm volatile("cp.async.wait_all;" ::: "memory");
                } else {
                    const uint32_t lo = p_issued > (uint32_t)NST ? p_issued - NST : 0;
                    for (uint32_t k = lo; k < p_issued; ++k)
                        mbar_wait_warp(&full_bar[k % NST], (k / NST) & 1, &never, nullptr, lim_ns);
                }
            }
        } else if (warp == 1) {
            // ================================================================ MMA issuer
            if (lane == 0) {
                constexpr uint32_t idesc_s = umma_idesc_bf16(64, TOK, false, false);
                constexpr uint32_t idesc_pv = umma_idesc_bf16(64, C::DC, false, true);
                const uint32_t st0 = smem_u32(stage_s);
                const uint64_t dq0 = umma_desc(smem_u32(q_s), 16, 1024, 2);
                bool ok = true;
                auto issue_s = [&](uint32_t gt) -> bool {
                    const uint32_t stage = gt % NST;
                    if (!mbar_wait_one(&full_bar[stage], (gt / NST) & 1, &abort_sh, a.err, lim_ns)) return false;
                    tc_fence_after();
                    if (a.gather) fence_proxy_async();  // rows written by cp.async, read by the tensor core
                    // S(j) goes into buffer j & 1, over P(j - 2): the MMAs of one thread run in issue
                    // order, so this product, issued after the P.V product of tile j - 2, cannot
                    // overwrite that P before it is read
                    const uint32_t d = tmem + C::S_COL + (m_s & 1) * TOK;
                    const uint64_t dk0 = umma_desc(st0 + stage * C::STAGE, 16, 1024, 2);
#pragma unroll
                    for (int kc = 0; kc < C::KCH; ++kc)
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk)
                            umma_bf16(d, dq0 + (uint64_t)((kc * C::QCHUNK + kk * 32) >> 4),
                                      dk0 + (uint64_t)((kc * C::CHUNK + kk * 32) >> 4), idesc_s, (kc | kk) != 0);
                    umma_commit(&sfull_bar[m_s & 1]);
                    ++m_s;
                    return true;
                };
                for (int si = 0; si < nseg && ok; ++si) {
                    const int n = segs[si].t1 - segs[si].t0;
                    if (!mbar_wait_one(&qfull_bar, m_q & 1, &abort_sh, a.err, lim_ns)) break;
                    ++m_q;
                    tc_fence_after();
                    fence_proxy_async();  // q rows written by cp.async
                    if (!issue_s(m_tile)) break;
                    for (int j = 0; j < n; ++j) {
                        if (j + 1 < n && !issue_s(m_tile + j + 1)) {
                            ok = false;
                            break;
                        }
                        const uint32_t pb = m_pv & 1;
                        if (!mbar_wait_one(&pfull_bar[pb], (m_pv >> 1) & 1, &abort_sh, a.err, lim_ns)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                        const uint32_t stage = (m_tile + j) % NST;
                        const uint64_t dv0 = umma_desc(st0 + stage * C::STAGE, C::CHUNK, 1024, 2);
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
        } else if (smx_warp) {
            // ================================================================ softmax / epilogue
            const int st_id = threadIdx.x - 128;  // 0 .. 127
            bool ok = true;
            // wait until P.V number k has completed (O settled): the commit that frees tile k's
            // stage.  P(k) needed S(k), issued after P.V k - 2, so every earlier P.V is complete
            // and the barrier is at most one phase short of the one waited for.
            auto wait_pv = [&](uint32_t k) -> bool {
                return mbar_wait_warp(&empty_bar[k % NST], (k / NST) & 1, &abort_sh, a.err, lim_ns);
            };
            bool q_ready = false;  // this segment's q rows are already on their way
            for (int si = 0; si < nseg && ok; ++si) {
                const Seg sg = segs[si];
                const int b = sg.b;
                const int T = clamp_len(__ldg(a.seqlens + b), max_tokens, a.L, nullptr);
                const int lim = row_ok ? T - a.L + i_row : -1;  // causal: row (i, h) sees t <= T - L + i
                const int lim_all = T - a.L;                     // visible to every row
                if (!q_ready) load_q(b);  // the q buffer is free: the previous segment's scores are done
                q_ready = false;
                // l: sum of the fp32 P (gives lse); lq: sum of the bf16-rounded P the product uses
                float m_ref = -INFINITY, l = 0.f, lq = 0.f;
                for (int tile = sg.t0; tile < sg.t1; ++tile) {
                    const int tok0 = tile * TOK;
                    const uint32_t sb = x_s & 1;
                    if (!mbar_wait_warp(&sfull_bar[sb], (x_s >> 1) & 1, &abort_sh, a.err, lim_ns)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    ++x_s;
                    // the segment's last score product is done: q may be overwritten by the next
                    // segment's rows while this tile and the epilogue run
                    if (tile + 1 == sg.t1 && si + 1 < nseg) {
                        load_q(segs[si + 1].b);
                        q_ready = true;
                    }
                    float s[NS];
                    const int tok0_t = tok0 + half * NS;  // this thread's first token
                    float mx = -INFINITY;
                    const bool full = tok0 + TOK - 1 <= lim_all;  // nothing masked in the tile
                    if (warp_live) {
                        load_half_row<NS>(tmem + s_lanes + C::S_COL + sb * TOK, s);
                        mx = tile_max(s, full, tok0_t, lim, a.scale_log2);
                        if (!row_ok) mx = -INFINITY;
                    }
                    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
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
                        // half h rescales O columns [128 h, 128 h + 128) of its row
#pragma unroll 1
                        for (int ch = 0; ch < C::DC / 64; ++ch) {
                            float o[32];
                            tmem_ld16x2_32<C::DC / 2>(tmem + s_lanes + ch * 32, o);
#pragma unroll
                            for (int k = 0; k < 32; ++k) o[k] *= alpha;
                            tmem_st16x2_32<C::DC / 2>(tmem + s_lanes + ch * 32, o);
                        }
                        tmem_st_wait();
                    }
                    if (warp_live) l += tile_exp(s, full, tok0_t, lim, a.scale_log2, m_ref);

                    // tokens past T_b in this tile hold garbage or were never loaded: zero their
                    // value rows (P is 0 there, but 0 * NaN would still poison the product)
                    const uint32_t stage = x_tile % NST;
                    if (tok0 + TOK > T) {
                        const int k0 = max(T - tok0, 0);
                        uint8_t *v0 = stage_s + (size_t)stage * C::STAGE;
                        const int units = (TOK - k0) * C::NV * 8;  // 16-byte units: rows x chunks x 8
                        for (int u = st_id; u < units; u += 32 * NSMX) {
                            const int row = k0 + u / (C::NV * 8), ch = (u / 8) % C::NV, k = u & 7;
                            *(uint4 *)(v0 + ch * C::CHUNK + row * 128 + k * 16) = make_uint4(0, 0, 0, 0);
                        }
                    }
                    // P (bf16 pairs) over S in the same buffer (this thread has read its scores)
                    if (warp_live) {
                        uint32_t w[NS / 2];
                        float sum = 0.f, sum2 = 0.f;
#pragma unroll
                        for (int k = 0; k < NS / 2; ++k) {
                            w[k] = pack_bf16(s[2 * k], s[2 * k + 1]);
                            sum += bf16_lo(w[k]);
                            sum2 += bf16_hi(w[k]);
                        }
                        store_half_row<NS>(tmem + s_lanes + C::S_COL + sb * TOK, w);
                        tmem_st_wait();
                        lq += sum + sum2;
                    }
                    if (tok0 + TOK > T) fence_proxy_async();  // the zeroed value rows above
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
                l += __shfl_xor_sync(0xffffffffu, l, 16);  // the two threads of a row hold partial sums
                lq += __shfl_xor_sync(0xffffffffu, lq, 16);
                const float inv = lq > 0.f ? 1.f / lq : 0.f;
                const float lse_v = l > 0.f ? (m_ref + lg2(l)) * 0.69314718055994530942f : -INFINITY;
                const size_t rows_b = (size_t)a.L * a.h_q;
                const size_t r_out = (size_t)i_row * a.h_q + head;
                if (warp_live) {
#pragma unroll 1
                    for (int ch = 0; ch < C::DC / 64; ++ch) {
                        float o[32];
                        tmem_ld16x2_32<C::DC / 2>(tmem + s_lanes + ch * 32, o);
                        if (!row_ok) continue;
                        const int col = half * (C::DC / 2) + ch * 32;
                        if (sg.nsplit == 1) {
                            uint4 *op = (uint4 *)(a.out + ((size_t)b * rows_b + r_out) * C::DC + col);
#pragma unroll
                            for (int k = 0; k < 4; ++k)
                                op[k] = make_uint4(pack_bf16(o[8 * k] * inv, o[8 * k + 1] * inv),
                                                   pack_bf16(o[8 * k + 2] * inv, o[8 * k + 3] * inv),
                                                   pack_bf16(o[8 * k + 4] * inv, o[8 * k + 5] * inv),
                                                   pack_bf16(o[8 * k + 6] * inv, o[8 * k + 7] * inv));
                        } else {
                            float4 *op = (float4 *)(a.ws_o + ((size_t)sg.slot * rows_b + r_out) * C::DC + col);
#pragma unroll
                            for (int k = 0; k < 8; ++k)
                                op[k] = make_float4(o[4 * k] * inv, o[4 * k + 1] * inv, o[4 * k + 2] * inv,
                                                    o[4 * k + 3] * inv);
                        }
                    }
                }
                if (row_ok && half == 0) {
                    if (sg.nsplit == 1)
                        a.lse[(size_t)b * rows_b + r_out] = lse_v;
                    else
                        a.ws_lse[(size_t)sg.slot * rows_b + r_out] = lse_v;
                }
                tc_fence_before();
            }
            if (!ok) asm volatile("cp.async.wait_all;" ::: "memory");  // q copies in flight
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
    if (warp >= 4) asm volatile("cp.async.wait_all;" ::: "memory");
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem, C::TMEM_COLS);
}

template <int TOK, int GW>
cudaError_t launch_t(const CUtensorMap &lm, const CUtensorMap &rm, const LatentArgs &a, int grid, cudaStream_t st) {
    auto k = gla_narrow_kernel<TOK, GW>;
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)NarrowCfg<TOK>::SMEM);
    if (e != cudaSuccess) return e;
    k<<<grid, narrow_threads<GW>(), NarrowCfg<TOK>::SMEM, st>>>(lm, rm, a);
    return cudaGetLastError();
}

}  // namespace

int narrow_tile_tokens() { return NARROW_TOK; }
// A segment start costs the CTA about 4 us (its q copy, the refill of the ring, the epilogue of
// the segment before it) against ~1.5 us per 96-token tile at the HBM rate: a part that starts
// six sequences ended ~20 us after the median one when parts were cut by tiles alone.
int narrow_seg_cost() { return 3; }
size_t narrow_smem_bytes() { return NarrowCfg<NARROW_TOK>::SMEM; }

cudaError_t launch_gla_narrow(const CUtensorMap &lm, const CUtensorMap &rm, const LatentArgs &a, int grid,
                              cudaStream_t st) {
    // gathered tiles: more producer warps, as the copy-issue rate of three bounds the kernel; the
    // box path keeps the smaller block (and its register bound)
    return a.gather ? launch_t<NARROW_TOK, GATHER_WARPS>(lm, rm, a, grid, st)
                    : launch_t<NARROW_TOK, BOX_WARPS>(lm, rm, a, grid, st);
}

}  // namespace kvd
