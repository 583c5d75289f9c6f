// GQA and GTA decode over a paged KV cache: warp-level tensor-core kernel.
//
// "Hardware-Efficient Attention for Fast Decoding", section 3: with g_q query
// heads per KV head the decode step does about 2 g_q / m_kv FLOPs per loaded
// byte (about 4 for GQA and 7.5 for GTA at h_q = 32, h_kv = 8), far below the
// B200 ridge, so this kernel is built to stream the cache at HBM speed; the
// math uses mma.sync because g_q * q_len (4 rows per group) is far too small
// for a 128-row tcgen05 tile.
//
// One CTA owns one contiguous part of the (sequence, 16-token tile) stream and
// `gpc` KV groups.  Warp `gpc` is the producer: it resolves block-table entries
// for a whole warp's worth of pages at once and issues one TMA per operand per
// tile (128-byte swizzle) into an n-stage mbarrier ring.  Warps 0..gpc-1 each
// own one KV group; per tile they compute S^T = K q^T with tokens as the MMA's
// M dimension (so the 4 query rows only pad N = 8, not M = 16), run the online
// softmax in fp32 (base 2, scale folded in), transpose P with movmatrix into
// the B operand and accumulate O^T += V^T P^T (V^T via ldmatrix.trans).  GTA
// reads the tied tile twice from shared memory: its first d_h - d_r dims as the
// key and all d_h dims as the value; the shared rope tile supplies the rest of
// the key.  Sequences cut into several parts write fp32 partials that the
// combine kernel merges.
#include <cuda_bf16.h>

#include "common.cuh"
#include "kernels.h"

namespace kvd {

namespace {

constexpr int MAXSEG = 128;
// GW: producer warps when tiles are gathered token by token (the block has up to 8 + GW warps;
// box-load launches use one producer warp but keep the GW = 4 bound, so their code is unchanged)
template <bool TIED, int D, int DR, int NT, int TT, int GW>
__global__ void __launch_bounds__((8 + GW) * 32, 1)
    group_decode_kernel(const __grid_constant__ CUtensorMap map0, const __grid_constant__ CUtensorMap map1,
                        const GroupArgs a) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    __shared__ uint64_t full_bar[MAX_STAGES], empty_bar[MAX_STAGES];
    __shared__ Seg segs[MAXSEG];
    __shared__ int nseg_sh, more_sh;
    __shared__ volatile int abort_sh;

    uint8_t *smem = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int gpc = a.gpc;
    const int part = blockIdx.x / a.n_sub, sub = blockIdx.x % a.n_sub;
    const int nstage = a.nstage;
    const int g_q = a.h_q / a.h_kv;
    const int R = g_q * a.L;
    const int max_tokens = a.max_pages * a.page_size;
    constexpr int NH = TT / 16;                                // 16-token MMA blocks per stage
    const uint32_t kv_tile = (uint32_t)(gpc * D * TT * 2);    // bytes of one K / V / tied tile

    if (threadIdx.x == 0) {
        for (int s = 0; s < nstage; ++s) {
            mbar_init(&full_bar[s], a.gather ? 32 * GW : 1);  // gathered: every producer lane
            mbar_init(&empty_bar[s], gpc);
        }
        abort_sh = 0;
        fence_mbar_init();
    }
    if (warp == gpc && lane == 0 && !a.gather) {
        tma_prefetch_desc(&map0);
        tma_prefetch_desc(&map1);
    }
    pdl_launch_dependents();
    __syncthreads();

    uint32_t it = 0;  // tile counter, identical in every warp
    for (int skip = 0;; skip += MAXSEG) {
        if (warp == gpc) {
            int cnt = 0;
            plan_walk(a.seqlens, a.B, TT, a.seg_cost, max_tokens, a.L, part, a.parts, a.err, [&](const Seg &s) {
                if (cnt >= skip && cnt < skip + MAXSEG) segs[cnt - skip] = s;
                ++cnt;
            });
            if (lane == 0) {
                nseg_sh = cnt - skip < MAXSEG ? (cnt - skip > 0 ? cnt - skip : 0) : MAXSEG;
                more_sh = cnt > skip + MAXSEG;
            }
        }
        __syncthreads();
        const int nseg = nseg_sh;

        if (warp >= gpc) {
            // ------------------------------------------------------------ producer(s)
            const uint64_t pol = policy_evict_first();
            const int z0 = sub * gpc * (D / 64);  // first 64-wide chunk of this CTA's groups
            uint32_t issued = it;
            bool stop = false;
            for (int si = 0; si < nseg && !stop; ++si) {
                const Seg sg = segs[si];
                const int32_t *bt = a.block_table + (size_t)sg.b * a.max_pages;
                if (a.gather) {
                    // Pages smaller than a tile (down to one token) or not a multiple of it.  The
                    // GW producer warps all walk every tile; warp w copies the tokens
                    // k = w, w + GW, ...: one lane per token resolves its cache row
                    // (distributed offset calculation, fetched a tile ahead), then the warp copies
                    // each token's row with 16-byte cp.async into the same swizzled layout the box
                    // loads produce (a token's row is contiguous: 32 lanes move 512 consecutive
                    // bytes per instruction).  Every lane arrives on the stage's barrier when its
                    // copies have landed.
                    const int pw = warp - gpc;
                    constexpr int TPW = (TT + GW - 1) / GW;     // most tokens a warp takes per tile
                    const int nkw = (TT - pw + GW - 1) / GW;    // the tokens this warp takes
                    const int T = clamp_len(__ldg(a.seqlens + sg.b), max_tokens, a.L, nullptr);
                    const int nch = gpc * (D / 64);
                    const size_t row_elems = (size_t)a.h_kv * D;
                    const __nv_bfloat16 *c0 = (const __nv_bfloat16 *)a.cache0 + (size_t)z0 * 64;
                    const __nv_bfloat16 *c1 = (const __nv_bfloat16 *)a.cache1 + (TIED ? 0 : (size_t)z0 * 64);
                    constexpr int RU = TIED ? DR * 2 / 16 : 0;  // 16-byte units of a rope row
                    // token of this lane in tile t (tokens past T_b repeat the last one; masked later)
                    auto tok_of = [&](int t) { return min(t * TT + pw + GW * lane, T - 1); };
                    int nxt_tok = tok_of(sg.t0);
                    int nxt_page = lane < nkw ? __ldg(bt + nxt_tok / a.page_size) : 0;
                    for (int t = sg.t0; t < sg.t1 && !stop; ++t, ++issued) {
                        const int tok = nxt_tok;
                        int page = nxt_page;
                        if (t + 1 < sg.t1) {
                            nxt_tok = tok_of(t + 1);
                            if (lane < nkw) nxt_page = __ldg(bt + nxt_tok / a.page_size);
                        }
                        const uint32_t stage = issued % nstage;
                        if (!mbar_wait_warp(&empty_bar[stage], ((issued / nstage) & 1) ^ 1, &abort_sh, a.err,
                                            a.wait_limit_ns)) {
                            stop = true;
                            break;
                        }
                        if (lane < nkw && (page < 0 || page >= a.num_pages)) {
                            set_error(a.err, DEVERR_BAD_PAGE);
                            page = 0;
                        }
                        const int myrow = page * a.page_size + tok % a.page_size;
                        if (!(a.debug_flags & DEBUG_SKIP_FIRST_LOAD) || issued != 0) {
                            // lane l moves 16-byte unit l % 8 of chunk l / 8 + 4 j of each token: the
                            // per-lane parts of both addresses are fixed, a token adds its row and slot
                            const uint32_t st = smem_u32(smem + (size_t)stage * a.stage_bytes);
                            const uint32_t dst_l = st + (uint32_t)((lane >> 3) * TT) * 128u;
                            const uint32_t c_l = (uint32_t)(lane & 7);
                            const int nj = (nch * 8 - lane + 31) / 32;  // this lane's units of a row
#pragma unroll
                            for (int i = 0; i < TPW; ++i) {
                                if (i >= nkw) break;
                                const uint32_t k = (uint32_t)(pw + GW * i);
                                const size_t row = (size_t)__shfl_sync(0xffffffffu, myrow, i);
                                const uint32_t dst = dst_l + k * 128u + ((c_l ^ (k & 7u)) << 4);
                                const __nv_bfloat16 *s0 = c0 + row * row_elems + lane * 8;
#pragma unroll 4
                                for (int j = 0; j < nj; ++j) {
                                    const uint32_t d = dst + (uint32_t)(4 * j * TT) * 128u;
                                    cp_async16(d, s0 + 256 * j, pol);
                                    if (!TIED) cp_async16(d + kv_tile, c1 + row * row_elems + lane * 8 + 256 * j, pol);
                                }
                            }
                            if constexpr (TIED) {
                                // rope rows, 32 / RU tokens per instruction: lane l copies unit l % RU
                                // of token pw + GW (i0 + l / RU)
                                const uint32_t ru = (uint32_t)(lane % RU);
#pragma unroll
                                for (int i0 = 0; i0 < TPW; i0 += 32 / RU) {
                                    const int i = i0 + lane / RU;
                                    const size_t row = (size_t)__shfl_sync(0xffffffffu, myrow, i & 31);
                                    if (i < nkw) {
                                        const uint32_t k = (uint32_t)(pw + GW * i);
                                        cp_async16(st + kv_tile + (DR == 64 ? sw128(k, ru) : sw64(k, ru)),
                                                   c1 + row * DR + ru * 8, pol);
                                    }
                                }
                            }
                            cp_async_arrive(&full_bar[stage]);
                        }
                    }
                    continue;
                }
                if (warp != gpc) continue;  // whole-tile boxes: one producer warp
                const int tiles_per_page = a.page_size / TT;
                const int p_first = sg.t0 / tiles_per_page;
                const int p_last = (sg.t1 - 1) / tiles_per_page;
                for (int pb = p_first; pb <= p_last && !stop; pb += 32) {
                    // distributed offset calculation: one block-table entry per lane
                    int page = 0;
                    if (pb + lane <= p_last) {
                        page = __ldg(bt + pb + lane);
                        if (page < 0 || page >= a.num_pages) {
                            set_error(a.err, DEVERR_BAD_PAGE);
                            page = 0;
                        }
                    }
                    const int t_lo = max(sg.t0, pb * tiles_per_page);
                    const int t_hi = min(sg.t1, (pb + 32) * tiles_per_page);
                    for (int t = t_lo; t < t_hi; ++t) {
                        const int pg = __shfl_sync(0xffffffffu, page, t / tiles_per_page - pb);
                        const uint32_t stage = issued % nstage;
                        if (!mbar_wait_warp(&empty_bar[stage], ((issued / nstage) & 1) ^ 1, &abort_sh, a.err,
                                            a.wait_limit_ns)) {
                            stop = true;
                            break;
                        }
                        if (lane == 0) {
                            uint8_t *st = smem + (size_t)stage * a.stage_bytes;
                            const int row = pg * a.page_size + (t % tiles_per_page) * TT;
                            mbar_arrive_expect_tx(&full_bar[stage], a.stage_bytes_tx);
                            if (!(a.debug_flags & DEBUG_SKIP_FIRST_LOAD) || issued != 0) {
                                tma_load_3d(st, &map0, &full_bar[stage], 0, row, z0, pol);
                                if (TIED)
                                    tma_load_2d(st + kv_tile, &map1, &full_bar[stage], 0, row, pol);
                                else
                                    tma_load_3d(st + kv_tile, &map1, &full_bar[stage], 0, row, z0, pol);
                            }
                        }
                        ++issued;
                    }
                }
            }
            if (stop && a.gather) {
                asm volatile("cp.async.wait_all;" ::: "memory");  // this lane's copies have landed
            } else if (stop) {
                // Let every copy already issued land before the CTA can exit.
                const uint32_t lo = issued > (uint32_t)nstage ? issued - nstage : 0;
                for (uint32_t k = lo; k < issued; ++k) {
                    volatile int never = 0;
                    mbar_wait_warp(&full_bar[k % nstage], (k / nstage) & 1, &never, nullptr, a.wait_limit_ns);
                }
            }
            it = issued;
        } else {
            // ------------------------------------------------------------ consumers
            const int gl = warp;                      // local group
            const int g = sub * gpc + gl;             // KV group
            const int lr = lane >> 2, lc = lane & 3;  // fragment row / column-pair
            // Stage-relative shared-memory addresses of this lane's ldmatrix rows (the swizzle
            // depends only on the lane).  koff: K (x4: tokens 8*(mi&1).., dims 8*(mi>>1)..);
            // voff: V^T (x4.trans: dims 8*(mi&1).., tokens 8*(mi>>1)..).  The next 16 tokens sit
            // 16 rows further on: +2048 bytes in 128-byte rows, +1024 in the 64-byte rope rows.
            uint32_t koff[D / 16], khalf[D / 16], voff[D / 16];
            {
                const int mi = lane >> 3;
                const int tk_k = (lane & 7) + 8 * (mi & 1);
                const int tk_v = (lane & 7) + 8 * (mi >> 1);
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const int dim = kk * 16 + 8 * (mi >> 1);
                    if (!TIED || kk * 16 < D - DR) {
                        koff[kk] = sw128((gl * (D / 64) + dim / 64) * TT + tk_k, (dim & 63) >> 3);
                        khalf[kk] = 2048;
                    } else {
                        const int rd = dim - (D - DR);
                        koff[kk] = kv_tile + (DR == 64 ? sw128(tk_k, rd >> 3) : sw64(tk_k, rd >> 3));
                        khalf[kk] = DR == 64 ? 2048 : 1024;
                    }
                    const int vdim = kk * 16 + 8 * (mi & 1);
                    voff[kk] = (TIED ? 0u : kv_tile) + sw128((gl * (D / 64) + vdim / 64) * TT + tk_v, (vdim & 63) >> 3);
                }
            }
            for (int si = 0; si < nseg; ++si) {
                const Seg sg = segs[si];
                const int b = sg.b;
                const int T = clamp_len(__ldg(a.seqlens + b), max_tokens, a.L, nullptr);

                // q^T as B fragments: rows n = 8 nt + lr, dims kk*16 + 2 lc (+8)
                uint32_t qf[NT][D / 16][2];
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    const int n = 8 * nt + lr;
                    if (n < R) {
                        const int i = n / g_q, head = g * g_q + n % g_q;
                        const uint32_t *qp =
                            (const uint32_t *)(a.q + (((size_t)b * a.L + i) * a.h_q + head) * D);
#pragma unroll
                        for (int kk = 0; kk < D / 16; ++kk) {
                            qf[nt][kk][0] = __ldg(qp + kk * 8 + lc);
                            qf[nt][kk][1] = __ldg(qp + kk * 8 + 4 + lc);
                        }
                    } else {
#pragma unroll
                        for (int kk = 0; kk < D / 16; ++kk) qf[nt][kk][0] = qf[nt][kk][1] = 0u;
                    }
                }
                // causal limit of the two rows this lane's accumulators hold
                int lim[NT][2];
#pragma unroll
                for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                    for (int j = 0; j < 2; ++j) {
                        const int n = 8 * nt + 2 * lc + j;
                        lim[nt][j] = n < R ? T - a.L + n / g_q : -1;
                    }

                // m holds the reference maximum of each row (base 2, scale folded in).  It is
                // only raised when a score exceeds it by more than 2^8, so P stays <= 256 and
                // O is rescaled rarely.
                // l: sum of the fp32 P (gives lse); lr: sum of the bf16-rounded P the product
                // uses (normalises O, so the output is a convex combination of the rounded
                // weights and a dominant token comes out exactly).
                float m[NT][2], l[NT][2], lq[NT][2], o[NT][D / 16][4];
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    m[nt][0] = m[nt][1] = -INFINITY;
                    l[nt][0] = l[nt][1] = 0.f;
                    lq[nt][0] = lq[nt][1] = 0.f;
#pragma unroll
                    for (int mt = 0; mt < D / 16; ++mt) o[nt][mt][0] = o[nt][mt][1] = o[nt][mt][2] = o[nt][mt][3] = 0.f;
                }
                // smallest causal limit over the real rows: tiles entirely at or below it need no mask
                const int lim_all = T - a.L;

                bool ok = true;
                for (int tile = sg.t0; tile < sg.t1; ++tile, ++it) {
                    const uint32_t stage = it % nstage;
                    if (!mbar_wait_warp(&full_bar[stage], (it / nstage) & 1, &abort_sh, a.err, a.wait_limit_ns)) {
                        ok = false;
                        break;
                    }
                    const uint32_t base = smem_u32(smem + (size_t)stage * a.stage_bytes);
                    const int tok0 = tile * TT;

                    // ---- S^T = K q^T (tokens x rows), NH independent 16-token blocks
                    float s[NH][NT][4];
#pragma unroll
                    for (int h = 0; h < NH; ++h)
#pragma unroll
                        for (int nt = 0; nt < NT; ++nt) s[h][nt][0] = s[h][nt][1] = s[h][nt][2] = s[h][nt][3] = 0.f;
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk) {
#pragma unroll
                        for (int h = 0; h < NH; ++h) {
                            uint32_t A[4];
                            ldsm_x4(base + koff[kk] + h * khalf[kk], A);
#pragma unroll
                            for (int nt = 0; nt < NT; ++nt) mma_bf16(s[h][nt], A, qf[nt][kk][0], qf[nt][kk][1]);
                        }
                    }

                    // ---- mask (boundary tiles only), online softmax in base 2
                    const bool full = tok0 + TT - 1 <= lim_all;
#pragma unroll
                    for (int h = 0; h < NH; ++h)
#pragma unroll
                        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                const int t = tok0 + 16 * h + lr + 8 * (e >> 1);
                                const float v = s[h][nt][e] * a.scale_log2;
                                s[h][nt][e] = (full || t <= lim[nt][e & 1]) ? v : -INFINITY;
                            }
                    float alpha[NT][2];
                    bool rescale = false;
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                        for (int j = 0; j < 2; ++j) {
                            float mx = -INFINITY;
#pragma unroll
                            for (int h = 0; h < NH; ++h) mx = fmaxf(mx, fmaxf(s[h][nt][j], s[h][nt][2 + j]));
                            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
                            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
                            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
                            float al = 1.f;
                            if (mx != -INFINITY) {
                                if (m[nt][j] == -INFINITY) {
                                    m[nt][j] = mx;  // first visible score: O and l still hold zeros
                                } else if (mx > m[nt][j] + 8.f) {
                                    al = ex2(m[nt][j] - mx);
                                    m[nt][j] = mx;
                                }
                            }
                            alpha[nt][j] = al;
                            rescale |= (al != 1.f);
                            const float mr = m[nt][j] == -INFINITY ? 0.f : m[nt][j];
#pragma unroll
                            for (int h = 0; h < NH; ++h) {
                                s[h][nt][j] = ex2(s[h][nt][j] - mr);
                                s[h][nt][2 + j] = ex2(s[h][nt][2 + j] - mr);
                            }
                        }
                    if (__any_sync(0xffffffffu, rescale)) {
#pragma unroll
                        for (int nt = 0; nt < NT; ++nt) {
                            l[nt][0] *= alpha[nt][0];
                            l[nt][1] *= alpha[nt][1];
                            lq[nt][0] *= alpha[nt][0];
                            lq[nt][1] *= alpha[nt][1];
#pragma unroll
                            for (int mt = 0; mt < D / 16; ++mt) {
                                o[nt][mt][0] *= alpha[nt][0];
                                o[nt][mt][1] *= alpha[nt][1];
                                o[nt][mt][2] *= alpha[nt][0];
                                o[nt][mt][3] *= alpha[nt][1];
                            }
                        }
                    }

                    // ---- P^T as B fragments (tokens x rows) via 8x8 transposes.  The normaliser
                    // sums the same bf16-rounded P the product uses.
                    uint32_t pb[NH][NT][2];
#pragma unroll
                    for (int h = 0; h < NH; ++h)
#pragma unroll
                        for (int nt = 0; nt < NT; ++nt) {
                            const uint32_t x0 = pack_bf16(s[h][nt][0], s[h][nt][1]);
                            const uint32_t x1 = pack_bf16(s[h][nt][2], s[h][nt][3]);
                            // (after the rescale above: l and lq were scaled to the current m first)
                            l[nt][0] += s[h][nt][0] + s[h][nt][2];
                            l[nt][1] += s[h][nt][1] + s[h][nt][3];
                            lq[nt][0] += bf16_lo(x0) + bf16_lo(x1);
                            lq[nt][1] += bf16_hi(x0) + bf16_hi(x1);
                            pb[h][nt][0] = movmatrix_t(x0);
                            pb[h][nt][1] = movmatrix_t(x1);
                        }

                    // ---- O^T += V^T P^T; tokens past T_b hold garbage (NaN poison): zero them
                    uint32_t mlo[NH], mhi[NH];
#pragma unroll
                    for (int h = 0; h < NH; ++h) {
                        mlo[h] = mhi[h] = 0xffffffffu;
                        const int t0 = tok0 + 16 * h + 2 * lc;
                        if (tok0 + TT > T) {
                            mlo[h] = (t0 < T ? 0x0000ffffu : 0u) | (t0 + 1 < T ? 0xffff0000u : 0u);
                            mhi[h] = (t0 + 8 < T ? 0x0000ffffu : 0u) | (t0 + 9 < T ? 0xffff0000u : 0u);
                        }
                    }
#pragma unroll
                    for (int mt = 0; mt < D / 16; ++mt)
#pragma unroll
                        for (int h = 0; h < NH; ++h) {
                            uint32_t A[4];
                            ldsm_x4_t(base + voff[mt] + h * 2048, A);
                            A[0] &= mlo[h];
                            A[1] &= mlo[h];
                            A[2] &= mhi[h];
                            A[3] &= mhi[h];
#pragma unroll
                            for (int nt = 0; nt < NT; ++nt) mma_bf16(o[nt][mt], A, pb[h][nt][0], pb[h][nt][1]);
                        }
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&empty_bar[stage]);
                }
                if (!ok) {
                    // skip the rest; keep the tile counter in step with the producer
                    break;
                }

                // ---- epilogue
#pragma unroll
                for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                    for (int j = 0; j < 2; ++j) {
                        float v = l[nt][j], w = lq[nt][j];
                        v += __shfl_xor_sync(0xffffffffu, v, 4);
                        w += __shfl_xor_sync(0xffffffffu, w, 4);
                        v += __shfl_xor_sync(0xffffffffu, v, 8);
                        w += __shfl_xor_sync(0xffffffffu, w, 8);
                        v += __shfl_xor_sync(0xffffffffu, v, 16);
                        w += __shfl_xor_sync(0xffffffffu, w, 16);
                        l[nt][j] = v;
                        lq[nt][j] = w;
                    }
                const int rows_b = a.L * a.h_q;
#pragma unroll
                for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                    for (int j = 0; j < 2; ++j) {
                        const int n = 8 * nt + 2 * lc + j;
                        if (n >= R) continue;
                        const int i = n / g_q, head = g * g_q + n % g_q;
                        const float lv = l[nt][j];
                        const float inv = lq[nt][j] > 0.f ? 1.f / lq[nt][j] : 0.f;
                        const float lse_v = lv > 0.f ? (m[nt][j] + lg2(lv)) * 0.69314718055994530942f : -INFINITY;
                        const int r = i * a.h_q + head;
                        if (sg.nsplit == 1) {
                            __nv_bfloat16 *op = a.out + ((size_t)b * rows_b + r) * D;
#pragma unroll
                            for (int mt = 0; mt < D / 16; ++mt) {
                                op[mt * 16 + lr] = __float2bfloat16_rn(o[nt][mt][j] * inv);
                                op[mt * 16 + 8 + lr] = __float2bfloat16_rn(o[nt][mt][2 + j] * inv);
                            }
                            if (lr == 0) a.lse[(size_t)b * rows_b + r] = lse_v;
                        } else {
                            float *op = a.ws_o + ((size_t)sg.slot * rows_b + r) * D;
#pragma unroll
                            for (int mt = 0; mt < D / 16; ++mt) {
                                op[mt * 16 + lr] = o[nt][mt][j] * inv;
                                op[mt * 16 + 8 + lr] = o[nt][mt][2 + j] * inv;
                            }
                            if (lr == 0) a.ws_lse[(size_t)sg.slot * rows_b + r] = lse_v;
                        }
                    }
            }
        }
        __syncthreads();
        if (!more_sh || abort_sh) break;
        __syncthreads();
    }
}

template <bool TIED, int D, int DR, int NT, int TT, int GW = 4>
cudaError_t launch_t(const CUtensorMap &m0, const CUtensorMap &m1, const GroupArgs &a, int grid, size_t smem,
                     cudaStream_t st) {
    auto k = group_decode_kernel<TIED, D, DR, NT, TT, GW>;
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    k<<<grid, (a.gpc + (a.gather ? GW : 1)) * 32, smem, st>>>(m0, m1, a);
    return cudaGetLastError();
}

template <bool TIED, int D, int DR>
cudaError_t launch_nt(int nt, const CUtensorMap &m0, const CUtensorMap &m1, const GroupArgs &a, int grid,
                      size_t smem, cudaStream_t st) {
    // gathered 32-token tiles (GTA at small page sizes): six producer warps keep more copies in flight
    if (a.tile == 32 && nt == 1)
        return a.gather ? launch_t<TIED, D, DR, 1, 32, 6>(m0, m1, a, grid, smem, st)
                        : launch_t<TIED, D, DR, 1, 32>(m0, m1, a, grid, smem, st);
    if (a.tile != 16) return cudaErrorInvalidValue;
    switch (nt) {
        case 1: return launch_t<TIED, D, DR, 1, 16>(m0, m1, a, grid, smem, st);
        case 2: return launch_t<TIED, D, DR, 2, 16>(m0, m1, a, grid, smem, st);
        case 4: return launch_t<TIED, D, DR, 4, 16>(m0, m1, a, grid, smem, st);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace

cudaError_t launch_group_decode(bool tied, int d, int d_r, int nt, const CUtensorMap &m0, const CUtensorMap &m1,
                                const GroupArgs &a, int grid, size_t smem, cudaStream_t st) {
    if (!tied && d == 128) return launch_nt<false, 128, 0>(nt, m0, m1, a, grid, smem, st);
    if (!tied && d == 64) return launch_nt<false, 64, 0>(nt, m0, m1, a, grid, smem, st);
    if (tied && d == 128 && d_r == 64) return launch_nt<true, 128, 64>(nt, m0, m1, a, grid, smem, st);
    if (tied && d == 64 && d_r == 32) return launch_nt<true, 64, 32>(nt, m0, m1, a, grid, smem, st);
    if (tied && d == 128 && d_r == 32) return launch_nt<true, 128, 32>(nt, m0, m1, a, grid, smem, st);
    if (tied && d == 64 && d_r == 64) return launch_nt<true, 64, 64>(nt, m0, m1, a, grid, smem, st);
    return cudaErrorInvalidValue;
}

}  // namespace kvd
