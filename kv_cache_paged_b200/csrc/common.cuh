// Shared device helpers for the decode kernels: PTX wrappers (mbarrier, TMA,
// ldmatrix, mma.sync, movmatrix), bounded waits, error flags and the split plan.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

namespace kvd {

constexpr uint32_t DEVERR_TIMEOUT = 1u;
constexpr uint32_t DEVERR_BAD_PAGE = 2u;
constexpr uint32_t DEVERR_BAD_SEQLEN = 4u;

// Workspace layout: [0, 256) header (error word at 0); then partial lse, then partial O.
constexpr size_t WS_HEADER = 256;

// Tokens per pipeline tile for the warp-MMA kernels (one m16 row block).
constexpr int TILE = 16;

// Default limit for one pipeline wait before the kernel gives up (ns).
constexpr uint64_t WAIT_LIMIT_NS = 2000000000ull;

// ----------------------------------------------------------------------------- split plan
// The (sequence, tile) stream is the concatenation over b of ceil(T_b / tile)
// tiles, N in all.  It is cut into P = min(parts, N) parts; part c < P covers
// tiles [floor(c N / P), floor((c+1) N / P)), so every part is non-empty and
// the parts holding one sequence's tiles are consecutive.  Parts c >= P are idle.
struct Seg {
    int32_t b, t0, t1, split, nsplit, slot;
};

__host__ __device__ inline int64_t part_begin(int64_t c, int64_t N, int64_t parts) { return (c * N) / parts; }

// The part containing tile x (0 <= x < N): the largest c with part_begin(c) <= x.
__host__ __device__ inline int64_t part_of(int64_t x, int64_t N, int64_t parts) {
    return ((x + 1) * parts - 1) / N;
}

// Clamp a sequence length to [0, max_tokens]; report whether it needed it.
__host__ __device__ inline int32_t clamp_len(int32_t T, int32_t max_tokens, int32_t L, bool *bad) {
    bool b = (T < 0) || (T > max_tokens) || (T > 0 && T < L);
    if (bad) *bad = b;
    if (T < 0) return 0;
    if (T > max_tokens) return max_tokens;
    return T;
}

__host__ __device__ inline int32_t tiles_of(int32_t T, int32_t tile) { return (T + tile - 1) / tile; }

// Fill `seg` for sequence b whose tiles are [cu, cu + n) intersected with part c's range.
__host__ __device__ inline Seg make_seg(int32_t b, int64_t cu, int32_t n, int64_t lo, int64_t hi, int64_t c,
                                        int64_t N, int64_t parts) {
    Seg s;
    s.b = b;
    int64_t a = lo > cu ? lo : cu;
    int64_t e = hi < cu + n ? hi : cu + n;
    s.t0 = (int32_t)(a - cu);
    s.t1 = (int32_t)(e - cu);
    int64_t first = part_of(cu, N, parts);
    int64_t last = part_of(cu + n - 1, N, parts);
    s.split = (int32_t)(c - first);
    s.nsplit = (int32_t)(last - first + 1);
    s.slot = (int32_t)(b + c);
    return s;
}

#ifdef __CUDACC__

__device__ __forceinline__ uint32_t smem_u32(const void *p) { return (uint32_t)__cvta_generic_to_shared(p); }

__device__ __forceinline__ uint64_t globaltimer() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ void set_error(uint32_t *err, uint32_t bits) {
    if (err) atomicOr(err, bits);
}

// The (sequence, tile) stream, with a cost: every non-empty sequence contributes seg_cost
// units before its tiles (the fixed work of starting a segment: its q, the pipeline's refill,
// its epilogue, counted in tiles), so the parts, cut into equal numbers of units, give fewer
// tiles to a part that starts more sequences.  Sequence b's tiles are the units
// [cu_b, cu_b + n_b) and its first tile is unit cu_b; seg_cost 0 is the plain tile stream.
__host__ __device__ inline int64_t units_of(int32_t n, int32_t seg_cost) { return n > 0 ? (int64_t)n + seg_cost : 0; }

// Warp-cooperative plan walk.  Every lane of the calling warp must call it with
// the same arguments.  Calls emit(seg) on lane 0 for each segment of part c, in
// order, up to the end of the part; returns N (total units).  The sequence lengths
// are read PLAN_K per lane at a time, all loads in flight together, and the first
// 32 PLAN_K tile counts are kept for the second pass: with up to 128 sequences the
// walk costs one global-memory round trip instead of one per 32 sequences and pass.
constexpr int PLAN_K = 4;
template <typename Emit>
__device__ __forceinline__ int64_t plan_walk(const int32_t *__restrict__ seqlens, int32_t B, int32_t tile,
                                             int32_t seg_cost, int32_t max_tokens, int32_t L, int64_t c,
                                             int64_t parts, uint32_t *err, Emit emit) {
    const int lane = threadIdx.x & 31;
    int64_t N = 0;
    int32_t keep[PLAN_K];  // tile counts of sequences 32 k + lane (the first batch)
    for (int32_t base = 0; base < B; base += 32 * PLAN_K) {
        int32_t raw[PLAN_K];
#pragma unroll
        for (int k = 0; k < PLAN_K; ++k) {
            const int32_t b = base + 32 * k + lane;
            raw[k] = b < B ? __ldg(seqlens + b) : 0;
        }
        int32_t tot = 0;
#pragma unroll
        for (int k = 0; k < PLAN_K; ++k) {
            const int32_t b = base + 32 * k + lane;
            int32_t n = 0;
            if (b < B) {
                bool bad;
                const int32_t T = clamp_len(raw[k], max_tokens, L, &bad);
                if (bad && c == 0) set_error(err, DEVERR_BAD_SEQLEN);
                n = tiles_of(T, tile);
            }
            if (base == 0) keep[k] = n;
            tot += (int32_t)units_of(n, seg_cost);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) tot += __shfl_xor_sync(0xffffffffu, tot, o);
        N += tot;
    }
    if (N == 0) return 0;
    if (parts > N) parts = N;
    if (c >= parts) return N;
    const int64_t lo = part_begin(c, N, parts), hi = part_begin(c + 1, N, parts);
    if (lo >= hi) return N;
    int64_t run = 0;
    for (int32_t base = 0; base < B && run < hi; base += 32) {
        int32_t b = base + lane;
        int32_t n = 0;
        if (base < 32 * PLAN_K) {
#pragma unroll
            for (int k = 0; k < PLAN_K; ++k)
                if (base == 32 * k) n = keep[k];
        } else if (b < B) {
            n = tiles_of(clamp_len(__ldg(seqlens + b), max_tokens, L, nullptr), tile);
        }
        int32_t incl = (int32_t)units_of(n, seg_cost);
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            int32_t v = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += v;
        }
        int64_t cu = run + (incl - n);  // the unit of this sequence's first tile
        bool hit = (b < B) && n > 0 && cu < hi && cu + n > lo;
        uint32_t mask = __ballot_sync(0xffffffffu, hit);
        while (mask) {
            int src = __ffs(mask) - 1;
            mask &= mask - 1;
            int64_t cu_s = __shfl_sync(0xffffffffu, cu, src);
            int32_t n_s = __shfl_sync(0xffffffffu, n, src);
            if (lane == 0) emit(make_seg(base + src, cu_s, n_s, lo, hi, c, N, parts));
        }
        run += __shfl_sync(0xffffffffu, incl, 31);
    }
    return N;
}

// ----------------------------------------------------------------------------- mbarrier
__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}
__device__ __forceinline__ void fence_mbar_init() { asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory"); }
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}
// Complete `bytes` of the current phase's transaction count without a copy (bytes that will
// never arrive).
__device__ __forceinline__ void mbar_complete_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile("mbarrier.complete_tx.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes) : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}\n"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// Wait, by all 32 lanes of a warp together, for phase `parity` of `bar` to
// complete.  Every lane gets the same answer.  Gives up (returns false) when
// *abort becomes nonzero or after limit_ns; on running out it records
// DEVERR_TIMEOUT in *err (when err is not null) and raises *abort so that the
// other warps stop too.
__device__ __forceinline__ bool mbar_wait_warp(uint64_t *bar, uint32_t parity, volatile int *abort, uint32_t *err,
                                               uint64_t limit_ns) {
    if (__all_sync(0xffffffffu, mbar_try_wait(bar, parity))) return true;
    const uint64_t t0 = globaltimer();
    while (true) {
#pragma unroll 1
        for (int i = 0; i < 32; ++i)
            if (__all_sync(0xffffffffu, mbar_try_wait(bar, parity))) return true;
        int stop = 0;
        if ((threadIdx.x & 31) == 0) {
            if (*abort) {
                stop = 1;
            } else if (globaltimer() - t0 > limit_ns) {
                set_error(err, DEVERR_TIMEOUT);
                *abort = 1;
                stop = 1;
            }
        }
        if (__shfl_sync(0xffffffffu, stop, 0)) return false;
    }
}

// ----------------------------------------------------------------------------- TMA
__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap *m) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(m) : "memory");
}
__device__ __forceinline__ void tma_load_2d(void *dst, const CUtensorMap *m, uint64_t *bar, int x, int y,
                                            uint64_t policy) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1, {%3, %4}], [%2], %5;" ::"r"(smem_u32(dst)),
        "l"(m), "r"(smem_u32(bar)), "r"(x), "r"(y), "l"(policy)
        : "memory");
}
__device__ __forceinline__ void tma_load_3d(void *dst, const CUtensorMap *m, uint64_t *bar, int x, int y, int z,
                                            uint64_t policy) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1, {%3, %4, %5}], [%2], %6;" ::"r"(smem_u32(dst)),
        "l"(m), "r"(smem_u32(bar)), "r"(x), "r"(y), "r"(z), "l"(policy)
        : "memory");
}
// Bring a box of a tensor into L2 ahead of its load (no shared memory, no barrier).
__device__ __forceinline__ void tma_prefetch_l2_2d(const CUtensorMap *m, int x, int y) {
    asm volatile("cp.async.bulk.prefetch.tensor.2d.L2.global.tile [%0, {%1, %2}];" ::"l"(m), "r"(x), "r"(y)
                 : "memory");
}
__device__ __forceinline__ void tma_prefetch_l2_3d(const CUtensorMap *m, int x, int y, int z) {
    asm volatile("cp.async.bulk.prefetch.tensor.3d.L2.global.tile [%0, {%1, %2, %3}];" ::"l"(m), "r"(x), "r"(y),
                 "r"(z)
                 : "memory");
}
// Bring `bytes` (a multiple of 16) of contiguous global memory at a 16-byte aligned address into L2.
__device__ __forceinline__ void bulk_prefetch_l2(const void *p, uint32_t bytes) {
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}
// 16-byte copy global -> shared through L2 only (cp.async.cg), with an L2 cache policy.
__device__ __forceinline__ void cp_async16(uint32_t dst_smem, const void *src, uint64_t policy) {
    asm volatile("cp.async.cg.shared.global.L2::cache_hint [%0], [%1], 16, %2;" ::"r"(dst_smem), "l"(src), "l"(policy)
                 : "memory");
}
// Arrive on `bar` once every cp.async this thread issued so far has landed (no count increment:
// the barrier's expected count must include this arrival).
__device__ __forceinline__ void cp_async_arrive(uint64_t *bar) {
    asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(bar)) : "memory");
}
// L2 policy for data read exactly once (the KV stream).
__device__ __forceinline__ uint64_t policy_evict_first() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
    return p;
}
// L2 policy for data that another CTA reads soon after (the rope rows every latent head reads).
__device__ __forceinline__ uint64_t policy_evict_normal() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_normal.b64 %0, 1.0;" : "=l"(p));
    return p;
}

// ----------------------------------------------------------------------------- warp MMA
__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t (&r)[4]) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t (&r)[4]) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
}
// D = A(16x16, row) * B(16x8, col) + D, bf16 in, fp32 accumulate.
__device__ __forceinline__ void mma_bf16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
// Transpose an 8x8 b16 matrix held one bf16x2 per lane in fragment order.
__device__ __forceinline__ uint32_t movmatrix_t(uint32_t x) {
    uint32_t y;
    asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
    return y;
}
// Pack two fp32 into bf16x2 (round to nearest even): lo -> bits [0,16), hi -> [16,32).
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
    uint32_t r;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}
// The two bf16 halves of a packed pair, widened exactly to fp32.
__device__ __forceinline__ float bf16_lo(uint32_t x) { return __uint_as_float(x << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t x) { return __uint_as_float(x & 0xffff0000u); }
__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
__device__ __forceinline__ float lg2(float x) {
    float y;
    asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// 128-byte-swizzled tile of 128-byte rows (TMA SWIZZLE_128B): byte offset of
// 16-byte chunk k of row r.  The tile base must be 1024-byte aligned.
__device__ __forceinline__ uint32_t sw128(uint32_t r, uint32_t k) { return r * 128u + ((k ^ (r & 7u)) << 4); }
// 64-byte rows, TMA SWIZZLE_64B (address bits [4,6) ^= bits [7,9)).
__device__ __forceinline__ uint32_t sw64(uint32_t r, uint32_t k) {
    uint32_t off = r * 64u + k * 16u;
    return off ^ (((off >> 7) & 3u) << 4);
}

// Warps copy a tile, token by token, into the layout a tile box load produces: NCH 64-wide
// chunks of the latent row (row stride lat_stride) as [chunk][tile rows][128 B] with the
// 128-byte swizzle, chunk_bytes apart, then RW 16-byte units of the rope row as
// [tile rows][16 RW bytes] at rope_dst (128-byte swizzle for 8 units, 64-byte for 4).  This
// warp copies the tokens k = k0, k0 + kstep, ... (nk <= 32 of them); lane i holds `myrow`, the
// cache row of its i-th token.  A 16-byte cp.async instruction moves at most 512 bytes and
// the SM retires only so many of them per cycle, so every instruction is made full: per token
// 512 consecutive bytes of the latent row (lane l: 16-byte unit l % 8 of chunk l / 8 + 4 j),
// and the rope rows of 32 / RW tokens at once.  The per-lane parts of the addresses are fixed
// for the whole call.
template <int NCH, int RW>
__device__ __forceinline__ void gather_tile(uint32_t st, uint32_t chunk_bytes, const __nv_bfloat16 *lat,
                                            size_t lat_stride, const __nv_bfloat16 *rope, size_t rope_stride,
                                            uint32_t rope_dst, int myrow, int k0, int kstep, int nk, int lane,
                                            uint64_t pol) {
    constexpr int UNITS = NCH * 8, NJ = (UNITS + 31) / 32, TPI = 32 / RW;
    const uint32_t dst_l = st + (uint32_t)(lane >> 3) * chunk_bytes;
    const uint32_t c_l = (uint32_t)(lane & 7);
    const __nv_bfloat16 *lat_l = lat + lane * 8;
#pragma unroll 2
    for (int i = 0; i < nk; ++i) {
        const uint32_t k = (uint32_t)(k0 + i * kstep);
        const size_t row = (size_t)__shfl_sync(0xffffffffu, myrow, i);
        const uint32_t dst = dst_l + k * 128u + ((c_l ^ (k & 7u)) << 4);
        const __nv_bfloat16 *src = lat_l + row * lat_stride;
#pragma unroll
        for (int j = 0; j < NJ; ++j)
            if (UNITS % 32 == 0 || lane + 32 * j < UNITS) cp_async16(dst + (uint32_t)(4 * j) * chunk_bytes, src + 256 * j, pol);
    }
    // rope: lane l copies unit l % RW of the warp's token i0 + l / RW
    const uint32_t ru = (uint32_t)(lane % RW);
    const __nv_bfloat16 *rope_l = rope + ru * 8;
    for (int i0 = 0; i0 < nk; i0 += TPI) {
        const int i = i0 + lane / RW;
        const size_t row = (size_t)__shfl_sync(0xffffffffu, myrow, i & 31);
        if (i < nk) {
            const uint32_t k = (uint32_t)(k0 + i * kstep);
            cp_async16(rope_dst + (RW == 8 ? sw128(k, ru) : sw64(k, ru)), rope_l + row * rope_stride, pol);
        }
    }
}

// Programmatic dependent launch.
__device__ __forceinline__ void pdl_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

#endif  // __CUDACC__

}  // namespace kvd

#ifdef __CUDACC__
namespace kvd {

// Single-thread bounded wait (for roles run by one elected lane).
__device__ __forceinline__ bool mbar_wait_one(uint64_t *bar, uint32_t parity, volatile int *abort, uint32_t *err,
                                              uint64_t limit_ns) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer();
    while (true) {
#pragma unroll 1
        for (int i = 0; i < 32; ++i)
            if (mbar_try_wait(bar, parity)) return true;
        if (*abort) return false;
        if (globaltimer() - t0 > limit_ns) {
            set_error(err, DEVERR_TIMEOUT);
            *abort = 1;
            return false;
        }
    }
}

// ----------------------------------------------------------------------------- softmax of a row slice
// A thread holds N raw scores s[k] (fp32 q.k) of one query row for tokens tok0 + k; the row sees
// tokens t <= lim.  c = softmax scale * log2(e), so exp(scale * s - m') = 2^(c * s - m).

// max over the visible k of c * s[k] (-inf if none).  On a tile with nothing masked (`full`) the
// raw scores are reduced first, since scaling by c is monotone (a min when c < 0).
template <int N>
__device__ __forceinline__ float tile_max(const float (&s)[N], bool full, int tok0, int lim, float c) {
    if (full) {
        float r[4] = {s[0], s[1], s[2], s[3]};
        if (c >= 0.f) {
#pragma unroll
            for (int k = 4; k < N; ++k) r[k & 3] = fmaxf(r[k & 3], s[k]);
            return fmaxf(fmaxf(r[0], r[1]), fmaxf(r[2], r[3])) * c;
        }
#pragma unroll
        for (int k = 4; k < N; ++k) r[k & 3] = fminf(r[k & 3], s[k]);
        return fminf(fminf(r[0], r[1]), fminf(r[2], r[3])) * c;
    }
    float m = -INFINITY;
#pragma unroll
    for (int k = 0; k < N; ++k)
        if (tok0 + k <= lim) m = fmaxf(m, s[k] * c);
    return m;
}

// s[k] <- 2^(c * s[k] - m) for visible k and 0 elsewhere (all 0 while m = -inf: nothing visible
// yet); returns the fp32 sum of the new s.
template <int N>
__device__ __forceinline__ float tile_exp(float (&s)[N], bool full, int tok0, int lim, float c, float m) {
    if (m == -INFINITY) {
#pragma unroll
        for (int k = 0; k < N; ++k) s[k] = 0.f;
        return 0.f;
    }
    const float nm = -m;
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    if (full) {
#pragma unroll
        for (int k = 0; k < N; ++k) {
            s[k] = ex2(fmaf(s[k], c, nm));
            acc[k & 3] += s[k];
        }
    } else {
#pragma unroll
        for (int k = 0; k < N; ++k) {
            s[k] = tok0 + k <= lim ? ex2(fmaf(s[k], c, nm)) : 0.f;
            acc[k & 3] += s[k];
        }
    }
    return (acc[0] + acc[1]) + (acc[2] + acc[3]);
}

// ----------------------------------------------------------------------------- tcgen05 (5th-gen tensor cores)
// Shared-memory matrix descriptor: start address, leading / stride byte offsets,
// version 1 (sm_100), layout type (2 = 128-byte swizzle, 4 = 64-byte swizzle).
__device__ __forceinline__ uint64_t umma_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo, uint32_t layout) {
    const uint32_t lo = ((saddr & 0x3FFFFu) >> 4) | (((lbo >> 4) & 0x3FFFu) << 16);
    const uint32_t hi = ((sbo >> 4) & 0x3FFFu) | (1u << 14) | (layout << 29);
    return ((uint64_t)hi << 32) | lo;
}
// Instruction descriptor for kind::f16 with bf16 A/B and fp32 accumulation.
__host__ __device__ constexpr uint32_t umma_idesc_bf16(int M, int N, bool a_mn_major, bool b_mn_major) {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((a_mn_major ? 1u : 0u) << 15) | ((b_mn_major ? 1u : 0u) << 16) |
           ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}
__device__ __forceinline__ void umma_bf16(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
        "l"(a), "l"(b), "r"(idesc), "r"(acc)
        : "memory");
}
// Arrive on `bar` once every tcgen05.mma issued so far by this thread has completed.
__device__ __forceinline__ void umma_commit(uint64_t *bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
                 : "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void fence_proxy_async() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

// Warp-wide TMEM allocation of `ncols` columns; the base address lands in *dst (shared).
__device__ __forceinline__ void tmem_alloc(uint32_t *dst, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst)), "r"(ncols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

// 32 consecutive fp32 columns of this thread's TMEM lane (warp w reads lanes 32*(w%4)..+31).
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
    uint32_t r[32];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
        "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
          "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const float (&v)[32]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
        "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};" ::"r"(taddr),
        "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])),
        "r"(__float_as_uint(v[3])), "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])),
        "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])), "r"(__float_as_uint(v[8])),
        "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])), "r"(__float_as_uint(v[11])),
        "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])), "r"(__float_as_uint(v[14])),
        "r"(__float_as_uint(v[15])), "r"(__float_as_uint(v[16])), "r"(__float_as_uint(v[17])),
        "r"(__float_as_uint(v[18])), "r"(__float_as_uint(v[19])), "r"(__float_as_uint(v[20])),
        "r"(__float_as_uint(v[21])), "r"(__float_as_uint(v[22])), "r"(__float_as_uint(v[23])),
        "r"(__float_as_uint(v[24])), "r"(__float_as_uint(v[25])), "r"(__float_as_uint(v[26])),
        "r"(__float_as_uint(v[27])), "r"(__float_as_uint(v[28])), "r"(__float_as_uint(v[29])),
        "r"(__float_as_uint(v[30])), "r"(__float_as_uint(v[31]))
        : "memory");
}
__device__ __forceinline__ void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// Half-warp split access (shape 16x32bx2) to the 16 TMEM lanes starting at taddr's lane: lanes
// 0-15 of the warp access N consecutive 32-bit columns from taddr's column, lanes 16-31 the
// same 16 TMEM lanes OFF columns further on: two threads per TMEM lane, one per column range.
template <int OFF>
__device__ __forceinline__ void tmem_ld16x2_32(uint32_t taddr, float (&v)[32]) {
    uint32_t r[32];
    asm volatile(
        "tcgen05.ld.sync.aligned.16x32bx2.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, "
        "%14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32], %33;"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
          "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr), "n"(OFF));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}
// As tmem_ld16x2_32 / tmem_ld16x2_16, without the wait: the registers are valid only after
// tmem_ld_wait(), so several loads can be in flight together.
template <int OFF>
__device__ __forceinline__ void tmem_ld16x2_32_nw(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.16x32bx2.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, "
        "%14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32], %33;"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
          "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr), "n"(OFF));
}
template <int OFF>
__device__ __forceinline__ void tmem_ld16x2_16_nw(uint32_t taddr, uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.16x32bx2.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, "
        "%14, %15}, [%16], %17;"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr), "n"(OFF));
}
__device__ __forceinline__ void tmem_ld_wait() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
template <int OFF>
__device__ __forceinline__ void tmem_ld16x2_16(uint32_t taddr, float (&v)[16]) {
    uint32_t r[16];
    asm volatile(
        "tcgen05.ld.sync.aligned.16x32bx2.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, "
        "%14, %15}, [%16], %17;"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr), "n"(OFF));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}
template <int OFF>
__device__ __forceinline__ void tmem_st16x2_32(uint32_t taddr, const float (&v)[32]) {
    asm volatile(
        "tcgen05.st.sync.aligned.16x32bx2.x32.b32 [%0], %33, {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, "
        "%13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};"
        ::"r"(taddr), "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])),
        "r"(__float_as_uint(v[3])), "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])),
        "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])), "r"(__float_as_uint(v[8])),
        "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])), "r"(__float_as_uint(v[11])),
        "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])), "r"(__float_as_uint(v[14])),
        "r"(__float_as_uint(v[15])), "r"(__float_as_uint(v[16])), "r"(__float_as_uint(v[17])),
        "r"(__float_as_uint(v[18])), "r"(__float_as_uint(v[19])), "r"(__float_as_uint(v[20])),
        "r"(__float_as_uint(v[21])), "r"(__float_as_uint(v[22])), "r"(__float_as_uint(v[23])),
        "r"(__float_as_uint(v[24])), "r"(__float_as_uint(v[25])), "r"(__float_as_uint(v[26])),
        "r"(__float_as_uint(v[27])), "r"(__float_as_uint(v[28])), "r"(__float_as_uint(v[29])),
        "r"(__float_as_uint(v[30])), "r"(__float_as_uint(v[31])), "n"(OFF)
        : "memory");
}
template <int OFF>
__device__ __forceinline__ void tmem_st16x2_16u(uint32_t taddr, const uint32_t (&v)[16]) {
    asm volatile(
        "tcgen05.st.sync.aligned.16x32bx2.x16.b32 [%0], %17, {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, "
        "%13, %14, %15, %16};" ::"r"(taddr),
        "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]),
        "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15]), "n"(OFF)
        : "memory");
}
template <int OFF>
__device__ __forceinline__ void tmem_st16x2_8u(uint32_t taddr, const uint32_t (&v)[8]) {
    asm volatile("tcgen05.st.sync.aligned.16x32bx2.x8.b32 [%0], %9, {%1, %2, %3, %4, %5, %6, %7, %8};" ::"r"(taddr),
                 "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "n"(OFF)
                 : "memory");
}

}  // namespace kvd
#endif  // __CUDACC__

#ifdef __CUDACC__
namespace kvd {
// O += A(TMEM) * B(smem descriptor): the A operand (K-major, bf16 pairs packed per
// 32-bit column, lane = row) is read from tensor memory.
__device__ __forceinline__ void umma_bf16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b, uint32_t idesc,
                                             uint32_t acc) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}\n" ::"r"(d_tmem),
        "r"(a_tmem), "l"(b), "r"(idesc), "r"(acc)
        : "memory");
}
__device__ __forceinline__ void tmem_st16u(uint32_t taddr, const uint32_t (&v)[16]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, "
        "%14, %15, %16};" ::"r"(taddr),
        "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]),
        "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15])
        : "memory");
}
}  // namespace kvd
#endif  // __CUDACC__

#ifdef __CUDACC__
namespace kvd {
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float (&v)[16]) {
    uint32_t r[16];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
        "%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}
__device__ __forceinline__ void tmem_st8u(uint32_t taddr, const uint32_t (&v)[8]) {
    asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"r"(taddr),
                 "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7])
                 : "memory");
}
}  // namespace kvd
#endif  // __CUDACC__

#ifdef __CUDACC__
namespace kvd {
// ----------------------------------------------------------------------------- thread-block clusters
__device__ __forceinline__ uint32_t cluster_rank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
// The shared::cluster address of `saddr` (a shared::cta address) in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t mapa_shared(uint32_t saddr, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(saddr), "r"(rank));
    return r;
}
__device__ __forceinline__ void st_cluster_v4(uint32_t caddr, float a, float b, float c, float d) {
    asm volatile("st.shared::cluster.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(caddr), "f"(a), "f"(b), "f"(c), "f"(d)
                 : "memory");
}
// Arrive on an mbarrier of another CTA of the cluster (default semantics: release at CTA scope).
// This is how a consumer hands a buffer back to a producer in the other CTA: its reads of the
// buffer are done before the arrival.  A cluster-scope release would also wait for every earlier
// memory operation of the thread to become visible cluster-wide, which costs thousands of cycles.
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t caddr_bar) {
    asm volatile("mbarrier.arrive.shared::cluster.b64 _, [%0];" ::"r"(caddr_bar) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait_cluster(uint64_t *bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}\n"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}
// As mbar_wait_warp, acquiring at cluster scope (for barriers that another CTA arrives on).
__device__ __forceinline__ bool mbar_wait_warp_cluster(uint64_t *bar, uint32_t parity, volatile int *abort,
                                                       uint32_t *err, uint64_t limit_ns) {
    if (__all_sync(0xffffffffu, mbar_try_wait_cluster(bar, parity))) return true;
    const uint64_t t0 = globaltimer();
    while (true) {
#pragma unroll 1
        for (int i = 0; i < 32; ++i)
            if (__all_sync(0xffffffffu, mbar_try_wait_cluster(bar, parity))) return true;
        int stop = 0;
        if ((threadIdx.x & 31) == 0) {
            if (*abort) {
                stop = 1;
            } else if (globaltimer() - t0 > limit_ns) {
                set_error(err, DEVERR_TIMEOUT);
                *abort = 1;
                stop = 1;
            }
        }
        if (__shfl_sync(0xffffffffu, stop, 0)) return false;
    }
}
__device__ __forceinline__ void cluster_sync() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
}  // namespace kvd
#endif  // __CUDACC__

#ifdef __CUDACC__
namespace kvd {
// Asynchronous store of 16 bytes into another CTA's shared memory; completes `bytes` of the
// transaction count of that CTA's mbarrier at caddr_bar (same CTA as the destination).
__device__ __forceinline__ void st_async_v4(uint32_t caddr, float a, float b, float c, float d, uint32_t caddr_bar) {
    asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.v4.f32 [%0], {%1, %2, %3, %4}, [%5];" ::"r"(
                     caddr),
                 "f"(a), "f"(b), "f"(c), "f"(d), "r"(caddr_bar)
                 : "memory");
}
// Bulk copy (the async copy engine) of `bytes` (a multiple of 16, both addresses 16-byte
// aligned) from this CTA's shared memory to another CTA's; completes `bytes` of the
// transaction count of the destination CTA's mbarrier at caddr_bar.  The source may be
// rewritten once that mbarrier's phase has completed.
__device__ __forceinline__ void bulk_copy_to_peer(uint32_t caddr_dst, uint32_t saddr_src, uint32_t bytes,
                                                  uint32_t caddr_bar) {
    asm volatile("cp.async.bulk.shared::cluster.shared::cta.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                     caddr_dst),
                 "r"(saddr_src), "r"(bytes), "r"(caddr_bar)
                 : "memory");
}
}  // namespace kvd
#endif  // __CUDACC__
