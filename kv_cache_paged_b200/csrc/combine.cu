// LSE combine of split-KV partials, and the plan-inspection kernel.
//
// A sequence whose tile range was cut into n parts has n partial results
// (O_s normalised by its own softmax denominator, lse_s = ln of that
// denominator).  The whole is the softmax-denominator-weighted mix:
//   lse = ln sum_s exp(lse_s),  out = sum_s exp(lse_s - lse) O_s,
// the decomposition Hydragen uses to merge prefix and suffix attention.  An
// empty part (lse_s = -inf) has weight 0; a sequence with no tokens gets
// out = 0 and lse = -inf.  Memory-bound and small next to the KV stream.
#include <cuda_bf16.h>

#include "common.cuh"
#include "kernels.h"

namespace kvd {

namespace {

// 4 rows per CTA (one 16-byte column group of one row per thread at d_v 256), loads of 4 parts
// per round trip, at most 40 registers: 6 CTAs per SM, so that the grid runs in fewer waves
// once the decode grid has drained (the combine's time is a chain of round trips per CTA)
constexpr int CROWS = 4;
constexpr int CPARTS = 4;

__global__ void __launch_bounds__(256, 6) combine_kernel(const CombineArgs a) {
    __shared__ int first_sh, nsplit_sh;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int b = blockIdx.x;
    const int row0 = blockIdx.y * CROWS;
    const int nrow = min(CROWS, a.rows - row0);

    if (warp == 0) {
        // the sequence's part range from seqlens: PLAN_K lengths per lane per round trip
        int64_t N = 0, cu = 0;
        int32_t nb = 0;
        for (int base = 0; base < a.B; base += 32 * PLAN_K) {
            int32_t raw[PLAN_K];
#pragma unroll
            for (int k = 0; k < PLAN_K; ++k) {
                const int idx = base + 32 * k + lane;
                raw[k] = idx < a.B ? __ldg(a.seqlens + idx) : 0;
            }
            int32_t n = 0, before = 0, mine = 0;
#pragma unroll
            for (int k = 0; k < PLAN_K; ++k) {
                const int idx = base + 32 * k + lane;
                const int32_t t = idx < a.B ? tiles_of(clamp_len(raw[k], a.max_tokens, a.L, nullptr), a.tile) : 0;
                const int32_t u = (int32_t)units_of(t, a.seg_cost);
                n += u;
                before += idx < b ? u : (idx == b ? u - t : 0);  // up to this sequence's first tile
                mine += idx == b ? t : 0;
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                n += __shfl_xor_sync(0xffffffffu, n, o);
                before += __shfl_xor_sync(0xffffffffu, before, o);
                mine += __shfl_xor_sync(0xffffffffu, mine, o);
            }
            N += n;
            cu += before;
            nb += mine;
        }
        if (lane == 0) {
            if (nb == 0) {
                first_sh = 0;
                nsplit_sh = 0;
            } else {
                const int64_t P = a.parts < N ? a.parts : N;
                const int64_t f = part_of(cu, N, P), l = part_of(cu + nb - 1, N, P);
                first_sh = (int)f;
                nsplit_sh = (int)(l - f + 1);
            }
        }
    }
    __syncthreads();
    const int nsplit = nsplit_sh;
    if (nsplit == 1) return;  // the decode kernel wrote this sequence's output itself
    // The part range above needs only seqlens (an input), so it overlaps the decode grid's tail;
    // the partials are read only once the decode grid has finished and they are visible.
    pdl_wait();
    const int first = first_sh;
    const size_t rows = (size_t)a.rows;

    // Each thread owns four consecutive outputs of one row and loads that row's lse and its four
    // columns from CPARTS parts per round trip (one round trip for up to CPARTS parts), reducing
    // locally.
    const int dv4 = a.d_v / 4;
    for (int idx = threadIdx.x; idx < nrow * dv4; idx += blockDim.x) {
        const int r = row0 + idx / dv4, c4 = idx % dv4;
        float mx = -INFINITY, sum = 0.f;
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int s0 = 0; s0 < nsplit; s0 += CPARTS) {
            float ls[CPARTS];
            float4 x[CPARTS];
#pragma unroll
            for (int k = 0; k < CPARTS; ++k) {
                const size_t slot = (size_t)(b + first) + min(s0 + k, nsplit - 1);
                ls[k] = s0 + k < nsplit ? __ldcs(a.ws_lse + slot * rows + r) : -INFINITY;
                x[k] = __ldcs((const float4 *)(a.ws_o + (slot * rows + r) * a.d_v) + c4);
            }
            // streaming log-sum-exp over the parts, rescaling what is summed so far
#pragma unroll
            for (int k = 0; k < CPARTS; ++k) {
                if (ls[k] == -INFINITY) continue;
                const float mn = fmaxf(mx, ls[k]);
                const float sc = mx == -INFINITY ? 0.f : expf(mx - mn);
                const float wk = expf(ls[k] - mn);
                sum = sum * sc + wk;
                acc.x = acc.x * sc + wk * x[k].x;
                acc.y = acc.y * sc + wk * x[k].y;
                acc.z = acc.z * sc + wk * x[k].z;
                acc.w = acc.w * sc + wk * x[k].w;
                mx = mn;
            }
        }
        const float inv = sum > 0.f ? 1.f / sum : 0.f;
        uint2 o;
        o.x = pack_bf16(acc.x * inv, acc.y * inv);
        o.y = pack_bf16(acc.z * inv, acc.w * inv);
        *(uint2 *)(a.out + ((size_t)b * rows + r) * a.d_v + 4 * c4) = o;
        if (c4 == 0) a.lse[(size_t)b * rows + r] = mx == -INFINITY ? -INFINITY : mx + logf(sum);
    }
}

__global__ void plan_kernel(const int32_t *seqlens, int B, int tile, int seg_cost, int max_tokens, int L, int parts,
                            int32_t *segs, int32_t *counts, int cap) {
    const int c = blockIdx.x;
    int cnt = 0;
    plan_walk(seqlens, B, tile, seg_cost, max_tokens, L, c, parts, nullptr, [&](const Seg &s) {
        if (cnt < cap) {
            int32_t *o = segs + ((size_t)c * cap + cnt) * 6;
            o[0] = s.b;
            o[1] = s.t0;
            o[2] = s.t1;
            o[3] = s.split;
            o[4] = s.nsplit;
            o[5] = s.slot;
        }
        ++cnt;
    });
    if ((threadIdx.x & 31) == 0) counts[c] = cnt;
}

// Merge two attention states over disjoint key sets of the same query rows (a shared
// prefix and a sequence's own continuation): with m = max(lse_a, lse_b),
// lse = m + ln(e^(lse_a - m) + e^(lse_b - m)) and out = e^(lse_a - lse) out_a + e^(lse_b - lse) out_b.
// A state with lse = -inf (no key) has weight 0; two empty states give out = 0, lse = -inf.
// One thread per 8 output elements (16 bytes of bf16).
__global__ void __launch_bounds__(256) merge_kernel(const __nv_bfloat16 *out_a, const float *lse_a,
                                                    const __nv_bfloat16 *out_b, const float *lse_b,
                                                    __nv_bfloat16 *out, float *lse, int rows, int d_v) {
    const int per_row = d_v / 8;
    const long long u = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (u >= (long long)rows * per_row) return;
    const int row = (int)(u / per_row), k = (int)(u % per_row);
    const float la = __ldg(lse_a + row), lb = __ldg(lse_b + row);
    const float m = fmaxf(la, lb);
    float wa = 0.f, wb = 0.f, l = -INFINITY;
    if (m != -INFINITY) {
        const float ea = expf(la - m), eb = expf(lb - m);
        const float inv = 1.f / (ea + eb);
        wa = ea * inv;
        wb = eb * inv;
        l = m + logf(ea + eb);
    }
    const uint4 va = __ldg((const uint4 *)(out_a + (size_t)row * d_v) + k);
    const uint4 vb = __ldg((const uint4 *)(out_b + (size_t)row * d_v) + k);
    const uint32_t xa[4] = {va.x, va.y, va.z, va.w}, xb[4] = {vb.x, vb.y, vb.z, vb.w};
    uint32_t y[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        // a state of weight 0 contributes nothing (its out may hold anything, e.g. zeros)
        const float lo = (wa > 0.f ? wa * bf16_lo(xa[i]) : 0.f) + (wb > 0.f ? wb * bf16_lo(xb[i]) : 0.f);
        const float hi = (wa > 0.f ? wa * bf16_hi(xa[i]) : 0.f) + (wb > 0.f ? wb * bf16_hi(xb[i]) : 0.f);
        y[i] = pack_bf16(lo, hi);
    }
    *((uint4 *)(out + (size_t)row * d_v) + k) = make_uint4(y[0], y[1], y[2], y[3]);
    if (k == 0) lse[row] = l;
}

}  // namespace

cudaError_t launch_merge(const void *out_a, const float *lse_a, const void *out_b, const float *lse_b, void *out,
                         float *lse, int rows, int d_v, cudaStream_t st) {
    if (rows == 0) return cudaSuccess;
    const long long units = (long long)rows * (d_v / 8);
    merge_kernel<<<(unsigned)((units + 255) / 256), 256, 0, st>>>(
        (const __nv_bfloat16 *)out_a, lse_a, (const __nv_bfloat16 *)out_b, lse_b, (__nv_bfloat16 *)out, lse, rows, d_v);
    return cudaGetLastError();
}

cudaError_t launch_combine(const CombineArgs &a, cudaStream_t st) {
    if (a.B == 0 || a.rows == 0) return cudaSuccess;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)a.B, (unsigned)((a.rows + CROWS - 1) / CROWS), 1);
    cfg.blockDim = dim3(256, 1, 1);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t e = cudaLaunchKernelEx(&cfg, combine_kernel, a);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

cudaError_t launch_plan(const int32_t *seqlens, int B, int tile, int seg_cost, int max_tokens, int L, int parts,
                        int32_t *segs, int32_t *counts, int cap, cudaStream_t st) {
    plan_kernel<<<parts, 32, 0, st>>>(seqlens, B, tile, seg_cost, max_tokens, L, parts, segs, counts, cap);
    return cudaGetLastError();
}

}  // namespace kvd
