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

constexpr int CROWS = 8;   // rows per CTA, one warp each for the lse step
constexpr int MAXW = 64;   // weights cached in shared memory per row

__global__ void __launch_bounds__(256) combine_kernel(const CombineArgs a) {
    __shared__ float w_sh[CROWS][MAXW];
    __shared__ float lse_sh[CROWS];
    __shared__ int first_sh, nsplit_sh;

    // Wait for the decode grid to finish and its partials to be visible.
    pdl_wait();

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int b = blockIdx.x;
    const int row0 = blockIdx.y * CROWS;
    const int nrow = min(CROWS, a.rows - row0);

    if (warp == 0) {
        int64_t N = 0, cu = 0;
        int32_t nb = 0;
        for (int base = 0; base < a.B; base += 32) {
            const int idx = base + lane;
            int32_t n = 0;
            if (idx < a.B) n = tiles_of(clamp_len(__ldg(a.seqlens + idx), a.max_tokens, a.L, nullptr), a.tile);
            int32_t before = idx < b ? n : 0;
            int32_t mine = idx == b ? n : 0;
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
    const int first = first_sh;
    const size_t rows = (size_t)a.rows;

    if (warp < nrow) {
        const int r = row0 + warp;
        float m = -INFINITY;
        for (int s = lane; s < nsplit; s += 32) m = fmaxf(m, a.ws_lse[(size_t)(b + first + s) * rows + r]);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        float sum = 0.f;
        if (m != -INFINITY)
            for (int s = lane; s < nsplit; s += 32) sum += expf(a.ws_lse[(size_t)(b + first + s) * rows + r] - m);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
        const float L = m == -INFINITY ? -INFINITY : m + logf(sum);
        for (int s = lane; s < min(nsplit, MAXW); s += 32)
            w_sh[warp][s] = L == -INFINITY ? 0.f : expf(a.ws_lse[(size_t)(b + first + s) * rows + r] - L);
        if (lane == 0) {
            lse_sh[warp] = L;
            a.lse[(size_t)b * rows + r] = L;
        }
    }
    __syncthreads();

    // out = sum_s w_s O_s: four consecutive columns per thread, the loads of all splits
    // independent of each other so that they are in flight together
    const int dv4 = a.d_v / 4;
    for (int idx = threadIdx.x; idx < nrow * dv4; idx += blockDim.x) {
        const int w = idx / dv4, c4 = idx % dv4;
        const int r = row0 + w;
        const float L = lse_sh[w];
        const float4 *src = (const float4 *)(a.ws_o + ((size_t)(b + first) * rows + r) * a.d_v) + c4;
        const size_t step4 = rows * a.d_v / 4;
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 4
        for (int s = 0; s < nsplit; ++s) {
            const float wt = s < MAXW ? w_sh[w][s]
                                      : (L == -INFINITY ? 0.f : expf(a.ws_lse[(size_t)(b + first + s) * rows + r] - L));
            const float4 x = __ldcs(src + (size_t)s * step4);
            acc.x += wt * x.x;
            acc.y += wt * x.y;
            acc.z += wt * x.z;
            acc.w += wt * x.w;
        }
        uint2 o;
        o.x = pack_bf16(acc.x, acc.y);
        o.y = pack_bf16(acc.z, acc.w);
        *(uint2 *)(a.out + ((size_t)b * rows + r) * a.d_v + 4 * c4) = o;
    }
}

__global__ void plan_kernel(const int32_t *seqlens, int B, int tile, int max_tokens, int L, int parts,
                            int32_t *segs, int32_t *counts, int cap) {
    const int c = blockIdx.x;
    int cnt = 0;
    plan_walk(seqlens, B, tile, max_tokens, L, c, parts, nullptr, [&](const Seg &s) {
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

}  // namespace

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

cudaError_t launch_plan(const int32_t *seqlens, int B, int tile, int max_tokens, int L, int parts, int32_t *segs,
                        int32_t *counts, int cap, cudaStream_t st) {
    plan_kernel<<<parts, 32, 0, st>>>(seqlens, B, tile, max_tokens, L, parts, segs, counts, cap);
    return cudaGetLastError();
}

}  // namespace kvd
