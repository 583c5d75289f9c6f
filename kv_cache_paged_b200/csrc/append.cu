// Cache append with RoPE (the step before decode) and in-place RoPE of the queries.
//
// "Hardware-Efficient Attention for Fast Decoding", sections 3.3.1 (GTA: tied state per
// group plus one shared RoPE key slice per token) and 3.3.2 (GLA/MLA: latent heads plus
// one shared RoPE key slice); the GQA baseline stores K and V heads with RoPE on the key.
// One warp per new token; a token has two fields, each a [heads, dim] bf16 row whose last
// `rope_w` dims of every head are rotated and the rest copied.  The copy moves 16-byte
// units; the rotation works on the (j, j + rope_w / 2) pairs in fp64 (angle, sin, cos and
// products; theta_j from the host, in fp64, by the same formula as the reference) and
// rounds once to bf16.  Each pair's sine and cosine are computed once per token and reused
// by every head.  A few KB per token: HBM-bound for large appends, launch-bound for one
// decode step's tokens.
#include <cuda_bf16.h>

#include <algorithm>
#include <cmath>

#include "common.cuh"
#include "kernels.h"
#include "kvappend.h"

namespace kvd {

namespace {

struct AppendField {
    const __nv_bfloat16 *src;  // [N, heads, dim]
    __nv_bfloat16 *dst;        // [num_rows, heads, dim]
    int heads, dim, rope_w;
};

constexpr int MAX_HALF = 64;  // d_r <= 128

struct AppendArgs {
    AppendField f[2];
    const int32_t *pos, *slot;
    uint32_t *err;
    int N, num_rows;
    double theta[MAX_HALF];  // rope_base^(-2 j / d_r), computed on the host in fp64
};

// y = rotation of the pair (x0, x1) by the angle with sine s and cosine c, rounded to bf16.
__device__ __forceinline__ void rotate(float x0, float x1, double s, double c, __nv_bfloat16 &y0,
                                       __nv_bfloat16 &y1) {
    y0 = __double2bfloat16((double)x0 * c - (double)x1 * s);
    y1 = __double2bfloat16((double)x1 * c + (double)x0 * s);
}

// One warp per new token at a time (grid-stride over tokens, a few CTAs per SM): the lanes
// copy the plain dims in 16-byte units, then lane j computes the sine and cosine of pair j
// once and rotates that pair in every head of the field.
__device__ __forceinline__ void append_token(const AppendArgs &a, int n, int lane) {
    const int slot = __ldg(a.slot + n);
    if (slot < 0) return;
    if (slot >= a.num_rows) {
        if (lane == 0 && a.err) set_error(a.err, DEVERR_BAD_PAGE);
        return;
    }
    const double pos = (double)__ldg(a.pos + n);
#pragma unroll
    for (int fi = 0; fi < 2; ++fi) {
        const AppendField &f = a.f[fi];
        const size_t row = (size_t)f.heads * f.dim;
        const __nv_bfloat16 *src = f.src + (size_t)n * row;
        __nv_bfloat16 *dst = f.dst + (size_t)slot * row;
        const int plain = f.dim - f.rope_w, units = plain / 8;
        for (int u = lane; u < f.heads * units; u += 32) {
            const int h = u / units, k = u - h * units;
            *(uint4 *)(dst + (size_t)h * f.dim + 8 * k) = __ldg((const uint4 *)(src + (size_t)h * f.dim) + k);
        }
        const int half = f.rope_w / 2;
        for (int j = lane; j < half; j += 32) {
            double sn, cs;
            sincos(pos * a.theta[j], &sn, &cs);
            for (int h = 0; h < f.heads; ++h) {
                const __nv_bfloat16 *x = src + (size_t)h * f.dim + plain;
                __nv_bfloat16 *y = dst + (size_t)h * f.dim + plain;
                rotate(__bfloat162float(x[j]), __bfloat162float(x[j + half]), sn, cs, y[j], y[j + half]);
            }
        }
    }
}

__global__ void __launch_bounds__(256) append_kernel(const AppendArgs a) {
    const int lane = threadIdx.x & 31;
    const int warps = gridDim.x * 8;
    for (int n = blockIdx.x * 8 + (threadIdx.x >> 5); n < a.N; n += warps) append_token(a, n, lane);
}

struct RopeQArgs {
    __nv_bfloat16 *q;
    const int32_t *seqlens;
    int rows, L, heads, d_qk, off, w;
    double theta[MAX_HALF];
};

// q [B, L, heads, d_qk]: rotate dims [off, off + w) of every head of row (b, i) to position
// seqlens[b] - L + i; one warp per row.
__global__ void __launch_bounds__(256) rope_q_kernel(const RopeQArgs a) {
    const int lane = threadIdx.x & 31;
    const int row = blockIdx.x * 8 + (threadIdx.x >> 5);
    if (row >= a.rows) return;
    const int b = row / a.L, i = row - b * a.L;
    const int p = __ldg(a.seqlens + b) - a.L + i;
    if (p < 0) return;
    const int half = a.w / 2;
    __nv_bfloat16 *base_row = a.q + (size_t)row * a.heads * a.d_qk + a.off;
    for (int j = lane; j < half; j += 32) {
        double sn, cs;
        sincos((double)p * a.theta[j], &sn, &cs);
        for (int h = 0; h < a.heads; ++h) {
            __nv_bfloat16 *x = base_row + (size_t)h * a.d_qk;
            rotate(__bfloat162float(x[j]), __bfloat162float(x[j + half]), sn, cs, x[j], x[j + half]);
        }
    }
}

void fill_theta(double *theta, int w, double base) {
    for (int j = 0; j < w / 2; ++j) theta[j] = std::pow(base, -2.0 * (double)j / (double)w);
}

bool aligned16(const void *p) { return p && ((uintptr_t)p & 15u) == 0; }

int launch_append(AppendArgs &a, int rope_w, double base, cudaStream_t st) {
    if (a.N == 0) return KVD_OK;
    fill_theta(a.theta, rope_w, base);
    const int sms = num_sms_current();
    if (sms <= 0) return KVD_ERR_CUDA;
    const int blocks = std::min((a.N + 7) / 8, sms * 8);
    append_kernel<<<(unsigned)blocks, 256, 0, st>>>(a);
    return cudaGetLastError() == cudaSuccess ? KVD_OK : KVD_ERR_CUDA;
}

// shared checks: counts, rope base, the index arrays and one field's layout
bool common_ok(int N, int num_rows, float base, const int32_t *pos, const int32_t *slot) {
    if (N < 0 || num_rows <= 0 || !(base > 0.f) || !std::isfinite(base)) return false;
    if (N > 0 && (!pos || !slot || ((uintptr_t)pos & 3u) || ((uintptr_t)slot & 3u))) return false;
    return true;
}
bool field_ok(const void *src, const void *dst, int heads, int dim, int rope_w) {
    return aligned16(src) && aligned16(dst) && heads > 0 && dim > 0 && dim % 8 == 0 && rope_w >= 0 &&
           rope_w <= dim && rope_w <= 2 * MAX_HALF && rope_w % 2 == 0 && (dim - rope_w) % 8 == 0;
}

}  // namespace

}  // namespace kvd

using namespace kvd;

extern "C" int kvd_gqa_append(const kvd_gqa_append_params *p, kvd_stream_t stream) {
    if (!p || !common_ok(p->N, p->num_rows, p->rope_base, p->positions, p->slot_mapping) ||
        !field_ok(p->k_new, p->k_cache, p->h_kv, p->d, p->d_r) || !field_ok(p->v_new, p->v_cache, p->h_kv, p->d, 0))
        return KVD_ERR_INVALID_ARG;
    AppendArgs a{};
    a.f[0] = {(const __nv_bfloat16 *)p->k_new, (__nv_bfloat16 *)p->k_cache, p->h_kv, p->d, p->d_r};
    a.f[1] = {(const __nv_bfloat16 *)p->v_new, (__nv_bfloat16 *)p->v_cache, p->h_kv, p->d, 0};
    a.pos = p->positions, a.slot = p->slot_mapping, a.err = p->error_word;
    a.N = p->N, a.num_rows = p->num_rows;
    return launch_append(a, p->d_r, p->rope_base, (cudaStream_t)stream);
}

extern "C" int kvd_gta_append(const kvd_gta_append_params *p, kvd_stream_t stream) {
    if (!p || !common_ok(p->N, p->num_rows, p->rope_base, p->positions, p->slot_mapping) ||
        !field_ok(p->tied_new, p->tied_cache, p->h_kv, p->d_h, 0) ||
        !field_ok(p->rope_new, p->rope_cache, 1, p->d_r, p->d_r) || p->d_r <= 0)
        return KVD_ERR_INVALID_ARG;
    AppendArgs a{};
    a.f[0] = {(const __nv_bfloat16 *)p->tied_new, (__nv_bfloat16 *)p->tied_cache, p->h_kv, p->d_h, 0};
    a.f[1] = {(const __nv_bfloat16 *)p->rope_new, (__nv_bfloat16 *)p->rope_cache, 1, p->d_r, p->d_r};
    a.pos = p->positions, a.slot = p->slot_mapping, a.err = p->error_word;
    a.N = p->N, a.num_rows = p->num_rows;
    return launch_append(a, p->d_r, p->rope_base, (cudaStream_t)stream);
}

extern "C" int kvd_gla_append(const kvd_gla_append_params *p, kvd_stream_t stream) {
    if (!p || !common_ok(p->N, p->num_rows, p->rope_base, p->positions, p->slot_mapping) ||
        !field_ok(p->latent_new, p->latent_cache, p->h_c, p->d_c, 0) ||
        !field_ok(p->rope_new, p->rope_cache, 1, p->d_r, p->d_r) || p->d_r <= 0)
        return KVD_ERR_INVALID_ARG;
    AppendArgs a{};
    a.f[0] = {(const __nv_bfloat16 *)p->latent_new, (__nv_bfloat16 *)p->latent_cache, p->h_c, p->d_c, 0};
    a.f[1] = {(const __nv_bfloat16 *)p->rope_new, (__nv_bfloat16 *)p->rope_cache, 1, p->d_r, p->d_r};
    a.pos = p->positions, a.slot = p->slot_mapping, a.err = p->error_word;
    a.N = p->N, a.num_rows = p->num_rows;
    return launch_append(a, p->d_r, p->rope_base, (cudaStream_t)stream);
}

extern "C" int kvd_rope_q(void *q, const int32_t *seqlens, int32_t B, int32_t L, int32_t heads, int32_t d_qk,
                          int32_t rope_off, int32_t d_r, float rope_base, kvd_stream_t stream) {
    if (!q || ((uintptr_t)q & 15u) || !seqlens || ((uintptr_t)seqlens & 3u) || B < 0 || L <= 0 || heads <= 0 ||
        d_qk <= 0 || d_r <= 0 || d_r % 2 || d_r > 2 * MAX_HALF || rope_off < 0 || rope_off + d_r > d_qk || !(rope_base > 0.f) ||
        !std::isfinite(rope_base))
        return KVD_ERR_INVALID_ARG;
    if (B == 0) return KVD_OK;
    RopeQArgs a{};
    a.q = (__nv_bfloat16 *)q, a.seqlens = seqlens, a.rows = B * L, a.L = L, a.heads = heads, a.d_qk = d_qk;
    a.off = rope_off, a.w = d_r;
    fill_theta(a.theta, d_r, rope_base);
    rope_q_kernel<<<(unsigned)((B * L + 7) / 8), 256, 0, (cudaStream_t)stream>>>(a);
    return cudaGetLastError() == cudaSuccess ? KVD_OK : KVD_ERR_CUDA;
}
