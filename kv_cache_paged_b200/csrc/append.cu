// Cache append with RoPE (the step before decode) and in-place RoPE of the queries.
//
// "Hardware-Efficient Attention for Fast Decoding", sections 3.3.1 (GTA: tied state per
// group plus one shared RoPE key slice per token) and 3.3.2 (GLA/MLA: latent heads plus
// one shared RoPE key slice); the GQA baseline stores K and V heads with RoPE on the key.
// One CTA per (new token, field): a field is a [heads, dim] bf16 row whose last `rope_w`
// dims of every head are rotated and the rest copied.  The copy moves 16-byte units; the
// rotation works on the (j, j + rope_w / 2) pairs in fp64 (angle, sin, cos and products)
// and rounds once to bf16.  The work is a few hundred bytes per token: HBM-bound for
// large appends, launch-bound for one decode step's tokens.
#include <cuda_bf16.h>

#include <cmath>

#include "common.cuh"
#include "kvappend.h"

namespace kvd {

namespace {

struct AppendField {
    const __nv_bfloat16 *src;  // [N, heads, dim]
    __nv_bfloat16 *dst;        // [num_rows, heads, dim]
    int heads, dim, rope_w;
};

struct AppendArgs {
    AppendField f[2];
    const int32_t *pos, *slot;
    uint32_t *err;
    int N, num_rows;
    double base;
};

// y = rotation of the pair (x0, x1) by position * base^(-2 j / w), rounded to bf16.
__device__ __forceinline__ void rope_pair(float x0, float x1, int j, int w, double pos, double base,
                                          __nv_bfloat16 &y0, __nv_bfloat16 &y1) {
    const double theta = pow(base, -2.0 * (double)j / (double)w);
    double s, c;
    sincos(pos * theta, &s, &c);
    y0 = __double2bfloat16((double)x0 * c - (double)x1 * s);
    y1 = __double2bfloat16((double)x1 * c + (double)x0 * s);
}

__global__ void __launch_bounds__(128) append_kernel(const AppendArgs a) {
    const int n = blockIdx.x;
    const AppendField f = a.f[blockIdx.y];
    const int slot = __ldg(a.slot + n);
    if (slot < 0) return;
    if (slot >= a.num_rows) {
        if (threadIdx.x == 0 && a.err) set_error(a.err, DEVERR_BAD_PAGE);
        return;
    }
    const size_t row = (size_t)f.heads * f.dim;
    const __nv_bfloat16 *src = f.src + (size_t)n * row;
    __nv_bfloat16 *dst = f.dst + (size_t)slot * row;
    // copied dims: 16-byte units of the first dim - rope_w dims of every head
    const int plain = f.dim - f.rope_w, units = plain / 8;
    for (int u = threadIdx.x; u < f.heads * units; u += blockDim.x) {
        const int h = u / units, k = u % units;
        *(uint4 *)(dst + (size_t)h * f.dim + 8 * k) = __ldg((const uint4 *)(src + (size_t)h * f.dim) + k);
    }
    if (f.rope_w == 0) return;
    const int half = f.rope_w / 2;
    const double pos = (double)__ldg(a.pos + n);
    for (int u = threadIdx.x; u < f.heads * half; u += blockDim.x) {
        const int h = u / half, j = u % half;
        const __nv_bfloat16 *x = src + (size_t)h * f.dim + plain;
        __nv_bfloat16 *y = dst + (size_t)h * f.dim + plain;
        rope_pair(__bfloat162float(x[j]), __bfloat162float(x[j + half]), j, f.rope_w, pos, a.base, y[j], y[j + half]);
    }
}

// q [B, L, heads, d_qk]: rotate dims [off, off + w) of every head of row (b, i) to position
// seqlens[b] - L + i; one CTA per row.
__global__ void __launch_bounds__(128) rope_q_kernel(__nv_bfloat16 *q, const int32_t *seqlens, int L, int heads,
                                                     int d_qk, int off, int w, double base) {
    const int row = blockIdx.x, b = row / L, i = row % L;
    const int p = __ldg(seqlens + b) - L + i;
    if (p < 0) return;
    const int half = w / 2;
    __nv_bfloat16 *base_row = q + (size_t)row * heads * d_qk + off;
    for (int u = threadIdx.x; u < heads * half; u += blockDim.x) {
        const int h = u / half, j = u % half;
        __nv_bfloat16 *x = base_row + (size_t)h * d_qk;
        const float x0 = __bfloat162float(x[j]), x1 = __bfloat162float(x[j + half]);
        rope_pair(x0, x1, j, w, (double)p, base, x[j], x[j + half]);
    }
}

bool aligned16(const void *p) { return p && ((uintptr_t)p & 15u) == 0; }

int launch_append(const AppendArgs &a, int nf, cudaStream_t st) {
    if (a.N == 0) return KVD_OK;
    append_kernel<<<dim3((unsigned)a.N, (unsigned)nf), 128, 0, st>>>(a);
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
           rope_w <= dim && rope_w % 2 == 0 && (dim - rope_w) % 8 == 0;
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
    a.N = p->N, a.num_rows = p->num_rows, a.base = p->rope_base;
    return launch_append(a, 2, (cudaStream_t)stream);
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
    a.N = p->N, a.num_rows = p->num_rows, a.base = p->rope_base;
    return launch_append(a, 2, (cudaStream_t)stream);
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
    a.N = p->N, a.num_rows = p->num_rows, a.base = p->rope_base;
    return launch_append(a, 2, (cudaStream_t)stream);
}

extern "C" int kvd_rope_q(void *q, const int32_t *seqlens, int32_t B, int32_t L, int32_t heads, int32_t d_qk,
                          int32_t rope_off, int32_t d_r, float rope_base, kvd_stream_t stream) {
    if (!q || ((uintptr_t)q & 15u) || !seqlens || ((uintptr_t)seqlens & 3u) || B < 0 || L <= 0 || heads <= 0 ||
        d_qk <= 0 || d_r <= 0 || d_r % 2 || rope_off < 0 || rope_off + d_r > d_qk || !(rope_base > 0.f) ||
        !std::isfinite(rope_base))
        return KVD_ERR_INVALID_ARG;
    if (B == 0) return KVD_OK;
    rope_q_kernel<<<(unsigned)(B * L), 128, 0, (cudaStream_t)stream>>>((__nv_bfloat16 *)q, seqlens, L, heads, d_qk,
                                                                       rope_off, d_r, (double)rope_base);
    return cudaGetLastError() == cudaSuccess ? KVD_OK : KVD_ERR_CUDA;
}
