// Internal interface between the C-ABI layer (api.cu) and the kernels.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace kvd {

// SM count of the calling thread's current device (cached per device; -1 on a CUDA error).
int num_sms_current();

constexpr int MAX_STAGES = 8;

// Test knobs (kvd_debug_set): make the first tile's copy never start so that the
// bounded waits run out, exercising the timeout path without a GPU fault.
constexpr int DEBUG_SKIP_FIRST_LOAD = 1;

struct GroupArgs {
    const __nv_bfloat16 *q;
    const int32_t *block_table;
    const int32_t *seqlens;
    __nv_bfloat16 *out;
    float *lse;
    float *ws_lse;  // [slots][L * h_q]
    float *ws_o;    // [slots][L * h_q][d]
    uint32_t *err;
    int B, L, h_q, h_kv, page_size, num_pages, max_pages;
    int tile;   // tokens per pipeline stage (16 or 32)
    int seg_cost;  // plan: units a segment start costs, in tiles
    int gather; // pages hold fewer tokens than a tile (or not a multiple): rows copied token by token
    const void *cache0, *cache1;  // K / tied and V / rope caches (the gathered path reads them directly)
    int gpc;    // KV groups per CTA (consumer warps)
    int n_sub;  // CTAs per part = h_kv / gpc
    int parts;
    int nstage;
    uint32_t stage_bytes;     // smem bytes per stage (multiple of 1024)
    uint32_t stage_bytes_tx;  // bytes the TMA copies deliver per stage
    float scale_log2;         // softmax scale * log2(e)
    uint64_t wait_limit_ns;
    int debug_flags;
};

cudaError_t launch_group_decode(bool tied, int d, int d_r, int nt, const CUtensorMap &m0, const CUtensorMap &m1,
                                const GroupArgs &a, int grid, size_t smem, cudaStream_t st);

struct LatentArgs {
    const __nv_bfloat16 *q;
    const int32_t *block_table;
    const int32_t *seqlens;
    __nv_bfloat16 *out;
    float *lse;
    float *ws_lse;  // [slots][L * h_q]
    float *ws_o;    // [slots][L * h_q][d_c]
    uint32_t *err;
    int B, L, h_q, h_c, page_size, num_pages, max_pages;
    int n_sub;  // CTAs per part = h_c * row blocks * value slices
    int n_rt;   // 128-row blocks per latent head
    int row_spread;  // <= 64 rows spread over the TMEM lane quadrants: rows per quadrant (0: off)
    int gather;      // pages hold fewer tokens than a tile (or not a multiple): rows copied token by token
    int noncausal;   // every row sees all T tokens (a shared prefix attended by all query rows)
    int box_tok;     // narrow kernel: tokens per TMA box (divides the tile and the page)
    int seg_cost;    // plan: units a segment start costs, in tiles
    const void *cache0, *cache1;  // latent and rope caches (the gathered path reads them directly)
    int parts;
    int nstage;
    float scale_log2;
    uint64_t wait_limit_ns;
    int debug_flags;
};

// Compile-time geometry of the latent kernel for a latent width (0 fields: unsupported).
struct LatentShape {
    int tok;               // tokens per tile
    uint32_t q_bytes;      // shared memory for the q block
    uint32_t stage_bytes;  // one KV tile
    uint32_t p_bytes;      // the P block
};
LatentShape latent_shape(int d_c);

// GTA prefix attention on the latent kernel (latent_decode.cu): state = one tied group
// (d_h 128), key = its first 64 dims + the 64-wide rope, every row sees the whole prefix.
LatentShape tied_prefix_shape();
cudaError_t launch_tied_prefix(const CUtensorMap &qm, const CUtensorMap &lm, const CUtensorMap &rm,
                               const LatentArgs &a, int grid, size_t smem, cudaStream_t st);

// GLA with at most 64 query rows per latent head (latent_narrow.cu): tiles of
// narrow_tile_tokens() tokens, M = 64 MMAs, q in shared memory; no q tensor map.
int narrow_tile_tokens();
int narrow_seg_cost();  // the plan's cost of a segment start, in tiles
size_t narrow_smem_bytes();
cudaError_t launch_gla_narrow(const CUtensorMap &lm, const CUtensorMap &rm, const LatentArgs &a, int grid,
                              cudaStream_t st);

// GLA with more than 64 query rows per latent head (latent_m128.cu), in blocks of 128 rows (one
// CTA each): 64-token tiles, M = 128 MMAs, two softmax warps per lane quadrant; no q tensor map.
int m128_tile_tokens();
int m128_seg_cost();
size_t m128_smem_bytes();
cudaError_t launch_gla_m128(const CUtensorMap &lm, const CUtensorMap &rm, const LatentArgs &a, int grid,
                            cudaStream_t st);

// d_c = 512 (MLA): CTA pairs splitting the key dimension (latent_pair.cu).
uint32_t mla_pair_fixed_smem();   // q half + the exchange buffer
uint32_t mla_pair_stage_bytes();  // one 64-token tile half
cudaError_t launch_mla_pair(const CUtensorMap &qm, const CUtensorMap &qrm, const CUtensorMap &lm,
                            const CUtensorMap &rm, const LatentArgs &a, int grid, size_t smem, cudaStream_t st);

struct CombineArgs {
    const int32_t *seqlens;
    const float *ws_lse;
    const float *ws_o;
    __nv_bfloat16 *out;
    float *lse;
    int B, L, tile, seg_cost, max_tokens, parts;
    int rows;  // L * h_q
    int d_v;
};

// Merges two attention states (out bf16 [rows, d_v], lse fp32 [rows]) over disjoint key sets.
cudaError_t launch_merge(const void *out_a, const float *lse_a, const void *out_b, const float *lse_b, void *out,
                         float *lse, int rows, int d_v, cudaStream_t st);

// Merges split partials (launched as a programmatic dependent of the decode kernel).
cudaError_t launch_combine(const CombineArgs &a, cudaStream_t st);

// Writes the plan of every part (see kvd_plan).
cudaError_t launch_plan(const int32_t *seqlens, int B, int tile, int seg_cost, int max_tokens, int L, int parts,
                        int32_t *segs, int32_t *counts, int cap, cudaStream_t st);

}  // namespace kvd
