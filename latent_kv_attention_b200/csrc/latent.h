// latent.h -- launch interfaces of the GQLA latent-path kernels.
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace lka {

enum GemmMode { GEMM_ABSORB = 0, GEMM_UPPROJ = 1, GEMM_EXPAND = 2 };

struct GemmParams {
    void* out;         // bf16 output
    uint32_t* status;  // workspace status word
    int M_rows;        // UPPROJ: rows per group (B*HPG*s_q)
    int K, N;          // reduction length (multiple of 64), output row length
    int B, HPG, s_q, h_q, g, Lmax;
    int tiles_per_b;   // EXPAND: 128-token tiles per sequence
};

cudaError_t gemm_absorb(const CUtensorMap& a, const CUtensorMap& b, const GemmParams& p, cudaStream_t st);
cudaError_t gemm_upproj(const CUtensorMap& a, const CUtensorMap& b, const GemmParams& p, cudaStream_t st);
cudaError_t gemm_expand(const CUtensorMap& a, const CUtensorMap& b, const GemmParams& p, cudaStream_t st);

struct LatentParams {
    const int32_t* lens;   // device [B]
    const __nv_bfloat16* q_t;  // [B*s_q*h_q][r_kv] absorbed query q~ (rows (b, t, h))
    const __nv_bfloat16* q_r;  // [B, h_q, s_q, d_r] RoPE query
    __nv_bfloat16* o_lat;  // [g][B*HPG*s_q][r_kv] bf16 latent-space output (rows (b, hh, t) per group)
    float* lse;            // [B, h_q, s_q] natural log, or nullptr
    float* part_o;         // [B*s_q*h_q][nsplit][r_kv] fp32 partials (nsplit > 1)
    float* part_lse;       // [B*s_q*h_q][nsplit] log2-domain
    uint32_t* status;
    int B, h_q, g, s_q, Lmax, causal;
    float scale_log2;
    int split_tokens, nsplit;
    // paged latent cache (block_table == nullptr: contiguous [B, Lmax, r_kv + d_r])
    const int32_t* block_table;  // device [B][max_pages] page indices, or nullptr
    int page_size, max_pages, num_pages;
    int box_rows;                // rows per TMA box: min(page_size, tile)
    // FP8 (e4m3) latent cache: dequantisation scales of the latent part and of the RoPE key (device [2]), or
    // nullptr for a bf16 cache
    const float* kv_scale;
};

cudaError_t latent_attn_launch(const CUtensorMap& tm_lat, const LatentParams& p, cudaStream_t st);
int latent_tile_tokens();

}  // namespace lka
