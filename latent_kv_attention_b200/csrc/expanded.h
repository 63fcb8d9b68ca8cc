// expanded.h -- launch interface of the GQLA per-group (expanded-cache) GQA path.
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/lka.h"

namespace lka {

struct ExpParams {
    const int32_t* lens;   // device [B]
    __nv_bfloat16* out;    // [B, h_q, s_q, 128]
    float* lse;            // [B, h_q, s_q] natural log, or nullptr
    float* part_o;         // [B*h_q*s_q][nsplit][128] (nsplit > 1)
    float* part_lse;       // [B*h_q*s_q][nsplit] log2 domain
    uint32_t* status;
    int B, h_q, g, s_q, Lmax, causal;
    float scale_log2;
    int split_tokens, nsplit;
    // paged caches (block_table == nullptr: contiguous kc, vc [B, g, Lmax, 128], kr [B, Lmax, 64])
    const int32_t* block_table;  // device [B][max_pages] page indices, or nullptr
    int page_size, max_pages, num_pages;
    int box_rows;                // rows per TMA box: min(page_size, tile)
};

cudaError_t expanded_attn_launch(const CUtensorMap& qc, const CUtensorMap& qr, const CUtensorMap& kc,
                                 const CUtensorMap& kr, const CUtensorMap& vc, const ExpParams& p, cudaStream_t st);

// Prefill (s_q >= kExpPrefillMinQueries) of the per-group path on the tensor-core prefill kernel (gta_attn.cu):
// keys [kc[gamma] ; k^R] of d_h + d_r = 192 values, values vc[gamma]; paged pools when block_table != nullptr.
constexpr int kExpPrefillMinQueries = 64;
size_t expanded_prefill_ws_bytes(int B, int h_q, int s_q, int Lmax);
lka_status_t expanded_prefill_tc(const void* q_c, const void* q_r, const void* kc, const void* vc, const void* kr,
                                 const int32_t* cache_lens, void* out, float* lse, int B, int h_q, int g, int s_q,
                                 int Lmax, int causal, float scale, void* ws, size_t ws_bytes, cudaStream_t st,
                                 const int32_t* block_table, int page_size, int max_pages, int num_pages);

}  // namespace lka
