// gqa_decode.h -- launch interface of the split-KV GQA decode kernels.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/lka.h"

namespace lka {

struct GqaParams {
    const void* q;          // [B, h_q, s_q, D]
    void* out;              // [B, h_q, s_q, D]
    float* lse;             // [B, h_q, s_q] natural log, or nullptr
    const int32_t* lens;    // device [B]
    float* part_o;          // [B*h_q*s_q][nsplit_max][D] fp32 partials
    float* part_lse;        // [B*h_q*s_q][nsplit_max] log2-domain partial lse
    uint32_t* status;       // workspace status word
    int B, h_q, h_kv, s_q, Lmax, causal;
    float scale_log2;       // scale * log2(e)
    int split_tokens;       // keys per split (multiple of the tile)
    int nsplit_max;         // ceil(Lmax / split_tokens)
    int n_rb;               // row blocks per KV head
    int ratio;              // h_q / h_kv
    // paged cache (block_table == nullptr: contiguous [B, h_kv, Lmax, D])
    const int32_t* block_table;  // device [B][max_pages] page indices, or nullptr
    int page_size, max_pages, num_pages;
    int box_rows;           // rows per TMA box: min(page_size, tile)
    // quantised (e4m3) cache: per-KV-head dequantisation scales, device [h_kv] (nullptr otherwise)
    const float* k_scale;
    const float* v_scale;
};

// The e4m3-cache instances (bf16 q/out): d = 128 on the tensor-core instance (rb = 16), d = 256 on the CUDA-core
// one (rb <= 4: a 16-byte chunk holds 16 values, so more rows per CTA would not fit the query slice in registers).
int gqa_fp8_tile_tokens(int d, int rb, int* ctas_per_sm);
cudaError_t gqa_fp8_decode_launch(const CUtensorMap& tk, const CUtensorMap& tv, const GqaParams& p, int d, int rb,
                                  int nsplit, cudaStream_t st);
// Merge of split partials for rows [B*h_q*s_q] of D values (rows needing one split are skipped).
cudaError_t gqa_combine_launch(const GqaParams& p, int dtype_bytes, int d, cudaStream_t st);
// Tokens per TMA tile of the kernel instance (0 if the instance does not exist) and its resident CTAs per SM.
int gqa_tile_tokens(int dtype_bytes, int d, int rb, int* ctas_per_sm);
// Launches the decode kernel (grid nsplit x h_kv*n_rb x B) and, when nsplit > 1, the merge.
cudaError_t gqa_decode_launch(const CUtensorMap& tk, const CUtensorMap& tv, const GqaParams& p, int dtype_bytes,
                              int d, int rb, int nsplit, cudaStream_t st);

// Causal (or full) prefill on the tensor cores for bf16, d = 128 (gta_attn.cu): one CTA per (128-query tile,
// query head, sequence, key split), keys and values of the head's KV head h / (h_q / h_kv); paged caches when
// block_table != nullptr (pools [num_pages, h_kv, page_size, 128]).  gqa_prefill_ws_bytes is its workspace.
size_t gqa_prefill_ws_bytes(int B, int h_q, int s_q, int Lmax);
int gqa_prefill_nsplit(int B, int h_q, int s_q, int Lmax);  // key splits of the prefill plan
lka_status_t gqa_prefill_tc(const void* q, const void* k, const void* v, const int32_t* cache_lens, void* out,
                            float* lse, int B, int h_q, int h_kv, int s_q, int Lmax, int causal, float scale, void* ws,
                            size_t ws_bytes, cudaStream_t st, const int32_t* block_table, int page_size, int max_pages,
                            int num_pages);
// Query tokens from which gqa_attn (bf16, d = 128) runs the tensor-core prefill instead of the split-KV kernel.
constexpr int kGqaPrefillMinQueries = 64;

}  // namespace lka
