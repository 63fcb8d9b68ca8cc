// latent_api.cu -- C ABI of the GQLA latent paths: latent_absorbed_attn (MQA-
// absorbed attention over the latent cache) and latent_expand_cache (the
// one-time conversion to the per-group cache).  Validation, workspace carving,
// TMA descriptors and the launch sequence
//   absorb GEMM (q~ = W^UK^T q^C) -> latent attention (+ split merge) -> up-projection GEMM (W^UV o~).
#include <math.h>

#include <algorithm>

#include "common.cuh"
#include "host_util.h"
#include "latent.h"

namespace lka {

struct LatentPlan {
    int split_tokens, nsplit;
    size_t off_qt, off_olat, off_plse, off_po, ws_bytes;
};

static lka_status_t latent_plan(int B, int h_q, int g, int s_q, int d_h, int r_kv, int d_r, int Lmax,
                                LatentPlan* pl, bool paged = false) {
    if (B < 0 || h_q < 1 || g < 1 || s_q < 1 || d_h < 1 || r_kv < 1 || d_r < 0 || Lmax < 1) return LKA_ERR_INVALID_ARG;
    if (h_q % g) return LKA_ERR_INVALID_ARG;
    // the kernels are specialised to the GQLA/MLA shape (h_q, d_h, r_kv, d_h^R) = (128, 128, 512, 64)
    if (h_q != 128 || d_h != 128 || r_kv != 512 || d_r != 64) return LKA_ERR_UNSUPPORTED;
    const int HPG = h_q / g;
    if (HPG < 16 || 128 % (HPG * s_q) != 0) return LKA_ERR_UNSUPPORTED;
    if ((!paged && (long long)B * Lmax >= (1ll << 31)) || B > 65535) return LKA_ERR_UNSUPPORTED;
    const int NT = latent_tile_tokens();
    int st = split_tokens_knob();
    if (st <= 0) {
        // One CTA pair per (sequence, query token, key split).  Pick the split count n that
        // minimises waves x (work per split + writing its partial result), in units of the work of
        // a whole sequence: ceil(units * n / pairs) * (1/n + part), where part = the partial's
        // bytes per CTA (128 x 256 fp32) over the cache bytes a CTA reads for a whole sequence
        // (Lmax x 576); no partial when n = 1.  Ties go to fewer splits.
        const long long units = (long long)(B > 0 ? B : 1) * s_q;
        const long long pairs = sm_count() / 2;
        const double part = (128.0 * 256.0 * 4.0) / ((double)Lmax * 576.0);
        int best = 1;
        double best_cost = 1e30;
        const int max_n = std::max(1, std::min(256, Lmax / (8 * NT)));
        for (int n = 1; n <= max_n; ++n) {
            const double cost = (double)((units * n + pairs - 1) / pairs) * (1.0 / n + (n > 1 ? part : 0.0));
            if (cost < best_cost - 1e-9) {
                best_cost = cost;
                best = n;
            }
        }
        st = (Lmax + best - 1) / best;
        if (st < 8 * NT) st = 8 * NT;
    }
    st = cdiv(st, NT) * NT;
    pl->split_tokens = st;
    pl->nsplit = cdiv(Lmax, st);
    WsCarve c;
    const size_t rows = (size_t)B * s_q * h_q;
    pl->off_qt = c.take(rows * r_kv * 2);
    pl->off_olat = c.take(rows * r_kv * 2);
    if (pl->nsplit > 1) {
        pl->off_plse = c.take(rows * pl->nsplit * 4);
        pl->off_po = c.take(rows * pl->nsplit * (size_t)r_kv * 4);
    } else {
        pl->off_plse = pl->off_po = 0;
    }
    pl->ws_bytes = c.off;
    return LKA_OK;
}

static lka_status_t st_of(cudaError_t e) { return e == cudaSuccess ? LKA_OK : LKA_ERR_CUDA; }

}  // namespace lka

using namespace lka;

extern "C" {

size_t latent_absorbed_attn_workspace_size(int B, int h_q, int g, int s_q, int d_h, int r_kv, int d_r, int Lmax) {
    LatentPlan pl;
    return latent_plan(B, h_q, g, s_q, d_h, r_kv, d_r, Lmax, &pl) == LKA_OK ? pl.ws_bytes : 0;
}

}  // extern "C"

namespace lka {
struct LatentPages {
    const int32_t* block_table;
    int page_size, max_pages, num_pages;
};

static lka_status_t latent_run(const void* q_c, const void* q_r, const void* w_uk, const void* w_uv,
                               const void* latent, const int32_t* cache_lens, void* out, float* lse, int B, int h_q,
                               int g, int s_q, int d_h, int r_kv, int d_r, int Lmax, int causal, float scale,
                               lka_dtype_t dtype, void* ws, size_t ws_bytes, void* stream, const LatentPages* pg,
                               const float* kv_scale = nullptr) {
    // kv_scale != nullptr: the latent cache holds e4m3 bytes (query and output stay bf16)
    if (dtype != LKA_BF16) return LKA_ERR_UNSUPPORTED;
    if (kv_scale && pg) return LKA_ERR_UNSUPPORTED;  // an FP8 cache is contiguous
    if (kv_scale && ((uintptr_t)kv_scale & 3)) return LKA_ERR_INVALID_ARG;
    LatentPlan pl;
    lka_status_t s = latent_plan(B, h_q, g, s_q, d_h, r_kv, d_r, Lmax, &pl, pg != nullptr);
    if (s != LKA_OK) return s;
    if (B == 0) return LKA_OK;
    const void* ptrs[] = {q_c, q_r, w_uk, w_uv, latent, cache_lens, out};
    for (const void* ptr : ptrs)
        if (!ptr || !aligned16(ptr)) return LKA_ERR_INVALID_ARG;
    if (!isfinite(scale)) return LKA_ERR_INVALID_ARG;
    if (!ws || ws_bytes < pl.ws_bytes) return LKA_ERR_WORKSPACE;
    if (!aligned16(ws)) return LKA_ERR_INVALID_ARG;
    cudaStream_t st = (cudaStream_t)stream;
    uint8_t* w = static_cast<uint8_t*>(ws);
    uint32_t* status = reinterpret_cast<uint32_t*>(w);
    const int HPG = h_q / g;
    const int slab = HPG * s_q;
    const auto BF = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    __nv_bfloat16* qt = reinterpret_cast<__nv_bfloat16*>(w + pl.off_qt);
    __nv_bfloat16* olat = reinterpret_cast<__nv_bfloat16*>(w + pl.off_olat);

    // 1) absorption q~ = W^UK_gamma^T q^C
    CUtensorMap tm_qc, tm_wuk;
    {
        const uint64_t dims[3] = {(uint64_t)d_h, (uint64_t)h_q * s_q, (uint64_t)B};
        const uint64_t str[2] = {(uint64_t)d_h * 2, (uint64_t)h_q * s_q * d_h * 2};
        const uint32_t box[3] = {64, (uint32_t)slab, (uint32_t)(128 / slab)};
        if (!make_tmap_nd(&tm_qc, BF, q_c, 3, dims, str, box)) return LKA_ERR_CUDA;
        if (!make_tmap_2d(&tm_wuk, BF, w_uk, r_kv, (uint64_t)g * d_h, (uint64_t)r_kv * 2, 64, 64)) return LKA_ERR_CUDA;
    }
    GemmParams ga{};
    ga.out = qt;
    ga.status = status;
    ga.K = d_h;
    ga.N = r_kv;
    ga.B = B;
    ga.HPG = HPG;
    ga.s_q = s_q;
    ga.h_q = h_q;
    ga.g = g;
    ga.Lmax = Lmax;
    if ((s = st_of(gemm_absorb(tm_qc, tm_wuk, ga, st))) != LKA_OK) return s;

    // 2) attention of all heads over the latent cache (+ merge of key splits)
    CUtensorMap tm_lat;
    const uint64_t lat_rows = pg ? (uint64_t)pg->num_pages * pg->page_size : (uint64_t)B * Lmax;
    const int box_rows = pg && pg->page_size < latent_tile_tokens() ? pg->page_size : latent_tile_tokens();
    if (kv_scale) {
        // e4m3 rows of r_kv + d_r bytes, 64-byte boxes without swizzle (the kernel widens them in shared memory)
        if (!make_tmap_2d(&tm_lat, CU_TENSOR_MAP_DATA_TYPE_UINT8, latent, r_kv + d_r, lat_rows, (uint64_t)(r_kv + d_r),
                          64, box_rows, CU_TENSOR_MAP_SWIZZLE_NONE))
            return LKA_ERR_CUDA;
    } else if (!make_tmap_2d(&tm_lat, BF, latent, r_kv + d_r, lat_rows, (uint64_t)(r_kv + d_r) * 2, 64, box_rows)) {
        return LKA_ERR_CUDA;
    }
    LatentParams lp{};
    lp.lens = cache_lens;
    lp.q_t = qt;
    lp.q_r = static_cast<const __nv_bfloat16*>(q_r);
    lp.o_lat = olat;
    lp.lse = lse;
    lp.part_o = pl.nsplit > 1 ? reinterpret_cast<float*>(w + pl.off_po) : nullptr;
    lp.part_lse = pl.nsplit > 1 ? reinterpret_cast<float*>(w + pl.off_plse) : nullptr;
    lp.status = status;
    lp.B = B;
    lp.h_q = h_q;
    lp.g = g;
    lp.s_q = s_q;
    lp.Lmax = Lmax;
    lp.causal = causal ? 1 : 0;
    lp.scale_log2 = scale * 1.4426950408889634f;
    lp.split_tokens = pl.split_tokens;
    lp.nsplit = pl.nsplit;
    lp.block_table = pg ? pg->block_table : nullptr;
    lp.page_size = pg ? pg->page_size : 0;
    lp.max_pages = pg ? pg->max_pages : 0;
    lp.num_pages = pg ? pg->num_pages : 0;
    lp.box_rows = box_rows;
    lp.kv_scale = kv_scale;
    if ((s = st_of(latent_attn_launch(tm_lat, lp, st))) != LKA_OK) return s;

    // 3) up-projection out = W^UV_gamma o~
    CUtensorMap tm_ol, tm_wuv;
    const int M_rows = B * slab;
    if (!make_tmap_2d(&tm_ol, BF, olat, r_kv, (uint64_t)g * M_rows, (uint64_t)r_kv * 2, 64, 128) ||
        !make_tmap_2d(&tm_wuv, BF, w_uv, r_kv, (uint64_t)g * d_h, (uint64_t)r_kv * 2, 64, 128))
        return LKA_ERR_CUDA;
    GemmParams gu = ga;
    gu.out = out;
    gu.M_rows = M_rows;
    gu.K = r_kv;
    gu.N = d_h;
    return st_of(gemm_upproj(tm_ol, tm_wuv, gu, st));
}


}  // namespace lka

extern "C" {

lka_status_t latent_absorbed_attn(const void* q_c, const void* q_r, const void* w_uk, const void* w_uv,
                                  const void* latent, const int32_t* cache_lens, void* out, float* lse, int B, int h_q,
                                  int g, int s_q, int d_h, int r_kv, int d_r, int Lmax, int causal, float scale,
                                  lka_dtype_t dtype, void* ws, size_t ws_bytes, void* stream) {
    return latent_run(q_c, q_r, w_uk, w_uv, latent, cache_lens, out, lse, B, h_q, g, s_q, d_h, r_kv, d_r, Lmax, causal,
                      scale, dtype, ws, ws_bytes, stream, nullptr);
}

size_t latent_absorbed_attn_fp8kv_workspace_size(int B, int h_q, int g, int s_q, int d_h, int r_kv, int d_r,
                                                  int Lmax) {
    return latent_absorbed_attn_workspace_size(B, h_q, g, s_q, d_h, r_kv, d_r, Lmax);
}

lka_status_t latent_absorbed_attn_fp8kv(const void* q_c, const void* q_r, const void* w_uk, const void* w_uv,
                                        const void* latent, const float* kv_scale, const int32_t* cache_lens, void* out,
                                        float* lse, int B, int h_q, int g, int s_q, int d_h, int r_kv, int d_r,
                                        int Lmax, int causal, float scale, void* ws, size_t ws_bytes, void* stream) {
    if (!kv_scale) return LKA_ERR_INVALID_ARG;
    return latent_run(q_c, q_r, w_uk, w_uv, latent, cache_lens, out, lse, B, h_q, g, s_q, d_h, r_kv, d_r, Lmax, causal,
                      scale, LKA_BF16, ws, ws_bytes, stream, nullptr, kv_scale);
}

size_t latent_absorbed_attn_paged_workspace_size(int B, int h_q, int g, int s_q, int d_h, int r_kv, int d_r,
                                                 int page_size, int max_pages) {
    if (page_size < 8 || (page_size & (page_size - 1)) || max_pages < 1 ||
        (long long)page_size * max_pages >= (1ll << 31))
        return 0;
    LatentPlan pl;
    return latent_plan(B, h_q, g, s_q, d_h, r_kv, d_r, page_size * max_pages, &pl, true) == LKA_OK ? pl.ws_bytes : 0;
}

lka_status_t latent_absorbed_attn_paged(const void* q_c, const void* q_r, const void* w_uk, const void* w_uv,
                                        const void* latent_pages, const int32_t* block_table,
                                        const int32_t* cache_lens, void* out, float* lse, int B, int h_q, int g,
                                        int s_q, int d_h, int r_kv, int d_r, int page_size, int max_pages,
                                        int num_pages, int causal, float scale, lka_dtype_t dtype, void* ws,
                                        size_t ws_bytes, void* stream) {
    if (page_size < 8 || (page_size & (page_size - 1)) || max_pages < 1 || num_pages < 1) return LKA_ERR_INVALID_ARG;
    if ((long long)page_size * max_pages >= (1ll << 31) || (long long)num_pages * page_size >= (1ll << 31))
        return LKA_ERR_UNSUPPORTED;
    if (B > 0 && (!block_table || (reinterpret_cast<uintptr_t>(block_table) & 3u))) return LKA_ERR_INVALID_ARG;
    const LatentPages pg{block_table, page_size, max_pages, num_pages};
    return latent_run(q_c, q_r, w_uk, w_uv, latent_pages, cache_lens, out, lse, B, h_q, g, s_q, d_h, r_kv, d_r,
                      page_size * max_pages, causal, scale, dtype, ws, ws_bytes, stream, &pg);
}

}  // extern "C"

namespace lka {
// kr[b, j, :] = latent[b, j, r_kv : r_kv + d_r]  (16-byte pieces)
__global__ void copy_rope_key_kernel(const uint8_t* latent, uint8_t* kr, long long n_tokens, int row_bytes,
                                     int off_bytes, int kr_bytes) {
    const int per = kr_bytes / 16;
    const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= n_tokens * per) return;
    const long long tok = i / per;
    const int c = (int)(i % per);
    *reinterpret_cast<uint4*>(kr + tok * kr_bytes + c * 16) =
        *reinterpret_cast<const uint4*>(latent + tok * row_bytes + off_bytes + c * 16);
}
}  // namespace lka

extern "C" lka_status_t latent_expand_cache(const void* latent, const void* w_uk, const void* w_uv, int B, int Lmax,
                                            int g, int d_h, int r_kv, int d_r, void* kc, void* vc, void* kr,
                                            lka_dtype_t dtype, void* stream) {
    if (dtype != LKA_BF16) return LKA_ERR_UNSUPPORTED;
    if (B < 0 || Lmax < 1 || g < 1 || d_h < 1 || r_kv < 1 || d_r < 0) return LKA_ERR_INVALID_ARG;
    if (d_h % 128 || r_kv % 64 || d_r % 8 || ((r_kv + d_r) * 2) % 16) return LKA_ERR_UNSUPPORTED;
    if ((long long)B * Lmax >= (1ll << 31)) return LKA_ERR_UNSUPPORTED;
    if (B == 0) return LKA_OK;
    const void* ptrs[] = {latent, w_uk, w_uv, kc, vc};
    for (const void* p : ptrs)
        if (!p || !aligned16(p)) return LKA_ERR_INVALID_ARG;
    if (d_r > 0 && (!kr || !aligned16(kr))) return LKA_ERR_INVALID_ARG;
    cudaStream_t st = (cudaStream_t)stream;
    const auto BF = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    CUtensorMap ta, tk, tv;
    if (!make_tmap_2d(&ta, BF, latent, r_kv + d_r, (uint64_t)B * Lmax, (uint64_t)(r_kv + d_r) * 2, 64, 128) ||
        !make_tmap_2d(&tk, BF, w_uk, r_kv, (uint64_t)g * d_h, (uint64_t)r_kv * 2, 64, 128) ||
        !make_tmap_2d(&tv, BF, w_uv, r_kv, (uint64_t)g * d_h, (uint64_t)r_kv * 2, 64, 128))
        return LKA_ERR_CUDA;
    GemmParams p{};
    p.status = nullptr;
    p.K = r_kv;
    p.N = d_h;
    p.B = B;
    p.g = g;
    p.Lmax = Lmax;
    p.tiles_per_b = cdiv(Lmax, 128);
    // the helper takes no workspace, so it has no status word: a timed-out wait only ends the kernel
    p.status = nullptr;
    p.out = kc;
    if (gemm_expand(ta, tk, p, st) != cudaSuccess) return LKA_ERR_CUDA;
    p.out = vc;
    if (gemm_expand(ta, tv, p, st) != cudaSuccess) return LKA_ERR_CUDA;
    if (d_r > 0) {
        const long long n = (long long)B * Lmax * (d_r * 2 / 16);
        copy_rope_key_kernel<<<(unsigned)((n + 255) / 256), 256, 0, st>>>(
            static_cast<const uint8_t*>(latent), static_cast<uint8_t*>(kr), (long long)B * Lmax, (r_kv + d_r) * 2,
            r_kv * 2, d_r * 2);
        if (cudaPeekAtLastError() != cudaSuccess) return LKA_ERR_CUDA;
    }
    return LKA_OK;
}
