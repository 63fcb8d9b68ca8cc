// api.cu -- the C ABI entry points (include/lka.h): argument validation,
// split planning, workspace carving, TMA descriptors and kernel dispatch.
// No allocation happens here: all scratch space is the caller's workspace.
#include <math.h>
#include <string.h>

#include <atomic>
#include <mutex>
#include <utility>
#include <vector>

#include "common.cuh"
#include "gqa_decode.h"
#include "host_util.h"

namespace lka {

// Test and benchmark hooks.  Both are per host thread: a setting made on one thread never changes the
// plan or the launches of calls made on another, so concurrent callers stay independent.
static thread_local int t_split_tokens = 0;
int split_tokens_knob() { return t_split_tokens; }

// ---------------------------------------------------------------- kernel timing hook
struct TimingRegistry {
    std::mutex mu;
    std::atomic<bool> on{false};
    std::vector<cudaEvent_t> pool;
    std::vector<std::pair<cudaEvent_t, cudaEvent_t>> pending;
};
static TimingRegistry& timing_reg() {
    static thread_local TimingRegistry r;
    return r;
}
bool kernel_timing_on() { return timing_reg().on.load(std::memory_order_relaxed); }
cudaEvent_t kernel_timing_event() {
    auto& r = timing_reg();
    std::lock_guard<std::mutex> g(r.mu);
    if (!r.pool.empty()) {
        cudaEvent_t e = r.pool.back();
        r.pool.pop_back();
        return e;
    }
    cudaEvent_t e = nullptr;
    if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
    return e;
}
void kernel_timing_push(cudaEvent_t a, cudaEvent_t b) {
    auto& r = timing_reg();
    std::lock_guard<std::mutex> g(r.mu);
    r.pending.emplace_back(a, b);
}

// ---------------------------------------------------------------- GQA plan
struct GqaPlan {
    int rb, n_rb, tile, split_tokens, nsplit;
    size_t off_lse, off_o, ws_bytes;
};

static int pick_rb(int rows, int d, int dtype_bytes, bool fp8kv) {
    // bf16 caches with d <= 128 and e4m3 caches with d = 128: the tensor-core instances, whose MMA tile holds
    // 16 query rows
    if ((!fp8kv && dtype_bytes == 2 && d <= 128) || (fp8kv && d == 128)) return 16;
    int cap = fp8kv ? 4 : 16;
    if (d == 256) cap = fp8kv ? 4 : 8;
    int rb = 1;
    while (rb < rows && rb < cap) rb *= 2;
    return rb;
}

static lka_status_t gqa_plan(int B, int h_q, int h_kv, int s_q, int d_h, int Lmax, int dtype_bytes, GqaPlan* pl,
                             bool paged = false, bool fp8kv = false) {
    if (B < 0 || h_q < 1 || h_kv < 1 || s_q < 1 || Lmax < 1 || d_h < 1) return LKA_ERR_INVALID_ARG;
    if (h_q % h_kv) return LKA_ERR_INVALID_ARG;
    const bool d_ok = fp8kv ? (d_h == 128 || d_h == 256)
                            : dtype_bytes == 2 ? (d_h == 64 || d_h == 128 || d_h == 256) : (d_h == 64 || d_h == 128);
    if (!d_ok) return LKA_ERR_UNSUPPORTED;
    if (!paged && (long long)B * h_kv * Lmax >= (1ll << 31)) return LKA_ERR_UNSUPPORTED;
    const int R = (h_q / h_kv) * s_q;
    pl->rb = pick_rb(R, d_h, dtype_bytes, fp8kv);
    pl->n_rb = cdiv(R, pl->rb);
    if ((long long)h_kv * pl->n_rb > 65535 || B > 65535) return LKA_ERR_UNSUPPORTED;
    int per_sm = 1;  // resident CTAs per SM of the kernel instance
    pl->tile = fp8kv ? gqa_fp8_tile_tokens(d_h, pl->rb, &per_sm) : gqa_tile_tokens(dtype_bytes, d_h, pl->rb, &per_sm);
    if (pl->tile <= 0) return LKA_ERR_UNSUPPORTED;
    int st = split_tokens_knob();
    if (st <= 0) {
        // One CTA per (sequence, KV head, row block, key split).  Pick the split count n that minimises
        // waves x (tiles per split + a fixed cost per CTA of about two tiles: filling the TMA ring at the
        // start, merging the warps and writing at the end), sizing splits for every sequence at Lmax.
        // With w = units * n / slots, the waves are max(ceil(w), w + 1/4): whole waves when the lengths
        // are equal, and some tail beyond the average when they differ (CTAs of short sequences end early
        // and the longest splits run last), which a plan of one long wave cannot absorb.  Ties go to fewer
        // splits.
        const double units = (double)(B > 0 ? B : 1) * h_kv * pl->n_rb;
        const double slots = (double)sm_count() * per_sm;
        const int lt = cdiv(Lmax, pl->tile);
        int best = 1;
        double best_cost = -1.0;
        for (int n = 1; n <= lt && n <= 256; ++n) {
            const double w = units * n / slots;
            const double cost = fmax(ceil(w - 1e-9), w + 0.25) * (cdiv(lt, n) + 2);
            if (best_cost < 0.0 || cost < best_cost - 1e-9) {
                best_cost = cost;
                best = n;
            }
        }
        st = cdiv(lt, best) * pl->tile;
    }
    st = cdiv(st, pl->tile) * pl->tile;
    pl->split_tokens = st;
    pl->nsplit = cdiv(Lmax, st);
    WsCarve c;
    const size_t rows = (size_t)B * h_q * s_q;
    if (pl->nsplit > 1) {
        pl->off_lse = c.take(rows * pl->nsplit * sizeof(float));
        pl->off_o = c.take(rows * pl->nsplit * (size_t)d_h * sizeof(float));
    } else {
        pl->off_lse = pl->off_o = 0;
    }
    pl->ws_bytes = c.off;
    return LKA_OK;
}

static lka_status_t launch_status(cudaError_t e) { return e == cudaSuccess ? LKA_OK : LKA_ERR_CUDA; }

lka_status_t status_from_word(uint32_t st) {
    if (st & kDevTimeout) return LKA_ERR_TIMEOUT;
    if (st & kDevBadLength) return LKA_ERR_BAD_LENGTH;
    if (st & kDevBadPage) return LKA_ERR_BAD_PAGE;
    if (st & kDevRange) return LKA_ERR_RANGE;
    return LKA_OK;
}

// Whether a GQA call runs the tensor-core prefill (bf16, d = 128, at least kGqaPrefillMinQueries queries).
static bool gqa_tc_prefill(int dtype_bytes, int d_h, int s_q, bool fp8kv) {
    return !fp8kv && dtype_bytes == 2 && d_h == 128 && s_q >= kGqaPrefillMinQueries;
}

// Workspace bytes of a GQA call; the size does not depend on the dtype beyond the supported head dims: plan
// with bf16 (the split-KV kernel, or the tensor-core prefill), then fp32, and take the larger.
static size_t gqa_ws_size(int B, int h_q, int h_kv, int s_q, int d_h, int Lmax, bool paged) {
    if (B < 0 || h_q < 1 || h_kv < 1 || s_q < 1 || Lmax < 1 || h_q % h_kv) return 0;
    size_t best = 0;
    bool any = false;
    GqaPlan pl;
    if (gqa_tc_prefill(2, d_h, s_q, false)) {
        best = gqa_prefill_ws_bytes(B, h_q, s_q, Lmax);
        any = true;
    } else if (gqa_plan(B, h_q, h_kv, s_q, d_h, Lmax, 2, &pl, paged) == LKA_OK) {
        best = pl.ws_bytes;
        any = true;
    }
    if (gqa_plan(B, h_q, h_kv, s_q, d_h, Lmax, 4, &pl, paged) == LKA_OK) {
        best = pl.ws_bytes > best ? pl.ws_bytes : best;
        any = true;
    }
    return any ? best : 0;
}

}  // namespace lka

using namespace lka;

extern "C" {

const char* lka_status_string(lka_status_t s) {
    switch (s) {
        case LKA_OK: return "LKA_OK";
        case LKA_ERR_INVALID_ARG: return "LKA_ERR_INVALID_ARG";
        case LKA_ERR_UNSUPPORTED: return "LKA_ERR_UNSUPPORTED";
        case LKA_ERR_WORKSPACE: return "LKA_ERR_WORKSPACE";
        case LKA_ERR_CUDA: return "LKA_ERR_CUDA";
        case LKA_ERR_TIMEOUT: return "LKA_ERR_TIMEOUT";
        case LKA_ERR_BAD_LENGTH: return "LKA_ERR_BAD_LENGTH";
        case LKA_ERR_BAD_PAGE: return "LKA_ERR_BAD_PAGE";
        case LKA_ERR_RANGE: return "LKA_ERR_RANGE";
    }
    return "LKA_ERR_UNKNOWN";
}

int lka_set_split_tokens(int tokens) {
    const int prev = t_split_tokens;
    t_split_tokens = tokens < 0 ? 0 : tokens;
    return prev;
}

lka_status_t lka_kernel_timing(int enable) {
    auto& r = timing_reg();
    std::lock_guard<std::mutex> g(r.mu);
    for (auto& pr : r.pending) {
        r.pool.push_back(pr.first);
        r.pool.push_back(pr.second);
    }
    r.pending.clear();
    r.on.store(enable != 0);
    return LKA_OK;
}

lka_status_t lka_kernel_timing_read(int* launches, double* total_ms) {
    if (!launches || !total_ms) return LKA_ERR_INVALID_ARG;
    auto& r = timing_reg();
    std::lock_guard<std::mutex> g(r.mu);
    double ms = 0.0;
    for (auto& pr : r.pending) {
        if (cudaEventSynchronize(pr.second) != cudaSuccess) return LKA_ERR_CUDA;
        float t = 0.f;
        if (cudaEventElapsedTime(&t, pr.first, pr.second) != cudaSuccess) return LKA_ERR_CUDA;
        ms += t;
    }
    *launches = (int)r.pending.size();
    *total_ms = ms;
    return LKA_OK;
}

lka_status_t lka_device_status(const void* ws, void* stream) {
    if (!ws) return LKA_ERR_INVALID_ARG;
    if (cudaStreamSynchronize((cudaStream_t)stream) != cudaSuccess) return LKA_ERR_CUDA;
    uint32_t st = 0;
    if (cudaMemcpy(&st, ws, sizeof(st), cudaMemcpyDeviceToHost) != cudaSuccess) return LKA_ERR_CUDA;
    return status_from_word(st);
}

lka_status_t lka_clear_status(void* ws, void* stream) {
    if (!ws) return LKA_ERR_INVALID_ARG;
    return launch_status(cudaMemsetAsync(ws, 0, sizeof(uint32_t), (cudaStream_t)stream));
}

size_t gqa_attn_workspace_size(int B, int h_q, int h_kv, int s_q, int d_h, int Lmax) {
    return gqa_ws_size(B, h_q, h_kv, s_q, d_h, Lmax, false);
}

int gqa_attn_split_count(int B, int h_q, int h_kv, int s_q, int d_h, int Lmax, lka_dtype_t dtype) {
    if (dtype != LKA_BF16 && dtype != LKA_FP32) return 0;
    if (gqa_tc_prefill(dtype == LKA_BF16 ? 2 : 4, d_h, s_q, false)) {
        if (B < 0 || h_q < 1 || h_kv < 1 || Lmax < 1 || h_q % h_kv) return 0;
        return gqa_prefill_nsplit(B, h_q, s_q, Lmax);
    }
    GqaPlan pl;
    return gqa_plan(B, h_q, h_kv, s_q, d_h, Lmax, dtype == LKA_BF16 ? 2 : 4, &pl) == LKA_OK ? pl.nsplit : 0;
}

}  // extern "C"

namespace lka {
struct PagedDesc {
    const int32_t* block_table;
    int page_size, max_pages, num_pages;
};

// Shared by gqa_attn (pg == nullptr: contiguous cache [B, h_kv, Lmax, d]) and gqa_attn_paged.
static lka_status_t gqa_run(const void* q, const void* k, const void* v, const int32_t* cache_lens, void* out,
                            float* lse, int B, int h_q, int h_kv, int s_q, int d_h, int Lmax, int causal, float scale,
                            lka_dtype_t dtype, void* ws, size_t ws_bytes, void* stream, const PagedDesc* pg,
                            const float* k_scale = nullptr, const float* v_scale = nullptr) {
    if (dtype != LKA_BF16 && dtype != LKA_FP32) return LKA_ERR_UNSUPPORTED;
    const bool fp8kv = k_scale != nullptr;  // e4m3 cache with per-KV-head scales (bf16 q / out)
    if (fp8kv && dtype != LKA_BF16) return LKA_ERR_UNSUPPORTED;
    const int eb = dtype == LKA_BF16 ? 2 : 4;
    const int kvb = fp8kv ? 1 : eb;  // bytes of one cache element
    if (gqa_tc_prefill(eb, d_h, s_q, fp8kv)) {
        // prefill: the tensor-core kernel, one CTA per (128-query tile, query head, sequence, key split)
        if (B < 0 || h_q < 1 || h_kv < 1 || Lmax < 1 || h_q % h_kv) return LKA_ERR_INVALID_ARG;
        if (!pg && (long long)B * h_kv * Lmax >= (1ll << 31)) return LKA_ERR_UNSUPPORTED;
        if (B == 0) return LKA_OK;
        if (!q || !k || !v || !cache_lens || !out) return LKA_ERR_INVALID_ARG;
        if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || !aligned16(cache_lens))
            return LKA_ERR_INVALID_ARG;
        if (!isfinite(scale)) return LKA_ERR_INVALID_ARG;
        if (ws && !aligned16(ws)) return LKA_ERR_INVALID_ARG;
        return gqa_prefill_tc(q, k, v, cache_lens, out, lse, B, h_q, h_kv, s_q, Lmax, causal, scale, ws, ws_bytes,
                              (cudaStream_t)stream, pg ? pg->block_table : nullptr, pg ? pg->page_size : 0,
                              pg ? pg->max_pages : 0, pg ? pg->num_pages : 0);
    }
    GqaPlan pl;
    lka_status_t s = gqa_plan(B, h_q, h_kv, s_q, d_h, Lmax, eb, &pl, pg != nullptr, fp8kv);
    if (s != LKA_OK) return s;
    if (B == 0) return LKA_OK;
    if (!q || !k || !v || !cache_lens || !out) return LKA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || !aligned16(cache_lens))
        return LKA_ERR_INVALID_ARG;
    if (!isfinite(scale)) return LKA_ERR_INVALID_ARG;
    if (!ws || ws_bytes < pl.ws_bytes) return LKA_ERR_WORKSPACE;
    if (!aligned16(ws)) return LKA_ERR_INVALID_ARG;

    const CUtensorMapDataType tdt = fp8kv ? CU_TENSOR_MAP_DATA_TYPE_UINT8
                                    : eb == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
    uint64_t rows = (uint64_t)B * h_kv * Lmax;
    uint32_t box_rows = (uint32_t)pl.tile;
    if (pg) {
        rows = (uint64_t)pg->num_pages * h_kv * pg->page_size;
        box_rows = (uint32_t)(pg->page_size < pl.tile ? pg->page_size : pl.tile);
    }
    CUtensorMap tk, tv;
    if (!make_tmap_2d(&tk, tdt, k, d_h, rows, (uint64_t)d_h * kvb, 128 / kvb, box_rows) ||
        !make_tmap_2d(&tv, tdt, v, d_h, rows, (uint64_t)d_h * kvb, 128 / kvb, box_rows))
        return LKA_ERR_CUDA;

    GqaParams p;
    p.q = q;
    p.out = out;
    p.lse = lse;
    p.lens = cache_lens;
    uint8_t* w = static_cast<uint8_t*>(ws);
    p.part_lse = pl.nsplit > 1 ? reinterpret_cast<float*>(w + pl.off_lse) : nullptr;
    p.part_o = pl.nsplit > 1 ? reinterpret_cast<float*>(w + pl.off_o) : nullptr;
    p.status = reinterpret_cast<uint32_t*>(w);
    p.B = B;
    p.h_q = h_q;
    p.h_kv = h_kv;
    p.s_q = s_q;
    p.Lmax = Lmax;
    p.causal = causal ? 1 : 0;
    p.scale_log2 = scale * 1.4426950408889634f;
    p.split_tokens = pl.split_tokens;
    p.nsplit_max = pl.nsplit;
    p.n_rb = pl.n_rb;
    p.ratio = h_q / h_kv;
    p.block_table = pg ? pg->block_table : nullptr;
    p.page_size = pg ? pg->page_size : 0;
    p.max_pages = pg ? pg->max_pages : 0;
    p.num_pages = pg ? pg->num_pages : 0;
    p.box_rows = (int)box_rows;
    p.k_scale = k_scale;
    p.v_scale = v_scale;
    if (fp8kv) return launch_status(gqa_fp8_decode_launch(tk, tv, p, d_h, pl.rb, pl.nsplit, (cudaStream_t)stream));
    return launch_status(gqa_decode_launch(tk, tv, p, eb, d_h, pl.rb, pl.nsplit, (cudaStream_t)stream));
}

// Paged-cache arguments: page_size a power of two >= 8, a table of max_pages entries per sequence, a pool
// of num_pages pages that TMA coordinates can address.
static lka_status_t paged_args_ok(int h_kv, int page_size, int max_pages, int num_pages) {
    if (page_size < 8 || (page_size & (page_size - 1)) || max_pages < 1 || num_pages < 1 || h_kv < 1)
        return LKA_ERR_INVALID_ARG;
    if ((long long)max_pages * page_size >= (1ll << 31) ||
        (long long)num_pages * h_kv * page_size >= (1ll << 31))
        return LKA_ERR_UNSUPPORTED;
    return LKA_OK;
}
}  // namespace lka

extern "C" {

lka_status_t gqa_attn(const void* q, const void* k, const void* v, const int32_t* cache_lens, void* out, float* lse,
                      int B, int h_q, int h_kv, int s_q, int d_h, int Lmax, int causal, float scale,
                      lka_dtype_t dtype, void* ws, size_t ws_bytes, void* stream) {
    return gqa_run(q, k, v, cache_lens, out, lse, B, h_q, h_kv, s_q, d_h, Lmax, causal, scale, dtype, ws, ws_bytes,
                   stream, nullptr);
}

size_t gqa_attn_fp8kv_workspace_size(int B, int h_q, int h_kv, int s_q, int d_h, int Lmax) {
    GqaPlan pl;
    return gqa_plan(B, h_q, h_kv, s_q, d_h, Lmax, 2, &pl, false, true) == LKA_OK ? pl.ws_bytes : 0;
}

lka_status_t gqa_attn_fp8kv(const void* q, const void* k, const void* v, const float* k_scale, const float* v_scale,
                            const int32_t* cache_lens, void* out, float* lse, int B, int h_q, int h_kv, int s_q,
                            int d_h, int Lmax, int causal, float scale, void* ws, size_t ws_bytes, void* stream) {
    if (B > 0 && (!k_scale || !v_scale || (reinterpret_cast<uintptr_t>(k_scale) & 3u) ||
                  (reinterpret_cast<uintptr_t>(v_scale) & 3u)))
        return LKA_ERR_INVALID_ARG;
    if (B == 0) {
        GqaPlan pl;
        return gqa_plan(B, h_q, h_kv, s_q, d_h, Lmax, 2, &pl, false, true);
    }
    return gqa_run(q, k, v, cache_lens, out, lse, B, h_q, h_kv, s_q, d_h, Lmax, causal, scale, LKA_BF16, ws, ws_bytes,
                   stream, nullptr, k_scale, v_scale);
}

size_t gqa_attn_paged_workspace_size(int B, int h_q, int h_kv, int s_q, int d_h, int page_size, int max_pages) {
    if (paged_args_ok(h_kv, page_size, max_pages, 1) != LKA_OK) return 0;
    return gqa_ws_size(B, h_q, h_kv, s_q, d_h, page_size * max_pages, true);
}

lka_status_t gqa_attn_paged(const void* q, const void* k_pages, const void* v_pages, const int32_t* block_table,
                            const int32_t* cache_lens, void* out, float* lse, int B, int h_q, int h_kv, int s_q,
                            int d_h, int page_size, int max_pages, int num_pages, int causal, float scale,
                            lka_dtype_t dtype, void* ws, size_t ws_bytes, void* stream) {
    lka_status_t s = paged_args_ok(h_kv, page_size, max_pages, num_pages);
    if (s != LKA_OK) return s;
    if (B > 0 && (!block_table || (reinterpret_cast<uintptr_t>(block_table) & 3u))) return LKA_ERR_INVALID_ARG;
    const PagedDesc pg{block_table, page_size, max_pages, num_pages};
    return gqa_run(q, k_pages, v_pages, cache_lens, out, lse, B, h_q, h_kv, s_q, d_h, page_size * max_pages, causal,
                   scale, dtype, ws, ws_bytes, stream, &pg);
}

}  // extern "C"
