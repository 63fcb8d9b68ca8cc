// sparse.cu -- top-k sparse attention of the GQLA latent paths, given the
// selected token indices.
//
// Operation ("GQLA: Group-Query Latent Attention ..." section 1, "TransGQLA and
// sparse GQLA", and section 2, "Sparse and long-context attention"): a
// token-dependent top-k selection of past keys/values (as in DeepSeek sparse
// attention); both GQLA decode paths attend over the selected tokens only.  The
// selection itself (the indexer) is the caller's: this file takes, for every
// query token, a list of topk cache positions.  Entry j of the list of query t
// of sequence b counts when 0 <= j <= L_b - s_q + t (a key the query may see
// under bottom-right causality); other entries (-1 for padding) are skipped, and
// every entry that counts is one key of the softmax.
//
// Execution: a gather pass compacts, for every (sequence, query token) pair, the
// listed rows of the cache into a dense cache in the workspace, then the dense
// kernels of the path run over it with one "sequence" per pair (s_q = 1, no mask:
// the list already respects causality), and a last pass puts the outputs back in
// [B, h_q, s_q, d] order.  A pair whose list has no entry that counts gets out = 0
// and lse = -inf.
#include <math.h>

#include "common.cuh"
#include "host_util.h"

namespace lka {

namespace sp {
constexpr int TILE = 128;  // the compacted caches are padded to whole tiles of the dense kernels
}

// One CTA of 256 threads per (sequence, query token): the entries that count, in list order, and how many there
// are.  Warp w scans the w-th eighth of the list; the warps' counts are scanned in shared memory.
__global__ void __launch_bounds__(256) sparse_select_kernel(const int32_t* indices, const int32_t* lens, int B, int s_q,
                                                            int topk, int Lmax, int32_t* sel, int32_t* count,
                                                            uint32_t* status) {
    __shared__ int s_cnt[8];
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int pair = blockIdx.x;  // b * s_q + t
    const int b = pair / s_q, t = pair % s_q;
    const int L = clamp_len(lens, b, Lmax, s_q, 1, status, t == 0 && threadIdx.x == 0);
    const int last = L - s_q + t;  // last key query t may see
    const int32_t* in = indices + (size_t)pair * topk;
    int32_t* out = sel + (size_t)pair * topk;
    const int chunk = cdiv(cdiv(topk, 8), 32) * 32;
    const int j_lo = min(topk, warp * chunk), j_hi = min(topk, j_lo + chunk);
    int n = 0;
    for (int j0 = j_lo; j0 < j_hi; j0 += 32) {
        const int j = j0 + lane;
        const int idx = j < j_hi ? in[j] : -1;
        n += __popc(__ballot_sync(0xffffffffu, idx >= 0 && idx <= last));
    }
    if (lane == 0) s_cnt[warp] = n;
    __syncthreads();
    int base = 0, total = 0;
    for (int w = 0; w < 8; ++w) {
        base += w < warp ? s_cnt[w] : 0;
        total += s_cnt[w];
    }
    for (int j0 = j_lo; j0 < j_hi; j0 += 32) {
        const int j = j0 + lane;
        const int idx = j < j_hi ? in[j] : -1;
        const bool ok = idx >= 0 && idx <= last;
        const uint32_t m = __ballot_sync(0xffffffffu, ok);
        if (ok) out[base + __popc(m & ((1u << lane) - 1u))] = idx;
        base += __popc(m);
    }
    if (threadIdx.x == 0) count[pair] = total;
}

// Copies row sel[pair][r] of a per-sequence cache (rows of `row_bytes` bytes; sequence b's rows start at
// (b * heads + h) * Lmax, h < heads) to row r of the compacted cache of the pair ((pair * heads + h) * cap).
// One thread per 16-byte piece, consecutive threads on consecutive pieces of a row; rows r >= count are left
// as they are (the dense kernels mask them).
__global__ void __launch_bounds__(256) sparse_gather_kernel(const uint8_t* src, uint8_t* dst, const int32_t* sel,
                                                            const int32_t* count, int pairs, int s_q, int heads,
                                                            int topk, int cap, int Lmax, int row_bytes) {
    const int per_row = row_bytes / 16;
    const long long total = (long long)pairs * heads * topk * per_row;
    for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < total;
         i += (long long)gridDim.x * blockDim.x) {
        const int c = (int)(i % per_row);
        const long long row = i / per_row;  // (pair, h, r)
        const int r = (int)(row % topk);
        const int h = (int)((row / topk) % heads);
        const int pair = (int)(row / ((long long)topk * heads));
        if (r >= __ldg(count + pair)) continue;
        const int b = pair / s_q;
        const int tok = __ldg(sel + (size_t)pair * topk + r);
        const uint4 v = __ldg(reinterpret_cast<const uint4*>(src + ((size_t)(b * heads + h) * Lmax + tok) * row_bytes) + c);
        reinterpret_cast<uint4*>(dst + ((size_t)(pair * heads + h) * cap + r) * row_bytes)[c] = v;
    }
}

static unsigned gather_grid(long long rows, int row_bytes) {
    const long long pieces = rows * (row_bytes / 16);
    const long long blocks = (pieces + 255) / 256;
    const long long cap = (long long)sm_count() * 16;  // grid-stride beyond 16 CTAs per SM
    return (unsigned)(blocks < cap ? blocks : cap);
}

// [B, h, s_q, D] <-> [B * s_q, h, 1, D] (to_pairs = 1: into pair order; 0: back), D elements of 2 bytes.
__global__ void sparse_reorder_kernel(const uint16_t* src, uint16_t* dst, int B, int h, int s_q, int D, int to_pairs) {
    const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    const long long n = (long long)B * h * s_q * D;
    if (i >= n) return;
    const int d = (int)(i % D);
    const int t = (int)((i / D) % s_q);
    const int hh = (int)((i / ((long long)D * s_q)) % h);
    const int b = (int)(i / ((long long)D * s_q * h));
    const size_t a = (((size_t)b * h + hh) * s_q + t) * D + d;       // [B, h, s_q, D]
    const size_t p = (((size_t)(b * s_q + t) * h + hh)) * D + d;     // [B * s_q, h, 1, D]
    if (to_pairs)
        dst[p] = src[a];
    else
        dst[a] = src[p];
}

// Outputs of the pairs back into [B, h_q, s_q, d] (when s_q > 1) and the pairs without any key: out = 0,
// lse = -inf.  One thread per output element (lse by the thread of element 0).
__global__ void sparse_finish_kernel(const __nv_bfloat16* out_pairs, const float* lse_pairs, const int32_t* count,
                                     __nv_bfloat16* out, float* lse, int B, int h, int s_q, int D) {
    const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    const long long n = (long long)B * h * s_q * D;
    if (i >= n) return;
    const int d = (int)(i % D);
    const int t = (int)((i / D) % s_q);
    const int hh = (int)((i / ((long long)D * s_q)) % h);
    const int b = (int)(i / ((long long)D * s_q * h));
    const int pair = b * s_q + t;
    const size_t pr = (size_t)pair * h + hh;
    const bool empty = count[pair] == 0;
    if (out_pairs != out) out[i] = empty ? __float2bfloat16_rn(0.f) : out_pairs[pr * D + d];
    else if (empty) out[i] = __float2bfloat16_rn(0.f);
    if (lse && d == 0) {
        const size_t li = ((size_t)b * h + hh) * s_q + t;
        if (lse_pairs != lse) lse[li] = empty ? -INFINITY : lse_pairs[pr];
        else if (empty) lse[li] = -INFINITY;
    }
}

struct SparsePlan {
    int cap;  // compacted tokens per pair (topk rounded up to whole tiles)
    size_t off_sel, off_count, off_qc, off_qr, off_out, off_lse, off_cache, off_inner, inner_bytes, ws_bytes;
};

// Workspace of a sparse call: selection, compacted caches, reordered q and outputs, then the dense call's own.
static bool sparse_plan(int B, int h_q, int s_q, int d_h, int d_r, int topk, size_t cache_bytes_per_pair,
                        size_t inner_bytes, SparsePlan* pl) {
    if (B < 0 || s_q < 1 || topk < 1 || inner_bytes == 0) return false;
    pl->cap = cdiv(topk, sp::TILE) * sp::TILE;
    const size_t pairs = (size_t)B * s_q;
    WsCarve c;
    pl->off_sel = c.take(pairs * topk * 4);
    pl->off_count = c.take(pairs * 4);
    pl->off_qc = c.take(pairs * h_q * d_h * 2);
    pl->off_qr = c.take(pairs * h_q * d_r * 2);
    pl->off_out = c.take(pairs * h_q * d_h * 2);
    pl->off_lse = c.take(pairs * h_q * 4);
    pl->off_cache = c.take(pairs * cache_bytes_per_pair * pl->cap);
    pl->off_inner = c.off;
    pl->inner_bytes = inner_bytes;
    pl->ws_bytes = c.off + inner_bytes;
    return true;
}

static lka_status_t cuda_ok() { return cudaPeekAtLastError() == cudaSuccess ? LKA_OK : LKA_ERR_CUDA; }

// The dense call keeps its device status in its own workspace header: fold it into the caller's.
__global__ void sparse_status_merge_kernel(uint32_t* outer, uint32_t* inner) {
    if (*inner) atomicOr(outer, *inner);
    *inner = 0u;
}

// Selection, query reordering (s_q > 1); returns the pair-ordered q_c / q_r to hand to the dense call.
static lka_status_t sparse_prologue(const void* q_c, const void* q_r, const int32_t* indices, const int32_t* lens,
                                    int B, int h_q, int s_q, int d_h, int d_r, int topk, int Lmax,
                                    const SparsePlan& pl, uint8_t* w, cudaStream_t st, const void** qc_p,
                                    const void** qr_p) {
    uint32_t* status = reinterpret_cast<uint32_t*>(w);
    const int pairs = B * s_q;
    if (cudaMemsetAsync(w + pl.off_inner, 0, sizeof(uint32_t), st) != cudaSuccess) return LKA_ERR_CUDA;
    sparse_select_kernel<<<pairs, 256, 0, st>>>(indices, lens, B, s_q, topk, Lmax,
                                                         reinterpret_cast<int32_t*>(w + pl.off_sel),
                                                         reinterpret_cast<int32_t*>(w + pl.off_count), status);
    if (cuda_ok() != LKA_OK) return LKA_ERR_CUDA;
    *qc_p = q_c;
    *qr_p = q_r;
    if (s_q > 1) {
        const long long nc = (long long)pairs * h_q * d_h, nr = (long long)pairs * h_q * d_r;
        sparse_reorder_kernel<<<(unsigned)((nc + 255) / 256), 256, 0, st>>>(
            static_cast<const uint16_t*>(q_c), reinterpret_cast<uint16_t*>(w + pl.off_qc), B, h_q, s_q, d_h, 1);
        sparse_reorder_kernel<<<(unsigned)((nr + 255) / 256), 256, 0, st>>>(
            static_cast<const uint16_t*>(q_r), reinterpret_cast<uint16_t*>(w + pl.off_qr), B, h_q, s_q, d_r, 1);
        if (cuda_ok() != LKA_OK) return LKA_ERR_CUDA;
        *qc_p = w + pl.off_qc;
        *qr_p = w + pl.off_qr;
    }
    return LKA_OK;
}

// lens of the dense call: max(count, 1) (a pair without keys reads one row and is cleared afterwards)
__global__ void sparse_lens_kernel(const int32_t* count, int32_t* lens, int pairs) {
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i < pairs) lens[i] = count[i] > 0 ? count[i] : 1;
}

static lka_status_t sparse_epilogue(void* out, float* lse, int B, int h_q, int s_q, int d_h, const SparsePlan& pl,
                                    uint8_t* w, cudaStream_t st) {
    const long long n = (long long)B * h_q * s_q * d_h;
    const __nv_bfloat16* op = s_q > 1 ? reinterpret_cast<const __nv_bfloat16*>(w + pl.off_out)
                                      : static_cast<const __nv_bfloat16*>(out);
    const float* lp = s_q > 1 ? reinterpret_cast<const float*>(w + pl.off_lse) : lse;
    sparse_finish_kernel<<<(unsigned)((n + 255) / 256), 256, 0, st>>>(
        op, lp, reinterpret_cast<const int32_t*>(w + pl.off_count), static_cast<__nv_bfloat16*>(out), lse, B, h_q, s_q,
        d_h);
    sparse_status_merge_kernel<<<1, 1, 0, st>>>(reinterpret_cast<uint32_t*>(w),
                                                reinterpret_cast<uint32_t*>(w + pl.off_inner));
    return cuda_ok();
}

}  // namespace lka

using namespace lka;

extern "C" {

size_t latent_absorbed_attn_sparse_workspace_size(int B, int h_q, int g, int s_q, int d_h, int r_kv, int d_r,
                                                  int topk) {
    if (topk < 1) return 0;
    const int cap = cdiv(topk, sp::TILE) * sp::TILE;
    const size_t inner = latent_absorbed_attn_workspace_size(B * s_q, h_q, g, 1, d_h, r_kv, d_r, cap);
    SparsePlan pl;
    if (!sparse_plan(B, h_q, s_q, d_h, d_r, topk, (size_t)(r_kv + d_r) * 2, inner, &pl)) return 0;
    return pl.ws_bytes;
}

lka_status_t latent_absorbed_attn_sparse(const void* q_c, const void* q_r, const void* w_uk, const void* w_uv,
                                         const void* latent, const int32_t* indices, const int32_t* cache_lens,
                                         void* out, float* lse, int B, int h_q, int g, int s_q, int d_h, int r_kv,
                                         int d_r, int Lmax, int topk, float scale, lka_dtype_t dtype, void* ws,
                                         size_t ws_bytes, void* stream) {
    if (dtype != LKA_BF16) return LKA_ERR_UNSUPPORTED;
    if (B < 0 || s_q < 1 || s_q > 2 || topk < 1 || Lmax < 1) return LKA_ERR_INVALID_ARG;
    const size_t need = latent_absorbed_attn_sparse_workspace_size(B, h_q, g, s_q, d_h, r_kv, d_r, topk);
    if (need == 0) return LKA_ERR_UNSUPPORTED;
    if (B == 0) return LKA_OK;
    const void* ptrs[] = {q_c, q_r, w_uk, w_uv, latent, indices, cache_lens, out};
    for (const void* ptr : ptrs)
        if (!ptr || !aligned16(ptr)) return LKA_ERR_INVALID_ARG;
    if ((long long)B * Lmax >= (1ll << 31) || (long long)B * s_q * topk >= (1ll << 31)) return LKA_ERR_UNSUPPORTED;
    if (!ws || ws_bytes < need) return LKA_ERR_WORKSPACE;
    if (!aligned16(ws)) return LKA_ERR_INVALID_ARG;
    const int cap = cdiv(topk, sp::TILE) * sp::TILE;
    SparsePlan pl;
    sparse_plan(B, h_q, s_q, d_h, d_r, topk, (size_t)(r_kv + d_r) * 2,
                latent_absorbed_attn_workspace_size(B * s_q, h_q, g, 1, d_h, r_kv, d_r, cap), &pl);
    uint8_t* w = static_cast<uint8_t*>(ws);
    cudaStream_t st = (cudaStream_t)stream;
    const void *qc_p, *qr_p;
    lka_status_t s = sparse_prologue(q_c, q_r, indices, cache_lens, B, h_q, s_q, d_h, d_r, topk, Lmax, pl, w, st,
                                     &qc_p, &qr_p);
    if (s != LKA_OK) return s;
    const int pairs = B * s_q;
    const long long items = (long long)pairs * topk;
    sparse_gather_kernel<<<gather_grid(items, (r_kv + d_r) * 2), 256, 0, st>>>(
        static_cast<const uint8_t*>(latent), w + pl.off_cache, reinterpret_cast<const int32_t*>(w + pl.off_sel),
        reinterpret_cast<const int32_t*>(w + pl.off_count), pairs, s_q, 1, topk, cap, Lmax, (r_kv + d_r) * 2);
    // the dense call's lens (max(count, 1)) reuse the selection buffer's head: the selection is consumed
    int32_t* lens_p = reinterpret_cast<int32_t*>(w + pl.off_sel);
    sparse_lens_kernel<<<cdiv(pairs, 256), 256, 0, st>>>(reinterpret_cast<const int32_t*>(w + pl.off_count), lens_p,
                                                         pairs);
    if (cuda_ok() != LKA_OK) return LKA_ERR_CUDA;
    void* out_p = s_q > 1 ? (void*)(w + pl.off_out) : out;
    float* lse_p = s_q > 1 ? reinterpret_cast<float*>(w + pl.off_lse) : lse;
    s = latent_absorbed_attn(qc_p, qr_p, w_uk, w_uv, w + pl.off_cache, lens_p, out_p, lse_p, pairs, h_q, g, 1, d_h,
                             r_kv, d_r, cap, 0, scale, dtype, w + pl.off_inner, pl.inner_bytes, stream);
    if (s != LKA_OK) return s;
    return sparse_epilogue(out, lse, B, h_q, s_q, d_h, pl, w, st);
}

size_t latent_expand_gqa_attn_sparse_workspace_size(int B, int h_q, int g, int s_q, int d_h, int d_r, int topk) {
    if (topk < 1 || g < 1) return 0;
    const int cap = cdiv(topk, sp::TILE) * sp::TILE;
    const size_t inner = latent_expand_gqa_attn_workspace_size(B * s_q, h_q, g, 1, d_h, d_r, cap);
    SparsePlan pl;
    // compacted kc and vc ([g] rows each) and kr per token
    if (!sparse_plan(B, h_q, s_q, d_h, d_r, topk, (size_t)(2 * g * d_h + d_r) * 2, inner, &pl)) return 0;
    return pl.ws_bytes;
}

lka_status_t latent_expand_gqa_attn_sparse(const void* q_c, const void* q_r, const void* kc, const void* vc,
                                           const void* kr, const int32_t* indices, const int32_t* cache_lens,
                                           void* out, float* lse, int B, int h_q, int g, int s_q, int d_h, int d_r,
                                           int Lmax, int topk, float scale, lka_dtype_t dtype, void* ws,
                                           size_t ws_bytes, void* stream) {
    if (dtype != LKA_BF16) return LKA_ERR_UNSUPPORTED;
    if (B < 0 || g < 1 || s_q < 1 || s_q > 2 || topk < 1 || Lmax < 1) return LKA_ERR_INVALID_ARG;
    const size_t need = latent_expand_gqa_attn_sparse_workspace_size(B, h_q, g, s_q, d_h, d_r, topk);
    if (need == 0) return LKA_ERR_UNSUPPORTED;
    if (B == 0) return LKA_OK;
    const void* ptrs[] = {q_c, q_r, kc, vc, kr, indices, cache_lens, out};
    for (const void* ptr : ptrs)
        if (!ptr || !aligned16(ptr)) return LKA_ERR_INVALID_ARG;
    if ((long long)B * g * Lmax >= (1ll << 31) || (long long)B * s_q * topk * g >= (1ll << 31))
        return LKA_ERR_UNSUPPORTED;
    if (!ws || ws_bytes < need) return LKA_ERR_WORKSPACE;
    if (!aligned16(ws)) return LKA_ERR_INVALID_ARG;
    const int cap = cdiv(topk, sp::TILE) * sp::TILE;
    SparsePlan pl;
    sparse_plan(B, h_q, s_q, d_h, d_r, topk, (size_t)(2 * g * d_h + d_r) * 2,
                latent_expand_gqa_attn_workspace_size(B * s_q, h_q, g, 1, d_h, d_r, cap), &pl);
    uint8_t* w = static_cast<uint8_t*>(ws);
    cudaStream_t st = (cudaStream_t)stream;
    const void *qc_p, *qr_p;
    lka_status_t s = sparse_prologue(q_c, q_r, indices, cache_lens, B, h_q, s_q, d_h, d_r, topk, Lmax, pl, w, st,
                                     &qc_p, &qr_p);
    if (s != LKA_OK) return s;
    const int pairs = B * s_q;
    uint8_t* kc_c = w + pl.off_cache;
    uint8_t* vc_c = kc_c + (size_t)pairs * g * cap * d_h * 2;
    uint8_t* kr_c = vc_c + (size_t)pairs * g * cap * d_h * 2;
    const int32_t* sel = reinterpret_cast<const int32_t*>(w + pl.off_sel);
    const int32_t* cnt = reinterpret_cast<const int32_t*>(w + pl.off_count);
    const long long items_g = (long long)pairs * g * topk, items_r = (long long)pairs * topk;
    sparse_gather_kernel<<<gather_grid(items_g, d_h * 2), 256, 0, st>>>(static_cast<const uint8_t*>(kc), kc_c, sel, cnt,
                                                                      pairs, s_q, g, topk, cap, Lmax, d_h * 2);
    sparse_gather_kernel<<<gather_grid(items_g, d_h * 2), 256, 0, st>>>(static_cast<const uint8_t*>(vc), vc_c, sel, cnt,
                                                                      pairs, s_q, g, topk, cap, Lmax, d_h * 2);
    sparse_gather_kernel<<<gather_grid(items_r, d_r * 2), 256, 0, st>>>(static_cast<const uint8_t*>(kr), kr_c, sel, cnt,
                                                                      pairs, s_q, 1, topk, cap, Lmax, d_r * 2);
    int32_t* lens_p = reinterpret_cast<int32_t*>(w + pl.off_sel);
    sparse_lens_kernel<<<cdiv(pairs, 256), 256, 0, st>>>(cnt, lens_p, pairs);
    if (cuda_ok() != LKA_OK) return LKA_ERR_CUDA;
    void* out_p = s_q > 1 ? (void*)(w + pl.off_out) : out;
    float* lse_p = s_q > 1 ? reinterpret_cast<float*>(w + pl.off_lse) : lse;
    s = latent_expand_gqa_attn(qc_p, qr_p, kc_c, vc_c, kr_c, lens_p, out_p, lse_p, pairs, h_q, g, 1, d_h, d_r, cap, 0,
                               scale, dtype, w + pl.off_inner, pl.inner_bytes, stream);
    if (s != LKA_OK) return s;
    return sparse_epilogue(out, lse, B, h_q, s_q, d_h, pl, w, st);
}

}  // extern "C"
