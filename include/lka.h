/*
 * lka.h -- C ABI of latent_kv_attention_b200: grouped / latent-KV scaled-dot-
 * product attention on NVIDIA B200 (sm_100a).
 *
 * Four attention entry points, one per cache layout the pages describe, plus
 * the one-time cache conversion and a few helpers.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - All tensor pointers are DEVICE pointers owned by the caller, row-major
 *    with the last dimension contiguous, 16-byte aligned.  The library never
 *    allocates device memory and keeps no per-call state: scratch space is the
 *    caller's workspace `ws` (size from the matching *_workspace_size call).
 *    A workspace must be zero-filled before its first use: its first 256
 *    bytes hold the sticky status word (see lka_device_status).
 *  - Work is enqueued asynchronously on `stream` (a cudaStream_t; NULL is the
 *    legacy default stream).  Calls on one workspace must not overlap.
 *  - cache_lens is a DEVICE int32 array [B]: cache_lens[b] = L_b counts the
 *    valid cache tokens of sequence b INCLUDING the s_q new query tokens,
 *    whose keys/values the caller has already written at positions
 *    L_b - s_q .. L_b - 1.  Requirement: 1 <= L_b <= Lmax, and L_b >= s_q when
 *    causal.  The device cannot report a bad length synchronously: an entry
 *    outside the range is clamped into it and LKA_ERR_BAD_LENGTH is raised in
 *    the workspace status word (read it with lka_device_status).
 *  - causal != 0 selects bottom-right aligned causal masking: query t
 *    (0 <= t < s_q) sees keys 0 .. L_b - s_q + t.  causal == 0 lets every query
 *    see keys 0 .. L_b - 1.  Prefill is s_q == L_b; decode is s_q = 1, or 2 for
 *    multi-token prediction.
 *  - scale multiplies the query-key dot products before the softmax.
 *  - Outputs have the input dtype (bf16 results are rounded to nearest even);
 *    lse (optional, may be NULL) is fp32, natural log of the softmax
 *    normaliser of each query row.
 *  - Errors are return codes; on a validation error nothing is enqueued and
 *    nothing is written.  Asynchronous CUDA launch failures are reported as
 *    LKA_ERR_CUDA.
 *
 * Sources (web pages on the subject, cited by title and section):
 *  [GQA]  "Grouped Query Attention (GQA)" glossary page, "How GQA works" and
 *         "How GQA shrinks the KV cache".
 *  [GQLA] "GQLA: Group-Query Latent Attention for Hardware-Adaptive Large
 *         Language Model Decoding", section 1 and section 3.1 with eq. (1) and
 *         Figure 2.
 *  [GTA]  "GTA: Grouped-head latenT Attention" press article, section on the
 *         grouped shared attention matrix.
 */
#ifndef LKA_H
#define LKA_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define LKA_API __attribute__((visibility("default")))
#else
#define LKA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    LKA_OK = 0,
    LKA_ERR_INVALID_ARG = 1,  /* a host-visible argument is out of range or a pointer is NULL/misaligned */
    LKA_ERR_UNSUPPORTED = 2,  /* valid arguments the library has no kernel for (dtype, head dim, ...) */
    LKA_ERR_WORKSPACE = 3,    /* ws is NULL or ws_bytes is below the *_workspace_size value */
    LKA_ERR_CUDA = 4,         /* a CUDA call or kernel launch failed */
    LKA_ERR_TIMEOUT = 5,      /* device status: a bounded in-kernel wait ran out (the kernel exited early) */
    LKA_ERR_BAD_LENGTH = 6,   /* device status: a cache_lens entry was outside its range and was clamped */
    LKA_ERR_BAD_PAGE = 7,     /* device status: a block-table entry a call needed was outside the page pool */
    LKA_ERR_RANGE = 8         /* device status: an intermediate value left the range of its internal format and
                                 was saturated (the output is finite but not accurate); see (b) */
} lka_status_t;

typedef enum { LKA_BF16 = 0, LKA_FP32 = 1 } lka_dtype_t;

/* ------------------------------------------------------------------------ */
/* (a) GQA attention  [GQA "How GQA works"]                                 */
/*  Query head i (0 <= i < h_q) attends with KV head floor(i / (h_q/h_kv)):  */
/*  each KV head serves a contiguous group of h_q/h_kv query heads.          */
/*  h_kv == h_q is MHA, h_kv == 1 is MQA.                                    */
/*   q   [B, h_q,  s_q,  d_h]     k, v [B, h_kv, Lmax, d_h]                  */
/*   out [B, h_q,  s_q,  d_h]     lse  [B, h_q, s_q] fp32 or NULL            */
/*  dtype: LKA_BF16 (d_h in {64, 128, 256}) or LKA_FP32 (d_h in {64, 128}).  */
/*  Split-KV flash decoding: long caches are split over CTAs and merged by   */
/*  log-sum-exp; the split partials live in ws.                              */
/*  Prefill (bf16, d_h = 128, s_q >= 64, any of the paged forms below but    */
/*  the FP8 cache) runs on the tcgen05 prefill kernel instead: one CTA per   */
/*  128-query tile, query head, sequence and key split; S = Q K^T and O +=   */
/*  P V on the tensor cores with the accumulators in tensor memory.          */
/* ------------------------------------------------------------------------ */
LKA_API size_t gqa_attn_workspace_size(int B, int h_q, int h_kv, int s_q, int d_h, int Lmax);
/* Key splits per sequence that gqa_attn plans for these sizes and dtype (decode: the grid is splits x h_kv x
 * row blocks x B CTAs; prefill: query tiles x splits x h_q x B; a sequence shorter than Lmax uses only the
 * splits its keys reach), or 0 for arguments gqa_attn rejects.  The plan depends only on the sizes, the dtype, the device's SM count and the split
 * knob (lka_set_split_tokens); host-only, no device work. */
LKA_API int gqa_attn_split_count(int B, int h_q, int h_kv, int s_q, int d_h, int Lmax, lka_dtype_t dtype);
LKA_API lka_status_t gqa_attn(const void *q, const void *k, const void *v, const int32_t *cache_lens, void *out,
                      float *lse, int B, int h_q, int h_kv, int s_q, int d_h, int Lmax, int causal, float scale,
                      lka_dtype_t dtype, void *ws, size_t ws_bytes, void *stream);

/* (a') GQA attention over a paged KV cache  [GQA "GQA compared with related
 *  techniques": PagedAttention allocates the cache in fixed-size blocks;
 *  GQLA sec. 2: paged KV caches are complementary system techniques].
 *  Same computation, arguments and dtypes as gqa_attn, with the cache held
 *  in a pool of fixed-size pages instead of one [Lmax] slab per sequence:
 *   k_pages, v_pages [num_pages, h_kv, page_size, d_h]   (device)
 *   block_table      [B, max_pages] int32 (device): token t of sequence b
 *                    is row t % page_size of page block_table[b][t / page_size]
 *  page_size is a power of two >= 8; the logical capacity of a sequence is
 *  max_pages * page_size (cache_lens entries above it are clamped, raising
 *  LKA_ERR_BAD_LENGTH).  Table entries of pages a sequence does not use may
 *  hold anything; an entry the call needs that is outside [0, num_pages) is
 *  replaced by page 0 and LKA_ERR_BAD_PAGE is raised in the workspace status.
 *  The workspace is sized by gqa_attn_paged_workspace_size. */
LKA_API size_t gqa_attn_paged_workspace_size(int B, int h_q, int h_kv, int s_q, int d_h, int page_size, int max_pages);
LKA_API lka_status_t gqa_attn_paged(const void *q, const void *k_pages, const void *v_pages,
                            const int32_t *block_table, const int32_t *cache_lens, void *out, float *lse, int B,
                            int h_q, int h_kv, int s_q, int d_h, int page_size, int max_pages, int num_pages,
                            int causal, float scale, lka_dtype_t dtype, void *ws, size_t ws_bytes, void *stream);

/* (a'') GQA attention over an FP8 (e4m3) KV cache  [GQLA sec. 2: quantised KV
 *  storage is a complementary system technique that lowers the bytes per
 *  cached token].  Same computation and layouts as gqa_attn with K and V held
 *  as e4m3 bytes and one fp32 dequantisation scale per KV head:
 *    K[b,h,t,:] = k_scale[h] * k[b,h,t,:],  V[b,h,t,:] = v_scale[h] * v[b,h,t,:]
 *   q, out [B,h_q,s_q,d_h] bf16;  k, v [B,h_kv,Lmax,d_h] e4m3 (one byte each);
 *   k_scale, v_scale [h_kv] fp32 (device);  lse as in gqa_attn.
 *  d_h in {128, 256}.  The e4m3 values are widened exactly; the scales are
 *  applied in fp32 (the key scale with the softmax scale to the query, the
 *  value scale to the output). */
LKA_API size_t gqa_attn_fp8kv_workspace_size(int B, int h_q, int h_kv, int s_q, int d_h, int Lmax);
LKA_API lka_status_t gqa_attn_fp8kv(const void *q, const void *k, const void *v, const float *k_scale,
                            const float *v_scale, const int32_t *cache_lens, void *out, float *lse, int B, int h_q,
                            int h_kv, int s_q, int d_h, int Lmax, int causal, float scale, void *ws, size_t ws_bytes,
                            void *stream);

/* gqa_attn for callers that cannot allocate device memory.  No counterpart in
 * the papers: it exists for callers that are handed only their input and
 * output buffers (a plugin or custom operator inside another runtime) or run
 * where the host framework forbids device allocations, and so cannot provide
 * the workspace gqa_attn takes.  Same arguments, result and dtypes as
 * gqa_attn minus the workspace: the split-KV scratch lives in a 16 MiB device
 * array inside the library (held by every GPU that loads the library until
 * the process exits).  This call allocates nothing.  Its first call on a
 * device looks up that array's device address (cudaGetSymbolAddress), so make
 * the first call on each device before any stream capture; the address is
 * cached per device ordinal, so do not use this variant on a device after
 * cudaDeviceReset.  Returns LKA_ERR_WORKSPACE, enqueuing nothing, when the
 * split plan of the call's sizes and dtype needs more than 16 MiB.  All calls
 * share the one array: calls that overlap on the GPU (other streams, other
 * host threads) race and must be serialised by the caller.  Device-side
 * status flags (LKA_ERR_TIMEOUT, LKA_ERR_BAD_LENGTH) accumulate in the
 * array's status word; read them with gqa_attn_noalloc_status. */
LKA_API lka_status_t gqa_attn_noalloc(const void *q, const void *k, const void *v, const int32_t *cache_lens,
                              void *out, float *lse, int B, int h_q, int h_kv, int s_q, int d_h, int Lmax,
                              int causal, float scale, lka_dtype_t dtype, void *stream);
/* The device status of the no-allocation variant on the current device: synchronises `stream`, reads the
 * status word of the library's scratch array (flags raised by gqa_attn_noalloc calls since the last read,
 * returned like lka_device_status), then enqueues its reset on `stream`.  Allocates nothing. */
LKA_API lka_status_t gqa_attn_noalloc_status(void *stream);

/* ------------------------------------------------------------------------ */
/* (b) GQLA MQA-absorbed latent attention  [GQLA sec. 1, sec. 3.1 eq. (1),  */
/*     Figure 2(b)]                                                         */
/*  The cache holds, per token, the joint latent c^KV (r_kv values) followed */
/*  by the shared RoPE key k^R (d_r values).  Head i belongs to group        */
/*  gamma = floor(i / (h_q/g)); W^UK_gamma, W^UV_gamma are d_h x r_kv.       */
/*  Computes, for every head i and query t:                                  */
/*     q~  = W^UK_gamma^T q^C                (absorption into the query)     */
/*     s_j = scale * (<q~, c_j> + <q^R, k^R_j>)                              */
/*     o~  = sum_j softmax(s)_j c_j          (attention over the latent)     */
/*     out = W^UV_gamma o~                   (up-projection of the output)   */
/*  which equals GQA over the per-group expanded keys/values (see (c)).      */
/*   q_c [B,h_q,s_q,d_h]  q_r [B,h_q,s_q,d_r]  w_uk, w_uv [g,d_h,r_kv]       */
/*   latent [B,Lmax,r_kv+d_r]  out [B,h_q,s_q,d_h]  lse [B,h_q,s_q] or NULL  */
/*  Supported: bf16, r_kv = 512, d_r = 64, d_h = 128, h_q = 128, s_q <= 2.   */
/*  The score contraction is split over two CTAs whose partial scores are    */
/*  exchanged as fp16 after multiplication by scale*log2(e); a scaled        */
/*  partial beyond the fp16 range (|x| > 65504) is saturated and raises      */
/*  LKA_ERR_RANGE in the workspace status (finite, inaccurate output).       */
/* ------------------------------------------------------------------------ */
LKA_API size_t latent_absorbed_attn_workspace_size(int B, int h_q, int g, int s_q, int d_h, int r_kv, int d_r, int Lmax);
LKA_API lka_status_t latent_absorbed_attn(const void *q_c, const void *q_r, const void *w_uk, const void *w_uv,
                                  const void *latent, const int32_t *cache_lens, void *out, float *lse, int B,
                                  int h_q, int g, int s_q, int d_h, int r_kv, int d_r, int Lmax, int causal,
                                  float scale, lka_dtype_t dtype, void *ws, size_t ws_bytes, void *stream);

/* (b') The same over a paged latent cache  [GQA "GQA compared with related
 *  techniques" (PagedAttention); GQLA sec. 2 (paged KV caches)].
 *   latent_pages [num_pages, page_size, r_kv + d_r]  (device)
 *   block_table  [B, max_pages] int32 (device): token t of sequence b is
 *                row t % page_size of page block_table[b][t / page_size]
 *  page_size a power of two >= 8; capacity max_pages * page_size per
 *  sequence; out-of-pool entries a call needs are replaced by page 0 and
 *  raise LKA_ERR_BAD_PAGE.  Other arguments and results as in (b). */
LKA_API size_t latent_absorbed_attn_paged_workspace_size(int B, int h_q, int g, int s_q, int d_h, int r_kv, int d_r,
                                                         int page_size, int max_pages);
LKA_API lka_status_t latent_absorbed_attn_paged(const void *q_c, const void *q_r, const void *w_uk,
                                        const void *w_uv, const void *latent_pages, const int32_t *block_table,
                                        const int32_t *cache_lens, void *out, float *lse, int B, int h_q, int g,
                                        int s_q, int d_h, int r_kv, int d_r, int page_size, int max_pages,
                                        int num_pages, int causal, float scale, lka_dtype_t dtype, void *ws,
                                        size_t ws_bytes, void *stream);

/* (b'') The same over an FP8 (e4m3) latent cache  [GQLA sec. 2: quantised KV
 *  storage is a complementary system technique that lowers the bytes per
 *  cached token].  latent [B, Lmax, r_kv + d_r] holds e4m3 bytes (576 per token,
 *  half the bf16 cache) with two fp32 dequantisation scales (device [2]):
 *    c^KV[b,t,:] = kv_scale[0] * latent[b,t,0:r_kv]
 *    k^R[b,t,:]  = kv_scale[1] * latent[b,t,r_kv:r_kv+d_r]
 *  q_c, q_r, w_uk, w_uv, out stay bf16; other arguments, results and shape
 *  limits as in (b); contiguous cache only.  The e4m3 values are widened
 *  exactly (to f16) in shared memory; the scales are applied in fp32 to the
 *  query and to the latent-space output (the query and P enter the tensor
 *  cores as f16). */
LKA_API size_t latent_absorbed_attn_fp8kv_workspace_size(int B, int h_q, int g, int s_q, int d_h, int r_kv, int d_r,
                                                         int Lmax);
LKA_API lka_status_t latent_absorbed_attn_fp8kv(const void *q_c, const void *q_r, const void *w_uk,
                                        const void *w_uv, const void *latent, const float *kv_scale,
                                        const int32_t *cache_lens, void *out, float *lse, int B, int h_q, int g,
                                        int s_q, int d_h, int r_kv, int d_r, int Lmax, int causal, float scale,
                                        void *ws, size_t ws_bytes, void *stream);

/* ------------------------------------------------------------------------ */
/* (c) GQLA GQA path over the per-group expanded cache  [GQLA sec. 1,       */
/*     sec. 3.1, Figure 2(a)]                                               */
/*  Key of group gamma at token j: [kc[b,gamma,j,:] ; kr[b,j,:]] (the RoPE   */
/*  key is stored once and shared by all groups); value: vc[b,gamma,j,:];    */
/*  query of head i: [q_c ; q_r].  h_q/g query heads per group.              */
/*   kc, vc [B,g,Lmax,d_h]  kr [B,Lmax,d_r]  other arguments as in (b).      */
/*  Supported: bf16, d_h = 128, d_r = 64, and either h_q/g = 16, s_q <= 2    */
/*  (decode kernel: one CTA per group and key split, the group's 16 heads x  */
/*  s_q query rows as the MMA rows), or s_q >= 64 with any h_q/g (prefill:   */
/*  the tcgen05 prefill kernel of (a) with 192-wide keys [kc ; kr], one CTA  */
/*  per 128-query tile, head, sequence and key split).                       */
/* ------------------------------------------------------------------------ */
LKA_API size_t latent_expand_gqa_attn_workspace_size(int B, int h_q, int g, int s_q, int d_h, int d_r, int Lmax);
LKA_API lka_status_t latent_expand_gqa_attn(const void *q_c, const void *q_r, const void *kc, const void *vc,
                                    const void *kr, const int32_t *cache_lens, void *out, float *lse, int B,
                                    int h_q, int g, int s_q, int d_h, int d_r, int Lmax, int causal, float scale,
                                    lka_dtype_t dtype, void *ws, size_t ws_bytes, void *stream);

/* (c') The same over paged caches  [GQA "GQA compared with related
 *  techniques" (PagedAttention); GQLA sec. 2 (paged KV caches)].
 *   kc_pages, vc_pages [num_pages, g, page_size, d_h]   kr_pages [num_pages, page_size, d_r]
 *   block_table [B, max_pages] int32: token t of sequence b is row t % page_size of
 *   page block_table[b][t / page_size] in all three pools.  latent_expand_cache with
 *   B = num_pages and Lmax = page_size converts a paged latent pool into these pools.
 *  page_size a power of two >= 8; out-of-pool entries a call needs are replaced by
 *  page 0 and raise LKA_ERR_BAD_PAGE.  Other arguments and results as in (c). */
LKA_API size_t latent_expand_gqa_attn_paged_workspace_size(int B, int h_q, int g, int s_q, int d_h, int d_r,
                                                           int page_size, int max_pages);
LKA_API lka_status_t latent_expand_gqa_attn_paged(const void *q_c, const void *q_r, const void *kc_pages,
                                          const void *vc_pages, const void *kr_pages, const int32_t *block_table,
                                          const int32_t *cache_lens, void *out, float *lse, int B, int h_q, int g,
                                          int s_q, int d_h, int d_r, int page_size, int max_pages, int num_pages,
                                          int causal, float scale, lka_dtype_t dtype, void *ws, size_t ws_bytes,
                                          void *stream);

/* (c'') Top-k sparse attention of both GQLA paths, given the selection
 *  [GQLA sec. 1 "TransGQLA and sparse GQLA", sec. 2 "Sparse and long-context
 *  attention": a token-dependent top-k selection of past keys/values; sparse
 *  GQLA keeps both decode paths].  The indexer that picks the tokens is the
 *  caller's.  indices [B, s_q, topk] int32 (device): for query token t of
 *  sequence b, the cache positions it attends to; entry j counts when
 *  0 <= j <= L_b - s_q + t, other entries (-1 for padding) are skipped, and
 *  each entry that counts is one key of the softmax (lists should not repeat
 *  a position).  A query whose list has no entry that counts gets out = 0 and
 *  lse = -inf.  s_q <= 2; other arguments, layouts and shape limits as in (b)
 *  (latent cache) and (c) (expanded caches).  The selected rows are gathered
 *  into the workspace before the dense kernels run over them. */
LKA_API size_t latent_absorbed_attn_sparse_workspace_size(int B, int h_q, int g, int s_q, int d_h, int r_kv, int d_r,
                                                          int topk);
LKA_API lka_status_t latent_absorbed_attn_sparse(const void *q_c, const void *q_r, const void *w_uk,
                                         const void *w_uv, const void *latent, const int32_t *indices,
                                         const int32_t *cache_lens, void *out, float *lse, int B, int h_q, int g,
                                         int s_q, int d_h, int r_kv, int d_r, int Lmax, int topk, float scale,
                                         lka_dtype_t dtype, void *ws, size_t ws_bytes, void *stream);
LKA_API size_t latent_expand_gqa_attn_sparse_workspace_size(int B, int h_q, int g, int s_q, int d_h, int d_r,
                                                            int topk);
LKA_API lka_status_t latent_expand_gqa_attn_sparse(const void *q_c, const void *q_r, const void *kc,
                                           const void *vc, const void *kr, const int32_t *indices,
                                           const int32_t *cache_lens, void *out, float *lse, int B, int h_q, int g,
                                           int s_q, int d_h, int d_r, int Lmax, int topk, float scale,
                                           lka_dtype_t dtype, void *ws, size_t ws_bytes, void *stream);

/* ------------------------------------------------------------------------ */
/* (d) GTA shared-score attention  [GTA, grouped shared attention matrix]   */
/*  H heads in G groups of H/G; head h uses group gamma = floor(h/(H/G)).    */
/*  One score matrix softmax(scale q_g k_g^T) per group is computed once and */
/*  applied to the values of every head of the group.                        */
/*   q_g [B,G,s_q,d_qk]  k_g [B,G,Lmax,d_qk]  v [B,H,Lmax,d_v]               */
/*   out [B,H,s_q,d_v]   lse [B,G,s_q] (one per group and query) or NULL     */
/*  Supported: bf16, d_qk = d_v = 64, H/G <= 4.                              */
/* ------------------------------------------------------------------------ */
LKA_API size_t gta_shared_score_attn_workspace_size(int B, int G, int H, int s_q, int d_qk, int d_v, int Lmax);
LKA_API lka_status_t gta_shared_score_attn(const void *q_g, const void *k_g, const void *v, const int32_t *cache_lens,
                                   void *out, float *lse, int B, int G, int H, int s_q, int d_qk, int d_v,
                                   int Lmax, int causal, float scale, lka_dtype_t dtype, void *ws, size_t ws_bytes,
                                   void *stream);

/* (d') The same over paged caches (chunked prefill against a paged cache)
 *  [GQA "GQA compared with related techniques" (PagedAttention); GQLA sec. 2
 *  (paged KV caches)].
 *   k_pages [num_pages, G, page_size, d_qk]   v_pages [num_pages, H, page_size, d_v]
 *   block_table [B, max_pages] int32 (device): token t of sequence b is row
 *   t % page_size of page block_table[b][t / page_size] in both pools.
 *  page_size a power of two >= 8; capacity max_pages * page_size per sequence
 *  (cache_lens entries above it are clamped, raising LKA_ERR_BAD_LENGTH); table
 *  entries a call needs that are outside [0, num_pages) are replaced by page 0
 *  and raise LKA_ERR_BAD_PAGE.  Other arguments and results as in (d). */
LKA_API size_t gta_shared_score_attn_paged_workspace_size(int B, int G, int H, int s_q, int d_qk, int d_v,
                                                          int page_size, int max_pages);
LKA_API lka_status_t gta_shared_score_attn_paged(const void *q_g, const void *k_pages, const void *v_pages,
                                         const int32_t *block_table, const int32_t *cache_lens, void *out,
                                         float *lse, int B, int G, int H, int s_q, int d_qk, int d_v, int page_size,
                                         int max_pages, int num_pages, int causal, float scale, lka_dtype_t dtype,
                                         void *ws, size_t ws_bytes, void *stream);

/* ------------------------------------------------------------------------ */
/* One-time cache conversion latent -> per-group expanded cache             */
/* [GQLA sec. 3.1: switching paths needs a one-time compression/expansion   */
/*  of the KV cache at deployment, never at run time]                       */
/*   kc[b,gamma,j,:] = W^UK_gamma c_j,  vc[b,gamma,j,:] = W^UV_gamma c_j,     */
/*   kr[b,j,:] = k^R_j  for every slot j < Lmax.  bf16 in/out, fp32 sums.   */
/* ------------------------------------------------------------------------ */
LKA_API lka_status_t latent_expand_cache(const void *latent, const void *w_uk, const void *w_uv, int B, int Lmax, int g,
                                 int d_h, int r_kv, int d_r, void *kc, void *vc, void *kr, lka_dtype_t dtype,
                                 void *stream);

/* ------------------------------------------------------------------------ */
/* Helpers                                                                  */
/* ------------------------------------------------------------------------ */
/* Synchronises `stream`, then returns the sticky status word of workspace ws: LKA_OK, or the first raised
 * flag in the order LKA_ERR_TIMEOUT, LKA_ERR_BAD_LENGTH, LKA_ERR_BAD_PAGE, LKA_ERR_RANGE. */
LKA_API lka_status_t lka_device_status(const void *ws, void *stream);
/* Enqueues a reset of the workspace status word to LKA_OK on `stream`. */
LKA_API lka_status_t lka_clear_status(void *ws, void *stream);
/* Human-readable name of a status code (static string, never NULL). */
LKA_API const char *lka_status_string(lka_status_t status);
/* Split size (KV tokens per CTA) for the split-KV kernels of the calls made FROM THE CALLING HOST THREAD;
 * 0 restores the automatic choice.  A tuning and test knob: results do not depend on it beyond rounding,
 * and calls made from other threads keep their own setting (default 0).  Returns the thread's previous value. */
LKA_API int lka_set_split_tokens(int tokens);
/* Timing hook for benchmarks, per host thread: lka_kernel_timing(1) discards the calling thread's earlier
 * records and starts recording a pair of CUDA events around the main (dominant) kernel of every later
 * entry-point call made from that thread, on that call's stream; lka_kernel_timing(0) stops recording.
 * lka_kernel_timing_read waits for the calling thread's recorded events and returns the number of timed
 * launches and their summed duration in milliseconds.  Calls from other threads are never timed by it. */
LKA_API lka_status_t lka_kernel_timing(int enable);
LKA_API lka_status_t lka_kernel_timing_read(int *launches, double *total_ms);
/* Self-test of the bounded in-kernel wait: launches one CTA that waits on a barrier nobody arrives at,
 * for at most limit_us microseconds, then records LKA_ERR_TIMEOUT in ws's status word and exits.
 * Used to check the timeout path without hanging the GPU. */
LKA_API lka_status_t lka_selftest_wait_timeout(void *ws, size_t ws_bytes, int limit_us, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* LKA_H */
