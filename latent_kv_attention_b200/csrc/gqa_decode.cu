// gqa_decode.cu -- split-KV flash decoding for grouped-query attention on
// CUDA cores, and the log-sum-exp merge of its split partials.
//
// Operation ("Grouped Query Attention (GQA)" glossary page, "How GQA works"):
// per query head plain scaled-dot-product attention, with each KV head shared
// by a contiguous group of h_q/h_kv query heads.  Decode is bound by reading
// the KV cache ("How GQA shrinks the KV cache": every new token reads the whole
// cache), at 4 FLOPs per cache byte for 4 heads per group, far below the
// tensor-core ridge, so the contraction runs on the FP32 pipes and the design
// goal is streaming the cache at HBM speed.
//
// One CTA = (sequence b, KV head, block of RB query rows of that group, split
// of the key range).  A producer warp streams K and V tiles of T_TILE tokens
// with TMA (128-byte swizzle) through an NSTAGE ring of mbarrier-guarded
// stages; each KV tile is read from HBM once and used by all query rows of the
// group.  Four consumer warps each own a quarter of every tile and run an
// independent online softmax over it:
//   scores: LPT lanes per token, each lane holding its slice of the RB query
//           rows in registers (pre-scaled by scale*log2 e), a shuffle
//           reduce-scatter over the LPT lanes;
//   softmax: running max / sum per row with warp shuffles, exp2;
//   P*V:    each lane owns D/32 output dims of all RB rows, P is broadcast from
//           shared memory.
// The four warp states are merged in shared memory at the end.  A split whose
// sequence needs a single split writes the final output directly; otherwise it
// writes an fp32 partial (normalised O and log2-domain lse) that
// gqa_combine_kernel merges.
#include <cuda_fp16.h>
#include <cuda_fp8.h>

#include "common.cuh"
#include "gqa_decode.h"
#include "host_util.h"
#include "tc.cuh"

// Tuning knobs of the build: shared-memory budget of the TMA ring per CTA (KiB) and
// the number of CTAs per SM the small-row instances are compiled for.
#ifndef LKA_GQA_STAGE_KB
#define LKA_GQA_STAGE_KB 96
#endif
#ifndef LKA_GQA_MINB
#define LKA_GQA_MINB 2
#endif
// fp32 query values each lane keeps in registers in the score phase
#ifndef LKA_GQA_QREGS
#define LKA_GQA_QREGS 64
#endif

namespace lka {

// One byte of an e4m3 (fp8) cache value.
struct e4m3 {
    uint8_t bits;
};

// Geometry of an instance: KV is the element type of the K/V cache (bf16, fp32 or e4m3), D the head dim,
// RB the query rows per CTA.
template <typename KV, int D, int RB>
struct GqaCfg {
    static constexpr int E = sizeof(KV);
    static constexpr int EPC = 16 / E;           // elements per 16-byte chunk
    static constexpr int CPR = D * E / 16;       // chunks per row
    static constexpr int NSEG = D * E / 128;     // 128-byte swizzle segments per row
    static constexpr int SEG_ELEMS = 128 / E;    // elements per segment (TMA box width)
    // lanes per token in the score phase: enough that the query slice held per
    // lane stays at LKA_GQA_QREGS fp32 registers, never fewer than the rows (so that the
    // reduce-scatter leaves one row per lane), at most one chunk per lane
    static constexpr int LPT0 = RB * D / LKA_GQA_QREGS > RB ? RB * D / LKA_GQA_QREGS : RB;
    static constexpr int LPT1 = LPT0 < CPR ? LPT0 : CPR;
    static constexpr int LPT = LPT1 < 32 ? LPT1 : 32;
    static constexpr int CPL = CPR / LPT;        // chunks per lane
    static constexpr int DUP = LPT / RB;         // lanes holding the same row after the reduction
    static constexpr int P = 32 / LPT;           // tokens per warp pass
    static constexpr int TW = P > 16 ? P : 16;   // tokens per warp per tile
    static constexpr int NPASS = TW / P;
    static constexpr int T_TILE = 4 * TW;
    static constexpr int DPLV = D / 32;          // value dims per lane
    static constexpr int MAT_BYTES = T_TILE * D * E;
    static constexpr int STAGE_BYTES = 2 * MAT_BYTES;
    static constexpr int NSTAGE0 = (LKA_GQA_STAGE_KB * 1024) / STAGE_BYTES;
    static constexpr int NSTAGE_CAP = E == 1 ? 6 : 4;  // the 1-byte cache has half-size stages: keep more
    static constexpr int NSTAGE = NSTAGE0 < 2 ? 2 : (NSTAGE0 > NSTAGE_CAP ? NSTAGE_CAP : NSTAGE0);
    static constexpr int P_BYTES = 4 * TW * RB * 8 + 4 * RB * 4;  // probabilities (stored as pairs) + rescale
    static constexpr int MERGE_BYTES = 4 * RB * D * 4 + 2 * 4 * RB * 4;
    static constexpr int SMEM = 1024 /*align slack*/ + NSTAGE * STAGE_BYTES + P_BYTES + 256 /*barriers*/;
    static constexpr int MINB0 = (RB <= 8 && SMEM <= 110 * 1024) ? 2 : 1;  // resident CTAs per SM
    static constexpr int MINB = (RB <= 4 && LKA_GQA_MINB > MINB0 && SMEM * LKA_GQA_MINB <= 225 * 1024) ? LKA_GQA_MINB
                                                                                                    : MINB0;
    static_assert(D * E >= 128 && (D * E) % 128 == 0, "row must be whole 128-byte segments");
    static_assert(LPT >= RB && LPT <= 32 && LPT <= CPR && CPR % LPT == 0, "lane split must own whole chunks");
    static_assert(MERGE_BYTES <= NSTAGE * STAGE_BYTES, "merge scratch reuses the stage ring");
    static_assert(D % 32 == 0 && (DPLV * E) % 4 == 0, "value slice per lane");
};

// Byte offset of 16-byte chunk `chunk` of segment `seg` of tile row `row`
// inside one TMA-loaded matrix of the stage (SWIZZLE_128B: chunk ^= row % 8).
template <int T_TILE>
__device__ __forceinline__ uint32_t swz_off(int seg, int row, int chunk) {
    return (uint32_t)(seg * T_TILE * 128 + row * 128 + ((chunk ^ (row & 7)) << 4));
}

template <typename T, int DPLV>
__device__ __forceinline__ void load_v_slice(const uint8_t* p, float* v);

template <>
__device__ __forceinline__ void load_v_slice<__nv_bfloat16, 2>(const uint8_t* p, float* v) {
    uint32_t w = *reinterpret_cast<const uint32_t*>(p);
    bf16x2_to_f32(w, v[0], v[1]);
}
template <>
__device__ __forceinline__ void load_v_slice<__nv_bfloat16, 4>(const uint8_t* p, float* v) {
    uint2 w = *reinterpret_cast<const uint2*>(p);
    bf16x2_to_f32(w.x, v[0], v[1]);
    bf16x2_to_f32(w.y, v[2], v[3]);
}
template <>
__device__ __forceinline__ void load_v_slice<__nv_bfloat16, 8>(const uint8_t* p, float* v) {
    uint4 w = *reinterpret_cast<const uint4*>(p);
    bf16x8_to_f32(w, v);
}
template <>
__device__ __forceinline__ void load_v_slice<float, 2>(const uint8_t* p, float* v) {
    float2 w = *reinterpret_cast<const float2*>(p);
    v[0] = w.x;
    v[1] = w.y;
}
template <>
__device__ __forceinline__ void load_v_slice<float, 4>(const uint8_t* p, float* v) {
    float4 w = *reinterpret_cast<const float4*>(p);
    v[0] = w.x;
    v[1] = w.y;
    v[2] = w.z;
    v[3] = w.w;
}

template <typename T>
__device__ __forceinline__ void load_chunk(const uint8_t* p, float* f);
template <>
__device__ __forceinline__ void load_chunk<__nv_bfloat16>(const uint8_t* p, float* f) {
    bf16x8_to_f32(*reinterpret_cast<const uint4*>(p), f);
}
template <>
__device__ __forceinline__ void load_chunk<float>(const uint8_t* p, float* f) {
    float4 w = *reinterpret_cast<const float4*>(p);
    f[0] = w.x;
    f[1] = w.y;
    f[2] = w.z;
    f[3] = w.w;
}

// Two e4m3 values (the low 16 bits of w) as fp32, exactly (e4m3 -> f16 is exact, f16 -> f32 too).
__device__ __forceinline__ float2 e4m3x2_to_f32x2(uint32_t w) {
    const __half2_raw h = __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(w & 0xffffu), __NV_E4M3);
    return __half22float2(*reinterpret_cast<const __half2*>(&h));
}
template <>
__device__ __forceinline__ void load_chunk<e4m3>(const uint8_t* p, float* f) {
    const uint4 w = *reinterpret_cast<const uint4*>(p);
    const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float2 a = e4m3x2_to_f32x2(ws[i]), b = e4m3x2_to_f32x2(ws[i] >> 16);
        f[4 * i] = a.x;
        f[4 * i + 1] = a.y;
        f[4 * i + 2] = b.x;
        f[4 * i + 3] = b.y;
    }
}
template <>
__device__ __forceinline__ void load_v_slice<e4m3, 4>(const uint8_t* p, float* v) {
    const uint32_t w = *reinterpret_cast<const uint32_t*>(p);
    const float2 a = e4m3x2_to_f32x2(w), b = e4m3x2_to_f32x2(w >> 16);
    v[0] = a.x;
    v[1] = a.y;
    v[2] = b.x;
    v[3] = b.y;
}
template <>
__device__ __forceinline__ void load_v_slice<e4m3, 8>(const uint8_t* p, float* v) {
    const uint2 w = *reinterpret_cast<const uint2*>(p);
    load_v_slice<e4m3, 4>(reinterpret_cast<const uint8_t*>(&w.x), v);
    load_v_slice<e4m3, 4>(reinterpret_cast<const uint8_t*>(&w.y), v + 4);
}

// (segment, chunk) of the c-th chunk owned by lane li of a token's LPT lanes.
// Chosen so that every 8-lane shared-memory phase of a 16-byte load touches 8
// distinct bank groups under the 128-byte swizzle.
template <int LPT, int NSEG>
__device__ __forceinline__ void lane_chunk(int li, int c, int& seg, int& chunk) {
    if constexpr (LPT <= 8) {
        constexpr int PER_SEG = 8 / LPT;
        seg = c / PER_SEG;
        chunk = li * PER_SEG + c % PER_SEG;
    } else {
        seg = li / 8 + c * (LPT / 8);
        chunk = li % 8;
    }
}

// Row of token `tok` of sequence b, KV head kvh, in the paged cache [num_pages][h_kv][page_size][D]
// ("Grouped Query Attention (GQA)" glossary page, comparison with related techniques: PagedAttention
// allocates the cache in fixed-size blocks): page block_table[b][tok / page_size], offset tok % page_size.
// Table entries outside [0, num_pages) are replaced by page 0; for a token the attention needs (`live`)
// that raises kDevBadPage.  Tokens past the table's capacity (the tail of a last tile) read page 0.
__device__ __forceinline__ int paged_row(const GqaParams& p, int b, int kvh, int tok, bool live) {
    int page = 0;
    const int j = tok / p.page_size;
    if (j < p.max_pages) {
        page = p.block_table[(size_t)b * p.max_pages + j];
        if (page < 0 || page >= p.num_pages) {
            if (live) atomicOr(p.status, kDevBadPage);
            page = 0;
        }
    }
    return (page * p.h_kv + kvh) * p.page_size + tok % p.page_size;
}

// Whether `pred` holds in any of the 128 consumer threads (named barrier 1 with an OR reduction): a value every
// consumer sees the same.
__device__ __forceinline__ bool consumers_any(bool pred) {
    uint32_t r;
    asm volatile("{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %1, 0;\n\tbar.red.or.pred q, 1, 128, p;\n\t"
                 "selp.u32 %0, 1, 0, q;\n\t}"
                 : "=r"(r)
                 : "r"((uint32_t)pred)
                 : "memory");
    return r != 0;
}

// Issues the copies of one KV tile (K and V of C::T_TILE tokens from token tok0 of sequence b, KV head kvh, as
// 128-byte swizzled segments of C::SEG_ELEMS values) into kdst / vdst, completing on `full`.
template <class C>
__device__ __forceinline__ void gqa_issue_tile(const CUtensorMap* tmK, const CUtensorMap* tmV, const GqaParams& p,
                                               uint32_t kdst, uint32_t vdst, uint32_t full, int b, int kvh, int L,
                                               int tok0) {
    if (!p.block_table) {
        const int y = (b * p.h_kv + kvh) * p.Lmax + tok0;
#pragma unroll
        for (int sg = 0; sg < C::NSEG; ++sg) {
            tma_load_2d(kdst + sg * C::T_TILE * 128, tmK, sg * C::SEG_ELEMS, y, full);
            tma_load_2d(vdst + sg * C::T_TILE * 128, tmV, sg * C::SEG_ELEMS, y, full);
        }
    } else {
        // paged cache: the tile is box_rows-row pieces, each inside one page of the block table
        for (int r0 = 0; r0 < C::T_TILE; r0 += p.box_rows) {
            const int tok = tok0 + r0;
            const int y = paged_row(p, b, kvh, tok, tok < L);
#pragma unroll
            for (int sg = 0; sg < C::NSEG; ++sg) {
                tma_load_2d(kdst + sg * C::T_TILE * 128 + r0 * 128, tmK, sg * C::SEG_ELEMS, y, full);
                tma_load_2d(vdst + sg * C::T_TILE * 128 + r0 * 128, tmV, sg * C::SEG_ELEMS, y, full);
            }
        }
    }
}

// The producer warp's lane 0: streams the split's n_tiles KV tiles through the C::NSTAGE ring of full / empty
// mbarriers, then waits until every copy it issued has landed (a CTA must not exit with copies in flight).
template <class C>
__device__ __forceinline__ void gqa_produce(const CUtensorMap* tmK, const CUtensorMap* tmV, const GqaParams& p,
                                            uint8_t* stages, uint64_t* bars, int* s_abort, int b, int kvh, int L,
                                            int kbeg, int n_tiles) {
    prefetch_tensormap(tmK);
    prefetch_tensormap(tmV);
    int issued = 0;
    for (int it = 0; it < n_tiles; ++it) {
        const int s = it % C::NSTAGE;
        if (it >= C::NSTAGE) {
            if (!mbar_wait(smem_u32(&bars[C::NSTAGE + s]), ((it / C::NSTAGE) - 1) & 1, p.status)) {
                *s_abort = 1;
                break;
            }
        }
        if (*(volatile int*)s_abort) break;
        const uint32_t full = smem_u32(&bars[s]);
        mbar_arrive_expect_tx(full, C::STAGE_BYTES);
        const uint32_t kdst = smem_u32(stages + s * C::STAGE_BYTES);
        gqa_issue_tile<C>(tmK, tmV, p, kdst, kdst + C::MAT_BYTES, full, b, kvh, L, kbeg + it * C::T_TILE);
        ++issued;
    }
    for (int it = issued - 1; it >= 0 && it >= issued - C::NSTAGE; --it)
        mbar_wait(smem_u32(&bars[it % C::NSTAGE]), (it / C::NSTAGE) & 1, p.status);
}

// Merge of the four consumer warps' states of the block's rows (om [4][RB][D] normalisable outputs, mm / lm
// [4][RB] log2-domain maxima and row sums, in shared memory) and the write of each row's result: the output (and
// lse) when the row's keys fit one split, else the split's normalised fp32 partial and lse for the merge kernel.
template <typename T, int D, int RB>
__device__ __forceinline__ void gqa_merge_store(const float* om, const float* mm, const float* lm, const GqaParams& p,
                                                int b, int kvh, int row0, int rows_here, int L, int kbeg, int split,
                                                float v_mul) {
    for (int idx = threadIdx.x; idx < rows_here * D; idx += 128) {
        const int r = idx / D, d = idx % D;
        const int gr = row0 + r;
        const int t = gr % p.s_q;
        const int hq = kvh * p.ratio + gr / p.s_q;
        const size_t orow = ((size_t)b * p.h_q + hq) * p.s_q + t;
        const int n_t = p.causal ? (L - p.s_q + t + 1) : L;
        const int nsp = cdiv(n_t, p.split_tokens);
        if (kbeg >= n_t) continue;  // this row has no keys in this split
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < 4; ++w) M = fmaxf(M, mm[w * RB + r]);
        float lsum = 0.f, acc = 0.f;
#pragma unroll
        for (int w = 0; w < 4; ++w) {
            const float f = exp2f(mm[w * RB + r] - M);  // warps without keys: exp2(-inf) = 0
            lsum += f * lm[w * RB + r];
            acc += f * om[(w * RB + r) * D + d];
        }
        const float ov = acc / lsum * v_mul;
        const float lse2 = M + log2f(lsum);
        if (nsp == 1) {
            reinterpret_cast<T*>(p.out)[orow * D + d] = from_f32<T>(ov);
            if (p.lse && d == 0) p.lse[orow] = lse2 * 0.69314718055994530942f;
        } else {
            p.part_o[(orow * p.nsplit_max + split) * D + d] = ov;
            if (d == 0) p.part_lse[orow * p.nsplit_max + split] = lse2;
        }
    }
}

template <typename T, int D, int RB, typename KV>
__global__ void __launch_bounds__(160, GqaCfg<KV, D, RB>::MINB)
    gqa_decode_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                      const GqaParams p) {
    using C = GqaCfg<KV, D, RB>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(align_up(reinterpret_cast<uintptr_t>(smem_raw), 1024));
    uint8_t* stages = smem;
    float2* p_buf = reinterpret_cast<float2*>(smem + C::NSTAGE * C::STAGE_BYTES);  // [4][TW][RB] (p, p) pairs
    float* a_buf = reinterpret_cast<float*>(p_buf + 4 * C::TW * RB);                 // [4][RB]
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::NSTAGE * C::STAGE_BYTES + C::P_BYTES);
    __shared__ int s_abort;

    const int split = blockIdx.x;
    const int kvh = blockIdx.y / p.n_rb;
    const int rb = blockIdx.y % p.n_rb;
    const int b = blockIdx.z;
    const int R = p.ratio * p.s_q;  // query rows of this group
    const int row0 = rb * RB;
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;

    const int L = clamp_len(p.lens, b, p.Lmax, p.s_q, p.causal, p.status,
                            threadIdx.x == 0 && split == 0 && kvh == 0 && rb == 0);
    // keys needed by the rows of this block: causal row t sees L - s_q + t + 1
    int rows_here = R - row0 < RB ? R - row0 : RB;
    int need = L;
    if (p.causal) {
        int tmax = 0;
        for (int r = 0; r < rows_here; ++r) {
            int t = (row0 + r) % p.s_q;
            tmax = t > tmax ? t : tmax;
        }
        need = L - p.s_q + tmax + 1;
    }
    const int kbeg = split * p.split_tokens;
    if (kbeg >= need) return;  // no row of this block has keys in this split
    const int kend = min(need, kbeg + p.split_tokens);
    const int n_tiles = cdiv(kend - kbeg, C::T_TILE);

    if (threadIdx.x == 0) {
        s_abort = 0;
        for (int s = 0; s < C::NSTAGE; ++s) {
            mbar_init(smem_u32(&bars[s]), 1);                 // full: producer arrival + tx bytes
            mbar_init(smem_u32(&bars[C::NSTAGE + s]), 4);     // empty: one arrival per consumer warp
        }
        fence_barrier_init();
    }
    __syncthreads();

    if (warp == 4) {
        // ------------------------------ producer ------------------------------
        if (lane == 0) gqa_produce<C>(&tmK, &tmV, p, stages, bars, &s_abort, b, kvh, L, kbeg, n_tiles);
        return;
    }

    // -------------------------------- consumers --------------------------------
    const int li = lane % C::LPT;           // lane within the token's lane group
    const int tok_in_pass = lane / C::LPT;  // token of this lane within a pass
    const int my_row = li / C::DUP;         // row this lane holds after the reduction
    const int g_row = row0 + my_row;        // row index within the group
    const bool row_ok = g_row < R;
    const int my_t = row_ok ? g_row % p.s_q : 0;
    const int my_last = p.causal ? (L - p.s_q + my_t) : (L - 1);  // last visible key of my row

    // query slice of this lane, pre-scaled into the log2 domain
    // the two halves of each pair multiply consecutive key elements (packed fp32x2 FMAs)
    float qreg[RB][C::CPL * C::EPC];
    // the softmax scale in the log2 domain, and the dequantisation scale of a quantised key cache
    const float q_mul = p.scale_log2 * (p.k_scale ? p.k_scale[kvh] : 1.f);
    {
        const T* qbase = reinterpret_cast<const T*>(p.q) +
                         ((size_t)(b * p.h_q + kvh * p.ratio) * p.s_q) * D;  // first row of the group
#pragma unroll
        for (int r = 0; r < RB; ++r) {
            const bool ok = row0 + r < R;
#pragma unroll
            for (int c = 0; c < C::CPL; ++c) {
                int seg, chunk;
                lane_chunk<C::LPT, C::NSEG>(li, c, seg, chunk);
                const int e0 = seg * C::SEG_ELEMS + chunk * C::EPC;
#pragma unroll
                for (int e = 0; e < C::EPC; ++e)
                    qreg[r][c * C::EPC + e] = ok ? to_f32<T>(qbase[(size_t)(row0 + r) * D + e0 + e]) * q_mul : 0.f;
            }
        }
    }

    float m_run = -INFINITY, l_run = 0.f;
    float2 o[RB][C::DPLV / 2];
#pragma unroll
    for (int r = 0; r < RB; ++r)
#pragma unroll
        for (int d = 0; d < C::DPLV / 2; ++d) o[r][d] = make_float2(0.f, 0.f);

    float2* pw = p_buf + warp * C::TW * RB;
    float* aw = a_buf + warp * RB;
    bool aborted = false;
    // keys below mask_from are visible to every row of the block: tiles below it need no mask
    int mask_from = kend;
    for (int r = 0; r < rows_here; ++r) {
        const int last = p.causal ? L - p.s_q + (row0 + r) % p.s_q : L - 1;
        mask_from = min(mask_from, last + 1);
    }

    // Byte offsets, inside a stage, of the chunks this lane reads.  Score phase: token row jt = warp * TW +
    // ps * P + tok_in_pass; TW is a multiple of 8, so the swizzle phase jt & 7 only depends on ps through
    // (ps * P) & 7, which takes NCLS values.  Value phase: row warp * TW + jj has swizzle phase jj & 7.
    constexpr int NCLS = C::P >= 8 ? 1 : 8 / C::P;
    uint32_t koff[NCLS][C::CPL];
#pragma unroll
    for (int cls = 0; cls < NCLS; ++cls)
#pragma unroll
        for (int c = 0; c < C::CPL; ++c) {
            int seg, chunk;
            lane_chunk<C::LPT, C::NSEG>(li, c, seg, chunk);
            koff[cls][c] = swz_off<C::T_TILE>(seg, warp * C::TW + cls * C::P + tok_in_pass, chunk);
        }
    const int v_ob = lane * C::DPLV * C::E;  // byte offset of this lane's value slice in a row
    const int v_seg = v_ob / 128, v_chunk = (v_ob % 128) / 16, v_in = v_ob % 16;
    uint32_t voff[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) voff[k] = swz_off<C::T_TILE>(v_seg, warp * C::TW + k, v_chunk) + v_in;

    for (int it = 0; it < n_tiles; ++it) {
        const int s = it % C::NSTAGE;
        if (!mbar_wait(smem_u32(&bars[s]), (it / C::NSTAGE) & 1, p.status)) {
            aborted = true;
            s_abort = 1;
            break;
        }
        const uint8_t* kt = stages + s * C::STAGE_BYTES;
        const uint8_t* vt = kt + C::MAT_BYTES;
        const int tbase = kbeg + it * C::T_TILE;

        // ---- scores for this warp's TW tokens ----
        float sc[C::NPASS];
#pragma unroll
        for (int ps = 0; ps < C::NPASS; ++ps) {
            const int jt = warp * C::TW + ps * C::P + tok_in_pass;  // token row in the tile
            float2 acc2[RB];
#pragma unroll
            for (int r = 0; r < RB; ++r) acc2[r] = make_float2(0.f, 0.f);
#pragma unroll
            for (int c = 0; c < C::CPL; ++c) {
                float kf[C::EPC];
                load_chunk<KV>(kt + koff[ps % NCLS][c] + (ps / NCLS) * NCLS * C::P * 128, kf);
#pragma unroll
                for (int r = 0; r < RB; ++r)
#pragma unroll
                    for (int e = 0; e < C::EPC; e += 2)
                        acc2[r] = __ffma2_rn(make_float2(qreg[r][c * C::EPC + e], qreg[r][c * C::EPC + e + 1]),
                                             make_float2(kf[e], kf[e + 1]), acc2[r]);
            }
            float acc[RB];
#pragma unroll
            for (int r = 0; r < RB; ++r) acc[r] = acc2[r].x + acc2[r].y;
            // reduce-scatter over the LPT lanes of the token: lane li ends with row li / DUP
            int nr = RB;
#pragma unroll
            for (int m = C::LPT / 2; m >= 1; m /= 2) {
                if (nr > 1) {
                    const bool upper = (li & m) != 0;
                    const int half = nr / 2;
#pragma unroll
                    for (int k2 = 0; k2 < RB / 2; ++k2) {
                        if (k2 < half) {
                            float send = upper ? acc[k2] : acc[half + k2];
                            float keep = upper ? acc[half + k2] : acc[k2];
                            acc[k2] = keep + __shfl_xor_sync(0xffffffffu, send, m);
                        }
                    }
                    nr = half;
                } else {
                    acc[0] += __shfl_xor_sync(0xffffffffu, acc[0], m);
                }
            }
            if (tbase + C::T_TILE > mask_from) {
                const int kpos = tbase + jt;
                const bool ok = row_ok && kpos < kend && kpos <= my_last;
                sc[ps] = ok ? acc[0] : -INFINITY;
            } else {
                sc[ps] = acc[0];
            }
        }

        // ---- online softmax over this warp's tokens (per row), lazily rescaled: p is taken against a
        // reference maximum m_run that only moves when a score exceeds it by more than 2^8 (the final
        // O / l is exact); the row maximum is only reduced across the lanes when that happens ----
        float mx = sc[0];
#pragma unroll
        for (int ps = 1; ps < C::NPASS; ++ps) mx = fmaxf(mx, sc[ps]);
        if (__any_sync(0xffffffffu, mx > m_run + 8.0f)) {  // (an unset reference is exceeded by any key)
#pragma unroll
            for (int m = C::LPT; m < 32; m *= 2) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, m));
            const float m_new = fmaxf(m_run, mx);
            float alpha = 1.f;
            if (m_run == -INFINITY) {
                m_run = m_new;  // O and l of the row are still zero
            } else if (m_new > m_run + 8.0f) {
                alpha = fast_exp2(m_run - m_new);
                m_run = m_new;
            }
            if (__any_sync(0xffffffffu, alpha != 1.f)) {
                l_run *= alpha;
                if (tok_in_pass == 0 && li % C::DUP == 0) aw[my_row] = alpha;
                __syncwarp();
                float al[RB];
#pragma unroll
                for (int r = 0; r < RB; ++r) al[r] = aw[r];
#pragma unroll
                for (int r = 0; r < RB; ++r)
#pragma unroll
                    for (int d = 0; d < C::DPLV / 2; ++d)
                        o[r][d] = __fmul2_rn(o[r][d], make_float2(al[r], al[r]));
                __syncwarp();
            }
        }
        {
            const float m_sub = m_run == -INFINITY ? 0.f : m_run;  // no visible key yet: p = 2^-inf = 0
#pragma unroll
            for (int ps = 0; ps < C::NPASS; ++ps) {
                const float pv = fast_exp2(sc[ps] - m_sub);
                l_run += pv;  // this lane's share; summed over the lanes of the row at the end
                if (li % C::DUP == 0) pw[(ps * C::P + tok_in_pass) * RB + my_row] = make_float2(pv, pv);
            }
        }
        __syncwarp();

        // ---- O += P V over this warp's tokens ----
        {
            int nvalid = kend - (tbase + warp * C::TW);
            nvalid = nvalid < 0 ? 0 : (nvalid > C::TW ? C::TW : nvalid);
            if (nvalid == C::TW) {
                // every token of this warp's quarter is a key: fully unrolled, constant offsets
#pragma unroll
                for (int jj = 0; jj < C::TW; ++jj) {
                    float vf[C::DPLV];
                    load_v_slice<KV, C::DPLV>(vt + voff[jj & 7] + (jj & ~7) * 128, vf);
                    float2 pj[RB];
                    if constexpr (RB % 2 == 0) {
                        const float4* pr4 = reinterpret_cast<const float4*>(pw + jj * RB);
#pragma unroll
                        for (int rp = 0; rp < RB / 2; ++rp) {
                            const float4 v4 = pr4[rp];
                            pj[2 * rp] = make_float2(v4.x, v4.y);
                            pj[2 * rp + 1] = make_float2(v4.z, v4.w);
                        }
                    } else {
#pragma unroll
                        for (int r = 0; r < RB; ++r) pj[r] = pw[jj * RB + r];
                    }
#pragma unroll
                    for (int r = 0; r < RB; ++r)
#pragma unroll
                        for (int d = 0; d < C::DPLV / 2; ++d)
                            o[r][d] = __ffma2_rn(pj[r], make_float2(vf[2 * d], vf[2 * d + 1]), o[r][d]);
                }
            } else {
#pragma unroll 4
                for (int jj = 0; jj < nvalid; ++jj) {
                    const int jt = warp * C::TW + jj;
                    float vf[C::DPLV];
                    load_v_slice<KV, C::DPLV>(vt + swz_off<C::T_TILE>(v_seg, jt, v_chunk) + v_in, vf);
                    const float2* pr = pw + jj * RB;
#pragma unroll
                    for (int r = 0; r < RB; ++r) {
                        const float2 pj = pr[r];
#pragma unroll
                        for (int d = 0; d < C::DPLV / 2; ++d)
                            o[r][d] = __ffma2_rn(pj, make_float2(vf[2 * d], vf[2 * d + 1]), o[r][d]);
                    }
                }
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&bars[C::NSTAGE + s]));
    }

    // the row sums: this lane's share summed over the token groups of the warp
#pragma unroll
    for (int m = C::LPT; m < 32; m *= 2) l_run += __shfl_xor_sync(0xffffffffu, l_run, m);

    // all consumer warps reach here; aborted CTAs stop without writing results (the decision is the same in
    // every consumer thread)
    if (consumers_any(aborted || *(volatile int*)&s_abort)) return;

    // ---- merge the four warp states in shared memory (reusing the stage ring) ----
    float* om = reinterpret_cast<float*>(stages);  // [4][RB][D]
    float* mm = om + 4 * RB * D;                    // [4][RB]
    float* lm = mm + 4 * RB;                        // [4][RB]
#pragma unroll
    for (int r = 0; r < RB; ++r)
#pragma unroll
        for (int d = 0; d < C::DPLV / 2; ++d)
            *reinterpret_cast<float2*>(&om[(warp * RB + r) * D + lane * C::DPLV + 2 * d]) = o[r][d];
    if (tok_in_pass == 0 && li % C::DUP == 0) {
        mm[warp * RB + my_row] = m_run;
        lm[warp * RB + my_row] = l_run;
    }
    named_barrier(1, 128);

    const float v_mul = p.v_scale ? p.v_scale[kvh] : 1.f;  // dequantisation scale of a quantised value cache
    gqa_merge_store<T, D, RB>(om, mm, lm, p, b, kvh, row0, rows_here, L, kbeg, split, v_mul);
}


// ---- tensor-core instances: bf16 caches (d in {64, 128}) and e4m3 caches (d = 128) -------------------------------
// The block's query rows (up to 16: h_q / h_kv heads x s_q tokens; rows past R are zero padding) are the M = 16
// rows of mma.sync m16n8k16 MMAs with fp32 accumulators.  Per tile each consumer warp takes 16 tokens: the scores
// are d/16 k-steps x 2 n-tiles of MMAs, and the accumulator layout of the score MMA is the A-operand layout of the
// P*V MMA, so P goes from the softmax to the d/8 P*V MMAs in registers.  At about 4 FLOPs per cache byte the MMAs
// are not there for throughput: they replace the score / value FMAs, shuffles and conversions of the CUDA-core loop
// (about 34 warp instructions per token and KV head) with a handful, so that the consumers keep up with the TMA
// stream at two CTAs per SM.
//   bf16 cache: bf16 MMAs; ldmatrix reads K (and, transposed, V) straight from the swizzled stage; P is bf16 (as in
//     every tensor-core path of the library).
//   e4m3 cache: f16 MMAs (e4m3 -> f16 is exact; q bf16 -> f16 too, for values of ordinary size).  The score
//     contraction runs over the head dim in a permuted order, the same for q and k, so that each lane reads 16
//     consecutive key bytes per token with one shared-memory load and widens them in registers: in 64-value
//     group G, lane tq's k-step 4 G + j covers values 64 G + 16 tq + 4 j + {0, 1} (as k = 2 tq, 2 tq + 1) and
//     + {2, 3} (as k = 2 tq + 8, 2 tq + 9).  The n-th token column of an n-tile is token pi(n) = n / 2 + 4 (n % 2)
//     of its 8 (so that the two rows a shared-memory phase reads fall in different bank halves).  Values go from
//     the stage to the P*V MMA in registers: each lane reads the 16 value bytes of one head-dim chunk of the four
//     tokens of its k-pairs, pairs the two tokens of each k-pair byte by byte (prmt) and widens the pair with one
//     conversion, the output columns following the chunk order.  P is f16; the per-KV-head scales are applied to
//     the fp32 scores and to the merged output.
template <int D, bool F8, bool R8 = false>
struct GqaMmaCfg {
    static constexpr int RB = 16;                  // query rows per CTA (the MMA's M)
    static constexpr int TW = 16;                  // tokens per warp per tile
    static constexpr int T_TILE = 4 * TW;
    static constexpr int E = F8 ? 1 : 2;           // bytes per cache element
    static constexpr int SEG_ELEMS = 128 / E;      // elements per 128-byte swizzle segment (TMA box width)
    static constexpr int NSEG = D * E / 128;
    static constexpr int MAT_BYTES = T_TILE * D * E;
    static constexpr int STAGE_BYTES = 2 * MAT_BYTES;
    static constexpr int NSTAGE0 = (LKA_GQA_STAGE_KB * 1024) / STAGE_BYTES;
    // R8: the 8-row form.  Its e4m3 instance runs three CTAs per SM (four stages each); every other instance runs
    // two (the 16-row e4m3 form does not fit three in registers)
    static constexpr int NSTAGE_CAP = F8 && R8 ? 4 : 6;
    static constexpr int NSTAGE = NSTAGE0 > NSTAGE_CAP ? NSTAGE_CAP : NSTAGE0;
    static constexpr int RING = NSTAGE * STAGE_BYTES;
    static constexpr int OFF_BAR = RING;
    static constexpr int MERGE_BYTES = 4 * RB * D * 4 + 2 * 4 * RB * 4;
    static constexpr int SMEM = 1024 + OFF_BAR + 256;
    static constexpr int MINB = F8 && R8 ? 3 : 2;
    static_assert(F8 ? D == 128 : (D == 64 || D == 128), "head dim of the tensor-core instances");
    static_assert(MERGE_BYTES <= RING && NSTAGE >= 2 && MINB * (SMEM + 1024) <= 228 * 1024, "shared memory");
};

template <bool F16>
__device__ __forceinline__ void mma_16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    if constexpr (F16)
        asm volatile("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
                     "{%8, %9}, {%0, %1, %2, %3};"
                     : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
                     : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
    else
        asm volatile("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
                     "{%8, %9}, {%0, %1, %2, %3};"
                     : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
                     : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
// Four 8x8 b16 matrices from shared memory; lane l gives the address of row l % 8 of matrix l / 8.
__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t (&r)[4]) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr)
                 : "memory");
}
// The same, each matrix transposed on the way into the registers.
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t (&r)[4]) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr)
                 : "memory");
}
// The two e4m3 values of the low (bytes 0, 1) or high (bytes 2, 3) half of w as an f16 pair, exactly; the lower
// byte becomes the lower half.  One conversion instruction reading the register half in place.
__device__ __forceinline__ uint32_t e4m3x2_lo_to_f16x2(uint32_t w) {
    uint32_t r;
    asm("{\n\t.reg .b16 lo, hi;\n\tmov.b32 {lo, hi}, %1;\n\tcvt.rn.f16x2.e4m3x2 %0, lo;\n\t}" : "=r"(r) : "r"(w));
    return r;
}
__device__ __forceinline__ uint32_t e4m3x2_hi_to_f16x2(uint32_t w) {
    uint32_t r;
    asm("{\n\t.reg .b16 lo, hi;\n\tmov.b32 {lo, hi}, %1;\n\tcvt.rn.f16x2.e4m3x2 %0, hi;\n\t}" : "=r"(r) : "r"(w));
    return r;
}
__device__ __forceinline__ uint32_t pack_f16x2_rn(float lo, float hi) {
    const __half2 v = __floats2half2_rn(lo, hi);  // .x = lo (low 16 bits), .y = hi
    return *reinterpret_cast<const uint32_t*>(&v);
}
// Physical token (of 8) of token column n of an n-tile in the e4m3 instance, and the inverse.
__device__ __forceinline__ int f8_tok(int n) { return (n >> 1) + 4 * (n & 1); }
__device__ __forceinline__ int f8_col(int t) { return 2 * (t & 3) + (t >> 2); }

template <int D, bool F8>
__global__ void __launch_bounds__(160, GqaMmaCfg<D, F8>::MINB)
    gqa_decode_mma_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                          const GqaParams p) {
    using C = GqaMmaCfg<D, F8>;
    constexpr int RB = C::RB, KS = D / 16, NT = D / 8;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(align_up(reinterpret_cast<uintptr_t>(smem_raw), 1024));
    uint8_t* stages = smem;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
    __shared__ int s_abort;

    const int split = blockIdx.x;
    const int kvh = blockIdx.y / p.n_rb;
    const int rb = blockIdx.y % p.n_rb;
    const int b = blockIdx.z;
    const int R = p.ratio * p.s_q;  // query rows of this group
    const int row0 = rb * RB;
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;

    const int L = clamp_len(p.lens, b, p.Lmax, p.s_q, p.causal, p.status,
                            threadIdx.x == 0 && split == 0 && kvh == 0 && rb == 0);
    const int rows_here = R - row0 < RB ? R - row0 : RB;
    int need = L;  // keys needed by the rows of this block: causal row t sees L - s_q + t + 1
    if (p.causal) {
        int tmax = 0;
        for (int r = 0; r < rows_here; ++r) tmax = max(tmax, (row0 + r) % p.s_q);
        need = L - p.s_q + tmax + 1;
    }
    const int kbeg = split * p.split_tokens;
    if (kbeg >= need) return;  // no row of this block has keys in this split
    const int kend = min(need, kbeg + p.split_tokens);
    const int n_tiles = cdiv(kend - kbeg, C::T_TILE);

    if (threadIdx.x == 0) {
        s_abort = 0;
        for (int s = 0; s < C::NSTAGE; ++s) {
            mbar_init(smem_u32(&bars[s]), 1);              // full: producer arrival + tx bytes
            mbar_init(smem_u32(&bars[C::NSTAGE + s]), 4);  // empty: one arrival per consumer warp
        }
        fence_barrier_init();
    }
    __syncthreads();

    if (warp == 4) {
        if (lane == 0) gqa_produce<C>(&tmK, &tmV, p, stages, bars, &s_abort, b, kvh, L, kbeg, n_tiles);
        return;
    }

    // -------------------------------- consumers --------------------------------
    // Fragment coordinates: lane = 4 g + tq holds rows g and g + 8 of the block and, in a score n-tile, the
    // token columns 2 tq and 2 tq + 1.
    const int g = lane >> 2, tq = lane & 3;
    int last[2];  // last visible key of the lane's two rows (-1: a padding row, nothing visible)
    uint32_t qa[KS][4];  // A fragments of the score MMA: the queries as given (the scale goes on the fp32 scores)
    {
        const __nv_bfloat16* qbase = reinterpret_cast<const __nv_bfloat16*>(p.q) +
                                     ((size_t)(b * p.h_q + kvh * p.ratio) * p.s_q) * D;  // first row of the group
        const uint32_t* qrow[2];
        bool ok[2];
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            const int gr = row0 + g + 8 * i;
            ok[i] = gr < R;
            last[i] = ok[i] ? (p.causal ? L - p.s_q + gr % p.s_q : L - 1) : -1;
            qrow[i] = reinterpret_cast<const uint32_t*>(qbase + (size_t)(ok[i] ? gr : 0) * D);
        }
        // bf16 pair u (values 2u, 2u + 1) of row i, as the MMA's operand type
        auto qpair = [&](int i, int u) -> uint32_t {
            const uint32_t w = ok[i] ? qrow[i][u] : 0u;
            if constexpr (F8) {
                float lo, hi;
                bf16x2_to_f32(w, lo, hi);
                return pack_f16x2_rn(lo, hi);
            } else {
                return w;
            }
        };
#pragma unroll
        for (int ks = 0; ks < KS; ++ks) {
            // pairs of values: bf16 layout 16 ks + 2 tq (+ 8); e4m3 permuted layout 64 G + 16 tq + 4 j (+ 2)
            const int u0 = F8 ? 32 * (ks >> 2) + 8 * tq + 2 * (ks & 3) : 8 * ks + tq;
            const int u1 = F8 ? u0 + 1 : u0 + 4;
            qa[ks][0] = qpair(0, u0);
            qa[ks][1] = qpair(1, u0);
            qa[ks][2] = qpair(0, u1);
            qa[ks][3] = qpair(1, u1);
        }
    }
    float o[NT][4];
#pragma unroll
    for (int j = 0; j < NT; ++j) o[j][0] = o[j][1] = o[j][2] = o[j][3] = 0.f;
    float m_run[2] = {-INFINITY, -INFINITY}, l_run[2] = {0.f, 0.f};
    // the softmax scale in the log2 domain, and the dequantisation scale of an e4m3 key cache
    const float s_mul = F8 ? p.scale_log2 * p.k_scale[kvh] : p.scale_log2;
    // keys below mask_from are visible to every row of the block: tiles below it need no mask
    int mask_from = kend;
    for (int r = 0; r < rows_here; ++r)
        mask_from = min(mask_from, p.causal ? L - p.s_q + (row0 + r) % p.s_q + 1 : L);
    // token (of the warp's 16) of score element (nt, e) of this lane
    auto tok_of = [&](int nt, int e) { return 8 * nt + (F8 ? f8_tok(2 * tq + (e & 1)) : 2 * tq + (e & 1)); };

    // ldmatrix row addresses of the bf16 stage (byte offsets, 128-byte swizzle: chunk ^ row % 8).  Keys: matrix
    // l / 8 = (token half l / 16, 8-value chunk parity (l / 8) % 2) of the warp's 16 tokens: the b0 / b1 fragments
    // of n-tiles 0 and 1 for one k-step.  Values (transposed): matrix l / 8 = (chunk parity l / 16, token half
    // (l / 8) % 2): b0 / b1 of two adjacent 8-column output n-tiles.
    const int r8 = lane & 7;
    const uint32_t k_row = (uint32_t)(16 * warp + 8 * (lane >> 4) + r8) * 128;
    const uint32_t v_row = (uint32_t)(16 * warp + 8 * ((lane >> 3) & 1) + r8) * 128;
    constexpr int V_SEG = C::T_TILE * 128;  // bytes per 64-value segment of a bf16 value tile
    uint32_t k_off[4], v_off[4];
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        k_off[c] = k_row + ((uint32_t)((2 * c + ((lane >> 3) & 1)) ^ r8) << 4);
        v_off[c] = v_row + ((uint32_t)((2 * c + (lane >> 4)) ^ r8) << 4);
    }
    // e4m3: this lane's key row of n-tile nt (token column g), and its head-dim chunk of the values: column n of
    // output n-tile nt is head-dim value 16 vch(n) + nt, vch putting the chunks of lanes g = 2 i, 2 i + 1 in
    // different halves of the swizzled row (the 8 lanes of a shared-memory phase read 8 different columns)
    const int kf_row0 = 16 * warp + f8_tok(g);
    auto vch = [](int n) { return ((n & 1) << 2) | (n >> 1); };

    bool aborted = false;
    for (int it = 0; it < n_tiles; ++it) {
        const int s = it % C::NSTAGE;
        if (!mbar_wait(smem_u32(&bars[s]), (it / C::NSTAGE) & 1, p.status)) {
            aborted = true;
            s_abort = 1;
            break;
        }
        const uint32_t kt = smem_u32(stages + s * C::STAGE_BYTES);
        const uint32_t vt = kt + C::MAT_BYTES;
        const int tbase = kbeg + it * C::T_TILE;

        // ---- S = Q K^T for the warp's 16 tokens (two accumulators per n-tile: even / odd k-steps) ----
        float sc[2][2][4];
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
            for (int h = 0; h < 2; ++h) sc[nt][h][0] = sc[nt][h][1] = sc[nt][h][2] = sc[nt][h][3] = 0.f;
        if constexpr (F8) {
            const uint8_t* kst = stages + s * C::STAGE_BYTES;
#pragma unroll
            for (int nt = 0; nt < 2; ++nt) {
                const int row = kf_row0 + 8 * nt;
#pragma unroll
                for (int G = 0; G < D / 64; ++G) {
                    const int seg = G >> 1, chunk = 4 * (G & 1) + tq;
                    const uint4 w = *reinterpret_cast<const uint4*>(kst + seg * C::T_TILE * 128 + row * 128 +
                                                                    ((chunk ^ (row & 7)) << 4));
                    const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
                    for (int j = 0; j < 4; ++j)
                        mma_16816<true>(sc[nt][j & 1], qa[4 * G + j], e4m3x2_lo_to_f16x2(ws[j]),
                                        e4m3x2_hi_to_f16x2(ws[j]));
                }
            }
        } else {
#pragma unroll
            for (int ks = 0; ks < KS; ++ks) {
                uint32_t kb[4];
                ldsm_x4(kt + (ks >> 2) * C::T_TILE * 128 + k_off[ks & 3], kb);
                mma_16816<false>(sc[0][ks & 1], qa[ks], kb[0], kb[1]);
                mma_16816<false>(sc[1][ks & 1], qa[ks], kb[2], kb[3]);
            }
        }
        // x[nt][e]: row g (e < 2) or g + 8, token tbase + 16 warp + tok_of(nt, e), in the log2 domain
        float x[2][4];
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) x[nt][e] = (sc[nt][0][e] + sc[nt][1][e]) * s_mul;
        if (tbase + C::T_TILE > mask_from) {
#pragma unroll
            for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int tok = tbase + 16 * warp + tok_of(nt, e);
                    x[nt][e] = (tok < kend && tok <= last[e >> 1]) ? x[nt][e] : -INFINITY;
                }
        }
        // ---- online softmax of the two rows, lazily rescaled: p is taken against a reference maximum m_run
        // that only moves when a score exceeds it by more than 2^8 (the final O / l is exact) ----
        float mx[2];
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            mx[i] = fmaxf(fmaxf(x[0][2 * i], x[0][2 * i + 1]), fmaxf(x[1][2 * i], x[1][2 * i + 1]));
            mx[i] = fmaxf(mx[i], __shfl_xor_sync(0xffffffffu, mx[i], 1));
            mx[i] = fmaxf(mx[i], __shfl_xor_sync(0xffffffffu, mx[i], 2));
        }
        if (__any_sync(0xffffffffu, mx[0] > m_run[0] + 8.0f || mx[1] > m_run[1] + 8.0f)) {
            float alpha[2];
#pragma unroll
            for (int i = 0; i < 2; ++i) {
                const float m_new = fmaxf(m_run[i], mx[i]);
                alpha[i] = 1.f;
                if (m_run[i] == -INFINITY) {
                    m_run[i] = m_new;  // O and l of the row are still zero
                } else if (m_new > m_run[i] + 8.0f) {
                    alpha[i] = fast_exp2(m_run[i] - m_new);
                    m_run[i] = m_new;
                }
                l_run[i] *= alpha[i];
            }
#pragma unroll
            for (int j = 0; j < NT; ++j) {
                o[j][0] *= alpha[0];
                o[j][1] *= alpha[0];
                o[j][2] *= alpha[1];
                o[j][3] *= alpha[1];
            }
        }
        uint32_t pa[4];  // A fragment of the P*V MMA (k = the warp's 16 tokens in score-column order)
        {
            const float ms0 = m_run[0] == -INFINITY ? 0.f : m_run[0];  // no visible key yet: p = 2^-inf = 0
            const float ms1 = m_run[1] == -INFINITY ? 0.f : m_run[1];
            float pr[2][4];
#pragma unroll
            for (int nt = 0; nt < 2; ++nt) {
                pr[nt][0] = fast_exp2(x[nt][0] - ms0);
                pr[nt][1] = fast_exp2(x[nt][1] - ms0);
                pr[nt][2] = fast_exp2(x[nt][2] - ms1);
                pr[nt][3] = fast_exp2(x[nt][3] - ms1);
                l_run[0] += pr[nt][0] + pr[nt][1];  // this lane's share; summed over the row's lanes at the end
                l_run[1] += pr[nt][2] + pr[nt][3];
            }
#pragma unroll
            for (int nt = 0; nt < 2; ++nt) {
                pa[2 * nt] = F8 ? pack_f16x2_rn(pr[nt][0], pr[nt][1]) : pack_bf16x2(pr[nt][0], pr[nt][1]);
                pa[2 * nt + 1] = F8 ? pack_f16x2_rn(pr[nt][2], pr[nt][3]) : pack_bf16x2(pr[nt][2], pr[nt][3]);
            }
        }
        const int nvalid = kend - (tbase + 16 * warp);  // value rows of the warp that are keys of the split
        if constexpr (F8) {
            // ---- O += P V straight from the e4m3 stage: lane (g, tq) reads value chunk vch(g) of the warp's
            // tokens tq, tq + 4, 8 + tq, 12 + tq (k-indices 2 tq, 2 tq + 1, 2 tq + 8, 2 tq + 9 in score-column
            // order); byte permutes pair the two tokens of each k-pair, one conversion widens a pair into a B
            // register.  Rows past the split's keys may hold anything (even NaN), which P = 0 would not cancel in
            // the MMA: they become 0 ----
            const uint8_t* vsrc = stages + s * C::STAGE_BYTES + C::MAT_BYTES;
            const int ch = vch(g);
            uint32_t vw[4][4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int t = tq + 4 * j;  // token of the warp's 16
                const int row = 16 * warp + t;
                uint4 w = *reinterpret_cast<const uint4*>(vsrc + row * 128 + ((ch ^ (row & 7)) << 4));
                if (t >= nvalid) w = make_uint4(0u, 0u, 0u, 0u);
                vw[j][0] = w.x;
                vw[j][1] = w.y;
                vw[j][2] = w.z;
                vw[j][3] = w.w;
            }
#pragma unroll
            for (int q = 0; q < 4; ++q) {  // value bytes 4 q .. 4 q + 3 of the chunk: n-tiles 4 q .. 4 q + 3
                const uint32_t lo01 = __byte_perm(vw[0][q], vw[1][q], 0x5140), hi01 = __byte_perm(vw[0][q], vw[1][q], 0x7362);
                const uint32_t lo23 = __byte_perm(vw[2][q], vw[3][q], 0x5140), hi23 = __byte_perm(vw[2][q], vw[3][q], 0x7362);
                mma_16816<true>(o[4 * q], pa, e4m3x2_lo_to_f16x2(lo01), e4m3x2_lo_to_f16x2(lo23));
                mma_16816<true>(o[4 * q + 1], pa, e4m3x2_hi_to_f16x2(lo01), e4m3x2_hi_to_f16x2(lo23));
                mma_16816<true>(o[4 * q + 2], pa, e4m3x2_lo_to_f16x2(hi01), e4m3x2_lo_to_f16x2(hi23));
                mma_16816<true>(o[4 * q + 3], pa, e4m3x2_hi_to_f16x2(hi01), e4m3x2_hi_to_f16x2(hi23));
            }
        } else {
            if (nvalid < 16) {
                // value rows of the warp past the split's keys (the last tile) may hold anything, even NaN, and
                // P = 0 does not cancel that in the MMA: zero them
                const int first = nvalid < 0 ? 0 : nvalid;
                uint8_t* vrow = stages + s * C::STAGE_BYTES + C::MAT_BYTES;
                for (int idx = lane; idx < (16 - first) * C::NSEG * 8; idx += 32) {
                    const int row = 16 * warp + first + idx / (C::NSEG * 8), rem = idx % (C::NSEG * 8);
                    *reinterpret_cast<uint4*>(vrow + (rem / 8) * C::T_TILE * 128 + row * 128 + (rem % 8) * 16) =
                        make_uint4(0u, 0u, 0u, 0u);
                }
                asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // before the ring's next copy
                __syncwarp();
            }
            // ---- O += P V ----
#pragma unroll
            for (int cc = 0; cc < NT / 2; ++cc) {
                uint32_t vb[4];
                ldsm_x4_t(vt + (cc >> 2) * V_SEG + v_off[cc & 3], vb);
                mma_16816<false>(o[2 * cc], pa, vb[0], vb[1]);
                mma_16816<false>(o[2 * cc + 1], pa, vb[2], vb[3]);
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&bars[C::NSTAGE + s]));
    }

    // the row sums: this lane's share summed over the four lanes of the row
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        l_run[i] += __shfl_xor_sync(0xffffffffu, l_run[i], 1);
        l_run[i] += __shfl_xor_sync(0xffffffffu, l_run[i], 2);
    }
    // all consumer warps reach here; a CTA that gave up on a wait writes no results
    if (!consumers_any(aborted || *(volatile int*)&s_abort)) {
        // ---- merge the four warp states in shared memory (reusing the stage ring) ----
        float* om = reinterpret_cast<float*>(stages);  // [4][RB][D]
        float* mm = om + 4 * RB * D;                    // [4][RB]
        float* lm = mm + 4 * RB;                        // [4][RB]
#pragma unroll
        for (int j = 0; j < NT; ++j) {
            float* r0 = om + (warp * RB + g) * D;  // row g (r0 + D: row g + 8)
            if constexpr (F8) {  // columns 2 tq, 2 tq + 1 of n-tile j: head-dim values 16 vch(n) + j
                const int d0 = 16 * vch(2 * tq) + j, d1 = 16 * vch(2 * tq + 1) + j;
                r0[d0] = o[j][0];
                r0[d1] = o[j][1];
                r0[8 * D + d0] = o[j][2];
                r0[8 * D + d1] = o[j][3];
            } else {
                *reinterpret_cast<float2*>(r0 + 8 * j + 2 * tq) = make_float2(o[j][0], o[j][1]);
                *reinterpret_cast<float2*>(r0 + 8 * D + 8 * j + 2 * tq) = make_float2(o[j][2], o[j][3]);
            }
        }
        if (tq == 0) {
            mm[warp * RB + g] = m_run[0];
            mm[warp * RB + g + 8] = m_run[1];
            lm[warp * RB + g] = l_run[0];
            lm[warp * RB + g + 8] = l_run[1];
        }
        named_barrier(1, 128);
        gqa_merge_store<__nv_bfloat16, D, RB>(om, mm, lm, p, b, kvh, row0, rows_here, L, kbeg, split,
                                              F8 ? p.v_scale[kvh] : 1.f);
    }
}

// The swapped form for blocks of at most 8 query rows (the common GQA groups of 4 or 8 heads at s_q = 1): the
// warp's 16 tokens are the M = 16 rows of the MMAs and the query rows the N = 8 columns, so that a 16-token tile
// costs d/16 score MMAs (S^T = K Q^T, K read by ldmatrix as the A operand, Q^T held in registers) and d/16 P*V
// MMAs (O^T = V^T P^T, V^T the A operand: read by the transposing ldmatrix from a bf16 stage, paired and widened
// in registers from an e4m3 one) instead of twice that with 8 of 16 rows empty.  The score accumulator holds P^T
// (tokens x rows); movmatrix transposes its two 8 x 8 halves into the B operand of the P*V MMA.  Everything else
// (softmax, scales, the e4m3 key handling with its permuted head-dim order and token order, the merge) is as in
// the 16-row form above.
//
// Per-warp state of the 8-row form over one work item: the query slice as B fragments of the score MMA, the
// last visible key of the lane's two query rows, the O^T accumulators and the lazily moved maxima with this
// lane's shares of the row sums.
template <int D>
struct Mma8Warp {
    uint32_t qb[D / 16][2];  // query row g: bf16 pairs as given, or f16 pairs in the permuted e4m3 order
    int last[2];             // last visible key of query rows 2 tq, 2 tq + 1 (-1: a padding row, nothing visible)
    float o[D / 16][4];      // O^T rows g, g + 8 of m-tile mt (head-dim values 16 mt + g, + 8 for bf16; 16 vch(g)
                             // + 2 mt, + 1 for e4m3), query rows 2 tq, 2 tq + 1
    float m_run[2], l_run[2];
};

// Query row g of the block into the B fragments of lane (g, tq) (zeros when ok is false); qrow points at the
// row's D bf16 values.  The scale goes on the fp32 scores, so the values are taken as given.
template <int D, bool F8>
__device__ __forceinline__ void mma8_load_q(uint32_t (&qb)[D / 16][2], const uint32_t* qrow, bool ok, int tq) {
    auto qpair = [&](int u) -> uint32_t {
        const uint32_t w = ok ? qrow[u] : 0u;
        if constexpr (F8) {
            float lo, hi;
            bf16x2_to_f32(w, lo, hi);
            return pack_f16x2_rn(lo, hi);
        } else {
            return w;
        }
    };
#pragma unroll
    for (int ks = 0; ks < D / 16; ++ks) {
        // pairs of values: bf16 layout 16 ks + 2 tq (+ 8); e4m3 permuted layout 64 G + 16 tq + 4 j (+ 2)
        const int u0 = F8 ? 32 * (ks >> 2) + 8 * tq + 2 * (ks & 3) : 8 * ks + tq;
        qb[ks][0] = qpair(u0);
        qb[ks][1] = qpair(F8 ? u0 + 1 : u0 + 4);
    }
}

// A fresh online-softmax state and the row limits of lane (g, tq) for the block of rows row0 .. row0 + 7 of a
// group of R query rows (row gr of the group is query position gr mod s_q) over L cache tokens.
template <int D>
__device__ __forceinline__ void mma8_reset(Mma8Warp<D>& st, const GqaParams& p, int row0, int R, int L, int tq) {
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        const int gr = row0 + 2 * tq + i;
        st.last[i] = gr < R ? (p.causal ? L - p.s_q + gr % p.s_q : L - 1) : -1;
        st.m_run[i] = -INFINITY;
        st.l_run[i] = 0.f;
    }
#pragma unroll
    for (int j = 0; j < D / 16; ++j) st.o[j][0] = st.o[j][1] = st.o[j][2] = st.o[j][3] = 0.f;
}

// One tile of the 8-row form for consumer warp `warp`: the scores of its 16 tokens of the stage (keys at
// `stage`, values MAT_BYTES after them), the online softmax and O^T += V^T P^T.  tbase: the tile's first key;
// kend: the split's end; keys below mask_from are visible to every row.  The warp arrives on `empty` after its
// P*V MMAs, when it no longer reads the stage.
template <int D, bool F8>
__device__ __forceinline__ void mma8_tile(Mma8Warp<D>& st, uint8_t* stage, int tbase, int kend, int mask_from,
                                          float s_mul, const uint32_t (&k_off)[4], const uint32_t (&v_off)[4],
                                          const int (&tok_g)[2], uint32_t empty, int warp, int lane) {
    using C = GqaMmaCfg<D, F8, true>;
    constexpr int KS = D / 16, MT = D / 16;
    constexpr int V_SEG = C::T_TILE * 128;  // bytes per 64-value segment of a bf16 value tile
    const int g = lane >> 2, tq = lane & 3;
    const uint32_t kt = smem_u32(stage);
    const uint32_t vt = kt + C::MAT_BYTES;
    // ---- S^T = K Q^T for the warp's 16 tokens (two accumulators: even / odd k-steps) ----
    float sc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
    if constexpr (F8) {
#pragma unroll
        for (int G = 0; G < D / 64; ++G) {
            const int seg = G >> 1, chunk = 4 * (G & 1) + tq;
            uint4 w[2];
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int row = 16 * warp + tok_g[h];
                w[h] = *reinterpret_cast<const uint4*>(stage + seg * C::T_TILE * 128 + row * 128 +
                                                       ((chunk ^ (row & 7)) << 4));
            }
            const uint32_t w0[4] = {w[0].x, w[0].y, w[0].z, w[0].w}, w1[4] = {w[1].x, w[1].y, w[1].z, w[1].w};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const uint32_t a[4] = {e4m3x2_lo_to_f16x2(w0[j]), e4m3x2_lo_to_f16x2(w1[j]),
                                       e4m3x2_hi_to_f16x2(w0[j]), e4m3x2_hi_to_f16x2(w1[j])};
                mma_16816<true>(sc[j & 1], a, st.qb[4 * G + j][0], st.qb[4 * G + j][1]);
            }
        }
    } else {
#pragma unroll
        for (int ks = 0; ks < KS; ++ks) {
            uint32_t a[4];
            ldsm_x4(kt + (ks >> 2) * C::T_TILE * 128 + k_off[ks & 3], a);
            // ldmatrix order (tokens 0-7 lo, tokens 0-7 hi, tokens 8-15 lo, tokens 8-15 hi) -> a0 a2 a1 a3
            const uint32_t af[4] = {a[0], a[2], a[1], a[3]};
            mma_16816<false>(sc[ks & 1], af, st.qb[ks][0], st.qb[ks][1]);
        }
    }
    // x[e]: token tbase + 16 warp + tok_g[e / 2], query row 2 tq + e % 2, in the log2 domain
    float x[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) x[e] = (sc[0][e] + sc[1][e]) * s_mul;
    if (tbase + C::T_TILE > mask_from) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int tok = tbase + 16 * warp + tok_g[e >> 1];
            x[e] = (tok < kend && tok <= st.last[e & 1]) ? x[e] : -INFINITY;
        }
    }
    // ---- online softmax of the two rows (over the 8 lanes that share tq), lazily rescaled ----
    float mx[2];
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        mx[i] = fmaxf(x[i], x[2 + i]);
        mx[i] = fmaxf(mx[i], __shfl_xor_sync(0xffffffffu, mx[i], 4));
        mx[i] = fmaxf(mx[i], __shfl_xor_sync(0xffffffffu, mx[i], 8));
        mx[i] = fmaxf(mx[i], __shfl_xor_sync(0xffffffffu, mx[i], 16));
    }
    if (__any_sync(0xffffffffu, mx[0] > st.m_run[0] + 8.0f || mx[1] > st.m_run[1] + 8.0f)) {
        float alpha[2];
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            const float m_new = fmaxf(st.m_run[i], mx[i]);
            alpha[i] = 1.f;
            if (st.m_run[i] == -INFINITY) {
                st.m_run[i] = m_new;  // O and l of the row are still zero
            } else if (m_new > st.m_run[i] + 8.0f) {
                alpha[i] = fast_exp2(st.m_run[i] - m_new);
                st.m_run[i] = m_new;
            }
            st.l_run[i] *= alpha[i];
        }
#pragma unroll
        for (int j = 0; j < MT; ++j) {
            st.o[j][0] *= alpha[0];
            st.o[j][1] *= alpha[1];
            st.o[j][2] *= alpha[0];
            st.o[j][3] *= alpha[1];
        }
    }
    uint32_t pb[2];  // B fragment of the P*V MMA: query row g, tokens 2 tq, 2 tq + 1 (+ 8)
    {
        const float ms0 = st.m_run[0] == -INFINITY ? 0.f : st.m_run[0];  // no visible key yet: p = 2^-inf = 0
        const float ms1 = st.m_run[1] == -INFINITY ? 0.f : st.m_run[1];
        const float p0 = fast_exp2(x[0] - ms0), p1 = fast_exp2(x[1] - ms1);
        const float p2 = fast_exp2(x[2] - ms0), p3 = fast_exp2(x[3] - ms1);
        st.l_run[0] += p0 + p2;  // this lane's share; summed over the row's lanes at the end
        st.l_run[1] += p1 + p3;
        // P^T halves (tokens g / g + 8 x rows 2 tq, 2 tq + 1) transposed into P halves (row g x tokens)
        const uint32_t t0 = F8 ? pack_f16x2_rn(p0, p1) : pack_bf16x2(p0, p1);
        const uint32_t t1 = F8 ? pack_f16x2_rn(p2, p3) : pack_bf16x2(p2, p3);
        asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(pb[0]) : "r"(t0));
        asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(pb[1]) : "r"(t1));
    }
    const int nvalid = kend - (tbase + 16 * warp);  // value rows of the warp that are keys of the split
    if constexpr (F8) {
        // ---- O^T += V^T P^T straight from the e4m3 stage ----
        // Lane (g, tq) reads the 16 value bytes of head-dim chunk vch(g) of the warp's tokens tq, tq + 4, 8 + tq and
        // 12 + tq: the tokens of the MMA's k-indices 2 tq, 2 tq + 1, 2 tq + 8, 2 tq + 9 in the permuted token order.
        // A byte permute pairs the two tokens of a k-pair value by value and one conversion widens the pair, so
        // that A-fragment rows g and g + 8 of m-tile mt hold head-dim values 16 vch(g) + 2 mt and + 1.  vch puts
        // the chunks of lanes g = 2 i and 2 i + 1 in different halves of the swizzled row, so the 8 lanes of a
        // shared-memory phase read 8 different 16-byte columns.  Rows past the split's keys may hold anything
        // (even NaN), which P = 0 would not cancel in the MMA: they become 0.
        const int vch = ((g & 1) << 2) | (g >> 1);
        const uint8_t* vsrc = stage + C::MAT_BYTES;
        uint32_t vw[4][4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int t = tq + 4 * j;  // token of the warp's 16
            const int row = 16 * warp + t;
            uint4 w = *reinterpret_cast<const uint4*>(vsrc + row * 128 + ((vch ^ (row & 7)) << 4));
            if (t >= nvalid) w = make_uint4(0u, 0u, 0u, 0u);
            vw[j][0] = w.x;
            vw[j][1] = w.y;
            vw[j][2] = w.z;
            vw[j][3] = w.w;
        }
#pragma unroll
        for (int q = 0; q < 4; ++q) {  // value bytes 4 q .. 4 q + 3 of the chunk: m-tiles 2 q and 2 q + 1
            const uint32_t lo01 = __byte_perm(vw[0][q], vw[1][q], 0x5140), hi01 = __byte_perm(vw[0][q], vw[1][q], 0x7362);
            const uint32_t lo23 = __byte_perm(vw[2][q], vw[3][q], 0x5140), hi23 = __byte_perm(vw[2][q], vw[3][q], 0x7362);
            const uint32_t a0[4] = {e4m3x2_lo_to_f16x2(lo01), e4m3x2_hi_to_f16x2(lo01), e4m3x2_lo_to_f16x2(lo23),
                                    e4m3x2_hi_to_f16x2(lo23)};
            mma_16816<true>(st.o[2 * q], a0, pb[0], pb[1]);
            const uint32_t a1[4] = {e4m3x2_lo_to_f16x2(hi01), e4m3x2_hi_to_f16x2(hi01), e4m3x2_lo_to_f16x2(hi23),
                                    e4m3x2_hi_to_f16x2(hi23)};
            mma_16816<true>(st.o[2 * q + 1], a1, pb[0], pb[1]);
        }
    } else {
        if (nvalid < 16) {
            // value rows of the warp past the split's keys (the last tile) may hold anything, even NaN, and
            // P = 0 does not cancel that in the MMA: zero them
            const int first = nvalid < 0 ? 0 : nvalid;
            uint8_t* vrow = stage + C::MAT_BYTES;
            for (int idx = lane; idx < (16 - first) * C::NSEG * 8; idx += 32) {
                const int row = 16 * warp + first + idx / (C::NSEG * 8), rem = idx % (C::NSEG * 8);
                *reinterpret_cast<uint4*>(vrow + (rem / 8) * C::T_TILE * 128 + row * 128 + (rem % 8) * 16) =
                    make_uint4(0u, 0u, 0u, 0u);
            }
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // before the ring's next copy
            __syncwarp();
        }
        // ---- O^T += V^T P^T: one MMA per 16 head-dim values ----
#pragma unroll
        for (int mt = 0; mt < MT; ++mt) {
            uint32_t a[4];
            ldsm_x4_t(vt + (mt >> 2) * V_SEG + v_off[mt & 3], a);
            // ldmatrix order (tokens 0-7 x d lo, tokens 0-7 x d hi, tokens 8-15 x d lo, tokens 8-15 x d hi),
            // transposed: (d lo, k lo) (d hi, k lo) (d lo, k hi) (d hi, k hi) = a0 a1 a2 a3
            mma_16816<false>(st.o[mt], a, pb[0], pb[1]);
        }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(empty);
}

// Sums this lane's row-sum shares over the row's eight lanes and writes the warp's state for the merge:
// om [4][8][D] (the O^T fragments back in row-major order), mm / lm [4][8].
template <int D, bool F8>
__device__ __forceinline__ void mma8_stash(Mma8Warp<D>& st, float* om, float* mm, float* lm, int warp, int lane) {
    constexpr int RB = 8;
    const int g = lane >> 2, tq = lane & 3;
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        st.l_run[i] += __shfl_xor_sync(0xffffffffu, st.l_run[i], 4);
        st.l_run[i] += __shfl_xor_sync(0xffffffffu, st.l_run[i], 8);
        st.l_run[i] += __shfl_xor_sync(0xffffffffu, st.l_run[i], 16);
    }
    float* o0 = om + (warp * RB + 2 * tq) * D;  // query row 2 tq (o1: 2 tq + 1)
    float* o1 = o0 + D;
#pragma unroll
    for (int mt = 0; mt < D / 16; ++mt) {
        if constexpr (F8) {  // rows g, g + 8 of m-tile mt: head-dim values d, d + 1 for d = 16 vch(g) + 2 mt
            const int d = 16 * (((g & 1) << 2) | (g >> 1)) + 2 * mt;
            *reinterpret_cast<float2*>(o0 + d) = make_float2(st.o[mt][0], st.o[mt][2]);
            *reinterpret_cast<float2*>(o1 + d) = make_float2(st.o[mt][1], st.o[mt][3]);
        } else {  // rows g, g + 8 of m-tile mt: head-dim values 16 mt + g, + 8
            o0[16 * mt + g] = st.o[mt][0];
            o1[16 * mt + g] = st.o[mt][1];
            o0[16 * mt + g + 8] = st.o[mt][2];
            o1[16 * mt + g + 8] = st.o[mt][3];
        }
    }
    if (g == 0) {
        mm[warp * RB + 2 * tq] = st.m_run[0];
        mm[warp * RB + 2 * tq + 1] = st.m_run[1];
        lm[warp * RB + 2 * tq] = st.l_run[0];
        lm[warp * RB + 2 * tq + 1] = st.l_run[1];
    }
}

// ldmatrix row addresses of lane `lane` in warp `warp` for a bf16 stage (byte offsets, 128-byte swizzle), and
// the token of the warp's 16 held by MMA row g + 8 h.  Both operands are A fragments read from token rows: matrix
// l / 8 = (token half l / 16, 8-value chunk parity (l / 8) % 2).  Keys: non-transposed, one k-step; values
// (transposed): one 16-value m-tile of O^T.
template <bool F8>
__device__ __forceinline__ void mma8_offsets(uint32_t (&k_off)[4], uint32_t (&v_off)[4], int (&tok_g)[2], int warp,
                                             int lane) {
    const int g = lane >> 2, r8 = lane & 7;
    const uint32_t k_row = (uint32_t)(16 * warp + 8 * (lane >> 4) + r8) * 128;
    const uint32_t v_row = k_row;
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        k_off[c] = k_row + ((uint32_t)((2 * c + ((lane >> 3) & 1)) ^ r8) << 4);
        v_off[c] = v_row + ((uint32_t)((2 * c + ((lane >> 3) & 1)) ^ r8) << 4);
    }
    tok_g[0] = F8 ? f8_tok(g) : g;
    tok_g[1] = 8 + tok_g[0];
}

template <int D, bool F8>
__global__ void __launch_bounds__(160, GqaMmaCfg<D, F8, true>::MINB)
    gqa_decode_mma8_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                           const GqaParams p) {
    using C = GqaMmaCfg<D, F8, true>;
    constexpr int RB = 8;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(align_up(reinterpret_cast<uintptr_t>(smem_raw), 1024));
    uint8_t* stages = smem;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
    __shared__ int s_abort;

    const int split = blockIdx.x;
    const int kvh = blockIdx.y / p.n_rb;
    const int rb = blockIdx.y % p.n_rb;
    const int b = blockIdx.z;
    const int R = p.ratio * p.s_q;  // query rows of this group
    const int row0 = rb * RB;
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;

    const int L = clamp_len(p.lens, b, p.Lmax, p.s_q, p.causal, p.status,
                            threadIdx.x == 0 && split == 0 && kvh == 0 && rb == 0);
    const int rows_here = R - row0 < RB ? R - row0 : RB;
    int need = L;  // keys needed by the rows of this block: causal row t sees L - s_q + t + 1
    if (p.causal) {
        int tmax = 0;
        for (int r = 0; r < rows_here; ++r) tmax = max(tmax, (row0 + r) % p.s_q);
        need = L - p.s_q + tmax + 1;
    }
    const int kbeg = split * p.split_tokens;
    if (kbeg >= need) return;  // no row of this block has keys in this split
    const int kend = min(need, kbeg + p.split_tokens);
    const int n_tiles = cdiv(kend - kbeg, C::T_TILE);

    if (threadIdx.x == 0) {
        s_abort = 0;
        for (int s = 0; s < C::NSTAGE; ++s) {
            mbar_init(smem_u32(&bars[s]), 1);              // full: producer arrival + tx bytes
            mbar_init(smem_u32(&bars[C::NSTAGE + s]), 4);  // empty: one arrival per consumer warp
        }
        fence_barrier_init();
    }
    __syncthreads();

    if (warp == 4) {
        if (lane == 0) gqa_produce<C>(&tmK, &tmV, p, stages, bars, &s_abort, b, kvh, L, kbeg, n_tiles);
        return;
    }

    // -------------------------------- consumers --------------------------------
    // Fragment coordinates: lane = 4 g + tq.  Score accumulator: tokens (MMA rows) g and g + 8 of the warp's 16,
    // query rows (MMA columns) 2 tq and 2 tq + 1.  B operand of the score MMA: query row g.
    const int g = lane >> 2, tq = lane & 3;
    Mma8Warp<D> st;
    mma8_reset<D>(st, p, row0, R, L, tq);
    {
        const __nv_bfloat16* qbase = reinterpret_cast<const __nv_bfloat16*>(p.q) +
                                     ((size_t)(b * p.h_q + kvh * p.ratio) * p.s_q) * D;  // first row of the group
        const bool ok = row0 + g < R;
        mma8_load_q<D, F8>(st.qb, reinterpret_cast<const uint32_t*>(qbase + (size_t)(ok ? row0 + g : 0) * D), ok,
                           tq);
    }
    const float s_mul = F8 ? p.scale_log2 * p.k_scale[kvh] : p.scale_log2;
    int mask_from = kend;  // keys below mask_from are visible to every row of the block
    for (int r = 0; r < rows_here; ++r)
        mask_from = min(mask_from, p.causal ? L - p.s_q + (row0 + r) % p.s_q + 1 : L);
    uint32_t k_off[4], v_off[4];
    int tok_g[2];
    mma8_offsets<F8>(k_off, v_off, tok_g, warp, lane);

    bool aborted = false;
    for (int it = 0; it < n_tiles; ++it) {
        const int s = it % C::NSTAGE;
        if (!mbar_wait(smem_u32(&bars[s]), (it / C::NSTAGE) & 1, p.status)) {
            aborted = true;
            s_abort = 1;
            break;
        }
        mma8_tile<D, F8>(st, stages + s * C::STAGE_BYTES, kbeg + it * C::T_TILE, kend, mask_from, s_mul, k_off,
                         v_off, tok_g, smem_u32(&bars[C::NSTAGE + s]), warp, lane);
    }

    // all consumer warps reach here; a CTA that gave up on a wait writes no results
    if (!consumers_any(aborted || *(volatile int*)&s_abort)) {
        // ---- merge the four warp states in shared memory (reusing the stage ring) ----
        float* om = reinterpret_cast<float*>(stages);  // [4][RB][D]
        float* mm = om + 4 * RB * D;                    // [4][RB]
        float* lm = mm + 4 * RB;                        // [4][RB]
        mma8_stash<D, F8>(st, om, mm, lm, warp, lane);
        named_barrier(1, 128);
        gqa_merge_store<__nv_bfloat16, D, RB>(om, mm, lm, p, b, kvh, row0, rows_here, L, kbeg, split,
                                              F8 ? p.v_scale[kvh] : 1.f);
    }
}


// Merge of split partials: with w_i = 2^(lse_i - max lse),
// O = sum_i w_i O_i / sum_i w_i and lse = max lse + log2(sum_i w_i).
// One warp per output row; rows that needed a single split were written
// directly by the decode kernel and are skipped.
template <typename T, int D>
__global__ void __launch_bounds__(128) gqa_combine_kernel(const GqaParams p) {
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const size_t row = (size_t)blockIdx.x * 4 + warp;
    const size_t nrows = (size_t)p.B * p.h_q * p.s_q;
    if (row >= nrows) return;
    const int t = (int)(row % p.s_q);
    const int b = (int)(row / ((size_t)p.h_q * p.s_q));
    const int L = clamp_len(p.lens, b, p.Lmax, p.s_q, p.causal, p.status, false);
    const int n_t = p.causal ? (L - p.s_q + t + 1) : L;
    const int nsp = cdiv(n_t, p.split_tokens);
    if (nsp == 1) return;
    const float* pl = p.part_lse + row * p.nsplit_max;
    float M = -INFINITY;
    for (int i = lane; i < nsp; i += 32) M = fmaxf(M, pl[i]);
#pragma unroll
    for (int m = 16; m >= 1; m /= 2) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, m));
    constexpr int DPL = D / 32;
    float acc[DPL];
#pragma unroll
    for (int d = 0; d < DPL; ++d) acc[d] = 0.f;
    float wsum = 0.f;
    const float* po = p.part_o + row * p.nsplit_max * D;
    // lane i holds the weight of split i (of each group of 32); 8 splits' values are loaded together
    for (int i32 = 0; i32 < nsp; i32 += 32) {
        const float w_lane = i32 + lane < nsp ? exp2f(pl[i32 + lane] - M) : 0.f;
        const int n = min(32, nsp - i32);
        for (int u0 = 0; u0 < n; u0 += 8) {
            float v[8][DPL];
#pragma unroll
            for (int u = 0; u < 8; ++u)
#pragma unroll
                for (int d = 0; d < DPL; ++d)
                    v[u][d] = u0 + u < n ? po[(size_t)(i32 + u0 + u) * D + d * 32 + lane] : 0.f;
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const float ws = __shfl_sync(0xffffffffu, w_lane, (u0 + u) & 31);
                const float w = u0 + u < n ? ws : 0.f;
                wsum += w;
#pragma unroll
                for (int d = 0; d < DPL; ++d) acc[d] = fmaf(w, v[u][d], acc[d]);
            }
        }
    }
    T* out = reinterpret_cast<T*>(p.out) + row * D;
#pragma unroll
    for (int d = 0; d < DPL; ++d) out[d * 32 + lane] = from_f32<T>(acc[d] / wsum);
    if (p.lse && lane == 0) p.lse[row] = (M + log2f(wsum)) * 0.69314718055994530942f;
}

// ---- host-side dispatch -------------------------------------------------------
template <typename T, int D, int RB, typename KV = T>
static cudaError_t launch_one(const CUtensorMap& tk, const CUtensorMap& tv, const GqaParams& p, int nsplit,
                              cudaStream_t st) {
    using C = GqaCfg<KV, D, RB>;
    auto kern = gqa_decode_kernel<T, D, RB, KV>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    if (e != cudaSuccess) return e;
    dim3 grid(nsplit, p.h_kv * p.n_rb, p.B);
    TimedLaunch timer(st);
    kern<<<grid, 160, C::SMEM, st>>>(tk, tv, p);
    timer.stop();
    e = cudaPeekAtLastError();
    if (e != cudaSuccess) return e;
    const size_t nrows = (size_t)p.B * p.h_q * p.s_q;
    if (nsplit > 1) {
        gqa_combine_kernel<T, D><<<(unsigned)((nrows + 3) / 4), 128, 0, st>>>(p);
        e = cudaPeekAtLastError();
    }
    return e;
}

template <int D, bool F8>
static cudaError_t launch_mma(const CUtensorMap& tk, const CUtensorMap& tv, const GqaParams& p, int nsplit,
                              cudaStream_t st) {
    using C = GqaMmaCfg<D, F8>;
    const bool rows8 = p.n_rb == 1 && p.ratio * p.s_q <= 8;
    auto kern = rows8 ? gqa_decode_mma8_kernel<D, F8> : gqa_decode_mma_kernel<D, F8>;
    const int smem = rows8 ? GqaMmaCfg<D, F8, true>::SMEM : C::SMEM;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    dim3 grid(nsplit, p.h_kv * p.n_rb, p.B);
    TimedLaunch timer(st);
    kern<<<grid, 160, smem, st>>>(tk, tv, p);
    timer.stop();
    e = cudaPeekAtLastError();
    if (e != cudaSuccess) return e;
    const size_t nrows = (size_t)p.B * p.h_q * p.s_q;
    if (nsplit > 1) {
        gqa_combine_kernel<__nv_bfloat16, D><<<(unsigned)((nrows + 3) / 4), 128, 0, st>>>(p);
        e = cudaPeekAtLastError();
    }
    return e;
}

cudaError_t gqa_combine_launch(const GqaParams& p, int dtype_bytes, int d, cudaStream_t st) {
    const size_t nrows = (size_t)p.B * p.h_q * p.s_q;
    const unsigned grid = (unsigned)((nrows + 3) / 4);
    if (dtype_bytes == 2 && d == 128) gqa_combine_kernel<__nv_bfloat16, 128><<<grid, 128, 0, st>>>(p);
    else if (dtype_bytes == 2 && d == 64) gqa_combine_kernel<__nv_bfloat16, 64><<<grid, 128, 0, st>>>(p);
    else if (dtype_bytes == 2 && d == 256) gqa_combine_kernel<__nv_bfloat16, 256><<<grid, 128, 0, st>>>(p);
    else if (dtype_bytes == 4 && d == 128) gqa_combine_kernel<float, 128><<<grid, 128, 0, st>>>(p);
    else if (dtype_bytes == 4 && d == 64) gqa_combine_kernel<float, 64><<<grid, 128, 0, st>>>(p);
    else return cudaErrorInvalidValue;
    return cudaPeekAtLastError();
}

int gqa_tile_tokens(int dtype_bytes, int d, int rb, int* ctas_per_sm) {
#define LKA_TILE_CASE(T, DD, R)                                  \
    if (dtype_bytes == (int)sizeof(T) && d == DD && rb == R) {   \
        if (ctas_per_sm) *ctas_per_sm = GqaCfg<T, DD, R>::MINB; \
        return GqaCfg<T, DD, R>::T_TILE;                         \
    }
    if (dtype_bytes == 2 && (d == 64 || d == 128) && rb == 16) {  // the tensor-core instance
        if (ctas_per_sm) *ctas_per_sm = d == 64 ? GqaMmaCfg<64, false>::MINB : GqaMmaCfg<128, false>::MINB;
        return d == 64 ? GqaMmaCfg<64, false>::T_TILE : GqaMmaCfg<128, false>::T_TILE;
    }
    LKA_TILE_CASE(__nv_bfloat16, 256, 1) LKA_TILE_CASE(__nv_bfloat16, 256, 2) LKA_TILE_CASE(__nv_bfloat16, 256, 4)
    LKA_TILE_CASE(__nv_bfloat16, 256, 8)
    LKA_TILE_CASE(float, 64, 1) LKA_TILE_CASE(float, 64, 2) LKA_TILE_CASE(float, 64, 4) LKA_TILE_CASE(float, 64, 8)
    LKA_TILE_CASE(float, 64, 16)
    LKA_TILE_CASE(float, 128, 1) LKA_TILE_CASE(float, 128, 2) LKA_TILE_CASE(float, 128, 4)
    LKA_TILE_CASE(float, 128, 8) LKA_TILE_CASE(float, 128, 16)
#undef LKA_TILE_CASE
    return 0;
}

cudaError_t gqa_decode_launch(const CUtensorMap& tk, const CUtensorMap& tv, const GqaParams& p, int dtype_bytes,
                              int d, int rb, int nsplit, cudaStream_t st) {
#define LKA_LAUNCH_CASE(T, DD, R) \
    if (dtype_bytes == (int)sizeof(T) && d == DD && rb == R) return launch_one<T, DD, R>(tk, tv, p, nsplit, st);
    if (dtype_bytes == 2 && d == 64 && rb == 16) return launch_mma<64, false>(tk, tv, p, nsplit, st);
    if (dtype_bytes == 2 && d == 128 && rb == 16) return launch_mma<128, false>(tk, tv, p, nsplit, st);
    LKA_LAUNCH_CASE(__nv_bfloat16, 256, 1) LKA_LAUNCH_CASE(__nv_bfloat16, 256, 2)
    LKA_LAUNCH_CASE(__nv_bfloat16, 256, 4) LKA_LAUNCH_CASE(__nv_bfloat16, 256, 8)
    LKA_LAUNCH_CASE(float, 64, 1) LKA_LAUNCH_CASE(float, 64, 2) LKA_LAUNCH_CASE(float, 64, 4)
    LKA_LAUNCH_CASE(float, 64, 8) LKA_LAUNCH_CASE(float, 64, 16)
    LKA_LAUNCH_CASE(float, 128, 1) LKA_LAUNCH_CASE(float, 128, 2) LKA_LAUNCH_CASE(float, 128, 4)
    LKA_LAUNCH_CASE(float, 128, 8) LKA_LAUNCH_CASE(float, 128, 16)
#undef LKA_LAUNCH_CASE
    return cudaErrorInvalidValue;
}

int gqa_fp8_tile_tokens(int d, int rb, int* ctas_per_sm) {
    if (d == 128 && rb == 16) {  // the tensor-core instance
        // (the plan assumes the 8-row form of the usual GQA groups: three CTAs per SM)
        if (ctas_per_sm) *ctas_per_sm = GqaMmaCfg<128, true, true>::MINB;
        return GqaMmaCfg<128, true, true>::T_TILE;
    }
#define LKA_TILE_CASE(DD, R)                                       \
    if (d == DD && rb == R) {                                      \
        if (ctas_per_sm) *ctas_per_sm = GqaCfg<e4m3, DD, R>::MINB; \
        return GqaCfg<e4m3, DD, R>::T_TILE;                        \
    }
    LKA_TILE_CASE(256, 1) LKA_TILE_CASE(256, 2) LKA_TILE_CASE(256, 4)
#undef LKA_TILE_CASE
    return 0;
}

cudaError_t gqa_fp8_decode_launch(const CUtensorMap& tk, const CUtensorMap& tv, const GqaParams& p, int d, int rb,
                                  int nsplit, cudaStream_t st) {
    if (d == 128 && rb == 16) return launch_mma<128, true>(tk, tv, p, nsplit, st);
#define LKA_LAUNCH_CASE(DD, R) \
    if (d == DD && rb == R) return launch_one<__nv_bfloat16, DD, R, e4m3>(tk, tv, p, nsplit, st);
    LKA_LAUNCH_CASE(256, 1) LKA_LAUNCH_CASE(256, 2) LKA_LAUNCH_CASE(256, 4)
#undef LKA_LAUNCH_CASE
    return cudaErrorInvalidValue;
}

}  // namespace lka
