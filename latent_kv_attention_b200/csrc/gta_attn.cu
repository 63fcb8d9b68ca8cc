// gta_attn.cu -- GTA-style grouped shared-score attention on the 5th-generation
// tensor cores.
//
// Operation ("GTA: Grouped-head latenT Attention" press article, section on
// the grouped shared attention matrix): the heads are split into groups (for
// example 4 heads per group) and the members of a group share one attention
// matrix: the scores are computed once per group and then used by every head
// of the group with that head's own values:
//     P_gamma = softmax(scale * Q_gamma K_gamma^T)  (causal: bottom-right mask)
//     O_h     = P_gamma V_h        for every head h of group gamma.
// Prefill is dense in both contractions, so both run as tcgen05 MMAs.
//
// One CTA = (128-query tile, group, sequence); q-tiles are scheduled longest
// first.  Warp 8 streams 128-key tiles of K_gamma and the V tiles of the
// group's heads with TMA (2 stages of 80 KB); warp 9 issues S = Q K^T
// (M = N = 128, K = 64) into tensor memory and, once the softmax has written P
// back to tensor memory as bf16, P*V for all heads of the group at once
// (M = 128, N = 64 x heads, K = 128; A = P from tensor memory; the heads' value
// tiles sit one box apart, which is the stride between the 64-column blocks of
// the B operand) -- the score tile is computed and normalised once and reused
// by all heads of the group.  A tcgen05.mma costs about the same for any N up
// to 256, so one wide MMA replaces one per head.  Warps 0-7 run the mask and
// the online softmax, two warps per group of 32 query rows (warps w and w + 4
// take the two 64-key halves of the tile and combine their row maxima through
// shared memory), with lazy rescaling (the running maximum only moves when it
// grows by more than 2^8); P goes to tensor memory.
//
// The same pipeline runs the causal prefill of grouped-query attention
// ("Grouped Query Attention (GQA)" glossary page, "How GQA works"): every query
// head is then a group of its own, its keys and values are those of its KV head
// floor(h / (h_q / h_kv)), and the head dimension d = 128 is two 64-column
// boxes of the query and key tiles and two 64-column blocks of the value tile
// (the N = 128 of P*V).  The prefill of the GQLA per-group GQA path (GQLA
// section 1: prefill expands the latent, MHA-like) is the same with a query
// and key of 192 values: two boxes of q^C / the group's key kc and a third box
// of q^R / the RoPE key k^R, which all groups share.
#include "common.cuh"
#include "host_util.h"
#include "tc.cuh"

namespace lka {

struct GtaParams {
    const int32_t* lens;
    __nv_bfloat16* out;  // [B, H, s_q, 64]
    float* lse;          // [B, G, s_q] or nullptr
    uint32_t* status;
    int B, G, H, s_q, Lmax, causal;
    float scale_log2;
    // paged caches (block_table == nullptr: contiguous [B][heads][Lmax] slabs)
    const int32_t* block_table;  // [B, max_pages]
    int page_size, max_pages, num_pages;
    int box_rows;                // rows per TMA box: min(128, page_size), or 128 when contiguous
    // key splits (nsplit > 1): split k covers keys [k * split_tokens, (k + 1) * split_tokens); a row whose keys
    // need more than one split writes normalised fp32 partials that gta_combine_kernel merges
    int split_tokens, nsplit;
    float* part_o;    // [B * H * s_q][nsplit][64]  (GQA: [B * h_q * s_q][nsplit][d])
    float* part_lse;  // [B * G * s_q][nsplit] log2 domain (one per group: the score matrix is the group's)
    // GQA mode: G = H = h_q query heads, h_kv KV heads; head h reads KV head h / kv_ratio
    int h_kv, kv_ratio;
};

namespace gta {
constexpr int TQ = 128, TK = 128;
constexpr int NSV = 2;              // V ring depth: value tiles live until their P*V MMAs complete
constexpr int BOX = TK * 128;       // 128 rows x 64 bf16
constexpr int NSW = 8;              // softmax warps: 4 lane quarters x 2 key halves
constexpr int CW = TK / 2;          // score columns per softmax warp
constexpr int NTHREADS = 32 * (NSW + 2);
constexpr int K_LEAD = 2;           // key tiles the producer keeps ahead of the value tiles
constexpr uint32_t T_O = 0;         // up to 4 x 64 fp32 columns (GTA: one block per head; GQA: the head's d)
constexpr uint32_t T_S = 256;       // 128 fp32 columns
constexpr uint32_t T_P = 384;       // 2 x 64 columns of bf16 pairs (double-buffered P)
// Shared-memory layout of an instance with NQB 64-column boxes of query / key (d_qk = 64 NQB) and NVB
// 64-column value blocks per tile (GTA: the group's heads; GQA: the head's d_v = 64 NVB).
template <int NQB, int NVB>
struct Cfg {
    // K ring depth: key tiles are released right after S = Q K^T
    static constexpr int NSK = NQB == 1 ? 4 : (NQB == 2 ? 3 : 2);
    static constexpr int VSTAGE = NVB * BOX;
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_K = NQB * BOX;
    static constexpr int OFF_V = OFF_K + NSK * NQB * BOX;
    static constexpr int OFF_RED = OFF_V + NSV * VSTAGE;  // float [2][NSW][32] row maxima + [NSW][32] row sums
    static constexpr int OFF_BAR = OFF_RED + 3 * NSW * 32 * 4;
    static constexpr int SMEM = 1024 + OFF_BAR + 256;
    static_assert(SMEM <= 232448, "shared memory budget");
    static_assert(NVB * 64 <= (int)T_S, "output columns");
};
}  // namespace gta

// GQA = false: GTA, value blocks = the group's heads (NVB = 4 slots, H / G of them used);
// GQA = true: one query head per group, K / V of its KV head, value blocks = the NVB column blocks of d.
// NQB = 3 (GQA): the third query box comes from tm_q2 (q^R rows) and the third key box from tm_k2 (the RoPE
// key, one row per token shared by all heads).
template <int NQB, int NVB, bool GQA>
__global__ void __launch_bounds__(gta::NTHREADS, 1)
    gta_attn_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_q2,
                    const __grid_constant__ CUtensorMap tm_k2, const GtaParams p) {
    using namespace gta;
    using CF = Cfg<NQB, NVB>;
    constexpr int NSK = CF::NSK, VSTAGE = CF::VSTAGE, OFF_Q = CF::OFF_Q, OFF_K = CF::OFF_K, OFF_V = CF::OFF_V;
    constexpr int OFF_RED = CF::OFF_RED, OFF_BAR = CF::OFF_BAR;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(align_up(reinterpret_cast<uintptr_t>(smem_raw), 1024));
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + OFF_BAR);
    uint64_t* q_full = bars;
    uint64_t* k_full = bars + 1;
    uint64_t* k_empty = k_full + NSK;
    uint64_t* v_full = k_empty + NSK;
    uint64_t* v_empty = v_full + NSV;
    uint64_t* s_ready = v_empty + NSV;
    uint64_t* s_free = s_ready + 1;
    uint64_t* p_ready = s_free + 1;   // [2] P(j) in buffer j&1 written
    uint64_t* o_ready = p_ready + 2;  // [2] PV(j) done
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(o_ready + 2);
    __shared__ int s_abort;

    const int n_qt = cdiv(p.s_q, TQ);
    const int qt = n_qt - 1 - (int)blockIdx.x / p.nsplit;  // longest tiles first
    const int split = (int)blockIdx.x % p.nsplit;
    const int grp = blockIdx.y, b = blockIdx.z;
    const int HPG = p.H / p.G;
    const int nvb = GQA ? NVB : HPG;                     // value blocks of a tile (64 columns each)
    const int kv_head = GQA ? grp / p.kv_ratio : grp;    // the head whose keys (and GQA: values) are read
    const int k_heads = GQA ? p.h_kv : p.G;              // heads of the key (GQA: and value) cache
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int L = clamp_len(p.lens, b, p.Lmax, p.s_q, p.causal, p.status,
                            threadIdx.x == 0 && blockIdx.x == 0 && grp == 0);
    const int q0 = qt * TQ;
    const int q_last = min(q0 + TQ, p.s_q) - 1;
    const int key_all = p.causal ? (L - p.s_q + q_last + 1) : L;  // keys any row of the tile may see
    const int kbeg = split * p.split_tokens;
    const int key_end = min(key_all, kbeg + p.split_tokens);      // this split's share of them
    if (key_end <= kbeg) return;                                   // no key of this split is visible
    const int n_tiles = cdiv(key_end - kbeg, TK);

    if (threadIdx.x == 0) {
        s_abort = 0;
        mbar_init(smem_u32(q_full), 1);
        for (int s = 0; s < NSK; ++s) {
            mbar_init(smem_u32(&k_full[s]), 1);
            mbar_init(smem_u32(&k_empty[s]), 1);
        }
        for (int s = 0; s < NSV; ++s) {
            mbar_init(smem_u32(&v_full[s]), 1);
            mbar_init(smem_u32(&v_empty[s]), 1);
        }
        mbar_init(smem_u32(s_ready), 1);
        mbar_init(smem_u32(s_free), NSW);
        for (int i = 0; i < 2; ++i) {
            mbar_init(smem_u32(&p_ready[i]), NSW);
            mbar_init(smem_u32(&o_ready[i]), 1);
        }
        fence_barrier_init();
    }
    if (warp == NSW + 1) {
        tmem_alloc(tmem_slot, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == NSW) {
        // ------------------------------ producer ------------------------------
        // issue order K(0..K_LEAD-1), then per tile i: K(i + K_LEAD), V(i)
        if (lane == 0) {
            const uint32_t qb = smem_u32(q_full);
            mbar_arrive_expect_tx(qb, NQB * BOX);
#pragma unroll
            for (int kb = 0; kb < NQB; ++kb) {
                if (kb < 2)
                    tma_load_2d(smem_u32(smem + OFF_Q + kb * BOX), &tm_q, kb * 64, (b * p.G + grp) * p.s_q + q0, qb);
                else
                    tma_load_2d(smem_u32(smem + OFF_Q + kb * BOX), &tm_q2, 0, (b * p.G + grp) * p.s_q + q0, qb);
            }
            int k_issued = 0, v_issued = 0;
            bool ok = true;
            // row of token `tok` of head `head` (of `heads`) of this sequence: contiguous [B][heads][Lmax], or
            // row tok % page_size of that head's block in page block_table[b][tok / page_size]; an entry outside
            // the pool is replaced by page 0, which is reported when the tile's queries need the token
            auto cache_row = [&](int tok, int heads, int head) -> int {
                if (!p.block_table) return (b * heads + head) * p.Lmax + tok;
                int page = 0;
                const int jp = tok / p.page_size;
                if (jp < p.max_pages) {
                    page = p.block_table[(size_t)b * p.max_pages + jp];
                    if (page < 0 || page >= p.num_pages) {
                        if (tok < key_end) atomicOr(p.status, kDevBadPage);
                        page = 0;
                    }
                }
                return (page * heads + head) * p.page_size + tok % p.page_size;
            };
            auto issue_k = [&](int i) {
                const int s = i % NSK;
                if (i >= NSK && !mbar_wait(smem_u32(&k_empty[s]), ((i / NSK) - 1) & 1, p.status)) return false;
                const uint32_t fb = smem_u32(&k_full[s]);
                mbar_arrive_expect_tx(fb, NQB * BOX);
                for (int r0 = 0; r0 < TK; r0 += p.box_rows) {  // one box, or one per page piece of the tile
                    const int tok = kbeg + i * TK + r0;
                    const int y = cache_row(tok, k_heads, kv_head);
#pragma unroll
                    for (int kb = 0; kb < NQB; ++kb) {
                        const uint32_t dst = smem_u32(smem + OFF_K + (s * NQB + kb) * BOX) + r0 * 128;
                        if (kb < 2)
                            tma_load_2d(dst, &tm_k, kb * 64, y, fb);
                        else  // the shared RoPE key: one row per token ([B, Lmax] or [num_pages, page_size])
                            tma_load_2d(dst, &tm_k2, 0, cache_row(tok, 1, 0), fb);
                    }
                }
                ++k_issued;
                return true;
            };
            auto issue_v = [&](int i) {
                const int s = i % NSV;
                if (i >= NSV && !mbar_wait(smem_u32(&v_empty[s]), ((i / NSV) - 1) & 1, p.status)) return false;
                const uint32_t fb = smem_u32(&v_full[s]);
                mbar_arrive_expect_tx(fb, nvb * BOX);
                const uint32_t d = smem_u32(smem + OFF_V + s * VSTAGE);
                for (int hh = 0; hh < nvb; ++hh)
                    for (int r0 = 0; r0 < TK; r0 += p.box_rows) {
                        if (GQA)  // column block hh of the KV head's value rows
                            tma_load_2d(d + hh * BOX + r0 * 128, &tm_v, hh * 64,
                                        cache_row(kbeg + i * TK + r0, k_heads, kv_head), fb);
                        else      // the value tile of the group's head hh
                            tma_load_2d(d + hh * BOX + r0 * 128, &tm_v, 0,
                                        cache_row(kbeg + i * TK + r0, p.H, grp * HPG + hh), fb);
                    }
                ++v_issued;
                return true;
            };
            for (int i = 0; ok && i < K_LEAD && i < n_tiles; ++i) ok = issue_k(i);
            for (int i = 0; ok && i < n_tiles; ++i) {
                if (*(volatile int*)&s_abort) break;
                if (i + K_LEAD < n_tiles) ok = issue_k(i + K_LEAD);
                if (ok) ok = issue_v(i);
            }
            if (!ok) s_abort = 1;
            // drain: every issued copy must land before the CTA may exit
            for (int i = k_issued - 1; i >= 0 && i >= k_issued - NSK; --i)
                mbar_wait(smem_u32(&k_full[i % NSK]), (i / NSK) & 1, p.status);
            for (int i = v_issued - 1; i >= 0 && i >= v_issued - NSV; --i)
                mbar_wait(smem_u32(&v_full[i % NSV]), (i / NSV) & 1, p.status);
            mbar_wait(qb, 0, p.status);
        }
    } else if (warp == NSW + 1) {
        // ------------------------------ MMA issuer ------------------------------
        constexpr uint32_t idesc_qk = idesc_bf16_f32(128, 128, false, false);
        const uint32_t idesc_pv = idesc_bf16_f32(128, 64 * nvb, false, true);
        bool ok = mbar_wait(smem_u32(q_full), 0, p.status);
        // zero the rows of a tile past the cache length (they may hold anything, even NaN)
        auto zero_tail = [&](uint8_t* base, int nbox, int j) {
            const int nvalid = min(TK, L - (kbeg + j * TK));
            if (nvalid >= TK) return;
            const int rows = TK - nvalid;
            for (int idx = lane; idx < nbox * rows * 8; idx += 32) {
                const int bx = idx / (rows * 8), rr = (idx / 8) % rows, c = idx % 8;
                *reinterpret_cast<uint4*>(base + bx * BOX + (nvalid + rr) * 128 + c * 16) = make_uint4(0, 0, 0, 0);
            }
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            __syncwarp();
        };
        auto issue_qk = [&](int j) -> bool {
            const int s = j % NSK;
            if (!mbar_wait(smem_u32(&k_full[s]), (j / NSK) & 1, p.status)) return false;
            uint8_t* kt = smem + OFF_K + s * NQB * BOX;
            zero_tail(kt, NQB, j);
            if (j >= 1 && !mbar_wait(smem_u32(s_free), (j - 1) & 1, p.status)) return false;
            tc_fence_after();
            if (lane == 0) {
                const uint32_t qa = smem_u32(smem + OFF_Q), ka = smem_u32(kt);
#pragma unroll
                for (int k = 0; k < 4 * NQB; ++k)  // K = 16 steps: box k / 4, 32 bytes apart inside it
                    umma_ss(tmem + T_S, smem_desc_sw128(qa + (k / 4) * BOX + (k % 4) * 32, 16, 1024),
                            smem_desc_sw128(ka + (k / 4) * BOX + (k % 4) * 32, 16, 1024), idesc_qk, k != 0);
                umma_commit(smem_u32(s_ready));
                umma_commit(smem_u32(&k_empty[s]));  // the key tile is free once the scores are computed
            }
            __syncwarp();
            return true;
        };
        if (ok) ok = issue_qk(0);
        for (int j = 0; ok && j < n_tiles; ++j) {
            if (j + 1 < n_tiles && !issue_qk(j + 1)) break;
            const int sv = j % NSV;
            if (!mbar_wait(smem_u32(&v_full[sv]), (j / NSV) & 1, p.status)) break;
            uint8_t* vt = smem + OFF_V + sv * VSTAGE;
            zero_tail(vt, nvb, j);
            if (!mbar_wait(smem_u32(&p_ready[j & 1]), (j >> 1) & 1, p.status)) break;
            tc_fence_after();
            if (lane == 0) {
                const uint32_t va = smem_u32(vt);
#pragma unroll
                for (int kk = 0; kk < TK / 16; ++kk)
                    umma_ts(tmem + T_O, tmem + T_P + (j & 1) * 64 + kk * 8, smem_desc_sw128(va + kk * 2048, BOX, 1024),
                            idesc_pv, (j | kk) != 0);
                umma_commit(smem_u32(&v_empty[sv]));
                umma_commit(smem_u32(&o_ready[j & 1]));
            }
            __syncwarp();
        }
    } else {
        // --------------------------- softmax warps 0-7 ---------------------------
        // Warp w: query rows 32(w%4) .. +31 (its TMEM lane quarter), key columns [64(w/4), +64)
        // of every tile; output columns are split between the two warps in alternate 16-column
        // chunks.
        const int qw = warp & 3, half = warp >> 2;
        const int row = qw * 32 + lane;  // query row in the tile == TMEM lane
        const int q = q0 + row;
        const bool row_ok = q < p.s_q;
        const int vis_end = row_ok ? (p.causal ? L - p.s_q + q + 1 : L) : 0;  // keys < vis_end are visible
        const uint32_t lane_base = (uint32_t)(qw * 32) << 16;
        const int col0 = half * CW;
        float* red_max = reinterpret_cast<float*>(smem + OFF_RED);  // [2][NSW][32]
        float* red_sum = red_max + 2 * NSW * 32;                    // [NSW][32]
        float m_ref = -INFINITY, l = 0.f;
        bool ok = true;
        for (int j = 0; j < n_tiles; ++j) {
            if (ok) ok = mbar_wait(smem_u32(s_ready), j & 1, p.status);
            tc_fence_after();
            uint32_t sr[CW];
#pragma unroll
            for (int c0 = 0; c0 < CW; c0 += 16) tmem_ld16(tmem + lane_base + T_S + col0 + c0, sr + c0);
            tmem_ld_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(s_free));  // the next score tile may be written
            const int k0 = kbeg + j * TK + col0;
            float* sf = reinterpret_cast<float*>(sr);
            if (kbeg + j * TK + TK <= vis_end) {
                const float2 sc2 = make_float2(p.scale_log2, p.scale_log2);
#pragma unroll
                for (int c = 0; c < CW; c += 2) {
                    const float2 v = __fmul2_rn(make_float2(__uint_as_float(sr[c]), __uint_as_float(sr[c + 1])), sc2);
                    sf[c] = v.x;
                    sf[c + 1] = v.y;
                }
            } else {
#pragma unroll
                for (int c = 0; c < CW; ++c)
                    sf[c] = (k0 + c < vis_end) ? __uint_as_float(sr[c]) * p.scale_log2 : -INFINITY;
            }
            // row maximum of the whole tile: this warp's half and the partner warp's half
            float mx = tree_max<CW>(sf);
            red_max[((j & 1) * NSW + warp) * 32 + lane] = mx;
            named_barrier(1 + qw, 64);
            mx = fmaxf(mx, red_max[((j & 1) * NSW + (warp ^ 4)) * 32 + lane]);
            const float m_new = fmaxf(m_ref, mx);
            bool resc = false;
            float alpha = 1.f, m_use = m_ref;
            if (m_ref == -INFINITY) {
                m_use = m_new;
            } else if (m_new > m_ref + 8.0f) {
                resc = true;
                alpha = fast_exp2(m_ref - m_new);
                m_use = m_new;
            }
            uint32_t pk[CW / 2];
            const float m_sub = m_use == -INFINITY ? 0.f : m_use;  // all scores -inf: p = 2^-inf = 0
            const float2 nm2 = make_float2(-m_sub, -m_sub);
#pragma unroll
            for (int c = 0; c < CW; c += 2) {
                const float2 v = __fadd2_rn(make_float2(sf[c], sf[c + 1]), nm2);
                sf[c] = fast_exp2(v.x);
                sf[c + 1] = fast_exp2(v.y);
                pk[c / 2] = pack_bf16x2(sf[c], sf[c + 1]);
            }
            const float rs = tree_sum<CW>(sf);
            l = (resc ? l * alpha : l) + rs;  // this warp's share of the row sum
            m_ref = m_use;
            // P buffer j&1 was last read by PV(j-2); O may only be rescaled after PV(j-1)
            if (ok && j >= 2) ok = mbar_wait(smem_u32(&o_ready[j & 1]), ((j >> 1) - 1) & 1, p.status);
            const bool any_resc = __any_sync(0xffffffffu, resc);
            if (any_resc && ok && j >= 1)
                ok = mbar_wait(smem_u32(&o_ready[(j - 1) & 1]), ((j - 1) >> 1) & 1, p.status);
            tc_fence_after();
#pragma unroll
            for (int c0 = 0; c0 < CW / 2; c0 += 16)
                tmem_st16(tmem + lane_base + T_P + (j & 1) * 64 + half * (CW / 2) + c0, pk + c0);
            if (any_resc) {
                for (int c0 = half * 16; c0 < 64 * nvb; c0 += 32) {
                    uint32_t o[16];
                    tmem_ld16(tmem + lane_base + T_O + c0, o);
                    tmem_ld_wait();
#pragma unroll
                    for (int e = 0; e < 16; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
                    tmem_st16(tmem + lane_base + T_O + c0, o);
                }
            }
            tmem_st_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(&p_ready[j & 1]));
        }
        // the full row sum
        red_sum[warp * 32 + lane] = l;
        named_barrier(1 + qw, 64);
        l += red_sum[(warp ^ 4) * 32 + lane];
        if (ok) ok = mbar_wait(smem_u32(&o_ready[(n_tiles - 1) & 1]), ((n_tiles - 1) >> 1) & 1, p.status);
        if (!ok) {
            s_abort = 1;
        } else {
            tc_fence_after();
            const float inv_l = l > 0.f ? 1.f / l : 0.f;
            // only a split that holds keys of the row writes for it: its normalised partial when the row's keys
            // span several splits, else the result
            const int nsp_row = row_ok ? cdiv(vis_end, p.split_tokens) : 0;
            const bool mine = row_ok && kbeg < vis_end;
            const bool partial = mine && nsp_row > 1;
            // output row of the head and its column: GTA head grp * HPG + c0 / 64, 64 values; GQA head grp, 64 nvb
            constexpr int DOUT = GQA ? 64 * NVB : 64;
            for (int c0 = half * 16; c0 < 64 * nvb; c0 += 32) {
                const int head = GQA ? grp : grp * HPG + c0 / 64;
                const int col = GQA ? c0 : c0 % 64;
                uint32_t o[16];
                tmem_ld16(tmem + lane_base + T_O + c0, o);
                tmem_ld_wait();
                if (partial) {
                    float4* d = reinterpret_cast<float4*>(
                        p.part_o + ((((size_t)b * p.H + head) * p.s_q + q) * p.nsplit + split) * DOUT + col);
#pragma unroll
                    for (int e = 0; e < 4; ++e)
                        d[e] = make_float4(__uint_as_float(o[4 * e]) * inv_l, __uint_as_float(o[4 * e + 1]) * inv_l,
                                           __uint_as_float(o[4 * e + 2]) * inv_l, __uint_as_float(o[4 * e + 3]) * inv_l);
                } else if (mine) {
                    uint32_t pkk[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e)
                        pkk[e] = pack_bf16x2(__uint_as_float(o[2 * e]) * inv_l, __uint_as_float(o[2 * e + 1]) * inv_l);
                    uint4* d = reinterpret_cast<uint4*>(p.out + (((size_t)b * p.H + head) * p.s_q + q) * DOUT + col);
                    d[0] = make_uint4(pkk[0], pkk[1], pkk[2], pkk[3]);
                    d[1] = make_uint4(pkk[4], pkk[5], pkk[6], pkk[7]);
                }
            }
            if (partial && half == 0)
                p.part_lse[(((size_t)b * p.G + grp) * p.s_q + q) * p.nsplit + split] = m_ref + log2f(l);
            else if (mine && p.lse && half == 0)
                p.lse[((size_t)b * p.G + grp) * p.s_q + q] =
                    (l > 0.f ? m_ref + log2f(l) : -INFINITY) * 0.69314718055994530942f;
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == NSW + 1) tmem_dealloc(tmem, 512);
}

// Merge of the key splits of the rows that needed several: 16 threads per (sequence, head, query) row, each
// with 4 of its 64 values (float4 loads, many rows in flight), weights 2^(lse_i - max lse) from the group's
// log2-domain lse of each split; writes the bf16 output and, for the first head of the group, the group's
// natural-log lse.
template <int DOUT>
__global__ void __launch_bounds__(256) gta_combine_kernel(const GtaParams p) {
    constexpr int TPR = DOUT / 4;                                             // threads per row
    const size_t row = (size_t)blockIdx.x * (256 / TPR) + threadIdx.x / TPR;  // ((b * H + h) * s_q + q)
    const int d4 = threadIdx.x % TPR;                                         // values 4 d4 .. 4 d4 + 3
    const size_t nrows = (size_t)p.B * p.H * p.s_q;
    if (row >= nrows) return;
    const int q = (int)(row % p.s_q);
    const int h = (int)((row / p.s_q) % p.H);
    const int b = (int)(row / ((size_t)p.H * p.s_q));
    const int HPG = p.H / p.G, grp = h / HPG;
    const int L = clamp_len(p.lens, b, p.Lmax, p.s_q, p.causal, p.status, false);
    const int n_t = p.causal ? L - p.s_q + q + 1 : L;
    const int nsp = cdiv(n_t, p.split_tokens);
    if (nsp <= 1) return;  // written by the attention kernel
    const float* pl = p.part_lse + (((size_t)b * p.G + grp) * p.s_q + q) * p.nsplit;
    float M = -INFINITY;
    for (int i = 0; i < nsp; ++i) M = fmaxf(M, pl[i]);
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    float wsum = 0.f;
    const float4* po = reinterpret_cast<const float4*>(p.part_o + row * p.nsplit * DOUT) + d4;
    for (int i = 0; i < nsp; ++i) {
        const float w = exp2f(pl[i] - M);
        const float4 v = po[(size_t)i * TPR];
        wsum += w;
        acc = make_float4(fmaf(w, v.x, acc.x), fmaf(w, v.y, acc.y), fmaf(w, v.z, acc.z), fmaf(w, v.w, acc.w));
    }
    const float inv = 1.f / wsum;
    uint2 o;
    o.x = pack_bf16x2(acc.x * inv, acc.y * inv);
    o.y = pack_bf16x2(acc.z * inv, acc.w * inv);
    reinterpret_cast<uint2*>(p.out + row * DOUT)[d4] = o;
    if (p.lse && d4 == 0 && h % HPG == 0)
        p.lse[((size_t)b * p.G + grp) * p.s_q + q] = (M + log2f(wsum)) * 0.69314718055994530942f;
}
}  // namespace lka

using namespace lka;

extern "C" {

}  // extern "C"

namespace {

// Key splits: one CTA per (query tile, group, sequence) and key split.  When the query tiles alone give less
// than about two waves of CTAs (a prefill chunk over a long cached prefix), the keys are split so that they
// do; the split size stays >= 512 keys.  The split partials (normalised O per head, lse per group) live in
// the workspace after the status header.
struct GtaPlan {
    int split_tokens, nsplit;
    size_t off_lse, off_o, ws_bytes;
};

void gta_plan(int B, int G, int H, int s_q, int Lmax, GtaPlan* pl, int dout = 64) {
    int st = split_tokens_knob();
    if (st <= 0) {
        const long long units = (long long)cdiv(s_q, gta::TQ) * G * (B > 0 ? B : 1);
        const long long target = 2LL * sm_count();
        const long long nsp = units >= target ? 1 : (target + units - 1) / units;
        st = (int)((Lmax + nsp - 1) / nsp);
        if (st < 512) st = 512;
    }
    st = cdiv(st, gta::TK) * gta::TK;
    pl->split_tokens = st;
    pl->nsplit = cdiv(Lmax, st);
    WsCarve c;
    pl->off_lse = pl->off_o = 0;
    if (pl->nsplit > 1) {
        pl->off_lse = c.take((size_t)B * G * s_q * pl->nsplit * sizeof(float));
        pl->off_o = c.take((size_t)B * H * s_q * pl->nsplit * dout * sizeof(float));
    }
    pl->ws_bytes = c.off;
}

}  // namespace

extern "C" size_t gta_shared_score_attn_workspace_size(int B, int G, int H, int s_q, int d_qk, int d_v, int Lmax) {
    if (B < 0 || G < 1 || H < 1 || s_q < 1 || Lmax < 1 || H % G) return 0;
    (void)d_qk;
    (void)d_v;
    GtaPlan pl;
    gta_plan(B, G, H, s_q, Lmax, &pl);
    return pl.ws_bytes;
}

namespace {

// Launches the attention kernel instance over grid (query tiles x splits, groups, sequences) and, with key
// splits, the merge.
template <int NQB, int NVB, bool GQA>
lka_status_t gta_launch(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv, const CUtensorMap& tq2,
                        const CUtensorMap& tk2, const GtaParams& p, cudaStream_t st) {
    constexpr int SMEM = gta::Cfg<NQB, NVB>::SMEM;
    auto kern = gta_attn_kernel<NQB, NVB, GQA>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM) != cudaSuccess)
        return LKA_ERR_CUDA;
    if ((long long)cdiv(p.s_q, gta::TQ) * p.nsplit >= (1ll << 31)) return LKA_ERR_UNSUPPORTED;
    dim3 grid(cdiv(p.s_q, gta::TQ) * p.nsplit, p.G, p.B);
    {
        TimedLaunch timer(st);
        kern<<<grid, gta::NTHREADS, SMEM, st>>>(tq, tk, tv, tq2, tk2, p);
        timer.stop();
    }
    if (cudaPeekAtLastError() != cudaSuccess) return LKA_ERR_CUDA;
    if (p.nsplit > 1) {
        constexpr int DOUT = GQA ? 64 * NVB : 64;
        constexpr int RPB = 256 / (DOUT / 4);  // rows per merge block
        const size_t rows = (size_t)p.B * p.H * p.s_q;
        gta_combine_kernel<DOUT><<<(unsigned)((rows + RPB - 1) / RPB), 256, 0, st>>>(p);
    }
    return cudaPeekAtLastError() == cudaSuccess ? LKA_OK : LKA_ERR_CUDA;
}

struct GtaPages {
    const int32_t* block_table;
    int page_size, max_pages, num_pages;
};

// Validates the arguments and launches the kernel.  Contiguous caches: pg == nullptr, k_g [B,G,Lmax,64],
// v [B,H,Lmax,64].  Paged: k_g [num_pages,G,page_size,64], v [num_pages,H,page_size,64], and Lmax is the
// capacity max_pages * page_size.
lka_status_t gta_run(const void* q_g, const void* k_g, const void* v, const int32_t* cache_lens, void* out,
                     float* lse, int B, int G, int H, int s_q, int d_qk, int d_v, int Lmax, int causal, float scale,
                     lka_dtype_t dtype, void* ws, size_t ws_bytes, void* stream, const GtaPages* pg) {
    if (B < 0 || G < 1 || H < 1 || s_q < 1 || Lmax < 1 || d_qk < 1 || d_v < 1) return LKA_ERR_INVALID_ARG;
    if (H % G) return LKA_ERR_INVALID_ARG;
    if (dtype != LKA_BF16 || d_qk != 64 || d_v != 64 || H / G > 4) return LKA_ERR_UNSUPPORTED;
    if ((long long)B * H * Lmax >= (1ll << 31) || (long long)B * G * s_q >= (1ll << 31) || B > 65535 || G > 65535)
        return LKA_ERR_UNSUPPORTED;
    if (pg && (long long)pg->num_pages * H * pg->page_size >= (1ll << 31)) return LKA_ERR_UNSUPPORTED;
    if (B == 0) return LKA_OK;
    const void* ptrs[] = {q_g, k_g, v, cache_lens, out};
    for (const void* ptr : ptrs)
        if (!ptr || !aligned16(ptr)) return LKA_ERR_INVALID_ARG;
    if (pg && !pg->block_table) return LKA_ERR_INVALID_ARG;
    if (!isfinite(scale)) return LKA_ERR_INVALID_ARG;
    GtaPlan pl;
    gta_plan(B, G, H, s_q, Lmax, &pl);
    if (!ws || ws_bytes < pl.ws_bytes) return LKA_ERR_WORKSPACE;
    if (!aligned16(ws)) return LKA_ERR_INVALID_ARG;
    const auto BF = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    const int box_rows = pg ? std::min(gta::TK, pg->page_size) : gta::TK;
    const uint64_t k_rows = pg ? (uint64_t)pg->num_pages * G * pg->page_size : (uint64_t)B * G * Lmax;
    const uint64_t v_rows = pg ? (uint64_t)pg->num_pages * H * pg->page_size : (uint64_t)B * H * Lmax;
    CUtensorMap tq, tk, tv;
    if (!make_tmap_2d(&tq, BF, q_g, 64, (uint64_t)B * G * s_q, 128, 64, 128) ||
        !make_tmap_2d(&tk, BF, k_g, 64, k_rows, 128, 64, box_rows) ||
        !make_tmap_2d(&tv, BF, v, 64, v_rows, 128, 64, box_rows))
        return LKA_ERR_CUDA;
    GtaParams p{};
    p.lens = cache_lens;
    p.out = static_cast<__nv_bfloat16*>(out);
    p.lse = lse;
    p.status = static_cast<uint32_t*>(ws);
    p.B = B;
    p.G = G;
    p.H = H;
    p.s_q = s_q;
    p.Lmax = Lmax;
    p.causal = causal ? 1 : 0;
    p.scale_log2 = scale * 1.4426950408889634f;
    p.box_rows = box_rows;
    p.split_tokens = pl.split_tokens;
    p.nsplit = pl.nsplit;
    p.part_lse = pl.nsplit > 1 ? reinterpret_cast<float*>(static_cast<uint8_t*>(ws) + pl.off_lse) : nullptr;
    p.part_o = pl.nsplit > 1 ? reinterpret_cast<float*>(static_cast<uint8_t*>(ws) + pl.off_o) : nullptr;
    if (pg) {
        p.block_table = pg->block_table;
        p.page_size = pg->page_size;
        p.max_pages = pg->max_pages;
        p.num_pages = pg->num_pages;
    }
    return gta_launch<1, 4, false>(tq, tk, tv, tq, tk, p, (cudaStream_t)stream);
}

bool gta_pages_ok(int page_size, int max_pages, int num_pages) {
    return page_size >= 8 && (page_size & (page_size - 1)) == 0 && max_pages >= 1 && num_pages >= 1 &&
           (long long)max_pages * page_size < (1ll << 31);
}

}  // namespace

extern "C" {

lka_status_t gta_shared_score_attn(const void* q_g, const void* k_g, const void* v, const int32_t* cache_lens,
                                   void* out, float* lse, int B, int G, int H, int s_q, int d_qk, int d_v, int Lmax,
                                   int causal, float scale, lka_dtype_t dtype, void* ws, size_t ws_bytes,
                                   void* stream) {
    return gta_run(q_g, k_g, v, cache_lens, out, lse, B, G, H, s_q, d_qk, d_v, Lmax, causal, scale, dtype, ws,
                   ws_bytes, stream, nullptr);
}

size_t gta_shared_score_attn_paged_workspace_size(int B, int G, int H, int s_q, int d_qk, int d_v, int page_size,
                                                  int max_pages) {
    if (!gta_pages_ok(page_size, max_pages, 1)) return 0;
    return gta_shared_score_attn_workspace_size(B, G, H, s_q, d_qk, d_v, page_size * max_pages);
}

lka_status_t gta_shared_score_attn_paged(const void* q_g, const void* k_pages, const void* v_pages,
                                         const int32_t* block_table, const int32_t* cache_lens, void* out,
                                         float* lse, int B, int G, int H, int s_q, int d_qk, int d_v, int page_size,
                                         int max_pages, int num_pages, int causal, float scale, lka_dtype_t dtype,
                                         void* ws, size_t ws_bytes, void* stream) {
    if (!gta_pages_ok(page_size, max_pages, num_pages)) return LKA_ERR_INVALID_ARG;
    const GtaPages pg{block_table, page_size, max_pages, num_pages};
    return gta_run(q_g, k_pages, v_pages, cache_lens, out, lse, B, G, H, s_q, d_qk, d_v, page_size * max_pages,
                   causal, scale, dtype, ws, ws_bytes, stream, &pg);
}

}  // extern "C"

namespace lka {

// Causal (or full) prefill of grouped-query attention with d = 128 on the tensor cores (the kernel above in its
// GQA form): one CTA per (128-query tile, query head, sequence, key split).
size_t gqa_prefill_ws_bytes(int B, int h_q, int s_q, int Lmax) {
    GtaPlan pl;
    gta_plan(B, h_q, h_q, s_q, Lmax, &pl, 128);
    return pl.ws_bytes;
}

int gqa_prefill_nsplit(int B, int h_q, int s_q, int Lmax) {
    GtaPlan pl;
    gta_plan(B, h_q, h_q, s_q, Lmax, &pl, 128);
    return pl.nsplit;
}

lka_status_t gqa_prefill_tc(const void* q, const void* k, const void* v, const int32_t* cache_lens, void* out,
                            float* lse, int B, int h_q, int h_kv, int s_q, int Lmax, int causal, float scale, void* ws,
                            size_t ws_bytes, cudaStream_t st, const int32_t* block_table, int page_size, int max_pages,
                            int num_pages) {
    GtaPlan pl;
    gta_plan(B, h_q, h_q, s_q, Lmax, &pl, 128);
    if (!ws || ws_bytes < pl.ws_bytes) return LKA_ERR_WORKSPACE;
    if ((long long)B * h_q * s_q >= (1ll << 31) || B > 65535 || h_q > 65535) return LKA_ERR_UNSUPPORTED;
    const auto BF = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    const int box_rows = block_table ? std::min(gta::TK, page_size) : gta::TK;
    const uint64_t kv_rows = block_table ? (uint64_t)num_pages * h_kv * page_size : (uint64_t)B * h_kv * Lmax;
    CUtensorMap tq, tk, tv;
    if (!make_tmap_2d(&tq, BF, q, 128, (uint64_t)B * h_q * s_q, 256, 64, 128) ||
        !make_tmap_2d(&tk, BF, k, 128, kv_rows, 256, 64, box_rows) ||
        !make_tmap_2d(&tv, BF, v, 128, kv_rows, 256, 64, box_rows))
        return LKA_ERR_CUDA;
    GtaParams p{};
    p.lens = cache_lens;
    p.out = static_cast<__nv_bfloat16*>(out);
    p.lse = lse;
    p.status = static_cast<uint32_t*>(ws);
    p.B = B;
    p.G = h_q;
    p.H = h_q;
    p.s_q = s_q;
    p.Lmax = Lmax;
    p.causal = causal ? 1 : 0;
    p.scale_log2 = scale * 1.4426950408889634f;
    p.box_rows = box_rows;
    p.split_tokens = pl.split_tokens;
    p.nsplit = pl.nsplit;
    p.part_lse = pl.nsplit > 1 ? reinterpret_cast<float*>(static_cast<uint8_t*>(ws) + pl.off_lse) : nullptr;
    p.part_o = pl.nsplit > 1 ? reinterpret_cast<float*>(static_cast<uint8_t*>(ws) + pl.off_o) : nullptr;
    p.h_kv = h_kv;
    p.kv_ratio = h_q / h_kv;
    if (block_table) {
        p.block_table = block_table;
        p.page_size = page_size;
        p.max_pages = max_pages;
        p.num_pages = num_pages;
    }
    return gta_launch<2, 2, true>(tq, tk, tv, tq, tk, p, st);
}

// Prefill of the GQLA per-group GQA path (bf16, d_h = 128, d_h^R = 64): keys [kc[gamma] ; k^R] of 192 values,
// values vc[gamma], h_q / g query heads per group; contiguous caches kc, vc [B, g, Lmax, 128], kr [B, Lmax, 64],
// or paged pools [num_pages, g, page_size, 128] and [num_pages, page_size, 64] with block_table.
size_t expanded_prefill_ws_bytes(int B, int h_q, int s_q, int Lmax) { return gqa_prefill_ws_bytes(B, h_q, s_q, Lmax); }

lka_status_t expanded_prefill_tc(const void* q_c, const void* q_r, const void* kc, const void* vc, const void* kr,
                                 const int32_t* cache_lens, void* out, float* lse, int B, int h_q, int g, int s_q,
                                 int Lmax, int causal, float scale, void* ws, size_t ws_bytes, cudaStream_t st,
                                 const int32_t* block_table, int page_size, int max_pages, int num_pages) {
    GtaPlan pl;
    gta_plan(B, h_q, h_q, s_q, Lmax, &pl, 128);
    if (!ws || ws_bytes < pl.ws_bytes) return LKA_ERR_WORKSPACE;
    if ((long long)B * h_q * s_q >= (1ll << 31) || B > 65535 || h_q > 65535) return LKA_ERR_UNSUPPORTED;
    const auto BF = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    const int box_rows = block_table ? std::min(gta::TK, page_size) : gta::TK;
    const uint64_t kv_rows = block_table ? (uint64_t)num_pages * g * page_size : (uint64_t)B * g * Lmax;
    const uint64_t r_rows = block_table ? (uint64_t)num_pages * page_size : (uint64_t)B * Lmax;
    const uint64_t q_rows = (uint64_t)B * h_q * s_q;
    CUtensorMap tq, tq2, tk, tk2, tv;
    if (!make_tmap_2d(&tq, BF, q_c, 128, q_rows, 256, 64, 128) || !make_tmap_2d(&tq2, BF, q_r, 64, q_rows, 128, 64, 128) ||
        !make_tmap_2d(&tk, BF, kc, 128, kv_rows, 256, 64, box_rows) ||
        !make_tmap_2d(&tk2, BF, kr, 64, r_rows, 128, 64, box_rows) ||
        !make_tmap_2d(&tv, BF, vc, 128, kv_rows, 256, 64, box_rows))
        return LKA_ERR_CUDA;
    GtaParams p{};
    p.lens = cache_lens;
    p.out = static_cast<__nv_bfloat16*>(out);
    p.lse = lse;
    p.status = static_cast<uint32_t*>(ws);
    p.B = B;
    p.G = h_q;
    p.H = h_q;
    p.s_q = s_q;
    p.Lmax = Lmax;
    p.causal = causal ? 1 : 0;
    p.scale_log2 = scale * 1.4426950408889634f;
    p.box_rows = box_rows;
    p.split_tokens = pl.split_tokens;
    p.nsplit = pl.nsplit;
    p.part_lse = pl.nsplit > 1 ? reinterpret_cast<float*>(static_cast<uint8_t*>(ws) + pl.off_lse) : nullptr;
    p.part_o = pl.nsplit > 1 ? reinterpret_cast<float*>(static_cast<uint8_t*>(ws) + pl.off_o) : nullptr;
    p.h_kv = g;
    p.kv_ratio = h_q / g;
    if (block_table) {
        p.block_table = block_table;
        p.page_size = page_size;
        p.max_pages = max_pages;
        p.num_pages = num_pages;
    }
    return gta_launch<3, 2, true>(tq, tk, tv, tq2, tk2, p, st);
}

}  // namespace lka
