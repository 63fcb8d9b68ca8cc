// expanded_attn.cu -- the GQA decode path of GQLA over the per-group expanded
// cache, on the 5th-generation tensor cores.
//
// Operation ("GQLA: Group-Query Latent Attention ..." section 1, section 3.1,
// Figure 2(a)): every group gamma of h_q/g = 16 query heads attends with keys
// [K_C[gamma] ; k^R] (128 + 64 values, the RoPE key stored once and shared by
// the groups) and values V[gamma] (128 values); query of head i is
// [q^C_i ; q^R_i].  The paper notes that 16 query heads per KV head match a
// tensor-core MMA tile; with s_q = 1 or 2 (multi-token prediction) one group
// has 16 or 32 query rows, too few for the 128-row MMA, so the kernel swaps
// the operands:
//     S^T [128 tokens x NR rows] = K_tile [128 x 192] * Q^T [192 x NR]
//     O^T [128 dims  x NR rows] += V_tile^T [128 x 128 tokens] * P^T [128 tokens x NR]
// Both accumulators live in tensor memory (lanes = tokens or value dims,
// columns = query rows).  The softmax runs down the lanes: the score tile is
// transposed through shared memory and each 16-lane half-warp reduces one
// query row over the 128 tokens, writing P^T straight into the swizzled
// shared-memory layout the P*V MMA reads.
//
// One CTA = (sequence b, group gamma, split of the keys): warp 4 streams
// 128-token tiles of K_C, k^R and V with TMA (2 stages of 80 KB), warp 5 issues
// the MMAs, warps 0-3 run the softmax with lazy rescaling of O^T.
#include "common.cuh"
#include "expanded.h"
#include "gqa_decode.h"
#include "host_util.h"
#include "tc.cuh"

namespace lka {

template <int NR>
struct ExpCfg {
    static constexpr int TK = 128;                 // tokens per tile (MMA M)
    static constexpr int NST = 2;                  // depth of the key ring and of the value ring
    static constexpr int BOX = TK * 128;           // 128 tokens x 64 bf16
    static constexpr int Q_BYTES = 3 * NR * 128;   // Q^T: 3 K-blocks (q_c 0..63, 64..127, q_r)
    static constexpr int KSTAGE = 3 * BOX;         // kc x2, kr (released after S^T = K Q^T)
    static constexpr int VSTAGE = 2 * BOX;         // vc x2 (released after O^T += V^T P^T)
    static constexpr int STAGE = KSTAGE + VSTAGE;
    static constexpr int SC_BYTES = NR * TK * 4;   // transposed scores
    static constexpr int PT_BYTES = 2 * NR * 128;  // P^T: 2 K-blocks of 64 tokens
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_KV = 16384;           // Q region padded to keep 1024-alignment
    static constexpr int OFF_SC = OFF_KV + NST * STAGE;
    static constexpr int OFF_PT = OFF_SC + 2 * SC_BYTES;
    static constexpr int OFF_AUX = OFF_PT + 2 * PT_BYTES;  // alpha[NR], l[NR], m[NR]
    static constexpr int OFF_BAR = OFF_AUX + 3 * NR * 4;
    static constexpr int SMEM = 1024 + OFF_BAR + 256;
    static constexpr uint32_t T_S = 0;             // 2 x NR columns
    static constexpr uint32_t T_O = 2 * NR;        // NR columns
    static constexpr int NSW = 8;                  // softmax warps: 4 TMEM lane quarters x 2 column halves
    static constexpr int HALF = NR / 2;            // score / output columns per softmax warp
    static constexpr int K_ITEMS = NR * 16 / (32 * NSW);  // (row, 8-token chunk) items per softmax thread
    static constexpr int NTHREADS = 32 * (NSW + 2);
    static_assert(Q_BYTES <= OFF_KV, "Q region");
};

// 8 consecutive columns of this warp's 32 TMEM lanes
__device__ __forceinline__ void tmem_ld8(uint32_t taddr, uint32_t* r) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
                 : "r"(taddr));
}
template <int N>
__device__ __forceinline__ void tmem_ld_cols(uint32_t taddr, uint32_t* r) {
    static_assert(N == 8 || N == 16, "8 or 16 columns");
    if constexpr (N == 8)
        tmem_ld8(taddr, r);
    else
        tmem_ld16(taddr, r);
}
template <int N>
__device__ __forceinline__ void tmem_st_cols(uint32_t taddr, const uint32_t* r) {
    static_assert(N == 8 || N == 16, "8 or 16 columns");
    if constexpr (N == 8)
        tmem_st8(taddr, r);
    else
        tmem_st16(taddr, r);
}

template <int NR>
__global__ void __launch_bounds__(ExpCfg<NR>::NTHREADS, 1)
    expanded_attn_kernel(const __grid_constant__ CUtensorMap tm_qc, const __grid_constant__ CUtensorMap tm_qr,
                         const __grid_constant__ CUtensorMap tm_kc, const __grid_constant__ CUtensorMap tm_kr,
                         const __grid_constant__ CUtensorMap tm_vc, const ExpParams p) {
    using C = ExpCfg<NR>;
    constexpr int TK = C::TK, NST = C::NST;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(align_up(reinterpret_cast<uintptr_t>(smem_raw), 1024));
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
    uint64_t* q_full = bars;
    uint64_t* k_full = bars + 1;
    uint64_t* k_empty = k_full + NST;
    uint64_t* v_full = k_empty + NST;
    uint64_t* v_empty = v_full + NST;
    uint64_t* s_ready = v_empty + NST;   // [2] QK(j) done
    uint64_t* s_free = s_ready + 2;      // [2] S(j) loaded by the softmax warps
    uint64_t* p_ready = s_free + 2;      // [2] P^T(j) written
    uint64_t* o_ready = p_ready + 2;     // [2] PV(j) done
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(o_ready + 2);
    float* alpha_buf = reinterpret_cast<float*>(smem + C::OFF_AUX);
    float* l_buf = alpha_buf + NR;
    float* m_buf = l_buf + NR;
    __shared__ int s_abort;
    __shared__ int s_resc[2];  // [tile & 1] some row of the tile moved its reference maximum

    const int split = blockIdx.x, grp = blockIdx.y, b = blockIdx.z;
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int HPG = p.h_q / p.g;  // 16
    const int L = clamp_len(p.lens, b, p.Lmax, p.s_q, p.causal, p.status,
                            threadIdx.x == 0 && split == 0 && grp == 0);
    const int kbeg = split * p.split_tokens;
    const int kend = min(L, kbeg + p.split_tokens);  // the last query row sees keys < L
    const int n_tiles = kend > kbeg ? cdiv(kend - kbeg, TK) : 0;
    if (n_tiles == 0) return;

    if (threadIdx.x == 0) {
        s_abort = 0;
        s_resc[0] = s_resc[1] = 0;
        mbar_init(smem_u32(q_full), 1);
        for (int s = 0; s < NST; ++s) {
            mbar_init(smem_u32(&k_full[s]), 1);
            mbar_init(smem_u32(&k_empty[s]), 1);
            mbar_init(smem_u32(&v_full[s]), 1);
            mbar_init(smem_u32(&v_empty[s]), 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(smem_u32(&s_ready[i]), 1);
            mbar_init(smem_u32(&s_free[i]), C::NSW);
            mbar_init(smem_u32(&p_ready[i]), C::NSW);
            mbar_init(smem_u32(&o_ready[i]), 1);
        }
        fence_barrier_init();
    }
    if (warp == C::NSW + 1) {
        tmem_alloc(tmem_slot, 128);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == C::NSW) {
        // --------------------------------- producer ---------------------------------
        if (lane == 0) {
            const uint32_t qb = smem_u32(q_full);
            mbar_arrive_expect_tx(qb, C::Q_BYTES);
            const int qrow = (b * p.h_q + grp * HPG) * p.s_q;
            const uint32_t qd = smem_u32(smem + C::OFF_Q);
            tma_load_2d(qd, &tm_qc, 0, qrow, qb);
            tma_load_2d(qd + NR * 128, &tm_qc, 64, qrow, qb);
            tma_load_2d(qd + 2 * NR * 128, &tm_qr, 0, qrow, qb);
            // issue order K(0), then per tile i: K(i+1), V(i); key tiles are released as soon as
            // their score MMAs complete, value tiles after their P*V MMAs
            int k_issued = 0, v_issued = 0;
            bool ok = true;
            // rows of token `tok` in the per-group cache (kc, vc) and in the RoPE-key cache (kr): contiguous
            // [B][g][Lmax] / [B][Lmax] slabs, or a page of the block table ([num_pages][g][page_size] /
            // [num_pages][page_size]); entries outside the pool are replaced by page 0 (reported when the
            // attention needs the token)
            auto rows_of = [&](int tok, int& yg, int& yr) {
                if (!p.block_table) {
                    yg = (b * p.g + grp) * p.Lmax + tok;
                    yr = b * p.Lmax + tok;
                    return;
                }
                int page = 0;
                const int j = tok / p.page_size;
                if (j < p.max_pages) {
                    page = p.block_table[(size_t)b * p.max_pages + j];
                    if (page < 0 || page >= p.num_pages) {
                        if (tok < L) atomicOr(p.status, kDevBadPage);
                        page = 0;
                    }
                }
                yg = (page * p.g + grp) * p.page_size + tok % p.page_size;
                yr = page * p.page_size + tok % p.page_size;
            };
            auto issue_k = [&](int i) {
                const int s = i % NST;
                if (i >= NST && !mbar_wait(smem_u32(&k_empty[s]), ((i / NST) - 1) & 1, p.status)) return false;
                const uint32_t fb = smem_u32(&k_full[s]);
                mbar_arrive_expect_tx(fb, C::KSTAGE);
                const uint32_t d = smem_u32(smem + C::OFF_KV + s * C::STAGE);
                for (int r0 = 0; r0 < TK; r0 += p.box_rows) {  // one box, or one per page piece of the tile
                    int yg, yr;
                    rows_of(kbeg + i * TK + r0, yg, yr);
                    tma_load_2d(d + r0 * 128, &tm_kc, 0, yg, fb);
                    tma_load_2d(d + C::BOX + r0 * 128, &tm_kc, 64, yg, fb);
                    tma_load_2d(d + 2 * C::BOX + r0 * 128, &tm_kr, 0, yr, fb);
                }
                ++k_issued;
                return true;
            };
            auto issue_v = [&](int i) {
                const int s = i % NST;
                if (i >= NST && !mbar_wait(smem_u32(&v_empty[s]), ((i / NST) - 1) & 1, p.status)) return false;
                const uint32_t fb = smem_u32(&v_full[s]);
                mbar_arrive_expect_tx(fb, C::VSTAGE);
                const uint32_t d = smem_u32(smem + C::OFF_KV + s * C::STAGE + C::KSTAGE);
                for (int r0 = 0; r0 < TK; r0 += p.box_rows) {
                    int yg, yr;
                    rows_of(kbeg + i * TK + r0, yg, yr);
                    tma_load_2d(d + r0 * 128, &tm_vc, 0, yg, fb);
                    tma_load_2d(d + C::BOX + r0 * 128, &tm_vc, 64, yg, fb);
                }
                ++v_issued;
                return true;
            };
            ok = issue_k(0);
            for (int i = 0; ok && i < n_tiles; ++i) {
                if (*(volatile int*)&s_abort) break;
                if (i + 1 < n_tiles) ok = issue_k(i + 1);
                if (ok) ok = issue_v(i);
            }
            if (!ok) s_abort = 1;
            for (int i = k_issued - 1; i >= 0 && i >= k_issued - NST; --i)
                mbar_wait(smem_u32(&k_full[i % NST]), (i / NST) & 1, p.status);
            for (int i = v_issued - 1; i >= 0 && i >= v_issued - NST; --i)
                mbar_wait(smem_u32(&v_full[i % NST]), (i / NST) & 1, p.status);
            mbar_wait(qb, 0, p.status);
        }
    } else if (warp == C::NSW + 1) {
        // -------------------------------- MMA issuer --------------------------------
        // per step j: QK(j) (needs S(j-2) loaded by the softmax warps) and PV(j-1)
        constexpr uint32_t idesc_qk = idesc_bf16_f32(128, NR, false, false);
        constexpr uint32_t idesc_pv = idesc_bf16_f32(128, NR, true, false);
        bool ok = mbar_wait(smem_u32(q_full), 0, p.status);
        for (int j = 0; ok && j < n_tiles + 1; ++j) {
            if (j < n_tiles) {
                const int s = j % NST;
                if (!mbar_wait(smem_u32(&k_full[s]), (j / NST) & 1, p.status)) break;
                uint8_t* st = smem + C::OFF_KV + s * C::STAGE;
                const int nvalid = min(TK, kend - (kbeg + j * TK));
                if (nvalid < TK) {
                    // keys past the key range may hold anything (even NaN): zero them
                    const int rows = TK - nvalid;
                    for (int idx = lane; idx < 3 * rows * 8; idx += 32) {
                        const int bx = idx / (rows * 8), rr = (idx / 8) % rows, c = idx % 8;
                        *reinterpret_cast<uint4*>(st + bx * C::BOX + (nvalid + rr) * 128 + c * 16) =
                            make_uint4(0, 0, 0, 0);
                    }
                    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                    __syncwarp();
                }
                if (j >= 2 && !mbar_wait(smem_u32(&s_free[j & 1]), ((j >> 1) - 1) & 1, p.status)) break;
                tc_fence_after();
                if (lane == 0) {
                    const uint32_t ka = smem_u32(st);
                    const uint32_t qa = smem_u32(smem + C::OFF_Q);
                    for (int kb = 0; kb < 3; ++kb)
#pragma unroll
                        for (int k = 0; k < 4; ++k)
                            umma_ss(tmem + C::T_S + (j & 1) * NR, smem_desc_sw128(ka + kb * C::BOX + k * 32, 16, 1024),
                                    smem_desc_sw128(qa + kb * NR * 128 + k * 32, 16, 1024), idesc_qk, (kb | k) != 0);
                    umma_commit(smem_u32(&s_ready[j & 1]));
                    umma_commit(smem_u32(&k_empty[s]));
                }
                __syncwarp();
            }
            if (j >= 1) {
                const int i = j - 1;
                const int sv = i % NST;
                if (!mbar_wait(smem_u32(&v_full[sv]), (i / NST) & 1, p.status)) break;
                uint8_t* vt = smem + C::OFF_KV + sv * C::STAGE + C::KSTAGE;
                const int nvalid = min(TK, kend - (kbeg + i * TK));
                if (nvalid < TK) {
                    // values past the key range may hold anything (even NaN): zero them so P = 0 adds nothing
                    const int rows = TK - nvalid;
                    for (int idx = lane; idx < 2 * rows * 8; idx += 32) {
                        const int bx = idx / (rows * 8), rr = (idx / 8) % rows, c = idx % 8;
                        *reinterpret_cast<uint4*>(vt + bx * C::BOX + (nvalid + rr) * 128 + c * 16) =
                            make_uint4(0, 0, 0, 0);
                    }
                    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                    __syncwarp();
                }
                if (!mbar_wait(smem_u32(&p_ready[i & 1]), (i >> 1) & 1, p.status)) break;
                tc_fence_after();
                if (lane == 0) {
                    const uint32_t va = smem_u32(vt);
                    const uint32_t pa = smem_u32(smem + C::OFF_PT + (i & 1) * C::PT_BYTES);
#pragma unroll
                    for (int kk = 0; kk < TK / 16; ++kk)
                        umma_ss(tmem + C::T_O, smem_desc_sw128(va + kk * 2048, C::BOX, 1024),
                                smem_desc_sw128(pa + (kk / 4) * NR * 128 + (kk % 4) * 32, 16, 1024), idesc_pv,
                                (i | kk) != 0);
                    umma_commit(smem_u32(&v_empty[sv]));
                    umma_commit(smem_u32(&o_ready[i & 1]));
                }
                __syncwarp();
            }
        }
    } else {
        // ----------------------------- softmax warps (0-7) -----------------------------
        // Warp w reads TMEM lane quarter w % 4 (tokens of S^T, value dims of O^T) and the column half w / 4
        // (query rows); after the transpose through shared memory the (row, 8-token chunk) items are
        // spread over all 256 threads.
        const int tid = (warp & 3) * 32 + lane;  // token lane of S^T, value dim of O^T
        const int half = warp >> 2;
        const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
        float m_ref[C::K_ITEMS], lsum[C::K_ITEMS];
#pragma unroll
        for (int k = 0; k < C::K_ITEMS; ++k) {
            m_ref[k] = -INFINITY;
            lsum[k] = 0.f;
        }
        const int c8 = lane % 16;  // 8-token chunk of this thread's items
        bool ok = true;
        for (int i = 0; i < n_tiles; ++i) {
            const int x = i & 1;
            if (ok) ok = mbar_wait(smem_u32(&s_ready[x]), (i >> 1) & 1, p.status);
            tc_fence_after();
            float* sc = reinterpret_cast<float*>(smem + C::OFF_SC + x * C::SC_BYTES);
            {
                uint32_t v[C::HALF];
                tmem_ld_cols<C::HALF>(tmem + lane_base + C::T_S + x * NR + half * C::HALF, v);
                tmem_ld_wait();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(smem_u32(&s_free[x]));  // the score buffer may be rewritten
#pragma unroll
                for (int r = 0; r < C::HALF; ++r) sc[(half * C::HALF + r) * TK + tid] = __uint_as_float(v[r]);
            }
            // P^T buffer x was last read by PV(i-2)
            if (ok && i >= 2) ok = mbar_wait(smem_u32(&o_ready[x]), ((i >> 1) - 1) & 1, p.status);
            // the rescale flag of this buffer was last read in tile i-2, before every thread passed the
            // barriers of tile i-1
            if (threadIdx.x == 0) s_resc[x] = 0;
            named_barrier(1, 32 * C::NSW);
            uint8_t* pt = smem + C::OFF_PT + x * C::PT_BYTES;
            const int k0 = kbeg + i * TK;
#pragma unroll
            for (int k = 0; k < C::K_ITEMS; ++k) {
                const int r = 2 * C::NSW * k + 2 * warp + lane / 16;  // query row: hh * s_q + t (16 lanes per row)
                const int t = r % p.s_q;
                const int rend = min(p.causal ? L - p.s_q + t + 1 : L, kbeg + p.split_tokens);
                const float4 a = *reinterpret_cast<const float4*>(sc + r * TK + 8 * c8);
                const float4 bq = *reinterpret_cast<const float4*>(sc + r * TK + 8 * c8 + 4);
                float s[8] = {a.x, a.y, a.z, a.w, bq.x, bq.y, bq.z, bq.w};
#pragma unroll
                for (int e = 0; e < 8; ++e) s[e] = (k0 + 8 * c8 + e < rend) ? s[e] * p.scale_log2 : -INFINITY;
                // lazy rescaling: the reference maximum of a row only moves when one of its scores exceeds it
                // by more than 2^8, so the row maximum is only reduced over the 16 lanes of the row then (the
                // warp's two rows together); the row sums stay per lane until the end
                float mx = tree_max<8>(s);
                float alpha = 1.f, m_use = m_ref[k];
                if (__any_sync(0xffffffffu, !(mx <= m_ref[k] + 8.0f))) {
#pragma unroll
                    for (int m = 8; m >= 1; m /= 2) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, m));
                    const float m_new = fmaxf(m_ref[k], mx);
                    if (m_ref[k] == -INFINITY) {
                        m_use = m_new;
                    } else if (m_new > m_ref[k] + 8.0f) {
                        alpha = fast_exp2(m_ref[k] - m_new);
                        m_use = m_new;
                    }
                }
                float pv[8];
                const float m_sub = m_use == -INFINITY ? 0.f : m_use;  // all scores -inf: p = 0
#pragma unroll
                for (int e = 0; e < 8; ++e) pv[e] = fast_exp2(s[e] - m_sub);
                lsum[k] = lsum[k] * alpha + tree_sum<8>(pv);  // this lane's share of the row sum
                m_ref[k] = m_use;
                const int kb2 = c8 / 8, cc = c8 % 8;
                *reinterpret_cast<uint4*>(pt + kb2 * NR * 128 + r * 128 + ((cc ^ (r & 7)) << 4)) =
                    make_uint4(pack_bf16x2(pv[0], pv[1]), pack_bf16x2(pv[2], pv[3]), pack_bf16x2(pv[4], pv[5]),
                               pack_bf16x2(pv[6], pv[7]));
                if (c8 == 0) alpha_buf[r] = alpha;
                if (alpha != 1.f) s_resc[x] = 1;
            }
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            named_barrier(1, 32 * C::NSW);  // alpha_buf and the rescale flag complete
            if (*(volatile int*)&s_resc[x]) {
                // O^T may only be rescaled once PV(i-1) has been accumulated into it
                if (ok && i >= 1) ok = mbar_wait(smem_u32(&o_ready[(i - 1) & 1]), ((i - 1) >> 1) & 1, p.status);
                tc_fence_after();
                uint32_t o[C::HALF];
                tmem_ld_cols<C::HALF>(tmem + lane_base + C::T_O + half * C::HALF, o);
                tmem_ld_wait();
#pragma unroll
                for (int r = 0; r < C::HALF; ++r)
                    o[r] = __float_as_uint(__uint_as_float(o[r]) * alpha_buf[half * C::HALF + r]);
                tmem_st_cols<C::HALF>(tmem + lane_base + C::T_O + half * C::HALF, o);
                tmem_st_wait();
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(&p_ready[x]));
        }
        // ---- epilogue ----
        if (ok) ok = mbar_wait(smem_u32(&o_ready[(n_tiles - 1) & 1]), ((n_tiles - 1) >> 1) & 1, p.status);
#pragma unroll
        for (int k = 0; k < C::K_ITEMS; ++k) {
            const int r = 2 * C::NSW * k + 2 * warp + lane / 16;
#pragma unroll
            for (int m = 8; m >= 1; m /= 2) lsum[k] += __shfl_xor_sync(0xffffffffu, lsum[k], m);  // the row sum
            if (c8 == 0) {
                l_buf[r] = lsum[k];
                m_buf[r] = m_ref[k];
            }
        }
        named_barrier(1, 32 * C::NSW);
        if (!ok) {
            s_abort = 1;
        } else {
            tc_fence_after();
            uint32_t o[C::HALF];
            tmem_ld_cols<C::HALF>(tmem + lane_base + C::T_O + half * C::HALF, o);
            tmem_ld_wait();
#pragma unroll
            for (int rr = 0; rr < C::HALF; ++rr) {
                const int r = half * C::HALF + rr;
                const int hh = r / p.s_q, t = r % p.s_q;
                const int n_t = p.causal ? L - p.s_q + t + 1 : L;
                if (kbeg >= n_t) continue;  // no keys of this row in this split
                const int nsp = cdiv(n_t, p.split_tokens);
                const size_t orow = ((size_t)b * p.h_q + grp * HPG + hh) * p.s_q + t;
                const float l = l_buf[r];
                const float ov = __uint_as_float(o[rr]) / l;
                const float lse2 = m_buf[r] + log2f(l);
                if (nsp == 1) {
                    p.out[orow * 128 + tid] = __float2bfloat16_rn(ov);
                    if (p.lse && tid == 0) p.lse[orow] = lse2 * 0.69314718055994530942f;
                } else {
                    p.part_o[(orow * p.nsplit + split) * 128 + tid] = ov;
                    if (tid == 0) p.part_lse[orow * p.nsplit + split] = lse2;
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == C::NSW + 1) tmem_dealloc(tmem, 128);
}

cudaError_t expanded_attn_launch(const CUtensorMap& qc, const CUtensorMap& qr, const CUtensorMap& kc,
                                 const CUtensorMap& kr, const CUtensorMap& vc, const ExpParams& p, cudaStream_t st) {
    dim3 grid(p.nsplit, p.g, p.B);
    cudaError_t e;
    TimedLaunch timer(st);
    if (p.s_q == 1) {
        e = cudaFuncSetAttribute(expanded_attn_kernel<16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 ExpCfg<16>::SMEM);
        if (e != cudaSuccess) return e;
        expanded_attn_kernel<16><<<grid, ExpCfg<16>::NTHREADS, ExpCfg<16>::SMEM, st>>>(qc, qr, kc, kr, vc, p);
    } else {
        e = cudaFuncSetAttribute(expanded_attn_kernel<32>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 ExpCfg<32>::SMEM);
        if (e != cudaSuccess) return e;
        expanded_attn_kernel<32><<<grid, ExpCfg<32>::NTHREADS, ExpCfg<32>::SMEM, st>>>(qc, qr, kc, kr, vc, p);
    }
    timer.stop();
    return cudaPeekAtLastError();
}

}  // namespace lka

using namespace lka;

namespace {
struct ExpPlan {
    int split_tokens, nsplit;
    size_t off_lse, off_o, ws_bytes;
};
lka_status_t exp_plan(int B, int h_q, int g, int s_q, int d_h, int d_r, int Lmax, ExpPlan* pl, bool paged = false) {
    if (B < 0 || h_q < 1 || g < 1 || s_q < 1 || d_h < 1 || d_r < 0 || Lmax < 1) return LKA_ERR_INVALID_ARG;
    if (h_q % g) return LKA_ERR_INVALID_ARG;
    if (h_q / g != 16 || d_h != 128 || d_r != 64 || s_q > 2) return LKA_ERR_UNSUPPORTED;
    if ((!paged && (long long)B * g * Lmax >= (1ll << 31)) || B > 65535 || g > 65535) return LKA_ERR_UNSUPPORTED;
    int st = split_tokens_knob();
    if (st <= 0) {
        const long long units = (long long)(B > 0 ? B : 1) * g;
        long long nsp = (6LL * sm_count() + units - 1) / units;
        if (nsp < 1) nsp = 1;
        st = (int)((Lmax + nsp - 1) / nsp);
        if (st < 512) st = 512;
    }
    st = cdiv(st, 128) * 128;
    pl->split_tokens = st;
    pl->nsplit = cdiv(Lmax, st);
    WsCarve c;
    const size_t rows = (size_t)B * h_q * s_q;
    if (pl->nsplit > 1) {
        pl->off_lse = c.take(rows * pl->nsplit * 4);
        pl->off_o = c.take(rows * pl->nsplit * (size_t)d_h * 4);
    } else {
        pl->off_lse = pl->off_o = 0;
    }
    pl->ws_bytes = c.off;
    return LKA_OK;
}
}  // namespace

extern "C" {

// Whether a call of the per-group path runs the tensor-core prefill (d_h = 128, d_h^R = 64, many queries).
static bool exp_tc_prefill(int d_h, int d_r, int s_q) {
    return d_h == 128 && d_r == 64 && s_q >= kExpPrefillMinQueries;
}

size_t latent_expand_gqa_attn_workspace_size(int B, int h_q, int g, int s_q, int d_h, int d_r, int Lmax) {
    if (exp_tc_prefill(d_h, d_r, s_q)) {
        if (B < 0 || h_q < 1 || g < 1 || Lmax < 1 || h_q % g) return 0;
        return expanded_prefill_ws_bytes(B, h_q, s_q, Lmax);
    }
    ExpPlan pl;
    return exp_plan(B, h_q, g, s_q, d_h, d_r, Lmax, &pl) == LKA_OK ? pl.ws_bytes : 0;
}

}  // extern "C"

namespace {
struct ExpPages {
    const int32_t* block_table;
    int page_size, max_pages, num_pages;
};

static lka_status_t expanded_run(const void* q_c, const void* q_r, const void* kc, const void* vc, const void* kr,
                                 const int32_t* cache_lens, void* out, float* lse, int B, int h_q, int g, int s_q,
                                 int d_h, int d_r, int Lmax, int causal, float scale, lka_dtype_t dtype, void* ws,
                                 size_t ws_bytes, void* stream, const ExpPages* pg) {
    if (dtype != LKA_BF16) return LKA_ERR_UNSUPPORTED;
    if (exp_tc_prefill(d_h, d_r, s_q)) {
        // prefill (GQLA section 1: MHA-like, compute-bound) on the tensor-core prefill kernel
        if (B < 0 || h_q < 1 || g < 1 || Lmax < 1 || h_q % g) return LKA_ERR_INVALID_ARG;
        if (!pg && (long long)B * g * Lmax >= (1ll << 31)) return LKA_ERR_UNSUPPORTED;
        if (B == 0) return LKA_OK;
        const void* ptrs[] = {q_c, q_r, kc, vc, kr, cache_lens, out};
        for (const void* ptr : ptrs)
            if (!ptr || !aligned16(ptr)) return LKA_ERR_INVALID_ARG;
        if (!isfinite(scale)) return LKA_ERR_INVALID_ARG;
        if (ws && !aligned16(ws)) return LKA_ERR_INVALID_ARG;
        return expanded_prefill_tc(q_c, q_r, kc, vc, kr, cache_lens, out, lse, B, h_q, g, s_q, Lmax, causal, scale,
                                   ws, ws_bytes, (cudaStream_t)stream, pg ? pg->block_table : nullptr,
                                   pg ? pg->page_size : 0, pg ? pg->max_pages : 0, pg ? pg->num_pages : 0);
    }
    ExpPlan pl;
    lka_status_t s = exp_plan(B, h_q, g, s_q, d_h, d_r, Lmax, &pl, pg != nullptr);
    if (s != LKA_OK) return s;
    if (B == 0) return LKA_OK;
    const void* ptrs[] = {q_c, q_r, kc, vc, kr, cache_lens, out};
    for (const void* ptr : ptrs)
        if (!ptr || !aligned16(ptr)) return LKA_ERR_INVALID_ARG;
    if (!isfinite(scale)) return LKA_ERR_INVALID_ARG;
    if (!ws || ws_bytes < pl.ws_bytes) return LKA_ERR_WORKSPACE;
    if (!aligned16(ws)) return LKA_ERR_INVALID_ARG;
    const auto BF = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    const int NR = 16 * s_q;
    CUtensorMap t_qc, t_qr, t_kc, t_kr, t_vc;
    // cache rows: per sequence (contiguous) or per page (paged); boxes are a whole 128-token tile or a page piece
    const uint64_t seqs = pg ? (uint64_t)pg->num_pages : (uint64_t)B;
    const int rows_per = pg ? pg->page_size : Lmax;
    const uint32_t box_rows = pg && pg->page_size < 128 ? (uint32_t)pg->page_size : 128u;
    if (!make_tmap_2d(&t_qc, BF, q_c, d_h, (uint64_t)B * h_q * s_q, (uint64_t)d_h * 2, 64, NR) ||
        !make_tmap_2d(&t_qr, BF, q_r, d_r, (uint64_t)B * h_q * s_q, (uint64_t)d_r * 2, 64, NR) ||
        !make_tmap_2d(&t_kc, BF, kc, d_h, seqs * g * rows_per, (uint64_t)d_h * 2, 64, box_rows) ||
        !make_tmap_2d(&t_kr, BF, kr, d_r, seqs * rows_per, (uint64_t)d_r * 2, 64, box_rows) ||
        !make_tmap_2d(&t_vc, BF, vc, d_h, seqs * g * rows_per, (uint64_t)d_h * 2, 64, box_rows))
        return LKA_ERR_CUDA;
    uint8_t* w = static_cast<uint8_t*>(ws);
    ExpParams p{};
    p.lens = cache_lens;
    p.out = static_cast<__nv_bfloat16*>(out);
    p.lse = lse;
    p.part_o = pl.nsplit > 1 ? reinterpret_cast<float*>(w + pl.off_o) : nullptr;
    p.part_lse = pl.nsplit > 1 ? reinterpret_cast<float*>(w + pl.off_lse) : nullptr;
    p.status = reinterpret_cast<uint32_t*>(w);
    p.B = B;
    p.h_q = h_q;
    p.g = g;
    p.s_q = s_q;
    p.Lmax = Lmax;
    p.causal = causal ? 1 : 0;
    p.scale_log2 = scale * 1.4426950408889634f;
    p.split_tokens = pl.split_tokens;
    p.nsplit = pl.nsplit;
    p.block_table = pg ? pg->block_table : nullptr;
    p.page_size = pg ? pg->page_size : 0;
    p.max_pages = pg ? pg->max_pages : 0;
    p.num_pages = pg ? pg->num_pages : 0;
    p.box_rows = (int)box_rows;
    cudaStream_t st = (cudaStream_t)stream;
    if (expanded_attn_launch(t_qc, t_qr, t_kc, t_kr, t_vc, p, st) != cudaSuccess) return LKA_ERR_CUDA;
    if (pl.nsplit > 1) {
        GqaParams gp{};
        gp.out = out;
        gp.lse = lse;
        gp.lens = cache_lens;
        gp.part_o = p.part_o;
        gp.part_lse = p.part_lse;
        gp.status = p.status;
        gp.B = B;
        gp.h_q = h_q;
        gp.h_kv = g;
        gp.s_q = s_q;
        gp.Lmax = Lmax;
        gp.causal = p.causal;
        gp.split_tokens = pl.split_tokens;
        gp.nsplit_max = pl.nsplit;
        if (gqa_combine_launch(gp, 2, d_h, st) != cudaSuccess) return LKA_ERR_CUDA;
    }
    return LKA_OK;
}


}  // namespace

extern "C" {

lka_status_t latent_expand_gqa_attn(const void* q_c, const void* q_r, const void* kc, const void* vc, const void* kr,
                                    const int32_t* cache_lens, void* out, float* lse, int B, int h_q, int g, int s_q,
                                    int d_h, int d_r, int Lmax, int causal, float scale, lka_dtype_t dtype, void* ws,
                                    size_t ws_bytes, void* stream) {
    return expanded_run(q_c, q_r, kc, vc, kr, cache_lens, out, lse, B, h_q, g, s_q, d_h, d_r, Lmax, causal, scale,
                        dtype, ws, ws_bytes, stream, nullptr);
}

size_t latent_expand_gqa_attn_paged_workspace_size(int B, int h_q, int g, int s_q, int d_h, int d_r, int page_size,
                                                   int max_pages) {
    if (page_size < 8 || (page_size & (page_size - 1)) || max_pages < 1 ||
        (long long)page_size * max_pages >= (1ll << 31))
        return 0;
    if (exp_tc_prefill(d_h, d_r, s_q)) {
        if (B < 0 || h_q < 1 || g < 1 || h_q % g) return 0;
        return expanded_prefill_ws_bytes(B, h_q, s_q, page_size * max_pages);
    }
    ExpPlan pl;
    return exp_plan(B, h_q, g, s_q, d_h, d_r, page_size * max_pages, &pl, true) == LKA_OK ? pl.ws_bytes : 0;
}

lka_status_t latent_expand_gqa_attn_paged(const void* q_c, const void* q_r, const void* kc_pages,
                                          const void* vc_pages, const void* kr_pages, const int32_t* block_table,
                                          const int32_t* cache_lens, void* out, float* lse, int B, int h_q, int g,
                                          int s_q, int d_h, int d_r, int page_size, int max_pages, int num_pages,
                                          int causal, float scale, lka_dtype_t dtype, void* ws, size_t ws_bytes,
                                          void* stream) {
    if (page_size < 8 || (page_size & (page_size - 1)) || max_pages < 1 || num_pages < 1 || g < 1)
        return LKA_ERR_INVALID_ARG;
    if ((long long)page_size * max_pages >= (1ll << 31) || (long long)num_pages * g * page_size >= (1ll << 31))
        return LKA_ERR_UNSUPPORTED;
    if (B > 0 && (!block_table || (reinterpret_cast<uintptr_t>(block_table) & 3u))) return LKA_ERR_INVALID_ARG;
    const ExpPages pg{block_table, page_size, max_pages, num_pages};
    return expanded_run(q_c, q_r, kc_pages, vc_pages, kr_pages, cache_lens, out, lse, B, h_q, g, s_q, d_h, d_r,
                        page_size * max_pages, causal, scale, dtype, ws, ws_bytes, stream, &pg);
}

}  // extern "C"
