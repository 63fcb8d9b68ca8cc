// latent_attn.cu -- MQA-absorbed attention over the GQLA/MLA latent cache on
// the 5th-generation tensor cores, and the merge of its split partials.
//
// Operation ("GQLA: Group-Query Latent Attention ..." section 1, section 3.1
// eq. (1) and Figure 2(b)): after W^UK is folded into the query, all h_q = 128
// heads attend to the cached latent itself.  The key of token j is the
// 576-value row [c_j ; k^R_j] (r_kv = 512 latent values and the shared d_h^R =
// 64 RoPE key); the value is its first 512 values.  For query row (head) h:
//     s_j = scale * <[q~_h ; q^R_h], [c_j ; k^R_j]>,  o~_h = sum_j softmax(s)_j c_j.
// The 128 x 576 x tokens score contraction and the 128 x tokens x 512 value
// contraction are dense, so both run as tcgen05 MMAs with M = 128 heads.
//
// Tensor memory holds 512 fp32 columns per SM and the output alone needs
// 128 x 512, so each work item is processed by a CLUSTER OF TWO CTAs: rank r
// accumulates output columns [256 r, 256 r + 256) and computes the split-K
// partial of the scores over key values [288 r, 288 r + 288).  For that it
// loads latent values [256 r, 256 r + 320) of every token (rank 0: [0, 320),
// rank 1: [256, 576), i.e. its 256 value columns plus the rest of its score
// range; the 64 values [256, 320) are read by both ranks, the second read
// coming from L2).  The two score partials are exchanged through distributed
// shared memory, each rank sending its partial multiplied by scale * log2 e
// and rounded to fp16 (half the shared-memory and DSMEM bytes of fp32): a rank
// adds the peer's rounded partial to its own fp32 one, so the two ranks' scores
// differ by that rounding (at most 2^-11 of the peer's scaled partial) and each
// normalises its half of the output with its own row sums.  The rounding is
// absolute in the score, so it grows with the partial's magnitude (a scaled
// partial of 20 moves by at most 0.01).  A scaled partial beyond the fp16
// range (|x| > 65504, a softmax that is one-hot many times over) is saturated
// and raises kDevRange in the status word (LKA_ERR_RANGE): the output stays
// finite but is not accurate.
//
// Each tcgen05.mma with M = 128 and K = 16 takes about the same time whatever
// its N (up to 256), so the tiles are as wide as memory allows: 64 tokens.  The
// query slice lives in tensor memory (the A operand of the score MMA), which
// leaves shared memory to a 4-stage TMA ring, one exchange buffer and an
// outbox: a partial is written to the outbox and sent with one bulk copy per
// block (the copy engine moves it; the warp does not wait for the transfer).
// Sender warps load each partial from tensor memory as soon as it is computed
// and send it; the softmax warps load their own copy of tile i+1 before they
// work on tile i, and the score MMA runs two tiles ahead of P*V, so the
// exchange overlaps the softmax of the previous tile.
//
// Per CTA: warp 8 streams 64-token tiles of the latent through the ring; warp 9
// issues the score MMAs (S = Q K^T into the TMEM score tile) and, with a bf16
// cache, warp 14 the P*V MMAs (O += P V with P read from TMEM; with an FP8
// cache warp 9 issues both); warps 10-13 (one per TMEM lane quarter) send the
// score partials;
// warps 0-7 write the query slice to TMEM once, then per tile add the peer's
// partial to their own, mask and run the online softmax, two warps per group
// of 32 head rows (warps w and w + 4 take the two 32-token halves of the tile
// and swap their row maxima through two spare TMEM columns), with lazy
// rescaling (the running maximum is only moved when it grows by more than 2^8,
// which leaves the final O / l exact); P is written back to TMEM as bf16.
#include <cuda_fp16.h>
#include <cuda_fp8.h>

#include "common.cuh"
#include "host_util.h"
#include "latent.h"
#include "tc.cuh"

namespace lka {

// f16 operands (FP8 cache: the widened cache, the query and P): instruction descriptor of kind::f16 with
// A = B = f16 (format 0), D = fp32, dense, and the f16 pair packing
__host__ __device__ constexpr uint32_t idesc_f16_f32(int M, int N, bool a_mn, bool b_mn) {
    return (1u << 4)                      // D format fp32
           | ((a_mn ? 1u : 0u) << 15)     // A major
           | ((b_mn ? 1u : 0u) << 16)     // B major
           | ((uint32_t)(N >> 3) << 17)   // N / 8
           | ((uint32_t)(M >> 4) << 24);  // M / 16
}
__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi) {
    __half2 v = __floats2half2_rn(lo, hi);  // .x = lo (low 16 bits), .y = hi
    return *reinterpret_cast<uint32_t*>(&v);
}

namespace lat {
constexpr int NT = 64;          // tokens per tile (the N of the score MMA)
constexpr int NST = 4;          // TMA ring depth
constexpr int PF = 6;           // L2 prefetch distance in tiles
constexpr int NKB = 5;          // 64-value boxes per rank and tile
constexpr int KSTEPS = 18;      // K = 16 steps of this rank's 288 score values
constexpr int BOX = NT * 128;   // one 64-value box of NT tokens
constexpr int BOX8 = NT * 64;   // the same box of e4m3 values (FP8 cache), landing in the upper half of a stage
constexpr int STAGE = NKB * BOX;
constexpr int NSW = 8;          // softmax warps: 4 lane quarters x 2 column halves
constexpr int NXW = 4;          // sender warps: one per lane quarter
constexpr int NCW = 2;          // converter warps (FP8 cache only)
constexpr int CW = NT / 2;      // score columns per softmax warp
constexpr int NTHREADS = 32 * (NSW + 2 + NXW);
constexpr int NTHREADS_F8 = NTHREADS + 32 * NCW;
// bf16 cache: one more warp, which issues the P*V MMAs, so that the score chain (waiting for key tiles and a
// free score buffer) and the P*V chain (waiting for P) do not hold each other up in one issuing thread.  (The
// FP8 instance, with its converter warps, keeps one issuer: 17 warps would not fit 128 registers a thread.)
constexpr int PV_WARP = NSW + 2 + NXW;
constexpr int NTHREADS_BF = NTHREADS + 32;
constexpr int XROW = CW * 2;    // bytes of one row of one half of an exchanged partial (fp16)
constexpr int XBUF = 2 * 128 * XROW;  // [half][head row][CW] fp16; each warp's block is contiguous
constexpr int XSPACE = 2 * XBUF;      // room reserved for each of the exchange buffer and the outbox
constexpr int OFF_KV = 0;
constexpr int OFF_X = OFF_KV + NST * STAGE;
constexpr int OFF_OUT = OFF_X + XSPACE;  // this CTA's partial on its way to the peer
constexpr int OFF_BAR = OFF_OUT + XSPACE;
// The query slice is staged once through shared memory that is idle at the start: the last ring
// stage, the exchange buffer and the first part of the outbox (five 128-row x 64-value boxes).
constexpr int NQB = 5;
constexpr int QBOX = 128 * 128;
constexpr int OFF_QST = OFF_KV + (NST - 1) * STAGE;
static_assert(OFF_QST % 1024 == 0 && OFF_QST + NQB * QBOX <= OFF_BAR, "query staging area");
constexpr int SMEM = 1024 + OFF_BAR + 512;
static_assert(SMEM <= 232448, "shared memory budget");
// tensor memory columns
constexpr uint32_t T_O = 0;          // 256 fp32 columns: this rank's half of the output
constexpr uint32_t T_Q = 256;        // 144 columns: this rank's 288 query values as bf16 pairs
constexpr uint32_t T_P = 400;        // NT/2 columns of bf16 pairs
constexpr uint32_t T_R = 432;        // 6 columns: row maxima (2 tiles x 2 halves) and row sums of the warp pairs
constexpr uint32_t T_S = 448;        // NT fp32 score partials
static_assert(T_Q + KSTEPS * 8 <= T_P && T_P + NT / 2 <= T_R && T_R + 6 <= T_S && T_S + NT <= 512,
              "tensor memory budget");
constexpr float RESCALE_THRESHOLD = 8.0f;  // log2 domain
constexpr float kF16Max = 65504.f;         // largest finite fp16 value
}  // namespace lat

__device__ __forceinline__ uint32_t cluster_rank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
__device__ __forceinline__ uint32_t mapa_peer(uint32_t saddr, uint32_t peer) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(saddr), "r"(peer));
    return r;
}
__device__ __forceinline__ void cluster_sync() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// Bulk copy of `bytes` from this CTA's shared memory to the peer's (cluster address `dst`),
// completing `bytes` of the transaction count of the peer's barrier `rbar`.
__device__ __forceinline__ void bulk_copy_to_peer(uint32_t dst, uint32_t src, uint32_t bytes, uint32_t rbar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.shared::cta.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
        "r"(src), "r"(bytes), "r"(rbar)
        : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// Wait until the bulk copies this thread committed have finished reading their sources.
__device__ __forceinline__ void bulk_wait_read() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
// Wait until they have completed entirely.
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }
// Arrival on the peer's "buffer free" barrier.  Relaxed: it only follows local shared-memory
// loads whose values have already been consumed, and a release fence here would also wait for
// this thread's outstanding remote stores.
__device__ __forceinline__ void remote_arrive(uint32_t rbar) {
    asm volatile("mbarrier.arrive.relaxed.cluster.shared::cluster.b64 _, [%0];" ::"r"(rbar) : "memory");
}
// Waits on the exchange barriers use the default (CTA-scope) acquire: the peer's partial scores
// arrive through bulk copies, whose bytes complete the local barrier's transaction count, and the
// peer's "buffer free" arrival (release at cluster scope) is only ever followed by new remote
// copies, never by reads of data the peer produced.

// 15 warps (16 with an FP8 cache): an SM sub-partition holds up to 4 of them, so at most
// 16384 / (4 * 32) = 128 registers each
template <bool F8>
__global__ void __cluster_dims__(2, 1, 1) __maxnreg__(128)
    latent_attn_kernel(const __grid_constant__ CUtensorMap tm_lat, const __grid_constant__ CUtensorMap tm_qt,
                       const __grid_constant__ CUtensorMap tm_qr, const LatentParams p) {
    using namespace lat;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(align_up(reinterpret_cast<uintptr_t>(smem_raw), 1024));
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + OFF_BAR);
    uint64_t* q_full = bars + 0;          // the query slice is in tensor memory (all softmax warps arrived)
    uint64_t* q_loaded = bars + 1;        // the query slice is in shared memory
    uint64_t* kv_full = bars + 2;
    uint64_t* kv_empty = kv_full + NST;
    uint64_t* s_ready = kv_empty + NST;   // QK(j) done
    uint64_t* s_free = s_ready + 1;       // S(j) loaded by all softmax and sender warps
    uint64_t* p_ready = s_free + 1;       // P(j) written by all softmax warps
    uint64_t* o_ready = p_ready + 1;      // PV(j) done
    uint64_t* xfull = o_ready + 1;        // [NSW] the peer's partial of warp w's block arrived
    uint64_t* xempty = xfull + NSW;       // [NSW] the peer has consumed this CTA's partial of warp w's block
    uint64_t* conv_full = xempty + NSW;   // [NST] FP8 cache: the stage has been widened to bf16
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(conv_full + NST);
    __shared__ int s_abort;
    __shared__ int s_conv_bad;  // FP8 cache: a converter thread gave up waiting (read by all converters)

    const uint32_t rank = cluster_rank();
    const uint32_t peer = rank ^ 1u;
    const int pair = blockIdx.x >> 1;
    const int t = pair % p.s_q;
    const int split = pair / p.s_q;
    const int b = blockIdx.y;
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;

    const int L = clamp_len(p.lens, b, p.Lmax, p.s_q, p.causal, p.status,
                            threadIdx.x == 0 && rank == 0 && pair == 0);
    const int last_key = p.causal ? L - p.s_q + t : L - 1;  // last key query t may see
    const int kbeg = split * p.split_tokens;
    const int kend = min(last_key + 1, kbeg + p.split_tokens);
    const int n_tiles = kend > kbeg ? cdiv(kend - kbeg, NT) : 0;

    if (threadIdx.x == 0) {
        s_abort = 0;
        s_conv_bad = 0;
        mbar_init(smem_u32(q_full), NSW);
        mbar_init(smem_u32(q_loaded), 1);
        for (int s = 0; s < NST; ++s) {
            mbar_init(smem_u32(&kv_full[s]), 1);
            mbar_init(smem_u32(&kv_empty[s]), 1);
        }
        mbar_init(smem_u32(s_ready), 1);
        mbar_init(smem_u32(s_free), NSW + NXW);
        mbar_init(smem_u32(p_ready), NSW);
        mbar_init(smem_u32(o_ready), 1);
        for (int i = 0; i < NSW; ++i) {
            mbar_init(smem_u32(&xfull[i]), 1);
            mbar_init(smem_u32(&xempty[i]), 1);
        }
        for (int s = 0; s < NST; ++s) mbar_init(smem_u32(&conv_full[s]), NCW);
        fence_barrier_init();
        // the exchange buffer starts open for the peer's partial scores
        for (int i = 0; i < NSW; ++i) mbar_arrive_expect_tx(smem_u32(&xfull[i]), XBUF / NSW);
    }
    if (warp == NSW + 1) {
        tmem_alloc(tmem_slot, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    cluster_sync();  // barriers of both CTAs initialised before any remote traffic
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (n_tiles > 0 && warp == NSW) {
        // ------------------------------- TMA producer -------------------------------
        if (lane == 0) {
            prefetch_tensormap(&tm_lat);
            // this rank's 288 values of the 128 query rows [q~ ; q^R] of (b, t): rank 0 q~[0:320) (the
            // last 32 unused), rank 1 q~[288:544) (the last 32 past the row: zero fill) and q^R[0:64)
            {
                const uint32_t qb = smem_u32(q_loaded);
                mbar_arrive_expect_tx(qb, NQB * QBOX);
                const int qrow = (b * p.s_q + t) * 128;
                const uint32_t qdst = smem_u32(smem + OFF_QST);
                for (int k = 0; k < (rank ? NQB - 1 : NQB); ++k)
                    tma_load_2d(qdst + k * QBOX, &tm_qt, (int)rank * 288 + k * 64, qrow, qb);
                if (rank) tma_load_3d(qdst + (NQB - 1) * QBOX, &tm_qr, 0, t, b * 128, qb);
            }
            // tiles PF ahead of the one being loaded are prefetched into L2, so that the ring (whose
            // stages stay busy until P*V) is refilled from L2 rather than from DRAM
            // row of token `tok` of this sequence in the cache: contiguous [B][Lmax] slabs, or a page of the
            // block table ([num_pages][page_size] rows; entries outside the pool are replaced by page 0, which
            // is reported when the attention needs the token)
            auto cache_row = [&](int tok) -> int {
                if (!p.block_table) return b * p.Lmax + tok;
                int page = 0;
                const int j = tok / p.page_size;
                if (j < p.max_pages) {
                    page = p.block_table[(size_t)b * p.max_pages + j];
                    if (page < 0 || page >= p.num_pages) {
                        if (tok < kend) atomicOr(p.status, kDevBadPage);
                        page = 0;
                    }
                }
                return page * p.page_size + tok % p.page_size;
            };
            auto prefetch = [&](int i) {
                for (int r0 = 0; r0 < NT; r0 += p.box_rows) {
                    const int y = cache_row(kbeg + i * NT + r0);
                    for (int kb = 0; kb < NKB; ++kb) tma_prefetch_2d(&tm_lat, (int)rank * 256 + kb * 64, y);  // bytes = values for e4m3
                }
            };
            for (int i = NST; i < min(n_tiles, PF); ++i) prefetch(i);
            int issued = 0;
            for (int i = 0; i < n_tiles; ++i) {
                const int s = i % NST;
                if (i >= NST && !mbar_wait(smem_u32(&kv_empty[s]), ((i / NST) - 1) & 1, p.status)) {
                    s_abort = 1;
                    break;
                }
                if (*(volatile int*)&s_abort) break;
                // the last stage holds part of the staged query until it is in tensor memory
                if (i == NST - 1 && !mbar_wait(smem_u32(q_full), 0, p.status)) {
                    s_abort = 1;
                    break;
                }
                const uint32_t fb = smem_u32(&kv_full[s]);
                mbar_arrive_expect_tx(fb, NKB * (F8 ? BOX8 : BOX));
                const uint32_t dst = smem_u32(smem + OFF_KV + s * STAGE) + (F8 ? STAGE / 2 : 0);
                for (int r0 = 0; r0 < NT; r0 += p.box_rows) {  // one box, or one per page piece of the tile
                    const int y = cache_row(kbeg + i * NT + r0);
                    for (int kb = 0; kb < NKB; ++kb) {
                        if (F8)
                            tma_load_2d(dst + kb * BOX8 + r0 * 64, &tm_lat, (int)rank * 256 + kb * 64, y, fb);
                        else
                            tma_load_2d(dst + kb * BOX + r0 * 128, &tm_lat, (int)rank * 256 + kb * 64, y, fb);
                    }
                }
                if (i + PF < n_tiles) prefetch(i + PF);
                ++issued;
            }
            for (int i = issued - 1; i >= 0 && i >= issued - NST; --i)
                mbar_wait(smem_u32(&kv_full[i % NST]), (i / NST) & 1, p.status);
        }
    } else if (n_tiles > 0 && warp == NSW + 1) {
        // ------------------------------- MMA issuer -------------------------------
        // Per step j: QK(j) once the softmax and sender warps have loaded S(j-1), then PV(j-2) once
        // P(j-2) is in tensor memory.  The softmax warps load S(j-1) before they compute P(j-2), so
        // QK(j) runs while tile j-2 is being finished.
        // an FP8 cache is widened to f16 (exact), and the query and P are f16 as well
        constexpr uint32_t idesc_qk = F8 ? idesc_f16_f32(128, NT, false, false) : idesc_bf16_f32(128, NT, false, false);
        constexpr uint32_t idesc_pv = F8 ? idesc_f16_f32(128, 256, false, true) : idesc_bf16_f32(128, 256, false, true);
        bool ok = mbar_wait(smem_u32(q_full), 0, p.status);
        for (int j = 0; ok && j < (F8 ? n_tiles + 2 : n_tiles); ++j) {
            if (j < n_tiles) {
                const int s = j % NST;
                if (!mbar_wait(smem_u32(F8 ? &conv_full[s] : &kv_full[s]), (j / NST) & 1, p.status)) break;
                uint8_t* st = smem + OFF_KV + s * STAGE;
                const int nvalid = min(NT, kend - (kbeg + j * NT));
                if (nvalid < NT) {
                    // rows past the last visible key may hold anything (even NaN): zero them so
                    // that P = 0 times V contributes exactly 0
                    const int rows = NT - nvalid;
                    for (int idx = lane; idx < NKB * rows * 8; idx += 32) {
                        const int kb = idx / (rows * 8), rr = (idx / 8) % rows, c = idx % 8;
                        *reinterpret_cast<uint4*>(st + kb * BOX + (nvalid + rr) * 128 + c * 16) =
                            make_uint4(0, 0, 0, 0);
                    }
                    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                    __syncwarp();
                }
                if (j >= 1 && !mbar_wait(smem_u32(s_free), (j - 1) & 1, p.status)) break;
                tc_fence_after();
                if (lane == 0) {
                    const uint32_t kva = smem_u32(st);
#pragma unroll
                    for (int ks = 0; ks < KSTEPS; ++ks) {
                        // score value 288 rank + 16 ks sits at offset 32 rank + 16 ks of this rank's tile
                        const int off = (int)rank * 32 + ks * 16;
                        umma_ts(tmem + T_S, tmem + T_Q + ks * 8,
                                smem_desc_sw128(kva + (off / 64) * BOX + (off % 64) * 2, 16, 1024), idesc_qk, ks != 0);
                    }
                    umma_commit(smem_u32(s_ready));
                }
                __syncwarp();
            }
            if (F8 && j >= 2) {
                const int i = j - 2;
                if (!mbar_wait(smem_u32(p_ready), i & 1, p.status)) break;
                tc_fence_after();
                if (lane == 0) {
                    const uint32_t va = smem_u32(smem + OFF_KV + (i % NST) * STAGE);
#pragma unroll
                    for (int kk = 0; kk < NT / 16; ++kk)
                        umma_ts(tmem + T_O, tmem + T_P + kk * 8, smem_desc_sw128(va + kk * 2048, BOX, 1024), idesc_pv,
                                (i | kk) != 0);
                    umma_commit(smem_u32(&kv_empty[i % NST]));
                    umma_commit(smem_u32(o_ready));
                }
                __syncwarp();
            }
        }
    } else if (!F8 && n_tiles > 0 && warp == PV_WARP) {
        // ----------------------------- P*V MMA issuer (bf16) -----------------------------
        // O += P(i) V(i) once P(i) is in tensor memory; the stage was zeroed past the last key before the score
        // MMA of the tile, and its commit to kv_empty releases it (this chain reads it last).  The commits track
        // this thread's MMAs only.
        constexpr uint32_t idesc_pv = idesc_bf16_f32(128, 256, false, true);
        for (int i = 0; i < n_tiles; ++i) {
            if (!mbar_wait(smem_u32(p_ready), i & 1, p.status)) break;
            tc_fence_after();
            if (lane == 0) {
                const uint32_t va = smem_u32(smem + OFF_KV + (i % NST) * STAGE);
#pragma unroll
                for (int kk = 0; kk < NT / 16; ++kk)
                    umma_ts(tmem + T_O, tmem + T_P + kk * 8, smem_desc_sw128(va + kk * 2048, BOX, 1024), idesc_pv,
                            (i | kk) != 0);
                umma_commit(smem_u32(&kv_empty[i % NST]));
                umma_commit(smem_u32(o_ready));
            }
            __syncwarp();
        }
    } else if (F8 && n_tiles > 0 && warp >= NSW + 2 + NXW) {
        // ------------------------------ converter warps ------------------------------
        // FP8 cache: a tile lands as e4m3 in the upper half of its stage (five boxes of NT rows x 64
        // bytes); the two converter warps widen it in place to the five f16 boxes (NT rows x 128 bytes,
        // 128-byte swizzle) the MMAs read.  e4m3 -> f16 is exact: every e4m3 value is an f16 value.  Box k
        // of the result overlaps only source boxes below k, or (k = 4) its own source: each source box is
        // read into registers and all 64 threads meet at a barrier before its result is written.
        // A thread that gives up waiting for a tile sets s_conv_bad before the first barrier of the tile, and all
        // 64 threads leave together after it, so that no barrier is left with a missing thread.
        const int ct = threadIdx.x - 32 * (NSW + 2 + NXW);  // 0 .. 63
        bool bad = false;
        for (int j = 0; !bad && j < n_tiles; ++j) {
            const int s = j % NST;
            if (!mbar_wait(smem_u32(&kv_full[s]), (j / NST) & 1, p.status)) s_conv_bad = 1;
            uint8_t* st = smem + OFF_KV + s * STAGE;
            const uint8_t* src = st + STAGE / 2;
#pragma unroll 1
            for (int k = 0; k < NKB; ++k) {
                constexpr int PER = BOX8 / 16 / 64;  // 16-byte source chunks per thread and box
                uint4 v[PER];
#pragma unroll
                for (int u = 0; u < PER; ++u) v[u] = *reinterpret_cast<const uint4*>(src + k * BOX8 + (ct + 64 * u) * 16);
                named_barrier(5, 64);
                if (k == 0 && *(volatile int*)&s_conv_bad) {
                    bad = true;
                    break;
                }
#pragma unroll
                for (int u = 0; u < PER; ++u) {
                    const int c = ct + 64 * u;        // chunk of the source box: 4 per 64-byte row
                    const int r = c >> 2, q = c & 3;  // token row, group of 16 values in the row
                    const uint32_t ws[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
                    uint32_t w[8];
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const __half2_raw lo =
                            __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(ws[i] & 0xffffu), __NV_E4M3);
                        const __half2_raw hi =
                            __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(ws[i] >> 16), __NV_E4M3);
                        w[2 * i] = (uint32_t)lo.x | ((uint32_t)lo.y << 16);
                        w[2 * i + 1] = (uint32_t)hi.x | ((uint32_t)hi.y << 16);
                    }
                    uint8_t* drow = st + k * BOX + r * 128;
                    *reinterpret_cast<uint4*>(drow + (((2 * q) ^ (r & 7)) << 4)) = make_uint4(w[0], w[1], w[2], w[3]);
                    *reinterpret_cast<uint4*>(drow + (((2 * q + 1) ^ (r & 7)) << 4)) =
                        make_uint4(w[4], w[5], w[6], w[7]);
                }
            }
            if (bad) break;
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // visible to the tensor cores
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(&conv_full[s]));
        }
        if (bad) s_abort = 1;
    } else if (n_tiles > 0 && warp >= NSW + 2 && warp < NSW + 2 + NXW) {
        // ------------------------------- sender warps -------------------------------
        // Sender warp q (= warp % 4) owns TMEM lane quarter q (head rows 32q .. +31): per tile it loads
        // this rank's partial scores of all NT columns from tensor memory, writes them to the outbox and
        // sends the two 32-column blocks of the quarter to the peer's exchange buffer once the peer's
        // softmax warps have consumed the previous tile there.  The softmax warps only wait for what
        // the peer sent; the sending (outbox store, proxy fence, waits, copies) is off their path.
        const int qx = warp & 3;
        const uint32_t lane_base = (uint32_t)(qx * 32) << 16;
        const int sw = (lane >> 1) & 3;  // 16-byte chunk swizzle of a 64-byte row: 8 lanes hit 8 bank groups
        int xblk[2];
        uint32_t xrem[2], xfull_rem[2];
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
            xblk[hf] = hf * 128 * XROW + qx * 32 * XROW;  // the block of softmax warp 4 hf + q
            xrem[hf] = mapa_peer(smem_u32(smem + OFF_X + xblk[hf]), peer);
            xfull_rem[hf] = mapa_peer(smem_u32(&xfull[hf * 4 + qx]), peer);
        }
        uint32_t own[NT];
        bool ok = mbar_wait(smem_u32(q_full), 0, p.status);  // the outbox holds part of the staged query
        for (int j = 0; ok && j < n_tiles; ++j) {
            ok = mbar_wait(smem_u32(s_ready), j & 1, p.status);
            tc_fence_after();
#pragma unroll
            for (int c0 = 0; c0 < NT; c0 += 16) tmem_ld16(tmem + lane_base + T_S + c0, own + c0);
            tmem_ld_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(s_free));
            if (lane == 0) bulk_wait_read();  // the previous copies have read the outbox
            __syncwarp();
            // the partial goes out already scaled into the log2 domain (scale * log2 e), saturated to the
            // fp16 range; a partial beyond it (|scaled partial| > 65504) raises kDevRange
            float amax = 0.f;
#pragma unroll
            for (int hf = 0; hf < 2; ++hf) {
                uint8_t* orow = smem + OFF_OUT + xblk[hf] + lane * XROW;
#pragma unroll
                for (int c = 0; c < CW / 8; ++c) {
                    const uint32_t* o8 = own + hf * CW + 8 * c;
                    uint32_t w4[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float y0 = __uint_as_float(o8[2 * e]) * p.scale_log2;
                        const float y1 = __uint_as_float(o8[2 * e + 1]) * p.scale_log2;
                        amax = fmaxf(amax, fmaxf(fabsf(y0), fabsf(y1)));
                        w4[e] = pack_f16x2(fminf(fmaxf(y0, -kF16Max), kF16Max), fminf(fmaxf(y1, -kF16Max), kF16Max));
                    }
                    *reinterpret_cast<uint4*>(orow + ((c ^ sw) << 4)) = make_uint4(w4[0], w4[1], w4[2], w4[3]);
                }
            }
            if (__any_sync(0xffffffffu, !(amax <= kF16Max)) && lane == 0) atomicOr(p.status, kDevRange);
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // visible to the copy engine
            __syncwarp();
            if (lane == 0) {
#pragma unroll
                for (int hf = 0; hf < 2; ++hf) {
                    // the peer's block is free once its softmax warps are done with the staged query
                    // (phase 0) and its softmax warp has consumed partial j-1 (phase j)
                    if (ok) ok = mbar_wait(smem_u32(&xempty[hf * 4 + qx]), j & 1, p.status);
                    if (ok) bulk_copy_to_peer(xrem[hf], smem_u32(smem + OFF_OUT + xblk[hf]), 32 * XROW, xfull_rem[hf]);
                }
                bulk_commit();
            }
            ok = __shfl_sync(0xffffffffu, ok, 0);
        }
        if (lane == 0) bulk_wait_all();
        if (!ok) s_abort = 1;
    } else if (warp < NSW) {
        // -------------------------------- softmax warps --------------------------------
        // Warp w owns head rows 32(w%4) .. +31 (its TMEM lane quarter) and score columns
        // [32(w/4), +32) of every tile, with its own exchange barriers; the two warps of a lane
        // quarter meet once per tile to combine their row maxima.
        const int qw = warp & 3, half = warp >> 2;
        const int h = qw * 32 + lane;  // head row == TMEM lane
        const uint32_t lane_base = (uint32_t)(qw * 32) << 16;
        const int col0 = half * CW;
        const int blk = half * 128 * XROW + qw * 32 * XROW;  // this warp's block in the exchange buffer
        // the peer's "buffer free" barrier of this warp's block
        const uint32_t xempty_rem = mapa_peer(smem_u32(&xempty[warp]), peer);
        const int sw = (lane >> 1) & 3;  // the sender's chunk swizzle
        float m_ref = -INFINITY, l = 0.f;
        bool ok = true;
        if (n_tiles > 0) {
            // this rank's 288 values of query row h, staged in shared memory -> tensor memory (A operand
            // of the score MMA, K-major: column c holds values 2c and 2c+1).  Nine 16-column chunks of
            // 32 values: the first warp of the lane quarter writes chunks 0-4, the second 5-8.
            if (ok) ok = mbar_wait(smem_u32(q_loaded), 0, p.status);
            for (int c0 = half * 5; c0 < (half ? KSTEPS / 2 : 5); ++c0) {
                const int v0 = c0 * 32;  // first value of the chunk within this rank's slice
                const bool rope = rank == 1 && v0 >= 224;
                const int box = rope ? NQB - 1 : v0 / 64, u0 = rope ? (v0 - 224) / 8 : (v0 % 64) / 8;
                const uint8_t* row = smem + OFF_QST + box * QBOX + h * 128;
                uint32_t w[16];
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const uint4 v = *reinterpret_cast<const uint4*>(row + (((u0 + q) ^ (h & 7)) << 4));
                    w[4 * q] = v.x;
                    w[4 * q + 1] = v.y;
                    w[4 * q + 2] = v.z;
                    w[4 * q + 3] = v.w;
                }
                if (F8) {
                    // FP8 cache: the dequantisation scale of the latent part (or of the RoPE key) goes into
                    // the query, which becomes f16 like the widened cache
                    const float qs = p.kv_scale[rope ? 1 : 0];
#pragma unroll
                    for (int e = 0; e < 16; ++e) {
                        const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[e]));
                        w[e] = pack_f16x2(f.x * qs, f.y * qs);
                    }
                }
                tmem_st16(tmem + lane_base + T_Q + c0 * 16, w);
            }
            tmem_st_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(q_full));
            // the staging area overlaps the exchange buffer: once every softmax warp of this CTA is done
            // with it, the peer may send its first partial (phase 0 of the buffer-free barrier)
            if (ok) ok = mbar_wait(smem_u32(q_full), 0, p.status);
            if (lane == 0) remote_arrive(xempty_rem);
        }
        uint32_t cur[CW];
        // this warp's block of this rank's partial of tile j into registers (the sender warps send it)
        auto fetch = [&](int j) {
            if (ok) ok = mbar_wait(smem_u32(s_ready), j & 1, p.status);
            tc_fence_after();
            tmem_ld16(tmem + lane_base + T_S + col0, cur);
            tmem_ld16(tmem + lane_base + T_S + col0 + 16, cur + 16);
            tmem_ld_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(s_free));
        };
        // combine a per-row value with the partner warp's through TMEM column T_R + col (+ 1 for
        // the partner's); both warps of the lane quarter call it with the same col
        auto swap_with_partner = [&](float v, uint32_t col) -> float {
            tmem_st1(tmem + lane_base + T_R + col + half, __float_as_uint(v));
            tmem_st_wait();
            tc_fence_before();
            named_barrier(1 + qw, 64);
            tc_fence_after();
            const uint32_t o = tmem_ld1(tmem + lane_base + T_R + col + (half ^ 1));
            tmem_ld_wait();
            return __uint_as_float(o);
        };
        if (n_tiles > 0) fetch(0);
        for (int i = 0; i < n_tiles; ++i) {
            // ---- the peer's partial of this block, added to this rank's ----
            if (ok) ok = mbar_wait(smem_u32(&xfull[warp]), i & 1, p.status);
            float s[CW];
            const uint8_t* xr = smem + OFF_X + blk + lane * XROW;
#pragma unroll
            for (int c = 0; c < CW / 8; ++c) {
                const uint4 v = *reinterpret_cast<const uint4*>(xr + ((c ^ sw) << 4));
                const uint32_t vw[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    // own partial scaled into the log2 domain plus the peer's (sent scaled)
                    const float2 pf = __half22float2(*reinterpret_cast<const __half2*>(&vw[k]));
                    const float2 a = __ffma2_rn(
                        make_float2(__uint_as_float(cur[8 * c + 2 * k]), __uint_as_float(cur[8 * c + 2 * k + 1])),
                        make_float2(p.scale_log2, p.scale_log2), pf);
                    s[8 * c + 2 * k] = a.x;
                    s[8 * c + 2 * k + 1] = a.y;
                }
            }
            __syncwarp();
            if (lane == 0 && i + 1 < n_tiles) {
                mbar_arrive_expect_tx(smem_u32(&xfull[warp]), XBUF / NSW);  // reopen for tile i + 1 ...
                remote_arrive(xempty_rem);                                   // ... and tell the peer
            }
            // ---- this rank's partial of tile i+1 (the score MMA may move on to tile i+2) ----
            if (i + 1 < n_tiles) fetch(i + 1);
            // ---- mask, online softmax ----
            const int k0 = kbeg + i * NT + col0;
            if (kbeg + (i + 1) * NT > kend) {
#pragma unroll
                for (int j = 0; j < CW; ++j) s[j] = (k0 + j < kend) ? s[j] : -INFINITY;
            }
            // row maximum of the whole tile: this warp's half and the partner warp's half
            float mx = tree_max<CW>(s);
            mx = fmaxf(mx, swap_with_partner(mx, 2u * (i & 1)));
            const float m_new = fmaxf(m_ref, mx);
            bool resc = false;
            float alpha = 1.f;
            float m_use = m_ref;
            if (m_ref == -INFINITY) {
                m_use = m_new;
            } else if (m_new > m_ref + RESCALE_THRESHOLD) {
                resc = true;
                alpha = fast_exp2(m_ref - m_new);
                m_use = m_new;
            }
            uint32_t pk[CW / 2];
            const float m_sub = m_use == -INFINITY ? 0.f : m_use;  // all scores -inf: p = 2^-inf = 0
            const float2 nm2 = make_float2(-m_sub, -m_sub);
#pragma unroll
            for (int j = 0; j < CW; j += 2) {
                const float2 v = __fadd2_rn(make_float2(s[j], s[j + 1]), nm2);
                s[j] = fast_exp2(v.x);
                s[j + 1] = fast_exp2(v.y);
                pk[j / 2] = F8 ? pack_f16x2(s[j], s[j + 1]) : pack_bf16x2(s[j], s[j + 1]);
            }
            const float rs = tree_sum<CW>(s);
            l = (resc ? l * alpha : l) + rs;  // this warp's share of the row sum
            m_ref = m_use;
            // PV(i-1) must be done: it reads the P buffer, and a rescale of O must follow its update
            if (ok && i >= 1) ok = mbar_wait(smem_u32(o_ready), (i - 1) & 1, p.status);
            tc_fence_after();
            if (__any_sync(0xffffffffu, resc)) {
                // each warp of the pair rescales half of this rank's 256 output columns
                for (int c0 = half * 128; c0 < half * 128 + 128; c0 += 16) {
                    uint32_t o[16];
                    tmem_ld16(tmem + lane_base + T_O + c0, o);
                    tmem_ld_wait();
#pragma unroll
                    for (int q = 0; q < 16; ++q) o[q] = __float_as_uint(__uint_as_float(o[q]) * alpha);
                    tmem_st16(tmem + lane_base + T_O + c0, o);
                }
            }
            tmem_st16(tmem + lane_base + T_P + half * (CW / 2), pk);
            tmem_st_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(p_ready));
        }
        if (!ok) s_abort = 1;
        // ---- epilogue: the full row sum, then normalise this warp's 128 output columns ----
        l += swap_with_partner(l, 4u);
        const int last = n_tiles - 1;
        if (ok && n_tiles > 0 && mbar_wait(smem_u32(o_ready), last & 1, p.status)) {
            tc_fence_after();
            // (FP8 cache: times the latent part's dequantisation scale, the value being the latent itself)
            const float inv_l = (l > 0.f ? 1.f / l : 0.f) * (F8 ? p.kv_scale[0] : 1.f);
            const int HPG = p.h_q / p.g;
            const int grp = h / HPG, hh = h % HPG;
            const size_t prow = ((size_t)(b * p.s_q + t) * p.h_q + h);
            __nv_bfloat16* orow =
                p.o_lat + ((size_t)grp * p.B * HPG * p.s_q + (size_t)(b * HPG + hh) * p.s_q + t) * 512 + rank * 256;
            float* prt = p.nsplit > 1 ? p.part_o + (prow * p.nsplit + split) * 512 + rank * 256 : nullptr;
            for (int c1 = half * 128; c1 < half * 128 + 128; c1 += 32) {
                uint32_t o2[32];  // two 16-column loads per wait
                tmem_ld16(tmem + lane_base + T_O + c1, o2);
                tmem_ld16(tmem + lane_base + T_O + c1 + 16, o2 + 16);
                tmem_ld_wait();
#pragma unroll
                for (int u = 0; u < 2; ++u) {
                    const int c0 = c1 + 16 * u;
                    const uint32_t* o = o2 + 16 * u;
                    if (prt) {
                        float4* d = reinterpret_cast<float4*>(prt + c0);
#pragma unroll
                        for (int q = 0; q < 4; ++q)
                            d[q] = make_float4(__uint_as_float(o[4 * q]) * inv_l, __uint_as_float(o[4 * q + 1]) * inv_l,
                                               __uint_as_float(o[4 * q + 2]) * inv_l,
                                               __uint_as_float(o[4 * q + 3]) * inv_l);
                    } else {
                        uint32_t pkk[8];
#pragma unroll
                        for (int q = 0; q < 8; ++q)
                            pkk[q] = pack_bf16x2(__uint_as_float(o[2 * q]) * inv_l, __uint_as_float(o[2 * q + 1]) * inv_l);
                        uint4* d = reinterpret_cast<uint4*>(orow + c0);
                        d[0] = make_uint4(pkk[0], pkk[1], pkk[2], pkk[3]);
                        d[1] = make_uint4(pkk[4], pkk[5], pkk[6], pkk[7]);
                    }
                }
            }
            if (rank == 0 && half == 0) {
                const float lse2 = l > 0.f ? m_ref + log2f(l) : -INFINITY;
                if (p.nsplit > 1)
                    p.part_lse[prow * p.nsplit + split] = lse2;
                else if (p.lse)
                    p.lse[((size_t)b * p.h_q + h) * p.s_q + t] = lse2 * 0.69314718055994530942f;
            }
        }
    }
    // both CTAs stay resident until the peer is done writing into their shared memory
    tc_fence_before();
    __syncwarp();
    cluster_sync();
    if (warp == NSW + 1) tmem_dealloc(tmem, 512);
}

// Merge of the split partials of the latent attention (same rule as the GQA
// merge: weights 2^(lse_i - max lse)); writes o~ in the layout the
// up-projection reads and the natural-log lse.  One warp per (b, t, head) row.
__global__ void __launch_bounds__(128) latent_combine_kernel(const LatentParams p) {
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const size_t row = (size_t)blockIdx.x * 4 + warp;  // ((b*s_q + t)*h_q + h)
    const size_t nrows = (size_t)p.B * p.s_q * p.h_q;
    if (row >= nrows) return;
    const int h = (int)(row % p.h_q);
    const int t = (int)((row / p.h_q) % p.s_q);
    const int b = (int)(row / ((size_t)p.h_q * p.s_q));
    const int L = clamp_len(p.lens, b, p.Lmax, p.s_q, p.causal, p.status, false);
    const int n_t = p.causal ? L - p.s_q + t + 1 : L;
    const int nsp = cdiv(n_t, p.split_tokens);
    const float* pl = p.part_lse + row * p.nsplit;
    float M = -INFINITY;
    for (int i = lane; i < nsp; i += 32) M = fmaxf(M, pl[i]);
#pragma unroll
    for (int m = 16; m >= 1; m /= 2) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, m));
    float acc[16];
#pragma unroll
    for (int q = 0; q < 16; ++q) acc[q] = 0.f;
    float wsum = 0.f;
    for (int i = 0; i < nsp; ++i) {
        const float w = exp2f(pl[i] - M);
        wsum += w;
        const float4* src = reinterpret_cast<const float4*>(p.part_o + (row * p.nsplit + i) * 512);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const float4 v = src[q * 32 + lane];
            acc[4 * q] = fmaf(w, v.x, acc[4 * q]);
            acc[4 * q + 1] = fmaf(w, v.y, acc[4 * q + 1]);
            acc[4 * q + 2] = fmaf(w, v.z, acc[4 * q + 2]);
            acc[4 * q + 3] = fmaf(w, v.w, acc[4 * q + 3]);
        }
    }
    const float inv = 1.f / wsum;
    const int HPG = p.h_q / p.g;
    const int grp = h / HPG, hh = h % HPG;
    __nv_bfloat16* orow = p.o_lat + ((size_t)grp * p.B * HPG * p.s_q + (size_t)(b * HPG + hh) * p.s_q + t) * 512;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        uint2 v;
        v.x = pack_bf16x2(acc[4 * q] * inv, acc[4 * q + 1] * inv);
        v.y = pack_bf16x2(acc[4 * q + 2] * inv, acc[4 * q + 3] * inv);
        *reinterpret_cast<uint2*>(orow + (q * 32 + lane) * 4) = v;
    }
    if (p.lse && lane == 0) p.lse[((size_t)b * p.h_q + h) * p.s_q + t] = (M + log2f(wsum)) * 0.69314718055994530942f;
}

int latent_tile_tokens() { return lat::NT; }

cudaError_t latent_attn_launch(const CUtensorMap& tm_lat, const LatentParams& p, cudaStream_t st) {
    const bool f8 = p.kv_scale != nullptr;
    // the query slices: q~ [B*s_q*h_q][512] and q^R [B][h_q][s_q][64], 128 rows of 64 values per box
    CUtensorMap tm_qt, tm_qr;
    const auto BF = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    if (!make_tmap_2d(&tm_qt, BF, p.q_t, 512, (uint64_t)p.B * p.s_q * p.h_q, 1024, 64, 128))
        return cudaErrorInvalidValue;
    {
        const uint64_t dims[3] = {64, (uint64_t)p.s_q, (uint64_t)p.B * p.h_q};
        const uint64_t strides[2] = {128, (uint64_t)p.s_q * 128};
        const uint32_t box[3] = {64, 1, 128};
        if (!make_tmap_nd(&tm_qr, BF, p.q_r, 3, dims, strides, box)) return cudaErrorInvalidValue;
    }
    cudaError_t e = f8 ? cudaFuncSetAttribute(latent_attn_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                              lat::SMEM)
                       : cudaFuncSetAttribute(latent_attn_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                              lat::SMEM);
    if (e != cudaSuccess) return e;
    dim3 grid(2 * p.s_q * p.nsplit, p.B);
    {
        TimedLaunch timer(st);
        if (f8)
            latent_attn_kernel<true><<<grid, lat::NTHREADS_F8, lat::SMEM, st>>>(tm_lat, tm_qt, tm_qr, p);
        else
            latent_attn_kernel<false><<<grid, lat::NTHREADS_BF, lat::SMEM, st>>>(tm_lat, tm_qt, tm_qr, p);
        timer.stop();
    }
    e = cudaPeekAtLastError();
    if (e != cudaSuccess || p.nsplit == 1) return e;
    const size_t nrows = (size_t)p.B * p.s_q * p.h_q;
    latent_combine_kernel<<<(unsigned)((nrows + 3) / 4), 128, 0, st>>>(p);
    return cudaPeekAtLastError();
}

}  // namespace lka
