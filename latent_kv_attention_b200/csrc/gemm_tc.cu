// gemm_tc.cu -- per-group projection GEMMs of the GQLA latent paths on the
// 5th-generation tensor cores (tcgen05, accumulators in tensor memory).
//
// Three uses, all C = A * B^T with bf16 operands and fp32 accumulation, one
// weight matrix per head group gamma ("GQLA ..." section 3.1, eq. (1): W^UK,
// W^UV in R^{g*d_h x r_kv}, block gamma maps the latent to group gamma):
//  ABSORB  q~[b,t,i,:] = W^UK_gamma^T q^C[b,i,t,:]   (M = B*HPG*s_q rows per group, N = r_kv, K = d_h)
//          -- W^UK folded into the query of the MQA-absorbed path;
//  UPPROJ  out[b,i,t,:] = W^UV_gamma o~[gamma][(b,i,t)] (N = d_h, K = r_kv)
//          -- W^UV applied to the latent-space attention output;
//  EXPAND  kc[b,gamma,j,:] = W_gamma c_j for every cache slot (N = d_h, K = r_kv)
//          -- the one-time conversion of the latent cache to the per-group cache.
//
// One CTA computes a 128 x N_TILE output tile: warp 0 streams A and B k-blocks
// of 64 with TMA (128-byte swizzle) through a 4-stage ring, warp 1 issues the
// MMAs (M = 128, N = N_TILE, K = 16 per instruction) into tensor memory, and
// all four warps drain the accumulator (one TMEM lane = one output row).
#include "common.cuh"
#include "host_util.h"
#include "latent.h"
#include "tc.cuh"

namespace lka {

template <int N_TILE, int MODE>
struct GemmCfg {
    static constexpr bool B_MN = (MODE == GEMM_ABSORB);  // W^UK^T is N-contiguous
    static constexpr int NST = 4;
    static constexpr int A_BYTES = 128 * 128;            // 128 rows x 64 bf16
    static constexpr int B_BYTES = N_TILE * 128;         // N_TILE rows (or 64-wide blocks) x 64 bf16
    static constexpr int STAGE = A_BYTES + B_BYTES;
    static constexpr int SMEM = 1024 + NST * STAGE + 256;
};

template <int N_TILE, int MODE>
__global__ void __launch_bounds__(128, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                   const GemmParams p) {
    using C = GemmCfg<N_TILE, MODE>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(align_up(reinterpret_cast<uintptr_t>(smem_raw), 1024));
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::NST * C::STAGE);
    uint64_t* empty = full + C::NST;
    uint64_t* done = empty + C::NST;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);

    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int tm = blockIdx.x, tn = blockIdx.y, grp = blockIdx.z;
    const int nkb = p.K / 64;

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::NST; ++s) {
            mbar_init(smem_u32(&full[s]), 1);
            mbar_init(smem_u32(&empty[s]), 1);
        }
        mbar_init(smem_u32(done), 1);
        fence_barrier_init();
    }
    if (warp == 0) {
        tmem_alloc(tmem_slot, N_TILE);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0 && lane == 0) {
        // ---------------- TMA producer ----------------
        prefetch_tensormap(&tmA);
        prefetch_tensormap(&tmB);
        int issued = 0;
        for (int kb = 0; kb < nkb; ++kb) {
            const int s = kb % C::NST;
            if (kb >= C::NST && !mbar_wait(smem_u32(&empty[s]), ((kb / C::NST) - 1) & 1, p.status)) break;
            const uint32_t bar = smem_u32(&full[s]);
            mbar_arrive_expect_tx(bar, C::STAGE);
            const uint32_t a_dst = smem_u32(smem + s * C::STAGE);
            const uint32_t b_dst = a_dst + C::A_BYTES;
            if constexpr (MODE == GEMM_ABSORB) {
                const int slab = p.HPG * p.s_q;  // rows of one (sequence, group) in q_c
                tma_load_3d(a_dst, &tmA, kb * 64, grp * slab, tm * (128 / slab), bar);
#pragma unroll
                for (int nb = 0; nb < N_TILE / 64; ++nb)
                    tma_load_2d(b_dst + nb * 64 * 128, &tmB, tn * N_TILE + nb * 64, grp * p.K + kb * 64, bar);
            } else if constexpr (MODE == GEMM_UPPROJ) {
                tma_load_2d(a_dst, &tmA, kb * 64, grp * p.M_rows + tm * 128, bar);
                tma_load_2d(b_dst, &tmB, kb * 64, grp * p.N + tn * N_TILE, bar);
            } else {
                const int b = tm / p.tiles_per_b, j0 = (tm % p.tiles_per_b) * 128;
                tma_load_2d(a_dst, &tmA, kb * 64, b * p.Lmax + j0, bar);
                tma_load_2d(b_dst, &tmB, kb * 64, grp * p.N + tn * N_TILE, bar);
            }
            ++issued;
        }
        for (int kb = issued - 1; kb >= 0 && kb >= issued - C::NST; --kb)
            mbar_wait(smem_u32(&full[kb % C::NST]), (kb / C::NST) & 1, p.status);
    } else if (warp == 1 && lane == 0) {
        // ---------------- MMA issuer ----------------
        constexpr uint32_t idesc = idesc_bf16_f32(128, N_TILE, false, C::B_MN);
        bool ok = true;
        for (int kb = 0; kb < nkb; ++kb) {
            const int s = kb % C::NST;
            if (!mbar_wait(smem_u32(&full[s]), (kb / C::NST) & 1, p.status)) {
                ok = false;
                break;
            }
            tc_fence_after();
            const uint32_t a_base = smem_u32(smem + s * C::STAGE);
            const uint32_t b_base = a_base + C::A_BYTES;
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const uint64_t ad = smem_desc_sw128(a_base + k * 32, 16, 1024);
                const uint64_t bd = C::B_MN ? smem_desc_sw128(b_base + k * 2048, 64 * 128, 1024)
                                            : smem_desc_sw128(b_base + k * 32, 16, 1024);
                umma_ss(tmem, ad, bd, idesc, (kb | k) != 0);
            }
            umma_commit(smem_u32(&empty[s]));
        }
        if (ok) umma_commit(smem_u32(done));
    }

    // ---------------- epilogue: TMEM -> registers -> global (bf16) ----------------
    __syncwarp();
    const bool have = mbar_wait(smem_u32(done), 0, p.status);
    tc_fence_after();
    if (have) {
        const int r = warp * 32 + lane;  // tile row == TMEM lane
        __nv_bfloat16* orow = nullptr;
        if constexpr (MODE == GEMM_ABSORB) {
            const int slab = p.HPG * p.s_q;
            const int b = tm * (128 / slab) + r / slab;
            const int rr = r % slab, hh = rr / p.s_q, t = rr % p.s_q;
            if (b < p.B)
                orow = reinterpret_cast<__nv_bfloat16*>(p.out) +
                       ((size_t)(b * p.s_q + t) * p.h_q + grp * p.HPG + hh) * p.N;
        } else if constexpr (MODE == GEMM_UPPROJ) {
            const int R = tm * 128 + r;
            if (R < p.M_rows) {
                const int slab = p.HPG * p.s_q;
                const int b = R / slab, rem = R % slab;
                orow = reinterpret_cast<__nv_bfloat16*>(p.out) +
                       ((size_t)b * p.h_q * p.s_q + grp * slab + rem) * p.N;
            }
        } else {
            const int b = tm / p.tiles_per_b, j = (tm % p.tiles_per_b) * 128 + r;
            if (j < p.Lmax)
                orow = reinterpret_cast<__nv_bfloat16*>(p.out) + ((size_t)(b * p.g + grp) * p.Lmax + j) * p.N;
        }
#pragma unroll 1
        for (int c0 = 0; c0 < N_TILE; c0 += 16) {
            uint32_t v[16];
            tmem_ld16(tmem + ((uint32_t)(warp * 32) << 16) + c0, v);
            tmem_ld_wait();
            if (orow) {
                uint32_t pk[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) pk[i] = pack_bf16x2(__uint_as_float(v[2 * i]), __uint_as_float(v[2 * i + 1]));
                uint4* dst = reinterpret_cast<uint4*>(orow + tn * N_TILE + c0);
                dst[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
                dst[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, N_TILE);
}

template <int N_TILE, int MODE>
static cudaError_t gemm_launch(const CUtensorMap& a, const CUtensorMap& b, const GemmParams& p, dim3 grid,
                               cudaStream_t st) {
    using C = GemmCfg<N_TILE, MODE>;
    auto kern = gemm_tc_kernel<N_TILE, MODE>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    if (e != cudaSuccess) return e;
    kern<<<grid, 128, C::SMEM, st>>>(a, b, p);
    return cudaPeekAtLastError();
}

cudaError_t gemm_absorb(const CUtensorMap& a, const CUtensorMap& b, const GemmParams& p, cudaStream_t st) {
    // rows per group B*HPG*s_q, 128 per tile; N = r_kv in tiles of 256
    const int slab = p.HPG * p.s_q;
    dim3 grid(cdiv(p.B, 128 / slab), p.N / 256, p.g);
    return gemm_launch<256, GEMM_ABSORB>(a, b, p, grid, st);
}
cudaError_t gemm_upproj(const CUtensorMap& a, const CUtensorMap& b, const GemmParams& p, cudaStream_t st) {
    dim3 grid(cdiv(p.M_rows, 128), p.N / 128, p.g);
    return gemm_launch<128, GEMM_UPPROJ>(a, b, p, grid, st);
}
cudaError_t gemm_expand(const CUtensorMap& a, const CUtensorMap& b, const GemmParams& p, cudaStream_t st) {
    dim3 grid(p.tiles_per_b * p.B, p.N / 128, p.g);
    return gemm_launch<128, GEMM_EXPAND>(a, b, p, grid, st);
}

}  // namespace lka
