// common.cuh -- device-side building blocks shared by the kernels of this
// library: mbarriers with bounded waits, TMA bulk-tensor loads, bf16 helpers,
// and the workspace status word.
//
// Every wait on an mbarrier is bounded (by %globaltimer): when it runs out the
// kernel records LKA_DEV_TIMEOUT in the caller's workspace status word and
// leaves its loops, so a scheduling bug shows up as an error code instead of a
// hung GPU.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace lka {

// ---- workspace header ------------------------------------------------------
// Every workspace starts with a 256-byte header; word 0 is the sticky status.
constexpr size_t kWsHeaderBytes = 256;
constexpr uint32_t kDevTimeout = 1u;    // a bounded wait ran out
constexpr uint32_t kDevBadLength = 2u;  // a cache_lens entry was clamped
constexpr uint32_t kDevBadPage = 4u;    // a block-table entry outside the page pool was replaced
constexpr uint32_t kDevRange = 8u;      // an intermediate exceeded the range of its internal format (saturated)

// Default limit of a bounded wait (nanoseconds of %globaltimer).
constexpr uint64_t kWaitLimitNs = 2000000000ull;

__host__ __device__ constexpr inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }
__host__ __device__ constexpr inline int cdiv(int a, int b) { return (a + b - 1) / b; }

// Length of sequence b as the kernels use it: clamped into [lo, Lmax] with
// lo = s_q for causal attention (1 otherwise); a clamp raises kDevBadLength.
__device__ __forceinline__ int clamp_len(const int32_t* lens, int b, int Lmax, int s_q, int causal,
                                         uint32_t* status, bool report) {
    int L = lens[b];
    int lo = causal ? s_q : 1;
    if (L < lo || L > Lmax) {
        if (report) atomicOr(status, kDevBadLength);
        L = L < lo ? lo : Lmax;
    }
    return L;
}

// ---- PTX wrappers -----------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t globaltimer() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

// Makes mbarrier initialisation visible to the async proxy (TMA, tcgen05).
__device__ __forceinline__ void fence_barrier_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}

// Waits until the phase with the given parity has completed, for at most
// limit_ns.  Returns false (and records kDevTimeout) when the limit runs out.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, uint32_t* status,
                                          uint64_t limit_ns = kWaitLimitNs) {
#pragma unroll 1
    for (int i = 0; i < 32; ++i)
        if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer();
#pragma unroll 1
    while (true) {
        if (mbar_try_wait(bar, parity)) return true;
        if (globaltimer() - t0 > limit_ns) {
            if (status) atomicOr(status, kDevTimeout);
            return false;
        }
    }
}

// 2-D tiled TMA load of one box into shared memory, completing on `bar`.
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, int x, int y, uint32_t bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
            dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar)
        : "memory");
}

// Prefetch of one box of a tiled tensor into L2 (no shared memory, no completion to wait for;
// out-of-range boxes are dropped by the copy engine).
__device__ __forceinline__ void tma_prefetch_2d(const CUtensorMap* map, int x, int y) {
    asm volatile("cp.async.bulk.prefetch.tensor.2d.L2.global.tile [%0, {%1, %2}];" ::"l"(
                     reinterpret_cast<uint64_t>(map)),
                 "r"(x), "r"(y)
                 : "memory");
}

__device__ __forceinline__ void prefetch_tensormap(const CUtensorMap* map) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// Named barrier over `count` threads (id 0 is __syncthreads).
__device__ __forceinline__ void named_barrier(int id, int count) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}

// 2^x with the hardware approximation (MUFU; ftz; 2^-inf = +0).
__device__ __forceinline__ float fast_exp2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// Pairwise (tree) max and sum of N register values: log2(N) dependent steps instead of N,
// so a single warp per scheduler is not bound by the add/max latency chain.
template <int N>
__device__ __forceinline__ float tree_max(const float* v) {
    if constexpr (N == 1) {
        return v[0];
    } else {
        return fmaxf(tree_max<N / 2>(v), tree_max<N - N / 2>(v + N / 2));
    }
}
template <int N>
__device__ __forceinline__ float tree_sum(const float* v) {
    if constexpr (N == 1) {
        return v[0];
    } else {
        return tree_sum<N / 2>(v) + tree_sum<N - N / 2>(v + N / 2);
    }
}

// ---- element conversion -------------------------------------------------------
// Unpack 8 bf16 values held in 16 bytes into fp32 (exact).
__device__ __forceinline__ void bf16x8_to_f32(const uint4 u, float* f) {
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        f[2 * i] = __uint_as_float(w[i] << 16);
        f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
}

__device__ __forceinline__ void bf16x2_to_f32(uint32_t w, float& lo, float& hi) {
    lo = __uint_as_float(w << 16);
    hi = __uint_as_float(w & 0xffff0000u);
}

template <typename T>
__device__ __forceinline__ float to_f32(T x);
template <>
__device__ __forceinline__ float to_f32<float>(float x) { return x; }
template <>
__device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T>
__device__ __forceinline__ T from_f32(float x);
template <>
__device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <>
__device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) { return __float2bfloat16_rn(x); }

}  // namespace lka
