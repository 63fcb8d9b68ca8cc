// host_util.h -- host-side helpers of the C ABI: TMA descriptor encoding,
// argument checks, workspace carving and device properties.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>
#include <stddef.h>
#include <stdint.h>

#include <atomic>
#include <mutex>

#include "../../include/lka.h"

namespace lka {

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// cuTensorMapEncodeTiled, fetched once through the runtime (no -lcuda link).
inline PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

// A 2-D row-major tensor [rows][inner] of `elem_bytes` elements, row stride
// `row_stride_bytes`, loaded in boxes of box_inner x box_rows with 128-byte
// swizzle (box_inner * elem_bytes must be 128) or no swizzle.
inline bool make_tmap_2d(CUtensorMap* map, CUtensorMapDataType dt, const void* base, uint64_t inner, uint64_t rows,
                         uint64_t row_stride_bytes, uint32_t box_inner, uint32_t box_rows,
                         CUtensorMapSwizzle swz = CU_TENSOR_MAP_SWIZZLE_128B) {
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {inner, rows};
    cuuint64_t strides[1] = {row_stride_bytes};
    cuuint32_t box[2] = {box_inner, box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(map, dt, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// An N-D (N <= 5) row-major tensor; dims[0] is the contiguous one, strides_bytes has N-1 entries.
inline bool make_tmap_nd(CUtensorMap* map, CUtensorMapDataType dt, const void* base, int rank, const uint64_t* dims,
                         const uint64_t* strides_bytes, const uint32_t* box,
                         CUtensorMapSwizzle swz = CU_TENSOR_MAP_SWIZZLE_128B) {
    auto fn = encode_fn();
    if (!fn || rank < 1 || rank > 5) return false;
    cuuint64_t d[5], s[4];
    cuuint32_t bx[5], es[5];
    for (int i = 0; i < rank; ++i) {
        d[i] = dims[i];
        bx[i] = box[i];
        es[i] = 1;
        if (i + 1 < rank) s[i] = strides_bytes[i];
    }
    CUresult r = fn(map, dt, rank, const_cast<void*>(base), d, s, bx, es, CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

inline int sm_count() {
    static std::atomic<int> cache[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
    int v = cache[dev].load(std::memory_order_relaxed);
    if (v == 0) {
        if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v <= 0) v = 148;
        cache[dev].store(v, std::memory_order_relaxed);
    }
    return v;
}

// The status code of a workspace status word (the first raised flag in the order timeout, clamped length,
// bad page, range).
lka_status_t status_from_word(uint32_t word);

// Split size knob of the calling host thread (0 = automatic).
int split_tokens_knob();

// Optional timing of the main kernel of each entry point (see
// lka_kernel_timing): when enabled on the calling thread, a pair of CUDA events is recorded on the
// launch stream around that kernel.  The events come from a pool that is only
// created, never device memory.
bool kernel_timing_on();
cudaEvent_t kernel_timing_event();
void kernel_timing_push(cudaEvent_t a, cudaEvent_t b);

struct TimedLaunch {
    cudaStream_t st;
    cudaEvent_t a = nullptr, b = nullptr;
    explicit TimedLaunch(cudaStream_t s) : st(s) {
        if (kernel_timing_on()) {
            a = kernel_timing_event();
            b = kernel_timing_event();
            if (a && b) cudaEventRecord(a, st);
        }
    }
    void stop() {
        if (a && b) {
            cudaEventRecord(b, st);
            kernel_timing_push(a, b);
            a = b = nullptr;
        }
    }
};

// Carves consecutive 256-byte aligned regions out of a workspace.
struct WsCarve {
    size_t off = 256;  // the first 256 bytes hold the status header
    size_t take(size_t bytes) {
        size_t o = off;
        off += (bytes + 255) / 256 * 256;
        return o;
    }
};

}  // namespace lka
