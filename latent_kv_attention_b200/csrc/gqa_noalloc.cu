// gqa_noalloc.cu -- gqa_attn for callers that cannot allocate device memory.
//
// The regular entry point takes a caller-provided workspace for its split-KV
// partial results.  Some callers have no way to provide one: a plugin or custom
// operator hosted by a runtime that hands it only its input and output buffers,
// code on a path where the host framework forbids cudaMalloc/cudaFree (for
// example because an allocation there would synchronise the device or break the
// framework's memory accounting), or a caller without access to any allocator.
// This variant keeps the scratch in a file-scope device array instead, of fixed
// size kNoAllocScratchBytes, which every GPU that loads the library holds until
// the process exits.  It launches the same kernels as gqa_attn and allocates
// nothing itself.
#include <math.h>

#include <atomic>

#include "common.cuh"
#include "gqa_decode.h"
#include "host_util.h"

namespace lka {

// Maximum scratch of the no-allocation variant: 16 MiB (the first 256 bytes
// are the status header, the rest holds the split partials).
constexpr size_t kNoAllocScratchBytes = 16u << 20;

static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];

// The array's name is only a host-side stand-in on the host: its device address
// is looked up once per device, with that device current, and cached.  The cache
// is keyed by the device ordinal only: after cudaDeviceReset on a device the
// library's module is loaded again and the cached address is stale, so this
// variant must not be used on a device after it has been reset.
static std::atomic<uint8_t*> g_noalloc_addr[64];

static uint8_t* noalloc_scratch_address() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
    uint8_t* p = g_noalloc_addr[dev].load(std::memory_order_acquire);
    if (p) return p;
    void* addr = nullptr;
    if (cudaGetSymbolAddress(&addr, g_noalloc_scratch) != cudaSuccess || !addr) return nullptr;
    g_noalloc_addr[dev].store(static_cast<uint8_t*>(addr), std::memory_order_release);
    return static_cast<uint8_t*>(addr);
}

}  // namespace lka

extern "C" lka_status_t gqa_attn_noalloc(const void* q, const void* k, const void* v, const int32_t* cache_lens,
                                         void* out, float* lse, int B, int h_q, int h_kv, int s_q, int d_h, int Lmax,
                                         int causal, float scale, lka_dtype_t dtype, void* stream) {
    if (dtype != LKA_BF16 && dtype != LKA_FP32) return LKA_ERR_UNSUPPORTED;
    if (gqa_attn_workspace_size(B, h_q, h_kv, s_q, d_h, Lmax) == 0) {
        // invalid or unsupported arguments: let gqa_attn report which, without touching the scratch
        return gqa_attn(q, k, v, cache_lens, out, lse, B, h_q, h_kv, s_q, d_h, Lmax, causal, scale, dtype, nullptr,
                        0, stream);
    }
    uint8_t* ws = lka::noalloc_scratch_address();
    if (!ws) return LKA_ERR_CUDA;
    // gqa_attn checks the scratch size against the split plan of this call's dtype and returns
    // LKA_ERR_WORKSPACE, before enqueuing anything, when the plan needs more than the array holds.
    // Nothing in the scratch has to start at zero: every split partial the merge reads is written by the
    // same call first.  The status word at its head accumulates the device-side flags (timeouts, clamped
    // lengths) until gqa_attn_noalloc_status reads and clears it.
    return gqa_attn(q, k, v, cache_lens, out, lse, B, h_q, h_kv, s_q, d_h, Lmax, causal, scale, dtype, ws,
                    lka::kNoAllocScratchBytes, stream);
}

extern "C" lka_status_t gqa_attn_noalloc_status(void* stream) {
    uint8_t* ws = lka::noalloc_scratch_address();
    if (!ws) return LKA_ERR_CUDA;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    uint32_t word = 0;
    // the flags of every call enqueued before this one on `stream` (and, through the one shared array, of
    // any other call that has completed), then an enqueued reset for the calls that follow
    if (cudaStreamSynchronize(st) != cudaSuccess) return LKA_ERR_CUDA;
    if (cudaMemcpyAsync(&word, ws, sizeof(word), cudaMemcpyDeviceToHost, st) != cudaSuccess ||
        cudaStreamSynchronize(st) != cudaSuccess)
        return LKA_ERR_CUDA;
    if (cudaMemsetAsync(ws, 0, sizeof(uint32_t), st) != cudaSuccess) return LKA_ERR_CUDA;
    return lka::status_from_word(word);
}
