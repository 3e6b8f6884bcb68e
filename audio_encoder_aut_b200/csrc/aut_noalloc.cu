// Window attention for callers that cannot allocate device memory.
//
// aut_window_attention needs a small device scratch area: the window
// boundaries (cu_seqlens) are copied there before the kernel reads them, and
// the caller normally passes that area as `workspace`.  Some callers cannot
// provide one: code whose device memory is owned by another allocator that
// forbids raw cudaMalloc, or that runs where allocation is not allowed at all
// (for example while a stream is being captured into a CUDA graph in a mode
// that rejects allocation calls).  aut_window_attention_noalloc keeps that
// scratch in a file-scope device array instead, so the caller passes only the
// inputs and the output.
#include <cuda_runtime.h>

#include <mutex>

#include "aut_internal.h"
#include "aut_kernels.h"

namespace aut {
namespace {

constexpr int kNoAllocMaxWindows = 32766;  // status word + cu_seqlens: 32768 words (128 KiB)

// Word 0 is the call's status word (a bounded wait that runs out writes
// AUT_ERR_TIMEOUT there), words 1 .. num_windows + 1 the uploaded cu_seqlens.
// Every GPU that loads the library holds this array until the process exits.
// All calls share it: calls that overlap on the GPU (different streams without
// ordering between them) race on it.
__device__ __align__(256) int32_t g_cu_seqlens_scratch[kNoAllocMaxWindows + 2];

// The array's device address for the current device.  In host code the
// array's name is only a host-side stand-in, so the address is looked up once
// per device (with that device current) and cached.
aut_status scratch_for_current_device(int32_t **out) {
    static std::mutex mu;
    static int32_t *addr[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return AUT_ERR_CUDA;
    if (dev < 0 || dev >= 64) return AUT_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(mu);
    if (!addr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_cu_seqlens_scratch) != cudaSuccess || !p) return AUT_ERR_CUDA;
        addr[dev] = static_cast<int32_t *>(p);
    }
    *out = addr[dev];
    return AUT_OK;
}

}  // namespace

aut_status noalloc_status_word(int32_t **out) { return scratch_for_current_device(out); }

}  // namespace aut

extern "C" aut_status aut_window_attention_noalloc(const void *qkv, void *out, int32_t T, int32_t d,
                                                   int32_t heads, const int32_t *cu_seqlens,
                                                   int32_t num_windows, aut_stream_t stream) {
    using namespace aut;
    if (T < 0 || d <= 0 || heads <= 0 || d % heads || num_windows < 0 || !cu_seqlens)
        return AUT_ERR_INVALID_ARG;
    if (num_windows > kNoAllocMaxWindows) return AUT_ERR_WORKSPACE;
    const int hd = d / heads;
    if (hd != 16 && hd != 32 && hd != 64 && hd != 128) return AUT_ERR_UNSUPPORTED;
    if (cu_seqlens[0] != 0 || cu_seqlens[num_windows] != T) return AUT_ERR_INVALID_ARG;
    for (int i = 0; i < num_windows; ++i) {
        const int len = cu_seqlens[i + 1] - cu_seqlens[i];
        if (len < 0 || len > kMaxWindowTokens) return AUT_ERR_INVALID_ARG;
    }
    if (T > 0 && (!qkv || !out)) return AUT_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(qkv) | reinterpret_cast<uintptr_t>(out)) & 15u)
        return AUT_ERR_INVALID_ARG;
    int32_t *scratch = nullptr;
    const aut_status st = scratch_for_current_device(&scratch);  // first call per device: set-up
    if (st != AUT_OK) return st;
    if (T == 0) return AUT_OK;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    // One upload rewrites, in stream order, everything the kernel reads: the
    // status word (cleared to 0) and the whole cu_seqlens prefix.  Entries past
    // it, left by an earlier call with more windows, are never read.
    std::vector<int32_t> words(1, 0);
    words.insert(words.end(), cu_seqlens, cu_seqlens + num_windows + 1);
    if (launch_upload(words.data(), words.size(), scratch, s) != cudaSuccess) return AUT_ERR_CUDA;
    return launch_window_attention(qkv, out, scratch + 1, num_windows, d, heads, s, T, scratch) ==
                   cudaSuccess
               ? AUT_OK
               : AUT_ERR_CUDA;
}
