// Audio injection into the decoder's input sequence (cubic.dev "Audio Encoder
// Component", Audio Injection Logic): the encoder's output rows replace the
// embeddings at the <|audio_pad|> placeholder positions of the token sequence,
// in sequence order (the j-th placeholder takes packed row j).
//
//   inject_rank_kernel  one CTA scans the token ids: src[i] = the number of
//                       placeholders before position i if i is one, else -1;
//                       a count that differs from the number of audio rows
//                       writes AUT_ERR_INVALID_ARG to the status word
//   inject_copy_kernel  every placeholder row <- its audio row (fp32 -> bf16,
//                       round to nearest even); ranks past the audio rows
//                       (after a count mismatch) are skipped
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "aut_internal.h"
#include "aut_kernels.h"
#include "aut_ptx.cuh"

namespace aut {
namespace {

constexpr int kScanThreads = 1024;

__global__ void __launch_bounds__(kScanThreads) inject_rank_kernel(const int32_t *__restrict__ ids,
                                                                   int L, int pad_id, int T,
                                                                   int32_t *__restrict__ src,
                                                                   int *__restrict__ status) {
    pdl_trigger();
    pdl_wait();
    __shared__ int warp_sums[kScanThreads / 32];
    __shared__ int carry;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    if (threadIdx.x == 0) carry = 0;
    __syncthreads();
    for (int base = 0; base < L; base += kScanThreads) {
        const int i = base + threadIdx.x;
        const int is_pad = (i < L && ids[i] == pad_id) ? 1 : 0;
        int incl = is_pad;  // inclusive scan inside the warp
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int v = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += v;
        }
        if (lane == 31) warp_sums[warp] = incl;
        __syncthreads();
        if (warp == 0) {
            int w = warp_sums[lane];
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int v = __shfl_up_sync(0xffffffffu, w, o);
                if (lane >= o) w += v;
            }
            warp_sums[lane] = w;  // inclusive over warps
        }
        __syncthreads();
        const int before = carry + (warp ? warp_sums[warp - 1] : 0) + incl - is_pad;
        if (i < L) src[i] = is_pad ? before : -1;
        __syncthreads();
        if (threadIdx.x == 0) carry += warp_sums[kScanThreads / 32 - 1];
        __syncthreads();
    }
    if (threadIdx.x == 0 && carry != T && status) atomicCAS(status, 0, (int)AUT_ERR_INVALID_ARG);
}

// One warp per row; the row moves as 16-byte groups where the alignment allows.
__global__ void inject_copy_kernel(const int32_t *__restrict__ src, int L, int T, int D,
                                   const float *__restrict__ audio,
                                   __nv_bfloat16 *__restrict__ embeds) {
    pdl_trigger();
    pdl_wait();
    const int lane = threadIdx.x & 31;
    const int warps = (gridDim.x * blockDim.x) >> 5;
    for (int i = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; i < L; i += warps) {
        const int j = src[i];
        if (j < 0 || j >= T) continue;  // a text row, or a rank past the audio rows
        const float *a = audio + (size_t)j * D;
        __nv_bfloat16 *e = embeds + (size_t)i * D;
        if (D % 4 == 0) {
            for (int c = lane * 4; c < D; c += 128) {
                const float4 v = *reinterpret_cast<const float4 *>(a + c);
                uint2 o;
                o.x = pack_bf16x2(v.x, v.y);
                o.y = pack_bf16x2(v.z, v.w);
                *reinterpret_cast<uint2 *>(e + c) = o;
            }
        } else {
            for (int c = lane; c < D; c += 32) e[c] = __float2bfloat16_rn(a[c]);
        }
    }
}

struct InjectLayout {
    size_t status, src, total;
};
InjectLayout inject_layout(int L) {
    InjectLayout l{};
    l.status = 0;
    l.src = 256;
    l.total = 256 + ((size_t)std::max(L, 1) * 4 + 255) / 256 * 256;
    return l;
}

}  // namespace
}  // namespace aut

using namespace aut;

extern "C" size_t aut_inject_workspace_bytes(int32_t L) {
    return L < 0 ? 0 : inject_layout(L).total;
}

extern "C" aut_status aut_inject_audio(void *embeds, const int32_t *token_ids, int32_t L,
                                       int32_t audio_pad_id, const void *audio, int32_t T,
                                       int32_t D, void *workspace, size_t ws_bytes,
                                       aut_stream_t stream) {
    if (L < 0 || T < 0 || D <= 0) return AUT_ERR_INVALID_ARG;
    if (L > 0 && (!embeds || !token_ids)) return AUT_ERR_INVALID_ARG;
    if (T > 0 && !audio) return AUT_ERR_INVALID_ARG;
    if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u)) return AUT_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(token_ids) & 3u) || (reinterpret_cast<uintptr_t>(audio) & 15u) ||
        (reinterpret_cast<uintptr_t>(embeds) & 7u))
        return AUT_ERR_INVALID_ARG;
    const InjectLayout lay = inject_layout(L);
    if (ws_bytes < lay.total) return AUT_ERR_WORKSPACE;
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    int *status = reinterpret_cast<int *>(ws + lay.status);
    int32_t *src = reinterpret_cast<int32_t *>(ws + lay.src);
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const int32_t zero = 0;
    if (launch_upload(&zero, 1, status, st) != cudaSuccess) return AUT_ERR_CUDA;
    if (L == 0) {
        // No placeholders: the count matches only when there are no audio rows.
        return T == 0 ? AUT_OK : AUT_ERR_INVALID_ARG;
    }
    if (launch_pdl(inject_rank_kernel, dim3(1), dim3(kScanThreads), 0, st, 1, token_ids, (int)L,
                   (int)audio_pad_id, (int)T, src, status) != cudaSuccess)
        return AUT_ERR_CUDA;
    const int blocks = std::min((L + 7) / 8, 8 * sm_count_cached());
    if (launch_pdl(inject_copy_kernel, dim3(blocks), dim3(256), 0, st, 1,
                   static_cast<const int32_t *>(src), (int)L, (int)T, (int)D,
                   static_cast<const float *>(audio), static_cast<__nv_bfloat16 *>(embeds)) !=
        cudaSuccess)
        return AUT_ERR_CUDA;
    return AUT_OK;
}
