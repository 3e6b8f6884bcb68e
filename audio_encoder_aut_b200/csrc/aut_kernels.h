// Host launchers of the encoder's kernels (implemented in aut_kernels.cu and
// aut_gemm.cu), used by the C-ABI layer in aut_api.cu.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include <cstddef>
#include <cstdint>
#include <mutex>
#include <utility>

namespace aut {

// Raises `Kernel`'s dynamic shared-memory limit to `bytes`, once per device;
// safe when several host threads make their first call at the same time.
template <auto Kernel>
cudaError_t smem_attr_once(int bytes) {
    static std::mutex mu;
    static bool done[64] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(mu);
    if (!done[dev]) {
        e = cudaFuncSetAttribute(Kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
        if (e != cudaSuccess) return e;
        done[dev] = true;
    }
    return cudaSuccess;
}

// Multiprocessor count of the current device (cached per device, thread-safe).
int sm_count_cached();

// Launches a forward-path kernel that may start while the previous kernel in
// the stream finishes (programmatic dependent launch); the kernel itself waits
// before touching global memory.  cluster_x > 1 launches CTA clusters.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t st, int cluster_x, Args &&...args) {
    cudaLaunchConfig_t lc{};
    lc.gridDim = grid;
    lc.blockDim = block;
    lc.dynamicSmemBytes = smem;
    lc.stream = st;
    cudaLaunchAttribute attr[2];
    int n = 0;
    attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[n].val.programmaticStreamSerializationAllowed = 1;
    ++n;
    if (cluster_x > 1) {
        attr[n].id = cudaLaunchAttributeClusterDimension;
        attr[n].val.clusterDim.x = cluster_x;
        attr[n].val.clusterDim.y = 1;
        attr[n].val.clusterDim.z = 1;
        ++n;
    }
    lc.attrs = attr;
    lc.numAttrs = n;
    return cudaLaunchKernelEx(&lc, kernel, std::forward<Args>(args)...);
}

enum GemmEpilogue : int {
    kEpiBf16 = 0,        // out bf16 [M, ldo] = acc + bias
    kEpiBf16Gelu = 1,    // out bf16 [M, ldo] = GELU(acc + bias)
    kEpiResidF32 = 2,    // out fp32 [M, ldo] += acc + bias
    kEpiConvPlanes = 3,  // conv2: GELU(acc + bias) -> conv3's phase planes
    kEpiConvFlat = 4,    // conv3: GELU(acc + bias) -> [chunk * 13 + t][f * C + c]
    kEpiPackTokens = 5,  // conv_out: acc (+ bias) (+ pos[t]) -> packed fp32 rows
    kEpiF32 = 6,         // out fp32 [M, ldo] = acc + bias
    kEpiBf16GeluSplit = 7,  // out bf16 [M, 2N]: GELU(acc + bias) as hi | lo halves
};

struct UploadPayload {
    static constexpr int kWords = 8000;  // 32,000 bytes: within the kernel-parameter limit
    int n, offset;
    int32_t words[kWords];
};

// conv1 + GELU into conv2's input phase planes (`planes`, borders included);
// also clears the zero borders of conv3's input planes (`planes2`) for the
// same chunk slots.
cudaError_t launch_conv1(const void *feats, int T_max, const int4 *chunks, int chunk_base,
                         int n_chunks, const void *w, const void *b, void *planes, int plane_rows,
                         void *planes2, int plane2_rows, int C, cudaStream_t st,
                         int *status = nullptr);
// conv1 + GELU on the tensor cores (aut_conv1.cu): the same output as
// launch_conv1, conv2's input planes and both plane sets' zero borders, for
// C a multiple of 32 in [64, 512].
bool conv1_tc_supported(int C);
cudaError_t launch_conv1_tc(const void *feats, int T_max, const int4 *chunks, int chunk_base,
                            int n_chunks, const void *w, const void *b, void *planes, int plane_rows,
                            void *planes2, int plane2_rows, int C, cudaStream_t st, int *status,
                            unsigned long long timeout_ns = 0);
cudaError_t launch_layernorm(const float *x, const void *g, const void *b, void *y, int T, int d,
                             float eps, cudaStream_t st, bool split = false);
cudaError_t launch_duplicate_k(const void *src, void *dst, int N, int K, cudaStream_t st);
cudaError_t launch_to_f16(const void *src, void *dst, size_t n, cudaStream_t st);
// v_f16: the v third of qkv already holds fp16 (the qkv GEMM wrote it so); only
// the head_dim-64 tensor-core path (T > 0) accepts it.
// wins (device, optional, tensor-core path only): the windows as (first token,
// length) pairs, longest first; the kernel walks its (window, head) tiles in
// that order.  Null: cu_seqlens order.
cudaError_t launch_window_attention(const void *qkv, void *out, const int *cu_dev, int n_windows,
                                    int d, int heads, cudaStream_t st, int T = -1,
                                    int *status = nullptr, bool v_f16 = false,
                                    unsigned long long timeout_ns = 0, int fault_inject = 0,
                                    const int2 *wins = nullptr);
// Whether launch_window_attention takes the tensor-core path.
inline bool window_attention_uses_tc(int d, int heads, int T) { return d / heads == 64 && T > 0; }
// tcgen05 variant for head_dim 64 (aut_attention.cu); T = rows of qkv.
// timeout_ns bounds every pipeline wait (0: 4 s); fault_inject leaves the first
// block's first stage unfilled (tests of the time-out path only).
cudaError_t launch_window_attention_tc(const void *qkv, void *out, const int *cu_dev, int n_windows,
                                       int d, int heads, int T, int *status, cudaStream_t st,
                                       bool v_f16 = false, unsigned long long timeout_ns = 0,
                                       int fault_inject = 0, const int2 *wins = nullptr);
// bf16 tensor map with 128-byte swizzle (aut_gemm.cu): dims innermost first,
// strides in bytes for dims 1.., box in elements.
bool make_tensor_map_bf16_sw128(CUtensorMap *m, int rank, const void *ptr, const uint64_t *dims,
                                const uint64_t *strides, const uint32_t *box);
// The same with 64-byte swizzle (an inner box of at most 64 bytes): the 16-byte
// chunk c of a box row at shared address a sits at chunk c ^ ((a >> 7) & 3).
bool make_tensor_map_bf16_sw64(CUtensorMap *m, int rank, const void *ptr, const uint64_t *dims,
                               const uint64_t *strides, const uint32_t *box);
cudaError_t launch_prepare(const void *conv2_w, const void *conv3_w, const void *conv_out_w,
                           void *conv2_tap, void *conv3_tap, void *conv_out_fc, float *pos, int C,
                           int d, cudaStream_t st);
cudaError_t launch_upload(const int32_t *host_words, size_t n, int32_t *dst, cudaStream_t st);

// ---- tensor-core GEMMs (aut_gemm.cu) ----
enum class GemmStatus { kOk, kBadShape, kTensorMap, kLaunch };

struct LinearLaunch {
    const void *a;     // bf16 (fp16 with f16) [M, K]
    const void *w;     // bf16 (fp16 with f16) [N, K]
    const void *bias;  // bf16 [N] or null
    void *out;
    size_t out_elems = 0;  // elements of `out` (0: M * ldo)
    int M, N, K, ldo;
    int epi;           // GemmEpilogue
    // pack-tokens epilogue
    const int4 *chunks;
    int chunk_base;
    const float *pos;
    int *status;
    unsigned long long timeout_ns;
    int fault_inject;
    bool single_cta = false;  // force one CTA per MMA (no CTA pairs)
    bool f16 = false;         // A and W are fp16 instead of bf16
    int f16_col = 1 << 30;    // kEpiBf16: output columns from here on written as fp16
};
GemmStatus launch_linear(const LinearLaunch &L, cudaStream_t st);

struct ConvLaunch {
    const void *planes;  // bf16 [4][plane_rows_cap][cols_in][C]: input phase planes
    int plane_rows_cap;  // rows of one plane in the buffer
    int chunks;          // chunks in this group
    int chunk_rows;      // plane rows per chunk (33 for conv2, 17 for conv3), zero row included
    int cols_in;         // plane columns, zero column included (26 / 14)
    int out_cols;        // output columns (25 / 13)
    int rows_per_tile;   // virtual rows per 128-row M tile (5 / 9)
    int C;
    const void *w_tap;   // bf16 [C][9][C]
    const void *bias;    // bf16 [C]
    int epi;             // kEpiConvPlanes (conv2) or kEpiConvFlat (conv3)
    void *out;
    size_t out_elems;    // elements of `out`
    int dst_plane_rows, dst_chunk_rows, dst_cols;  // kEpiConvPlanes destination geometry
    int *status;
    unsigned long long timeout_ns;
    bool single_cta = false;
};
GemmStatus launch_conv_gemm(const ConvLaunch &L, cudaStream_t st);

}  // namespace aut
