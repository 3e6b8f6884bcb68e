// Window attention on the 5th-generation tensor cores, for head_dim 64.
//
// Bidirectional attention inside one cu_seqlens window for one head
// (aut_encoder page, AuTAttention: block-diagonal over the packed windows, no
// cache; openarchlab "1A . AuT Audio Encoder", section 3: non-causal within each
// segment).  A window has at most 128 tokens, so one (window, head) is one
// 128-row tile and the softmax is exact in one pass over the tile:
//
//   TMA:      Q, K, V tiles [128 x 64] bf16 (128-byte swizzle) from qkv [T, 3d];
//             rows past the window's end are the next window's rows (or zero
//             past T) and are masked below
//   tcgen05:  S = Q K^T            M = 128, N = 128, K = 64 -> TMEM columns 0..127
//   threads:  two warps per TMEM lane quadrant, each over half of the keys, own
//             query row r: row max over the valid keys, then
//             p = exp2((s - max) * log2(e) / sqrt(64)), row sum, and P written to
//             shared memory as fp16 (P lies in [0, 1]; fp16 keeps 11 significant
//             bits, 8x finer than bf16) in the swizzled K-major layout the MMA
//             reads, over the Q and K tiles the first MMA no longer needs; V is
//             converted in place to fp16 (exact for bf16 values in fp16's range)
//   tcgen05:  O = P V              M = 128, N = 64, K = 128, f16 inputs, V read
//                                  MN-major -> TMEM columns 0..63 (S is dead)
//   threads:  O / rowsum written as [hi | lo] bf16 halves of a 2 d row (rows past
//             the window's end are not written)
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "aut_internal.h"
#include "aut_kernels.h"
#include "aut_ptx.cuh"

namespace aut {

namespace {

using bf16 = __nv_bfloat16;

constexpr int kTile = 128;                 // query / key rows per tile
constexpr int kHd = 64;                    // head dim (one 128-byte swizzle row)
constexpr int kTileBytes = kTile * kHd * 2;  // 16 KiB
// Shared memory: Q | K | V; P (fp16, 128 x 128) overwrites Q | K once S is done.
constexpr int kOffQ = 0, kOffK = kTileBytes, kOffV = 2 * kTileBytes;
constexpr int kOffRed = 3 * kTileBytes;               // row max / sum of the two column halves
constexpr int kOffBar = kOffRed + 2 * 2 * kTile * 4;
constexpr int kSmem = 1024 + kOffBar + 64;
constexpr int kThreads = 256;  // 8 warps: TMEM lane quadrant x half of the key (or O) columns
constexpr uint32_t kTmemCols = 128;        // S: 0..127, then O: 0..63
// kind::f16 with fp16 A and B, fp32 accumulate, A K-major, B MN-major.
__host__ __device__ constexpr uint32_t idesc_f16_f32_bmn(int M, int N) {
    return (1u << 4) | (1u << 16) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}
constexpr unsigned long long kTimeoutNs = 4000ull * 1000ull * 1000ull;

// Byte offset of the 16-byte chunk `chunk` (8 keys) of row `r` in a K-major
// operand of 128 rows x 128 keys held as two 128-byte-swizzled atoms of 64 keys.
__device__ __forceinline__ uint32_t p_chunk_offset(int r, int chunk) {
    const int atom = chunk >> 3, c = chunk & 7;
    return (uint32_t)(atom * kTileBytes + r * 128 + ((c ^ (r & 7)) << 4));
}

__global__ void __launch_bounds__(kThreads) window_attn_tc_kernel(
    const __grid_constant__ CUtensorMap tm_qkv, bf16 *__restrict__ out, const int *__restrict__ cu,
    int d, float scale_log2e, int *status) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint8_t *sQ = sm + kOffQ, *sK = sm + kOffK, *sV = sm + kOffV;
    uint8_t *sP = sQ;  // reuses Q | K after the S MMAs completed
    float *red_max = reinterpret_cast<float *>(sm + kOffRed);  // [2 halves][128 rows]
    float *red_sum = red_max + 2 * kTile;
    uint64_t *bar = reinterpret_cast<uint64_t *>(sm + kOffBar);  // load, S done, O done
    uint32_t *tslot = reinterpret_cast<uint32_t *>(bar + 3);
    volatile int *fail = reinterpret_cast<volatile int *>(tslot + 1);  // the load timed out
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int quad = warp & 3, half = warp >> 2;
    const int row = quad * 32 + lane;  // query row of this thread (TMEM lane)

    pdl_trigger();
    if (tid == 0) {
        mbar_init(bar + 0, 1);
        mbar_init(bar + 1, 1);
        mbar_init(bar + 2, 1);
        *fail = 0;
        fence_barrier_init();
        tma_prefetch_desc(&tm_qkv);
    }
    if (warp == 0) {
        tmem_alloc(tslot, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tslot;
    pdl_wait();

    const int seg = blockIdx.x, h = blockIdx.y;
    const int s0 = cu[seg], len = cu[seg + 1] - s0;
    bool ok = len > 0;

    if (ok && tid == 0) {
        mbar_arrive_expect_tx(bar + 0, 3 * kTileBytes);
        tma_load_2d(sQ, &tm_qkv, bar + 0, h * kHd, s0);
        tma_load_2d(sK, &tm_qkv, bar + 0, d + h * kHd, s0);
        tma_load_2d(sV, &tm_qkv, bar + 0, 2 * d + h * kHd, s0);
        if (mbar_wait(bar + 0, 0, nullptr, kTimeoutNs)) {
            tc_fence_after();
            constexpr uint32_t idesc_s = idesc_bf16_f32(kTile, kTile);
#pragma unroll
            for (int kk = 0; kk < kHd / 16; ++kk)
                tc_mma_bf16(tmem, smem_desc_sw128(sQ) + 2 * kk, smem_desc_sw128(sK) + 2 * kk,
                            idesc_s, kk > 0);
            tc_commit(bar + 1);
        } else {
            if (status) atomicCAS(status, 0, kDevTimeout);
            *fail = 1;  // nothing was issued to the tensor cores; release the row threads
            mbar_arrive(bar + 1);
        }
    }

    // ---- softmax of row `row` over the window's keys (two warps per row) ----
    const uint32_t trow = tmem + ((uint32_t)(quad * 32) << 16);
    float row_sum = 1.f;
    if (ok) {
        if (!mbar_wait(bar + 1, 0, nullptr, kTimeoutNs)) {
            if (status) atomicCAS(status, 0, kDevTimeout);
        }
        ok = *fail == 0;
    }
    tc_fence_after();
    if (ok) {  // block-uniform: every thread shares `len`
        float v[2][32];
        tmem_ld32(trow + half * 64, v[0]);
        tmem_ld32(trow + half * 64 + 32, v[1]);
        tc_wait_ld();
        float mx = -INFINITY;
#pragma unroll
        for (int c = 0; c < 2; ++c)
#pragma unroll
            for (int j = 0; j < 32; ++j)
                if (half * 64 + c * 32 + j < len) mx = fmaxf(mx, v[c][j]);
        red_max[half * kTile + row] = mx;
        __syncthreads();
        mx = fmaxf(red_max[row], red_max[kTile + row]);
        float sum = 0.f;
#pragma unroll
        for (int c = 0; c < 2; ++c) {
#pragma unroll
            for (int q = 0; q < 4; ++q) {  // 8 keys = one 16-byte chunk of P
                uint32_t ph[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int j = q * 8 + 2 * e, key = half * 64 + c * 32 + j;
                    const float p0 = key < len ? exp2f((v[c][j] - mx) * scale_log2e) : 0.f;
                    const float p1 = key + 1 < len ? exp2f((v[c][j + 1] - mx) * scale_log2e) : 0.f;
                    sum += p0 + p1;
                    __half2 hp = __floats2half2_rn(p0, p1);
                    ph[e] = *reinterpret_cast<uint32_t *>(&hp);
                }
                *reinterpret_cast<uint4 *>(sP + p_chunk_offset(row, half * 8 + c * 4 + q)) =
                    make_uint4(ph[0], ph[1], ph[2], ph[3]);
            }
        }
        red_sum[half * kTile + row] = sum;
        // V to fp16 in place (same positions, so the swizzled layout is kept).  Every
        // thread acquires the TMA barrier (long complete) before reading V directly.
        mbar_wait(bar + 0, 0, nullptr, kTimeoutNs);
        uint4 *vv = reinterpret_cast<uint4 *>(sV) + tid * 4;
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            uint4 w = vv[u];
            uint32_t *e = reinterpret_cast<uint32_t *>(&w);
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&e[k]));
                __half2 hv = __floats2half2_rn(f.x, f.y);
                e[k] = *reinterpret_cast<uint32_t *>(&hv);
            }
            vv[u] = w;
        }
    } else {
        __syncthreads();  // matches the row-max exchange above
    }
    fence_proxy_async_smem();  // P and V (generic-proxy writes) visible to the MMA
    tc_fence_before();
    __syncthreads();
    if (ok) row_sum = red_sum[row] + red_sum[kTile + row];

    if (ok && tid == 0) {
        tc_fence_after();
        // O = P V over 128 keys: k-step s covers keys 16 s .. 16 s + 16.
        constexpr uint32_t idesc_o = idesc_f16_f32_bmn(kTile, kHd);
#pragma unroll
        for (int s = 0; s < 8; ++s)
            tc_mma_bf16(tmem, smem_desc_sw128(sP + (s >> 2) * kTileBytes) + 2 * (s & 3),
                        smem_desc_sw128_mn(sV + s * 16 * 128), idesc_o, s > 0);
        tc_commit(bar + 2);
    }
    if (ok) {
        if (!mbar_wait(bar + 2, 0, nullptr, kTimeoutNs)) {
            if (status) atomicCAS(status, 0, kDevTimeout);
        }
    }
    tc_fence_after();
    if (ok) {  // O columns half * 32 .. + 32 of row `row`
        const float inv = 1.f / row_sum;
        float v[32];
        tmem_ld32(trow + half * 32, v);
        tc_wait_ld();
        if (row < len) {
            bf16 *o = out + (size_t)(s0 + row) * 2 * d + h * kHd + half * 32;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                uint32_t hi[4], lo[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float a = v[q * 8 + 2 * e] * inv, b = v[q * 8 + 2 * e + 1] * inv;
                    hi[e] = pack_bf16x2(a, b);
                    const float2 hf =
                        __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&hi[e]));
                    lo[e] = pack_bf16x2(a - hf.x, b - hf.y);
                }
                *reinterpret_cast<uint4 *>(o + q * 8) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
                *reinterpret_cast<uint4 *>(o + d + q * 8) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
            }
        }
    }
    if (tid == 0 && *fail) mbar_wait(bar + 0, 0, nullptr, kTimeoutNs);  // copies in flight land
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

}  // namespace

cudaError_t launch_window_attention_tc(const void *qkv, void *out, const int *cu_dev, int n_windows,
                                       int d, int heads, int T, int *status, cudaStream_t st) {
    if (n_windows <= 0) return cudaSuccess;
    if (d / heads != kHd || T <= 0) return cudaErrorInvalidValue;
    static bool attr_done[64] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev >= 0 && dev < 64 && !attr_done[dev]) {
        const cudaError_t e = cudaFuncSetAttribute(
            window_attn_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
        if (e != cudaSuccess) return e;
        attr_done[dev] = true;
    }
    CUtensorMap tm;
    const uint64_t dims[2] = {(uint64_t)3 * d, (uint64_t)T};
    const uint64_t strides[1] = {(uint64_t)3 * d * 2};
    const uint32_t box[2] = {kHd, kTile};
    if (!make_tensor_map_bf16_sw128(&tm, 2, qkv, dims, strides, box)) return cudaErrorInvalidValue;
    const float scale_log2e = 1.4426950408889634f / 8.0f;  // log2(e) / sqrt(64)
    return launch_pdl(window_attn_tc_kernel, dim3(n_windows, heads), dim3(kThreads), kSmem, st, 1, tm,
                      static_cast<bf16 *>(out), cu_dev, d, scale_log2e, status);
}

}  // namespace aut
