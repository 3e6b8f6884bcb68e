// Window attention on the 5th-generation tensor cores, for head_dim 64.
//
// Bidirectional attention inside one cu_seqlens window for one head
// (aut_encoder page, AuTAttention: block-diagonal over the packed windows, no
// cache; openarchlab "1A . AuT Audio Encoder", section 3: non-causal within each
// segment).  A window has at most 128 tokens, so one (window, head) is one
// 128-row tile and the softmax is exact in one pass over the tile.
//
// The kernel is persistent (one CTA per SM) and walks the (window, head)
// tiles with a grid stride.  Warp roles:
//   warp 0     TMA producer: Q, K, V tiles [128 x 64] bf16 (128-byte swizzle)
//              from qkv [T, 3d] into a ring of kStages stages; rows past the
//              window's end are the next window's rows (or zero past T) and
//              are masked below
//   warp 1     MMA issuer: S = Q K^T (M = 128, N = the window length rounded
//              up to 16, K = 64) into the S buffer of the tile's softmax
//              group; once that group has written P, O = P V (M = 128, N = 64,
//              K = window length rounded up to 16, fp16 inputs, V read
//              MN-major) into one of the group's two O buffers, then S of the
//              group's next tile
//   warps 2-9  two softmax groups of four warps (one per TMEM lane quadrant);
//              group g takes the CTA's tiles g, g + 2, g + 4, ...  Every
//              thread owns one query row and all of its keys, so the row max
//              and sum need no exchange between threads: max over the row,
//              p = exp2(s log2(e) / sqrt(64) - max log2(e) / sqrt(64)) written
//              as fp16 (P lies in [0, 1]; 11 significant bits, 8x finer than
//              bf16) in the swizzled K-major layout the MMA reads, over the Q
//              and K tiles the S product no longer needs; V converted in place
//              to fp16 (saturating) unless the qkv GEMM already wrote it as fp16
//              (v_f16); then, while the tensor cores compute this tile's O and
//              the group's next S, O / rowsum of the group's previous tile
//              written as fp16 [T, d] (rows past the window's end are not
//              written)
// While one group runs its softmax the other's S and O products run on the
// tensor cores, and the producer stays up to kStages tiles ahead.
//
// Tensor memory (512 columns): S buffers of the two groups at 0 and 128; O
// buffers (64 columns) at 256 + 64 (2 g + j), j alternating over the group's
// tiles.  Two TMEM users never share an SM between kernels of the forward:
// this kernel's shared memory (about 197 KB) leaves no room for a GEMM CTA
// (about 197 KB either), so a CTA launched early by programmatic dependent
// launch cannot hold TMEM columns that a CTA of the previous kernel still needs.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "aut_internal.h"
#include "aut_kernels.h"
#include "aut_ptx.cuh"

namespace aut {

namespace {

using bf16 = __nv_bfloat16;

constexpr int kTile = 128;                   // query / key rows per tile
constexpr int kHd = 64;                      // head dim (one 128-byte swizzle row)
constexpr int kTileBytes = kTile * kHd * 2;  // 16 KiB
constexpr int kStages = 4;
constexpr int kStageBytes = 3 * kTileBytes;  // Q | K | V; P (fp16, 128 x 128) overwrites Q | K
constexpr int kGroups = 2;                   // softmax groups (four warps each)
constexpr int kOffWin = kStages * kStageBytes;
constexpr int kWinCache = 512;  // (row0, length) of a CTA's first local tiles' windows
constexpr int kOffBar = kOffWin + kWinCache * 8;
// full[kStages], empty[kStages], s_full[2], p_full[2], o_full[4], o_empty[4], mma_done
constexpr int kNumBars = 2 * kStages + 2 * kGroups + 4 + 4 + 1;
constexpr int kSmem = 1024 + kOffBar + kNumBars * 8 + 16;
constexpr int kComputeWarps = 4 * kGroups;
constexpr int kThreads = 64 + 32 * kComputeWarps;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColO = 256;  // O buffer b (0..3) at kColO + 64 b

// kind::f16 with fp16 A and B, fp32 accumulate, A K-major, B MN-major.
__host__ __device__ constexpr uint32_t idesc_f16_f32_bmn(int M, int N) {
    return (1u << 4) | (1u << 16) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

// Byte offset of the 16-byte chunk `chunk` (8 keys) of row `r` in a K-major
// operand of 128 rows x 128 keys held as two 128-byte-swizzled atoms of 64 keys.
__device__ __forceinline__ uint32_t p_chunk_offset(int r, int chunk) {
    const int atom = chunk >> 3, c = chunk & 7;
    return (uint32_t)(atom * kTileBytes + r * 128 + ((c ^ (r & 7)) << 4));
}

__device__ __forceinline__ void signal_abort(int *status, volatile int *abort) {
    if (status) atomicCAS(status, 0, kDevTimeout);
    *abort = 1;
}

// Tokens of window w (the last 16-row step of the MMAs covers the ragged end).
__device__ __forceinline__ void window_of(const int *cu, int w, int *s0, int *len, int *n16) {
    *s0 = cu[w];
    *len = cu[w + 1] - *s0;
    *n16 = max(1, (*len + 15) >> 4);
}
// The same from the CTA's shared-memory cache of its local tiles' windows
// (entries past the cache are read from cu_seqlens).
__device__ __forceinline__ void local_window(const int2 *cache, const int *cu, int k, int w, int *s0,
                                             int *len, int *n16) {
    if (k < kWinCache) {
        const int2 e = cache[k];
        *s0 = e.x;
        *len = e.y;
        *n16 = max(1, (e.y + 15) >> 4);
    } else {
        window_of(cu, w, s0, len, n16);
    }
}

__global__ void __launch_bounds__(kThreads, 1) window_attn_tc_kernel(
    const __grid_constant__ CUtensorMap tm_qkv, __half *__restrict__ out, const int *__restrict__ cu,
    int n_windows, int heads, int d, float scale_log2e, int *status, int v_f16,
    unsigned long long lim, int fault_inject, int T) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    int2 *wcache = reinterpret_cast<int2 *>(sm + kOffWin);
    uint64_t *full = reinterpret_cast<uint64_t *>(sm + kOffBar);
    uint64_t *empty = full + kStages;
    uint64_t *s_full = empty + kStages;  // [2] S of the group's tile in TMEM
    uint64_t *p_full = s_full + kGroups; // [2] P (and fp16 V) in shared memory, S read
    uint64_t *o_full = p_full + kGroups; // [4] O buffer complete
    uint64_t *o_empty = o_full + 4;      // [4] O buffer read out of TMEM
    uint64_t *mma_done = o_empty + 4;
    uint32_t *tslot = reinterpret_cast<uint32_t *>(mma_done + 1);
    int *abort_flag = reinterpret_cast<int *>(tslot + 1);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    pdl_trigger();
    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(full + s, 1);
            mbar_init(empty + s, 1);
        }
        for (int g = 0; g < kGroups; ++g) {
            mbar_init(s_full + g, 1);
            mbar_init(p_full + g, 4);
        }
        for (int b = 0; b < 4; ++b) {
            mbar_init(o_full + b, 1);
            mbar_init(o_empty + b, 4);
        }
        mbar_init(mma_done, 1);
        *abort_flag = 0;
        fence_barrier_init();
        tma_prefetch_desc(&tm_qkv);
    }
    if (warp == 1) {
        tmem_alloc(tslot, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tslot;
    volatile int *abort_v = abort_flag;
    pdl_wait();
    const int n_tiles = n_windows * heads;
    // This CTA's tiles: blockIdx.x + k gridDim.x for k < n_local.
    const int n_local = blockIdx.x < n_tiles ? (n_tiles - 1 - (int)blockIdx.x) / (int)gridDim.x + 1 : 0;
    auto tile_of = [&](int k) { return (int)blockIdx.x + k * (int)gridDim.x; };
    // Every role needs each tile's window: read them from cu_seqlens once, in
    // parallel, instead of one dependent global load per tile and role.
    for (int k = threadIdx.x; k < min(n_local, kWinCache); k += kThreads) {
        const int w = tile_of(k) / heads;
        const int a = cu[w];
        wcache[k] = make_int2(a, cu[w + 1] - a);
    }
    __syncthreads();

    if (warp == 0) {
        if (lane == 0) {
            // ------------------------------------------------ TMA producer --
            uint32_t issued = 0, parity = 0;
            bool ok = true;
            for (int k = 0; k < n_local; ++k) {
                const int t = tile_of(k), w = t / heads, h = t - w * heads;
                const int s = k % kStages;
                const uint32_t use = (uint32_t)(k / kStages);
                if (k >= kStages && !mbar_wait(empty + s, (use - 1) & 1u, abort_v, lim)) {
                    ok = false;
                    break;
                }
                if (fault_inject && blockIdx.x == 0 && k == 0) continue;  // never filled
                uint8_t *st = sm + s * kStageBytes;
                int s0, len, n16;
                local_window(wcache, cu, k, w, &s0, &len, &n16);
                mbar_arrive_expect_tx(full + s, kStageBytes);
                tma_load_2d(st, &tm_qkv, full + s, h * kHd, s0);
                tma_load_2d(st + kTileBytes, &tm_qkv, full + s, d + h * kHd, s0);
                tma_load_2d(st + 2 * kTileBytes, &tm_qkv, full + s, 2 * d + h * kHd, s0);
                issued |= 1u << s;
                parity = (parity & ~(1u << s)) | ((use & 1u) << s);
            }
            if (!ok) signal_abort(status, abort_v);
            // The last load issued on every stage has landed before the block
            // may exit (one shared time limit for all of them).
            const uint64_t t0 = global_timer_ns();
            for (int s = 0; s < kStages; ++s) {
                const uint64_t used = global_timer_ns() - t0;
                if ((issued >> s & 1u) && used < lim)
                    mbar_wait(full + s, parity >> s & 1u, nullptr, lim - used);
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            // -------------------------------------------------- MMA issuer --
            constexpr uint32_t idesc_o = idesc_f16_f32_bmn(kTile, kHd);
            bool ok = true;
            // S of local tile k into its group's S buffer.
            auto issue_s = [&](int k) -> bool {
                int s0, len, n16;
                local_window(wcache, cu, k, tile_of(k) / heads, &s0, &len, &n16);
                const int s = k % kStages;
                if (!mbar_wait(full + s, (uint32_t)(k / kStages) & 1u, abort_v, lim)) return false;
                tc_fence_after();
                uint8_t *st = sm + s * kStageBytes;
                const uint32_t idesc_s = idesc_bf16_f32(kTile, 16 * n16);
#pragma unroll
                for (int q = 0; q < kHd / 16; ++q)
                    tc_mma_bf16(tmem + (k & 1) * kTile, smem_desc_sw128(st) + 2 * q,
                                smem_desc_sw128(st + kTileBytes) + 2 * q, idesc_s, q > 0);
                tc_commit(s_full + (k & 1));
                return true;
            };
            for (int k = 0; ok && k < n_local && k < kGroups; ++k) ok = issue_s(k);
            for (int k = 0; ok && k < n_local; ++k) {
                int s0, len, n16;
                local_window(wcache, cu, k, tile_of(k) / heads, &s0, &len, &n16);
                const int g = k & 1, ob = 2 * g + ((k >> 1) & 1);
                uint8_t *st = sm + (k % kStages) * kStageBytes;
                // P of tile k is in shared memory (and S has been read); the O
                // buffer was last drained by the epilogue of the group's tile k - 4.
                if (!mbar_wait(p_full + g, (uint32_t)(k >> 1) & 1u, abort_v, lim) ||
                    (k >= 4 && !mbar_wait(o_empty + ob, (uint32_t)((k >> 2) - 1) & 1u, abort_v, lim))) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                // O = P V: k-step j covers keys 16 j .. 16 j + 16.
                for (int j = 0; j < n16; ++j)
                    tc_mma_bf16(tmem + kColO + ob * kHd,
                                smem_desc_sw128(st + (j >> 2) * kTileBytes) + 2 * (j & 3),
                                smem_desc_sw128_mn(st + 2 * kTileBytes + j * 16 * 128), idesc_o,
                                j > 0);
                tc_commit(o_full + ob);
                tc_commit(empty + k % kStages);  // Q | K (now P) and V free once O is done
                // The group's next S reuses the S buffer this tile's softmax has read.
                if (k + kGroups < n_local && !issue_s(k + kGroups)) ok = false;
            }
            if (!ok) signal_abort(status, abort_v);
            // Every MMA this thread issued has completed before TMEM is released.
            tc_commit(mma_done);
            mbar_wait(mma_done, 0, nullptr, lim);
        }
    } else {
        // --------------------------------------------- softmax, epilogue --
        const int cw = warp - 2, g = cw >> 2;
        const int quad = warp & 3;  // TMEM lanes [32 quad, 32 quad + 32)
        const int row = quad * 32 + lane;
        const int gtid = (cw & 3) * 32 + lane;  // 0 .. 127 inside the group
        const uint32_t trow = tmem + ((uint32_t)(quad * 32) << 16);
        bool fail = false;
        // Epilogue of local tile kk: O / rowsum to fp16 rows.
        auto epilogue = [&](int kk, float inv) {
            const int t = tile_of(kk), w = t / heads, h = t - w * heads;
            int s0, len, n16;
            local_window(wcache, cu, kk, w, &s0, &len, &n16);
            const int ob = 2 * g + ((kk >> 1) & 1);
            fail = fail || !mbar_wait_warp(o_full + ob, (uint32_t)(kk >> 2) & 1u, abort_v, lim);
            if (fail) return;
            tc_fence_after();
            const bool active = quad * 32 < len;
            __half *dst = out + (size_t)(s0 + row) * d + h * kHd;
            if (active) {
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {  // 32 output columns per TMEM load
                    float o[32];
                    tmem_ld32(trow + kColO + ob * kHd + 32 * hh, o);
                    tc_wait_ld();
                    if (row < len && AUT_IN_BOUNDS(s0 + row < T, status)) {
#pragma unroll
                        for (int q = 0; q < 4; ++q) {
                            uint32_t pk[4];
#pragma unroll
                            for (int e = 0; e < 4; ++e)
                                pk[e] = pack_f16x2_sat(o[q * 8 + 2 * e] * inv, o[q * 8 + 2 * e + 1] * inv);
                            *reinterpret_cast<uint4 *>(dst + 32 * hh + q * 8) =
                                make_uint4(pk[0], pk[1], pk[2], pk[3]);
                        }
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(o_empty + ob);
        };
        int prev_k = -1;
        float prev_inv = 0.f;
        for (int k = g; k < n_local; k += kGroups) {
            int s0, len, n16;
            local_window(wcache, cu, k, tile_of(k) / heads, &s0, &len, &n16);
            const int s = k % kStages;
            uint8_t *st = sm + s * kStageBytes;
            const uint32_t t_s = trow + g * kTile;
            const bool active = quad * 32 < len;  // warp-uniform: some rows are valid
            const int nch = (len + 31) >> 5;      // 32-key chunks holding the window's keys
            fail = fail || !mbar_wait_warp(s_full + g, (uint32_t)(k >> 1) & 1u, abort_v, lim);
            if (fail) break;
            tc_fence_after();
            // Row max over the window's keys: the scores come out of TMEM 64 keys
            // (two 32-key chunks) per wait.
            float mx = -INFINITY;
            if (active) {
#pragma unroll
                for (int c0 = 0; c0 < 4; c0 += 2) {
                    if (c0 < nch) {
                        float v[2][32];
                        tmem_ld32(t_s + c0 * 32, v[0]);
                        if (c0 + 1 < nch) tmem_ld32(t_s + c0 * 32 + 32, v[1]);
                        tc_wait_ld();
#pragma unroll
                        for (int u = 0; u < 2; ++u) {
                            const int key0 = (c0 + u) * 32;
                            if (key0 + 32 <= len) {
#pragma unroll
                                for (int j = 0; j < 32; ++j) mx = fmaxf(mx, v[u][j]);
                            } else if (key0 < len) {  // the chunk holding the window's end
#pragma unroll
                                for (int j = 0; j < 32; ++j)
                                    if (key0 + j < len) mx = fmaxf(mx, v[u][j]);
                            }
                        }
                    }
                }
            }
            // P = exp2(s * scale - max * scale); zero past the window's end.
            const float neg = -mx * scale_log2e;
            float sum = 0.f;
            if (active) {
#pragma unroll
                for (int c0 = 0; c0 < 4; c0 += 2) {
                    if (c0 < nch) {
                        float v[2][32];
                        tmem_ld32(t_s + c0 * 32, v[0]);
                        if (c0 + 1 < nch) tmem_ld32(t_s + c0 * 32 + 32, v[1]);
                        tc_wait_ld();
#pragma unroll
                        for (int u = 0; u < 2; ++u) {
                            const int key0 = (c0 + u) * 32;
                            if (key0 < len) {
                                const bool whole = key0 + 32 <= len;
#pragma unroll
                                for (int q = 0; q < 4; ++q) {  // 8 keys = one 16-byte chunk of P
                                    uint32_t ph[4];
#pragma unroll
                                    for (int e = 0; e < 4; ++e) {
                                        const int j = q * 8 + 2 * e;
                                        float p0 = ex2_approx(fmaf(v[u][j], scale_log2e, neg));
                                        float p1 = ex2_approx(fmaf(v[u][j + 1], scale_log2e, neg));
                                        if (!whole) {
                                            p0 = key0 + j < len ? p0 : 0.f;
                                            p1 = key0 + j + 1 < len ? p1 : 0.f;
                                        }
                                        sum += p0 + p1;
                                        __half2 hp = __floats2half2_rn(p0, p1);
                                        ph[e] = *reinterpret_cast<uint32_t *>(&hp);
                                    }
                                    *reinterpret_cast<uint4 *>(st + p_chunk_offset(row, key0 / 8 + q)) =
                                        make_uint4(ph[0], ph[1], ph[2], ph[3]);
                                }
                            }
                        }
                    }
                }
            }
            const float inv = 1.f / sum;
            // V rows the MMA reads, to fp16 in place (same positions, so the
            // swizzled layout is kept).  Reading V directly needs the TMA
            // barrier's phase observed by this thread (it completed long ago).
            if (!v_f16) {
                fail = !mbar_wait_warp(full + s, (uint32_t)(k / kStages) & 1u, abort_v, lim);
                if (fail) break;
                uint4 *vv = reinterpret_cast<uint4 *>(st + 2 * kTileBytes);
                for (int i = gtid; i < n16 * 128; i += 128) {
                    uint4 u = vv[i];
                    uint32_t *e = reinterpret_cast<uint32_t *>(&u);
#pragma unroll
                    for (int m = 0; m < 4; ++m) {
                        const float2 f =
                            __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&e[m]));
                        e[m] = pack_f16x2_sat(f.x, f.y);
                    }
                    vv[i] = u;
                }
            }
            fence_proxy_async_smem();  // P and V (generic-proxy writes) visible to the MMA
            tc_fence_before();         // S reads done before the next S overwrites it
            __syncwarp();
            if (lane == 0) mbar_arrive(p_full + g);
            // The group's previous tile's output, while O of this tile and S of
            // the group's next tile compute.
            if (prev_k >= 0) epilogue(prev_k, prev_inv);
            prev_k = k;
            prev_inv = inv;
        }
        if (!fail && prev_k >= 0) epilogue(prev_k, prev_inv);
        if (fail && lane == 0) signal_abort(status, abort_v);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

}  // namespace

cudaError_t launch_window_attention_tc(const void *qkv, void *out, const int *cu_dev, int n_windows,
                                       int d, int heads, int T, int *status, cudaStream_t st,
                                       bool v_f16, unsigned long long timeout_ns, int fault_inject) {
    if (n_windows <= 0) return cudaSuccess;
    if (d / heads != kHd || T <= 0) return cudaErrorInvalidValue;
    const cudaError_t e = smem_attr_once<window_attn_tc_kernel>(kSmem);
    if (e != cudaSuccess) return e;
    CUtensorMap tm;
    const uint64_t dims[2] = {(uint64_t)3 * d, (uint64_t)T};
    const uint64_t strides[1] = {(uint64_t)3 * d * 2};
    const uint32_t box[2] = {kHd, kTile};
    if (!make_tensor_map_bf16_sw128(&tm, 2, qkv, dims, strides, box)) return cudaErrorInvalidValue;
    const float scale_log2e = 1.4426950408889634f / 8.0f;  // log2(e) / sqrt(64)
    const long tiles = (long)n_windows * heads;
    const int grid = (int)std::min<long>(tiles, (long)sm_count_cached());
    return launch_pdl(window_attn_tc_kernel, dim3(grid), dim3(kThreads), kSmem, st, 1, tm,
                      static_cast<__half *>(out), cu_dev, n_windows, heads, d, scale_log2e, status,
                      v_f16 ? 1 : 0, timeout_ns ? timeout_ns : 4000ull * 1000ull * 1000ull,
                      fault_inject, T);
}

}  // namespace aut
