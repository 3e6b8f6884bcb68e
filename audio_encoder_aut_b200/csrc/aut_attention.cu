// Window attention on the 5th-generation tensor cores, for head_dim 64.
//
// Bidirectional attention inside one cu_seqlens window for one head
// (aut_encoder page, AuTAttention: block-diagonal over the packed windows, no
// cache; openarchlab "1A . AuT Audio Encoder", section 3: non-causal within each
// segment).  A window has at most 128 tokens, so one (window, head) is one
// 128-row tile and the softmax is exact in one pass over the tile.
//
// The kernel is persistent (one CTA per SM) and walks the (window, head)
// tiles with a grid stride, over the windows in the order of an optional
// table (the encoder passes them longest first, so that every CTA gets a
// similar mix of long and short windows).  Warp roles:
//   warp 0     TMA producer: Q, K, V tiles [128 x 64] bf16 (128-byte swizzle)
//              from qkv [T, 3d] into a ring of kStages stages; rows past the
//              window's end are the next window's rows (or zero past T) and
//              are masked below
//   warps 1, 10  MMA issuers, one thread per softmax group: S = Q K^T
//              (M = 128, N = the window length rounded up to 16, K = 64) into
//              the group's S buffer; once the group has written P, O = P V
//              (M = 128, N = 64, K = window length rounded up to 16, fp16
//              inputs, V read MN-major) into one of the group's two O buffers,
//              then S of the group's next tile
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
// full[kStages], empty[kStages], s_full[2], p_full[2], o_full[4], o_empty[4], mma_done[2]
constexpr int kNumBars = 2 * kStages + 2 * kGroups + 4 + 4 + kGroups;
constexpr int kSmem = 1024 + kOffBar + kNumBars * 8 + 16;
constexpr int kComputeWarps = 4 * kGroups;
constexpr int kMmaWarp1 = 2 + kComputeWarps;  // group 1's MMA issuer (group 0's: warp 1)
constexpr int kThreads = 64 + 32 * kComputeWarps + 32;
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

// Local tile k of this CTA: its position in the tile list is
// blockIdx.x + k gridDim.x, which names a window slot (list position / heads)
// and a head.  The window of a slot is wins[slot] when the caller passes the
// length-ordered table, else window `slot` of cu_seqlens.
struct TileGeom {
    int s0, len, n16, h;
};
__device__ __forceinline__ int2 window_at(const int *cu, const int2 *wins, int slot) {
    if (wins) return wins[slot];
    const int a = cu[slot];
    return make_int2(a, cu[slot + 1] - a);
}
// The same from the CTA's shared-memory cache of its local tiles' windows
// (entries past the cache are read from global memory).
__device__ __forceinline__ TileGeom local_tile(const int2 *cache, const int *cu, const int2 *wins,
                                               int heads, int k) {
    const int i = (int)blockIdx.x + k * (int)gridDim.x, slot = i / heads;
    const int2 e = k < kWinCache ? cache[k] : window_at(cu, wins, slot);
    TileGeom t;
    t.s0 = e.x;
    t.len = e.y;
    t.n16 = max(1, (e.y + 15) >> 4);  // the last 16-row step of the MMAs covers the ragged end
    t.h = i - slot * heads;
    return t;
}

__global__ void __launch_bounds__(kThreads, 1) window_attn_tc_kernel(
    const __grid_constant__ CUtensorMap tm_qkv, __half *__restrict__ out, const int *__restrict__ cu,
    const int2 *__restrict__ wins, int n_windows, int heads, int d, float scale_log2e, int *status,
    int v_f16, unsigned long long lim, int fault_inject, int T) {
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
    uint64_t *mma_done = o_empty + 4;    // [2] per MMA issuer
    uint32_t *tslot = reinterpret_cast<uint32_t *>(mma_done + kGroups);
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
        for (int g = 0; g < kGroups; ++g) mbar_init(mma_done + g, 1);
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
    // Every role needs each tile's window: read them once, in parallel,
    // instead of one dependent global load per tile and role.
    for (int k = threadIdx.x; k < min(n_local, kWinCache); k += kThreads)
        wcache[k] = window_at(cu, wins, ((int)blockIdx.x + k * (int)gridDim.x) / heads);
    __syncthreads();

    if (warp == 0) {
        if (lane == 0) {
            // ------------------------------------------------ TMA producer --
            uint32_t issued = 0, parity = 0;
            bool ok = true;
            for (int k = 0; k < n_local; ++k) {
                const int s = k % kStages;
                const uint32_t use = (uint32_t)(k / kStages);
                if (k >= kStages && !mbar_wait(empty + s, (use - 1) & 1u, abort_v, lim)) {
                    ok = false;
                    break;
                }
                if (fault_inject && blockIdx.x == 0 && k == 0) continue;  // never filled
                uint8_t *st = sm + s * kStageBytes;
                const TileGeom tg = local_tile(wcache, cu, wins, heads, k);
                mbar_arrive_expect_tx(full + s, kStageBytes);
                tma_load_2d(st, &tm_qkv, full + s, tg.h * kHd, tg.s0);
                tma_load_2d(st + kTileBytes, &tm_qkv, full + s, d + tg.h * kHd, tg.s0);
                tma_load_2d(st + 2 * kTileBytes, &tm_qkv, full + s, 2 * d + tg.h * kHd, tg.s0);
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
    } else if (warp == 1 || warp == kMmaWarp1) {
        if (lane == 0) {
            // ------------------------------------------------- MMA issuers --
            // One thread per softmax group (warp 1: group 0, kMmaWarp1: group
            // 1), so that neither group's products wait behind the other's
            // barriers.  Group g's tiles go S = Q K^T -> softmax -> O = P V, and
            // S of its next tile reuses the S buffer once the softmax has read
            // it (that is, once P is in).
            const int g = warp == 1 ? 0 : 1;
            constexpr uint32_t idesc_o = idesc_f16_f32_bmn(kTile, kHd);
            bool ok = true;
            auto issue_s = [&](int k) -> bool {
                const int s = k % kStages;
                if (!mbar_wait(full + s, (uint32_t)(k / kStages) & 1u, abort_v, lim)) return false;
                tc_fence_after();
                const TileGeom tg = local_tile(wcache, cu, wins, heads, k);
                uint8_t *st = sm + s * kStageBytes;
                const uint32_t idesc_s = idesc_bf16_f32(kTile, 16 * tg.n16);
#pragma unroll
                for (int q = 0; q < kHd / 16; ++q)
                    tc_mma_bf16(tmem + g * kTile, smem_desc_sw128(st) + 2 * q,
                                smem_desc_sw128(st + kTileBytes) + 2 * q, idesc_s, q > 0);
                tc_commit(s_full + g);
                return true;
            };
            if (g < n_local) ok = issue_s(g);
            for (int k = g; ok && k < n_local; k += kGroups) {
                const int ob = 2 * g + ((k >> 1) & 1);
                // P of tile k is in shared memory (and S has been read); the O
                // buffer was last drained by the epilogue of the group's tile k - 4.
                if (!mbar_wait(p_full + g, (uint32_t)(k >> 1) & 1u, abort_v, lim) ||
                    (k >= 4 && !mbar_wait(o_empty + ob, (uint32_t)((k >> 2) - 1) & 1u, abort_v, lim))) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const TileGeom tg = local_tile(wcache, cu, wins, heads, k);
                uint8_t *st = sm + (k % kStages) * kStageBytes;
                // O = P V: k-step j covers keys 16 j .. 16 j + 16.
                for (int j = 0; j < tg.n16; ++j)
                    tc_mma_bf16(tmem + kColO + ob * kHd,
                                smem_desc_sw128(st + (j >> 2) * kTileBytes) + 2 * (j & 3),
                                smem_desc_sw128_mn(st + 2 * kTileBytes + j * 16 * 128), idesc_o,
                                j > 0);
                tc_commit(o_full + ob);
                tc_commit(empty + k % kStages);  // Q | K (now P) and V free once O is done
                if (k + kGroups < n_local) ok = issue_s(k + kGroups);
            }
            if (!ok) signal_abort(status, abort_v);
            // Every MMA this thread issued has completed before TMEM is released.
            tc_commit(mma_done + g);
            mbar_wait(mma_done + g, 0, nullptr, lim);
        }
    } else {
        // --------------------------------------------- softmax, epilogue --
        const int cw = warp - 2, g = cw >> 2;  // warps 2 .. 2 + kComputeWarps - 1
        const int quad = warp & 3;  // TMEM lanes [32 quad, 32 quad + 32)
        const int row = quad * 32 + lane;
        const int gtid = (cw & 3) * 32 + lane;  // 0 .. 127 inside the group
        const uint32_t trow = tmem + ((uint32_t)(quad * 32) << 16);
        const float2 scale2 = make_float2(scale_log2e, scale_log2e);
        bool fail = false;
        // Epilogue of local tile kk: O / rowsum to fp16 rows.
        auto epilogue = [&](int kk, float inv) {
            const TileGeom tg = local_tile(wcache, cu, wins, heads, kk);
            const int ob = 2 * g + ((kk >> 1) & 1);
            fail = fail || !mbar_wait_warp(o_full + ob, (uint32_t)(kk >> 2) & 1u, abort_v, lim);
            if (fail) return;
            tc_fence_after();
            const bool active = quad * 32 < tg.len;
            __half *dst = out + (size_t)(tg.s0 + row) * d + tg.h * kHd;
            if (active) {
                float o[2][32];  // the row's 64 output columns, one wait
                tmem_ld32(trow + kColO + ob * kHd, o[0]);
                tmem_ld32(trow + kColO + ob * kHd + 32, o[1]);
                tc_wait_ld();
                if (row < tg.len && AUT_IN_BOUNDS(tg.s0 + row < T, status)) {
#pragma unroll
                    for (int hh = 0; hh < 2; ++hh)
#pragma unroll
                        for (int q = 0; q < 4; ++q) {
                            uint32_t pk[4];
#pragma unroll
                            for (int e = 0; e < 4; ++e)
                                pk[e] = pack_f16x2_sat(o[hh][q * 8 + 2 * e] * inv,
                                                       o[hh][q * 8 + 2 * e + 1] * inv);
                            *reinterpret_cast<uint4 *>(dst + 32 * hh + q * 8) =
                                make_uint4(pk[0], pk[1], pk[2], pk[3]);
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
            const TileGeom tg = local_tile(wcache, cu, wins, heads, k);
            const int len = tg.len;
            const int s = k % kStages;
            uint8_t *st = sm + s * kStageBytes;
            const uint32_t t_s = trow + g * kTile;
            const bool active = quad * 32 < len;  // warp-uniform: some rows are valid
            const int nch = (len + 31) >> 5;      // 32-key chunks holding the window's keys
            fail = fail || !mbar_wait_warp(s_full + g, (uint32_t)(k >> 1) & 1u, abort_v, lim);
            if (fail) break;
            tc_fence_after();
            // Scores come out of TMEM two 32-key chunks (64 keys) per wait, into
            // v.  Row max over the window's keys (keys past the end read as
            // -inf), then P = 2^(s scale - max scale), zero past the window's
            // end.  The pair of chunks loaded last for the max is still in v and
            // is exponentiated first, so a window of up to 64 keys is read from
            // TMEM once and a longer one three times instead of four.  Partial
            // maxima and sums run in four independent chains.
            float v[2][32];
            auto load_pair = [&](int c0) {
                tmem_ld32(t_s + c0 * 32, v[0]);
                if (c0 + 1 < nch) tmem_ld32(t_s + c0 * 32 + 32, v[1]);
                tc_wait_ld();
            };
            float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
            auto max_pair = [&](int c0) {
#pragma unroll
                for (int u = 0; u < 2; ++u) {
                    const int key0 = (c0 + u) * 32;
                    if (key0 < len) {
                        if (key0 + 32 > len) {  // the chunk holding the window's end
#pragma unroll
                            for (int j = 0; j < 32; ++j) v[u][j] = key0 + j < len ? v[u][j] : -INFINITY;
                        }
#pragma unroll
                        for (int j = 0; j < 32; j += 8)
#pragma unroll
                            for (int e = 0; e < 4; ++e) m4[e] = fmax3(m4[e], v[u][j + 2 * e], v[u][j + 2 * e + 1]);
                    }
                }
            };
            float2 s4[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                            make_float2(0.f, 0.f)};
            float2 neg2 = make_float2(0.f, 0.f);
            auto exp_pair = [&](int c0) {
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
                                const float2 x = ffma2(make_float2(v[u][j], v[u][j + 1]), scale2, neg2);
                                float2 p = make_float2(ex2_approx(x.x), ex2_approx(x.y));
                                if (!whole) {
                                    p.x = key0 + j < len ? p.x : 0.f;
                                    p.y = key0 + j + 1 < len ? p.y : 0.f;
                                }
                                s4[e] = fadd2(s4[e], p);
                                __half2 hp = __floats2half2_rn(p.x, p.y);
                                ph[e] = *reinterpret_cast<uint32_t *>(&hp);
                            }
                            *reinterpret_cast<uint4 *>(st + p_chunk_offset(row, key0 / 8 + q)) =
                                make_uint4(ph[0], ph[1], ph[2], ph[3]);
                        }
                    }
                }
            };
            if (active) {
                load_pair(0);
                max_pair(0);
                if (nch > 2) {
                    load_pair(2);
                    max_pair(2);
                }
                const float mx = fmaxf(fmax3(m4[0], m4[1], m4[2]), m4[3]);
                neg2 = make_float2(-mx * scale_log2e, -mx * scale_log2e);
                if (nch > 2) {
                    exp_pair(2);
                    load_pair(0);
                }
                exp_pair(0);
            }
            const float2 sum2 = fadd2(fadd2(s4[0], s4[1]), fadd2(s4[2], s4[3]));
            const float inv = 1.f / (sum2.x + sum2.y);
            // V rows the MMA reads, to fp16 in place (same positions, so the
            // swizzled layout is kept).  Reading V directly needs the TMA
            // barrier's phase observed by this thread (it completed long ago).
            if (!v_f16) {
                fail = !mbar_wait_warp(full + s, (uint32_t)(k / kStages) & 1u, abort_v, lim);
                if (fail) break;
                uint4 *vv = reinterpret_cast<uint4 *>(st + 2 * kTileBytes);
                for (int i = gtid; i < tg.n16 * 128; i += 128) {
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
    __syncwarp();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

}  // namespace

cudaError_t launch_window_attention_tc(const void *qkv, void *out, const int *cu_dev, int n_windows,
                                       int d, int heads, int T, int *status, cudaStream_t st,
                                       bool v_f16, unsigned long long timeout_ns, int fault_inject,
                                       const int2 *wins) {
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
                      static_cast<__half *>(out), cu_dev, wins, n_windows, heads, d, scale_log2e,
                      status, v_f16 ? 1 : 0, timeout_ns ? timeout_ns : 4000ull * 1000ull * 1000ull,
                      fault_inject, T);
}

}  // namespace aut
