// conv1 + GELU of the stem on the tensor cores, written into conv2's phase planes.
//
// conv1 is Conv2d(1 -> C, 3x3, stride 2, padding 1) on one chunk's mel tile
// [128 bins, 100 frames] (aut_encoder page, AuTEncoder.frontend; openarchlab
// "1A . AuT Audio Encoder", section 3), then GELU.  Per output position it is a
// 9-term dot product plus the bias for each of the C channels: a GEMM with
// M = positions, N = C, K = 10 (9 taps and a constant 1 against the bias,
// zero-padded to one K = 16 step).  The products run on the tensor cores
// (bf16 x bf16, fp32 accumulate, exact products); the CUDA cores only apply
// GELU, which is most of conv1's arithmetic.
//
// Tiles follow the layout conv2 reads: the output position (h, w) belongs to
// phase plane (h & 1, w & 1) at plane row (h >> 1) + 1 and column (w >> 1) + 1
// (row 0 and column 0 are conv2's zero padding).  One tile is 5 plane rows x
// 25 columns of one plane of one chunk (125 positions in M = 128 rows; the
// last tile of a plane has 2 rows), so its output is one TMA store box per
// 32-channel block, [32 channels, 25 columns, 5 rows], straight into the plane.
//
// The accumulator is split in two halves, channels [0, 256) and [256, C), each
// its own MMA (N <= 256) with its own full/empty barriers, so the next tile's
// first half is computed while the epilogue still drains this tile's second.
//
// Block = 20 warps:
//   warp 0     writes each tile's A operand (9 taps per row, 128-byte swizzle)
//              into one of two buffers, from the chunk's mel tile
//   warps 18-19  stage the CTA's chunks' mel tiles in shared memory (zero
//              outside the mel bins and past the request's valid frames), two
//              buffers, many loads in flight per lane
//   warp 1     allocates tensor memory and issues the tile's MMAs (one per
//              accumulator half) from one thread
//   warps 2-17 epilogue: four groups of four warps (one per TMEM lane
//              quadrant) take every fourth 32-channel block; per block, GELU
//              to bf16 into a 64-byte-swizzled staging box, then one TMA
//              store.  They also write the zero borders of both plane sets
//              for the chunks whose first tile their CTA owns.
// Tiles are split into contiguous ranges, one per CTA (a CTA meets at most a
// few chunks).  Every mbarrier wait is bounded; on time-out the kernel records
// AUT_ERR_TIMEOUT and stops.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "aut_internal.h"
#include "aut_kernels.h"
#include "aut_ptx.cuh"

namespace aut {

namespace {

using bf16 = __nv_bfloat16;

constexpr int kRowsPerTile = 5;                                       // plane rows per tile
constexpr int kBlocksPerPlane = (kP1Rows - 1 + kRowsPerTile - 1) / kRowsPerTile;  // 7
constexpr int kTilesPerChunk = 4 * kBlocksPerPlane;                   // 28
constexpr int kTailRows = (kP1Rows - 1) - (kBlocksPerPlane - 1) * kRowsPerTile;  // 2
constexpr int kPlaneCols = kP1Cols - 1;                               // 25 output columns
constexpr int kMelRowsPad = kMelBins + 2;                             // bins -1 .. 128
constexpr int kMelColsPad = 104;                                      // frames -1 .. 102
constexpr int kMaxC = 512;
constexpr int kHalfN = 256;       // accumulator half: channels [0, 256) and [256, C)
constexpr int kGroups = 4;        // epilogue groups of four warps
constexpr int kEpiWarps = 4 * kGroups;
constexpr int kThreadsC1 = 32 * (2 + kEpiWarps + 2);
constexpr int kLoaderWarp0 = 2 + kEpiWarps;  // the last two warps stage mel tiles
constexpr int kBoxBytes = 128 * 64;          // 128 positions x 32 channels
constexpr int kMelBytes = ((kMelRowsPad * kMelColsPad * 2 + 1023) / 1024) * 1024;
constexpr int kOffB = 0;                                   // C rows x 128 B
constexpr int kOffA = kOffB + kMaxC * 128;                 // 2 x 16 KB
constexpr int kOffOut = kOffA + 2 * 16384;                 // 4 groups x 2 boxes x 8 KB
constexpr int kOffMel = kOffOut + kGroups * 2 * kBoxBytes;  // 2 x bf16 [130][104]
constexpr int kOffBar = kOffMel + 2 * kMelBytes;
constexpr int kSmemC1 = 1024 + kOffBar + 128;

static_assert(kP1Rows - 1 == 32 && kPlaneCols == 25, "conv1 output 64 x 50");
static_assert(kRowsPerTile * kPlaneCols <= 128, "a tile fits M = 128");
static_assert(kSmemC1 <= 227 * 1024, "shared memory of one CTA");
static_assert(kThreadsC1 <= 1024 && kEpiWarps % 4 == 0, "whole lane quadrants per group");
static_assert(kBoxBytes % 512 == 0 && kOffOut % 1024 == 0, "64-byte swizzle boxes on 512-byte atoms");
static_assert(kOffA % 1024 == 0 && kOffMel % 16 == 0, "128-byte swizzle operands on 1024-byte atoms");
static_assert((kGroups & (kGroups - 1)) == 0, "groups take blocks by a power-of-two stride");

AUT_DEV void bar_named(int id, int count) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}
AUT_DEV void tma_store_3d(const CUtensorMap *m, const void *src, int c0, int c1, int c2) {
    asm volatile("cp.async.bulk.tensor.3d.global.shared::cta.bulk_group [%0, {%2, %3, %4}], [%1];" ::"l"(
                     reinterpret_cast<uint64_t>(m)),
                 "r"(smem_addr(src)), "r"(c0), "r"(c1), "r"(c2)
                 : "memory");
}

__device__ __forceinline__ void c1_abort(int *status, volatile int *abort) {
    if (status) atomicCAS(status, 0, kDevTimeout);
    *abort = 1;
}

__global__ void __launch_bounds__(kThreadsC1, 1) conv1_tc_kernel(
    const __grid_constant__ CUtensorMap tm_out5, const __grid_constant__ CUtensorMap tm_out2,
    const bf16 *__restrict__ feats, int T_max, const int4 *__restrict__ chunks, int chunk_base,
    int n_chunks, const bf16 *__restrict__ w, const bf16 *__restrict__ b,
    bf16 *__restrict__ planes, int plane_rows, bf16 *__restrict__ planes2, int plane2_rows, int C,
    int *status, unsigned long long lim) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint8_t *sB = sm + kOffB;
    uint8_t *sA = sm + kOffA;
    uint8_t *sOut = sm + kOffOut;
    uint8_t *mel_base = sm + kOffMel;
    uint64_t *a_full = reinterpret_cast<uint64_t *>(sm + kOffBar);  // [2]
    uint64_t *a_empty = a_full + 2;                                  // [2]
    uint64_t *t_full = a_empty + 2;   // [2] per accumulator half
    uint64_t *t_empty = t_full + 2;   // [2] count 16: every epilogue warp has read the half
    uint64_t *mma_done = t_empty + 2;
    uint64_t *mel_full = mma_done + 1;   // [2] count 2: both loader warps have staged the tile
    uint64_t *mel_empty = mel_full + 2;  // [2] the builder is done with the tile
    uint32_t *tslot = reinterpret_cast<uint32_t *>(mel_empty + 2);
    int *abort_flag = reinterpret_cast<int *>(tslot + 1);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n0 = C < kHalfN ? C : kHalfN;  // channels in the first accumulator half
    const int n_half = C > kHalfN ? 2 : 1;

    pdl_trigger();
    if (threadIdx.x == 0) {
        for (int i = 0; i < 2; ++i) {
            mbar_init(a_full + i, 1);
            mbar_init(a_empty + i, 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(t_full + i, 1);
            mbar_init(t_empty + i, kEpiWarps);
        }
        mbar_init(mma_done, 1);
        for (int i = 0; i < 2; ++i) {
            mbar_init(mel_full + i, 2);
            mbar_init(mel_empty + i, 1);
        }
        *abort_flag = 0;
        fence_barrier_init();
        tma_prefetch_desc(&tm_out5);
        tma_prefetch_desc(&tm_out2);
    }
    if (warp == 1) {
        tmem_alloc(tslot, 512);
        tmem_relinquish();
    }
    // B operand: per channel the 9 conv1 weights, then the bias (against A's
    // constant 1), then zeros: 16 bf16 in the first 32 bytes of a 128-byte
    // swizzled row.
    for (int r = threadIdx.x; r < C; r += kThreadsC1) {
        uint32_t wd[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            const int t0 = 2 * k, t1 = 2 * k + 1;
            const bf16 z = __float2bfloat16_rn(0.f);
            __nv_bfloat162 p2;
            p2.x = t0 < 9 ? w[r * 9 + t0] : t0 == 9 ? b[r] : z;
            p2.y = t1 < 9 ? w[r * 9 + t1] : t1 == 9 ? b[r] : z;
            wd[k] = *reinterpret_cast<uint32_t *>(&p2);
        }
        uint8_t *row = sB + r * 128;
        *reinterpret_cast<uint4 *>(row + ((0 ^ (r & 7)) << 4)) = make_uint4(wd[0], wd[1], wd[2], wd[3]);
        *reinterpret_cast<uint4 *>(row + ((1 ^ (r & 7)) << 4)) = make_uint4(wd[4], wd[5], wd[6], wd[7]);
    }
    fence_proxy_async_smem();  // B (generic writes) visible to the MMA
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tslot;
    volatile int *abort_v = abort_flag;
    pdl_wait();  // the plan upload (chunk table) is complete

    const int total = n_chunks * kTilesPerChunk;
    const int t_begin = (int)((long)total * blockIdx.x / gridDim.x);
    const int t_end = (int)((long)total * (blockIdx.x + 1) / gridDim.x);
    const int n_my = t_end - t_begin;
    const int cl_first = t_begin / kTilesPerChunk;  // the CTA's chunks: cl_first + k
    const int n_cl = n_my > 0 ? (t_end - 1) / kTilesPerChunk - cl_first + 1 : 0;

    if (warp == 0) {
        // ------------------------------------------------ A operand builder --
        int cur = -1;
        const bf16 *mel = nullptr;
        bool ok = true;
        for (int t = 0; t < n_my && ok; ++t) {
            const int gt = t_begin + t, cl = gt / kTilesPerChunk, r = gt - cl * kTilesPerChunk;
            const int plane = r / kBlocksPerPlane, rb = r - plane * kBlocksPerPlane;
            const int ph = plane >> 1, pw = plane & 1;
            if (cl != cur) {
                const int k = cl - cl_first;
                // Done with the previous chunk's mel tile; wait for this one.
                if (k > 0 && lane == 0) mbar_arrive(mel_empty + ((k - 1) & 1));
                if (!mbar_wait_warp(mel_full + (k & 1), (uint32_t)(k >> 1) & 1u, abort_v, lim)) {
                    ok = false;
                    break;
                }
                mel = reinterpret_cast<const bf16 *>(mel_base + (k & 1) * kMelBytes);
                cur = cl;
            }
            const int buf = t & 1;
            if (t >= 2 && !mbar_wait_warp(a_empty + buf, (uint32_t)((t >> 1) - 1) & 1u, abort_v, lim)) {
                ok = false;
                break;
            }
            uint8_t *a = sA + buf * 16384;
            const int rows = rb == kBlocksPerPlane - 1 ? kTailRows : kRowsPerTile;
            for (int m = lane; m < 128; m += 32) {
                uint32_t xd[8] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
                if (m < rows * kPlaneCols) {
                    const int i = rb * kRowsPerTile + m / kPlaneCols, j = m % kPlaneCols;
                    const int h = 2 * i + ph, wo = 2 * j + pw;
                    // tap (kh, kw) reads bin 2h + kh - 1 and frame 2wo + kw - 1,
                    // i.e. padded row 2h + kh and padded column 2wo + kw
                    const bf16 *base = mel + (2 * h) * kMelColsPad + 2 * wo;
                    bf16 x[10];
#pragma unroll
                    for (int kh = 0; kh < 3; ++kh)
#pragma unroll
                        for (int kw = 0; kw < 3; ++kw) x[kh * 3 + kw] = base[kh * kMelColsPad + kw];
                    x[9] = __float2bfloat16_rn(1.f);  // against the bias
#pragma unroll
                    for (int k = 0; k < 5; ++k) {
                        __nv_bfloat162 p2;
                        p2.x = x[2 * k];
                        p2.y = x[2 * k + 1];
                        xd[k] = *reinterpret_cast<uint32_t *>(&p2);
                    }
                }
                uint8_t *row = a + m * 128;
                *reinterpret_cast<uint4 *>(row + ((0 ^ (m & 7)) << 4)) = make_uint4(xd[0], xd[1], xd[2], xd[3]);
                *reinterpret_cast<uint4 *>(row + ((1 ^ (m & 7)) << 4)) = make_uint4(xd[4], xd[5], xd[6], xd[7]);
            }
            fence_proxy_async_smem();  // A (generic writes) visible to the MMA
            __syncwarp();
            if (lane == 0) mbar_arrive(a_full + buf);
        }
        if (!ok && lane == 0) c1_abort(status, abort_v);
    } else if (warp >= kLoaderWarp0) {
        // -------------------------------------------------- mel tile loaders --
        // Chunk k's mel tile, bins -1 .. 128 and frames -1 .. 102, into buffer
        // k & 1: zero outside the bins and past the request's valid frames.
        // Each lane keeps 16 loads in flight before it stores them.
        const int lt = (warp - kLoaderWarp0) * 32 + lane;  // 0 .. 63
        constexpr int kElems = kMelRowsPad * kMelColsPad, kBatch = 16;
        bool ok = true;
        for (int k = 0; k < n_cl && ok; ++k) {
            if (k >= 2 && !mbar_wait_warp(mel_empty + (k & 1), (uint32_t)((k >> 1) - 1) & 1u, abort_v, lim)) {
                ok = false;
                break;
            }
            bf16 *mel = reinterpret_cast<bf16 *>(mel_base + (k & 1) * kMelBytes);
            const int4 ci = chunks[chunk_base + cl_first + k];
            const bf16 *src = feats + ((size_t)ci.x * kMelBins) * T_max + ci.y;
            for (int i0 = lt; i0 < kElems; i0 += 64 * kBatch) {
                bf16 vals[kBatch];
#pragma unroll
                for (int u = 0; u < kBatch; ++u) {
                    const int idx = i0 + 64 * u;
                    const int rr = idx / kMelColsPad, cc = idx - rr * kMelColsPad;
                    const int bin = rr - 1, fr = cc - 1;
                    vals[u] = (idx < kElems && bin >= 0 && bin < kMelBins && fr >= 0 && fr < ci.z)
                                  ? src[(size_t)bin * T_max + fr]
                                  : __float2bfloat16_rn(0.f);
                }
#pragma unroll
                for (int u = 0; u < kBatch; ++u)
                    if (i0 + 64 * u < kElems) mel[i0 + 64 * u] = vals[u];
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(mel_full + (k & 1));  // release: the stores above
        }
        if (!ok && lane == 0) c1_abort(status, abort_v);
    } else if (warp == 1) {
        if (lane == 0) {
            // -------------------------------------------------- MMA issuer --
            // Half h: channels [h * 256, h * 256 + N_h), N_h a multiple of 32.
            const uint32_t idesc0 = idesc_bf16_f32(128, n0);
            const uint32_t idesc1 = idesc_bf16_f32(128, n_half > 1 ? C - kHalfN : 32);
            bool ok = true;
            for (int t = 0; t < n_my && ok; ++t) {
                const int buf = t & 1;
                if (!mbar_wait(a_full + buf, (uint32_t)(t >> 1) & 1u, abort_v, lim)) {
                    ok = false;
                    break;
                }
                const uint64_t a_desc = smem_desc_sw128(sA + buf * 16384);
                for (int h = 0; h < n_half; ++h) {
                    // The epilogue has read this half of the previous tile.
                    if (t > 0 && !mbar_wait(t_empty + h, (uint32_t)(t - 1) & 1u, abort_v, lim)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    tc_mma_bf16(tmem + h * kHalfN, a_desc, smem_desc_sw128(sB + h * kHalfN * 128),
                                h ? idesc1 : idesc0, 0);
                    tc_commit(t_full + h);
                }
                if (ok) tc_commit(a_empty + buf);
            }
            if (!ok) c1_abort(status, abort_v);
            tc_commit(mma_done);
            mbar_wait(mma_done, 0, nullptr, lim);
        }
    } else {
        // ------------------------------------------------------- epilogue --
        const int ew = warp - 2;                     // 0 .. 15
        const int quad = warp & 3, grp = ew >> 2;   // TMEM lane quadrant, group
        const int row = quad * 32 + lane;            // TMEM lane = position of the tile
        const uint32_t t_row = tmem + ((uint32_t)(quad * 32) << 16);
        const bool issuer = (ew & 3) == 0 && lane == 0;
        const int n_blk = C / 32, n_blk0 = n0 / 32;  // 32-channel blocks: all, first half
        uint8_t *my_out = sOut + grp * 2 * kBoxBytes;
        uint32_t stored = 0;  // boxes this group has stored (group-uniform)
        // Warp-uniform; false once a wait of this warp has given up.  A warp that
        // gives up raises the abort and then still walks every remaining block
        // with its group, skipping its waits, TMEM loads and stores, so that no
        // warp of the group is left at a group barrier (which has no time limit).
        bool ok = true;
        const int gtid = ew * 32 + lane;  // 0 .. 511
        for (int t = 0; t < n_my; ++t) {
            const int gt = t_begin + t, cl = gt / kTilesPerChunk, r = gt - cl * kTilesPerChunk;
            const int plane = r / kBlocksPerPlane, rb = r - plane * kBlocksPerPlane;
            if (r == 0 && ok) {
                // This chunk's zero borders: row 0 and column 0 of its four conv2
                // input planes, and of conv3's input planes (conv2's output) row 0,
                // column 0 and, in odd-column planes, the missing last column.
                const int c16 = C / 8;  // 16-byte pieces per pixel
                const size_t r1 = (size_t)cl * kP1Rows;
                for (int idx = gtid; idx < 4 * (kP1Cols + kP1Rows - 1) * c16; idx += 32 * kEpiWarps) {
                    const int pix = idx / c16, q = idx - pix * c16;
                    const int pl = pix / (kP1Cols + kP1Rows - 1), e = pix - pl * (kP1Cols + kP1Rows - 1);
                    const size_t prow = (size_t)pl * plane_rows + r1 + (e < kP1Cols ? 0 : e - kP1Cols + 1);
                    const int col = e < kP1Cols ? e : 0;
                    if (!AUT_IN_BOUNDS(prow < (size_t)4 * plane_rows, status)) continue;
                    reinterpret_cast<uint4 *>(planes + (prow * kP1Cols + col) * C)[q] = make_uint4(0u, 0u, 0u, 0u);
                }
                const size_t r2 = (size_t)cl * kP2Rows;
                constexpr int kB2 = kP2Cols + 2 * (kP2Rows - 1);  // row 0, column 0, last column
                for (int idx = gtid; idx < 4 * kB2 * c16; idx += 32 * kEpiWarps) {
                    const int pix = idx / c16, q = idx - pix * c16;
                    const int pl = pix / kB2, e = pix - pl * kB2;
                    size_t prow;
                    int col;
                    if (e < kP2Cols) {
                        prow = r2;
                        col = e;
                    } else if (e < kP2Cols + kP2Rows - 1) {
                        prow = r2 + (e - kP2Cols + 1);
                        col = 0;
                    } else {
                        if (!(pl & 1)) continue;
                        prow = r2 + (e - kP2Cols - (kP2Rows - 1) + 1);
                        col = kP2Cols - 1;
                    }
                    prow += (size_t)pl * plane2_rows;
                    if (!AUT_IN_BOUNDS(prow < (size_t)4 * plane2_rows, status)) continue;
                    reinterpret_cast<uint4 *>(planes2 + (prow * kP2Cols + col) * C)[q] = make_uint4(0u, 0u, 0u, 0u);
                }
            }
            const bool tail = rb == kBlocksPerPlane - 1;
            const bool live = quad * 32 < (tail ? kTailRows : kRowsPerTile) * kPlaneCols;  // warp-uniform
            const int out_row = plane * plane_rows + cl * kP1Rows + 1 + rb * kRowsPerTile;
            for (int h = 0; h < n_half; ++h) {
                if (ok && !mbar_wait_warp(t_full + h, (uint32_t)t & 1u, abort_v, lim)) {
                    ok = false;
                    if (lane == 0) c1_abort(status, abort_v);
                }
                tc_fence_after();
                // This group's blocks of the half: every fourth, counted from block 0.
                const int b_lo = h ? n_blk0 : 0, b_hi = h ? n_blk : n_blk0;
                for (int bk = b_lo + ((grp - b_lo) & (kGroups - 1)); bk < b_hi; bk += kGroups) {
                    const int c0 = 32 * bk;
                    uint8_t *box = my_out + (stored & 1u) * kBoxBytes;
                    // The store issued from this box two blocks ago has read it.
                    if (issuer && stored >= 2) bulk_wait_read_1();
                    bar_named(1 + grp, 128);
                    if (live && ok) {  // a quadrant past the tile's positions is never stored
                        float v[32];
                        tmem_ld32(t_row + c0, v);
                        tc_wait_ld();
                        uint32_t pk[16];
#pragma unroll
                        for (int j = 0; j < 32; j += 2) {
                            const float2 g = gelu_fast2(make_float2(v[j], v[j + 1]));
                            pk[j / 2] = pack_bf16x2(g.x, g.y);
                        }
                        // 64-byte rows, 64-byte swizzle: the 16-byte chunk j of row m
                        // sits at chunk j ^ ((m >> 1) & 3).
                        uint8_t *rp = box + row * 64;
#pragma unroll
                        for (int j = 0; j < 4; ++j)
                            *reinterpret_cast<uint4 *>(rp + ((j ^ ((row >> 1) & 3)) << 4)) =
                                make_uint4(pk[4 * j], pk[4 * j + 1], pk[4 * j + 2], pk[4 * j + 3]);
                    }
                    fence_proxy_async_smem();
                    bar_named(1 + grp, 128);
                    if (issuer && ok) {
                        tma_store_3d(tail ? &tm_out2 : &tm_out5, box, c0, 1, out_row);
                        bulk_commit();
                    }
                    ++stored;
                }
                // Every TMEM read of this half is done: the next tile's MMA may write it.
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(t_empty + h);
            }
        }
        if (issuer) bulk_wait_read_all();  // the staged boxes are read before the block exits
    }
    tc_fence_before();
    __syncwarp();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

}  // namespace

bool conv1_tc_supported(int C) { return C % 32 == 0 && C >= 64 && C <= kMaxC; }

cudaError_t launch_conv1_tc(const void *feats, int T_max, const int4 *chunks, int chunk_base,
                            int n_chunks, const void *w, const void *b, void *planes, int plane_rows,
                            void *planes2, int plane2_rows, int C, cudaStream_t st, int *status,
                            unsigned long long timeout_ns) {
    if (n_chunks <= 0) return cudaSuccess;
    if (!conv1_tc_supported(C)) return cudaErrorInvalidValue;
    const cudaError_t e = smem_attr_once<conv1_tc_kernel>(kSmemC1);
    if (e != cudaSuccess) return e;
    // conv2's input planes as [4 * plane_rows rows][kP1Cols columns][C]: boxes of
    // 32 channels x 25 columns x 5 (or 2) rows, 64-byte swizzle.
    CUtensorMap tm5, tm2;
    const uint64_t dims[3] = {(uint64_t)C, (uint64_t)kP1Cols, (uint64_t)4 * plane_rows};
    const uint64_t strides[2] = {(uint64_t)C * 2, (uint64_t)kP1Cols * C * 2};
    const uint32_t box5[3] = {32, (uint32_t)kPlaneCols, (uint32_t)kRowsPerTile};
    const uint32_t box2[3] = {32, (uint32_t)kPlaneCols, (uint32_t)kTailRows};
    if (!make_tensor_map_bf16_sw64(&tm5, 3, planes, dims, strides, box5) ||
        !make_tensor_map_bf16_sw64(&tm2, 3, planes, dims, strides, box2))
        return cudaErrorInvalidValue;
    const int tiles = n_chunks * kTilesPerChunk;
    const int grid = std::min(tiles, sm_count_cached());
    return launch_pdl(conv1_tc_kernel, dim3(grid), dim3(kThreadsC1), kSmemC1, st, 1, tm5, tm2,
                      static_cast<const bf16 *>(feats), T_max, chunks, chunk_base, n_chunks,
                      static_cast<const bf16 *>(w), static_cast<const bf16 *>(b),
                      static_cast<bf16 *>(planes), plane_rows, static_cast<bf16 *>(planes2),
                      plane2_rows, C, status, timeout_ns ? timeout_ns : 4000ull * 1000ull * 1000ull);
}

}  // namespace aut
