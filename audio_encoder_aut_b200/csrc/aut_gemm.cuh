// Persistent tcgen05 GEMM for sm_100a: D[M, N] = A[M, K] * B[N, K]^T (bf16 in,
// fp32 accumulate in tensor memory) with fused epilogues.
//
// Every GEMM of the encoder runs through this kernel:
//   - the linear layers (qkv_proj, o_proj, fc1, fc2, proj1, proj2) with bias,
//     bias + GELU, or bias + residual add into the fp32 residual stream;
//   - conv2 and conv3 of the stem as implicit GEMMs: the A operand of filter
//     tap (kh, kw) is a plain rectangle of one stride-2 phase plane of the
//     previous conv's output, so TMA loads it directly (no im2col buffer);
//   - conv_out, whose epilogue adds the chunk's sinusoid row, drops the tokens
//     past the chunk's valid length and writes each kept row to its packed
//     position (token packing fused into the GEMM).
//
// Block = 10 warps: warp 0 issues TMA loads into a STAGES-deep shared-memory
// ring, warp 1 owns the tensor-memory allocation and issues tcgen05.mma from
// one thread, warps 2-9 drain the accumulator (tcgen05.ld) and run the
// epilogue (two warps per 32-lane TMEM quadrant).  Two accumulators in tensor memory let the epilogue of one tile
// overlap the MMAs of the next.  Tiles are 128 x BN x 64 (bf16, 128-byte
// swizzle); the grid is persistent (one CTA per SM, tiles strided by gridDim).
// Every mbarrier wait is bounded: on time-out the kernel records
// AUT_ERR_TIMEOUT in the status word, stops all roles, waits for its own copies
// and MMAs in flight, frees tensor memory and returns.
#pragma once

#include "aut_kernels.h"
#include "aut_ptx.cuh"

namespace aut {

constexpr int kTokensPerChunkDev = 13;  // tokens out of one 100-frame chunk
constexpr int kEpilogueWarps = 8;
constexpr int kGemmThreads = 64 + 32 * kEpilogueWarps;  // producer warp, MMA warp, epilogue

// Epilogue codes (GemmEpilogue) are declared in aut_kernels.h.

struct GemmArgs {
    int M, N;
    int f16;  // A and B are fp16 (1) or bf16 (0)
    int num_m_tiles, num_n_tiles, num_k_blocks;
    // implicit-GEMM convolution operand (conv = 1)
    int conv;
    int conv_rows;     // virtual plane rows per M tile
    int conv_cols;     // output columns per virtual row
    int conv_vrows;    // virtual rows per chunk: output rows + 1 spare
    int conv_cblocks;  // 64-channel blocks per filter tap
    int conv_chunks;   // chunks in this group
    // epilogue
    int epi;
    const __nv_bfloat16 *bias;  // [N] or nullptr
    void *out;
    size_t out_elems;  // elements of the output buffer (bounds checks of debug builds)
    int ldo;
    int C;               // conv channels (conv epilogues)
    int dst_plane_rows;  // rows of one destination phase plane (kEpiConvPlanes)
    int dst_chunk_rows;  // destination plane rows per chunk, zero row included
    int dst_cols;        // destination plane columns, zero column included
    const int4 *chunks;  // chunk records {request, frame0, valid_frames, token0}
    int chunk_base;      // global index of the group's first chunk (kEpiPackTokens)
    const float *pos;    // sinusoid table [13][N] or nullptr (kEpiPackTokens)
    // failure reporting
    int *status;
    unsigned long long timeout_ns;
    int fault_inject;
    // Epilogue stores through shared memory and TMA (tmC): plain row-major
    // outputs (kEpiBf16, kEpiBf16Gelu, kEpiResidF32, kEpiF32) whose per-warp
    // column range is a whole number of 128-byte pieces.
    int tma_out;
    // bf16 epilogues: output columns from here on are written as fp16 instead
    // (the V part of qkv for the tensor-core attention); a multiple of 64.
    int f16_col;
};

// BN: tile width of one MMA (N).  CG: CTAs per MMA (1, or 2 for a CTA pair
// whose MMA is M = 256: each CTA holds 128 rows of A and BN / 2 rows of B).
// A tile wider than one MMA (BN > 256) is two MMAs of BN / 2 per K step into
// one accumulator of BN columns: the A operand then serves twice the columns
// per byte an SM takes in, and the second accumulator (which would hide a
// tile's drain behind the next tile's MMAs) no longer fits in tensor memory.
template <int BN, int CG>
struct GemmCfg {
    static constexpr int BM = 128, BK = 64;
    static constexpr int NSPLIT = BN > 256 ? 2 : 1;  // MMAs per K step
    static constexpr int MMA_N = BN / NSPLIT;
    static constexpr int ACCS = NSPLIT == 1 ? 2 : 1;  // accumulators in tensor memory
    static constexpr int A_BYTES = BM * BK * 2;
    static constexpr int B_ROWS = BN / CG;
    static constexpr int B_SPLIT_ROWS = MMA_N / CG;  // B rows per MMA in this CTA
    static constexpr int B_BYTES = B_ROWS * BK * 2;
    static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
    // Output staging for the TMA-store epilogue: two boxes of 32 rows x 128
    // bytes per epilogue warp (128-byte-swizzled), used alternately so that one
    // piece's store drains while the next piece is computed; only for tile
    // widths whose half is a whole number of 32-column fp32 pieces (no other
    // width can use it, and shared memory left unallocated serves as L1 cache).
    static constexpr int STAGING_BYTES = (BN / 2) % 32 == 0 ? kEpilogueWarps * 2 * 4096 : 0;
    static constexpr int BAR_BYTES = 384;
    static constexpr int SMEM_LIMIT = 232448;  // dynamic shared memory per block on sm_100
    static constexpr int STAGES_FIT =
        (SMEM_LIMIT - 1024 - STAGING_BYTES - BAR_BYTES) / STAGE_BYTES;
    static constexpr int STAGES = STAGES_FIT > 8 ? 8 : STAGES_FIT;
    static constexpr int TMEM_COLS = (ACCS * BN <= 32)    ? 32
                                     : (ACCS * BN <= 64)  ? 64
                                     : (ACCS * BN <= 128) ? 128
                                     : (ACCS * BN <= 256) ? 256
                                                          : 512;
    static constexpr int SMEM_BYTES =
        1024 /*alignment slack*/ + STAGES * STAGE_BYTES + STAGING_BYTES + BAR_BYTES;
    static_assert(STAGES >= 3, "at least three operand stages");
    static_assert(MMA_N % 16 == 0 && MMA_N >= 16 && MMA_N <= 256 && ACCS * BN <= 512, "UMMA N");
    static_assert(B_SPLIT_ROWS % 8 == 0, "each CTA holds whole 8-row swizzle atoms of B");
    static_assert(A_BYTES % 1024 == 0 && B_BYTES % 1024 == 0, "swizzle atoms stay aligned");
};

AUT_DEV void gemm_signal_abort(const GemmArgs &args, volatile int *abort_flag) {
    if (args.status) atomicCAS(args.status, 0, kDevTimeout);
    *abort_flag = 1;
}

AUT_DEV int stem_tokens_dev(int v) {
    v = v > 0 ? (v + 1) / 2 : 0;
    v = v > 0 ? (v + 1) / 2 : 0;
    return v > 0 ? (v + 1) / 2 : 0;
}

// Converts 16 fp32 values to bf16 and stores them (32 contiguous bytes).
AUT_DEV void store_bf16x16(__nv_bfloat16 *p, const float (&v)[16]) {
    uint4 a, b;
    a.x = pack_bf16x2(v[0], v[1]);
    a.y = pack_bf16x2(v[2], v[3]);
    a.z = pack_bf16x2(v[4], v[5]);
    a.w = pack_bf16x2(v[6], v[7]);
    b.x = pack_bf16x2(v[8], v[9]);
    b.y = pack_bf16x2(v[10], v[11]);
    b.z = pack_bf16x2(v[12], v[13]);
    b.w = pack_bf16x2(v[14], v[15]);
    reinterpret_cast<uint4 *>(p)[0] = a;
    reinterpret_cast<uint4 *>(p)[1] = b;
}

// The same as fp16 (saturating at +-65504).
AUT_DEV void store_f16x16(__nv_bfloat16 *p, const float (&v)[16]) {
    uint4 a, b;
    a.x = pack_f16x2_sat(v[0], v[1]);
    a.y = pack_f16x2_sat(v[2], v[3]);
    a.z = pack_f16x2_sat(v[4], v[5]);
    a.w = pack_f16x2_sat(v[6], v[7]);
    b.x = pack_f16x2_sat(v[8], v[9]);
    b.y = pack_f16x2_sat(v[10], v[11]);
    b.z = pack_f16x2_sat(v[12], v[13]);
    b.w = pack_f16x2_sat(v[14], v[15]);
    reinterpret_cast<uint4 *>(p)[0] = a;
    reinterpret_cast<uint4 *>(p)[1] = b;
}

AUT_DEV void add_bias16(float (&v)[16], const __nv_bfloat16 *bias, int n0) {
    if (!bias) return;
    const uint4 *bp = reinterpret_cast<const uint4 *>(bias + n0);
    const uint4 b0 = __ldg(bp), b1 = __ldg(bp + 1);
    const __nv_bfloat162 *h0 = reinterpret_cast<const __nv_bfloat162 *>(&b0);
    const __nv_bfloat162 *h1 = reinterpret_cast<const __nv_bfloat162 *>(&b1);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        float2 f0 = __bfloat1622float2(h0[i]);
        float2 f1 = __bfloat1622float2(h1[i]);
        v[2 * i] += f0.x;
        v[2 * i + 1] += f0.y;
        v[8 + 2 * i] += f1.x;
        v[8 + 2 * i + 1] += f1.y;
    }
}

template <int BN, int CG>
__global__ void __launch_bounds__(kGemmThreads, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                   const __grid_constant__ CUtensorMap tmC, const GemmArgs args) {
    using Cfg = GemmCfg<BN, CG>;
    constexpr int STAGES = Cfg::STAGES;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint8_t *sA = smem;
    uint8_t *sB = smem + STAGES * Cfg::A_BYTES;
    uint8_t *staging = smem + STAGES * Cfg::STAGE_BYTES;  // 1024-aligned: whole stages before it
    uint64_t *full = reinterpret_cast<uint64_t *>(staging + Cfg::STAGING_BYTES);
    uint64_t *empty = full + STAGES;
    uint64_t *tfull = empty + STAGES;
    uint64_t *tempty = tfull + 2;
    uint64_t *mma_done = tempty + 2;
    uint64_t *xbar = mma_done + 1;  // [8] per epilogue warp: residual piece landed
    // Even CTA of a pair: the odd CTA has reported how many phases of every
    // stage it loaded (odd_cnt) before exiting its producer loop.
    uint64_t *exit_bar = xbar + kEpilogueWarps;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(exit_bar + 1);
    int *abort_flag = reinterpret_cast<int *>(tmem_slot + 1);
    uint32_t *odd_cnt = reinterpret_cast<uint32_t *>(abort_flag + 1);  // [STAGES]
    int *mma_exit = reinterpret_cast<int *>(odd_cnt + STAGES);  // the MMA issuer left its loop

    pdl_trigger();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = CG == 2 ? cluster_ctarank() : 0;  // 0 issues the MMAs
    const int group = blockIdx.x / CG, n_groups = gridDim.x / CG;
    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(full + s, 1);
            mbar_init(empty + s, 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(tfull + a, 1);
            mbar_init(tempty + a, kEpilogueWarps * CG);
        }
        mbar_init(mma_done, 1);
        for (int w = 0; w < kEpilogueWarps; ++w) mbar_init(xbar + w, 1);
        mbar_init(exit_bar, 1);
        *abort_flag = 0;
        *mma_exit = 0;
        fence_barrier_init();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&tmA);
        tma_prefetch_desc(&tmB);
        if (args.tma_out) tma_prefetch_desc(&tmC);
    }
    if (warp == 1) {
        if constexpr (CG == 2) {
            tmem_alloc_pair(tmem_slot, Cfg::TMEM_COLS);
            tmem_relinquish_pair();
        } else {
            tmem_alloc(tmem_slot, Cfg::TMEM_COLS);
            tmem_relinquish();
        }
    }
    tc_fence_before();
    __syncwarp();
    if constexpr (CG == 2)
        cluster_sync();  // barriers of both CTAs initialised before any remote use
    else
        __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    volatile int *abort_v = abort_flag;
    const int total_tiles = args.num_m_tiles * args.num_n_tiles;
    const uint64_t lim = args.timeout_ns;

    if (warp == 0) {
        if (lane == 0) {
            // ------------------------------------------------ TMA producer --
            // Both CTAs of a pair load their own A rows and B half; the loads of
            // both complete on the even CTA's `full` barrier, which the even CTA
            // arms with the pair's byte count.
            const uint32_t a_bytes =
                args.conv ? 128u * args.conv_rows * args.conv_cols : (uint32_t)Cfg::A_BYTES;
            const uint32_t cta_bytes = a_bytes + Cfg::B_BYTES;  // one CTA's loads per stage
            auto arm = [&](int stage) {
                if (rank == 0) mbar_arrive_expect_tx(full + stage, CG * cta_bytes);
            };
            // Weights (B): k-block kb of the tile whose B rows start at b_row.
            // With two MMAs per K step, this CTA's B rows of each MMA come from
            // their own place in the weights (one box each, B_SPLIT_ROWS rows).
            auto load_b = [&](int stage, int kb, int b_row) {
#pragma unroll
                for (int h = 0; h < Cfg::NSPLIT; ++h) {
                    uint8_t *b_dst = sB + stage * Cfg::B_BYTES + h * Cfg::B_SPLIT_ROWS * 128;
                    const int row = b_row + h * Cfg::MMA_N;
                    if (!args.conv) {
                        if constexpr (CG == 2)
                            tma_load_2d_pair(b_dst, &tmB, map_to_rank(full + stage, 0), kb * 64, row);
                        else
                            tma_load_2d(b_dst, &tmB, full + stage, kb * 64, row);
                    } else {
                        const int tap = kb / args.conv_cblocks;
                        const int cb = kb - tap * args.conv_cblocks;
                        if constexpr (CG == 2)
                            tma_load_3d_pair(b_dst, &tmB, map_to_rank(full + stage, 0), cb * 64, tap,
                                             row);
                        else
                            tma_load_3d(b_dst, &tmB, full + stage, cb * 64, tap, row);
                    }
                }
            };
            // Activations (A): k-block kb of the tile at 128-row slot m_slot.
            auto load_a = [&](int stage, int kb, int m_slot) {
                uint8_t *a_dst = sA + stage * Cfg::A_BYTES;
                if (!args.conv) {
                    if constexpr (CG == 2)
                        tma_load_2d_pair(a_dst, &tmA, map_to_rank(full + stage, 0), kb * 64,
                                         m_slot * 128);
                    else
                        tma_load_2d(a_dst, &tmA, full + stage, kb * 64, m_slot * 128);
                } else {
                    const int tap = kb / args.conv_cblocks;
                    const int cb = kb - tap * args.conv_cblocks;
                    const int kh = tap / 3, kw = tap - 3 * (tap / 3);
                    // tap kh reads input row 2i + kh - 1: phase 1 for kh in {0, 2},
                    // phase 0 for kh = 1; plane row i (kh = 0) or i + 1 (kh = 1, 2)
                    // counting the leading zero row.  Same for kw along columns.
                    const int plane = (kh == 1 ? 0 : 2) + (kw == 1 ? 0 : 1);
                    const int dh = kh == 0 ? 0 : 1, dw = kw == 0 ? 0 : 1;
                    const int vrow = m_slot * args.conv_rows + dh;
                    if constexpr (CG == 2)
                        tma_load_4d_pair(a_dst, &tmA, map_to_rank(full + stage, 0), cb * 64, dw,
                                         vrow, plane);
                    else
                        tma_load_4d(a_dst, &tmA, full + stage, cb * 64, dw, vrow, plane);
                }
            };
            pdl_wait();  // the previous kernel's outputs (this GEMM's A) are complete
            int stage = 0;
            uint32_t phase = 0;
            uint32_t cnt[STAGES];  // phases of each stage this CTA has loaded
#pragma unroll
            for (int s = 0; s < STAGES; ++s) cnt[s] = 0;
            bool ok = true, skip = args.fault_inject != 0 && blockIdx.x == 0;
            for (int tile = group; ok && tile < total_tiles; tile += n_groups) {
                const int n_blk = tile % args.num_n_tiles, m_blk = tile / args.num_n_tiles;
                const int m_slot = m_blk * CG + (int)rank;  // this CTA's 128-row slot
                const int b_row = n_blk * BN + (int)rank * Cfg::B_SPLIT_ROWS;
                for (int kb = 0; kb < args.num_k_blocks; ++kb) {
                    if (!mbar_wait(empty + stage, phase ^ 1u, abort_v, lim)) {
                        ok = false;
                        break;
                    }
                    if (skip) {
                        skip = false;  // injected fault: this stage is never filled
                    } else {
                        arm(stage);
                        load_b(stage, kb, b_row);
                        load_a(stage, kb, m_slot);
#pragma unroll
                        for (int s = 0; s < STAGES; ++s) cnt[s] += s == stage ? 1u : 0u;
                    }
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            if (!ok) gemm_signal_abort(args, abort_v);
            // Before the block may exit, the last phase loaded into every stage
            // has landed.  A pair's loads all count on the even CTA's barriers,
            // and the odd CTA leaves only through the cluster barrier at the end,
            // which the even CTA reaches after these waits.  After a failure the
            // two producers may have stopped one phase apart on a stage: the odd
            // CTA reports its counts, and the even CTA completes the odd half of
            // a phase the odd CTA never loaded, or arms a phase only the odd CTA
            // loaded.  One shared time limit bounds all the waits.
            uint64_t t0 = global_timer_ns();
            auto left = [&]() -> uint64_t {
                const uint64_t used = global_timer_ns() - t0;
                return used < lim ? lim - used : 0;
            };
            if constexpr (CG == 2) {
                if (rank == 1) {
#pragma unroll
                    for (int s = 0; s < STAGES; ++s)
                        st_shared_cluster_u32(map_to_rank(odd_cnt + s, 0), cnt[s]);
                    mbar_arrive_cluster(map_to_rank(exit_bar, 0));
                } else {
                    // Settle phases only once the MMA issuer has stopped consuming
                    // them, so that a phase completed here is never read as data.
                    // The issuer leaves its loop within one wait limit of a
                    // failure; the bound here is well past that, so this spin
                    // cannot run out first and settle a phase it still waits on.
                    volatile int *mx = mma_exit;
                    while (!*mx && global_timer_ns() - t0 < 4 * lim)
                        __nanosleep(128);  // the last tile's MMAs and drain use the issue slots
                    t0 = global_timer_ns();
                    const bool got = mbar_wait_cluster(exit_bar, 0, left());
#pragma unroll
                    for (int s = 0; s < STAGES; ++s) {
                        const uint32_t ce = cnt[s], co = got ? odd_cnt[s] : cnt[s];
                        if (ce > 0 && co + 1 == ce) mbar_complete_tx(full + s, cta_bytes);
                        if (ce > 0 && left() > 0) mbar_wait(full + s, (ce - 1) & 1u, nullptr, left());
                        if (co == ce + 1) {
                            mbar_arrive_expect_tx(full + s, cta_bytes);
                            if (left() > 0) mbar_wait(full + s, ce & 1u, nullptr, left());
                        }
                    }
                }
            } else {
#pragma unroll
                for (int s = 0; s < STAGES; ++s)
                    if (cnt[s] > 0 && left() > 0) mbar_wait(full + s, (cnt[s] - 1) & 1u, nullptr, left());
            }
        }
    } else if (warp == 1) {
        if (lane == 0 && rank == 0) {
            // -------------------------------------------------- MMA issuer --
            const uint32_t idesc = args.f16 ? idesc_f16_f32(128 * CG, Cfg::MMA_N)
                                            : idesc_bf16_f32(128 * CG, Cfg::MMA_N);
            constexpr uint16_t kPair = 0x3;
            int stage = 0, it = 0;
            uint32_t phase = 0;
            bool ok = true;
            for (int tile = group; ok && tile < total_tiles; tile += n_groups, ++it) {
                const int acc = it % Cfg::ACCS;
                const uint32_t acc_phase = (uint32_t)(it / Cfg::ACCS) & 1u;
                // Wait for the epilogue to have drained the accumulator (the
                // phase before the first use counts as complete).
                if (!mbar_wait(tempty + acc, acc_phase ^ 1u, abort_v, lim)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + acc * BN;
                for (int kb = 0; kb < args.num_k_blocks; ++kb) {
                    if (!mbar_wait(full + stage, phase, abort_v, lim)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint64_t a_desc = smem_desc_sw128(sA + stage * Cfg::A_BYTES);
                    // A convolution's last channel block of each tap may be partly
                    // past C (zero fill): only its K steps that hold channels run.
                    int ksteps = 4;
                    if (args.conv) {
                        const int cb = kb % args.conv_cblocks;
                        const int left = args.C - cb * 64;
                        if (left < 64) ksteps = (left + 15) >> 4;
                    }
#pragma unroll
                    for (int h = 0; h < Cfg::NSPLIT; ++h) {
                        const uint64_t b_desc = smem_desc_sw128(sB + stage * Cfg::B_BYTES +
                                                                h * Cfg::B_SPLIT_ROWS * 128);
                        const uint32_t d = d_tmem + h * Cfg::MMA_N;
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk) {  // K = 16 per MMA: +32 bytes in the row
                            if (kk >= ksteps) break;
                            const uint32_t accumulate = (kb | kk) != 0;
                            if constexpr (CG == 2)
                                tc_mma_bf16_pair(d, a_desc + 2 * kk, b_desc + 2 * kk, idesc,
                                                 accumulate);
                            else
                                tc_mma_bf16(d, a_desc + 2 * kk, b_desc + 2 * kk, idesc, accumulate);
                        }
                    }
                    if constexpr (CG == 2)
                        tc_commit_pair(empty + stage, kPair);
                    else
                        tc_commit(empty + stage);
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (!ok) break;
                if constexpr (CG == 2)
                    tc_commit_pair(tfull + acc, kPair);
                else
                    tc_commit(tfull + acc);
            }
            if (!ok) gemm_signal_abort(args, abort_v);
            *reinterpret_cast<volatile int *>(mma_exit) = 1;
            // Every MMA this thread issued has completed before TMEM is released.
            if constexpr (CG == 2)
                tc_commit_pair(mma_done, 0x1);
            else
                tc_commit(mma_done);
            mbar_wait(mma_done, 0, nullptr, lim);
        }
    } else {
        // ------------------------------------------------------- epilogue --
        // Eight warps: TMEM lane quadrant (warp % 4) x column half.  A residual
        // add is acc + (x + bias) on every path, so that a row's result does not
        // depend on the tile shape its launch happens to use.
        pdl_wait();  // the residual and the output buffers belong to the previous kernel
        const int quad = warp & 3;  // TMEM lanes [32 quad, 32 quad + 32)
        const int half = (warp - 2) >> 2;
        const int r = quad * 32 + lane;
        constexpr int NC = BN / 16;
        const bool resid = args.epi == kEpiResidF32;
        // Single tile per CTA: the residual (x + bias) goes to accumulator 1
        // while the MMAs fill accumulator 0; the drain adds the two.
        const bool resid_once = Cfg::ACCS == 2 && resid && args.tma_out && total_tiles <= n_groups;
        // Several tiles per CTA: the drain brings each residual piece in by TMA
        // (into the staging box it then stores from) and adds it there.
        const bool resid_drain = resid && args.tma_out && !resid_once;
        uint64_t *my_xbar = xbar + (warp - 2);
        uint32_t xph = 0;        // phase of my_xbar
        bool x_pending = false;  // lane 0: a residual load has not been waited for
        // Residual piece (32 rows x 32 fp32) of `tile` at column offset `col`
        // into this warp's staging box; lane 0 only.
        uint8_t *const my_boxes = staging + (warp - 2) * 8192;  // two 4 KB boxes
        // Stores this warp has issued (warp-uniform); a piece fills box piece & 1,
        // so the most recent store, the only one wait_group.read 1 leaves
        // running, always reads the other box.
        uint32_t piece = 0;
        auto load_x = [&](int tile, int col, uint8_t *box) {
            const int m0 = ((tile / args.num_n_tiles) * CG + (int)rank) * 128 + quad * 32;
            bulk_wait_read_all();  // every earlier store has read its box
            mbar_arrive_expect_tx(my_xbar, 4096);
            tma_load_2d(box, &tmC, my_xbar,
                        (tile % args.num_n_tiles) * BN + half * (BN / 2) + col, m0);
            x_pending = true;
        };
        bool ok = true;
        const uint32_t tempty_even = CG == 2 ? map_to_rank(tempty, 0) : 0;
        auto release = [&](int acc) {  // accumulator `acc` may be (re)written by the MMAs
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                if constexpr (CG == 2)
                    mbar_arrive_cluster(tempty_even + acc * 8);
                else
                    mbar_arrive(tempty + acc);
            }
        };
        // Where this thread's accumulator row of `tile` goes.
        auto locate = [&](int tile, bool &valid, size_t &dst_row, int &pos_row) {
            const int m_blk = (tile / args.num_n_tiles) * CG + (int)rank;  // 128-row slot
            valid = true;
            dst_row = 0;
            pos_row = 0;
            if (args.conv) {
                const int vr_local = r / args.conv_cols;
                const int j = r - vr_local * args.conv_cols;
                const int vr = m_blk * args.conv_rows + vr_local;
                const int chunk = vr / args.conv_vrows;
                const int i = vr - chunk * args.conv_vrows;
                valid = vr_local < args.conv_rows && i < args.conv_vrows - 1 &&
                        chunk < args.conv_chunks;
                if (args.epi == kEpiConvPlanes) {
                    // conv2 output (row i, col j) -> phase plane ((i&1), (j&1)) of conv3's
                    // input, behind one zero row and one zero column.
                    const int plane = (i & 1) * 2 + (j & 1);
                    const size_t prow = (size_t)plane * args.dst_plane_rows +
                                        (size_t)chunk * args.dst_chunk_rows + (i >> 1) + 1;
                    dst_row = (prow * (size_t)args.dst_cols + (j >> 1) + 1) * (size_t)args.C;
                } else {
                    // conv3 output (mel row f = i, time j) -> token row chunk * 13 + j, column f*C.
                    dst_row = ((size_t)(chunk * args.conv_cols + j) * (args.conv_vrows - 1) + i) *
                              (size_t)args.C;
                }
            } else {
                const int m = m_blk * 128 + r;
                valid = m < args.M;
                if (args.epi == kEpiPackTokens) {
                    const int cl = m / kTokensPerChunkDev;
                    const int t = m - cl * kTokensPerChunkDev;
                    if (valid) {
                        const int4 ci = args.chunks[args.chunk_base + cl];
                        valid = t < stem_tokens_dev(ci.z);
                        dst_row = (size_t)(ci.w + t) * args.ldo;
                    }
                    pos_row = t;
                } else {
                    dst_row = (size_t)m * args.ldo;
                }
            }
        };
        // Single-tile residual GEMMs (TMA-store epilogue): accumulator `acc` <-
        // x + bias over this warp's 32 rows and its half of the columns, so that
        // the drain adds acc + (x + bias).  x comes in by TMA through the warp's
        // two staging boxes, 64 columns (two 128-byte boxes) per round, while
        // the MMAs run.
        auto preload = [&](int tile, int acc) {
            constexpr int HW = BN / 2;
            const int m0 = ((tile / args.num_n_tiles) * CG + (int)rank) * 128 + quad * 32;
            const bool slab = m0 < args.M;  // warp-uniform
            const int n_first = (tile % args.num_n_tiles) * BN + half * HW;
            const uint32_t t_addr = tmem_base + ((uint32_t)(quad * 32) << 16) + acc * BN + half * HW;
#pragma unroll 1
            for (int c0 = 0; c0 < HW; c0 += 64) {
                const int nb = HW - c0 >= 64 ? 2 : 1;  // boxes this round (warp-uniform)
                if (slab && lane == 0) {
                    mbar_arrive_expect_tx(my_xbar, nb * 4096);
                    for (int b = 0; b < nb; ++b)
                        tma_load_2d(my_boxes + b * 4096, &tmC, my_xbar, n_first + c0 + 32 * b, m0);
                    x_pending = true;
                }
                __syncwarp();
                if (slab) {
                    if (!mbar_wait_warp(my_xbar, xph, abort_v, lim)) {
                        ok = false;
                        gemm_signal_abort(args, abort_v);
                        return;
                    }
                    x_pending = false;
                    xph ^= 1u;
                }
                for (int b = 0; b < nb; ++b) {
                    float xr[2][16];
                    const uint8_t *row = my_boxes + b * 4096 + lane * 128;
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        const float4 x4 = slab ? *reinterpret_cast<const float4 *>(
                                                     row + ((j ^ (lane & 7)) << 4))
                                               : make_float4(0.f, 0.f, 0.f, 0.f);
                        float *q = &xr[j >> 2][(j & 3) * 4];
                        q[0] = x4.x;
                        q[1] = x4.y;
                        q[2] = x4.z;
                        q[3] = x4.w;
                    }
                    add_bias16(xr[0], args.bias, n_first + c0 + 32 * b);
                    add_bias16(xr[1], args.bias, n_first + c0 + 32 * b + 16);
                    tmem_st16(t_addr + c0 + 32 * b, xr[0]);
                    tmem_st16(t_addr + c0 + 32 * b + 16, xr[1]);
                }
                // These reads of the boxes come before the next round's TMA writes.
                fence_proxy_async_smem();
                __syncwarp();
            }
            tc_wait_st();
        };

        // Drain through shared memory: this warp's 32 rows x BN / 2 columns go
        // out in pieces of 32 rows x 128 bytes (32 fp32 or 64 bf16 columns),
        // each written to the warp's 128-byte-swizzled staging box and stored
        // by one TMA tile store (whole lines, rows past M clipped by the map).
        auto drain_tma = [&](int tile, uint32_t t_acc) {
            constexpr int HW = BN / 2;
            const bool f32 = args.epi == kEpiResidF32 || args.epi == kEpiF32;
            const int pcols = f32 ? 32 : 64;

            const int m0 = ((tile / args.num_n_tiles) * CG + (int)rank) * 128 + quad * 32;
            const bool slab = m0 < args.M;  // warp-uniform
            const int n_first = (tile % args.num_n_tiles) * BN + half * HW;
            const uint32_t t_res = tmem_base + ((uint32_t)(quad * 32) << 16) + BN + half * HW;
            t_acc += half * HW;
#pragma unroll 1
            for (int p = 0; p < HW / pcols; ++p) {
                uint8_t *stg = my_boxes + (piece & 1u) * 4096;
                uint32_t w[32];  // this row's 128-byte piece as 8 chunks of 4 words
                if (f32) {
                    float v[2][16];
                    tmem_ld16(t_acc + p * pcols, v[0]);
                    tmem_ld16(t_acc + p * pcols + 16, v[1]);
                    if (resid_once) {
                        float r[2][16];
                        tmem_ld16(t_res + p * pcols, r[0]);
                        tmem_ld16(t_res + p * pcols + 16, r[1]);
                        tc_wait_ld();
#pragma unroll
                        for (int i = 0; i < 2; ++i)
#pragma unroll
                            for (int j = 0; j < 16; ++j) v[i][j] += r[i][j];
                    } else {
                        if (resid_drain && slab && p > 0 && lane == 0) load_x(tile, p * pcols, stg);
                        __syncwarp();  // the warp-wide TMEM wait needs every lane here
                        tc_wait_ld();
                        if (!resid) {
                            add_bias16(v[0], args.bias, n_first + p * pcols);
                            add_bias16(v[1], args.bias, n_first + p * pcols + 16);
                        }
                        if (resid_drain && slab) {
                            // + (residual piece from the box + bias): the same order
                            // of additions as the single-tile path, acc + (x + b),
                            // so that a row's result does not depend on how many
                            // tiles its launch has.
                            if (!mbar_wait_warp(my_xbar, xph, abort_v, lim)) {
                                ok = false;
                                gemm_signal_abort(args, abort_v);
                            } else {
                                x_pending = false;
                            }
                            xph ^= 1u;
                            const uint8_t *row = stg + lane * 128;
                            float xr[2][16];
#pragma unroll
                            for (int j = 0; j < 8; ++j) {
                                const float4 x4 = *reinterpret_cast<const float4 *>(
                                    row + ((j ^ (lane & 7)) << 4));
                                float *q = &xr[j >> 2][(j & 3) * 4];
                                q[0] = x4.x;
                                q[1] = x4.y;
                                q[2] = x4.z;
                                q[3] = x4.w;
                            }
                            add_bias16(xr[0], args.bias, n_first + p * pcols);
                            add_bias16(xr[1], args.bias, n_first + p * pcols + 16);
#pragma unroll
                            for (int i = 0; i < 2; ++i)
#pragma unroll
                                for (int j = 0; j < 16; ++j) v[i][j] += xr[i][j];
                        }
                    }
#pragma unroll
                    for (int j = 0; j < 32; ++j) w[j] = __float_as_uint(v[j >> 4][j & 15]);
                } else {
                    const bool as_f16 = n_first + p * pcols >= args.f16_col;
#pragma unroll
                    for (int h = 0; h < 2; ++h) {  // 32 columns at a time
                        float v[2][16];
                        tmem_ld16(t_acc + p * pcols + 32 * h, v[0]);
                        tmem_ld16(t_acc + p * pcols + 32 * h + 16, v[1]);
                        tc_wait_ld();
#pragma unroll
                        for (int i = 0; i < 2; ++i) {
                            add_bias16(v[i], args.bias, n_first + p * pcols + 32 * h + 16 * i);
                            if (args.epi == kEpiBf16Gelu) {
#pragma unroll
                                for (int j = 0; j < 16; j += 2) {
                                    const float2 g = gelu_fast2(make_float2(v[i][j], v[i][j + 1]));
                                    v[i][j] = g.x;
                                    v[i][j + 1] = g.y;
                                }
                            }
#pragma unroll
                            for (int j = 0; j < 8; ++j)
                                w[16 * h + 8 * i + j] =
                                    as_f16 ? pack_f16x2_sat(v[i][2 * j], v[i][2 * j + 1])
                                           : pack_bf16x2(v[i][2 * j], v[i][2 * j + 1]);
                        }
                    }
                }
                // The store issued from this box two pieces ago has read it (the
                // previous piece's store, from the other box, may still run).
                if (lane == 0) bulk_wait_read_1();
                __syncwarp();
                uint8_t *row = stg + lane * 128;
#pragma unroll
                for (int j = 0; j < 8; ++j)  // 16-byte chunk j of this row, 128-byte swizzle
                    *reinterpret_cast<uint4 *>(row + ((j ^ (lane & 7)) << 4)) =
                        make_uint4(w[4 * j], w[4 * j + 1], w[4 * j + 2], w[4 * j + 3]);
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0 && slab) {
                    tma_store_2d(&tmC, stg, n_first + p * pcols, m0);
                    bulk_commit();
                }
                if (slab) ++piece;
                __syncwarp();  // converged again before the next warp-wide TMEM load
            }
        };

        if (resid_once && group < total_tiles) preload(group, 1);
        int it = 0;
        for (int tile = group; tile < total_tiles; tile += n_groups, ++it) {
            const int acc = it % Cfg::ACCS;
            const uint32_t acc_phase = (uint32_t)(it / Cfg::ACCS) & 1u;
            if (args.tma_out && args.bias && (!resid || resid_drain) && lane * 4 < BN / 2)
                prefetch_l1(args.bias + (tile % args.num_n_tiles) * BN + half * (BN / 2) + lane * 4);
            if (resid_drain && lane == 0 &&  // first residual piece lands during the mainloop
                ((tile / args.num_n_tiles) * CG + (int)rank) * 128 + quad * 32 < args.M)
                load_x(tile, 0, my_boxes + (piece & 1u) * 4096);
            __syncwarp();  // lane 0's residual load above is the only divergent step
            if (!mbar_wait_warp(tfull + acc, acc_phase, abort_v, lim)) {
                ok = false;
                break;
            }
            tc_fence_after();
            const int n_blk = tile % args.num_n_tiles;
            bool valid;
            size_t dst_row;
            int pos_row;
            locate(tile, valid, dst_row, pos_row);
            const uint32_t t_addr = tmem_base + ((uint32_t)(quad * 32) << 16) + acc * BN;
            if (args.tma_out) {
                drain_tma(tile, t_addr);
            } else {
#pragma unroll 1
            for (int c0 = half; c0 < NC; c0 += 4) {
                const int c1 = c0 + 2;
                const bool two = c1 < NC;  // warp-uniform
                float v0[16], v1[16];
                __syncwarp();  // lanes past the tile's valid rows skip ahead below
                tmem_ld16(t_addr + c0 * 16, v0);
                if (two) tmem_ld16(t_addr + c1 * 16, v1);
                tc_wait_ld();
                if (!valid) continue;
                float *rp = reinterpret_cast<float *>(args.out) + dst_row;
#pragma unroll
                for (int k = 0; k < 2; ++k) {
                    if (k == 1 && !two) break;
                    float(&v)[16] = k ? v1 : v0;
                    const int n0 = n_blk * BN + (k ? c1 : c0) * 16;
                    const size_t end = dst_row + n0 + (args.epi == kEpiBf16GeluSplit ? args.N : 0) + 16;
                    if (!AUT_IN_BOUNDS(end <= args.out_elems, args.status)) continue;
                    if (!resid) add_bias16(v, args.bias, n0);
                    switch (args.epi) {
                        case kEpiBf16:
                            if (n0 >= args.f16_col)
                                store_f16x16(reinterpret_cast<__nv_bfloat16 *>(args.out) + dst_row + n0, v);
                            else
                                store_bf16x16(reinterpret_cast<__nv_bfloat16 *>(args.out) + dst_row + n0, v);
                            break;
                        case kEpiBf16Gelu:
                        case kEpiConvPlanes:
                        case kEpiConvFlat: {
#pragma unroll
                            for (int i = 0; i < 16; i += 2) {
                                const float2 g = gelu_fast2(make_float2(v[i], v[i + 1]));
                                v[i] = g.x;
                                v[i + 1] = g.y;
                            }
                            store_bf16x16(reinterpret_cast<__nv_bfloat16 *>(args.out) + dst_row + n0, v);
                            break;
                        }
                        case kEpiBf16GeluSplit: {
                            // GELU, then the value as hi + lo bf16 halves [hi | lo] of a 2N row.
                            float lo[16];
#pragma unroll
                            for (int i = 0; i < 16; i += 2) {
                                const float2 g = gelu_fast2(make_float2(v[i], v[i + 1]));
                                v[i] = g.x;
                                v[i + 1] = g.y;
                            }
#pragma unroll
                            for (int i = 0; i < 16; ++i)
                                lo[i] = v[i] - __bfloat162float(__float2bfloat16_rn(v[i]));
                            __nv_bfloat16 *o = reinterpret_cast<__nv_bfloat16 *>(args.out) + dst_row + n0;
                            store_bf16x16(o, v);
                            store_bf16x16(o + args.N, lo);
                            break;
                        }
                        case kEpiResidF32: {  // acc + (x + bias), x read back from the output
                            float r[16];
                            const float4 *xp = reinterpret_cast<const float4 *>(rp + n0);
#pragma unroll
                            for (int q = 0; q < 4; ++q) {
                                const float4 e = xp[q];
                                r[4 * q] = e.x;
                                r[4 * q + 1] = e.y;
                                r[4 * q + 2] = e.z;
                                r[4 * q + 3] = e.w;
                            }
                            add_bias16(r, args.bias, n0);
                            float4 *p = reinterpret_cast<float4 *>(rp + n0);
#pragma unroll
                            for (int q = 0; q < 4; ++q)
                                p[q] = make_float4(v[4 * q] + r[4 * q], v[4 * q + 1] + r[4 * q + 1],
                                                   v[4 * q + 2] + r[4 * q + 2], v[4 * q + 3] + r[4 * q + 3]);
                            break;
                        }
                        case kEpiF32:
                        case kEpiPackTokens: {
                            if (args.epi == kEpiPackTokens && args.pos) {
                                const float4 *pp = reinterpret_cast<const float4 *>(
                                    args.pos + (size_t)pos_row * args.N + n0);
#pragma unroll
                                for (int q = 0; q < 4; ++q) {
                                    const float4 e = __ldg(pp + q);
                                    v[4 * q] += e.x;
                                    v[4 * q + 1] += e.y;
                                    v[4 * q + 2] += e.z;
                                    v[4 * q + 3] += e.w;
                                }
                            }
                            float4 *p = reinterpret_cast<float4 *>(rp + n0);
#pragma unroll
                            for (int q = 0; q < 4; ++q)
                                p[q] = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
                            break;
                        }
                        default:
                            break;
                    }
                }
            }
            }
            release(acc);
        }
        if (!ok && lane == 0) gemm_signal_abort(args, abort_v);
        // The staged stores have read shared memory before the block may exit;
        // their global writes complete with the grid, before any dependent
        // launch passes its griddepcontrol.wait.
        if (args.tma_out && lane == 0) bulk_wait_read_all();
        if (x_pending) mbar_wait(my_xbar, xph, nullptr, lim);  // a residual load in flight lands
        __syncwarp();
    }

    __syncwarp();
    if constexpr (CG == 2) {
        cluster_sync();  // both CTAs done with TMEM and with each other's barriers
        if (warp == 1) {
            tc_fence_after();
            tmem_dealloc_pair(tmem_base, Cfg::TMEM_COLS);
        }
    } else {
        __syncthreads();
        if (warp == 1) {
            tc_fence_after();
            tmem_dealloc(tmem_base, Cfg::TMEM_COLS);
        }
    }
}

}  // namespace aut
