// Host side of the tcgen05 GEMM: TMA tensor maps, tile-width choice, launch.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <mutex>

#include "aut_gemm.cuh"
#include "aut_internal.h"
#include "aut_kernels.h"

namespace aut {

namespace {

using EncodeTiledFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                   const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                   const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault,
                                             &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

// bf16 tensor map (128-byte swizzle unless asked otherwise); dims innermost
// first, strides in bytes for dims 1.., box in elements.  Out-of-range elements
// of a box read as zero.
bool make_map(CUtensorMap *m, int rank, const void *ptr, const cuuint64_t *dims,
              const cuuint64_t *strides, const cuuint32_t *box,
              CUtensorMapDataType dtype = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16,
              CUtensorMapSwizzle swizzle = CU_TENSOR_MAP_SWIZZLE_128B) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const cuuint32_t es[5] = {1, 1, 1, 1, 1};
    return fn(m, dtype, (cuuint32_t)rank, const_cast<void *>(ptr), dims,
              strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool make_map_bf16(CUtensorMap *m, int rank, const void *ptr, const uint64_t *dims,
                   const uint64_t *strides, const uint32_t *box, CUtensorMapSwizzle swizzle) {
    if (rank < 1 || rank > 5) return false;
    cuuint64_t dd[5], ss[4];
    cuuint32_t bb[5];
    for (int i = 0; i < rank; ++i) {
        dd[i] = dims[i];
        bb[i] = box[i];
        if (i + 1 < rank) ss[i] = strides[i];
    }
    return make_map(m, rank, ptr, dd, ss, bb, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, swizzle);
}

}  // namespace

bool make_tensor_map_bf16_sw128(CUtensorMap *m, int rank, const void *ptr, const uint64_t *dims,
                                const uint64_t *strides, const uint32_t *box) {
    return make_map_bf16(m, rank, ptr, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B);
}

bool make_tensor_map_bf16_sw64(CUtensorMap *m, int rank, const void *ptr, const uint64_t *dims,
                               const uint64_t *strides, const uint32_t *box) {
    return make_map_bf16(m, rank, ptr, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_64B);
}

namespace {

int sm_count() { return sm_count_cached(); }

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

template <int BN, int CG>
GemmStatus run(const CUtensorMap &ta, const CUtensorMap &tb, const CUtensorMap &tc,
               const GemmArgs &args,
               cudaStream_t st) {
    using Cfg = GemmCfg<BN, CG>;
    if (smem_attr_once<gemm_tc_kernel<BN, CG>>(Cfg::SMEM_BYTES) != cudaSuccess)
        return GemmStatus::kLaunch;
    const int tiles = args.num_m_tiles * args.num_n_tiles;
    const int groups = std::min(tiles, sm_count() / CG);
    const cudaError_t e = launch_pdl(gemm_tc_kernel<BN, CG>, dim3(groups * CG), dim3(kGemmThreads),
                                     Cfg::SMEM_BYTES, st, CG, ta, tb, tc, args);
    return e == cudaSuccess ? GemmStatus::kOk : GemmStatus::kLaunch;
}

GemmStatus dispatch(int bn, int cg, const CUtensorMap &ta, const CUtensorMap &tb,
                    const CUtensorMap &tc,
                    const GemmArgs &args, cudaStream_t st) {
    if (cg == 2) {
        switch (bn) {
            case 64: return run<64, 2>(ta, tb, tc, args, st);
            case 128: return run<128, 2>(ta, tb, tc, args, st);
            case 192: return run<192, 2>(ta, tb, tc, args, st);
            case 240: return run<240, 2>(ta, tb, tc, args, st);
            case 256: return run<256, 2>(ta, tb, tc, args, st);
            case 480: return run<480, 2>(ta, tb, tc, args, st);  // two N = 240 MMAs per K step
            default: return GemmStatus::kBadShape;
        }
    }
    switch (bn) {
        case 16: return run<16, 1>(ta, tb, tc, args, st);
        case 32: return run<32, 1>(ta, tb, tc, args, st);
        case 64: return run<64, 1>(ta, tb, tc, args, st);
        case 128: return run<128, 1>(ta, tb, tc, args, st);
        case 192: return run<192, 1>(ta, tb, tc, args, st);
        case 240: return run<240, 1>(ta, tb, tc, args, st);
        case 256: return run<256, 1>(ta, tb, tc, args, st);
        default: return GemmStatus::kBadShape;
    }
}

bool pair_ok(int bn) { return bn == 64 || bn == 128 || bn == 192 || bn == 240 || bn == 256; }

// Tile shape for a plain GEMM: the (width, CTAs per MMA) with the fewest waves
// x per-tile time.  Per k-block a tile costs about (BN + 512) column-units:
// the A tile arrives whatever the width, so halving BN saves far less than
// half (measured on B200: a 256 x 128 pair k-block takes ~0.32 us against
// ~0.37 us at 256 x 256).  A CTA pair streams a third less operand data per
// FLOP than a single SM, so it is credited as 4/6 of the single-SM time.
void choose_tile(int M, int N, int sms, bool allow_pair, int *bn_out, int *cg_out) {
    static const int cand[] = {256, 128, 64, 32, 16};
    long best_cost = -1;
    *bn_out = 0;
    *cg_out = 1;
    for (int cg = 1; cg <= 2; ++cg) {
        if (cg == 2 && (!allow_pair || M <= 128)) continue;
        for (int bn : cand) {
            if (N % bn || (cg == 2 && !pair_ok(bn))) continue;
            const long mt = (M + 128 * cg - 1) / (128 * cg);
            const long tiles = mt * (N / bn);
            const long slots = sms / cg;
            const long waves = (tiles + slots - 1) / slots;
            const long cost = waves * (bn + 512) * (cg == 2 ? 4 : 6);
            if (best_cost < 0 || cost < best_cost) {
                best_cost = cost;
                *bn_out = bn;
                *cg_out = cg;
            }
        }
    }
}

}  // namespace

GemmStatus launch_linear(const LinearLaunch &L, cudaStream_t st) {
    if (L.M <= 0) return GemmStatus::kOk;
    if (L.N <= 0 || L.K <= 0 || L.K % 64 || L.N % 16 || !L.a || !L.w || !L.out)
        return GemmStatus::kBadShape;
    if (!aligned16(L.a) || !aligned16(L.w) || !aligned16(L.out) || (L.bias && !aligned16(L.bias)))
        return GemmStatus::kBadShape;
    int bn = 0, cg = 1;
    choose_tile(L.M, L.N, sm_count(), !L.single_cta, &bn, &cg);
    if (!bn) return GemmStatus::kBadShape;
    CUtensorMap ta, tb;
    const cuuint64_t da[2] = {(cuuint64_t)L.K, (cuuint64_t)L.M};
    const cuuint64_t sa[1] = {(cuuint64_t)L.K * 2};
    const cuuint32_t ba[2] = {64, 128};
    const cuuint64_t db[2] = {(cuuint64_t)L.K, (cuuint64_t)L.N};
    const cuuint32_t bb[2] = {64, (cuuint32_t)(bn / cg)};
    // fp16 operands use the same maps: the copies move bytes, and the zero fill
    // of out-of-range rows is zero in both types.
    if (!make_map(&ta, 2, L.a, da, sa, ba) || !make_map(&tb, 2, L.w, db, sa, bb))
        return GemmStatus::kTensorMap;
    GemmArgs args{};
    args.f16 = L.f16 ? 1 : 0;
    args.f16_col = L.f16_col;
    args.M = L.M;
    args.N = L.N;
    args.num_m_tiles = (L.M + 128 * cg - 1) / (128 * cg);
    args.num_n_tiles = L.N / bn;
    args.num_k_blocks = L.K / 64;
    args.conv = 0;
    args.epi = L.epi;
    args.bias = static_cast<const __nv_bfloat16 *>(L.bias);
    args.out = L.out;
    args.out_elems = L.out_elems ? L.out_elems : (size_t)L.M * L.ldo;
    args.ldo = L.ldo;
    args.chunks = L.chunks;
    args.chunk_base = L.chunk_base;
    args.pos = L.pos;
    args.status = L.status;
    args.timeout_ns = L.timeout_ns;
    args.fault_inject = L.fault_inject;
    // Row-major outputs whose per-warp column range (bn / 2) is a whole number
    // of 128-byte pieces leave through shared memory and TMA stores.
    CUtensorMap tc = tb;  // unused unless tma_out
    const bool f32 = L.epi == kEpiResidF32 || L.epi == kEpiF32;
    const bool row_major = f32 || L.epi == kEpiBf16 || L.epi == kEpiBf16Gelu;
    const int pcols = f32 ? 32 : 64;
    if (row_major && (bn / 2) % pcols == 0 && L.ldo >= L.N) {
        const size_t es = f32 ? 4 : 2;
        const cuuint64_t dc[2] = {(cuuint64_t)L.N, (cuuint64_t)L.M};
        const cuuint64_t sc[1] = {(cuuint64_t)L.ldo * es};
        const cuuint32_t bc[2] = {(cuuint32_t)pcols, 32};
        if (!make_map(&tc, 2, L.out, dc, sc, bc,
                      f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16))
            return GemmStatus::kTensorMap;
        args.tma_out = 1;
    }
    return dispatch(bn, cg, ta, tb, tc, args, st);
}

GemmStatus launch_conv_gemm(const ConvLaunch &L, cudaStream_t st) {
    if (L.chunks <= 0) return GemmStatus::kOk;
    const int bn = conv_tile_n(L.C);
    if (!bn || L.rows_per_tile * L.out_cols > 128) return GemmStatus::kBadShape;
    if (!aligned16(L.planes) || !aligned16(L.w_tap) || !aligned16(L.out) || !aligned16(L.bias))
        return GemmStatus::kBadShape;
    const int cg = (!L.single_cta && pair_ok(bn)) ? 2 : 1;
    // C = 480 on CTA pairs: one tile covers all 480 output channels as two
    // N = 240 MMAs per K step, so each SM loads its A tile once for 480
    // channels instead of twice for 240 (the conv mainloop is bound by the
    // operand bytes an SM takes in).
    const int tile_n = (cg == 2 && bn == 240 && L.C == 480) ? 480 : bn;
    const long rows_total = (long)L.chunks * L.chunk_rows;
    CUtensorMap ta, tb;
    const cuuint64_t da[4] = {(cuuint64_t)L.C, (cuuint64_t)L.cols_in, (cuuint64_t)rows_total, 4};
    const cuuint64_t sa[3] = {(cuuint64_t)L.C * 2, (cuuint64_t)L.cols_in * L.C * 2,
                              (cuuint64_t)L.plane_rows_cap * L.cols_in * L.C * 2};
    const cuuint32_t ba[4] = {64, (cuuint32_t)L.out_cols, (cuuint32_t)L.rows_per_tile, 1};
    const cuuint64_t db[3] = {(cuuint64_t)L.C, 9, (cuuint64_t)L.C};
    const cuuint64_t sb[2] = {(cuuint64_t)L.C * 2, (cuuint64_t)9 * L.C * 2};
    const cuuint32_t bb[3] = {64, 1, (cuuint32_t)(bn / cg)};
    if (!make_map(&ta, 4, L.planes, da, sa, ba) || !make_map(&tb, 3, L.w_tap, db, sb, bb))
        return GemmStatus::kTensorMap;
    GemmArgs args{};
    args.f16_col = 1 << 30;
    args.M = (int)rows_total;
    args.N = L.C;
    const long slot_rows = (long)L.rows_per_tile * cg;
    args.num_m_tiles = (int)((rows_total + slot_rows - 1) / slot_rows);
    args.num_n_tiles = L.C / tile_n;
    args.conv = 1;
    args.conv_rows = L.rows_per_tile;
    args.conv_cols = L.out_cols;
    args.conv_vrows = L.chunk_rows;
    args.conv_cblocks = (L.C + 63) / 64;
    args.conv_chunks = L.chunks;
    args.num_k_blocks = 9 * args.conv_cblocks;
    args.epi = L.epi;
    args.bias = static_cast<const __nv_bfloat16 *>(L.bias);
    args.out = L.out;
    args.out_elems = L.out_elems;
    args.C = L.C;
    args.dst_plane_rows = L.dst_plane_rows;
    args.dst_chunk_rows = L.dst_chunk_rows;
    args.dst_cols = L.dst_cols;
    args.status = L.status;
    args.timeout_ns = L.timeout_ns;
    return dispatch(tile_n, cg, ta, tb, tb, args, st);  // no TMA-store epilogue
}

}  // namespace aut
