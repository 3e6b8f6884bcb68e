// Non-GEMM kernels of the encoder: conv1 of the stem, LayerNorm, window
// attention, one-time weight preparation, and small helpers.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "aut_internal.h"
#include "aut_kernels.h"
#include "aut_ptx.cuh"

namespace aut {

using bf16 = __nv_bfloat16;

// ------------------------------------------------------------------ conv1 --
// conv1 of the stem (aut_encoder page, module docstring; openarchlab "1A . AuT
// Audio Encoder", section 3): Conv2d(1 -> C, k3, s2, p1) + GELU over one
// 128 x 100 chunk whose frames at or after the request's length are zero (the
// last chunk of a request is zero-padded to a full chunk, AuTEncoder.frontend).
//
// The 64 x 50 x C output goes to four phase planes P[(h&1)*2 + (w&1)], each
// [33][26][C] per chunk with a zero row 0 and zero column 0 in front, holding
// output (h, w) at (h/2 + 1, w/2 + 1).  conv2's filter tap (kh, kw) then reads
// one plane at a fixed offset, a plain rectangle a TMA box can fetch.
//
// Block (chunk, 8 output rows); each thread computes eight channels (packed
// fp32x2 arithmetic) for a strided set of positions, so a warp writes 32
// consecutive 16-byte channel octets.  This CUDA-core version serves the
// channel counts the tensor-core conv1 (aut_conv1.cu) does not take.
__global__ void __launch_bounds__(256) conv1_kernel(const bf16 *__restrict__ feats, int T_max,
                                                    const int4 *__restrict__ chunks,
                                                    int chunk_base, const bf16 *__restrict__ w,
                                                    const bf16 *__restrict__ b,
                                                    bf16 *__restrict__ planes, int plane_rows,
                                                    bf16 *__restrict__ planes2, int plane2_rows,
                                                    int C, int *status) {
    pdl_trigger();
    pdl_wait();
    const int cl = blockIdx.x, hg = blockIdx.y;
    const int4 ci = chunks[chunk_base + cl];
    __shared__ float xs[17][101];  // mel rows 16 hg - 1 .. 16 hg + 15, frames -1 .. 99
    const bf16 *src = feats + ((size_t)ci.x * kMelBins) * T_max + ci.y;
    // All of this thread's loads are issued before any is used (one round trip).
    constexpr int kTile = 17 * 101, kPer = (kTile + 255) / 256;
    float vals[kPer];
#pragma unroll
    for (int u = 0; u < kPer; ++u) {
        const int idx = threadIdx.x + u * blockDim.x;
        const int rr = idx / 101, cc = idx - rr * 101;
        const int mel = 16 * hg - 1 + rr, fr = cc - 1;
        vals[u] = (idx < kTile && mel >= 0 && mel < kMelBins && fr >= 0 && fr < ci.z)
                      ? __bfloat162float(src[(size_t)mel * T_max + fr])
                      : 0.f;
    }
#pragma unroll
    for (int u = 0; u < kPer; ++u) {
        const int idx = threadIdx.x + u * blockDim.x;
        if (idx < kTile) (&xs[0][0])[idx] = vals[u];
    }
    __syncthreads();

    const int CO = C >> 3;  // channel octets
    const int slices = blockDim.x / CO;
    const int co = threadIdx.x % CO, slice = threadIdx.x / CO;
    if (slice >= slices) return;
    float2 wt[4][9], bias[4];  // channel pairs (2p, 2p + 1) of this thread's octet
#pragma unroll
    for (int p = 0; p < 4; ++p) {
        const int c = 8 * co + 2 * p;
#pragma unroll
        for (int k = 0; k < 9; ++k)
            wt[p][k] = make_float2(__bfloat162float(w[c * 9 + k]), __bfloat162float(w[(c + 1) * 9 + k]));
        bias[p] = make_float2(__bfloat162float(b[c]), __bfloat162float(b[c + 1]));
    }
    const size_t chunk_row0 = (size_t)cl * kP1Rows;
    for (int pos = slice; pos < 8 * kC1Cols; pos += slices) {
        const int hl = pos / kC1Cols, wo = pos - hl * kC1Cols;
        float2 x[9];
#pragma unroll
        for (int kh = 0; kh < 3; ++kh)
#pragma unroll
            for (int kw = 0; kw < 3; ++kw) {
                const float v = xs[2 * hl + kh][2 * wo + kw];
                x[kh * 3 + kw] = make_float2(v, v);
            }
        uint32_t packed[4];
#pragma unroll
        for (int p = 0; p < 4; ++p) {
            float2 a = bias[p];
#pragma unroll
            for (int k = 0; k < 9; ++k) a = ffma2(wt[p][k], x[k], a);
            const float2 g = gelu_fast2(a);
            packed[p] = pack_bf16x2(g.x, g.y);
        }
        const int h = 8 * hg + hl;
        const int plane = (h & 1) * 2 + (wo & 1);
        const size_t row = (size_t)plane * plane_rows + chunk_row0 + (h >> 1) + 1;
        if (!AUT_IN_BOUNDS(row < (size_t)4 * plane_rows && (wo >> 1) + 1 < kP1Cols, status)) continue;
        uint4 *dst = reinterpret_cast<uint4 *>(planes + (row * kP1Cols + (wo >> 1) + 1) * C) + co;
        *dst = make_uint4(packed[0], packed[1], packed[2], packed[3]);
    }
    // Zero column of the plane rows this block owns, and (first block) the zero row.
    for (int idx = slice; idx < 16; idx += slices) {
        const int plane = idx >> 2, r = 4 * hg + (idx & 3) + 1;
        const size_t row = (size_t)plane * plane_rows + chunk_row0 + r;
        reinterpret_cast<uint4 *>(planes + row * kP1Cols * C)[co] = make_uint4(0u, 0u, 0u, 0u);
    }
    if (hg == 0)
        for (int idx = slice; idx < 4 * kP1Cols; idx += slices) {
            const int plane = idx / kP1Cols, col = idx - plane * kP1Cols;
            const size_t row = (size_t)plane * plane_rows + chunk_row0;
            reinterpret_cast<uint4 *>(planes + (row * kP1Cols + col) * C)[co] =
                make_uint4(0u, 0u, 0u, 0u);
        }
    // The zero borders of conv3's input planes (conv2's output, [4][.][kP2Cols][C])
    // for this chunk, which conv2's epilogue never writes: this block clears
    // column 0 and, in odd-column planes, the missing last column of plane rows
    // 2 hg + 1 and 2 hg + 2; the first block also clears row 0.
    const size_t chunk2_row0 = (size_t)cl * kP2Rows;
    for (int idx = slice; idx < 4 * 2 * 2; idx += slices) {
        const int plane = idx >> 2, r = 2 * hg + 1 + ((idx >> 1) & 1), side = idx & 1;
        if (side == 1 && !(plane & 1)) continue;
        const size_t row = (size_t)plane * plane2_rows + chunk2_row0 + r;
        const int col = side ? kP2Cols - 1 : 0;
        if (!AUT_IN_BOUNDS(row < (size_t)4 * plane2_rows, status)) continue;
        reinterpret_cast<uint4 *>(planes2 + (row * kP2Cols + col) * C)[co] = make_uint4(0u, 0u, 0u, 0u);
    }
    if (hg == 0)
        for (int idx = slice; idx < 4 * kP2Cols; idx += slices) {
            const int plane = idx / kP2Cols, col = idx - plane * kP2Cols;
            const size_t row = (size_t)plane * plane2_rows + chunk2_row0;
            reinterpret_cast<uint4 *>(planes2 + (row * kP2Cols + col) * C)[co] =
                make_uint4(0u, 0u, 0u, 0u);
        }
}

// -------------------------------------------------------------- layernorm --
// LayerNorm with bias (cubic.dev "Audio Encoder Component", Transformer Encoder
// Layers), fp32 in, bf16 out; one warp per row, the row held in registers,
// two passes (mean, then centred variance).  With `split`, the output row is
// [hi | lo] (2 d wide): hi = bf16(y), lo = bf16(y - hi), so that a GEMM over
// the doubled K against [W | W] sees y to about 16 significant bits.
constexpr int kLnRowsPerBlock = 8;  // one warp per row

template <int VPL>  // float4 per lane
__global__ void __launch_bounds__(32 * kLnRowsPerBlock) layernorm_kernel(const float *__restrict__ x,
                                                        const bf16 *__restrict__ g,
                                                        const bf16 *__restrict__ bt,
                                                        bf16 *__restrict__ y, int T, int d,
                                                        float eps, int split) {
    pdl_trigger();
    pdl_wait();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int row = blockIdx.x * kLnRowsPerBlock + warp;
    if (row >= T) return;
    const int n4 = d >> 2;
    const float4 *xr = reinterpret_cast<const float4 *>(x + (size_t)row * d);
    const uint2 *gr = reinterpret_cast<const uint2 *>(g);
    const uint2 *br = reinterpret_cast<const uint2 *>(bt);
    float4 v[VPL];
    float s = 0.f;
#pragma unroll
    for (int i = 0; i < VPL; ++i) {
        const int idx = lane + 32 * i;
        if (idx < n4) {
            v[i] = xr[idx];
            s += (v[i].x + v[i].y) + (v[i].z + v[i].w);
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    const float mean = s / d;
    float ss = 0.f;
#pragma unroll
    for (int i = 0; i < VPL; ++i) {
        const int idx = lane + 32 * i;
        if (idx < n4) {
            const float a = v[i].x - mean, b = v[i].y - mean, c = v[i].z - mean, e = v[i].w - mean;
            ss += (a * a + b * b) + (c * c + e * e);
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    const float rstd = rsqrtf(ss / d + eps);
    uint2 *yr = reinterpret_cast<uint2 *>(y + (size_t)row * (split ? 2 * d : d));
#pragma unroll
    for (int i = 0; i < VPL; ++i) {
        const int idx = lane + 32 * i;
        if (idx < n4) {
            const uint2 gg = __ldg(gr + idx), bb = __ldg(br + idx);  // same for every row: L1 hits
            const float2 g0 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&gg.x));
            const float2 g1 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&gg.y));
            const float2 c0 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&bb.x));
            const float2 c1 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&bb.y));
            const float o0 = (v[i].x - mean) * rstd * g0.x + c0.x;
            const float o1 = (v[i].y - mean) * rstd * g0.y + c0.y;
            const float o2 = (v[i].z - mean) * rstd * g1.x + c1.x;
            const float o3 = (v[i].w - mean) * rstd * g1.y + c1.y;
            uint2 o;
            o.x = pack_bf16x2(o0, o1);
            o.y = pack_bf16x2(o2, o3);
            yr[idx] = o;
            if (split) {  // second half of the row: what bf16 rounding left out
                const __nv_bfloat162 h0 = *reinterpret_cast<const __nv_bfloat162 *>(&o.x);
                const __nv_bfloat162 h1 = *reinterpret_cast<const __nv_bfloat162 *>(&o.y);
                const float2 f0 = __bfloat1622float2(h0), f1 = __bfloat1622float2(h1);
                yr[n4 + idx] = make_uint2(pack_bf16x2(o0 - f0.x, o1 - f0.y),
                                          pack_bf16x2(o2 - f1.x, o3 - f1.y));
            }
        }
    }
}

// --------------------------------------------------------- window attention --
AUT_DEV void ldmatrix_x4(uint32_t (&r)[4], const void *p) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(smem_addr(p)));
}
AUT_DEV void ldmatrix_x4_trans(uint32_t (&r)[4], const void *p) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(smem_addr(p)));
}
AUT_DEV void mma_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, "
        "{%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Bidirectional attention inside one cu_seqlens window for one head (aut_encoder
// page, AuTAttention: block-diagonal over the packed windows, no cache; openarchlab
// "1A . AuT Audio Encoder", section 3: non-causal within each segment).  A window
// has at most 128 tokens, so Q, K and V of one (window, head) sit in shared memory
// whole and the softmax is exact in one pass: S = Q K^T (fp32), row max, exp,
// row sum, O = P V / sum.  Keys past the window's length are masked; rows past it
// are computed on zeros and not written.  Each of the 8 warps owns 16-row query
// tiles.  P carries a second bf16 term (hi + lo); the output is fp16, which the
// o_proj GEMM consumes with fp16 weights (11 significant bits).
constexpr int kAttnWarps = 8;

template <int HD>
__global__ void __launch_bounds__(32 * kAttnWarps) window_attn_kernel(const bf16 *__restrict__ qkv,
                                                          __half *__restrict__ out,
                                                          const int *__restrict__ cu, int d,
                                                          float scale_log2e) {
    constexpr int LD = HD + 8;  // padded row: conflict-free ldmatrix
    extern __shared__ __align__(16) uint8_t attn_smem[];
    bf16 *sK = reinterpret_cast<bf16 *>(attn_smem);
    bf16 *sV = sK + kMaxWindowTokens * LD;
    pdl_trigger();
    pdl_wait();
    const int seg = blockIdx.x, h = blockIdx.y;
    const int s0 = cu[seg], len = cu[seg + 1] - s0;
    if (len <= 0) return;
    const int nkt = (len + 15) >> 4;
    const int rows = nkt * 16;
    constexpr int CH = HD / 8;
    // K and V: asynchronous 16-byte copies straight into shared memory, all in
    // flight at once; rows past the window's end are zero-filled (source size 0).
    for (int idx = threadIdx.x; idx < 2 * rows * CH; idx += blockDim.x) {
        const int part = idx / (rows * CH);
        const int rem = idx - part * rows * CH;
        const int r = rem / CH, c = rem - (rem / CH) * CH;
        const bf16 *src =
            qkv + (size_t)(s0 + (r < len ? r : 0)) * 3 * d + (part + 1) * d + h * HD + c * 8;
        bf16 *dst = (part == 0 ? sK : sV) + r * LD + c * 8;
        asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_addr(dst)),
                     "l"(src), "r"(r < len ? 16 : 0)
                     : "memory");
    }
    asm volatile("cp.async.commit_group;" ::: "memory");

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, t = lane & 3;
    // Q: a window has at most 128 tokens = 8 tiles of 16 rows, one per warp; each
    // warp reads its A fragments straight from global memory (rows past the
    // window's end read row len - 1 and are dropped).
    constexpr int KS = HD / 16;
    static_assert(kMaxWindowTokens <= 16 * kAttnWarps, "one query tile per warp");
    const int mt = warp;
    uint32_t qa[KS][4];
    if (mt < nkt) {
        const int r0 = min(mt * 16 + g, len - 1), r1 = min(mt * 16 + g + 8, len - 1);
        const bf16 *q0 = qkv + (size_t)(s0 + r0) * 3 * d + h * HD + 2 * t;
        const bf16 *q1 = qkv + (size_t)(s0 + r1) * 3 * d + h * HD + 2 * t;
#pragma unroll
        for (int kk = 0; kk < KS; ++kk) {
            qa[kk][0] = __ldg(reinterpret_cast<const unsigned int *>(q0 + kk * 16));
            qa[kk][1] = __ldg(reinterpret_cast<const unsigned int *>(q1 + kk * 16));
            qa[kk][2] = __ldg(reinterpret_cast<const unsigned int *>(q0 + kk * 16 + 8));
            qa[kk][3] = __ldg(reinterpret_cast<const unsigned int *>(q1 + kk * 16 + 8));
        }
    }
    asm volatile("cp.async.wait_all;" ::: "memory");
    __syncthreads();

    if (mt < nkt) {
        float s[16][4];
#pragma unroll
        for (int j = 0; j < 16; ++j) s[j][0] = s[j][1] = s[j][2] = s[j][3] = 0.f;
#pragma unroll
        for (int kk = 0; kk < KS; ++kk) {
#pragma unroll
            for (int nt = 0; nt < 8; ++nt) {
                if (nt < nkt) {
                    uint32_t b[4];
                    ldmatrix_x4(b, sK + (nt * 16 + (lane & 7) + ((lane >> 4) << 3)) * LD + kk * 16 +
                                       ((lane >> 3) & 1) * 8);
                    mma_16816(s[2 * nt], qa[kk], b[0], b[1]);
                    mma_16816(s[2 * nt + 1], qa[kk], b[2], b[3]);
                }
            }
        }
        // exact softmax over the window's keys (rows g and g + 8 of the tile)
        float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
        for (int j = 0; j < 16; ++j) {
            if (j < 2 * nkt) {
                const int c0 = j * 8 + 2 * t;
                if (c0 >= len) s[j][0] = s[j][2] = -INFINITY;
                if (c0 + 1 >= len) s[j][1] = s[j][3] = -INFINITY;
                mx0 = fmaxf(mx0, fmaxf(s[j][0], s[j][1]));
                mx1 = fmaxf(mx1, fmaxf(s[j][2], s[j][3]));
            }
        }
#pragma unroll
        for (int o = 1; o <= 2; o <<= 1) {
            mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, o));
            mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, o));
        }
        float sum0 = 0.f, sum1 = 0.f;
#pragma unroll
        for (int j = 0; j < 16; ++j) {
            if (j < 2 * nkt) {
                s[j][0] = exp2f((s[j][0] - mx0) * scale_log2e);
                s[j][1] = exp2f((s[j][1] - mx0) * scale_log2e);
                s[j][2] = exp2f((s[j][2] - mx1) * scale_log2e);
                s[j][3] = exp2f((s[j][3] - mx1) * scale_log2e);
                sum0 += s[j][0] + s[j][1];
                sum1 += s[j][2] + s[j][3];
            }
        }
#pragma unroll
        for (int o = 1; o <= 2; o <<= 1) {
            sum0 += __shfl_xor_sync(0xffffffffu, sum0, o);
            sum1 += __shfl_xor_sync(0xffffffffu, sum1, o);
        }
        float o_acc[HD / 8][4];
#pragma unroll
        for (int j = 0; j < HD / 8; ++j) o_acc[j][0] = o_acc[j][1] = o_acc[j][2] = o_acc[j][3] = 0.f;
#pragma unroll
        for (int kt = 0; kt < 8; ++kt) {
            if (kt < nkt) {
                // P as hi + lo bf16 terms: two MMAs against the same V fragment.
                uint32_t ph[4], pl[4];
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const float(&sa)[4] = s[2 * kt + (q >> 1)];
                    const float a = sa[(q & 1) * 2], b = sa[(q & 1) * 2 + 1];
                    ph[q] = pack_bf16x2(a, b);
                    const float2 hf = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&ph[q]));
                    pl[q] = pack_bf16x2(a - hf.x, b - hf.y);
                }
#pragma unroll
                for (int np = 0; np < HD / 16; ++np) {
                    uint32_t b[4];
                    ldmatrix_x4_trans(b, sV + (kt * 16 + (lane & 7) + ((lane >> 3) & 1) * 8) * LD +
                                             np * 16 + (lane >> 4) * 8);
                    mma_16816(o_acc[2 * np], ph, b[0], b[1]);
                    mma_16816(o_acc[2 * np + 1], ph, b[2], b[3]);
                    mma_16816(o_acc[2 * np], pl, b[0], b[1]);
                    mma_16816(o_acc[2 * np + 1], pl, b[2], b[3]);
                }
            }
        }
        // O / rowsum written as fp16 [T, d] (saturating at +-65504).
        const float inv0 = 1.f / sum0, inv1 = 1.f / sum1;
        const int r0 = mt * 16 + g, r1 = r0 + 8;
#pragma unroll
        for (int j = 0; j < HD / 8; ++j) {
            const int col = h * HD + j * 8 + 2 * t;
            if (r0 < len)
                *reinterpret_cast<uint32_t *>(out + (size_t)(s0 + r0) * d + col) =
                    pack_f16x2_sat(o_acc[j][0] * inv0, o_acc[j][1] * inv0);
            if (r1 < len)
                *reinterpret_cast<uint32_t *>(out + (size_t)(s0 + r1) * d + col) =
                    pack_f16x2_sat(o_acc[j][2] * inv1, o_acc[j][3] * inv1);
        }
    }
}

// -------------------------------------------------------------- prepare ----
// conv weights [co][ci][kh][kw] -> [co][kh*3 + kw][ci] (channel-last per tap,
// the "weight transposition" of the cubic.dev Audio Encoder page).
__global__ void conv_tap_major_kernel(const bf16 *__restrict__ src, bf16 *__restrict__ dst, int C) {
    const size_t n = (size_t)C * 9 * C;
    for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n;
         i += (size_t)gridDim.x * blockDim.x) {
        const int ci = (int)(i % C);
        const size_t rest = i / C;
        const int tap = (int)(rest % 9);
        const int co = (int)(rest / 9);
        dst[i] = src[((size_t)co * C + ci) * 9 + tap];
    }
}

// conv_out weight [d][c*16 + f] -> [d][f*C + c]: the stem writes its output
// channel-fastest, so conv_out's K index is reordered once instead.
__global__ void conv_out_reorder_kernel(const bf16 *__restrict__ src, bf16 *__restrict__ dst, int d,
                                        int C) {
    const size_t K = (size_t)kStemRows * C;
    const size_t n = (size_t)d * K;
    for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n;
         i += (size_t)gridDim.x * blockDim.x) {
        const size_t row = i / K;
        const int k = (int)(i - row * K);
        const int f = k / C, c = k - f * C;
        dst[i] = src[row * K + (size_t)c * kStemRows + f];
    }
}

// Sinusoid table [13][d] (aut_encoder page, module docstring: the same 13
// positions for every chunk; cubic.dev page: computed, never loaded), in the
// Whisper form: row t = [sin(t g_k) | cos(t g_k)], g_k = exp(-k ln(1e4) / (d/2 - 1)),
// evaluated in double and stored as fp32.
__global__ void position_table_kernel(float *pos, int d) {
    const int half = d / 2;
    for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < kTokensPerChunk * d;
         i += gridDim.x * blockDim.x) {
        const int t = i / d, c = i - t * d;
        const int k = c < half ? c : c - half;
        const double inc = log(10000.0) / (double)(half - 1);
        const double ang = (double)t * exp(-inc * (double)k);
        pos[i] = (float)(c < half ? sin(ang) : cos(ang));
    }
}

// Copies a block of 32-bit words carried in the kernel's parameters to device
// memory: plan tables reach the device without a host buffer that has to
// outlive the call.
__global__ void upload_words_kernel(const UploadPayload p, int32_t *dst) {
    pdl_trigger();
    pdl_wait();
    for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < p.n; i += gridDim.x * blockDim.x)
        dst[p.offset + i] = p.words[i];
}

// ------------------------------------------------------------ launchers ----
int sm_count_cached() {
    static std::mutex mu;
    static int n[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
    std::lock_guard<std::mutex> lock(mu);
    if (!n[dev]) {
        int v = 0;
        cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev);
        n[dev] = v > 0 ? v : 1;
    }
    return n[dev];
}

cudaError_t launch_conv1(const void *feats, int T_max, const int4 *chunks, int chunk_base,
                         int n_chunks, const void *w, const void *b, void *planes, int plane_rows,
                         void *planes2, int plane2_rows, int C, cudaStream_t st, int *status) {
    if (n_chunks <= 0) return cudaSuccess;
    static_assert(kC1Rows / 8 * 2 == kP2Rows - 1, "two conv3-input plane rows per conv1 block");
    return launch_pdl(conv1_kernel, dim3(n_chunks, kC1Rows / 8), dim3(256), 0, st, 1,
                      static_cast<const bf16 *>(feats), T_max, chunks, chunk_base,
                      static_cast<const bf16 *>(w), static_cast<const bf16 *>(b),
                      static_cast<bf16 *>(planes), plane_rows, static_cast<bf16 *>(planes2),
                      plane2_rows, C, status);
}

cudaError_t launch_layernorm(const float *x, const void *g, const void *b, void *y, int T, int d,
                             float eps, cudaStream_t st, bool split) {
    if (T <= 0) return cudaSuccess;
    const int vpl = (d / 4 + 31) / 32;  // float4 per lane, exact so the row stays in registers
    const dim3 grid((T + kLnRowsPerBlock - 1) / kLnRowsPerBlock), block(32 * kLnRowsPerBlock);
    const bf16 *gg = static_cast<const bf16 *>(g), *bb = static_cast<const bf16 *>(b);
    bf16 *yy = static_cast<bf16 *>(y);
    const int sp = split ? 1 : 0;
#define AUT_LN_CASE(V)                                                                         \
    case V:                                                                                    \
        return launch_pdl(layernorm_kernel<V>, grid, block, 0, st, 1, x, gg, bb, yy, T, d, eps, sp);
    switch (vpl) {
        AUT_LN_CASE(1)
        AUT_LN_CASE(2)
        AUT_LN_CASE(3)
        AUT_LN_CASE(4)
        AUT_LN_CASE(5)
        AUT_LN_CASE(6)
        AUT_LN_CASE(7)
        AUT_LN_CASE(8)
        AUT_LN_CASE(10)
        AUT_LN_CASE(12)
        AUT_LN_CASE(16)
        default:
            if (vpl <= 12)
                return launch_pdl(layernorm_kernel<12>, grid, block, 0, st, 1, x, gg, bb, yy, T, d,
                                  eps, sp);
            return launch_pdl(layernorm_kernel<16>, grid, block, 0, st, 1, x, gg, bb, yy, T, d, eps,
                              sp);
    }
#undef AUT_LN_CASE
}

template <int HD>
cudaError_t run_window_attention(const bf16 *q, __half *o, const int *cu_dev, int n_windows, int d,
                                 int heads, float scale_log2e, cudaStream_t st) {
    constexpr int smem = 2 * kMaxWindowTokens * (HD + 8) * (int)sizeof(bf16);
    const cudaError_t e = smem_attr_once<window_attn_kernel<HD>>(smem);
    if (e != cudaSuccess) return e;
    return launch_pdl(window_attn_kernel<HD>, dim3(n_windows, heads), dim3(32 * kAttnWarps), smem, st,
                      1, q, o, cu_dev, d, scale_log2e);
}

cudaError_t launch_window_attention(const void *qkv, void *out, const int *cu_dev, int n_windows,
                                    int d, int heads, cudaStream_t st, int T, int *status,
                                    bool v_f16, unsigned long long timeout_ns, int fault_inject,
                                    const int2 *wins) {
    if (n_windows <= 0) return cudaSuccess;
    const int hd = d / heads;
    if (window_attention_uses_tc(d, heads, T))
        return launch_window_attention_tc(qkv, out, cu_dev, n_windows, d, heads, T, status, st,
                                          v_f16, timeout_ns, fault_inject, wins);
    if (v_f16 || fault_inject) return cudaErrorInvalidValue;
    const float scale_log2e = 1.4426950408889634f / sqrtf((float)hd);
    const bf16 *q = static_cast<const bf16 *>(qkv);
    __half *o = static_cast<__half *>(out);
    switch (hd) {
        case 16: return run_window_attention<16>(q, o, cu_dev, n_windows, d, heads, scale_log2e, st);
        case 32: return run_window_attention<32>(q, o, cu_dev, n_windows, d, heads, scale_log2e, st);
        case 64: return run_window_attention<64>(q, o, cu_dev, n_windows, d, heads, scale_log2e, st);
        case 128: return run_window_attention<128>(q, o, cu_dev, n_windows, d, heads, scale_log2e, st);
        default: return cudaErrorInvalidValue;
    }
}

// [W | W]: a weight repeated along K, so that one GEMM over a [hi | lo] operand
// accumulates W hi + W lo.
__global__ void duplicate_k_kernel(const bf16 *__restrict__ src, bf16 *__restrict__ dst, int N,
                                   int K) {
    const size_t n = (size_t)N * 2 * K;
    for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n;
         i += (size_t)gridDim.x * blockDim.x) {
        const size_t row = i / (2 * K);
        const int k = (int)(i - row * 2 * K);
        dst[i] = src[row * K + (k < K ? k : k - K)];
    }
}

cudaError_t launch_duplicate_k(const void *src, void *dst, int N, int K, cudaStream_t st) {
    duplicate_k_kernel<<<592, 256, 0, st>>>(static_cast<const bf16 *>(src), static_cast<bf16 *>(dst),
                                            N, K);
    return cudaGetLastError();
}

// bf16 -> fp16 (saturating), n elements, n a multiple of 2.
__global__ void to_f16_kernel(const bf16 *__restrict__ src, uint32_t *__restrict__ dst, size_t n2) {
    for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n2;
         i += (size_t)gridDim.x * blockDim.x) {
        const float2 f = __bfloat1622float2(reinterpret_cast<const __nv_bfloat162 *>(src)[i]);
        dst[i] = pack_f16x2_sat(f.x, f.y);
    }
}

cudaError_t launch_to_f16(const void *src, void *dst, size_t n, cudaStream_t st) {
    if (n % 2) return cudaErrorInvalidValue;
    to_f16_kernel<<<592, 256, 0, st>>>(static_cast<const bf16 *>(src), static_cast<uint32_t *>(dst),
                                       n / 2);
    return cudaGetLastError();
}

cudaError_t launch_prepare(const void *conv2_w, const void *conv3_w, const void *conv_out_w,
                           void *conv2_tap, void *conv3_tap, void *conv_out_fc, float *pos, int C,
                           int d, cudaStream_t st) {
    conv_tap_major_kernel<<<592, 256, 0, st>>>(static_cast<const bf16 *>(conv2_w),
                                               static_cast<bf16 *>(conv2_tap), C);
    conv_tap_major_kernel<<<592, 256, 0, st>>>(static_cast<const bf16 *>(conv3_w),
                                               static_cast<bf16 *>(conv3_tap), C);
    conv_out_reorder_kernel<<<592, 256, 0, st>>>(static_cast<const bf16 *>(conv_out_w),
                                                 static_cast<bf16 *>(conv_out_fc), d, C);
    position_table_kernel<<<(kTokensPerChunk * d + 255) / 256, 256, 0, st>>>(pos, d);
    return cudaGetLastError();
}

cudaError_t launch_upload(const int32_t *host_words, size_t n, int32_t *dst, cudaStream_t st) {
    UploadPayload p;
    for (size_t off = 0; off < n; off += UploadPayload::kWords) {
        p.n = (int)std::min<size_t>(UploadPayload::kWords, n - off);
        p.offset = (int)off;
        std::copy(host_words + off, host_words + off + p.n, p.words);
        cudaError_t e = launch_pdl(upload_words_kernel, dim3((p.n + 255) / 256), dim3(256), 0, st, 1,
                                   p, dst);
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

}  // namespace aut
