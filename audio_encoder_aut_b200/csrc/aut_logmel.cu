// Log-mel front end: 16 kHz mono waveform -> the encoder's 128-bin features.
//
// The pages fix 16 kHz mono input (cubic.dev "Audio Encoder Component",
// Feature Extraction Pipeline), 128 mel bins and 100 frames per second, and
// call the features Whisper-style (m-star.org "mstar.model.components.aut_encoder",
// module docstring).  The steps left open follow Whisper's recipe: 400-sample
// periodic Hann frames every 160 samples, centred, with the signal reflected
// by 200 samples at both ends; the power of the 400-point DFT (bins 0..200);
// 128 Slaney mel filters (unit area) over 0..8000 Hz; log10 of
// max(energy, 1e-10); the transform's last frame dropped (n // 160 frames);
// per request, values raised to at least (max - 8); then (x + 4) / 4.
//
// Kernels (fp32 on the CUDA cores; the DFT is a dense 400-term contraction
// per bin, done as a register-tiled product, with the window folded into the
// basis):
//   logmel_tables_kernel   windowed DFT basis [400][224][re, im] and the mel
//                          filter table (weights + support per filter)
//   logmel_kernel          one CTA = 64 frames of one request: samples into
//                          shared memory (reflected at the request's ends),
//                          C[64 x 224 x 2] = frames x basis, power, mel
//                          filters, log10; each warp folds its maximum into
//                          the request's (ordered-integer atomicMax)
//   logmel_finish_kernel   clamp to max - 8, (x + 4) / 4, bf16 features
//                          [B, 128, T_max] with zeros past each request's
//                          frames
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cmath>
#include <vector>

#include "aut_internal.h"
#include "aut_kernels.h"
#include "aut_ptx.cuh"

namespace aut {
namespace {

constexpr int kNfft = 400, kHop = 160, kBins = 201, kBinsPad = 224, kMels = 128;
constexpr int kFramesPerCta = 64, kThreads = 256;
constexpr int kKChunk = 16;                                     // basis rows per stage
constexpr int kSamples = kFramesPerCta * kHop + kNfft - kHop;  // 10480
constexpr int kChunkFloats = kKChunk * kBinsPad * 2;          // 7168
constexpr int kPowLd = kBinsPad + 1;                           // padded power row
constexpr int kSmemFloats = kSamples + 2 * kChunkFloats;  // the power aliases samples + stages
static_assert(kFramesPerCta * kPowLd <= kSmemFloats, "power fits over samples and stages");
constexpr int kSmemBytes = kSmemFloats * 4;

struct MelFilter {
    int k0, n;  // support: bins [k0, k0 + n)
};

// Workspace carve-up (byte offsets).
struct LogmelLayout {
    size_t status, keys, nsamp, basis, fb, support, logmel, total;
};
LogmelLayout logmel_layout(int n_req, int T_max) {
    auto up = [](size_t v) { return (v + 255) / 256 * 256; };
    LogmelLayout L{};
    size_t o = 0;
    L.status = o;
    o = up(o + 4);
    L.keys = o;
    o = up(o + 4 * (size_t)std::max(n_req, 1));
    L.nsamp = o;
    o = up(o + 4 * (size_t)std::max(n_req, 1));
    L.basis = o;
    o = up(o + (size_t)kNfft * kBinsPad * 2 * 4);
    L.fb = o;
    o = up(o + (size_t)kMels * kBins * 4);
    L.support = o;
    o = up(o + (size_t)kMels * sizeof(MelFilter));
    L.logmel = o;
    o = up(o + (size_t)std::max(n_req, 1) * kMels * std::max(T_max, 1) * 4);
    L.total = o;
    return L;
}

// Float order as signed-integer order (for atomicMax on floats of any sign).
__device__ __forceinline__ int float_key(float f) {
    const int i = __float_as_int(f);
    return i >= 0 ? i : i ^ 0x7fffffff;
}
__device__ __forceinline__ float key_float(int k) { return __int_as_float(k >= 0 ? k : k ^ 0x7fffffff); }

// Slaney's mel scale (linear below 1 kHz, 27 mels per factor 6.4 above).
__device__ double hz_to_mel(double f) {
    const double logstep = log(6.4) / 27.0;
    return f >= 1000.0 ? 15.0 + log(f / 1000.0) / logstep : f / (200.0 / 3.0);
}
__device__ double mel_to_hz(double m) {
    const double logstep = log(6.4) / 27.0;
    return m >= 15.0 ? 1000.0 * exp(logstep * (m - 15.0)) : m * (200.0 / 3.0);
}

__global__ void logmel_tables_kernel(float2 *__restrict__ basis, float *__restrict__ fb,
                                     MelFilter *__restrict__ support, int *__restrict__ keys,
                                     int n_req) {
    pdl_trigger();
    pdl_wait();
    const int tid = blockIdx.x * blockDim.x + threadIdx.x, nth = gridDim.x * blockDim.x;
    const double two_pi = 6.283185307179586476925;
    // basis[n][k] = w[n] (cos, -sin)(2 pi k n / 400); (k n) mod 400 keeps the angle exact.
    for (int i = tid; i < kNfft * kBinsPad; i += nth) {
        const int n = i / kBinsPad, k = i - n * kBinsPad;
        float2 v = make_float2(0.f, 0.f);
        if (k < kBins) {
            const double w = 0.5 - 0.5 * cos(two_pi * n / kNfft);
            const double a = two_pi * (double)((k * n) % kNfft) / kNfft;
            v = make_float2((float)(w * cos(a)), (float)(-w * sin(a)));
        }
        basis[i] = v;
    }
    // Filter m: triangle over Slaney-mel points m, m + 1, m + 2 (130 points
    // equally spaced in mels over 0 .. 8000 Hz), scaled to unit area.
    const double mmax = hz_to_mel(8000.0);
    for (int m = tid; m < kMels; m += nth) {
        const double lo = mel_to_hz(mmax * m / (kMels + 1));
        const double ce = mel_to_hz(mmax * (m + 1) / (kMels + 1));
        const double hi = mel_to_hz(mmax * (m + 2) / (kMels + 1));
        int k0 = -1, k1 = -1;
        for (int k = 0; k < kBins; ++k) {
            const double f = k * 16000.0 / kNfft;
            const double t = fmax(0.0, fmin((f - lo) / (ce - lo), (hi - f) / (hi - ce)));
            const float v = (float)(t * 2.0 / (hi - lo));
            fb[m * kBins + k] = v;
            if (v != 0.f) {
                if (k0 < 0) k0 = k;
                k1 = k;
            }
        }
        support[m] = k0 < 0 ? MelFilter{0, 0} : MelFilter{k0, k1 - k0 + 1};
    }
    for (int r = tid; r < n_req; r += nth) keys[r] = float_key(-INFINITY);
}

// Loads one stage (kKChunk basis rows) global -> shared.
__device__ __forceinline__ void load_basis_chunk(float *dst, const float2 *basis, int chunk) {
    const float4 *src = reinterpret_cast<const float4 *>(basis + (size_t)chunk * kKChunk * kBinsPad);
    float4 *d = reinterpret_cast<float4 *>(dst);
    for (int i = threadIdx.x; i < kChunkFloats / 4; i += kThreads) d[i] = __ldg(src + i);
}

__global__ void __launch_bounds__(kThreads, 1)
    logmel_kernel(const float *__restrict__ wave, long long S_max, const int *__restrict__ nsamp,
                  const float2 *__restrict__ basis, const float *__restrict__ fb,
                  const MelFilter *__restrict__ support, float *__restrict__ logmel, int T_max,
                  int *__restrict__ keys) {
    extern __shared__ float4 smem4[];
    float *xs = reinterpret_cast<float *>(smem4);
    float *stage = xs + kSamples;
    pdl_trigger();
    pdl_wait();
    const int r = blockIdx.y, t0 = blockIdx.x * kFramesPerCta;
    const int n = nsamp[r], frames = n / kHop;
    if (t0 >= frames) return;
    // Samples of frames t0 .. t0 + 63: index 160 t - 200 + i, reflected at both ends.
    const float *x = wave + (size_t)r * S_max;
    const long long j0 = (long long)t0 * kHop - kNfft / 2;
    for (int i = threadIdx.x; i < kSamples; i += kThreads) {
        long long j = j0 + i;
        if (j < 0) j = -j;
        if (j >= n) j = 2LL * (n - 1) - j;
        xs[i] = (j >= 0 && j < n) ? __ldg(x + j) : 0.f;
    }
    load_basis_chunk(stage, basis, 0);
    __syncthreads();

    // Warp w: frames 8w .. 8w + 7; lane c: bins c + 32 j (j < 7), re and im.
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    float2 acc[8][7];
#pragma unroll
    for (int f = 0; f < 8; ++f)
#pragma unroll
        for (int j = 0; j < 7; ++j) acc[f][j] = make_float2(0.f, 0.f);
    constexpr int kChunks = kNfft / kKChunk;
    for (int ch = 0; ch < kChunks; ++ch) {
        float *cur = stage + (ch & 1) * kChunkFloats;
        if (ch + 1 < kChunks) load_basis_chunk(stage + ((ch + 1) & 1) * kChunkFloats, basis, ch + 1);
        const float2 *b2 = reinterpret_cast<const float2 *>(cur);
#pragma unroll 4
        for (int kk = 0; kk < kKChunk; ++kk) {
            const int nn = ch * kKChunk + kk;
            float a[8];
#pragma unroll
            for (int f = 0; f < 8; ++f) a[f] = xs[(warp * 8 + f) * kHop + nn];
#pragma unroll
            for (int j = 0; j < 7; ++j) {
                const float2 b = b2[kk * kBinsPad + lane + 32 * j];
#pragma unroll
                for (int f = 0; f < 8; ++f) {
                    acc[f][j].x = fmaf(a[f], b.x, acc[f][j].x);
                    acc[f][j].y = fmaf(a[f], b.y, acc[f][j].y);
                }
            }
        }
        __syncthreads();  // this stage is read; the next one has landed
    }
    // Power into shared memory (over the samples and the basis stages, all
    // read by now): pw[f][k], rows padded so a warp's 32 frames hit 32 banks.
    float *pw = xs;
#pragma unroll
    for (int f = 0; f < 8; ++f)
#pragma unroll
        for (int j = 0; j < 7; ++j) {
            const float2 v = acc[f][j];
            pw[(warp * 8 + f) * kPowLd + lane + 32 * j] = v.x * v.x + v.y * v.y;
        }
    __syncthreads();
    // Thread: frame f = tid % 64, mel filters m = tid / 64 + 4 i.
    const int f = threadIdx.x & 63, t = t0 + f;
    const bool valid = t < frames;
    float mx = -INFINITY;
    float *dst = logmel + (size_t)r * kMels * T_max + t;
    for (int m = threadIdx.x >> 6; m < kMels; m += kThreads / 64) {
        const MelFilter s = support[m];
        const float *w = fb + m * kBins;
        float e = 0.f;
        for (int k = s.k0; k < s.k0 + s.n; ++k) e = fmaf(pw[f * kPowLd + k], __ldg(w + k), e);
        const float v = log10f(fmaxf(e, 1e-10f));
        if (valid) {
            dst[(size_t)m * T_max] = v;
            mx = fmaxf(mx, v);
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    if (lane == 0 && mx > -INFINITY) atomicMax(keys + r, float_key(mx));
}

__global__ void logmel_finish_kernel(const float *__restrict__ logmel, const int *__restrict__ nsamp,
                                     const int *__restrict__ keys, __nv_bfloat16 *__restrict__ out,
                                     int n_req, int T_max) {
    pdl_trigger();
    pdl_wait();
    const size_t total = (size_t)n_req * kMels * T_max;
    for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < total;
         i += (size_t)gridDim.x * blockDim.x) {
        const int t = (int)(i % T_max);
        const int r = (int)(i / ((size_t)kMels * T_max));
        float v = 0.f;
        if (t < nsamp[r] / kHop) {
            const float lo = key_float(keys[r]) - 8.0f;
            v = (fmaxf(logmel[i], lo) + 4.0f) * 0.25f;
        }
        out[i] = __float2bfloat16_rn(v);
    }
}

}  // namespace
}  // namespace aut

using namespace aut;

extern "C" size_t aut_logmel_workspace_bytes(int32_t n_req, int32_t T_max) {
    if (n_req < 0 || T_max < 0) return 0;
    return logmel_layout(n_req, T_max).total;
}

extern "C" aut_status aut_logmel(const void *waveform, int64_t S_max, const int32_t *sample_lens,
                                 int32_t n_req, void *features, int32_t T_max,
                                 int32_t *feature_lens, void *workspace, size_t ws_bytes,
                                 aut_stream_t stream) {
    if (n_req < 0 || S_max < 0 || T_max < 0 || (n_req > 0 && !sample_lens))
        return AUT_ERR_INVALID_ARG;
    int frames_max = 0;
    for (int r = 0; r < n_req; ++r) {
        const int64_t n = sample_lens[r];
        // Reflection by 200 samples needs more than 200 samples (or none at all).
        if (n < 0 || n > S_max || (n > 0 && n <= kNfft / 2) || n / kHop > 0x7fffffff)
            return AUT_ERR_INVALID_ARG;
        frames_max = std::max(frames_max, (int)(n / kHop));
    }
    if (frames_max > T_max) return AUT_ERR_INVALID_ARG;
    if (feature_lens)
        for (int r = 0; r < n_req; ++r) feature_lens[r] = sample_lens[r] / kHop;
    if (n_req == 0 || T_max == 0) return AUT_OK;
    if (!waveform || !features || !workspace) return AUT_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(waveform) & 3u) || (reinterpret_cast<uintptr_t>(features) & 1u) ||
        (reinterpret_cast<uintptr_t>(workspace) & 255u))
        return AUT_ERR_INVALID_ARG;
    const LogmelLayout L = logmel_layout(n_req, T_max);
    if (ws_bytes < L.total) return AUT_ERR_WORKSPACE;
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    std::vector<int32_t> words(1, 0);  // status word, cleared
    if (launch_upload(words.data(), 1, reinterpret_cast<int32_t *>(ws + L.status), st) != cudaSuccess ||
        launch_upload(sample_lens, n_req, reinterpret_cast<int32_t *>(ws + L.nsamp), st) != cudaSuccess)
        return AUT_ERR_CUDA;
    auto *basis = reinterpret_cast<float2 *>(ws + L.basis);
    auto *fb = reinterpret_cast<float *>(ws + L.fb);
    auto *sup = reinterpret_cast<MelFilter *>(ws + L.support);
    auto *keys = reinterpret_cast<int *>(ws + L.keys);
    auto *lm = reinterpret_cast<float *>(ws + L.logmel);
    const int *ns = reinterpret_cast<const int *>(ws + L.nsamp);
    if (launch_pdl(logmel_tables_kernel, dim3(2 * sm_count_cached()), dim3(256), 0, st, 1, basis,
                   fb, sup, keys, (int)n_req) != cudaSuccess)
        return AUT_ERR_CUDA;
    if (smem_attr_once<logmel_kernel>(kSmemBytes) != cudaSuccess) return AUT_ERR_CUDA;
    const dim3 grid((frames_max + kFramesPerCta - 1) / kFramesPerCta, n_req);
    if (frames_max > 0 &&
        launch_pdl(logmel_kernel, grid, dim3(kThreads), kSmemBytes, st, 1,
                   static_cast<const float *>(waveform), (long long)S_max, ns,
                   static_cast<const float2 *>(basis), static_cast<const float *>(fb),
                   static_cast<const MelFilter *>(sup), lm, (int)T_max, keys) != cudaSuccess)
        return AUT_ERR_CUDA;
    if (launch_pdl(logmel_finish_kernel, dim3(4 * sm_count_cached()), dim3(256), 0, st, 1,
                   static_cast<const float *>(lm), ns, static_cast<const int *>(keys),
                   static_cast<__nv_bfloat16 *>(features), (int)n_req, (int)T_max) != cudaSuccess)
        return AUT_ERR_CUDA;
    return AUT_OK;
}
