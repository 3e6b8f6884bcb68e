// C-ABI entry points (include/aut.h): argument checks, workspace carve-up and
// the launch sequence of the encoder forward pass.
//
// Forward (aut_encoder page, AuTEncoder.forward = layout + frontend + encode):
//   front end, per group of at most conv_chunksize chunks:
//     conv1 + GELU (CUDA cores) -> phase planes
//     conv2 + GELU (tcgen05 implicit GEMM) -> phase planes
//     conv3 + GELU (tcgen05 implicit GEMM) -> [chunk * 13 + t][f * C + c]
//     conv_out (tcgen05 GEMM) + sinusoid row + trim + pack -> x0 (fp32)
//   per layer: LN1 -> qkv (GEMM + bias) -> window attention -> o_proj (GEMM +
//     bias + residual) -> LN2 -> fc1 (GEMM + bias + GELU) -> fc2 (GEMM + bias +
//     residual)
//   final LN -> proj1 (GEMM + bias + GELU) -> proj2 (GEMM + bias) -> out (fp32)
#include <cuda_runtime.h>
#include <nvtx3/nvToolsExt.h>

#include <algorithm>
#include <cstring>

#include "aut_internal.h"
#include "aut_kernels.h"

namespace aut {

namespace {

// NVTX range over one stage of the forward (the stem, a layer, the projector),
// for profilers; a host-side marker only, so it costs nothing on the device and
// is recorded once when the forward is captured into a graph.
struct NvtxRange {
    explicit NvtxRange(const char *name) { nvtxRangePushA(name); }
    ~NvtxRange() { nvtxRangePop(); }
    NvtxRange(const NvtxRange &) = delete;
    NvtxRange &operator=(const NvtxRange &) = delete;
};

constexpr unsigned long long kDefaultTimeoutNs = 4000ull * 1000ull * 1000ull;  // 4 s

size_t align_up(size_t v, size_t a = 1024) { return (v + a - 1) / a * a; }

struct Region {
    size_t off = 0;
    size_t take(size_t bytes) {
        const size_t o = off;
        off = align_up(off + bytes);
        return o;
    }
};

struct PreparedLayout {
    size_t conv2, conv3, conv_out, pos, proj1_dup, proj2_dup, o_f16, total;
};

PreparedLayout prepared_layout(const aut_config *c) {
    Region r;
    PreparedLayout p;
    const size_t C = c->conv_ch, d = c->d_model;
    p.conv2 = r.take(C * 9 * C * 2);
    p.conv3 = r.take(C * 9 * C * 2);
    p.conv_out = r.take(d * kStemRows * C * 2);
    p.pos = r.take((size_t)kTokensPerChunk * d * 4);
    p.proj1_dup = r.take(d * 2 * d * 2);
    p.proj2_dup = r.take((size_t)c->output_dim * 2 * d * 2);
    p.o_f16 = r.take((size_t)std::max(c->layers, 1) * d * d * 2);
    p.total = r.off;
    return p;
}

aut_status cuda_status(cudaError_t e) { return e == cudaSuccess ? AUT_OK : AUT_ERR_CUDA; }

aut_status gemm_status(GemmStatus s) {
    switch (s) {
        case GemmStatus::kOk: return AUT_OK;
        case GemmStatus::kBadShape: return AUT_ERR_INVALID_ARG;
        default: return AUT_ERR_CUDA;
    }
}

#define AUT_TRY(expr)                          \
    do {                                       \
        const aut_status _s = (expr);          \
        if (_s != AUT_OK) return _s;           \
    } while (0)

bool weights_complete(const aut_config *c, const aut_weights *w, int n_layers, bool stem,
                      bool projector) {
    if (!w) return false;
    if (stem && (!w->conv1_w || !w->conv1_b || !w->conv2_b || !w->conv3_b || !w->conv2_w_tap ||
                 !w->conv3_w_tap || !w->conv_out_w_fc || !w->pos_table))
        return false;
    if (n_layers > 0 && (!w->layers || !w->o_w_f16)) return false;
    for (int i = 0; i < n_layers; ++i) {
        const aut_layer_weights &l = w->layers[i];
        if (!l.ln1_w || !l.ln1_b || !l.qkv_w || !l.qkv_b || !l.o_w || !l.o_b || !l.ln2_w ||
            !l.ln2_b || !l.fc1_w || !l.fc1_b || !l.fc2_w || !l.fc2_b)
            return false;
    }
    if (projector && (!w->ln_post_w || !w->ln_post_b || !w->proj1_b || !w->proj2_b ||
                      !w->proj1_w_dup || !w->proj2_w_dup))
        return false;
    (void)c;
    return true;
}

struct Ctx {
    const aut_config *cfg;
    const aut_weights *w;
    uint8_t *ws;
    WorkspaceLayout L;
    cudaStream_t st;
    int *status;
    aut_trace *trace = nullptr;

    // Records the trace event after a kernel launch (no-op without a trace).
    aut_status mark(int kind) const {
        if (!trace) return AUT_OK;
        const int i = trace->count++;
        if (i < trace->capacity) {
            if (trace->kinds) trace->kinds[i] = kind;
            if (trace->events &&
                cudaEventRecordWithFlags(static_cast<cudaEvent_t>(trace->events[i]), st,
                                         cudaEventRecordExternal) != cudaSuccess)
                return AUT_ERR_CUDA;
        }
        return AUT_OK;
    }

    template <class T>
    T *at(size_t off) const {
        return reinterpret_cast<T *>(ws + off);
    }
};

aut_status linear(const Ctx &c, const void *a, const void *w, const void *b, void *out, int M,
                  int N, int K, int epi, int kind, int ldo = 0, bool f16 = false,
                  int f16_col = 1 << 30) {
    LinearLaunch L{};
    L.f16 = f16;
    L.f16_col = f16_col;
    L.a = a;
    L.w = w;
    L.bias = b;
    L.out = out;
    L.M = M;
    L.N = N;
    L.K = K;
    L.ldo = ldo ? ldo : N;
    L.epi = epi;
    L.status = c.status;
    L.timeout_ns = kDefaultTimeoutNs;
    AUT_TRY(gemm_status(launch_linear(L, c.st)));
    return c.mark(kind);
}

// cu_seqlens followed by the window table the tensor-core attention walks:
// (first token, length) per window, longest first, ties in window order, so
// that its grid stride gives every CTA a similar mix of long and short
// windows.  The table starts on an even word of the region (8-byte aligned).
void append_windows(std::vector<int32_t> &words, const std::vector<int32_t> &cu) {
    const int nW = (int)cu.size() - 1;
    words.insert(words.end(), cu.begin(), cu.end());
    if (words.size() & 1) words.push_back(0);
    std::vector<int> order(nW);
    for (int i = 0; i < nW; ++i) order[i] = i;
    std::stable_sort(order.begin(), order.end(), [&](int a, int b) {
        return cu[a + 1] - cu[a] > cu[b + 1] - cu[b];
    });
    for (int w : order) {
        words.push_back(cu[w]);
        words.push_back(cu[w + 1] - cu[w]);
    }
}

// Device address of the window table behind cu_seqlens (append_windows).
const int2 *window_table(const Ctx &c, int nW) {
    return reinterpret_cast<const int2 *>(c.at<int32_t>(c.L.cu) + nW + 1 + ((nW + 1) & 1));
}

// The chunk table, cu_seqlens and the window table lie next to each other in
// the workspace (chunks, padding, cu, windows); one upload writes the span.
aut_status upload_plan(const Ctx &c, const Plan &p) {
    const size_t cu_word = (c.L.cu - c.L.chunks) / 4;
    std::vector<int32_t> words(cu_word, 0);
    size_t i = 0;
    for (const ChunkInfo &ci : p.chunks) {
        words[i++] = ci.request;
        words[i++] = ci.frame0;
        words[i++] = ci.valid_frames;
        words[i++] = ci.token0;
    }
    append_windows(words, p.cu_seqlens);
    AUT_TRY(cuda_status(launch_upload(words.data(), words.size(), c.at<int32_t>(c.L.chunks), c.st)));
    return c.mark(AUT_K_UPLOAD);
}

// AuTEncoder.frontend: chunks -> conv stem -> conv_out + positions -> packed x0.
aut_status run_frontend(const Ctx &c, const Plan &p, const void *feats, int T_max, float *x0,
                        bool with_positions) {
    const aut_config *cfg = c.cfg;
    const int C = cfg->conv_ch, d = cfg->d_model;
    const int n_ch = (int)p.chunks.size();
    const int G = c.L.group_chunks;
    if (n_ch == 0) return AUT_OK;
    NvtxRange range("aut stem");
    const int4 *chunks = c.at<int4>(c.L.chunks);
    void *planes1 = c.at<void>(c.L.planes1);
    void *planes2 = c.at<void>(c.L.planes2);
    void *y3 = c.at<void>(c.L.y3);
    const int p1_rows = G * kP1Rows, p2_rows = G * kP2Rows;
    for (int c0 = 0; c0 < n_ch; c0 += G) {
        const int g = std::min(G, n_ch - c0);
        if (conv1_tc_supported(C))
            AUT_TRY(cuda_status(launch_conv1_tc(feats, T_max, chunks, c0, g, c.w->conv1_w,
                                                c.w->conv1_b, planes1, p1_rows, planes2, p2_rows, C,
                                                c.st, c.status, kDefaultTimeoutNs)));
        else
            AUT_TRY(cuda_status(launch_conv1(feats, T_max, chunks, c0, g, c.w->conv1_w, c.w->conv1_b,
                                             planes1, p1_rows, planes2, p2_rows, C, c.st, c.status)));
        AUT_TRY(c.mark(AUT_K_CONV1));
        ConvLaunch k2{};
        k2.planes = planes1;
        k2.plane_rows_cap = p1_rows;
        k2.chunks = g;
        k2.chunk_rows = kP1Rows;
        k2.cols_in = kP1Cols;
        k2.out_cols = kC2Cols;
        k2.rows_per_tile = 128 / kC2Cols;
        k2.C = C;
        k2.w_tap = c.w->conv2_w_tap;
        k2.bias = c.w->conv2_b;
        k2.epi = kEpiConvPlanes;
        k2.out = planes2;
        k2.out_elems = (size_t)4 * p2_rows * kP2Cols * C;
        k2.dst_plane_rows = p2_rows;
        k2.dst_chunk_rows = kP2Rows;
        k2.dst_cols = kP2Cols;
        k2.status = c.status;
        k2.timeout_ns = kDefaultTimeoutNs;
        AUT_TRY(gemm_status(launch_conv_gemm(k2, c.st)));
        AUT_TRY(c.mark(AUT_K_CONV2));
        ConvLaunch k3 = k2;
        k3.planes = planes2;
        k3.plane_rows_cap = p2_rows;
        k3.chunk_rows = kP2Rows;
        k3.cols_in = kP2Cols;
        k3.out_cols = kC3Cols;
        k3.rows_per_tile = 128 / kC3Cols;
        k3.w_tap = c.w->conv3_w_tap;
        k3.bias = c.w->conv3_b;
        k3.epi = kEpiConvFlat;
        k3.out = y3;
        k3.out_elems = (size_t)G * kTokensPerChunk * kStemRows * C;
        AUT_TRY(gemm_status(launch_conv_gemm(k3, c.st)));
        AUT_TRY(c.mark(AUT_K_CONV3));
        LinearLaunch lo{};
        lo.a = y3;
        lo.w = c.w->conv_out_w_fc;
        lo.bias = c.w->conv_out_b;
        lo.out = x0;
        lo.out_elems = (size_t)p.total_tokens * d;
        lo.M = g * kTokensPerChunk;
        lo.N = d;
        lo.K = kStemRows * C;
        lo.ldo = d;
        lo.epi = kEpiPackTokens;
        lo.chunks = chunks;
        lo.chunk_base = c0;
        lo.pos = with_positions ? static_cast<const float *>(c.w->pos_table) : nullptr;
        lo.status = c.status;
        lo.timeout_ns = kDefaultTimeoutNs;
        AUT_TRY(gemm_status(launch_linear(lo, c.st)));
        AUT_TRY(c.mark(AUT_K_CONV_OUT));
    }
    return AUT_OK;
}

// AuTEncoder.encode: layers [0, n_layers) on the residual stream x, then (if out)
// the final LayerNorm and projector.
aut_status run_encode(const Ctx &c, float *x, int T, int nW, int n_layers, void *out) {
    const aut_config *cfg = c.cfg;
    const int d = cfg->d_model, F = cfg->ffn;
    if (T == 0) return AUT_OK;
    void *xn = c.at<void>(c.L.xn), *qkv = c.at<void>(c.L.qkv), *attn = c.at<void>(c.L.attn),
         *ffn = c.at<void>(c.L.ffn);
    const int *cu = c.at<int>(c.L.cu);
    static const char *const kLayerNames[] = {
        "aut layer 0",  "aut layer 1",  "aut layer 2",  "aut layer 3",  "aut layer 4",
        "aut layer 5",  "aut layer 6",  "aut layer 7",  "aut layer 8",  "aut layer 9",
        "aut layer 10", "aut layer 11", "aut layer 12", "aut layer 13", "aut layer 14",
        "aut layer 15", "aut layer 16", "aut layer 17", "aut layer 18", "aut layer 19",
        "aut layer 20", "aut layer 21", "aut layer 22", "aut layer 23", "aut layer"};
    for (int l = 0; l < n_layers; ++l) {
        NvtxRange range(kLayerNames[l < 24 ? l : 24]);
        const aut_layer_weights &lw = c.w->layers[l];
        AUT_TRY(cuda_status(launch_layernorm(x, lw.ln1_w, lw.ln1_b, xn, T, d, cfg->ln_eps, c.st)));
        AUT_TRY(c.mark(AUT_K_LAYERNORM));
        // With the tensor-core attention the qkv GEMM writes v as fp16, the
        // type of the attention's P V product.
        const bool v_f16 = window_attention_uses_tc(d, cfg->heads, T);
        AUT_TRY(linear(c, xn, lw.qkv_w, lw.qkv_b, qkv, T, 3 * d, d, kEpiBf16, AUT_K_QKV, 0, false,
                       v_f16 ? 2 * d : 1 << 30));
        AUT_TRY(cuda_status(launch_window_attention(qkv, attn, cu, nW, d, cfg->heads, c.st, T,
                                                    c.status, v_f16, 0, 0, window_table(c, nW))));
        AUT_TRY(c.mark(AUT_K_ATTENTION));
        // fp16 attention output against the fp16 copy of o_w
        const void *o_w16 = static_cast<const uint8_t *>(c.w->o_w_f16) + (size_t)l * d * d * 2;
        AUT_TRY(linear(c, attn, o_w16, lw.o_b, x, T, d, d, kEpiResidF32, AUT_K_O_PROJ, 0, true));
        AUT_TRY(cuda_status(launch_layernorm(x, lw.ln2_w, lw.ln2_b, xn, T, d, cfg->ln_eps, c.st)));
        AUT_TRY(c.mark(AUT_K_LAYERNORM));
        AUT_TRY(linear(c, xn, lw.fc1_w, lw.fc1_b, ffn, T, F, d, kEpiBf16Gelu, AUT_K_FC1));
        AUT_TRY(linear(c, ffn, lw.fc2_w, lw.fc2_b, x, T, d, F, kEpiResidF32, AUT_K_FC2));
    }
    if (!out) return AUT_OK;
    NvtxRange range("aut projector");
    // Projector operands as hi + lo bf16 pairs ([hi | lo] rows against K-repeated
    // weights): its two roundings would otherwise add as much error as a layer.
    AUT_TRY(cuda_status(
        launch_layernorm(x, c.w->ln_post_w, c.w->ln_post_b, xn, T, d, cfg->ln_eps, c.st, true)));
    AUT_TRY(c.mark(AUT_K_LAYERNORM));
    AUT_TRY(linear(c, xn, c.w->proj1_w_dup, c.w->proj1_b, ffn, T, d, 2 * d, kEpiBf16GeluSplit,
                   AUT_K_PROJ1, 2 * d));
    return linear(c, ffn, c.w->proj2_w_dup, c.w->proj2_b, out, T, cfg->output_dim, 2 * d,
                  kEpiF32, AUT_K_PROJ2);
}

aut_status make_ctx(const aut_config *cfg, const aut_weights *w, void *ws, size_t ws_bytes,
                    const Plan &p, cudaStream_t st, Ctx *c, aut_trace *trace = nullptr) {
    c->cfg = cfg;
    c->trace = trace;
    if (trace) {
        if (trace->capacity < 0 || (trace->capacity > 0 && !trace->events && !trace->kinds))
            return AUT_ERR_INVALID_ARG;
        trace->count = 0;
    }
    c->w = w;
    c->ws = static_cast<uint8_t *>(ws);
    c->st = st;
    c->L = workspace_layout(cfg, p.total_tokens, (int64_t)p.cu_seqlens.size() - 1,
                            (int64_t)p.chunks.size());
    if (!ws || (reinterpret_cast<uintptr_t>(ws) & 255u)) return AUT_ERR_INVALID_ARG;
    if (ws_bytes < c->L.total) return AUT_ERR_WORKSPACE;
    c->status = c->at<int>(c->L.status);
    return cuda_status(cudaMemsetAsync(c->status, 0, sizeof(int), st));
}

aut_status check_features(const Plan &p, const void *feats, int T_max, const int32_t *lens,
                          int n_req) {
    for (int r = 0; r < n_req; ++r)
        if (lens[r] > T_max) return AUT_ERR_INVALID_ARG;
    if (!p.chunks.empty() && (!feats || T_max <= 0)) return AUT_ERR_INVALID_ARG;
    return AUT_OK;
}

}  // namespace

WorkspaceLayout workspace_layout(const aut_config *c, int64_t T, int64_t nW, int64_t n_ch) {
    WorkspaceLayout L{};
    Region r;
    const size_t d = c->d_model, F = c->ffn, C = c->conv_ch;
    L.status = r.take(256);
    L.chunks = r.take((size_t)std::max<int64_t>(n_ch, 1) * 16);
    L.cu = r.take((size_t)(3 * nW + 2) * 4);  // cu_seqlens, one padding word, window table
    L.x = r.take((size_t)T * d * 4);
    // The stem buffers and the layer buffers are never live together: overlay them.
    const size_t base = r.off;
    Region a{base};
    L.xn = a.take((size_t)T * 2 * d * 2);  // [hi | lo] rows for the projector
    L.qkv = a.take((size_t)T * 3 * d * 2);
    L.attn = a.take((size_t)T * d * 2);  // fp16
    L.ffn = a.take((size_t)T * std::max(F, 2 * d) * 2);
    const int G = (int)std::min<int64_t>(n_ch, c->conv_chunksize);
    L.group_chunks = G;
    Region b{base};
    L.planes1 = b.take((size_t)4 * G * kP1Rows * kP1Cols * C * 2);
    L.planes2 = b.take((size_t)4 * G * kP2Rows * kP2Cols * C * 2);
    L.y3 = b.take((size_t)G * kTokensPerChunk * kStemRows * C * 2);
    L.total = std::max(a.off, b.off);
    return L;
}

}  // namespace aut

using namespace aut;

extern "C" size_t aut_workspace_bytes(const aut_config *cfg, int32_t total_tokens,
                                      int32_t num_windows, int32_t num_chunks) {
    if (check_config(cfg) != AUT_OK || total_tokens < 0 || num_windows < 0 || num_chunks < 0)
        return 0;
    return workspace_layout(cfg, total_tokens, num_windows, num_chunks).total;
}

extern "C" size_t aut_prepared_bytes(const aut_config *cfg) {
    if (check_config(cfg) != AUT_OK) return 0;
    return prepared_layout(cfg).total;
}

extern "C" aut_status aut_prepare_weights(const aut_config *cfg, const aut_weights *src, void *dst,
                                          size_t dst_bytes, aut_weights *prepared,
                                          aut_stream_t stream) {
    AUT_TRY(check_config(cfg));
    if (!src || !dst || !prepared || !src->conv2_w || !src->conv3_w || !src->conv_out_w ||
        !src->proj1_w || !src->proj2_w)
        return AUT_ERR_INVALID_ARG;
    const PreparedLayout p = prepared_layout(cfg);
    if (dst_bytes < p.total) return AUT_ERR_WORKSPACE;
    if (reinterpret_cast<uintptr_t>(dst) & 255u) return AUT_ERR_INVALID_ARG;
    uint8_t *base = static_cast<uint8_t *>(dst);
    aut_weights out = *src;
    out.conv2_w_tap = base + p.conv2;
    out.conv3_w_tap = base + p.conv3;
    out.conv_out_w_fc = base + p.conv_out;
    out.pos_table = base + p.pos;
    out.proj1_w_dup = base + p.proj1_dup;
    out.proj2_w_dup = base + p.proj2_dup;
    out.o_w_f16 = base + p.o_f16;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    for (int l = 0; l < cfg->layers; ++l) {
        if (!src->layers || !src->layers[l].o_w) return AUT_ERR_INVALID_ARG;
        AUT_TRY(cuda_status(launch_to_f16(src->layers[l].o_w,
                                          base + p.o_f16 + (size_t)l * cfg->d_model * cfg->d_model * 2,
                                          (size_t)cfg->d_model * cfg->d_model, st)));
    }
    AUT_TRY(cuda_status(launch_duplicate_k(src->proj1_w, base + p.proj1_dup, cfg->d_model,
                                           cfg->d_model, st)));
    AUT_TRY(cuda_status(launch_duplicate_k(src->proj2_w, base + p.proj2_dup, cfg->output_dim,
                                           cfg->d_model, st)));
    AUT_TRY(cuda_status(launch_prepare(src->conv2_w, src->conv3_w, src->conv_out_w,
                                       base + p.conv2, base + p.conv3, base + p.conv_out,
                                       reinterpret_cast<float *>(base + p.pos), cfg->conv_ch,
                                       cfg->d_model, reinterpret_cast<cudaStream_t>(stream))));
    *prepared = out;
    return AUT_OK;
}

extern "C" aut_status aut_encode(const aut_config *cfg, const aut_weights *prepared,
                                 const void *features, int32_t T_max, const int32_t *feature_lens,
                                 int32_t n_req, void *out, void *workspace, size_t ws_bytes,
                                 aut_stream_t stream) {
    return aut_encode_traced(cfg, prepared, features, T_max, feature_lens, n_req, out, workspace,
                             ws_bytes, stream, nullptr);
}

extern "C" aut_status aut_encode_traced(const aut_config *cfg, const aut_weights *prepared,
                                        const void *features, int32_t T_max,
                                        const int32_t *feature_lens, int32_t n_req, void *out,
                                        void *workspace, size_t ws_bytes, aut_stream_t stream,
                                        aut_trace *trace) {
    Plan p;
    AUT_TRY(build_plan(cfg, feature_lens, n_req, &p));
    AUT_TRY(check_features(p, features, T_max, feature_lens, n_req));
    if (!weights_complete(cfg, prepared, cfg->layers, true, true)) return AUT_ERR_INVALID_ARG;
    if (p.total_tokens > 0 && !out) return AUT_ERR_INVALID_ARG;
    if (reinterpret_cast<uintptr_t>(out) & 15u) return AUT_ERR_INVALID_ARG;
    Ctx c;
    AUT_TRY(make_ctx(cfg, prepared, workspace, ws_bytes, p, reinterpret_cast<cudaStream_t>(stream),
                     &c, trace));
    if (p.total_tokens == 0) return AUT_OK;
    AUT_TRY(upload_plan(c, p));
    float *x = c.at<float>(c.L.x);
    AUT_TRY(run_frontend(c, p, features, T_max, x, true));
    return run_encode(c, x, p.total_tokens, (int)p.cu_seqlens.size() - 1, cfg->layers, out);
}

extern "C" aut_status aut_frontend(const aut_config *cfg, const aut_weights *prepared,
                                   const void *features, int32_t T_max,
                                   const int32_t *feature_lens, int32_t n_req, void *x0,
                                   int32_t with_positions, void *workspace, size_t ws_bytes,
                                   aut_stream_t stream) {
    Plan p;
    AUT_TRY(build_plan(cfg, feature_lens, n_req, &p));
    AUT_TRY(check_features(p, features, T_max, feature_lens, n_req));
    if (!weights_complete(cfg, prepared, 0, true, false)) return AUT_ERR_INVALID_ARG;
    if (p.total_tokens > 0 && !x0) return AUT_ERR_INVALID_ARG;
    if (reinterpret_cast<uintptr_t>(x0) & 15u) return AUT_ERR_INVALID_ARG;
    Ctx c;
    AUT_TRY(make_ctx(cfg, prepared, workspace, ws_bytes, p, reinterpret_cast<cudaStream_t>(stream), &c));
    if (p.total_tokens == 0) return AUT_OK;
    AUT_TRY(upload_plan(c, p));
    return run_frontend(c, p, features, T_max, static_cast<float *>(x0), with_positions != 0);
}

extern "C" aut_status aut_encode_packed(const aut_config *cfg, const aut_weights *prepared,
                                        void *hidden, int32_t total_tokens,
                                        const int32_t *cu_seqlens, int32_t num_windows,
                                        int32_t n_layers, void *out, void *workspace,
                                        size_t ws_bytes, aut_stream_t stream) {
    AUT_TRY(check_config(cfg));
    if (total_tokens < 0 || num_windows < 0 || n_layers < 0 || n_layers > cfg->layers)
        return AUT_ERR_INVALID_ARG;
    if (!cu_seqlens || cu_seqlens[0] != 0 || cu_seqlens[num_windows] != total_tokens)
        return AUT_ERR_INVALID_ARG;
    for (int i = 0; i < num_windows; ++i) {
        const int len = cu_seqlens[i + 1] - cu_seqlens[i];
        if (len < 0 || len > kMaxWindowTokens) return AUT_ERR_INVALID_ARG;
    }
    if (!weights_complete(cfg, prepared, n_layers, false, out != nullptr)) return AUT_ERR_INVALID_ARG;
    if (total_tokens > 0 && !hidden) return AUT_ERR_INVALID_ARG;
    if (reinterpret_cast<uintptr_t>(hidden) & 15u) return AUT_ERR_INVALID_ARG;
    Plan p;
    p.total_tokens = total_tokens;
    p.cu_seqlens.assign(cu_seqlens, cu_seqlens + num_windows + 1);
    Ctx c;
    AUT_TRY(make_ctx(cfg, prepared, workspace, ws_bytes, p, reinterpret_cast<cudaStream_t>(stream), &c));
    if (total_tokens == 0) return AUT_OK;
    std::vector<int32_t> words;
    append_windows(words, p.cu_seqlens);
    AUT_TRY(cuda_status(launch_upload(words.data(), words.size(), c.at<int32_t>(c.L.cu), c.st)));
    return run_encode(c, static_cast<float *>(hidden), total_tokens, num_windows, n_layers, out);
}

extern "C" aut_status aut_linear(const void *x, const void *w, const void *bias, void *y, int32_t M,
                                 int32_t N, int32_t K, int32_t epilogue, int32_t *status,
                                 int32_t timeout_ms, int32_t flags, aut_stream_t stream) {
    if (M < 0 || N <= 0 || K <= 0 || epilogue < 0 || epilogue > 3 || timeout_ms < 0)
        return AUT_ERR_INVALID_ARG;
    if (M > 0 && (!x || !w || !y)) return AUT_ERR_INVALID_ARG;
    if (K % 64 || N % 16) return AUT_ERR_UNSUPPORTED;
    LinearLaunch L{};
    L.a = x;
    L.w = w;
    L.bias = bias;
    L.out = y;
    L.M = M;
    L.N = N;
    L.K = K;
    L.ldo = N;
    L.epi = epilogue == 3 ? kEpiF32 : epilogue;
    L.status = reinterpret_cast<int *>(status);
    L.timeout_ns = timeout_ms ? (unsigned long long)timeout_ms * 1000000ull : kDefaultTimeoutNs;
    L.fault_inject = (flags & AUT_LINEAR_FAULT_INJECT) ? 1 : 0;
    L.single_cta = (flags & AUT_LINEAR_SINGLE_CTA) != 0;
    L.f16 = (flags & AUT_LINEAR_F16) != 0;
    return gemm_status(launch_linear(L, reinterpret_cast<cudaStream_t>(stream)));
}

extern "C" aut_status aut_layernorm(const void *x, const void *gamma, const void *beta, void *y,
                                    int32_t T, int32_t d, float eps, aut_stream_t stream) {
    if (T < 0 || d <= 0 || d % 4 || d > 2048 || !(eps >= 0.f)) return AUT_ERR_INVALID_ARG;
    if (T > 0 && (!x || !gamma || !beta || !y)) return AUT_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(x) | reinterpret_cast<uintptr_t>(y) |
         reinterpret_cast<uintptr_t>(gamma) | reinterpret_cast<uintptr_t>(beta)) & 7u)
        return AUT_ERR_INVALID_ARG;
    return cuda_status(launch_layernorm(static_cast<const float *>(x), gamma, beta, y, T, d, eps,
                                        reinterpret_cast<cudaStream_t>(stream)));
}

extern "C" aut_status aut_window_attention(const void *qkv, void *out, int32_t T, int32_t d,
                                           int32_t heads, const int32_t *cu_seqlens,
                                           int32_t num_windows, void *workspace, size_t ws_bytes,
                                           aut_stream_t stream) {
    return aut_window_attention_ex(qkv, out, T, d, heads, cu_seqlens, num_windows, workspace,
                                   ws_bytes, 0, 0, stream);
}

extern "C" aut_status aut_window_attention_ex(const void *qkv, void *out, int32_t T, int32_t d,
                                              int32_t heads, const int32_t *cu_seqlens,
                                              int32_t num_windows, void *workspace,
                                              size_t ws_bytes, int32_t timeout_ms, int32_t flags,
                                              aut_stream_t stream) {
    if (timeout_ms < 0 || (flags & ~AUT_ATTN_FAULT_INJECT)) return AUT_ERR_INVALID_ARG;
    if (T < 0 || d <= 0 || heads <= 0 || d % heads || num_windows < 0 || !cu_seqlens)
        return AUT_ERR_INVALID_ARG;
    const int hd = d / heads;
    if (hd != 16 && hd != 32 && hd != 64 && hd != 128) return AUT_ERR_UNSUPPORTED;
    if (cu_seqlens[0] != 0 || cu_seqlens[num_windows] != T) return AUT_ERR_INVALID_ARG;
    for (int i = 0; i < num_windows; ++i) {
        const int len = cu_seqlens[i + 1] - cu_seqlens[i];
        if (len < 0 || len > kMaxWindowTokens) return AUT_ERR_INVALID_ARG;
    }
    if (T > 0 && (!qkv || !out)) return AUT_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(qkv) | reinterpret_cast<uintptr_t>(out)) & 15u)
        return AUT_ERR_INVALID_ARG;
    if (!workspace || ws_bytes < (size_t)(num_windows + 2) * 4) return AUT_ERR_WORKSPACE;
    if (reinterpret_cast<uintptr_t>(workspace) & 3u) return AUT_ERR_INVALID_ARG;
    if (T == 0) return AUT_OK;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    // Workspace words: [0] the status word (cleared here), [1 ..] cu_seqlens.
    std::vector<int32_t> words(1, 0);
    words.insert(words.end(), cu_seqlens, cu_seqlens + num_windows + 1);
    int32_t *ws = static_cast<int32_t *>(workspace);
    AUT_TRY(cuda_status(launch_upload(words.data(), words.size(), ws, st)));
    const bool fault = (flags & AUT_ATTN_FAULT_INJECT) != 0;
    if (fault && !window_attention_uses_tc(d, heads, T)) return AUT_ERR_UNSUPPORTED;
    return cuda_status(launch_window_attention(
        qkv, out, ws + 1, num_windows, d, heads, st, T, ws, false,
        timeout_ms ? (unsigned long long)timeout_ms * 1000000ull : 0ull, fault ? 1 : 0));
}

extern "C" aut_status aut_check_status_word(int32_t *status) {
    if (!status) AUT_TRY(noalloc_status_word(&status));
    int32_t v = 0;
    if (cudaMemcpy(&v, status, sizeof(v), cudaMemcpyDeviceToHost) != cudaSuccess) return AUT_ERR_CUDA;
    const int32_t zero = 0;
    if (cudaMemcpy(status, &zero, sizeof(zero), cudaMemcpyHostToDevice) != cudaSuccess)
        return AUT_ERR_CUDA;
    return static_cast<aut_status>(v);
}

extern "C" aut_status aut_check(void *workspace) {
    if (!workspace) return AUT_ERR_INVALID_ARG;
    return aut_check_status_word(static_cast<int32_t *>(workspace));
}
