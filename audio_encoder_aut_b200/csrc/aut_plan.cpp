// Host-side layout planner: token counts, cu_seqlens and the chunk table.
//
// Follows the m-star.org page "mstar.model.components.aut_encoder":
// AuTEncoder.layout ("host-side arithmetic only"), AuTEncoderConfig.tokens_for_frames
// (13 tokens per full 100-frame chunk plus three stride-2 convolutions' worth of
// the remainder) and window_lengths (full windows, then the remainder), with the
// per-axis output size of Conv2d(k3, s2, p1) from openarchlab "1A . AuT Audio
// Encoder", section 3: L_out = floor((L_in + 1) / 2).
#include "aut_internal.h"

#include <limits>

namespace aut {

int stride2_len(int n) { return n > 0 ? (n + 1) / 2 : 0; }

int stem_len(int n) { return stride2_len(stride2_len(stride2_len(n))); }

aut_status check_config(const aut_config *c) {
    if (!c) return AUT_ERR_INVALID_ARG;
    if (c->d_model <= 0 || c->layers < 0 || c->heads <= 0 || c->ffn <= 0 || c->conv_ch <= 0 ||
        c->output_dim <= 0 || c->n_window <= 0 || c->n_window_infer <= 0 ||
        c->conv_chunksize <= 0 || !(c->ln_eps >= 0.f))
        return AUT_ERR_INVALID_ARG;
    if (c->mel_bins != kMelBins || c->n_window != kChunkFrames / 2) return AUT_ERR_UNSUPPORTED;
    if (c->n_window_infer % kChunkFrames != 0) return AUT_ERR_UNSUPPORTED;
    if (window_tokens(c) > kMaxWindowTokens) return AUT_ERR_UNSUPPORTED;
    if (c->d_model % c->heads != 0) return AUT_ERR_UNSUPPORTED;
    int hd = c->d_model / c->heads;
    if (hd != 16 && hd != 32 && hd != 64 && hd != 128) return AUT_ERR_UNSUPPORTED;
    if (c->d_model % 64 != 0 || c->d_model > 2048 || c->ffn % 64 != 0) return AUT_ERR_UNSUPPORTED;
    if (c->output_dim % 16 != 0) return AUT_ERR_UNSUPPORTED;
    if (conv_tile_n(c->conv_ch) == 0) return AUT_ERR_UNSUPPORTED;
    return AUT_OK;
}

int window_tokens(const aut_config *c) {
    return stem_len(kChunkFrames) * (c->n_window_infer / kChunkFrames);
}

int conv_tile_n(int C) {
    // Conv GEMM tile widths the library instantiates; C above 256 takes two tiles.
    static const int kWidths[] = {16, 32, 64, 128, 192, 240, 256};
    auto has = [](int v) {
        for (int w : kWidths)
            if (w == v) return true;
        return false;
    };
    if (C <= 256) return has(C) ? C : 0;
    if (C % 2 == 0 && has(C / 2)) return C / 2;
    return 0;
}

aut_status build_plan(const aut_config *cfg, const int32_t *lens, int32_t n_req, Plan *p) {
    aut_status st = check_config(cfg);
    if (st != AUT_OK) return st;
    if (n_req < 0 || (n_req > 0 && !lens)) return AUT_ERR_INVALID_ARG;
    const int w = window_tokens(cfg);
    const int tpc = stem_len(kChunkFrames);
    p->tokens_per_request.assign(n_req, 0);
    p->cu_seqlens.assign(1, 0);
    p->chunks.clear();
    int64_t row = 0;
    for (int r = 0; r < n_req; ++r) {
        const int64_t n = lens[r];
        if (n < 0) return AUT_ERR_INVALID_ARG;
        const int64_t full = n / kChunkFrames, rem = n % kChunkFrames;
        const int64_t t = full * tpc + stem_len((int)rem);
        if (row + t > std::numeric_limits<int32_t>::max()) return AUT_ERR_INVALID_ARG;
        p->tokens_per_request[r] = (int32_t)t;
        for (int64_t k = 0; k < t / w; ++k) p->cu_seqlens.push_back(p->cu_seqlens.back() + w);
        if (t % w) p->cu_seqlens.push_back(p->cu_seqlens.back() + (int32_t)(t % w));
        const int64_t nchunks = full + (rem ? 1 : 0);
        for (int64_t k = 0; k < nchunks; ++k) {
            ChunkInfo ci;
            ci.request = r;
            ci.frame0 = (int32_t)(k * kChunkFrames);
            ci.valid_frames = (int32_t)std::min<int64_t>(kChunkFrames, n - k * kChunkFrames);
            ci.token0 = (int32_t)row;
            row += stem_len(ci.valid_frames);
            p->chunks.push_back(ci);
        }
    }
    p->total_tokens = (int32_t)row;
    return AUT_OK;
}

}  // namespace aut

extern "C" aut_status aut_plan(const aut_config *cfg, const int32_t *feature_lens, int32_t n_req,
                               int32_t *tokens_per_request, int32_t *cu_seqlens,
                               int32_t *total_tokens, int32_t *num_windows, int32_t *num_chunks) {
    aut::Plan p;
    aut_status st = aut::build_plan(cfg, feature_lens, n_req, &p);
    if (st != AUT_OK) return st;
    if (tokens_per_request)
        std::copy(p.tokens_per_request.begin(), p.tokens_per_request.end(), tokens_per_request);
    if (cu_seqlens) std::copy(p.cu_seqlens.begin(), p.cu_seqlens.end(), cu_seqlens);
    if (total_tokens) *total_tokens = p.total_tokens;
    if (num_windows) *num_windows = (int32_t)p.cu_seqlens.size() - 1;
    if (num_chunks) *num_chunks = (int32_t)p.chunks.size();
    return AUT_OK;
}

extern "C" const char *aut_status_string(aut_status s) {
    switch (s) {
        case AUT_OK: return "ok";
        case AUT_ERR_INVALID_ARG: return "invalid argument";
        case AUT_ERR_UNSUPPORTED: return "unsupported configuration";
        case AUT_ERR_WORKSPACE: return "workspace or destination too small";
        case AUT_ERR_CUDA: return "CUDA error";
        case AUT_ERR_TIMEOUT: return "device pipeline wait timed out";
        case AUT_ERR_BOUNDS: return "device index out of bounds (debug build)";
    }
    return "unknown status";
}
