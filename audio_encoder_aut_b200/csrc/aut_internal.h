// Internal host-side declarations shared by the planner, the launch code and
// the kernels' host wrappers.  Not part of the public ABI (that is include/aut.h).
#pragma once

#include <algorithm>
#include <cstddef>
#include <cstdint>
#include <vector>

#include "../../include/aut.h"

namespace aut {

constexpr int kMelBins = 128;        // num_mel_bins the stem geometry is built for
constexpr int kChunkFrames = 100;    // 2 * n_window
constexpr int kMaxWindowTokens = 128;
constexpr int kTokensPerChunk = 13;  // stem_len(100)
constexpr int kStemRows = 16;        // stem_len(128): mel rows after the stem

// Stem geometry (one 128 x 100 chunk).  The outputs of conv1 and conv2 are
// stored as four stride-2 phase planes with one zero row and one zero column in
// front (see the conv kernels), so that every filter tap of the next conv reads
// a plain rectangle.
constexpr int kC1Rows = 64, kC1Cols = 50;                       // conv1 output (H, W)
constexpr int kP1Rows = kC1Rows / 2 + 1, kP1Cols = kC1Cols / 2 + 1;  // 33 x 26 planes
constexpr int kC2Rows = 32, kC2Cols = 25;                       // conv2 output
constexpr int kP2Rows = kC2Rows / 2 + 1, kP2Cols = (kC2Cols + 1) / 2 + 1;  // 17 x 14 planes
constexpr int kC3Rows = 16, kC3Cols = 13;                       // conv3 output

struct ChunkInfo {  // mirrors the device int4 chunk record
    int32_t request, frame0, valid_frames, token0;
};

struct Plan {
    std::vector<int32_t> tokens_per_request;
    std::vector<int32_t> cu_seqlens;
    std::vector<ChunkInfo> chunks;
    int32_t total_tokens = 0;
};

int stride2_len(int n);
int stem_len(int n);
int window_tokens(const aut_config *c);
int conv_tile_n(int C);
aut_status check_config(const aut_config *c);
aut_status build_plan(const aut_config *cfg, const int32_t *lens, int32_t n_req, Plan *p);

// Device workspace carve-up (byte offsets, every region 1024-aligned).
struct WorkspaceLayout {
    size_t status, chunks, cu, x, xn, qkv, attn, ffn, planes1, planes2, y3, total;
    int group_chunks;  // chunk capacity of the stem buffers
};
WorkspaceLayout workspace_layout(const aut_config *c, int64_t T, int64_t nW, int64_t n_ch);

// Device address, on the current device, of the status word the
// allocation-free window attention writes (aut_noalloc.cu).
aut_status noalloc_status_word(int32_t **out);

}  // namespace aut
