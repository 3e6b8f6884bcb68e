/*
 * aut.h -- C ABI of the AuT (Qwen3-family) audio encoder forward pass on B200.
 *
 * The library computes what the m-star.org page "mstar.model.components.aut_encoder"
 * calls AuTEncoder.forward(features, feature_lens): a host-side layout step
 * (AuTEncoder.layout) followed by the device-side front end (AuTEncoder.frontend:
 * 100-frame chunks -> three Conv2d(k3, s2, p1) + GELU -> conv_out -> + sinusoids ->
 * packed tokens) and the packed transformer stack and projector
 * (AuTEncoder.encode: pre-LayerNorm layers whose attention is block-diagonal over
 * cu_seqlens windows, then a final LayerNorm and a Linear-GELU-Linear projector).
 *
 * Conventions shared by every entry point
 *   - Ownership: the caller allocates every buffer.  The library allocates no
 *     device memory and keeps no per-call state; device pointers are plain
 *     addresses on the current CUDA device.
 *   - Streams: device work is enqueued on `stream` and returns before it ends
 *     (asynchronous); host buffers passed in are read before the call returns.
 *   - Types: every parameter and the features are bf16 (stored as 16-bit
 *     words); the residual stream ("hidden") and the encoder output are fp32.
 *   - Layouts are row-major.  Linear weights follow PyTorch: [out, in].  Conv
 *     weights are [C_out, C_in, 3, 3].  The fused qkv weight stacks q, k, v on
 *     dim 0 ([3 d, d]) and head h uses columns [h*hd, (h+1)*hd) of each.
 *   - Errors: argument errors return before anything is launched.  A failed
 *     launch returns AUT_ERR_CUDA.  Faults found on the device (a pipeline wait
 *     that ran out of time) are written to a status word in the workspace and
 *     returned by aut_check() after the caller has synchronised the stream.
 */
#ifndef AUT_H_
#define AUT_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st *aut_stream_t; /* a cudaStream_t; NULL = legacy default stream */

typedef enum {
    AUT_OK = 0,
    AUT_ERR_INVALID_ARG = 1,  /* null pointer, negative length, length > T_max, ... */
    AUT_ERR_UNSUPPORTED = 2,  /* configuration outside what the kernels implement */
    AUT_ERR_WORKSPACE = 3,    /* workspace or destination buffer too small */
    AUT_ERR_CUDA = 4,         /* a CUDA runtime call or launch failed */
    AUT_ERR_TIMEOUT = 5,      /* a device pipeline wait ran out of time (from aut_check) */
    AUT_ERR_BOUNDS = 6        /* debug builds (libaut_debug.so, -DAUT_DEBUG_BOUNDS): a kernel
                               * computed an address outside its buffer and skipped the
                               * access (from aut_check) */
} aut_status;

/* Encoder hyper-parameters; field meaning follows AuTEncoderConfig on the
 * aut_encoder page.  Supported: mel_bins = 128, n_window = 50 (100-frame chunks),
 * n_window_infer a multiple of 100 with at most 128 tokens per window,
 * head_dim = d_model / heads in {16, 32, 64, 128}, d_model a multiple of 64 and
 * at most 2048, ffn a multiple of 64, output_dim a multiple of 16, conv_ch one of
 * 16, 32, 64, 128, 192, 240, 256, 384, 480, 512. */
typedef struct {
    int32_t d_model;         /* d */
    int32_t layers;          /* encoder_layers */
    int32_t heads;           /* encoder_attention_heads */
    int32_t ffn;             /* encoder_ffn_dim */
    int32_t mel_bins;        /* num_mel_bins (128) */
    int32_t n_window;        /* half the chunk length in frames (50) */
    int32_t n_window_infer;  /* attention window in frames (800 -> 104 tokens) */
    int32_t conv_ch;         /* downsample_hidden_size C */
    int32_t output_dim;      /* projector output width */
    int32_t conv_chunksize;  /* chunks the conv stem processes per group */
    float ln_eps;            /* LayerNorm epsilon */
} aut_config;

/* One encoder layer's parameters (device pointers, bf16).  Shapes:
 * ln1_w/ln1_b/ln2_w/ln2_b/o_b/fc2_b [d]; qkv_w [3d, d]; qkv_b [3d]; o_w [d, d];
 * fc1_w [ffn, d]; fc1_b [ffn]; fc2_w [d, ffn]. */
typedef struct {
    const void *ln1_w, *ln1_b, *qkv_w, *qkv_b, *o_w, *o_b;
    const void *ln2_w, *ln2_b, *fc1_w, *fc1_b, *fc2_w, *fc2_b;
} aut_layer_weights;

/* Whole-encoder parameters.  All pointers are device bf16 except `layers`,
 * a HOST array of cfg.layers entries that must outlive every call using it.
 * conv1_w [C,1,3,3]; conv2_w, conv3_w [C,C,3,3]; conv{1,2,3}_b [C];
 * conv_out_w [d, C*16] with input index c*16 + f (f = mel row after the stem);
 * conv_out_b [d] or NULL; ln_post_w/b [d]; proj1_w [d,d]; proj1_b [d];
 * proj2_w [output_dim, d]; proj2_b [output_dim]. */
typedef struct {
    const void *conv1_w, *conv1_b, *conv2_w, *conv2_b, *conv3_w, *conv3_b;
    const void *conv_out_w, *conv_out_b;
    const aut_layer_weights *layers;
    const void *ln_post_w, *ln_post_b, *proj1_w, *proj1_b, *proj2_w, *proj2_b;
    /* Filled by aut_prepare_weights, NULL in caller-built structs: kernel-layout
     * copies of conv2_w/conv3_w ([C][9][C]: out, tap, in), conv_out_w
     * ([d][16*C]: index f*C + c), the fp32 sinusoid table [13][d], and the
     * projector weights repeated along K ([d][2d], [output_dim][2d]) for the
     * two-term (hi + lo bf16) projector operands. */
    const void *conv2_w_tap, *conv3_w_tap, *conv_out_w_fc, *pos_table;
    const void *proj1_w_dup, *proj2_w_dup;
    const void *o_w_f16; /* fp16 [layers][d][d]: every layer's o_proj weight in fp16 (the
                          * operand type of the attention output) */
} aut_weights;

/* aut_encoder page, AuTEncoder.layout / AuTEncoderConfig.tokens_for_frames /
 * window_lengths / AuTLayout.  Host arithmetic only; nothing touches a GPU.
 * feature_lens [n_req] are mel frame counts (>= 0; 0 gives an empty request).
 * Outputs (each may be NULL): tokens_per_request [n_req]; cu_seqlens
 * [num_windows + 1] (call once with cu_seqlens = NULL to learn num_windows);
 * total_tokens; num_windows; num_chunks (100-frame chunks, the partial last
 * chunk of each request included).  Requests are packed in input order and a
 * window never spans two requests. */
aut_status aut_plan(const aut_config *cfg, const int32_t *feature_lens, int32_t n_req,
                    int32_t *tokens_per_request, int32_t *cu_seqlens,
                    int32_t *total_tokens, int32_t *num_windows, int32_t *num_chunks);

/* No passage: a library helper.  Bytes of device workspace that aut_encode /
 * aut_frontend / aut_encode_packed need for a batch with these plan totals
 * (from aut_plan).  Returns 0 for an unsupported configuration. */
size_t aut_workspace_bytes(const aut_config *cfg, int32_t total_tokens, int32_t num_windows,
                           int32_t num_chunks);

/* No passage: a library helper.  Bytes of the device buffer aut_prepare_weights
 * fills. */
size_t aut_prepared_bytes(const aut_config *cfg);

/* One-time weight preparation (cubic.dev "Audio Encoder Component", Weight
 * Transposition: conv weights are re-laid-out channel-last for the kernels).
 * Writes into `dst` (device, dst_bytes >= aut_prepared_bytes) the tap-major conv2
 * and conv3 weights, conv_out's columns reordered to the stem's output order,
 * the sinusoid table (aut_encoder page, module docstring: the same 13 positions
 * for every chunk), every layer's o_proj weight converted to fp16, and the
 * K-repeated projector weights.  Copies `src` into `*prepared` and points the
 * seven prepared fields into `dst`.  Asynchronous on `stream`; src stays owned
 * by the caller and must stay alive while `prepared` is used. */
aut_status aut_prepare_weights(const aut_config *cfg, const aut_weights *src, void *dst,
                               size_t dst_bytes, aut_weights *prepared, aut_stream_t stream);

/* aut_encoder page, AuTEncoder.forward: features -> [total_tokens, output_dim].
 * features: device bf16 [n_req, mel_bins, T_max], time fastest; frames at or
 * after feature_lens[r] are treated as zero whatever the buffer holds.
 * feature_lens: HOST int32 [n_req], each in [0, T_max].  out: device fp32
 * [total_tokens, output_dim], rows in packed order (requests in input order,
 * tokens in time order).  workspace: device, ws_bytes >= aut_workspace_bytes.
 * `prepared` comes from aut_prepare_weights. */
aut_status aut_encode(const aut_config *cfg, const aut_weights *prepared, const void *features,
                      int32_t T_max, const int32_t *feature_lens, int32_t n_req, void *out,
                      void *workspace, size_t ws_bytes, aut_stream_t stream);

/* Kernel kinds reported by aut_encode_traced. */
typedef enum {
    AUT_K_UPLOAD = 0,    /* plan tables to the device */
    AUT_K_ZERO_PADS = 1, /* (no longer launched: conv1 writes the planes' zero borders) */
    AUT_K_CONV1 = 2,
    AUT_K_CONV2 = 3,
    AUT_K_CONV3 = 4,
    AUT_K_CONV_OUT = 5,  /* conv_out + positions + packing */
    AUT_K_LAYERNORM = 6,
    AUT_K_QKV = 7,
    AUT_K_ATTENTION = 8,
    AUT_K_O_PROJ = 9,
    AUT_K_FC1 = 10,
    AUT_K_FC2 = 11,
    AUT_K_PROJ1 = 12,
    AUT_K_PROJ2 = 13
} aut_kernel_kind;

/* Per-kernel trace, the CUDA-event timing of each stage.  events: caller-created
 * cudaEvent_t handles (NULL with capacity 0 to only count); kinds: int32
 * [capacity] or NULL.  The library records events[i] on the stream right after
 * its i-th kernel launch and stores the kernel's aut_kernel_kind in kinds[i];
 * count receives the number of kernels launched (even beyond capacity).  The
 * records are external (cudaEventRecordExternal), so under stream capture they
 * become event-record nodes of the graph, re-recorded on every replay. */
typedef struct {
    void **events;
    int32_t capacity;
    int32_t count;
    int32_t *kinds;
} aut_trace;

/* aut_encode with a per-kernel trace (trace may be NULL). */
aut_status aut_encode_traced(const aut_config *cfg, const aut_weights *prepared,
                             const void *features, int32_t T_max, const int32_t *feature_lens,
                             int32_t n_req, void *out, void *workspace, size_t ws_bytes,
                             aut_stream_t stream, aut_trace *trace);

/* aut_encoder page, AuTEncoder.frontend: features -> packed chunk embeddings
 * x0, device fp32 [total_tokens, d_model].  with_positions = 0 leaves out the
 * sinusoid add (the conv_out output itself, for stage-wise checking).
 * Other arguments as for aut_encode. */
aut_status aut_frontend(const aut_config *cfg, const aut_weights *prepared, const void *features,
                        int32_t T_max, const int32_t *feature_lens, int32_t n_req, void *x0,
                        int32_t with_positions, void *workspace, size_t ws_bytes,
                        aut_stream_t stream);

/* aut_encoder page, AuTEncoder.encode: the transformer stack (and projector)
 * over a packed sequence.  hidden: device fp32 [total_tokens, d_model], the
 * residual stream, updated in place by layers [0, n_layers).  cu_seqlens: HOST
 * int32 [num_windows + 1], non-decreasing from 0 to total_tokens, every window at
 * most 128 tokens.  If out (device fp32 [total_tokens, output_dim]) is not NULL,
 * the final LayerNorm and projector run after the layers and write it. */
aut_status aut_encode_packed(const aut_config *cfg, const aut_weights *prepared, void *hidden,
                             int32_t total_tokens, const int32_t *cu_seqlens,
                             int32_t num_windows, int32_t n_layers, void *out, void *workspace,
                             size_t ws_bytes, aut_stream_t stream);

/* A linear layer Y = X W^T + b on the tensor cores (every GEMM of the path: the
 * fused qkv_proj of the aut_encoder page, o_proj, fc1/fc2 of the FFN, the
 * projector), exposed for kernel-level checks.  x: device bf16 [M, K]; w: device
 * bf16 [N, K]; bias: device bf16 [N] or NULL.  epilogue 0: y bf16 [M, N] =
 * acc + b; 1: y bf16 = GELU(acc + b); 2: y fp32 [M, N] += acc + b (residual add);
 * 3: y fp32 [M, N] = acc + b.
 * K must be a multiple of 64 and N a multiple of 16.  status: device int32 word
 * for device-side faults (may be NULL).  timeout_ms bounds every pipeline wait
 * (0 = default of 4000 ms).  flags: AUT_LINEAR_FAULT_INJECT makes the first block
 * skip its first operand load so that its consumer's wait runs out (tests of the
 * timeout path only); AUT_LINEAR_SINGLE_CTA keeps every MMA on one SM (no CTA
 * pairs); AUT_LINEAR_F16 takes x and w as fp16 instead of bf16 (the o_proj
 * GEMM over the fp16 attention output); 0 for normal use. */
#define AUT_LINEAR_FAULT_INJECT 1
#define AUT_LINEAR_SINGLE_CTA 2
#define AUT_LINEAR_F16 4
aut_status aut_linear(const void *x, const void *w, const void *bias, void *y, int32_t M,
                      int32_t N, int32_t K, int32_t epilogue, int32_t *status,
                      int32_t timeout_ms, int32_t flags, aut_stream_t stream);

/* LayerNorm with bias over the last dim (cubic.dev "Audio Encoder Component",
 * Transformer Encoder Layers): y = (x - mean) / sqrt(var + eps) * gamma + beta,
 * biased variance.  x: device fp32 [T, d]; gamma, beta: device bf16 [d];
 * y: device bf16 [T, d].  d a multiple of 4, at most 2048. */
aut_status aut_layernorm(const void *x, const void *gamma, const void *beta, void *y,
                         int32_t T, int32_t d, float eps, aut_stream_t stream);

/* Window attention (aut_encoder page, AuTAttention; openarchlab "1A . AuT Audio
 * Encoder", section 3: non-causal attention limited to each cu_seqlens segment):
 * for every segment and head, softmax(Q K^T / sqrt(hd)) V.  qkv: device bf16
 * [T, 3 d] (q | k | v); out: device fp16 [T, d] (11 significant bits, 8x
 * finer than bf16; values beyond +-65504 saturate), the operand of the fp16
 * o_proj GEMM.  The probabilities P enter the P V product as fp16 for head_dim
 * 64 (tensor-core path) and as two bf16 terms otherwise.  cu_seqlens: HOST int32
 * [num_windows + 1], every window at most 128 tokens.  workspace: device, 4-byte
 * aligned, at least 4 * (num_windows + 2) bytes: word 0 is the call's status
 * word (aut_check(workspace) reads it after the stream is synchronised), the
 * rest the uploaded cu_seqlens. */
aut_status aut_window_attention(const void *qkv, void *out, int32_t T, int32_t d, int32_t heads,
                                const int32_t *cu_seqlens, int32_t num_windows,
                                void *workspace, size_t ws_bytes, aut_stream_t stream);

/* aut_window_attention with control over its failure path, for tests:
 * timeout_ms bounds every pipeline wait of the head_dim-64 tensor-core kernel
 * (0 = default of 4000 ms); flags AUT_ATTN_FAULT_INJECT leaves the first
 * block's first operand stage unfilled, so that its consumers' waits run out,
 * the kernel writes AUT_ERR_TIMEOUT to the workspace's status word and returns
 * (head_dim 64 only; AUT_ERR_UNSUPPORTED otherwise); 0 for normal use. */
#define AUT_ATTN_FAULT_INJECT 1
aut_status aut_window_attention_ex(const void *qkv, void *out, int32_t T, int32_t d,
                                   int32_t heads, const int32_t *cu_seqlens, int32_t num_windows,
                                   void *workspace, size_t ws_bytes, int32_t timeout_ms,
                                   int32_t flags, aut_stream_t stream);

/* Window attention that allocates nothing, for callers that cannot allocate
 * device memory: code whose device memory belongs to another allocator that
 * forbids raw cudaMalloc, or code running where allocation is not allowed
 * (for example during a CUDA-graph capture that rejects allocation calls).
 * There is no counterpart in the paper; this computes exactly what
 * aut_window_attention computes, with the same argument meanings, but keeps
 * its scratch (the uploaded cu_seqlens) in a file-scope device array of the
 * library instead of a caller workspace.
 * Limits and behaviour:
 *   - num_windows at most 32766 (128 KiB of scratch: one status word and
 *     cu_seqlens); larger returns AUT_ERR_WORKSPACE before anything is
 *     launched.
 *   - Device-side faults (a pipeline wait that ran out of time) go to a status
 *     word in the same array, cleared by every call; aut_check_status_word(NULL)
 *     reads and clears it for the current device after the stream is
 *     synchronised.
 *   - The first call on each device looks up the array's device address (with
 *     that device current) and caches it; make that first call before any
 *     stream capture.
 *   - Every GPU that loads the library holds the array until the process
 *     exits.
 *   - All calls share the array, which keeps the last call's contents: calls
 *     that overlap on the GPU (unordered streams) race and must not be issued.
 *   - No cudaMalloc, cudaFree or allocating library routine is called. */
aut_status aut_window_attention_noalloc(const void *qkv, void *out, int32_t T, int32_t d,
                                        int32_t heads, const int32_t *cu_seqlens,
                                        int32_t num_windows, aut_stream_t stream);

/* Log-mel front end (cubic.dev "Audio Encoder Component", Feature Extraction
 * Pipeline: 16 kHz mono audio -> 128-bin mel spectrogram; m-star.org
 * aut_encoder page, module docstring: Whisper-style log-mel, 100 frames/s).
 * The steps the pages leave open follow Whisper's recipe: 400-sample periodic
 * Hann frames every 160 samples, centred, the signal reflected by 200 samples
 * at both ends; power of the 400-point DFT; 128 Slaney mel filters of unit
 * area over 0..8000 Hz; log10 of max(energy, 1e-10); the transform's last
 * frame dropped, so n samples give n / 160 frames; per request, values raised
 * to at least (that request's maximum - 8); then (x + 4) / 4.
 * waveform: device fp32 [n_req, S_max] (request r's first sample_lens[r]
 * samples are used).  sample_lens: HOST int32 [n_req], each 0 or in
 * (200, S_max].  features: device bf16 [n_req, 128, T_max], T_max at least the
 * longest request's frames; written whole (zeros past each request's frames),
 * ready for aut_encode.  feature_lens: HOST int32 [n_req] out (may be NULL):
 * sample_lens[r] / 160.  workspace: device, 256-byte aligned, at least
 * aut_logmel_workspace_bytes(n_req, T_max).  Argument errors return before any
 * launch; asynchronous on `stream`. */
aut_status aut_logmel(const void *waveform, int64_t S_max, const int32_t *sample_lens,
                      int32_t n_req, void *features, int32_t T_max, int32_t *feature_lens,
                      void *workspace, size_t ws_bytes, aut_stream_t stream);

/* No passage: a library helper.  Bytes of device workspace aut_logmel needs. */
size_t aut_logmel_workspace_bytes(int32_t n_req, int32_t T_max);

/* Audio injection into the decoder's input (cubic.dev "Audio Encoder
 * Component", Audio Injection Logic: the encoder's features replace the
 * embeddings at the <|audio_pad|> placeholder positions).  The j-th position
 * (in sequence order) whose token id equals audio_pad_id receives row j of
 * `audio`; every other row of `embeds` is left as it is.
 * embeds: device bf16 [L, D], updated in place (8-byte aligned); token_ids:
 * device int32 [L]; audio: device fp32 [T, D] (16-byte aligned), e.g. the
 * output of aut_encode (rows in packed order), rounded to bf16 (nearest even)
 * on the way in.  workspace: device, 256-byte aligned, at least
 * aut_inject_workspace_bytes(L).  The number of placeholders is counted on the
 * device: if it is not T, aut_check(workspace) reports AUT_ERR_INVALID_ARG
 * after the stream is synchronised and no row past T is read (placeholders
 * beyond the T-th keep their embeddings).  Asynchronous on `stream`. */
aut_status aut_inject_audio(void *embeds, const int32_t *token_ids, int32_t L,
                            int32_t audio_pad_id, const void *audio, int32_t T, int32_t D,
                            void *workspace, size_t ws_bytes, aut_stream_t stream);

/* No passage: a library helper.  Bytes of device workspace aut_inject_audio needs. */
size_t aut_inject_workspace_bytes(int32_t L);

/* No passage: a library helper.  Reads and clears the device status word of a
 * workspace used by aut_window_attention or by aut_encode /
 * aut_frontend / aut_encode_packed (synchronous: call after the stream is
 * synchronised).  Each of those calls clears the word when it starts, so this
 * reports the first device-side fault of the latest call on the workspace. */
aut_status aut_check(void *workspace);

/* No passage: a library helper.  Reads and clears a status word given to
 * aut_linear (synchronous).  NULL
 * selects the status word of aut_window_attention_noalloc on the current
 * device. */
aut_status aut_check_status_word(int32_t *status);

/* No passage: a library helper.  Static text for a status code. */
const char *aut_status_string(aut_status status);

#ifdef __cplusplus
}
#endif

#endif /* AUT_H_ */
