"""Plain CPU oracle of the AuT (Qwen3-family) audio encoder forward pass.

TEST INFRASTRUCTURE ONLY: imported by the tests, the smoke check and the
benchmark's CPU-baseline leg, never by the product path.

Sources (page title, then section / item):
  [aut_encoder]  m-star.org "mstar.model.components.aut_encoder": module
                 docstring, AuTEncoder.layout / frontend / encode, AuTEncoderConfig
                 (tokens_for_frames, window_lengths), AuTLayout, AuTAttention.
  [AuT 1A]       openarchlab "1A . AuT Audio Encoder (3x Conv2d Stride-2 &
                 Windowed Attention)": section 3 (conv output-size formula,
                 flatten C_conv x 16, non-causal attention within cu_seqlens),
                 section 4 (8x compression, window isolation), section 6 (terms).
  [AuT wiki]     cubic.dev "Audio Encoder Component": LayerNorm with bias,
                 computed sinusoidal positions, weight transposition.

Readings taken where the pages are silent (each also listed in the design
notes): the last chunk is always zero-padded to a full chunk before the stem;
GELU is the exact erf form; LayerNorm eps 1e-5 with biased variance; the
sinusoid table is Whisper's [sin | cos] with timescale 1e4 and increment
ln(1e4) / (d/2 - 1), indexed by the token's position inside its chunk; the
attention scale is 1/sqrt(head_dim); q, k, v are stacked on the output dim of
the fused qkv weight; the layers are pre-LayerNorm.

Every floating-point step runs in the dtype passed in (fp64 by default) on the
bf16-rounded inputs, with no intermediate rounding.
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np
from scipy.special import erf as _erf

__all__ = [
    "conv_out_len", "chunk_frames", "tokens_per_chunk", "tokens_for_frames",
    "window_tokens", "window_lengths", "Chunk", "Layout", "plan",
    "gelu", "sinusoids", "conv2d_k3s2p1", "chunk_mel", "stem", "frontend",
    "layer_norm", "window_attention", "encoder_layer", "projector", "encode",
    "forward",
]


# --------------------------------------------------------------------------
# Host-side layout arithmetic: [aut_encoder] AuTEncoder.layout, AuTEncoderConfig
# --------------------------------------------------------------------------

def conv_out_len(n: int) -> int:
    """Output length of one Conv2d(kernel 3, stride 2, padding 1) along an
    axis of length n: floor((n + 1) / 2) [AuT 1A, section 3, the L_out formula];
    an empty axis stays empty."""
    return (n + 1) // 2 if n > 0 else 0


def chunk_frames(cfg) -> int:
    """Frames per conv chunk: 2 * n_window [aut_encoder, module docstring]."""
    return 2 * cfg.n_window


def tokens_per_chunk(cfg) -> int:
    """Tokens out of one full chunk: three stride-2 convs (100 -> 13)
    [aut_encoder, module docstring]."""
    return conv_out_len(conv_out_len(conv_out_len(chunk_frames(cfg))))


def tokens_for_frames(cfg, num_frames: int) -> int:
    """Tokens for num_frames mel frames: one chunk's worth per full chunk plus
    three stride-2 convolutions' worth of the remainder
    [aut_encoder, AuTEncoderConfig.tokens_for_frames]."""
    cf = chunk_frames(cfg)
    full, rem = divmod(num_frames, cf)
    return full * tokens_per_chunk(cfg) + conv_out_len(conv_out_len(conv_out_len(rem)))


def window_tokens(cfg) -> int:
    """Tokens per attention window: n_window_infer frames cover
    n_window_infer / chunk_frames whole chunks (800 frames -> 104 tokens)
    [aut_encoder, module docstring]."""
    cf = chunk_frames(cfg)
    if cfg.n_window_infer % cf != 0:
        raise ValueError("n_window_infer must be a multiple of 2 * n_window")
    return tokens_per_chunk(cfg) * (cfg.n_window_infer // cf)


def window_lengths(num_tokens: int, w: int) -> list[int]:
    """Attention segments of one request: full windows, then the remainder
    [aut_encoder, AuTEncoderConfig.window_lengths]."""
    out = [w] * (num_tokens // w)
    if num_tokens % w:
        out.append(num_tokens % w)
    return out


@dataclasses.dataclass(frozen=True)
class Chunk:
    request: int          # index of the request the chunk belongs to
    frame0: int           # first frame of the chunk inside its request
    valid_frames: int     # frames of the chunk that lie before the request's end
    token0: int           # packed row of the chunk's first kept token
    valid_tokens: int     # tokens the chunk keeps after trimming


@dataclasses.dataclass(frozen=True)
class Layout:
    """[aut_encoder, AuTLayout]: where the packed tokens come from and how they
    attend, plus the chunk list the front end walks."""
    tokens_per_request: list
    cu_seqlens: list
    chunks: list

    @property
    def total_tokens(self) -> int:
        return self.cu_seqlens[-1]

    @property
    def window_lengths(self) -> list:
        return [b - a for a, b in zip(self.cu_seqlens[:-1], self.cu_seqlens[1:])]


def plan(cfg, feature_lens) -> Layout:
    """Token counts, cu_seqlens and the chunk list for a batch of mel lengths,
    host arithmetic only [aut_encoder, AuTEncoder.layout].  Requests are packed
    in input order; a request's windows never span into the next request."""
    cf = chunk_frames(cfg)
    w = window_tokens(cfg)
    tokens, cu, chunks = [], [0], []
    row = 0
    for r, n in enumerate(feature_lens):
        if n < 0:
            raise ValueError("negative feature length")
        t = tokens_for_frames(cfg, n)
        tokens.append(t)
        for seg in window_lengths(t, w):
            cu.append(cu[-1] + seg)
        for k in range((n + cf - 1) // cf):
            vf = min(cf, n - k * cf)
            vt = conv_out_len(conv_out_len(conv_out_len(vf)))
            chunks.append(Chunk(r, k * cf, vf, row, vt))
            row += vt
    assert row == cu[-1]
    return Layout(tokens, cu, chunks)


# --------------------------------------------------------------------------
# Elementwise pieces
# --------------------------------------------------------------------------

def gelu(x: np.ndarray) -> np.ndarray:
    """activation_function 'gelu' [aut_encoder, AuTEncoderConfig], exact form:
    x * (1 + erf(x / sqrt 2)) / 2."""
    return x * 0.5 * (1.0 + _erf(x / math.sqrt(2.0)))


def sinusoids(length: int, channels: int, dtype=np.float64) -> np.ndarray:
    """Computed (never loaded) sinusoidal position table [AuT wiki, Positional
    Embeddings; AuT 1A, section 6 SinusoidsPositionEmbedding], Whisper form:
    row t = [sin(t * g_k) for k < d/2] + [cos(t * g_k) for k < d/2],
    g_k = exp(-k * ln(10000) / (d/2 - 1)).  Built in fp64."""
    half = channels // 2
    inc = math.log(10000.0) / (half - 1)
    g = np.exp(-inc * np.arange(half, dtype=np.float64))
    ang = np.arange(length, dtype=np.float64)[:, None] * g[None, :]
    return np.concatenate([np.sin(ang), np.cos(ang)], axis=1).astype(dtype)


def layer_norm(x: np.ndarray, gamma, beta, eps: float) -> np.ndarray:
    """LayerNorm with bias over the last axis, biased variance
    [AuT wiki, Transformer Encoder Layers]."""
    mu = x.mean(axis=-1, keepdims=True)
    var = ((x - mu) ** 2).mean(axis=-1, keepdims=True)
    return (x - mu) / np.sqrt(var + eps) * gamma + beta


# --------------------------------------------------------------------------
# Front end: [aut_encoder, AuTEncoder.frontend]; [AuT 1A, sections 3 and 6]
# --------------------------------------------------------------------------

def conv2d_k3s2p1(x: np.ndarray, w: np.ndarray, b: np.ndarray) -> np.ndarray:
    """Conv2d(kernel 3, stride 2, padding 1) + bias on channel-last input.

    x: [N, H, W, C_in]; w: [C_out, C_in, 3, 3] (PyTorch layout); b: [C_out].
    y[n, i, j, o] = b[o] + sum_{c, kh, kw} w[o, c, kh, kw] * x[n, 2i+kh-1, 2j+kw-1, c],
    with x = 0 outside the input.  One matmul per filter tap."""
    n, h, wd, cin = x.shape
    ho, wo = conv_out_len(h), conv_out_len(wd)
    xp = np.zeros((n, h + 2, wd + 2, cin), dtype=x.dtype)
    xp[:, 1:h + 1, 1:wd + 1, :] = x
    y = np.zeros((n * ho * wo, w.shape[0]), dtype=x.dtype)
    for kh in range(3):
        for kw in range(3):
            xs = np.ascontiguousarray(xp[:, kh:kh + 2 * ho:2, kw:kw + 2 * wo:2, :])
            y += xs.reshape(-1, cin) @ w[:, :, kh, kw].T.astype(x.dtype)
    y += b.astype(x.dtype)[None, :]
    return y.reshape(n, ho, wo, w.shape[0])


def chunk_mel(cfg, feats: np.ndarray, layout: Layout, chunks=None, dtype=np.float64) -> np.ndarray:
    """Cut every request into chunk_frames pieces; frames at or after the
    request's length are zero, so the last piece is zero-padded to a full chunk
    [aut_encoder, AuTEncoder.frontend].  Returns [n_chunks, mel, chunk_frames]."""
    cf = chunk_frames(cfg)
    chunks = layout.chunks if chunks is None else chunks
    out = np.zeros((len(chunks), feats.shape[1], cf), dtype=dtype)
    for i, c in enumerate(chunks):
        out[i, :, :c.valid_frames] = feats[c.request, :, c.frame0:c.frame0 + c.valid_frames]
    return out


def stem(cfg, w: dict, mel: np.ndarray, dtype=np.float64) -> np.ndarray:
    """Three Conv2d(3, s2, p1) + GELU, flatten C x 16 in C-major order, then the
    conv_out linear [aut_encoder, module docstring; AuT 1A, section 3].
    mel: [n_chunks, mel_bins, chunk_frames] (H = mel bin, W = frame).
    Returns [n_chunks, tokens_per_chunk, d_model] (no positions yet)."""
    x = mel.astype(dtype)[..., None]                     # [N, H, W, 1]
    for i in (1, 2, 3):
        x = gelu(conv2d_k3s2p1(x, w[f"conv{i}_w"].astype(dtype), w[f"conv{i}_b"].astype(dtype)))
    n, f3, t3, c = x.shape                               # [N, 16, 13, C]
    v = x.transpose(0, 2, 3, 1).reshape(n, t3, c * f3)  # v_j[c * 16 + f] = y3[c, f, j]
    h = v @ w["conv_out_w"].astype(dtype).T
    if w.get("conv_out_b") is not None:
        h = h + w["conv_out_b"].astype(dtype)
    return h


def frontend(cfg, w: dict, feats: np.ndarray, feature_lens, dtype=np.float64,
             with_positions: bool = True, chunk_batch: int = 16,
             stem_rows: dict | None = None) -> np.ndarray:
    """(B, mel, T_max) zero-padded mel + valid lengths -> packed
    [total_tokens, d_model] [aut_encoder, AuTEncoder.frontend]: every chunk gets
    the same tokens_per_chunk positions, then is trimmed to its valid tokens and
    packed chunk by chunk, request by request.  If `stem_rows` is a dict, the
    packed rows before the positions are added are also stored under "stem"."""
    layout = plan(cfg, feature_lens)
    tpc = tokens_per_chunk(cfg)
    pe = sinusoids(tpc, cfg.d_model, dtype)
    x0 = np.zeros((layout.total_tokens, cfg.d_model), dtype=dtype)
    raw = np.zeros_like(x0) if stem_rows is not None else None
    for s in range(0, len(layout.chunks), chunk_batch):
        part = layout.chunks[s:s + chunk_batch]
        h = stem(cfg, w, chunk_mel(cfg, feats, layout, part, dtype), dtype)
        if raw is not None:
            for c, hc in zip(part, h):
                raw[c.token0:c.token0 + c.valid_tokens] = hc[:c.valid_tokens]
        if with_positions:
            h = h + pe[None]
        for c, hc in zip(part, h):
            x0[c.token0:c.token0 + c.valid_tokens] = hc[:c.valid_tokens]
    if stem_rows is not None:
        stem_rows["stem"] = raw
    return x0


# --------------------------------------------------------------------------
# Transformer stack: [aut_encoder, AuTEncoderLayer / AuTAttention / encode]
# --------------------------------------------------------------------------

def window_attention(qkv: np.ndarray, cu_seqlens, heads: int) -> np.ndarray:
    """Bidirectional attention inside each cu_seqlens segment, none across
    segments, no cache: per segment and head, softmax(Q K^T / sqrt(hd)) V
    [aut_encoder, AuTAttention ('SDPA per window from cu_seqlens');
     AuT 1A, section 3 (is_causal = False within cu_seqlens segments)]."""
    t, three_d = qkv.shape
    d = three_d // 3
    hd = d // heads
    out = np.zeros((t, d), dtype=qkv.dtype)
    scale = 1.0 / math.sqrt(hd)
    for a, b in zip(cu_seqlens[:-1], cu_seqlens[1:]):
        if b == a:
            continue
        q = qkv[a:b, :d].reshape(b - a, heads, hd).transpose(1, 0, 2)
        k = qkv[a:b, d:2 * d].reshape(b - a, heads, hd).transpose(1, 0, 2)
        v = qkv[a:b, 2 * d:].reshape(b - a, heads, hd).transpose(1, 0, 2)
        s = (q @ k.transpose(0, 2, 1)) * scale
        s = s - s.max(axis=-1, keepdims=True)
        p = np.exp(s)
        p = p / p.sum(axis=-1, keepdims=True)
        out[a:b] = (p @ v).transpose(1, 0, 2).reshape(b - a, d)
    return out


def encoder_layer(cfg, lw: dict, x: np.ndarray, cu_seqlens) -> np.ndarray:
    """One pre-LayerNorm layer [aut_encoder, AuTEncoderLayer; AuT wiki,
    Transformer Encoder Layers]:
      x += o_proj(attn(qkv_proj(LN1(x)))),  x += fc2(gelu(fc1(LN2(x))))."""
    dt = x.dtype
    g = lambda k: lw[k].astype(dt)
    hn = layer_norm(x, g("ln1_w"), g("ln1_b"), cfg.ln_eps)
    qkv = hn @ g("qkv_w").T + g("qkv_b")
    a = window_attention(qkv, cu_seqlens, cfg.encoder_attention_heads)
    x = x + (a @ g("o_w").T + g("o_b"))
    hn = layer_norm(x, g("ln2_w"), g("ln2_b"), cfg.ln_eps)
    f = gelu(hn @ g("fc1_w").T + g("fc1_b"))
    return x + (f @ g("fc2_w").T + g("fc2_b"))


def projector(cfg, w: dict, x: np.ndarray) -> np.ndarray:
    """Final LayerNorm and the two-layer GELU projector to the LLM width
    [aut_encoder, module docstring; AuT 1A, section 1 (1280 -> 1280 -> 2048)]."""
    dt = x.dtype
    g = lambda k: w[k].astype(dt)
    hn = layer_norm(x, g("ln_post_w"), g("ln_post_b"), cfg.ln_eps)
    return gelu(hn @ g("proj1_w").T + g("proj1_b")) @ g("proj2_w").T + g("proj2_b")


def encode(cfg, w: dict, x0: np.ndarray, cu_seqlens, hidden: dict | None = None) -> np.ndarray:
    """The transformer stack and projector over a packed sequence:
    (total_tokens, d_model) -> (total_tokens, output_dim) [aut_encoder,
    AuTEncoder.encode].  If `hidden` is a dict, the residual stream after each
    layer is stored in it under the layer index."""
    x = x0
    for i, lw in enumerate(w["layers"]):
        x = encoder_layer(cfg, lw, x, cu_seqlens)
        if hidden is not None:
            hidden[i] = x
    return projector(cfg, w, x)


def forward(cfg, w: dict, feats: np.ndarray, feature_lens, dtype=np.float64,
            hidden: dict | None = None):
    """features, feature_lens -> (out [total_tokens, output_dim], layout)
    [aut_encoder, AuTEncoder.forward].  If `hidden` is a dict it receives the
    stem rows before positions ("stem"), x0 ("x0") and the residual stream
    after every layer (layer index)."""
    layout = plan(cfg, feature_lens)
    x0 = frontend(cfg, w, feats, feature_lens, dtype, stem_rows=hidden)
    if hidden is not None:
        hidden["x0"] = x0
    return encode(cfg, w, x0, layout.cu_seqlens, hidden), layout
