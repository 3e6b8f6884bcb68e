"""Pins of the CPU oracle against things other than itself: values the pages
print, closed forms, brute force on tiny inputs, and library routines (torch
fp64 conv2d, LayerNorm, SDPA and TransformerEncoderLayer) that compute the same
textbook operations.  CPU only."""
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import aut_synth as S
import oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "worked_sizes.txt")


def _golden():
    rows = {}
    with open(GOLDEN) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            name, a, b, _src = line.rstrip("\n").split("\t")
            rows[name] = (int(a), int(b))
    return rows


# ----------------------------------------------------------------- sizes ----

def test_worked_sizes_from_pages():
    g = _golden()
    a, b = g["mel_bins_after_three_convs"]
    assert O.conv_out_len(O.conv_out_len(O.conv_out_len(a))) == b
    a, b = g["frames_to_tokens_full_chunk"]
    assert O.tokens_for_frames(S.OMNI, a) == b
    a, b = g["window_frames_to_tokens"]
    assert O.window_tokens(S.OMNI) == b and S.OMNI.n_window_infer == a
    a, b = g["chunk_frames_from_n_window"]
    assert S.OMNI.n_window == a and O.chunk_frames(S.OMNI) == b


@pytest.mark.parametrize("n", [1, 2, 3, 5, 37, 99, 100, 101, 128, 237, 800, 3000])
def test_conv_out_len_matches_torch_conv_shape(n):
    # Library routine: PyTorch's Conv2d(k=3, s=2, p=1) output shape.
    x = torch.zeros(1, 1, 4, n, dtype=torch.float64)
    y = F.conv2d(x, torch.zeros(1, 1, 3, 3, dtype=torch.float64), stride=2, padding=1)
    assert y.shape[-1] == O.conv_out_len(n)


def test_tokens_closed_form_and_not_ceil_div_8():
    # 13 per full chunk plus ceil(rem / 8) for the remainder (the three
    # halvings with rounding up compose to a ceiling division by 8).
    for n in range(0, 5001):
        full, rem = divmod(n, 100)
        assert O.tokens_for_frames(S.OMNI, n) == 13 * full + (rem + 7) // 8
    assert O.tokens_for_frames(S.OMNI, 200) == 26 != math.ceil(200 / 8)


def test_tokens_by_torch_conv_chain_on_partial_chunks():
    # Brute force: run three real stride-2 convolutions on each chunk's frames.
    def chain(n):
        x = torch.zeros(1, 1, 8, n, dtype=torch.float64)
        k = torch.zeros(1, 1, 3, 3, dtype=torch.float64)
        for _ in range(3):
            x = F.conv2d(x, k, stride=2, padding=1)
        return x.shape[-1]
    for n in [1, 37, 99, 100, 137, 250, 1234]:
        chunks = [min(100, n - s) for s in range(0, n, 100)]
        assert O.tokens_for_frames(S.OMNI, n) == sum(chain(c) for c in chunks)


def test_compression_about_eight():
    # openarchlab 1A, section 4: T_aud ~ T_mel / 8 (13 tokens per 100 frames).
    for n in [1000, 3000, 120000]:
        t = O.tokens_for_frames(S.OMNI, n)
        assert 7.0 < n / t < 8.0


def test_window_lengths_invariants():
    for n in range(0, 700):
        wl = O.window_lengths(n, 104)
        assert sum(wl) == n
        assert all(v == 104 for v in wl[:-1])
        assert all(0 < v <= 104 for v in wl)


def test_plan_worked_configs():
    lay = O.plan(S.TINY, [237])           # 2*13 + ceil(37/8)=5 -> 31; window 26
    assert lay.tokens_per_request == [31] and lay.cu_seqlens == [0, 26, 31]
    lay = O.plan(S.ASR_06B, [3000])       # 30 chunks * 13 = 390 = 3*104 + 78
    assert lay.total_tokens == 390 and lay.cu_seqlens == [0, 104, 208, 312, 390]
    lay = O.plan(S.OMNI, [120000])        # 1200 chunks * 13 = 15600 = 150 * 104
    assert lay.total_tokens == 15600 and lay.cu_seqlens == list(range(0, 15601, 104))
    lay = O.plan(S.OMNI, [119950])        # 1199*13 + ceil(50/8)=7 = 15594 = 149*104 + 98
    assert lay.total_tokens == 15594 and lay.window_lengths[-1] == 98
    assert len(lay.cu_seqlens) == 151


def test_plan_chunks_and_windows_tile_requests():
    lens = [0, 1, 99, 100, 101, 800, 801, 1999, 0, 5]
    lay = O.plan(S.OMNI, lens)
    # chunk rows are contiguous and cover every token exactly once
    row = 0
    for c in lay.chunks:
        assert c.token0 == row and 0 < c.valid_frames <= 100
        row += c.valid_tokens
    assert row == lay.total_tokens == sum(lay.tokens_per_request)
    # no window straddles two requests
    starts = np.cumsum([0] + lay.tokens_per_request)
    bounds = set(lay.cu_seqlens)
    assert set(int(s) for s in starts) <= bounds


# --------------------------------------------------------------- sinusoid ----

def test_sinusoid_closed_form():
    d = 1280
    pe = O.sinusoids(13, d)
    assert np.all(pe[0, :d // 2] == 0.0) and np.all(pe[0, d // 2:] == 1.0)
    np.testing.assert_allclose(pe[:, :d // 2] ** 2 + pe[:, d // 2:] ** 2, 1.0, atol=1e-15)
    for t in range(13):
        assert pe[t, 0] == pytest.approx(math.sin(t), abs=1e-15)                 # g_0 = 1
        assert pe[t, d // 2 - 1] == pytest.approx(math.sin(t * 1e-4), abs=1e-15)  # g_last = 1e-4
        assert pe[t, d - 1] == pytest.approx(math.cos(t * 1e-4), abs=1e-15)
        k = 7
        g = math.exp(-k * math.log(10000.0) / (d // 2 - 1))
        assert pe[t, k] == pytest.approx(math.sin(t * g), abs=1e-14)


# ------------------------------------------------------------------- gelu ----

def test_gelu_against_math_erf_and_torch():
    x = np.linspace(-6, 6, 1001)
    ref = np.array([v * 0.5 * (1 + math.erf(v / math.sqrt(2))) for v in x])
    np.testing.assert_allclose(O.gelu(x), ref, rtol=0, atol=1e-15)
    t = F.gelu(torch.from_numpy(x)).numpy()
    np.testing.assert_allclose(O.gelu(x), t, rtol=0, atol=1e-14)


# ------------------------------------------------------------------- conv ----

def _brute_conv(x, w, b):
    n, h, wd, cin = x.shape
    cout = w.shape[0]
    ho, wo = (h + 1) // 2, (wd + 1) // 2
    y = np.zeros((n, ho, wo, cout))
    for a in range(n):
        for i in range(ho):
            for j in range(wo):
                for o in range(cout):
                    s = b[o]
                    for c in range(cin):
                        for kh in range(3):
                            for kw in range(3):
                                hi, wj = 2 * i + kh - 1, 2 * j + kw - 1
                                if 0 <= hi < h and 0 <= wj < wd:
                                    s += w[o, c, kh, kw] * x[a, hi, wj, c]
                    y[a, i, j, o] = s
    return y


@pytest.mark.parametrize("shape", [(1, 7, 5, 1, 3), (2, 16, 12, 3, 4), (1, 4, 9, 2, 2)])
def test_conv_brute_force_and_torch(shape):
    n, h, wd, cin, cout = shape
    rng = np.random.default_rng(5)
    x = rng.standard_normal((n, h, wd, cin))
    w = rng.standard_normal((cout, cin, 3, 3))
    b = rng.standard_normal(cout)
    y = O.conv2d_k3s2p1(x, w, b)
    np.testing.assert_allclose(y, _brute_conv(x, w, b), rtol=0, atol=1e-12)
    yt = F.conv2d(torch.from_numpy(x).permute(0, 3, 1, 2), torch.from_numpy(w),
                  torch.from_numpy(b), stride=2, padding=1).permute(0, 2, 3, 1).numpy()
    np.testing.assert_allclose(y, yt, rtol=0, atol=1e-12)


def test_conv_impulse_returns_kernel_tap():
    # An impulse at input (2i0 + kh - 1, 2j0 + kw - 1) lands on output (i0, j0)
    # weighted by tap (kh, kw).
    rng = np.random.default_rng(1)
    w = rng.standard_normal((3, 1, 3, 3))
    for kh in range(3):
        for kw in range(3):
            x = np.zeros((1, 10, 10, 1))
            x[0, 2 * 2 + kh - 1, 2 * 3 + kw - 1, 0] = 1.0
            y = O.conv2d_k3s2p1(x, w, np.zeros(3))
            np.testing.assert_allclose(y[0, 2, 3], w[:, 0, kh, kw], atol=1e-15)


def test_partial_chunk_padding_reading():
    """The last chunk is padded to a full chunk before the stem.  With zero
    biases the padded region stays zero through the GELUs and the kept tokens
    equal those of convolving the short chunk alone; with non-zero biases the
    padded positions carry GELU(bias) into the last kept tokens, so the two
    differ (the reading this oracle takes, with the aut_encoder frontend page)."""
    cfg = S.TINY
    w = S.weights(cfg, conv_scale=20.0)
    rng = np.random.default_rng(3)
    short = rng.standard_normal((1, 128, 37))
    padded = np.zeros((1, 128, 100)); padded[..., :37] = short
    keep = O.tokens_for_frames(cfg, 37)

    def stem_short(wts):
        x = short[..., None]
        for i in (1, 2, 3):
            x = O.gelu(O.conv2d_k3s2p1(x, wts[f"conv{i}_w"], wts[f"conv{i}_b"]))
        n, f3, t3, c = x.shape
        return (x.transpose(0, 2, 3, 1).reshape(n, t3, c * f3) @ wts["conv_out_w"].T)[0]

    w0 = dict(w)
    for i in (1, 2, 3):
        w0[f"conv{i}_b"] = np.zeros_like(w[f"conv{i}_b"])
    a = O.stem(cfg, w0, padded)[0, :keep]
    np.testing.assert_allclose(a, stem_short(w0)[:keep], atol=1e-12)
    a = O.stem(cfg, w, padded)[0, :keep]
    assert np.abs(a - stem_short(w)[:keep]).max() > 1e-6


# ------------------------------------------------------------- layernorm ----

def test_layernorm_unit_and_torch():
    rng = np.random.default_rng(2)
    x = rng.standard_normal((17, 96)) * 3 + 1
    y = O.layer_norm(x, np.ones(96), np.zeros(96), 1e-5)
    np.testing.assert_allclose(y.mean(-1), 0, atol=1e-12)
    np.testing.assert_allclose(y.var(-1), 1, atol=1e-5)
    g, b = rng.standard_normal(96), rng.standard_normal(96)
    yt = F.layer_norm(torch.from_numpy(x), (96,), torch.from_numpy(g), torch.from_numpy(b), 1e-5)
    np.testing.assert_allclose(O.layer_norm(x, g, b, 1e-5), yt.numpy(), atol=1e-12)


# ------------------------------------------------------------- attention ----

def _sdpa(q, k, v, mask=None):
    return F.scaled_dot_product_attention(q, k, v, attn_mask=mask).numpy()


def test_attention_per_window_equals_block_diagonal_and_dense():
    rng = np.random.default_rng(4)
    heads, hd, t = 3, 8, 23
    d = heads * hd
    qkv = rng.standard_normal((t, 3 * d))
    cu = [0, 10, 20, 23]
    out = O.window_attention(qkv, cu, heads)

    def split(x):
        return torch.from_numpy(x.reshape(t, heads, hd).transpose(1, 0, 2).copy())
    q, k, v = split(qkv[:, :d]), split(qkv[:, d:2 * d]), split(qkv[:, 2 * d:])
    # (1) one T x T block-diagonal mask through the library's SDPA
    mask = torch.full((t, t), float("-inf"), dtype=torch.float64)
    for a, b in zip(cu[:-1], cu[1:]):
        mask[a:b, a:b] = 0.0
    ref = _sdpa(q, k, v, mask).transpose(1, 0, 2).reshape(t, d)
    np.testing.assert_allclose(out, ref, atol=1e-12)
    # (2) a single window covering the whole sequence is dense attention
    dense = _sdpa(q, k, v).transpose(1, 0, 2).reshape(t, d)
    np.testing.assert_allclose(O.window_attention(qkv, [0, t], heads), dense, atol=1e-12)
    # (3) a constant-V check: softmax rows sum to one, so O = V's constant row
    qkv2 = qkv.copy(); qkv2[:, 2 * d:] = 0.75
    np.testing.assert_allclose(O.window_attention(qkv2, cu, heads), 0.75, atol=1e-14)


# ----------------------------------------------------- layer / encoder ----

def _torch_layer(cfg, lw):
    d, H, F_ = cfg.d_model, cfg.encoder_attention_heads, cfg.encoder_ffn_dim
    m = torch.nn.TransformerEncoderLayer(d, H, F_, dropout=0.0, activation="gelu",
                                         layer_norm_eps=cfg.ln_eps, batch_first=True,
                                         norm_first=True).double().eval()
    t = lambda a: torch.from_numpy(np.asarray(a, dtype=np.float64))
    with torch.no_grad():
        m.self_attn.in_proj_weight.copy_(t(lw["qkv_w"]))
        m.self_attn.in_proj_bias.copy_(t(lw["qkv_b"]))
        m.self_attn.out_proj.weight.copy_(t(lw["o_w"]))
        m.self_attn.out_proj.bias.copy_(t(lw["o_b"]))
        m.linear1.weight.copy_(t(lw["fc1_w"])); m.linear1.bias.copy_(t(lw["fc1_b"]))
        m.linear2.weight.copy_(t(lw["fc2_w"])); m.linear2.bias.copy_(t(lw["fc2_b"]))
        m.norm1.weight.copy_(t(lw["ln1_w"])); m.norm1.bias.copy_(t(lw["ln1_b"]))
        m.norm2.weight.copy_(t(lw["ln2_w"])); m.norm2.bias.copy_(t(lw["ln2_b"]))
    return m


def test_encoder_layer_equals_torch_transformer_layer():
    cfg = S.TINY
    w = S.randomize_layernorm(S.weights(cfg, std=0.1))
    lw = w["layers"][0]
    rng = np.random.default_rng(6)
    x = rng.standard_normal((31, cfg.d_model))
    cu = [0, 26, 31]
    mask = torch.full((31, 31), float("-inf"), dtype=torch.float64)
    for a, b in zip(cu[:-1], cu[1:]):
        mask[a:b, a:b] = 0.0
    with torch.no_grad():
        ref = _torch_layer(cfg, lw)(torch.from_numpy(x)[None], src_mask=mask)[0].numpy()
    np.testing.assert_allclose(O.encoder_layer(cfg, lw, x, cu), ref, atol=1e-11)


def test_full_forward_equals_torch_composition():
    """The whole tiny encoder rebuilt from torch fp64 library modules (conv2d on
    NCHW with H = mel, W = frame; the HF-style permute/flatten; TransformerEncoderLayer
    with a block-diagonal mask; LayerNorm; Linear) matches the oracle."""
    cfg = S.TINY
    lens = [237, 40, 0, 100]
    w = S.randomize_layernorm(S.weights(cfg, conv_out_bias=True, conv_scale=10.0, std=0.05))
    feats = S.features(lens)
    out, lay = O.forward(cfg, w, feats, lens)
    t = lambda a: torch.from_numpy(np.asarray(a, dtype=np.float64))
    rows = []
    pe = t(O.sinusoids(13, cfg.d_model))
    for r, n in enumerate(lens):
        for s in range(0, n, 100):
            x = torch.zeros(1, 1, 128, 100, dtype=torch.float64)
            v = min(100, n - s)
            x[0, 0, :, :v] = t(feats[r, :, s:s + v])
            for i in (1, 2, 3):
                x = F.gelu(F.conv2d(x, t(w[f"conv{i}_w"]), t(w[f"conv{i}_b"]), stride=2, padding=1))
            n_, c, f, tt = x.shape
            v_ = x.permute(0, 3, 1, 2).reshape(tt, c * f)
            h = F.linear(v_, t(w["conv_out_w"]), t(w["conv_out_b"])) + pe
            k = (v + 7) // 8 if v < 100 else 13
            rows.append(h[:k])
    x = torch.cat(rows)
    T = x.shape[0]
    assert T == lay.total_tokens
    mask = torch.full((T, T), float("-inf"), dtype=torch.float64)
    for a, b in zip(lay.cu_seqlens[:-1], lay.cu_seqlens[1:]):
        mask[a:b, a:b] = 0.0
    with torch.no_grad():
        for lw in w["layers"]:
            x = _torch_layer(cfg, lw)(x[None], src_mask=mask)[0]
        x = F.layer_norm(x, (cfg.d_model,), t(w["ln_post_w"]), t(w["ln_post_b"]), cfg.ln_eps)
        x = F.linear(F.gelu(F.linear(x, t(w["proj1_w"]), t(w["proj1_b"]))),
                     t(w["proj2_w"]), t(w["proj2_b"]))
    np.testing.assert_allclose(out, x.numpy(), atol=1e-10)


def test_window_isolation_exact():
    """openarchlab 1A, section 4: perturbing the second window's spectrogram
    leaves the first window's output unchanged (difference exactly 0)."""
    cfg = S.TINY                     # window = 200 frames = 26 tokens
    lens = [237]
    w = S.weights(cfg)
    feats = S.features(lens)
    a, lay = O.forward(cfg, w, feats, lens)
    f2 = feats.copy()
    f2[0, :, 200:237] += 1.0         # frames of window 2 only
    b, _ = O.forward(cfg, w, f2, lens)
    w1 = lay.cu_seqlens[1]
    assert np.array_equal(a[:w1], b[:w1])
    assert np.abs(a[w1:] - b[w1:]).max() > 0


def test_packing_order_invariance_exact():
    cfg = S.TINY
    lens = [137, 250, 60]
    w = S.weights(cfg)
    feats = S.features(lens)
    a, la = O.forward(cfg, w, feats, lens)
    perm = [2, 0, 1]
    b, lb = O.forward(cfg, w, feats[perm], [lens[i] for i in perm])
    sa = np.cumsum([0] + la.tokens_per_request)
    sb = np.cumsum([0] + lb.tokens_per_request)
    for j, i in enumerate(perm):
        assert np.array_equal(a[sa[i]:sa[i + 1]], b[sb[j]:sb[j + 1]])


def test_window_subrequest_equals_full_rows():
    """A window is whole chunks of one request, so the oracle can compute any
    window of a long request from that window's frames alone; this is how the
    full-size parity tests sample rows.  BLAS blocks a shorter matrix
    differently, so rows agree to fp64 rounding rather than bit for bit."""
    cfg = S.TINY
    lens = [530]
    w = S.weights(cfg)
    feats = S.features(lens)
    full, lay = O.forward(cfg, w, feats, lens)
    for k, (a, b) in enumerate(zip(lay.cu_seqlens[:-1], lay.cu_seqlens[1:])):
        f0 = k * cfg.n_window_infer
        sub_len = min(cfg.n_window_infer, lens[0] - f0)
        sub, _ = O.forward(cfg, w, feats[:, :, f0:f0 + sub_len], [sub_len])
        np.testing.assert_allclose(sub, full[a:b], rtol=0, atol=1e-12)


def test_bf16_rounding_of_inputs():
    x = np.array([1.0, 1.00390625, 1.005859375, -3.14159, 1e-3], dtype=np.float32)
    r = S.round_bf16(x)
    t = torch.from_numpy(x).to(torch.bfloat16).to(torch.float32).numpy()
    assert np.array_equal(r, t)
