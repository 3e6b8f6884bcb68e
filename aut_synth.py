"""Seeded synthetic inputs for the AuT audio encoder: configurations, request
lengths, log-mel features and random-init weights.

This module is shared by the CPU oracle's tests and by the GPU path's tests and
benchmark. It holds no arithmetic of the encoder itself (no token counts, no
windows, no convolution): only the workload shapes and the random draws.

Conventions (PyTorch layouts, every parameter bf16-representable):
  conv{1,2,3}_w  [C_out, C_in, 3, 3]      conv{1,2,3}_b [C_out]
  conv_out_w     [d_model, C * f3]          (input index c * f3 + f, f3 = 16 mel rows)
  conv_out_b     [d_model] or None
  per layer: ln1_w, ln1_b [d]; qkv_w [3d, d] (q, k, v stacked on dim 0); qkv_b [3d];
             o_w [d, d]; o_b [d]; ln2_w, ln2_b [d]; fc1_w [F, d]; fc1_b [F];
             fc2_w [d, F]; fc2_b [d]
  ln_post_w, ln_post_b [d]; proj1_w [d, d]; proj1_b [d]; proj2_w [O, d]; proj2_b [O]

Values are drawn in fp32 from numpy's PCG64 and rounded once to bf16
(round-to-nearest-even); both the oracle and the GPU see the same rounded values.
Seeds: lengths 0, features 1, weights 2, waveforms 3.
"""
from __future__ import annotations

import dataclasses
import numpy as np

SEED_LENGTHS = 0
SEED_FEATURES = 1
SEED_WEIGHTS = 2
SEED_WAVES = 3


@dataclasses.dataclass(frozen=True)
class AuTConfig:
    """Encoder hyper-parameters (field names follow AuTEncoderConfig on the
    m-star.org aut_encoder page)."""
    d_model: int
    encoder_layers: int
    encoder_attention_heads: int
    encoder_ffn_dim: int
    downsample_hidden_size: int      # conv channels C
    output_dim: int
    num_mel_bins: int = 128
    n_window: int = 50
    n_window_infer: int = 800
    conv_chunksize: int = 500
    ln_eps: float = 1e-5

    @property
    def head_dim(self) -> int:
        return self.d_model // self.encoder_attention_heads


# The five workloads: tiny, 0.6B-class, Omni-class 16 requests, long-form 20 min,
# throughput batch.  The last three share the Omni-class dimensions.
TINY = AuTConfig(d_model=64, encoder_layers=2, encoder_attention_heads=4,
                 encoder_ffn_dim=256, downsample_hidden_size=16, output_dim=128,
                 n_window_infer=200)
ASR_06B = AuTConfig(d_model=896, encoder_layers=18, encoder_attention_heads=14,
                    encoder_ffn_dim=3584, downsample_hidden_size=480, output_dim=1024)
OMNI = AuTConfig(d_model=1280, encoder_layers=24, encoder_attention_heads=20,
                 encoder_ffn_dim=5120, downsample_hidden_size=480, output_dim=2048)

WORKLOADS = {
    "tiny": TINY,
    "asr06b_30s": ASR_06B,
    "omni_16req": OMNI,
    "omni_20min": OMNI,
    "omni_20min_ragged": OMNI,
    "omni_256req": OMNI,
}


def round_bf16(x: np.ndarray) -> np.ndarray:
    """Round fp32 values to the nearest bf16 (ties to even); returns float32."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return (u.astype(np.uint32) << 16).view(np.float32)


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """bf16 bit patterns (uint16) of already bf16-representable float32 values."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    return (x.view(np.uint32) >> 16).astype(np.uint16)


def request_lengths(workload: str, seed: int = SEED_LENGTHS) -> list[int]:
    """Mel frame counts per request for a named workload.

    tiny: one 2.37 s request; asr06b_30s: one 30 s request; omni_16req: 16
    requests uniform on [100, 3000] frames, redrawn when a multiple of 100;
    omni_20min: 120000 frames; omni_20min_ragged: 119950 frames;
    omni_256req: 256 requests, round(100 * exp(U[ln 0.5, ln 60])) frames.
    """
    rng = np.random.Generator(np.random.PCG64(seed))
    if workload == "tiny":
        return [237]
    if workload == "asr06b_30s":
        return [3000]
    if workload == "omni_16req":
        out = []
        while len(out) < 16:
            n = int(rng.integers(100, 3001))
            if n % 100 != 0:
                out.append(n)
        return out
    if workload == "omni_20min":
        return [120000]
    if workload == "omni_20min_ragged":
        return [119950]
    if workload == "omni_256req":
        u = rng.uniform(np.log(0.5), np.log(60.0), size=256)
        return [max(1, int(round(100.0 * np.exp(v)))) for v in u]
    raise KeyError(workload)


def random_lengths(n: int, lo: int, hi: int, seed: int) -> list[int]:
    """n frame counts uniform on [lo, hi] (inclusive), for planner property tests."""
    rng = np.random.Generator(np.random.PCG64(seed))
    return [int(v) for v in rng.integers(lo, hi + 1, size=n)]


def log_uniform_request(rng: np.random.Generator) -> int:
    """One request length in frames, log-uniform on [0.5, 60] s."""
    return max(1, int(round(100.0 * np.exp(rng.uniform(np.log(0.5), np.log(60.0))))))


def features(lens: list[int], num_mel_bins: int = 128, t_max: int | None = None,
             seed: int = SEED_FEATURES, fill_beyond: float = 0.0) -> np.ndarray:
    """Log-mel stand-in [B, num_mel_bins, T_max] (time fastest): N(0,1) on each
    request's valid frames, `fill_beyond` after them; bf16-rounded float32."""
    if t_max is None:
        t_max = max([1] + list(lens))
    rng = np.random.Generator(np.random.PCG64(seed))
    out = np.full((len(lens), num_mel_bins, t_max), fill_beyond, dtype=np.float32)
    for r, n in enumerate(lens):
        if n > 0:
            out[r, :, :n] = rng.standard_normal((num_mel_bins, n), dtype=np.float32)
    return round_bf16(out)


def weights(cfg: AuTConfig, seed: int = SEED_WEIGHTS, conv_out_bias: bool = False,
            conv_scale: float = 1.0, std: float = 0.02) -> dict:
    """Random-init parameters, N(0, std) for matrices and biases, LayerNorm
    gamma = 1 and beta = 0.  `conv_scale` multiplies the three conv weights
    (a value well above 1 drives the stem's GELUs into their non-linear range)."""
    rng = np.random.Generator(np.random.PCG64(seed))
    d, F, C, O = cfg.d_model, cfg.encoder_ffn_dim, cfg.downsample_hidden_size, cfg.output_dim
    f3 = 16  # mel rows after the stem for 128 bins; a shape, fixed by the workloads

    def n(*shape, scale=1.0):
        return round_bf16(rng.standard_normal(shape, dtype=np.float32) * np.float32(std * scale))

    w = {
        "conv1_w": n(C, 1, 3, 3, scale=conv_scale), "conv1_b": n(C),
        "conv2_w": n(C, C, 3, 3, scale=conv_scale), "conv2_b": n(C),
        "conv3_w": n(C, C, 3, 3, scale=conv_scale), "conv3_b": n(C),
        "conv_out_w": n(d, C * f3),
    }
    w["conv_out_b"] = n(d) if conv_out_bias else None
    layers = []
    for _ in range(cfg.encoder_layers):
        layers.append({
            "ln1_w": np.ones(d, np.float32), "ln1_b": np.zeros(d, np.float32),
            "qkv_w": n(3 * d, d), "qkv_b": n(3 * d),
            "o_w": n(d, d), "o_b": n(d),
            "ln2_w": np.ones(d, np.float32), "ln2_b": np.zeros(d, np.float32),
            "fc1_w": n(F, d), "fc1_b": n(F),
            "fc2_w": n(d, F), "fc2_b": n(d),
        })
    w["layers"] = layers
    w["ln_post_w"] = np.ones(d, np.float32)
    w["ln_post_b"] = np.zeros(d, np.float32)
    w["proj1_w"] = n(d, d)
    w["proj1_b"] = n(d)
    w["proj2_w"] = n(O, d)
    w["proj2_b"] = n(O)
    return w


def randomize_layernorm(w: dict, seed: int = 7) -> dict:
    """Replace every LayerNorm gamma/beta by bf16 values near (1, 0) so that the
    affine part of LayerNorm is exercised (gamma = 1, beta = 0 hides it)."""
    rng = np.random.Generator(np.random.PCG64(seed))
    def g(n):
        return round_bf16(1.0 + 0.1 * rng.standard_normal(n, dtype=np.float32))
    def b(n):
        return round_bf16(0.1 * rng.standard_normal(n, dtype=np.float32))
    for lw in w["layers"]:
        d = lw["ln1_w"].shape[0]
        lw["ln1_w"], lw["ln1_b"] = g(d), b(d)
        lw["ln2_w"], lw["ln2_b"] = g(d), b(d)
    d = w["ln_post_w"].shape[0]
    w["ln_post_w"], w["ln_post_b"] = g(d), b(d)
    return w


def waveforms(n_samples: list[int], seed: int = SEED_WAVES, sample_rate: int = 16000) -> list:
    """Speech-like 16 kHz mono stand-ins, one float64 array per request: a
    voiced source (20 harmonics of a pitch that wanders over 90 - 250 Hz)
    shaped by two random formant bumps that move every 0.25 s, a 3 - 6 Hz
    syllable envelope with occasional pauses, and a little white noise
    (peak amplitude about 0.3).  For front-end workloads only: the encoder's
    own workloads start from features()."""
    rng = np.random.Generator(np.random.PCG64(seed))
    out = []
    for n in n_samples:
        if n <= 0:
            out.append(np.zeros(0))
            continue
        t = np.arange(n) / sample_rate
        seg = max(1, int(0.25 * sample_rate))
        n_seg = -(-n // seg) + 1
        knots = np.arange(n_seg) * seg
        f0 = np.interp(np.arange(n), knots, rng.uniform(90.0, 250.0, n_seg))
        f1 = np.interp(np.arange(n), knots, rng.uniform(300.0, 900.0, n_seg))
        f2 = np.interp(np.arange(n), knots, rng.uniform(900.0, 2500.0, n_seg))
        phase = 2 * np.pi * np.cumsum(f0) / sample_rate
        x = np.zeros(n)
        for h in range(1, 21):
            fh = h * f0
            amp = (np.exp(-((fh - f1) / 150.0) ** 2) + 0.6 * np.exp(-((fh - f2) / 250.0) ** 2)
                   + 0.05) / h
            x += amp * np.sin(h * phase)
        env = 0.5 + 0.5 * np.sin(2 * np.pi * rng.uniform(3.0, 6.0) * t + rng.uniform(0, 2 * np.pi))
        gate = np.interp(np.arange(n), knots, (rng.uniform(size=n_seg) > 0.15).astype(float))
        x = x * env * gate
        x = 0.3 * x / max(1e-9, np.abs(x).max()) + 0.003 * rng.standard_normal(n)
        out.append(x)
    return out
