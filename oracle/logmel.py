"""Plain CPU oracle of the encoder's log-mel front end (waveform -> features).

TEST INFRASTRUCTURE ONLY: imported by the tests and the benchmark's
CPU-baseline leg, never by the product path.

What the pages fix: 16 kHz mono audio in (cubic.dev "Audio Encoder Component",
Feature Extraction Pipeline; soniqo.audio Arabic transcribe guide, pipeline
table), 128 mel bins at 100 frames per second, "Whisper-style" (m-star.org
"mstar.model.components.aut_encoder", module docstring).  What they leave open
is read as Whisper's recipe, each step below:
  - frames every 160 samples (100 frames/s at 16 kHz), 400-sample periodic
    Hann window, the signal reflected by 200 samples at both ends so frame t
    is centred on sample 160 t;
  - power spectrum |X_k|^2 of the 400-point DFT, bins k = 0 .. 200;
  - 128 triangular mel filters on Slaney's mel scale over 0 .. 8000 Hz, each
    scaled to unit area (Slaney normalisation);
  - log10 of max(mel energy, 1e-10); the last frame of the transform dropped,
    so a request of n samples gives n // 160 frames;
  - per request, values below (that request's maximum - 8) raised to it, then
    (x + 4) / 4.
Every step runs in fp64.
"""
from __future__ import annotations

import math

import numpy as np

__all__ = ["SAMPLE_RATE", "N_FFT", "HOP", "N_MELS", "hann_periodic", "frames_for_samples",
           "stft_power", "hz_to_mel_slaney", "mel_to_hz_slaney", "mel_filterbank",
           "log_mel", "log_mel_batch"]

SAMPLE_RATE = 16000
N_FFT = 400
HOP = 160
N_MELS = 128
F_MAX = 8000.0


def hann_periodic(n: int = N_FFT) -> np.ndarray:
    """w[i] = (1 - cos(2 pi i / n)) / 2 for i < n (the periodic Hann window)."""
    i = np.arange(n, dtype=np.float64)
    return 0.5 - 0.5 * np.cos(2.0 * math.pi * i / n)


def frames_for_samples(n: int) -> int:
    """Feature frames of an n-sample request: one per hop, the transform's last
    frame dropped (100 frames per second of 16 kHz audio)."""
    return n // HOP


def stft_power(wave: np.ndarray) -> np.ndarray:
    """|X_t(k)|^2 for t = 0 .. n // 160 (every centred frame, the last one
    included) and k = 0 .. 200: the 400-sample frame centred on sample 160 t of
    the signal reflected by 200 samples at both ends, times the periodic Hann
    window, through a 400-point DFT (numpy's FFT as the library step).
    Returns [n // 160 + 1, 201]."""
    x = np.asarray(wave, dtype=np.float64)
    if x.shape[0] <= N_FFT // 2:
        raise ValueError("reflection needs more than 200 samples")
    xp = np.pad(x, N_FFT // 2, mode="reflect")
    n_frames = 1 + x.shape[0] // HOP
    idx = np.arange(n_frames)[:, None] * HOP + np.arange(N_FFT)[None, :]
    spec = np.fft.rfft(xp[idx] * hann_periodic()[None, :], axis=-1)
    return spec.real ** 2 + spec.imag ** 2


def hz_to_mel_slaney(f):
    """Slaney's mel scale: linear below 1 kHz (3 mels per 200 Hz), logarithmic
    above (27 mels per factor 6.4)."""
    f = np.asarray(f, dtype=np.float64)
    lin = f / (200.0 / 3.0)
    logstep = math.log(6.4) / 27.0
    return np.where(f >= 1000.0, 15.0 + np.log(np.maximum(f, 1e-300) / 1000.0) / logstep, lin)


def mel_to_hz_slaney(m):
    """Inverse of hz_to_mel_slaney."""
    m = np.asarray(m, dtype=np.float64)
    logstep = math.log(6.4) / 27.0
    return np.where(m >= 15.0, 1000.0 * np.exp(logstep * (m - 15.0)), m * (200.0 / 3.0))


def mel_filterbank(n_mels: int = N_MELS, n_fft: int = N_FFT, sr: int = SAMPLE_RATE,
                   f_max: float = F_MAX) -> np.ndarray:
    """[n_mels, n_fft // 2 + 1] triangular filters: n_mels + 2 points equally
    spaced in Slaney mels over [0, f_max]; filter m rises from point m to point
    m + 1 and falls to point m + 2 (linear in Hz, evaluated at the DFT bin
    frequencies k sr / n_fft), scaled by 2 / (f_{m+2} - f_m) so every filter
    has unit area."""
    bins = np.arange(n_fft // 2 + 1, dtype=np.float64) * sr / n_fft
    pts = mel_to_hz_slaney(np.linspace(hz_to_mel_slaney(0.0), hz_to_mel_slaney(f_max), n_mels + 2))
    fb = np.zeros((n_mels, bins.shape[0]))
    for m in range(n_mels):
        lo, ce, hi = pts[m], pts[m + 1], pts[m + 2]
        up = (bins - lo) / (ce - lo)
        down = (hi - bins) / (hi - ce)
        fb[m] = np.maximum(0.0, np.minimum(up, down)) * (2.0 / (hi - lo))
    return fb


def log_mel(wave: np.ndarray) -> np.ndarray:
    """One request's features [128, n // 160] from n samples of 16 kHz audio
    (the recipe in the module docstring)."""
    p = stft_power(wave)[:-1]                    # drop the transform's last frame
    mel = p @ mel_filterbank().T                 # [frames, 128]
    lg = np.log10(np.maximum(mel, 1e-10))
    if lg.size:
        lg = np.maximum(lg, lg.max() - 8.0)
    return ((lg + 4.0) / 4.0).T


def log_mel_batch(waves, t_max: int | None = None):
    """Requests of different lengths -> (features [B, 128, T_max] with zeros past
    each request's frames, feature_lens).  Empty requests give no frames."""
    lens = [frames_for_samples(len(w)) for w in waves]
    t = max(lens + [1]) if t_max is None else t_max
    out = np.zeros((len(waves), N_MELS, t))
    for i, w in enumerate(waves):
        if len(w):
            out[i, :, :lens[i]] = log_mel(w)
    return out, lens
