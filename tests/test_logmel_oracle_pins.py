"""Pins of the log-mel oracle (oracle/logmel.py) against things other than
itself: a brute-force DFT with the reflection written out, torch.stft and
torch's Hann window, the Slaney filterbank and the Whisper feature extractor
of the transformers library, and closed-form invariants (Parseval, silence,
gain, a pure tone)."""
import math

import numpy as np
import pytest

import aut_synth as S
from oracle import logmel as LM

torch = pytest.importorskip("torch")


def _wave(n, seed=0):
    return np.random.default_rng(seed).standard_normal(n)


def test_hann_is_torch_periodic_window():
    np.testing.assert_allclose(LM.hann_periodic(), torch.hann_window(400, periodic=True,
                                                                      dtype=torch.float64).numpy(),
                               rtol=0, atol=1e-15)


def test_stft_power_matches_brute_force_dft_with_explicit_reflection():
    x = _wave(1003, 1)
    n = x.shape[0]
    w = [(1 - math.cos(2 * math.pi * i / 400)) / 2 for i in range(400)]
    got = LM.stft_power(x)
    assert got.shape == (1 + n // 160, 201)
    for t in (0, 1, 3, n // 160):
        for k in (0, 1, 7, 100, 199, 200):
            re = im = 0.0
            for i in range(400):
                j = 160 * t - 200 + i
                if j < 0:
                    j = -j
                elif j >= n:
                    j = 2 * (n - 1) - j
                a = -2 * math.pi * k * i / 400
                re += x[j] * w[i] * math.cos(a)
                im += x[j] * w[i] * math.sin(a)
            assert got[t, k] == pytest.approx(re * re + im * im, rel=1e-9, abs=1e-9)


def test_stft_power_matches_torch_stft():
    x = _wave(16000 * 2 + 77, 2)
    ref = torch.stft(torch.from_numpy(x), 400, 160, window=torch.hann_window(400, dtype=torch.float64),
                     center=True, pad_mode="reflect", return_complex=True).abs() ** 2
    np.testing.assert_allclose(LM.stft_power(x), ref.numpy().T, rtol=1e-9, atol=1e-9)


def test_parseval_per_frame():
    """One-sided power, doubled for k = 1 .. 199, sums to 400 * sum((x w)^2)."""
    x = _wave(4000, 3)
    p = LM.stft_power(x)
    xp = np.pad(x, 200, mode="reflect")
    for t in (0, 5, 25):
        seg = xp[160 * t:160 * t + 400] * LM.hann_periodic()
        one_sided = p[t, 0] + 2 * p[t, 1:200].sum() + p[t, 200]
        assert one_sided == pytest.approx(400 * (seg ** 2).sum(), rel=1e-12)


def test_slaney_mel_scale_closed_forms():
    assert LM.hz_to_mel_slaney(0.0) == 0.0
    assert LM.hz_to_mel_slaney(1000.0) == pytest.approx(15.0, abs=1e-12)
    assert LM.hz_to_mel_slaney(6400.0) == pytest.approx(15.0 + 27.0, abs=1e-12)
    assert LM.hz_to_mel_slaney(200.0) == pytest.approx(3.0, abs=1e-12)
    f = np.array([0.0, 50.0, 999.0, 1000.0, 1234.5, 8000.0])
    np.testing.assert_allclose(LM.mel_to_hz_slaney(LM.hz_to_mel_slaney(f)), f, rtol=1e-12, atol=1e-9)


def test_filterbank_matches_transformers_slaney_bank():
    from transformers.audio_utils import mel_filter_bank
    ref = mel_filter_bank(num_frequency_bins=201, num_mel_filters=128, min_frequency=0.0,
                          max_frequency=8000.0, sampling_rate=16000, norm="slaney",
                          mel_scale="slaney")
    np.testing.assert_allclose(LM.mel_filterbank(), ref.T, rtol=1e-9, atol=1e-12)


def test_filterbank_triangles_have_unit_area_in_hz():
    fb = LM.mel_filterbank(n_mels=8, n_fft=4000, sr=16000, f_max=8000.0)  # fine bins: 4 Hz
    area = fb.sum(axis=1) * (16000 / 4000)
    np.testing.assert_allclose(area, 1.0, rtol=2e-2)


@pytest.mark.parametrize("n", [16000, 16000 * 3 + 123, 4817])
def test_log_mel_matches_whisper_feature_extractor(n):
    from transformers import WhisperFeatureExtractor
    fe = WhisperFeatureExtractor(feature_size=128)
    x = S.waveforms([n], seed=5)[0]
    ref = fe._np_extract_fbank_features(x[None].astype(np.float64), "cpu")[0]
    got = LM.log_mel(x)
    assert got.shape == (128, n // 160) == ref.shape
    np.testing.assert_allclose(got, ref, rtol=0, atol=2e-5)


def test_log_mel_silence_gain_and_tone():
    assert np.all(LM.log_mel(np.zeros(3200)) == (-10.0 + 4.0) / 4.0)
    x = S.waveforms([8000], seed=6)[0]
    a = LM.log_mel(x)
    b = LM.log_mel(10.0 * x)  # energy x100: log10 + 2, the clamp moves with the max
    np.testing.assert_allclose(b - a, 0.5, atol=1e-9)
    t = np.arange(16000) / 16000.0
    tone = np.sin(2 * math.pi * 1000.0 * t)
    m = LM.log_mel(tone)[:, 10:-10].mean(axis=1)
    pts = LM.mel_to_hz_slaney(np.linspace(0, LM.hz_to_mel_slaney(8000.0), 130))[1:-1]
    assert abs(pts[int(np.argmax(m))] - 1000.0) < 60.0


def test_batch_zero_fills_and_lengths():
    waves = S.waveforms([0, 16000, 4817], seed=7)
    feats, lens = LM.log_mel_batch(waves)
    assert lens == [0, 100, 30]
    assert feats.shape == (3, 128, 100)
    assert np.all(feats[0] == 0) and np.all(feats[2, :, 30:] == 0)
    np.testing.assert_array_equal(feats[2, :, :30], LM.log_mel(waves[2]))
