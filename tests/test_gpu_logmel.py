"""The GPU log-mel front end (aut_logmel) against the log-mel oracle on the
same seeded speech-like waveforms: element by element within the bf16 output
bound, per frame within the acceptance bound; ragged lengths, empty requests,
the shortest request, zero fill past each request's frames, silence; and
waveform -> features -> encoder output against the oracle's composition."""
import numpy as np
import pytest

import aut_synth as S
import oracle as O
from gpu_util import assert_bf16_output_close, assert_rows_close
from oracle import logmel as LM

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

from audio_encoder_aut_b200 import _lib as A  # noqa: E402
from audio_encoder_aut_b200.encoder import Encoder  # noqa: E402

_ENC = {}


def _enc(name="tiny"):
    if name not in _ENC:
        cfg = S.WORKLOADS[name]
        w = S.weights(cfg, conv_scale=10.0)
        _ENC[name] = (cfg, w, Encoder(cfg, w, 0))
    return _ENC[name]


def _gpu_logmel(enc, waves, t_max=None):
    s_max = max([len(x) for x in waves] + [1])
    buf = np.zeros((len(waves), s_max), np.float32)
    for i, x in enumerate(waves):
        buf[i, :len(x)] = x
    wd = torch.from_numpy(buf).to(enc.device)
    feats, lens = enc.logmel(wd, [len(x) for x in waves], t_max)
    torch.cuda.synchronize()
    return feats.float().cpu().numpy(), lens


def _ref(waves, t_max=None):
    # The oracle in fp64 on the fp32 samples the GPU sees.
    return LM.log_mel_batch([np.asarray(x, np.float32).astype(np.float64) for x in waves], t_max)


@pytest.mark.parametrize("n_samples", [
    [16000 * 3 + 57],
    [201, 16000, 0, 4817, 160 * 64, 160 * 64 + 159, 160 * 65],
    [16000 * 30],
])
def test_logmel_matches_oracle(n_samples):
    cfg, w, enc = _enc()
    waves = S.waveforms(n_samples, seed=11)
    got, lens = _gpu_logmel(enc, waves)
    ref, ref_lens = _ref(waves)
    assert lens == ref_lens == [n // 160 for n in n_samples]
    assert got.shape == ref.shape
    for r, n in enumerate(lens):
        assert np.all(got[r, :, n:] == 0)
        if n:
            # fp32 DFT and filters, then one bf16 rounding of values in [-1.5, 2.5]
            assert_bf16_output_close(got[r, :, :n].T, ref[r, :, :n].T, f"log-mel request {r}",
                                     atol=2e-3)
            assert_rows_close(got[r, :, :n].T, ref[r, :, :n].T, f"log-mel frames of request {r}")


def test_logmel_zero_fill_beyond_frames_and_silence():
    cfg, w, enc = _enc()
    waves = [np.zeros(3200), S.waveforms([1000], seed=3)[0]]
    got, lens = _gpu_logmel(enc, waves, t_max=40)
    assert lens == [20, 6] and got.shape == (2, 128, 40)
    assert np.all(got[0, :, :20] == -1.5) and np.all(got[0, :, 20:] == 0)
    assert np.all(got[1, :, 6:] == 0)


def test_logmel_rejects_short_and_oversized_requests():
    cfg, w, enc = _enc()
    wd = torch.zeros((1, 1000), device="cuda")
    for lens, t_max in (([150], 8), ([200], 8), ([1001], 8), ([1000], 5)):
        st, _ = A.aut_logmel(wd.data_ptr(), 1000, lens, 0, t_max, 0, 0, 0)
        assert st == A.AUT_ERR_INVALID_ARG


@pytest.mark.parametrize("name,n_samples", [("tiny", [37920, 9600]),
                                            ("asr06b_30s", [16000 * 30])])
def test_waveform_to_encoder_output(name, n_samples):
    """Waveform -> GPU log-mel -> GPU encoder, against oracle log-mel -> oracle
    encoder, within the acceptance bound."""
    cfg, w, enc = _enc(name)
    waves = S.waveforms(n_samples, seed=12)
    s_max = max(n_samples)
    buf = np.zeros((len(waves), s_max), np.float32)
    for i, x in enumerate(waves):
        buf[i, :len(x)] = x
    feats, lens = enc.logmel(torch.from_numpy(buf).cuda(), n_samples)
    out = enc.encode(feats, lens)
    torch.cuda.synchronize()
    assert enc.check() == A.AUT_OK
    ref_feats, ref_lens = _ref(waves)
    ref, _ = O.forward(cfg, w, S.round_bf16(ref_feats.astype(np.float32)), ref_lens,
                       dtype=np.float64 if name == "tiny" else np.float32)
    assert_rows_close(out.cpu().numpy(), ref, f"waveform -> {name} output")
