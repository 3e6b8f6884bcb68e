"""Pins of the audio-injection oracle (oracle/inject.py): torch's
masked_scatter (the library routine that writes a source's rows, in order,
into the masked rows of a tensor) and the invariants of the definition."""
import numpy as np
import pytest

from oracle import inject as I

torch = pytest.importorskip("torch")


def _case(L, D, n_pad, seed, pad_id=151646):
    rng = np.random.default_rng(seed)
    ids = rng.integers(0, 150000, size=L)
    where = rng.choice(L, size=n_pad, replace=False)
    ids[where] = pad_id
    return rng.standard_normal((L, D)), ids, pad_id, rng.standard_normal((n_pad, D))


@pytest.mark.parametrize("L,D,n_pad", [(50, 8, 13), (300, 16, 300), (40, 4, 0), (1, 3, 1)])
def test_inject_matches_torch_masked_scatter(L, D, n_pad):
    emb, ids, pad, audio = _case(L, D, n_pad, L + n_pad)
    mask = torch.from_numpy(ids == pad)[:, None].expand(L, D)
    ref = torch.from_numpy(emb).masked_scatter(mask, torch.from_numpy(audio))
    np.testing.assert_array_equal(I.inject_audio(emb, ids, pad, audio), ref.numpy())


def test_inject_keeps_text_rows_and_fills_placeholders_in_order():
    emb, ids, pad, audio = _case(120, 6, 31, 3)
    out = I.inject_audio(emb, ids, pad, audio)
    text = ids != pad
    np.testing.assert_array_equal(out[text], emb[text])
    np.testing.assert_array_equal(out[~text], audio)


def test_inject_rejects_count_mismatch():
    emb, ids, pad, audio = _case(60, 4, 10, 4)
    with pytest.raises(ValueError):
        I.inject_audio(emb, ids, pad, audio[:9])
