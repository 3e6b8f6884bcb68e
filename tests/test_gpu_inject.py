"""The GPU audio injection (aut_inject_audio) against the injection oracle:
bit-exact (a copy with one round-to-nearest-even to bf16 on both sides);
placeholders everywhere, nowhere, at the ends; a count mismatch reported
through the status word with nothing written past the audio rows; and the
encoder's own output injected into a synthetic prompt."""
import numpy as np
import pytest

import aut_synth as S
from oracle import inject as I

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

from audio_encoder_aut_b200 import _lib as A  # noqa: E402

PAD = 151646


def _run(emb, ids, audio, pad=PAD):
    L, D = emb.shape
    ed = torch.from_numpy(S.round_bf16(emb.astype(np.float32))).cuda().to(torch.bfloat16)
    idd = torch.from_numpy(np.asarray(ids, np.int32)).cuda()
    ad = torch.from_numpy(np.ascontiguousarray(audio, np.float32)).cuda()
    ws = torch.empty(A.aut_inject_workspace_bytes(L), dtype=torch.uint8, device="cuda")
    st = A.aut_inject_audio(ed.data_ptr(), idd.data_ptr(), L, pad, ad.data_ptr(), audio.shape[0],
                            D, ws.data_ptr(), ws.numel(), torch.cuda.current_stream().cuda_stream)
    torch.cuda.synchronize()
    return st, A.aut_check(ws.data_ptr()), ed.float().cpu().numpy()


def _ids(L, pads, seed):
    rng = np.random.default_rng(seed)
    ids = rng.integers(0, 150000, size=L)
    ids[pads] = PAD
    return ids


@pytest.mark.parametrize("L,D,where", [
    (3000, 2048, "random"), (777, 1024, "all"), (500, 2048, "none"), (4097, 12, "ends"),
    (1, 2048, "all")])
def test_inject_matches_oracle_bit_exact(L, D, where):
    rng = np.random.default_rng(L)
    if where == "random":
        pads = np.sort(rng.choice(L, size=L // 3, replace=False))
    elif where == "all":
        pads = np.arange(L)
    elif where == "none":
        pads = np.arange(0)
    else:
        pads = np.r_[0:5, L - 5:L]
    ids = _ids(L, pads, L + 1)
    emb = rng.standard_normal((L, D)).astype(np.float32)
    audio = rng.standard_normal((len(pads), D)).astype(np.float32)
    st, dev, got = _run(emb, ids, audio)
    assert st == A.AUT_OK and dev == A.AUT_OK
    ref = I.inject_audio(S.round_bf16(emb), ids, PAD, S.round_bf16(audio))
    np.testing.assert_array_equal(got, ref)


def test_inject_count_mismatch_is_reported_and_bounded():
    rng = np.random.default_rng(5)
    L, D = 200, 64
    pads = np.sort(rng.choice(L, size=40, replace=False))
    ids = _ids(L, pads, 6)
    emb = rng.standard_normal((L, D)).astype(np.float32)
    audio = rng.standard_normal((30, D)).astype(np.float32)  # 10 rows short
    st, dev, got = _run(emb, ids, audio)
    assert st == A.AUT_OK and dev == A.AUT_ERR_INVALID_ARG
    # the first 30 placeholders filled, the last 10 untouched, text rows untouched
    np.testing.assert_array_equal(got[pads[:30]], S.round_bf16(audio))
    np.testing.assert_array_equal(got[pads[30:]], S.round_bf16(emb)[pads[30:]])


def test_inject_encoder_output_into_prompt():
    from audio_encoder_aut_b200.encoder import Encoder
    cfg = S.TINY
    w = S.weights(cfg)
    enc = Encoder(cfg, w, 0)
    lens = [237, 61]
    out = enc.encode(enc.features_to_device(S.features(lens)), lens)
    T = out.shape[0]
    ids = np.r_[np.arange(5), np.full(T, PAD), np.arange(7)]
    emb = np.random.default_rng(1).standard_normal((len(ids), cfg.output_dim)).astype(np.float32)
    st, dev, got = _run(emb, ids, out.cpu().numpy())
    assert st == A.AUT_OK and dev == A.AUT_OK
    np.testing.assert_array_equal(got[5:5 + T], S.round_bf16(out.cpu().numpy()))
