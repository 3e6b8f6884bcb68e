"""Runs workloads through the bounds-checked library (AUT_LIB=debug, set by the
caller before this module is imported) and prints one JSON line: which library
was loaded, every device status read back, and the tiny forward's worst
element error against the oracle relative to its row RMS."""
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

import aut_synth as S  # noqa: E402
import oracle as O  # noqa: E402
from audio_encoder_aut_b200 import _lib as A  # noqa: E402
from audio_encoder_aut_b200.encoder import Encoder  # noqa: E402


def main():
    out = {"lib": os.path.basename(A.LIB_PATH), "status": {}}
    # The tiny encoder, non-linear stem and a conv_out bias, ragged requests.
    cfg = S.TINY
    w = S.weights(cfg, conv_scale=25.0, conv_out_bias=True)
    lens = [237, 0, 61, 100, 9]
    feats = S.features(lens)
    enc = Encoder(cfg, w, 0)
    got = enc.encode(enc.features_to_device(feats), lens).cpu().numpy().astype(np.float64)
    torch.cuda.synchronize()
    out["status"]["tiny"] = int(enc.check())
    ref, _ = O.forward(cfg, w, feats, lens)
    rms = np.sqrt((ref ** 2).mean(1, keepdims=True))
    out["tiny_max_err_over_rms"] = float((np.abs(got - ref) / rms).max())
    # Omni dims: the stem's conv epilogues and the pack, the layers' per-row and
    # TMA-store epilogues, the tensor-core attention.
    cfg = S.OMNI
    w = S.weights(cfg)
    lens = [1734, 90, 610, 333]
    enc = Encoder(cfg, w, 0)
    enc.encode(enc.features_to_device(S.features(lens)), lens)
    torch.cuda.synchronize()
    out["status"]["omni"] = int(enc.check())
    # Kernel level: narrow tiles use the per-row epilogue (M not a multiple of 128).
    st = torch.cuda.current_stream().cuda_stream
    for (M, N, K, epi) in [(77, 16, 64, 2), (300, 240, 128, 1), (31, 48, 64, 0), (129, 2048, 1280, 3)]:
        x = torch.randn(M, K, device="cuda").to(torch.bfloat16)
        wt = (torch.randn(N, K, device="cuda") * 0.05).to(torch.bfloat16)
        y = torch.zeros(M, N, device="cuda", dtype=torch.float32 if epi in (2, 3) else torch.bfloat16)
        s = torch.zeros(1, dtype=torch.int32, device="cuda")
        assert A.aut_linear(x.data_ptr(), wt.data_ptr(), None, y.data_ptr(), M, N, K, epi,
                            s.data_ptr(), 0, A.LINEAR_SINGLE_CTA, st) == A.AUT_OK
        torch.cuda.synchronize()
        out["status"][f"linear_{M}x{N}x{K}"] = int(A.aut_check_status_word(s.data_ptr()))
    print(json.dumps(out), flush=True)


if __name__ == "__main__":
    main()
