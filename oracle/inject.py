"""Plain CPU oracle of the audio injection into the decoder's input sequence.

TEST INFRASTRUCTURE ONLY: imported by the tests, never by the product path.

cubic.dev "Audio Encoder Component", Audio Injection Logic: the encoder's
output rows are not appended to the text; they replace the embeddings at the
<|audio_pad|> placeholder positions of the decoder's token sequence.  Reading
taken where the page is silent: the placeholders are filled in sequence order
by the encoder's rows in packed order (request by request, token by token), so
their count must equal the number of encoder rows; every other row is kept.
"""
from __future__ import annotations

import numpy as np

__all__ = ["inject_audio"]


def inject_audio(text_embeds: np.ndarray, token_ids, audio_pad_id: int,
                 audio_rows: np.ndarray) -> np.ndarray:
    """[L, D] text embeddings, L token ids, [T, D] encoder rows -> [L, D] with
    the j-th placeholder position (in sequence order) holding audio row j."""
    out = np.array(text_embeds, copy=True)
    pos = [i for i, t in enumerate(token_ids) if t == audio_pad_id]
    if len(pos) != audio_rows.shape[0]:
        raise ValueError(f"{len(pos)} placeholders for {audio_rows.shape[0]} audio rows")
    for j, i in enumerate(pos):
        out[i] = audio_rows[j]
    return out
