"""The window-attention entry point that allocates nothing, for callers that
cannot allocate device memory (their memory belongs to another allocator, or
they run where allocation is not allowed, such as during some CUDA-graph
captures).  It must give the same output as the workspace entry point.  This
file sorts last so that a run stopping at the first failure has run every
other test first."""
import numpy as np
import pytest

import aut_synth as S
from audio_encoder_aut_b200 import _lib as A


def test_noalloc_rejects_too_many_windows_before_any_launch():
    # Checked on the host before anything touches a GPU (none is needed): the
    # array holds a status word and at most 32767 cu_seqlens entries.
    assert A.aut_window_attention_noalloc(1024, 1024, 0, 64, 4, [0] * 32768, 0) == \
        A.AUT_ERR_WORKSPACE


@pytest.mark.gpu
def test_noalloc_attention_matches_workspace_attention_on_two_calls():
    """Calls in a row, each checked against the workspace entry point; the
    third has a single window after one with six, so it must ignore the stale
    cu_seqlens entries the earlier call left in the shared array.  After every
    call the status word of the allocation-free entry reads OK."""
    torch = pytest.importorskip("torch")
    st = torch.cuda.current_stream().cuda_stream
    cases = [(20, 64, [104, 104, 1, 17, 128, 50]), (4, 16, [26, 5, 26, 26, 3]),
             (20, 64, [77])]
    for call, (heads, hd, lens) in enumerate(cases):
        d = heads * hd
        cu = [0]
        for n in lens:
            cu.append(cu[-1] + n)
        T = cu[-1]
        rng = np.random.default_rng(100 + call)
        qkv = torch.from_numpy(S.round_bf16(rng.standard_normal((T, 3 * d)).astype(np.float32)))
        qkv = qkv.to("cuda").to(torch.bfloat16)
        ref = torch.zeros((T, d), dtype=torch.float16, device="cuda")
        got = torch.full((T, d), float("nan"), dtype=torch.float16, device="cuda")
        ws = torch.empty(4 * (len(cu) + 1), dtype=torch.uint8, device="cuda")
        assert A.aut_window_attention(qkv.data_ptr(), ref.data_ptr(), T, d, heads, cu,
                                      ws.data_ptr(), ws.numel(), st) == A.AUT_OK
        assert A.aut_window_attention_noalloc(qkv.data_ptr(), got.data_ptr(), T, d, heads, cu,
                                              st) == A.AUT_OK
        torch.cuda.synchronize()
        g = got.float().cpu().numpy()
        r = ref.float().cpu().numpy()
        # Same kernel on the same inputs: the tests' attention bound, and in fact
        # bit-identical output.
        assert np.isfinite(g).all()
        np.testing.assert_allclose(g, r, rtol=1e-4, atol=1e-4 * np.abs(r).max())
        assert np.array_equal(g, r)
        assert A.aut_check_status_word(None) == A.AUT_OK
        assert A.aut_check(ws.data_ptr()) == A.AUT_OK
