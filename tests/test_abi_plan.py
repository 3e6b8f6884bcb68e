"""The C ABI without a GPU: the library loads and exports every symbol the
header declares; the host planner matches the oracle's planner bit for bit;
argument errors are rejected before anything is launched."""
import ctypes

import numpy as np
import pytest

import aut_synth as S
import oracle as O
from audio_encoder_aut_b200 import _lib as A


def test_library_exports_every_header_symbol():
    lib = A.lib()
    names = A.header_symbols()
    assert len(names) >= 13
    for n in names:
        assert hasattr(lib, n), n


def _check_plan(cfg, lens):
    tpr, cu, total, nw, nch = A.aut_plan(A.make_config(cfg), lens)
    lay = O.plan(cfg, lens)
    assert tpr == lay.tokens_per_request
    assert cu == lay.cu_seqlens
    assert total == lay.total_tokens and nw == len(lay.cu_seqlens) - 1
    assert nch == len(lay.chunks)


@pytest.mark.parametrize("workload", ["tiny", "asr06b_30s", "omni_16req", "omni_20min",
                                      "omni_256req"])
def test_plan_matches_oracle_on_workloads(workload):
    _check_plan(S.WORKLOADS[workload], S.request_lengths(workload))


def test_plan_ragged_long_form():
    _check_plan(S.OMNI, S.request_lengths("omni_20min_ragged"))


@pytest.mark.parametrize("seed", range(6))
def test_plan_matches_oracle_random(seed):
    lens = S.random_lengths(40, 0, 2500, seed)
    _check_plan(S.OMNI, lens)
    _check_plan(S.TINY, lens)


def test_plan_edge_lengths():
    _check_plan(S.OMNI, [0])
    _check_plan(S.OMNI, [])
    _check_plan(S.OMNI, [1, 2, 7, 8, 9, 99, 100, 101, 799, 800, 801, 1599, 1600])
    assert A.aut_plan(A.make_config(S.OMNI), [0, 0])[2] == 0


def test_plan_rejects_bad_arguments():
    c = A.make_config(S.OMNI)
    assert A.aut_plan_status(c, [5, -1]) == A.AUT_ERR_INVALID_ARG
    bad = A.make_config(S.OMNI)
    bad.n_window_infer = 850
    assert A.aut_plan_status(bad, [100]) == A.AUT_ERR_UNSUPPORTED
    bad = A.make_config(S.OMNI)
    bad.n_window_infer = 1000      # 130 tokens per window: more than one 128-row tile
    assert A.aut_plan_status(bad, [100]) == A.AUT_ERR_UNSUPPORTED
    bad = A.make_config(S.OMNI)
    bad.mel_bins = 80
    assert A.aut_plan_status(bad, [100]) == A.AUT_ERR_UNSUPPORTED
    bad = A.make_config(S.OMNI)
    bad.heads = 7
    assert A.aut_plan_status(bad, [100]) == A.AUT_ERR_UNSUPPORTED
    assert A.lib().aut_plan(None, None, 0, None, None, None, None, None) == A.AUT_ERR_INVALID_ARG


def test_workspace_and_prepared_sizes():
    c = A.make_config(S.OMNI)
    ws = A.aut_workspace_bytes(c, 3200, 31, 250)
    # at least the fp32 residual stream plus the bf16 qkv buffer
    assert ws >= 3200 * 1280 * 4 + 3200 * 3840 * 2
    assert A.aut_workspace_bytes(c, 6400, 62, 500) > ws
    assert A.aut_prepared_bytes(c) >= 2 * 480 * 9 * 480 * 2 + 1280 * 7680 * 2
    bad = A.make_config(S.OMNI)
    bad.conv_ch = 100
    assert A.aut_workspace_bytes(bad, 10, 1, 1) == 0


def test_conv_widths_accepted_are_the_documented_set():
    """aut.h documents conv_ch as one of 16, 32, 64, 128, 192, 240, 256, 384,
    480, 512; every other width up to 1024 is refused before any launch."""
    documented = {16, 32, 64, 128, 192, 240, 256, 384, 480, 512}
    for C in range(1, 1025):
        c = A.make_config(S.OMNI)
        c.conv_ch = C
        assert (A.aut_prepared_bytes(c) > 0) == (C in documented), C
        assert (A.aut_plan_status(c, [100]) == A.AUT_OK) == (C in documented), C


def test_entry_points_reject_before_launch():
    """Argument errors come back without touching a GPU (none is present here)."""
    L = A.lib()
    c = A.make_config(S.TINY)
    w = A.aut_weights()
    lens = (ctypes.c_int32 * 1)(237)
    # incomplete weights
    assert L.aut_encode(ctypes.byref(c), ctypes.byref(w), 1024, 300, lens, 1, 1024, 1024,
                        1 << 30, None) == A.AUT_ERR_INVALID_ARG
    # length beyond T_max
    assert L.aut_encode(ctypes.byref(c), ctypes.byref(w), 1024, 200, lens, 1, 1024, 1024,
                        1 << 30, None) == A.AUT_ERR_INVALID_ARG
    # GEMM shapes the kernel does not take
    assert A.aut_linear(1024, 1024, None, 1024, 128, 64, 100, 0, None, 0, 0, 0) == \
        A.AUT_ERR_UNSUPPORTED
    assert A.aut_linear(1024, 1024, None, 1024, 128, 64, 64, 7, None, 0, 0, 0) == \
        A.AUT_ERR_INVALID_ARG
    # a window longer than one tile
    assert A.aut_window_attention(1024, 1024, 200, 64, 4, [0, 200], 1024, 1024, 0) == \
        A.AUT_ERR_INVALID_ARG
    assert A.aut_layernorm(1024, 1024, 1024, 1024, 4, 6, 1e-5, 0) == A.AUT_ERR_INVALID_ARG
    assert A.status_string(A.AUT_ERR_TIMEOUT) == "device pipeline wait timed out"


def test_missing_library_fails_loudly(monkeypatch, tmp_path):
    monkeypatch.setattr(A, "_lib", None)
    monkeypatch.setattr(A, "LIB_PATH", str(tmp_path / "libaut.so"))
    with pytest.raises(RuntimeError, match="no CPU fallback"):
        A.lib()
