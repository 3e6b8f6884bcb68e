"""ctypes binding of libaut.so (include/aut.h).  Argument marshalling only:
every step of the encoder runs in the library's kernels.  Raises when the
library has not been built; there is no fallback."""
from __future__ import annotations

import ctypes
import os
import re
from ctypes import POINTER, c_char_p, c_float, c_int32, c_size_t, c_void_p

# AUT_LIB=debug selects the bounds-checked build (libaut_debug.so, built by
# `python -m audio_encoder_aut_b200.build --debug-bounds`).
LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)),
                        "libaut_debug.so" if os.environ.get("AUT_LIB") == "debug" else "libaut.so")
HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include",
                      "aut.h")

AUT_OK, AUT_ERR_INVALID_ARG, AUT_ERR_UNSUPPORTED, AUT_ERR_WORKSPACE, AUT_ERR_CUDA, \
    AUT_ERR_TIMEOUT, AUT_ERR_BOUNDS = range(7)

EPI_BF16, EPI_BF16_GELU, EPI_RESID_F32, EPI_F32 = 0, 1, 2, 3
LINEAR_FAULT_INJECT, LINEAR_SINGLE_CTA, LINEAR_F16 = 1, 2, 4

KERNEL_KINDS = ["upload", "zero_pads", "conv1", "conv2", "conv3", "conv_out", "layernorm",
                "qkv", "attention", "o_proj", "fc1", "fc2", "proj1", "proj2"]
GEMM_KINDS = {"conv2", "conv3", "conv_out", "qkv", "o_proj", "fc1", "fc2", "proj1", "proj2"}


class aut_config(ctypes.Structure):
    _fields_ = [("d_model", c_int32), ("layers", c_int32), ("heads", c_int32),
                ("ffn", c_int32), ("mel_bins", c_int32), ("n_window", c_int32),
                ("n_window_infer", c_int32), ("conv_ch", c_int32), ("output_dim", c_int32),
                ("conv_chunksize", c_int32), ("ln_eps", c_float)]


LAYER_FIELDS = ["ln1_w", "ln1_b", "qkv_w", "qkv_b", "o_w", "o_b",
                "ln2_w", "ln2_b", "fc1_w", "fc1_b", "fc2_w", "fc2_b"]


class aut_layer_weights(ctypes.Structure):
    _fields_ = [(n, c_void_p) for n in LAYER_FIELDS]


class aut_weights(ctypes.Structure):
    _fields_ = ([(n, c_void_p) for n in ["conv1_w", "conv1_b", "conv2_w", "conv2_b", "conv3_w",
                                         "conv3_b", "conv_out_w", "conv_out_b"]]
                + [("layers", POINTER(aut_layer_weights))]
                + [(n, c_void_p) for n in ["ln_post_w", "ln_post_b", "proj1_w", "proj1_b",
                                           "proj2_w", "proj2_b", "conv2_w_tap", "conv3_w_tap",
                                           "conv_out_w_fc", "pos_table", "proj1_w_dup",
                                           "proj2_w_dup", "o_w_f16"]])


class aut_trace(ctypes.Structure):
    _fields_ = [("events", POINTER(c_void_p)), ("capacity", c_int32), ("count", c_int32),
                ("kinds", POINTER(c_int32))]


class AutError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)} (status {status})")


_lib = None

_SIGNATURES = {
    "aut_plan": (c_int32, [POINTER(aut_config), POINTER(c_int32), c_int32, POINTER(c_int32),
                           POINTER(c_int32), POINTER(c_int32), POINTER(c_int32),
                           POINTER(c_int32)]),
    "aut_workspace_bytes": (c_size_t, [POINTER(aut_config), c_int32, c_int32, c_int32]),
    "aut_prepared_bytes": (c_size_t, [POINTER(aut_config)]),
    "aut_prepare_weights": (c_int32, [POINTER(aut_config), POINTER(aut_weights), c_void_p,
                                      c_size_t, POINTER(aut_weights), c_void_p]),
    "aut_encode": (c_int32, [POINTER(aut_config), POINTER(aut_weights), c_void_p, c_int32,
                             POINTER(c_int32), c_int32, c_void_p, c_void_p, c_size_t, c_void_p]),
    "aut_encode_traced": (c_int32, [POINTER(aut_config), POINTER(aut_weights), c_void_p, c_int32,
                                    POINTER(c_int32), c_int32, c_void_p, c_void_p, c_size_t,
                                    c_void_p, POINTER(aut_trace)]),
    "aut_frontend": (c_int32, [POINTER(aut_config), POINTER(aut_weights), c_void_p, c_int32,
                               POINTER(c_int32), c_int32, c_void_p, c_int32, c_void_p, c_size_t,
                               c_void_p]),
    "aut_encode_packed": (c_int32, [POINTER(aut_config), POINTER(aut_weights), c_void_p, c_int32,
                                    POINTER(c_int32), c_int32, c_int32, c_void_p, c_void_p,
                                    c_size_t, c_void_p]),
    "aut_linear": (c_int32, [c_void_p, c_void_p, c_void_p, c_void_p, c_int32, c_int32, c_int32,
                             c_int32, c_void_p, c_int32, c_int32, c_void_p]),
    "aut_layernorm": (c_int32, [c_void_p, c_void_p, c_void_p, c_void_p, c_int32, c_int32,
                                c_float, c_void_p]),
    "aut_window_attention": (c_int32, [c_void_p, c_void_p, c_int32, c_int32, c_int32,
                                       POINTER(c_int32), c_int32, c_void_p, c_size_t, c_void_p]),
    "aut_window_attention_ex": (c_int32, [c_void_p, c_void_p, c_int32, c_int32, c_int32,
                                          POINTER(c_int32), c_int32, c_void_p, c_size_t, c_int32,
                                          c_int32, c_void_p]),
    "aut_window_attention_noalloc": (c_int32, [c_void_p, c_void_p, c_int32, c_int32, c_int32,
                                               POINTER(c_int32), c_int32, c_void_p]),
    "aut_logmel": (c_int32, [c_void_p, ctypes.c_int64, POINTER(c_int32), c_int32, c_void_p,
                             c_int32, POINTER(c_int32), c_void_p, c_size_t, c_void_p]),
    "aut_logmel_workspace_bytes": (c_size_t, [c_int32, c_int32]),
    "aut_inject_audio": (c_int32, [c_void_p, c_void_p, c_int32, c_int32, c_void_p, c_int32,
                                   c_int32, c_void_p, c_size_t, c_void_p]),
    "aut_inject_workspace_bytes": (c_size_t, [c_int32]),
    "aut_check": (c_int32, [c_void_p]),
    "aut_check_status_word": (c_int32, [c_void_p]),
    "aut_status_string": (c_char_p, [c_int32]),
}


def lib():
    """The loaded library; raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"{LIB_PATH} is missing: build it with `python -m audio_encoder_aut_b200.build` "
                "(the encoder has no CPU fallback)")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGNATURES.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def header_symbols() -> list[str]:
    """Names of the functions include/aut.h declares."""
    text = open(HEADER).read()
    return sorted(set(re.findall(r"^\s*(?:aut_status|size_t|const char \*)\s*\*?\s*(aut_\w+)\(",
                                 text, flags=re.M)))


def _i32(values):
    arr = (c_int32 * max(1, len(values)))()
    for i, v in enumerate(values):
        arr[i] = int(v)
    return arr


def _check(status: int, where: str) -> None:
    if status != AUT_OK:
        raise AutError(status, where)


def status_string(status: int) -> str:
    return lib().aut_status_string(status).decode()


def make_config(cfg) -> aut_config:
    """aut_config from any object with AuTEncoderConfig-style attribute names."""
    return aut_config(cfg.d_model, cfg.encoder_layers, cfg.encoder_attention_heads,
                      cfg.encoder_ffn_dim, cfg.num_mel_bins, cfg.n_window, cfg.n_window_infer,
                      cfg.downsample_hidden_size, cfg.output_dim, cfg.conv_chunksize,
                      float(cfg.ln_eps))


# ---------------------------------------------------------- C-ABI names ----

def aut_plan(cfg: aut_config, feature_lens):
    """-> (tokens_per_request, cu_seqlens, total_tokens, num_windows, num_chunks)."""
    L = lib()
    lens = _i32(feature_lens)
    total, nw, nch = c_int32(), c_int32(), c_int32()
    _check(L.aut_plan(ctypes.byref(cfg), lens, len(feature_lens), None, None,
                      ctypes.byref(total), ctypes.byref(nw), ctypes.byref(nch)), "aut_plan")
    tpr = (c_int32 * max(1, len(feature_lens)))()
    cu = (c_int32 * (nw.value + 1))()
    _check(L.aut_plan(ctypes.byref(cfg), lens, len(feature_lens), tpr, cu, None, None, None),
           "aut_plan")
    return (list(tpr)[:len(feature_lens)], list(cu), total.value, nw.value, nch.value)


def aut_plan_status(cfg: aut_config, feature_lens) -> int:
    lens = _i32(feature_lens)
    t = c_int32()
    return lib().aut_plan(ctypes.byref(cfg), lens, len(feature_lens), None, None,
                          ctypes.byref(t), None, None)


def aut_workspace_bytes(cfg: aut_config, total_tokens: int, num_windows: int,
                        num_chunks: int) -> int:
    return lib().aut_workspace_bytes(ctypes.byref(cfg), total_tokens, num_windows, num_chunks)


def aut_prepared_bytes(cfg: aut_config) -> int:
    return lib().aut_prepared_bytes(ctypes.byref(cfg))


def aut_prepare_weights(cfg, src: aut_weights, dst: int, dst_bytes: int, stream: int) -> aut_weights:
    out = aut_weights()
    _check(lib().aut_prepare_weights(ctypes.byref(cfg), ctypes.byref(src), dst, dst_bytes,
                                     ctypes.byref(out), stream), "aut_prepare_weights")
    return out


def aut_encode(cfg, prepared, features: int, t_max: int, feature_lens, out: int, workspace: int,
               ws_bytes: int, stream: int) -> int:
    return lib().aut_encode(ctypes.byref(cfg), ctypes.byref(prepared), features, t_max,
                            _i32(feature_lens), len(feature_lens), out, workspace, ws_bytes,
                            stream)


def aut_encode_traced(cfg, prepared, features: int, t_max: int, feature_lens, out: int,
                      workspace: int, ws_bytes: int, stream: int, trace: aut_trace | None) -> int:
    return lib().aut_encode_traced(ctypes.byref(cfg), ctypes.byref(prepared), features, t_max,
                                   _i32(feature_lens), len(feature_lens), out, workspace, ws_bytes,
                                   stream, ctypes.byref(trace) if trace is not None else None)


def aut_frontend(cfg, prepared, features: int, t_max: int, feature_lens, x0: int,
                 with_positions: bool, workspace: int, ws_bytes: int, stream: int) -> int:
    return lib().aut_frontend(ctypes.byref(cfg), ctypes.byref(prepared), features, t_max,
                              _i32(feature_lens), len(feature_lens), x0, int(with_positions),
                              workspace, ws_bytes, stream)


def aut_encode_packed(cfg, prepared, hidden: int, total_tokens: int, cu_seqlens, n_layers: int,
                      out: int | None, workspace: int, ws_bytes: int, stream: int) -> int:
    return lib().aut_encode_packed(ctypes.byref(cfg), ctypes.byref(prepared), hidden,
                                   total_tokens, _i32(cu_seqlens), len(cu_seqlens) - 1, n_layers,
                                   out, workspace, ws_bytes, stream)


def aut_linear(x: int, w: int, bias: int | None, y: int, M: int, N: int, K: int, epilogue: int,
               status: int | None, timeout_ms: int, flags: int, stream: int) -> int:
    return lib().aut_linear(x, w, bias, y, M, N, K, epilogue, status, timeout_ms, flags, stream)


def aut_layernorm(x: int, gamma: int, beta: int, y: int, T: int, d: int, eps: float,
                  stream: int) -> int:
    return lib().aut_layernorm(x, gamma, beta, y, T, d, eps, stream)


def aut_window_attention(qkv: int, out: int, T: int, d: int, heads: int, cu_seqlens,
                         workspace: int, ws_bytes: int, stream: int) -> int:
    return lib().aut_window_attention(qkv, out, T, d, heads, _i32(cu_seqlens),
                                      len(cu_seqlens) - 1, workspace, ws_bytes, stream)


def aut_window_attention_ex(qkv: int, out: int, T: int, d: int, heads: int, cu_seqlens,
                            workspace: int, ws_bytes: int, timeout_ms: int, flags: int,
                            stream: int) -> int:
    return lib().aut_window_attention_ex(qkv, out, T, d, heads, _i32(cu_seqlens),
                                         len(cu_seqlens) - 1, workspace, ws_bytes, timeout_ms,
                                         flags, stream)


ATTN_FAULT_INJECT = 1


def aut_window_attention_noalloc(qkv: int, out: int, T: int, d: int, heads: int, cu_seqlens,
                                 stream: int) -> int:
    """Window attention without a caller workspace (scratch in the library's own
    device array; see include/aut.h for its limits)."""
    return lib().aut_window_attention_noalloc(qkv, out, T, d, heads, _i32(cu_seqlens),
                                              len(cu_seqlens) - 1, stream)


def aut_logmel(waveform: int, s_max: int, sample_lens, features: int, t_max: int,
               workspace: int, ws_bytes: int, stream: int):
    """-> (status, feature_lens)."""
    fl = (c_int32 * max(1, len(sample_lens)))()
    st = lib().aut_logmel(waveform, s_max, _i32(sample_lens), len(sample_lens), features, t_max,
                          fl, workspace, ws_bytes, stream)
    return st, list(fl)[:len(sample_lens)]


def aut_logmel_workspace_bytes(n_req: int, t_max: int) -> int:
    return lib().aut_logmel_workspace_bytes(n_req, t_max)


def aut_inject_audio(embeds: int, token_ids: int, L: int, audio_pad_id: int, audio: int, T: int,
                     D: int, workspace: int, ws_bytes: int, stream: int) -> int:
    return lib().aut_inject_audio(embeds, token_ids, L, audio_pad_id, audio, T, D, workspace,
                                  ws_bytes, stream)


def aut_inject_workspace_bytes(L: int) -> int:
    return lib().aut_inject_workspace_bytes(L)


def aut_check(workspace: int) -> int:
    return lib().aut_check(workspace)


def aut_check_status_word(status: int) -> int:
    return lib().aut_check_status_word(status)
