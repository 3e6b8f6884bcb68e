"""B200-native AuT (Qwen3-family) audio encoder forward pass.

The computation lives in libaut.so (CUDA for sm_100a, C ABI in include/aut.h);
`_lib` is its ctypes binding and `encoder.Encoder` the PyTorch plumbing
(device memory and streams) around it.
"""
from . import _lib  # noqa: F401

__all__ = ["_lib", "Encoder"]


def __getattr__(name):
    if name == "Encoder":
        from .encoder import Encoder
        return Encoder
    raise AttributeError(name)
