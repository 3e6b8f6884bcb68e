"""CPU oracle for the AuT audio encoder forward pass.

TEST INFRASTRUCTURE ONLY.  Only the test suite, the package entry's smoke()
check and the benchmark's CPU-baseline leg may import, call or execute anything
here; the product path (the CUDA library and its Python binding) never does,
and fails loudly when its extension is missing instead of falling back to this.

The oracle is a plain, slow, obviously correct restatement of what the pages
say the encoder computes, in fp64 (or fp32 for the large workloads), sharing no
code, tables or constants with the CUDA path.
"""
from .aut_oracle import *  # noqa: F401,F403
from . import inject, logmel  # noqa: F401
