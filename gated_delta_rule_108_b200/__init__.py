"""B200-native Kimi Delta Attention (gated delta rule) recurrence.

The compute lives in ``libkda_b200.so`` (hand-written CUDA for sm_100a behind a
C ABI, declared in ``include/kda.h``); :mod:`.kda` is the thin Python binding.
Importing this package does not load the library: the first call does, and it
raises if the library is missing -- there is no CPU fallback.
"""
from .kda import (  # noqa: F401
    KDAError,
    chunk_fwd,
    chunk_fwd_workspace_size,
    recurrent_step,
    library_path,
)
