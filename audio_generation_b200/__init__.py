"""B200 (sm_100a) MiniMax-H3 transformer-block library: Python binding.

The computation lives in libh3.so (hand-written CUDA for sm_100a, C ABI in
include/h3.h); ``audio_generation_b200.h3`` marshals arguments to it.
"""

from . import h3  # noqa: F401
