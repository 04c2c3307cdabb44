"""B200 (sm_100a) QSA decode hot path: C-ABI library libqsa.so and its thin binding.

The compute lives in csrc/ (hand-written CUDA for sm_100a behind the C ABI declared in
include/qsa.h); qsa.py only marshals torch device tensors and streams into that ABI.
"""
from .qsa import (Qsa, QsaConfig, QsaError, alloc_layer, alloc_step_outputs, buffer_bytes,  # noqa: F401
                  load_library, make_config, sparse_attend_noalloc)
