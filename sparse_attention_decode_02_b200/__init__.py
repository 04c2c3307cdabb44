"""B200 (sm_100a) QSA decode hot path: C-ABI library libqsa.so and its thin binding.

The compute lives in csrc/ (hand-written CUDA for sm_100a behind the C ABI declared in
include/qsa.h); qsa.py only marshals torch device tensors and streams into that ABI.
"""
from .qsa import (QSA_INPUTS_EARLY, QSA_INPUTS_ORDERED, QSA_KV_F16, QSA_KV_FP8, QSA_MAX_QUERIES,  # noqa: F401
                  QSA_POOLED_F16, QSA_POOLED_FP8, QSA_SCAN_CUDA_CORES, QSA_SCAN_TENSOR, Qsa, QsaConfig, QsaError, alloc_layer,
                  alloc_multi_outputs, alloc_step_outputs, buffer_bytes, cp_merge, cp_select, load_library, make_config,
                  sparse_attend_noalloc)
