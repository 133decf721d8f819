"""Batch-1 hybrid Gated-DeltaNet + attention inference on B200 (sm_100a).

The compute path is libmk.so (C ABI, include/mk.h); this package is its thin
Python binding. There is no CPU fallback.
"""
from ._abi import (MK_DEVERR_BAD_TOKEN, MK_DEVERR_BARRIER_TIMEOUT, MK_DEVERR_CAPACITY,  # noqa: F401
                   MK_DEVERR_PIPE_TIMEOUT, MkError, load_library)
from .model import Model, make_config, query_sizes, weights_to_device  # noqa: F401
