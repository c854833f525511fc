"""B200 (sm_100a) implementation of the Faster Flash Decoding decode path.

The compute path lives in the CUDA library ``libffd_b200.so`` (C ABI in
``include/ffd.h``); :mod:`sparse_long_context_ffd_b200.ffd` is its ctypes
binding.
"""
from . import ffd  # noqa: F401
from .ffd import (FFDError, Shape, DecodeBuffers, decode, quantize_keys, make_shape,  # noqa: F401
                  workspace_init, decode_workspace_bytes, check_device_status,
                  FFD_LAST_BLOCK)
from .step import DecodeStep, StandInAttentionLayer  # noqa: F401,E402
