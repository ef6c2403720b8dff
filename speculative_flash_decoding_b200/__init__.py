"""Speculative flash-decode attention (attention-level speculation) for B200.

For every decode query the library computes, in CUDA kernels for sm_100a,
the attention-sink approximation O_spec (softmax attention over the first S
and last W cached tokens, published early by a kernel launched first at high
priority, with the exact path running beside it), the exact attention
O_exact over the whole cache (split-K flash decoding), the per-token
relative L2 error of O_spec and the commit/discard flag.

The C ABI is include/alspec.h (libalspec.so); ``alspec`` is its ctypes
binding.  Importing the package raises if libalspec.so is missing.
"""
from .alspec import *  # noqa: F401,F403
from .alspec import Decoder, AlspecError, make_desc, SIGNATURES, LIB_PATH  # noqa: F401

__version__ = "0.1.0"
