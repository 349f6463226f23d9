"""MosaicQuant / ZipperEngine on B200: NVFP4 dense base + sparse 4-bit residual GEMM.

The compute lives in ``libmosaic.so`` (hand-written CUDA for sm_100a, C ABI in
``include/mosaic.h``); ``mosaic`` is its ctypes binding.
"""
from . import mosaic  # noqa: F401
from .mosaic import Layer, MosaicError, lib  # noqa: F401
