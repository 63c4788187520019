"""POET-X orthogonal-equivalence linear layer for NVIDIA B200 (sm_100a).

The compute lives in ``libpoetx.so`` (C ABI in ``include/poetx.h``); ``poetx`` is its
ctypes binding.
"""
from . import poetx  # noqa: F401
from .poetx import PoetxLinear  # noqa: F401

__all__ = ["poetx", "PoetxLinear"]
