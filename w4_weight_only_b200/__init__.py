"""w4a: int4 weight-only (AWQ-format) decode of an OLMo-3-32B-shaped decoder on
one NVIDIA B200 (sm_100a).

The compute path is ``libw4a.so`` (CUDA kernels behind the C ABI declared in
``include/w4a.h``); this package is its thin torch binding.  Importing the
package does not load the library; the first call does, and raises if it is
missing (there is no CPU fallback).
"""
from . import _abi  # noqa: F401
from .config import Config, olmo3_32b, tiny  # noqa: F401

__all__ = ["Config", "olmo3_32b", "tiny", "lib_path"]


def lib_path():
    return _abi.lib_path()
