"""B200-native (sm_100a) forward + backward training step of a depth-dialled GPT.

The step lives in ``libgpt.so`` (C ABI in ``include/gpt.h``, CUDA kernels in
``csrc/``); ``binding`` marshals arguments to it through ctypes and
``runtime`` owns device buffers (torch for memory and streams).
"""
from . import binding  # noqa: F401

__all__ = ["binding"]
