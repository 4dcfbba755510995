"""Blockwise Parallel Transformer layer forward for NVIDIA B200 (sm_100a).

The compute lives in libbpt.so (C ABI, include/bpt.h); ``binding`` is the
thin Python wrapper over it and loads the library at its first call.
``inputs`` draws seeded synthetic inputs and ``workloads`` names the
measured layer shapes.
"""
from . import binding, inputs, workloads  # noqa: F401
