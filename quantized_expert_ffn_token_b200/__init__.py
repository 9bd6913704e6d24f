"""Quantized sparse-MoE feed-forward layer for one NVIDIA B200 (sm_100a).

The compute path is the CUDA library ``libqeffn.so`` behind the C ABI in
``include/moe.h``; ``capi`` is its ctypes binding and ``session`` a small
convenience layer that owns a context, loads seeded synthetic layers and
runs forwards.  PyTorch provides device memory and streams only.
"""
from . import capi  # noqa: F401  (fails loudly when the library is not built)
