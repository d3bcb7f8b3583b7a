"""B200-native routed MoE layer: router top-k, count/scan, permute, grouped SwiGLU GEMM, combine.

The compute path lives in ``libmoe_b200.so`` (hand-written CUDA for sm_100a behind
the C ABI declared in ``include/moe.h``); :mod:`.binding` is a thin ctypes layer
over it that marshals torch tensors into pointers.  There is no CPU fallback:
every call raises if the shared library is missing or no CUDA device is present.
"""
from .config import MoEConfig, ALL as CONFIGS, get as get_config  # noqa: F401

__all__ = ["MoEConfig", "CONFIGS", "get_config"]
