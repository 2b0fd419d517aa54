"""B200-native MoE layer: route -> dispatch -> grouped expert FFN -> combine.

The compute path is the CUDA library ``libmoe.so`` (C ABI declared in
``include/moe.h``); ``combine_softmax_top_b200.moe`` is its thin Python
binding. The library is loaded on first use and a missing or stale build
raises: there is no CPU fallback.
"""
from . import workloads  # noqa: F401  (pure input generation, no CUDA needed)

__all__ = ["workloads"]
