"""B200-native RG-LRU recurrent-block core (causal depthwise conv1d k=4,
block-diagonal gates, fp32 linear scan with document resets, GELU-tanh
product), behind the C ABI declared in ``include/rglru.h``.

``lm_causal_depthwise_b200.api`` holds the Python binding (argument
marshalling only; every step runs in the CUDA library ``librglru.so``).
``lm_causal_depthwise_b200.workloads`` holds the seeded synthetic inputs.
Importing the package loads nothing; the library is loaded on first use and
a missing library is an error, never a fallback.
"""
__all__ = ["api", "workloads"]
