"""B200-native (sm_100a) fused Mixture-of-Experts layer forward.

The compute path lives in ``libmoe.so`` (hand-written CUDA for sm_100a behind a C ABI,
declared in ``include/moe.h``).  ``mixture_experts_layer_35_b200.moe`` is the thin
ctypes binding; it raises if the library is missing, and nothing here falls back to
the CPU.  ``inputs`` draws the seeded synthetic workloads.
"""
__version__ = "0.1.0"
