"""B200-native forward pass of a Mixture-of-Experts SwiGLU FFN layer.

The compute path is the C-ABI library libmoe_b200.so (hand-written sm_100a
CUDA kernels, declared in include/moe.h).  `binding` is a thin ctypes layer
over it: argument marshalling only.  The library is loaded on first use and
a missing or unloadable library raises; there is no CPU fallback.
"""
__all__ = ["binding", "synth"]
