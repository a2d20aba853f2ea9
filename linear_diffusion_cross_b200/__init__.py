"""B200-native fused linear diffusion cross-entropy (LM-head loss, fwd + bwd).

The computation lives in libfldce.so (hand-written sm_100a CUDA, C ABI in
include/fldce.h); ``binding`` is its ctypes binding and ``synth`` draws the
seeded synthetic workloads.  Importing the package loads nothing: the
library is loaded on first use, and a missing library is an error.
"""
__all__ = ["binding", "synth"]
