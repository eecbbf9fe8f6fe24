"""B200-native inner loop of end-to-end test-time training (TTT-E2E) with the
E2-TTT closed-form chunk update.

The compute path is libttt.so (hand-written sm_100a CUDA behind a C ABI,
include/ttt.h); `weight_long_context_b200.ttt` is its ctypes binding and
`weight_long_context_b200.inputs` the seeded synthetic input generator.
Importing the package loads nothing; the library is loaded on first use and
the binding raises if it is missing (there is no CPU fallback).
"""
__all__ = ["ttt", "inputs", "build"]
