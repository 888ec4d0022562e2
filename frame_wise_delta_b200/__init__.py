"""B200 (sm_100a) frame-wise delta-rule memory (VDA) of Video DeltaNet.

The kernels live in libvdn.so (C ABI in include/vdn.h); `vdn` is its thin
ctypes binding and `synth` the seeded workload generator. Importing the
package does not load the library; the first binding call does, and fails
loudly if it is missing.
"""
__all__ = ["vdn", "synth"]
