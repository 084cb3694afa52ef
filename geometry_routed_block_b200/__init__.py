"""Velox geometry-routed block-sparse attention for B200 (sm_100a).

The CUDA library (libvelox.so, C ABI declared in include/velox.h) does every step
of the path; `geometry_routed_block_b200.velox` is its thin ctypes binding and is
imported on demand, so `synth` can be used without a GPU.
"""
__all__ = ["synth", "velox"]
