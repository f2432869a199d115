"""2D Neighborhood Attention for the B200 (sm_100a).

The operator lives in the C-ABI library libna2d.so (include/na2d.h, CUDA
sources under csrc/); `vision_sliding_window_b200.na2d` is its Python
binding and `vision_sliding_window_b200.inputs` the seeded input generators.
"""
__all__ = ["na2d", "inputs", "build"]
