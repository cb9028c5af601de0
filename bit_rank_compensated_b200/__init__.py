"""libsvdq for B200: SVDQuant NVFP4 W4A4 + low-rank linear layer (C ABI + thin binding).

``bit_rank_compensated_b200.svdq`` is the Python binding of the C ABI declared in
include/svdq.h; ``bit_rank_compensated_b200.build`` compiles libsvdq.so in-tree.
Importing this package does not load the CUDA library.
"""
__all__ = ["svdq", "build"]
