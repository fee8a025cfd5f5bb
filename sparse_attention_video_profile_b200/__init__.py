"""B200-native spatial/temporal sparse 3D attention (Sparse VideoGen style).

The compute path lives in the CUDA library ``libsvg.so`` built from ``csrc/``;
``svg`` is its thin ctypes binding.  Importing this package does not load the
library; ``from sparse_attention_video_profile_b200 import svg`` does, and
fails loudly if it has not been built.
"""
__version__ = "0.1.0"
