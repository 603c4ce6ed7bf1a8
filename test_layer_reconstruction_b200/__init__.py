"""B200 (sm_100a) implementation of the VGG-T^3 test-time-training layer.

``ttt`` binds the C ABI of libttt.so (include/ttt.h); ``inputs`` draws the
seeded synthetic workloads; ``build`` compiles the CUDA library in-tree.
"""
from . import inputs  # noqa: F401

__all__ = ["inputs", "ttt", "build"]
