"""Quantised-base + LoRA linear for NVIDIA B200 (sm_100a): CUDA kernels behind a C ABI.

``qlr`` is the Python binding of include/qlr.h; ``build`` compiles libqlr.so in-tree.
"""
__all__ = ["qlr", "build"]
