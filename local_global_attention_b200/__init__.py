"""PACK3D local-global attention on NVIDIA B200 (sm_100a).

The operator lives in the CUDA library built from ``csrc/`` (C ABI in
``include/pack3d.h``); :mod:`local_global_attention_b200.pack3d` is its Python
binding.  Importing this package does not load the library.
"""
__all__ = ["pack3d", "inputs", "configs", "build"]
