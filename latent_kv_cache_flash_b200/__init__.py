"""GQLA decode attention on B200 (sm_100a).

The compute path is the C-ABI library ``libgqla.so`` (CUDA kernels, declared in
``include/gqla.h``); :mod:`latent_kv_cache_flash_b200.gqla` is a thin ctypes
binding over it.  Nothing is imported eagerly so that the input generators in
:mod:`latent_kv_cache_flash_b200.synth` load without the library.
"""
__all__ = ["gqla", "synth"]
