"""Chunk-causal 3D-RoPE attention for the Causal WAN DiT on NVIDIA B200 (sm_100a).

The compute path is the C-ABI library ``libdz.so`` (include/dz.h); ``dz``
is its ctypes binding and ``synth`` draws seeded synthetic inputs.  Importing
the package does not load the library; ``dz.load()`` (or the first call)
does, and fails loudly if it has not been built.
"""
__all__ = ["dz", "synth"]
