"""IndexMem hot path on B200: learned KV-cache eviction with latent memory.

The CUDA library (libindexmem.so, C ABI in include/indexmem.h) does all the
work; ``binding`` marshals arguments to it, ``layer`` wraps one layer's
buffers, ``synth`` draws seeded synthetic workloads. Importing the package
does not load the library; the first binding call does, and fails loudly if it
is missing.
"""
__all__ = ["binding", "synth", "layer"]
