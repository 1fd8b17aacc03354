"""B200-native MLA against the compressed latent cache: libmla (CUDA, sm_100a)
and its Python binding -- absorbed decode (dense and top-k sparse), cache
append, output projection, and prefill in the materialised factorisation.

``binding`` is the ctypes layer over include/mla.h; ``runner`` moves a
generated workload onto the GPU and drives the library; ``inputs`` holds the
seeded synthetic inputs.  Importing the package loads nothing; the library is
loaded on first use and a missing build raises.
"""
__all__ = ["binding", "inputs", "roofline", "runner"]
