"""libbsattn: block-sparse (keep-or-drop) and piecewise (PISA) attention on B200.

The compute lives in the CUDA library ``libbsattn.so`` (C ABI: include/bsattn.h);
``bsattn`` is its Python binding and ``synth`` the seeded synthetic-input generators.
Importing the package loads nothing; the first call into ``bsattn`` loads the library
and raises if it is missing.
"""
__all__ = ["bsattn", "synth"]
