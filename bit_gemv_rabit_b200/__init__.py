"""librabit: the RaBiT residual-binary linear layer on NVIDIA B200 (sm_100a).

The compute path is the C-ABI shared library ``librabit.so`` built from ``csrc/``; the
Python binding in :mod:`bit_gemv_rabit_b200.rabit` only marshals arguments to it.  Importing
this package loads nothing; the library is loaded on first use of the binding and a missing
or unbuilt library raises an error (there is no fallback path).
"""
__all__ = ["inputs"]
