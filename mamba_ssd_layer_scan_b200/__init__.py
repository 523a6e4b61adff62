"""B200-native (sm_100a) Mamba-2 SSD sequence mixer: chunked scan and recurrent decode update.

The compute path lives in the C-ABI shared library built from ``csrc/`` (declared in
``include/ssd.h``); ``ssd`` is the thin ctypes binding over it.  Submodules are imported lazily so
that the input generator can be used on machines without the CUDA library.
"""
__all__ = ["configs", "inputs", "ssd"]
