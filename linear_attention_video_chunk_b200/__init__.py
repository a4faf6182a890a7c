"""ReHyAt temporally chunked hybrid attention on NVIDIA B200 (sm_100a).

The compute path is the C-ABI library ``librehyat.so`` (hand-written CUDA);
``rehyat`` is its thin ctypes binding.  Importing this package does not load
the library; the first call through ``rehyat`` does, and fails loudly if the
library is missing.
"""
__all__ = ["rehyat", "inputs"]
