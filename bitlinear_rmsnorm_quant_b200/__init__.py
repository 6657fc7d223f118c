"""Fused RMSNorm + BitLinear (ternary weights, int8 activations) for B200.

The compute path is the CUDA library ``libmmf.so`` (declared in
``include/mmf.h``); ``mmf`` is its thin ctypes binding.  Importing this package
does not load the library; the first call into ``mmf`` does, and fails loudly
if it is missing.
"""
