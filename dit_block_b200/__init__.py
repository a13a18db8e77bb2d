"""B200-native fused DiT-block per-token operators.

The kernels live in ``libsol.so`` (CUDA, sm_100a) behind the C ABI declared in
``include/sol.h``; :mod:`dit_block_b200.sol` is the ctypes binding with the same names.
Importing this package does not load the library; the first op call does, and it
raises if the library is missing.  There is no CPU fallback.
"""
