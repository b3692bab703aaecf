"""B200-native learnable channel permutation (PermLLM LCP) hot path.

The compute path is the CUDA library ``csrc/liblcp.so`` (sm_100a); the
``binding`` module only marshals arguments into it.  Importing this package
does not load the library; the first call into ``binding`` does, and raises
if the library is missing.
"""
