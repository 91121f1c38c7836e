"""B200-native decode hot path of Simplified Sparse Attention (gist tokens).

``gist_token_chunk_b200.ssa`` binds the C-ABI library ``libssa.so`` (built
from ``csrc/`` for sm_100a); importing it fails loudly when the library is
missing.  ``gist_token_chunk_b200.inputs`` draws the seeded synthetic
workloads.  This package root imports neither, so the input generator can be
used without the native library.
"""
