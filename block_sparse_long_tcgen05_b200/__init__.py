"""B200 (sm_100a) hot path of MiniMax Sparse Attention (MSA).

The computation lives in libmsa.so (hand-written CUDA, C ABI in include/msa.h);
``msa`` is its Python binding and ``synth`` draws the seeded synthetic workloads.
"""
from . import synth  # noqa: F401
