"""Block-causal linear attention with a constant-memory fp32 state, for B200.

The compute lives in ``libla_b200.so`` (hand-written sm_100a CUDA kernels behind
a C ABI, declared in ``include/la.h``).  ``block_causal_linear_b200.la`` is the
thin ctypes binding with the same entry-point names.  Nothing is imported here,
so that the input generator in ``synth`` loads without the CUDA library.
"""
