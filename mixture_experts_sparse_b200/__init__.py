"""B200-native forward pass of one sparse Mixture-of-Experts FFN layer.

The compute path is the C-ABI library ``libmoe_b200.so`` (hand-written sm_100a
CUDA kernels); ``mixture_experts_sparse_b200.native`` is a thin ctypes binding
with the same entry-point names.  The binding loads the library lazily and raises
if it is missing: there is no CPU fallback.
"""
