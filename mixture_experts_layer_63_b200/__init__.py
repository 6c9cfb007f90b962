"""B200-native forward pass of a sparse Mixture-of-Experts FFN layer.

The compute path lives in ``libmoe.so`` (hand-written CUDA for sm_100a behind
a C ABI, declared in ``include/moe.h``).  ``mixture_experts_layer_63_b200.api`` is a thin ctypes
binding with the same entry-point names; it marshals torch tensors into plain
device pointers and the current CUDA stream.  Importing this package does not
load the library; the first call into ``api`` does, and raises if it is
missing.
"""
