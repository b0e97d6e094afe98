"""B200-native Compressed Sparse Attention (CSA) / Heavily Compressed Attention (HCA).

The compute path is the C-ABI library ``libcsa_b200.so`` (hand-written CUDA
for sm_100a, declared in ``include/csa_b200.h``); ``api`` is its thin Python
binding.  ``synth`` draws the seeded synthetic workloads.  Importing the
package does not load the library; the first call through ``api`` does, and
raises if it is missing.
"""
__all__ = ["api", "synth"]
