"""SVDQuant W4A4 linear layer with a 16-bit low-rank branch, for B200 (sm_100a).

The compute lives in ``libsvdq.so`` (CUDA, include/svdq.h); ``svdq`` is its
Python binding and ``workloads`` the seeded synthetic inputs.
"""
__version__ = "0.2.0"
