"""TTQ linear layer on B200 (sm_100a): activation-aware test-time
quantisation with hand-written CUDA kernels behind a C ABI (include/ttq.h).

The compiled library is loaded on first use by ``ttq`` (the ctypes binding);
importing the package itself does not touch the GPU.
"""
__version__ = "0.1.0"
