"""libdit3d: B200 (sm_100a) kernels for the hot path of a video Diffusion Transformer block.

The C library (``libdit3d.so``, ABI in ``include/dit3d.h``) holds every kernel;
``dit3d`` is its ctypes binding (the library is loaded on first use) and
``workloads`` the synthetic-input generator.
"""
from . import dit3d, workloads  # noqa: F401

__all__ = ["dit3d", "workloads"]
