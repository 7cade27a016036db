"""B200-native CSA/HCA compressed long-context attention layer.

The compute path is the C-ABI library ``libcsa_b200.so`` (hand-written sm_100a
CUDA kernels, declared in ``include/csa.h``); ``ops`` is its thin ctypes binding.
"""
from . import configs  # noqa: F401
