"""B200-native blockwise packed causal RoPE attention.

The compute lives in ``liblwm_blockattn.so`` (CUDA for sm_100a, C ABI in
``include/lwm_blockattn.h``); ``ops`` is a thin ctypes binding over it.
Import of this package stays light: the shared library is loaded on first
use, and a missing library raises instead of falling back to anything.
"""

__all__ = ["ops", "workloads"]
