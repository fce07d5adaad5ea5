"""B200-native (sm_100a) DeepSeek-V4 hybrid CSA/HCA attention hot path.

The kernels and their C ABI live in ``csrc/`` (built into
``_lib/libds4a.so``); ``ds4a`` is the thin ctypes binding with the same
entry-point names.  PyTorch serves only for device memory and streams.
"""
from .ds4a import *  # noqa: F401,F403
