"""B200-native (sm_100a) TurboQuant hot path: online vector quantization with
near-optimal distortion, and inner-product / attention scoring over the codes.

The compute lives in ``libtq_b200.so`` (hand-written CUDA, C ABI in
``include/tq.h``); this package is its ctypes binding.  Importing it without
the built library raises: there is no CPU fallback.
"""
from .api import *  # noqa: F401,F403
from .api import __all__  # noqa: F401
