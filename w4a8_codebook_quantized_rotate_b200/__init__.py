"""B200-native asym_w4a8_int8 ConvRot linear layer.

The layer itself is the C-ABI CUDA library declared in ``include/w4a8.h``
(built into ``lib/libw4a8.so``); :mod:`.binding` is its ctypes binding.
"""

from . import build as build  # noqa: F401
