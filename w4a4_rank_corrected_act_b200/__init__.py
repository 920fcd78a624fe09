"""B200-native (sm_100a) SVDQuant W4A4 linear layer.

The compute path lives in the shared library ``libsvdq_b200.so`` (C ABI in
``include/svdq.h``); this package only builds it and binds it with ctypes.
"""
from .binding import *  # noqa: F401,F403
from .binding import SvdqLinear, SvdqError, lib, LIB_PATH, svdq_weight, calibrate_lambda  # noqa: F401
